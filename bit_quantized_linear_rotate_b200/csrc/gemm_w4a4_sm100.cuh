// K2: W4A4 / W4A8 integer GEMM on the sm_100a tensor cores, one CTA pair per
// 256 x 256 output tile.
//
//   acc[m, n] = sum_k qa[m, k] * w[n, k]        (int8 x int8 -> int32 in TMEM)
//   y[m, n]   = bf16( (float(acc) * a_scale[m]) * w_scale[n] (+ bias[n]) )
//
// The integer matmul on unpacked int4 weights is the Ascend W4A4 path of
// comfy-kitchen PR #212 ("Summary": packed weights unpacked before each
// integer matmul); the epilogue is the shared "EpiRowwise" of comfy-kitchen
// PR #182 ("Description"). The packed formats are "convrot_w4a4" and
// "asym_w4a8_int8" of stable-diffusion.cpp PR #2276 ("Summary").
//
// Layout of the work. A cluster of two CTAs computes a 256 (activation rows) x
// 256 (weight rows) tile with tcgen05.mma.cta_group::2.kind::i8, M=256 N=256
// K=32, issued by one thread of the even CTA: each CTA holds 128 activation
// rows (A) and 128 of the 256 weight rows (B) of every k-block in its own
// shared memory, and 128 accumulator rows x 256 columns in its TMEM. Splitting
// B across the pair halves the operand bytes each SM's shared memory serves
// per MMA. The grid is persistent (as many pairs as fit at once); pairs walk
// the output tiles with the weight-tile index fastest, so concurrently
// resident pairs share activation rows in L2.
//
// Operand paths (per operand):
//   OP_INT8      int8 tile straight from TMA (128-byte swizzle)
//   OP_PACKED4   packed int4 (64 bytes per row per k-block) from TMA, decoded to
//                signed int8 u - 8 in natural k order by the decode warps
//   OP_PACKED4_U weights only: decoded to unsigned u with the k order of each
//                8-column group permuted to (0 2 4 6 1 3 5 7) -- three logical
//                ops per 8 nibbles; the activations arrive in the same permuted
//                order and the epilogue subtracts 8 * sum_k qa[m, k]
// Decoded tiles use the same K-major 128-byte-swizzled layout as the TMA
// writes and the UMMA shared-memory descriptor reads (rows of 128 bytes,
// 16-byte chunk c of row r at chunk c ^ (r % 8)).
//
// Warps: 0 packed-tile TMA producer, 1 MMA issue (even CTA) and TMEM
// allocation, 2..11 nibble decode (two per operand slot, 64 rows each; the
// first of each pair also issues that slot's int8-tile TMA as soon as the slot
// is free; without a decode path warp 2 issues all int8 tiles), 12..15
// epilogue.
// TMEM holds two accumulators (2 x 256 columns): the epilogue of one tile
// overlaps the main loop of the next. Every barrier wait is bounded
// (ck_common.cuh); on a timeout the CTA stops issuing, drains what it issued,
// meets its peer, frees TMEM and returns with the device error word set.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "ck_common.cuh"

namespace ck {
namespace gemm {

constexpr int BM = 128;            // activation rows per CTA (pair: 256 = UMMA M)
constexpr int BN = 256;            // weight rows per pair tile (UMMA N)
constexpr int BNH = BN / 2;        // weight rows held by each CTA
constexpr int BK = 128;            // k per stage = bytes per int8 operand row
constexpr int PKB = BK / 2;        // packed bytes per row per stage
constexpr int A_U = BM * BK;       // 16 KiB
constexpr int B_U = BNH * BK;      // 16 KiB
constexpr int A_P = BM * PKB;      // 8 KiB
constexpr int B_P = BNH * PKB;     // 8 KiB
constexpr int kDecWarps = 10;       // two per operand slot (at most 5 slots with a decode path)
constexpr int kEpiWarps = 4;
constexpr int W_PACK = 0, W_MMA = 1, W_DEC0 = 2, W_EPI0 = W_DEC0 + kDecWarps;
constexpr int kThreads = (W_EPI0 + kEpiWarps) * 32;
constexpr int kDecThreads = kDecWarps * 32;
constexpr uint32_t kTmemCols = 512;  // two 256-column accumulators

enum Operand { OP_PACKED4 = 0, OP_INT8 = 1, OP_PACKED4_U = 2 };
enum Epi { EPI_I32 = 0, EPI_BF16 = 1 };

template <int A_MODE, int B_MODE>
struct Cfg {
  static constexpr bool AP = A_MODE == OP_PACKED4;
  static constexpr bool BP = B_MODE != OP_INT8;
  static constexpr bool BU = B_MODE == OP_PACKED4_U;
  static constexpr bool ANY_P = AP || BP;
  static constexpr bool ANY_I8 = !AP || !BP;
  // With a decode path, the packed ring and the operand ring have the same
  // depth and decode warp dw owns slot dw of both: every wait it makes is on
  // the phase right after the one it saw last, so parity waits cannot alias.
  static constexpr int NU = !ANY_P ? 6 : ((AP && BP) ? 4 : 5);   // operand stages
  static constexpr int NP = !ANY_P ? 1 : NU;                      // packed stages
  static constexpr int NDEC = ANY_P ? 2 * NU : 0;                 // active decode warps (2 per slot)
  static_assert(NDEC <= kDecWarps, "decode warps");
  static constexpr int P_STAGE = (AP ? A_P : 0) + (BP ? B_P : 0);
  static constexpr int I8_CTA_BYTES = (AP ? 0 : A_U) + (BP ? 0 : B_U);
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + NU * A_U;
  static constexpr int OFF_P = OFF_B + NU * B_U;
  static constexpr int OFF_BAR = OFF_P + (ANY_P ? NP * P_STAGE : 0);
  // full_p, empty_p [NP]; full_u, empty_u [NU]; acc_full, acc_empty [2]; drain
  static constexpr int NBAR = 2 * NP + 2 * NU + 5;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr size_t SMEM = BYTES + 1024;                    // slack for 1024-byte alignment
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(!(A_MODE == OP_PACKED4_U), "the permuted unsigned path is for the weights");
};

struct Params {
  int M, N, K;
  int tiles_m, tiles_n;           // 256 x 256 pair tiles
  const float* a_scale;           // (M)      EPI_BF16
  const int32_t* a_rowsum;        // (M)      OP_PACKED4_U: sum_k qa[m, k]
  const __nv_bfloat16* w_scale;   // (N)      EPI_BF16
  const __nv_bfloat16* bias;      // (N) or null
  void* out;                      // (M, N) int32 or bf16
  int out_vec_ok;                 // 16-byte vector stores allowed
  int col_vec_ok;                 // w_scale (and bias) 16-byte aligned: vector loads
};

// Writes one decoded 16-byte chunk (k = 16 * uc .. 16 * uc + 15 of the stage)
// of operand row r into a 128-byte-swizzled K-major tile.
__device__ __forceinline__ void st_sw128(uint8_t* tile, int r, int uc, uint4 v) {
  *reinterpret_cast<uint4*>(tile + r * 128 + ((uc ^ (r & 7)) << 4)) = v;
}

// One warp decodes 64 packed rows (64 bytes each, rows [64 h, 64 h + 64)) of a
// stage into the operand tile: all eight 16-byte loads are issued first.
template <bool UNSIGNED_PERM>
__device__ __forceinline__ void decode_half(const uint8_t* src, uint8_t* dst, int h, int lane, int kbase, int K) {
  uint4 pk[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int c = 256 * h + 32 * i + lane, r = c >> 2, pc = c & 3;
    pk[i] = *reinterpret_cast<const uint4*>(src + r * PKB + pc * 16);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int c = 256 * h + 32 * i + lane, r = c >> 2, pc = c & 3;
    uint4 o0 = make_uint4(0, 0, 0, 0), o1 = o0;
    if (kbase + pc * 32 < K) {   // columns past K decode to 0 (unsigned: weight 8 against code 0)
      if (UNSIGNED_PERM) decode_nibbles_u8_perm(pk[i], o0, o1);
      else decode_nibbles_s8(pk[i], o0, o1);
    }
    st_sw128(dst, r, 2 * pc, o0);
    st_sw128(dst, r, 2 * pc + 1, o1);
  }
}

template <int A_MODE, int B_MODE, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_w4_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                   const Params p) {
  using C = Cfg<A_MODE, B_MODE>;
  constexpr int NU = C::NU, NP = C::NP;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_u = sm + C::OFF_A;
  uint8_t* b_u = sm + C::OFF_B;
  uint8_t* pk = sm + C::OFF_P;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR);
  uint64_t* full_p = bars;
  uint64_t* empty_p = bars + NP;
  uint64_t* full_u = bars + 2 * NP;
  uint64_t* empty_u = bars + 2 * NP + NU;
  uint64_t* acc_full = bars + 2 * NP + 2 * NU;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_full + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::OFF_MISC);
  int* abort_flag = reinterpret_cast<int*>(sm + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();        // 0: leader (issues the MMAs), 1: peer
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  const int ntiles = p.tiles_m * p.tiles_n;
  const int nkb = (p.K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NP; ++s) {
      mbar_init(&full_p[s], 1);
      mbar_init(&empty_p[s], 2);
    }
    for (int s = 0; s < NU; ++s) {
      mbar_init(&full_u[s], (C::ANY_P ? 4 : 0) + (C::ANY_I8 ? 1 : 0));
      mbar_init(&empty_u[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if ((warp == W_PACK || warp == W_DEC0) && lane == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
  }
  if (warp == W_MMA) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();            // both CTAs' barriers exist before any cross-CTA arrive or copy
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  volatile int* abort = abort_flag;
  // launched as a programmatic dependent: the set-up above overlaps the end of
  // the previous kernel; the operands and the output belong to it until here
  grid_dep_launch();
  grid_dep_wait();

  if (warp == W_PACK) {
    // ------------------------------------------------------ packed-tile producer
    if (C::ANY_P && lane == 0) {
      int g = 0;
      bool ok = true;
      for (int t = pair; t < ntiles && ok; t += npairs) {
        const int m_row = (t / p.tiles_n) * 256 + (int)rank * BM;
        const int n_row = (t % p.tiles_n) * BN + (int)rank * BNH;
        for (int kb = 0; kb < nkb; ++kb, ++g) {
          const int sp = g % NP;
          if (!mbar_wait(&empty_p[sp], ((g / NP) & 1) ^ 1, abort, 1)) { ok = false; break; }
          mbar_arrive_expect_tx(&full_p[sp], C::P_STAGE);
          uint8_t* st = pk + sp * C::P_STAGE;
          if (C::AP) tma_load_2d(st, &tm_a, &full_p[sp], kb * PKB, m_row);
          if (C::BP) tma_load_2d(st + (C::AP ? A_P : 0), &tm_b, &full_p[sp], kb * PKB, n_row);
        }
      }
      if (!ok)   // drain: the copies issued into the packed ring land before the CTA exits
        for (int h = g - 1; h >= 0 && h >= g - NP; --h)
          mbar_wait(&full_p[h % NP], (h / NP) & 1, nullptr, 3, 100000000ull);
    }
  } else if (warp == W_MMA) {
    // ------------------------------------------------ MMA issue (leader CTA)
    if (rank == 0 && lane == 0) {
      constexpr uint32_t idesc = idesc_i8(2 * BM, BN, true, !C::BU);
      int g = 0, i = 0;
      bool ok = true;
      for (int t = pair; t < ntiles && ok; t += npairs, ++i) {
        const int ab = i & 1;
        if (!mbar_wait_cluster(&acc_empty[ab], ((i >> 1) & 1) ^ 1, abort, 4)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(ab * BN);
        for (int kb = 0; kb < nkb; ++kb, ++g) {
          const int su = g % NU;
          if (!mbar_wait_cluster(&full_u[su], (g / NU) & 1, abort, 5)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk) {
            const uint64_t ad = desc_kmajor_sw128(a_u + su * A_U, kk * 32);
            const uint64_t bd = desc_kmajor_sw128(b_u + su * B_U, kk * 32);
            mma_i8_pair(d, ad, bd, idesc, (kb | kk) != 0);
          }
          mma_commit_pair(&empty_u[su], 0x3);
        }
        if (ok) mma_commit_pair(&acc_full[ab], 0x3);
      }
      if (!ok) {   // drain the MMAs in flight before TMEM is released
        mma_commit_pair(drain, 0x1);
        mbar_wait(drain, 0, nullptr, 9, 100000000ull);
      }
    }
  } else if (warp < W_EPI0) {
    // ------------------------------------------------ decode (warps 2..11)
    // Stage g belongs to the decode warps 2 (g % NU) and 2 (g % NU) + 1 (slot
    // g % NU of both rings), each taking half of the rows: a pair of warps
    // turns a whole stage around (one proxy fence and one arrive per warp and
    // stage), and up to NU stages are decoded concurrently.
    const int dw = warp - W_DEC0;
    if (C::ANY_P && dw < C::NDEC) {
      const int half = dw & 1, slot = dw >> 1;
      int g = 0, last_i8 = -1;
      bool ok = true;
      for (int t = pair; t < ntiles && ok; t += npairs) {
        const int m_row = (t / p.tiles_n) * 256 + (int)rank * BM;
        const int n_row = (t % p.tiles_n) * BN + (int)rank * BNH;
        for (int kb = 0; kb < nkb; ++kb, ++g) {
          if (g % NU != slot) continue;
          const int sp = g % NP, su = g % NU;
          if (!warp_wait(&empty_u[su], ((g / NU) & 1) ^ 1, abort, 7)) { ok = false; break; }
          if (C::ANY_I8 && half == 0 && lane == 0) {   // the slot is free: fetch its int8 tiles
            if (rank == 0) mbar_arrive_expect_tx(&full_u[su], 2 * C::I8_CTA_BYTES);
            const uint32_t bar = mapa_shared(smem_u32(&full_u[su]), 0);
            if (!C::AP) tma_load_2d_pair(a_u + su * A_U, &tm_a, bar, kb * BK, m_row);
            if (!C::BP) tma_load_2d_pair(b_u + su * B_U, &tm_b, bar, kb * BK, n_row);
            last_i8 = g;
          }
          if (!warp_wait(&full_p[sp], (g / NP) & 1, abort, 6)) { ok = false; break; }
          const uint8_t* st = pk + sp * C::P_STAGE;
          if (C::BP) decode_half<C::BU>(st + (C::AP ? A_P : 0), b_u + su * B_U, half, lane, kb * BK, p.K);
          if (C::AP) decode_half<false>(st, a_u + su * A_U, half, lane, kb * BK, p.K);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&empty_p[sp]);
            if (rank == 0) mbar_arrive(&full_u[su]);
            else mbar_arrive_remote(mapa_shared(smem_u32(&full_u[su]), 0));
          }
        }
      }
      if (!ok && rank == 0 && lane == 0 && last_i8 >= 0)   // drain the int8 tiles this warp requested
        mbar_wait_cluster(&full_u[last_i8 % NU], (last_i8 / NU) & 1, nullptr, 3, 100000000ull);
    } else if (!C::ANY_P && dw == 0 && lane == 0) {
      // ------------------------------------------- int8-tile producer (no decode path)
      int g = 0;
      bool ok = true;
      for (int t = pair; t < ntiles && ok; t += npairs) {
        const int m_row = (t / p.tiles_n) * 256 + (int)rank * BM;
        const int n_row = (t % p.tiles_n) * BN + (int)rank * BNH;
        for (int kb = 0; kb < nkb; ++kb, ++g) {
          const int su = g % NU;
          if (!mbar_wait(&empty_u[su], ((g / NU) & 1) ^ 1, abort, 2)) { ok = false; break; }
          if (rank == 0) mbar_arrive_expect_tx(&full_u[su], 2 * C::I8_CTA_BYTES);
          const uint32_t bar = mapa_shared(smem_u32(&full_u[su]), 0);
          tma_load_2d_pair(a_u + su * A_U, &tm_a, bar, kb * BK, m_row);
          tma_load_2d_pair(b_u + su * B_U, &tm_b, bar, kb * BK, n_row);
        }
      }
      if (!ok && rank == 0)   // drain (the leader's barrier counts both CTAs' bytes)
        for (int h = g - 1; h >= 0 && h >= g - NU; --h)
          mbar_wait_cluster(&full_u[h % NU], (h / NU) & 1, nullptr, 3, 100000000ull);
    }
  } else {
    // ------------------------------------------------ epilogue (warps 12..15)
    const int quarter = warp & 3;               // TMEM lanes this warp may read
    const int rl = quarter * 32 + lane;         // accumulator row of this thread
    const bool has_bias = p.bias != nullptr;
    int i = 0;
    for (int t = pair; t < ntiles; t += npairs, ++i) {
      const int ab = i & 1;
      if (!warp_wait(&acc_full[ab], (i >> 1) & 1, abort, 8)) break;
      tc_fence_after();
      const int m = (t / p.tiles_n) * 256 + (int)rank * BM + rl;
      const int n0 = (t % p.tiles_n) * BN;
      const bool row_ok = m < p.M;
      const float srow = (EPI == EPI_BF16 && row_ok) ? p.a_scale[m] : 0.0f;
      const int corr = (C::BU && row_ok) ? 8 * p.a_rowsum[m] : 0;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 16) {
        uint32_t r[16];
        tmem_ld_32x32b_x16(tmem + (uint32_t)(ab * BN) + ((uint32_t)(quarter * 32) << 16) + (uint32_t)c0, r);
        tmem_ld_wait();
        const int nb = n0 + c0;
        if (!row_ok || nb >= p.N) continue;
        const bool full = (nb + 16 <= p.N) && p.out_vec_ok;
        if (EPI == EPI_I32) {
          int32_t* orow = reinterpret_cast<int32_t*>(p.out) + (int64_t)m * p.N + nb;
          if (full) {
#pragma unroll
            for (int j = 0; j < 16; j += 4)
              *reinterpret_cast<uint4*>(orow + j) =
                  make_uint4(r[j] - corr, r[j + 1] - corr, r[j + 2] - corr, r[j + 3] - corr);
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (nb + j < p.N) orow[j] = (int32_t)r[j] - corr;
          }
        } else {
          // per-column scale and bias of these 16 columns, as bf16 pairs (broadcast loads)
          uint32_t cs[8], cb[8];
          if (full && p.col_vec_ok) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const uint4 a = __ldg(reinterpret_cast<const uint4*>(p.w_scale + nb) + j);
              cs[4 * j] = a.x; cs[4 * j + 1] = a.y; cs[4 * j + 2] = a.z; cs[4 * j + 3] = a.w;
              const uint4 b = has_bias ? __ldg(reinterpret_cast<const uint4*>(p.bias + nb) + j) : make_uint4(0, 0, 0, 0);
              cb[4 * j] = b.x; cb[4 * j + 1] = b.y; cb[4 * j + 2] = b.z; cb[4 * j + 3] = b.w;
            }
          } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int n = nb + 2 * j;
              const uint32_t s0 = n < p.N ? __bfloat16_as_ushort(p.w_scale[n]) : 0u;
              const uint32_t s1 = n + 1 < p.N ? __bfloat16_as_ushort(p.w_scale[n + 1]) : 0u;
              const uint32_t b0 = (has_bias && n < p.N) ? __bfloat16_as_ushort(p.bias[n]) : 0u;
              const uint32_t b1 = (has_bias && n + 1 < p.N) ? __bfloat16_as_ushort(p.bias[n + 1]) : 0u;
              cs[j] = s0 | (s1 << 16);
              cb[j] = b0 | (b1 << 16);
            }
          }
          uint32_t hh[8];
#pragma unroll
          for (int j = 0; j < 16; j += 2) {
            const float sw0 = __uint_as_float(cs[j >> 1] << 16);
            const float sw1 = __uint_as_float(cs[j >> 1] & 0xFFFF0000u);
            float v0 = __fmul_rn(__fmul_rn((float)((int32_t)r[j] - corr), srow), sw0);
            float v1 = __fmul_rn(__fmul_rn((float)((int32_t)r[j + 1] - corr), srow), sw1);
            if (has_bias) {
              v0 = __fadd_rn(v0, __uint_as_float(cb[j >> 1] << 16));
              v1 = __fadd_rn(v1, __uint_as_float(cb[j >> 1] & 0xFFFF0000u));
            }
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(v0, v1);
            hh[j >> 1] = *reinterpret_cast<const uint32_t*>(&b2);
          }
          __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.out) + (int64_t)m * p.N + nb;
          if (full) {
            *reinterpret_cast<uint4*>(orow) = make_uint4(hh[0], hh[1], hh[2], hh[3]);
            *reinterpret_cast<uint4*>(orow + 8) = make_uint4(hh[4], hh[5], hh[6], hh[7]);
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              if (nb + j < p.N) {
                const uint32_t hw = hh[j >> 1];
                reinterpret_cast<unsigned short*>(orow)[j] =
                    (j & 1) ? (unsigned short)(hw >> 16) : (unsigned short)(hw & 0xFFFFu);
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(mapa_shared(smem_u32(&acc_empty[ab]), 0));
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();            // the peer is done with the pair's TMEM and barriers
  if (warp == W_MMA) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

// Unpacks a packed int4 matrix (R, C/2) into int8 (R, C), value u - 8: the
// weight preparation that PR #212 caches ("Summary"), as a standalone pass.
__global__ void unpack_int4_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, int64_t n16) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n16; i += (int64_t)gridDim.x * blockDim.x) {
    uint4 o0, o1;
    decode_nibbles_s8(__ldcs(src + i), o0, o1);
    __stcs(dst + 2 * i, o0);
    __stcs(dst + 2 * i + 1, o1);
  }
}

}  // namespace gemm
}  // namespace ck
