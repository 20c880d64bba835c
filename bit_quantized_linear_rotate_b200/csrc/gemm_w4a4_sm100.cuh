// K2: W4A4 / W4A8 integer GEMM on the sm_100a tensor cores.
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
// Each operand is either packed int4 (OP_PACKED4: TMA stages 64-byte packed
// rows, the decode warps unpack nibbles to int8 u - 8 into the MMA operand
// tile) or int8 (OP_INT8: TMA writes the operand tile directly, 128-byte
// swizzle). One CTA computes one 128 x 256 output tile:
//   warp 0      TMA producer of the packed ring
//   warp 1      TMEM allocation (256 columns); one thread issues
//               tcgen05.mma.cta_group::1.kind::i8 (M=128, N=256, K=32), four per
//               k-block, and commits each operand stage back to its producers
//   warps 2..5  nibble decode into the operand ring, then the epilogue:
//               tcgen05.ld of their 32 TMEM lanes, rowwise scales, bf16, stores
//   warp 6      TMA producer of int8 operand tiles
// Operand tiles are K-major with the 128-byte swizzle (rows of 128 bytes,
// 16-byte chunk c of row r at chunk c ^ (r % 8)), the layout both the TMA
// swizzle and the UMMA shared-memory descriptor use.
// Every barrier wait is bounded (ck_common.cuh); on a timeout the CTA drains
// what it issued, frees TMEM and returns with the device error word set.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "ck_common.cuh"

namespace ck {
namespace gemm {

constexpr int BM = 128;            // activation rows per tile (UMMA M)
constexpr int BN = 256;            // weight rows per tile (UMMA N)
constexpr int BK = 128;            // k per stage = bytes per int8 operand row
constexpr int PKB = BK / 2;        // packed bytes per row per stage
constexpr int A_U = BM * BK;       // 16 KiB
constexpr int B_U = BN * BK;       // 32 KiB
constexpr int A_P = BM * PKB;      // 8 KiB
constexpr int B_P = BN * PKB;      // 16 KiB
constexpr int kThreads = 224;
constexpr int kDecThreads = 128;   // warps 2..5
constexpr uint32_t kTmemCols = 256;

enum Operand { OP_PACKED4 = 0, OP_INT8 = 1 };
enum Epi { EPI_I32 = 0, EPI_BF16 = 1 };

template <int A_MODE, int B_MODE>
struct Cfg {
  static constexpr bool AP = A_MODE == OP_PACKED4;
  static constexpr bool BP = B_MODE == OP_PACKED4;
  static constexpr bool ANY_P = AP || BP;
  static constexpr bool ANY_I8 = !AP || !BP;
  static constexpr int NU = (AP && BP) ? 2 : (ANY_P ? 3 : 4);   // operand stages
  static constexpr int NP = ANY_P ? 4 : 1;                        // packed stages
  static constexpr int P_STAGE = (AP ? A_P : 0) + (BP ? B_P : 0);
  static constexpr int I8_BYTES = (AP ? 0 : A_U) + (BP ? 0 : B_U);
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + NU * A_U;
  static constexpr int OFF_P = OFF_B + NU * B_U;
  static constexpr int OFF_BAR = OFF_P + (ANY_P ? NP * P_STAGE : 0);
  // barriers: full_p, empty_p [NP], full_u, empty_u [NU], acc_full, drain
  static constexpr int NBAR = 2 * NP + 2 * NU + 2;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int OFF_COL = (OFF_MISC + 16 + 15) / 16 * 16;
  static constexpr int BYTES = OFF_COL + 2 * BN * 4;
  static constexpr size_t SMEM = BYTES + 1024;                   // slack for 1024-byte alignment
  static_assert(SMEM <= 232448, "shared memory budget");
};

struct Params {
  int M, N, K;
  const float* a_scale;          // (M)      EPI_BF16
  const __nv_bfloat16* w_scale;  // (N)      EPI_BF16
  const __nv_bfloat16* bias;     // (N) or null
  void* out;                     // (M, N) int32 or bf16
  int out_vec_ok;                // 16-byte vector stores allowed
};

// Writes one decoded 16-byte chunk (k = 16 * uc .. 16 * uc + 15 of the stage)
// of operand row r into a 128-byte-swizzled K-major tile.
__device__ __forceinline__ void st_sw128(uint8_t* tile, int r, int uc, uint4 v) {
  *reinterpret_cast<uint4*>(tile + r * 128 + ((uc ^ (r & 7)) << 4)) = v;
}

// Decodes ROWS packed rows (64 bytes each) of a stage into the operand tile.
template <int ROWS>
__device__ __forceinline__ void decode_tile(const uint8_t* src, uint8_t* dst, int dt, int kbase, int K) {
#pragma unroll 4
  for (int c = dt; c < ROWS * 4; c += kDecThreads) {
    const int r = c >> 2, pc = c & 3;
    uint4 o0 = make_uint4(0, 0, 0, 0), o1 = o0;
    if (kbase + pc * 32 < K) {   // columns past K decode to 0, not to -8
      const uint4 pk = *reinterpret_cast<const uint4*>(src + r * PKB + pc * 16);
      decode_nibbles_s8(pk, o0, o1);
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
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::OFF_MISC);
  int* abort_flag = reinterpret_cast<int*>(sm + C::OFF_MISC + 4);
  float* col_scale = reinterpret_cast<float*>(sm + C::OFF_COL);
  float* col_bias = col_scale + BN;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BN;
  const int m0 = blockIdx.y * BM;
  const int nkb = (p.K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NP; ++s) {
      mbar_init(&full_p[s], 1);
      mbar_init(&empty_p[s], kDecThreads);
    }
    for (int s = 0; s < NU; ++s) {
      mbar_init(&full_u[s], (C::ANY_P ? kDecThreads : 0) + (C::ANY_I8 ? 1 : 0));
      mbar_init(&empty_u[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if ((warp == 0 || warp == 6) && lane == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  volatile int* abort = abort_flag;

  if (warp == 0) {
    // ---------------------------------------------------- packed-ring producer
    if (C::ANY_P && lane == 0) {
      int issued = 0;
      for (int kb = 0; kb < nkb; ++kb) {
        const int sp = kb % NP;
        if (!mbar_wait(&empty_p[sp], ((kb / NP) & 1) ^ 1, abort, 1)) break;
        mbar_arrive_expect_tx(&full_p[sp], C::P_STAGE);
        uint8_t* st = pk + sp * C::P_STAGE;
        if (C::AP) tma_load_2d(st, &tm_a, &full_p[sp], kb * PKB, m0);
        if (C::BP) tma_load_2d(st + (C::AP ? A_P : 0), &tm_b, &full_p[sp], kb * PKB, n0);
        issued = kb + 1;
      }
      if (*abort)
        for (int kb = issued - 1; kb >= 0 && kb >= issued - NP; --kb)
          mbar_wait(&full_p[kb % NP], (kb / NP) & 1, nullptr, 3, 100000000ull);
    }
  } else if (warp == 6) {
    // ------------------------------------------------- int8 operand producer
    if (C::ANY_I8 && lane == 0) {
      int issued = 0;
      for (int kb = 0; kb < nkb; ++kb) {
        const int su = kb % NU;
        if (!mbar_wait(&empty_u[su], ((kb / NU) & 1) ^ 1, abort, 2)) break;
        mbar_arrive_expect_tx(&full_u[su], C::I8_BYTES);
        if (!C::AP) tma_load_2d(a_u + su * A_U, &tm_a, &full_u[su], kb * BK, m0);
        if (!C::BP) tma_load_2d(b_u + su * B_U, &tm_b, &full_u[su], kb * BK, n0);
        issued = kb + 1;
      }
      if (*abort)
        for (int kb = issued - 1; kb >= 0 && kb >= issued - NU; --kb)
          mbar_wait(&full_u[kb % NU], (kb / NU) & 1, nullptr, 3, 100000000ull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issue
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(BM, BN);
      for (int kb = 0; kb < nkb; ++kb) {
        const int su = kb % NU;
        if (!mbar_wait(&full_u[su], (kb / NU) & 1, abort, 4)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BK / 32; ++kk) {
          const uint64_t ad = desc_kmajor_sw128(a_u + su * A_U, kk * 32);
          const uint64_t bd = desc_kmajor_sw128(b_u + su * B_U, kk * 32);
          mma_i8(tmem, ad, bd, idesc, (kb | kk) != 0);
        }
        mma_commit(&empty_u[su]);
      }
      if (*abort) {
        mma_commit(drain);
        mbar_wait(drain, 0, nullptr, 5, 100000000ull);
      } else {
        mma_commit(acc_full);
      }
    }
  } else {
    // --------------------------------------------------- decode (warps 2..5)
    const int dt = threadIdx.x - 64;
    if (C::ANY_P) {
      for (int kb = 0; kb < nkb; ++kb) {
        const int sp = kb % NP, su = kb % NU;
        if (!mbar_wait(&full_p[sp], (kb / NP) & 1, abort, 6)) break;
        if (!mbar_wait(&empty_u[su], ((kb / NU) & 1) ^ 1, abort, 7)) break;
        const uint8_t* st = pk + sp * C::P_STAGE;
        if (C::BP) decode_tile<BN>(st + (C::AP ? A_P : 0), b_u + su * B_U, dt, kb * BK, p.K);
        if (C::AP) decode_tile<BM>(st, a_u + su * A_U, dt, kb * BK, p.K);
        fence_proxy_async_smem();
        mbar_arrive(&empty_p[sp]);
        mbar_arrive(&full_u[su]);
      }
    }

    // -------------------------------------------------------------- epilogue
    if (EPI == EPI_BF16) {
      for (int j = dt; j < BN; j += kDecThreads) {
        const int n = n0 + j;
        col_scale[j] = n < p.N ? __bfloat162float(p.w_scale[n]) : 0.0f;
        col_bias[j] = (n < p.N && p.bias != nullptr) ? __bfloat162float(p.bias[n]) : 0.0f;
      }
      asm volatile("bar.sync 1, %0;" ::"r"(kDecThreads) : "memory");
    }
    if (mbar_wait(acc_full, 0, abort, 8)) {
      tc_fence_after();
      const int quarter = warp & 3;               // TMEM lanes this warp may read
      const int rl = quarter * 32 + lane;         // tile row of this thread
      const int m = m0 + rl;
      const bool row_ok = m < p.M;
      const float srow = (EPI == EPI_BF16 && row_ok) ? p.a_scale[m] : 0.0f;
      const bool has_bias = p.bias != nullptr;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)c0, r);
        tmem_ld_wait();
        if (!row_ok) continue;
        const int nb = n0 + c0;
        const bool full = (nb + 32 <= p.N) && p.out_vec_ok;
        if (EPI == EPI_I32) {
          int32_t* orow = reinterpret_cast<int32_t*>(p.out) + (int64_t)m * p.N + nb;
          if (full) {
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              *reinterpret_cast<uint4*>(orow + j) = make_uint4(r[j], r[j + 1], r[j + 2], r[j + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (nb + j < p.N) orow[j] = (int32_t)r[j];
          }
        } else {
          uint32_t h[16];
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            float v0 = __fmul_rn(__fmul_rn((float)(int32_t)r[j], srow), col_scale[c0 + j]);
            float v1 = __fmul_rn(__fmul_rn((float)(int32_t)r[j + 1], srow), col_scale[c0 + j + 1]);
            if (has_bias) {
              v0 = __fadd_rn(v0, col_bias[c0 + j]);
              v1 = __fadd_rn(v1, col_bias[c0 + j + 1]);
            }
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(v0, v1);
            h[j >> 1] = *reinterpret_cast<const uint32_t*>(&b2);
          }
          __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.out) + (int64_t)m * p.N + nb;
          if (full) {
#pragma unroll
            for (int j = 0; j < 16; j += 4)
              *reinterpret_cast<uint4*>(orow + 2 * j) = make_uint4(h[j], h[j + 1], h[j + 2], h[j + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (nb + j < p.N) {
                const uint32_t hw = h[j >> 1];
                reinterpret_cast<unsigned short*>(orow)[j] =
                    (j & 1) ? (unsigned short)(hw >> 16) : (unsigned short)(hw & 0xFFFFu);
              }
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
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
