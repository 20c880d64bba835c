// W4A8 decode GEMV on the sm_100a tensor cores (tcgen05), M <= 16 activation rows.
//
//   acc[n, m] = sum_k u[n, k] * xq[m, k] - 8 * sum_k xq[m, k]      (u = offset-binary nibble)
//   y[m, n]   = bf16( (float(acc) * x_scale[m]) * w_scale[n] (+ bias[n]) )
//
// The W4A8 decode of comfy-kitchen PR #182 ("Description": int4 weights decoded
// in registers, int8 products with int32 accumulation, the shared EpiRowwise
// epilogue, bit-identical to the large-M path). Here the weights are the
// operand that fills the tensor core:
//   - 128 weight rows are the M = 128 operand of tcgen05.mma.kind::i8, as
//     unsigned bytes u: decode warps split each packed k-block (TMA-loaded, 64
//     bytes per row) into nibbles and write them in natural k order into a
//     128-byte-swizzled K-major tile;
//   - the activation rows, padded to 16, are the N = 16 operand (signed),
//     TMA-loaded once per CTA with the same swizzle (rows past M read as 0);
//   - the 128 x 16 int32 accumulator lives in TMEM.
// The offset comes out once per output: sum (u - 8) x = sum u x - 8 sum x.
//
// Work split. When the 128-row blocks are fewer than the SMs (N = 3840: 30
// blocks), or one CTA's activations would not fit in shared memory, a cluster
// of S CTAs shares one block and splits its k-blocks S ways. Each CTA writes
// its partial accumulator, less 8 times its partial activation sums, to its
// own shared memory; CTA 0 of the cluster adds the others' through
// distributed shared memory, applies the epilogue and writes y. No global
// scratch is needed.
//
// Warps: 0 TMA producer (activations once, weight stages through the packed
// ring), 1 TMEM allocation and MMA issue, 2..7 decode (two per decoded slot,
// 64 rows each), 8..11 epilogue (one TMEM lane quarter each). Every barrier wait is
// bounded (ck_common.cuh); on a timeout the CTA stops, drains what it issued,
// still meets its cluster, frees TMEM and returns with the device error word
// set. The first weight stages are constant data and stream before the
// programmatic-dependency wait; activations and y wait for it.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "ck_common.cuh"

namespace ck {
namespace gtc {

constexpr int BM = 128;            // weight rows per CTA (UMMA M)
constexpr int BN = 16;             // activation rows, padded (UMMA N)
constexpr int BK = 128;            // k per stage = bytes per decoded row
constexpr int PKB = BK / 2;        // packed bytes per weight row per stage
constexpr int W_U = BM * BK;       // 16 KiB decoded stage
constexpr int W_P = BM * PKB;      // 8 KiB packed stage
constexpr int X_KB = BN * BK;      // 2 KiB activation tile per k-block
// Two rings: packed weight stages (8 KiB, the deeper one: they carry the bytes
// in flight from HBM) and decoded stages (16 KiB). Two decode warps serve each
// decoded slot. The depths are the fastest of a measured sweep (packed 4..12,
// decoded 2..7).
constexpr int NP = 8;
constexpr int NU = 3;
// A decode pair waits for fill g / NP of packed slot g % NP only once fill
// g / NP - 1 is complete (every stage before g - NU has been consumed), which
// needs NP > NU; otherwise parity waits could alias.
static_assert(NP > NU, "packed ring deeper than the decoded ring");
constexpr int kDecWarps = 2 * NU;
// the epilogue warps start at a multiple of 4 (warp w reads TMEM lanes 32 (w % 4) ..)
constexpr int W_PROD = 0, W_MMA = 1, W_DEC0 = 2, W_DEC1 = W_DEC0 + kDecWarps, W_EPI0 = (W_DEC1 + 3) / 4 * 4;
constexpr int kEpiWarps = 4;
constexpr int kThreads = (W_EPI0 + kEpiWarps) * 32;
constexpr uint32_t kTmemCols = 32;  // the smallest allocation; 16 columns are used
constexpr int RED_BYTES = BM * BN * 4;
constexpr int kBars = 2 * NP + 2 * NU + 3;
static_assert(W_EPI0 % 4 == 0, "epilogue warp w reads TMEM lanes 32 (w % 4) ..");

// Dynamic shared memory for a CTA holding `nkbc_max` activation k-blocks.
__host__ __device__ constexpr int smem_bytes(int nkbc_max) {
  return NU * W_U + NP * W_P + nkbc_max * X_KB + RED_BYTES + kBars * 8 + 8 + BN * 4 + 1024;
}

struct Params {
  int M, K, N;
  int S;          // CTAs per cluster: the split of K
  int nkb;        // K / 128
  int nkbc_max;   // most k-blocks one CTA takes: ceil(nkb / S)
  const float* xs;
  const __nv_bfloat16* sw;
  const __nv_bfloat16* bias;
  __nv_bfloat16* y;
};

// 16 packed bytes (32 nibbles, k = 0..31, low nibble = even k) -> the 32
// unsigned nibbles in natural k order: o0 holds k 0..15, o1 holds k 16..31.
__device__ __forceinline__ void nibbles_u8(const uint4 p, uint4& o0, uint4& o1) {
  const uint32_t w[4] = {p.x, p.y, p.z, p.w};
  uint32_t r[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t lo = w[j] & 0x0F0F0F0Fu, hi = (w[j] >> 4) & 0x0F0F0F0Fu;
    r[2 * j] = __byte_perm(lo, hi, 0x5140);       // k 8j .. 8j + 3
    r[2 * j + 1] = __byte_perm(lo, hi, 0x7362);   // k 8j + 4 .. 8j + 7
  }
  o0 = make_uint4(r[0], r[1], r[2], r[3]);
  o1 = make_uint4(r[4], r[5], r[6], r[7]);
}

// One warp decodes packed rows [64 h, 64 h + 64) of a stage (64 bytes each)
// into the 128-byte-swizzled tile: 16-byte chunk c of row r at c ^ (r % 8).
__device__ __forceinline__ void decode_rows(const uint8_t* src, uint8_t* dst, int h, int lane) {
  uint4 pk[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int c = 256 * h + 32 * i + lane, r = c >> 2, pc = c & 3;
    pk[i] = *reinterpret_cast<const uint4*>(src + r * PKB + pc * 16);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int c = 256 * h + 32 * i + lane, r = c >> 2, pc = c & 3;
    uint4 o0, o1;
    nibbles_u8(pk[i], o0, o1);
    *reinterpret_cast<uint4*>(dst + r * 128 + (((2 * pc) ^ (r & 7)) << 4)) = o0;
    *reinterpret_cast<uint4*>(dst + r * 128 + (((2 * pc + 1) ^ (r & 7)) << 4)) = o1;
  }
}

// 16 bytes of another CTA's shared memory (a shared::cluster address).
__device__ __forceinline__ int4 ld_dsmem_v4(uint32_t addr) {
  int4 v;
  asm volatile("ld.shared::cluster.v4.s32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ void epi_bar_sync() {   // the four epilogue warps only
  asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory");
}

__global__ void __launch_bounds__(kThreads, 1)
    gemv_w4a8_tc_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                        const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* wu = sm;                                  // [NU][16 KiB] decoded weights
  uint8_t* wp = wu + NU * W_U;                       // [NP][8 KiB] packed weights
  uint8_t* xt = wp + NP * W_P;                       // [nkbc_max][2 KiB] activations
  int32_t* red = reinterpret_cast<int32_t*>(xt + p.nkbc_max * X_KB);   // [128][16] partial sums
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(red) + RED_BYTES);
  uint64_t* full_p = bars;
  uint64_t* empty_p = bars + NP;
  uint64_t* full_u = bars + 2 * NP;
  uint64_t* empty_u = bars + 2 * NP + NU;
  uint64_t* x_full = bars + 2 * NP + 2 * NU;
  uint64_t* acc_full = x_full + 1;
  uint64_t* drain = x_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kBars);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* xsum = abort_flag + 1;                        // [16]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = p.S;
  const uint32_t rank = cluster_ctarank();
  const int n0 = (int)(blockIdx.x / S) * BM;
  const int kb0 = (int)((int64_t)rank * p.nkb / S);
  const int nkbc = (int)((int64_t)(rank + 1) * p.nkb / S) - kb0;   // >= 1: S <= nkb

  if (threadIdx.x == 0) {
    for (int s = 0; s < NP; ++s) {
      mbar_init(&full_p[s], 1);
      mbar_init(&empty_p[s], 2);
    }
    for (int s = 0; s < NU; ++s) {
      mbar_init(&full_u[s], 2);
      mbar_init(&empty_u[s], 1);
    }
    mbar_init(x_full, 1);
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == W_PROD && lane == 0) {
    prefetch_tmap(&tm_w);
    prefetch_tmap(&tm_x);
  }
  if (warp == W_MMA) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  volatile int* abort = abort_flag;
  const int first = nkbc < NP ? nkbc : NP;
  if (warp == W_PROD && lane == 0)   // constant weights: start streaming before the dependency wait
    for (int g = 0; g < first; ++g) {
      mbar_arrive_expect_tx(&full_p[g], W_P);
      tma_load_2d(wp + g * W_P, &tm_w, &full_p[g], (kb0 + g) * PKB, n0);
    }
  grid_dep_launch();
  grid_dep_wait();   // the activations and y belong to the previous kernel until here

  if (warp == W_PROD) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      mbar_arrive_expect_tx(x_full, (uint32_t)(nkbc * X_KB));
      for (int j = 0; j < nkbc; ++j) tma_load_2d(xt + j * X_KB, &tm_x, x_full, (kb0 + j) * BK, 0);
      int g = first;
      bool ok = true;
      for (; g < nkbc; ++g) {
        const int s = g % NP;
        if (!mbar_wait(&empty_p[s], ((g / NP) & 1) ^ 1, abort, 40)) { ok = false; break; }
        mbar_arrive_expect_tx(&full_p[s], W_P);
        tma_load_2d(wp + s * W_P, &tm_w, &full_p[s], (kb0 + g) * PKB, n0);
      }
      if (!ok) {   // drain: every copy issued lands before the CTA exits
        for (int h = g - 1; h >= 0 && h >= g - NP; --h)
          mbar_wait(&full_p[h % NP], (h / NP) & 1, nullptr, 41, 100000000ull);
        mbar_wait(x_full, 0, nullptr, 41, 100000000ull);
      }
    }
  } else if (warp == W_MMA) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(BM, BN, false, true);   // u8 weights x s8 activations
      bool ok = mbar_wait(x_full, 0, abort, 42);
      tc_fence_after();
      for (int g = 0; ok && g < nkbc; ++g) {
        const int s = g % NU;
        if (!mbar_wait(&full_u[s], (g / NU) & 1, abort, 43)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BK / 32; ++kk) {
          const uint64_t ad = desc_kmajor_sw128(wu + s * W_U, kk * 32);
          const uint64_t bd = desc_kmajor_sw128(xt + g * X_KB, kk * 32);
          mma_i8(tmem, ad, bd, idesc, (g | kk) != 0);
        }
        mma_commit(&empty_u[s]);
      }
      if (ok) {
        mma_commit(acc_full);
      } else {   // the MMAs in flight finish before TMEM is released
        mma_commit(drain);
        mbar_wait(drain, 0, nullptr, 44, 100000000ull);
      }
    }
  } else if (warp < W_DEC1) {
    // --------------------------------------------------------------- decode
    // the warp pair of decoded slot su takes stages g = su, su + NU, ..., each
    // read from packed slot g % NP: phase g / NP of that slot belongs to stage g
    // alone, and the producer refills it only after both halves have arrived
    const int dw = warp - W_DEC0, half = dw & 1, su = dw >> 1;
    for (int g = su; g < nkbc; g += NU) {
      const int sp = g % NP;
      if (!warp_wait(&empty_u[su], ((g / NU) & 1) ^ 1, abort, 45)) break;
      if (!warp_wait(&full_p[sp], (g / NP) & 1, abort, 46)) break;
      decode_rows(wp + sp * W_P, wu + su * W_U, half, lane);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&empty_p[sp]);
        mbar_arrive(&full_u[su]);
      }
    }
  } else if (warp >= W_EPI0) {
    // ------------------------------------------------------------- epilogue
    const int q = warp & 3, r = q * 32 + lane;
    // partial activation sums of this CTA's k-range: thread r adds 16-byte chunk
    // r % 8 of activation row r / 8 in every k-block (a row's sum ignores the
    // swizzle, which only moves chunks within the row)
    bool ok = warp_wait(x_full, 0, abort, 47);
    if (ok) {
      const int t = r >> 3, part = r & 7;
      int sacc = 0;
      for (int j = 0; j < nkbc; ++j) {
        const uint4 v = *reinterpret_cast<const uint4*>(xt + j * X_KB + t * 128 + part * 16);
        sacc = __dp4a((int)v.x, 0x01010101, sacc);
        sacc = __dp4a((int)v.y, 0x01010101, sacc);
        sacc = __dp4a((int)v.z, 0x01010101, sacc);
        sacc = __dp4a((int)v.w, 0x01010101, sacc);
      }
      sacc += __shfl_xor_sync(0xffffffffu, sacc, 1);
      sacc += __shfl_xor_sync(0xffffffffu, sacc, 2);
      sacc += __shfl_xor_sync(0xffffffffu, sacc, 4);
      if (part == 0) xsum[t] = sacc;
    }
    epi_bar_sync();
    if (ok) ok = warp_wait(acc_full, 0, abort, 48);
    if (ok) {
      tc_fence_after();
      uint32_t v[16];
      tmem_ld_32x32b_x16(tmem + ((uint32_t)(q * 32) << 16), v);
      tmem_ld_wait();
      int4* dst = reinterpret_cast<int4*>(red + r * BN);
#pragma unroll
      for (int j = 0; j < BN; j += 4)
        dst[j / 4] = make_int4((int)v[j] - 8 * xsum[j], (int)v[j + 1] - 8 * xsum[j + 1],
                               (int)v[j + 2] - 8 * xsum[j + 2], (int)v[j + 3] - 8 * xsum[j + 3]);
    }
  }

  // every CTA of the cluster has its partial sums in shared memory
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (rank == 0 && warp >= W_EPI0 && *abort == 0) {
    const int r = (warp & 3) * 32 + lane, n = n0 + r;
    int acc[BN];
    const int4* own = reinterpret_cast<const int4*>(red + r * BN);
#pragma unroll
    for (int j = 0; j < BN / 4; ++j) {
      const int4 a = own[j];
      acc[4 * j] = a.x; acc[4 * j + 1] = a.y; acc[4 * j + 2] = a.z; acc[4 * j + 3] = a.w;
    }
    for (int c = 1; c < S; ++c) {   // fixed order: the sum is exact in int32 either way
      const uint32_t base = mapa_shared(smem_u32(red + r * BN), (uint32_t)c);
#pragma unroll
      for (int j = 0; j < BN / 4; ++j) {
        const int4 a = ld_dsmem_v4(base + 16 * j);
        acc[4 * j] += a.x; acc[4 * j + 1] += a.y; acc[4 * j + 2] += a.z; acc[4 * j + 3] += a.w;
      }
    }
    if (n < p.N) {
      const float sw = __bfloat162float(p.sw[n]);
      const bool has_bias = p.bias != nullptr;
      const float b = has_bias ? __bfloat162float(p.bias[n]) : 0.0f;
#pragma unroll
      for (int t = 0; t < BN; ++t) {
        if (t < p.M) {
          float v = __fmul_rn(__fmul_rn((float)acc[t], p.xs[t]), sw);
          if (has_bias) v = __fadd_rn(v, b);
          p.y[(int64_t)t * p.N + n] = __float2bfloat16_rn(v);
        }
      }
    }
  }
  cluster_sync();   // CTA 0 has read the others' partial sums
  if (warp == W_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace gtc
}  // namespace ck
