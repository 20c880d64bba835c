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
// Design (one CTA per 128 x 256 output tile, one tile per CTA):
//   warp 0        TMA producer: packed tiles (64 bytes = 128 k per row) of the
//                 weights (and of int4 activations) into a 4-stage ring; int8
//                 activations go straight into the MMA operand ring with the
//                 128-byte swizzle.
//   warp 1        allocates 256 TMEM columns; one thread issues
//                 tcgen05.mma.cta_group::1.kind::i8, M=128 N=256 K=32, four per
//                 stage, and commits each stage back to the decoders.
//   warps 2..5    decode nibbles to int8 (u - 8) from the packed ring into the
//                 2-stage MMA operand ring (K-major, 128-byte swizzle), then run
//                 the epilogue: tcgen05.ld of their 32 TMEM lanes, the rowwise
//                 scales, bf16 rounding and 16-byte stores.
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
constexpr int BK = 128;            // k per stage = bytes per unpacked operand row
constexpr int PKB = BK / 2;        // packed bytes per row per stage
constexpr int NP = 4;              // packed stages
constexpr int NU = 2;              // operand (unpacked) stages
constexpr int A_U = BM * BK;       // 16 KiB
constexpr int B_U = BN * BK;       // 32 KiB
constexpr int A_P = BM * PKB;      // 8 KiB
constexpr int B_P = BN * PKB;      // 16 KiB
constexpr int kThreads = 192;
constexpr int kDecThreads = 128;   // warps 2..5
constexpr uint32_t kTmemCols = 256;

struct Smem {
  uint8_t a_u[NU][A_U];            // 1024-byte aligned (offset 0)
  uint8_t b_u[NU][B_U];
  uint8_t a_p[NP][A_P];
  uint8_t b_p[NP][B_P];
  uint64_t full_p[NP];
  uint64_t empty_p[NP];
  uint64_t full_u[NU];
  uint64_t empty_u[NU];
  uint64_t acc_full;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  float col_scale[BN];
  float col_bias[BN];
};
constexpr size_t kSmemBytes = sizeof(Smem) + 1024;   // + slack for 1024-byte alignment

enum Epi { EPI_I32 = 0, EPI_BF16 = 1 };

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

template <bool A_PACKED, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_w4_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                   const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                     ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BN;
  const int m0 = blockIdx.y * BM;
  const int nkb = (p.K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NP; ++s) {
      mbar_init(&S.full_p[s], 1);
      mbar_init(&S.empty_p[s], kDecThreads);
    }
    for (int s = 0; s < NU; ++s) {
      mbar_init(&S.full_u[s], kDecThreads + (A_PACKED ? 0 : 1));
      mbar_init(&S.empty_u[s], 1);
    }
    mbar_init(&S.acc_full, 1);
    mbar_init(&S.drain, 1);
    S.abort = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
  }
  if (warp == 1) {
    tmem_alloc(&S.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  volatile int* abort = &S.abort;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0;
      for (int kb = 0; kb < nkb; ++kb) {
        const int sp = kb % NP;
        if (!mbar_wait(&S.empty_p[sp], ((kb / NP) & 1) ^ 1, abort, 1)) break;
        mbar_arrive_expect_tx(&S.full_p[sp], B_P + (A_PACKED ? A_P : 0));
        tma_load_2d(S.b_p[sp], &tm_b, &S.full_p[sp], kb * PKB, n0);
        if (A_PACKED) tma_load_2d(S.a_p[sp], &tm_a, &S.full_p[sp], kb * PKB, m0);
        if (!A_PACKED) {
          const int su = kb % NU;
          if (!mbar_wait(&S.empty_u[su], ((kb / NU) & 1) ^ 1, abort, 2)) { issued = kb + 1; break; }
          mbar_arrive_expect_tx(&S.full_u[su], A_U);
          tma_load_2d(S.a_u[su], &tm_a, &S.full_u[su], kb * BK, m0);
        }
        issued = kb + 1;
      }
      if (*abort) {
        // drain: wait (bounded) for the copies issued into the packed ring
        for (int kb = issued - 1; kb >= 0 && kb >= issued - NP; --kb)
          mbar_wait(&S.full_p[kb % NP], (kb / NP) & 1, nullptr, 3, 100000000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issue
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(BM, BN);
      for (int kb = 0; kb < nkb; ++kb) {
        const int su = kb % NU;
        if (!mbar_wait(&S.full_u[su], (kb / NU) & 1, abort, 4)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BK / 32; ++kk) {
          const uint64_t ad = desc_kmajor_sw128(S.a_u[su], kk * 32);
          const uint64_t bd = desc_kmajor_sw128(S.b_u[su], kk * 32);
          mma_i8(tmem, ad, bd, idesc, (kb | kk) != 0);
        }
        mma_commit(&S.empty_u[su]);
      }
      if (*abort) {
        mma_commit(&S.drain);
        mbar_wait(&S.drain, 0, nullptr, 5, 100000000ull);
      } else {
        mma_commit(&S.acc_full);
      }
    }
  } else {
    // ------------------------------------------------------ decode (warps 2..5)
    const int dt = threadIdx.x - 64;
    for (int kb = 0; kb < nkb; ++kb) {
      const int sp = kb % NP, su = kb % NU;
      if (!mbar_wait(&S.full_p[sp], (kb / NP) & 1, abort, 6)) break;
      if (!mbar_wait(&S.empty_u[su], ((kb / NU) & 1) ^ 1, abort, 7)) break;
      const int kbase = kb * BK;
      // weight tile: 256 rows x 4 packed chunks of 16 bytes
#pragma unroll 4
      for (int c = dt; c < BN * 4; c += kDecThreads) {
        const int r = c >> 2, pc = c & 3;
        uint4 o0 = make_uint4(0, 0, 0, 0), o1 = o0;
        if (kbase + pc * 32 < p.K) {
          const uint4 pk = *reinterpret_cast<const uint4*>(S.b_p[sp] + r * PKB + pc * 16);
          decode_nibbles_s8(pk, o0, o1);
        }
        st_sw128(S.b_u[su], r, 2 * pc, o0);
        st_sw128(S.b_u[su], r, 2 * pc + 1, o1);
      }
      if (A_PACKED) {
#pragma unroll 4
        for (int c = dt; c < BM * 4; c += kDecThreads) {
          const int r = c >> 2, pc = c & 3;
          uint4 o0 = make_uint4(0, 0, 0, 0), o1 = o0;
          if (kbase + pc * 32 < p.K) {
            const uint4 pk = *reinterpret_cast<const uint4*>(S.a_p[sp] + r * PKB + pc * 16);
            decode_nibbles_s8(pk, o0, o1);
          }
          st_sw128(S.a_u[su], r, 2 * pc, o0);
          st_sw128(S.a_u[su], r, 2 * pc + 1, o1);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&S.empty_p[sp]);
      mbar_arrive(&S.full_u[su]);
    }

    // -------------------------------------------------------------- epilogue
    if (EPI == EPI_BF16) {
      for (int j = dt; j < BN; j += kDecThreads) {
        const int n = n0 + j;
        S.col_scale[j] = n < p.N ? __bfloat162float(p.w_scale[n]) : 0.0f;
        S.col_bias[j] = (n < p.N && p.bias != nullptr) ? __bfloat162float(p.bias[n]) : 0.0f;
      }
      asm volatile("bar.sync 1, %0;" ::"r"(kDecThreads) : "memory");
    }
    if (mbar_wait(&S.acc_full, 0, abort, 8)) {
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
            float v0 = __fmul_rn(__fmul_rn((float)(int32_t)r[j], srow), S.col_scale[c0 + j]);
            float v1 = __fmul_rn(__fmul_rn((float)(int32_t)r[j + 1], srow), S.col_scale[c0 + j + 1]);
            if (has_bias) {
              v0 = __fadd_rn(v0, S.col_bias[c0 + j]);
              v1 = __fadd_rn(v1, S.col_bias[c0 + j + 1]);
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

}  // namespace gemm
}  // namespace ck
