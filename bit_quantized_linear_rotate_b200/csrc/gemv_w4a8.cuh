// K3: W4A8 decode GEMV, M <= 16 activation rows.
//
//   acc[m, n] = sum_k xq[m, k] * (u[n, k] - 8)
//   y[m, n]   = bf16( (float(acc) * x_scale[m]) * w_scale[n] (+ bias[n]) )
//
// comfy-kitchen PR #182 ("Description"): the decode GEMV decodes the int4
// weights in registers (no INT4 -> INT8 decode pass through memory) and shares
// the codec and the EpiRowwise epilogue with the large-M path, so both are
// bit-identical. Here the weight stream is the only HBM traffic that matters:
// each byte is loaded once with 128-bit loads, split into its two nibbles with
// two logical ops and fed as the unsigned 16-row A operand of
// mma.sync.m16n8k32.u8.s8 (weights are the M side; the <= 16 activation rows
// are one or two n8 tiles). The offset is applied once per output:
// sum (u - 8) x = sum u x - 8 sum x, with sum x from dp4a against 0x01010101.
//
// k-order inside one mma is permuted identically for A and B (lane t, step j:
// fragment slot 4t+i holds k = 32t + 8j + 2i, slot 16+4t+i holds k + 1), so
// the nibble split needs no byte shuffles on the weight side.
#pragma once

#include <cuda_bf16.h>

#include "ck_common.cuh"

namespace ck {
namespace w4a8 {

constexpr int kWarps = 8;
constexpr int kRows = 16;        // weight rows per CTA
constexpr int kChunk = 128;      // k per warp step (64 packed bytes per row)

__device__ __forceinline__ void mma_u8s8(int (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int MT>  // number of 8-row activation tiles (1: M <= 8, 2: M <= 16)
__global__ void __launch_bounds__(kWarps * 32) gemv_w4a8_kernel(
    const int8_t* __restrict__ xq, const float* __restrict__ xs, int M, int K, int N,
    const uint8_t* __restrict__ w, const __nv_bfloat16* __restrict__ sw,
    const __nv_bfloat16* __restrict__ bias, __nv_bfloat16* __restrict__ y) {
  __shared__ int red[kWarps][kRows][8 * MT];
  __shared__ int xsum_s[kWarps][8 * MT];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int n0 = blockIdx.x * kRows;
  const int nchunk = K / kChunk;
  const int64_t wld = K >> 1;

  const bool r0ok = n0 + g < N, r1ok = n0 + g + 8 < N;
  const uint8_t* wr0 = w + (int64_t)(n0 + g) * wld + 16 * t;
  const uint8_t* wr1 = w + (int64_t)(n0 + g + 8) * wld + 16 * t;

  int acc[MT][4];
  int xsum[MT];
#pragma unroll
  for (int j = 0; j < MT; ++j) {
    xsum[j] = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[j][i] = 0;
  }

  constexpr int PF = 4;  // chunks loaded ahead of use
  for (int c0 = warp; c0 < nchunk; c0 += kWarps * PF) {
    uint4 wa[PF], wb[PF];
#pragma unroll
    for (int u = 0; u < PF; ++u) {
      const int c = c0 + u * kWarps;
      wa[u] = make_uint4(0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u);
      wb[u] = wa[u];
      if (c < nchunk) {
        if (r0ok) wa[u] = __ldcs(reinterpret_cast<const uint4*>(wr0 + (int64_t)c * (kChunk / 2)));
        if (r1ok) wb[u] = __ldcs(reinterpret_cast<const uint4*>(wr1 + (int64_t)c * (kChunk / 2)));
      }
    }
#pragma unroll
    for (int u = 0; u < PF; ++u) {
      const int c = c0 + u * kWarps;
      if (c >= nchunk) break;
      // activations for this lane's token column g of each tile: 32 bytes at k = c*128 + 32t
      uint32_t xv[MT][8];
#pragma unroll
      for (int j = 0; j < MT; ++j) {
        const int m = 8 * j + g;
        uint4 x0 = make_uint4(0, 0, 0, 0), x1 = x0;
        if (m < M) {
          const int8_t* xp = xq + (int64_t)m * K + (int64_t)c * kChunk + 32 * t;
          x0 = __ldg(reinterpret_cast<const uint4*>(xp));
          x1 = __ldg(reinterpret_cast<const uint4*>(xp + 16));
        }
        xv[j][0] = x0.x; xv[j][1] = x0.y; xv[j][2] = x0.z; xv[j][3] = x0.w;
        xv[j][4] = x1.x; xv[j][5] = x1.y; xv[j][6] = x1.z; xv[j][7] = x1.w;
#pragma unroll
        for (int q = 0; q < 8; ++q) xsum[j] = __dp4a((int)xv[j][q], 0x01010101, xsum[j]);
      }
      const uint32_t pa[4] = {wa[u].x, wa[u].y, wa[u].z, wa[u].w};
      const uint32_t pb[4] = {wb[u].x, wb[u].y, wb[u].z, wb[u].w};
#pragma unroll
      for (int s = 0; s < 4; ++s) {  // word s covers k = 32t + 8s .. 8s+7
        uint32_t a[4];
        a[0] = pa[s] & 0x0F0F0F0Fu;           // row g,   even k
        a[1] = pb[s] & 0x0F0F0F0Fu;           // row g+8, even k
        a[2] = (pa[s] >> 4) & 0x0F0F0F0Fu;    // row g,   odd k
        a[3] = (pb[s] >> 4) & 0x0F0F0F0Fu;    // row g+8, odd k
#pragma unroll
        for (int j = 0; j < MT; ++j) {
          const uint32_t lo = xv[j][2 * s], hi = xv[j][2 * s + 1];
          mma_u8s8(acc[j], a, __byte_perm(lo, hi, 0x6420), __byte_perm(lo, hi, 0x7531));
        }
      }
    }
  }

  // per-token sums: lanes t = 0..3 of group g hold quarters of the token's k range
#pragma unroll
  for (int j = 0; j < MT; ++j) {
    xsum[j] += __shfl_xor_sync(0xffffffffu, xsum[j], 1);
    xsum[j] += __shfl_xor_sync(0xffffffffu, xsum[j], 2);
    if (t == 0) xsum_s[warp][8 * j + g] = xsum[j];
    red[warp][g][8 * j + 2 * t] = acc[j][0];
    red[warp][g][8 * j + 2 * t + 1] = acc[j][1];
    red[warp][g + 8][8 * j + 2 * t] = acc[j][2];
    red[warp][g + 8][8 * j + 2 * t + 1] = acc[j][3];
  }
  __syncthreads();

  for (int idx = threadIdx.x; idx < kRows * 8 * MT; idx += kWarps * 32) {
    const int m = idx / kRows, r = idx % kRows;
    const int n = n0 + r;
    if (m >= M || n >= N) continue;
    int tot = 0, xsm = 0;
#pragma unroll
    for (int wv = 0; wv < kWarps; ++wv) {
      tot += red[wv][r][m];
      xsm += xsum_s[wv][m];
    }
    const int a = tot - 8 * xsm;
    float v = __fmul_rn(__fmul_rn((float)a, xs[m]), __bfloat162float(sw[n]));
    if (bias != nullptr) v = __fadd_rn(v, __bfloat162float(bias[n]));
    y[(int64_t)m * N + n] = __float2bfloat16_rn(v);
  }
}

}  // namespace w4a8
}  // namespace ck
