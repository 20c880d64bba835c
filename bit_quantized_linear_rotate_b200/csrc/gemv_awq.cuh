// K4: AWQ W4A16 GEMV, M <= 8 activation rows.
//
//   W[n, k] = (u[n, k] - 8) * wscales[k / G, n] + wzeros[k / G, n]
//   y[m, n] = sum_k x[m, k] W[n, k] (+ bias[n])
//
// comfy_kitchen/tensor/awq_w4a16.py (module docstring: packed layout and the
// dequantization formula; _awq_forward: y = x W^T + bias through
// ck.gemv_awq_w4a16). The weight is never dequantized in memory: per 64-wide
// k sub-block (inside one quantization group, G % 64 == 0)
//   y += s[g, n] * P + z[g, n] * X,   P = sum_k (u - 8) x,   X = sum_k x,
// an exact rewrite of the formula. P comes from mma.sync.m16n8k16 with fp32
// accumulation: the 16 weight rows of a tile are the A operand, decoded in
// registers from nibbles to exact bf16/fp16 values (u - 8) with one logical op
// and one packed subtract per pair (0x4300 | u is the bf16 number 128 + u;
// 0x6400 | u is the fp16 number 1024 + u); the activation rows are the n8 B
// operand. X comes from the same B fragments times an all-ones A operand, so
// each lane receives exactly the token sums its accumulators need.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ck_common.cuh"

namespace ck {
namespace awq {

constexpr int kWarps = 8;
constexpr int kRT = 2;            // 16-row tiles per CTA
constexpr int kRows = 16 * kRT;
constexpr int kSub = 64;          // k per sub-block (32 packed bytes per row)

template <typename T> struct Traits;
template <> struct Traits<__nv_bfloat16> {
  static constexpr uint32_t kMagic = 0x43004300u;    // bf16x2 (128 + u)
  static constexpr uint32_t kBias = 0x43084308u;     // bf16x2 (136, 136)
  static constexpr uint32_t kOnes = 0x3F803F80u;     // bf16x2 (1, 1)
  static __device__ __forceinline__ uint32_t sub2(uint32_t a, uint32_t b) {
    __nv_bfloat162 r = __hsub2(*reinterpret_cast<__nv_bfloat162*>(&a), *reinterpret_cast<__nv_bfloat162*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
  }
  static __device__ __forceinline__ float tof(__nv_bfloat16 v) { return __bfloat162float(v); }
  static __device__ __forceinline__ __nv_bfloat16 fromf(float v) { return __float2bfloat16_rn(v); }
  static __device__ __forceinline__ void mma(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
};
template <> struct Traits<__half> {
  static constexpr uint32_t kMagic = 0x64006400u;    // fp16x2 (1024 + u)
  static constexpr uint32_t kBias = 0x64086408u;     // fp16x2 (1032, 1032)
  static constexpr uint32_t kOnes = 0x3C003C00u;     // fp16x2 (1, 1)
  static __device__ __forceinline__ uint32_t sub2(uint32_t a, uint32_t b) {
    __half2 r = __hsub2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
  }
  static __device__ __forceinline__ float tof(__half v) { return __half2float(v); }
  static __device__ __forceinline__ __half fromf(float v) { return __float2half_rn(v); }
  static __device__ __forceinline__ void mma(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
};

// Nibbles s and s+4 of a packed word (k_rel s and s+4) as a decoded (u - 8) pair.
template <typename T>
__device__ __forceinline__ uint32_t nib_pair(uint32_t w, int s) {
  return Traits<T>::sub2(((w >> (4 * s)) & 0x000F000Fu) | Traits<T>::kMagic, Traits<T>::kBias);
}

// The same pair without the subtraction: (128 + u) as bf16, (1024 + u) as
// fp16, one shift and one logical op. A sum of such products carries an
// extra kOffset * sum(x), which the streaming kernel removes with the group's
// zero term: s * (P' - kOffset X) + z X = s P' + (z - kOffset s) X.
template <typename T>
__device__ __forceinline__ uint32_t nib_pair_raw(uint32_t w, int s) {
  return ((w >> (4 * s)) & 0x000F000Fu) | Traits<T>::kMagic;
}
template <typename T> struct RawOffset;
template <> struct RawOffset<__nv_bfloat16> { static constexpr float v = 136.0f; };   // 128 + 8
template <> struct RawOffset<__half> { static constexpr float v = 1032.0f; };         // 1024 + 8

template <typename T>
__global__ void __launch_bounds__(kWarps * 32) gemv_awq_kernel(
    const T* __restrict__ x, int M, int K, int N, int G, const uint8_t* __restrict__ qw,
    const T* __restrict__ ws, const T* __restrict__ wz, const T* __restrict__ bias,
    T* __restrict__ y) {
  __shared__ float red[kWarps][kRows][8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int n0 = blockIdx.x * kRows;
  const int nsub = K / kSub;
  const int64_t wld = K >> 1;
  const bool tok_ok = g < M;
  const uint32_t ones[4] = {Traits<T>::kOnes, Traits<T>::kOnes, Traits<T>::kOnes, Traits<T>::kOnes};

  float yacc[kRT][4];
#pragma unroll
  for (int r = 0; r < kRT; ++r)
#pragma unroll
    for (int i = 0; i < 4; ++i) yacc[r][i] = 0.0f;

  constexpr int PF = 4;
  for (int sb0 = warp; sb0 < nsub; sb0 += kWarps * PF) {
    uint2 wv[PF][kRT][2];
#pragma unroll
    for (int u = 0; u < PF; ++u) {
      const int sb = sb0 + u * kWarps;
#pragma unroll
      for (int r = 0; r < kRT; ++r)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int n = n0 + 16 * r + g + 8 * h;
          wv[u][r][h] = make_uint2(0x88888888u, 0x88888888u);
          if (sb < nsub && n < N)
            wv[u][r][h] = __ldcs(reinterpret_cast<const uint2*>(qw + (int64_t)n * wld + sb * (kSub / 2) + 8 * t));
        }
    }
#pragma unroll
    for (int u = 0; u < PF; ++u) {
      const int sb = sb0 + u * kWarps;
      if (sb >= nsub) break;
      // B fragments: this lane's token g, k = sb*64 + 16t .. +15, regrouped into (k, k+4) pairs
      uint4 xa = make_uint4(0, 0, 0, 0), xb = xa;
      if (tok_ok) {
        const T* xp = x + (int64_t)g * K + sb * kSub + 16 * t;
        xa = __ldg(reinterpret_cast<const uint4*>(xp));
        xb = __ldg(reinterpret_cast<const uint4*>(xp + 8));
      }
      uint32_t bp[8];
      bp[0] = __byte_perm(xa.x, xa.z, 0x5410);  // (0, 4)
      bp[1] = __byte_perm(xa.x, xa.z, 0x7632);  // (1, 5)
      bp[2] = __byte_perm(xa.y, xa.w, 0x5410);  // (2, 6)
      bp[3] = __byte_perm(xa.y, xa.w, 0x7632);  // (3, 7)
      bp[4] = __byte_perm(xb.x, xb.z, 0x5410);  // (8, 12)
      bp[5] = __byte_perm(xb.x, xb.z, 0x7632);  // (9, 13)
      bp[6] = __byte_perm(xb.y, xb.w, 0x5410);  // (10, 14)
      bp[7] = __byte_perm(xb.y, xb.w, 0x7632);  // (11, 15)

      float X[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int j = 0; j < 4; ++j) Traits<T>::mma(X, ones, bp[2 * j], bp[2 * j + 1]);

      const int grp = (sb * kSub) / G;
#pragma unroll
      for (int r = 0; r < kRT; ++r) {
        float P[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        const uint32_t w0[2] = {wv[u][r][0].x, wv[u][r][0].y};   // row g
        const uint32_t w1[2] = {wv[u][r][1].x, wv[u][r][1].y};   // row g+8
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          // pairs 2j and 2j+1: word (2j)/4, nibble offsets (2j)%4 and (2j+1)%4
          const int wd = j >> 1, s0 = (2 * j) & 3, s1 = (2 * j + 1) & 3;
          uint32_t a[4];
          a[0] = nib_pair<T>(w0[wd], s0);
          a[1] = nib_pair<T>(w1[wd], s0);
          a[2] = nib_pair<T>(w0[wd], s1);
          a[3] = nib_pair<T>(w1[wd], s1);
          Traits<T>::mma(P, a, bp[2 * j], bp[2 * j + 1]);
        }
        const int na = n0 + 16 * r + g, nb = na + 8;
        float sa = 0.f, za = 0.f, sbb = 0.f, zb = 0.f;
        if (na < N) { sa = Traits<T>::tof(ws[(int64_t)grp * N + na]); za = Traits<T>::tof(wz[(int64_t)grp * N + na]); }
        if (nb < N) { sbb = Traits<T>::tof(ws[(int64_t)grp * N + nb]); zb = Traits<T>::tof(wz[(int64_t)grp * N + nb]); }
        yacc[r][0] += sa * P[0] + za * X[0];
        yacc[r][1] += sa * P[1] + za * X[1];
        yacc[r][2] += sbb * P[2] + zb * X[2];
        yacc[r][3] += sbb * P[3] + zb * X[3];
      }
    }
  }

#pragma unroll
  for (int r = 0; r < kRT; ++r) {
    red[warp][16 * r + g][2 * t] = yacc[r][0];
    red[warp][16 * r + g][2 * t + 1] = yacc[r][1];
    red[warp][16 * r + g + 8][2 * t] = yacc[r][2];
    red[warp][16 * r + g + 8][2 * t + 1] = yacc[r][3];
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < kRows * 8; idx += kWarps * 32) {
    const int m = idx / kRows, rr = idx % kRows;
    const int n = n0 + rr;
    if (m >= M || n >= N) continue;
    float v = 0.0f;
#pragma unroll
    for (int wv2 = 0; wv2 < kWarps; ++wv2) v += red[wv2][rr][m];
    if (bias != nullptr) v += Traits<T>::tof(bias[n]);
    y[(int64_t)m * N + n] = Traits<T>::fromf(v);
  }
}

}  // namespace awq
}  // namespace ck
