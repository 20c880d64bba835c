// K1: fused groupwise Hadamard rotation + rowwise symmetric quantization.
//
// Follows "quantize_and_rotate_rowwise" (comfy-kitchen PR #155 "[Feat][Ascend]
// Add fused RotateQuant backend", "What this PR does": group rotation, rowwise
// dynamic quantization, positive scale, zero-row handling) with a register /
// warp-shuffle Hadamard transform as in the CUDA INT8 rowwise ConvRot quantizer
// named by comfy-kitchen PR #182 ("Description").
//
// One CTA per row; thread t owns the 32 contiguous columns [32t, 32t + 32)
// (four 128-bit loads). The transform runs in fp32: log2(min(G, 32)) butterfly
// stages inside the thread, then log2(G / 32) stages across lanes
// (__shfl_xor_sync, one shuffle and one FMA per element and stage), then the
// 1/sqrt(G) normalisation (a power of two for G = 16, 64, 256). The rotated row
// never leaves registers: amax is reduced across the CTA, then every thread
// quantizes its 32 values and writes 16 bytes (packed int4) or 32 bytes (int8).
//
// Quantization multiplies by the reciprocal of the scale; when the product lies
// within 1e-4 of a rounding boundary it is recomputed with the correctly
// rounded quotient y / s, so ties are decided as by division.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ck_common.cuh"

namespace ck {
namespace rq {

constexpr int EPT = 32;   // columns per thread

enum Store { STORE_PACKED4 = 0, STORE_INT8 = 1 };

template <typename T>
__device__ __forceinline__ void load8(const T* p, float* f);

template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float* f) {
  const uint4 raw = __ldcs(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    f[2 * j] = __uint_as_float(w[j] << 16);
    f[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
  }
}

template <>
__device__ __forceinline__ void load8<__half>(const __half* p, float* f) {
  const uint4 raw = __ldcs(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 v = __half22float2(*reinterpret_cast<const __half2*>(&w[j]));
    f[2 * j] = v.x;
    f[2 * j + 1] = v.y;
  }
}

// Sylvester butterflies on element-index bits below min(G, 32): for index bit h,
// (a, b) -> (a + b, a - b) where a has the bit clear.
__device__ __forceinline__ void fht_in_thread(float (&v)[EPT], int G) {
#pragma unroll
  for (int h = 1; h < EPT; h <<= 1) {
    if (h < G) {
#pragma unroll
      for (int e = 0; e < EPT; ++e) {
        if ((e & h) == 0) {
          const float a = v[e], b = v[e + h];
          v[e] = a + b;
          v[e + h] = a - b;
        }
      }
    }
  }
}

// Index bits 5.. live in lane bits 0..: new = partner + v (bit clear) or partner - v (bit set).
__device__ __forceinline__ void fht_across_lanes(float (&v)[EPT], int G, int lane) {
  for (int j = 1; EPT * j < G; j <<= 1) {
    const float sgn = (lane & j) ? -1.0f : 1.0f;
#pragma unroll
    for (int e = 0; e < EPT; ++e) {
      const float other = __shfl_xor_sync(0xffffffffu, v[e], j);
      v[e] = fmaf(sgn, v[e], other);
    }
  }
}

__device__ __forceinline__ int quant1(float y, float r, float s, float qmax) {
  float t = __fmul_rn(y, r);
  const float f = t - truncf(t);
  if (fabsf(fabsf(f) - 0.5f) < 1e-4f) t = __fdiv_rn(y, s);
  return (int)fminf(fmaxf(rintf(t), -qmax), qmax);
}

template <int QBITS, int STORE, typename T>
__global__ void __launch_bounds__(1024) rotate_quant_kernel(const T* __restrict__ x, int K, int64_t ldx,
                                                            int G, float rnorm, uint8_t* __restrict__ q,
                                                            float* __restrict__ scale) {
  constexpr float kQmax = QBITS == 4 ? 7.0f : 127.0f;
  __shared__ float red[32];
  const int64_t row = blockIdx.x;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int e0 = tid * EPT;
  const T* xr = x + row * ldx;

  float v[EPT];
#pragma unroll
  for (int j = 0; j < EPT / 8; ++j) {
    if (e0 + 8 * j < K) {
      load8<T>(xr + e0 + 8 * j, v + 8 * j);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) v[8 * j + e] = 0.0f;
    }
  }

  if (G > 1) {
    fht_in_thread(v, G);
    fht_across_lanes(v, G, lane);   // every lane runs it; columns past K hold zeros
#pragma unroll
    for (int e = 0; e < EPT; ++e) v[e] *= rnorm;
  }
  float amax = 0.0f;
#pragma unroll
  for (int e = 0; e < EPT; ++e) amax = fmaxf(amax, fabsf(v[e]));

#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (lane == 0) red[tid >> 5] = amax;
  __syncthreads();
  if (tid < 32) {
    float a = tid < (int)(blockDim.x >> 5) ? red[tid] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if (tid == 0) red[0] = a;
  }
  __syncthreads();
  amax = red[0];

  // positive-scale contract: an all-zero row gets scale 1 and all-zero codes
  const float s = amax > 0.0f ? __fdiv_rn(amax, kQmax) : 1.0f;
  const float r = __frcp_rn(s);
  if (tid == 0) scale[row] = s;
  if (e0 >= K) return;

  if (STORE == STORE_PACKED4) {
    // 32 codes -> 16 bytes, u = q + 8, low nibble = even column
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t acc = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc |= (uint32_t)(quant1(v[8 * j + e], r, s, kQmax) + 8) << (4 * e);
      w[j] = acc;
    }
    uint8_t* qr = q + row * (int64_t)(K >> 1) + (e0 >> 1);
    if ((K & 31) == 0) {          // rows of K/2 bytes are 16-byte aligned
      *reinterpret_cast<uint4*>(qr) = make_uint4(w[0], w[1], w[2], w[3]);
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (e0 + 8 * j < K) reinterpret_cast<uint32_t*>(qr)[j] = w[j];
    }
  } else {
    uint32_t w[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint32_t acc = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) acc |= (uint32_t)(quant1(v[4 * j + e], r, s, kQmax) & 0xFF) << (8 * e);
      w[j] = acc;
    }
    uint8_t* qr = q + row * (int64_t)K + e0;
    if ((K & 31) == 0) {
      reinterpret_cast<uint4*>(qr)[0] = make_uint4(w[0], w[1], w[2], w[3]);
      reinterpret_cast<uint4*>(qr)[1] = make_uint4(w[4], w[5], w[6], w[7]);
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (e0 + 8 * j < K) reinterpret_cast<uint2*>(qr)[j] = make_uint2(w[2 * j], w[2 * j + 1]);
    }
  }
}

}  // namespace rq
}  // namespace ck
