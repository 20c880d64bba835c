// K1: fused groupwise Hadamard rotation + rowwise symmetric quantization.
//
// Follows "quantize_and_rotate_rowwise" (comfy-kitchen PR #155 "[Feat][Ascend]
// Add fused RotateQuant backend", "What this PR does": group rotation, rowwise
// dynamic quantization, positive scale, zero-row handling) with the
// warp-shuffle Hadamard transform named in comfy-kitchen PR #182
// ("Description": the CUDA INT8 rowwise ConvRot quantizer of #176).
//
// One CTA per row. Thread t owns 8-element vectors v = i * blockDim + t
// (i < VPT) loaded with 128-bit loads, so a warp covers 256 consecutive
// columns per iteration and every Hadamard group (G <= 256 columns = G/8
// vectors) sits in G/8 consecutive lanes. The transform runs in fp32:
// three butterfly stages inside the thread, log2(G/8) stages across lanes
// with __shfl_xor_sync, then the 1/sqrt(G) normalisation (exact for G = 16,
// 64, 256). The rotated row never leaves registers: amax is reduced across the
// CTA, then each thread quantizes and stores its own values (4 bytes of packed
// int4 or 8 bytes of int8 per vector, coalesced across the warp).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ck_common.cuh"

namespace ck {
namespace rq {

template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&f)[8]);

template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&f)[8]) {
  const uint4 raw = __ldcs(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    f[2 * j] = __uint_as_float(w[j] << 16);
    f[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
  }
}

template <>
__device__ __forceinline__ void load8<__half>(const __half* p, float (&f)[8]) {
  const uint4 raw = __ldcs(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 v = __half22float2(*reinterpret_cast<const __half2*>(&w[j]));
    f[2 * j] = v.x;
    f[2 * j + 1] = v.y;
  }
}

// y[e] for e in 0..7 -> Sylvester butterflies on element-index bits 0..2 (only
// the bits below G). Index bit b set => new = x(bit clear) - x(bit set).
__device__ __forceinline__ void fht_in_thread(float (&v)[8], int G) {
#pragma unroll
  for (int h = 1; h < 8; h <<= 1) {
    if (h < G) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if ((e & h) == 0) {
          const float a = v[e], b = v[e + h];
          v[e] = a + b;
          v[e + h] = a - b;
        }
      }
    }
  }
}

// Stages on element-index bits 3.. (lane bits 0..): partner lane = lane ^ j.
__device__ __forceinline__ void fht_across_lanes(float (&v)[8], int G, int lane) {
  for (int j = 1; 8 * j < G; j <<= 1) {
    const bool upper = (lane & j) != 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float other = __shfl_xor_sync(0xffffffffu, v[e], j);
      v[e] = upper ? (other - v[e]) : (v[e] + other);
    }
  }
}

// Threads per CTA allowed for VPT vectors per thread (keeps VPT = 8 in registers).
__host__ __device__ constexpr int max_threads(int vpt) { return vpt >= 8 ? 512 : 1024; }

template <int VPT, int BITS, typename T>
__global__ void __launch_bounds__(max_threads(VPT)) rotate_quant_kernel(const T* __restrict__ x, int K,
                                                            int64_t ldx, int G, float rnorm,
                                                            uint8_t* __restrict__ q,
                                                            float* __restrict__ scale) {
  constexpr float kQmax = BITS == 4 ? 7.0f : 127.0f;
  __shared__ float red[32];
  const int64_t row = blockIdx.x;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int nvec = K >> 3;
  const T* xr = x + row * ldx;

  float v[VPT][8];
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int vi = i * blockDim.x + tid;
    if (vi < nvec) {
      load8<T>(xr + 8 * vi, v[i]);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) v[i][e] = 0.0f;
    }
  }

  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    // every lane of the warp runs the shuffles; vectors past the row are zeros
    if (i * (int)blockDim.x < nvec) {
      if (G > 1) {
        fht_in_thread(v[i], G);
        fht_across_lanes(v[i], G, lane);
#pragma unroll
        for (int e = 0; e < 8; ++e) v[i][e] *= rnorm;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[i][e]));
    }
  }

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

#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int vi = i * blockDim.x + tid;
    if (vi < nvec) {
      int qi[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float t = rintf(__fmul_rn(v[i][e], r));
        qi[e] = (int)fminf(fmaxf(t, -kQmax), kQmax);
      }
      if (BITS == 4) {
        uint32_t packed = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) packed |= (uint32_t)(qi[e] + 8) << (4 * e);
        reinterpret_cast<uint32_t*>(q + row * (int64_t)(K >> 1))[vi] = packed;
      } else {
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          lo |= (uint32_t)(qi[e] & 0xFF) << (8 * e);
          hi |= (uint32_t)(qi[e + 4] & 0xFF) << (8 * e);
        }
        reinterpret_cast<uint2*>(q + row * (int64_t)K)[vi] = make_uint2(lo, hi);
      }
    }
  }
}

}  // namespace rq
}  // namespace ck
