// Rowwise quantization after a GENERAL group rotation: y_g = x_g . R for an
// arbitrary G x G matrix R (row vector times R), then the same rowwise
// symmetric quantization and storage as K1.
//
// The pages' fused RotateQuant is tested with "asymmetric-rotation inputs"
// (comfy-kitchen PR #155, "How was this patch tested?"): the rotation is a
// parameter of quantize_and_rotate_rowwise, not always the Hadamard matrix.
// Without a fast transform this is a small dense product per group, G
// multiply-adds per output element, done here on the CUDA cores in fp32:
// one CTA per row (grid-stride), the row staged in shared memory as fp32,
// each thread producing output columns with R read through the L1 cache
// (R is at most 256 x 256 and shared by every row).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ck_common.cuh"

namespace ck {
namespace rqg {

constexpr int kThreads = 256;

template <typename T> __device__ __forceinline__ float load_f(const T* p);
template <> __device__ __forceinline__ float load_f<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(*p); }
template <> __device__ __forceinline__ float load_f<__half>(const __half* p) { return __half2float(*p); }

// Shared memory: xs[K] (the row as fp32), ys[K] (the rotated row), red[32].
template <typename T, int QBITS>
__global__ void __launch_bounds__(kThreads) rotate_quant_general_kernel(const T* __restrict__ x, int64_t M, int K,
                                                                         int64_t ldx, int G,
                                                                         const float* __restrict__ R,
                                                                         uint8_t* __restrict__ q,
                                                                         float* __restrict__ scale) {
  constexpr float kQmax = QBITS == 4 ? 7.0f : 127.0f;
  extern __shared__ float smf[];
  float* xs = smf;
  float* ys = smf + K;
  __shared__ float red[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  grid_dep_launch();
  grid_dep_wait();
  for (int64_t row = blockIdx.x; row < M; row += gridDim.x) {
    const T* xr = x + row * ldx;
    for (int c = tid; c < K; c += kThreads) xs[c] = load_f<T>(xr + c);
    __syncthreads();
    float amax = 0.0f;
    for (int c = tid; c < K; c += kThreads) {
      const int g0 = c - c % G, j = c - g0;
      float acc = 0.0f;
      for (int i = 0; i < G; ++i) acc = fmaf(xs[g0 + i], __ldg(R + i * G + j), acc);
      ys[c] = acc;
      amax = fmaxf(amax, fabsf(acc));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (lane == 0) red[warp] = amax;
    __syncthreads();
    amax = 0.0f;
    for (int w = 0; w < kThreads / 32; ++w) amax = fmaxf(amax, red[w]);
    const float s = amax > 0.0f ? amax / kQmax : 1.0f;   // positive-scale contract: an all-zero row gets 1
    if (tid == 0) scale[row] = s;
    if (QBITS == 8) {
      int8_t* qr = reinterpret_cast<int8_t*>(q) + row * K;
      for (int c = tid; c < K; c += kThreads)
        qr[c] = (int8_t)fminf(fmaxf(rintf(ys[c] / s), -kQmax), kQmax);
    } else {
      uint8_t* qr = q + row * (K / 2);
      for (int b = tid; b < K / 2; b += kThreads) {
        const int lo = (int)fminf(fmaxf(rintf(ys[2 * b] / s), -kQmax), kQmax);
        const int hi = (int)fminf(fmaxf(rintf(ys[2 * b + 1] / s), -kQmax), kQmax);
        qr[b] = (uint8_t)((lo + 8) | ((hi + 8) << 4));   // offset binary, low nibble = even column
      }
    }
    __syncthreads();   // xs, ys and red are rewritten for the next row
  }
}

}  // namespace rqg
}  // namespace ck
