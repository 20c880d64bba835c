// K1: fused groupwise Hadamard rotation + rowwise symmetric quantization.
//
// Follows "quantize_and_rotate_rowwise" (comfy-kitchen PR #155 "[Feat][Ascend]
// Add fused RotateQuant backend", "What this PR does": group rotation, rowwise
// dynamic quantization, positive scale, zero-row handling) with a register /
// warp-shuffle Hadamard transform as in the CUDA INT8 rowwise ConvRot quantizer
// named by comfy-kitchen PR #182 ("Description").
//
// A persistent grid of CTAs walks the rows, one row per CTA at a time, the next
// row's loads issued before the current row is processed; thread t owns the 64
// contiguous columns [64t, 64t + 64) (eight 128-bit loads, issued coalesced and
// regrouped through shared memory). The transform runs in fp32: log2(min(G, 64)) butterfly
// stages inside the thread, then log2(G / 64) stages across lanes
// (__shfl_xor_sync, one shuffle and one FMA per element and stage), then the
// 1/sqrt(G) normalisation (a power of two for G = 16, 64, 256). The rotated row
// never leaves registers: amax is reduced across the CTA, then every thread
// quantizes its 32 values and writes 16 bytes (packed int4) or 32 bytes (int8).
//
// Arithmetic is packed two lanes at a time (sm_100 f32x2 add/mul/fma). Codes
// are rounded by adding 1.5 * 2^23 (round to nearest, ties to even, no float to
// int conversion) and packed with byte permutes. Quantization multiplies by
// the reciprocal of the scale; for unrotated rows (G = 1, where exact halves
// are common) codes near a half integer are decided exactly by the sign of
// y - h s, as division would.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ck_common.cuh"

namespace ck {
namespace rq {

constexpr int EPT = 64;   // columns per thread
constexpr int CPT = EPT / 8;   // 16-byte chunks per thread

// STORE_INT8_PERM: int8 codes with the columns of each 8-column group stored in
// the order (0 2 4 6 1 3 5 7), plus the row sum of the codes -- the activation
// format of the linear's GEMM (it pairs with weights split into low / high
// nibbles without byte shuffles).
enum Store { STORE_PACKED4 = 0, STORE_INT8 = 1, STORE_INT8_PERM = 2 };

// Coalesced 128-bit loads of the warp's 32 * EPT columns: lane l takes 16-byte
// chunks l, 32 + l, ... of the warp's span (zero past K).
__device__ __forceinline__ void load_raw(const void* row, int warp, int lane, int K, uint4 (&raw)[CPT]) {
#pragma unroll
  for (int j = 0; j < CPT; ++j) {
    const int c = 32 * CPT * warp + 32 * j + lane;      // 16-byte chunk index in the row
    raw[j] = (8 * c < K) ? __ldcs(reinterpret_cast<const uint4*>(row) + c) : make_uint4(0, 0, 0, 0);
  }
}

// 16-byte slot of chunk c in a warp's transpose buffer: the low three bits
// (position in a 128-byte line) are XORed with the line index, so both the
// coalesced writes and the contiguous per-thread reads are bank-conflict free.
__device__ __forceinline__ int tslot(int c) { return c ^ ((c >> 3) & 7); }

// Regroups the coalesced chunks so that lane l holds chunks CPT*l .. CPT*l + CPT-1
// (its EPT contiguous columns).
__device__ __forceinline__ void transpose_raw(uint4* buf, int lane, uint4 (&raw)[CPT]) {
#pragma unroll
  for (int j = 0; j < CPT; ++j) buf[tslot(32 * j + lane)] = raw[j];
  __syncwarp();
#pragma unroll
  for (int j = 0; j < CPT; ++j) raw[j] = buf[tslot(CPT * lane + j)];
  __syncwarp();
}

template <typename T>
__device__ __forceinline__ void to_float8(const uint4 raw, float* f);

template <>
__device__ __forceinline__ void to_float8<__nv_bfloat16>(const uint4 raw, float* f) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    f[2 * j] = __uint_as_float(w[j] << 16);
    f[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
  }
}

template <>
__device__ __forceinline__ void to_float8<__half>(const uint4 raw, float* f) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 v = __half22float2(*reinterpret_cast<const __half2*>(&w[j]));
    f[2 * j] = v.x;
    f[2 * j + 1] = v.y;
  }
}

// The 32 values of a thread live as 16 float2 pairs v[j] = (y[2j], y[2j+1]);
// sm_100 executes one f32x2 add / fma per pair, two lanes of fp32 work.
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {       // a - b, one rounding
  return __ffma2_rn(b, make_float2(-1.0f, -1.0f), a);
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Sylvester butterflies on element-index bits below min(G, 32): for index bit h,
// (a, b) -> (a + b, a - b) where a has the bit clear. G is a compile-time
// constant for the common group sizes (the stage tests then vanish).
__device__ __forceinline__ void fht_in_thread(float2 (&v)[EPT / 2], int G) {
  if (G > 1) {
#pragma unroll
    for (int j = 0; j < EPT / 2; ++j) {
      const float a = v[j].x, b = v[j].y;
      v[j] = make_float2(a + b, a - b);
    }
  }
#pragma unroll
  for (int hb = 1; hb < EPT / 2; hb <<= 1) {       // element bit 1.. = pair-index bit 0..
    if (2 * hb < G) {
#pragma unroll
      for (int j = 0; j < EPT / 2; ++j) {
        if ((j & hb) == 0) {
          const float2 a = v[j], b = v[j + hb];
          v[j] = __fadd2_rn(a, b);
          v[j + hb] = sub2(a, b);
        }
      }
    }
  }
}

// Index bits log2(EPT).. live in lane bits 0..: new = partner + v (bit clear) or partner - v (bit set).
__device__ __forceinline__ void fht_across_lanes(float2 (&v)[EPT / 2], int G, int lane) {
  for (int j = 1; EPT * j < G; j <<= 1) {
    const float sg = (lane & j) ? -1.0f : 1.0f;
    const float2 sgn = make_float2(sg, sg);
#pragma unroll
    for (int e = 0; e < EPT / 2; ++e) {
      const float2 other = make_float2(__shfl_xor_sync(0xffffffffu, v[e].x, j),
                                       __shfl_xor_sync(0xffffffffu, v[e].y, j));
      v[e] = __ffma2_rn(sgn, v[e], other);
    }
  }
}

// Adding 1.5 * 2^23 rounds |t| < 2^22 to an integer (nearest, ties to even) in
// the low mantissa bits: the float's bit pattern is 0x4B400000 + round(t).
constexpr float kRoundMagic = 12582912.0f;

// Exact round-half-even of y / s for an unrotated row (y = x exactly): the
// reciprocal product decides every code that is not within 1e-3 of a half
// integer; near one, the sign of the single-rounding residual y - h s decides.
__device__ __forceinline__ float quant_exact(float y, float r, float s) {
  const float t = __fmul_rn(y, r);
  const float fl = floorf(t);
  const float d = t - fl;
  if (fabsf(d - 0.5f) >= 1e-3f) return rintf(t);
  const float h = fl + 0.5f;
  const float e = fmaf(-h, s, y);
  return e > 0.0f ? fl + 1.0f : (e < 0.0f ? fl : rintf(h));
}

// GT: the group size when it is 1, 16, 64 or 256 (compile time), 0 otherwise
// (then taken from G at run time).
template <int QBITS, int STORE, int GT, typename T>
__global__ void __launch_bounds__(512) rotate_quant_kernel(const T* __restrict__ x, int64_t M, int K, int64_t ldx,
                                                            int G_rt, float rnorm, uint8_t* __restrict__ q,
                                                            float* __restrict__ scale,
                                                            int32_t* __restrict__ rowsum) {
  constexpr float kQmax = QBITS == 4 ? 7.0f : 127.0f;
  const int G = GT ? GT : G_rt;
  __shared__ float red[4][32];   // [2 * (it & 1)]: amax, [2 * (it & 1) + 1]: row sum
  extern __shared__ uint4 tbuf_all[];              // 32 * CPT chunks per warp
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int e0 = tid * EPT;
  uint4* tbuf = tbuf_all + 32 * CPT * warp;

  // persistent over rows; the next row's 128-bit loads are in flight while the
  // current row is transformed, reduced and quantized (not for G = 256 or a
  // run-time G, whose cross-lane stages need those registers)
  constexpr bool kPrefetch = GT != 0 && GT <= EPT;
  // launched as a programmatic dependent: x and the outputs belong to the
  // previous kernel in the stream until grid_dep_wait returns
  grid_dep_launch();
  grid_dep_wait();
  int64_t row = blockIdx.x;
  uint4 raw[CPT];
  if (kPrefetch && row < M) load_raw(x + row * ldx, warp, lane, K, raw);
  for (int it = 0; row < M; row += gridDim.x, ++it) {
    if (!kPrefetch) load_raw(x + row * ldx, warp, lane, K, raw);
    transpose_raw(tbuf, lane, raw);
    float2 v[EPT / 2];
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      float f[8];
      to_float8<T>(raw[j], f);
#pragma unroll
      for (int e = 0; e < 4; ++e) v[4 * j + e] = make_float2(f[2 * e], f[2 * e + 1]);
    }
    const int64_t next = row + gridDim.x;
    if (kPrefetch && next < M) load_raw(x + next * ldx, warp, lane, K, raw);

    // unnormalised transform z = x H; the 1/sqrt(G) factor is folded into the scale
    fht_in_thread(v, G);
    if (G > EPT) fht_across_lanes(v, G, lane);   // every lane runs it; columns past K hold zeros
    float amax = 0.0f;
#pragma unroll
    for (int e = 0; e < EPT / 2; ++e) amax = max3(amax, fabsf(v[e].x), fabsf(v[e].y));

    // block reductions alternate between buffer pairs, so one barrier per reduction suffices
    float* rb = red[2 * (it & 1)];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (lane == 0) rb[tid >> 5] = amax;
    __syncthreads();
    amax = 0.0f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) amax = fmaxf(amax, rb[w]);
    amax = __fmul_rn(amax, rnorm);               // amax of y = z / sqrt(G)

    // positive-scale contract: an all-zero row gets scale 1 and all-zero codes
    const float s = amax > 0.0f ? __fdiv_rn(amax, kQmax) : 1.0f;
    const float r = __frcp_rn(s);
    if (tid == 0) scale[row] = s;

    // codes: bit patterns whose low byte is q (int8) or q + 8 (offset-binary int4)
    uint32_t u[EPT];
    const float magic = STORE == STORE_PACKED4 ? kRoundMagic + 8.0f : kRoundMagic;
    if (G == 1) {
#pragma unroll
      for (int e = 0; e < EPT / 2; ++e) {
        u[2 * e] = __float_as_uint(quant_exact(v[e].x, r, s) + magic);
        u[2 * e + 1] = __float_as_uint(quant_exact(v[e].y, r, s) + magic);
      }
    } else {
      // t = z * (r / sqrt(G)) + magic in one rounding: the nearest integer to the
      // exact product (r / sqrt(G) is exact for G = 4^k)
      const float rr = __fmul_rn(r, rnorm);
      const float2 r2 = make_float2(rr, rr), m2 = make_float2(magic, magic);
#pragma unroll
      for (int e = 0; e < EPT / 2; ++e) {
        const float2 t = __ffma2_rn(v[e], r2, m2);
        u[2 * e] = __float_as_uint(t.x);
        u[2 * e + 1] = __float_as_uint(t.y);
      }
    }
    // low bytes of four codes -> one word (natural order, or (0 2 4 6)(1 3 5 7) per 8 columns)
    uint32_t g[EPT / 4];
#pragma unroll
    for (int j = 0; j < EPT / 4; ++j) {
      const int b = STORE == STORE_INT8_PERM ? 8 * (j >> 1) + (j & 1) : 4 * j;
      const int st = STORE == STORE_INT8_PERM ? 2 : 1;
      g[j] = __byte_perm(__byte_perm(u[b], u[b + st], 0x5140), __byte_perm(u[b + 2 * st], u[b + 3 * st], 0x5140),
                         0x5410);
    }
    if (STORE == STORE_INT8_PERM) {
      int sum = 0;
#pragma unroll
      for (int j = 0; j < EPT / 4; ++j) sum = __dp4a((int)g[j], 0x01010101, sum);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      float* rs = red[2 * (it & 1) + 1];
      if (lane == 0) rs[tid >> 5] = __int_as_float(sum);
      __syncthreads();
      if (tid == 0) {
        int a = 0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) a += __float_as_int(rs[w]);
        rowsum[row] = a;
      }
    }

    if (e0 < K) {
      if (STORE == STORE_PACKED4) {
        // bytes hold u = q + 8 < 16: fold neighbours into nibbles, low nibble = even column
        uint32_t w[EPT / 8];
#pragma unroll
        for (int j = 0; j < EPT / 8; ++j) {
          const uint32_t ta = g[2 * j] | (g[2 * j] >> 4), tb = g[2 * j + 1] | (g[2 * j + 1] >> 4);
          w[j] = __byte_perm(ta, tb, 0x6420);
        }
        uint8_t* qr = q + row * (int64_t)(K >> 1) + (e0 >> 1);
        if ((K & 31) == 0 && e0 + EPT <= K) {          // whole, 16-byte aligned pieces
#pragma unroll
          for (int j = 0; j < EPT / 32; ++j)
            reinterpret_cast<uint4*>(qr)[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
        } else {
#pragma unroll
          for (int j = 0; j < EPT / 8; ++j)
            if (e0 + 8 * j < K) reinterpret_cast<uint32_t*>(qr)[j] = w[j];
        }
      } else {
        uint8_t* qr = q + row * (int64_t)K + e0;
        if ((K & 31) == 0 && e0 + EPT <= K) {
#pragma unroll
          for (int j = 0; j < EPT / 16; ++j)
            reinterpret_cast<uint4*>(qr)[j] = make_uint4(g[4 * j], g[4 * j + 1], g[4 * j + 2], g[4 * j + 3]);
        } else {
#pragma unroll
          for (int j = 0; j < EPT / 8; ++j)
            if (e0 + 8 * j < K) reinterpret_cast<uint2*>(qr)[j] = make_uint2(g[2 * j], g[2 * j + 1]);
        }
      }
    }
  }
}

}  // namespace rq
}  // namespace ck
