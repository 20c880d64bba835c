// Streaming decode GEMVs (the fast path of K3 and K4 for K <= 4096).
//
// Both are bound by reading the packed weights once from HBM. One CTA per SM
// owns a contiguous, balanced range of weight-row tiles:
//   warp 8     producer: streams each tile's weight rows (contiguous bytes in
//              memory) into a ring of shared-memory stages with one 1-D
//              cp.async.bulk copy per tile (and, for AWQ, the tile's scales and
//              zeros with two 2-D TMA copies), several tiles ahead;
//   warps 0..7 consumers: split K. Each keeps the activation fragments of its
//              k-slice in registers for the whole kernel, decodes the weight
//              nibbles of every tile from shared memory in registers and runs
//              legacy warp-level MMAs (mma.sync) on them;
//   warp 9     epilogue: reduces the eight partial tiles in a fixed order,
//              applies the scales and writes y.
// All barrier waits are bounded; a timeout sets the device error word.
//
// For W4A8 with at most 8 activation rows, w4a8_stream_m8_kernel swaps the
// MMA operands (16 weight rows as the m16 operand) and moves each 16-row tile
// with ONE tensor copy through a 3-D view of the weight matrix (see
// wtile_addr); it also hands a weight stage back as soon as it has been read,
// with the partial sums passing through their own small ring.
//
// Back-to-back calls overlap: a CTA takes at most half of an SM's shared
// memory, the kernels are launched as programmatic dependents, each lets the
// next one be scheduled once its consumers have their activations (trigger
// note: a next call's weight prefetch would otherwise queue ahead of those
// loads), and a new call streams its first weight tiles (constant data) into
// its ring while the previous call is still running; only the activation
// reads and the output writes wait for the previous kernel (grid_dep_wait).
// A decode loop of GEMVs thus keeps HBM streaming across kernel boundaries
// instead of paying each launch's ramp-up and drain.
//
// W4A8 (comfy-kitchen PR #182, "Description": register-side int4 decode, int32
// accumulation, EpiRowwise): weights are the n8 operand of
// mma.m16n8k32.s8.u8 (8 weight rows per tile), the <= 16 activation rows the
// m16 operand; nibbles enter unsigned and sum (u - 8) x = sum u x - 8 sum x.
// AWQ W4A16 (comfy_kitchen/tensor/awq_w4a16.py, dequantize / _awq_forward):
// weights are the m16 operand of mma.m16n8k16 (16 rows per tile), decoded to
// exact (u - 8) bf16/fp16 values; per 64-column sub-block of a group,
// y += s * P + z * X with P = sum (u - 8) x and X = sum x.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ck_common.cuh"
#include "gemv_awq.cuh"

namespace ck {
namespace gstream {

constexpr int kCons = 8;
constexpr int W_PROD = kCons, W_EPI = kCons + 1;
constexpr int kThreads = (kCons + 2) * 32;
constexpr int kMaxStages = 8;
constexpr int kRed = 3;          // partial-sum slots of w4a8_stream_m8_kernel
constexpr int kRedBytes = kCons * 32 * 4 * 4;

// Shared-memory layout, computed on the host: [stages][red][misc][barriers].
struct Layout {
  int ns;            // stages
  int stage_bytes;
  int off_red;       // ns x kCons x 32 lanes x 4 values x 4 bytes
  int off_misc;
  int off_bar;
  int total;
};

// Tiles of w4a8_stream_m8_kernel: small copies are slow on this hardware (a
// 2 KB bulk copy per weight row runs at a fraction of HBM bandwidth), so a
// 16-row tile moves in one copy through a 3-D view of the weight matrix:
// 64-byte slices of the rows outermost, the tile's rows in the middle. It
// lands as [slice][row][64 B] with the 64-byte swizzle, which XORs each row's
// 16-byte chunks with (row >> 1) & 3, so MMA-fragment reads of eight rows at
// the same k hit different banks.
// Shared-memory address of byte b of weight row r in a tile of R rows copied
// as [b / 64][r][64 B] with the 64-byte swizzle (16-byte chunk c of a 64-byte
// line L stored at chunk c ^ ((L >> 1) & 3); R even, so (L >> 1) & 3 only
// depends on r).
template <int R>
__device__ __forceinline__ int wtile_addr(int r, int b) {
  return ((b >> 6) * R + r) * 64 + ((((b >> 4) & 3) ^ ((r >> 1) & 3)) << 4) + (b & 15);
}

__device__ __forceinline__ void mma_s8u8(int (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.u8.s32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// ============================================================== W4A8

struct W4A8Params {
  const int8_t* xq;              // (M, K)
  const float* xs;               // (M)
  const uint8_t* w;              // (N, K/2)
  const __nv_bfloat16* sw;       // (N)
  const __nv_bfloat16* bias;     // (N) or null
  __nv_bfloat16* y;              // (M, N)
  int M, K, N;
  int ntiles;                    // 8-row weight tiles
  int srow;                      // shared-memory row stride: K/2 + 64 (bank-conflict-free reads)
  Layout L;
};

template <int CPW>   // 128-column chunks per consumer warp (K <= 8 * 128 * CPW)
__global__ void __launch_bounds__(kThreads, 2) w4a8_stream_kernel(const W4A8Params p) {
  extern __shared__ __align__(1024) uint8_t sm[];
  const Layout& L = p.L;
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L.off_bar);
  uint64_t* consumed = full + kMaxStages;
  uint64_t* epi_done = consumed + kMaxStages;
  int* red = reinterpret_cast<int*>(sm + L.off_red);
  int* xsum_part = reinterpret_cast<int*>(sm + L.off_misc);           // [kCons][16]
  float* colv = reinterpret_cast<float*>(xsum_part + kCons * 16);     // [2][rows of this CTA]
  int* abort_flag = reinterpret_cast<int*>(colv + 2 * 8 * ((p.ntiles + gridDim.x - 1) / gridDim.x));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int t0 = (int)((int64_t)blockIdx.x * p.ntiles / gridDim.x);
  const int t1 = (int)((int64_t)(blockIdx.x + 1) * p.ntiles / gridDim.x);
  const int nt = t1 - t0;
  const int wld = p.K >> 1;
  const int nchunk = p.K >> 7;
  const int ns = L.ns;

  // the producer initialises the barriers and starts streaming at once: the
  // first ns tiles need no free-slot wait, so their copies overlap the prologue
  auto issue = [&](int i) {
    const int s = i % ns;
    const int tile = t0 + i;
    const int rows = min(8, p.N - 8 * tile);
    mbar_arrive_expect_tx(&full[s], (uint32_t)(rows * wld));
    for (int r = 0; r < rows; ++r)
      bulk_load(sm + s * L.stage_bytes + r * p.srow, p.w + ((int64_t)tile * 8 + r) * wld, (uint32_t)wld, &full[s]);
  };
  if (warp == W_PROD && lane == 0) {
    for (int s = 0; s < ns; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&consumed[s], kCons);
      mbar_init(&epi_done[s], 1);
    }
    *abort_flag = 0;
    fence_mbarrier_init();
    for (int i = 0; i < min(ns, nt); ++i) issue(i);
  }
  if (warp == W_EPI) {
    // this CTA's column scales and biases: constant data, read before the dependency wait
    const int r0 = 8 * t0, nr = min(8 * nt, p.N - r0);
    for (int r = lane; r < nr; r += 32) {
      colv[r] = __bfloat162float(p.sw[r0 + r]);
      colv[8 * ((p.ntiles + gridDim.x - 1) / gridDim.x) + r] = p.bias ? __bfloat162float(p.bias[r0 + r]) : 0.0f;
    }
  }
  grid_dep_wait();   // the activations and the output belong to the previous kernel until here

  uint32_t af[CPW][4][4];
  if (warp < kCons) {
    // activation fragments of this warp's chunks (tokens g and g + 8), and their sums
    int xs_g = 0, xs_g8 = 0;
#pragma unroll
    for (int ci = 0; ci < CPW; ++ci) {
      const int c = warp + kCons * ci;
      uint4 a0 = make_uint4(0, 0, 0, 0), a1 = a0, b0 = a0, b1 = a0;
      if (c < nchunk) {
        if (g < p.M) {
          const uint4* xp = reinterpret_cast<const uint4*>(p.xq + (int64_t)g * p.K + c * 128 + 32 * t);
          a0 = __ldg(xp);
          a1 = __ldg(xp + 1);
        }
        if (g + 8 < p.M) {
          const uint4* xp = reinterpret_cast<const uint4*>(p.xq + (int64_t)(g + 8) * p.K + c * 128 + 32 * t);
          b0 = __ldg(xp);
          b1 = __ldg(xp + 1);
        }
      }
      const uint32_t xa[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const uint32_t xb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        xs_g = __dp4a((int)xa[q], 0x01010101, xs_g);
        xs_g8 = __dp4a((int)xb[q], 0x01010101, xs_g8);
      }
      // mma step j, lane (g, t): fragment slot 4t + i holds k = c*128 + 32t + 8j + 2i,
      // slot 16 + 4t + i holds k + 1 (even / odd bytes of the 8 activations)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        af[ci][j][0] = __byte_perm(xa[2 * j], xa[2 * j + 1], 0x6420);
        af[ci][j][1] = __byte_perm(xb[2 * j], xb[2 * j + 1], 0x6420);
        af[ci][j][2] = __byte_perm(xa[2 * j], xa[2 * j + 1], 0x7531);
        af[ci][j][3] = __byte_perm(xb[2 * j], xb[2 * j + 1], 0x7531);
      }
    }
    xs_g += __shfl_xor_sync(0xffffffffu, xs_g, 1);
    xs_g += __shfl_xor_sync(0xffffffffu, xs_g, 2);
    xs_g8 += __shfl_xor_sync(0xffffffffu, xs_g8, 1);
    xs_g8 += __shfl_xor_sync(0xffffffffu, xs_g8, 2);
    if (t == 0) {
      xsum_part[warp * 16 + g] = xs_g;
      xsum_part[warp * 16 + g + 8] = xs_g8;
    }
  }
  __syncthreads();
  grid_dep_launch();   // once every consumer has its activations (the trigger note above)
  volatile int* abort = abort_flag;

  if (warp < kCons) {
    for (int i = 0; i < nt; ++i) {
      const int s = i % ns;
      if (!warp_wait(&full[s], (i / ns) & 1, abort, 20)) break;
      const uint8_t* st = sm + s * L.stage_bytes;
      int acc[4] = {0, 0, 0, 0};
#pragma unroll
      for (int ci = 0; ci < CPW; ++ci) {
        const int c = warp + kCons * ci;
        if (c < nchunk) {
          const uint4 wv = *reinterpret_cast<const uint4*>(st + g * p.srow + c * 64 + 16 * t);
          const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
          for (int j = 0; j < 4; ++j)   // word j: k = 32t + 8j .. +7; low nibbles = even k
            mma_s8u8(acc, af[ci][j], ww[j] & 0x0F0F0F0Fu, (ww[j] >> 4) & 0x0F0F0F0Fu);
        }
      }
      *reinterpret_cast<int4*>(red + ((s * kCons + warp) * 32 + lane) * 4) = make_int4(acc[0], acc[1], acc[2], acc[3]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&consumed[s]);
    }
  } else if (warp == W_PROD) {
    if (lane == 0) {
      int issued = min(ns, nt);
      for (int i = issued; i < nt; ++i) {
        if (!mbar_wait(&epi_done[i % ns], ((i / ns) & 1) ^ 1, abort, 21)) break;
        issue(i);
        issued = i + 1;
      }
      if (*abort)
        for (int i = issued - 1; i >= 0 && i >= issued - ns; --i)
          mbar_wait(&full[i % ns], (i / ns) & 1, nullptr, 23, 100000000ull);
    }
  } else {
    // epilogue: lane (g, t) finishes tokens g, g + 8 x weight rows 2t, 2t + 1 of each tile
    int xsg = 0, xsg8 = 0;
#pragma unroll
    for (int w = 0; w < kCons; ++w) {
      xsg += xsum_part[w * 16 + g];
      xsg8 += xsum_part[w * 16 + g + 8];
    }
    const float sg = g < p.M ? p.xs[g] : 0.0f, sg8 = g + 8 < p.M ? p.xs[g + 8] : 0.0f;
    const int cb = 8 * ((p.ntiles + gridDim.x - 1) / gridDim.x);
    const bool has_bias = p.bias != nullptr;
    for (int i = 0; i < nt; ++i) {
      const int s = i % ns;
      if (!warp_wait(&consumed[s], (i / ns) & 1, abort, 22)) break;
      int acc[4] = {0, 0, 0, 0};
#pragma unroll
      for (int w = 0; w < kCons; ++w) {
        const int4 v = *reinterpret_cast<const int4*>(red + ((s * kCons + w) * 32 + lane) * 4);
        acc[0] += v.x; acc[1] += v.y; acc[2] += v.z; acc[3] += v.w;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&epi_done[s]);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int token = g + 8 * (k >> 1);
        const int rl = 8 * i + 2 * t + (k & 1);              // row within this CTA's range
        const int n = 8 * t0 + rl;
        if (token < p.M && n < p.N) {
          const int a = acc[k] - 8 * ((k >> 1) ? xsg8 : xsg);
          float v = __fmul_rn(__fmul_rn((float)a, (k >> 1) ? sg8 : sg), colv[rl]);
          if (has_bias) v = __fadd_rn(v, colv[cb + rl]);
          p.y[(int64_t)token * p.N + n] = __float2bfloat16_rn(v);
        }
      }
    }
  }
  __syncthreads();
}

// ============================================== W4A8, at most 8 activation rows

__device__ __forceinline__ void mma_u8s8(int (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// The same product with the operands' roles swapped, for M <= 8: 16 weight
// rows per tile are the m16 (unsigned) operand and the activation rows the n8
// operand, so every MMA spends half of its work on real rows instead of
// 1/16 .. 1/4 (the legacy mma.sync path has little throughput to spare).
// Each lane holds, per 128-column chunk, the 16 bytes of weight rows g and
// g + 8 at k = 32t .. 32t + 31 of the chunk; MMA step j takes word j of them,
// its low nibbles (even k) in fragment slots 4t..4t+3 and its high nibbles
// (odd k) in slots 16+4t..16+4t+3; the activation fragments follow the same
// k order. Shared memory: [ns weight stages][kRed partial-sum slots][misc]
// [barriers full, wfree (kMaxStages); rfull, rfree (kRed)]: a weight stage is
// refilled once every consumer warp has read it; the epilogue reduces the
// partial sums from their own ring.
template <int CPW>   // 128-column chunks per consumer warp (K <= 8 * 128 * CPW)
__global__ void __launch_bounds__(kThreads, 2)
    w4a8_stream_m8_kernel(const __grid_constant__ CUtensorMap tm_w, const W4A8Params p) {
  extern __shared__ uint8_t sm_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));
  const Layout& L = p.L;
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L.off_bar);
  uint64_t* wfree = full + kMaxStages;
  uint64_t* rfull = wfree + kMaxStages;
  uint64_t* rfree = rfull + kRed;
  int* red = reinterpret_cast<int*>(sm + L.off_red);
  int* xsum_part = reinterpret_cast<int*>(sm + L.off_misc);           // [kCons][8]
  float* colv = reinterpret_cast<float*>(xsum_part + kCons * 8);      // [2][rows of this CTA]
  const int rows_cta = 16 * ((p.ntiles + gridDim.x - 1) / gridDim.x);
  int* abort_flag = reinterpret_cast<int*>(colv + 2 * rows_cta);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int t0 = (int)((int64_t)blockIdx.x * p.ntiles / gridDim.x);
  const int t1 = (int)((int64_t)(blockIdx.x + 1) * p.ntiles / gridDim.x);
  const int nt = t1 - t0;
  const int wld = p.K >> 1;
  const int nchunk = p.K >> 7;
  const int ns = L.ns;

  auto issue = [&](int i) {   // rows past N arrive as zeros (and are never stored)
    const int s = i % ns;
    mbar_arrive_expect_tx(&full[s], (uint32_t)(16 * wld));
    tma_load_3d(sm + s * L.stage_bytes, &tm_w, &full[s], 0, 16 * (t0 + i), 0);
  };
  if (warp == W_PROD && lane == 0) {
    prefetch_tmap(&tm_w);
    for (int s = 0; s < ns; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&wfree[s], kCons);
    }
    for (int r = 0; r < kRed; ++r) {
      mbar_init(&rfull[r], kCons);
      mbar_init(&rfree[r], 1);
    }
    *abort_flag = 0;
    fence_mbarrier_init();
    for (int i = 0; i < min(ns, nt); ++i) issue(i);
  }
  grid_dep_wait();   // the activations and the output belong to the previous kernel until here

  uint32_t bf[CPW][4][2];   // activation fragments of token g
  if (warp < kCons) {
    int xs_g = 0;
#pragma unroll
    for (int ci = 0; ci < CPW; ++ci) {
      const int c = warp + kCons * ci;
      uint4 a0 = make_uint4(0, 0, 0, 0), a1 = a0;
      if (c < nchunk && g < p.M) {
        const uint4* xp = reinterpret_cast<const uint4*>(p.xq + (int64_t)g * p.K + c * 128 + 32 * t);
        a0 = __ldg(xp);
        a1 = __ldg(xp + 1);
      }
      const uint32_t xa[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
      for (int q = 0; q < 8; ++q) xs_g = __dp4a((int)xa[q], 0x01010101, xs_g);
#pragma unroll
      for (int j = 0; j < 4; ++j) {   // k = c*128 + 32t + 8j + (0 2 4 6) and + (1 3 5 7)
        bf[ci][j][0] = __byte_perm(xa[2 * j], xa[2 * j + 1], 0x6420);
        bf[ci][j][1] = __byte_perm(xa[2 * j], xa[2 * j + 1], 0x7531);
      }
    }
    xs_g += __shfl_xor_sync(0xffffffffu, xs_g, 1);
    xs_g += __shfl_xor_sync(0xffffffffu, xs_g, 2);
    if (t == 0) xsum_part[warp * 8 + g] = xs_g;
  } else if (warp == W_EPI) {
    const int r0 = 16 * t0, nr = min(16 * nt, p.N - r0);
    for (int r = lane; r < nr; r += 32) {
      colv[r] = __bfloat162float(p.sw[r0 + r]);
      colv[rows_cta + r] = p.bias ? __bfloat162float(p.bias[r0 + r]) : 0.0f;
    }
  }
  __syncthreads();
  grid_dep_launch();   // once every consumer has its activations (the trigger note above)
  volatile int* abort = abort_flag;

  if (warp < kCons) {
    // = wtile_addr<16>(g, c * 64 + 16 * t) for c = warp + 8 * ci; row g + 8 is 8 lines on
    const int wb = (warp * 16 + g) * 64 + ((t ^ ((g >> 1) & 3)) << 4);
    for (int i = 0; i < nt; ++i) {
      const int s = i % ns, rs = i % kRed;
      if (!warp_wait(&full[s], (i / ns) & 1, abort, 30)) break;
      const uint8_t* st = sm + s * L.stage_bytes;
      uint4 wg[CPW], wg8[CPW];
#pragma unroll
      for (int ci = 0; ci < CPW; ++ci) {
        const bool live = warp + kCons * ci < nchunk;
        wg[ci] = live ? *reinterpret_cast<const uint4*>(st + wb + 8192 * ci) : make_uint4(0, 0, 0, 0);
        wg8[ci] = live ? *reinterpret_cast<const uint4*>(st + wb + 8192 * ci + 512) : make_uint4(0, 0, 0, 0);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&wfree[s]);
      int accc[CPW][4];
#pragma unroll
      for (int ci = 0; ci < CPW; ++ci) {
        accc[ci][0] = accc[ci][1] = accc[ci][2] = accc[ci][3] = 0;
        if (warp + kCons * ci < nchunk) {
          const uint32_t u[4] = {wg[ci].x, wg[ci].y, wg[ci].z, wg[ci].w};
          const uint32_t v[4] = {wg8[ci].x, wg8[ci].y, wg8[ci].z, wg8[ci].w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t a[4] = {u[j] & 0x0F0F0F0Fu, v[j] & 0x0F0F0F0Fu, (u[j] >> 4) & 0x0F0F0F0Fu,
                                   (v[j] >> 4) & 0x0F0F0F0Fu};
            mma_u8s8(accc[ci], a, bf[ci][j][0], bf[ci][j][1]);
          }
        }
      }
      int acc[4] = {0, 0, 0, 0};
#pragma unroll
      for (int ci = 0; ci < CPW; ++ci) {
        acc[0] += accc[ci][0]; acc[1] += accc[ci][1]; acc[2] += accc[ci][2]; acc[3] += accc[ci][3];
      }
      if (!warp_wait(&rfree[rs], ((i / kRed) & 1) ^ 1, abort, 31)) break;
      *reinterpret_cast<int4*>(red + ((rs * kCons + warp) * 32 + lane) * 4) = make_int4(acc[0], acc[1], acc[2], acc[3]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&rfull[rs]);
    }
  } else if (warp == W_PROD) {
    if (lane == 0) {
      int issued = min(ns, nt);
      for (int i = issued; i < nt; ++i) {
        if (!mbar_wait(&wfree[i % ns], ((i / ns) & 1) ^ 1, abort, 32)) break;
        issue(i);
        issued = i + 1;
      }
      if (*abort)
        for (int i = issued - 1; i >= 0 && i >= issued - ns; --i)
          mbar_wait(&full[i % ns], (i / ns) & 1, nullptr, 33, 100000000ull);
    }
  } else {
    // epilogue: lane (g, t) finishes weight rows g, g + 8 x tokens 2t, 2t + 1 of each tile
    int xs2[2] = {0, 0};
#pragma unroll
    for (int w = 0; w < kCons; ++w) {
      xs2[0] += xsum_part[w * 8 + 2 * t];
      xs2[1] += xsum_part[w * 8 + 2 * t + 1];
    }
    const float sx[2] = {2 * t < p.M ? p.xs[2 * t] : 0.0f, 2 * t + 1 < p.M ? p.xs[2 * t + 1] : 0.0f};
    const bool has_bias = p.bias != nullptr;
    for (int i = 0; i < nt; ++i) {
      const int rs = i % kRed;
      if (!warp_wait(&rfull[rs], (i / kRed) & 1, abort, 34)) break;
      int acc[4] = {0, 0, 0, 0};
#pragma unroll
      for (int w = 0; w < kCons; ++w) {
        const int4 v = *reinterpret_cast<const int4*>(red + ((rs * kCons + w) * 32 + lane) * 4);
        acc[0] += v.x; acc[1] += v.y; acc[2] += v.z; acc[3] += v.w;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&rfree[rs]);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int token = 2 * t + (k & 1);
        const int rl = 16 * i + g + 8 * (k >> 1);           // row within this CTA's range
        const int n = 16 * t0 + rl;
        if (token < p.M && n < p.N) {
          const int a = acc[k] - 8 * xs2[k & 1];
          float v = __fmul_rn(__fmul_rn((float)a, sx[k & 1]), colv[rl]);
          if (has_bias) v = __fadd_rn(v, colv[rows_cta + rl]);
          p.y[(int64_t)token * p.N + n] = __float2bfloat16_rn(v);
        }
      }
    }
  }
  __syncthreads();
}

// ============================================================== AWQ W4A16

struct AwqParams {
  const void* x;                 // (M, K) T
  const uint8_t* qw;             // (N, K/2)
  const void* bias;              // (N) T or null
  void* y;                       // (M, N) T
  int M, K, N, G;
  int gshift;                    // log2(G / 64): 64-column sub-block -> quantization group
  int ntiles;                    // 16-row weight tiles
  int w_bytes;                   // 16 * K / 2
  int sz_bytes;                  // (K / G) * 16 * 2: one of scales / zeros per stage
  int sz_stride;                 // sz_bytes rounded up to 128: TMA destinations are 128-byte aligned
  int srow;                      // shared-memory row stride: K/2 + 32 (bank-conflict-free reads)
  Layout L;
};

template <typename T, int SPW>   // 64-column sub-blocks per consumer warp (K <= 8 * 64 * SPW)
__global__ void __launch_bounds__(kThreads, 2)
    awq_stream_kernel(const __grid_constant__ CUtensorMap tm_s, const __grid_constant__ CUtensorMap tm_z,
                      const AwqParams p) {
  using Tr = awq::Traits<T>;
  extern __shared__ __align__(1024) uint8_t sm[];
  const Layout& L = p.L;
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L.off_bar);
  uint64_t* consumed = full + kMaxStages;
  uint64_t* epi_done = consumed + kMaxStages;
  float* red = reinterpret_cast<float*>(sm + L.off_red);
  float* colb = reinterpret_cast<float*>(sm + L.off_misc);          // bias of this CTA's rows
  int* abort_flag = reinterpret_cast<int*>(colb + 16 * ((p.ntiles + gridDim.x - 1) / gridDim.x));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int t0 = (int)((int64_t)blockIdx.x * p.ntiles / gridDim.x);
  const int t1 = (int)((int64_t)(blockIdx.x + 1) * p.ntiles / gridDim.x);
  const int nt = t1 - t0;
  const int wld = p.K >> 1;
  const int nsub = p.K >> 6;
  const int ns = L.ns;
  const T* x = reinterpret_cast<const T*>(p.x);

  // the producer initialises the barriers and starts streaming at once (see the W4A8 kernel)
  auto issue = [&](int i) {
    const int s = i % ns;
    const int tile = t0 + i;
    const int rows = min(16, p.N - 16 * tile);
    uint8_t* st = sm + s * L.stage_bytes;
    mbar_arrive_expect_tx(&full[s], (uint32_t)(rows * wld) + 2u * (uint32_t)p.sz_bytes);
    for (int r = 0; r < rows; ++r)
      bulk_load(st + r * p.srow, p.qw + ((int64_t)tile * 16 + r) * wld, (uint32_t)wld, &full[s]);
    tma_load_2d(st + p.w_bytes, &tm_s, &full[s], 16 * tile, 0);
    tma_load_2d(st + p.w_bytes + p.sz_stride, &tm_z, &full[s], 16 * tile, 0);
  };
  if (warp == W_PROD && lane == 0) {
    prefetch_tmap(&tm_s);
    prefetch_tmap(&tm_z);
    for (int s = 0; s < ns; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&consumed[s], kCons);
      mbar_init(&epi_done[s], 1);
    }
    *abort_flag = 0;
    fence_mbarrier_init();
    for (int i = 0; i < min(ns, nt); ++i) issue(i);
  }
  if (warp == W_EPI) {   // bias of this CTA's rows: constant data, read before the dependency wait
    const int r0 = 16 * t0, nr = min(16 * nt, p.N - r0);
    for (int r = lane; r < nr; r += 32) colb[r] = p.bias ? Tr::tof(reinterpret_cast<const T*>(p.bias)[r0 + r]) : 0.0f;
  }
  grid_dep_wait();   // the activations and the output belong to the previous kernel until here

  uint32_t bp[SPW][8];    // activation fragments (token g, k = sb*64 + 16t + (k, k+4) pairs)
  float X[SPW][2];        // sum_k x for tokens 2t, 2t + 1 over each sub-block
  if (warp < kCons) {
    const uint32_t ones[4] = {Tr::kOnes, Tr::kOnes, Tr::kOnes, Tr::kOnes};
#pragma unroll
    for (int i = 0; i < SPW; ++i) {
      const int sb = warp + kCons * i;
      uint4 xa = make_uint4(0, 0, 0, 0), xb = xa;
      if (sb < nsub && g < p.M) {
        const T* xp = x + (int64_t)g * p.K + sb * 64 + 16 * t;
        xa = __ldg(reinterpret_cast<const uint4*>(xp));
        xb = __ldg(reinterpret_cast<const uint4*>(xp + 8));
      }
      bp[i][0] = __byte_perm(xa.x, xa.z, 0x5410);  // (0, 4)
      bp[i][1] = __byte_perm(xa.x, xa.z, 0x7632);  // (1, 5)
      bp[i][2] = __byte_perm(xa.y, xa.w, 0x5410);  // (2, 6)
      bp[i][3] = __byte_perm(xa.y, xa.w, 0x7632);  // (3, 7)
      bp[i][4] = __byte_perm(xb.x, xb.z, 0x5410);  // (8, 12)
      bp[i][5] = __byte_perm(xb.x, xb.z, 0x7632);  // (9, 13)
      bp[i][6] = __byte_perm(xb.y, xb.w, 0x5410);  // (10, 14)
      bp[i][7] = __byte_perm(xb.y, xb.w, 0x7632);  // (11, 15)
      float Xc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int j = 0; j < 4; ++j) Tr::mma(Xc, ones, bp[i][2 * j], bp[i][2 * j + 1]);
      X[i][0] = Xc[0];
      X[i][1] = Xc[1];
    }
  }
  __syncthreads();
  grid_dep_launch();   // once every consumer has its activations (the trigger note above)
  volatile int* abort = abort_flag;

  if (warp < kCons) {
    for (int i = 0; i < nt; ++i) {
      const int s = i % ns;
      if (!warp_wait(&full[s], (i / ns) & 1, abort, 24)) break;
      const uint8_t* st = sm + s * L.stage_bytes;
      const T* sc = reinterpret_cast<const T*>(st + p.w_bytes);                 // [K/G][16]
      const T* zr = reinterpret_cast<const T*>(st + p.w_bytes + p.sz_stride);
      float yacc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int i2 = 0; i2 < SPW; ++i2) {
        const int sb = warp + kCons * i2;
        if (sb < nsub) {
          const uint2 w0 = *reinterpret_cast<const uint2*>(st + g * p.srow + sb * 32 + 8 * t);
          const uint2 w1 = *reinterpret_cast<const uint2*>(st + (g + 8) * p.srow + sb * 32 + 8 * t);
          const uint32_t r0[2] = {w0.x, w0.y}, r1[2] = {w1.x, w1.y};
          // weights enter the MMA as (offset + u); the group's zero term takes the offset back out
          float P[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int wd = j >> 1, s0 = (2 * j) & 3, s1 = (2 * j + 1) & 3;
            uint32_t a[4];
            a[0] = awq::nib_pair_raw<T>(r0[wd], s0);
            a[1] = awq::nib_pair_raw<T>(r1[wd], s0);
            a[2] = awq::nib_pair_raw<T>(r0[wd], s1);
            a[3] = awq::nib_pair_raw<T>(r1[wd], s1);
            Tr::mma(P, a, bp[i2][2 * j], bp[i2][2 * j + 1]);
          }
          const int grp = sb >> p.gshift;
          constexpr float kOff = awq::RawOffset<T>::v;
          const float sa = Tr::tof(sc[grp * 16 + g]), sbb = Tr::tof(sc[grp * 16 + g + 8]);
          const float za = fmaf(-kOff, sa, Tr::tof(zr[grp * 16 + g]));
          const float zb = fmaf(-kOff, sbb, Tr::tof(zr[grp * 16 + g + 8]));
          yacc[0] += sa * P[0] + za * X[i2][0];
          yacc[1] += sa * P[1] + za * X[i2][1];
          yacc[2] += sbb * P[2] + zb * X[i2][0];
          yacc[3] += sbb * P[3] + zb * X[i2][1];
        }
      }
      *reinterpret_cast<float4*>(red + ((s * kCons + warp) * 32 + lane) * 4) = make_float4(yacc[0], yacc[1], yacc[2], yacc[3]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&consumed[s]);
    }
  } else if (warp == W_PROD) {
    if (lane == 0) {
      int issued = min(ns, nt);
      for (int i = issued; i < nt; ++i) {
        if (!mbar_wait(&epi_done[i % ns], ((i / ns) & 1) ^ 1, abort, 25)) break;
        issue(i);
        issued = i + 1;
      }
      if (*abort)
        for (int i = issued - 1; i >= 0 && i >= issued - ns; --i)
          mbar_wait(&full[i % ns], (i / ns) & 1, nullptr, 26, 100000000ull);
    }
  } else {
    // epilogue: lane (g, t) finishes weight rows g, g + 8 x tokens 2t, 2t + 1 of each tile
    T* y = reinterpret_cast<T*>(p.y);
    for (int i = 0; i < nt; ++i) {
      const int s = i % ns;
      if (!warp_wait(&consumed[s], (i / ns) & 1, abort, 27)) break;
      float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int w = 0; w < kCons; ++w) {
        const float4 v = *reinterpret_cast<const float4*>(red + ((s * kCons + w) * 32 + lane) * 4);
        acc[0] += v.x; acc[1] += v.y; acc[2] += v.z; acc[3] += v.w;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&epi_done[s]);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int rl = 16 * i + g + 8 * (k >> 1);
        const int n = 16 * t0 + rl;
        const int token = 2 * t + (k & 1);
        if (token < p.M && n < p.N) y[(int64_t)token * p.N + n] = Tr::fromf(acc[k] + colb[rl]);
      }
    }
  }
  __syncthreads();
}

}  // namespace gstream
}  // namespace ck
