// K3, W4A8 decode GEMV for at most 8 activation rows: the streaming kernel.
//
//   acc[m, n] = sum_k xq[m, k] * (u[n, k] - 8)
//   y[m, n]   = bf16( (float(acc) * x_scale[m]) * w_scale[n] (+ bias[n]) )
//
// comfy-kitchen PR #182 "HIP port of #176: W4A8 decode GEMV and fused
// GatedDeltaNet decode", Description: int4 weights decoded in registers, int8
// dot products with int32 accumulation, the shared rowwise epilogue.
//
// The kernel reads the packed weights once from HBM and is built around what
// delays such a stream on B200:
//
// * Work split. CTA b of a grid of G (one per SM) owns output rows
//   [n0, n1), whole octets of rows split evenly, moved in 16-row tiles (the
//   m16 operand of mma.sync.m16n8k32 u8 x s8). A last tile that would run
//   past n1 is moved back to end at n1 (its first rows, already produced by
//   the previous tile, are computed again and not stored), so no CTA carries
//   more than one tile beyond the average.
// * Weight tiles. One tensor copy per tile through a 3-D view of the weight
//   matrix ([K/128 slices][rows][64 B], 64-byte swizzle, see wtile_addr).
//   The producer warp reads only constant data, so it does not wait for the
//   previous kernel: while that kernel runs, this CTA (co-resident: at most
//   half an SM's shared memory) fills its ring, `fill` tiles in flight at a
//   time, so that the activation loads made after the dependency wait do not
//   queue behind a whole ring of weight tiles. The weight scales and bias of
//   the CTA's rows come by bulk copy on their own barrier.
// * Compute. 8 consumer warps split K; each holds its activation fragments in
//   registers. A packed word costs two logical ops: the low nibbles (even k)
//   and the high nibbles left in place (16 x odd-k value) go to two MMAs with
//   separate accumulators, and the high sum, a multiple of 16, is shifted
//   back exactly. Nibbles enter unsigned: sum (u - 8) x = sum u x - 8 sum x.
// * Reduction. Each consumer warp adds its partial tile into a shared-memory
//   slot of that tile (integer adds commute: the result does not depend on
//   the order) and arrives on the tile's barrier; an epilogue warp waits for
//   the tiles in order and writes y. No warp waits for the epilogue, and no
//   memory fence sits on the consumers' path.
// All barrier waits are bounded; a timeout sets the device error word.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "ck_common.cuh"

namespace ck {
namespace w4s {

constexpr int kCons = 8;                        // consumer warps
constexpr int W_PROD = kCons, W_EPI = kCons + 1;
constexpr int kThreads = (kCons + 2) * 32;
constexpr int TR = 16;                          // weight rows per tile
constexpr int kMaxStages = 8;

struct Params {
  const int8_t* xq;               // (M, K)
  const float* xs;                // (M)
  const __nv_bfloat16* sw;        // (N)
  const __nv_bfloat16* bias;      // (N) or null
  __nv_bfloat16* y;               // (M, N)
  int M, K, N;
  int ns, stage_bytes;            // ring stages and their size (16 * K / 2, 1024-aligned)
  int max_rows, max_tiles;        // per CTA
  int fill;                       // ring tiles in flight at most while the ring first fills
  int off_acc, off_misc, off_bar; // shared-memory offsets
};

__device__ __forceinline__ void mma_u8s8(int (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Rows [n0, n1) of CTA b: whole octets, split evenly.
__device__ __forceinline__ void cta_rows(int N, int& n0, int& n1) {
  const int no = N >> 3;
  n0 = 8 * (int)((int64_t)blockIdx.x * no / gridDim.x);
  n1 = 8 * (int)((int64_t)(blockIdx.x + 1) * no / gridDim.x);
}

template <int CPW>   // 128-column chunks per consumer warp (K <= 8 * 128 * CPW)
__global__ void __launch_bounds__(kThreads, 2)
    w4a8_rowsplit_kernel(const __grid_constant__ CUtensorMap tm_w, const Params p) {
  extern __shared__ uint8_t sm_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));
  int* acc_sl = reinterpret_cast<int*>(sm + p.off_acc);                 // [max_tiles][16 rows][8 tokens]
  int* xsum = reinterpret_cast<int*>(sm + p.off_misc);                  // [8] sum_k xq[m, k]
  float* xsv = reinterpret_cast<float*>(xsum + 8);                      // [8] x_scale
  __nv_bfloat16* colv = reinterpret_cast<__nv_bfloat16*>(xsv + 8);     // [2][max_rows]: w_scale, bias
  int* abort_flag = reinterpret_cast<int*>(colv + 2 * p.max_rows);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + p.off_bar);
  uint64_t* wfree = full + kMaxStages;
  uint64_t* cbar = wfree + kMaxStages;
  uint64_t* tdone = cbar + 1;                                           // [max_tiles]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  int n0, n1;
  cta_rows(p.N, n0, n1);
  const int nrows = n1 - n0;
  const int ntile = (nrows + TR - 1) / TR;
  const int nchunk = p.K >> 7;
  const int ns = p.ns;
  const int wld = p.K >> 1;
  auto tstart = [&](int i) { return (i == ntile - 1 && nrows >= TR) ? n1 - TR : n0 + TR * i; };
  auto issue = [&](int i) {
    const int s = i % ns;
    mbar_arrive_expect_tx(&full[s], (uint32_t)(TR * wld));
    tma_load_3d(sm + s * p.stage_bytes, &tm_w, &full[s], 0, tstart(i), 0);
  };

  if (warp == W_PROD && lane == 0) {
    prefetch_tmap(&tm_w);
    for (int s = 0; s < ns; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&wfree[s], kCons);
    }
    mbar_init(cbar, 1);
    for (int i = 0; i < ntile; ++i) mbar_init(&tdone[i], kCons);
    *abort_flag = 0;
    fence_mbarrier_init();
    if (nrows > 0) {   // this CTA's weight scales (and bias): constant data
      mbar_arrive_expect_tx(cbar, (uint32_t)(2 * nrows * (p.bias ? 2 : 1)));
      bulk_load(colv, p.sw + n0, (uint32_t)(2 * nrows), cbar);
      if (p.bias) bulk_load(colv + p.max_rows, p.bias + n0, (uint32_t)(2 * nrows), cbar);
    } else {
      mbar_arrive(cbar);
    }
  }
  for (int i = threadIdx.x; i < ntile * TR * 8; i += blockDim.x) acc_sl[i] = 0;
  if (threadIdx.x < 8) xsum[threadIdx.x] = 0;
  __syncthreads();
  grid_dep_launch();
  volatile int* abort = abort_flag;

  if (warp == W_PROD) {
    // weight tiles only: no dependency wait
    if (lane == 0) {
      const int nfill = min(ns, ntile);
      int issued = 0;
      bool ok = true;
      for (int i = 0; i < nfill && ok; ++i) {
        if (i >= p.fill) ok = mbar_wait(&full[(i - p.fill) % ns], 0, abort, 35);
        if (ok) {
          issue(i);
          issued = i + 1;
        }
      }
      for (int i = nfill; i < ntile && ok; ++i) {
        if (!mbar_wait(&wfree[i % ns], ((i / ns) & 1) ^ 1, abort, 32)) break;
        issue(i);
        issued = i + 1;
      }
      if (*abort)   // the copies in flight land before the CTA exits
        for (int i = issued - 1; i >= 0 && i >= issued - ns; --i)
          mbar_wait(&full[i % ns], (i / ns) & 1, nullptr, 33, 100000000ull);
    }
  } else {
    // the activations, their scales and the output belong to the previous kernel until here
    grid_dep_wait();
    if (warp < kCons) {
      // fragments of token g for k = c*128 + 32t + 8j + (0 2 4 6) [.0] and + (1 3 5 7) [.1]
      uint32_t bf[CPW][4][2];
      const float xsl = lane < p.M ? __ldg(p.xs + lane) : 0.0f;
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
        for (int j = 0; j < 4; ++j) {
          bf[ci][j][0] = __byte_perm(xa[2 * j], xa[2 * j + 1], 0x6420);
          bf[ci][j][1] = __byte_perm(xa[2 * j], xa[2 * j + 1], 0x7531);
        }
      }
      xs_g += __shfl_xor_sync(0xffffffffu, xs_g, 1);
      xs_g += __shfl_xor_sync(0xffffffffu, xs_g, 2);
      // published to the epilogue through the tile barriers (each warp adds before arriving)
      if (t == 0) atomicAdd(&xsum[g], xs_g);
      if (warp == 0 && lane < 8) xsv[lane] = xsl;

      // row g of chunk c sits at line (c * 16 + g) of the swizzled tile; row g + 8 eight lines on
      const int wb = (warp * 16 + g) * 64 + ((t ^ ((g >> 1) & 3)) << 4);
      for (int i = 0; i < ntile; ++i) {
        const int s = i % ns;
        if (!warp_wait(&full[s], (i / ns) & 1, abort, 30)) break;
        const uint8_t* st = sm + s * p.stage_bytes;
        uint4 wg[CPW], wg8[CPW];
#pragma unroll
        for (int ci = 0; ci < CPW; ++ci) {
          const bool live = warp + kCons * ci < nchunk;
          wg[ci] = live ? *reinterpret_cast<const uint4*>(st + wb + (kCons * 1024) * ci) : make_uint4(0, 0, 0, 0);
          wg8[ci] = live ? *reinterpret_cast<const uint4*>(st + wb + (kCons * 1024) * ci + 512) : make_uint4(0, 0, 0, 0);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&wfree[s]);
        // word j of a lane holds k = 32t + 8j .. + 7 of the chunk, low nibbles at even k
        int alo[4] = {0, 0, 0, 0}, ahi[4] = {0, 0, 0, 0};
#pragma unroll
        for (int ci = 0; ci < CPW; ++ci) {
          if (warp + kCons * ci < nchunk) {
            const uint32_t u[4] = {wg[ci].x, wg[ci].y, wg[ci].z, wg[ci].w};
            const uint32_t v[4] = {wg8[ci].x, wg8[ci].y, wg8[ci].z, wg8[ci].w};
#pragma unroll
            for (int pr = 0; pr < 2; ++pr) {
              const uint32_t lo[4] = {u[2 * pr] & 0x0F0F0F0Fu, v[2 * pr] & 0x0F0F0F0Fu, u[2 * pr + 1] & 0x0F0F0F0Fu,
                                      v[2 * pr + 1] & 0x0F0F0F0Fu};
              const uint32_t hi[4] = {u[2 * pr] & 0xF0F0F0F0u, v[2 * pr] & 0xF0F0F0F0u, u[2 * pr + 1] & 0xF0F0F0F0u,
                                      v[2 * pr + 1] & 0xF0F0F0F0u};
              mma_u8s8(alo, lo, bf[ci][2 * pr][0], bf[ci][2 * pr + 1][0]);
              mma_u8s8(ahi, hi, bf[ci][2 * pr][1], bf[ci][2 * pr + 1][1]);
            }
          }
        }
        // accumulator of lane (g, t): weight rows g (e 0, 1) and g + 8 (e 2, 3) x tokens 2t, 2t + 1
        int* sl = acc_sl + i * (TR * 8);
        atomicAdd(&sl[g * 8 + 2 * t], alo[0] + (ahi[0] >> 4));
        atomicAdd(&sl[g * 8 + 2 * t + 1], alo[1] + (ahi[1] >> 4));
        atomicAdd(&sl[(g + 8) * 8 + 2 * t], alo[2] + (ahi[2] >> 4));
        atomicAdd(&sl[(g + 8) * 8 + 2 * t + 1], alo[3] + (ahi[3] >> 4));
        __syncwarp();
        if (lane == 0) mbar_arrive(&tdone[i]);   // release: the adds above reach the epilogue
      }
    } else {
      // epilogue: lane (r, h) writes weight row r of the tile for tokens h, h + 2, ...
      const bool cols_ok = ntile == 0 || warp_wait(cbar, 0, abort, 36);
      const bool has_bias = p.bias != nullptr;
      for (int i = 0; cols_ok && i < ntile; ++i) {
        if (!warp_wait(&tdone[i], 0, abort, 34)) break;
        const int* sl = acc_sl + i * (TR * 8);
        const int ts = tstart(i);
        const int lo = n0 + TR * i, hi = min(ts + TR, n1);   // rows no earlier tile wrote
        const int r = lane & 15;
        const int n = ts + r;
        if (n >= lo && n < hi) {
          const float swv = __bfloat162float(colv[n - n0]);
          const float bv = has_bias ? __bfloat162float(colv[p.max_rows + n - n0]) : 0.0f;
          for (int tk = lane >> 4; tk < p.M; tk += 2) {
            float v = __fmul_rn(__fmul_rn((float)(sl[r * 8 + tk] - 8 * xsum[tk]), xsv[tk]), swv);
            if (has_bias) v = __fadd_rn(v, bv);
            p.y[(int64_t)tk * p.N + n] = __float2bfloat16_rn(v);
          }
        }
      }
    }
  }
  __syncthreads();
}

}  // namespace w4s
}  // namespace ck
