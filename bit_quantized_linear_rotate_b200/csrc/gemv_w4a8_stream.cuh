// K3, W4A8 decode GEMV for at most 32 activation rows: the streaming kernel.
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
//   m16 operand of mma.sync.m16n8k32 u8 x s8; the tokens, in NT groups of 8,
//   are the n8 operands). A last tile that would run past n1 is moved back to
//   end at n1 (its first rows, already produced by the previous tile, are
//   computed again and not stored), so no CTA carries more than one tile
//   beyond the average.
// * Weight tiles. One tensor copy per tile through a 3-D view of the weight
//   matrix ([K/128 slices][rows][64 B], 64-byte swizzle, see wtile_addr).
//   The producer warp reads only constant data, so it does not wait for the
//   previous kernel: while that kernel runs, this CTA (for NT = 1 at most
//   half an SM's shared memory and registers, so that it is co-resident with
//   the previous call's CTA) fills its ring, `fill` tiles in flight at a
//   time, so that the activation loads made after the dependency wait do not
//   queue behind a whole ring of weight tiles. The weight scales and bias of
//   the CTA's rows come by bulk copy on their own barrier.
// * Dependent launch. The next kernel on the stream is released only once
//   every consumer warp of the CTA has its activation fragments and has
//   finished the first tile: a next call's weight prefetch would otherwise
//   queue ahead of this call's activation loads (measured: 6.8 -> 6.3 us a
//   call at M = 1..4, K = 4096, N = 12288).
// * Compute. NC consumer warps split K (8 for one token group, 16 and one CTA
//   per SM for more); each holds its activation fragments in registers (read
//   as int8, or as int4 codes packed two per byte for the small-batch linear,
//   A4). A packed weight word costs two logical ops: the low nibbles (even k)
//   and the high nibbles (odd k) go to two MMAs; with one token group the
//   high nibbles stay in place (16 x the value) in an accumulator of their
//   own, shifted back exactly at the end, with more groups they are shifted
//   down first. Nibbles enter unsigned: sum (u - 8) x = sum u x - 8 sum x.
// * Reduction. Each consumer warp adds its partial tile into a shared-memory
//   slot of that tile (integer adds commute: the result does not depend on
//   the order). One token group: the warp arrives on the tile's barrier and
//   an epilogue warp waits for the tiles in order and writes y; no warp waits
//   for the epilogue, and no memory fence sits on the consumers' path. More
//   groups: the consumer warps meet at a named barrier and write the tile's
//   outputs themselves, one per lane.
// All barrier waits are bounded; a timeout sets the device error word.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "ck_common.cuh"

namespace ck {
namespace w4s {

constexpr int TR = 16;                          // weight rows per tile
constexpr int TS = TR + 4;                      // words per token in a tile slot (bank-conflict-free adds)
constexpr int kMaxTokens = 32;
constexpr int kMaxStages = 8;

// Consumer warps for NT token groups, and the CTA's threads (plus producer and epilogue warps).
// One token group: 8 consumer warps, a producer and an epilogue warp, two CTAs per SM. More
// groups: 16 consumer warps that also write the outputs, a producer, one CTA per SM.
__host__ __device__ constexpr int cons_warps(int nt) { return nt == 1 ? 8 : 16; }
__host__ __device__ constexpr int threads_for(int nt) { return (cons_warps(nt) + (nt == 1 ? 2 : 1)) * 32; }

struct Params {
  const int8_t* xq;               // (M, K) int8, or (M, K / 2) packed int4 codes (A4)
  const float* xs;                // (M)
  const __nv_bfloat16* sw;        // (N)
  const __nv_bfloat16* bias;      // (N) or null
  __nv_bfloat16* y;               // (M, N)
  int M, K, N;                    // M <= 8 * NT
  int ns, stage_bytes;            // ring stages and their size (16 * K / 2, 1024-aligned)
  int max_rows, max_tiles;        // per CTA
  int fill;                       // ring tiles in flight at most while the ring first fills
  int off_acc, off_misc, off_bar; // shared-memory offsets
};

// The consumer warps' named barrier (id 1; __syncthreads takes id 0).
template <int NC>
__device__ __forceinline__ void cons_bar_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(NC * 32) : "memory");
}

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

// NT: token groups of 8 (M <= 8 NT); CPW: 128-column chunks per consumer warp
// (K <= NC * 128 * CPW).
// A4: the activations are int4 codes packed two per byte (offset binary u = q + 8,
// low nibble = even column, (M, K / 2) bytes) instead of int8: half the bytes every
// CTA pulls from L2.
template <int NT, int CPW, bool A4 = false>
__global__ void __launch_bounds__(threads_for(NT), NT == 1 ? 2 : 1)
    w4a8_rowsplit_kernel(const __grid_constant__ CUtensorMap tm_w, const Params p) {
  constexpr int NC = cons_warps(NT), W_PROD = NC;   // then the epilogue warp, NC + 1, if NT == 1
  constexpr bool kConsEpi = NT > 1;                 // the consumer warps write the outputs
  constexpr int SLOT = NT * 8 * TS;   // words of one tile's slot: [token][TS], rows 0..15 used
  extern __shared__ uint8_t sm_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));
  int* acc_sl = reinterpret_cast<int*>(sm + p.off_acc);                 // [max_tiles][SLOT]
  int* xsum = reinterpret_cast<int*>(sm + p.off_misc);                  // [32] sum_k xq[m, k]
  float* xsv = reinterpret_cast<float*>(xsum + kMaxTokens);             // [32] x_scale
  __nv_bfloat16* colv = reinterpret_cast<__nv_bfloat16*>(xsv + kMaxTokens);   // [2][max_rows]: w_scale, bias
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
      mbar_init(&wfree[s], NC);
    }
    mbar_init(cbar, 1);
    for (int i = 0; i < ntile; ++i) mbar_init(&tdone[i], NC);
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
  for (int i = threadIdx.x; i < ntile * SLOT; i += blockDim.x) acc_sl[i] = 0;
  if (threadIdx.x < kMaxTokens) xsum[threadIdx.x] = 0;
  __syncthreads();
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
    if (warp < NC) {
      // fragments of token g + 8 nt for k = c*128 + 32t + 8j + (0 2 4 6) [.0] and + (1 3 5 7) [.1].
      // Every load is issued before the first is used (one L2 round trip, not one per chunk and
      // group); the raw words land in the fragment registers and are permuted in place.
      uint32_t bf[CPW][4][2][NT];
      const float xsl = lane < p.M ? __ldg(p.xs + lane) : 0.0f;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int tok = g + 8 * nt;
#pragma unroll
        for (int ci = 0; ci < CPW; ++ci) {
          const int c = warp + NC * ci;
          uint4 a0 = make_uint4(0, 0, 0, 0), a1 = a0;
          if constexpr (A4) {   // word j: the 8 codes of k = 32t + 8j .. + 7; u = 8 (code 0) where absent
            a0 = make_uint4(0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u);
            if (c < nchunk && tok < p.M)
              a0 = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(p.xq) +
                                                        (int64_t)tok * (p.K >> 1) + c * 64 + 16 * t));
            bf[ci][0][0][nt] = a0.x; bf[ci][1][0][nt] = a0.y; bf[ci][2][0][nt] = a0.z; bf[ci][3][0][nt] = a0.w;
          } else {
            if (c < nchunk && tok < p.M) {
              const uint4* xp = reinterpret_cast<const uint4*>(p.xq + (int64_t)tok * p.K + c * 128 + 32 * t);
              a0 = __ldg(xp);
              a1 = __ldg(xp + 1);
            }
            bf[ci][0][0][nt] = a0.x; bf[ci][0][1][nt] = a0.y; bf[ci][1][0][nt] = a0.z; bf[ci][1][1][nt] = a0.w;
            bf[ci][2][0][nt] = a1.x; bf[ci][2][1][nt] = a1.y; bf[ci][3][0][nt] = a1.z; bf[ci][3][1][nt] = a1.w;
          }
        }
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        int xs_g = 0;
#pragma unroll
        for (int ci = 0; ci < CPW; ++ci)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            if constexpr (A4) {
              // even / odd k nibbles to signed bytes: (u + 0x78) ^ 0x80 = u - 8, no carry between bytes
              const uint32_t w = bf[ci][j][0][nt];
              const uint32_t ev = ((w & 0x0F0F0F0Fu) + 0x78787878u) ^ 0x80808080u;
              const uint32_t od = (((w >> 4) & 0x0F0F0F0Fu) + 0x78787878u) ^ 0x80808080u;
              xs_g = __dp4a((int)ev, 0x01010101, __dp4a((int)od, 0x01010101, xs_g));
              bf[ci][j][0][nt] = ev;
              bf[ci][j][1][nt] = od;
            } else {
              const uint32_t w0 = bf[ci][j][0][nt], w1 = bf[ci][j][1][nt];
              xs_g = __dp4a((int)w0, 0x01010101, __dp4a((int)w1, 0x01010101, xs_g));
              bf[ci][j][0][nt] = __byte_perm(w0, w1, 0x6420);
              bf[ci][j][1][nt] = __byte_perm(w0, w1, 0x7531);
            }
          }
        xs_g += __shfl_xor_sync(0xffffffffu, xs_g, 1);
        xs_g += __shfl_xor_sync(0xffffffffu, xs_g, 2);
        // published to the epilogue through the tile barriers (each warp adds before arriving)
        if (t == 0) atomicAdd(&xsum[g + 8 * nt], xs_g);
      }
      if (warp == 0) xsv[lane] = xsl;

      // row g of chunk c sits at line (c * 16 + g) of the swizzled tile; row g + 8 eight lines on
      const int wb = (warp * 16 + g) * 64 + ((t ^ ((g >> 1) & 3)) << 4);
      // With consumer-written outputs the consumer warps meet at a named barrier once per tile;
      // after a timeout a warp skips the work but still takes every barrier, so that all of
      // them reach the same count (every other wait is bounded).
      bool ok = true;
      for (int i = 0; i < ntile; ++i) {
        const int s = i % ns;
        if constexpr (kConsEpi) {
          ok = ok && warp_wait(&full[s], (i / ns) & 1, abort, 30);
          if (!ok) {
            cons_bar_sync<NC>();
            continue;
          }
        } else {
          if (!warp_wait(&full[s], (i / ns) & 1, abort, 30)) break;
        }
        const uint8_t* st = sm + s * p.stage_bytes;
        // with four token groups the activation fragments fill most registers: the weight words
        // of a chunk are read just before its MMAs and the stage is handed back after the last
        constexpr bool kEarlyFree = NT < 4;
        uint4 wg[CPW], wg8[CPW];
        auto load_w = [&](int ci) {
          const bool live = warp + NC * ci < nchunk;
          wg[ci] = live ? *reinterpret_cast<const uint4*>(st + wb + (NC * 1024) * ci) : make_uint4(0, 0, 0, 0);
          wg8[ci] = live ? *reinterpret_cast<const uint4*>(st + wb + (NC * 1024) * ci + 512) : make_uint4(0, 0, 0, 0);
        };
        if constexpr (kEarlyFree) {
#pragma unroll
          for (int ci = 0; ci < CPW; ++ci) load_w(ci);
          __syncwarp();
          if (lane == 0) mbar_arrive(&wfree[s]);
        }
        // word j of a lane holds k = 32t + 8j .. + 7 of the chunk, low nibbles at even k. One token
        // group: the high nibbles stay in place (16 x the odd-k value) and get an accumulator of
        // their own, shifted back exactly at the end. More groups: the high nibbles are shifted
        // down once per word, and one accumulator per group keeps the registers in bounds.
        constexpr bool kSplitHi = NT == 1;
        int alo[NT][4], ahi[kSplitHi ? NT : 1][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) alo[nt][e] = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) ahi[0][e] = 0;
#pragma unroll
        for (int ci = 0; ci < CPW; ++ci) {
          if constexpr (!kEarlyFree) load_w(ci);
          if (warp + NC * ci < nchunk) {
            const uint32_t u[4] = {wg[ci].x, wg[ci].y, wg[ci].z, wg[ci].w};
            const uint32_t v[4] = {wg8[ci].x, wg8[ci].y, wg8[ci].z, wg8[ci].w};
#pragma unroll
            for (int pr = 0; pr < 2; ++pr) {
              const uint32_t lo[4] = {u[2 * pr] & 0x0F0F0F0Fu, v[2 * pr] & 0x0F0F0F0Fu, u[2 * pr + 1] & 0x0F0F0F0Fu,
                                      v[2 * pr + 1] & 0x0F0F0F0Fu};
              if constexpr (kSplitHi) {
                const uint32_t hi[4] = {u[2 * pr] & 0xF0F0F0F0u, v[2 * pr] & 0xF0F0F0F0u, u[2 * pr + 1] & 0xF0F0F0F0u,
                                        v[2 * pr + 1] & 0xF0F0F0F0u};
                mma_u8s8(alo[0], lo, bf[ci][2 * pr][0][0], bf[ci][2 * pr + 1][0][0]);
                mma_u8s8(ahi[0], hi, bf[ci][2 * pr][1][0], bf[ci][2 * pr + 1][1][0]);
              } else {
                const uint32_t hi[4] = {(u[2 * pr] >> 4) & 0x0F0F0F0Fu, (v[2 * pr] >> 4) & 0x0F0F0F0Fu,
                                        (u[2 * pr + 1] >> 4) & 0x0F0F0F0Fu, (v[2 * pr + 1] >> 4) & 0x0F0F0F0Fu};
                // the groups' MMAs interleave, so that two on one accumulator are NT apart
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma_u8s8(alo[nt], lo, bf[ci][2 * pr][0][nt], bf[ci][2 * pr + 1][0][nt]);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma_u8s8(alo[nt], hi, bf[ci][2 * pr][1][nt], bf[ci][2 * pr + 1][1][nt]);
              }
            }
          }
        }
        if constexpr (kSplitHi) {
#pragma unroll
          for (int e = 0; e < 4; ++e) alo[0][e] += ahi[0][e] >> 4;
        }
        if constexpr (!kEarlyFree) {
          __syncwarp();
          if (lane == 0) mbar_arrive(&wfree[s]);
        }
        // accumulator of lane (g, t): weight rows g (e 0, 1) and g + 8 (e 2, 3) x tokens
        // 8 nt + 2t, + 1; slot word (token * TS + row): the 32 lanes hit 32 banks
        int* sl = acc_sl + i * SLOT;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          int* so = sl + (8 * nt + 2 * t) * TS + g;
          atomicAdd(so, alo[nt][0]);
          atomicAdd(so + TS, alo[nt][1]);
          atomicAdd(so + 8, alo[nt][2]);
          atomicAdd(so + TS + 8, alo[nt][3]);
        }
        if constexpr (!kConsEpi) {
          __syncwarp();
          if (lane == 0) mbar_arrive(&tdone[i]);   // release: the adds above reach the epilogue
        } else {
          // once every consumer warp has added its part, output o = 32 warp + lane of the
          // tile's 16 x 8 NT: token o / 16, row o % 16 (a half warp stores 16 adjacent rows)
          if (i == 0) ok = warp_wait(cbar, 0, abort, 36);
          cons_bar_sync<NC>();
          if (!ok) continue;
          if (i == 0) grid_dep_launch();   // every consumer warp is past its activation loads
          const int o = warp * 32 + lane;
          const int tk = o >> 4, r = o & 15;
          const int ts = tstart(i);
          const int lo = n0 + TR * i, hi = min(ts + TR, n1);   // rows no earlier tile wrote
          const int n = ts + r;
          if (tk < p.M && n >= lo && n < hi) {
            const float swv = __bfloat162float(colv[n - n0]);
            float v = __fmul_rn(__fmul_rn((float)(sl[tk * TS + r] - 8 * xsum[tk]), xsv[tk]), swv);
            if (p.bias != nullptr) v = __fadd_rn(v, __bfloat162float(colv[p.max_rows + n - n0]));
            p.y[(int64_t)tk * p.N + n] = __float2bfloat16_rn(v);
          }
        }
      }
    } else if constexpr (!kConsEpi) {
      // epilogue: lane (r, h) writes weight row r of the tile for tokens h, h + 2, ... The
      // per-token terms are read once (the token sums are complete once every consumer warp
      // has arrived on the first tile's barrier), and each tile's slot values are read in one
      // batch before any output is formed.
      constexpr int TPL = 4 * NT;   // tokens per lane
      const bool cols_ok = ntile == 0 || warp_wait(cbar, 0, abort, 36);
      const bool has_bias = p.bias != nullptr;
      const int r = lane & 15, h = lane >> 4;
      int xo[TPL];
      float xsc[TPL];
      for (int i = 0; cols_ok && i < ntile; ++i) {
        if (!warp_wait(&tdone[i], 0, abort, 34)) break;
        if (i == 0) grid_dep_launch();   // every consumer warp is past its activation loads
        if (i == 0) {
#pragma unroll
          for (int q = 0; q < TPL; ++q) {
            xo[q] = 8 * xsum[h + 2 * q];
            xsc[q] = xsv[h + 2 * q];
          }
        }
        const int* sl = acc_sl + i * SLOT;
        int a[TPL];
#pragma unroll
        for (int q = 0; q < TPL; ++q) a[q] = sl[(h + 2 * q) * TS + r];
        const int ts = tstart(i);
        const int lo = n0 + TR * i, hi = min(ts + TR, n1);   // rows no earlier tile wrote
        const int n = ts + r;
        if (n >= lo && n < hi) {
          const float swv = __bfloat162float(colv[n - n0]);
          const float bv = has_bias ? __bfloat162float(colv[p.max_rows + n - n0]) : 0.0f;
#pragma unroll
          for (int q = 0; q < TPL; ++q) {
            const int tk = h + 2 * q;
            if (tk < p.M) {
              float v = __fmul_rn(__fmul_rn((float)(a[q] - xo[q]), xsc[q]), swv);
              if (has_bias) v = __fadd_rn(v, bv);
              p.y[(int64_t)tk * p.N + n] = __float2bfloat16_rn(v);
            }
          }
        }
      }
    }
  }
  __syncthreads();
}

}  // namespace w4s
}  // namespace ck
