// Host side of the C ABI declared in include/ck.h: argument validation, TMA
// tensor maps, kernel selection and launches. Everything is enqueued on the
// caller's stream; nothing here allocates, frees or synchronises, except
// ck_device_error_check (documented as synchronising).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <algorithm>
#include <atomic>
#include <cstring>
#include <mutex>
#include <string>
#include <utility>

#include "../../include/ck.h"
#include "ck_common.cuh"
#include "gemm_w4a4_sm100.cuh"
#include "gemv_awq.cuh"
#include "gemv_stream.cuh"
#include "gemv_w4a8.cuh"
#include "gemv_w4a8_stream.cuh"
#include "gemv_w4a8_tc.cuh"
#include "rotate_quant.cuh"
#include "rotate_quant_general.cuh"

namespace {

thread_local std::string g_last_error;

ck_status fail(ck_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

ck_status ok() {
  g_last_error.clear();
  return CK_OK;
}

ck_status launch_status(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(CK_ERR_CUDA, "%s: launch failed: %s", what, cudaGetErrorString(e));
  return ok();
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
bool is_pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }
cudaStream_t S(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// Launches `kern` on `st` as a programmatic dependent of the previous kernel in
// the stream: it may start while that kernel finishes and orders itself after
// it with grid_dep_wait (ck_common.cuh).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// ------------------------------------------------------------- tensor maps

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Row-major matrix (rows x cols elements of `dt`) with row stride `ld` bytes,
// box = (box_cols x box_rows) elements.
ck_status make_tmap(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t ld,
                    uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw,
                    CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_UINT8) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return fail(CK_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {ld};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(CK_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return CK_OK;
}

// 3-D tensor map over a packed weight matrix (N rows of K/2 bytes) viewed as
// [K/128 slices of 64 bytes][N rows][64 bytes], slices outermost, with the
// 64-byte swizzle; one box is `rows` rows x all slices (the streaming GEMVs'
// tile layout, gemv_stream.cuh).
ck_status make_tmap_wtile(CUtensorMap* m, const void* w, uint64_t N, uint64_t K, uint32_t rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return fail(CK_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[3] = {64, N, K / 128};
  const cuuint64_t strides[2] = {K / 2, 64};
  const cuuint32_t box[3] = {64, rows, (cuuint32_t)(K / 128)};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(w), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(CK_ERR_CUDA, "cuTensorMapEncodeTiled (weight tiles) failed (%d)", (int)r);
  return CK_OK;
}

// Shared-memory layout of w4a8_stream_m8_kernel: as many 1024-aligned weight
// stages as fit, then kRed partial-sum slots, the misc block and the barriers.
ck::gstream::Layout stream_layout_m8(int stage_bytes, int misc_bytes);

// Dynamic shared memory of one streaming-GEMV CTA: two CTAs (plus the 1 KB
// the runtime reserves per CTA) fit in an SM's 228 KB.
constexpr int kStreamSmemMax = 112 * 1024;

// The host-side caches below hold per-device facts (a kernel attribute that was
// set, an occupancy, an SM count). Each entry is an atomic, so calls from
// several host threads may race to fill one; they compute the same value, and
// setting a kernel attribute twice to the same value is harmless.
constexpr int kMaxDevices = 64;

// The current device, or -1 when it cannot be read or is beyond the caches.
int current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  return dev;
}

// Raises a stream kernel's dynamic shared-memory limit to max_bytes (the most
// any of its launches asks for, `bytes` <= max_bytes; kStreamSmemMax unless the
// kernel runs one CTA per SM) once per device, cached per kernel instantiation
// through Tag.
template <typename Tag, typename KernelT>
cudaError_t set_smem_max(KernelT kern, int bytes, int max_bytes = kStreamSmemMax) {
  static std::atomic<bool> done[kMaxDevices];
  const int dev = current_device();
  if (dev < 0) return cudaErrorInvalidDevice;
  if (bytes > max_bytes) return cudaErrorInvalidValue;
  if (done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, max_bytes);
  if (e == cudaSuccess) done[dev].store(true, std::memory_order_release);
  return e;
}

ck::gstream::Layout stream_layout_m8(int stage_bytes, int misc_bytes) {
  using namespace ck::gstream;
  Layout L;
  L.stage_bytes = (stage_bytes + 1023) / 1024 * 1024;   // swizzled tile copies start on 1024-byte boundaries
  const int bar_bytes = (2 * kMaxStages + 2 * kRed) * 8;
  const int budget = kStreamSmemMax - 1024 - kRed * kRedBytes - misc_bytes - bar_bytes - 256;   // 1024: base alignment
  L.ns = std::min(kMaxStages, budget / L.stage_bytes);
  L.off_red = L.ns * L.stage_bytes;
  L.off_misc = L.off_red + kRed * kRedBytes;
  L.off_bar = (L.off_misc + misc_bytes + 15) / 16 * 16;
  L.total = L.off_bar + bar_bytes + 1024;   // the kernel aligns its base up to 1024 bytes
  return L;
}

// Shared-memory layout of a streaming GEMV: as many stages as fit in half of
// an SM's shared memory, so that the next call's CTA can be resident (and
// streaming its first tiles) while this one runs. The per-CTA slices of the
// weight scales and bias (misc_bytes) grow with N / SMs; when they leave room
// for fewer than two stages (L.ns < 2, possibly negative) the streaming
// kernel cannot run and the caller takes the general kernel. The same holds
// for stream_layout_m8.
ck::gstream::Layout stream_layout(int stage_bytes, int misc_bytes) {
  using namespace ck::gstream;
  Layout L;
  L.stage_bytes = (stage_bytes + 127) / 128 * 128;
  const int red_stage = kCons * 32 * 4 * 4;
  const int budget = kStreamSmemMax - misc_bytes - 3 * kMaxStages * 8 - 256;
  L.ns = std::min(kMaxStages, budget / (L.stage_bytes + red_stage));
  L.off_red = L.ns * L.stage_bytes;
  L.off_misc = L.off_red + L.ns * red_stage;
  L.off_bar = (L.off_misc + misc_bytes + 15) / 16 * 16;
  L.total = L.off_bar + 3 * kMaxStages * 8;
  return L;
}


// ------------------------------------------------------------------ kernels

// Sets a kernel's dynamic shared-memory limit to `bytes` (the fixed size of
// all its launches) once per device, cached per kernel instantiation (Tag).
template <typename Tag, typename KernelT>
ck_status ensure_smem_attr(KernelT kernel, size_t bytes) {
  static std::atomic<bool> done[kMaxDevices];
  const int dev = current_device();
  if (dev < 0) return fail(CK_ERR_CUDA, "cudaGetDevice failed");
  if (!done[dev].load(std::memory_order_acquire)) {
    const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return fail(CK_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    done[dev].store(true, std::memory_order_release);
  }
  return CK_OK;
}

int sm_count() {
  static std::atomic<int> cache[kMaxDevices];
  const int dev = current_device();
  if (dev < 0) return 148;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

// Persistent grid: as many CTAs of `nt` threads (a multiple of 32, at most
// 1024) and `smem` dynamic bytes as are co-resident, at most `work`. The
// kernel's dynamic shared-memory limit is raised once per device to
// `smem_max`, the most ANY launch of this kernel asks for: raising it to each
// launch's own size would lower it again for a smaller launch and make a later
// larger one fail. The occupancy is cached per kernel instantiation (Tag),
// device and nt.
template <typename Tag, typename KernelT>
unsigned persistent_grid(KernelT kern, int nt, size_t smem, size_t smem_max, int64_t work) {
  static std::atomic<bool> limit_set[kMaxDevices];
  static std::atomic<int> cache[kMaxDevices][32];   // [dev][nt / 32 - 1]: CTAs per SM, 0 = not known
  const int dev = current_device();
  const int slot = nt / 32 - 1;
  const bool cached = dev >= 0 && nt % 32 == 0 && slot >= 0 && slot < 32;
  if (smem_max > 48 * 1024 && !(cached && limit_set[dev].load(std::memory_order_acquire))) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_max) == cudaSuccess &&
        cached)
      limit_set[dev].store(true, std::memory_order_release);
  }
  int blocks = cached ? cache[dev][slot].load(std::memory_order_relaxed) : 0;
  if (blocks <= 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, kern, nt, smem) != cudaSuccess || blocks <= 0)
      blocks = 1;
    if (cached) cache[dev][slot].store(blocks, std::memory_order_relaxed);
  }
  return (unsigned)std::min<int64_t>(work, (int64_t)blocks * sm_count());
}

template <int QBITS, int STORE, int GT, typename T>
void launch_rq_g(const T* x, int64_t M, int K, int64_t ldx, int G, float rnorm, uint8_t* q, float* s, int32_t* rs,
                 int nt, cudaStream_t st) {
  auto kern = ck::rq::rotate_quant_kernel<QBITS, STORE, GT, T>;
  const size_t smem = (size_t)(nt / 32) * 32 * ck::rq::CPT * 16;   // one transpose buffer per warp
  const size_t smem_max = (size_t)512 * ck::rq::CPT * 16;            // at the most threads a launch takes
  struct Tag {};
  launch_pdl(kern, dim3(persistent_grid<Tag>(kern, nt, smem, smem_max, M)), dim3(nt), smem, st, x, M, K, ldx, G,
             rnorm, q, s, rs);
}

// in_scale: the caller's tensor-wise input scale a >= 0. The kernel's transform
// is unnormalised (z = x H) and it scales z by rnorm both for the row amax and
// for the codes, so rnorm = a / sqrt(G) yields the rotation and quantization of
// a * x; a = 1 leaves rnorm = 1 / sqrt(G), exactly the unscaled launch. (G = 1
// decides its codes from z and s alone and must have a = 1.)
template <int QBITS, int STORE, typename T>
void launch_rq(const void* x, int64_t M, int K, int64_t ldx, int G, void* q, float* s, int32_t* rs, int nt,
               float in_scale, cudaStream_t st) {
  const float rnorm = (float)((double)in_scale / std::sqrt((double)G));
  const T* xx = reinterpret_cast<const T*>(x);
  uint8_t* qq = reinterpret_cast<uint8_t*>(q);
  switch (G) {
    case 1: launch_rq_g<QBITS, STORE, 1, T>(xx, M, K, ldx, G, rnorm, qq, s, rs, nt, st); break;
    case 16: launch_rq_g<QBITS, STORE, 16, T>(xx, M, K, ldx, G, rnorm, qq, s, rs, nt, st); break;
    case 64: launch_rq_g<QBITS, STORE, 64, T>(xx, M, K, ldx, G, rnorm, qq, s, rs, nt, st); break;
    case 256: launch_rq_g<QBITS, STORE, 256, T>(xx, M, K, ldx, G, rnorm, qq, s, rs, nt, st); break;
    default: launch_rq_g<QBITS, STORE, 0, T>(xx, M, K, ldx, G, rnorm, qq, s, rs, nt, st); break;
  }
}

template <typename T>
void launch_rq_store(int bits, int store, const void* x, int64_t M, int K, int64_t ldx, int G, void* q,
                     float* s, int32_t* rs, int nt, float a, cudaStream_t st) {
  using namespace ck::rq;
  if (store == STORE_PACKED4) launch_rq<4, STORE_PACKED4, T>(x, M, K, ldx, G, q, s, rs, nt, a, st);
  else if (store == STORE_INT8_PERM && bits == 4) launch_rq<4, STORE_INT8_PERM, T>(x, M, K, ldx, G, q, s, rs, nt, a, st);
  else if (store == STORE_INT8_PERM) launch_rq<8, STORE_INT8_PERM, T>(x, M, K, ldx, G, q, s, rs, nt, a, st);
  else if (bits == 4) launch_rq<4, STORE_INT8, T>(x, M, K, ldx, G, q, s, rs, nt, a, st);
  else launch_rq<8, STORE_INT8, T>(x, M, K, ldx, G, q, s, rs, nt, a, st);
}

// store: STORE_PACKED4 (bits 4), STORE_INT8 (codes as int8 bytes) or STORE_INT8_PERM
// (bits 4 or 8, the linears' GEMM-ready activations with row sums in `rs`). in_scale:
// the tensor-wise input scale, validated by the caller (finite, >= 0, 1 when G = 1).
ck_status rotate_quant_impl(const void* x, ck_dtype xt, int64_t M, int64_t K, int64_t ldx, int G,
                            int bits, int store, void* q, float* s, int32_t* rs, cudaStream_t st,
                            float in_scale = 1.0f) {
  using namespace ck::rq;
  const int64_t nt = ((K + EPT - 1) / EPT + 31) / 32 * 32;
  if (nt > 512) return fail(CK_ERR_UNSUPPORTED, "rotate_quant: K=%lld too large (max 32768)", (long long)K);
  if (xt == CK_BF16)
    launch_rq_store<__nv_bfloat16>(bits, store, x, M, (int)K, ldx, G, q, s, rs, (int)nt, in_scale, st);
  else launch_rq_store<__half>(bits, store, x, M, (int)K, ldx, G, q, s, rs, (int)nt, in_scale, st);
  return launch_status("rotate_quant");
}

// The tensor-wise input scale's contract: a finite a >= 0, and a = 1 when G = 1.
ck_status check_input_scale(const char* who, float a, int group_size) {
  if (!std::isfinite(a) || a < 0.0f)
    return fail(CK_ERR_INVALID_ARG, "%s: input_scale=%g must be finite and >= 0", who, (double)a);
  if (group_size == 1 && a != 1.0f)
    return fail(CK_ERR_UNSUPPORTED, "%s: group_size 1 (no rotation) takes only input_scale 1", who);
  return CK_OK;
}

// Largest |a * w| of one product term, per operand pair: the int32 accumulator
// holds sum_k a * w exactly only while K * term <= INT32_MAX.
constexpr int64_t kTermS8 = 128 * 128;      // int8 x int8
constexpr int64_t kTermW4A8 = 128 * 8;      // int8 x (u - 8)
constexpr int64_t kTermW4A4 = 8 * 8;        // (u - 8) x (u - 8)
constexpr int64_t kTermLinear = 7 * 15;     // int4 code x unsigned nibble u (the linear's GEMM)
constexpr int64_t kTermGemv = 128 * 15;     // int8 x unsigned nibble u (the W4A8 GEMV)

ck_status check_acc_range(const char* who, int64_t K, int64_t term) {
  if (K > (int64_t)INT32_MAX / term)
    return fail(CK_ERR_UNSUPPORTED, "%s: K=%lld could overflow the int32 accumulator (K * %lld > 2^31 - 1)", who,
                (long long)K, (long long)term);
  return CK_OK;
}

ck_status check_gemm_shape(const char* who, int64_t M, int64_t K, int64_t N, int64_t term) {
  if (M <= 0 || K <= 0 || N <= 0) return fail(CK_ERR_INVALID_ARG, "%s: M, K, N must be > 0", who);
  if (K % 32 != 0) return fail(CK_ERR_UNSUPPORTED, "%s: K=%lld must be a multiple of 32", who, (long long)K);
  if (M > (int64_t)INT32_MAX / 2 || N > (int64_t)INT32_MAX / 2 || K > (int64_t)INT32_MAX / 2)
    return fail(CK_ERR_UNSUPPORTED, "%s: dimension too large", who);
  ck_status r = check_acc_range(who, K, term);
  if (r != CK_OK) return r;
  if ((M + ck::gemm::BM - 1) / ck::gemm::BM > 65535)
    return fail(CK_ERR_UNSUPPORTED, "%s: M=%lld too large for one launch", who, (long long)M);
  return CK_OK;
}

// Largest number of CTA pairs of this kernel that are co-resident on the device (cached per device).
template <typename Tag, typename KernelT>
ck_status max_pairs(KernelT kernel, size_t smem, int* out) {
  static std::atomic<int> cache[kMaxDevices];
  const int dev = current_device();
  if (dev < 0) return fail(CK_ERR_CUDA, "cudaGetDevice failed");
  int pairs = cache[dev].load(std::memory_order_relaxed);
  if (pairs == 0) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(ck::gemm::kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    const cudaError_t e = cudaOccupancyMaxActiveClusters(&n, kernel, &cfg);
    if (e != cudaSuccess || n <= 0) return fail(CK_ERR_CUDA, "cudaOccupancyMaxActiveClusters: %s (%d)", cudaGetErrorString(e), n);
    cache[dev].store(n, std::memory_order_relaxed);
    pairs = n;
  }
  *out = pairs;
  return CK_OK;
}

template <int A_MODE, int B_MODE, int EPI>
ck_status gemm_impl(const void* qa, int64_t M, int64_t K, int64_t N, const void* w, const float* a_scale,
                    const int32_t* a_rowsum, const uint16_t* w_scale, const uint16_t* bias, void* out,
                    cudaStream_t st) {
  using namespace ck::gemm;
  using C = Cfg<A_MODE, B_MODE>;
  CUtensorMap ta, tb;
  ck_status r;
  if (C::AP) r = make_tmap(&ta, qa, (uint64_t)K / 2, (uint64_t)M, (uint64_t)K / 2, PKB, BM, CU_TENSOR_MAP_SWIZZLE_NONE);
  else r = make_tmap(&ta, qa, (uint64_t)K, (uint64_t)M, (uint64_t)K, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B);
  if (r != CK_OK) return r;
  if (C::BP) r = make_tmap(&tb, w, (uint64_t)K / 2, (uint64_t)N, (uint64_t)K / 2, PKB, BNH, CU_TENSOR_MAP_SWIZZLE_NONE);
  else r = make_tmap(&tb, w, (uint64_t)K, (uint64_t)N, (uint64_t)K, BK, BNH, CU_TENSOR_MAP_SWIZZLE_128B);
  if (r != CK_OK) return r;
  auto kern = gemm_w4_kernel<A_MODE, B_MODE, EPI>;
  struct Tag {};
  if ((r = ensure_smem_attr<Tag>(kern, C::SMEM)) != CK_OK) return r;
  int pairs_max = 0;
  if ((r = max_pairs<Tag>(kern, C::SMEM, &pairs_max)) != CK_OK) return r;
  Params p;
  p.M = (int)M; p.N = (int)N; p.K = (int)K;
  p.tiles_m = (int)((M + 2 * BM - 1) / (2 * BM));
  p.tiles_n = (int)((N + BN - 1) / BN);
  p.a_scale = a_scale;
  p.a_rowsum = a_rowsum;
  p.w_scale = reinterpret_cast<const __nv_bfloat16*>(w_scale);
  p.bias = reinterpret_cast<const __nv_bfloat16*>(bias);
  p.out = out;
  const size_t esz = EPI == EPI_I32 ? 4 : 2;
  p.out_vec_ok = aligned(out, 16) && ((N * (int64_t)esz) % 16 == 0);
  p.col_vec_ok = (w_scale == nullptr || aligned(w_scale, 16)) && (bias == nullptr || aligned(bias, 16));
  const int64_t tiles = (int64_t)p.tiles_m * p.tiles_n;
  const int pairs = (int)std::min<int64_t>(tiles, pairs_max);

  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, ta, tb, p);
  if (e != cudaSuccess) return fail(CK_ERR_CUDA, "gemm_w4: launch failed: %s", cudaGetErrorString(e));
  return launch_status("gemm_w4");
}

size_t align256(size_t v) { return (v + 255) / 256 * 256; }
bool linear_small_m(int64_t M, int64_t K);

// The codes' region of the linear's workspace. Small batches: the codes packed two
// per byte, then room for them one per byte (used only when the matmul phase must
// take a GEMV path that reads int8).
size_t linear_q_bytes(int64_t M, int64_t K) {
  if (linear_small_m(M, K)) return align256((size_t)M * (size_t)K / 2) + align256((size_t)M * (size_t)K);
  return align256((size_t)M * (size_t)K);
}

// The linear's workspace: the codes (int8 (M, K) in the GEMM's permuted column
// order; for small batches packed int4 or, in the W4A8 linear, int8 in natural
// order), float32 row scales (M), int32 row sums of the codes (M), each 256-byte
// aligned.
struct LinearWs {
  int8_t* q;
  int8_t* q8;   // small batches: room for the packed codes unpacked to int8
  float* scale;
  int32_t* rowsum;
};

LinearWs linear_ws(void* base, int64_t M, int64_t K) {
  uint8_t* b = reinterpret_cast<uint8_t*>(base);
  LinearWs w;
  w.q = reinterpret_cast<int8_t*>(b);
  w.q8 = linear_small_m(M, K) ? reinterpret_cast<int8_t*>(b + align256((size_t)M * (size_t)K / 2)) : nullptr;
  w.scale = reinterpret_cast<float*>(b + linear_q_bytes(M, K));
  w.rowsum = reinterpret_cast<int32_t*>(b + linear_q_bytes(M, K) + align256((size_t)M * sizeof(float)));
  return w;
}

size_t linear_ws_bytes(int64_t M, int64_t K) {
  return linear_q_bytes(M, K) + align256((size_t)M * sizeof(float)) + (size_t)M * sizeof(int32_t);
}

// Small batches of the linear take the decode-GEMV kernels instead of the
// tensor-core GEMM: with M <= 64 the GEMM's 256 x 256 pair tiles leave most
// SMs idle (K = N = 3840: 15 of 74 pairs busy), while the streaming GEMV
// spreads the weights over every SM. The codes then stay in natural column
// order (the GEMV computes its own row sums). The epilogue arithmetic is the
// same, so the results do not depend on the route. Both phases of the linear
// take the decision from (M, K) alone.
bool linear_small_m(int64_t M, int64_t K) { return M <= 64 && K % 128 == 0 && K <= 4096; }

// What phase 1 of a linear stores: the GEMM's permuted int8 codes with row sums, or
// for small batches the codes in natural order, packed two per byte when they are
// int4 (the row-split GEMV then pulls half the bytes from L2).
int linear_store(int64_t M, int64_t K, int bits) {
  if (!linear_small_m(M, K)) return ck::rq::STORE_INT8_PERM;
  return bits == 4 ? ck::rq::STORE_PACKED4 : ck::rq::STORE_INT8;
}
constexpr int64_t kSmallMChunk = 16;           // rows per GEMV call
constexpr int64_t kSmallMChunkRowsplit = 32;   // rows per row-split GEMV call

ck_status gemv_w4a8_rowsplit(const int8_t* xq, const float* x_scale, int64_t M, int64_t K, int64_t N,
                             const uint8_t* w_packed, const __nv_bfloat16* sw, const __nv_bfloat16* bb,
                             __nv_bfloat16* yy, cudaStream_t st, bool a4 = false);

ck_status check_linear_workspace(const char* who, int64_t M, int64_t K, const void* ws, size_t bytes) {
  if (ws == nullptr || bytes < linear_ws_bytes(M, K))
    return fail(CK_ERR_INVALID_ARG, "%s: workspace smaller than ck_linear_w4a4_workspace_bytes", who);
  if (!aligned(ws, 256)) return fail(CK_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", who);
  return CK_OK;
}

}  // namespace

extern "C" {

const char* ck_last_error(void) { return g_last_error.c_str(); }

const char* ck_version(void) { return "ck 0.1 (sm_100a)"; }

}  // extern "C"

namespace {

ck_status rotate_quant_entry(const char* who, const void* x, ck_dtype xt, int64_t M, int64_t K, int64_t ldx,
                             int group_size, int bits, float in_scale, void* q_out, float* scale_out,
                             void* stream) {
  if (M < 0 || K <= 0) return fail(CK_ERR_INVALID_ARG, "%s: need M >= 0 and K > 0", who);
  if (xt != CK_BF16 && xt != CK_FP16) return fail(CK_ERR_INVALID_ARG, "%s: unknown dtype", who);
  if (bits != 4 && bits != 8) return fail(CK_ERR_INVALID_ARG, "%s: bits must be 4 or 8", who);
  if (!is_pow2(group_size) || group_size > 256)
    return fail(CK_ERR_UNSUPPORTED, "%s: group_size=%d must be a power of two <= 256", who, group_size);
  ck_status r = check_input_scale(who, in_scale, group_size);
  if (r != CK_OK) return r;
  if (K % group_size != 0) return fail(CK_ERR_INVALID_ARG, "%s: K %% group_size != 0", who);
  if (K % 8 != 0) return fail(CK_ERR_UNSUPPORTED, "%s: K must be a multiple of 8", who);
  if (ldx < K) return fail(CK_ERR_INVALID_ARG, "%s: ldx < K", who);
  if (M == 0) return ok();
  if (x == nullptr || q_out == nullptr || scale_out == nullptr)
    return fail(CK_ERR_INVALID_ARG, "%s: null pointer", who);
  if (!aligned(x, 16) || ldx % 8 != 0) return fail(CK_ERR_INVALID_ARG, "%s: x rows must be 16-byte aligned", who);
  if (!aligned(q_out, 16) || !aligned(scale_out, 4)) return fail(CK_ERR_INVALID_ARG, "%s: misaligned output", who);
  if (M > INT32_MAX) return fail(CK_ERR_UNSUPPORTED, "%s: M too large", who);
  return rotate_quant_impl(x, xt, M, K, ldx, group_size, bits,
                           bits == 4 ? ck::rq::STORE_PACKED4 : ck::rq::STORE_INT8, q_out, scale_out,
                           nullptr, S(stream), in_scale);
}

}  // namespace

extern "C" {

ck_status ck_rotate_quant_rowwise(const void* x, ck_dtype xt, int64_t M, int64_t K, int64_t ldx,
                                  int group_size, int bits, void* q_out, float* scale_out,
                                  void* stream) {
  return rotate_quant_entry("rotate_quant", x, xt, M, K, ldx, group_size, bits, 1.0f, q_out, scale_out, stream);
}

ck_status ck_rotate_quant_rowwise_scaled(const void* x, ck_dtype xt, int64_t M, int64_t K, int64_t ldx,
                                         int group_size, int bits, float input_scale, void* q_out,
                                         float* scale_out, void* stream) {
  return rotate_quant_entry("rotate_quant_scaled", x, xt, M, K, ldx, group_size, bits, input_scale, q_out,
                            scale_out, stream);
}

ck_status ck_rotate_quant_rowwise_i8(const void* x, ck_dtype xt, int64_t M, int64_t K, int64_t ldx,
                                     int group_size, int bits, int8_t* q_out, float* scale_out,
                                     void* stream) {
  if (M < 0 || K <= 0) return fail(CK_ERR_INVALID_ARG, "rotate_quant_i8: need M >= 0 and K > 0");
  if (xt != CK_BF16 && xt != CK_FP16) return fail(CK_ERR_INVALID_ARG, "rotate_quant_i8: unknown dtype");
  if (bits != 4 && bits != 8) return fail(CK_ERR_INVALID_ARG, "rotate_quant_i8: bits must be 4 or 8");
  if (!is_pow2(group_size) || group_size > 256)
    return fail(CK_ERR_UNSUPPORTED, "rotate_quant_i8: group_size=%d must be a power of two <= 256", group_size);
  if (K % group_size != 0) return fail(CK_ERR_INVALID_ARG, "rotate_quant_i8: K %% group_size != 0");
  if (K % 8 != 0) return fail(CK_ERR_UNSUPPORTED, "rotate_quant_i8: K must be a multiple of 8");
  if (ldx < K) return fail(CK_ERR_INVALID_ARG, "rotate_quant_i8: ldx < K");
  if (M == 0) return ok();
  if (x == nullptr || q_out == nullptr || scale_out == nullptr)
    return fail(CK_ERR_INVALID_ARG, "rotate_quant_i8: null pointer");
  if (!aligned(x, 16) || ldx % 8 != 0) return fail(CK_ERR_INVALID_ARG, "rotate_quant_i8: x rows must be 16-byte aligned");
  if (!aligned(q_out, 16) || !aligned(scale_out, 4)) return fail(CK_ERR_INVALID_ARG, "rotate_quant_i8: misaligned output");
  if (M > INT32_MAX) return fail(CK_ERR_UNSUPPORTED, "rotate_quant_i8: M too large");
  return rotate_quant_impl(x, xt, M, K, ldx, group_size, bits, ck::rq::STORE_INT8, q_out, scale_out, nullptr,
                           S(stream));
}

ck_status ck_rotate_quant_rowwise_r(const void* x, ck_dtype xt, int64_t M, int64_t K, int64_t ldx,
                                    int group_size, const float* R, int bits, void* q_out, float* scale_out,
                                    void* stream) {
  if (xt != CK_BF16 && xt != CK_FP16) return fail(CK_ERR_INVALID_ARG, "rotate_quant_rowwise_r: unknown dtype");
  if (bits != 4 && bits != 8) return fail(CK_ERR_INVALID_ARG, "rotate_quant_rowwise_r: bits must be 4 or 8");
  if (M < 0 || K <= 0) return fail(CK_ERR_INVALID_ARG, "rotate_quant_rowwise_r: M >= 0 and K > 0 required");
  if (group_size < 1 || group_size > 256)
    return fail(CK_ERR_UNSUPPORTED, "rotate_quant_rowwise_r: group_size=%d outside [1, 256]", group_size);
  if (K % group_size != 0) return fail(CK_ERR_INVALID_ARG, "rotate_quant_rowwise_r: K %% group_size != 0");
  if (K % 2 != 0) return fail(CK_ERR_INVALID_ARG, "rotate_quant_rowwise_r: K must be even");
  if (K > 16384) return fail(CK_ERR_UNSUPPORTED, "rotate_quant_rowwise_r: K=%lld > 16384", (long long)K);
  if (ldx < K) return fail(CK_ERR_INVALID_ARG, "rotate_quant_rowwise_r: ldx < K");
  if (M == 0) return ok();
  if (!x || !R || !q_out || !scale_out) return fail(CK_ERR_INVALID_ARG, "rotate_quant_rowwise_r: null pointer");
  if (!aligned(x, 2) || !aligned(R, 4) || !aligned(scale_out, 4))
    return fail(CK_ERR_INVALID_ARG, "rotate_quant_rowwise_r: misaligned pointer");
  const size_t smem = 2 * (size_t)K * sizeof(float);
  const size_t smem_max = 2 * (size_t)16384 * sizeof(float);   // K <= 16384: the limit, set once per device
  const unsigned grid = (unsigned)std::min<int64_t>(M, 8 * (int64_t)sm_count());
  cudaError_t e = cudaSuccess;
  ck_status r = CK_OK;
#define CK_RQG(T, B)                                                                                 \
  {                                                                                                  \
    auto kern = ck::rqg::rotate_quant_general_kernel<T, B>;                                          \
    struct Tag {};                                                                                   \
    r = ensure_smem_attr<Tag>(kern, smem_max);                                                       \
    if (r == CK_OK)                                                                                  \
      e = launch_pdl(kern, dim3(grid), dim3(ck::rqg::kThreads), smem, S(stream), reinterpret_cast<const T*>(x), M, \
                     (int)K, ldx, group_size, R, reinterpret_cast<uint8_t*>(q_out), scale_out);       \
  }
  if (xt == CK_BF16) {
    if (bits == 4) CK_RQG(__nv_bfloat16, 4) else CK_RQG(__nv_bfloat16, 8)
  } else {
    if (bits == 4) CK_RQG(__half, 4) else CK_RQG(__half, 8)
  }
#undef CK_RQG
  if (r != CK_OK) return r;
  if (e != cudaSuccess) return fail(CK_ERR_CUDA, "rotate_quant_rowwise_r: %s", cudaGetErrorString(e));
  return launch_status("rotate_quant_rowwise_r");
}

ck_status ck_unpack_int4(const uint8_t* packed, int64_t R, int64_t C, int8_t* out, void* stream) {
  if (R <= 0 || C <= 0) return fail(CK_ERR_INVALID_ARG, "unpack_int4: R, C must be > 0");
  if (!packed || !out) return fail(CK_ERR_INVALID_ARG, "unpack_int4: null pointer");
  const int64_t nbytes = R * (C / 2);
  if (C % 2 != 0 || nbytes % 16 != 0) return fail(CK_ERR_UNSUPPORTED, "unpack_int4: R*C/2 must be a multiple of 16");
  if (!aligned(packed, 16) || !aligned(out, 16)) return fail(CK_ERR_INVALID_ARG, "unpack_int4: pointers must be 16-byte aligned");
  const int64_t n16 = nbytes / 16;
  const unsigned grid = (unsigned)std::min<int64_t>((n16 + 255) / 256, 148 * 16);
  ck::gemm::unpack_int4_kernel<<<grid, 256, 0, S(stream)>>>(reinterpret_cast<const uint4*>(packed),
                                                            reinterpret_cast<uint4*>(out), n16);
  return launch_status("unpack_int4");
}

ck_status ck_gemm_s8(const int8_t* qa, const float* a_scale, int64_t M, int64_t K, int64_t N,
                     const int8_t* w, const uint16_t* w_scale, const uint16_t* bias, uint16_t* y,
                     void* stream) {
  ck_status r = check_gemm_shape("gemm_s8", M, K, N, kTermS8);
  if (r != CK_OK) return r;
  if (!qa || !a_scale || !w || !w_scale || !y) return fail(CK_ERR_INVALID_ARG, "gemm_s8: null pointer");
  if (!aligned(qa, 16) || !aligned(w, 16)) return fail(CK_ERR_UNSUPPORTED, "gemm_s8: operands must be 16-byte aligned");
  if (!aligned(a_scale, 4) || !aligned(w_scale, 2) || !aligned(y, 2) || (bias && !aligned(bias, 2)))
    return fail(CK_ERR_INVALID_ARG, "gemm_s8: misaligned scale, bias or output");
  return gemm_impl<ck::gemm::OP_INT8, ck::gemm::OP_INT8, ck::gemm::EPI_BF16>(qa, M, K, N, w, a_scale, nullptr, w_scale, bias, y, S(stream));
}

ck_status ck_gemm_w4a8(const int8_t* qa, const float* a_scale, int64_t M, int64_t K, int64_t N,
                       const uint8_t* w_packed, const uint16_t* w_scale, const uint16_t* bias,
                       uint16_t* y, void* stream) {
  ck_status r = check_gemm_shape("gemm_w4a8", M, K, N, kTermW4A8);
  if (r != CK_OK) return r;
  if (!qa || !a_scale || !w_packed || !w_scale || !y) return fail(CK_ERR_INVALID_ARG, "gemm_w4a8: null pointer");
  if (!aligned(qa, 16) || !aligned(w_packed, 16)) return fail(CK_ERR_UNSUPPORTED, "gemm_w4a8: operands must be 16-byte aligned");
  if (!aligned(a_scale, 4) || !aligned(w_scale, 2) || !aligned(y, 2) || (bias && !aligned(bias, 2)))
    return fail(CK_ERR_INVALID_ARG, "gemm_w4a8: misaligned scale, bias or output");
  return gemm_impl<ck::gemm::OP_INT8, ck::gemm::OP_PACKED4, ck::gemm::EPI_BF16>(qa, M, K, N, w_packed, a_scale, nullptr, w_scale, bias, y, S(stream));
}

ck_status ck_gemm_s8_i32(const int8_t* qa, const int8_t* w, int64_t M, int64_t K, int64_t N, int32_t* acc,
                         void* stream) {
  ck_status r = check_gemm_shape("gemm_s8_i32", M, K, N, kTermS8);
  if (r != CK_OK) return r;
  if (!qa || !w || !acc) return fail(CK_ERR_INVALID_ARG, "gemm_s8_i32: null pointer");
  if (!aligned(qa, 16) || !aligned(w, 16)) return fail(CK_ERR_UNSUPPORTED, "gemm_s8_i32: operands must be 16-byte aligned");
  if (!aligned(acc, 4)) return fail(CK_ERR_INVALID_ARG, "gemm_s8_i32: misaligned output");
  return gemm_impl<ck::gemm::OP_INT8, ck::gemm::OP_INT8, ck::gemm::EPI_I32>(qa, M, K, N, w, nullptr, nullptr, nullptr, nullptr, acc, S(stream));
}

ck_status ck_gemm_w4a4(const uint8_t* qa_packed, const float* a_scale, int64_t M, int64_t K,
                       int64_t N, const uint8_t* w_packed, const uint16_t* w_scale,
                       const uint16_t* bias, uint16_t* y, void* stream) {
  ck_status r = check_gemm_shape("gemm_w4a4", M, K, N, kTermW4A4);
  if (r != CK_OK) return r;
  if (!qa_packed || !a_scale || !w_packed || !w_scale || !y) return fail(CK_ERR_INVALID_ARG, "gemm_w4a4: null pointer");
  if (!aligned(qa_packed, 16) || !aligned(w_packed, 16)) return fail(CK_ERR_UNSUPPORTED, "gemm_w4a4: operands must be 16-byte aligned");
  if (!aligned(a_scale, 4) || !aligned(w_scale, 2) || !aligned(y, 2) || (bias && !aligned(bias, 2)))
    return fail(CK_ERR_INVALID_ARG, "gemm_w4a4: misaligned scale, bias or output");
  return gemm_impl<ck::gemm::OP_PACKED4, ck::gemm::OP_PACKED4, ck::gemm::EPI_BF16>(qa_packed, M, K, N, w_packed, a_scale, nullptr, w_scale, bias, y, S(stream));
}

size_t ck_linear_w4a4_workspace_bytes(int64_t M, int64_t K) {
  if (M <= 0 || K <= 0) return 0;
  return linear_q_bytes(M, K) + align256((size_t)M * sizeof(float)) + (size_t)M * sizeof(int32_t);
}

}  // extern "C"

namespace {

// The linears' activation code widths: int4 codes (the W4A4 linear) or int8
// codes (the W4A8 linear); the GEMM multiplies either with unsigned nibbles.
int64_t linear_term(int bits) { return bits == 4 ? kTermLinear : kTermGemv; }

// Phase 1 of a linear: rotate + quantize x into the workspace. `perm` selects
// the GEMM-ready format (codes in permuted column order plus row sums, for the
// tensor-core GEMM with unsigned weight decode); otherwise the codes stay in
// natural order (the decode-GEMV route and the pre-decoded-weight GEMM).
ck_status linear_quantize_entry(const char* who, const void* x, ck_dtype xt, int64_t M, int64_t K, int64_t ldx,
                                int group_size, int bits, float in_scale, int store, void* workspace,
                                size_t ws_bytes, void* stream) {
  ck_status r = check_gemm_shape(who, M, K, 1, linear_term(bits));
  if (r != CK_OK) return r;
  if ((r = check_linear_workspace(who, M, K, workspace, ws_bytes)) != CK_OK) return r;
  if (xt != CK_BF16 && xt != CK_FP16) return fail(CK_ERR_INVALID_ARG, "%s: unknown dtype", who);
  if (!is_pow2(group_size) || group_size > 256)
    return fail(CK_ERR_UNSUPPORTED, "%s: group_size=%d must be a power of two <= 256", who, group_size);
  if ((r = check_input_scale(who, in_scale, group_size)) != CK_OK) return r;
  if (K % group_size != 0) return fail(CK_ERR_INVALID_ARG, "%s: K %% group_size != 0", who);
  if (ldx < K) return fail(CK_ERR_INVALID_ARG, "%s: ldx < K", who);
  if (x == nullptr) return fail(CK_ERR_INVALID_ARG, "%s: null pointer", who);
  if (!aligned(x, 16) || ldx % 8 != 0) return fail(CK_ERR_INVALID_ARG, "%s: x rows must be 16-byte aligned", who);
  LinearWs ws = linear_ws(workspace, M, K);
  return rotate_quant_impl(x, xt, M, K, ldx, group_size, bits, store, ws.q, ws.scale, ws.rowsum, S(stream),
                           in_scale);
}

// Phase 2 of a linear on packed int4 weights: the small-batch decode GEMV or
// the tensor-core GEMM with unsigned weight decode, on the codes phase 1 wrote.
ck_status linear_matmul_entry(const char* who, int64_t M, int64_t K, int64_t N, int bits, const uint8_t* w_packed,
                              const uint16_t* w_scale, const uint16_t* bias, uint16_t* y, const void* workspace,
                              size_t ws_bytes, void* stream) {
  ck_status r = check_gemm_shape(who, M, K, N, linear_term(bits));
  if (r != CK_OK) return r;
  if ((r = check_linear_workspace(who, M, K, workspace, ws_bytes)) != CK_OK) return r;
  if (!w_packed || !w_scale || !y) return fail(CK_ERR_INVALID_ARG, "%s: null pointer", who);
  if (!aligned(w_packed, 16)) return fail(CK_ERR_UNSUPPORTED, "%s: weights must be 16-byte aligned", who);
  if (!aligned(w_scale, 2) || !aligned(y, 2) || (bias && !aligned(bias, 2)))
    return fail(CK_ERR_INVALID_ARG, "%s: misaligned scale, bias or output", who);
  LinearWs ws = linear_ws(const_cast<void*>(workspace), M, K);
  if (linear_small_m(M, K)) {
    // 32-row pieces through the row-split kernel where it applies (int4 codes read packed),
    // else 16-row GEMV calls on int8 codes (unpacked first when phase 1 packed them)
    const bool a4 = bits == 4;
    const bool rowsplit = N % 8 == 0 && aligned(w_scale, 16) && (bias == nullptr || aligned(bias, 16));
    const int8_t* q8 = ws.q;
    bool unpacked = false;
    for (int64_t r0 = 0; r0 < M; r0 += kSmallMChunkRowsplit) {
      const int64_t mc = std::min<int64_t>(kSmallMChunkRowsplit, M - r0);
      r = CK_ERR_UNSUPPORTED;
      if (rowsplit)
        r = gemv_w4a8_rowsplit(a4 ? ws.q + r0 * (K / 2) : ws.q + r0 * K, ws.scale + r0, mc, K, N, w_packed,
                               reinterpret_cast<const __nv_bfloat16*>(w_scale),
                               reinterpret_cast<const __nv_bfloat16*>(bias),
                               reinterpret_cast<__nv_bfloat16*>(y + r0 * N), S(stream), a4);
      if (r == CK_ERR_UNSUPPORTED) {   // nothing launched: 16-row GEMV calls
        if (a4 && !unpacked) {
          if ((r = ck_unpack_int4(reinterpret_cast<const uint8_t*>(ws.q), M, K, ws.q8, stream)) != CK_OK) return r;
          q8 = ws.q8;
          unpacked = true;
        }
        for (int64_t q0 = r0; q0 < r0 + mc; q0 += kSmallMChunk) {
          const int64_t qc = std::min<int64_t>(kSmallMChunk, r0 + mc - q0);
          r = ck_gemv_w4a8(q8 + q0 * K, ws.scale + q0, qc, K, N, w_packed, w_scale, bias, y + q0 * N, stream);
          if (r != CK_OK) return r;
        }
      }
      if (r != CK_OK) return r;
    }
    return ok();
  }
  return gemm_impl<ck::gemm::OP_INT8, ck::gemm::OP_PACKED4_U, ck::gemm::EPI_BF16>(
      ws.q, M, K, N, w_packed, ws.scale, ws.rowsum, w_scale, bias, y, S(stream));
}

}  // namespace

extern "C" {

ck_status ck_linear_w4a4_quantize(const void* x, ck_dtype xt, int64_t M, int64_t K, int64_t ldx, int group_size,
                                  void* workspace, size_t ws_bytes, void* stream) {
  return linear_quantize_entry("linear_w4a4_quantize", x, xt, M, K, ldx, group_size, 4, 1.0f,
                               linear_store(M, K, 4), workspace, ws_bytes, stream);
}

ck_status ck_linear_w4a4_matmul(int64_t M, int64_t K, int64_t N, const uint8_t* w_packed, const uint16_t* w_scale,
                                const uint16_t* bias, uint16_t* y, const void* workspace, size_t ws_bytes,
                                void* stream) {
  return linear_matmul_entry("linear_w4a4_matmul", M, K, N, 4, w_packed, w_scale, bias, y, workspace, ws_bytes,
                             stream);
}

}  // extern "C"

namespace {

ck_status linear_entry(const char* who, const void* x, ck_dtype xt, int64_t M, int64_t K, int64_t N, int64_t ldx,
                       int group_size, int bits, float in_scale, const uint8_t* w_packed, const uint16_t* w_scale,
                       const uint16_t* bias, uint16_t* y, void* workspace, size_t ws_bytes, void* stream) {
  ck_status r = check_gemm_shape(who, M, K, N, linear_term(bits));
  if (r != CK_OK) return r;
  // validate both phases before enqueuing either
  if ((r = check_linear_workspace(who, M, K, workspace, ws_bytes)) != CK_OK) return r;
  if (!w_packed || !w_scale || !y) return fail(CK_ERR_INVALID_ARG, "%s: null pointer", who);
  if (!aligned(w_packed, 16)) return fail(CK_ERR_UNSUPPORTED, "%s: weights must be 16-byte aligned", who);
  if (!aligned(w_scale, 2) || !aligned(y, 2) || (bias && !aligned(bias, 2)))
    return fail(CK_ERR_INVALID_ARG, "%s: misaligned scale, bias or output", who);
  r = linear_quantize_entry(who, x, xt, M, K, ldx, group_size, bits, in_scale, linear_store(M, K, bits), workspace,
                            ws_bytes, stream);
  if (r != CK_OK) return r;
  return linear_matmul_entry(who, M, K, N, bits, w_packed, w_scale, bias, y, workspace, ws_bytes, stream);
}

}  // namespace

extern "C" {

ck_status ck_linear_w4a4(const void* x, ck_dtype xt, int64_t M, int64_t K, int64_t N, int64_t ldx,
                         int group_size, const uint8_t* w_packed, const uint16_t* w_scale,
                         const uint16_t* bias, uint16_t* y, void* workspace, size_t ws_bytes,
                         void* stream) {
  return linear_entry("linear_w4a4", x, xt, M, K, N, ldx, group_size, 4, 1.0f, w_packed, w_scale, bias, y,
                      workspace, ws_bytes, stream);
}

ck_status ck_linear_w4a4_scaled(const void* x, ck_dtype xt, int64_t M, int64_t K, int64_t N, int64_t ldx,
                                int group_size, float input_scale, const uint8_t* w_packed,
                                const uint16_t* w_scale, const uint16_t* bias, uint16_t* y, void* workspace,
                                size_t ws_bytes, void* stream) {
  return linear_entry("linear_w4a4_scaled", x, xt, M, K, N, ldx, group_size, 4, input_scale, w_packed, w_scale,
                      bias, y, workspace, ws_bytes, stream);
}

size_t ck_linear_w4a8_workspace_bytes(int64_t M, int64_t K) { return ck_linear_w4a4_workspace_bytes(M, K); }

ck_status ck_linear_w4a8(const void* x, ck_dtype xt, int64_t M, int64_t K, int64_t N, int64_t ldx,
                         int group_size, const uint8_t* w_packed, const uint16_t* w_scale,
                         const uint16_t* bias, uint16_t* y, void* workspace, size_t ws_bytes,
                         void* stream) {
  return linear_entry("linear_w4a8", x, xt, M, K, N, ldx, group_size, 8, 1.0f, w_packed, w_scale, bias, y,
                      workspace, ws_bytes, stream);
}

ck_status ck_linear_w4a4_predecoded(const void* x, ck_dtype xt, int64_t M, int64_t K, int64_t N, int64_t ldx,
                                    int group_size, const int8_t* w_s8, const uint16_t* w_scale,
                                    const uint16_t* bias, uint16_t* y, void* workspace, size_t ws_bytes,
                                    void* stream) {
  const char* who = "linear_w4a4_predecoded";
  ck_status r = check_gemm_shape(who, M, K, N, kTermLinear);
  if (r != CK_OK) return r;
  if ((r = check_linear_workspace(who, M, K, workspace, ws_bytes)) != CK_OK) return r;
  if (!w_s8 || !w_scale || !y) return fail(CK_ERR_INVALID_ARG, "%s: null pointer", who);
  if (!aligned(w_s8, 16)) return fail(CK_ERR_UNSUPPORTED, "%s: weights must be 16-byte aligned", who);
  if (!aligned(w_scale, 2) || !aligned(y, 2) || (bias && !aligned(bias, 2)))
    return fail(CK_ERR_INVALID_ARG, "%s: misaligned scale, bias or output", who);
  r = linear_quantize_entry(who, x, xt, M, K, ldx, group_size, 4, 1.0f, ck::rq::STORE_INT8, workspace, ws_bytes,
                            stream);
  if (r != CK_OK) return r;
  LinearWs ws = linear_ws(workspace, M, K);
  return gemm_impl<ck::gemm::OP_INT8, ck::gemm::OP_INT8, ck::gemm::EPI_BF16>(
      ws.q, M, K, N, w_s8, ws.scale, nullptr, w_scale, bias, y, S(stream));
}

}  // extern "C"

// ---------------------------------------------- linear with a static scratch

// The scratch of ck_linear_w4a4_static: one fixed block of global memory per
// device, reserved when the module loads on that device. It holds the same
// layout as the caller workspace of ck_linear_w4a4 (codes, scales, row sums).
static __device__ __align__(256) unsigned char g_linear_scratch[CK_LINEAR_STATIC_SCRATCH_BYTES];

namespace {

constexpr int kMaxScratchDevices = 64;
std::mutex g_scratch_mu;
struct ScratchEntry {
  void* addr;   // device address of g_linear_scratch
  void* ctx;    // the context it was looked up in
};
ScratchEntry g_scratch[kMaxScratchDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

// The calling thread's current CUDA context (null if it cannot be read).
void* current_context() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  CUcontext c = nullptr;
  if (fn == nullptr || fn(&c) != CUDA_SUCCESS) return nullptr;
  return reinterpret_cast<void*>(c);
}

// Device address of g_linear_scratch on the current device, looked up on the
// first call for that device and cached together with the current context; a
// different context (the device was reset and its context made anew, say)
// triggers a new lookup, since the module, and the array with it, was loaded
// again. Fails if `x` does not live on the current device, whose scratch the
// call would otherwise pair with another device's data.
ck_status static_scratch_addr(const void* x, void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess)
    return fail(CK_ERR_CUDA, "linear_w4a4_static: cudaGetDevice failed: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxScratchDevices)
    return fail(CK_ERR_UNSUPPORTED, "linear_w4a4_static: device ordinal %d >= %d", dev, kMaxScratchDevices);
  cudaPointerAttributes pa;
  e = cudaPointerGetAttributes(&pa, x);
  if (e != cudaSuccess) {
    cudaGetLastError();   // clear the error this records, so that a later launch check does not see it
    return fail(CK_ERR_INVALID_ARG, "linear_w4a4_static: x is not a device pointer (%s)", cudaGetErrorString(e));
  }
  if (pa.type != cudaMemoryTypeDevice && pa.type != cudaMemoryTypeManaged)
    return fail(CK_ERR_INVALID_ARG, "linear_w4a4_static: x is not device memory");
  if (pa.device != dev)
    return fail(CK_ERR_INVALID_ARG,
                "linear_w4a4_static: x is on device %d but device %d is current; make x's device current",
                pa.device, dev);
  void* ctx = current_context();
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchEntry& ent = g_scratch[dev];
  if (ent.addr == nullptr || ent.ctx != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_linear_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(CK_ERR_CUDA, "linear_w4a4_static: cudaGetSymbolAddress failed on device %d: %s", dev,
                  cudaGetErrorString(e));
    ent.addr = p;
    ent.ctx = ctx;
  }
  *out = ent.addr;
  return CK_OK;
}

}  // namespace

extern "C" {

ck_status ck_linear_w4a4_static(const void* x, ck_dtype xt, int64_t M, int64_t K, int64_t N,
                                int64_t ldx, int group_size, const uint8_t* w_packed,
                                const uint16_t* w_scale, const uint16_t* bias, uint16_t* y,
                                void* stream) {
  ck_status r = check_gemm_shape("linear_w4a4_static", M, K, N, kTermLinear);
  if (r != CK_OK) return r;
  const size_t need = linear_ws_bytes(M, K);
  if (need > (size_t)CK_LINEAR_STATIC_SCRATCH_BYTES)
    return fail(CK_ERR_UNSUPPORTED,
                "linear_w4a4_static: M=%lld, K=%lld need %zu bytes of scratch, more than the %zu-byte "
                "static scratch; call ck_linear_w4a4 with a workspace instead",
                (long long)M, (long long)K, need, (size_t)CK_LINEAR_STATIC_SCRATCH_BYTES);
  if (x == nullptr) return fail(CK_ERR_INVALID_ARG, "linear_w4a4_static: null pointer");
  void* scratch = nullptr;
  if ((r = static_scratch_addr(x, &scratch)) != CK_OK) return r;
  return ck_linear_w4a4(x, xt, M, K, N, ldx, group_size, w_packed, w_scale, bias, y, scratch,
                        (size_t)CK_LINEAR_STATIC_SCRATCH_BYTES, stream);
}

ck_status ck_gemm_w4a4_i32(const uint8_t* qa_packed, const uint8_t* w_packed, int64_t M, int64_t K,
                           int64_t N, int32_t* acc, void* stream) {
  ck_status r = check_gemm_shape("gemm_w4a4_i32", M, K, N, kTermW4A4);
  if (r != CK_OK) return r;
  if (!qa_packed || !w_packed || !acc) return fail(CK_ERR_INVALID_ARG, "gemm_w4a4_i32: null pointer");
  if (!aligned(qa_packed, 16) || !aligned(w_packed, 16)) return fail(CK_ERR_UNSUPPORTED, "gemm_w4a4_i32: operands must be 16-byte aligned");
  if (!aligned(acc, 4)) return fail(CK_ERR_INVALID_ARG, "gemm_w4a4_i32: misaligned output");
  return gemm_impl<ck::gemm::OP_PACKED4, ck::gemm::OP_PACKED4, ck::gemm::EPI_I32>(qa_packed, M, K, N, w_packed, nullptr, nullptr, nullptr, nullptr, acc, S(stream));
}

ck_status ck_gemm_w4a8_i32(const int8_t* qa, const uint8_t* w_packed, int64_t M, int64_t K, int64_t N,
                           int32_t* acc, void* stream) {
  ck_status r = check_gemm_shape("gemm_w4a8_i32", M, K, N, kTermW4A8);
  if (r != CK_OK) return r;
  if (!qa || !w_packed || !acc) return fail(CK_ERR_INVALID_ARG, "gemm_w4a8_i32: null pointer");
  if (!aligned(qa, 16) || !aligned(w_packed, 16)) return fail(CK_ERR_UNSUPPORTED, "gemm_w4a8_i32: operands must be 16-byte aligned");
  if (!aligned(acc, 4)) return fail(CK_ERR_INVALID_ARG, "gemm_w4a8_i32: misaligned output");
  return gemm_impl<ck::gemm::OP_INT8, ck::gemm::OP_PACKED4, ck::gemm::EPI_I32>(qa, M, K, N, w_packed, nullptr, nullptr, nullptr, nullptr, acc, S(stream));
}

}  // extern "C"

namespace {

// W4A8 GEMV on the tensor cores: ceil(N / 128) row blocks, each one cluster of
// `split` CTAs dividing K. One wave at one CTA per SM sets the split (at most 8
// and at most K / 128), raised where a CTA's activations would not fit.
ck_status gemv_w4a8_tc_launch(const int8_t* xq, const float* x_scale, int64_t M, int64_t K, int64_t N,
                              const uint8_t* w_packed, const __nv_bfloat16* sw, const __nv_bfloat16* bb,
                              __nv_bfloat16* yy, cudaStream_t st) {
  using namespace ck::gtc;
  constexpr int kSmemMax = 227 * 1024;
  const int nkb = (int)(K / BK);
  const int64_t rb = (N + BM - 1) / BM;
  const int split_max = std::min(8, nkb);
  int split = (int)std::max<int64_t>(1, std::min<int64_t>(split_max, sm_count() / rb));
  while (split < split_max && smem_bytes((nkb + split - 1) / split) > kSmemMax) ++split;
  const int nkbc_max = (nkb + split - 1) / split;
  const int smem = smem_bytes(nkbc_max);
  if (smem > kSmemMax) return fail(CK_ERR_UNSUPPORTED, "gemv_w4a8_tc: K=%lld too large", (long long)K);
  if (rb * split > INT32_MAX) return fail(CK_ERR_UNSUPPORTED, "gemv_w4a8_tc: N=%lld too large", (long long)N);
  CUtensorMap tw, tx;
  ck_status r = make_tmap(&tw, w_packed, (uint64_t)K / 2, (uint64_t)N, (uint64_t)K / 2, PKB, BM,
                          CU_TENSOR_MAP_SWIZZLE_NONE);
  if (r != CK_OK) return r;
  r = make_tmap(&tx, xq, (uint64_t)K, (uint64_t)M, (uint64_t)K, BK, BN, CU_TENSOR_MAP_SWIZZLE_128B);
  if (r != CK_OK) return r;
  auto kern = gemv_w4a8_tc_kernel;
  struct Tag {};
  if ((r = ensure_smem_attr<Tag>(kern, kSmemMax)) != CK_OK) return r;
  Params p;
  p.M = (int)M; p.K = (int)K; p.N = (int)N;
  p.S = split; p.nkb = nkb; p.nkbc_max = nkbc_max;
  p.xs = x_scale; p.sw = sw; p.bias = bb; p.y = yy;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)split;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3((unsigned)(rb * split), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tw, tx, p);
  if (e != cudaSuccess) return fail(CK_ERR_CUDA, "gemv_w4a8_tc: launch failed: %s", cudaGetErrorString(e));
  return launch_status("gemv_w4a8_tc");
}

// Tiles the row-split W4A8 kernel fills while the previous kernel still runs, at most
// this many in flight (see gemv_w4a8_stream.cuh): 3 with one token group (two CTAs per
// SM); 1 with several, whose activation loads then queue behind fewer weight bytes
// (measured at M = 16: 8.9 against 9.4 us with 3).
constexpr int kRowsplitFill = 3;
constexpr int kRowsplitFillWide = 1;
// Dynamic shared memory of a row-split CTA for more than 8 tokens: one CTA per SM
// (the 228 KB of an SM less the 1 KB the runtime reserves per CTA).
constexpr int kRowsplitSmemBig = 227 * 1024;

// The row-split W4A8 GEMV (M <= 32, K <= 4096, K % 128 == 0, N % 8 == 0, 16-byte
// aligned scales and bias). CK_ERR_UNSUPPORTED, with nothing launched, when a
// CTA's share of rows would leave its ring fewer than two stages.
ck_status gemv_w4a8_rowsplit(const int8_t* xq, const float* x_scale, int64_t M, int64_t K, int64_t N,
                             const uint8_t* w_packed, const __nv_bfloat16* sw, const __nv_bfloat16* bb,
                             __nv_bfloat16* yy, cudaStream_t st, bool a4) {
  using namespace ck::w4s;
  if (M > kMaxTokens || K > 4096 || K % 128 != 0 || N % 8 != 0) return CK_ERR_UNSUPPORTED;
  const int nt = M <= 8 ? 1 : M <= 16 ? 2 : 4;
  const int ncons = cons_warps(nt), nthreads = threads_for(nt);
  const int smax = nt == 1 ? kStreamSmemMax : kRowsplitSmemBig;
  const int64_t octets = N / 8;
  const int grid = (int)std::min<int64_t>(octets, sm_count());
  Params p;
  p.xq = xq; p.xs = x_scale; p.sw = sw; p.bias = bb; p.y = yy;
  p.M = (int)M; p.K = (int)K; p.N = (int)N;
  p.stage_bytes = (int)((16 * (K / 2) + 1023) / 1024 * 1024);
  p.max_rows = (int)(8 * ((octets + grid - 1) / grid));
  p.max_tiles = (p.max_rows + TR - 1) / TR;
  const int acc_bytes = p.max_tiles * nt * 8 * TS * 4;
  const int misc_bytes = (2 * kMaxTokens * 4 + 2 * 2 * p.max_rows + 4 + 15) / 16 * 16;
  const int bar_bytes = (2 * kMaxStages + 1 + p.max_tiles) * 8;
  const int fixed = acc_bytes + misc_bytes + bar_bytes + 1024;   // 1024: base alignment slack
  if (fixed > smax) return CK_ERR_UNSUPPORTED;
  p.ns = std::min(kMaxStages, (smax - fixed) / p.stage_bytes);
  if (p.ns < 2) return CK_ERR_UNSUPPORTED;
  // no more stages than a CTA has tiles: the shared memory left over lets the neighbouring
  // kernels' CTAs stay resident beside this one
  p.ns = std::min(p.ns, std::max(2, p.max_tiles));
  p.fill = nt == 1 ? kRowsplitFill : kRowsplitFillWide;
  p.off_acc = p.ns * p.stage_bytes;
  p.off_misc = p.off_acc + acc_bytes;
  p.off_bar = p.off_misc + misc_bytes;
  const int total = p.off_bar + bar_bytes + 1024;
  CUtensorMap tw;
  ck_status r = make_tmap_wtile(&tw, w_packed, (uint64_t)N, (uint64_t)K, TR);
  if (r != CK_OK) return r;
  const int cpw = (int)((K / 128 + ncons - 1) / ncons);
  cudaError_t e = cudaSuccess;
#define CK_W4A8_ROWSPLIT_A(NT, CPW, A4)                                                            \
  {                                                                                                \
    auto kern = w4a8_rowsplit_kernel<NT, CPW, A4>;                                                 \
    struct Tag {};                                                                                 \
    e = set_smem_max<Tag>(kern, total, smax);                                                      \
    if (e == cudaSuccess) e = launch_pdl(kern, dim3(grid), dim3(nthreads), total, st, tw, p);      \
  }
#define CK_W4A8_ROWSPLIT(NT, CPW)                                                                  \
  {                                                                                                \
    if (a4) CK_W4A8_ROWSPLIT_A(NT, CPW, true)                                                      \
    else CK_W4A8_ROWSPLIT_A(NT, CPW, false)                                                        \
  }
  if (nt == 1) {
    if (cpw <= 1) CK_W4A8_ROWSPLIT(1, 1)
    else if (cpw == 2) CK_W4A8_ROWSPLIT(1, 2)
    else if (cpw == 3) CK_W4A8_ROWSPLIT(1, 3)
    else CK_W4A8_ROWSPLIT(1, 4)
  } else if (nt == 2) {
    if (cpw <= 1) CK_W4A8_ROWSPLIT(2, 1)
    else CK_W4A8_ROWSPLIT(2, 2)
  } else {
    if (cpw <= 1) CK_W4A8_ROWSPLIT(4, 1)
    else CK_W4A8_ROWSPLIT(4, 2)
  }
#undef CK_W4A8_ROWSPLIT
#undef CK_W4A8_ROWSPLIT_A
  if (e != cudaSuccess) return fail(CK_ERR_CUDA, "gemv_w4a8: %s", cudaGetErrorString(e));
  return launch_status("gemv_w4a8");
}

}  // namespace

extern "C" {

ck_status ck_gemv_w4a8(const int8_t* xq, const float* x_scale, int64_t M, int64_t K, int64_t N,
                       const uint8_t* w_packed, const uint16_t* w_scale, const uint16_t* bias,
                       uint16_t* y, void* stream) {
  if (M <= 0 || K <= 0 || N <= 0) return fail(CK_ERR_INVALID_ARG, "gemv_w4a8: M, K, N must be > 0");
  if (M > 16) return fail(CK_ERR_UNSUPPORTED, "gemv_w4a8: M=%lld > 16", (long long)M);
  if (K % 128 != 0) return fail(CK_ERR_UNSUPPORTED, "gemv_w4a8: K must be a multiple of 128");
  if (K > INT32_MAX / 2 || N > INT32_MAX / 2) return fail(CK_ERR_UNSUPPORTED, "gemv_w4a8: dimension too large");
  if (check_acc_range("gemv_w4a8", K, kTermGemv) != CK_OK) return CK_ERR_UNSUPPORTED;
  if (!xq || !x_scale || !w_packed || !w_scale || !y) return fail(CK_ERR_INVALID_ARG, "gemv_w4a8: null pointer");
  if (!aligned(xq, 16) || !aligned(w_packed, 16)) return fail(CK_ERR_UNSUPPORTED, "gemv_w4a8: operands must be 16-byte aligned");
  if (!aligned(x_scale, 4) || !aligned(w_scale, 2) || !aligned(y, 2) || (bias && !aligned(bias, 2)))
    return fail(CK_ERR_INVALID_ARG, "gemv_w4a8: misaligned scale, bias or output");
  const auto* sw = reinterpret_cast<const __nv_bfloat16*>(w_scale);
  const auto* bb = reinterpret_cast<const __nv_bfloat16*>(bias);
  auto* yy = reinterpret_cast<__nv_bfloat16*>(y);
  if (K <= 4096 && N % 8 == 0 && aligned(sw, 16) && (bb == nullptr || aligned(bb, 16))) {
    // row-split streaming path: whole octets of rows per CTA, 16-row tiles (gemv_w4a8_stream.cuh)
    ck_status r = gemv_w4a8_rowsplit(xq, x_scale, M, K, N, w_packed, sw, bb, yy, S(stream));
    if (r != CK_ERR_UNSUPPORTED) return r;
  }
  if (K <= 4096 && M <= 8) {
    // streaming path for up to 8 activation rows: 16-row weight tiles as the m16 operand
    using namespace ck::gstream;
    W4A8Params sp;
    sp.xq = xq; sp.xs = x_scale; sp.w = w_packed; sp.sw = sw; sp.bias = bb; sp.y = yy;
    sp.M = (int)M; sp.K = (int)K; sp.N = (int)N;
    sp.ntiles = (int)((N + 15) / 16);
    const int grid = std::min(sp.ntiles, sm_count());
    const int tpc = (sp.ntiles + grid - 1) / grid;
    CUtensorMap tw;
    ck_status r = make_tmap_wtile(&tw, w_packed, (uint64_t)N, (uint64_t)K, 16);
    if (r != CK_OK) return r;
    sp.L = stream_layout_m8((int)(16 * (K / 2)), kCons * 8 * 4 + 2 * 16 * tpc * 4 + 16);
    if (sp.L.ns >= 2) {   // else too many tiles per CTA for the ring: general kernel
      const int nchunk = (int)(K / 128), cpw = (nchunk + kCons - 1) / kCons;
      cudaError_t e;
#define CK_W4A8_STREAM_M8(CPW)                                                                   \
      {                                                                                            \
        auto kern = w4a8_stream_m8_kernel<CPW>;                                                    \
        struct Tag {};                                                                             \
        e = set_smem_max<Tag>(kern, sp.L.total);                                                   \
        if (e == cudaSuccess) e = launch_pdl(kern, dim3(grid), dim3(kThreads), sp.L.total, S(stream), tw, sp); \
      }
      if (cpw <= 1) CK_W4A8_STREAM_M8(1)
      else if (cpw == 2) CK_W4A8_STREAM_M8(2)
      else if (cpw == 3) CK_W4A8_STREAM_M8(3)
      else CK_W4A8_STREAM_M8(4)
#undef CK_W4A8_STREAM_M8
      if (e != cudaSuccess) return fail(CK_ERR_CUDA, "gemv_w4a8: %s", cudaGetErrorString(e));
      return launch_status("gemv_w4a8");
    }
  }
  if (K <= 4096) {
    // streaming path: 8-row weight tiles through a shared-memory ring, one CTA per SM
    using namespace ck::gstream;
    W4A8Params sp;
    sp.xq = xq; sp.xs = x_scale; sp.w = w_packed; sp.sw = sw; sp.bias = bb; sp.y = yy;
    sp.M = (int)M; sp.K = (int)K; sp.N = (int)N;
    sp.ntiles = (int)((N + 7) / 8);
    const int grid = std::min(sp.ntiles, sm_count());
    const int tpc = (sp.ntiles + grid - 1) / grid;
    sp.srow = (int)(K / 2) + 64;
    sp.L = stream_layout(8 * sp.srow, kCons * 16 * 4 + 2 * 8 * tpc * 4 + 16);
    if (sp.L.ns >= 2) {   // else too many tiles per CTA for the ring: general kernel
      const int nchunk = (int)(K / 128), cpw = (nchunk + kCons - 1) / kCons;
      cudaError_t e;
#define CK_W4A8_STREAM(CPW)                                                                      \
      {                                                                                            \
        auto kern = w4a8_stream_kernel<CPW>;                                                       \
        struct Tag {};                                                                             \
        e = set_smem_max<Tag>(kern, sp.L.total);                                                   \
        if (e == cudaSuccess) e = launch_pdl(kern, dim3(grid), dim3(kThreads), sp.L.total, S(stream), sp); \
      }
      if (cpw <= 1) CK_W4A8_STREAM(1)
      else if (cpw == 2) CK_W4A8_STREAM(2)
      else if (cpw == 3) CK_W4A8_STREAM(3)
      else CK_W4A8_STREAM(4)
#undef CK_W4A8_STREAM
      if (e != cudaSuccess) return fail(CK_ERR_CUDA, "gemv_w4a8: %s", cudaGetErrorString(e));
      return launch_status("gemv_w4a8");
    }
  }
  const unsigned grid = (unsigned)((N + ck::w4a8::kRows - 1) / ck::w4a8::kRows);
  if (M <= 8)
    ck::w4a8::gemv_w4a8_kernel<1><<<grid, ck::w4a8::kWarps * 32, 0, S(stream)>>>(xq, x_scale, (int)M, (int)K, (int)N, w_packed, sw, bb, yy);
  else
    ck::w4a8::gemv_w4a8_kernel<2><<<grid, ck::w4a8::kWarps * 32, 0, S(stream)>>>(xq, x_scale, (int)M, (int)K, (int)N, w_packed, sw, bb, yy);
  return launch_status("gemv_w4a8");
}

ck_status ck_gemv_w4a8_tc(const int8_t* xq, const float* x_scale, int64_t M, int64_t K, int64_t N,
                          const uint8_t* w_packed, const uint16_t* w_scale, const uint16_t* bias,
                          uint16_t* y, void* stream) {
  if (M <= 0 || K <= 0 || N <= 0) return fail(CK_ERR_INVALID_ARG, "gemv_w4a8_tc: M, K, N must be > 0");
  if (M > 16) return fail(CK_ERR_UNSUPPORTED, "gemv_w4a8_tc: M=%lld > 16", (long long)M);
  if (K % 128 != 0) return fail(CK_ERR_UNSUPPORTED, "gemv_w4a8_tc: K must be a multiple of 128");
  if (K > 8192) return fail(CK_ERR_UNSUPPORTED, "gemv_w4a8_tc: K=%lld > 8192", (long long)K);
  if (N > INT32_MAX / 2) return fail(CK_ERR_UNSUPPORTED, "gemv_w4a8_tc: dimension too large");
  if (!xq || !x_scale || !w_packed || !w_scale || !y) return fail(CK_ERR_INVALID_ARG, "gemv_w4a8_tc: null pointer");
  if (!aligned(xq, 16) || !aligned(w_packed, 16))
    return fail(CK_ERR_UNSUPPORTED, "gemv_w4a8_tc: operands must be 16-byte aligned");
  if (!aligned(x_scale, 4) || !aligned(w_scale, 2) || !aligned(y, 2) || (bias && !aligned(bias, 2)))
    return fail(CK_ERR_INVALID_ARG, "gemv_w4a8_tc: misaligned scale, bias or output");
  return gemv_w4a8_tc_launch(xq, x_scale, M, K, N, w_packed, reinterpret_cast<const __nv_bfloat16*>(w_scale),
                             reinterpret_cast<const __nv_bfloat16*>(bias), reinterpret_cast<__nv_bfloat16*>(y),
                             S(stream));
}

ck_status ck_gemv_awq_w4a16(const void* x, ck_dtype dt, int64_t M, int64_t K, int64_t N, int group_size,
                            const uint8_t* qweight, const void* wscales, const void* wzeros,
                            const void* bias, void* y, void* stream) {
  if (M <= 0 || K <= 0 || N <= 0) return fail(CK_ERR_INVALID_ARG, "gemv_awq_w4a16: M, K, N must be > 0");
  if (dt != CK_BF16 && dt != CK_FP16) return fail(CK_ERR_INVALID_ARG, "gemv_awq_w4a16: unknown dtype");
  if (M > 8) return fail(CK_ERR_UNSUPPORTED, "gemv_awq_w4a16: M=%lld > 8", (long long)M);
  if (group_size <= 0 || group_size % 64 != 0)
    return fail(CK_ERR_UNSUPPORTED, "gemv_awq_w4a16: group_size=%d must be a multiple of 64", group_size);
  if (K % group_size != 0) return fail(CK_ERR_INVALID_ARG, "gemv_awq_w4a16: K %% group_size != 0");
  if (K > INT32_MAX / 2 || N > INT32_MAX / 2) return fail(CK_ERR_UNSUPPORTED, "gemv_awq_w4a16: dimension too large");
  if (!x || !qweight || !wscales || !wzeros || !y) return fail(CK_ERR_INVALID_ARG, "gemv_awq_w4a16: null pointer");
  if (!aligned(x, 16) || !aligned(qweight, 16)) return fail(CK_ERR_UNSUPPORTED, "gemv_awq_w4a16: x and qweight must be 16-byte aligned");
  if (!aligned(wscales, 2) || !aligned(wzeros, 2) || !aligned(y, 2) || (bias && !aligned(bias, 2)))
    return fail(CK_ERR_INVALID_ARG, "gemv_awq_w4a16: misaligned scales, zeros, bias or output");
  if (K <= 4096 && K / group_size <= 256 && N % 8 == 0 && is_pow2(group_size / 64) && aligned(wscales, 16) &&
      aligned(wzeros, 16)) {
    // streaming path: 16-row weight tiles plus their scales and zeros through a shared-memory ring
    using namespace ck::gstream;
    CUtensorMap ts, tz;
    const uint32_t ngrp = (uint32_t)(K / group_size);
    ck_status r = make_tmap(&ts, wscales, (uint64_t)N, ngrp, (uint64_t)N * 2, 16, ngrp, CU_TENSOR_MAP_SWIZZLE_NONE,
                            CU_TENSOR_MAP_DATA_TYPE_UINT16);
    if (r != CK_OK) return r;
    r = make_tmap(&tz, wzeros, (uint64_t)N, ngrp, (uint64_t)N * 2, 16, ngrp, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_DATA_TYPE_UINT16);
    if (r != CK_OK) return r;
    AwqParams ap;
    ap.x = x; ap.qw = qweight; ap.bias = bias; ap.y = y;
    ap.M = (int)M; ap.K = (int)K; ap.N = (int)N; ap.G = group_size;
    ap.gshift = 0;
    while ((64 << ap.gshift) < group_size) ++ap.gshift;
    ap.ntiles = (int)((N + 15) / 16);
    ap.srow = (int)(K / 2) + 32;
    ap.w_bytes = (16 * ap.srow + 127) / 128 * 128;    // padded rows; the scale tiles follow 128-byte aligned
    ap.sz_bytes = (int)ngrp * 16 * 2;
    ap.sz_stride = (ap.sz_bytes + 127) / 128 * 128;    // every tensor-copy destination 128-byte aligned
    // two CTAs per SM within a call: the call is bound by the consumers' issue, not by the
    // weight stream, so 16 consumer warps per SM beat keeping a slot for the next call's CTA
    // (measured at K = 3072, N = 18432: 13.7 -> 12.4 us)
    const int grid = std::min(ap.ntiles, 2 * sm_count());
    const int tpc = (ap.ntiles + grid - 1) / grid;
    ap.L = stream_layout(ap.w_bytes + 2 * ap.sz_stride, 16 * tpc * 4 + 16);
    if (ap.L.ns >= 2) {   // else too many tiles per CTA for the ring: general kernel
      const int nsub = (int)(K / 64), spw = (nsub + kCons - 1) / kCons;
      cudaError_t e = cudaSuccess;
#define CK_AWQ_STREAM(T, SPW)                                                                    \
      {                                                                                            \
        auto kern = awq_stream_kernel<T, SPW>;                                                     \
        struct Tag {};                                                                             \
        e = set_smem_max<Tag>(kern, ap.L.total);                                                   \
        if (e == cudaSuccess) e = launch_pdl(kern, dim3(grid), dim3(kThreads), ap.L.total, S(stream), ts, tz, ap); \
      }
      if (dt == CK_BF16) {
        if (spw <= 2) CK_AWQ_STREAM(__nv_bfloat16, 2)
        else if (spw <= 4) CK_AWQ_STREAM(__nv_bfloat16, 4)
        else if (spw <= 6) CK_AWQ_STREAM(__nv_bfloat16, 6)
        else CK_AWQ_STREAM(__nv_bfloat16, 8)
      } else {
        if (spw <= 2) CK_AWQ_STREAM(__half, 2)
        else if (spw <= 4) CK_AWQ_STREAM(__half, 4)
        else if (spw <= 6) CK_AWQ_STREAM(__half, 6)
        else CK_AWQ_STREAM(__half, 8)
      }
#undef CK_AWQ_STREAM
      if (e != cudaSuccess) return fail(CK_ERR_CUDA, "gemv_awq_w4a16: %s", cudaGetErrorString(e));
      return launch_status("gemv_awq_w4a16");
    }
  }
  const unsigned grid = (unsigned)((N + ck::awq::kRows - 1) / ck::awq::kRows);
  if (dt == CK_BF16) {
    using T = __nv_bfloat16;
    ck::awq::gemv_awq_kernel<T><<<grid, ck::awq::kWarps * 32, 0, S(stream)>>>(
        (const T*)x, (int)M, (int)K, (int)N, group_size, qweight, (const T*)wscales, (const T*)wzeros,
        (const T*)bias, (T*)y);
  } else {
    using T = __half;
    ck::awq::gemv_awq_kernel<T><<<grid, ck::awq::kWarps * 32, 0, S(stream)>>>(
        (const T*)x, (int)M, (int)K, (int)N, group_size, qweight, (const T*)wscales, (const T*)wzeros,
        (const T*)bias, (T*)y);
  }
  return launch_status("gemv_awq_w4a16");
}

ck_status ck_device_error_check(void* stream) {
  cudaError_t e = cudaStreamSynchronize(S(stream));
  if (e != cudaSuccess) return fail(CK_ERR_CUDA, "stream error: %s", cudaGetErrorString(e));
  unsigned int w = 0;
  e = cudaMemcpyFromSymbol(&w, ck::g_err_word, sizeof(w));
  if (e != cudaSuccess) return fail(CK_ERR_CUDA, "reading the error word: %s", cudaGetErrorString(e));
  if (w != 0) {
    const unsigned int zero = 0;
    cudaMemcpyToSymbol(ck::g_err_word, &zero, sizeof(zero));
    return fail(CK_ERR_TIMEOUT, "a bounded barrier wait gave up (error word 0x%08x, site %u)", w, (w >> 8) & 0xffu);
  }
  return ok();
}

}  // extern "C"

namespace {
__global__ void selftest_wait_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    ck::mbar_init(&bar, 1);
    abort_flag = 0;
    ck::fence_mbarrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) ck::mbar_wait(&bar, 0, &abort_flag, 0x7f, limit_ns);  // nothing arrives
  __syncthreads();
}
}  // namespace

extern "C" ck_status ck_selftest_bounded_wait(int64_t timeout_ns, void* stream) {
  if (timeout_ns < 1000 || timeout_ns > 5000000000ll)
    return fail(CK_ERR_INVALID_ARG, "selftest_bounded_wait: timeout_ns outside [1e3, 5e9]");
  selftest_wait_kernel<<<1, 32, 0, S(stream)>>>((uint64_t)timeout_ns);
  return launch_status("selftest_bounded_wait");
}
