/*
 * ck.h -- C ABI of the ConvRot packed-INT4 quantized linear for NVIDIA B200 (sm_100a).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every pointer argument is a DEVICE pointer owned by the caller, unless the
 *   argument's comment says otherwise. Nothing is allocated, freed or
 *   synchronised inside a compute call: arguments are validated on the host,
 *   then the kernels are enqueued on `stream` and the call returns.
 * - `stream` is a cudaStream_t passed as an opaque pointer (NULL = the legacy
 *   default stream).
 * - Matrices are row-major. A "packed int4" matrix of logical shape (R, C) is
 *   stored as (R, C/2) bytes: bits 0..3 hold column 2j and bits 4..7 column
 *   2j+1 (comfy_kitchen/tensor/awq_w4a16.py, module docstring). Each nibble is
 *   offset binary, u = q + 8, so the signed value is q = u - 8 in [-8, 7];
 *   int8 and uint8 storage are the same bytes.
 * - bf16 / fp16 values are passed as 16-bit storage (uint16_t).
 * - Errors: CK_ERR_INVALID_ARG for null pointers, non-positive sizes,
 *   inconsistent strides or misaligned pointers; CK_ERR_UNSUPPORTED for shapes
 *   the kernels decline (the pages' "unsupported-shape decline"); CK_ERR_CUDA
 *   when a launch fails. Nothing is enqueued when validation fails.
 *   ck_last_error() returns a thread-local message for the last failure.
 * - Integer accumulation is exact int32. A shape whose K could overflow it is
 *   CK_ERR_UNSUPPORTED: K must satisfy K * max|a * w| <= 2^31 - 1. The
 *   largest term is 128 * 128 for int8 x int8 (K <= 131071), 128 * 8 for
 *   int8 x int4 (K <= 2097151), 8 * 8 for int4 x int4, 7 * 15 in the linear,
 *   and 128 * 15 in the W4A8 GEMV (K <= 1118481).
 * - Kernels that wait on shared-memory barriers give up after a bounded time
 *   and set a device error word instead of hanging; ck_device_error_check()
 *   reports it.
 * - Back-to-back calls overlap: every kernel is launched as a programmatic
 *   dependent of the previous kernel on the stream and waits for it before it
 *   reads activations or writes outputs. The decode GEMVs (and the linears'
 *   small-batch route, which runs them) treat their WEIGHT operands --
 *   packed weights, weight scales, zeros and bias -- as constant data and
 *   start streaming them before that wait. So do not let the kernel launched
 *   immediately before such a call on the same stream write those weights;
 *   any other operation in between (another kernel, a copy, an event wait)
 *   makes the ordering complete again.
 */
#ifndef CK_H_
#define CK_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  CK_OK = 0,
  CK_ERR_INVALID_ARG = 1,
  CK_ERR_UNSUPPORTED = 2,
  CK_ERR_CUDA = 3,
  CK_ERR_TIMEOUT = 4
} ck_status;

typedef enum { CK_BF16 = 0, CK_FP16 = 1 } ck_dtype;

/*
 * Fused group rotation + rowwise symmetric quantization
 * ("quantize_and_rotate_rowwise" of comfy-kitchen PR #155 "[Feat][Ascend] Add
 * fused RotateQuant backend", section "What this PR does").
 *
 * For every row m of x and every group g of `group_size` consecutive columns:
 *   y_g = x_g . H_G / sqrt(G)          (Sylvester-ordered Hadamard, fp32)
 *   s_m = max_k |y[m,k]| / qmax         (qmax = 7 for bits=4, 127 for bits=8;
 *                                        s_m = 1 for an all-zero row)
 *   q[m,k] = clamp(round_half_even(y[m,k] / s_m), -qmax, qmax)
 *
 * x          : (M, K) bf16 or fp16 (xt), row stride ldx >= K elements,
 *              16-byte aligned rows (ldx % 8 == 0, x 16-byte aligned).
 * group_size : 1 (no rotation), 16, 64 or 256; K % group_size == 0, K % 8 == 0.
 * bits       : 4 -> q_out is (M, K/2) packed int4, u = q + 8, low nibble =
 *                   even column;
 *              8 -> q_out is (M, K) int8.
 * scale_out  : (M) float32, always > 0.
 * M may be any number of flattened leading dimensions; M == 0 is a no-op.
 */
ck_status ck_rotate_quant_rowwise(const void* x, ck_dtype xt, int64_t M, int64_t K,
                                  int64_t ldx, int group_size, int bits, void* q_out,
                                  float* scale_out, void* stream);

/*
 * Same rotation and quantization as ck_rotate_quant_rowwise, with the codes
 * stored one per byte: q_out is (M, K) int8 for bits = 4 (|q| <= 7) as well as
 * bits = 8 (|q| <= 127). This is the activation format the W4A4 linear feeds
 * its GEMM (comfy-kitchen PR #212 "Related work": PR #201 removes the
 * activation pack/unpack); the int4 code values are identical to the packed
 * output's.
 */
ck_status ck_rotate_quant_rowwise_i8(const void* x, ck_dtype xt, int64_t M, int64_t K,
                                     int64_t ldx, int group_size, int bits, int8_t* q_out,
                                     float* scale_out, void* stream);

/*
 * ck_rotate_quant_rowwise with a GENERAL rotation: y_g = x_g . R for every
 * group g of every row, R any G x G matrix (the pages test
 * quantize_and_rotate_rowwise with "asymmetric-rotation inputs", comfy-kitchen
 * PR #155, "How was this patch tested?"), followed by the same rowwise
 * symmetric quantization and the same output formats as
 * ck_rotate_quant_rowwise. The product runs in fp32 on the CUDA cores (G
 * multiply-adds per element): a functional path, not the Hadamard fast path.
 * R          : (G, G) float32, row-major, device memory: y[j] = sum_i x[i] R[i][j].
 * group_size : 1 .. 256 with K % group_size == 0; K even, K <= 16384.
 * Other arguments as for ck_rotate_quant_rowwise (x 2-byte aligned suffices).
 */
ck_status ck_rotate_quant_rowwise_r(const void* x, ck_dtype xt, int64_t M, int64_t K, int64_t ldx,
                                    int group_size, const float* R, int bits, void* q_out,
                                    float* scale_out, void* stream);

/*
 * ck_rotate_quant_rowwise of a * x, for a caller-supplied tensor-wise input
 * scale a. Two passages touch this scale:
 *   - comfy-kitchen PR #155, "How was this patch tested?": caller-provided
 *     zero tensor-wise scales follow eager quantization;
 *   - stable-diffusion.cpp PR #2276, review comments on docs/int8_convrot.md:
 *     inputs whose scale is not 1 are scaled, then quantized.
 * Neither gives a formula. The reading taken is that a multiplies x before
 * the rotation:
 *   y_g = (a x_g) . H_G / sqrt(G), then s_m and q as for ck_rotate_quant_rowwise.
 * a = 0 makes every row all-zero: s_m = 1 and q = 0. a = 1 gives exactly the
 * results of ck_rotate_quant_rowwise. Same kernel and speed: the scale folds
 * into the transform's normalisation.
 * input_scale : host value, finite and >= 0 (else CK_ERR_INVALID_ARG). The
 *               scaled rows must stay in fp32's normal range: a row whose
 *               nonzero scale s_m would fall below 2^-126, or overflow, gets
 *               unspecified codes.
 * group_size  : a power of two <= 256. 1 (no rotation) is accepted only
 *               with a = 1 (CK_ERR_UNSUPPORTED otherwise).
 * Other arguments, formats and errors as for ck_rotate_quant_rowwise.
 */
ck_status ck_rotate_quant_rowwise_scaled(const void* x, ck_dtype xt, int64_t M, int64_t K,
                                         int64_t ldx, int group_size, int bits, float input_scale,
                                         void* q_out, float* scale_out, void* stream);

/*
 * Integer matmul of packed int4 activations with packed int4 weights, int32
 * accumulation on the tcgen05 tensor cores, and the rowwise-scale epilogue
 * (the "EpiRowwise" of comfy-kitchen PR #182, Description):
 *   acc[m,n] = sum_k qa[m,k] * w[n,k]
 *   y[m,n]   = bf16_rne( (float(acc) * a_scale[m]) * float(w_scale[n]) (+ bias[n]) )
 *
 * qa_packed : (M, K/2) packed int4 (e.g. ck_rotate_quant_rowwise with bits=4).
 * a_scale   : (M) float32.
 * w_packed  : (N, K/2) packed int4 weights ("convrot_w4a4", stable-diffusion.cpp
 *             PR #2276, Summary); 16-byte aligned.
 * w_scale   : (N) bf16 per-output-row weight scale.
 * bias      : (N) bf16 or NULL.
 * y         : (M, N) bf16.
 * Requires K % 32 == 0 (packed rows are whole 16-byte units for the TMA) and
 * 16-byte aligned qa_packed / w_packed; otherwise CK_ERR_UNSUPPORTED.
 */
ck_status ck_gemm_w4a4(const uint8_t* qa_packed, const float* a_scale, int64_t M, int64_t K,
                       int64_t N, const uint8_t* w_packed, const uint16_t* w_scale,
                       const uint16_t* bias, uint16_t* y, void* stream);

/*
 * Large-M W4A8 GEMM ("asym_w4a8_int8", stable-diffusion.cpp PR #2276,
 * Summary): int8 activation codes times packed int4 weights, the same main
 * loop and epilogue as ck_gemm_w4a4 with the activation tile loaded by TMA
 * instead of decoded. ck_linear_w4a4 runs exactly ck_rotate_quant_rowwise_i8
 * (bits=4) followed by this call.
 * qa (M, K) int8 (any codes in [-127, 127]), 16-byte aligned; K % 32 == 0.
 */
ck_status ck_gemm_w4a8(const int8_t* qa, const float* a_scale, int64_t M, int64_t K, int64_t N,
                       const uint8_t* w_packed, const uint16_t* w_scale, const uint16_t* bias,
                       uint16_t* y, void* stream);

/*
 * Unpacks a packed int4 matrix (R, C/2) into int8 (R, C) with value u - 8: the
 * weight preparation that comfy-kitchen PR #212 ("Summary", "Memory and support
 * limits") caches across calls, as a standalone pass the caller can run once.
 * Requires C even, R*C/2 a multiple of 16 and 16-byte aligned pointers.
 */
ck_status ck_unpack_int4(const uint8_t* packed, int64_t R, int64_t C, int8_t* out, void* stream);

/*
 * ck_gemm_w4a4 with both operands already int8 (activation codes from
 * ck_rotate_quant_rowwise_i8, weights from ck_unpack_int4): the pre-decoded
 * weight variant, trading twice the weight bytes for no in-kernel decode.
 * qa (M, K) int8, w (N, K) int8, both 16-byte aligned; K % 32 == 0.
 */
ck_status ck_gemm_s8(const int8_t* qa, const float* a_scale, int64_t M, int64_t K, int64_t N,
                     const int8_t* w, const uint16_t* w_scale, const uint16_t* bias, uint16_t* y,
                     void* stream);

/* Bytes of device workspace ck_linear_w4a4 needs for M rows of logical width K. */
size_t ck_linear_w4a4_workspace_bytes(int64_t M, int64_t K);

/*
 * The ConvRot W4A4 linear ("public ConvRot W4A4 Linear dispatcher",
 * comfy-kitchen PR #212; packed formats of stable-diffusion.cpp PR #2276):
 * y = bf16(rotate-quantize(x) . W^T * scales (+ bias)), computed as
 * ck_linear_w4a4_quantize followed by ck_linear_w4a4_matmul. Results equal
 * ck_rotate_quant_rowwise(bits=4) followed by ck_gemm_w4a4 bit for bit.
 * K is the LOGICAL inner dimension (the packed weight has K/2 bytes per row);
 * K % 32 == 0 and K % group_size == 0.
 * workspace : device buffer of at least ck_linear_w4a4_workspace_bytes(M, K)
 *             bytes, 256-byte aligned; opaque scratch written by the quantize
 *             phase and read by the matmul phase.
 * Other arguments as for ck_rotate_quant_rowwise and ck_gemm_w4a4.
 */
ck_status ck_linear_w4a4(const void* x, ck_dtype xt, int64_t M, int64_t K, int64_t N,
                         int64_t ldx, int group_size, const uint8_t* w_packed,
                         const uint16_t* w_scale, const uint16_t* bias, uint16_t* y,
                         void* workspace, size_t ws_bytes, void* stream);

/*
 * The two phases of ck_linear_w4a4, callable separately (to time or overlap
 * them). Phase 1 rotates and quantizes x into `workspace`: the int4 codes
 * stored one per byte (as comfy-kitchen PR #212 "Related work" notes, #201
 * does away with the activation pack/unpack) -- for small batches packed two
 * per byte, since every SM of that route reads all of them -- and the row
 * scales, in a layout private to the library that depends only on (M, K). Phase 2 multiplies
 * those codes with the packed int4 weights and applies the rowwise-scale
 * epilogue: on the tensor-core GEMM, or for small batches (M <= 64, K <= 4096,
 * K % 128 == 0) on the streaming decode-GEMV kernels, which keep every SM
 * busy at such M. The result does not depend on the route. Call both phases
 * with the same M and K.
 */
ck_status ck_linear_w4a4_quantize(const void* x, ck_dtype xt, int64_t M, int64_t K, int64_t ldx,
                                  int group_size, void* workspace, size_t ws_bytes, void* stream);
ck_status ck_linear_w4a4_matmul(int64_t M, int64_t K, int64_t N, const uint8_t* w_packed,
                                const uint16_t* w_scale, const uint16_t* bias, uint16_t* y,
                                const void* workspace, size_t ws_bytes, void* stream);

/*
 * ck_linear_w4a4 of a * x, for a tensor-wise input scale a. It follows the
 * reading of ck_rotate_quant_rowwise_scaled. stable-diffusion.cpp PR #2276,
 * review comments on docs/int8_convrot.md: ggml_mul_mat_w4_convrot scales
 * inputs whose scale is not 1, then quantizes them. y is the linear of a * x
 * and is not divided by a afterwards. a = 1 gives exactly ck_linear_w4a4's
 * results, and a = 0 gives y = bias (or 0) in every row.
 * input_scale : as for ck_rotate_quant_rowwise_scaled.
 * Other arguments, the workspace and its size as for ck_linear_w4a4.
 */
ck_status ck_linear_w4a4_scaled(const void* x, ck_dtype xt, int64_t M, int64_t K, int64_t N,
                                int64_t ldx, int group_size, float input_scale,
                                const uint8_t* w_packed, const uint16_t* w_scale,
                                const uint16_t* bias, uint16_t* y, void* workspace,
                                size_t ws_bytes, void* stream);

/* Bytes of device workspace ck_linear_w4a8 needs (the same layout and size as the W4A4 linear's). */
size_t ck_linear_w4a8_workspace_bytes(int64_t M, int64_t K);

/*
 * The W4A8 ConvRot linear, for the "asym_w4a8_int8" packed format of
 * stable-diffusion.cpp PR #2276 (Summary; read as int4 weights against int8
 * activations, no weight zero point): every row of x is rotated as in
 * ck_rotate_quant_rowwise and quantized to INT8 codes (qmax = 127), then
 * multiplied with the packed int4 weights on the same routes as ck_linear_w4a4
 * (tensor-core GEMM, or the decode GEMV for M <= 64, K <= 4096,
 * K % 128 == 0), with the same epilogue:
 *   y[m,n] = bf16_rne( (float(sum_k q8[m,k] (u[n,k] - 8)) * s_m) * w_scale[n] (+ bias[n]) )
 * The result equals ck_rotate_quant_rowwise(bits=8) followed by ck_gemm_w4a8
 * bit for bit. K % 32 == 0 and K % group_size == 0; K <= 1118481 (int32
 * accumulator).
 * workspace : at least ck_linear_w4a8_workspace_bytes(M, K) bytes, 256-byte
 *             aligned, opaque.
 * Other arguments as for ck_linear_w4a4.
 */
ck_status ck_linear_w4a8(const void* x, ck_dtype xt, int64_t M, int64_t K, int64_t N,
                         int64_t ldx, int group_size, const uint8_t* w_packed,
                         const uint16_t* w_scale, const uint16_t* bias, uint16_t* y,
                         void* workspace, size_t ws_bytes, void* stream);

/*
 * ck_linear_w4a4 on weights already unpacked to int8: the weight-cache
 * trade of comfy-kitchen PR #212 ("[Perf][Ascend] Reuse unpacked W4A4 weights
 * within an explicit scope", Summary and "Memory and support limits"), where
 * the caller unpacks the packed weights once (ck_unpack_int4) and reuses the
 * int8 copy across calls. The int8 copy costs twice the packed bytes of
 * device memory; in exchange the GEMM loads both operands as int8 tiles and
 * decodes nothing. The result equals ck_linear_w4a4's bit for bit.
 * w_s8      : (N, K) int8, values u - 8 in [-8, 7] (the output of
 *             ck_unpack_int4 on the packed weights), 16-byte aligned.
 * workspace : at least ck_linear_w4a4_workspace_bytes(M, K) bytes.
 * Always runs the tensor-core GEMM (no small-batch route): meant for large M,
 * where the in-kernel weight decode is the cost it removes.
 * Other arguments as for ck_linear_w4a4.
 */
ck_status ck_linear_w4a4_predecoded(const void* x, ck_dtype xt, int64_t M, int64_t K, int64_t N,
                                    int64_t ldx, int group_size, const int8_t* w_s8,
                                    const uint16_t* w_scale, const uint16_t* bias, uint16_t* y,
                                    void* workspace, size_t ws_bytes, void* stream);

/* Size of the scratch built into the library for ck_linear_w4a4_static: 32 MiB per device. */
#define CK_LINEAR_STATIC_SCRATCH_BYTES (32u * 1024u * 1024u)

/*
 * ck_linear_w4a4 for callers that cannot hand the library a workspace. The
 * ConvRot pages have no counterpart to this entry point; it exists only
 * because of how some callers are built.
 *
 * Who needs it: a caller that owns the input and output buffers but has no
 * way to get device scratch -- for example a plugin whose host passes it
 * only tensors, or code running where cudaMalloc is not allowed because it
 * can block or synchronise the device, or where every byte of device memory
 * belongs to another allocator. Such a caller cannot use ck_linear_w4a4,
 * which needs a workspace of ck_linear_w4a4_workspace_bytes(M, K) bytes.
 *
 * What it does: the same computation as ck_linear_w4a4 with the same
 * arguments minus workspace/ws_bytes, and the same results bit for bit. The
 * scratch is a fixed CK_LINEAR_STATIC_SCRATCH_BYTES block of device memory
 * inside the library, reserved by the CUDA runtime when the library's GPU
 * code is loaded on a device. The call allocates and frees nothing.
 *
 * Cost to every user of the library: loading the library's GPU code on a
 * device reserves these 32 MiB there for the life of the process (or of the
 * device's context), whichever entry points the process calls.
 *
 * Limits and rules:
 * - The scratch must hold ck_linear_w4a4_workspace_bytes(M, K) bytes, i.e.
 *   about M*K + 8*M. Larger problems (for instance M = 8192, K = 10240) get
 *   CK_ERR_UNSUPPORTED with a message naming the sizes, and nothing runs.
 *   M = 8192, K = 3840 fits.
 * - Set-up: the first call on each device (with that device current) looks up
 *   the scratch's device address and caches it with the device's current
 *   context. Make that first call before starting any stream capture. If the
 *   context changes (after cudaDeviceReset, say) the next call looks the
 *   address up again.
 * - x must live on the current device (CK_ERR_INVALID_ARG otherwise): the
 *   scratch used is the current device's.
 * - Nothing in the scratch needs to start at zero: every byte the GEMM phase
 *   reads is written earlier in the same call by the quantize phase.
 * - There is one scratch per device, shared by every call on that device.
 *   Calls whose work can overlap on the GPU -- issued on different streams
 *   without ordering between them, or from several host threads -- race on
 *   it and may produce wrong results. Calls on one stream run one after
 *   another and are safe.
 */
ck_status ck_linear_w4a4_static(const void* x, ck_dtype xt, int64_t M, int64_t K, int64_t N,
                                int64_t ldx, int group_size, const uint8_t* w_packed,
                                const uint16_t* w_scale, const uint16_t* bias, uint16_t* y,
                                void* stream);

/*
 * W4A8 decode GEMV ("W4A8 decode GEMV" of comfy-kitchen PR #182, Description;
 * "asym_w4a8_int8" of stable-diffusion.cpp PR #2276): int8 activations times
 * packed int4 weights decoded in registers, int32 accumulation, same epilogue
 * as ck_gemm_w4a4 with a_scale = x_scale.
 * xq      : (M, K) int8, 16-byte aligned, 1 <= M <= 16.
 * x_scale : (M) float32.
 * Requires K % 128 == 0; otherwise CK_ERR_UNSUPPORTED.
 */
ck_status ck_gemv_w4a8(const int8_t* xq, const float* x_scale, int64_t M, int64_t K, int64_t N,
                       const uint8_t* w_packed, const uint16_t* w_scale, const uint16_t* bias,
                       uint16_t* y, void* stream);

/*
 * ck_gemv_w4a8 computed on the tcgen05 tensor cores: 128 weight rows are the
 * MMA's M operand (decoded to unsigned bytes in shared memory), the activation
 * rows padded to 16 its N operand, and clusters of CTAs split K where the
 * row blocks are too few. The results equal ck_gemv_w4a8's bit for bit. It
 * is an alternative path, not the default: on K = 4096, N = 12288 it is
 * currently about twice as slow as ck_gemv_w4a8, whose legacy-MMA streaming
 * kernels ck_gemv_w4a8 keeps using.
 * Arguments and errors as for ck_gemv_w4a8, with K <= 8192.
 */
ck_status ck_gemv_w4a8_tc(const int8_t* xq, const float* x_scale, int64_t M, int64_t K, int64_t N,
                          const uint8_t* w_packed, const uint16_t* w_scale, const uint16_t* bias,
                          uint16_t* y, void* stream);

/*
 * AWQ W4A16 GEMV ("ck.gemv_awq_w4a16(x, qdata, wscales, wzeros, bias=,
 * group_size=)", comfy_kitchen/tensor/awq_w4a16.py, _awq_forward):
 *   W[n,k] = (u[n,k] - 8) * wscales[k/G, n] + wzeros[k/G, n]
 *   y[m,n] = sum_k x[m,k] W[n,k] (+ bias[n])       (fp32 accumulation)
 * dt applies to x, wscales, wzeros, bias and y (bf16 or fp16).
 * x       : (M, K), 1 <= M <= 8, 16-byte aligned.
 * qweight : (N, K/2) packed uint4, 16-byte aligned.
 * wscales, wzeros : (K/G, N).
 * Requires group_size % 64 == 0 and K % group_size == 0; otherwise
 * CK_ERR_UNSUPPORTED.
 */
ck_status ck_gemv_awq_w4a16(const void* x, ck_dtype dt, int64_t M, int64_t K, int64_t N,
                            int group_size, const uint8_t* qweight, const void* wscales,
                            const void* wzeros, const void* bias, void* y, void* stream);

/*
 * Test hooks: raw int32 accumulators acc[m,n] = sum_k qa[m,k] * w[n,k] through
 * the same tensor-core main loop as ck_gemm_w4a4, so identical quantized
 * inputs can be compared bit for bit.
 * ck_gemm_w4a4_i32: qa packed int4 (M, K/2).  ck_gemm_w4a8_i32: qa int8 (M, K).
 * acc: (M, N) int32. Same shape rules as ck_gemm_w4a4.
 */
ck_status ck_gemm_w4a4_i32(const uint8_t* qa_packed, const uint8_t* w_packed, int64_t M,
                           int64_t K, int64_t N, int32_t* acc, void* stream);
ck_status ck_gemm_w4a8_i32(const int8_t* qa, const uint8_t* w_packed, int64_t M, int64_t K,
                           int64_t N, int32_t* acc, void* stream);
/* Test hook of ck_gemm_s8: int8 activations and int8 weights -> int32. */
ck_status ck_gemm_s8_i32(const int8_t* qa, const int8_t* w, int64_t M, int64_t K, int64_t N,
                         int32_t* acc, void* stream);

/*
 * Synchronises `stream`, then reads and clears the device error word set by a
 * kernel whose bounded barrier wait gave up. Returns CK_ERR_TIMEOUT if it was
 * set, CK_ERR_CUDA if the stream reported an error, CK_OK otherwise.
 */
ck_status ck_device_error_check(void* stream);

/*
 * Self-test of the bounded wait: launches one block that waits on a
 * shared-memory barrier nothing will ever complete, gives up after
 * `timeout_ns` nanoseconds (1e3 .. 5e9), sets the device error word and
 * returns. ck_device_error_check() must then report CK_ERR_TIMEOUT.
 */
ck_status ck_selftest_bounded_wait(int64_t timeout_ns, void* stream);

/* Thread-local message describing the last non-OK status ("" if none). */
const char* ck_last_error(void);

/* Library version string. */
const char* ck_version(void);

#ifdef __cplusplus
}
#endif

#endif /* CK_H_ */
