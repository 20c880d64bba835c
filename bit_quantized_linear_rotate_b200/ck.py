"""Python binding of libck.so (include/ck.h): argument marshalling only.

Every function takes CUDA tensors, passes their device pointers, sizes and the
current CUDA stream to the C entry point of the same name, and raises
``CKError`` on a non-OK status. All computation happens in the library's CUDA
kernels; there is no CPU fallback: importing this module without a built
libck.so raises ImportError.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libck.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m bit_quantized_linear_rotate_b200.build` "
        "(the ConvRot kernels have no CPU fallback)")

lib = ctypes.CDLL(LIB_PATH)

CK_OK, CK_ERR_INVALID_ARG, CK_ERR_UNSUPPORTED, CK_ERR_CUDA, CK_ERR_TIMEOUT = range(5)
CK_BF16, CK_FP16 = 0, 1
STATUS_NAMES = {0: "CK_OK", 1: "CK_ERR_INVALID_ARG", 2: "CK_ERR_UNSUPPORTED", 3: "CK_ERR_CUDA",
                4: "CK_ERR_TIMEOUT"}

_p = ctypes.c_void_p
_i64 = ctypes.c_int64
_int = ctypes.c_int
_f32 = ctypes.c_float

# name -> argument types (restype is ck_status = int unless listed below)
SIGNATURES = {
    "ck_rotate_quant_rowwise": [_p, _int, _i64, _i64, _i64, _int, _int, _p, _p, _p],
    "ck_rotate_quant_rowwise_i8": [_p, _int, _i64, _i64, _i64, _int, _int, _p, _p, _p],
    "ck_rotate_quant_rowwise_r": [_p, _int, _i64, _i64, _i64, _int, _p, _int, _p, _p, _p],
    "ck_rotate_quant_rowwise_scaled": [_p, _int, _i64, _i64, _i64, _int, _int, _f32, _p, _p, _p],
    "ck_gemm_w4a4": [_p, _p, _i64, _i64, _i64, _p, _p, _p, _p, _p],
    "ck_gemm_w4a8": [_p, _p, _i64, _i64, _i64, _p, _p, _p, _p, _p],
    "ck_unpack_int4": [_p, _i64, _i64, _p, _p],
    "ck_gemm_s8": [_p, _p, _i64, _i64, _i64, _p, _p, _p, _p, _p],
    "ck_gemm_s8_i32": [_p, _p, _i64, _i64, _i64, _p, _p],
    "ck_linear_w4a4_workspace_bytes": [_i64, _i64],
    "ck_linear_w4a4": [_p, _int, _i64, _i64, _i64, _i64, _int, _p, _p, _p, _p, _p, ctypes.c_size_t, _p],
    "ck_linear_w4a4_quantize": [_p, _int, _i64, _i64, _i64, _int, _p, ctypes.c_size_t, _p],
    "ck_linear_w4a4_matmul": [_i64, _i64, _i64, _p, _p, _p, _p, _p, ctypes.c_size_t, _p],
    "ck_linear_w4a4_scaled": [_p, _int, _i64, _i64, _i64, _i64, _int, _f32, _p, _p, _p, _p, _p, ctypes.c_size_t,
                              _p],
    "ck_linear_w4a4_static": [_p, _int, _i64, _i64, _i64, _i64, _int, _p, _p, _p, _p, _p],
    "ck_linear_w4a8_workspace_bytes": [_i64, _i64],
    "ck_linear_w4a8": [_p, _int, _i64, _i64, _i64, _i64, _int, _p, _p, _p, _p, _p, ctypes.c_size_t, _p],
    "ck_linear_w4a4_predecoded": [_p, _int, _i64, _i64, _i64, _i64, _int, _p, _p, _p, _p, _p, ctypes.c_size_t,
                                  _p],
    "ck_gemv_w4a8": [_p, _p, _i64, _i64, _i64, _p, _p, _p, _p, _p],
    "ck_gemv_w4a8_tc": [_p, _p, _i64, _i64, _i64, _p, _p, _p, _p, _p],
    "ck_gemv_awq_w4a16": [_p, _int, _i64, _i64, _i64, _int, _p, _p, _p, _p, _p, _p],
    "ck_gemm_w4a4_i32": [_p, _p, _i64, _i64, _i64, _p, _p],
    "ck_gemm_w4a8_i32": [_p, _p, _i64, _i64, _i64, _p, _p],
    "ck_device_error_check": [_p],
    "ck_selftest_bounded_wait": [_i64, _p],
    "ck_last_error": [],
    "ck_version": [],
}
_RESTYPES = {"ck_linear_w4a4_workspace_bytes": ctypes.c_size_t, "ck_linear_w4a8_workspace_bytes": ctypes.c_size_t,
             "ck_last_error": ctypes.c_char_p, "ck_version": ctypes.c_char_p}

for _name, _args in SIGNATURES.items():
    _f = getattr(lib, _name)
    _f.argtypes = _args
    _f.restype = _RESTYPES.get(_name, ctypes.c_int)


class CKError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib.ck_last_error().decode()
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {msg}")


def _check(status: int, where: str) -> None:
    if status != CK_OK:
        raise CKError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None, device=None):
    """The stream handle for a call on `device`: the given stream (which must belong to that
    device) or that device's current stream."""
    if stream is None:
        stream = torch.cuda.current_stream(device)
    elif device is not None and stream.device != device:
        raise ValueError(f"stream is on {stream.device}, the tensors on {device}")
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(dt) -> int:
    if dt == torch.bfloat16:
        return CK_BF16
    if dt == torch.float16:
        return CK_FP16
    raise TypeError(f"unsupported dtype {dt} (bf16 or fp16)")


_BYTES = (torch.uint8, torch.int8)      # codes and packed nibbles: either view of the same bytes
_HALF = (torch.bfloat16, torch.float16)
_F32 = (torch.float32,)
_BF16 = (torch.bfloat16,)
_I32 = (torch.int32,)


def _types(where: str, **named) -> None:
    """TypeError unless each named tensor (None is skipped) has one of its allowed dtypes.

    The C entry points see raw bytes, so a tensor of the wrong dtype would be
    read as garbage rather than rejected."""
    for name, (t, allowed) in named.items():
        if t is not None and t.dtype not in allowed:
            want = " or ".join(str(a).replace("torch.", "") for a in allowed)
            raise TypeError(f"{where}: {name} must be {want}, got {str(t.dtype).replace('torch.', '')}")


def _cuda(*ts):
    """The one CUDA device all given tensors (None is skipped) live on; ValueError otherwise.

    The library launches on the calling thread's current device, so every call below runs with
    this device made current (``torch.cuda.device``)."""
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"all tensors must be on one device ({dev} and {t.device} given)")
    return dev


def _rows(x):
    """(M, K, ldx) of a tensor whose last dim is contiguous; leading dims are flattened."""
    if x.stride(-1) != 1:
        raise ValueError("the last dimension must be contiguous")
    K = x.shape[-1]
    if x.dim() == 1:
        return 1, K, K, x
    x2 = x if x.dim() == 2 else x.reshape(-1, K)
    return x2.shape[0], K, x2.stride(0), x2


def version() -> str:
    return lib.ck_version().decode()


def last_error() -> str:
    return lib.ck_last_error().decode()


def _call(dev, name: str, *args, stream=None) -> None:
    """Calls the C entry point `name` with `dev` current and that device's stream appended."""
    with torch.cuda.device(dev):
        _check(getattr(lib, name)(*args, _stream(stream, dev)), name)


def _nbytes(t) -> int:
    return t.numel() * t.element_size()


def _codes_out(x, K, bits, q_out, scale_out):
    lead = tuple(x.shape[:-1])
    if q_out is None:
        q_out = torch.empty(lead + ((K // 2,) if bits == 4 else (K,)), device=x.device,
                            dtype=torch.uint8 if bits == 4 else torch.int8)
    if scale_out is None:
        scale_out = torch.empty(lead, device=x.device, dtype=torch.float32)
    return q_out, scale_out


def rotate_quant_rowwise(x, group_size: int, bits: int, q_out=None, scale_out=None, stream=None):
    """Returns (q, scale): q packed int4 (..., K/2) uint8 for bits=4, int8 (..., K) for bits=8."""
    _types("rotate_quant_rowwise", x=(x, _HALF), q_out=(q_out, _BYTES), scale_out=(scale_out, _F32))
    _cuda(x)
    M, K, ldx, x2 = _rows(x)
    q_out, scale_out = _codes_out(x, K, bits, q_out, scale_out)
    dev = _cuda(x, q_out, scale_out)
    _call(dev, "ck_rotate_quant_rowwise", _ptr(x2), _dtype_code(x.dtype), M, K, ldx, group_size, bits,
          _ptr(q_out), _ptr(scale_out), stream=stream)
    return q_out, scale_out


def rotate_quant_rowwise_i8(x, group_size: int, bits: int, q_out=None, scale_out=None, stream=None):
    """Returns (q, scale) with the codes stored one per byte: q (..., K) int8 for bits 4 or 8."""
    _types("rotate_quant_rowwise_i8", x=(x, _HALF), q_out=(q_out, _BYTES), scale_out=(scale_out, _F32))
    _cuda(x)
    M, K, ldx, x2 = _rows(x)
    q_out, scale_out = _codes_out(x, K, 8, q_out, scale_out)
    dev = _cuda(x, q_out, scale_out)
    _call(dev, "ck_rotate_quant_rowwise_i8", _ptr(x2), _dtype_code(x.dtype), M, K, ldx, group_size, bits,
          _ptr(q_out), _ptr(scale_out), stream=stream)
    return q_out, scale_out


def rotate_quant_rowwise_r(x, R, bits: int, q_out=None, scale_out=None, stream=None):
    """Rotation by a general (G, G) float32 matrix R (y_g = x_g @ R), then rowwise quantization.

    Returns (q, s) in the formats of rotate_quant_rowwise: bits=4 packed (..., K/2) uint8, bits=8
    (..., K) int8; s (...) float32.
    """
    _types("rotate_quant_rowwise_r", x=(x, _HALF), q_out=(q_out, _BYTES), scale_out=(scale_out, _F32))
    _cuda(x, R)
    if R.dtype != torch.float32 or R.dim() != 2 or R.shape[0] != R.shape[1] or not R.is_contiguous():
        raise ValueError("R must be a contiguous square float32 matrix")
    M, K, ldx, x2 = _rows(x)
    q_out, scale_out = _codes_out(x, K, bits, q_out, scale_out)
    dev = _cuda(x, R, q_out, scale_out)
    _call(dev, "ck_rotate_quant_rowwise_r", _ptr(x2), _dtype_code(x.dtype), M, K, ldx, R.shape[0], _ptr(R), bits,
          _ptr(q_out), _ptr(scale_out), stream=stream)
    return q_out, scale_out


def rotate_quant_rowwise_scaled(x, group_size: int, bits: int, input_scale: float, q_out=None,
                                scale_out=None, stream=None):
    """rotate_quant_rowwise of input_scale * x (a finite tensor-wise scale >= 0); same formats."""
    _types("rotate_quant_rowwise_scaled", x=(x, _HALF), q_out=(q_out, _BYTES), scale_out=(scale_out, _F32))
    _cuda(x)
    M, K, ldx, x2 = _rows(x)
    q_out, scale_out = _codes_out(x, K, bits, q_out, scale_out)
    dev = _cuda(x, q_out, scale_out)
    _call(dev, "ck_rotate_quant_rowwise_scaled", _ptr(x2), _dtype_code(x.dtype), M, K, ldx, group_size, bits,
          float(input_scale), _ptr(q_out), _ptr(scale_out), stream=stream)
    return q_out, scale_out


def unpack_int4(packed, out=None, stream=None):
    """(R, C/2) packed int4 -> (R, C) int8 with value u - 8."""
    _types("unpack_int4", packed=(packed, _BYTES), out=(out, _BYTES))
    _cuda(packed)
    R, Ch = packed.shape
    if out is None:
        out = torch.empty((R, 2 * Ch), device=packed.device, dtype=torch.int8)
    dev = _cuda(packed, out)
    _call(dev, "ck_unpack_int4", _ptr(packed), R, 2 * Ch, _ptr(out), stream=stream)
    return out


def _mn_out(a, M, N, out, dtype=torch.bfloat16):
    return torch.empty((M, N), device=a.device, dtype=dtype) if out is None else out


def gemm_w4a8(qa, a_scale, w_packed, w_scale, bias=None, out=None, stream=None):
    """int8 activation codes (M, K) x packed int4 weights (N, K/2) -> bf16 (M, N)."""
    _types("gemm_w4a8", qa=(qa, _BYTES), a_scale=(a_scale, _F32), w_packed=(w_packed, _BYTES),
           w_scale=(w_scale, _BF16), bias=(bias, _BF16), out=(out, _BF16))
    _cuda(qa, a_scale, w_packed, w_scale, bias, out)
    M, K = qa.shape
    N = w_packed.shape[0]
    out = _mn_out(qa, M, N, out)
    _call(_cuda(qa, out), "ck_gemm_w4a8", _ptr(qa), _ptr(a_scale), M, K, N, _ptr(w_packed), _ptr(w_scale),
          _ptr(bias), _ptr(out), stream=stream)
    return out


def gemm_s8(qa, a_scale, w8, w_scale, bias=None, out=None, stream=None):
    _types("gemm_s8", qa=(qa, _BYTES), a_scale=(a_scale, _F32), w8=(w8, _BYTES), w_scale=(w_scale, _BF16),
           bias=(bias, _BF16), out=(out, _BF16))
    _cuda(qa, a_scale, w8, w_scale, bias, out)
    M, K = qa.shape
    N = w8.shape[0]
    out = _mn_out(qa, M, N, out)
    _call(_cuda(qa, out), "ck_gemm_s8", _ptr(qa), _ptr(a_scale), M, K, N, _ptr(w8), _ptr(w_scale), _ptr(bias),
          _ptr(out), stream=stream)
    return out


def gemm_s8_i32(qa, w8, out=None, stream=None):
    _types("gemm_s8_i32", qa=(qa, _BYTES), w8=(w8, _BYTES), out=(out, _I32))
    _cuda(qa, w8, out)
    M, K = qa.shape
    N = w8.shape[0]
    out = _mn_out(qa, M, N, out, torch.int32)
    _call(_cuda(qa, out), "ck_gemm_s8_i32", _ptr(qa), _ptr(w8), M, K, N, _ptr(out), stream=stream)
    return out


def gemm_w4a4(qa_packed, a_scale, w_packed, w_scale, bias=None, out=None, stream=None):
    _types("gemm_w4a4", qa_packed=(qa_packed, _BYTES), a_scale=(a_scale, _F32), w_packed=(w_packed, _BYTES),
           w_scale=(w_scale, _BF16), bias=(bias, _BF16), out=(out, _BF16))
    _cuda(qa_packed, a_scale, w_packed, w_scale, bias, out)
    M, Kh = qa_packed.shape
    N = w_packed.shape[0]
    out = _mn_out(qa_packed, M, N, out)
    _call(_cuda(qa_packed, out), "ck_gemm_w4a4", _ptr(qa_packed), _ptr(a_scale), M, 2 * Kh, N, _ptr(w_packed),
          _ptr(w_scale), _ptr(bias), _ptr(out), stream=stream)
    return out


def linear_w4a4_workspace_bytes(M: int, K: int) -> int:
    return int(lib.ck_linear_w4a4_workspace_bytes(M, K))


def linear_w4a8_workspace_bytes(M: int, K: int) -> int:
    return int(lib.ck_linear_w4a8_workspace_bytes(M, K))


def _linear(name, x, w, w_scale, group_size, bias, workspace, out, stream, ws_fn, *extra, w_name="w_packed"):
    """Shared marshalling of the one-shot linears: (x, weights, scales) -> y (..., N) bf16."""
    _types(name, x=(x, _HALF), **{w_name: (w, _BYTES)}, w_scale=(w_scale, _BF16), bias=(bias, _BF16),
           out=(out, _BF16), workspace=(workspace, _BYTES))
    _cuda(x, w, w_scale, bias, workspace, out)
    M, K, ldx, x2 = _rows(x)
    N = w.shape[0]
    if workspace is None:
        workspace = torch.empty(ws_fn(M, K), device=x.device, dtype=torch.uint8)
    if out is None:
        out = torch.empty(tuple(x.shape[:-1]) + (N,), device=x.device, dtype=torch.bfloat16)
    dev = _cuda(x, workspace, out)
    _call(dev, "ck_" + name, _ptr(x2), _dtype_code(x.dtype), M, K, N, ldx, group_size, *extra, _ptr(w),
          _ptr(w_scale), _ptr(bias), _ptr(out), _ptr(workspace), _nbytes(workspace), stream=stream)
    return out


def linear_w4a4(x, w_packed, w_scale, group_size: int, bias=None, workspace=None, out=None,
                stream=None):
    """ConvRot W4A4 linear: y (..., N) bf16 from x (..., K) bf16/fp16 and packed (N, K/2) weights."""
    return _linear("linear_w4a4", x, w_packed, w_scale, group_size, bias, workspace, out, stream,
                   linear_w4a4_workspace_bytes)


def linear_w4a8(x, w_packed, w_scale, group_size: int, bias=None, workspace=None, out=None,
                stream=None):
    """ConvRot W4A8 linear: x rotated and quantized to int8 codes, times packed (N, K/2) int4 weights."""
    return _linear("linear_w4a8", x, w_packed, w_scale, group_size, bias, workspace, out, stream,
                   linear_w4a8_workspace_bytes)


def linear_w4a4_predecoded(x, w_s8, w_scale, group_size: int, bias=None, workspace=None, out=None,
                           stream=None):
    """linear_w4a4 with the weights already unpacked to int8 (N, K) by unpack_int4 (same results)."""
    return _linear("linear_w4a4_predecoded", x, w_s8, w_scale, group_size, bias, workspace, out, stream,
                   linear_w4a4_workspace_bytes, w_name="w_s8")


def linear_w4a4_scaled(x, w_packed, w_scale, group_size: int, input_scale: float, bias=None, workspace=None,
                       out=None, stream=None):
    """linear_w4a4 of input_scale * x (a finite tensor-wise scale >= 0); the output is not rescaled."""
    return _linear("linear_w4a4_scaled", x, w_packed, w_scale, group_size, bias, workspace, out, stream,
                   linear_w4a4_workspace_bytes, ctypes.c_float(float(input_scale)))


# Size of the library's built-in scratch for linear_w4a4_static (CK_LINEAR_STATIC_SCRATCH_BYTES).
LINEAR_STATIC_SCRATCH_BYTES = 32 * 1024 * 1024


def linear_w4a4_static(x, w_packed, w_scale, group_size: int, bias=None, out=None, stream=None):
    """linear_w4a4 without a workspace argument: the library uses its own fixed per-device scratch.

    Same results as linear_w4a4. Calls on one device share that scratch, so calls that may run
    at the same time on the GPU (different streams, several threads) must not be mixed. The call
    runs with x's device current: the scratch it uses is that device's.
    """
    _types("linear_w4a4_static", x=(x, _HALF), w_packed=(w_packed, _BYTES), w_scale=(w_scale, _BF16),
           bias=(bias, _BF16), out=(out, _BF16))
    _cuda(x, w_packed, w_scale, bias, out)
    M, K, ldx, x2 = _rows(x)
    N = w_packed.shape[0]
    if out is None:
        out = torch.empty(tuple(x.shape[:-1]) + (N,), device=x.device, dtype=torch.bfloat16)
    _call(_cuda(x, out), "ck_linear_w4a4_static", _ptr(x2), _dtype_code(x.dtype), M, K, N, ldx, group_size,
          _ptr(w_packed), _ptr(w_scale), _ptr(bias), _ptr(out), stream=stream)
    return out


def linear_w4a4_quantize(x, group_size: int, workspace, stream=None):
    """Phase 1 of linear_w4a4: rotate + quantize x into `workspace` (opaque)."""
    _types("linear_w4a4_quantize", x=(x, _HALF), workspace=(workspace, _BYTES))
    dev = _cuda(x, workspace)
    M, K, ldx, x2 = _rows(x)
    _call(dev, "ck_linear_w4a4_quantize", _ptr(x2), _dtype_code(x.dtype), M, K, ldx, group_size, _ptr(workspace),
          _nbytes(workspace), stream=stream)
    return workspace


def linear_w4a4_matmul(M: int, K: int, w_packed, w_scale, workspace, bias=None, out=None, stream=None):
    """Phase 2 of linear_w4a4: GEMM of the workspace codes with the packed weights -> y (M, N) bf16."""
    _types("linear_w4a4_matmul", w_packed=(w_packed, _BYTES), w_scale=(w_scale, _BF16), bias=(bias, _BF16),
           out=(out, _BF16), workspace=(workspace, _BYTES))
    _cuda(w_packed, w_scale, workspace, bias, out)
    N = w_packed.shape[0]
    out = _mn_out(w_packed, M, N, out)
    _call(_cuda(w_packed, workspace, out), "ck_linear_w4a4_matmul", M, K, N, _ptr(w_packed), _ptr(w_scale),
          _ptr(bias), _ptr(out), _ptr(workspace), _nbytes(workspace), stream=stream)
    return out


def _gemv_w4a8(name, xq, x_scale, w_packed, w_scale, bias, out, stream):
    _types(name, xq=(xq, _BYTES), x_scale=(x_scale, _F32), w_packed=(w_packed, _BYTES),
           w_scale=(w_scale, _BF16), bias=(bias, _BF16), out=(out, _BF16))
    _cuda(xq, x_scale, w_packed, w_scale, bias, out)
    M, K = xq.shape
    N = w_packed.shape[0]
    out = _mn_out(xq, M, N, out)
    _call(_cuda(xq, out), "ck_" + name, _ptr(xq), _ptr(x_scale), M, K, N, _ptr(w_packed), _ptr(w_scale),
          _ptr(bias), _ptr(out), stream=stream)
    return out


def gemv_w4a8(xq, x_scale, w_packed, w_scale, bias=None, out=None, stream=None):
    return _gemv_w4a8("gemv_w4a8", xq, x_scale, w_packed, w_scale, bias, out, stream)


def gemv_w4a8_tc(xq, x_scale, w_packed, w_scale, bias=None, out=None, stream=None):
    """gemv_w4a8 on the tcgen05 tensor cores (the same results bit for bit; an alternative path)."""
    return _gemv_w4a8("gemv_w4a8_tc", xq, x_scale, w_packed, w_scale, bias, out, stream)


def gemv_awq_w4a16(x, qweight, wscales, wzeros, bias=None, group_size: int = 64, out=None, stream=None):
    """``ck.gemv_awq_w4a16(x, qdata, wscales, wzeros, bias=, group_size=)``."""
    same = (x.dtype,) if x.dtype in _HALF else _HALF
    _types("gemv_awq_w4a16", x=(x, _HALF), qweight=(qweight, _BYTES), wscales=(wscales, same),
           wzeros=(wzeros, same), bias=(bias, same), out=(out, same))
    _cuda(x, qweight, wscales, wzeros, bias, out)
    M, K = x.shape
    N = qweight.shape[0]
    out = _mn_out(x, M, N, out, x.dtype)
    _call(_cuda(x, out), "ck_gemv_awq_w4a16", _ptr(x), _dtype_code(x.dtype), M, K, N, group_size, _ptr(qweight),
          _ptr(wscales), _ptr(wzeros), _ptr(bias), _ptr(out), stream=stream)
    return out


def gemm_w4a4_i32(qa_packed, w_packed, out=None, stream=None):
    _types("gemm_w4a4_i32", qa_packed=(qa_packed, _BYTES), w_packed=(w_packed, _BYTES), out=(out, _I32))
    _cuda(qa_packed, w_packed, out)
    M, Kh = qa_packed.shape
    N = w_packed.shape[0]
    out = _mn_out(qa_packed, M, N, out, torch.int32)
    _call(_cuda(qa_packed, out), "ck_gemm_w4a4_i32", _ptr(qa_packed), _ptr(w_packed), M, 2 * Kh, N, _ptr(out),
          stream=stream)
    return out


def gemm_w4a8_i32(qa, w_packed, out=None, stream=None):
    _types("gemm_w4a8_i32", qa=(qa, _BYTES), w_packed=(w_packed, _BYTES), out=(out, _I32))
    _cuda(qa, w_packed, out)
    M, K = qa.shape
    N = w_packed.shape[0]
    out = _mn_out(qa, M, N, out, torch.int32)
    _call(_cuda(qa, out), "ck_gemm_w4a8_i32", _ptr(qa), _ptr(w_packed), M, K, N, _ptr(out), stream=stream)
    return out


def device_error_check(stream=None) -> None:
    """Synchronises the stream and raises CKError(CK_ERR_TIMEOUT) if a bounded wait gave up."""
    _check(lib.ck_device_error_check(_stream(stream)), "ck_device_error_check")


def selftest_bounded_wait(timeout_ns: int, stream=None) -> None:
    _check(lib.ck_selftest_bounded_wait(int(timeout_ns), _stream(stream)), "ck_selftest_bounded_wait")
