"""ConvRot packed-INT4 quantized linear for NVIDIA B200 (sm_100a).

The compute lives in libck.so (C ABI: include/ck.h); ``ck`` is its thin
Python binding. Accessing any op below loads the library and raises
ImportError if it has not been built (there is no CPU fallback).
``workloads`` (seeded synthetic inputs) needs no GPU and no library.
"""

_OPS = ("rotate_quant_rowwise", "gemm_w4a4", "linear_w4a4", "linear_w4a4_workspace_bytes",
        "gemv_w4a8", "gemv_awq_w4a16", "gemm_w4a4_i32", "gemm_w4a8_i32", "device_error_check",
        "selftest_bounded_wait", "CKError", "version", "rotate_quant_rowwise_i8", "unpack_int4",
        "gemm_s8", "gemm_s8_i32", "gemm_w4a8", "linear_w4a4_quantize", "linear_w4a4_matmul")

__all__ = list(_OPS) + ["ck", "workloads"]


def __getattr__(name):
    import importlib
    if name in _OPS or name == "ck":
        mod = importlib.import_module(__name__ + ".ck")
        return mod if name == "ck" else getattr(mod, name)
    if name == "workloads":
        return importlib.import_module(__name__ + ".workloads")
    raise AttributeError(name)
