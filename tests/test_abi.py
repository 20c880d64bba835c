"""The C-ABI library loads, exports every symbol include/ck.h declares, and
rejects invalid arguments on the host before anything reaches the GPU."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def ck():
    from bit_quantized_linear_rotate_b200 import build
    build.build()
    from bit_quantized_linear_rotate_b200 import ck as _ck
    return _ck


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "ck.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ck_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ("ck_rotate_quant_rowwise", "ck_linear_w4a4", "ck_gemv_w4a8", "ck_gemv_awq_w4a16",
                 "ck_rotate_quant_rowwise_i8", "ck_gemm_w4a8", "ck_unpack_int4", "ck_gemm_s8",
                 "ck_gemm_w4a4", "ck_gemm_w4a4_i32", "ck_gemm_w4a8_i32", "ck_last_error"):
        assert name in syms


def test_library_exports_every_declared_symbol(ck):
    for name in declared_symbols():
        assert hasattr(ck.lib, name), name
        assert name in ck.SIGNATURES, f"binding lacks {name}"


def test_header_is_plain_c_and_links_from_c(ck, tmp_path):
    # the boundary is a C ABI: ck.h compiles as strict C99 and a C program links
    # against libck.so and calls it (M = 0 is a no-op that needs no GPU)
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_ck.c"
    src.write_text('#include "ck.h"\n#include <stdio.h>\n'
                   "int main(void) {\n"
                   '  printf("%s\\n", ck_version());\n'
                   "  return ck_rotate_quant_rowwise(0, CK_BF16, 0, 64, 64, 64, 4, 0, 0, 0) == CK_OK ? 0 : 1;\n"
                   "}\n")
    libdir = os.path.dirname(ck.LIB_PATH)
    exe = tmp_path / "use_ck"
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-L", libdir, "-l:libck.so", f"-Wl,-rpath,{libdir}", "-o", str(exe)],
                   check=True, capture_output=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0
    assert "sm_100a" in out.stdout


def test_version_and_last_error(ck):
    assert "sm_100a" in ck.version()
    assert isinstance(ck.last_error(), str)


def test_workspace_bytes(ck):
    # int8 activation codes, float32 scales, int32 row sums (each rounded up to 256 bytes)
    assert ck.linear_w4a4_workspace_bytes(8192, 3840) == 8192 * 3840 + 8192 * 4 + 8192 * 4
    assert ck.linear_w4a4_workspace_bytes(3, 64) == 256 + 256 + 12
    assert ck.linear_w4a4_workspace_bytes(0, 64) == 0
    # small batches (M <= 64, K % 128 == 0, K <= 4096): the codes packed two per byte, then
    # room for them one per byte
    assert ck.linear_w4a4_workspace_bytes(32, 3840) == 32 * 1920 + 32 * 3840 + 256 + 32 * 4
    assert ck.linear_w4a4_workspace_bytes(3, 128) == 256 + 512 + 256 + 12
    assert ck.linear_w4a8_workspace_bytes(32, 3840) == ck.linear_w4a4_workspace_bytes(32, 3840)


def _rq(ck, **kw):
    a = dict(x=1 << 20, xt=0, M=4, K=64, ldx=64, G=64, bits=4, q=1 << 21, s=1 << 22)
    a.update(kw)
    p = lambda v: ctypes.c_void_p(v) if v is not None else None
    return ck.lib.ck_rotate_quant_rowwise(p(a["x"]), a["xt"], a["M"], a["K"], a["ldx"], a["G"], a["bits"],
                                          p(a["q"]), p(a["s"]), None)


def test_rotate_quant_validation(ck):
    assert _rq(ck, bits=3) == ck.CK_ERR_INVALID_ARG
    assert "bits" in ck.last_error()                         # the message names the bad argument
    assert _rq(ck, G=48) == ck.CK_ERR_UNSUPPORTED
    assert _rq(ck, G=512, K=512, ldx=512) == ck.CK_ERR_UNSUPPORTED
    assert _rq(ck, K=96) == ck.CK_ERR_INVALID_ARG            # K % G != 0
    assert _rq(ck, ldx=32) == ck.CK_ERR_INVALID_ARG          # ldx < K
    assert _rq(ck, x=None) == ck.CK_ERR_INVALID_ARG
    assert _rq(ck, x=(1 << 20) + 2) == ck.CK_ERR_INVALID_ARG  # misaligned rows
    assert _rq(ck, ldx=68) == ck.CK_ERR_INVALID_ARG          # row stride not 16-byte aligned
    assert _rq(ck, xt=7) == ck.CK_ERR_INVALID_ARG
    assert _rq(ck, M=-1) == ck.CK_ERR_INVALID_ARG
    assert _rq(ck, M=0, x=None, q=None, s=None) == ck.CK_OK  # empty input: no-op
    assert ck.last_error() == ""                             # a successful call clears the message


def test_gemm_and_linear_validation(ck):
    P = lambda v: ctypes.c_void_p(v)
    L = ck.lib
    assert L.ck_gemm_w4a4(P(1 << 20), P(1 << 20), 8, 48, 8, P(1 << 20), P(1 << 20), None, P(1 << 20), None) == ck.CK_ERR_UNSUPPORTED
    assert L.ck_gemm_w4a4(None, P(1 << 20), 8, 64, 8, P(1 << 20), P(1 << 20), None, P(1 << 20), None) == ck.CK_ERR_INVALID_ARG
    assert L.ck_gemm_w4a4(P(1 << 20), P(1 << 20), 0, 64, 8, P(1 << 20), P(1 << 20), None, P(1 << 20), None) == ck.CK_ERR_INVALID_ARG
    assert L.ck_gemm_w4a4(P((1 << 20) + 8), P(1 << 20), 8, 64, 8, P(1 << 20), P(1 << 20), None, P(1 << 20), None) == ck.CK_ERR_UNSUPPORTED
    assert L.ck_gemm_w4a4_i32(P(1 << 20), P(1 << 20), 8, 64, -1, P(1 << 20), None) == ck.CK_ERR_INVALID_ARG
    assert L.ck_gemm_w4a8_i32(P(1 << 20), None, 8, 64, 8, P(1 << 20), None) == ck.CK_ERR_INVALID_ARG
    # workspace too small / misaligned
    assert L.ck_linear_w4a4(P(1 << 20), 0, 8, 64, 8, 64, 64, P(1 << 20), P(1 << 20), None, P(1 << 20),
                            P(1 << 20), 16, None) == ck.CK_ERR_INVALID_ARG
    assert L.ck_linear_w4a4(P(1 << 20), 0, 8, 64, 8, 64, 64, P(1 << 20), P(1 << 20), None, P(1 << 20),
                            P((1 << 20) + 16), 1 << 20, None) == ck.CK_ERR_INVALID_ARG


def test_linear_phase_validation(ck):
    P = lambda v: ctypes.c_void_p(v)
    L = ck.lib
    ws = ck.linear_w4a4_workspace_bytes(8, 64)
    assert L.ck_linear_w4a4_quantize(P(1 << 20), 0, 8, 64, 64, 64, P(1 << 21), ws - 1, None) == ck.CK_ERR_INVALID_ARG
    assert L.ck_linear_w4a4_quantize(P(1 << 20), 0, 8, 64, 64, 48, P(1 << 21), ws, None) == ck.CK_ERR_UNSUPPORTED
    assert L.ck_linear_w4a4_quantize(P(1 << 20), 0, 8, 48, 48, 16, P(1 << 21), ws, None) == ck.CK_ERR_UNSUPPORTED
    assert L.ck_linear_w4a4_matmul(8, 64, 8, None, P(1 << 20), None, P(1 << 20), P(1 << 21), ws, None) == ck.CK_ERR_INVALID_ARG
    assert L.ck_linear_w4a4_matmul(8, 64, 8, P(1 << 20), P(1 << 20), None, P(1 << 20), P((1 << 21) + 128), ws, None) == ck.CK_ERR_INVALID_ARG


def test_predecoded_path_validation(ck):
    P = lambda v: ctypes.c_void_p(v)
    L = ck.lib
    assert L.ck_unpack_int4(P(1 << 20), 3, 6, P(1 << 21), None) == ck.CK_ERR_UNSUPPORTED   # 9 bytes
    assert L.ck_unpack_int4(P(1 << 20), 4, 7, P(1 << 21), None) == ck.CK_ERR_UNSUPPORTED   # odd C
    assert L.ck_unpack_int4(None, 4, 8, P(1 << 21), None) == ck.CK_ERR_INVALID_ARG
    assert L.ck_unpack_int4(P((1 << 20) + 4), 4, 8, P(1 << 21), None) == ck.CK_ERR_INVALID_ARG
    assert L.ck_gemm_s8(P(1 << 20), P(1 << 20), 8, 40, 8, P(1 << 20), P(1 << 20), None, P(1 << 20), None) == ck.CK_ERR_UNSUPPORTED
    assert L.ck_gemm_w4a8(P(1 << 20), None, 8, 64, 8, P(1 << 20), P(1 << 20), None, P(1 << 20), None) == ck.CK_ERR_INVALID_ARG
    assert L.ck_gemm_s8_i32(P(1 << 20), P(1 << 20), 8, 64, 0, P(1 << 20), None) == ck.CK_ERR_INVALID_ARG
    assert L.ck_rotate_quant_rowwise_i8(P(1 << 20), 0, 4, 64, 64, 64, 5, P(1 << 21), P(1 << 22), None) == ck.CK_ERR_INVALID_ARG
    assert L.ck_rotate_quant_rowwise_i8(P(1 << 20), 0, 4, 64, 64, 3, 4, P(1 << 21), P(1 << 22), None) == ck.CK_ERR_UNSUPPORTED


def test_gemv_validation(ck):
    P = lambda v: ctypes.c_void_p(v)
    L = ck.lib
    assert L.ck_gemv_w4a8(P(1 << 20), P(1 << 20), 17, 128, 8, P(1 << 20), P(1 << 20), None, P(1 << 20), None) == ck.CK_ERR_UNSUPPORTED
    assert L.ck_gemv_w4a8(P(1 << 20), P(1 << 20), 4, 96, 8, P(1 << 20), P(1 << 20), None, P(1 << 20), None) == ck.CK_ERR_UNSUPPORTED
    assert L.ck_gemv_w4a8(P(1 << 20), None, 4, 128, 8, P(1 << 20), P(1 << 20), None, P(1 << 20), None) == ck.CK_ERR_INVALID_ARG
    assert L.ck_gemv_awq_w4a16(P(1 << 20), 0, 9, 128, 8, 64, P(1 << 20), P(1 << 20), P(1 << 20), None, P(1 << 20), None) == ck.CK_ERR_UNSUPPORTED
    assert L.ck_gemv_awq_w4a16(P(1 << 20), 0, 2, 128, 8, 32, P(1 << 20), P(1 << 20), P(1 << 20), None, P(1 << 20), None) == ck.CK_ERR_UNSUPPORTED
    assert L.ck_gemv_awq_w4a16(P(1 << 20), 0, 2, 192, 8, 128, P(1 << 20), P(1 << 20), P(1 << 20), None, P(1 << 20), None) == ck.CK_ERR_INVALID_ARG
    assert L.ck_gemv_awq_w4a16(P(1 << 20), 5, 2, 128, 8, 64, P(1 << 20), P(1 << 20), P(1 << 20), None, P(1 << 20), None) == ck.CK_ERR_INVALID_ARG


def test_tensor_core_gemv_validation(ck):
    P = lambda v: ctypes.c_void_p(v)
    L = ck.lib
    call = lambda M, K, N, xq=P(1 << 20): L.ck_gemv_w4a8_tc(xq, P(1 << 20), M, K, N, P(1 << 20), P(1 << 20), None,
                                                               P(1 << 20), None)
    assert call(17, 128, 8) == ck.CK_ERR_UNSUPPORTED        # M > 16
    assert call(4, 96, 8) == ck.CK_ERR_UNSUPPORTED          # K % 128
    assert call(4, 8320, 8) == ck.CK_ERR_UNSUPPORTED        # K > 8192
    assert call(0, 128, 8) == ck.CK_ERR_INVALID_ARG
    assert call(4, 128, 8, xq=None) == ck.CK_ERR_INVALID_ARG
    assert call(4, 128, 8, xq=P((1 << 20) + 8)) == ck.CK_ERR_UNSUPPORTED


def test_general_rotation_validation(ck):
    P = lambda v: ctypes.c_void_p(v)
    L = ck.lib
    ok = dict(x=P(1 << 20), xt=0, M=4, K=64, ldx=64, G=16, R=P(1 << 22), bits=4, q=P(1 << 21), s=P(1 << 23))
    def call(**kw):
        a = dict(ok); a.update(kw)
        return L.ck_rotate_quant_rowwise_r(a["x"], a["xt"], a["M"], a["K"], a["ldx"], a["G"], a["R"], a["bits"],
                                           a["q"], a["s"], None)
    assert call(G=0) == ck.CK_ERR_UNSUPPORTED
    assert call(G=512, K=512, ldx=512) == ck.CK_ERR_UNSUPPORTED
    assert call(G=48) == ck.CK_ERR_INVALID_ARG          # K % G != 0
    assert call(bits=2) == ck.CK_ERR_INVALID_ARG
    assert call(R=None) == ck.CK_ERR_INVALID_ARG
    assert call(K=63, ldx=64, G=1) == ck.CK_ERR_INVALID_ARG   # K odd
    assert call(M=0, x=None, R=None, q=None, s=None) == ck.CK_OK


@pytest.mark.parametrize("a", [float("nan"), float("inf"), -1.0, -1e-30])
def test_input_scale_must_be_finite_and_nonnegative(ck, a):
    P = lambda v: ctypes.c_void_p(v)
    L = ck.lib
    assert L.ck_rotate_quant_rowwise_scaled(P(1 << 20), 0, 4, 64, 64, 64, 4, a, P(1 << 21), P(1 << 22),
                                            None) == ck.CK_ERR_INVALID_ARG
    assert "input_scale" in ck.last_error()
    ws = ck.linear_w4a4_workspace_bytes(8, 64)
    assert L.ck_linear_w4a4_scaled(P(1 << 20), 0, 8, 64, 8, 64, 64, a, P(1 << 20), P(1 << 20), None,
                                   P(1 << 20), P(1 << 21), ws, None) == ck.CK_ERR_INVALID_ARG


def test_input_scale_other_checks(ck):
    P = lambda v: ctypes.c_void_p(v)
    L = ck.lib
    def rq(**kw):
        a = dict(x=P(1 << 20), M=4, K=64, G=64, bits=4, a=0.5)
        a.update(kw)
        return L.ck_rotate_quant_rowwise_scaled(a["x"], 0, a["M"], a["K"], a["K"], a["G"], a["bits"], a["a"],
                                                P(1 << 21), P(1 << 22), None)
    assert rq(G=1, a=2.0) == ck.CK_ERR_UNSUPPORTED        # no rotation: only a = 1
    assert rq(G=1, a=1.0, M=0) == ck.CK_OK
    assert rq(M=0, a=0.0) == ck.CK_OK                     # empty input: no-op
    assert rq(G=48) == ck.CK_ERR_UNSUPPORTED
    assert rq(bits=5) == ck.CK_ERR_INVALID_ARG
    assert rq(x=None) == ck.CK_ERR_INVALID_ARG
    assert rq(x=P((1 << 20) + 2)) == ck.CK_ERR_INVALID_ARG
    ws = ck.linear_w4a4_workspace_bytes(8, 64)
    lin = lambda G, a, ws_bytes=ws: L.ck_linear_w4a4_scaled(P(1 << 20), 0, 8, 64, 8, 64, G, a, P(1 << 20),
                                                            P(1 << 20), None, P(1 << 20), P(1 << 21), ws_bytes,
                                                            None)
    assert lin(1, 3.0) == ck.CK_ERR_UNSUPPORTED
    assert lin(48, 1.0) == ck.CK_ERR_UNSUPPORTED
    assert lin(64, 1.0, ws - 1) == ck.CK_ERR_INVALID_ARG


def test_k_that_could_overflow_the_int32_accumulator_is_rejected(ck):
    # |sum_k a w| <= K * max|a w|: int8 x int8 128 * 128, int8 x int4 128 * 8,
    # int4 x int4 8 * 8, int8 x unsigned nibble (GEMV) 128 * 15
    P = lambda v: ctypes.c_void_p(v)
    L = ck.lib
    g = (P(1 << 20), P(1 << 20), 8)
    tail = (P(1 << 20), P(1 << 20), None, P(1 << 20), None)
    assert L.ck_gemm_s8(*g[:2], 8, 131072, 8, *tail) == ck.CK_ERR_UNSUPPORTED
    assert "overflow" in ck.last_error()
    assert L.ck_gemm_s8_i32(P(1 << 20), P(1 << 20), 8, 131072, 8, P(1 << 20), None) == ck.CK_ERR_UNSUPPORTED
    assert L.ck_gemm_w4a8(*g[:2], 8, 2097152, 8, *tail) == ck.CK_ERR_UNSUPPORTED
    assert L.ck_gemm_w4a4(*g[:2], 8, 33554432, 8, *tail) == ck.CK_ERR_UNSUPPORTED
    assert L.ck_gemv_w4a8(P(1 << 20), P(1 << 20), 4, 1118592, 8, P(1 << 20), P(1 << 20), None, P(1 << 20),
                          None) == ck.CK_ERR_UNSUPPORTED
    assert "overflow" in ck.last_error()


def test_selftest_timeout_range_is_validated(ck):
    assert ck.lib.ck_selftest_bounded_wait(10, None) == ck.CK_ERR_INVALID_ARG
    assert ck.lib.ck_selftest_bounded_wait(10 ** 10, None) == ck.CK_ERR_INVALID_ARG


def test_package_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "bit_quantized_linear_rotate_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in src and "from oracle" not in src, f


def test_binding_rejects_wrong_dtypes_before_any_launch(ck):
    # the C entry points see bytes: the binding checks dtypes first (CPU tensors
    # with the right dtypes then fail the CUDA-tensor check, so no launch happens)
    import torch
    i8 = torch.zeros(4, 128, dtype=torch.int8)
    u8 = torch.zeros(8, 64, dtype=torch.uint8)
    f32 = torch.ones(4)
    bf = torch.ones(8, dtype=torch.bfloat16)
    with pytest.raises(TypeError, match="x_scale"):
        ck.gemv_w4a8(i8, f32.to(torch.bfloat16), u8, bf)
    with pytest.raises(TypeError, match="w_scale"):
        ck.gemv_w4a8(i8, f32, u8, bf.float())
    with pytest.raises(TypeError, match="xq"):
        ck.gemv_w4a8_tc(i8.float(), f32, u8, bf)
    with pytest.raises(ValueError, match="CUDA"):
        ck.gemv_w4a8(i8, f32, u8, bf)
    x = torch.zeros(4, 128, dtype=torch.bfloat16)
    with pytest.raises(TypeError, match="x"):
        ck.rotate_quant_rowwise(x.float(), 64, 4)
    with pytest.raises(TypeError, match="scale_out"):
        ck.rotate_quant_rowwise(x, 64, 4, scale_out=torch.empty(4, dtype=torch.float64))
    with pytest.raises(TypeError, match="w_packed"):
        ck.linear_w4a4(x, u8.float(), bf, 64)
    with pytest.raises(TypeError, match="bias"):
        ck.linear_w4a4_scaled(x, u8, bf, 64, 0.5, bias=bf.half())
    with pytest.raises(TypeError, match="wscales"):
        ck.gemv_awq_w4a16(x[:2], u8, bf.half().reshape(2, 4), bf.reshape(2, 4))
    with pytest.raises(TypeError, match="out"):
        ck.gemm_w4a8_i32(i8, u8, out=torch.empty(4, 8, dtype=torch.float32))
    with pytest.raises(ValueError, match="CUDA"):
        ck.gemv_awq_w4a16(x[:2], u8, bf.reshape(2, 4), bf.reshape(2, 4))
