"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Small shapes span several tiles and ragged tails; the five workload configs run
at full size, compared on every output: all rows of the M=8192 linears too, in chunks.
"""

import numpy as np
import pytest
import torch

import oracle as O
from bit_quantized_linear_rotate_b200 import workloads as WL
from tests.parity import (assert_codes_close, assert_out_close, assert_scales_close, bf16_tensor_bits,
                          code_flip_allowance, to_np_f64, unpack_codes)

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

DEV = "cuda:0"


@pytest.fixture(scope="module")
def ck():
    from bit_quantized_linear_rotate_b200 import ck as _ck
    return _ck


@pytest.fixture(autouse=True)
def _no_device_errors(ck):
    yield
    ck.device_error_check()


def _rand_x(M, K, seed, dtype=torch.bfloat16, outliers=0):
    g = torch.Generator().manual_seed(seed)
    return WL.activations(M, K, outliers, g, dtype)


# ------------------------------------------------------------- rotate_quant

@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("G", [16, 64, 256])
def test_rotate_quant_matches_oracle(ck, G, bits, dtype):
    M, K = 37, 768
    xf = _rand_x(M, K + 64, seed=G * 10 + bits, dtype=dtype, outliers=6)
    x = xf.to(DEV)[:, :K]                       # row stride K + 64: non-contiguous rows
    q, s = ck.rotate_quant_rowwise(x, G, bits)
    torch.cuda.synchronize()
    q_ref, s_ref = O.rotate_quant_rowwise(to_np_f64(xf[:, :K]), G, bits)
    assert_scales_close(s.cpu().numpy(), s_ref)
    q_gpu = unpack_codes(q) if bits == 4 else q.cpu().numpy()
    assert_codes_close(q_gpu, q_ref)
    if bits == 4:
        # packed bytes are bit-exact wherever the codes agree
        same = (O.pack_nibbles(q_ref) == q.cpu().numpy())
        agree = (q_gpu == q_ref).reshape(M, K // 2, 2).all(axis=2)
        assert np.array_equal(same[agree], np.ones(int(agree.sum()), dtype=bool))


@pytest.mark.parametrize("G,bits,dtype", [(16, 4, torch.bfloat16), (64, 8, torch.float16), (256, 4, torch.bfloat16),
                                          (3, 8, torch.bfloat16), (1, 4, torch.float16)])
def test_rotate_quant_general_R_matches_oracle(ck, G, bits, dtype):
    # a general rotation: non-symmetric, not orthogonal (y_g = x_g @ R)
    M, K = 37, 768 if G != 3 else 768 - 768 % 6
    xf = _rand_x(M, K + 32, seed=G * 7 + bits, dtype=dtype, outliers=4)
    xf[5] = 0                                    # an all-zero row gets scale 1
    g = torch.Generator().manual_seed(G)
    R = (torch.randn(G, G, generator=g, dtype=torch.float64) / max(G, 1) ** 0.5).float()
    x = xf.to(DEV)[:, :K]
    q, s = ck.rotate_quant_rowwise_r(x, R.to(DEV), bits)
    torch.cuda.synchronize()
    q_ref, s_ref = O.rotate_quant_rowwise(to_np_f64(xf[:, :K]), G, bits, R.double().numpy())
    assert s[5].item() == 1.0
    assert_scales_close(s.cpu().numpy(), s_ref)
    assert_codes_close(unpack_codes(q) if bits == 4 else q.cpu().numpy(), q_ref)


@pytest.mark.parametrize("G", [16, 64, 256])
def test_rotate_quant_general_R_with_hadamard_equals_fast_path(ck, G):
    M, K = 64, 1024
    x = _rand_x(M, K, seed=G, outliers=4).to(DEV)
    H = torch.tensor(O.hadamard_sylvester(G), dtype=torch.float32, device=DEV)
    qg, sg = ck.rotate_quant_rowwise_r(x, H, 8)
    qf, sf = ck.rotate_quant_rowwise(x, G, 8)
    torch.cuda.synchronize()
    assert_scales_close(sg.cpu().numpy(), sf.cpu().numpy().astype(np.float32))
    assert_codes_close(qg.cpu().numpy(), qf.cpu().numpy())


@pytest.mark.parametrize("G", [1, 2, 8, 32, 128])
def test_rotate_quant_other_group_sizes(ck, G):
    M, K = 19, 1024
    xf = _rand_x(M, K, seed=G)
    q, s = ck.rotate_quant_rowwise(xf.to(DEV), G, 8)
    q_ref, s_ref = O.rotate_quant_rowwise(to_np_f64(xf), G, 8)
    assert_scales_close(s.cpu().numpy(), s_ref)
    assert_codes_close(q.cpu().numpy(), q_ref)


def test_rotate_quant_special_rows(ck):
    G, K = 64, 256
    x = torch.zeros(6, K)
    x[1, 70] = 3.0                    # one-hot -> +-qmax Walsh row in group 1
    x[2, 128:192] = -1.5              # constant group -> [-qmax, 0, ...]
    x[3] = torch.linspace(-4, 4, K)
    x[5, 255] = 1e-30                 # tiny but nonzero (bf16 keeps it)
    xb = x.to(torch.bfloat16)
    for bits in (4, 8):
        q, s = ck.rotate_quant_rowwise(xb.to(DEV), G, bits)
        q_ref, s_ref = O.rotate_quant_rowwise(to_np_f64(xb), G, bits)
        q_gpu = unpack_codes(q) if bits == 4 else q.cpu().numpy()
        assert s.cpu()[0].item() == 1.0 and s.cpu()[4].item() == 1.0      # all-zero rows
        assert np.all(q_gpu[0] == 0) and np.all(q_gpu[4] == 0)
        np.testing.assert_array_equal(q_gpu[1], q_ref[1])
        np.testing.assert_array_equal(q_gpu[2], q_ref[2])
        assert_scales_close(s.cpu().numpy(), s_ref)
        assert_codes_close(q_gpu, q_ref, max_frac=1.0 / q_ref.size + 1e-12)


def test_rotate_quant_batched_and_empty(ck):
    xf = _rand_x(10, 512, seed=3).reshape(2, 5, 512)
    q, s = ck.rotate_quant_rowwise(xf.to(DEV), 64, 4)
    assert q.shape == (2, 5, 256) and s.shape == (2, 5)
    q_ref, s_ref = O.rotate_quant_rowwise(to_np_f64(xf.reshape(10, 512)), 64, 4)
    assert_codes_close(unpack_codes(q.reshape(10, 256)), q_ref)
    assert_scales_close(s.reshape(10).cpu().numpy(), s_ref)
    empty = torch.empty(0, 512, device=DEV, dtype=torch.bfloat16)
    q0, s0 = ck.rotate_quant_rowwise(empty, 64, 4)
    assert q0.shape == (0, 256) and s0.shape == (0,)


@pytest.mark.parametrize("M,K", [(3, 16384), (1500, 32768), (2048, 10240)])
def test_rotate_quant_long_rows(ck, M, K):
    xf = _rand_x(M, K, seed=K, outliers=K // 100)
    q, s = ck.rotate_quant_rowwise(xf.to(DEV), 256, 4)
    rows = np.unique(np.r_[0, 1, M // 2, M - 1])
    q_ref, s_ref = O.rotate_quant_rowwise(to_np_f64(xf[rows]), 256, 4)
    assert_scales_close(s.cpu().numpy()[rows], s_ref)
    assert_codes_close(unpack_codes(q.cpu()[rows]), q_ref)


def test_rotate_quant_alternating_row_lengths(ck):
    # launches of one kernel with different dynamic shared memory (64 KB at
    # K = 32768, 56 KB at K = 28672), a larger one after a smaller one
    for K in (32768, 28672, 32768, 24576, 32768):
        xf = _rand_x(3, K, seed=K + 1, outliers=K // 100)
        q, s = ck.rotate_quant_rowwise(xf.to(DEV), 64, 4)
        torch.cuda.synchronize()
        q_ref, s_ref = O.rotate_quant_rowwise(to_np_f64(xf), 64, 4)
        assert_scales_close(s.cpu().numpy(), s_ref)
        assert_codes_close(unpack_codes(q), q_ref)


def test_rotate_quant_mlp_down_G16_full(ck):
    w = WL.LINEAR_MLP_DOWN
    x = WL.linear_inputs(w)["x"]
    for bits in (4, 8):
        q, s = ck.rotate_quant_rowwise(x.to(DEV), w.rq_group, bits)
        q_ref, s_ref = O.rotate_quant_rowwise(to_np_f64(x), w.rq_group, bits)
        assert_scales_close(s.cpu().numpy(), s_ref)
        assert_codes_close(unpack_codes(q) if bits == 4 else q.cpu().numpy(), q_ref)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("G,K", [(64, 3840), (16, 1008), (256, 512)])
def test_rotate_quant_i8_codes_equal_packed_codes(ck, G, K, bits):
    M = 70
    xf = _rand_x(M, K, seed=K + bits, outliers=3)
    x = xf.to(DEV)
    q8, s8 = ck.rotate_quant_rowwise_i8(x, G, bits)
    q, s = ck.rotate_quant_rowwise(x, G, bits)
    q_ref, s_ref = O.rotate_quant_rowwise(to_np_f64(xf), G, bits)
    assert torch.equal(s8, s)
    q_other = unpack_codes(q) if bits == 4 else q.cpu().numpy()
    np.testing.assert_array_equal(q8.cpu().numpy(), q_other)
    assert_codes_close(q8.cpu().numpy(), q_ref)
    assert_scales_close(s8.cpu().numpy(), s_ref)


@pytest.mark.parametrize("R,C", [(3840, 3840), (7, 64), (1, 32)])
def test_unpack_int4_bit_exact(ck, R, C):
    g = torch.Generator().manual_seed(R + C)
    wp = torch.randint(0, 256, (R, C // 2), generator=g, dtype=torch.uint8)
    w8 = ck.unpack_int4(wp.to(DEV))
    np.testing.assert_array_equal(w8.cpu().numpy(), O.unpack_nibbles(wp.numpy()))


# ------------------------------------------------------- integer GEMM (exact)

GEMM_SHAPES = [(128, 128, 256), (300, 384, 520), (1, 32, 8), (257, 4096, 300), (129, 160, 257),
               (512, 3840, 768)]


@pytest.mark.parametrize("M,K,N", GEMM_SHAPES)
def test_gemm_w4a4_i32_bit_exact(ck, M, K, N):
    g = torch.Generator().manual_seed(M * 7 + N)
    qa = torch.randint(0, 256, (M, K // 2), generator=g, dtype=torch.uint8)
    wp = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.uint8)
    acc = ck.gemm_w4a4_i32(qa.to(DEV), wp.to(DEV))
    ref = O.int_matmul(O.unpack_nibbles(qa.numpy()), O.unpack_nibbles(wp.numpy()))
    np.testing.assert_array_equal(acc.cpu().numpy(), ref)


@pytest.mark.parametrize("M,K,N", GEMM_SHAPES)
def test_gemm_w4a8_i32_bit_exact(ck, M, K, N):
    g = torch.Generator().manual_seed(M * 11 + N)
    qa = torch.randint(-127, 128, (M, K), generator=g, dtype=torch.int8)
    wp = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.uint8)
    acc = ck.gemm_w4a8_i32(qa.to(DEV), wp.to(DEV))
    ref = O.int_matmul(qa.numpy().astype(np.int64), O.unpack_nibbles(wp.numpy()))
    np.testing.assert_array_equal(acc.cpu().numpy(), ref)


@pytest.mark.parametrize("M,K,N", GEMM_SHAPES)
def test_gemm_s8_i32_bit_exact(ck, M, K, N):
    g = torch.Generator().manual_seed(M * 13 + N)
    qa = torch.randint(-127, 128, (M, K), generator=g, dtype=torch.int8)
    w8 = torch.randint(-128, 128, (N, K), generator=g, dtype=torch.int8)
    acc = ck.gemm_s8_i32(qa.to(DEV), w8.to(DEV))
    ref = O.int_matmul(qa.numpy().astype(np.int64), w8.numpy().astype(np.int64))
    np.testing.assert_array_equal(acc.cpu().numpy(), ref)


def test_gemm_extreme_operands(ck):
    M, K, N = 130, 10240, 260
    qa = torch.full((M, K // 2), 0xFF, dtype=torch.uint8)      # +7 everywhere
    wp = torch.zeros((N, K // 2), dtype=torch.uint8)            # -8 everywhere
    acc = ck.gemm_w4a4_i32(qa.to(DEV), wp.to(DEV)).cpu()
    assert torch.all(acc == -56 * K)
    q8 = torch.full((M, K), -127, dtype=torch.int8)
    acc = ck.gemm_w4a8_i32(q8.to(DEV), wp.to(DEV)).cpu()
    assert torch.all(acc == 1016 * K)


@pytest.mark.parametrize("with_bias", [False, True])
@pytest.mark.parametrize("M,K,N", [(200, 512, 300), (128, 3840, 256), (33, 96, 40)])
def test_gemm_w4a4_epilogue_bit_exact(ck, M, K, N, with_bias):
    g = torch.Generator().manual_seed(M + N + int(with_bias))
    qa = torch.randint(0, 256, (M, K // 2), generator=g, dtype=torch.uint8)
    sa = (torch.rand(M, generator=g) * 0.5 + 0.01)
    wp = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.uint8)
    sw = WL.uniform((N,), 0.005, 0.02, g)
    bias = WL.uniform((N,), -1, 1, g) if with_bias else None
    y = ck.gemm_w4a4(qa.to(DEV), sa.to(DEV), wp.to(DEV), sw.to(DEV), None if bias is None else bias.to(DEV))
    acc = O.int_matmul(O.unpack_nibbles(qa.numpy()), O.unpack_nibbles(wp.numpy()))
    ref_bits = O.to_bf16_bits(O.epilogue_rowwise(acc, sa.numpy(), to_np_f64(sw),
                                                 None if bias is None else to_np_f64(bias)))
    np.testing.assert_array_equal(bf16_tensor_bits(y), ref_bits)


@pytest.mark.parametrize("M,K,N", [(200, 512, 300), (8192, 3840, 256), (45, 160, 70)])
def test_gemm_w4a8_and_s8_epilogue_bit_exact(ck, M, K, N):
    g = torch.Generator().manual_seed(M * 3 + N)
    qa = torch.randint(-127, 128, (M, K), generator=g, dtype=torch.int8)
    sa = torch.rand(M, generator=g) * 0.5 + 0.01
    wp = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.uint8)
    sw = WL.uniform((N,), 0.005, 0.02, g)
    bias = WL.uniform((N,), -1, 1, g)
    acc = O.int_matmul(qa.numpy().astype(np.int64), O.unpack_nibbles(wp.numpy()))
    ref_bits = O.to_bf16_bits(O.epilogue_rowwise(acc, sa.numpy(), to_np_f64(sw), to_np_f64(bias)))
    y = ck.gemm_w4a8(qa.to(DEV), sa.to(DEV), wp.to(DEV), sw.to(DEV), bias.to(DEV))
    np.testing.assert_array_equal(bf16_tensor_bits(y), ref_bits)
    w8 = ck.unpack_int4(wp.to(DEV))
    y8 = ck.gemm_s8(qa.to(DEV), sa.to(DEV), w8, sw.to(DEV), bias.to(DEV))
    np.testing.assert_array_equal(bf16_tensor_bits(y8), ref_bits)


# --------------------------------------------------------- W4A4 linear (e2e)

@pytest.mark.parametrize("M,K,N,G,bias,dtype", [
    (37, 512, 300, 64, True, torch.bfloat16),
    (129, 768, 260, 256, False, torch.float16),
    (300, 256, 520, 16, True, torch.bfloat16),
    (64, 3840, 3840, 64, False, torch.bfloat16),
    (24, 1024, 264, 16, True, torch.float16),      # small-batch route, fp16, packed codes
])
def test_linear_w4a4_matches_oracle(ck, M, K, N, G, bias, dtype):
    d = WL.small_linear_inputs(M, K, N, seed=M + K, n_outlier_cols=K // 100, dtype=dtype, with_bias=bias)
    b = d.get("bias")
    y = ck.linear_w4a4(d["x"].to(DEV), d["w_packed"].to(DEV), d["w_scale"].to(DEV), G,
                       bias=None if b is None else b.to(DEV))
    r = O.linear_w4a4(to_np_f64(d["x"]), d["w_packed"].numpy(), to_np_f64(d["w_scale"]), G,
                      bias=None if b is None else to_np_f64(b))
    assert_out_close(to_np_f64(y), O.bf16_bits_to_f64(r["y_bits"]))


# ------------------------------------------------- tensor-wise input scale

@pytest.mark.parametrize("G,bits,dtype,a", [
    (16, 4, torch.bfloat16, 0.37), (64, 8, torch.float16, 5.5), (256, 4, torch.bfloat16, 1e-3),
    (64, 4, torch.float16, 3.0e4), (32, 8, torch.bfloat16, 0.71), (64, 4, torch.bfloat16, 0.0),
])
def test_rotate_quant_scaled_matches_oracle(ck, G, bits, dtype, a):
    M, K = 37, 768
    xf = _rand_x(M, K + 64, seed=G + bits, dtype=dtype, outliers=6)
    x = xf.to(DEV)[:, :K]
    q, s = ck.rotate_quant_rowwise_scaled(x, G, bits, a)
    torch.cuda.synchronize()
    q_ref, s_ref = O.rotate_quant_rowwise(to_np_f64(xf[:, :K]), G, bits, input_scale=a)
    q_gpu = unpack_codes(q) if bits == 4 else q.cpu().numpy()
    if a == 0.0:
        assert np.all(s.cpu().numpy() == 1.0) and np.all(q_gpu == 0)
    assert_scales_close(s.cpu().numpy(), s_ref)
    assert_codes_close(q_gpu, q_ref)


@pytest.mark.parametrize("bits", [4, 8])
def test_rotate_quant_scaled_by_powers_of_two_is_exact(ck, bits):
    # a = 1 is the unscaled call bit for bit; a = 2^k keeps every code and
    # multiplies every scale by 2^k exactly (each step is exact in binary fp)
    M, K, G = 300, 1024, 64
    x = _rand_x(M, K, seed=9, outliers=10).to(DEV)
    q1, s1 = ck.rotate_quant_rowwise(x, G, bits)
    for a in (1.0, 0.125, 64.0):
        qa, sa = ck.rotate_quant_rowwise_scaled(x, G, bits, a)
        torch.cuda.synchronize()
        assert torch.equal(qa, q1)
        assert torch.equal(sa, s1 * a)


@pytest.mark.parametrize("M,K,N,G,bias,dtype,a", [
    (300, 1024, 520, 64, True, torch.bfloat16, 0.37),
    (129, 768, 260, 256, False, torch.float16, 12.0),
    (32, 3840, 520, 64, True, torch.bfloat16, 2.5),        # small-batch route
    (200, 512, 300, 16, True, torch.bfloat16, 0.0),
])
def test_linear_w4a4_scaled_matches_oracle(ck, M, K, N, G, bias, dtype, a):
    d = WL.small_linear_inputs(M, K, N, seed=M + N, n_outlier_cols=K // 100, dtype=dtype, with_bias=bias)
    b = d.get("bias")
    y = ck.linear_w4a4_scaled(d["x"].to(DEV), d["w_packed"].to(DEV), d["w_scale"].to(DEV), G, a,
                              bias=None if b is None else b.to(DEV))
    r = O.linear_w4a4(to_np_f64(d["x"]), d["w_packed"].numpy(), to_np_f64(d["w_scale"]), G,
                      bias=None if b is None else to_np_f64(b), input_scale=a)
    if a == 0.0:
        # every row quantizes to zero codes: y is the bias, exactly
        expect = b.expand(M, N) if b is not None else torch.zeros(M, N, dtype=torch.bfloat16)
        assert torch.equal(y.cpu(), expect.to(torch.bfloat16))
    assert_out_close(to_np_f64(y), O.bf16_bits_to_f64(r["y_bits"]))


def test_linear_w4a4_scaled_by_one_is_the_unscaled_call(ck):
    for M in (300, 32):
        d = WL.small_linear_inputs(M, 1024, 264, seed=3, n_outlier_cols=10, with_bias=True)
        args = (d["x"].to(DEV), d["w_packed"].to(DEV), d["w_scale"].to(DEV), 64)
        y1 = ck.linear_w4a4(*args, bias=d["bias"].to(DEV))
        ya = ck.linear_w4a4_scaled(*args, 1.0, bias=d["bias"].to(DEV))
        torch.cuda.synchronize()
        assert np.array_equal(bf16_tensor_bits(ya), bf16_tensor_bits(y1))


def _a256(v):
    return (v + 255) // 256 * 256


def _small_m_route(M, K):
    # small batches run the linear's product on the decode GEMV, with natural-order codes
    return M <= 64 and K % 128 == 0 and K <= 4096


def _linear_workspace(ws, M, K, bits=4):
    """(codes in natural column order, scales, row sums or None) from the linear's workspace.

    Small batches keep int4 codes packed two per byte (offset binary, low nibble = even column)
    followed by room for them one per byte; int8 codes (the W4A8 linear) one per byte."""
    small = _small_m_route(M, K)
    nq = _a256(M * K // 2) + _a256(M * K) if small else _a256(M * K)
    s = ws[nq:nq + 4 * M].view(torch.float32).cpu().numpy()
    if small and bits == 4:
        b = ws[:M * K // 2].cpu().numpy().reshape(M, K // 2).astype(np.int64)
        q = np.empty((M, K), dtype=np.int64)
        q[:, 0::2] = (b & 15) - 8
        q[:, 1::2] = (b >> 4) - 8
        return q, s, None
    q = ws[:M * K].view(torch.int8).view(M, K).cpu().numpy().astype(np.int64)
    if small:
        return q, s, None
    perm = np.array([0, 2, 4, 6, 1, 3, 5, 7])
    nat = np.empty_like(q)
    for j in range(8):
        nat[:, perm[j]::8] = q[:, j::8]
    rs = ws[nq + _a256(4 * M):nq + _a256(4 * M) + 4 * M].view(torch.int32).cpu().numpy()
    return nat, s, rs


@pytest.mark.parametrize("M,K,N", [(300, 1024, 520), (32, 3840, 520), (1, 1024, 96), (64, 1024, 520),
                                   (65, 1024, 520), (17, 128, 72), (24, 2048, 1000), (40, 512, 264),
                                   (33, 256, 100), (32, 4096, 4736)])
def test_linear_phases_equal_rotate_quant_plus_gemm_w4a4(ck, M, K, N):
    # both routes of the linear (tensor-core GEMM; decode GEMV for small batches) give the
    # result of rotate_quant(bits = 4) followed by the packed-activation GEMM, bit for bit
    d = WL.small_linear_inputs(M, K, N, seed=11 + M, n_outlier_cols=10, with_bias=True)
    x, wp, sw, b = d["x"].to(DEV), d["w_packed"].to(DEV), d["w_scale"].to(DEV), d["bias"].to(DEV)
    ws = torch.empty(ck.linear_w4a4_workspace_bytes(M, K), device=DEV, dtype=torch.uint8)
    ck.linear_w4a4_quantize(x, 64, ws)
    y2 = ck.linear_w4a4_matmul(M, K, wp, sw, ws, bias=b)
    y1 = ck.linear_w4a4(x, wp, sw, 64, bias=b)
    qp, sp = ck.rotate_quant_rowwise(x, 64, 4)
    y0 = ck.gemm_w4a4(qp, sp, wp, sw, bias=b)
    assert torch.equal(y1, y0) and torch.equal(y2, y0)
    q, s, rs = _linear_workspace(ws, M, K)
    np.testing.assert_array_equal(q, unpack_codes(qp))
    np.testing.assert_array_equal(s, sp.cpu().numpy())
    if rs is not None:
        np.testing.assert_array_equal(rs, q.sum(axis=1))


def _linear_full_config(ck, w, chunk_rows=2048, bits=4):
    """Runs the linear (W4A4, or W4A8 with bits=8) at full size and compares every row with the
    oracle, in row chunks (the oracle's float64 intermediates of one chunk stay within a few
    hundred MB)."""
    d = WL.linear_inputs(w)
    x, wp, sw = d["x"].to(DEV), d["w_packed"].to(DEV), d["w_scale"].to(DEV)
    ws = torch.empty(ck.linear_w4a4_workspace_bytes(w.M, w.K), device=DEV, dtype=torch.uint8)
    call = ck.linear_w4a4 if bits == 4 else ck.linear_w4a8
    oracle_linear = O.linear_w4a4 if bits == 4 else O.linear_w4a8
    y = call(x, wp, sw, w.G, workspace=ws)
    torch.cuda.synchronize()
    # the quantized activations the GEMM consumed (workspace: int8 codes with each 8-column group
    # stored as columns (0 2 4 6 1 3 5 7), row scales, row sums of the codes)
    qa_all, sa_all, rs_all = _linear_workspace(ws, w.M, w.K, bits)
    qmax = O.QMAX[bits]
    assert qa_all.min() >= -qmax and qa_all.max() <= qmax
    if rs_all is not None:
        np.testing.assert_array_equal(rs_all, qa_all.sum(axis=1))
    y_cpu = y.cpu()
    wq = O.unpack_nibbles(d["w_packed"].numpy())
    sw64 = to_np_f64(d["w_scale"])
    n_diff = n_flip_rows = 0
    err2 = ref2 = 0.0
    for r0 in range(0, w.M, chunk_rows):
        rows = slice(r0, min(w.M, r0 + chunk_rows))
        r = oracle_linear(to_np_f64(d["x"][rows]), d["w_packed"].numpy(), sw64, w.G)
        qa, sa = qa_all[rows], sa_all[rows]
        dq = np.abs(qa - r["q"])
        assert dq.max(initial=0) <= 1, f"rows {rows}: codes differ by {dq.max()}"
        n_diff += int((dq != 0).sum())
        assert_scales_close(sa, r["s"])
        y_ref = O.bf16_bits_to_f64(r["y_bits"])
        y_gpu = to_np_f64(y_cpu[rows])
        extra, flips = code_flip_allowance(qa, r["q"], wq, r["s"], sw64)
        n_flip_rows += int(np.any(dq != 0, axis=1).sum())
        assert_out_close(y_gpu, y_ref, extra=extra)
        err2 += float(np.sum((y_gpu - y_ref) ** 2))
        ref2 += float(np.sum(y_ref ** 2))
        # with identical quantized inputs the GEMM + epilogue is bit-exact
        exact = O.to_bf16_bits(O.epilogue_rowwise(O.int_matmul(qa, wq), sa, sw64))
        np.testing.assert_array_equal(bf16_tensor_bits(y_cpu[rows]), exact)
    frac = n_diff / float(w.M * w.K)
    assert frac <= 1e-3, f"{frac:.4%} of codes differ (limit 0.1 %)"
    rel = np.sqrt(err2 / ref2)
    assert rel <= 1e-2
    print(f"{w.name} bits={bits}: {n_diff} codes differ by one LSB ({frac:.2e}) in {n_flip_rows} rows; "
          f"normwise rel err {rel:.3e}")
    return rel


def test_linear_config_M32_full(ck):
    _linear_full_config(ck, WL.LINEAR_M32)


def test_linear_config_M8192_full(ck):
    _linear_full_config(ck, WL.LINEAR_M8192)


def test_linear_config_mlp_down_full(ck):
    _linear_full_config(ck, WL.LINEAR_MLP_DOWN)


# ------------------------------------------------------------- W4A8 linear

@pytest.mark.parametrize("M,K,N,G,bias,dtype", [
    (300, 1024, 520, 64, True, torch.bfloat16),     # tensor-core route, ragged M and N
    (129, 512, 256, 16, False, torch.float16),
    (257, 2048, 384, 256, True, torch.bfloat16),
    (32, 3840, 520, 64, True, torch.bfloat16),      # small-batch route (decode GEMV)
    (7, 256, 72, 64, False, torch.float16),
])
def test_linear_w4a8_matches_oracle(ck, M, K, N, G, bias, dtype):
    d = WL.small_linear_inputs(M, K, N, seed=40 + M, n_outlier_cols=6, with_bias=bias)
    x = d["x"].to(dtype)
    b = d["bias"].to(DEV) if bias else None
    y = ck.linear_w4a8(x.to(DEV), d["w_packed"].to(DEV), d["w_scale"].to(DEV), G, bias=b)
    r = O.linear_w4a8(to_np_f64(x), d["w_packed"].numpy(), to_np_f64(d["w_scale"]), G,
                      bias=to_np_f64(d["bias"]) if bias else None)
    assert_out_close(to_np_f64(y.cpu()), O.bf16_bits_to_f64(r["y_bits"]))


@pytest.mark.parametrize("M,K,N", [(300, 1024, 520), (32, 3840, 520), (65, 1024, 520), (1, 128, 40)])
def test_linear_w4a8_equals_rotate_quant_plus_gemm_w4a8(ck, M, K, N):
    # both routes give the result of rotate_quant(bits = 8) followed by the int8-activation GEMM, bit
    # for bit, and the workspace holds the same codes, scales and row sums
    d = WL.small_linear_inputs(M, K, N, seed=50 + M, n_outlier_cols=10, with_bias=True)
    x, wp, sw, b = d["x"].to(DEV), d["w_packed"].to(DEV), d["w_scale"].to(DEV), d["bias"].to(DEV)
    ws = torch.empty(ck.linear_w4a8_workspace_bytes(M, K), device=DEV, dtype=torch.uint8)
    y1 = ck.linear_w4a8(x, wp, sw, 64, bias=b, workspace=ws)
    q8, s8 = ck.rotate_quant_rowwise(x, 64, 8)
    y0 = ck.gemm_w4a8(q8, s8, wp, sw, bias=b)
    assert torch.equal(y1, y0)
    q, s, rs = _linear_workspace(ws, M, K, bits=8)
    np.testing.assert_array_equal(q, q8.cpu().numpy().astype(np.int64))
    np.testing.assert_array_equal(s, s8.cpu().numpy())
    if rs is not None:
        np.testing.assert_array_equal(rs, q.sum(axis=1))


def test_linear_w4a8_config_M8192_full(ck):
    # the W4A8 linear on the M = 8192, K = N = 3840, G = 64 workload, every row against the oracle
    _linear_full_config(ck, WL.LINEAR_M8192, bits=8)


# ------------------------------------------- linear on pre-unpacked int8 weights

@pytest.mark.parametrize("M,K,N,G,bias", [(300, 1024, 520, 64, True), (32, 3840, 256, 64, False),
                                          (129, 512, 72, 16, True), (8192, 3840, 3840, 64, False)])
def test_linear_w4a4_predecoded_equals_linear_w4a4(ck, M, K, N, G, bias):
    # the weight-cache variant: unpack once, then the linear on int8 weights gives the packed
    # linear's result bit for bit
    d = WL.small_linear_inputs(M, K, N, seed=60 + M, n_outlier_cols=8, with_bias=bias)
    x, wp, sw = d["x"].to(DEV), d["w_packed"].to(DEV), d["w_scale"].to(DEV)
    b = d["bias"].to(DEV) if bias else None
    w8 = ck.unpack_int4(wp)
    y0 = ck.linear_w4a4(x, wp, sw, G, bias=b)
    y1 = ck.linear_w4a4_predecoded(x, w8, sw, G, bias=b)
    assert torch.equal(y1, y0)
    if M <= 512:
        r = O.linear_w4a4(to_np_f64(d["x"]), d["w_packed"].numpy(), to_np_f64(sw.cpu()), G,
                          bias=to_np_f64(d["bias"]) if bias else None)
        assert_out_close(to_np_f64(y1.cpu()), O.bf16_bits_to_f64(r["y_bits"]))


# -------------------------------------------------------------------- GEMVs

def _w4a8_inputs_quantized(w, M):
    d = WL.gemv_w4a8_inputs(w, M)
    q, s = O.rotate_quant_rowwise(to_np_f64(d["x"]), 1, 8)     # rowwise int8, no rotation
    return d, torch.from_numpy(q.astype(np.int8)), torch.from_numpy(s)


@pytest.mark.parametrize("M", WL.GEMV_W4A8.Ms)
def test_gemv_w4a8_config_bit_exact(ck, M):
    w = WL.GEMV_W4A8
    d, xq, xs = _w4a8_inputs_quantized(w, M)
    y = ck.gemv_w4a8(xq.to(DEV), xs.to(DEV), d["w_packed"].to(DEV), d["w_scale"].to(DEV))
    r = O.gemv_w4a8(xq.numpy(), xs.numpy(), d["w_packed"].numpy(), to_np_f64(d["w_scale"]))
    np.testing.assert_array_equal(bf16_tensor_bits(y), r["y_bits"])


@pytest.mark.parametrize("M,K,N,bias", [(3, 256, 100, True), (9, 512, 37, False), (16, 1280, 48, True),
                                        (1, 128, 16, False)])
def test_gemv_w4a8_ragged_bit_exact(ck, M, K, N, bias):
    g = torch.Generator().manual_seed(M * N)
    xq = torch.randint(-127, 128, (M, K), generator=g, dtype=torch.int8)
    xs = torch.rand(M, generator=g) * 0.1 + 0.001
    wp = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.uint8)
    sw = WL.uniform((N,), 0.005, 0.02, g)
    b = WL.uniform((N,), -1, 1, g) if bias else None
    y = ck.gemv_w4a8(xq.to(DEV), xs.to(DEV), wp.to(DEV), sw.to(DEV), None if b is None else b.to(DEV))
    r = O.gemv_w4a8(xq.numpy(), xs.numpy(), wp.numpy(), to_np_f64(sw), None if b is None else to_np_f64(b))
    np.testing.assert_array_equal(bf16_tensor_bits(y), r["y_bits"])


@pytest.mark.parametrize("M,K,N,bias", [(1, 128, 8, False), (8, 128, 16, True), (5, 384, 24, True), (2, 4096, 40, False),
                                        (7, 1024, 1000, True), (4, 2048, 2376, False), (8, 4096, 4736, True),
                                        (3, 512, 12288, False), (9, 128, 8, True), (12, 384, 24, False),
                                        (16, 4096, 4736, True), (13, 3840, 3840, False), (16, 2048, 12288, True)])
def test_gemv_w4a8_rowsplit_shapes_bit_exact(ck, M, K, N, bias):
    # the row-split streaming kernel (M <= 16, N % 8 == 0; one token group up to M = 8, two
    # above): CTAs owning one octet of rows, the last tile of a CTA moved back over rows an
    # earlier tile wrote, K from one chunk to 32 chunks
    g = torch.Generator().manual_seed(M * 7919 + N)
    xq = torch.randint(-127, 128, (M, K), generator=g, dtype=torch.int8)
    xs = torch.rand(M, generator=g) * 0.1 + 0.001
    wp = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.uint8)
    sw = WL.uniform((N,), 0.005, 0.02, g)
    b = WL.uniform((N,), -1, 1, g) if bias else None
    y = ck.gemv_w4a8(xq.to(DEV), xs.to(DEV), wp.to(DEV), sw.to(DEV), None if b is None else b.to(DEV))
    r = O.gemv_w4a8(xq.numpy(), xs.numpy(), wp.numpy(), to_np_f64(sw), None if b is None else to_np_f64(b))
    np.testing.assert_array_equal(bf16_tensor_bits(y), r["y_bits"])


def test_gemv_w4a8_unaligned_scales_take_another_path(ck):
    # scales that are not 16-byte aligned cannot be bulk-copied: the call still gives the exact result
    M, K, N = 4, 512, 64
    g = torch.Generator().manual_seed(5)
    xq = torch.randint(-127, 128, (M, K), generator=g, dtype=torch.int8)
    xs = torch.rand(M, generator=g) * 0.1 + 0.001
    wp = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.uint8)
    sw = WL.uniform((N + 1,), 0.005, 0.02, g)
    y = ck.gemv_w4a8(xq.to(DEV), xs.to(DEV), wp.to(DEV), sw.to(DEV)[1:])
    r = O.gemv_w4a8(xq.numpy(), xs.numpy(), wp.numpy(), to_np_f64(sw[1:]))
    np.testing.assert_array_equal(bf16_tensor_bits(y), r["y_bits"])


def _tall_sample(N, seed):
    rng = np.random.default_rng(seed)
    return np.unique(np.r_[0, 1, 2, N // 2, N - 2, N - 1, rng.integers(0, N, 300)])


@pytest.mark.parametrize("M", [4, 12])
def test_gemv_w4a8_tall_weights_bit_exact(ck, M):
    # 2M weight rows of K = 128: each CTA's per-row scale and bias slices no
    # longer leave room for a ring of two weight stages, so the general kernel
    # runs; sampled output columns are checked bit for bit
    K, N = 128, 2_000_000
    g = torch.Generator().manual_seed(M + 77)
    xq = torch.randint(-127, 128, (M, K), generator=g, dtype=torch.int8)
    xs = torch.rand(M, generator=g) * 0.1 + 0.001
    wp = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.uint8)
    sw = WL.uniform((N,), 0.005, 0.02, g)
    b = WL.uniform((N,), -1, 1, g)
    y = ck.gemv_w4a8(xq.to(DEV), xs.to(DEV), wp.to(DEV), sw.to(DEV), b.to(DEV))
    idx = _tall_sample(N, M)
    r = O.gemv_w4a8(xq.numpy(), xs.numpy(), wp.numpy()[idx], to_np_f64(sw)[idx], to_np_f64(b)[idx])
    np.testing.assert_array_equal(bf16_tensor_bits(y)[:, idx], r["y_bits"])


def test_gemv_awq_tall_weights(ck):
    M, K, N, G = 2, 128, 4_000_000, 64
    g = torch.Generator().manual_seed(91)
    x = WL.activations(M, K, 0, g)
    qw = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.uint8)
    ws = WL.uniform((K // G, N), 0.001, 0.01, g)
    wz = (torch.randn((K // G, N), generator=g) * 0.01).to(torch.bfloat16)
    y = ck.gemv_awq_w4a16(x.to(DEV), qw.to(DEV), ws.to(DEV), wz.to(DEV), None, group_size=G)
    idx = _tall_sample(N, 5)
    r = O.gemv_awq_w4a16(to_np_f64(x), qw.numpy()[idx], to_np_f64(ws)[:, idx], to_np_f64(wz)[:, idx], G)
    assert_out_close(to_np_f64(y)[:, idx], r["y_f64"])


@pytest.mark.parametrize("M,K,N", [(5, 8192, 96), (16, 4224, 40)])
def test_gemv_w4a8_general_path_bit_exact(ck, M, K, N):
    # K > 4096 takes the general (non-streaming) kernel
    g = torch.Generator().manual_seed(K + N)
    xq = torch.randint(-127, 128, (M, K), generator=g, dtype=torch.int8)
    xs = torch.rand(M, generator=g) * 0.1 + 0.001
    wp = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.uint8)
    sw = WL.uniform((N,), 0.005, 0.02, g)
    y = ck.gemv_w4a8(xq.to(DEV), xs.to(DEV), wp.to(DEV), sw.to(DEV))
    r = O.gemv_w4a8(xq.numpy(), xs.numpy(), wp.numpy(), to_np_f64(sw))
    np.testing.assert_array_equal(bf16_tensor_bits(y), r["y_bits"])


@pytest.mark.parametrize("M,K,N,bias", [(3, 256, 100, True), (1, 128, 300, False), (9, 512, 37, True),
                                         (16, 1280, 48, True), (5, 8192, 96, False), (12, 4096, 1000, True),
                                         (16, 3840, 3840, False)])
def test_gemv_w4a8_tc_bit_exact(ck, M, K, N, bias):
    # the tensor-core GEMV against the oracle and the default GEMV, bit for bit
    g = torch.Generator().manual_seed(M * K + N)
    xq = torch.randint(-128, 128, (M, K), generator=g, dtype=torch.int8)
    xs = torch.rand(M, generator=g) * 0.1 + 0.001
    wp = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.uint8)
    sw = WL.uniform((N,), 0.005, 0.02, g)
    b = WL.uniform((N,), -1, 1, g) if bias else None
    args = (xq.to(DEV), xs.to(DEV), wp.to(DEV), sw.to(DEV), None if b is None else b.to(DEV))
    y = ck.gemv_w4a8_tc(*args)
    r = O.gemv_w4a8(xq.numpy(), xs.numpy(), wp.numpy(), to_np_f64(sw), None if b is None else to_np_f64(b))
    np.testing.assert_array_equal(bf16_tensor_bits(y), r["y_bits"])
    assert np.array_equal(bf16_tensor_bits(ck.gemv_w4a8(*args)), bf16_tensor_bits(y))


@pytest.mark.parametrize("M", WL.GEMV_W4A8.Ms)
def test_gemv_w4a8_tc_config_equals_default(ck, M):
    d = WL.gemv_w4a8_inputs(WL.GEMV_W4A8, M)
    xq, xs = ck.rotate_quant_rowwise(d["x"].to(DEV), 1, 8)
    wp, sw = d["w_packed"].to(DEV), d["w_scale"].to(DEV)
    y_tc = ck.gemv_w4a8_tc(xq, xs, wp, sw)
    y = ck.gemv_w4a8(xq, xs, wp, sw)
    torch.cuda.synchronize()
    assert torch.equal(y_tc.view(torch.int16), y.view(torch.int16))


def test_gemv_w4a8_agrees_with_large_m_gemm(ck):
    # the decode GEMV and the tensor-core GEMM share codec and epilogue: same int32 results
    g = torch.Generator().manual_seed(5)
    M, K, N = 16, 4096, 512
    xq = torch.randint(-127, 128, (M, K), generator=g, dtype=torch.int8)
    wp = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.uint8)
    ones = torch.ones(M)
    sw = torch.ones(N, dtype=torch.bfloat16)
    acc = ck.gemm_w4a8_i32(xq.to(DEV), wp.to(DEV)).cpu()
    y = ck.gemv_w4a8(xq.to(DEV), ones.to(DEV), wp.to(DEV), sw.to(DEV)).cpu()
    assert torch.equal(acc.float().to(torch.bfloat16), y)


@pytest.mark.parametrize("M", WL.GEMV_AWQ.Ms)
def test_gemv_awq_config(ck, M):
    w = WL.GEMV_AWQ
    d = WL.gemv_awq_inputs(w, M)
    y = ck.gemv_awq_w4a16(d["x"].to(DEV), d["qweight"].to(DEV), d["wscales"].to(DEV), d["wzeros"].to(DEV),
                          group_size=w.G)
    r = O.gemv_awq_w4a16(to_np_f64(d["x"]), d["qweight"].numpy(), to_np_f64(d["wscales"]),
                         to_np_f64(d["wzeros"]), w.G)
    assert_out_close(to_np_f64(y), r["y_f64"])


@pytest.mark.parametrize("M,K,N,G,dtype,bias", [
    (1, 128, 40, 64, torch.bfloat16, True),
    (5, 1024, 70, 128, torch.float16, False),      # N % 8 != 0: general kernel
    (8, 768, 33, 256, torch.bfloat16, True),       # general kernel
    (2, 3072, 96, 64, torch.float16, True),
    (3, 8192, 48, 64, torch.bfloat16, True),       # K > 4096: general kernel
    (4, 4096, 4104, 128, torch.bfloat16, False),   # ragged last 16-row tile
])
def test_gemv_awq_variants(ck, M, K, N, G, dtype, bias):
    g = torch.Generator().manual_seed(K + N)
    x = WL.activations(M, K, 0, g, dtype)
    qw = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.uint8)
    ws = WL.uniform((K // G, N), 0.001, 0.01, g, dtype)
    wz = (torch.randn((K // G, N), generator=g) * 0.01).to(dtype)
    b = WL.uniform((N,), -1, 1, g, dtype) if bias else None
    y = ck.gemv_awq_w4a16(x.to(DEV), qw.to(DEV), ws.to(DEV), wz.to(DEV), None if b is None else b.to(DEV),
                          group_size=G)
    r = O.gemv_awq_w4a16(to_np_f64(x), qw.numpy(), to_np_f64(ws), to_np_f64(wz), G,
                         None if b is None else to_np_f64(b))
    assert_out_close(to_np_f64(y), r["y_f64"])


# ------------------------------------------------------------- error paths

def test_bounded_wait_reports_timeout_and_context_survives(ck):
    ck.selftest_bounded_wait(2_000_000)          # 2 ms: nothing ever arrives
    with pytest.raises(ck.CKError) as e:
        ck.device_error_check()
    assert e.value.status == ck.CK_ERR_TIMEOUT
    ck.device_error_check()                       # cleared
    x = _rand_x(4, 256, seed=1).to(DEV)
    q, s = ck.rotate_quant_rowwise(x, 64, 8)      # the context still works
    torch.cuda.synchronize()
    assert torch.all(s > 0)


def test_invalid_arguments_raise(ck):
    x = torch.zeros(4, 96, device=DEV, dtype=torch.bfloat16)
    with pytest.raises(ck.CKError) as e:
        ck.rotate_quant_rowwise(x, 64, 4)
    assert e.value.status == ck.CK_ERR_INVALID_ARG
    with pytest.raises(ck.CKError) as e:
        ck.gemv_w4a8(torch.zeros(17, 128, device=DEV, dtype=torch.int8), torch.ones(17, device=DEV),
                     torch.zeros(8, 64, device=DEV, dtype=torch.uint8), torch.ones(8, device=DEV, dtype=torch.bfloat16))
    assert e.value.status == ck.CK_ERR_UNSUPPORTED


# ------------------------------------ back-to-back calls (programmatic dependents)

def test_back_to_back_linear_calls_share_a_workspace(ck):
    """Consecutive linears on one stream reuse one workspace with no host sync in between: the
    next call's rotate+quant may only overwrite the workspace once the previous GEMM is done."""
    M, K, N, G = 1024, 3840, 3840, 64
    ins = [WL.small_linear_inputs(M, K, N, 40 + i, n_outlier_cols=8) for i in range(4)]
    ds = [{k: v.to(DEV) for k, v in d.items()} for d in ins]
    refs = []
    for d in ds:   # one call at a time, synchronised
        refs.append(ck.linear_w4a4(d["x"], d["w_packed"], d["w_scale"], G).clone())
        torch.cuda.synchronize()
    ws = torch.empty(ck.linear_w4a4_workspace_bytes(M, K), device=DEV, dtype=torch.uint8)
    outs = [torch.empty(M, N, device=DEV, dtype=torch.bfloat16) for _ in ds]
    for rep in range(3):
        for d, o in zip(ds, outs):
            ck.linear_w4a4(d["x"], d["w_packed"], d["w_scale"], G, workspace=ws, out=o)
    torch.cuda.synchronize()
    for o, r in zip(outs, refs):
        assert torch.equal(o.view(torch.int16), r.view(torch.int16))
    ck.device_error_check()


def test_graph_replay_equals_eager_calls(ck):
    """Chains of calls captured once in a CUDA graph and replayed (how the bench times the GEMVs
    and the other configs): every output equals the eager call's, bit for bit."""
    g = torch.Generator().manual_seed(123)
    K8, N8 = 4096, 2048
    wps = [torch.randint(0, 256, (N8, K8 // 2), generator=g, dtype=torch.uint8).to(DEV) for _ in range(3)]
    sw = WL.uniform((N8,), 0.005, 0.02, g).to(DEV)
    xqs = {M: torch.randint(-127, 128, (M, K8), generator=g, dtype=torch.int8).to(DEV) for M in (4, 16)}
    xss = {M: (torch.rand(M, generator=g) * 0.1 + 0.001).to(DEV) for M in (4, 16)}
    Ka, Na, G = 3072, 2048, 64
    xa = WL.activations(2, Ka, 0, g).to(DEV)
    qws = [torch.randint(0, 256, (Na, Ka // 2), generator=g, dtype=torch.uint8).to(DEV) for _ in range(3)]
    wsa = WL.uniform((Ka // G, Na), 0.001, 0.01, g).to(DEV)
    wza = (torch.randn((Ka // G, Na), generator=g) * 0.01).to(torch.bfloat16).to(DEV)
    lin = {M: WL.small_linear_inputs(M, 1024, 520, seed=M, n_outlier_cols=10, with_bias=True) for M in (300, 32)}
    lin = {M: {k: v.to(DEV) for k, v in d.items()} for M, d in lin.items()}
    wss = {M: torch.empty(ck.linear_w4a4_workspace_bytes(M, 1024), device=DEV, dtype=torch.uint8) for M in lin}
    xr = WL.activations(257, 3840, 38, g).to(DEV)

    def chain(outs):
        i = 0
        for c in range(3):
            for M in (4, 16):
                ck.gemv_w4a8(xqs[M], xss[M], wps[c], sw, out=outs[i]); i += 1
            ck.gemv_awq_w4a16(xa, qws[c], wsa, wza, group_size=G, out=outs[i]); i += 1
        for M, d in lin.items():
            ck.linear_w4a4(d["x"], d["w_packed"], d["w_scale"], G, bias=d["bias"], workspace=wss[M], out=outs[i])
            i += 1
        ck.rotate_quant_rowwise(xr, 64, 4, q_out=outs[i], scale_out=outs[i + 1])

    def make_outs():
        o = []
        for c in range(3):
            o += [torch.empty(M, N8, device=DEV, dtype=torch.bfloat16) for M in (4, 16)]
            o.append(torch.empty(2, Na, device=DEV, dtype=torch.bfloat16))
        o += [torch.empty(M, 520, device=DEV, dtype=torch.bfloat16) for M in lin]
        o += [torch.empty(257, 1920, device=DEV, dtype=torch.uint8), torch.empty(257, device=DEV)]
        return o

    ref = make_outs()
    chain(ref)                 # eager; also fills the library's per-kernel caches before capture
    torch.cuda.synchronize()
    got = make_outs()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="relaxed"):
        chain(got)
    for _ in range(3):
        for t in got:
            t.zero_()
        graph.replay()
        torch.cuda.synchronize()
        for a, b in zip(got, ref):
            assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
    del graph
    ck.device_error_check()


def test_back_to_back_dependent_gemvs(ck):
    """A chain of GEMVs where each call reads the previous call's output, launched back to back:
    every activation read must see the previous kernel's writes."""
    K = N = 1024
    g = torch.Generator().manual_seed(77)
    x0 = WL.activations(2, K, 0, g)
    layers = []
    for _ in range(4):
        qw = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.uint8)
        ws_ = WL.uniform((K // 64, N), 0.001, 0.01, g)
        wz = (torch.randn((K // 64, N), generator=g) * 0.01).to(torch.bfloat16)
        layers.append((qw.to(DEV), ws_.to(DEV), wz.to(DEV)))
    # chained without syncs
    y = x0.to(DEV)
    for qw, ws_, wz in layers:
        y = ck.gemv_awq_w4a16(y, qw, ws_, wz, group_size=64)
    torch.cuda.synchronize()
    chained = y.clone()
    # the same chain with a sync after every call
    y = x0.to(DEV)
    for qw, ws_, wz in layers:
        y = ck.gemv_awq_w4a16(y, qw, ws_, wz, group_size=64)
        torch.cuda.synchronize()
    assert torch.equal(chained.view(torch.int16), y.view(torch.int16))
    # and the W4A8 GEMV reading codes that rotate_quant_rowwise (G = 1, int8) writes just before
    wp = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.uint8).to(DEV)
    sw = WL.uniform((N,), 0.005, 0.02, g).to(DEV)
    xs = [WL.activations(4, K, 0, g).to(DEV) for _ in range(3)]
    outs = []
    for xx in xs:
        xq, xsc = ck.rotate_quant_rowwise(xx, 1, 8)
        outs.append(ck.gemv_w4a8(xq, xsc, wp, sw))
    torch.cuda.synchronize()
    for xx, o in zip(xs, outs):
        xq, xsc = ck.rotate_quant_rowwise(xx, 1, 8)
        torch.cuda.synchronize()
        r = ck.gemv_w4a8(xq, xsc, wp, sw)
        torch.cuda.synchronize()
        assert torch.equal(o.view(torch.int16), r.view(torch.int16))
    ck.device_error_check()
