"""Pins of the CPU oracle against things other than itself.

Closed forms, invariants, brute force on tiny inputs, a library routine for
bf16 rounding, and hand-worked fixtures under tests/golden/ (each carrying the
page and section it restates). A plausible slip in the oracle (a transposed
rotation, a wrong nibble order, a dropped "- 8", swapped scale indices, a
wrong tie rule) fails at least one test here.
"""

import json
import os

import numpy as np
import pytest
import torch

import oracle as O

pytestmark = pytest.mark.filterwarnings("ignore")


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- rotation

@pytest.mark.parametrize("G", [1, 2, 4, 8, 16, 32, 64, 128, 256])
def test_two_hadamard_constructions_agree(G):
    np.testing.assert_array_equal(O.hadamard_sylvester(G), O.hadamard_closed_form(G))


@pytest.mark.parametrize("G", [16, 64, 256])
def test_hadamard_orthonormal_symmetric_involutory(G):
    H = O.hadamard_sylvester(G)
    I = np.eye(G)
    np.testing.assert_allclose(H @ H.T, I, atol=1e-12)
    np.testing.assert_array_equal(H, H.T)
    np.testing.assert_allclose(H @ H, I, atol=1e-12)
    # first row and column are all +1/sqrt(G) (natural / Sylvester order)
    np.testing.assert_array_equal(H[0], np.full(G, 1 / np.sqrt(G)))


@pytest.mark.parametrize("G", [16, 64, 256])
def test_rotation_preserves_each_group_norm(G):
    rng = np.random.default_rng(G)
    x = rng.standard_normal((5, 4 * G))
    y = O.rotate_groups(x, G)
    nx = np.linalg.norm(x.reshape(5, 4, G), axis=2)
    ny = np.linalg.norm(y.reshape(5, 4, G), axis=2)
    np.testing.assert_allclose(ny, nx, rtol=1e-13)
    # groups do not mix: rotating one group leaves the others at zero
    x2 = np.zeros_like(x)
    x2[:, G:2 * G] = x[:, G:2 * G]
    y2 = O.rotate_groups(x2, G)
    assert np.all(y2[:, :G] == 0) and np.all(y2[:, 2 * G:] == 0)


def test_rotation_golden(golden_dir):
    d = _load(golden_dir, "rotate_quant_hand.json")
    r = d["rotation_G4"]
    np.testing.assert_allclose(O.rotate_groups(np.array(r["x"]), 4), np.array(r["y"]), atol=1e-15)
    q, s = O.rotate_quant_rowwise(np.array(r["x"]), 4, 4)
    np.testing.assert_array_equal(q, np.array(r["q_int4"]))
    assert s[0] == np.float32(5.0 / 7.0)
    g = d["rotation_G2_general_R"]
    np.testing.assert_array_equal(O.rotate_groups(np.array(g["x"]), 2, np.array(g["R"])), np.array(g["y"]))


def test_rotation_G1_is_identity():
    x = np.random.default_rng(0).standard_normal((3, 10))
    np.testing.assert_array_equal(O.rotate_groups(x, 1), x)


@pytest.mark.parametrize("G,bits", [(16, 4), (64, 4), (256, 4), (16, 8), (64, 8), (256, 8)])
def test_one_hot_rotates_to_walsh_row_at_full_scale(G, bits):
    qmax = O.QMAX[bits]
    for i in (0, 1, G // 2 + 3, G - 1):
        x = np.zeros((1, 2 * G))
        x[0, G + i] = 3.0            # one-hot in the second group
        q, s = O.rotate_quant_rowwise(x, G, bits)
        assert np.all(q[0, :G] == 0)
        # y_j = 3 * (-1)^{<i, j>} / sqrt(G): every |y| equals the amax
        signs = np.array([(-1) ** bin(i & j).count("1") for j in range(G)])
        np.testing.assert_array_equal(q[0, G:], qmax * signs)
        assert s[0] == np.float32(3.0 / np.sqrt(G) / qmax)


@pytest.mark.parametrize("G,bits", [(16, 4), (64, 8), (256, 4)])
def test_constant_group_rotates_to_first_coordinate(G, bits):
    qmax = O.QMAX[bits]
    x = np.full((2, G), -1.5)
    x[1] = 0.75
    y = O.rotate_groups(x, G)
    np.testing.assert_allclose(y[:, 0], x[:, 0] * np.sqrt(G), rtol=1e-15)
    np.testing.assert_allclose(y[:, 1:], 0.0, atol=1e-14)
    q, _ = O.quantize_rowwise(y, bits)
    np.testing.assert_array_equal(q[:, 0], [-qmax, qmax])
    assert np.all(q[:, 1:] == 0)


@pytest.mark.parametrize("G", [16, 64, 256])
def test_groupwise_rotation_leaves_the_product_unchanged(G):
    # x W^T = (x H)(W H)^T blockwise, because H H^T = I; fails for x H^T vs x H
    # mixups only with a non-symmetric R, checked right after.
    rng = np.random.default_rng(7)
    K = 3 * G
    x = rng.standard_normal((4, K))
    W = rng.standard_normal((5, K))
    np.testing.assert_allclose(O.rotate_groups(x, G) @ O.rotate_groups(W, G).T, x @ W.T,
                               rtol=1e-11, atol=1e-11)
    Q, _ = np.linalg.qr(rng.standard_normal((G, G)))      # orthogonal, not symmetric
    np.testing.assert_allclose(O.rotate_groups(x, G, Q) @ O.rotate_groups(W, G, Q).T, x @ W.T,
                               rtol=1e-11, atol=1e-11)


# ------------------------------------------------------------ quantization

def test_quantize_ties_and_zero_row(golden_dir):
    d = _load(golden_dir, "rotate_quant_hand.json")
    for key, bits in (("quantize_ties_int4", 4), ("quantize_ties_int8", 8), ("quantize_zero_row", 4)):
        c = d[key]
        q, s = O.quantize_rowwise(np.array(c["y"]), bits)
        np.testing.assert_array_equal(q, np.array(c["q"]))
        np.testing.assert_array_equal(s, np.array(c["s"], dtype=np.float32))


def test_quantize_range_scale_and_clamp():
    rng = np.random.default_rng(3)
    y = rng.standard_normal((50, 64)) * rng.uniform(0.01, 100, size=(50, 1))
    for bits in (4, 8):
        qmax = O.QMAX[bits]
        q, s = O.quantize_rowwise(y, bits)
        assert q.min() >= -qmax and q.max() <= qmax
        assert np.all(s > 0)
        # the row maximum lands exactly on +-qmax
        idx = np.abs(y).argmax(axis=1)
        np.testing.assert_array_equal(np.abs(q[np.arange(50), idx]), qmax)
        # reconstruction error at most half a step (plus float32 scale rounding)
        err = np.abs(q * s.astype(np.float64)[:, None] - y)
        assert np.all(err <= 0.5 * s[:, None] * (1 + 1e-6))


def test_all_zero_rows_give_unit_scale_and_zero_output():
    x = np.zeros((3, 128))
    x[1, 5] = 2.0
    q, s = O.rotate_quant_rowwise(x, 64, 4)
    assert s[0] == 1.0 and s[2] == 1.0 and np.all(q[0] == 0) and np.all(q[2] == 0)
    wp = np.random.default_rng(1).integers(0, 256, size=(6, 64), dtype=np.uint8)
    bias = np.array([0.5, -0.25, 0, 1, 2, 3], dtype=np.float32)
    r = O.linear_w4a4(x, wp, np.full(6, 0.01, dtype=np.float32), 64, bias=bias)
    assert np.all(np.isfinite(r["y_f32"]))
    np.testing.assert_array_equal(r["y_f32"][0], bias)
    np.testing.assert_array_equal(r["y_f32"][2], bias)


# ------------------------------------------------- tensor-wise input scale

@pytest.mark.parametrize("G,bits", [(16, 4), (64, 8), (256, 4)])
def test_zero_input_scale_quantizes_like_all_zero_rows(G, bits):
    # a = 0 scales every row to zero: the positive-scale contract gives s = 1, q = 0
    x = np.random.default_rng(11).standard_normal((5, 2 * G)) * 40
    q, s = O.rotate_quant_rowwise(x, G, bits, input_scale=0.0)
    assert np.all(q == 0)
    np.testing.assert_array_equal(s, np.ones(5, dtype=np.float32))
    bias = np.linspace(-1, 1, 7).astype(np.float32)
    wp = np.random.default_rng(2).integers(0, 256, size=(7, G), dtype=np.uint8)
    r = O.linear_w4a4(x, wp, np.full(7, 0.01, dtype=np.float32), G, bias=bias, input_scale=0.0)
    np.testing.assert_array_equal(r["y_f32"], np.broadcast_to(bias, (5, 7)))


@pytest.mark.parametrize("G,bits", [(16, 4), (64, 8)])
def test_input_scale_multiplies_the_one_hot_amplitude(G, bits):
    # one-hot 3 scaled by a = 5: every rotated entry is +-15 / sqrt(G), so
    # s = 15 / sqrt(G) / qmax (dividing by a, or ignoring it, gives another s)
    qmax = O.QMAX[bits]
    i = G // 2 + 1
    x = np.zeros((1, G))
    x[0, i] = 3.0
    q, s = O.rotate_quant_rowwise(x, G, bits, input_scale=5.0)
    signs = np.array([(-1) ** bin(i & j).count("1") for j in range(G)])
    np.testing.assert_array_equal(q[0], qmax * signs)
    assert s[0] == np.float32(15.0 / np.sqrt(G) / qmax)


@pytest.mark.parametrize("k", [-6, -1, 3, 10])
def test_power_of_two_input_scale_keeps_codes_and_scales_s(k):
    # scaling by 2^k is exact in binary floating point: the codes are those of
    # x and every scale (and unbiased output) is 2^k times the unscaled one
    rng = np.random.default_rng(5)
    x = rng.standard_normal((6, 128)) * rng.uniform(0.1, 10, size=(6, 1))
    a = 2.0 ** k
    for bits in (4, 8):
        q1, s1 = O.rotate_quant_rowwise(x, 64, bits)
        qa, sa = O.rotate_quant_rowwise(x, 64, bits, input_scale=a)
        np.testing.assert_array_equal(qa, q1)
        np.testing.assert_array_equal(sa, (s1 * np.float32(a)).astype(np.float32))
    wp = rng.integers(0, 256, size=(9, 64), dtype=np.uint8)
    sw = rng.uniform(0.005, 0.02, size=9).astype(np.float32)
    r1 = O.linear_w4a4(x, wp, sw, 64)
    ra = O.linear_w4a4(x, wp, sw, 64, input_scale=a)
    np.testing.assert_array_equal(ra["acc"], r1["acc"])
    np.testing.assert_array_equal(ra["y_f32"], (r1["y_f32"] * np.float32(a)).astype(np.float32))


def test_general_input_scale_stays_within_half_a_step_of_the_scaled_rotation():
    rng = np.random.default_rng(8)
    x = rng.standard_normal((10, 256))
    a = 0.3712
    y = O.rotate_groups(a * x, 64)
    q, s = O.rotate_quant_rowwise(x, 64, 4, input_scale=a)
    err = np.abs(q * s.astype(np.float64)[:, None] - y)
    assert np.all(err <= 0.5 * s[:, None] * (1 + 1e-6))
    np.testing.assert_array_equal(np.abs(q).max(axis=1), 7)


@pytest.mark.parametrize("a", [-1.0, -0.0 - 1e-30, float("nan"), float("inf")])
def test_input_scale_must_be_finite_and_nonnegative(a):
    with pytest.raises(ValueError):
        O.rotate_quant_rowwise(np.ones((1, 16)), 16, 4, input_scale=a)


# -------------------------------------------------------------------- codec

def test_codec_golden(golden_dir):
    d = _load(golden_dir, "codec_hand.json")
    b = np.array(d["packed"], dtype=np.uint8)
    np.testing.assert_array_equal(O.unpack_nibbles(b) + 8, np.array(d["u4"]))
    np.testing.assert_array_equal(O.unpack_nibbles(b), np.array(d["signed"]))
    np.testing.assert_array_equal(O.pack_nibbles(np.array(d["signed"])), b)


def test_codec_round_trips_every_byte():
    b = np.arange(256, dtype=np.uint8).reshape(1, 256)
    q = O.unpack_nibbles(b)
    assert q.min() == -8 and q.max() == 7
    np.testing.assert_array_equal(O.pack_nibbles(q), b)
    # low nibble is the even column
    np.testing.assert_array_equal(q[0, 0::2] + 8, np.arange(256) & 15)
    np.testing.assert_array_equal(q[0, 1::2] + 8, np.arange(256) >> 4)


# ------------------------------------------------------------------- matmul

def _brute_int(qa, qw):
    M, K = len(qa), len(qa[0])
    N = len(qw)
    out = [[0] * N for _ in range(M)]
    for m in range(M):
        for n in range(N):
            acc = 0
            for k in range(K):
                acc += int(qa[m][k]) * int(qw[n][k])
            out[m][n] = acc
    return np.array(out, dtype=np.int64)


@pytest.mark.parametrize("M,N,K", [(1, 1, 2), (3, 5, 16), (7, 4, 64), (64, 33, 64)])
def test_int_matmul_matches_brute_force(M, N, K):
    rng = np.random.default_rng(M * 100 + N)
    qa = rng.integers(-127, 128, size=(M, K))
    qw = rng.integers(-8, 8, size=(N, K))
    np.testing.assert_array_equal(O.int_matmul(qa, qw), _brute_int(qa.tolist(), qw.tolist()))
    # asymmetric shapes: acc[m, n] uses row m of qa and row n of qw
    acc = O.int_matmul(qa, qw)
    assert acc.shape == (M, N)
    if M > 1 and N > 1:
        assert acc[0, 1] == int(np.dot(qa[0], qw[1]))


@pytest.mark.parametrize("K", [64, 3840, 10240])
def test_int_matmul_extreme_operands(K):
    a7 = np.full((1, K), 7)
    w_8 = np.full((1, K), -8)
    assert O.int_matmul(a7, w_8)[0, 0] == -8 * 7 * K
    assert O.int_matmul(a7, np.full((1, K), 7))[0, 0] == 49 * K
    assert O.int_matmul(np.full((1, K), -127), w_8)[0, 0] == 1016 * K


# ------------------------------------------------------------------ epilogue

def test_epilogue_golden(golden_dir):
    d = _load(golden_dir, "epilogue_hand.json")
    acc = np.array(d["acc"])
    t = O.epilogue_rowwise(acc, d["s_m"], d["sw_n"])
    np.testing.assert_array_equal(t, np.array(d["y_no_bias"], dtype=np.float32))
    t = O.epilogue_rowwise(acc, d["s_m"], d["sw_n"], d["bias"])
    np.testing.assert_array_equal(t, np.array(d["y_bias"], dtype=np.float32))
    c = d["bf16_round_cases"]
    np.testing.assert_array_equal(O.to_bf16_bits(np.array(c["values"])), np.array(c["bits"], dtype=np.uint16))
    assert O.to_bf16_bits(O.epilogue_rowwise(np.array([[1]]), [1.0], [1.0]))[0, 0] == 0x3F80


def test_bf16_rounding_matches_library_on_float32_values():
    rng = np.random.default_rng(11)
    v = np.concatenate([rng.standard_normal(20000).astype(np.float32) * 10,
                        (rng.standard_normal(2000) * 1e-30).astype(np.float32),
                        np.float32(1.0) + np.arange(-300, 300, dtype=np.float32) * np.float32(2 ** -9)])
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    np.testing.assert_array_equal(O.to_bf16_bits(v), ref)
    np.testing.assert_array_equal(O.bf16_bits_to_f64(ref), torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).double().numpy())


def test_bf16_rounding_from_float64_rounds_once():
    # 1 + 2^-8 + 2^-40: above the tie in float64, exactly the tie after a float32 detour
    v = 1.0 + 2.0 ** -8 + 2.0 ** -40
    assert O.to_bf16_bits(np.array([v]))[0] == 0x3F81


# ---------------------------------------------------------------------- AWQ

def test_awq_golden(golden_dir):
    d = _load(golden_dir, "awq_dequant_hand.json")
    W = O.awq_dequantize(np.array(d["qweight"], dtype=np.uint8), d["wscales"], d["wzeros"], d["G"])
    np.testing.assert_array_equal(W, np.array(d["W"]))
    r = O.gemv_awq_w4a16(np.array(d["x"]), np.array(d["qweight"], dtype=np.uint8), d["wscales"], d["wzeros"], d["G"])
    np.testing.assert_array_equal(r["y_f64"], np.array(d["y_no_bias"]))
    r = O.gemv_awq_w4a16(np.array(d["x"]), np.array(d["qweight"], dtype=np.uint8), d["wscales"], d["wzeros"], d["G"],
                         bias=np.array(d["bias"]))
    np.testing.assert_array_equal(r["y_f64"], np.array(d["y_bias"]))


def test_awq_special_cases():
    N, K, G = 3, 8, 4
    rng = np.random.default_rng(5)
    z = rng.standard_normal((K // G, N))
    s = rng.uniform(0.1, 1.0, (K // G, N))
    eights = np.full((N, K // 2), 0x88, dtype=np.uint8)          # every nibble = 8
    np.testing.assert_array_equal(O.awq_dequantize(eights, s, z, G), np.repeat(z.T, G, axis=1))
    qb = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    np.testing.assert_array_equal(O.awq_dequantize(qb, np.ones((K // G, N)), np.zeros((K // G, N)), G),
                                  O.unpack_nibbles(qb).astype(np.float64))


def test_awq_gemv_matches_group_algebra():
    # y = sum_g s[g,n] (sum_{k in g} u x - 8 X_g) + z[g,n] X_g, X_g = sum_{k in g} x
    M, N, K, G = 3, 7, 256, 64
    rng = np.random.default_rng(9)
    x = rng.standard_normal((M, K))
    qb = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    s = rng.uniform(0.001, 0.01, (K // G, N))
    z = rng.standard_normal((K // G, N)) * 0.01
    u = np.empty((N, K))
    u[:, 0::2] = qb & 15
    u[:, 1::2] = qb >> 4
    y = np.zeros((M, N))
    for g in range(K // G):
        sl = slice(g * G, (g + 1) * G)
        Xg = x[:, sl].sum(axis=1)[:, None]
        P = x[:, sl] @ u[:, sl].T
        y += s[g][None, :] * (P - 8 * Xg) + z[g][None, :] * Xg
    np.testing.assert_allclose(O.gemv_awq_w4a16(x, qb, s, z, G)["y_f64"], y, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------- composites

def test_w4a8_gemv_composite_small():
    rng = np.random.default_rng(2)
    xq = rng.integers(-127, 128, size=(4, 64))
    xs = rng.uniform(0.01, 0.1, 4).astype(np.float32)
    wp = rng.integers(0, 256, size=(5, 32), dtype=np.uint8)
    sw = rng.uniform(0.005, 0.02, 5).astype(np.float32)
    r = O.gemv_w4a8(xq, xs, wp, sw)
    np.testing.assert_array_equal(r["acc"], _brute_int(xq.tolist(), O.unpack_nibbles(wp).tolist()))
    # the dequantized float product agrees with the epilogue result to float32 rounding
    ref = (xq * xs[:, None].astype(np.float64)) @ (O.unpack_nibbles(wp) * sw[:, None].astype(np.float64)).T
    np.testing.assert_allclose(r["y_f32"], ref, rtol=1e-5, atol=1e-6)


def test_linear_w4a4_approximates_the_float_linear():
    # the stored weight lives in the rotated basis (the rotation is folded into it offline), so the
    # quantized linear tracks (x H)(sw W)^T; int4 activation rounding keeps it within ~15 %
    rng = np.random.default_rng(4)
    M, K, N, G = 8, 256, 16, 64
    x = rng.standard_normal((M, K))
    wp = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    sw = np.full(N, 0.01, dtype=np.float32)
    r = O.linear_w4a4(x, wp, sw, G)
    ref = O.rotate_groups(x, G) @ (O.unpack_nibbles(wp) * 0.01).T
    y = r["y_f32"].astype(np.float64)
    rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert rel < 0.25
    # exact identity on the quantized operands
    np.testing.assert_array_equal(O.unpack_nibbles(r["qa_packed"]), r["q"])


# ------------------------------------------------- W4A8 linear ([SD] asym_w4a8_int8)

def test_linear_w4a8_one_hot_groups_closed_form():
    # a row that is c at the first column of every group rotates to c / sqrt(G) everywhere (the
    # first row of the Sylvester matrix is all ones), so every int8 code is +127; weight bytes
    # 0x00 (all nibbles u = 0, w = -8) and 0xFF (u = 15, w = 7) then give acc = 127 * w * K
    M, K, G, c = 2, 256, 64, 3.0
    x = np.zeros((M, K))
    x[:, ::G] = c
    wp = np.zeros((2, K // 2), dtype=np.uint8)
    wp[1, :] = 0xFF
    sw = np.full(2, 0.01, dtype=np.float32)
    r = O.linear_w4a8(x, wp, sw, G)
    assert np.all(r["q"] == 127)
    np.testing.assert_array_equal(r["acc"], np.array([[-1016 * K, 889 * K]] * M))
    s = c / np.sqrt(G) / 127
    np.testing.assert_allclose(r["s"], s, rtol=2 ** -23)
    y_closed = np.array([-1016 * K * s * 0.01, 889 * K * s * 0.01])
    np.testing.assert_allclose(r["y_f32"], np.tile(y_closed, (M, 1)), rtol=1e-6)


def test_linear_w4a8_within_half_a_code_of_the_float_linear():
    # the stored weight lives in the rotated basis: the exact product is (x H)(sw Wq)^T, and the
    # only error int8 activation rounding adds is at most s_m / 2 per term
    rng = np.random.default_rng(8)
    M, K, N, G = 6, 512, 24, 64
    x = rng.standard_normal((M, K))
    x[:, 5] *= 20
    wp = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    sw = rng.uniform(0.005, 0.02, N).astype(np.float32)
    r = O.linear_w4a8(x, wp, sw, G)
    wq = O.unpack_nibbles(wp).astype(np.float64)
    ref = O.rotate_groups(x, G) @ (wq * sw[:, None].astype(np.float64)).T
    bound = 0.5 * r["s"].astype(np.float64)[:, None] * (np.abs(wq).sum(axis=1) * sw)[None, :]
    err = np.abs(r["y_f32"].astype(np.float64) - ref)
    assert np.all(err <= bound * (1 + 1e-5) + 1e-6 * np.abs(ref))
    # and it is far tighter than the int4 path on the same inputs (the int8 step is 127 / 7 finer)
    r4 = O.linear_w4a4(x, wp, sw, G)
    assert np.linalg.norm(r["y_f32"] - ref) < 0.2 * np.linalg.norm(r4["y_f32"] - ref)


def test_linear_w4a8_brute_force_tiny():
    # every step written out with scalar loops: closed-form Hadamard entries, Python's
    # round-half-even, the offset-binary nibbles and the float32 epilogue products
    rng = np.random.default_rng(9)
    M, K, N, G = 2, 16, 3, 4
    x = rng.standard_normal((M, K)).round(3)
    wp = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    sw = rng.uniform(0.005, 0.02, N).astype(np.float32)
    H = [[(-1) ** bin(i & j).count("1") / G ** 0.5 for j in range(G)] for i in range(G)]
    r = O.linear_w4a8(x, wp, sw, G)
    for m in range(M):
        rot = [sum(x[m, (k // G) * G + i] * H[i][k % G] for i in range(G)) for k in range(K)]
        amax = max(abs(v) for v in rot)
        s = np.float32(amax / 127) if amax > 0 else np.float32(1)
        q = [max(-127, min(127, round(v / float(s)))) for v in rot]
        assert r["q"][m].tolist() == q
        for n in range(N):
            w = [((int(wp[n, k // 2]) >> (4 * (k % 2))) & 0xF) - 8 for k in range(K)]
            acc = sum(qa * wv for qa, wv in zip(q, w))
            assert r["acc"][m, n] == acc
            y = np.float32(np.float32(np.float32(acc) * s) * sw[n])
            assert r["y_f32"][m, n] == y
