"""Plain float64 / integer restatement of the ConvRot packed-INT4 linear.

TEST INFRASTRUCTURE ONLY (see the package docstring): the product path never
imports this module.

Sources (page title, then the section or symbol each function follows):

* [RQ]  comfy-kitchen PR #155 "[Feat][Ascend] Add fused RotateQuant backend",
        "What this PR does": ``quantize_and_rotate_rowwise`` = group rotation
        followed by rowwise dynamic quantization with a positive scale;
        "How was this patch tested?": group sizes 16/64/256, all-zero rows,
        batched and non-contiguous inputs.
* [AWQ] ``comfy_kitchen/tensor/awq_w4a16.py``: module docstring (packed
        layout: bits 0..3 -> column 2j, bits 4..7 -> column 2j+1, uint4 in
        [0, 15]) and ``TensorCoreAWQW4A16Layout.dequantize`` /
        ``_awq_forward`` (W = (q - 8) * wscales[k // G, n] + wzeros[k // G, n],
        y = x W^T + bias).
* [W4A8] comfy-kitchen PR #182 "HIP port of #176: W4A8 decode GEMV and fused
        GatedDeltaNet decode", Description: int4 weight decode, int8 dot
        products with int32 accumulation and the rowwise ``EpiRowwise``
        epilogue shared by every path.
* [SD]  stable-diffusion.cpp PR #2276 "feat: support packed INT4 convrot
        models", Summary: ``convrot_w4a4`` and ``asym_w4a8_int8`` packed
        formats, group-size-64 ConvRot quantization.

Readings where the pages are silent:

* Rotation: orthonormal Sylvester Hadamard H_G / sqrt(G) applied to each
  contiguous group of G columns, y_g = x_g @ H; G = 1 is the identity
  (rowwise quantization without rotation).
* Scale: s = float32(amax / qmax) from the float64 amax of the rotated row;
  an all-zero row gets s = 1 (positive-scale contract). qmax = 7 (int4) or
  127 (int8); the range is symmetric, -8 / -128 never occur.
* Rounding: round half to even of y / s (float64 division), then clamp.
* Codec: offset binary, nibble u = q + 8, low nibble = even column, for
  weights and int4 activations alike.
* Tensor-wise input scale: a caller-supplied scalar a >= 0 multiplies x
  before the rotation ([SD] review comments on docs/int8_convrot.md: inputs
  whose scale is not 1 are scaled, then quantized; [RQ] "How was this patch
  tested?": caller-provided zero tensor-wise scales follow eager
  quantization). So a = 0 makes every row all-zero: s = 1, q = 0.
* Epilogue: float32 ((float(acc) * s_m) * sw_n) (+ bias_n), each product
  rounded to float32, then round-to-nearest-even to bfloat16.
"""

from __future__ import annotations

import numpy as np

QMAX = {4: 7, 8: 127}


# --------------------------------------------------------------------------
# Hadamard matrices [RQ] (the pages name the rotation, not its constant)
# --------------------------------------------------------------------------

def _check_pow2(G: int) -> None:
    if G < 1 or (G & (G - 1)) != 0:
        raise ValueError(f"group size must be a power of two, got {G}")


def hadamard_sylvester(G: int) -> np.ndarray:
    """Orthonormal Hadamard matrix of order G by Sylvester's doubling.

    H_1 = [1]; H_2n = [[H_n, H_n], [H_n, -H_n]]; returned as H_G / sqrt(G).
    """
    _check_pow2(G)
    H = np.ones((1, 1), dtype=np.float64)
    while H.shape[0] < G:
        H = np.block([[H, H], [H, -H]])
    return H / np.sqrt(float(G))


def hadamard_closed_form(G: int) -> np.ndarray:
    """Same matrix from its closed form H[i, j] = (-1)^popcount(i & j) / sqrt(G)."""
    _check_pow2(G)
    H = np.empty((G, G), dtype=np.float64)
    for i in range(G):
        for j in range(G):
            H[i, j] = -1.0 if bin(i & j).count("1") % 2 else 1.0
    return H / np.sqrt(float(G))


# --------------------------------------------------------------------------
# a1: group rotation [RQ]
# --------------------------------------------------------------------------

def rotate_groups(x, G: int, R=None) -> np.ndarray:
    """y[m, g*G:(g+1)*G] = x[m, g*G:(g+1)*G] @ R for every group g of every row.

    ``R`` defaults to the orthonormal Sylvester Hadamard matrix of order G; any
    G x G matrix may be given (the pages test "asymmetric-rotation inputs").
    """
    x = np.asarray(x, dtype=np.float64)
    M, K = x.shape
    if K % G != 0:
        raise ValueError(f"K={K} is not a multiple of G={G}")
    R = hadamard_sylvester(G) if R is None else np.asarray(R, dtype=np.float64)
    if R.shape != (G, G):
        raise ValueError("R must be G x G")
    return (x.reshape(M, K // G, G) @ R).reshape(M, K)


# --------------------------------------------------------------------------
# a2 + a3: rowwise symmetric quantization [RQ]
# --------------------------------------------------------------------------

def quantize_rowwise(y, bits: int):
    """Per-row symmetric quantization of an already rotated matrix.

    Returns (q, s): q int64 (M, K) in [-qmax, qmax], s float32 (M,) > 0.
    s = float32(max_k |y[m, k]| / qmax), or 1 for an all-zero row;
    q = clamp(round_half_even(y / s), -qmax, qmax).
    """
    y = np.asarray(y, dtype=np.float64)
    qmax = QMAX[bits]
    M, K = y.shape
    amax = np.abs(y).max(axis=1) if K > 0 else np.zeros(M)
    s = (amax / qmax).astype(np.float32)
    s[amax == 0.0] = np.float32(1.0)
    q = np.rint(y / s.astype(np.float64)[:, None])
    q = np.clip(q, -qmax, qmax).astype(np.int64)
    return q, s


def _check_input_scale(input_scale) -> float:
    a = float(input_scale)
    if not np.isfinite(a) or a < 0.0:
        raise ValueError(f"input_scale={input_scale!r} must be finite and >= 0")
    return a


def rotate_quant_rowwise(x, G: int, bits: int, R=None, input_scale=1.0):
    """``quantize_and_rotate_rowwise``: rotation a1 then quantization a2-a3.

    ``input_scale`` is the caller's tensor-wise scale a: the rotated and
    quantized matrix is that of a * x (the product taken in float64).
    """
    a = _check_input_scale(input_scale)
    x = np.asarray(x, dtype=np.float64)
    return quantize_rowwise(rotate_groups(a * x, G, R), bits)


# --------------------------------------------------------------------------
# Packed uint4 codec [AWQ docstring], offset binary for signed values
# --------------------------------------------------------------------------

def nibbles_u4(packed) -> np.ndarray:
    """(R, C/2) bytes -> (R, C) uint4 values: bits 0..3 -> column 2j, bits 4..7 -> 2j+1."""
    b = np.asarray(packed).astype(np.uint8)
    R, Ch = b.shape
    u = np.empty((R, 2 * Ch), dtype=np.int64)
    u[:, 0::2] = b & 0x0F
    u[:, 1::2] = (b >> 4) & 0x0F
    return u


def unpack_nibbles(packed) -> np.ndarray:
    """Signed values q = u - 8 in [-8, 7] of a packed (R, C/2) byte matrix."""
    return nibbles_u4(packed) - 8


def pack_nibbles(q) -> np.ndarray:
    """(R, C) signed values in [-8, 7] -> (R, C/2) uint8 with u = q + 8."""
    q = np.asarray(q, dtype=np.int64)
    if q.shape[1] % 2:
        raise ValueError("column count must be even")
    if q.size and (q.min() < -8 or q.max() > 7):
        raise ValueError("values outside [-8, 7]")
    u = (q + 8).astype(np.uint8)
    return (u[:, 0::2] | (u[:, 1::2] << 4)).astype(np.uint8)


# --------------------------------------------------------------------------
# a5: integer matmul [W4A8]
# --------------------------------------------------------------------------

def int_matmul(qa, qw) -> np.ndarray:
    """acc[m, n] = sum_k qa[m, k] * qw[n, k], exact, returned as int64.

    The products and partial sums are integers far below 2**53, so a float64
    matmul (any summation order) returns them exactly; the bound is checked.
    """
    qa = np.asarray(qa, dtype=np.int64)
    qw = np.asarray(qw, dtype=np.int64)
    K = qa.shape[1]
    if qw.shape[1] != K:
        raise ValueError("inner dimensions differ")
    bound = K * max(int(np.abs(qa).max(initial=0)), 1) * max(int(np.abs(qw).max(initial=0)), 1)
    if bound >= 2 ** 53:
        raise OverflowError("accumulator bound exceeds exact float64 range")
    acc = qa.astype(np.float64) @ qw.astype(np.float64).T
    acc = acc.astype(np.int64)
    if acc.size and np.abs(acc).max() >= 2 ** 31:
        raise OverflowError("accumulator leaves int32")
    return acc


# --------------------------------------------------------------------------
# a6: rowwise-scale epilogue and bf16 rounding [W4A8 EpiRowwise]
# --------------------------------------------------------------------------

def epilogue_rowwise(acc, s_m, sw_n, bias=None) -> np.ndarray:
    """float32 value of ((float(acc) * s_m) * sw_n) (+ bias_n), before bf16 rounding."""
    t = np.asarray(acc).astype(np.float32)
    t = t * np.asarray(s_m, dtype=np.float32)[:, None]
    t = t * np.asarray(sw_n, dtype=np.float32)[None, :]
    if bias is not None:
        t = t + np.asarray(bias, dtype=np.float32)[None, :]
    return t


def to_bf16_bits(v) -> np.ndarray:
    """Round float64/float32 values to bfloat16 (nearest, ties to even); uint16 bits.

    bfloat16 keeps 8 significant bits and float32's exponent range: the value is
    rounded to a multiple of its quantum 2^(e-8) (v = m 2^e, 0.5 <= |m| < 1),
    with the quantum fixed at 2^-133 below the normal range.
    """
    v = np.asarray(v, dtype=np.float64)
    _, e = np.frexp(v)
    e = np.maximum(e, -125)
    quantum = np.ldexp(np.ones_like(v), e - 8)
    r = np.rint(v / quantum) * quantum
    if not np.all(np.isfinite(r)) or np.abs(r).max(initial=0.0) > 3.3895313892515355e38:
        raise OverflowError("value outside the bfloat16 range")
    return (r.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)


def bf16_bits_to_f64(b) -> np.ndarray:
    """Exact float64 value of bfloat16 bit patterns."""
    b = np.asarray(b).astype(np.uint32)
    return (b << 16).view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------
# Composite paths
# --------------------------------------------------------------------------

def linear_w4a4(x, w_packed, w_scale, G: int, bias=None, R=None, input_scale=1.0) -> dict:
    """ConvRot W4A4 linear: rotate + int4 quantize x, int matmul with the
    packed int4 weight, rowwise-scale epilogue to bf16.

    With a tensor-wise ``input_scale`` a, the linear of a * x (the input is
    scaled, then quantized; the output is not rescaled).

    Returns every intermediate: ``q`` (M, K) int, ``qa_packed`` (M, K/2) u8,
    ``s`` (M,) float32, ``acc`` (M, N) int64, ``y_f32`` and ``y_bits`` (bf16).
    """
    q, s = rotate_quant_rowwise(x, G, 4, R, input_scale)
    acc = int_matmul(q, unpack_nibbles(w_packed))
    y32 = epilogue_rowwise(acc, s, w_scale, bias)
    return {"q": q, "qa_packed": pack_nibbles(q), "s": s, "acc": acc,
            "y_f32": y32, "y_bits": to_bf16_bits(y32)}


def linear_w4a8(x, w_packed, w_scale, G: int, bias=None) -> dict:
    """ConvRot W4A8 linear ([SD] Summary, ``asym_w4a8_int8``: int4 weights against int8
    activations): rotate + int8 quantize x (qmax 127), int matmul with the packed int4 weight,
    the same rowwise-scale epilogue to bf16.

    Returns ``q`` (M, K) int, ``s`` (M,) float32, ``acc`` (M, N) int64, ``y_f32`` and ``y_bits``.
    """
    q, s = rotate_quant_rowwise(x, G, 8)
    acc = int_matmul(q, unpack_nibbles(w_packed))
    y32 = epilogue_rowwise(acc, s, w_scale, bias)
    return {"q": q, "s": s, "acc": acc, "y_f32": y32, "y_bits": to_bf16_bits(y32)}


def gemv_w4a8(xq, x_scale, w_packed, w_scale, bias=None) -> dict:
    """W4A8 decode: int8 activations x int4 packed weights, same epilogue."""
    acc = int_matmul(xq, unpack_nibbles(w_packed))
    y32 = epilogue_rowwise(acc, x_scale, w_scale, bias)
    return {"acc": acc, "y_f32": y32, "y_bits": to_bf16_bits(y32)}


def awq_dequantize(qweight, wscales, wzeros, G: int) -> np.ndarray:
    """W[n, k] = (u[n, k] - 8) * wscales[k // G, n] + wzeros[k // G, n], float64."""
    u = nibbles_u4(qweight)
    N, K = u.shape
    if K % G:
        raise ValueError("K must be a multiple of G")
    s = np.asarray(wscales, dtype=np.float64)
    z = np.asarray(wzeros, dtype=np.float64)
    if s.shape != (K // G, N) or z.shape != (K // G, N):
        raise ValueError("wscales / wzeros must be (K // G, N)")
    grp = np.arange(K) // G
    return (u - 8.0) * s[grp, :].T + z[grp, :].T


def gemv_awq_w4a16(x, qweight, wscales, wzeros, G: int, bias=None) -> dict:
    """y = x W^T (+ bias) with W from ``awq_dequantize``; float64, then bf16."""
    W = awq_dequantize(qweight, wscales, wzeros, G)
    y = np.asarray(x, dtype=np.float64) @ W.T
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[None, :]
    return {"y_f64": y, "y_bits": to_bf16_bits(y)}
