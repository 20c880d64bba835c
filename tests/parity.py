"""Comparison rules shared by the GPU parity tests.

* Integer accumulators and packed bytes of identical quantized inputs: bit-exact.
* Quantized activations from the fp32 GPU rotation vs the fp64 oracle: at most
  1 code apart everywhere, and different on at most 0.1 % of the entries
  (rounding ties decided differently).
* Scales: relative difference <= 1e-5.
* bf16 outputs: normwise ||y - y*|| / ||y*|| <= 1e-2 and, per element,
  |y - y*| <= 1e-2 |y*| + 1e-2 rms(y*_row), so cancellation near zero does not
  fail a correct result; where quantized codes differ from the oracle's (the
  one-LSB ties above), the elementwise bound adds the exact output shift those
  codes cause (``code_flip_allowance``).
"""

import numpy as np
import torch

import oracle as O


def to_np_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def bf16_tensor_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def assert_codes_close(q_gpu: np.ndarray, q_ref: np.ndarray, max_frac: float = 1e-3):
    q_gpu = np.asarray(q_gpu, dtype=np.int64)
    q_ref = np.asarray(q_ref, dtype=np.int64)
    assert q_gpu.shape == q_ref.shape
    d = np.abs(q_gpu - q_ref)
    assert d.max(initial=0) <= 1, f"codes differ by {d.max()}"
    frac = float((d != 0).mean()) if d.size else 0.0
    assert frac <= max_frac, f"{frac:.4%} of codes differ (limit {max_frac:.2%})"
    return frac


def assert_scales_close(s_gpu, s_ref, rtol=1e-5):
    s_gpu = np.asarray(s_gpu, dtype=np.float64)
    s_ref = np.asarray(s_ref, dtype=np.float64)
    assert np.all(s_gpu > 0)
    np.testing.assert_allclose(s_gpu, s_ref, rtol=rtol, atol=0)


def assert_out_close(y_gpu: np.ndarray, y_ref: np.ndarray, rel=1e-2, extra=None):
    """Normwise and elementwise output check. ``extra`` (same shape, optional) widens the
    elementwise bound by the exact effect of quantized codes that legitimately differ from the
    oracle's (see ``code_flip_allowance``)."""
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    assert y_gpu.shape == y_ref.shape
    assert np.all(np.isfinite(y_gpu))
    nrm = np.linalg.norm(y_ref)
    err = np.linalg.norm(y_gpu - y_ref)
    assert err <= rel * max(nrm, 1e-30), f"normwise rel err {err / max(nrm, 1e-30):.3e}"
    rms = np.sqrt(np.mean(y_ref ** 2, axis=-1, keepdims=True))
    bound = rel * np.abs(y_ref) + rel * rms
    if extra is not None:
        bound = bound + extra
    bad = np.abs(y_gpu - y_ref) > bound
    assert not bad.any(), f"{int(bad.sum())} elements outside tolerance"
    return err / max(nrm, 1e-30)


def code_flip_allowance(q_gpu, q_ref, w_int, s_row, sw_col):
    """Elementwise effect on y = (acc * s_m) * sw_n of activation codes that differ by one LSB.

    A code of row m that differs by d at column k moves acc[m, n] by d * w[n, k] for every n, so
    y[m, n] by at most s_m * sw_n * sum_k |d_mk| |w[n, k]| (times a small margin for the float32
    and bfloat16 roundings of the shifted value). At int4 this is up to 8 s_m sw_n per flipped
    code, more than 1e-2 rms(y_row) at K in the thousands, so a row with one tie decided the other
    way would fail a bound that ignores it. Returns (allowance (M, N), number of flipped codes)."""
    d = np.abs(np.asarray(q_gpu, dtype=np.int64) - np.asarray(q_ref, dtype=np.int64))
    M = d.shape[0]
    N = w_int.shape[0]
    extra = np.zeros((M, N))
    ms, ks = np.nonzero(d)
    wabs = np.abs(np.asarray(w_int, dtype=np.float64))
    for m, k in zip(ms, ks):
        extra[m] += d[m, k] * wabs[:, k]
    extra *= np.asarray(s_row, dtype=np.float64)[:, None] * np.asarray(sw_col, dtype=np.float64)[None, :]
    return extra * 1.01, len(ms)


def unpack_codes(packed: torch.Tensor) -> np.ndarray:
    return O.unpack_nibbles(packed.cpu().numpy())
