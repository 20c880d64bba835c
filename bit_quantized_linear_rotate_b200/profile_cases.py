"""Runs one kernel case a few times on cuda:0, for profiler captures.

    python -m bit_quantized_linear_rotate_b200.profile_cases CASE [--iters N]

Cases (full workload sizes, a few GB at most on the device):
  rq_M8192         ck_rotate_quant_rowwise_i8, x 8192 x 3840 bf16, G=64, int4 codes
  rq_M8192_K10240_G16   ck_rotate_quant_rowwise, 8192 x 10240, G=16, bits=8
  gemm_w4a8_M8192  ck_gemm_w4a8, int8 codes 8192 x 3840 x packed weights 3840 x 1920
  gemm_s8_M8192    ck_gemm_s8 with pre-decoded int8 weights
  gemm_w4a4_M8192  ck_gemm_w4a4, packed int4 activations and weights
  linear_M8192     ck_linear_w4a4 (both kernels)
  linear_M32       ck_linear_w4a4 at M=32, K=N=3840 (the small-batch route)
  linmm_M8192      ck_linear_w4a4_matmul (the linear's GEMM phase alone)
  linq_M8192       ck_linear_w4a4_quantize (the linear's rotate + quantize phase alone)
  w4a8_M{1,4,16}   ck_gemv_w4a8, K=4096, N=12288
  w4a8tc_M{1,4,16} ck_gemv_w4a8_tc (the tcgen05 alternative), same shapes
  awq_M{1,2,4}     ck_gemv_awq_w4a16, K=3072, N=18432, G=64
One warm-up call precedes the timed iterations; the process exits non-zero if
a kernel reported an error.
"""

from __future__ import annotations

import argparse

import torch

from . import ck
from . import workloads as WL


def build_case(name: str, dev):
    if name.startswith(("rq_", "gemm_", "lin")):
        w = WL.LINEAR_M32 if name == "linear_M32" else WL.LINEAR_M8192
        if name == "rq_M8192_K10240_G16":
            x = WL.linear_inputs(WL.LINEAR_MLP_DOWN)["x"].to(dev)
            return lambda: ck.rotate_quant_rowwise(x, 16, 8)
        d = WL.linear_inputs(w)
        x, wp, sw = d["x"].to(dev), d["w_packed"].to(dev), d["w_scale"].to(dev)
        y = torch.empty(w.M, w.N, device=dev, dtype=torch.bfloat16)
        if name.startswith(("rq_", "gemm_")):   # setup launches only where the case needs them
            qa, sa = ck.rotate_quant_rowwise_i8(x, w.G, 4)
        if name == "rq_M8192":
            return lambda: ck.rotate_quant_rowwise_i8(x, w.G, 4, q_out=qa, scale_out=sa)
        if name == "gemm_w4a8_M8192":
            return lambda: ck.gemm_w4a8(qa, sa, wp, sw, out=y)
        if name == "gemm_s8_M8192":
            w8 = ck.unpack_int4(wp)
            return lambda: ck.gemm_s8(qa, sa, w8, sw, out=y)
        if name == "gemm_w4a4_M8192":
            qp, _ = ck.rotate_quant_rowwise(x, w.G, 4)
            return lambda: ck.gemm_w4a4(qp, sa, wp, sw, out=y)
        ws = torch.empty(ck.linear_w4a4_workspace_bytes(w.M, w.K), device=dev, dtype=torch.uint8)
        if name in ("linear_M8192", "linear_M32"):
            return lambda: ck.linear_w4a4(x, wp, sw, w.G, workspace=ws, out=y)
        if name == "linq_M8192":
            return lambda: ck.linear_w4a4_quantize(x, w.G, ws)
        if name == "linmm_M8192":
            ck.linear_w4a4_quantize(x, w.G, ws)
            return lambda: ck.linear_w4a4_matmul(w.M, w.K, wp, sw, ws, out=y)
    if name.startswith(("w4a8_M", "w4a8tc_M")):
        tc = name.startswith("w4a8tc_M")
        M = int(name[len("w4a8tc_M" if tc else "w4a8_M"):])
        d = WL.gemv_w4a8_inputs(WL.GEMV_W4A8, M)
        xq, xs = ck.rotate_quant_rowwise(d["x"].to(dev), 1, 8)
        wp, sw = d["w_packed"].to(dev), d["w_scale"].to(dev)
        y = torch.empty(M, WL.GEMV_W4A8.N, device=dev, dtype=torch.bfloat16)
        if tc:
            return lambda: ck.gemv_w4a8_tc(xq, xs, wp, sw, out=y)
        return lambda: ck.gemv_w4a8(xq, xs, wp, sw, out=y)
    if name.startswith("awq_M"):
        M = int(name[len("awq_M"):])
        w = WL.GEMV_AWQ
        d = WL.gemv_awq_inputs(w, M)
        t = {k: v.to(dev) for k, v in d.items()}
        y = torch.empty(M, w.N, device=dev, dtype=torch.bfloat16)
        return lambda: ck.gemv_awq_w4a16(t["x"], t["qweight"], t["wscales"], t["wzeros"], group_size=w.G, out=y)
    raise SystemExit(f"unknown case {name}")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("case")
    ap.add_argument("--iters", type=int, default=3)
    a = ap.parse_args()
    dev = torch.device("cuda:0")
    fn = build_case(a.case, dev)
    fn()
    ck.device_error_check()
    for _ in range(a.iters):
        fn()
    ck.device_error_check()
    print(f"{a.case}: ok")


if __name__ == "__main__":
    main()
