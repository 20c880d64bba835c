"""ck_linear_w4a4_static: the W4A4 linear with the library's own per-device
scratch instead of a caller workspace.

It must give the same output as ck_linear_w4a4 on the same inputs, on
consecutive calls (the second call reuses the scratch the first one wrote),
and refuse problems whose scratch would not fit. The file name keeps it last
in collection so it also runs after everything else has used the device; it
passes on its own as well.
"""

import pytest
import torch

from bit_quantized_linear_rotate_b200 import workloads as WL


@pytest.fixture(scope="module")
def ck():
    from bit_quantized_linear_rotate_b200 import build
    build.build()
    from bit_quantized_linear_rotate_b200 import ck as _ck
    return _ck


def _inputs(M, K, N, seed, dev, with_bias=False):
    d = WL.small_linear_inputs(M, K, N, seed, n_outlier_cols=4, with_bias=with_bias)
    return {k: v.to(dev) for k, v in d.items()}


def test_static_scratch_limit_is_checked_on_the_host(ck):
    # M = 8192, K = 10240 needs ~84 MB of scratch: refused before anything touches a device
    st = ck.lib.ck_linear_w4a4_static(None, 0, 8192, 10240, 3840, 10240, 256, None, None, None, None, None)
    assert st == ck.CK_ERR_UNSUPPORTED
    assert "scratch" in ck.last_error()
    assert ck.linear_w4a4_workspace_bytes(8192, 10240) > ck.LINEAR_STATIC_SCRATCH_BYTES
    assert ck.linear_w4a4_workspace_bytes(8192, 3840) <= ck.LINEAR_STATIC_SCRATCH_BYTES


@pytest.mark.gpu
def test_static_matches_workspace_entry_on_consecutive_calls(ck):
    dev = torch.device("cuda:0")
    cases = [(256, 3840, 3840, 64, 11, False),   # first call: does the set-up
             (97, 1024, 640, 16, 12, True),      # smaller ragged problem over a scratch that holds more
             (8192, 3840, 3840, 64, 13, False)]  # the M = 8192 linear at the scratch's upper range
    for M, K, N, G, seed, bias in cases:
        d = _inputs(M, K, N, seed, dev, with_bias=bias)
        b = d.get("bias")
        ref = ck.linear_w4a4(d["x"], d["w_packed"], d["w_scale"], G, bias=b)
        for _ in range(2):
            y = ck.linear_w4a4_static(d["x"], d["w_packed"], d["w_scale"], G, bias=b)
            torch.cuda.synchronize()
            # same kernels on the same inputs: the tolerance is zero
            assert torch.equal(y.view(torch.int16), ref.view(torch.int16)), (M, K, N, G)
    ck.device_error_check()


@pytest.mark.gpu
def test_static_rejects_oversize_and_keeps_working(ck):
    dev = torch.device("cuda:0")
    d = _inputs(64, 512, 256, 14, dev)
    big = torch.empty(8192, 4608, device=dev, dtype=torch.bfloat16)   # 8192*4608 > 32 MiB of codes
    wbig = torch.empty(128, 2304, device=dev, dtype=torch.uint8)
    sbig = torch.ones(128, device=dev, dtype=torch.bfloat16)
    with pytest.raises(ck.CKError, match="scratch"):
        ck.linear_w4a4_static(big, wbig, sbig, 64)
    y = ck.linear_w4a4_static(d["x"], d["w_packed"], d["w_scale"], 64)
    ref = ck.linear_w4a4(d["x"], d["w_packed"], d["w_scale"], 64)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), ref.view(torch.int16))
    ck.device_error_check()


@pytest.mark.gpu
def test_static_call_allocates_no_device_memory(ck):
    # the entry point's whole claim: with the output preallocated, a call changes neither
    # torch's allocator nor the device's free memory (after the first call's set-up)
    dev = torch.device("cuda:0")
    d = _inputs(512, 3840, 1024, 15, dev, with_bias=True)
    out = torch.empty(512, 1024, device=dev, dtype=torch.bfloat16)
    ck.linear_w4a4_static(d["x"], d["w_packed"], d["w_scale"], 64, bias=d["bias"], out=out)
    torch.cuda.synchronize()
    alloc0 = torch.cuda.memory_allocated(dev)
    free0, _ = torch.cuda.mem_get_info(dev)
    for _ in range(3):
        ck.linear_w4a4_static(d["x"], d["w_packed"], d["w_scale"], 64, bias=d["bias"], out=out)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated(dev) == alloc0
    free1, _ = torch.cuda.mem_get_info(dev)
    assert free1 == free0
    ref = ck.linear_w4a4(d["x"], d["w_packed"], d["w_scale"], 64, bias=d["bias"])
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    ck.device_error_check()


@pytest.mark.gpu
def test_static_rejects_input_not_on_the_current_device(ck):
    # the scratch belongs to the current device, so x must live there: host memory is refused
    x = torch.zeros(8, 128, dtype=torch.bfloat16)
    torch.cuda.init()
    st = ck.lib.ck_linear_w4a4_static(ck._ptr(x), 0, 8, 128, 64, 128, 64, ck._ptr(x), ck._ptr(x), None,
                                      ck._ptr(x), None)
    assert st == ck.CK_ERR_INVALID_ARG
    assert "device" in ck.last_error()
    ck.device_error_check()
