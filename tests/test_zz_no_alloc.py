"""The workspace-free quantization entry point against the regular one.

arc_quantize_act_nvfp4_static_scratch exists for callers that cannot allocate device memory while
they run (a process that reserves all of its GPU memory at start-up, or a plug-in with no access
to its host framework's allocator). It takes its temporary space from a fixed array inside the
library instead of a workspace argument. This test calls both entry points through the C ABI on
the same inputs, twice in a row with different inputs (the second call finds the first call's
leftovers in the shared array), and requires identical codes, scale bytes and tensor scales.
It also checks that a request larger than the array is refused before any launch, and that
repeated calls leave the device's free memory unchanged (the call allocates nothing).
"""
import ctypes

import numpy as np
import pytest
import torch

import nvfp4_block_scaled_arc_b200 as arc
import workloads as W

pytestmark = pytest.mark.gpu

ARC_ERR_WORKSPACE = 6


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _quantize_both(x, idx, gain=None):
    L = arc.lib()
    M, K = x.shape
    r = idx.numel()
    kaug = K + r
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    outs = []
    for which in ("workspace", "static"):
        codes = torch.full((arc.codes_bytes(M, kaug),), 0xA5, dtype=torch.uint8, device="cuda")
        sf = torch.full((arc.sf_bytes(M, kaug),), 0x5A, dtype=torch.uint8, device="cuda")
        scale = torch.zeros(1, dtype=torch.float32, device="cuda")
        args = [ctypes.c_void_p(x.data_ptr()), M, K, x.stride(0), ctypes.c_void_p(idx.data_ptr()), r,
                ctypes.c_void_p(gain.data_ptr()) if gain is not None else None, 1e-6, None,
                ctypes.c_void_p(codes.data_ptr()), ctypes.c_void_p(sf.data_ptr()), ctypes.c_void_p(scale.data_ptr())]
        if which == "workspace":
            ws = torch.empty(arc.quantize_workspace_bytes(M, r), dtype=torch.uint8, device="cuda")
            st = L.arc_quantize_act_nvfp4(*args, ctypes.c_void_p(ws.data_ptr()), ws.numel(), stream)
        else:
            st = L.arc_quantize_act_nvfp4_static_scratch(*args, stream)
        assert st == 0, st
        outs.append((codes, sf, scale))
    torch.cuda.synchronize()
    assert arc.last_device_status() == 0
    return outs


def test_static_scratch_matches_workspace_entry_on_two_calls():
    # two calls in a row on different inputs: the second one finds the first one's leftovers
    first = W.llama8b("qkv", rows=1000, with_w=False)
    second = W.stress(0.05, rows=600, w_rows=8)
    for x_bits, r in ((first["x"], 128), (second["x"], 256)):
        x = _dev(x_bits)
        idx = arc.calibrate_outliers(x, r)
        (c1, s1, a1), (c2, s2, a2) = _quantize_both(x, idx)
        assert torch.equal(c1, c2)
        assert torch.equal(s1, s2)
        assert torch.equal(a1, a2)


def test_static_scratch_with_rmsnorm_prologue():
    rec = W.recurrent(S=300, d=512, ffn=64)
    h = _dev(rec["h"])
    g = _dev(rec["layers"][0]["gain"])
    idx = arc.calibrate_outliers(h, 64)
    (c1, s1, a1), (c2, s2, a2) = _quantize_both(h, idx, gain=g)
    assert torch.equal(c1, c2) and torch.equal(s1, s2) and torch.equal(a1, a2)


def test_static_scratch_refuses_requests_beyond_its_size():
    L = arc.lib()
    x = _dev(W.matrix_bf16(3, 1, 16, 256, 1.0))
    idx = torch.arange(256, dtype=torch.int32, device="cuda")
    out = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    scale = torch.zeros(1, dtype=torch.float32, device="cuda")
    M = 1 << 20  # 8 bytes per row of RMSNorm statistics exceed the fixed array
    st = L.arc_quantize_act_nvfp4_static_scratch(
        ctypes.c_void_p(x.data_ptr()), M, 256, 256, ctypes.c_void_p(idx.data_ptr()), 256, None, 1e-6, None,
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(scale.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == ARC_ERR_WORKSPACE


def test_static_scratch_allocates_no_device_memory():
    L = arc.lib()
    d = W.llama8b("o", rows=512, with_w=False)
    x = _dev(d["x"])
    r = 128
    idx = arc.calibrate_outliers(x, r)
    M, K = x.shape
    codes = torch.empty(arc.codes_bytes(M, K + r), dtype=torch.uint8, device="cuda")
    sf = torch.empty(arc.sf_bytes(M, K + r), dtype=torch.uint8, device="cuda")
    scale = torch.zeros(1, dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    def call():
        st = L.arc_quantize_act_nvfp4_static_scratch(
            ctypes.c_void_p(x.data_ptr()), M, K, K, ctypes.c_void_p(idx.data_ptr()), r, None, 1e-6, None,
            ctypes.c_void_p(codes.data_ptr()), ctypes.c_void_p(sf.data_ptr()), ctypes.c_void_p(scale.data_ptr()),
            stream)
        assert st == 0, st

    call()  # the first call looks up the array's address
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(5):
        call()
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, (free0, free1)
    assert arc.last_device_status() == 0
