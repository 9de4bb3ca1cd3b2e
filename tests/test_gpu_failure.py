"""Failure detection on the GPU without a fault: a GEMM launch withholds one operand load (a
flag that nothing sets), its consumer's bounded wait runs out, the kernel stops cleanly and
reports ARC_ERR_TIMEOUT through the status word; the context stays usable afterwards."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_arc_b200 as arc
import workloads as W
from tests._helpers import to_dev

pytestmark = pytest.mark.gpu

TIMEOUT = 5


@pytest.mark.parametrize("kind", ["nvfp4", "bf16"])
def test_withheld_load_times_out_and_recovers(kind):
    x = to_dev(W.matrix_bf16(31, 1, 256, 512, 1.0))
    w = to_dev(W.matrix_bf16(31, 2, 512, 512, 0.05))
    assert arc.last_device_status() == 0
    if kind == "nvfp4":
        A = arc.quantize_act_nvfp4(x)
        B = arc.pack_weight_nvfp4(w)
        good = arc.gemm_nvfp4(A, B)
    else:
        good = arc.gemm_bf16(x, w)
    torch.cuda.synchronize()
    arc.set_wait_limit_ns(50_000_000)  # 50 ms
    try:
        arc.debug_inject(1)
        bad = arc.gemm_nvfp4(A, B) if kind == "nvfp4" else arc.gemm_bf16(x, w)
        assert arc.last_device_status() == TIMEOUT
    finally:
        arc.set_wait_limit_ns(2_000_000_000)
    again = arc.gemm_nvfp4(A, B) if kind == "nvfp4" else arc.gemm_bf16(x, w)
    torch.cuda.synchronize()
    assert arc.last_device_status() == 0
    assert torch.equal(again, good)


def test_withheld_row_copy_in_the_reordered_quantizer_times_out_and_recovers():
    # the reordered quantizer stages rows by bulk copies with bounded waits: a copy that never
    # comes must end in ARC_ERR_TIMEOUT, not a hang, and leave the context usable
    d = W.llama8b("o", rows=300, with_w=False)
    x = to_dev(d["x"])
    perm = arc.calibrate_order(x)
    good = arc.quantize_act_nvfp4_reordered(x, perm, 128)
    torch.cuda.synchronize()
    assert arc.last_device_status() == 0
    arc.set_wait_limit_ns(50_000_000)  # 50 ms
    try:
        arc.debug_inject(2)
        arc.quantize_act_nvfp4_reordered(x, perm, 128)
        assert arc.last_device_status() == TIMEOUT
    finally:
        arc.set_wait_limit_ns(2_000_000_000)
    again = arc.quantize_act_nvfp4_reordered(x, perm, 128)
    torch.cuda.synchronize()
    assert arc.last_device_status() == 0
    assert torch.equal(again.codes, good.codes) and torch.equal(again.sf, good.sf)
