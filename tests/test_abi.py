"""The C-ABI library (no GPU needed): it loads, exports every function include/arc.h declares,
its size queries follow the documented layout, and host-side argument checks reject bad calls
before any CUDA work."""
import ctypes
import os
import re

import numpy as np
import pytest

import nvfp4_block_scaled_arc_b200 as arc
import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from nvfp4_block_scaled_arc_b200 import _build

    _build.build()
    return arc.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "arc.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(arc_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(arc.exported_symbols())


def test_size_queries(L):
    for rows, kaug in [(16, 272), (4096, 4224), (130, 14464), (1, 64), (129, 65)]:
        kp = (kaug + 63) // 64 * 64
        assert L.arc_kpad(kaug) == kp == O.kpad(kaug)
        assert L.arc_nvfp4_codes_bytes(rows, kaug) == rows * kp // 2
        assert L.arc_nvfp4_sf_bytes(rows, kaug) == O.sf_swizzled_bytes(rows, kp // 16)
    assert L.arc_quantize_workspace_bytes(4096, 128) >= 4 + 4096 * 8  # partials, 1/rms per row
    assert L.arc_status_str(5) == b"ARC_ERR_TIMEOUT"


def test_host_checks_reject_before_any_launch(L):
    P = ctypes.c_void_p
    fake = P(0x10000)  # never dereferenced: the checks return first
    ws = P(0x20000)
    # K % 16 != 0
    assert L.arc_quantize_act_nvfp4(fake, 4, 40, 40, None, 0, None, 1e-6, None, fake, fake, fake, ws, 1 << 20, None) == 1
    # r % 16 != 0
    assert L.arc_quantize_act_nvfp4(fake, 4, 64, 64, fake, 8, None, 1e-6, None, fake, fake, fake, ws, 1 << 20, None) == 1
    # r > K
    assert L.arc_quantize_act_nvfp4(fake, 4, 64, 64, fake, 80, None, 1e-6, None, fake, fake, fake, ws, 1 << 20, None) == 1
    # NULL input
    assert L.arc_quantize_act_nvfp4(None, 4, 64, 64, None, 0, None, 1e-6, None, fake, fake, fake, ws, 1 << 20, None) == 1
    # misaligned codes
    assert L.arc_quantize_act_nvfp4(fake, 4, 64, 64, None, 0, None, 1e-6, None, P(0x10008), fake, fake, ws, 1 << 20, None) == 2
    # workspace too small
    assert L.arc_quantize_act_nvfp4(fake, 4, 64, 64, None, 0, None, 1e-6, None, fake, fake, fake, ws, 8, None) == 6
    # GEMM: N % 8 != 0, ldy < N
    assert L.arc_gemm_nvfp4(fake, fake, fake, fake, fake, fake, 4, 12, 64, fake, 12, None, 0, None) == 1
    assert L.arc_gemm_bf16(fake, 64, fake, 64, 4, 16, 64, fake, 8, None, 0, None) == 1
    assert L.arc_gemm_bf16(P(0x10004), 64, fake, 64, 4, 16, 64, fake, 16, None, 0, None) == 2
    assert L.arc_set_wait_limit_ns(0) == 1
    assert L.arc_debug_inject(7) == 1


def test_host_checks_of_the_reorder_fp8_and_schedule_calls(L):
    P = ctypes.c_void_p
    fake, ws = P(0x10000), P(0x20000)
    # calibration order: odd K, NULL output, small workspace, misaligned input
    assert L.arc_calibrate_order(fake, 4, 63, 64, fake, ws, 1 << 20, None) == 1
    assert L.arc_calibrate_order(fake, 4, 64, 64, None, ws, 1 << 20, None) == 1
    assert L.arc_calibrate_order(fake, 4, 64, 64, fake, ws, 8, None) == 6
    assert L.arc_calibrate_order(P(0x10002), 4, 64, 64, fake, ws, 1 << 20, None) == 2
    # reordered quantizer / packer: NULL order, rows too wide for the two row buffers, misaligned order
    assert L.arc_quantize_act_nvfp4_reordered(fake, 4, 64, 64, None, 16, None, 1e-6, None, fake, fake, fake, ws,
                                              1 << 20, None) == 1
    assert L.arc_quantize_act_nvfp4_reordered(fake, 4, 51216, 51216, fake, 16, None, 1e-6, None, fake, fake, fake,
                                              ws, 1 << 20, None) == 3
    assert L.arc_quantize_act_nvfp4_reordered(fake, 4, 64, 64, P(0x10004), 16, None, 1e-6, None, fake, fake, fake,
                                              ws, 1 << 20, None) == 2
    assert L.arc_pack_weight_nvfp4_reordered(fake, 4, 64, 64, None, 16, fake, fake, fake, ws, 1 << 20, None) == 1
    # FP8 quantizer: K % 16, ldc < K, ldc % 16, small workspace
    assert L.arc_quantize_fp8(fake, 4, 40, 40, None, fake, 48, fake, ws, 1 << 20, None) == 1
    assert L.arc_quantize_fp8(fake, 4, 64, 64, None, fake, 48, fake, ws, 1 << 20, None) == 1
    assert L.arc_quantize_fp8(fake, 4, 64, 64, None, fake, 72, fake, ws, 1 << 20, None) == 2
    assert L.arc_quantize_fp8(fake, 4, 64, 64, None, fake, 64, fake, ws, 8, None) == 6
    # FP8 GEMM: K % 16, lda % 16, N % 8
    assert L.arc_gemm_fp8(fake, 40, fake, fake, 40, fake, 4, 16, 40, fake, 16, None, 0, None) == 1
    assert L.arc_gemm_fp8(fake, 72, fake, fake, 64, fake, 4, 16, 64, fake, 16, None, 0, None) == 2
    assert L.arc_gemm_fp8(fake, 64, fake, fake, 64, fake, 4, 12, 64, fake, 16, None, 0, None) == 1
    # schedule driver: T > 0 steps and no flags
    assert L.arc_recurrent_prefill_schedule(fake, 16, None, 4, None, ws, 1 << 20, None) == 1


def test_static_scratch_reports_argument_errors_before_its_size_limit(L):
    # a request that is both too large for the fixed array and malformed reports the argument
    # error first, like the workspace entry point does
    P = ctypes.c_void_p
    fake = P(0x10000)
    big = 1 << 22  # rows: far beyond the array's limit
    assert L.arc_quantize_act_nvfp4_static_scratch(fake, big, 40, 40, None, 0, None, 1e-6, None, fake, fake, fake,
                                                   None) == 1  # K % 16 != 0
    assert L.arc_quantize_act_nvfp4_static_scratch(fake, big, 64, 64, None, 16, None, 1e-6, None, fake, fake, fake,
                                                   None) == 1  # r > 0 without idx
    assert L.arc_quantize_act_nvfp4_static_scratch(fake, big, 64, 64, None, 0, None, 1e-6, None, P(0x10008), fake,
                                                   fake, None) == 2  # misaligned codes
    assert L.arc_quantize_act_nvfp4_static_scratch(fake, big, 64, 64, None, 0, None, 1e-6, None, fake, fake, fake,
                                                   None) == 6  # well-formed, too large


def test_host_checks_of_the_mxfp4_calls(L):
    P = ctypes.c_void_p
    fake, idx = P(0x10000), P(0x30000)
    q, w = L.arc_quantize_act_mxfp4, L.arc_pack_weight_mxfp4
    for f in (q, w):
        # K % 32 != 0, r % 32 != 0, r > K, NULL idx with r > 0, NULL output, ld < K
        assert f(fake, 4, 48, 48, None, 0, fake, fake, None) == 1
        assert f(fake, 4, 64, 64, idx, 16, fake, fake, None) == 1
        assert f(fake, 4, 64, 64, idx, 96, fake, fake, None) == 1
        assert f(fake, 4, 64, 64, None, 32, fake, fake, None) == 1
        assert f(fake, 4, 64, 64, None, 0, None, fake, None) == 1
        assert f(fake, 4, 64, 32, None, 0, fake, fake, None) == 1
        # misaligned input rows or outputs
        assert f(P(0x10008), 4, 64, 64, None, 0, fake, fake, None) == 2
        assert f(fake, 4, 64, 68, None, 0, fake, fake, None) == 2
        assert f(fake, 4, 64, 64, None, 0, fake, P(0x10004), None) == 2
    g = L.arc_gemm_mxfp4
    # N % 8 != 0, ldy < N, ld_add < N with an add term, NULL operand, misaligned output
    assert g(fake, fake, fake, fake, 4, 12, 64, fake, 16, None, 0, None) == 1
    assert g(fake, fake, fake, fake, 4, 16, 64, fake, 8, None, 0, None) == 1
    assert g(fake, fake, fake, fake, 4, 16, 64, fake, 16, fake, 8, None) == 1
    assert g(None, fake, fake, fake, 4, 16, 64, fake, 16, None, 0, None) == 1
    assert g(fake, fake, fake, fake, 4, 16, 64, P(0x10002), 16, None, 0, None) == 2


def test_host_checks_of_calibration_and_the_elementwise_calls(L):
    P = ctypes.c_void_p
    fake, ws = P(0x10000), P(0x20000)
    big = 1 << 20
    c = L.arc_calibrate_outliers
    assert c(fake, 4, 63, 64, 8, fake, ws, big, None) == 1      # K odd
    assert c(fake, 4, 64, 64, 0, fake, ws, big, None) == 1      # r <= 0
    assert c(fake, 4, 64, 64, 65, fake, ws, big, None) == 1     # r > K
    assert c(fake, 4, 4096, 4096, 1025, fake, ws, big, None) == 1  # r > 1024
    assert c(fake, 4, 64, 32, 8, fake, ws, big, None) == 1      # ldx < K
    assert c(None, 4, 64, 64, 8, fake, ws, big, None) == 1
    assert c(fake, 4, 64, 64, 8, None, ws, big, None) == 1
    assert c(P(0x10002), 4, 64, 64, 8, fake, ws, big, None) == 2  # x not 4-byte aligned
    assert c(fake, 4, 64, 64, 8, fake, ws, 8, None) == 6        # workspace too small
    assert c(fake, 4, 64, 64, 8, fake, P(0x20010), big, None) == 2  # workspace not 256-byte aligned
    n = L.arc_rmsnorm_bf16
    assert n(fake, 4, 60, 64, fake, 1e-6, fake, 64, None) == 1   # d % 8
    assert n(fake, 4, 64, 56, fake, 1e-6, fake, 64, None) == 1   # ldh < d
    assert n(fake, 4, 64, 64, None, 1e-6, fake, 64, None) == 1   # no gain
    assert n(fake, 4, 64, 64, fake, 1e-6, P(0x10008), 64, None) == 2
    s = L.arc_silu_mul_bf16
    assert s(fake, 4, 60, 128, fake, 64, None) == 1              # F % 8
    assert s(fake, 4, 64, 120, fake, 64, None) == 1              # ld_gu < 2F
    assert s(fake, 4, 64, 128, fake, 56, None) == 1              # ldo < F
    assert s(P(0x10008), 4, 64, 128, fake, 64, None) == 2


def test_size_queries_of_mxfp4_calibration_and_the_recurrence(L):
    for rows, kaug in [(16, 272), (4096, 4224), (130, 14464), (1, 64), (129, 96), (300, 160)]:
        # one UE8M0 scale per 32 values of the padded depth, in the same 512-byte atoms
        assert L.arc_mxfp4_sf_bytes(rows, kaug) == O.sf_swizzled_bytes(rows, O.kpad(kaug) // 32)
    assert L.arc_mxfp4_sf_bytes(0, 64) == 0 and L.arc_mxfp4_sf_bytes(4, 0) == 0
    for K in (2, 256, 4096, 14336, 1000):
        w = L.arc_calibrate_workspace_bytes(K)
        assert w >= 12 * K and w % 256 == 0  # u32 column maxima + u64 sort keys
    assert L.arc_calibrate_workspace_bytes(0) == 0
    # the recurrence's workspace holds its codes, scale bytes, gate|up, activation, normed input
    # and a quantizer workspace, each rounded up to 256 bytes
    S, d, F, rg, rd = 4096, 2048, 8192, 64, 64
    subs = (arc.SwigluSublayer * 2)()
    for sl in subs:
        sl.r_gateup, sl.r_down = rg, rd
    blk = arc.SwigluBlock(d=d, ffn=F, eps=1e-6, n_sublayers=2, sublayers=subs)
    w = L.arc_recurrent_workspace_bytes(S, ctypes.byref(blk))
    parts = [max(L.arc_nvfp4_codes_bytes(S, d + rg), L.arc_nvfp4_codes_bytes(S, F + rd), S * max(d, F)),
             max(L.arc_nvfp4_sf_bytes(S, d + rg), L.arc_nvfp4_sf_bytes(S, F + rd)), 8, S * 2 * F * 2, S * F * 2,
             S * d * 2, L.arc_quantize_workspace_bytes(S, max(rg, rd))]
    assert sum(parts) <= w <= sum(parts) + 7 * 256
    assert L.arc_recurrent_workspace_bytes(0, ctypes.byref(blk)) == 0
    assert L.arc_recurrent_workspace_bytes(S, None) == 0
