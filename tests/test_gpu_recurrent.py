"""GPU parity of the recurrent SwiGLU block pieces and of the RAMP-style prefill driver.

Bit-exactness across many recurrent steps is not a meaningful target (one flipped bf16 rounding
in a GEMM output changes later codes), so each sublayer is checked teacher-forced: the oracle
takes the GPU's own input of that step; codes and scale bytes must match bit for bit, GEMM
outputs within the 2e-3 rule, the SwiGLU gate within one bf16 ulp. The driver is then checked
to produce exactly the composition of the individual calls.
"""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_arc_b200 as arc
import oracle as O
import workloads as W
from tests._helpers import (GEMM_TOL, assert_codes_equal, gpu_codes, gpu_sf_canonical, normalized_gemm_error,
                            row_norms, to_bits, to_dev)

pytestmark = pytest.mark.gpu

EPS = 1e-6


def make_block(S, d, ffn, r):
    rec = W.recurrent(S=S, d=d, ffn=ffn)
    h = to_dev(rec["h"])
    subs = []
    for L in rec["layers"]:
        wgu, wd, gain = to_dev(L["wgu"]), to_dev(L["wd"]), to_dev(L["gain"])
        # offline calibration on a BF16 pass of the block's first step
        n = arc.rmsnorm_bf16(h, gain, EPS)
        idx_gu = arc.calibrate_outliers(n, r)
        act = arc.silu_mul_bf16(arc.gemm_bf16(n, wgu))
        idx_d = arc.calibrate_outliers(act, r)
        subs.append(dict(gain=gain, wgu=wgu, wd=wd, idx_gu=idx_gu, idx_d=idx_d,
                         gu_q=arc.pack_weight_nvfp4(wgu, idx_gu), d_q=arc.pack_weight_nvfp4(wd, idx_d),
                         bits=L))
    torch.cuda.synchronize()
    return rec, h, subs


def silu_within_one_ulp(got_bits, gu_bits):
    want = O.bf16_bits_to_f32(O.silu_mul(gu_bits)).astype(np.float64)
    got = O.bf16_bits_to_f32(got_bits).astype(np.float64)
    ulp = np.maximum(np.abs(want), 1e-30) * 2.0 ** -7
    assert np.all(np.abs(got - want) <= ulp + 1e-38)


def nvfp4_sublayer_teacher_forced(h, L, r):
    S, d = h.shape
    hb = to_bits(h)
    g_bits = to_bits(L["gain"])
    idx_gu = L["idx_gu"].cpu().numpy()
    idx_d = L["idx_d"].cpu().numpy()
    # fused RMSNorm + quantize
    qa = arc.quantize_act_nvfp4(h, L["idx_gu"], rms_gain=L["gain"], eps=EPS)
    n_ref = O.rmsnorm(hb, g_bits, float(np.float32(EPS)))
    s_ref = O.tensor_scale(O.amax(n_ref))
    c_ref, sf_ref = O.quantize_act(hb, idx_gu, s_ref, rms_gain=g_bits, eps=float(np.float32(EPS)))
    torch.cuda.synchronize()
    assert qa.scale.item() == np.float32(s_ref)
    assert_codes_equal(gpu_codes(qa, S), c_ref)
    assert_codes_equal(gpu_sf_canonical(qa, S), sf_ref, "scale bytes")
    # gate|up GEMM
    gu = arc.gemm_nvfp4(qa, L["gu_q"])
    wgu_bits = to_bits(L["wgu"])
    sw = O.tensor_scale(O.amax(wgu_bits))
    bc, bsf = O.pack_weight(wgu_bits, idx_gu, sw)
    rows = np.r_[0:4, S - 4:S]
    ref = O.gemm_nvfp4_f64_matmul(c_ref, sf_ref, s_ref, bc, bsf, sw, rows=rows)
    gu_bits = to_bits(gu)
    assert normalized_gemm_error(gu_bits[rows], ref, row_norms(n_ref[rows]), row_norms(wgu_bits)) <= GEMM_TOL
    # SwiGLU gate
    act = arc.silu_mul_bf16(gu)
    act_bits = to_bits(act)
    silu_within_one_ulp(act_bits, gu_bits)
    # quantize the gate output (teacher-forced on the GPU's own act)
    qd = arc.quantize_act_nvfp4(act, L["idx_d"])
    s2 = O.tensor_scale(O.amax(act_bits))
    c2, sf2 = O.quantize_act(act_bits, idx_d, s2)
    torch.cuda.synchronize()
    assert qd.scale.item() == np.float32(s2)
    assert_codes_equal(gpu_codes(qd, S), c2)
    assert_codes_equal(gpu_sf_canonical(qd, S), sf2, "scale bytes")
    # down GEMM with the residual add in its epilogue (in place)
    h_new = arc.gemm_nvfp4(qd, L["d_q"], out=h.clone(), add=h)
    wd_bits = to_bits(L["wd"])
    swd = O.tensor_scale(O.amax(wd_bits))
    dc, dsf = O.pack_weight(wd_bits, idx_d, swd)
    ref = O.gemm_nvfp4_f64_matmul(c2, sf2, s2, dc, dsf, swd, rows=rows) + O.bf16_bits_to_f32(hb[rows])
    assert normalized_gemm_error(to_bits(h_new)[rows], ref, row_norms(act_bits[rows]), row_norms(wd_bits),
                                 with_add=True) <= GEMM_TOL
    return h_new


def bf16_sublayer_teacher_forced(h, L):
    S, d = h.shape
    hb = to_bits(h)
    g_bits = to_bits(L["gain"])
    n = arc.rmsnorm_bf16(h, L["gain"], EPS)
    n_bits = to_bits(n)
    np.testing.assert_array_equal(n_bits, O.rmsnorm(hb, g_bits, float(np.float32(EPS))))
    gu = arc.gemm_bf16(n, L["wgu"])
    rows = np.r_[0:4, S - 4:S]
    wgu_bits = to_bits(L["wgu"])
    ref = O.gemm_bf16_f64(n_bits, wgu_bits, rows=rows)
    gu_bits = to_bits(gu)
    assert normalized_gemm_error(gu_bits[rows], ref, row_norms(n_bits[rows]), row_norms(wgu_bits)) <= GEMM_TOL
    act = arc.silu_mul_bf16(gu)
    act_bits = to_bits(act)
    silu_within_one_ulp(act_bits, gu_bits)
    h_new = arc.gemm_bf16(act, L["wd"], out=h.clone(), add=h)
    wd_bits = to_bits(L["wd"])
    ref = O.gemm_bf16_f64(act_bits, wd_bits, rows=rows) + O.bf16_bits_to_f32(hb[rows])
    assert normalized_gemm_error(to_bits(h_new)[rows], ref, row_norms(act_bits[rows]), row_norms(wd_bits),
                                 with_add=True) <= GEMM_TOL
    return h_new


def test_sublayers_teacher_forced_full_width():
    rec, h, subs = make_block(S=160, d=2048, ffn=8192, r=64)
    h1 = nvfp4_sublayer_teacher_forced(h, subs[0], 64)
    h2 = bf16_sublayer_teacher_forced(h1, subs[1])
    assert torch.isfinite(h2.float()).all()


@pytest.mark.parametrize("T,k_low", [(3, 0), (3, 2), (2, 2)])
def test_driver_equals_composed_calls(T, k_low):
    rec, h0, subs = make_block(S=130, d=256, ffn=512, r=32)
    blk = arc.RecurrentBlock(256, 512, EPS, [{k: v for k, v in s.items() if k != "bits"} for s in subs])
    h_drv = arc.recurrent_prefill(h0.clone(), blk, T, k_low)
    h = h0.clone()
    for t in range(T):
        for L in subs:
            if t < k_low:
                qa = arc.quantize_act_nvfp4(h, L["idx_gu"], rms_gain=L["gain"], eps=EPS)
                gu = arc.gemm_nvfp4(qa, L["gu_q"])
                act = arc.silu_mul_bf16(gu)
                qd = arc.quantize_act_nvfp4(act, L["idx_d"])
                arc.gemm_nvfp4(qd, L["d_q"], out=h, add=h)
            else:
                n = arc.rmsnorm_bf16(h, L["gain"], EPS)
                gu = arc.gemm_bf16(n, L["wgu"])
                act = arc.silu_mul_bf16(gu)
                arc.gemm_bf16(act, L["wd"], out=h, add=h)
    torch.cuda.synchronize()
    assert arc.last_device_status() == 0
    assert torch.equal(h_drv, h)


def test_ramp_schedule_error_ordering():
    # fidelity of the mixed schedule against all-BF16 (hidden-state relative error)
    rec, h0, subs = make_block(S=256, d=256, ffn=512, r=32)
    blk = arc.RecurrentBlock(256, 512, EPS, [{k: v for k, v in s.items() if k != "bits"} for s in subs])
    T = 8
    ref = arc.recurrent_prefill(h0.clone(), blk, T, 0).float()
    errs = {}
    for k in (0, 4, 8):
        out = arc.recurrent_prefill(h0.clone(), blk, T, k).float()
        errs[k] = (torch.linalg.norm(out - ref) / torch.linalg.norm(ref)).item()
    assert errs[0] == 0.0
    assert 0.0 < errs[4] < errs[8]


@pytest.mark.parametrize("schedule", [[0, 1, 0, 1], [1, 1, 0, 0], [0, 0, 1, 1], [1, 0, 0, 1]])
def test_schedule_driver_equals_composed_steps(schedule):
    # any per-step precision schedule is the composition of its steps, each run on its own
    # (one step of the prefix driver: k_low = 1 for an NVFP4 step, 0 for a BF16 one)
    rec, h0, subs = make_block(S=130, d=256, ffn=512, r=32)
    blk = arc.RecurrentBlock(256, 512, EPS, [{k: v for k, v in s.items() if k != "bits"} for s in subs])
    h_drv = arc.recurrent_prefill_schedule(h0.clone(), blk, schedule)
    h = h0.clone()
    for f in schedule:
        arc.recurrent_prefill(h, blk, 1, 1 if f else 0)
    torch.cuda.synchronize()
    assert arc.last_device_status() == 0
    assert torch.equal(h_drv, h)
    # the prefix schedule is the k_low driver
    k = 2
    a = arc.recurrent_prefill_schedule(h0.clone(), blk, [1] * k + [0] * 2)
    b = arc.recurrent_prefill(h0.clone(), blk, 4, k)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
