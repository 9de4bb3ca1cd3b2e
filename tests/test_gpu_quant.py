"""GPU parity of the fused NVFP4 + residual-channel quantizer against the CPU oracle.

Codes, scale bytes (canonical form) and the tensor scale must match bit for bit.
"""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_arc_b200 as arc
import oracle as O
import workloads as W
from tests._helpers import assert_codes_equal, gpu_codes, gpu_sf_canonical, gpu_sf_swizzled, to_dev

pytestmark = pytest.mark.gpu


def run_and_compare(x_bits, r=None, idx=None, static=None, gain_bits=None, eps=1e-6, weights=False):
    M, K = x_bits.shape
    if idx is None:
        idx = O.calibrate(x_bits, r) if r else np.zeros(0, np.int32)
    idx = np.asarray(idx, np.int32)
    x = to_dev(x_bits)
    d_idx = torch.from_numpy(idx).cuda() if idx.size else None
    if weights:
        q = arc.pack_weight_nvfp4(x, d_idx)
        s_ref = O.tensor_scale(O.amax(x_bits))
        c_ref, sf_ref = O.pack_weight(x_bits, idx, s_ref)
    else:
        st = None if static is None else torch.tensor([static], dtype=torch.float32, device="cuda")
        g = None if gain_bits is None else to_dev(gain_bits)
        q = arc.quantize_act_nvfp4(x, d_idx, rms_gain=g, eps=eps, static_scale=st)
        eps32 = float(np.float32(eps))
        if static is not None:
            s_ref = float(np.float32(static))
        elif gain_bits is not None:
            s_ref = O.tensor_scale(O.amax(O.rmsnorm(x_bits, gain_bits, eps32)))
        else:
            s_ref = O.tensor_scale(O.amax(x_bits))
        c_ref, sf_ref = O.quantize_act(x_bits, idx, s_ref, rms_gain=gain_bits, eps=eps32)
    torch.cuda.synchronize()
    assert arc.last_device_status() == 0
    assert q.scale.item() == np.float32(s_ref), (q.scale.item(), s_ref)
    assert_codes_equal(gpu_codes(q, M), c_ref, "codes")
    assert_codes_equal(gpu_sf_canonical(q, M), sf_ref, "scale bytes")
    # padding rows of the swizzled layout are zero
    swz = gpu_sf_swizzled(q, M)
    np.testing.assert_array_equal(swz, O.sf_swizzle(sf_ref))
    return q, idx


def test_tiny_config():
    d = W.tiny()
    run_and_compare(d["x"], r=16)


@pytest.mark.parametrize("proj,rows", [("qkv", 300), ("down", 130), ("gateup", 129)])
def test_llama_shapes_ragged_rows(proj, rows):
    d = W.llama8b(proj, rows=rows, with_w=False)
    run_and_compare(d["x"], r=128)


@pytest.mark.parametrize("frac,r", [(0.0, 0), (0.001, 32), (0.01, 128), (0.05, 256)])
def test_outlier_stress(frac, r):
    d = W.stress(frac, rows=256, w_rows=8)
    run_and_compare(d["x"], r=r)


@pytest.mark.parametrize("K,r,M", [(272, 16, 40), (208, 48, 7), (64, 0, 1), (4160, 64, 131)])
def test_k_not_multiple_of_64_and_tiny_rows(K, r, M):
    x = W.matrix_bf16(9, 1, M, K, 1.0, col_mult=W.outlier_multipliers(9, 0, K, max(1, K // 50), 10.0, 60.0))
    run_and_compare(x, r=r)


@pytest.mark.parametrize("static", [0.01, 1.0, 1e-6])
def test_static_scale(static):
    d = W.llama8b("o", rows=64, with_w=False)
    run_and_compare(d["x"], r=32, static=static)


def test_rmsnorm_prologue_unit_gain():
    d = W.recurrent(S=200, d=2048, ffn=256)
    run_and_compare(d["h"], r=64, gain_bits=d["layers"][0]["gain"])


def test_rmsnorm_prologue_random_gain_and_static():
    h = W.matrix_bf16(21, 1, 96, 512, 3.0)
    g = W.matrix_bf16(21, 2, 1, 512, 1.0).reshape(-1)
    run_and_compare(h, r=32, gain_bits=g)
    run_and_compare(h, r=32, gain_bits=g, static=0.002)


@pytest.mark.parametrize("which", ["tiny", "qkv"])
def test_weight_pack(which):
    if which == "tiny":
        d = W.tiny()
        idx = O.calibrate(d["x"], 16)
        run_and_compare(d["w"], idx=idx, weights=True)
    else:
        d = W.llama8b("qkv", rows=64, w_rows=512)
        idx = O.calibrate(d["x"], 128)
        run_and_compare(d["w"], idx=idx, weights=True)


def test_ties_and_signed_zero_exact():
    # blocks whose values sit exactly on E2M1 rounding ties for a non-power-of-two decode scale,
    # plus small negatives that round to a signed zero; static tensor scale 1
    rng = np.random.default_rng(3)
    e4 = [0x30, 0x33, 0x35, 0x3B, 0x2D]  # E4M3 scale bytes, several with 3 mantissa bits set
    vals = []
    for b in range(64):
        sf = e4[b % len(e4)]
        e, m = (sf >> 3) & 15, sf & 7
        dval = (1 + m / 8) * 2.0 ** (e - 7)
        blk = [6 * dval]
        ties = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -1.25, -5.0, -0.1, -0.0, 0.0, 0.3]
        blk += [t * dval for t in ties]
        rng.shuffle(blk)
        vals.append(blk)
    x = np.array(vals, np.float32).reshape(8, 128)
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)  # truncation keeps -0.1*d as a small negative
    run_and_compare(bits, idx=np.arange(16, 32, dtype=np.int32), static=1.0)


def test_zero_tensor_and_zero_rows():
    x = np.zeros((70, 128), np.uint16)
    run_and_compare(x, idx=np.arange(16, dtype=np.int32))  # amax 0 -> scale 1, all codes 0
    y = W.matrix_bf16(5, 1, 70, 128, 1.0)
    y[3] = 0
    y[50] = 0x8000
    run_and_compare(y, r=16)


def test_calibration_matches_oracle():
    for x in (W.tiny()["x"], W.llama8b("down", rows=200, with_w=False)["x"],
              W.stress(0.05, rows=300, w_rows=8)["x"]):
        for r in (16, 128, 256):
            got = arc.calibrate_outliers(to_dev(x), r).cpu().numpy()
            np.testing.assert_array_equal(got, O.calibrate(x, r))


def test_rejects_bad_arguments():
    x = to_dev(W.matrix_bf16(1, 1, 16, 64, 1.0))
    with pytest.raises(arc.ArcError) as e:
        arc.quantize_act_nvfp4(x[:, :40])  # K % 16 != 0
    assert e.value.code == 1
    idx = torch.arange(17, dtype=torch.int32, device="cuda")
    with pytest.raises(arc.ArcError):
        arc.quantize_act_nvfp4(x, idx)  # r % 16 != 0


def test_graph_capture_and_replay_give_identical_bytes():
    # The quantizer captured in a CUDA graph (abs-max partials, then the coding kernel started by
    # programmatic dependent launch) and replayed twice gives the bytes of a direct call, and
    # both equal the oracle.
    d = W.llama8b("qkv", rows=300, with_w=False)
    x_bits = d["x"]
    idx = O.calibrate(x_bits, 128)
    x = to_dev(x_bits)
    d_idx = torch.from_numpy(idx).cuda()
    direct = arc.quantize_act_nvfp4(x, d_idx)
    out = arc.quantize_act_nvfp4(x, d_idx)  # the buffers the graph writes
    ws = torch.empty(arc.quantize_workspace_bytes(300, 128), dtype=torch.uint8, device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        arc.quantize_act_nvfp4(x, d_idx, out=out, workspace=ws, stream=side)  # warm-up outside capture
        torch.cuda.synchronize()
        for t in (out.codes, out.sf, out.scale):
            t.zero_()
        with torch.cuda.graph(g, stream=side):
            arc.quantize_act_nvfp4(x, d_idx, out=out, workspace=ws, stream=side)
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert arc.last_device_status() == 0
    assert torch.equal(out.codes, direct.codes) and torch.equal(out.sf, direct.sf)
    assert out.scale.item() == direct.scale.item()
    s_ref = O.tensor_scale(O.amax(x_bits))
    c_ref, sf_ref = O.quantize_act(x_bits, idx, s_ref)
    assert_codes_equal(gpu_codes(out, 300), c_ref, "codes")
    assert_codes_equal(gpu_sf_canonical(out, 300), sf_ref, "scale bytes")


@pytest.mark.parametrize("rows,proj,static", [(1776, "down", None), (9473, "qkv", None), (9473, "qkv", 0.02)])
def test_many_rows_per_warp(rows, proj, static):
    # several rows per warp (each warp codes rows blockIdx + gridDim * j), with the next row's
    # first segment prefetched across the row boundary, and a ragged row count past one full
    # wave of rows
    d = W.llama8b(proj, rows=rows, with_w=False)
    run_and_compare(d["x"], r=128, static=static)


def test_repeated_calls_with_one_workspace():
    # consecutive calls reuse the workspace's abs-max partials: each call must see only its own
    # maxima (a different tensor scale every call)
    x0 = W.llama8b("o", rows=512, with_w=False)["x"]
    idx = O.calibrate(x0, 64)
    d_idx = torch.from_numpy(idx).cuda()
    ws = torch.empty(arc.quantize_workspace_bytes(512, 64), dtype=torch.uint8, device="cuda")
    for k, scale in enumerate((1.0, 4.0, 0.25, 8.0)):  # powers of two: exact in bf16
        xb = (torch.from_numpy(O.bf16_bits_to_f32(x0)) * scale).bfloat16().view(torch.int16).numpy().view(np.uint16)
        q = arc.quantize_act_nvfp4(to_dev(xb), d_idx, workspace=ws)
        torch.cuda.synchronize()
        assert arc.last_device_status() == 0
        s_ref = O.tensor_scale(O.amax(xb))
        assert q.scale.item() == np.float32(s_ref), (k, q.scale.item(), s_ref)
        c_ref, sf_ref = O.quantize_act(xb, idx, s_ref)
        assert_codes_equal(gpu_codes(q, 512), c_ref, "codes")
        assert_codes_equal(gpu_sf_canonical(q, 512), sf_ref, "scale bytes")
