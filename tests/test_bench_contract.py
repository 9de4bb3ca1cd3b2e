"""The JSON line of bench.py, on CPU: the keys and units of our arm's line (built from a fixed
timing result), its roofline arithmetic against the measured peaks, the rule that the GEMM's
DRAM traffic is reported only for the kernel source it was captured on, and the reference arm's
line from the CPU oracle on the tiny workload.
"""
import json
import os
import shutil

import bench
import workloads as W

KEYS = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
        "vs_baseline", "dtype", "data", "config", "roofline", "quant_roofline", "e2e", "gpu_launches", "clocks")


def _args(fmt="nvfp4", no_e2e=False):
    class A:
        steps, warmup, workload, reorder = 10, 3, "llama8b", False

    A.format, A.no_e2e = fmt, no_e2e
    return A


def _res():
    return dict(total_ms=6.0, q_ms=1.5, g_ms=4.5, e2e_ms=60.0, per_layer={},
                clocks={"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": []}, h2d=100, d2h=200, launches=120)


def test_our_line_has_the_contract_keys_and_units():
    layers, desc = bench.layer_set("llama8b")
    line = bench.layers_line(_args(), 1, layers, desc, _res())
    for k in KEYS:
        assert k in line, k
    json.dumps(line)
    assert line["higher_is_better"] is True and line["scaling"] == "weak" and line["n_gpus"] == 1
    assert line["vs_baseline"] is None
    assert line["config"]["workload"].startswith("llama8b") and "flushed" in line["config"]["l2"]
    assert abs(line["ms_per_step"] - 0.6) < 1e-12
    flops = sum(bench.layer_flops(L) for L in layers)
    assert abs(line["value"] - flops * 10 / 6.0e-3 / 1e12) < 1e-9 * line["value"]
    # the dominant kernel's roofline: GEMM flops over its own time, against 4 x the measured BF16
    # burst (the nominal dense FP4 / BF16 ratio)
    pk, _ = bench.peaks()
    r = line["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert abs(r["peak"] - 4 * pk["bf16_tflops"]) < 1e-9
    assert abs(r["achieved"] - flops * 10 / 4.5e-3 / 1e12) < 1e-9 * r["achieved"]
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-12
    q = line["quant_roofline"]
    assert q["bound"] == "hbm" and q["unit"] == "GB/s" and abs(q["peak"] - pk["hbm_gbs"]) < 1e-9
    assert abs(q["achieved"] - sum(bench.layer_quant_bytes(L) for L in layers) * 10 / 1.5e-3 / 1e9) < 1e-6 * q["achieved"]
    # end to end: the same metric over the host-copy time, with the bytes copied per step
    e = line["e2e"]
    assert e["unit"] == line["unit"] and e["h2d_bytes_per_step"] == 100 and e["d2h_bytes_per_step"] == 200
    assert abs(e["value"] - flops * 10 / 60e-3 / 1e12) < 1e-9 * e["value"]
    assert line["gpu_launches"] == 120


def test_fp8_and_mxfp4_lines_use_their_own_peaks():
    layers, desc = bench.layer_set("llama8b")
    pk, _ = bench.peaks()
    fp8 = bench.layers_line(_args("fp8", no_e2e=True), 1, layers, desc, _res())
    assert abs(fp8["roofline"]["peak"] - 2 * pk["bf16_tflops"]) < 1e-9
    assert fp8["e2e"] is None and fp8["roofline"]["traffic"] is None
    mx = bench.layers_line(_args("mxfp4", no_e2e=True), 1, layers, desc, _res())
    assert abs(mx["roofline"]["peak"] - 4 * pk["bf16_tflops"]) < 1e-9
    assert mx["metric"] != fp8["metric"]


def test_traffic_only_for_the_kernel_source_it_was_taken_on(tmp_path, monkeypatch):
    src = os.path.join(bench.ROOT, "nvfp4_block_scaled_arc_b200", "csrc")
    dst = tmp_path / "nvfp4_block_scaled_arc_b200" / "csrc"
    dst.mkdir(parents=True)
    for f in ("arc_device.cuh", "gemm.cuh"):
        shutil.copy(os.path.join(src, f), dst / f)
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    fp = bench.gemm_kernel_fingerprint()
    prof = tmp_path / "profiles" / "gemm_nvfp4_llama8b.md"
    prof.write_text(f"kernel_source_fingerprint: {fp}\ndram_bytes_per_launch_step_avg: 12345\n")
    assert bench.ncu_traffic() == 12345.0
    prof.write_text("kernel_source_fingerprint: 0000000000000000\ndram_bytes_per_launch_step_avg: 12345\n")
    assert bench.ncu_traffic() is None
    # any edit of the kernel source after the capture withdraws the figure
    prof.write_text(f"kernel_source_fingerprint: {fp}\ndram_bytes_per_launch_step_avg: 12345\n")
    with open(dst / "gemm.cuh", "a") as fh:
        fh.write("\n")
    assert bench.ncu_traffic() is None


def test_reference_arm_line_from_the_oracle(capsys, monkeypatch):
    monkeypatch.setenv("ARC_ORACLE_THREADS", "2")
    layers = [dict(name="tiny", M=16, K=256, N=256, r=16, gen=lambda rows, row0: W.tiny(rows))]

    class A:
        steps, warmup, reorder, format = 2, 1, False, "nvfp4"

    bench.run_reference(A, 0, 1, layers, "tiny")
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == bench.UNIT
    assert line["metric"] == bench.METRIC and line["steps"] == 2 and line["warmup"] == 1
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["cpu_baseline"]["cores"] == 2
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    # other ranks print nothing
    bench.run_reference(A, 1, 2, layers, "tiny")
    assert capsys.readouterr().out == ""
