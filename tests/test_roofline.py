"""Measurement arithmetic, pinned to the decode-ceiling worked example printed
on "Small MoE Architecture, in depth" ("Worked example: the batch-1 budget on
a device") and to closed forms of the layer's work."""
import os

import numpy as np

from sparse_mixture_experts_sigmoid_b200 import roofline
from sparse_mixture_experts_sigmoid_b200.workloads import WORKLOADS

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "decode_ceiling.txt")


def test_decode_ceiling_worked_example():
    rows, params = [], {}
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        parts = line.split()
        if len(parts) == 2:
            params[parts[0]] = float(parts[1])
        else:
            rows.append((parts[0], *map(float, parts[1:])))
    assert len(rows) == 3
    for name, total, active, fp_gb, ceil_tps in rows:
        fp, tps = roofline.batch1_decode_ceiling(total, active, params["bytes_per_param"], params["mem_gb_s"])
        assert f"{fp:4.2f}" == f"{fp_gb:4.2f}", name
        assert round(tps) == ceil_tps, name


def test_layer_work_closed_forms():
    w = WORKLOADS["mixtral_prefill"]
    counts = np.full(w.E, w.R // w.E)
    lw = roofline.layer_work(w, counts)
    assert lw["flops"] == 2.0 * 4096 * 2 * 3 * 4096 * 14336 + 2.0 * 4096 * 8 * 4096
    # all 8 experts active: 8 * 3 * 14336 * 4096 * 2 bytes of weights, ~2.82 GB
    assert abs(lw["bytes"] - (8 * 3 * 14336 * 4096 * 2 + 8 * 4096 * 2 + 2 * 4096 * 4096 * 2)) == 0
    d = WORKLOADS["mixtral_decode"]
    dw = roofline.layer_work(d, np.r_[1, 1, np.zeros(6)])
    # decode reads only the two chosen experts: 704.6 MB of expert weights
    assert abs(2 * 3 * 14336 * 4096 * 2 / 1e6 - 704.6) < 0.1
    assert dw["bytes"] == 2 * 3 * 14336 * 4096 * 2 + 8 * 4096 * 2 + 2 * 4096 * 2
    # stage flops add up to the layer's
    for name in ("gemma_upcycle", "qwen_shared"):
        w = WORKLOADS[name]
        sw = roofline.stage_work(w, np.ones(w.E))
        assert abs(sum(v["flops"] for v in sw.values()) - w.flops()) < 1e-6 * w.flops()


def test_peaks_file_or_fallback(tmp_path):
    p = roofline.measured_peaks(str(tmp_path / "missing.json"))
    assert p["source"] == "fallback" and p["hbm_gbs"] == 6650.0


def test_fractions_name_the_binding_resource():
    """frac = max(F / peak_F, B / peak_B) / t, whichever side of the ridge the
    work lies on; both components are reported."""
    peaks = {"hbm_gbs": 6000.0}
    # 1 TFLOP and 1 GB in 1 ms: 1000 TFLOP/s (of 2000) and 1000 GB/s (of 6000)
    r = roofline.fractions(1e12, 1e9, 1e-3, peaks, 2000.0)
    assert r["bound"] == "tensor" and abs(r["tensor_frac"] - 0.5) < 1e-12
    assert abs(r["hbm_frac"] - 1 / 6) < 1e-12 and r["frac"] == r["tensor_frac"]
    # near the ridge (intensity 250 vs a ridge of 333): the bigger fraction wins
    r = roofline.fractions(250e9, 1e9, 1e-3, peaks, 2000.0)
    assert r["bound"] == "hbm" and abs(r["frac"] - 1 / 6) < 1e-12 and abs(r["tensor_frac"] - 0.125) < 1e-12


def test_load_spread():
    s = roofline.load_spread([4, 0, 2, 2])
    assert s["active_experts"] == 3 and s["max"] == 4 and s["min"] == 0 and s["mean"] == 2.0
    assert abs(s["cv"] - np.std([4, 0, 2, 2]) / 2.0) < 1e-15


def test_bench_names_the_kernel_each_stage_runs():
    """The kernel (and source) the bench line attributes each stage to: the
    batch-1 bf16 down projection runs the TMA-ring kernel unless the layer has
    a shared expert, 4-bit layers run the ring-streamed 4-bit kernels, and
    every named source exists (its hash keys the committed DRAM captures)."""
    import dataclasses

    import bench

    dec = WORKLOADS["mixtral_decode"]
    assert bench.kernel_of("down", dec, False) == ("down_tma_kernel", "segment_tma.cu")
    assert bench.kernel_of("gate_up", dec, False) == ("seg_gateup_kernel", "segment.cu")
    assert bench.kernel_of("down", dec, True) == ("q4t_down_kernel", "segment_q4_tma.cu")
    shared = dataclasses.replace(dec, h_shared=1024)
    assert bench.kernel_of("down", shared, False) == ("down_direct_kernel", "segment.cu")
    f32 = dataclasses.replace(dec, dtype="f32")
    assert bench.kernel_of("down", f32, False) == ("down_direct_kernel", "segment.cu")
    pre = WORKLOADS["mixtral_prefill"]
    assert bench.kernel_of("gate_up", pre, False) == ("grouped_gemm_kernel", bench.GG_SRC)
    tables = (bench.STAGE_KERNEL, bench.STAGE_KERNEL_SMALL, bench.STAGE_KERNEL_SMALL_TMA, bench.STAGE_KERNEL_Q4)
    for table in tables:
        for _, src in table.values():
            assert len(bench.source_hash(src)) == 16
