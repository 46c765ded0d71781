"""Host-side pieces of bench.py (CPU): workload descriptions, entry-point names,
kernel hashes, and the cpu_baseline leg's parity report."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
import oracle  # noqa: E402
from exact_attention_152_b200.workloads import HEADLINE, WORKLOADS  # noqa: E402


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_workload_config_and_names(name):
    w = WORKLOADS[name]
    cfg = bench.workload_config(w, 1)
    assert cfg["workload"] == name and cfg["per_gpu_problem"]
    assert w.flops > 0
    assert bench.launch_name(w).startswith("attn_fwd")
    assert bench.bwd_launch_name(w).startswith("attn_bwd")
    if w.colmask:
        assert bench.launch_name(w) == "attn_fwd_colmask" and "doc_lengths" in cfg
    if w.packed:
        assert bench.launch_name(w) == "attn_fwd_varlen" and cfg["num_seqs"] == len(w.seqlens)


def test_kernel_hash_ignores_comments_and_tracks_code(tmp_path, monkeypatch):
    h_fwd, h_bwd = bench.kernel_source_hash("fwd"), bench.kernel_source_hash("bwd")
    assert h_fwd != h_bwd and len(h_fwd) == 16
    # a copy of the sources with an extra comment hashes the same; a code change does not
    csrc = os.path.join(ROOT, "exact_attention_152_b200", "csrc")
    fake = tmp_path / "exact_attention_152_b200" / "csrc"
    fake.mkdir(parents=True)
    for n in bench.KERNEL_SOURCES["fwd"]:
        (fake / n).write_text(open(os.path.join(csrc, n)).read())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.kernel_source_hash("fwd") == h_fwd
    src = (fake / "attn_fwd.cu").read_text()
    (fake / "attn_fwd.cu").write_text(src + "\n// a comment\n/* another */\n")
    assert bench.kernel_source_hash("fwd") == h_fwd
    (fake / "attn_fwd.cu").write_text(src + "\nstatic int extra_code = 1;\n")
    assert bench.kernel_source_hash("fwd") != h_fwd


def test_recorded_traffic_matches_current_sources():
    """profiles/ncu_traffic.json holds the headline's counters for the current
    kernel sources (the bench reports them as roofline.traffic)."""
    t = bench.recorded_traffic(HEADLINE, "fwd")
    assert t is not None and 0.8e8 < t < 4e8
    assert bench.recorded_traffic(HEADLINE, "bwd") is not None


@pytest.mark.parametrize("name", ["tiny_b1h2n128d64", "varlen16_h16_d128_causal"])
def test_cpu_baseline_parity_report(name):
    """With the oracle's own result standing in for the GPU's, the parity report
    is exactly zero (indexing of dense and packed layouts); with zeros it is
    the oracle's magnitudes."""
    w = WORKLOADS[name]
    shape_o = (w.total, w.H, w.d) if w.packed else (w.B, w.H, w.Nq, w.d)
    shape_l = (w.H, w.total) if w.packed else (w.B, w.H, w.Nq)
    zeros = bench.cpu_baseline(w, 0.5, np.zeros(shape_o, np.float32), np.zeros(shape_l, np.float32))
    assert zeros["parity"]["rows"] > 0 and zeros["parity"]["max_abs_o"] > 0.1
    if not w.packed:
        o = np.zeros(shape_o)
        lse = np.zeros(shape_l)
        for b in range(w.B):
            for h in range(w.H):
                bh = b * w.H + h
                q = w.to_f64("q", w.head_bits("q", bh))
                k, v = (w.to_f64(x, w.head_bits(x, w.kv_head_of(bh))) for x in "kv")
                o[b, h], lse[b, h] = oracle.attn_rows(q, np.arange(w.Nq), k, v, w.scale, w.causal)
        exact = bench.cpu_baseline(w, 0.5, o, lse)["parity"]
        assert exact["max_abs_o"] == 0.0 and exact["max_abs_lse"] == 0.0


def test_peak_follows_the_timed_window():
    """A short window with no power-cap samples is a burst; a seconds-long
    window, or one that saw sw_power_cap, takes the sustained figure."""
    peaks = {"burst": 1636.8, "sustained": 1388.9, "hbm_gbs": 6551.4, "source": "measured"}
    cool = {"sm_mhz": 1965.0, "reasons": []}
    capped = {"sm_mhz": 1620.0, "reasons": ["sw_power_cap"]}
    assert bench.pick_peak(peaks, 18.0, cool)[0] == 1636.8
    assert bench.pick_peak(peaks, 18.0, None)[0] == 1636.8
    assert bench.pick_peak(peaks, 18.0, capped)[0] == 1388.9
    assert bench.pick_peak(peaks, 1800.0, cool)[0] == 1388.9
    assert bench.pick_peak(peaks, 18.0, cool, ratio=2.0)[0] == 2 * 1636.8
    # 148 SMs x 8192 FLOP/clk at 1965 MHz
    assert abs(bench.clock_peak(cool) - 2382.4) < 0.1
    assert bench.clock_peak(None) is None


def test_clock_samples_near_the_timed_region():
    """The clock summary keeps the nvidia-smi rows stamped within the margin of
    the timed region, and falls back to every row when none is."""
    import datetime
    rows = [
        "2026/12/03 10:00:00.000, 1965, 1965, 300.0, 0, Not Active, Not Active, Not Active, Not Active",
        "2026/12/03 10:00:00.500, 1600, 1965, 900.0, 100, Not Active, Not Active, Not Active, Active",
        "2026/12/03 10:00:00.520, 1620, 1965, 910.0, 100, Not Active, Not Active, Not Active, Active",
        "2026/12/03 10:00:02.000, 1965, 1965, 250.0, 0, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
    ]
    t0 = datetime.datetime(2026, 12, 3, 10, 0, 0, 480000)
    t1 = datetime.datetime(2026, 12, 3, 10, 0, 0, 500000)
    c = bench.ClockSampler.parse(rows, t0, t1, 0.06)
    assert c["samples"] == 2 and c["samples_in_window"] == 2
    assert c["sm_mhz"] == 1610.0 and c["reasons"] == ["sw_power_cap"] and c["power_w_max"] == 910.0
    far = datetime.datetime(2026, 12, 3, 11, 0, 0)
    c = bench.ClockSampler.parse(rows, far, far, 0.06)
    assert c["samples"] == 4 and c["samples_in_window"] == 0
    assert bench.ClockSampler.parse(["x"], t0, t1) is None


def test_colmask_launch_count():
    """The document workload's calls launch the mask summaries, the CTA plan
    and the attention kernel; a problem with more units than the plan holds
    launches two kernels."""
    import types
    w = WORKLOADS["docs_b2h16n8k_d128_causal"]
    assert bench.colmask_launches(w) == 3
    big = types.SimpleNamespace(B=64, Nq=65536, Nk=65536)
    assert bench.colmask_launches(big) == 2


def test_bwd_colmask_launch_count():
    """The document workload's backward launches row sums, mask summaries, the
    CTA plan, the main kernel and the dQ rounding."""
    assert bench.bwd_colmask_launches(WORKLOADS["docs_b2h16n8k_d128_causal"]) == 5
