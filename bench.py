#!/usr/bin/env python
"""Attention-forward benchmark on B200: one JSON line on stdout (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one call of the whole hot path -- one attn_fwd over the workload's full
batch (B x H heads, Nq queries, Nk keys) -- on inputs already resident in HBM.
The default workload is the non-causal B=2, H=16, N=8192, d=128 forward.  Its
Q+K+V (201 MB) exceed the 126 MB L2, so L2 is not flushed between steps.

Under torchrun (N > 1) every rank runs the same per-GPU workload on its own GPU
(independent problems: weak scaling, no data-path collective); the timed region
is bracketed by barrier + synchronize and its device time is the max over ranks.

--impl reference times the fp64 CPU oracle (the reference arm: there is no
runnable reference implementation) on bounded samples of query rows of the same
workload, in the same metric.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attention fwd TFLOP/s (BF16, 1×B200) and % of dense BF16 tensor peak"
METRIC_BWD = "attention bwd TFLOP/s (BF16, 1×B200; 2.5x the forward's FLOPs)"
UNIT = "TFLOP/s"
SPEC_DENSE_BF16_TFLOPS = 2250.0
L2_BYTES = 126 * 1024 * 1024


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=None)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--exp-mode", type=int, default=None, help="0 MUFU, 1 split, 2 polynomial")
    ap.add_argument("--threshold", type=float, default=None, help="rescale threshold (powers of 2)")
    ap.add_argument("--count-rescales", action="store_true",
                    help="after timing, one extra launch counts the (row, KV step) rescale events")
    ap.add_argument("--pass", dest="which", choices=["fwd", "bwd"], default="fwd",
                    help="time the forward (default) or the backward pass")
    return ap.parse_args(argv)


def dist_env():
    from exact_attention_152_b200 import parallel
    return parallel.rank_env()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"burst": float(p["bf16_tflops"]), "sustained": float(p["bf16_tflops_sustained"]),
                "hbm_gbs": float(p["hbm_gbs"]), "source": "measured"}
    except Exception:
        return {"burst": 1590.0, "sustained": 1400.0, "hbm_gbs": 6650.0, "source": "fallback"}


SMS = 148                       # streaming multiprocessors of a B200
DENSE_BF16_FLOP_PER_CLK_SM = 8192  # dense BF16 tensor FLOPs per SM per clock
SUSTAINED_WINDOW_MS = 1000.0    # a timed window shorter than this is a burst


def pick_peak(peaks, window_ms, clocks, ratio=1.0):
    """The measured peak that matches how the kernel was timed.

    The burst matmul figure fits a timed window under ~1 s in which the power
    cap never engaged; the seconds-long sustained figure fits a window that
    ran for seconds or saw sw_power_cap.  Returns (peak, kind)."""
    capped = bool(clocks) and "sw_power_cap" in (clocks.get("reasons") or [])
    if window_ms >= SUSTAINED_WINDOW_MS or capped:
        why = "power cap active" if capped else f"{window_ms / 1e3:.1f} s window"
        return peaks["sustained"] * ratio, f"bf16_tflops_sustained ({peaks['source']}; {why})"
    return (peaks["burst"] * ratio,
            f"bf16_tflops burst ({peaks['source']}; {window_ms:.0f} ms window, power cap not engaged)")


def clock_peak(clocks, ratio=1.0):
    """Dense tensor peak at the SM clock sampled during the timed region
    (148 SMs x 8192 BF16 FLOP/clk x median MHz), in TFLOP/s; None if no sample."""
    if not clocks or not clocks.get("sm_mhz"):
        return None
    return SMS * DENSE_BF16_FLOP_PER_CLK_SM * clocks["sm_mhz"] * 1e6 * ratio / 1e12


# The sources each timed kernel is built from: a recorded ncu capture stays
# attached to exactly this code.
# the sources a kernel's device code is compiled from (tmap.h is host-side
# tensor-map encoding; the box shapes it is given live in the kernel files)
KERNEL_SOURCES = {
    "fwd": ("attn_fwd.cu", "sm100.cuh", "exp2.cuh", "host_common.h"),
    "bwd": ("attn_bwd.cu", "sm100.cuh", "exp2.cuh", "host_common.h"),
}


def kernel_source_hash(kind="fwd"):
    """Hash of a kernel's CUDA sources with comments and whitespace removed."""
    import re
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "exact_attention_152_b200", "csrc")
    for name in KERNEL_SOURCES[kind]:
        with open(os.path.join(csrc, name)) as f:
            src = f.read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        src = "".join(src.split())
        h.update(name.encode() + b"\0" + src.encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload_name, kind="fwd"):
    """DRAM bytes per launch of the timed kernel from a committed ncu summary,
    if it was taken on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    e = rec.get(f"{kind}:{workload_name}")
    if not e or e.get("kernel_src_sha") != kernel_source_hash(kind):
        return None
    return e.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# nvidia-smi clock sampling during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi samples every 20 ms while a region is timed.  Each sample
    carries nvidia-smi's own timestamp, and the report uses the samples taken
    within 60 ms of the timed region (all samples if none falls there)."""
    FIELDS = ["timestamp", "clocks.sm", "clocks.max.sm", "power.draw", "utilization.gpu",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    INTERVAL_MS = 20
    MARGIN_S = 0.06

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="clocks", suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={','.join(self.FIELDS)}",
                 "--format=csv,noheader,nounits", "-lms", str(self.INTERVAL_MS)],
                stdout=self.out, stderr=subprocess.DEVNULL)
            # nvidia-smi's first start on a fresh box can take seconds: wait for
            # its first row, so a short timed region is not over before sampling
            t0 = time.time()
            while time.time() - t0 < 15.0 and os.path.getsize(self.path) == 0 \
                    and self.proc.poll() is None:
                time.sleep(0.01)
        except Exception:
            self.proc = None

    def mark_start(self):
        self.t0 = datetime.datetime.now()

    def mark_end(self):
        self.t1 = datetime.datetime.now()
        time.sleep(2 * self.INTERVAL_MS / 1e3)  # a sample after the region's end

    @staticmethod
    def parse(lines, t0=None, t1=None, margin_s=0.06):
        """Summary of nvidia-smi CSV rows (the FIELDS order); rows stamped
        within margin_s of [t0, t1] when there are any."""
        rows = []
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != len(ClockSampler.FIELDS):
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f")
                rows.append((ts, float(parts[1]), float(parts[2]), float(parts[3]), float(parts[4]),
                             parts[5:]))
            except ValueError:
                continue
        if not rows:
            return None
        sel = rows
        if t0 is not None and t1 is not None:
            m = datetime.timedelta(seconds=margin_s)
            near = [r for r in rows if t0 - m <= r[0] <= t1 + m]
            sel = near or rows
        reasons = sorted({ClockSampler.REASONS[i] for r in sel for i, s in enumerate(r[5])
                          if s.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[1] for r in sel),
                "sm_max_mhz": max(r[2] for r in sel),
                "power_w_max": max(r[3] for r in sel),
                "samples": len(sel), "samples_in_window": len(sel) if sel is not rows else 0,
                "reasons": reasons}

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        with open(self.path) as f:
            lines = f.readlines()
        os.unlink(self.path)
        return self.parse(lines, self.t0, self.t1, self.MARGIN_S)


def colmask_launches(w, Hm=1):
    """Kernels one attn_fwd_colmask call launches with a workspace of
    attn_colmask_workspace_size bytes: the mask summaries, the CTA plan when it
    fits (at most 8192 (mask row, 256-row block) units, mask rows x (key
    blocks + 1) at most 4096, Nq <= 4 Nk), and the attention kernel."""
    units = w.B * Hm * math.ceil(w.Nq / 256)
    n_kb = math.ceil(w.Nk / 128)
    fits = 0 < units <= 8192 and w.B * Hm * (n_kb + 1) <= 4096 and w.Nq <= 4 * w.Nk
    return 3 if fits else 2


def bwd_colmask_launches(w):
    """Kernels one attn_bwd_colmask call launches with a workspace of
    attn_bwd_colmask_workspace_size bytes: row sums, mask summaries, the CTA
    plan when it fits (at most 8192 CTAs, groups of key/value heads x (query
    tiles per CTA + 1) at most 4096 bins), the main kernel, dQ rounding."""
    hkv, group = w.kv_heads, w.H // w.kv_heads
    n_kb, n_qt = math.ceil(w.Nk / 128), math.ceil(w.Nq / 128)
    per_kv = group * w.Nq * w.d * 8
    g = max([c for c in range(1, hkv + 1) if hkv % c == 0 and c * per_kv <= 48 << 20] or [1])
    units = w.B * hkv * n_kb
    bins = math.ceil(w.B * hkv / g) * (group * n_qt + 1)
    return 5 if units <= 8192 and bins <= 4096 else 4


# ---------------------------------------------------------------------------
# End-to-end timing with host buffers
# ---------------------------------------------------------------------------
E2E_PATTERN = ("two buffer slots on three streams: step i+1's host-to-device copies overlap "
               "step i's call and its device-to-host read (PCIe is full duplex)")


def pipelined_e2e(comp, slots, n_steps, warmup=2):
    """Device milliseconds for n_steps end-to-end steps.  Each step copies its
    inputs from pinned host memory (upload stream), runs the call on `comp`
    (the stream the C-ABI call is given) and reads its results back to pinned
    host memory (download stream).  Steps alternate between two slots, each a
    dict with 'h2d' [(device dst, host src)], 'run' (issues the call on comp)
    and 'd2h' [(host dst, device src)]; a slot's inputs are rewritten only
    after the call two steps back has read them, and its outputs only after
    their read-back."""
    import torch
    up, down = torch.cuda.Stream(comp.device), torch.cuda.Stream(comp.device)
    in_free, out_free = [None, None], [None, None]
    last = [None]

    def step(i):
        s = i % 2
        sl = slots[s]
        if in_free[s] is not None:
            up.wait_event(in_free[s])
        with torch.cuda.stream(up):
            for dst, src in sl["h2d"]:
                dst.copy_(src, non_blocking=True)
        ready = torch.cuda.Event()
        ready.record(up)
        comp.wait_event(ready)
        if out_free[s] is not None:
            comp.wait_event(out_free[s])
        sl["run"]()
        done = torch.cuda.Event()
        done.record(comp)
        in_free[s] = done
        down.wait_event(done)
        with torch.cuda.stream(down):
            for dst, src in sl["d2h"]:
                dst.copy_(src, non_blocking=True)
        back = torch.cuda.Event()
        back.record(down)
        out_free[s] = back
        last[0] = back

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize(comp.device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    up.wait_event(e0)
    for i in range(n_steps):
        step(warmup + i)
    comp.wait_event(last[0])
    e1.record(comp)
    torch.cuda.synchronize(comp.device)
    return e0.elapsed_time(e1)


# ---------------------------------------------------------------------------
# CPU oracle timing (baseline / reference arm)
# ---------------------------------------------------------------------------
def oracle_units(w):
    """The oracle's units of work for a workload, one (batch, head) or one
    (sequence, head) at a time: yields (tag, Nq, Nk, key/value loader)."""
    from exact_attention_152_b200 import inputs
    if w.packed:
        kvh = w.H // w.kv_heads
        for s, n in enumerate(w.seqlens):
            if n == 0:
                continue
            for h in range(w.H):
                yield (s, h), n, n, (lambda s=s, h=h: tuple(
                    w.to_f64(x, w.seq_head_bits(x, s, h // kvh)) for x in "kv"))
    else:
        for bh in range(w.B * w.H):
            yield bh, w.Nq, w.Nk, (lambda bh=bh: tuple(
                w.to_f64(x, w.head_bits(x, w.kv_head_of(bh))) for x in "kv"))


def time_oracle_rows(w, n_rows, seed_off, keep=None):
    """Time the oracle on n_rows seeded query rows, taken unit by unit (all rows
    of a head, then the next) so large samples span several heads.  keep: a
    list that receives (unit tag, rows, O, LSE) of every unit."""
    import oracle
    from exact_attention_152_b200 import inputs, masks
    from exact_attention_152_b200.workloads import visible_keys
    tot_t, tot_f, done, units = 0.0, 0.0, 0, 0
    wl, wr = w.band
    cols_all = w.colmask_array() if w.colmask else None
    for i, (tag, nq, nk, load_kv) in enumerate(oracle_units(w)):
        if done >= n_rows:
            break
        k, v = load_kv()
        rows = inputs.sample_rows(w.seed + seed_off, i, nq, min(nq, n_rows - done))
        if w.packed:
            q = w.to_f64("q", w.seq_head_bits("q", tag[0], tag[1], rows))
        else:
            q = w.to_f64("q", w.q_rows_bits(tag, rows))
        if cols_all is not None:
            cols = cols_all[tag // w.H, 0]
            t0 = time.perf_counter()
            res = oracle.attn_rows_colmask(q, rows, k, v, w.scale, w.causal, cols)
            tot_t += time.perf_counter() - t0
            tot_f += 4.0 * w.d * float(masks.visible_per_row(cols, rows, w.causal).sum())
        else:
            t0 = time.perf_counter()
            res = oracle.attn_rows_window(q, rows, k, v, w.scale, wl, wr)
            tot_t += time.perf_counter() - t0
            tot_f += 4.0 * w.d * float(visible_keys(rows, nk, wl, wr).sum())
        if keep is not None:
            keep.append((tag, rows) + tuple(res))
        done += len(rows)
        units += 1
    return tot_t, tot_f, done, units


def total_rows(w):
    return (w.total if w.packed else w.B * w.Nq) * w.H


def calibrate_rows(w, seconds):
    dt, _, n, _ = time_oracle_rows(w, 256, 1000)
    return max(16, min(total_rows(w), int(n * seconds / max(dt, 1e-6))))


def cpu_baseline(w, seconds, o_gpu=None, lse_gpu=None):
    """The oracle timed on sampled rows; with the GPU's O and LSE of the same
    inputs (host arrays in the workload's layout) the same rows also give the
    errors of the GPU result."""
    import oracle
    n = calibrate_rows(w, seconds)
    units = []
    dt, flops, n, heads = time_oracle_rows(w, n, 2000, keep=units if o_gpu is not None else None)
    out = {"value": flops / dt / 1e12, "unit": UNIT, "cores": oracle.default_threads(),
           "kind": "oracle",
           "sample": f"{n} seeded query rows over {heads} head(s) of {w.name} (visible keys "
                     f"of {mask_words(w)}), fp64, {dt:.1f} s of oracle time; "
                     f"value = those rows' algorithmic FLOPs / time"}
    if o_gpu is not None:
        eo, el = [], []
        for tag, rows, o_ref, l_ref in units:
            if w.packed:
                s_, h_ = tag
                g = int(w.cu_seqlens[s_]) + rows
                og, lg = o_gpu[g, h_], lse_gpu[h_, g]
            else:
                b_, h_ = divmod(tag, w.H)
                og, lg = o_gpu[b_, h_, rows], lse_gpu[b_, h_, rows]
            eo.append(np.abs(og.astype(np.float64) - o_ref).ravel())
            both = np.isneginf(lg) & np.isneginf(l_ref)
            el.append(np.abs(np.where(both, 0.0, lg) - np.where(both, 0.0, l_ref)))
        eo, el = np.concatenate(eo), np.concatenate(el)
        out["parity"] = {"rows": int(n), "max_abs_o": float(eo.max()), "mean_abs_o": float(eo.mean()),
                         "max_abs_lse": float(el.max()),
                         "bound": ("E4M3 inputs: the per-element bound of the FP8 parity tests" if w.fp8 else
                                   "max|dO| <= 1e-2, mean|dO| <= 1e-3, max|dLSE| <= 1e-3")}
    return out


def mask_words(w):
    if w.colmask:
        return f"column-interval document mask, documents of {w.docs[0]}..{w.docs[1]} tokens" + \
            (", causal" if w.causal else "")
    return f"band {w.band}"


def workload_config(w, n_gpus):
    rows_q = w.total if w.packed else w.B * w.Nq
    rows_k = w.total if w.packed else w.B * w.Nk
    qkv_bytes = (w.H * rows_q + 2 * w.kv_heads * rows_k) * w.d * 2
    cfg = {"workload": w.name, "B": w.B, "H": w.H, "Hkv": w.kv_heads, "Nq": w.Nq, "Nk": w.Nk, "d": w.d,
           "causal": w.causal, "band": list(w.band), "scale": w.scale, "seed": w.seed,
           "per_gpu_problem": True, "global_batch": w.B * n_gpus,
           "l2": f"inputs {qkv_bytes / 1e6:.0f} MB {'>' if qkv_bytes > L2_BYTES else '<='} "
                 f"126 MB L2; not flushed between steps",
           "parallelism": f"independent problem per GPU x{n_gpus}"}
    if w.colmask:
        cfg.update({"mask": mask_words(w), "mask_layout": "int32 [B, 1, Nk, 4]",
                    "doc_lengths": [w.doc_lengths(b) for b in range(w.B)]})
    if w.packed:
        cfg.update({"layout": "packed [total, H, d]", "num_seqs": len(w.seqlens),
                    "total_tokens": w.total, "seqlen_min": min(w.seqlens),
                    "seqlen_max": max(w.seqlens)})
    return cfg


def run_reference_bwd(args, w, per_step):
    """Reference arm of --pass bwd: the oracle's backward, each step on the
    first n query rows of one head against all its keys (n sized to about
    per_step seconds), in the same metric (2.5x the forward's FLOPs)."""
    import oracle
    for _ in range(args.warmup):
        bwd_cpu_baseline(w, per_step)
    vals, secs = [], []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        r = bwd_cpu_baseline(w, per_step)
        secs.append(time.perf_counter() - t0)
        vals.append(r["value"])
    value = statistics.mean(vals)
    line = {
        "impl": "reference", "metric": METRIC_BWD, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.mean(secs) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": dict(workload_config(w, 1), **{"pass": "bwd"}),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": r["sample"]},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def bwd_launch_name(w):
    if w.colmask:
        return "attn_bwd_colmask"
    if w.packed:
        return "attn_bwd_varlen"
    return "attn_bwd_window" if w.window is not None else "attn_bwd"


def launch_name(w):
    if w.colmask:
        return "attn_fwd_colmask"
    if w.fp8:
        return "attn_fwd_fp8"
    if w.packed:
        return "attn_fwd_varlen"
    if w.window is not None:
        return "attn_fwd_window"
    return "attn_fwd_gqa" if w.kv_heads != w.H else "attn_fwd"


def run_reference(args):
    rank, world, _ = dist_env()
    from exact_attention_152_b200.workloads import HEADLINE, WORKLOADS
    if world > 1 and rank != 0:
        return 0
    import oracle
    w = WORKLOADS[args.workload or HEADLINE]
    budget = 150.0  # seconds for warmup + timed steps together
    per_step = budget / max(1, args.steps + args.warmup)
    if args.which == "bwd":
        return run_reference_bwd(args, w, per_step)
    n = calibrate_rows(w, per_step)
    for i in range(args.warmup):
        time_oracle_rows(w, n, 3000 + i)
    tot_t, tot_f = 0.0, 0.0
    for i in range(args.steps):
        dt, fl, n, _ = time_oracle_rows(w, n, 5000 + i)
        tot_t += dt
        tot_f += fl
    value = tot_f / tot_t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_t / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, 1),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.default_threads(), "kind": "oracle",
                         "sample": f"each step: {n} seeded query rows (head by head, visible keys of {mask_words(w)}), fp64"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------
def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    from exact_attention_152_b200 import binding, parallel
    from exact_attention_152_b200.workloads import HEADLINE, WORKLOADS

    rank, world, local_rank = dist_env()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        parallel.init("nccl", timeout_s=120, device=dev)
    w = WORKLOADS[args.workload or HEADLINE]
    peaks = load_peaks()

    # inputs: the workload's seeded BF16 tensors, resident in HBM
    host = {x: w.tensor_bits(x) for x in "qkv"}

    def as_tensor(bits):
        if w.fp8:
            return torch.from_numpy(bits)  # E4M3 codes, one byte each
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)

    q, k, v = (as_tensor(host[x]).to(dev) for x in "qkv")
    if w.packed:
        o = torch.empty((w.total, w.H, w.d), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((w.H, w.total), dtype=torch.float32, device=dev)
        host_cu = torch.from_numpy(w.cu_seqlens)
        cu = host_cu.to(dev)
    else:
        o = torch.empty((w.B, w.H, w.Nq, w.d), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=dev)
        host_cu = cu = None
    if w.colmask:
        host_mask = torch.from_numpy(w.colmask_array())
        mask = host_mask.to(dev)
        ws_bytes = binding.attn_colmask_workspace_size(w.B, 1, w.Nk)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    else:
        host_mask = mask = None
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    knobs = args.exp_mode is not None or args.threshold is not None or args.count_rescales
    thr = 8.0 if args.threshold is None else args.threshold
    em = 1 if args.exp_mode is None else args.exp_mode
    if knobs and (w.packed or w.window is not None or w.kv_heads != w.H or w.fp8 or w.colmask):
        raise SystemExit("--exp-mode/--threshold apply to dense workloads without a band only")

    def launch(qp=q, kp=k, vp=v, op=o, lp=lse, cp=cu, mp=mask):
        if w.colmask:
            rc = binding.attn_fwd_colmask(qp.data_ptr(), kp.data_ptr(), vp.data_ptr(), op.data_ptr(),
                                          lp.data_ptr(), w.B, w.H, w.kv_heads, w.Nq, w.Nk, w.d,
                                          w.scale, int(w.causal), mp.data_ptr(), 1, ws.data_ptr(),
                                          ws_bytes, sh)
        elif w.fp8:
            rc = binding.attn_fwd_fp8(qp.data_ptr(), kp.data_ptr(), vp.data_ptr(), op.data_ptr(),
                                      lp.data_ptr(), w.B, w.H, w.kv_heads, w.Nq, w.Nk, w.d, w.scale,
                                      *w.descale, int(w.causal), sh)
        elif w.packed:
            rc = binding.attn_fwd_varlen(qp.data_ptr(), kp.data_ptr(), vp.data_ptr(), op.data_ptr(),
                                         lp.data_ptr(), cp.data_ptr(), cp.data_ptr(), len(w.seqlens),
                                         max(w.seqlens), w.total, w.total, w.H, w.kv_heads, w.d,
                                         w.scale, w.band[0], w.band[1], sh)
        elif w.window is not None:
            rc = binding.attn_fwd_window(qp.data_ptr(), kp.data_ptr(), vp.data_ptr(), op.data_ptr(),
                                         lp.data_ptr(), w.B, w.H, w.kv_heads, w.Nq, w.Nk, w.d,
                                         w.scale, w.band[0], w.band[1], sh)
        elif w.kv_heads != w.H:
            rc = binding.attn_fwd_gqa(qp.data_ptr(), kp.data_ptr(), vp.data_ptr(), op.data_ptr(),
                                      lp.data_ptr(), w.B, w.H, w.kv_heads, w.Nq, w.Nk, w.d, w.scale,
                                      int(w.causal), sh)
        elif knobs:
            rc = binding.attn_fwd_config(qp.data_ptr(), kp.data_ptr(), vp.data_ptr(), op.data_ptr(),
                                         lp.data_ptr(), w.B, w.H, w.Nq, w.Nk, w.d, w.scale,
                                         int(w.causal), thr, em, None, sh)
        else:
            rc = binding.attn_fwd(qp.data_ptr(), kp.data_ptr(), vp.data_ptr(), op.data_ptr(),
                                  lp.data_ptr(), w.B, w.H, w.Nq, w.Nk, w.d, w.scale, int(w.causal), sh)
        binding.check(rc, "attn_fwd")

    # one checked launch before anything is timed
    launch()
    binding.check(binding.attn_status_sync(sh), "first launch")
    for _ in range(args.warmup):
        launch()
    binding.check(binding.attn_status_sync(sh), "warm-up")
    assert bool(torch.isfinite(o.float()).all()), "non-finite output"

    gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(gpu_id)
    K = args.steps
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(K + 1)]
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.mark_start()
    evs[0].record(stream)
    for i in range(K):
        launch()
        evs[i + 1].record(stream)
    torch.cuda.synchronize(dev)
    sampler.mark_end()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    binding.check(binding.attn_status_sync(sh), "timed region")
    total_ms = evs[0].elapsed_time(evs[K])
    per_launch = [evs[i].elapsed_time(evs[i + 1]) for i in range(K)]
    kernel_ms = sum(per_launch) / K
    total_ms, kernel_ms = parallel.max_over_ranks([total_ms, kernel_ms], dev)
    value = world * w.flops * K / (total_ms / 1e3) / 1e12
    achieved = w.flops / (kernel_ms / 1e3) / 1e12

    # end to end through the public API: pinned host inputs -> H2D, attn_fwd, D2H
    hq, hk, hv = (as_tensor(host[x]).pin_memory() for x in "qkv")
    hc = host_cu.pin_memory() if w.packed else None
    hm = host_mask.pin_memory() if w.colmask else None
    KE = args.e2e_steps
    slots = []
    for s_ in range(2):
        qd, kd, vd = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        od, ld = (o, lse) if s_ == 0 else (torch.empty_like(o), torch.empty_like(lse))
        cd = torch.empty_like(cu) if w.packed else None
        md = torch.empty_like(mask) if w.colmask else None
        ho = torch.empty(o.shape, dtype=torch.bfloat16).pin_memory()
        hl = torch.empty(lse.shape, dtype=torch.float32).pin_memory()
        h2d_pairs = [(qd, hq), (kd, hk), (vd, hv)] + ([(cd, hc)] if w.packed else []) + \
            ([(md, hm)] if w.colmask else [])
        slots.append({"h2d": h2d_pairs, "d2h": [(ho, od), (hl, ld)],
                      "run": (lambda a=(qd, kd, vd, od, ld, cd, md): launch(*a))})
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    te_ms = pipelined_e2e(stream, slots, KE)
    if world > 1:
        dist.barrier()
    binding.check(binding.attn_status_sync(sh), "e2e region")
    # the results read back through both slots equal the device-resident one
    for sl in slots:
        for h_, d_ in zip((sl["d2h"][0][0], sl["d2h"][1][0]), (o, lse)):
            assert torch.equal(h_.view(torch.int16) if h_.dtype == torch.bfloat16 else h_,
                               d_.cpu().view(torch.int16) if d_.dtype == torch.bfloat16 else d_.cpu()), \
                "end-to-end read-back differs from the device result"
    (te_ms,) = parallel.max_over_ranks([te_ms], dev)
    e2e_value = world * w.flops * KE / (te_ms / 1e3) / 1e12
    h2d = sum(x.numel() * x.element_size()
              for x in (hq, hk, hv) + ((hc,) if w.packed else ()) + ((hm,) if w.colmask else ()))
    d2h = o.numel() * o.element_size() + lse.numel() * lse.element_size()

    # rescale events of one launch (outside the timed region): rows whose
    # reference max moved at a KV step after their first
    rescales = None
    if args.count_rescales:
        cnt = torch.zeros(1, dtype=torch.int64, device=dev)
        rc = binding.attn_fwd_config(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                     w.B, w.H, w.Nq, w.Nk, w.d, w.scale, int(w.causal), thr, em,
                                     cnt.data_ptr(), sh)
        binding.check(rc, "attn_fwd_config")
        binding.check(binding.attn_status_sync(sh), "rescale count")
        n = int(cnt.item())
        rows = w.B * w.H * w.Nq
        # KV steps after the first, summed over rows: a CTA of 256 query rows
        # visits KV tiles of 128 keys up to its last row's (causal) or all
        n_all = (w.Nk + 127) // 128
        steps = 0.0
        for r0 in range(0, w.Nq, 256):
            r1 = min(r0 + 256, w.Nq)
            n_kv = min((r1 - 1) // 128 + 1, n_all) if w.causal else n_all
            steps += (r1 - r0) * (n_kv - 1)
        steps *= w.B * w.H
        rescales = {"threshold": thr, "events": n, "rows": rows, "per_row": n / rows,
                    "fraction_of_row_steps": n / steps if steps else 0.0}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, args.cpu_seconds, o.float().cpu().numpy(), lse.cpu().numpy())

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    # E4M3 contractions: the measured BF16 peak times the nominal FP8 / BF16
    # dense ratio (4.5 / 2.25 PFLOP/s)
    ratio = 2.0 if w.fp8 else 1.0
    peak, peak_kind = pick_peak(peaks, total_ms, clocks, ratio)
    cpk = clock_peak(clocks, ratio)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": total_ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3" if w.fp8 else "bf16",
        "data": "synthetic",
        "config": workload_config(w, world),
        "pct_of_dense_spec": 100.0 * value / world / (SPEC_DENSE_BF16_TFLOPS * ratio),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT,
                     "frac": achieved / peak, "traffic": recorded_traffic(w.name, "fwd"),
                     "peak_kind": peak_kind + (" x 2 (nominal E4M3/BF16 dense ratio)" if w.fp8 else ""),
                     "frac_of_burst": achieved / (peaks["burst"] * ratio),
                     "frac_of_sustained": achieved / (peaks["sustained"] * ratio),
                     "clock_peak": cpk,
                     "frac_of_clock_peak": achieved / cpk if cpk else None,
                     "frac_of_spec": achieved / (SPEC_DENSE_BF16_TFLOPS * ratio),
                     "algorithmic_flops_per_launch": w.flops,
                     "timed_window": ("mask-summary + CTA-plan + attention kernels" if w.colmask
                                      else "attention kernel")},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": KE, "pattern": E2E_PATTERN, "path": f"pinned host Q/K/V{' + offsets' if w.packed else ''}"
                        f"{' + mask' if w.colmask else ''} -> H2D -> "
                        f"{launch_name(w)} (C-ABI) -> D2H of O and LSE"},
        # attn_fwd_colmask launches the mask summaries (and, when it fits, the
        # CTA plan) before the attention kernel
        "gpu_launches": colmask_launches(w) * K if w.colmask else K,
        "clocks": clocks,
        "kernel_src_sha": kernel_source_hash("fwd"),
    }
    if knobs:
        line["config"]["rescale_threshold"] = thr
        line["config"]["exp_mode"] = em
    if rescales is not None:
        line["rescale_events"] = rescales
    print(json.dumps(line), flush=True)
    return 0


def bwd_cpu_baseline(w, seconds):
    """The oracle's backward on the first n query rows of one head (all of its
    keys), n sized to about `seconds` of CPU time; FLOPs counted as 2.5x the
    forward's 4*d per visible pair."""
    import oracle
    from exact_attention_152_b200 import inputs
    from exact_attention_152_b200.workloads import visible_keys
    wl, wr = w.band
    if w.packed:  # sequence 0, head 0
        nq = nk = w.seqlens[0]
        k, v = (inputs.bf16_bits_to_f64(w.seq_head_bits(x, 0, 0)) for x in "kv")
        q_of = lambda rows: w.seq_head_bits("q", 0, 0, rows)  # noqa: E731
        flat = lambda rows: (rows[:, None] * w.H) * w.d + np.arange(w.d)[None, :]  # noqa: E731
    else:
        nq, nk = w.Nq, w.Nk
        k, v = (inputs.bf16_bits_to_f64(w.head_bits(x, w.kv_head_of(0))) for x in "kv")
        q_of = lambda rows: w.q_rows_bits(0, rows)  # noqa: E731
        flat = lambda rows: rows[:, None] * w.d + np.arange(w.d)[None, :]  # noqa: E731
    cols = w.colmask_array()[0, 0] if w.colmask else None
    n, dt = 64, 0.0
    while True:
        rows = np.arange(min(n, nq), dtype=np.int64)
        q = inputs.bf16_bits_to_f64(q_of(rows))
        g = inputs.bf16_bits_to_f64(inputs.gen_bf16_at(w.seed + 1, "q", flat(rows)))
        t0 = time.perf_counter()
        if cols is not None:
            oracle.attn_bwd_colmask_head(q, k, v, g, w.scale, w.causal, cols)
        else:
            oracle.attn_bwd_head(q, k, v, g, w.scale, wl, wr)
        dt = time.perf_counter() - t0
        if dt > seconds / 4 or n >= nq:
            break
        n = min(nq, n * 4)
    if cols is not None:
        from exact_attention_152_b200 import masks
        pairs = float(masks.visible_per_row(cols, rows, w.causal).sum())
    else:
        pairs = float(visible_keys(rows, nk, wl, wr).sum())
    flops = 2.5 * 4.0 * w.d * pairs
    where = "sequence 0, head 0" if w.packed else "head 0"
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"backward of the first {len(rows)} query rows of {where} of {w.name} against "
                      f"all its keys, fp64, one thread, {dt:.1f} s"}


def run_ours_bwd(args):
    """The backward pass: each step is one attn_bwd call (row sums, main
    kernel, dQ rounding) over the whole workload, with O and LSE from one
    forward call before timing."""
    import torch

    from exact_attention_152_b200 import binding, inputs
    from exact_attention_152_b200.workloads import HEADLINE, WORKLOADS

    rank, world, local_rank = dist_env()
    if world > 1:
        raise SystemExit("--pass bwd runs on one GPU")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = WORKLOADS[args.workload or HEADLINE]
    if w.fp8:
        raise SystemExit("--pass bwd: no backward for E4M3 workloads")
    peaks = load_peaks()
    host = {x: w.tensor_bits(x) for x in "qkv"}
    host["do"] = inputs.gen_bf16(w.seed + 1, "q", w.shape("q"))
    to_dev = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)  # noqa: E731
    q, k, v, do = (to_dev(host[x]) for x in ("q", "k", "v", "do"))
    mask = None
    if w.packed:
        cu = torch.from_numpy(w.cu_seqlens).to(dev)
        o, lse = binding.fwd_varlen(q, k, v, cu, cu, max(w.seqlens), scale=w.scale, window=w.band)
        ws_bytes = binding.attn_bwd_workspace_size(1, w.H, w.total, w.d)
    elif w.colmask:
        cu = None
        mask = torch.from_numpy(w.colmask_array()).to(dev)
        o, lse = binding.fwd_colmask(q, k, v, mask, causal=w.causal, scale=w.scale)
        ws_bytes = binding.attn_bwd_colmask_workspace_size(w.B, w.H, w.Nq, w.d, 1, w.Nk)
    else:
        cu = None
        o, lse = binding.fwd(q, k, v, causal=w.causal, scale=w.scale, window=w.window)
        ws_bytes = binding.attn_bwd_workspace_size(w.B, w.H, w.Nq, w.d)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)

    def launch(ins=(q, k, v, o, do, lse, cu if w.packed else mask), outs=(dq, dk, dv)):
        ptrs = [t.data_ptr() for t in ins[:6]] + [t.data_ptr() for t in outs]
        if w.colmask:
            rc = binding.attn_bwd_colmask(*ptrs, ws.data_ptr(), ws_bytes, w.B, w.H, w.kv_heads, w.Nq,
                                          w.Nk, w.d, w.scale, int(w.causal), ins[6].data_ptr(), 1, sh)
        elif w.packed:
            c = ins[6].data_ptr()
            rc = binding.attn_bwd_varlen(*ptrs, ws.data_ptr(), ws_bytes, c, c, len(w.seqlens),
                                         max(w.seqlens), w.total, w.total, w.H, w.kv_heads, w.d,
                                         w.scale, w.band[0], w.band[1], sh)
        elif w.window is not None:
            rc = binding.attn_bwd_window(*ptrs, ws.data_ptr(), ws_bytes, w.B, w.H, w.kv_heads,
                                         w.Nq, w.Nk, w.d, w.scale, w.band[0], w.band[1], sh)
        else:
            rc = binding.attn_bwd(*ptrs, ws.data_ptr(), ws_bytes, w.B, w.H, w.kv_heads, w.Nq, w.Nk,
                                  w.d, w.scale, int(w.causal), sh)
        binding.check(rc, "attn_bwd")

    launch()
    binding.check(binding.attn_status_sync(sh), "first launch")
    for _ in range(args.warmup):
        launch()
    binding.check(binding.attn_status_sync(sh), "warm-up")
    for t in (dq, dk, dv):
        assert bool(torch.isfinite(t.float()).all()), "non-finite gradient"
    flops = 2.5 * w.flops
    sampler = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid))
    K = args.steps
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(K + 1)]
    sampler.start()
    torch.cuda.synchronize(dev)
    sampler.mark_start()
    evs[0].record(stream)
    for i in range(K):
        launch()
        evs[i + 1].record(stream)
    torch.cuda.synchronize(dev)
    sampler.mark_end()
    clocks = sampler.stop()
    binding.check(binding.attn_status_sync(sh), "timed region")
    total_ms = evs[0].elapsed_time(evs[K])
    call_ms = total_ms / K
    value = flops * K / (total_ms / 1e3) / 1e12

    # end to end: pinned host Q, K, V, O, dO, LSE -> H2D -> attn_bwd -> D2H dQ, dK, dV
    pin = lambda t: t.cpu().pin_memory()  # noqa: E731
    ins = (q, k, v, o, do, lse) + ((cu,) if w.packed else ()) + ((mask,) if w.colmask else ())
    h_in = [pin(t) for t in ins]
    slots = []
    for s_ in range(2):
        d_in = [torch.empty_like(t) for t in ins]
        d_out = (dq, dk, dv) if s_ == 0 else tuple(torch.empty_like(t) for t in (dq, dk, dv))
        h_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in d_out]
        args_in = tuple(d_in) + ((None,) if not (w.packed or w.colmask) else ())
        slots.append({"h2d": list(zip(d_in, h_in)), "d2h": list(zip(h_out, d_out)),
                      "run": (lambda a=args_in, o_=d_out: launch(a, o_))})
    te_ms = pipelined_e2e(stream, slots, args.e2e_steps)
    binding.check(binding.attn_status_sync(sh), "e2e region")
    # dK and dV read back through both slots equal the device-resident ones
    # (dQ's fp32 reductions may land in another order)
    for sl in slots:
        for (h_, _), d_ in zip(sl["d2h"][1:], (dk, dv)):
            assert torch.equal(h_.view(torch.int16), d_.cpu().view(torch.int16)), \
                "end-to-end read-back differs from the device result"
    e2e_value = flops * args.e2e_steps / (te_ms / 1e3) / 1e12
    cpu = None if args.no_cpu_baseline else bwd_cpu_baseline(w, args.cpu_seconds)
    peak, peak_kind = pick_peak(peaks, total_ms, clocks)
    cpk = clock_peak(clocks)
    achieved = flops / (call_ms / 1e3) / 1e12
    line = {
        "metric": METRIC_BWD, "value": value, "unit": UNIT, "n_gpus": 1, "steps": K,
        "warmup": args.warmup, "ms_per_step": call_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(workload_config(w, 1), **{"pass": "bwd", "dO": "N(0,1), seed + 1"}),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT,
                     "frac": achieved / peak, "traffic": recorded_traffic(w.name, "bwd"),
                     "peak_kind": peak_kind,
                     "frac_of_burst": achieved / peaks["burst"],
                     "frac_of_sustained": achieved / peaks["sustained"],
                     "clock_peak": cpk,
                     "frac_of_clock_peak": achieved / cpk if cpk else None,
                     "frac_of_spec_2250": achieved / SPEC_DENSE_BF16_TFLOPS,
                     "algorithmic_flops_per_launch": flops,
                     "timed": "the whole attn_bwd call: row sums + main kernel + dQ rounding"},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": UNIT,
                "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in h_in),
                "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in (dq, dk, dv)),
                "steps": args.e2e_steps, "pattern": E2E_PATTERN,
                "path": f"pinned host Q/K/V/O/dO/LSE{' + offsets' if w.packed else ''}"
                        f"{' + mask' if w.colmask else ''} -> H2D -> "
                        f"{bwd_launch_name(w)} (C-ABI) -> D2H of dQ/dK/dV"},
        # row sums, main kernel, dQ rounding (+ the mask summaries for column intervals)
        "gpu_launches": (bwd_colmask_launches(w) if w.colmask else 3) * K,
        "clocks": clocks,
        "kernel_src_sha": kernel_source_hash("bwd"),
    }
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.which == "bwd":
        return run_ours_bwd(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
