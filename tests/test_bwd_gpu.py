"""Backward pass (attn_bwd) against the fp64 oracle's chain rule.

The CUDA backward takes the CUDA forward's O and LSE (as a training step
would); the oracle differentiates the exact definition.  Tolerance, from the
arithmetic (harness.bwd_bound_head): every gradient element must lie within
2 * 2^-8 (twice the BF16 unit roundoff) times the magnitude sums of its own
rounding errors -- P or dS rounded to BF16 before a GEMM, the BF16 O inside
D = <dO, O>, the output's own rounding -- computed from the exact P in fp64.
The Frobenius-norm error must also stay below 1e-2 of the gradient's norm.
"""
import math

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

import harness  # noqa: E402
import oracle  # noqa: E402
from exact_attention_152_b200 import inputs  # noqa: E402

REL_FRO = 1e-2

CASES = [
    # B, H, Hkv, Nq, Nk, d, causal
    (1, 2, 2, 128, 128, 128, False),
    (1, 2, 2, 256, 256, 128, True),
    (2, 3, 3, 300, 300, 64, True),
    (1, 4, 2, 257, 257, 128, False),
    (1, 4, 1, 513, 513, 64, True),
    (1, 2, 2, 200, 517, 128, False),
    (1, 2, 2, 640, 130, 64, False),
    (1, 1, 1, 1, 1, 128, False),
    (2, 8, 2, 1024, 1024, 128, True),
]


def run_fwd_bwd(q_bits, k_bits, v_bits, do_bits, scale, causal):
    import torch
    from exact_attention_152_b200 import binding
    q, k, v, do = (harness.to_device_bf16(x) for x in (q_bits, k_bits, v_bits, do_bits))
    o, lse = binding.fwd(q, k, v, causal=causal, scale=scale)
    dq, dk, dv = binding.bwd(q, k, v, o, do, lse, causal=causal, scale=scale)
    assert binding.attn_status_sync(torch.cuda.current_stream().cuda_stream) == 0
    return tuple(x.float().cpu().numpy() for x in (dq, dk, dv))


def check_grads(got, ref, mags, label=""):
    """Norm-wise bound per gradient, and the element-wise bound of
    harness.check_grads_elementwise (mags: the magnitude sums).  A gradient
    that is zero in exact arithmetic (a band where every query sees one key:
    the softmax is constant) still carries fp32 rounding from P and
    D = <dO, O>; the floor of the norm bound is therefore 1e-4 of the largest
    gradient norm of the problem."""
    scale_nrm = max(np.linalg.norm(r) for r in ref)
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        g = g.astype(np.float64)
        err = np.linalg.norm(g - r)
        nrm = np.linalg.norm(r)
        print(label, name, "rel_fro", err / max(nrm, 1e-30))
        assert np.all(np.isfinite(g)), name
        assert err <= REL_FRO * nrm + 1e-4 * scale_nrm + 1e-6, (label, name, err, nrm)
    harness.check_grads_elementwise(got, ref, mags, label)


def band_mags(q, k, v, do, scale, wl, wr):
    """Magnitude sums of the element-wise bound for a key band (fp64 inputs)."""
    Nk = k.shape[2]
    return harness.bwd_bound_dense(q, k, v, do, scale, lambda b, h: harness.band_visible(wl, wr, Nk))


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_bwd_parity(case):
    B, H, Hkv, Nq, Nk, d, causal = case
    seed = 300 + Nq + Nk + d
    q = harness.random_bits(seed, (B, H, Nq, d), tensor="q")
    k = harness.random_bits(seed, (B, Hkv, Nk, d), tensor="k")
    v = harness.random_bits(seed, (B, Hkv, Nk, d), tensor="v")
    do = harness.random_bits(seed + 1, (B, H, Nq, d), tensor="q")
    scale = float(np.float32(1 / math.sqrt(d)))
    got = run_fwd_bwd(q, k, v, do, scale, causal)
    f = inputs.bf16_bits_to_f64
    ref = oracle.attn_bwd(f(q), f(k), f(v), f(do), scale, -1, 0 if causal else -1)
    mags = band_mags(f(q), f(k), f(v), f(do), scale, -1, 0 if causal else -1)
    check_grads(got, ref, mags, str(case))


def test_bwd_empty_sides():
    import torch
    from exact_attention_152_b200 import binding
    q = torch.randn(1, 2, 64, 64, device="cuda").bfloat16()
    k0 = torch.empty(1, 2, 0, 64, device="cuda", dtype=torch.bfloat16)
    o = torch.zeros_like(q)
    lse = torch.full((1, 2, 64), -math.inf, device="cuda")
    dq, dk, dv = binding.bwd(q, k0, k0, o, q, lse)
    torch.cuda.synchronize()
    assert torch.all(dq == 0) and dk.numel() == 0 and dv.numel() == 0
    k = torch.randn(1, 2, 50, 64, device="cuda").bfloat16()
    q0 = torch.empty(1, 2, 0, 64, device="cuda", dtype=torch.bfloat16)
    l0 = torch.empty(1, 2, 0, device="cuda")
    dq, dk, dv = binding.bwd(q0, k, k, q0, q0, l0)
    torch.cuda.synchronize()
    assert torch.all(dk == 0) and torch.all(dv == 0)


def test_bwd_repeatable_and_workspace_reuse():
    """Bitwise equal across calls except for the order of the fp32 dQ
    reductions, which may differ; dK and dV are exact repeats.  A reused,
    dirty workspace gives the same results."""
    import torch
    from exact_attention_152_b200 import binding
    B, H, N, d = 1, 4, 512, 128
    q, k, v, do = (harness.to_device_bf16(harness.random_bits(320, (B, H, N, d), tensor=t))
                   for t in ("q", "k", "v", "v"))
    o, lse = binding.fwd(q, k, v, causal=True)
    ws = torch.full((binding.attn_bwd_workspace_size(B, H, N, d),), 255, dtype=torch.uint8,
                    device="cuda")
    a = binding.bwd(q, k, v, o, do, lse, causal=True, workspace=ws)
    b = binding.bwd(q, k, v, o, do, lse, causal=True, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(a[1].view(torch.int16), b[1].view(torch.int16))
    assert torch.equal(a[2].view(torch.int16), b[2].view(torch.int16))
    assert torch.allclose(a[0].float(), b[0].float(), rtol=1e-2, atol=1e-3)


def test_bwd_workload_sampled():
    """Headline-sized causal backward (B=2, H=16, N=8192, d=128): the full
    oracle is too slow, so two heads are checked in full at N=8192."""
    import torch
    from exact_attention_152_b200 import binding
    B, H, N, d = 2, 16, 8192, 128
    seed = 330
    q = harness.random_bits(seed, (B, H, N, d), tensor="q")
    k = harness.random_bits(seed, (B, H, N, d), tensor="k")
    v = harness.random_bits(seed, (B, H, N, d), tensor="v")
    do = harness.random_bits(seed + 1, (B, H, N, d), tensor="q")
    scale = float(np.float32(1 / math.sqrt(d)))
    got = run_fwd_bwd(q, k, v, do, scale, True)
    f = inputs.bf16_bits_to_f64
    for b, h in [(0, 0), (1, 15)]:
        one = [f(x[b:b + 1, h:h + 1]) for x in (q, k, v, do)]
        ref = oracle.attn_bwd(*one, scale, -1, 0)
        check_grads(tuple(g[b:b + 1, h:h + 1] for g in got), ref, band_mags(*one, scale, -1, 0),
                    f"head {(b, h)}")


BAND_CASES = [
    # B, H, Hkv, Nq, Nk, d, (window_left, window_right)
    (1, 2, 2, 384, 384, 128, (63, 0)),        # causal sliding window
    (1, 2, 2, 300, 300, 64, (100, 50)),
    (1, 2, 2, 257, 257, 128, (0, 0)),          # diagonal only
    (1, 4, 2, 520, 520, 128, (-1, 10)),
    (1, 2, 2, 200, 517, 128, (10, 300)),       # Nq < Nk
    (1, 2, 2, 600, 100, 64, (50, 0)),          # Nq > Nk: rows >= 150 and some keys see nothing
    (2, 2, 1, 1024, 1024, 128, (255, 0)),
]


@pytest.mark.parametrize("case", BAND_CASES, ids=[str(c) for c in BAND_CASES])
def test_bwd_band_parity(case):
    import torch
    from exact_attention_152_b200 import binding
    B, H, Hkv, Nq, Nk, d, (wl, wr) = case
    seed = 340 + Nq + Nk + d + wl
    q = harness.random_bits(seed, (B, H, Nq, d), tensor="q")
    k = harness.random_bits(seed, (B, Hkv, Nk, d), tensor="k")
    v = harness.random_bits(seed, (B, Hkv, Nk, d), tensor="v")
    do = harness.random_bits(seed + 1, (B, H, Nq, d), tensor="q")
    scale = float(np.float32(1 / math.sqrt(d)))
    qd, kd, vd, dod = (harness.to_device_bf16(x) for x in (q, k, v, do))
    o, lse = binding.fwd(qd, kd, vd, scale=scale, window=(wl, wr))
    got = binding.bwd(qd, kd, vd, o, dod, lse, scale=scale, window=(wl, wr))
    assert binding.attn_status_sync(torch.cuda.current_stream().cuda_stream) == 0
    got = tuple(x.float().cpu().numpy() for x in got)
    f = inputs.bf16_bits_to_f64
    ref = oracle.attn_bwd(f(q), f(k), f(v), f(do), scale, wl, wr)
    check_grads(got, ref, band_mags(f(q), f(k), f(v), f(do), scale, wl, wr), str(case))


def test_bwd_band_limits_equal_causal_and_full_bitwise():
    """Band (-1, 0) is the causal backward and (-1, -1) the unmasked one, bit for
    bit for dK and dV (dQ: the fp32 reductions may reorder)."""
    import torch
    from exact_attention_152_b200 import binding
    B, H, N, d = 1, 4, 640, 128
    q, k, v, do = (harness.to_device_bf16(harness.random_bits(350, (B, H, N, d), tensor=t))
                   for t in ("q", "k", "v", "v"))
    for causal, band in ((True, (-1, 0)), (False, (-1, -1))):
        o, lse = binding.fwd(q, k, v, causal=causal)
        a = binding.bwd(q, k, v, o, do, lse, causal=causal)
        b = binding.bwd(q, k, v, o, do, lse, window=band)
        torch.cuda.synchronize()
        assert torch.equal(a[1].view(torch.int16), b[1].view(torch.int16))
        assert torch.equal(a[2].view(torch.int16), b[2].view(torch.int16))
        assert torch.allclose(a[0].float(), b[0].float(), rtol=1e-2, atol=1e-3)
