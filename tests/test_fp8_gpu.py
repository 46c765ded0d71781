"""FP8 forward (attn_fwd_fp8) against the fp64 oracle on the dequantized inputs.

Tolerance, from the arithmetic: Q.K^T of E4M3 codes is exact in the FP32
accumulator up to summation order; each weight P is rounded to E4M3 before
P.V.  E4M3 keeps 3 mantissa bits, so a normal weight is off by at most 2^-4 of
itself, and a subnormal one (below 2^-6) by at most 2^-10.  The kernel carries
P scaled by 2^4 relative to the row maximum (2^(4+delta) with 0 <= delta <= 4
under the lazy maximum), so with p_j = 2^4 exp(s_j - max s) the error of
O_ic is at most
    sum_j max(2^-4 p_j, 2^-10) |v_jc| / sum_j p_j  +  2^-8 |O_ic|
(the last term: BF16 rounding of O and FP32 sums).  The test computes that
bound per element from the decoded inputs and asserts |dO| <= bound; LSE uses
the unrounded weights and keeps the BF16 path's 1e-3.
"""
import math

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

import harness  # noqa: E402
import oracle  # noqa: E402
from exact_attention_152_b200 import inputs  # noqa: E402

CASES = [
    # B, H, Hkv, Nq, Nk, causal, descale (q, k, v)
    (1, 2, 2, 128, 128, False, (1.0, 1.0, 1.0)),
    (1, 2, 2, 300, 300, True, (0.5, 0.25, 2.0)),
    (2, 4, 2, 1000, 1000, True, (1.0, 0.5, 1.0)),
    (1, 2, 1, 200, 517, False, (0.125, 1.0, 0.5)),
    (1, 3, 3, 2048, 2048, False, (1.0, 1.0, 1.0)),
]


def _run(q8, k8, v8, scale, descale, causal):
    import torch
    from exact_attention_152_b200 import binding
    q, k, v = (torch.from_numpy(np.ascontiguousarray(x)).cuda() for x in (q8, k8, v8))
    o, lse = binding.fwd_fp8(q, k, v, descale, causal=causal, scale=scale)
    assert binding.attn_status_sync(torch.cuda.current_stream().cuda_stream) == 0
    return o.float().cpu().numpy(), lse.cpu().numpy()


def _bound(qf, kf, vf, scale, causal, o_ref):
    """Per-element error bound for one head (see the module docstring)."""
    s = scale * (qf @ kf.T)
    if causal:
        s = np.where(np.tril(np.ones(s.shape, dtype=bool)), s, -np.inf)
    p = 16.0 * np.exp(s - s.max(1, keepdims=True))
    err = np.maximum(p * 2.0 ** -4, 2.0 ** -10) * (p > 0)
    return (err @ np.abs(vf)) / p.sum(1, keepdims=True) + 2.0 ** -8 * np.abs(o_ref) + 1e-6


@pytest.mark.parametrize("case", CASES, ids=[str(c[:6]) for c in CASES])
def test_fp8_parity(case):
    B, H, Hkv, Nq, Nk, causal, descale = case
    seed = 600 + Nq + H
    q8 = inputs.gen_e4m3(seed, "q", (B, H, Nq, 128))
    k8 = inputs.gen_e4m3(seed, "k", (B, Hkv, Nk, 128))
    v8 = inputs.gen_e4m3(seed, "v", (B, Hkv, Nk, 128))
    scale = float(np.float32(1 / math.sqrt(128)))
    o, lse = _run(q8, k8, v8, scale, descale, causal)
    g = H // Hkv
    worst = 0.0
    for b in range(B):
        for h in range(H):
            qf = inputs.e4m3_to_f64(q8[b, h]) * descale[0]
            kf = inputs.e4m3_to_f64(k8[b, h // g]) * descale[1]
            vf = inputs.e4m3_to_f64(v8[b, h // g]) * descale[2]
            rows = np.arange(Nq, dtype=np.int64)
            o_ref, l_ref = oracle.attn_rows(qf, rows, kf, vf, scale, causal)
            bound = _bound(qf, kf, vf, scale, causal, o_ref)
            err = np.abs(o[b, h].astype(np.float64) - o_ref)
            worst = max(worst, float((err / bound).max()))
            assert np.all(err <= bound), (b, h, float((err / bound).max()))
            assert np.abs(lse[b, h] - l_ref).max() <= harness.MAX_ABS_LSE
    print(case, "max err / bound", worst)


def test_fp8_uniform_weights_exact():
    """scale = 0: every weight is 2^4 exactly (representable), so O is the
    descaled mean of V up to FP32 sums and BF16 rounding, and LSE = log Nk."""
    B, H, N = 1, 2, 384
    q8 = inputs.gen_e4m3(650, "q", (B, H, N, 128))
    k8 = inputs.gen_e4m3(650, "k", (B, H, N, 128))
    v8 = inputs.gen_e4m3(650, "v", (B, H, N, 128))
    o, lse = _run(q8, k8, v8, 0.0, (1.0, 1.0, 0.5), False)
    for h in range(H):
        ref = 0.5 * inputs.e4m3_to_f64(v8[0, h]).mean(0)
        np.testing.assert_allclose(o[0, h], np.broadcast_to(ref, (N, 128)), rtol=2.0 ** -8, atol=1e-6)
    np.testing.assert_allclose(lse, math.log(N), rtol=0, atol=1e-5)


def test_fp8_workloads_sampled():
    """The FP8 bench workloads (B=2, H=16, N=8192, d=128, causal and not) on
    sampled rows with the same bound."""
    from exact_attention_152_b200.workloads import WORKLOADS
    for name in ("fp8_b2h16n8k_d128", "fp8_b2h16n8k_d128_causal"):
        w = WORKLOADS[name]
        q8, k8, v8 = (w.tensor_bits(x) for x in "qkv")
        o, lse = _run(q8, k8, v8, w.scale, w.descale, w.causal)
        for bh in (0, 17, 31):
            b, h = divmod(bh, w.H)
            rows = w.sampled_rows(bh)
            qf = w.to_f64("q", q8[b, h, rows])
            kf, vf = w.to_f64("k", k8[b, h]), w.to_f64("v", v8[b, h])
            o_ref, l_ref = oracle.attn_rows(qf, rows, kf, vf, w.scale, w.causal)
            s = w.scale * (qf @ kf.T)
            if w.causal:
                s = np.where(np.arange(w.Nk)[None, :] <= rows[:, None], s, -np.inf)
            p = 16.0 * np.exp(s - s.max(1, keepdims=True))
            bound = (np.maximum(p * 2.0 ** -4, 2.0 ** -10) * (p > 0)) @ np.abs(vf) / p.sum(1, keepdims=True) \
                + 2.0 ** -8 * np.abs(o_ref) + 1e-6
            err = np.abs(o[b, h, rows].astype(np.float64) - o_ref)
            assert np.all(err <= bound), (name, bh, float((err / bound).max()))
            assert np.abs(lse[b, h, rows] - l_ref).max() <= harness.MAX_ABS_LSE
