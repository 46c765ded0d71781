"""The backward's element-wise tolerance (harness.bwd_bound_head) against a
CPU model of the BF16 roundings it accounts for (no GPU).

The model differentiates the exact definition in fp64 but rounds, as the CUDA
backward does, P to BF16 before dV = P^T dO, the forward's O to BF16 inside
D = <dO, O>, dS to BF16 before dK and dQ, and every gradient to BF16.  Its
error must stay within the bound at factor 1 (the GPU tests allow 2), and
must use a fair part of it (the bound is not vacuous)."""
import math

import numpy as np
import pytest

import harness
import oracle
from exact_attention_152_b200 import inputs


def _bf16(x):
    return inputs.bf16_bits_to_f64(inputs.f32_to_bf16_bits(np.asarray(x, dtype=np.float32)))


def _model_bwd(q, k, v, do, scale, vis):
    s = np.where(vis, scale * (q @ k.T), -np.inf)
    m = s.max(axis=1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    e = np.where(vis, np.exp(s - m), 0.0)
    l = e.sum(axis=1, keepdims=True)
    p = e / np.where(l > 0, l, 1.0)
    o = _bf16(p @ v)                         # the forward's BF16 output
    dv = _bf16(_bf16(p).T @ do)
    dd = (do * o).sum(axis=1, keepdims=True)
    ds = _bf16(p * (do @ v.T - dd))
    return _bf16(scale * ds @ k), _bf16(scale * ds.T @ q), dv


@pytest.mark.parametrize("N,d,wl,wr,mult", [(96, 64, -1, 0, 1.0), (80, 128, -1, -1, 1.0),
                                             (64, 64, 15, 3, 4.0), (70, 64, -1, 0, 8.0)])
def test_bound_covers_bf16_model(N, d, wl, wr, mult):
    seed = 900 + N + d
    f = inputs.bf16_bits_to_f64
    q = f(harness.random_bits(seed, (1, 1, N, d), tensor="q", mult=mult))
    k, v = (f(harness.random_bits(seed, (1, 1, N, d), tensor=t)) for t in "kv")
    do = f(harness.random_bits(seed + 1, (1, 1, N, d), tensor="q"))
    scale = 1.0 / math.sqrt(d)
    vis = harness.band_visible(wl, wr, N)(0, N)
    got = _model_bwd(q[0, 0], k[0, 0], v[0, 0], do[0, 0], scale, vis)
    ref = [r[0, 0] for r in oracle.attn_bwd(q, k, v, do, scale, wl, wr)]
    mags = harness.bwd_bound_head(q[0, 0], k[0, 0], v[0, 0], do[0, 0], scale, harness.band_visible(wl, wr, N))
    worst = 0.0
    for g, r, m in zip(got, ref, mags):
        lim = harness.BWD_U * (m + np.abs(r)) + 1e-12
        ratio = np.abs(g - r) / lim
        assert ratio.max() <= 1.0, ratio.max()
        worst = max(worst, float(ratio.max()))
    assert worst > 0.1, worst


def test_bound_catches_a_dropped_term():
    """A backward that forgets D (dS = P dP) is far outside the bound."""
    N, d = 64, 64
    f = inputs.bf16_bits_to_f64
    q, k, v = (f(harness.random_bits(910, (1, 1, N, d), tensor=t)) for t in "qkv")
    do = f(harness.random_bits(911, (1, 1, N, d), tensor="q"))
    scale = 1.0 / math.sqrt(d)
    ref = oracle.attn_bwd(q, k, v, do, scale, -1, -1)
    mags = harness.bwd_bound_dense(q, k, v, do, scale, lambda b, h: harness.band_visible(-1, -1, N))
    s = scale * q[0, 0] @ k[0, 0].T
    p = np.exp(s - s.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    ds = p * (do[0, 0] @ v[0, 0].T)
    bad = (scale * ds @ k[0, 0])[None, None], ref[1], ref[2]
    with pytest.raises(AssertionError):
        harness.check_grads_elementwise(bad, ref, mags, "dropped D")
