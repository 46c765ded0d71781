"""Sliding-window band (attn_fwd_window) against the oracle: key j is visible to
query i when i - window_left <= j <= i + window_right (-1: no bound)."""
import math

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

import harness  # noqa: E402
import oracle  # noqa: E402
from exact_attention_152_b200 import inputs  # noqa: E402

CASES = [
    # B, H, Hkv, Nq, Nk, d, (window_left, window_right)
    (1, 2, 2, 300, 300, 128, (0, 0)),
    (1, 2, 2, 300, 300, 64, (5, 3)),
    (2, 2, 2, 520, 520, 128, (127, 0)),
    (1, 3, 3, 520, 520, 128, (128, 0)),
    (1, 2, 2, 777, 777, 128, (255, 255)),
    (1, 2, 2, 640, 640, 64, (-1, 40)),
    (1, 2, 2, 1000, 1000, 128, (300, -1)),
    (2, 4, 2, 700, 700, 128, (200, 0)),        # grouped-query heads
    (1, 2, 2, 200, 520, 128, (10, 300)),      # Nq < Nk
    (1, 2, 2, 600, 100, 64, (50, 0)),         # Nq > Nk: rows >= 150 see no key
    (1, 2, 2, 1300, 1300, 128, (1, 1)),
]


def _oracle(q, k, v, scale, wl, wr):
    B, H, Nq, _ = q.shape
    g = H // k.shape[1]
    ref = {}
    for b in range(B):
        for h in range(H):
            rows = np.arange(Nq, dtype=np.int64)
            oo, ll = oracle.attn_rows_window(inputs.bf16_bits_to_f64(q[b, h]), rows,
                                             inputs.bf16_bits_to_f64(k[b, h // g]),
                                             inputs.bf16_bits_to_f64(v[b, h // g]), scale, wl, wr)
            ref[b * H + h] = (rows, oo, ll)
    return ref


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_window_parity(case):
    B, H, Hkv, Nq, Nk, d, (wl, wr) = case
    seed = 90 + Nq + d
    q = harness.random_bits(seed, (B, H, Nq, d), tensor="q")
    k = harness.random_bits(seed, (B, Hkv, Nk, d), tensor="k")
    v = harness.random_bits(seed, (B, Hkv, Nk, d), tensor="v")
    scale = float(np.float32(1 / math.sqrt(d)))
    o, lse = harness.run_cuda(q, k, v, scale, False, window=(wl, wr))
    m = harness.compare(o, lse, _oracle(q, k, v, scale, wl, wr))
    print(case, m)
    harness.assert_within(m)


def test_empty_band_rows_are_zero_and_neg_inf():
    B, H, Nq, Nk, d = 1, 2, 600, 100, 64
    q = harness.random_bits(95, (B, H, Nq, d), tensor="q")
    k = harness.random_bits(95, (B, H, Nk, d), tensor="k")
    v = harness.random_bits(95, (B, H, Nk, d), tensor="v")
    o, lse = harness.run_cuda(q, k, v, 0.125, False, window=(50, 0))
    # row i sees keys [i - 50, i] within [0, 99]: empty from row 150 on
    assert np.all(o[:, :, 150:] == 0.0)
    assert np.all(np.isneginf(lse[:, :, 150:]))
    assert np.all(np.isfinite(lse[:, :, :150]))


@pytest.mark.parametrize("d", [64, 128])
def test_band_limits_equal_causal_and_full_bitwise(d):
    """(-1, 0) is the causal kernel call and (-1, -1) the unmasked one, bit for
    bit; a band wider than the sequence equals the unmasked result."""
    import torch
    from exact_attention_152_b200 import binding
    B, H, N = 2, 3, 700
    q = harness.to_device_bf16(harness.random_bits(96, (B, H, N, d), tensor="q"))
    k = harness.to_device_bf16(harness.random_bits(96, (B, H, N, d), tensor="k"))
    v = harness.to_device_bf16(harness.random_bits(96, (B, H, N, d), tensor="v"))
    oc, lc = binding.fwd(q, k, v, causal=True)
    ow, lw = binding.fwd(q, k, v, window=(-1, 0))
    of, lf = binding.fwd(q, k, v, causal=False)
    on, ln = binding.fwd(q, k, v, window=(-1, -1))
    ob, lb = binding.fwd(q, k, v, window=(N, N))
    torch.cuda.synchronize()
    assert torch.equal(oc.view(torch.int16), ow.view(torch.int16)) and torch.equal(lc, lw)
    assert torch.equal(of.view(torch.int16), on.view(torch.int16)) and torch.equal(lf, ln)
    assert torch.equal(of.view(torch.int16), ob.view(torch.int16)) and torch.equal(lf, lb)


def test_window_sampled_rows_long():
    """A long causal sliding window (4096 keys) over 32k positions, sampled rows."""
    B, H, N, d, wl = 1, 2, 32768, 128, 4095
    q = harness.random_bits(97, (B, H, N, d), tensor="q")
    k = harness.random_bits(97, (B, H, N, d), tensor="k")
    v = harness.random_bits(97, (B, H, N, d), tensor="v")
    scale = float(np.float32(1 / math.sqrt(d)))
    o, lse = harness.run_cuda(q, k, v, scale, False, window=(wl, 0))
    ref = {}
    for h in range(H):
        rows = np.unique(np.concatenate([inputs.sample_rows(97, h, N, 200),
                                         [0, 4095, 4096, 4097, N - 1]])).astype(np.int64)
        oo, ll = oracle.attn_rows_window(inputs.bf16_bits_to_f64(q[0, h, rows]), rows,
                                         inputs.bf16_bits_to_f64(k[0, h]),
                                         inputs.bf16_bits_to_f64(v[0, h]), scale, wl, 0)
        ref[h] = (rows, oo, ll)
    harness.assert_within(harness.compare(o, lse, ref))
