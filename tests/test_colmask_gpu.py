"""Column-interval masks (attn_fwd_colmask) against the oracle: key j is hidden
from query rows [lo1_j, hi1_j) and [lo2_j, hi2_j), and from rows i < j when
causal.  Shapes span several 128-key blocks, 256-row CTAs and ragged tails."""
import math

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

import harness  # noqa: E402
import oracle  # noqa: E402
from exact_attention_152_b200 import inputs, masks  # noqa: E402


def _mask(kind, seed, B, H, Nq, Nk):
    if kind == "docs":
        return masks.documents([masks.document_lengths(seed + b, Nk, 40, 400) for b in range(B)], Nk), True
    if kind == "docs_bidir":
        return masks.documents([masks.document_lengths(seed + b, Nk, 100, 700) for b in range(B)], Nk,
                               bidirectional=True), False
    if kind == "prefix":
        return masks.prefix_lm(B, Nk, Nk // 3), False
    if kind == "random":
        return masks.random_intervals(seed, B, 1, Nq, Nk), False
    if kind == "random_heads":
        return masks.random_intervals(seed, B, H, Nq, Nk), False
    if kind == "random_causal":
        return masks.random_intervals(seed, B, 1, Nq, Nk), True
    raise ValueError(kind)


def _run(q, k, v, mask, causal, scale):
    import torch
    from exact_attention_152_b200 import binding
    qd, kd, vd = (harness.to_device_bf16(x) for x in (q, k, v))
    md = torch.from_numpy(mask).cuda()
    o, lse = binding.fwd_colmask(qd, kd, vd, md, causal=causal, scale=scale)
    assert binding.attn_status_sync(torch.cuda.current_stream().cuda_stream) == 0
    return o.float().cpu().numpy(), lse.cpu().numpy()


def _oracle(q, k, v, mask, causal, scale, rows_per_head=None, seed=0):
    B, H, Nq, _ = q.shape
    g = H // k.shape[1]
    ref = {}
    for b in range(B):
        for h in range(H):
            if rows_per_head is None:
                rows = np.arange(Nq, dtype=np.int64)
            else:
                rows = inputs.sample_rows(seed, b * H + h, Nq, rows_per_head)
            cols = mask[b, h if mask.shape[1] > 1 else 0]
            oo, ll = oracle.attn_rows_colmask(inputs.bf16_bits_to_f64(q[b, h, rows]), rows,
                                              inputs.bf16_bits_to_f64(k[b, h // g]),
                                              inputs.bf16_bits_to_f64(v[b, h // g]), scale, causal,
                                              cols)
            ref[b * H + h] = (rows, oo, ll)
    return ref


CASES = [
    # kind, B, H, Hkv, Nq, Nk, d
    ("docs", 2, 2, 2, 1000, 1000, 128),
    ("docs", 1, 3, 3, 777, 777, 64),
    ("docs_bidir", 1, 2, 2, 1300, 1300, 128),
    ("prefix", 2, 2, 2, 900, 900, 128),
    ("random", 1, 2, 2, 520, 520, 128),
    ("random", 1, 2, 2, 300, 1000, 64),          # Nq < Nk
    ("random_heads", 2, 4, 2, 600, 600, 128),    # one mask per head, grouped K/V
    ("random_causal", 1, 2, 2, 700, 700, 128),
    ("random", 1, 2, 2, 1000, 130, 128),         # Nq > Nk, one ragged key block
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_colmask_parity(case):
    kind, B, H, Hkv, Nq, Nk, d = case
    seed = 300 + Nq + d
    q = harness.random_bits(seed, (B, H, Nq, d), tensor="q")
    k = harness.random_bits(seed, (B, Hkv, Nk, d), tensor="k")
    v = harness.random_bits(seed, (B, Hkv, Nk, d), tensor="v")
    mask, causal = _mask(kind, seed, B, H, Nq, Nk)
    scale = float(np.float32(1 / math.sqrt(d)))
    o, lse = _run(q, k, v, mask, causal, scale)
    m = harness.compare(o, lse, _oracle(q, k, v, mask, causal, scale))
    print(case, m)
    harness.assert_within(m)


def test_hidden_rows_are_zero_and_neg_inf():
    """Every key hides rows [200, 520): those rows see nothing -- all of the
    CTA of rows 256..511 (no key block visited but one, fully masked) and parts
    of its neighbours -- while the other rows see every key."""
    B, H, N, d = 1, 2, 700, 128
    q = harness.random_bits(311, (B, H, N, d), tensor="q")
    k = harness.random_bits(311, (B, H, N, d), tensor="k")
    v = harness.random_bits(311, (B, H, N, d), tensor="v")
    mask = masks.empty(B, 1, N)
    mask[..., 2], mask[..., 3] = 200, 520
    o, lse = _run(q, k, v, mask, False, 0.1)
    assert np.all(o[:, :, 200:520] == 0.0) and np.all(np.isneginf(lse[:, :, 200:520]))
    keep = np.r_[0:200, 520:N]
    m = harness.compare(o, lse, _oracle(q, k, v, mask, False, 0.1))
    harness.assert_within(m)
    assert np.all(np.isfinite(lse[:, :, keep]))


@pytest.mark.parametrize("d", [64, 128])
def test_colmask_equals_band_and_plain_bitwise(d):
    """An all-empty mask is attn_fwd bit for bit (causal or not), and a band
    spelled as column intervals is attn_fwd_window bit for bit: blocks that the
    column mask hides entirely contribute exact zeros."""
    import torch
    from exact_attention_152_b200 import binding
    B, H, N = 2, 3, 900
    q, k, v = (harness.to_device_bf16(harness.random_bits(312, (B, H, N, d), tensor=t))
               for t in "qkv")
    for causal in (False, True):
        o0, l0 = binding.fwd(q, k, v, causal=causal)
        o1, l1 = binding.fwd_colmask(q, k, v, torch.from_numpy(masks.empty(B, 1, N)).cuda(),
                                     causal=causal)
        torch.cuda.synchronize()
        assert torch.equal(o0.view(torch.int16), o1.view(torch.int16)) and torch.equal(l0, l1)
    for wl, wr in [(200, 0), (100, 300), (0, 0)]:
        o0, l0 = binding.fwd(q, k, v, window=(wl, wr))
        o1, l1 = binding.fwd_colmask(q, k, v, torch.from_numpy(masks.band(B, N, wl, wr)).cuda())
        torch.cuda.synchronize()
        assert torch.equal(o0.view(torch.int16), o1.view(torch.int16)), (wl, wr)
        assert torch.equal(l0, l1), (wl, wr)


def test_colmask_documents_sampled_rows_long():
    """Document-causal mask over 16k positions (documents of 256 .. 4096
    tokens), sampled rows of every head."""
    B, H, N, d = 1, 4, 16384, 128
    q = harness.random_bits(313, (B, H, N, d), tensor="q")
    k = harness.random_bits(313, (B, H, N, d), tensor="k")
    v = harness.random_bits(313, (B, H, N, d), tensor="v")
    mask = masks.documents([masks.document_lengths(313, N, 256, 4096)], N)
    scale = float(np.float32(1 / math.sqrt(d)))
    o, lse = _run(q, k, v, mask, True, scale)
    harness.assert_within(harness.compare(o, lse, _oracle(q, k, v, mask, True, scale, 96, 313)))
