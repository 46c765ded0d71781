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


BWD_CASES = [
    # kind, B, H, Hkv, Nq, Nk, d
    ("docs", 1, 2, 2, 1000, 1000, 128),
    ("docs_bidir", 1, 2, 1, 777, 777, 64),
    ("prefix", 1, 2, 2, 900, 900, 128),
    ("random", 1, 2, 2, 520, 520, 128),
    ("random", 1, 2, 2, 300, 1000, 64),          # Nq < Nk
    ("random_heads", 1, 4, 2, 600, 600, 128),    # one mask per head, grouped K/V
    ("random_causal", 1, 2, 2, 700, 700, 128),
    ("random", 1, 2, 2, 1000, 130, 128),         # Nq > Nk, one ragged key block
]


@pytest.mark.parametrize("case", BWD_CASES, ids=[str(c) for c in BWD_CASES])
def test_colmask_bwd_parity(case):
    """attn_bwd_colmask against the oracle's chain rule under the same intervals
    (tolerance as the dense backward's)."""
    import torch
    from exact_attention_152_b200 import binding
    from test_bwd_gpu import check_grads
    kind, B, H, Hkv, Nq, Nk, d = case
    seed = 320 + Nq + d
    q = harness.random_bits(seed, (B, H, Nq, d), tensor="q")
    k = harness.random_bits(seed, (B, Hkv, Nk, d), tensor="k")
    v = harness.random_bits(seed, (B, Hkv, Nk, d), tensor="v")
    do = harness.random_bits(seed + 1, (B, H, Nq, d), tensor="q")
    mask, causal = _mask(kind, seed, B, H, Nq, Nk)
    scale = float(np.float32(1 / math.sqrt(d)))
    qd, kd, vd, dod = (harness.to_device_bf16(x) for x in (q, k, v, do))
    md = torch.from_numpy(mask).cuda()
    o, lse = binding.fwd_colmask(qd, kd, vd, md, causal=causal, scale=scale)
    grads = binding.bwd_colmask(qd, kd, vd, o, dod, lse, md, causal=causal, scale=scale)
    assert binding.attn_status_sync(torch.cuda.current_stream().cuda_stream) == 0
    got = tuple(x.float().cpu().numpy() for x in grads)
    f = inputs.bf16_bits_to_f64
    ref = oracle.attn_bwd_colmask(f(q), f(k), f(v), f(do), scale, causal, mask)
    Hm = mask.shape[1]
    mags = harness.bwd_bound_dense(f(q), f(k), f(v), f(do), scale,
                                   lambda b, h: harness.colmask_visible(mask[b, h if Hm > 1 else 0], causal))
    check_grads(got, ref, mags, str(case))


@pytest.mark.parametrize("d", [64, 128])
def test_colmask_bwd_equals_band_and_plain(d):
    """An all-empty mask gives attn_bwd's dK and dV bit for bit (causal or not),
    and a band spelled as intervals gives attn_bwd_window's: the same query
    tiles are visited and the same pairs masked.  dQ, reduced in no fixed
    order, agrees to fp32 rounding."""
    import torch
    from exact_attention_152_b200 import binding
    B, H, N = 1, 2, 900
    q, k, v = (harness.to_device_bf16(harness.random_bits(330, (B, H, N, d), tensor=t)) for t in "qkv")
    do = harness.to_device_bf16(harness.random_bits(331, (B, H, N, d), tensor="q"))
    cases = [(masks.empty(B, 1, N), False, dict(causal=False)),
             (masks.empty(B, 1, N), True, dict(causal=True)),
             (masks.band(B, N, 200, 0), False, dict(window=(200, 0))),
             (masks.band(B, N, 100, 300), False, dict(window=(100, 300)))]
    for mask, causal, kw in cases:
        o, lse = binding.fwd(q, k, v, **kw)
        ref = binding.bwd(q, k, v, o, do, lse, **kw)
        got = binding.bwd_colmask(q, k, v, o, do, lse, torch.from_numpy(mask).cuda(), causal=causal)
        torch.cuda.synchronize()
        assert torch.equal(got[1].view(torch.int16), ref[1].view(torch.int16)), kw
        assert torch.equal(got[2].view(torch.int16), ref[2].view(torch.int16)), kw
        torch.testing.assert_close(got[0].float(), ref[0].float(), rtol=1e-2, atol=1e-3)


def test_colmask_bwd_hidden_blocks():
    """Every key hides rows [200, 520) and keys 300..427 hide every row: the
    hidden query tiles are skipped, keys no query sees get dK = dV = 0, and the
    rest matches the oracle."""
    import torch
    from exact_attention_152_b200 import binding
    from test_bwd_gpu import check_grads
    B, H, N, d = 1, 2, 700, 128
    q, k, v = (harness.random_bits(332, (B, H, N, d), tensor=t) for t in "qkv")
    do = harness.random_bits(333, (B, H, N, d), tensor="q")
    mask = masks.empty(B, 1, N)
    mask[..., 2], mask[..., 3] = 200, 520
    mask[0, 0, 300:428, 0], mask[0, 0, 300:428, 1] = 0, N
    qd, kd, vd, dod = (harness.to_device_bf16(x) for x in (q, k, v, do))
    md = torch.from_numpy(mask).cuda()
    o, lse = binding.fwd_colmask(qd, kd, vd, md, scale=0.1)
    dq, dk, dv = binding.bwd_colmask(qd, kd, vd, o, dod, lse, md, scale=0.1)
    assert binding.attn_status_sync(torch.cuda.current_stream().cuda_stream) == 0
    assert torch.all(dk[:, :, 300:428] == 0) and torch.all(dv[:, :, 300:428] == 0)
    assert torch.all(dq[:, :, 200:520] == 0)
    f = inputs.bf16_bits_to_f64
    ref = oracle.attn_bwd_colmask(f(q), f(k), f(v), f(do), 0.1, False, mask)
    mags = harness.bwd_bound_dense(f(q), f(k), f(v), f(do), 0.1,
                                   lambda b, h: harness.colmask_visible(mask[b, 0], False))
    check_grads(tuple(x.float().cpu().numpy() for x in (dq, dk, dv)), ref, mags, "hidden")


def test_colmask_bwd_both_hidden_ranges_ragged():
    """Both hidden query-tile ranges of a key block, a partial last key block
    and a partial last query tile at once (Nq = 650, Nk = 333): every key
    hides rows [128, 384) by its first interval and [512, Nq) by its second,
    with per-key jitter in the middle block so the block summaries (max lo,
    min hi) differ from the keys' own bounds.  The backward skips tiles 1-2
    and 4-5 for the blocks where every key hides them; the result matches the
    oracle under the element-wise bound, and keys past Nk do not exist."""
    import torch
    from exact_attention_152_b200 import binding
    from test_bwd_gpu import check_grads
    B, H, Nq, Nk, d = 1, 2, 650, 333, 128
    q, k, v = (harness.random_bits(334, (B, H, n, d), tensor=t) for t, n in (("q", Nq), ("k", Nk), ("v", Nk)))
    do = harness.random_bits(335, (B, H, Nq, d), tensor="q")
    mask = masks.empty(B, 1, Nk)
    mask[..., 0], mask[..., 1] = 128, 384
    mask[..., 2], mask[..., 3] = 512, Nq
    rng = np.random.default_rng(5)
    mid = slice(128, 256)
    mask[0, 0, mid, 0] = 128 - rng.integers(0, 40, 128)     # max lo stays 128: tiles 1-2 still hidden
    mask[0, 0, mid, 1] = 384 + rng.integers(0, 40, 128)
    mask[0, 0, mid, 3] = Nq + rng.integers(0, 40, 128)       # ends past Nq: the last tile stays hidden
    qd, kd, vd, dod = (harness.to_device_bf16(x) for x in (q, k, v, do))
    md = torch.from_numpy(mask).cuda()
    o, lse = binding.fwd_colmask(qd, kd, vd, md, scale=0.1)
    dq, dk, dv = binding.bwd_colmask(qd, kd, vd, o, dod, lse, md, scale=0.1)
    assert binding.attn_status_sync(torch.cuda.current_stream().cuda_stream) == 0
    assert torch.all(dq[:, :, 128:384] == 0) and torch.all(dq[:, :, 512:] == 0)
    f = inputs.bf16_bits_to_f64
    ref = oracle.attn_bwd_colmask(f(q), f(k), f(v), f(do), 0.1, False, mask)
    mags = harness.bwd_bound_dense(f(q), f(k), f(v), f(do), 0.1,
                                   lambda b, h: harness.colmask_visible(mask[b, 0], False))
    check_grads(tuple(x.float().cpu().numpy() for x in (dq, dk, dv)), ref, mags, "two ranges, ragged")


def test_colmask_plan_order_changes_nothing():
    """A workspace of the required size (block summaries only) keeps the launch
    order; the full size runs the longest-first CTA plans.  Both give the same
    forward output bit for bit and the same dK and dV (dQ's fp32 reductions
    may land in another order)."""
    import torch
    from exact_attention_152_b200 import binding
    B, H, N, d = 2, 4, 1000, 128
    g = torch.Generator().manual_seed(21)
    q, k, v, do = (torch.randn(B, H, N, d, generator=g).to(torch.bfloat16).cuda() for _ in range(4))
    mask = torch.from_numpy(masks.documents([masks.document_lengths(31 + b, N, 40, 400) for b in range(B)],
                                            N)).cuda()
    n_kb = (N + 127) // 128
    o_plan, l_plan = binding.fwd_colmask(q, k, v, mask, causal=True)
    ws_min = torch.empty(B * n_kb * 32, dtype=torch.uint8, device="cuda")
    o_fix, l_fix = binding.fwd_colmask(q, k, v, mask, causal=True, workspace=ws_min)
    torch.cuda.synchronize()
    assert torch.equal(o_plan.view(torch.int16), o_fix.view(torch.int16))
    assert torch.equal(l_plan, l_fix)
    dq_p, dk_p, dv_p = binding.bwd_colmask(q, k, v, o_plan, do, l_plan, mask, causal=True)
    base = binding.attn_bwd_workspace_size(B, H, N, d)
    ws_bmin = torch.empty((base + 255) // 256 * 256 + B * n_kb * 32, dtype=torch.uint8, device="cuda")
    dq_f, dk_f, dv_f = binding.bwd_colmask(q, k, v, o_plan, do, l_plan, mask, causal=True, workspace=ws_bmin)
    torch.cuda.synchronize()
    assert torch.equal(dk_p.view(torch.int16), dk_f.view(torch.int16))
    assert torch.equal(dv_p.view(torch.int16), dv_f.view(torch.int16))
    assert torch.allclose(dq_p.float(), dq_f.float(), rtol=1e-2, atol=1e-3)
    assert binding.attn_status_sync(torch.cuda.current_stream().cuda_stream) == 0
