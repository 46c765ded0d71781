"""Backward of packed variable-length batches (attn_bwd_varlen) against the
oracle's per-sequence chain rule; tolerance as the dense backward's (see
test_bwd_gpu: an element-wise bound from the BF16 roundings, per sequence)."""
import math

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

import harness  # noqa: E402
import oracle  # noqa: E402
from exact_attention_152_b200 import inputs  # noqa: E402
from test_bwd_gpu import check_grads  # noqa: E402

CASES = [
    # name, q lengths, k lengths (None: same), H, Hkv, d, (window_left, window_right)
    ("ragged_causal", [1, 127, 128, 129, 300, 0, 513, 64], None, 2, 2, 128, (-1, 0)),
    ("ragged_full_d64", [1, 127, 128, 129, 300, 0, 513, 64], None, 2, 2, 64, (-1, -1)),
    ("gqa_causal", [700, 33, 256], None, 4, 2, 128, (-1, 0)),
    ("q_ne_k", [100, 300, 0, 257], [350, 40, 90, 0], 2, 1, 128, (-1, -1)),
    ("window", [900, 257], None, 2, 2, 128, (63, 0)),
    ("window_q_ne_k", [130, 600], [700, 20], 2, 2, 64, (5, 200)),
]


def _cu(lens):
    return np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)


def _run(q, k, v, do, cu_q, cu_k, max_q, max_k, scale, window):
    import torch
    from exact_attention_152_b200 import binding
    qd, kd, vd, dod = (harness.to_device_bf16(x) for x in (q, k, v, do))
    cq, ck = (torch.from_numpy(c).cuda() for c in (cu_q, cu_k))
    o, lse = binding.fwd_varlen(qd, kd, vd, cq, ck, max_q, scale=scale, window=window)
    dq, dk, dv = binding.bwd_varlen(qd, kd, vd, o, dod, lse, cq, ck, max_k, scale=scale,
                                    window=window)
    assert binding.attn_status_sync(torch.cuda.current_stream().cuda_stream) == 0
    return tuple(x.float().cpu().numpy() for x in (dq, dk, dv))


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_bwd_varlen_parity(case):
    name, lq, lk, H, Hkv, d, window = case
    lk = lq if lk is None else lk
    cu_q, cu_k = _cu(lq), _cu(lk)
    seed = 400 + sum(lq) % 89
    q = harness.random_bits(seed, (int(cu_q[-1]), H, d), tensor="q")
    k = harness.random_bits(seed, (int(cu_k[-1]), Hkv, d), tensor="k")
    v = harness.random_bits(seed, (int(cu_k[-1]), Hkv, d), tensor="v")
    do = harness.random_bits(seed + 1, (int(cu_q[-1]), H, d), tensor="q")
    scale = float(np.float32(1 / math.sqrt(d)))
    got = _run(q, k, v, do, cu_q, cu_k, max(lq), max(max(lk), 1), scale, window)
    f = inputs.bf16_bits_to_f64
    ref = oracle.attn_bwd_varlen(f(q), f(k), f(v), f(do), cu_q, cu_k, scale, *window)
    mags = harness.bwd_bound_varlen(f(q), f(k), f(v), f(do), cu_q, cu_k, scale, *window)
    check_grads(got, ref, mags, name)


@pytest.mark.parametrize("causal", [False, True])
def test_equal_lengths_match_dense(causal):
    """B sequences of one length, packed: dK and dV equal the dense backward's
    bit for bit (each is summed inside one CTA in a fixed order); dQ, whose
    key-block partial sums land in fp32 through reductions in no fixed order,
    agrees to fp32 rounding."""
    import torch
    from exact_attention_152_b200 import binding
    B, H, N, d = 3, 2, 300, 128
    q, k, v = (harness.to_device_bf16(harness.random_bits(410, (B, H, N, d), tensor=t)) for t in "qkv")
    do = harness.to_device_bf16(harness.random_bits(411, (B, H, N, d), tensor="q"))
    o, lse = binding.fwd(q, k, v, causal=causal)
    ref = binding.bwd(q, k, v, o, do, lse, causal=causal)
    pack = lambda x: x.transpose(1, 2).reshape(B * N, H, d).contiguous()  # noqa: E731
    cu = torch.arange(0, B * N + 1, N, dtype=torch.int32, device="cuda")
    lse_p = lse.permute(1, 0, 2).reshape(H, B * N).contiguous()
    got = binding.bwd_varlen(pack(q), pack(k), pack(v), pack(o), pack(do), lse_p, cu, cu, N,
                             causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(got[1].view(torch.int16), pack(ref[1]).view(torch.int16))
    assert torch.equal(got[2].view(torch.int16), pack(ref[2]).view(torch.int16))
    torch.testing.assert_close(got[0].float(), pack(ref[0]).float(), rtol=1e-2, atol=1e-3)


def test_rows_outside_sequences_and_bad_offsets():
    """Query rows no sequence owns get dQ = 0 and key rows no sequence owns are
    not written; offsets that run backwards or past the tensors are skipped and
    reported as ATTN_ERR_INVALID_ARG at the next status read."""
    import torch
    from exact_attention_152_b200 import binding
    H, d, T = 2, 64, 400
    q, k, v = (harness.to_device_bf16(harness.random_bits(412, (T, H, d), tensor=t)) for t in "qkv")
    do = harness.to_device_bf16(harness.random_bits(413, (T, H, d), tensor="q"))
    stream = torch.cuda.current_stream().cuda_stream
    cu = torch.tensor([10, 200, 330], dtype=torch.int32, device="cuda")
    o = torch.zeros_like(q)
    lse = torch.zeros((H, T), dtype=torch.float32, device="cuda")
    binding.fwd_varlen(q, k, v, cu, cu, 256, causal=True, out=o, lse=lse)
    dq, dk, dv = (torch.full_like(x, 7.0) for x in (q, k, v))
    ws = torch.empty(binding.attn_bwd_workspace_size(1, H, T, d), dtype=torch.uint8, device="cuda")

    def call(cu_q, cu_k, max_k):
        return binding.attn_bwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                       do.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                       dv.data_ptr(), ws.data_ptr(), ws.numel(), cu_q.data_ptr(),
                                       cu_k.data_ptr(), cu_q.numel() - 1, max_k, T, T, H, H, d,
                                       0.125, -1, 0, stream)
    assert call(cu, cu, 256) == 0
    assert binding.attn_status_sync(stream) == 0
    assert torch.all(dq[:10] == 0) and torch.all(dq[330:] == 0)
    assert torch.all(dk[:10] == 7.0) and torch.all(dv[330:] == 7.0)
    assert not torch.any(dk[10:330] == 7.0)
    # sequence 1 runs backwards, sequence 2 ends past the tensors
    bad = torch.tensor([0, 200, 100, 450], dtype=torch.int32, device="cuda")
    dk.fill_(7.0)
    assert call(bad, bad, 256) == 0
    assert binding.attn_status_sync(stream) == binding.ATTN_ERR_INVALID_ARG
    assert binding.attn_status_sync(stream) == 0
    assert not torch.any(dk[:200] == 7.0) and torch.all(dk[200:] == 7.0)
    # a key length beyond max_seqlen_k rounded up to 128 is refused too
    long = torch.tensor([0, 300, 400], dtype=torch.int32, device="cuda")
    assert call(long, long, 100) == 0
    assert binding.attn_status_sync(stream) == binding.ATTN_ERR_INVALID_ARG
