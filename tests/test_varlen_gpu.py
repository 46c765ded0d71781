"""Packed variable-length batches (attn_fwd_varlen) against the oracle: each
sequence attends only to its own keys, positions counted within the sequence."""
import math

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

import harness  # noqa: E402
import oracle  # noqa: E402
from exact_attention_152_b200 import inputs  # noqa: E402

CASES = [
    # name, q lengths, k lengths (None: same), H, Hkv, d, (window_left, window_right)
    ("ragged_causal", [1, 127, 128, 129, 300, 0, 513, 64], None, 4, 4, 128, (-1, 0)),
    ("ragged_full", [1, 127, 128, 129, 300, 0, 513, 64], None, 2, 2, 64, (-1, -1)),
    ("gqa_causal", [700, 33, 256, 1000], None, 8, 2, 128, (-1, 0)),
    ("q_ne_k", [100, 300, 0, 257], [350, 40, 90, 0], 2, 1, 128, (-1, -1)),
    ("window", [900, 257, 1024], None, 2, 2, 128, (63, 0)),
    ("window_q_ne_k", [130, 600], [700, 20], 3, 3, 64, (5, 200)),
    ("single_long", [4099], None, 2, 2, 128, (-1, 0)),
]


def _cu(lens):
    return np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_varlen_parity(case):
    name, lq, lk, H, Hkv, d, window = case
    lk = lq if lk is None else lk
    cu_q, cu_k = _cu(lq), _cu(lk)
    seed = 200 + sum(lq) % 97
    q = harness.random_bits(seed, (int(cu_q[-1]), H, d), tensor="q")
    k = harness.random_bits(seed, (int(cu_k[-1]), Hkv, d), tensor="k")
    v = harness.random_bits(seed, (int(cu_k[-1]), Hkv, d), tensor="v")
    scale = float(np.float32(1 / math.sqrt(d)))
    o, lse = harness.run_varlen(q, k, v, cu_q, cu_k, max(lq), scale, window)
    ref = oracle.attn_varlen(inputs.bf16_bits_to_f64(q), inputs.bf16_bits_to_f64(k),
                             inputs.bf16_bits_to_f64(v), cu_q, cu_k, scale, *window)
    m = harness.compare_varlen(o, lse, ref, cu_q)
    print(name, m)
    harness.assert_within(m)


@pytest.mark.parametrize("causal", [False, True])
def test_equal_lengths_match_dense_bitwise(causal):
    """B sequences of one length, packed, give the dense [B, H, N, d] result bit
    for bit (same tiles, same arithmetic; only the addressing differs)."""
    import torch
    from exact_attention_152_b200 import binding
    B, H, N, d = 3, 4, 640, 128
    qd = harness.to_device_bf16(harness.random_bits(210, (B, H, N, d), tensor="q"))
    kd = harness.to_device_bf16(harness.random_bits(210, (B, H, N, d), tensor="k"))
    vd = harness.to_device_bf16(harness.random_bits(210, (B, H, N, d), tensor="v"))
    o_d, l_d = binding.fwd(qd, kd, vd, causal=causal)
    pack = lambda t: t.transpose(1, 2).reshape(B * N, H, d).contiguous()  # noqa: E731
    cu = torch.arange(0, (B + 1) * N, N, dtype=torch.int32, device="cuda")
    o_p, l_p = binding.fwd_varlen(pack(qd), pack(kd), pack(vd), cu, cu, N, causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(pack(o_d).view(torch.int16), o_p.view(torch.int16))
    assert torch.equal(l_d.permute(1, 0, 2).reshape(H, B * N), l_p)


def test_no_writes_outside_outputs():
    import torch
    from exact_attention_152_b200 import binding
    lens = [129, 1, 300]
    H, d = 2, 128
    cu = torch.from_numpy(_cu(lens)).cuda()
    T = sum(lens)
    q = harness.to_device_bf16(harness.random_bits(211, (T, H, d), tensor="q"))
    k = harness.to_device_bf16(harness.random_bits(211, (T, H, d), tensor="k"))
    v = harness.to_device_bf16(harness.random_bits(211, (T, H, d), tensor="v"))
    pad = 8192
    o_buf = torch.full((pad + T * H * d + pad,), 7.0, dtype=torch.bfloat16, device="cuda")
    l_buf = torch.full((pad + H * T + pad,), 7.0, dtype=torch.float32, device="cuda")
    o = o_buf[pad:pad + T * H * d].view(T, H, d)
    lse = l_buf[pad:pad + H * T].view(H, T)
    binding.fwd_varlen(q, k, v, cu, cu, max(lens), causal=True, out=o, lse=lse)
    assert binding.attn_status_sync(torch.cuda.current_stream().cuda_stream) == 0
    assert torch.all(o_buf[:pad] == 7.0) and torch.all(o_buf[pad + T * H * d:] == 7.0)
    assert torch.all(l_buf[:pad] == 7.0) and torch.all(l_buf[pad + H * T:] == 7.0)
    assert not torch.any(o == 7.0) and not torch.any(lse == 7.0)


def test_bad_offsets_are_reported_and_skipped():
    """Offsets that do not describe sequences inside the tensors: the kernel
    skips those sequences (their outputs stay untouched), computes the others and
    reports ATTN_ERR_INVALID_ARG at the next status read."""
    import torch
    from exact_attention_152_b200 import binding
    H, d, T = 2, 64, 400
    q = harness.to_device_bf16(harness.random_bits(212, (T, H, d), tensor="q"))
    k = harness.to_device_bf16(harness.random_bits(212, (T, H, d), tensor="k"))
    v = harness.to_device_bf16(harness.random_bits(212, (T, H, d), tensor="v"))
    # sequence 1 runs backwards, sequence 2 ends past total: both skipped
    cu = torch.tensor([0, 200, 100, 450], dtype=torch.int32, device="cuda")
    o = torch.full((T, H, d), 7.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.full((H, T), 7.0, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    binding.fwd_varlen(q, k, v, cu, cu, 256, causal=True, out=o, lse=lse)
    assert binding.attn_status_sync(stream) == binding.ATTN_ERR_INVALID_ARG
    assert binding.attn_status_sync(stream) == 0  # read clears it
    assert not torch.any(o[:200] == 7.0)           # sequence 0 computed
    assert torch.all(o[200:] == 7.0) and torch.all(lse[:, 200:] == 7.0)
    # a sequence longer than max_seqlen_q rounded up to 256 is refused as well
    cu2 = torch.tensor([0, 300, 400], dtype=torch.int32, device="cuda")
    binding.fwd_varlen(q, k, v, cu2, cu2, 100, causal=True, out=o, lse=lse)
    assert binding.attn_status_sync(stream) == binding.ATTN_ERR_INVALID_ARG
