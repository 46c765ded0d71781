"""Grouped-query / multi-query attention (attn_fwd_gqa) against the oracle:
query head h of batch b attends to key/value head h / (H / Hkv)."""
import math

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

import harness  # noqa: E402
import oracle  # noqa: E402
from exact_attention_152_b200 import inputs  # noqa: E402

CASES = [
    # B, H, Hkv, Nq, Nk, d, causal
    (2, 8, 2, 300, 300, 128, True),
    (1, 16, 1, 1000, 1000, 64, False),
    (3, 6, 3, 200, 517, 128, False),
    (1, 4, 1, 129, 129, 64, True),
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_gqa_parity(case):
    B, H, Hkv, Nq, Nk, d, causal = case
    seed = 70 + H + Hkv
    q = harness.random_bits(seed, (B, H, Nq, d), tensor="q")
    k = harness.random_bits(seed, (B, Hkv, Nk, d), tensor="k")
    v = harness.random_bits(seed, (B, Hkv, Nk, d), tensor="v")
    scale = float(np.float32(1 / math.sqrt(d)))
    o, lse = harness.run_cuda(q, k, v, scale, causal)
    g = H // Hkv
    ref = {}
    for b in range(B):
        for h in range(H):
            rows = np.arange(Nq, dtype=np.int64)
            oo, ll = oracle.attn_rows(inputs.bf16_bits_to_f64(q[b, h]), rows,
                                      inputs.bf16_bits_to_f64(k[b, h // g]),
                                      inputs.bf16_bits_to_f64(v[b, h // g]), scale, causal)
            ref[b * H + h] = (rows, oo, ll)
    harness.assert_within(harness.compare(o, lse, ref))


def test_gqa_equals_repeated_heads_bitwise():
    import torch
    from exact_attention_152_b200 import binding
    B, H, Hkv, N, d = 2, 8, 2, 384, 128
    q = harness.to_device_bf16(harness.random_bits(80, (B, H, N, d), tensor="q"))
    k = harness.to_device_bf16(harness.random_bits(80, (B, Hkv, N, d), tensor="k"))
    v = harness.to_device_bf16(harness.random_bits(80, (B, Hkv, N, d), tensor="v"))
    o_g, l_g = binding.fwd(q, k, v, causal=True)
    k_rep = k.repeat_interleave(H // Hkv, dim=1).contiguous()
    v_rep = v.repeat_interleave(H // Hkv, dim=1).contiguous()
    o_m, l_m = binding.fwd(q, k_rep, v_rep, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o_g.view(torch.int16), o_m.view(torch.int16))
    assert torch.equal(l_g, l_m)
