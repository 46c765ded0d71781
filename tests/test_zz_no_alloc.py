"""attn_bwd_noalloc: the backward with its workspace in the library's static
device array.  Collected last; passes alone and after the other tests."""
import math

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

import harness  # noqa: E402
import oracle  # noqa: E402
from exact_attention_152_b200 import inputs  # noqa: E402

STATIC_BYTES = 96 << 20


def _case(B, H, Hkv, N, d, seed):
    q = harness.random_bits(seed, (B, H, N, d), tensor="q")
    k = harness.random_bits(seed, (B, Hkv, N, d), tensor="k")
    v = harness.random_bits(seed, (B, Hkv, N, d), tensor="v")
    do = harness.random_bits(seed + 1, (B, H, N, d), tensor="q")
    return q, k, v, do


def _run_noalloc(q, k, v, o, do, lse, causal, scale):
    import torch
    from exact_attention_152_b200 import binding
    B, H, N, d = q.shape
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    rc = binding.attn_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                  do.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                  dv.data_ptr(), B, H, k.shape[1], N, k.shape[2], d, scale,
                                  int(causal), torch.cuda.current_stream().cuda_stream)
    binding.check(rc, "attn_bwd_noalloc")
    return dq, dk, dv


@pytest.mark.parametrize("causal", [False, True])
def test_noalloc_matches_oracle_and_workspace_version(causal):
    import torch
    from exact_attention_152_b200 import binding
    B, H, Hkv, N, d = 1, 4, 2, 640, 128
    bits = _case(B, H, Hkv, N, d, 400)
    q, k, v, do = (harness.to_device_bf16(x) for x in bits)
    scale = float(np.float32(1 / math.sqrt(d)))
    o, lse = binding.fwd(q, k, v, causal=causal, scale=scale)
    ref_ws = binding.bwd(q, k, v, o, do, lse, causal=causal, scale=scale)
    # two calls in a row share the static array: the second must not see the
    # first one's accumulator
    runs = [_run_noalloc(q, k, v, o, do, lse, causal, scale) for _ in range(2)]
    assert binding.attn_status_sync(torch.cuda.current_stream().cuda_stream) == 0
    for got in runs:
        # dK, dV: same kernels, same order -> identical; dQ: fp32 reductions may reorder
        assert torch.equal(got[1].view(torch.int16), ref_ws[1].view(torch.int16))
        assert torch.equal(got[2].view(torch.int16), ref_ws[2].view(torch.int16))
        assert torch.allclose(got[0].float(), ref_ws[0].float(), rtol=1e-2, atol=1e-3)
    got = runs[1]
    f = inputs.bf16_bits_to_f64
    wr = 0 if causal else -1
    ref = oracle.attn_bwd(*(f(x) for x in bits), scale, -1, wr)
    mags = harness.bwd_bound_dense(*(f(x) for x in bits), scale,
                                   lambda b, h: harness.band_visible(-1, wr, N))
    harness.check_grads_elementwise(tuple(g.float().cpu().numpy() for g in got), ref, mags,
                                    f"noalloc causal={causal}")


def test_noalloc_allocates_nothing():
    import torch
    from exact_attention_152_b200 import binding
    B, H, N, d = 1, 2, 512, 64
    q, k, v, do = (harness.to_device_bf16(x) for x in _case(B, H, H, N, d, 410))
    o, lse = binding.fwd(q, k, v, causal=True)
    outs = [torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)]
    stream = torch.cuda.current_stream().cuda_stream

    def call():
        rc = binding.attn_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                      do.data_ptr(), lse.data_ptr(), *(t.data_ptr() for t in outs),
                                      B, H, H, N, N, d, 0.125, 1, stream)
        binding.check(rc, "attn_bwd_noalloc")

    call()  # first use: the library's module and its static array are resident from here on
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(5):
        call()
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert binding.attn_status_sync(stream) == 0


def test_noalloc_rejects_sizes_beyond_the_static_array():
    from exact_attention_152_b200 import binding
    B, H, N, d = 1, 64, 8192, 128
    assert binding.attn_bwd_workspace_size(B, H, N, d) > STATIC_BYTES
    fake = 0x10000  # never dereferenced: the size check comes first
    rc = binding.attn_bwd_noalloc(*([fake] * 9), B, H, H, N, N, d, 0.1, 0, None)
    assert rc == binding.ATTN_ERR_UNSUPPORTED
    # the largest headline-like problem that fits is accepted by the size check
    assert binding.attn_bwd_workspace_size(2, 8, 8192, 128) <= STATIC_BYTES
