"""Failure detection without a fault: a bounded device wait runs out, the kernel
records ATTN_ERR_TIMEOUT and exits normally, and the context stays usable."""
import pytest

pytestmark = pytest.mark.gpu

import harness  # noqa: E402


def test_timeout_is_reported_and_context_survives():
    import torch
    from exact_attention_152_b200 import binding
    s = torch.cuda.current_stream().cuda_stream
    assert binding.attn_status_sync(s) == binding.ATTN_OK
    assert binding.attn_selftest_timeout(20000, s) == binding.ATTN_OK  # 20 ms limit
    assert binding.attn_status_sync(s) == binding.ATTN_ERR_TIMEOUT
    assert binding.attn_status_sync(s) == binding.ATTN_OK  # read-and-clear
    # a normal forward still runs and is still correct afterwards
    q = harness.random_bits(60, (1, 2, 200, 64), tensor="q")
    k = harness.random_bits(60, (1, 2, 200, 64), tensor="k")
    v = harness.random_bits(60, (1, 2, 200, 64), tensor="v")
    o, lse = harness.run_cuda(q, k, v, 0.125, True)
    harness.assert_within(harness.compare(o, lse, harness.oracle_rows(q, k, v, 0.125, True)))
