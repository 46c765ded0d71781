"""The seeded input generator (CPU only)."""
import numpy as np
import torch

from exact_attention_152_b200 import inputs
from exact_attention_152_b200.workloads import WORKLOADS


def test_bf16_rounding_matches_torch():
    r = np.random.default_rng(0)
    x = np.concatenate([r.standard_normal(100000).astype(np.float32) * 10,
                        np.array([1.0, -2.5, 1 + 2**-8, 1 + 3 * 2**-9, 65504.0, 1e-30], np.float32)])
    ours = inputs.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_widening_is_exact():
    b = np.arange(0, 65536, 7, dtype=np.uint16)
    b = b[(b & 0x7F80) != 0x7F80]  # drop inf/nan patterns
    f = inputs.bf16_bits_to_f64(b)
    back = inputs.f32_to_bf16_bits(f.astype(np.float32))
    assert np.array_equal(back, b)


def test_subset_equals_full():
    full = inputs.gen_bf16(7, "k", (3, 50, 8))
    idx = np.array([0, 5, 77, 1199, 600])
    assert np.array_equal(inputs.gen_bf16_at(7, "k", idx), full.reshape(-1)[idx])


def test_streams_differ_and_are_deterministic():
    a = inputs.gen_bf16(1, "q", (1000,))
    assert np.array_equal(a, inputs.gen_bf16(1, "q", (1000,)))
    assert not np.array_equal(a, inputs.gen_bf16(1, "k", (1000,)))
    assert not np.array_equal(a, inputs.gen_bf16(2, "q", (1000,)))


def test_distributions():
    z = inputs.bf16_bits_to_f64(inputs.gen_bf16(3, "q", (200000,)))
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1) < 0.01
    z8 = inputs.bf16_bits_to_f64(inputs.gen_bf16(3, "q", (200000,), mult=8.0))
    assert np.array_equal(z8, 8 * z)  # power-of-two scaling is exact
    u = inputs.bf16_bits_to_f64(inputs.gen_bf16(3, "v", (200000,), dist="uniform"))
    assert u.min() >= -1 and u.max() <= 1 and abs(u.mean()) < 0.01  # bf16 rounding may reach 1.0
    assert abs(u.var() - 1 / 3) < 0.01


def test_sample_rows():
    rows = inputs.sample_rows(4, 3, 131072, 256)
    assert len(rows) == 256 and rows[0] == 0 and rows[-1] == 131071
    assert np.all(np.diff(rows) > 0)
    assert np.array_equal(rows, inputs.sample_rows(4, 3, 131072, 256))
    assert np.array_equal(inputs.sample_rows(0, 0, 10, 64), np.arange(10))


def test_workload_slices_agree():
    w = WORKLOADS["tiny_b1h2n128d64"]
    q = w.tensor_bits("q")
    assert q.shape == (1, 2, 128, 64)
    assert np.array_equal(w.head_bits("q", 1), q[0, 1])
    rows = np.array([0, 9, 127])
    assert np.array_equal(w.q_rows_bits(1, rows), q[0, 1, rows])
    assert WORKLOADS["mha_b2h16n8k_d128"].flops == 4 * 2 * 16 * 8192 * 8192 * 128


def test_gqa_workload_kv_heads():
    import dataclasses
    w = dataclasses.replace(WORKLOADS["gqa_b2h32kv8n8k_d128"], Nq=64, Nk=64)
    assert w.shape("q") == (2, 32, 64, 128) and w.shape("k") == (2, 8, 64, 128)
    k = w.tensor_bits("k")
    for bh in (0, 3, 4, 31, 32, 37, 63):
        b, h = divmod(bh, w.H)
        assert w.kv_head_of(bh) == b * 8 + h // 4
        assert np.array_equal(w.head_bits("k", w.kv_head_of(bh)), k[b, h // 4])


def test_e4m3_codes():
    """The E4M3 table follows the format's definition, and rounding to it agrees
    with torch's float8_e4m3fn conversion inside the finite range (torch does
    not saturate beyond it; this generator does, to +-448)."""
    import torch
    from exact_attention_152_b200 import inputs
    t = inputs.e4m3_decode_table()
    assert t[0x00] == 0.0 and t[0x01] == 2.0 ** -9 and t[0x08] == 2.0 ** -6
    assert t[0x38] == 1.0 and t[0x7E] == 448.0 and np.isnan(t[0x7F]) and t[0xB8] == -1.0
    x = np.random.default_rng(3).standard_normal(100000).astype(np.float32) * np.float32(40)
    x = np.concatenate([x, np.float32([0.0, -0.0, 2.0 ** -10, 1.5 * 2.0 ** -9, 1.0625, 1.1875, 448])])
    x = x[np.abs(x) <= 448]
    ours = inputs.e4m3_from_f32(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)
    assert inputs.e4m3_from_f32(np.float32([1000.0, -500.0])).tolist() == [0x7E, 0xFE]
    codes = inputs.gen_e4m3(5, "q", (4, 8))
    assert codes.dtype == np.uint8 and codes.shape == (4, 8)
