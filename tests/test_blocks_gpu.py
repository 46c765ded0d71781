"""Building blocks of the kernel, each alone on one tile, against plain host math."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu

from exact_attention_152_b200 import blocks_binding as bb  # noqa: E402
from exact_attention_152_b200 import inputs  # noqa: E402


def _stream():
    import torch
    return torch.cuda.current_stream().cuda_stream


def _dev(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("d", [64, 128])
def test_mma_ss_tile(d):
    import torch
    a_bits = inputs.gen_bf16(100 + d, "q", (128, d))
    b_bits = inputs.gen_bf16(100 + d, "k", (128, d))
    a, b = _dev(a_bits), _dev(b_bits)
    c = torch.full((128, 128), float("nan"), dtype=torch.float32, device="cuda")
    assert bb.blocks_mma_ss(a.data_ptr(), b.data_ptr(), c.data_ptr(), d, _stream()) == 0
    assert bb.blocks_status_sync(_stream()) == 0
    ref = inputs.bf16_bits_to_f64(a_bits) @ inputs.bf16_bits_to_f64(b_bits).T
    got = c.cpu().numpy().astype(np.float64)
    # BF16 products are exact in fp32; only the fp32 accumulation order differs.
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-4 * np.abs(ref).max())


@pytest.mark.parametrize("d", [64, 128])
def test_mma_ts_tile(d):
    import torch
    p_bits = inputs.gen_bf16(200 + d, "q", (128, 128), dist="uniform")
    v_bits = inputs.gen_bf16(200 + d, "v", (128, d))
    p, v = _dev(p_bits), _dev(v_bits)
    c = torch.full((128, d), float("nan"), dtype=torch.float32, device="cuda")
    assert bb.blocks_mma_ts(p.data_ptr(), v.data_ptr(), c.data_ptr(), d, _stream()) == 0
    assert bb.blocks_status_sync(_stream()) == 0
    ref = inputs.bf16_bits_to_f64(p_bits) @ inputs.bf16_bits_to_f64(v_bits)
    got = c.cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-4 * np.abs(ref).max())


@pytest.mark.parametrize("d", [64, 128])
def test_swizzle_roundtrip(d):
    import torch
    x_bits = inputs.gen_bf16(300 + d, "q", (128, d))
    x = _dev(x_bits)
    y_tma = torch.zeros_like(x)
    y_plain = torch.zeros_like(x)
    assert bb.blocks_swizzle_roundtrip(x.data_ptr(), y_tma.data_ptr(), y_plain.data_ptr(), d, _stream()) == 0
    assert bb.blocks_status_sync(_stream()) == 0
    assert torch.equal(y_plain.view(torch.int16), x.view(torch.int16))
    assert torch.equal(y_tma.view(torch.int16), x.view(torch.int16))


def test_exp2_mufu_and_polynomial():
    import torch
    xs = np.concatenate([np.linspace(-140.0, 10.0, 600001), [0.0, -0.0, -127.0, -126.5, -1e30, 1.0, 8.0],
                         np.arange(-126, 9, dtype=np.float64)]).astype(np.float32)
    x = torch.from_numpy(xs).cuda()
    ym = torch.empty_like(x)
    yp = torch.empty_like(x)
    assert bb.blocks_exp2(x.data_ptr(), ym.data_ptr(), yp.data_ptr(), x.numel(), _stream()) == 0
    torch.cuda.synchronize()
    ym, yp = ym.cpu().numpy().astype(np.float64), yp.cpu().numpy().astype(np.float64)
    ref = np.exp2(xs.astype(np.float64))
    normal = xs >= -125.0
    # polynomial: the fitted bound (1.02e-4 relative) in the normal range
    rel_p = np.abs(yp[normal] / ref[normal] - 1)
    assert rel_p.max() < 1.1e-4, rel_p.max()
    # hardware ex2.approx: a few ulp
    rel_m = np.abs(ym[normal] / ref[normal] - 1)
    assert rel_m.max() < 2e-6, rel_m.max()
    # exact points: 2^0 = 1 and integer powers of two (f = 0 -> p(0) = 1)
    ints = np.arange(-126, 9)
    yi = yp[-len(ints):]
    assert np.array_equal(yi, np.exp2(ints.astype(np.float64)))
    assert np.all(yp[xs == 0.0] == 1.0)
    # far below the range (masked scores) -> exactly +0
    assert np.all(yp[xs <= -127.0] == 0.0)
    assert np.all(ym[xs <= -127.0] < 1e-37)


def _dev_u8(codes):
    import torch
    return torch.from_numpy(np.ascontiguousarray(codes)).cuda()


def test_pack_e4m3_order_and_rounding():
    """Four fp32 -> four E4M3 bytes, x[4i] in the low byte, rounded as the
    host encoder rounds (nearest even, saturating)."""
    import torch
    x = np.random.default_rng(7).standard_normal(4096).astype(np.float32) * np.float32(50)
    x[:8] = [0.0, -0.0, 2.0 ** -10, 1.5 * 2.0 ** -9, 1.0625, 1.1875, 448.0, 1000.0]
    y = torch.zeros(1024, dtype=torch.int32, device="cuda")
    assert bb.blocks_pack_e4m3(torch.from_numpy(x).cuda().data_ptr(), y.data_ptr(), 1024, _stream()) == 0
    assert bb.blocks_status_sync(_stream()) == 0
    got = y.cpu().numpy().view(np.uint8)
    assert np.array_equal(got, inputs.e4m3_from_f32(x))


def test_mma_e4m3_ss_tile():
    import torch
    a = inputs.gen_e4m3(500, "q", (128, 128))
    b = inputs.gen_e4m3(500, "k", (128, 128))
    c = torch.full((128, 128), float("nan"), dtype=torch.float32, device="cuda")
    assert bb.blocks_mma_e4m3_ss(_dev_u8(a).data_ptr(), _dev_u8(b).data_ptr(), c.data_ptr(), _stream()) == 0
    assert bb.blocks_status_sync(_stream()) == 0
    ref = inputs.e4m3_to_f64(a) @ inputs.e4m3_to_f64(b).T
    got = c.cpu().numpy().astype(np.float64)
    # E4M3 products are exact in fp32; only the accumulation order differs
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-5 * np.abs(ref).max())


def test_mma_e4m3_ts_tile():
    import torch
    p = inputs.gen_e4m3(510, "q", (128, 128), dist="uniform", mult=4.0)
    v = inputs.gen_e4m3(510, "v", (128, 128))
    c = torch.full((128, 128), float("nan"), dtype=torch.float32, device="cuda")
    assert bb.blocks_mma_e4m3_ts(_dev_u8(p).data_ptr(), _dev_u8(v).data_ptr(), c.data_ptr(), _stream()) == 0
    assert bb.blocks_status_sync(_stream()) == 0
    ref = inputs.e4m3_to_f64(p) @ inputs.e4m3_to_f64(v)
    got = c.cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-5 * np.abs(ref).max())
