"""GPU checks of the sm_100a building blocks, one at a time, through the
self-test C ABI (include/fa_selftest.h)."""
import numpy as np
import pytest
import torch

from exact_io_aware_52_b200 import _binding as fb

pytestmark = pytest.mark.gpu


def _dev():
    return torch.device("cuda:0")


def _status():
    return torch.zeros(1, dtype=torch.int32, device=_dev())


def _p(t):
    return t.data_ptr()


def test_tma_128b_swizzle_image():
    """A 128x64 bf16 box lands in shared memory with the 128-byte swizzle:
    16-byte chunk c of row r sits at chunk position c xor (r mod 8)."""
    lib = fb.load_selftest()
    src = torch.arange(128 * 64, dtype=torch.int32).reshape(128, 64)
    src_bits = (src & 0x7FFF).to(torch.int16)  # distinct 16-bit patterns per element
    src_d = src_bits.view(torch.bfloat16).to(_dev())
    dst = torch.zeros(16384, dtype=torch.uint8, device=_dev())
    st = _status()
    assert lib.fa_selftest_tma_sw128(_p(src_d), _p(dst), _p(st), None) == 0
    assert st.item() == 0
    img = dst.cpu().numpy().view(np.int16)
    expect = np.zeros(128 * 64, dtype=np.int16)
    s = src_bits.numpy()
    for r in range(128):
        for c in range(64):
            chunk, within = divmod(c, 8)
            pos = r * 64 + ((chunk ^ (r % 8)) * 8) + within
            expect[pos] = s[r, c]
    np.testing.assert_array_equal(img, expect)


@pytest.mark.parametrize("K", [64, 128])
def test_tcgen05_ss_matches_matmul(K):
    """S = A B^T on the tensor cores (both operands K-major, 128-byte swizzle)
    equals the float64 product of the same bf16 values to fp32 accuracy."""
    lib = fb.load_selftest()
    g = torch.Generator().manual_seed(100 + K)
    a = torch.randn(128, K, generator=g).to(torch.bfloat16)
    b = torch.randn(128, K, generator=g).to(torch.bfloat16)
    s = torch.full((128, 128), float("nan"), device=_dev())
    st = _status()
    assert lib.fa_selftest_mma_ss(_p(a.to(_dev())), _p(b.to(_dev())), _p(s), K, _p(st), None) == 0
    assert st.item() == 0
    ref = a.double() @ b.double().T
    np.testing.assert_allclose(s.cpu().double().numpy(), ref.numpy(), rtol=0, atol=2e-4)


@pytest.mark.parametrize("D", [64, 128])
def test_tcgen05_ts_matches_matmul(D):
    """O = P V with P staged in tensor memory (two bf16 per column) and V
    MN-major in shared memory equals the float64 product."""
    lib = fb.load_selftest()
    g = torch.Generator().manual_seed(200 + D)
    p = torch.rand(128, 128, generator=g).to(torch.bfloat16)
    v = torch.randn(128, D, generator=g).to(torch.bfloat16)
    o = torch.full((128, D), float("nan"), device=_dev())
    st = _status()
    assert lib.fa_selftest_mma_ts(_p(p.to(_dev())), _p(v.to(_dev())), _p(o), D, _p(st), None) == 0
    assert st.item() == 0
    ref = p.double() @ v.double()
    np.testing.assert_allclose(o.cpu().double().numpy(), ref.numpy(), rtol=0, atol=2e-4)


def test_tcgen05_e4m3_ss_matches_matmul():
    """S = A B^T with E4M3 operands (kind::f8f6f4, K-major, 128-byte rows)
    equals the float64 product of the same E4M3 values."""
    lib = fb.load_selftest()
    g = torch.Generator().manual_seed(300)
    a = (torch.randn(128, 128, generator=g) * 3).to(torch.float8_e4m3fn)
    b = (torch.randn(128, 128, generator=g) * 3).to(torch.float8_e4m3fn)
    s = torch.full((128, 128), float("nan"), device=_dev())
    st = _status()
    assert lib.fa_selftest_mma_e4m3_ss(_p(a.to(_dev())), _p(b.to(_dev())), _p(s), _p(st), None) == 0
    assert st.item() == 0
    ref = a.double() @ b.double().T
    np.testing.assert_allclose(s.cpu().double().numpy(), ref.numpy(), rtol=1e-6, atol=1e-4)


def test_tcgen05_e4m3_ts_matches_matmul():
    """O = E4M3(P) V: P (fp32, spanning the E4M3 subnormals up to 256) rounded
    and packed four per TMEM column by the kernel's packer, V MN-major; equals
    the float64 product of torch's E4M3 rounding of P with V."""
    lib = fb.load_selftest()
    g = torch.Generator().manual_seed(301)
    p = torch.exp2(torch.rand(128, 128, generator=g) * 22 - 14)  # 2^-14 .. 2^8
    v = torch.randn(128, 128, generator=g).to(torch.float8_e4m3fn)
    o = torch.full((128, 128), float("nan"), device=_dev())
    st = _status()
    assert lib.fa_selftest_mma_e4m3_ts(_p(p.to(_dev())), _p(v.to(_dev())), _p(o), _p(st), None) == 0
    assert st.item() == 0
    ref = p.to(torch.float8_e4m3fn).double() @ v.double()
    np.testing.assert_allclose(o.cpu().double().numpy(), ref.numpy(), rtol=1e-5, atol=1e-4)


def test_bounded_wait_gives_up():
    """A wait on a barrier nothing arrives at gives up after its limit,
    reports FA_ERR_DEVICE_TIMEOUT, and the context stays usable."""
    import time
    lib = fb.load_selftest()
    st = _status()
    t0 = time.time()
    assert lib.fa_selftest_wait_timeout(_p(st), 200, None) == 0
    dt = time.time() - t0
    assert st.item() == fb.FA_ERR_DEVICE_TIMEOUT
    assert dt < 5.0
    x = torch.ones(16, device=_dev())
    assert float((x * 2).sum().item()) == 32.0


def test_polynomial_exp2_error_bound():
    """The FMA-pipe 2^x: relative error <= 4e-6 against float64 exp2 over the
    range the softmax feeds it ([-127, 8]), exact powers of two at integers
    (p(0) = 1), and +0 (to within the error) for inputs at or below -127."""
    lib = fb.load_selftest()
    x = torch.cat([torch.linspace(-126.0, 8.0, 1 << 20), torch.arange(-126, 9, dtype=torch.float32),
                   torch.tensor([-127.0, -200.0, -1e30, float("-inf")])])
    if x.numel() % 2:
        x = torch.cat([x, torch.zeros(1)])
    xd = x.to(_dev())
    y = torch.empty_like(xd)
    assert lib.fa_selftest_exp2_poly(_p(xd), _p(y), x.numel(), None) == 0
    yy = y.cpu().double()
    ref = torch.exp2(x.double())
    live = x >= -126
    rel = ((yy[live] - ref[live]) / ref[live]).abs()
    assert rel.max().item() <= 4e-6, rel.max().item()
    ints = (x == x.round()) & live
    assert torch.equal(yy[ints], ref[ints])
    assert (yy[~live].abs() <= 1e-43).all()



def test_exponential_unit_rate():
    """Measurement behind the softmax design: one SM sub-partition delivers at
    most 4 exp2 lanes per clock (16 per SM), and one warp alone gets less of
    that than two side by side, least with the softmax's own mix of work."""
    import ctypes
    lib = fb.load_selftest()
    rate = {}
    for mix in (0, 1):
        for w in (1, 2):
            c = ctypes.c_double(0.0)
            assert lib.fa_selftest_mufu_rate(w, mix, 200, ctypes.byref(c), None) == 0
            rate[mix, w] = 128 * 32 * w / c.value
    print("exp2 lanes per clock per sub-partition (ex2 only, 1 and 2 warps; softmax mix, 1 and 2 warps):",
          ", ".join(f"{rate[k]:.2f}" for k in sorted(rate)))
    assert all(0.0 < r <= 4.2 for r in rate.values()), rate
    assert rate[0, 2] >= rate[0, 1] and rate[1, 2] >= rate[1, 1], rate
    assert lib.fa_selftest_mufu_rate(0, 0, 10, ctypes.byref(ctypes.c_double()), None) == 1
