"""Host check of the INT8 rounding argument the CUDA path relies on.

The kernels form an INT8 code as the low byte of RN(RN(x * inv) + 1.5 * 2^23)
(the magic-number conversion) with inv = RN(127 / a) and |x| <= a, the block's
absolute maximum. This restates that step in IEEE fp32 with numpy and checks it
against round-half-to-even of RN(x * inv) and the [-127, 127] range, including
exact halfway products and extreme block maxima."""
import numpy as np

MAGIC = np.float32(12582912.0)   # 1.5 * 2^23


def magic_codes(x, inv):
    p = (x * inv).astype(np.float32)
    low = (p + MAGIC).astype(np.float32).view(np.uint32) & np.uint32(0xFF)
    low = low.astype(np.int32)
    return np.where(low >= 128, low - 256, low), p


def test_magic_rounding_is_round_half_even_and_in_range():
    rng = np.random.default_rng(11)
    for e in np.linspace(-36.0, 37.0, 147):
        a = np.float32(10.0 ** e)
        if not np.isfinite(np.float32(127.0) / a):
            continue
        x = (rng.uniform(-1.0, 1.0, 4096) * a).astype(np.float32)
        x[:2] = (a, -a)
        inv = np.float32(np.float32(127.0) / a)
        codes, p = magic_codes(x, inv)
        np.testing.assert_array_equal(codes, np.rint(p).astype(np.int32))
        assert np.abs(codes).max() <= 127


def test_magic_rounding_halfway_products_go_to_even():
    a = np.float32(127.0)
    inv = np.float32(1.0)
    x = (np.arange(-127, 127, dtype=np.float32) + np.float32(0.5)).astype(np.float32)
    codes, _ = magic_codes(x, inv)
    expect = np.rint(x).astype(np.int32)          # half to even
    np.testing.assert_array_equal(codes, expect)
    assert (codes % 2 == 0).all()
