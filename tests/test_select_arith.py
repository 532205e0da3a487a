"""The long-row selection's integer arithmetic (select_hist_kernel), emulated in fp32 with
NumPy: the two-part fixed-point mass is exact, its sums fit in int32, and the bucket map is
monotone.  These are the properties the kernel's exact-sum Top-p rests on; the GPU parity
tests check the masks themselves.  fp32 operations are emulated one rounding at a time;
an fma whose product is exact (a power-of-two scale) is an fp32 add."""
import numpy as np

SHIFT = np.float32(12582912.0)          # 1.5 * 2^23
SHIFT_BITS = np.int64(0x4B400000)


def mass_parts(w):
    """hh, hl with w * 2^32 = hh * 2^20 + hl, as the kernel forms them from an fp32 w."""
    w = np.asarray(w, np.float32)
    a = (w * np.float32(4096.0)).astype(np.float32)                  # exact
    t1 = (a + SHIFT).astype(np.float32)
    r = (t1 - SHIFT).astype(np.float32)
    lo = (a - r).astype(np.float32)
    t2 = (lo * np.float32(1048576.0) + SHIFT).astype(np.float32)   # lo * 2^20 exact, one rounding
    hh = t1.view(np.int32).astype(np.int64) - SHIFT_BITS
    hl = t2.view(np.int32).astype(np.int64) - SHIFT_BITS
    return hh, hl


def bucket(x, mx):
    """round(32 (max - x) + delta) clamped to [0, 511], from the bits of fl(cb - 32 x)."""
    x = np.asarray(x, np.float32)
    cb = (np.float32(mx) * np.float32(32.0) + SHIFT).astype(np.float32)
    u = (cb - x * np.float32(32.0)).astype(np.float32)               # 32 x exact
    b = u.view(np.int32).astype(np.int64) - SHIFT_BITS
    return np.clip(b, 0, 511)


def round_half_even(v):
    return np.round(v)      # NumPy rounds half to even


def test_mass_parts_encode_the_rounded_mass_exactly():
    rng = np.random.default_rng(3)
    w = np.concatenate([rng.random(200000), 2.0 ** -rng.uniform(0, 40, 200000), [1.0, 0.5, 2.0 ** -33, 0.0],
                        rng.random(50000) * rng.integers(1, 129, 50000)]).astype(np.float32)
    hh, hl = mass_parts(w)
    want = round_half_even(w.astype(np.float64) * 2.0 ** 32)        # exact in fp64 (w has 24 bits)
    assert np.array_equal(hh * 2 ** 20 + hl, want.astype(np.int64))
    assert (np.abs(hl) <= 2 ** 19).all()
    # a block's mass is at most 2^7 tokens times the row maximum's: hh <= 2^19, so over 2^11
    # blocks the high sums stay below 2^30 and the low sums within +-2^30
    assert hh.max() <= 2 ** 19 and hh.min() >= 0


def test_mass_sums_fit_int32_at_the_limits():
    w = np.full(2048, 128.0, np.float32)          # 2^11 blocks of 2^7 tokens at the maximum
    hh, hl = mass_parts(w)
    assert hh.sum() <= 2 ** 30 < 2 ** 31 - 1
    rng = np.random.default_rng(5)
    w = (rng.random(2048) * 128).astype(np.float32)
    hh, hl = mass_parts(w)
    assert abs(hl.sum()) <= 2 ** 30


def test_bucket_map_is_monotone_and_starts_at_the_maximum():
    rng = np.random.default_rng(11)
    for _ in range(200):
        row = (rng.normal(0, rng.uniform(0.1, 5), 1936) + rng.uniform(-50, 50)).astype(np.float32)
        mx = row.max()
        b = bucket(row, mx)
        order = np.argsort(-row.astype(np.float64), kind="stable")
        assert (np.diff(b[order]) >= 0).all()            # a higher logit never lands later
        assert b[row == mx].max() == 0
        assert ((b >= 0) & (b <= 511)).all()
    assert bucket(np.float32(-np.inf), np.float32(3.0)) == 511


def test_bucket_width_is_one_32nd_of_a_logit():
    mx = np.float32(1.25)
    x = (mx - np.arange(0, 400, dtype=np.float64) / 32.0).astype(np.float32)
    b = bucket(x, mx)
    assert np.array_equal(b, np.minimum(np.arange(400), 511))
