"""The query split of the tensor-core FP4 selection, checked on the host.

The kernel scales query row h by 2^(6 - E_h) (E_h the exponent of its largest
component, so the largest lands in [64, 128)) and feeds it to E4M3 products as
hi = rne(v) and lo = rne(v - hi).  The library states (include/cobs.h) that
two E4M3 parts hold a bf16 value exactly, that only components below 2^-8 of
the row's largest are rounded, and by at most 2^-16 of it (a component of at
least 1/4 after scaling has a last bit of at least 2^-9, the smallest E4M3
step, so its residual after hi is exact in E4M3).  E4M3 is emulated
here from its definition (bias 7, three mantissa bits, subnormals down to
2^-9, largest finite 448, round to nearest with ties to even)."""

import numpy as np

from workloads import bits_to_f64, to_bf16_bits


def e4m3_grid():
    mags = [m / 8 * 2.0 ** -6 for m in range(8)]                       # zero, subnormals
    mags += [(1 + m / 8) * 2.0 ** (e - 7) for e in range(1, 16) for m in range(8)
             if not (e == 15 and m == 7)]                                # normals, 448 last
    return np.array(sorted(set(mags)))


GRID = e4m3_grid()
CODES = np.arange(len(GRID))


def rne_e4m3(x):
    """Round to the nearest E4M3 value, ties to the even code, saturating."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), GRID[-1])
    i = np.clip(np.searchsorted(GRID, a), 1, len(GRID) - 1)
    lo, hi = GRID[i - 1], GRID[i]
    pick_hi = (a - lo > hi - a) | ((a - lo == hi - a) & (CODES[i] % 2 == 0))
    return np.sign(x) * np.where(pick_hi, hi, lo)


def split(row):
    m = np.max(np.abs(row))
    E = int(np.floor(np.log2(m))) if m > 0 else 0
    v = row * 2.0 ** (6 - E)
    hi = rne_e4m3(v)
    lo = rne_e4m3(v - hi)
    return v, hi, lo


def test_grid_is_e4m3():
    assert len(GRID) == 127 and GRID[1] == 2.0 ** -9 and GRID[-1] == 448.0
    assert GRID[8] == 2.0 ** -6                        # smallest normal
    assert rne_e4m3(2.0 ** -10) == 0.0                 # half the smallest subnormal: tie to 0
    assert rne_e4m3(1.0625) == 1.0 and rne_e4m3(1.1875) == 1.25   # ties to even mantissa
    assert rne_e4m3(1000.0) == 448.0                    # saturation


def test_two_parts_hold_bf16_rows():
    rng = np.random.default_rng(7)
    for trial in range(200):
        scale = 2.0 ** rng.integers(-20, 20)
        row = bits_to_f64(to_bf16_bits(rng.standard_normal(128) * scale
                                       * np.exp(rng.standard_normal(128) * (trial % 4))))
        v, hi, lo = split(row)
        mx = np.max(np.abs(v))
        assert 64.0 <= mx < 128.0
        err = np.abs(hi + lo - v)
        big = np.abs(v) >= 2.0 ** -8 * mx
        assert np.all(err[big] == 0.0)                  # exact from 2^-8 of the largest on
        assert np.all(err[np.abs(v) >= 0.25] == 0.0)    # i.e. from 1/4 after scaling
        assert np.all(err <= 2.0 ** -16 * mx)           # and at most 2^-16 of it below


def test_small_components_round_within_bound():
    # the largest at 64 (the weakest bound), components from 2^-4 down to 2^-12
    row = np.zeros(128)
    row[0] = 64.0
    row[1:] = bits_to_f64(to_bf16_bits(np.linspace(2.0 ** -4, 2.0 ** -12, 127)))
    v, hi, lo = split(row)
    assert np.max(np.abs(hi + lo - v)) <= 2.0 ** -16 * 64.0
