"""Pins of the oracle's FP4 (E2M1) storage of U against what fixes it from
outside the oracle: the E2M1 bit-field definition (1 sign bit, 2 exponent bits
with bias 1, 1 mantissa bit, subnormal when the exponent field is 0), brute
force over every code for round-to-nearest with ties to even, the defining
inequality of the scale exponent, and the rounding error bound that follows
from the grid spacing (COBS explainer §2.3, quantisation)."""

import math

import numpy as np
import pytest

import oracle.cobs_oracle as O


def e2m1_from_bits(c: int) -> float:
    sign = -1.0 if c & 8 else 1.0
    ex, man = (c >> 1) & 3, c & 1
    if ex == 0:
        return sign * man * 0.5                      # subnormal: 0.M x 2^(1-bias)
    return sign * 2.0 ** (ex - 1) * (1.0 + 0.5 * man)


ALL_VALUES = np.array([e2m1_from_bits(c) for c in range(16)])


def test_code_values_match_the_bit_field_definition():
    np.testing.assert_array_equal(O.e2m1_value(np.arange(16)), ALL_VALUES)
    assert sorted(set(np.abs(ALL_VALUES))) == list(O.E2M1_MAGNITUDES)


def test_rounding_is_nearest_with_ties_to_even_by_brute_force():
    rng = np.random.default_rng(1)
    mids = [(a + b) / 2 for a, b in zip(O.E2M1_MAGNITUDES, O.E2M1_MAGNITUDES[1:])]
    xs = np.concatenate([rng.uniform(-7.5, 7.5, 4000), np.array(mids), -np.array(mids),
                         np.array(O.E2M1_MAGNITUDES), [6.0 + 1e-12, 1e9, -1e9, 0.0, -0.0]])
    codes = O.round_to_e2m1(xs)
    for x, c in zip(xs, codes):
        v = O.e2m1_value(c)
        target = float(np.clip(x, -6.0, 6.0))
        dist = np.abs(ALL_VALUES - target)
        assert abs(v - target) == dist.min(), (x, c)
        nearest = [k for k in range(16) if dist[k] == dist.min()]
        mags = {k & 7 for k in nearest}
        if len(mags) > 1:                  # a tie between two magnitudes: the even one
            assert (int(c) & 7) % 2 == 0, (x, c)
        if v == 0.0:
            assert int(c) == 0             # zero is always the positive code


def test_known_ties():
    cases = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for x, want in cases.items():
        assert O.e2m1_value(O.round_to_e2m1(x)) == want
        assert O.e2m1_value(O.round_to_e2m1(-x)) == -want


def test_scale_exponent_is_the_smallest_that_fits():
    rng = np.random.default_rng(2)
    amaxes = list(np.exp(rng.uniform(-80, 80, 2000)))
    for k in range(-20, 21):               # exact boundaries and their neighbours
        amaxes += [6.0 * 2.0 ** k, np.nextafter(6.0 * 2.0 ** k, np.inf),
                   np.nextafter(6.0 * 2.0 ** k, 0.0), 2.0 ** k]
    for amax in amaxes:
        e = O.fp4_scale_exponent(float(amax))
        assert amax <= 6.0 * 2.0 ** e
        assert e == -126 or amax > 6.0 * 2.0 ** (e - 1)
    assert O.fp4_scale_exponent(6.0) == 0
    assert O.fp4_scale_exponent(6.0 * 2.0 ** -200) == -126
    assert O.fp4_scale_exponent(0.0) is None


def grid_step(mag):
    """Spacing of the E2M1 grid around a magnitude in [0, 6]."""
    return np.where(mag <= 2.0, 0.5, np.where(mag <= 4.0, 1.0, 2.0))


def test_quantised_components_within_half_a_grid_step():
    rng = np.random.default_rng(3)
    for scale in (1e-3, 0.1, 3.0, 1e4):
        u = rng.normal(size=(5, 128)) * scale
        u[1, 40:72] = 0.0                              # a group of zeros
        codes, sb = O.quantize_u_fp4(u)
        deq = O.dequantize_u_fp4(codes, sb)
        for j in range(5):
            for g in range(4):
                seg = u[j, 32 * g:32 * (g + 1)]
                if not np.any(seg):
                    assert sb[j, g] == 0 and not np.any(codes[j, 32 * g:32 * (g + 1)])
                    continue
                e = int(sb[j, g]) - 127
                assert e == O.fp4_scale_exponent(float(np.max(np.abs(seg))))
                x = seg / 2.0 ** e
                err = np.abs(deq[j, 32 * g:32 * (g + 1)] - seg) / 2.0 ** e
                assert np.all(err <= grid_step(np.abs(x)) / 2 + 1e-12)
                # the largest component never saturates
                assert np.max(np.abs(x)) <= 6.0


def test_grid_values_round_trip_exactly():
    rng = np.random.default_rng(4)
    mags = np.array(O.E2M1_MAGNITUDES)
    u = rng.choice(mags, size=(3, 64)) * rng.choice([-1.0, 1.0], size=(3, 64))
    u[:, 0] = 6.0                 # every group holds a +-6: its exponent is the one used
    u[:, 32] = -6.0
    u *= 2.0 ** np.array([-3, 0, 5])[:, None]
    codes, sb = O.quantize_u_fp4(u)
    np.testing.assert_array_equal(O.dequantize_u_fp4(codes, sb), u)


def test_fp4_record_keeps_mu_and_scores_from_the_dequantised_factor():
    """mu is the bf16 record's row 0; with U made exactly representable the FP4
    score equals the exact second-order score."""
    rng = np.random.default_rng(5)
    keys = O.round_to_bf16(rng.normal(0.0, 0.5, size=(64, 64)))
    mu, codes, sb = O.block_record_fp4(keys, 4)
    rec = O.block_record(keys, 4)
    np.testing.assert_array_equal(mu, rec[0])
    vals = O.fp4_record_values(mu[None], codes[None], sb[None])
    assert vals.shape == (1, 5, 64)
    np.testing.assert_array_equal(vals[0, 1:], O.dequantize_u_fp4(codes, sb))
    q = rng.normal(size=64)
    exact = O.head_block_scores(q, vals, np.array([64]))
    by_hand = (math.log(64) + vals[0, 0] @ q / 8.0
               + 0.5 * sum((vals[0, j] @ q) ** 2 for j in range(1, 5)) / 64.0)
    assert exact[0] == pytest.approx(by_hand, rel=1e-12)


def test_fp4_factor_error_bounded_by_the_grid():
    """Against the exact factor of a real block: every component within half
    a grid step of its group's scale."""
    rng = np.random.default_rng(6)
    keys = O.round_to_bf16(rng.normal(0.0, 0.5, size=(64, 128)))
    _, sigma = O.block_moments(keys)
    u, _ = O.covariance_factor(sigma, 8)
    _, codes, sb = O.block_record_fp4(keys, 8)
    deq = O.dequantize_u_fp4(codes, sb)
    step = np.repeat(np.exp2(sb.astype(float) - 127), 32, axis=1)
    assert np.all(np.abs(deq - u.T) <= step + 1e-15)


# ---------------------------------------------------------------------------
# plausible mistakes planted in the oracle (on the CPU) must trip a pin
# ---------------------------------------------------------------------------

def _expect_pin_failure(monkeypatch, name, bad, pin):
    monkeypatch.setattr(O, name, bad)
    with pytest.raises(AssertionError):
        pin()


def test_mutation_ties_to_odd(monkeypatch):
    def bad(x):
        x = np.asarray(x, dtype=np.float64)
        a = np.minimum(np.abs(x), 6.0)
        grid = np.asarray(O.E2M1_MAGNITUDES)
        dist = np.abs(a[..., None] - grid)
        nearest = dist == dist.min(axis=-1, keepdims=True)
        pick = len(grid) - 1 - np.argmax(nearest[..., ::-1], axis=-1)   # the larger code
        return np.where((x < 0) & (pick != 0), pick | 8, pick).astype(np.uint8)
    _expect_pin_failure(monkeypatch, "round_to_e2m1", bad, test_known_ties)


def test_mutation_saturating_exponent(monkeypatch):
    def bad(amax):   # floor(log2 amax) - 2: values in (6, 8) x 2^e would clip
        if amax == 0.0:
            return None
        return max(int(math.floor(math.log2(amax))) - 2, -126)
    _expect_pin_failure(monkeypatch, "fp4_scale_exponent", bad,
                        test_scale_exponent_is_the_smallest_that_fits)


def test_mutation_wrong_grid(monkeypatch):
    monkeypatch.setattr(O, "E2M1_MAGNITUDES", (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 5.0))
    with pytest.raises(AssertionError):
        test_code_values_match_the_bit_field_definition()


def test_mutation_groups_of_16(monkeypatch):
    def bad(u_rows):
        u_rows = np.asarray(u_rows, dtype=np.float64)
        r, d = u_rows.shape
        codes = np.zeros((r, d), dtype=np.uint8)
        scale_bytes = np.zeros((r, d // 32), dtype=np.uint8)
        for j in range(r):
            for g in range(d // 16):
                seg = u_rows[j, g * 16:(g + 1) * 16]
                e = O.fp4_scale_exponent(float(np.max(np.abs(seg))))
                if e is None:
                    continue
                scale_bytes[j, g // 2] = e + 127
                codes[j, g * 16:(g + 1) * 16] = O.round_to_e2m1(seg / 2.0 ** e)
        return codes, scale_bytes
    _expect_pin_failure(monkeypatch, "quantize_u_fp4", bad,
                        test_quantised_components_within_half_a_grid_step)
