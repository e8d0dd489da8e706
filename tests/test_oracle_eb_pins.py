"""Pins of the entropy-bounded sampler oracle: the pages' settings, closed forms,
hand-worked cases and a library entropy (no GPU)."""

import math

import numpy as np
import pytest
from scipy.stats import entropy as scipy_entropy

from oracle import eb_sampler as eb


def test_settings_are_the_pages_values():
    assert (eb.N_MAX_STEPS, eb.T_START, eb.T_END) == (48, 0.8, 0.4)
    assert (eb.ENTROPY_BOUND, eb.STOP_ENTROPY, eb.STOP_STABLE_STEPS) == (0.1, 0.005, 2)


def test_temperature_falls_linearly_between_the_endpoints():
    assert eb.eb_temperature(0) == pytest.approx(0.8)
    assert eb.eb_temperature(47) == pytest.approx(0.4)
    t = [eb.eb_temperature(s) for s in range(48)]
    d = np.diff(t)
    assert np.allclose(d, d[0]) and d[0] < 0
    with pytest.raises(ValueError):
        eb.eb_temperature(48)


def test_entropy_closed_forms_and_library():
    V, mask = 9, 4
    # equal logits: uniform over the V - 1 tokens that are not the mask
    H, a, p = eb.eb_row_stats(np.zeros((1, V)), mask, 0.8)
    assert H[0] == pytest.approx(math.log(V - 1))
    assert a[0] == 0 and p[0, mask] == 0
    # one dominant logit: entropy ~ 0 and that token is the argmax
    l = np.zeros((1, V)); l[0, 7] = 200.0
    H, a, _ = eb.eb_row_stats(l, mask, 0.5)
    assert H[0] < 1e-12 and a[0] == 7
    # a random row against scipy on the temperature-scaled distribution
    rng = np.random.default_rng(3)
    l = rng.standard_normal((1, V))
    T = 0.6
    H, _, p = eb.eb_row_stats(l, mask, T)
    q = np.exp(np.delete(l[0], mask) / T)
    assert H[0] == pytest.approx(scipy_entropy(q / q.sum()))
    assert p[0].sum() == pytest.approx(1.0)


def test_lower_temperature_lowers_entropy():
    l = np.random.default_rng(5).standard_normal((3, 17))
    hs = [eb.eb_row_stats(l, 0, T)[0] for T in (0.8, 0.6, 0.4)]
    assert np.all(hs[0] > hs[1]) and np.all(hs[1] > hs[2])


def test_inverse_cdf_sampling_hand_cases():
    p = np.array([[0.1, 0.2, 0.3, 0.4]])
    for u, want in ((0.05, 0), (0.1, 1), (0.25, 1), (0.31, 2), (0.61, 3), (0.999, 3)):
        assert eb.eb_sample(p, np.array([u]))[0] == want, u
    # a zero-probability token (the mask) is never drawn
    p = np.array([[0.5, 0.0, 0.5]])
    assert eb.eb_sample(p, np.array([0.5]))[0] == 2
    assert eb.eb_sample(p, np.array([0.4999]))[0] == 0


def test_unmask_takes_the_entropy_bounded_prefix():
    M = 9
    canvas = np.full((1, 5), M, np.int32)
    canvas[0, 4] = 2                                   # already committed
    H = np.array([[0.02, 0.05, 0.08, 0.001, 0.0]])
    tok = np.array([[10, 11, 12, 13, 14]], np.int32)
    new, com = eb.eb_unmask(canvas, H, tok, M, 0.1)
    # entropy order 3, 0, 1, 2: sums 0.001, 0.021, 0.071, 0.151 -> slots 3, 0, 1
    assert com[0].tolist() == [True, True, False, True, False]
    assert new[0].tolist() == [10, 11, M, 13, 2]
    # the lowest-entropy slot is committed even above the bound
    new, com = eb.eb_unmask(canvas, H + 1.0, tok, M, 0.1)
    assert com[0].tolist() == [False, False, False, True, False]
    # ties in entropy: the lower slot first
    new, com = eb.eb_unmask(np.full((1, 3), M, np.int32), np.full((1, 3), 0.06), tok[:, :3], M, 0.1)
    assert com[0].tolist() == [True, False, False]


def test_adaptive_stop_needs_low_entropy_and_stable_argmax():
    a, b = np.array([1, 2, 3]), np.array([1, 2, 4])
    assert not eb.eb_should_stop([0.004], [a])                  # one pass: no consensus yet
    assert eb.eb_should_stop([0.01, 0.004], [a, a])             # two consecutive passes agree
    assert not eb.eb_should_stop([0.004, 0.006], [a, a, a])     # entropy not low enough
    assert not eb.eb_should_stop([0.004], [a, a, b])            # the latest pass changed
    assert eb.eb_should_stop([0.004], [b, a, a])                # older changes do not matter
    assert not eb.eb_should_stop([0.004], [a, b])
    # with stable = 3 the latest three passes must agree
    assert not eb.eb_should_stop([0.004], [b, a, a], stable=3)
    assert eb.eb_should_stop([0.004], [a, a, a], stable=3)
