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


def test_commit_step_stop_and_cap_take_argmax_tokens():
    """E6: a canvas that stops (low mean entropy, argmax equal to the previous pass's)
    or reaches the last pass commits every masked slot with its argmax token; others
    commit by the entropy bound with the drawn tokens."""
    mask = 0
    canvas = np.array([[0, 5, 0, 0], [0, 0, 0, 0], [0, 0, 7, 0]], np.int32)
    H = np.array([[0.001, 0.0, 0.002, 0.003],        # mean 0.0015, stable -> stops
                  [0.06, 0.05, 0.04, 0.03],          # mean above the threshold
                  [0.001, 0.001, 0.001, 0.001]])     # low, but argmax changed
    a = np.array([[11, 12, 13, 14], [21, 22, 23, 24], [31, 32, 33, 34]], np.int32)
    prev = np.array([[11, 12, 13, 14], [21, 22, 23, 24], [31, 32, 33, 99]], np.int32)
    drawn = a + 100
    new, com, stop = eb.eb_commit_step(canvas, H, a, drawn, prev, mask, last=False)
    assert stop.tolist() == [True, False, False]
    assert new[0].tolist() == [11, 5, 13, 14]                 # argmax, committed slot kept
    # canvas 1: entropy order 3, 2, 1, 0: 0.03 + 0.04 = 0.07 <= 0.1 < 0.12
    assert new[1].tolist() == [0, 0, 123, 124]
    # canvas 2: all four fit in the bound (drawn tokens), the committed slot is kept
    assert new[2].tolist() == [131, 132, 7, 134]
    assert com.sum(axis=1).tolist() == [3, 2, 3]
    # the last pass commits everything left with argmax tokens; no previous pass -> no stop
    new2, com2, stop2 = eb.eb_commit_step(canvas, H, a, drawn, None, mask, last=True)
    assert not stop2.any()
    assert (new2 != mask).all() and new2[1].tolist() == [21, 22, 23, 24]


def _identity_layers_cfg(om, canvas_len):
    cfg = om.OracleConfig(n_layers=1, d_model=2, n_q_heads=1, n_kv_heads=1, head_dim=2,
                          n_experts=1, top_k=1, n_shared=0, d_ff=2, vocab=4,
                          canvas_len=canvas_len, window=4, global_every=1, rms_eps=1e-6)
    z = np.zeros((2, 2))

    class W(om.LayerWeights):
        def __init__(self):
            super().__init__(cfg, 0)
            self._cache.update({"wq": z, "wk": z, "wv": z, "wo": z, "wr": np.zeros((1, 2))})

        def expert(self, e):
            return (z, z, z)
    return cfg, [W()]


def test_block_stops_at_the_second_pass_on_peaked_identical_rows(monkeypatch):
    """Identity blocks and an embedding whose rows 0 (mask) and 1 point the same way:
    every slot's final-normed state is the same, so every pass sees the same
    entropy h(T) on all slots and argmax 1 everywhere.  Pass 0 commits, by the
    bound, the largest n with n * h(T0) <= 0.1; pass 1 sees the same argmax and a
    mean entropy below 0.005, so the canvas stops and the rest take token 1."""
    from oracle import model as om
    a = 4.6
    emb = np.array([[1.0, 0.0], [a, 0.0], [0.0, 0.0], [-a, 0.0]])
    monkeypatch.setattr(om, "embedding_rows", lambda cfg, rows: emb[np.asarray(rows).ravel()])
    monkeypatch.setattr(om, "embedding_block", lambda cfg, v0, v1: emb[v0:v1])
    Tc = 40
    cfg, weights = _identity_layers_cfg(om, Tc)
    kp = np.zeros((1, 1, 2, 2))
    u = np.full((48, 1, Tc), 0.5)
    hist = []
    canvas, passes = eb.eb_denoise_block(cfg, np.zeros((1, Tc), np.int32), [kp], [kp], u,
                                         weights=weights, history=hist)
    # h(T0): logits over tokens 1..3 are (a, 0, -a) * sqrt(2) / sqrt(1 + eps)
    s = math.sqrt(2.0) / math.sqrt(1.0 + 1e-6)
    z = np.array([0.0, -a * s, -2 * a * s]) / 0.8
    p = np.exp(z) / np.exp(z).sum()
    h0 = float(-(p * np.log(p)).sum())
    n1, tot = 0, 0.0
    while n1 < Tc and tot + h0 <= 0.1:
        tot += h0
        n1 += 1
    assert 1 < n1 < Tc and h0 < 0.005
    assert int(hist[0]["committed"].sum()) == n1 and not hist[0]["stopped"].any()
    assert hist[1]["stopped"].all() and int(hist[1]["committed"].sum()) == Tc - n1
    assert passes.tolist() == [2] and (canvas == 1).all()


def test_block_with_high_entropy_commits_one_slot_per_pass_then_all_at_the_cap():
    """Random weights give entropies near ln(vocab): the bound admits only the single
    lowest-entropy slot per pass (at least one), and the last allowed pass commits
    every remaining slot with its argmax token.  No slot ever reverts."""
    from oracle import model as om
    cfg = om.OracleConfig(n_layers=1, d_model=64, n_q_heads=2, n_kv_heads=1, head_dim=32,
                          n_experts=4, top_k=2, n_shared=1, d_ff=64, vocab=97, canvas_len=8,
                          window=4, global_every=1)
    g = np.random.default_rng(11)
    kp = [g.standard_normal((1, 1, 5, 32))]
    vp = [g.standard_normal((1, 1, 5, 32))]
    n_max = 4
    u = g.uniform(size=(n_max, 1, 8))
    hist = []
    canvas, passes = eb.eb_denoise_block(cfg, np.zeros((1, 8), np.int32), kp, vp, u,
                                         n_max=n_max, history=hist)
    assert [int(h["committed"].sum()) for h in hist] == [1, 1, 1, 5]
    assert passes.tolist() == [4] and (canvas != 0).all()
    prev = np.zeros((1, 8), np.int32)
    for h in hist:
        keep = prev != 0
        assert np.array_equal(h["canvas"][keep], prev[keep])
        c = h["committed"][0]
        if c.sum() == 1:   # the lowest-entropy masked slot, with its drawn token
            i = int(np.nonzero(c)[0][0])
            masked = prev[0] == 0
            assert h["H"][0, i] == h["H"][0][masked].min()
            assert h["canvas"][0, i] == h["drawn"][0, i]
        prev = h["canvas"]
