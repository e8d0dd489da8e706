"""Pins of the CPU oracle to things other than itself (CPU only).

Each test ties one oracle function to a published value, a closed form, an
identity, a library routine computing the same quantity a different way, or
a brute-force scalar restatement on tiny inputs.  A dropped term, a wrong
sign or index or a transposed operand in the oracle fails at least one.
"""

import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from oracle import model as om
from oracle import rng as orng

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


def tiny_cfg(**kw):
    base = dict(n_layers=1, d_model=64, n_q_heads=4, n_kv_heads=2, head_dim=16, n_experts=4,
                top_k=2, n_shared=1, d_ff=32, vocab=97, canvas_len=8, window=5, global_every=2,
                bf16_weights=True)
    base.update(kw)
    return om.OracleConfig(**base)


# ----------------------------------------------------------------------------- generator

def test_splitmix64_published_vectors():
    for line in open(os.path.join(GOLDEN, "splitmix64_vectors.txt")):
        if line.startswith("#") or not line.strip():
            continue
        vals = [int(v, 0) for v in line.split()]
        seed, expect = vals[0], vals[1:]
        # streaming form: state += GAMMA; out = mix(state)
        got = [int(u) for u in orng.splitmix64_outputs(seed, 0, len(expect))]
        assert got == expect
        # offset form: the i-th output alone
        for i, e in enumerate(expect):
            assert int(orng.splitmix64_outputs(seed, i, 1)[0]) == e
            assert orng.splitmix64_mix((seed + (i + 1) * orng.GAMMA) & orng.MASK64) == e


def test_irwin_hall_moments_and_bounds():
    key = orng.splitmix64_stream_key(0, 5)
    u = orng.splitmix64_outputs(key, 0, 1 << 21)
    x = orng.irwin_hall_normal_f32(u, 0.02).astype(np.float64)
    n = x.size
    # mean 0, variance std^2 * (1 - 2^-32) (sum of four discrete uniforms on 0..65535)
    assert abs(x.mean()) < 4 * 0.02 / math.sqrt(n)
    assert abs(x.var() / 0.02 ** 2 - 1) < 0.01
    assert np.abs(x).max() <= 131070 * np.float32(0.02 * math.sqrt(3) / 65536) * (1 + 1e-6)
    # fourth standardised moment of a 4-term Irwin-Hall sum: 3 - 6/(5*4) = 2.7
    k4 = np.mean(((x - x.mean()) / x.std()) ** 4)
    assert abs(k4 - 2.7) < 0.03
    # the 16-bit fields are what is summed: one hand-built output
    u1 = np.array([(1 << 48) | (2 << 32) | (3 << 16) | 4], dtype=np.uint64)
    z = orng.irwin_hall_normal_f32(u1, 1.0)[0]
    assert z == np.float32(10 - 131070) * np.float32(math.sqrt(3) / 65536)


def test_bf16_rounding_against_torch_and_hand_cases():
    one = 1.0
    cases = {one: one, one + 2 ** -8: one,                        # tie -> even (1.0)
             one + 3 * 2 ** -8: one + 2 ** -6,                    # tie -> even (upper)
             one + 2 ** -8 + 2 ** -20: one + 2 ** -7, -2.5: -2.5}
    for a, b in cases.items():
        assert orng.round_to_bf16(np.array([a], np.float32))[0] == np.float32(b)
    x = (RNG.standard_normal(100000) * np.exp(RNG.uniform(-20, 20, 100000))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(orng.round_to_bf16(x), ref)


def test_weight_tensor_slices_are_consistent():
    full = orng.weight_tensor(0, 77, (6, 10), 0.02, True)
    part = orng.weight_tensor(0, 77, (2, 10), 0.02, True, start=30)
    assert np.array_equal(full[3:5], part)
    other = orng.weight_tensor(0, 78, (6, 10), 0.02, True)
    assert not np.array_equal(full, other)


# ----------------------------------------------------------------------------- norm / rope

def test_rmsnorm_against_torch_and_closed_form():
    x = RNG.standard_normal((7, 33)) * 3
    w = RNG.standard_normal(33)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (33,), torch.from_numpy(w), eps=1e-6)
    assert np.allclose(om.rmsnorm(x, w, 1e-6), ref.numpy(), rtol=1e-12, atol=1e-12)
    y = om.rmsnorm(x, np.ones(33), 0.0)
    assert np.allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-12)
    assert np.allclose(om.rmsnorm(5.0 * x, w, 0.0), om.rmsnorm(x, w, 0.0), rtol=1e-12)


def test_rope_against_complex_rotation():
    dh, T, H = 16, 5, 3
    x = RNG.standard_normal((T, H, dh))
    pos = np.array([0, 1, 7, 100, 4099])
    for n_rot in (8, 3, 0):
        got = om.rope_rotate(x, pos, 10000.0, n_rot)
        z = x[..., :8] + 1j * x[..., 8:]
        j = np.arange(8)
        freq = np.where(j < n_rot, 10000.0 ** (-j / 8.0), 0.0)   # theta^(-2j/dh), dh=16
        z = z * np.exp(1j * pos[:, None, None] * freq[None, None, :])
        assert np.allclose(got[..., :8], z.real, atol=1e-12)
        assert np.allclose(got[..., 8:], z.imag, atol=1e-12)
    assert np.allclose(om.rope_rotate(x, np.zeros(T), 10000.0, 8), x)


def test_rope_relative_position_property():
    dh = 32
    q, k = RNG.standard_normal((1, 1, dh)), RNG.standard_normal((1, 1, dh))
    def dot(m, n):
        a = om.rope_rotate(q, np.array([m]), 10000.0, dh // 2)
        b = om.rope_rotate(k, np.array([n]), 10000.0, dh // 2)
        return float(np.sum(a * b))
    assert abs(dot(10, 3) - dot(107, 100)) < 1e-10
    assert abs(dot(10, 3) - dot(3, 10)) > 1e-6       # depends on the sign of m - n


def test_rope_pairs_local_global():
    c = tiny_cfg(head_dim=256, global_every=6, n_layers=6)
    assert [om.rope_pairs_rotated(c, l) for l in range(6)] == [128] * 5 + [32]
    c2 = tiny_cfg(head_dim=256, global_every=6, rope_enabled=False)
    assert om.rope_pairs_rotated(c2, 0) == 0 and om.rope_pairs_rotated(c2, 5) == 0
    c3 = tiny_cfg(head_dim=64, global_every=6, prope_fraction=0.0)
    assert om.rope_pairs_rotated(c3, 5) == 0


# ----------------------------------------------------------------------------- attention

def _brute_attention(q, kc, vc, kp, vp, n_vis):
    """Scalar loops: per query row and head, walk the key list and accumulate."""
    Tc, Hq, dh = q.shape
    Hkv, P = kp.shape[0], kp.shape[1]
    out = np.zeros_like(q)
    for h in range(Hq):
        g = (h * Hkv) // Hq
        keys = [(kp[g, p], vp[g, p]) for p in range(P - n_vis, P)] + \
               [(kc[i, g], vc[i, g]) for i in range(Tc)]
        for t in range(Tc):
            s = [sum(q[t, h, a] * kk[a] for a in range(dh)) / math.sqrt(dh) for kk, _ in keys]
            mx = max(s)
            e = [math.exp(v - mx) for v in s]
            z = sum(e)
            for a in range(dh):
                out[t, h, a] = sum(e[j] * keys[j][1][a] for j in range(len(keys))) / z
    return out


def test_attention_brute_force():
    Tc, Hq, Hkv, dh, P = 3, 4, 2, 4, 5
    q = RNG.standard_normal((Tc, Hq, dh))
    kc, vc = RNG.standard_normal((Tc, Hkv, dh)), RNG.standard_normal((Tc, Hkv, dh))
    kp, vp = RNG.standard_normal((Hkv, P, dh)), RNG.standard_normal((Hkv, P, dh))
    for n_vis in (5, 2, 0):
        got = om.attention(q, kc, vc, kp, vp, n_vis)
        assert np.allclose(got, _brute_attention(q, kc, vc, kp, vp, n_vis), atol=1e-12)


def test_attention_zero_query_is_mean_of_visible_values():
    Tc, Hq, Hkv, dh, P, n_vis = 4, 2, 1, 8, 9, 3
    q = np.zeros((Tc, Hq, dh))
    kc, vc = RNG.standard_normal((Tc, Hkv, dh)), RNG.standard_normal((Tc, Hkv, dh))
    kp, vp = RNG.standard_normal((Hkv, P, dh)), RNG.standard_normal((Hkv, P, dh))
    got = om.attention(q, kc, vc, kp, vp, n_vis)
    mean = (vp[0, P - n_vis:].sum(0) + vc[:, 0].sum(0)) / (n_vis + Tc)
    assert np.allclose(got, mean[None, None, :], atol=1e-12)


def test_attention_split_kv_merge_is_exact():
    q = RNG.standard_normal((6, 16)) * 2
    keys, vals = RNG.standard_normal((50, 16)), RNG.standard_normal((50, 16))
    s = q @ keys.T / 4.0
    ref = scipy.special.softmax(s, axis=1) @ vals
    for chunks in ([(0, 50)], [(0, 7), (7, 50)], [(0, 1), (1, 20), (20, 21), (21, 50)]):
        assert np.allclose(om.attention_split_kv(q, keys, vals, chunks), ref, atol=1e-12)


def test_attention_window_and_gqa_mapping():
    Tc, Hq, Hkv, dh, P = 3, 4, 2, 8, 10
    q = RNG.standard_normal((Tc, Hq, dh))
    kc, vc = RNG.standard_normal((Tc, Hkv, dh)), RNG.standard_normal((Tc, Hkv, dh))
    kp, vp = RNG.standard_normal((Hkv, P, dh)), RNG.standard_normal((Hkv, P, dh))
    base = om.attention(q, kc, vc, kp, vp, 4)
    kp2 = kp.copy(); kp2[:, :P - 4] += 5.0           # outside the window: no effect
    assert np.allclose(om.attention(q, kc, vc, kp2, vp, 4), base, atol=1e-12)
    kp3 = kp.copy(); kp3[:, P - 1] += 5.0            # inside the window: changes it
    assert not np.allclose(om.attention(q, kc, vc, kp3, vp, 4), base)
    # heads 0,1 read kv head 0; heads 2,3 read kv head 1
    vp4 = vp.copy(); vp4[1] += 1.0; vc4 = vc.copy(); vc4[:, 1] += 1.0
    o4 = om.attention(q, kc, vc4, kp, vp4, 4)
    assert np.allclose(o4[:, :2], base[:, :2], atol=1e-12)
    assert np.allclose(o4[:, 2:], base[:, 2:] + 1.0, atol=1e-12)


def test_canvas_attention_permutation_equivariant_without_positions():
    cfg = tiny_cfg(rope_enabled=False, n_experts=2, top_k=1, n_shared=0)
    W = om.layer_weights(cfg, 0)
    h = RNG.standard_normal((1, cfg.canvas_len, cfg.d_model))
    kp = RNG.standard_normal((1, cfg.n_kv_heads, 6, cfg.head_dim))
    vp = RNG.standard_normal((1, cfg.n_kv_heads, 6, cfg.head_dim))
    perm = RNG.permutation(cfg.canvas_len)
    a, b = {}, {}
    om.layer_forward(cfg, W, h, kp, vp, trace=a)
    om.layer_forward(cfg, W, h[:, perm], kp, vp, trace=b)
    assert np.allclose(b["attn_o"], a["attn_o"][:, perm], atol=1e-12)
    assert np.allclose(b["out"], a["out"][:, perm], atol=1e-10)
    # with positions on, equivariance breaks
    cfg2 = tiny_cfg(rope_enabled=True, n_experts=2, top_k=1, n_shared=0)
    a2, b2 = {}, {}
    om.layer_forward(cfg2, om.layer_weights(cfg2, 0), h, kp, vp, trace=a2)
    om.layer_forward(cfg2, om.layer_weights(cfg2, 0), h[:, perm], kp, vp, trace=b2)
    assert not np.allclose(b2["attn_o"], a2["attn_o"][:, perm])


# ----------------------------------------------------------------------------- router / MoE

def test_router_topk_against_stable_sort_and_softmax():
    logits = RNG.standard_normal((40, 16)).astype(np.float32)
    logits[3, [2, 9, 11]] = 5.0                        # exact ties -> lower index first
    logits[4, :] = 0.0
    idx, w = om.router_topk(logits, 4)
    ref_idx = np.lexsort((np.tile(np.arange(16), (40, 1)), -logits), axis=1)[:, :4]
    assert np.array_equal(idx, ref_idx)
    assert list(idx[3][:3]) == [2, 9, 11] and list(idx[4]) == [0, 1, 2, 3]
    p = scipy.special.softmax(logits.astype(np.float64), axis=1)
    sel = np.take_along_axis(p, idx.astype(np.int64), axis=1)
    assert np.allclose(w, sel / sel.sum(1, keepdims=True), rtol=1e-12)
    idx_all, w_all = om.router_topk(logits, 16)
    assert np.allclose(np.take_along_axis(w_all, np.argsort(idx_all, 1), 1), p, rtol=1e-12)


def test_router_permutation_against_stable_argsort():
    idx = np.stack([RNG.choice(12, 3, replace=False) for _ in range(30)]).astype(np.int32)
    offsets, perm = om.router_permutation(idx, 12)
    assert np.array_equal(np.diff(offsets), np.bincount(idx.ravel(), minlength=12))
    assert np.array_equal(perm, np.argsort(idx.ravel(), kind="stable"))
    assert sorted(perm.tolist()) == list(range(90))


class _FixedWeights(om.LayerWeights):
    """LayerWeights with hand-set tensors (for identities)."""

    def __init__(self, cfg, layer, tensors, experts):
        super().__init__(cfg, layer)
        self._cache.update(tensors)
        self._experts = experts

    def expert(self, e):
        return self._experts[e]


def _rand_expert(d, F):
    return (RNG.standard_normal((F, d)) * 0.2, RNG.standard_normal((F, d)) * 0.2,
            RNG.standard_normal((d, F)) * 0.2)


def test_silu_against_expit():
    x = RNG.standard_normal(100) * 5
    assert np.allclose(om.silu(x), x * scipy.special.expit(x), rtol=1e-13)


def test_moe_single_expert_equals_dense_ffn():
    d, F = 12, 10
    cfg = tiny_cfg(d_model=d, d_ff=F, n_experts=1, top_k=1, n_shared=0)
    ex = _rand_expert(d, F)
    W = _FixedWeights(cfg, 0, {"wr": RNG.standard_normal((1, d))}, [ex])
    x = RNG.standard_normal((9, d))
    y, _, idx, w = om.moe_ffn(cfg, W, x)
    h = np.maximum(0, 0)  # noqa: F841
    gate = x @ ex[0].T
    dense = ((gate * scipy.special.expit(gate)) * (x @ ex[1].T)) @ ex[2].T
    assert np.all(idx == 0) and np.allclose(w, 1.0)
    assert np.allclose(y, dense, atol=1e-12)


def test_moe_all_experts_is_softmax_mixture_plus_shared():
    d, F, E = 10, 6, 5
    cfg = tiny_cfg(d_model=d, d_ff=F, n_experts=E, top_k=E, n_shared=1)
    exps = [_rand_expert(d, F) for _ in range(E)]
    sh = _rand_expert(d, F)
    wr = RNG.standard_normal((E, d))
    W = _FixedWeights(cfg, 0, {"wr": wr, "sg": sh[0], "su": sh[1], "sd": sh[2]}, exps)
    x = RNG.standard_normal((7, d))
    y, _, _, _ = om.moe_ffn(cfg, W, x)
    p = scipy.special.softmax(x @ wr.T, axis=1)
    ref = np.zeros_like(x)
    for t in range(7):
        for e in range(E):
            ref[t] += p[t, e] * om.expert_mlp(x[t:t + 1], *exps[e])[0]
        ref[t] += om.expert_mlp(x[t:t + 1], *sh)[0]
    assert np.allclose(y, ref, atol=1e-12)


def test_moe_zero_router_is_uniform_lowest_index():
    d, F, E, k = 8, 4, 6, 3
    cfg = tiny_cfg(d_model=d, d_ff=F, n_experts=E, top_k=k, n_shared=0)
    exps = [_rand_expert(d, F) for _ in range(E)]
    W = _FixedWeights(cfg, 0, {"wr": np.zeros((E, d))}, exps)
    x = RNG.standard_normal((4, d))
    y, _, idx, w = om.moe_ffn(cfg, W, x)
    assert np.array_equal(idx, np.tile([0, 1, 2], (4, 1)))
    assert np.allclose(w, 1.0 / 3)
    ref = sum(om.expert_mlp(x, *exps[e]) for e in range(3)) / 3
    assert np.allclose(y, ref, atol=1e-12)


def test_layer_residual_wiring():
    cfg = tiny_cfg()
    d = cfg.d_model
    W = om.layer_weights(cfg, 0)
    h = RNG.standard_normal((1, cfg.canvas_len, d))
    kp = RNG.standard_normal((1, cfg.n_kv_heads, 6, cfg.head_dim))
    vp = RNG.standard_normal((1, cfg.n_kv_heads, 6, cfg.head_dim))
    tr = {}
    out = om.layer_forward(cfg, W, h, kp, vp, trace=tr)
    # the two residual branches, recomputed from their own definitions
    attn = tr["attn"]
    assert np.allclose(tr["h1"], h + om.rmsnorm(attn, 1.0, cfg.rms_eps), atol=1e-12)
    assert np.allclose(out, tr["h1"] + tr["moe"], atol=1e-12)
    # zero output projection -> attention branch is exactly zero (rmsnorm(0) = 0)
    W0 = om.layer_weights(cfg, 0)
    W0._cache["wo"] = np.zeros_like(W.get("wo"))
    tr0 = {}
    om.layer_forward(cfg, W0, h, kp, vp, trace=tr0)
    assert np.array_equal(tr0["h1"], h)


# ----------------------------------------------------------------------------- head / commit

def test_logit_stats_against_softmax_with_mask_excluded():
    logits = RNG.standard_normal((6, 50)) * 4
    logits[0, 0] = 100.0                              # mask id 0 would win if not excluded
    logits[1, [5, 17]] = 50.0                         # tie -> lower index
    conf, a, m, s = om.logit_stats(logits, 0)
    p = scipy.special.softmax(logits[:, 1:], axis=1)
    assert np.array_equal(a, 1 + np.argmax(logits[:, 1:], axis=1))
    assert a[1] == 5 and a[0] != 0
    assert np.allclose(conf, p.max(axis=1), rtol=1e-12)
    assert np.allclose(np.log(s) + m, scipy.special.logsumexp(logits[:, 1:], axis=1), rtol=1e-12)


def test_head_reduce_matches_explicit_embedding_rows():
    cfg = tiny_cfg(vocab=40, d_model=16, mask_id=3)
    hn = RNG.standard_normal((5, 16))
    E = om.embedding_rows(cfg, np.arange(40))
    conf, a, _, _ = om.head_reduce(cfg, hn, vocab_block=7)
    lg = hn @ E.T
    lg[:, 3] = -np.inf
    assert np.array_equal(a, np.argmax(lg, 1))
    assert np.allclose(conf, scipy.special.softmax(lg, 1).max(1), rtol=1e-12)


def test_commit_schedule_golden():
    for line in open(os.path.join(GOLDEN, "commit_schedule.txt")):
        if line.startswith("#") or not line.strip():
            continue
        v = [int(t) for t in line.split()]
        n, S, ks = v[0], v[1], v[2:]
        canvas = np.zeros((1, n), np.int32)
        got = []
        for s in range(S):
            conf = RNG.uniform(size=(1, n))
            before = int((canvas == 0).sum())
            canvas, committed = om.commit(canvas, conf, np.full((1, n), 7), S - s, 0)
            got.append(int(committed.sum()))
            assert int((canvas == 0).sum()) == before - got[-1]
        assert got == ks
        assert int((canvas == 0).sum()) == 0


def test_commit_picks_highest_confidence_ties_lowest_index_and_never_reverts():
    canvas = np.array([[0, 5, 0, 0, 0, 0]], np.int32)     # row 1 already committed
    conf = np.array([[0.2, 0.99, 0.5, 0.5, 0.1, 0.5]])
    tok = np.array([[11, 12, 13, 14, 15, 16]])
    new, com = om.commit(canvas, conf, tok, 2, 0)          # r=5, k=3
    assert com.tolist() == [[False, False, True, True, False, True]]
    assert new.tolist() == [[0, 5, 13, 14, 0, 16]]
    new2, com2 = om.commit(new, np.zeros((1, 6)), tok + 100, 1, 0)   # all remaining
    assert new2.tolist() == [[111, 5, 13, 14, 115, 16]]


# ----------------------------------------------------------------------------- whole step

def _tiny_prompt(cfg, P, seed=5):
    g = np.random.default_rng(seed)
    shape = (1, cfg.n_kv_heads, P, cfg.head_dim)
    return ([g.standard_normal(shape) for _ in range(cfg.n_layers)],
            [g.standard_normal(shape) for _ in range(cfg.n_layers)])


def test_denoise_block_invariants_and_resume():
    cfg = tiny_cfg(n_layers=2, canvas_len=8, vocab=61)
    kp, vp = _tiny_prompt(cfg, 6)
    weights = [om.layer_weights(cfg, l) for l in range(cfg.n_layers)]
    canvas0 = np.zeros((1, 8), np.int32)
    hist = []
    final = om.denoise_block(cfg, canvas0, kp, vp, 3, weights=weights, history=hist)
    masked = [8] + [int((hh["canvas"] == 0).sum()) for hh in hist]
    assert masked == [8, 5, 2, 0]                          # k = 3, 3, 2
    prev = canvas0
    for hh in hist:
        keep = prev != 0
        assert np.array_equal(hh["canvas"][keep], prev[keep])          # never revert
        assert np.all(hh["canvas"][hh["committed"]] == hh["tok"][hh["committed"]])
        assert np.all(hh["tok"] != 0)                                   # mask id never predicted
        prev = hh["canvas"]
    # resume: one step, then the remaining two from the saved canvas
    c1, _, _, _ = om.canvas_step(cfg, canvas0, kp, vp, 3, weights=weights)
    c3 = om.denoise_block(cfg, c1, kp, vp, 2, weights=weights)
    assert np.array_equal(c3, final)


def test_c_generator_matches_numpy_generator():
    for tid, shape, start, bf16 in [(1, (37, 64), 0, True), (77, (5, 1000), 12345, False),
                                    (64 * 3 + 5, (3, 2816), 7 * 704 * 2816, True)]:
        a = orng.weight_tensor_numpy(0, tid, shape, 0.02, bf16, start=start)
        b = orng.weight_tensor(0, tid, shape, 0.02, bf16, start=start)
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


# ----------------------------------------------------------------------------- layer assembly

def _wiring_cfg(**kw):
    """d = dh = 4, one query and one key/value head, layer 0 local (window 1),
    layer 1 global (p-RoPE with p = 0.25 rotates pair 0 only)."""
    base = dict(n_layers=2, d_model=4, n_q_heads=1, n_kv_heads=1, head_dim=4, n_experts=2,
                top_k=1, n_shared=0, d_ff=4, vocab=8, canvas_len=2, window=1, global_every=2,
                rope_theta=10000.0, prope_fraction=0.25)
    base.update(kw)
    return om.OracleConfig(**base)


def _wiring_weights(cfg, layer):
    """Hand-set projections on h = e0 (input norm gives x = 2 e0): q = e0, canvas keys
    0, canvas values e0, every other weight zero (the block adds nothing to h)."""
    z = np.zeros((4, 4))
    wq = z.copy(); wq[0, 0] = 0.5
    wv = z.copy(); wv[0, 0] = 0.5
    zero_expert = (np.zeros((4, 4)), np.zeros((4, 4)), np.zeros((4, 4)))
    return _FixedWeights(cfg, layer, {"wq": wq, "wk": z.copy(), "wv": wv, "wo": z.copy(),
                                      "wr": np.zeros((2, 4))}, [zero_expert] * 2)


def _wiring_prompt(a=(1.0, -2.0, 4.0)):
    """Three prompt keys a_j e0 and values (j + 1) e1, [B=1, Hkv=1, P=3, dh=4]."""
    kp = np.zeros((1, 1, 3, 4))
    vp = np.zeros((1, 1, 3, 4))
    for j, aj in enumerate(a):
        kp[0, 0, j, 0] = aj
        vp[0, 0, j, 1] = j + 1
    return kp, vp


def _hand_attention(pos, a_visible, v_index):
    """o at one canvas query, worked by hand: the rotated query at position `pos` is
    (cos pos, 0, sin pos, 0) (pair 0 turns at frequency theta^0 = 1), so prompt key
    a_j e0 scores a_j cos(pos) / sqrt(4); both canvas keys are 0 (score 0) and carry
    the value e0; prompt value j is (j + 1) e1."""
    e_p = [math.exp(aj * math.cos(pos) / 2.0) for aj in a_visible]
    z = sum(e_p) + 2.0
    return np.array([2.0 / z, sum(e * (j + 1) for e, j in zip(e_p, v_index)) / z, 0.0, 0.0])


def test_layer_canvas_positions_window_and_unrotated_values():
    """Canvas slot i attends from position P + i; a local layer sees only the last
    min(window, P) prompt keys and a global one all P; V is never rotated
    ("Hands-On with Diffusion Gemma", Detailed Specs: sliding-window local layers,
    global layers, RoPE / p-RoPE; the readings R2 and R4)."""
    cfg = _wiring_cfg()
    a = (1.0, -2.0, 4.0)
    kp, vp = _wiring_prompt(a)
    h = np.zeros((1, 2, 4))
    h[..., 0] = 1.0
    P = 3
    for layer, vis in ((0, [2]), (1, [0, 1, 2])):      # window 1 on the local layer
        tr = {}
        out = om.layer_forward(cfg, _wiring_weights(cfg, layer), h, kp, vp, trace=tr)
        assert np.array_equal(out, h)                   # zero o-projection and experts
        for i in range(2):
            want = _hand_attention(P + i, [a[j] for j in vis], vis)
            assert np.allclose(tr["attn_o"][0, i, 0], want, atol=1e-12), (layer, i)
    # keys outside the window do not matter on the local layer, and do on the global one
    kp2 = kp.copy()
    kp2[0, 0, :2, 0] = (7.0, 3.0)
    for layer, same in ((0, True), (1, False)):
        t1, t2 = {}, {}
        om.layer_forward(cfg, _wiring_weights(cfg, layer), h, kp, vp, trace=t1)
        om.layer_forward(cfg, _wiring_weights(cfg, layer), h, kp2, vp, trace=t2)
        assert np.array_equal(t1["attn_o"], t2["attn_o"]) == same, layer


def test_layer_window_longer_than_prompt_sees_every_key():
    """A window of 1024 over a 3-key prompt: the local layer sees all 3 (min(window, P))."""
    cfg = _wiring_cfg(window=1024)
    a = (1.0, -2.0, 4.0)
    kp, vp = _wiring_prompt(a)
    h = np.zeros((1, 2, 4))
    h[..., 0] = 1.0
    tr = {}
    om.layer_forward(cfg, _wiring_weights(cfg, 0), h, kp, vp, trace=tr)
    for i in range(2):
        assert np.allclose(tr["attn_o"][0, i, 0], _hand_attention(3 + i, a, [0, 1, 2]),
                           atol=1e-12)


def test_canvas_step_final_norm_and_embedding_row(monkeypatch):
    """A pass through identity blocks: the head scores the final-normed embedding row
    of the mask id against the tied embedding, mask id excluded ("Hands-On with
    Diffusion Gemma", Detailed Specs: tied embed_tokens / lm_head and the final norm).
    Embedding (vocab 4, d 2, mask id 0): rows (1, 1), (2, 0), (0, 1.5), (-1, 2).
    The canvas is all mask, so h = (1, 1); rms = 1, so the final norm leaves
    (1, 1) / sqrt(1 + eps).  Logits of tokens 1..3: 2, 1.5, 1 (over sqrt(1 + eps)):
    argmax 1 and confidence 1 / (1 + e^-0.5 + e^-1)."""
    emb = np.array([[1.0, 1.0], [2.0, 0.0], [0.0, 1.5], [-1.0, 2.0]])
    monkeypatch.setattr(om, "embedding_rows", lambda cfg, rows: emb[np.asarray(rows).ravel()])
    monkeypatch.setattr(om, "embedding_block", lambda cfg, v0, v1: emb[v0:v1])
    cfg = om.OracleConfig(n_layers=1, d_model=2, n_q_heads=1, n_kv_heads=1, head_dim=2,
                          n_experts=1, top_k=1, n_shared=0, d_ff=2, vocab=4, canvas_len=3,
                          window=4, global_every=1, rms_eps=1e-6)
    z = np.zeros((2, 2))
    W = _FixedWeights(cfg, 0, {"wq": z, "wk": z, "wv": z, "wo": z, "wr": np.zeros((1, 2))},
                      [(z, z, z)])
    kp = np.zeros((1, 1, 2, 2))
    canvas = np.zeros((1, 3), np.int32)
    new, conf, tok, com = om.canvas_step(cfg, canvas, [kp], [kp], 3, weights=[W])
    s = 1.0 / math.sqrt(1.0 + 1e-6)
    want = 1.0 / (1.0 + math.exp(-0.5 * s) + math.exp(-1.0 * s))
    assert np.all(tok == 1)
    assert np.allclose(conf, want, rtol=1e-12)
    # one slot of three commits (k = ceil(3 / 3)); equal confidences -> slot 0
    assert new.tolist() == [[1, 0, 0]] and com.tolist() == [[True, False, False]]


# ----------------------------------------------------------------------------- FP8 expert weights

def _e4m3_table():
    """Every finite E4M3 value, decoded from the format: sign, exponent field e
    (bias 7), mantissa m; e = 0 gives m * 2^-9, otherwise (1 + m/8) * 2^(e-7);
    S.1111.111 is NaN.  Returns (values, mantissa parity) of the 254 finite codes."""
    vals, even = [], []
    for code in range(256):
        sgn, e, m = code >> 7, (code >> 3) & 15, code & 7
        if e == 15 and m == 7:
            continue
        v = m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
        vals.append(-v if sgn else v)
        even.append(m % 2 == 0)
    return np.array(vals), np.array(even)


def test_e4m3_rounding_is_the_nearest_code_ties_to_even():
    from oracle import quant
    table, even = _e4m3_table()
    assert table.max() == 448.0 and table[table > 0].min() == 2.0 ** -9
    x = np.concatenate([RNG.standard_normal(4000) * np.exp(RNG.uniform(-9, 6, 4000)),
                        (table[np.abs(table) < 448][:-1] + table[np.abs(table) < 448][1:]) / 2])
    x = np.clip(x, -448, 448).astype(np.float32)
    got = quant.e4m3_round(x)
    for xi, gi in zip(x.astype(np.float64), got.astype(np.float64)):
        d = np.abs(table - xi)
        best = np.nonzero(d == d.min())[0]
        if len(best) > 1:                      # a tie: the code with the even mantissa
            best = [b for b in best if even[b]]
        assert gi == table[best[0]], (xi, gi, table[best])


def test_rowwise_fp8_scale_and_error_bound():
    from oracle import quant
    w = (RNG.standard_normal((6, 300)) * 0.02).astype(np.float32)
    w[2, 7] = -0.2                              # a large entry sets its row's scale
    w[3] = 0.0                                  # a zero row
    q, s = quant.e4m3_rowwise(w)
    amax = np.abs(w).max(axis=1)
    assert np.array_equal(s, (amax.astype(np.float32) / np.float32(448)).astype(np.float32))
    assert np.all(np.abs(q) <= 448) and np.all(q[3] == 0) and s[3] == 0
    assert q[2, 7] == -448.0                    # the row maximum maps to the largest code
    deq = quant.dequantized(w)
    # half an E4M3 ulp: relative 2^-4 for normal codes, absolute s * 2^-10 below 2^-6
    err = np.abs(deq - w.astype(np.float64))
    bound = np.maximum(np.abs(w) * 2.0 ** -4, s[:, None].astype(np.float64) * 2.0 ** -10)
    assert np.all(err <= bound * (1 + 1e-6))


def test_fp8_experts_are_the_dequantised_drawn_weights():
    from oracle import quant
    c16 = tiny_cfg(n_experts=4, d_model=64, d_ff=32)
    c8 = tiny_cfg(n_experts=4, d_model=64, d_ff=32, expert_fp8=True)
    W16, W8 = om.layer_weights(c16, 0), om.layer_weights(c8, 0)
    for a, b in zip(W16.expert(2), W8.expert(2)):
        assert np.array_equal(b, quant.dequantized(a.astype(np.float32)))
        assert 0 < np.abs(a - b).max() <= np.abs(a).max() * 2.0 ** -4
    for a, b in zip(W16.shared(), W8.shared()):
        assert np.array_equal(b, quant.dequantized(a.astype(np.float32)))
    assert np.array_equal(W16.get("wq"), W8.get("wq"))     # only the experts change
