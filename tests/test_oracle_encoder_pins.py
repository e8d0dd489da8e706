"""Pins of the causal encoder and the block-autoregressive loop (oracle/encoder.py).

Each pin ties the encoder to something outside it: the decoder's attention on
prefixes (pinned in test_oracle_pins.py against brute force), closed forms,
causality itself (encoding in chunks equals encoding at once), the window edge,
and the decoder's own block on a one-slot canvas, where causal and bidirectional
attention coincide.
"""

import numpy as np
import pytest

from oracle import encoder as oe
from oracle import model as om

RNG = np.random.default_rng(4321)


def small_cfg(**kw):
    base = dict(n_layers=2, d_model=64, n_q_heads=4, n_kv_heads=2, head_dim=16, n_experts=4,
                top_k=2, n_shared=1, d_ff=32, vocab=97, canvas_len=4, window=5, global_every=2,
                bf16_weights=True)
    base.update(kw)
    return om.OracleConfig(**base)


def _qkv(n, P0, Hq=4, Hkv=2, dh=8):
    q = RNG.standard_normal((n, Hq, dh))
    kn = RNG.standard_normal((n, Hkv, dh))
    vn = RNG.standard_normal((n, Hkv, dh))
    kc = RNG.standard_normal((Hkv, P0, dh))
    vc = RNG.standard_normal((Hkv, P0, dh))
    return q, kn, vn, kc, vc


@pytest.mark.parametrize("window", [None, 4, 2])
def test_causal_attention_is_the_decoder_attention_on_each_prefix(window):
    """Row i equals the decoder's joint attention of a one-query canvas whose prompt
    part is the visible cached positions and whose canvas part is the visible new
    tokens (the decoder's attention is pinned against brute force elsewhere)."""
    n, P0 = 6, 3
    q, kn, vn, kc, vc = _qkv(n, P0)
    got = oe.causal_attention(q, kn, vn, kc, vc, window)
    for i in range(n):
        p = P0 + i
        lo = 0 if window is None else max(0, p - window + 1)
        n_vis = max(0, P0 - lo)
        j0 = max(0, lo - P0)
        ref = om.attention(q[i:i + 1], kn[j0:i + 1], vn[j0:i + 1], kc, vc, n_vis)
        np.testing.assert_allclose(got[i], ref[0], rtol=1e-12, atol=1e-12)


def test_first_token_with_an_empty_cache_attends_only_to_itself():
    """Closed form: one visible key, so the output is that token's value exactly."""
    q, kn, vn, kc, vc = _qkv(3, 0)
    got = oe.causal_attention(q, kn, vn, kc, vc, None)
    for h in range(4):
        np.testing.assert_array_equal(got[0, h], vn[0, h // 2])


def test_window_edge():
    """On a local layer, a cached key just outside row i's window does not change row i,
    and the oldest key inside it does."""
    n, P0, W = 3, 6, 4
    q, kn, vn, kc, vc = _qkv(n, P0)
    base = oe.causal_attention(q, kn, vn, kc, vc, W)
    i = 1                               # position P0 + 1 sees P0 + 1 - W + 1 = 4 .. 7
    outside, inside = P0 + i - W, P0 + i - W + 1
    for pos, changes in ((outside, False), (inside, True)):
        k2 = kc.copy()
        k2[:, pos] += 3.0
        got = oe.causal_attention(q, kn, vn, k2, vc, W)
        assert (not np.allclose(got[i], base[i])) == changes, pos
    # a later new token does not reach an earlier row (causality)
    k3 = kn.copy()
    k3[2] += 3.0
    got = oe.causal_attention(q, k3, vn, kc, vc, W)
    np.testing.assert_array_equal(got[:2], base[:2])


def test_encoding_in_chunks_equals_encoding_at_once():
    """Causality: the cache after encoding 7 tokens at once equals the cache after
    encoding 3 and then 4 (positions, window and appending all line up)."""
    cfg = small_cfg()
    toks = RNG.integers(1, cfg.vocab, size=(2, 7))
    k0, v0 = oe.empty_cache(cfg, 2)
    ka, va = oe.encode(cfg, toks, k0, v0)
    kb, vb = oe.encode(cfg, toks[:, :3], k0, v0)
    kb, vb = oe.encode(cfg, toks[:, 3:], kb, vb)
    for l in range(cfg.n_layers):
        assert ka[l].shape == (2, cfg.n_kv_heads, 7, cfg.head_dim)
        np.testing.assert_allclose(kb[l], ka[l], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(vb[l], va[l], rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("layer", [0, 1])
def test_one_new_token_matches_the_decoder_block_on_a_one_slot_canvas(layer):
    """With one new token, causal and bidirectional attention see the same keys (all
    cached positions, fewer than the window, plus itself), and the decoder's canvas
    row 0 sits at position P, the encoder's new token too: the two blocks agree."""
    cfg = small_cfg(window=8)
    W = om.layer_weights(cfg, layer)
    B, P0 = 2, 5
    kc = RNG.standard_normal((B, cfg.n_kv_heads, P0, cfg.head_dim))
    vc = RNG.standard_normal((B, cfg.n_kv_heads, P0, cfg.head_dim))
    h = RNG.standard_normal((B, 1, cfg.d_model))
    h_enc, k_new, v_new = oe.encoder_layer_forward(cfg, W, h, kc, vc)
    trace = {}
    h_dec = om.layer_forward(cfg, W, h, kc, vc, trace=trace)
    np.testing.assert_allclose(h_enc, h_dec, rtol=1e-10, atol=1e-12)
    # the appended key is the decoder's rotated canvas key, the value its value
    n_rot = om.rope_pairs_rotated(cfg, layer)
    for b in range(B):
        k_rot = om.rope_rotate(trace["k"][b], np.array([P0]), cfg.rope_theta, n_rot)
        np.testing.assert_allclose(k_new[b, :, 0], k_rot[0], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(v_new[b, :, 0], trace["v"][b, 0], rtol=1e-12, atol=1e-12)


def test_generate_appends_each_finished_block_and_matches_one_shot_encoding():
    """Two blocks: every slot of each block is committed, the cache grows by the canvas
    length per block, and the final cache equals encoding prompt + both blocks at once."""
    cfg = small_cfg()
    prompt = RNG.integers(1, cfg.vocab, size=(2, 5))
    hist = []
    toks, kc, vc = oe.generate(cfg, prompt, n_blocks=2, n_steps=2, history=hist)
    assert toks.shape == (2, 2 * cfg.canvas_len)
    assert not np.any(toks == cfg.mask_id)
    assert [h["P"] for h in hist] == [5, 5 + cfg.canvas_len]
    k0, v0 = oe.empty_cache(cfg, 2)
    ka, va = oe.encode(cfg, np.concatenate([prompt, toks], axis=1), k0, v0)
    for l in range(cfg.n_layers):
        assert kc[l].shape[2] == 5 + 2 * cfg.canvas_len
        np.testing.assert_allclose(kc[l], ka[l], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(vc[l], va[l], rtol=1e-10, atol=1e-12)


def test_generate_with_fed_blocks_encodes_the_fed_tokens():
    """block_tokens replaces each finished block before it is encoded (the hook a test
    uses to compare one block of another implementation at a time)."""
    cfg = small_cfg()
    prompt = RNG.integers(1, cfg.vocab, size=(1, 3))
    fed = RNG.integers(1, cfg.vocab, size=(1, 2 * cfg.canvas_len))
    _, kc, _ = oe.generate(cfg, prompt, n_blocks=2, n_steps=1, block_tokens=fed)
    k0, v0 = oe.empty_cache(cfg, 1)
    ka, _ = oe.encode(cfg, np.concatenate([prompt, fed], axis=1), k0, v0)
    for l in range(cfg.n_layers):
        np.testing.assert_allclose(kc[l], ka[l], rtol=1e-10, atol=1e-12)
