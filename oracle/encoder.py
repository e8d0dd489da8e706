"""The causal encoder (prompt prefill, context building) and the block-autoregressive
outer loop, restated plainly in numpy float64 (test infrastructure only).

Page citations (title, then section):

[HO]  "Hands-On with Diffusion Gemma: Another Gemma with a Diffusion Mechanism",
      sections "How Is This Different from Previous Models?" and "Detailed Specs".
[EF]  "DiffusionGemma: The Diffusion Era Begins with 4x Faster Text Generation",
      section "DiffusionGemma's Technical Architecture".

What the pages fix: the causal part of the model serves as an encoder that
ingests the input once and fills the KV cache the decoder reads [HO How
Different; HO Detailed Specs: Encoder and Decoder; EF Technical
Architecture: the autoregressive encoder creates the prompt's KV cache, the
decoder reaches it by cross-attention]; the encoder has the structure of the
causal base model, with unidirectional attention [HO Detailed Specs]; the
encoder and decoder share their weights, embedding and norms included [HO
Detailed Specs: weight sharing]; after a 256-token canvas is finished the
model returns to causal context building for the next canvas [HO How
Different].

Readings taken where the pages are silent (kept with the design notes):
 G1 the encoder runs the decoder's blocks with the same weights (R4-R10
     unchanged), except that attention is causal: the token at position p
     attends to the positions <= p, on a local layer only to the last `window`
     of them (p - window + 1 .. p), on a global layer to all; RoPE uses the
     absolute positions 0, 1, ...; the KV cache of a layer holds the rotated k
     and the v of every token encoded so far, in position order;
 G2 a finished canvas (every slot committed) is encoded at the positions
     P .. P + Tc - 1 that its slots had in the decoder (R4) and appended to the
     cache; the next canvas starts all-mask with P grown by Tc;
 G3 only the encoder's KV cache is used: its output hidden states pass through
     no final norm and no head.
"""

from __future__ import annotations

import math
from typing import Optional

import numpy as np

from .model import (OracleConfig, denoise_block, embedding_rows, is_global_layer, layer_weights,
                    moe_ffn, rmsnorm, rope_pairs_rotated, rope_rotate)


def causal_attention(q, k_new, v_new, k_cache, v_cache, window: Optional[int]) -> np.ndarray:
    """G1: causal softmax attention of n new tokens over the cached keys and themselves.

    q [n, Hq, dh]; k_new, v_new [n, Hkv, dh] (the new tokens' rotated keys and
    values); k_cache, v_cache [Hkv, P0, dh] (the positions before them).  New
    token i sits at position P0 + i and sees the positions lo(i) .. P0 + i, with
    lo(i) = max(0, P0 + i - window + 1) on a local layer (window set) and 0 on a
    global one (window None).  Grouped-query heads as in the decoder.
    Returns o [n, Hq, dh].
    """
    n, Hq, dh = q.shape
    Hkv, P0 = k_cache.shape[0], k_cache.shape[1]
    group = Hq // Hkv
    out = np.empty((n, Hq, dh))
    for h in range(Hq):
        g = h // group
        for i in range(n):
            p = P0 + i
            lo = 0 if window is None else max(0, p - window + 1)
            keys, vals = [], []
            for pos in range(lo, p + 1):          # the visible positions, in order
                if pos < P0:
                    keys.append(k_cache[g, pos])
                    vals.append(v_cache[g, pos])
                else:
                    keys.append(k_new[pos - P0, g])
                    vals.append(v_new[pos - P0, g])
            K, V = np.stack(keys), np.stack(vals)
            s = K @ q[i, h] / math.sqrt(dh)
            e = np.exp(s - s.max())
            out[i, h] = (e / e.sum()) @ V
    return out


def encoder_layer_forward(cfg: OracleConfig, W, h: np.ndarray, k_cache, v_cache,
                          router_bias=None, trace: Optional[dict] = None):
    """One encoder block (G1) on n new tokens per sequence.

    h [B, n, d]; k_cache, v_cache [B, Hkv, P0, dh] (rotated keys).  The block is
    the decoder's (R7: input norm, q/k/v, attention, post-attention norm and
    residual, pre-FFN norm, MoE, residual) with causal attention.  Returns
    (h_out [B, n, d], k_new [B, Hkv, n, dh] rotated, v_new [B, Hkv, n, dh]).
    """
    c = cfg
    B, n, d = h.shape
    P0 = k_cache.shape[2]
    layer = W.layer
    dh, Hq, Hkv = c.head_dim, c.n_q_heads, c.n_kv_heads
    n_rot = rope_pairs_rotated(c, layer)
    window = None if is_global_layer(c, layer) else c.window
    pos = P0 + np.arange(n)
    h = np.asarray(h, dtype=np.float64)

    x = rmsnorm(h, W.norm("input"), c.rms_eps)
    q = (x @ W.get("wq").T).reshape(B, n, Hq, dh)
    k = (x @ W.get("wk").T).reshape(B, n, Hkv, dh)
    v = (x @ W.get("wv").T).reshape(B, n, Hkv, dh)
    o = np.empty((B, n, Hq, dh))
    k_rot = np.empty((B, n, Hkv, dh))
    for b in range(B):
        qb = rope_rotate(q[b], pos, c.rope_theta, n_rot)
        k_rot[b] = rope_rotate(k[b], pos, c.rope_theta, n_rot)
        o[b] = causal_attention(qb, k_rot[b], v[b], np.asarray(k_cache[b], np.float64),
                                np.asarray(v_cache[b], np.float64), window)
    attn = o.reshape(B, n, Hq * dh) @ W.get("wo").T
    h1 = h + rmsnorm(attn, W.norm("post_attn"), c.rms_eps)
    x2 = rmsnorm(h1, W.norm("pre_ff"), c.rms_eps)
    y, _, _, _ = moe_ffn(c, W, x2.reshape(B * n, d), router_bias)
    h2 = h1 + y.reshape(B, n, d)
    if trace is not None:
        trace.update(q=q, k=k_rot, v=v, attn_o=o, h1=h1, x2=x2, out=h2)
    return h2, k_rot.transpose(0, 2, 1, 3), v.transpose(0, 2, 1, 3)


def empty_cache(cfg: OracleConfig, batch: int):
    """Per-layer key and value caches holding no position yet: [B, Hkv, 0, dh] each."""
    z = np.zeros((batch, cfg.n_kv_heads, 0, cfg.head_dim))
    return [z.copy() for _ in range(cfg.n_layers)], [z.copy() for _ in range(cfg.n_layers)]


def encode(cfg: OracleConfig, tokens: np.ndarray, k_caches, v_caches, router_bias=None,
           weights=None):
    """Encode n new tokens per sequence after the cached ones and append their keys and
    values to every layer's cache (G1-G3).

    tokens int [B, n]; k_caches[l], v_caches[l] [B, Hkv, P0, dh].  The tokens are
    embedded with the shared embedding [HO Detailed Specs: weight sharing] and run
    through every block; layer l's cache grows by that layer's k and v.
    Returns the new (k_caches, v_caches), [B, Hkv, P0 + n, dh] each.
    """
    c = cfg
    tokens = np.asarray(tokens)
    B, n = tokens.shape
    h = embedding_rows(c, tokens.reshape(-1)).reshape(B, n, c.d_model)
    k_out, v_out = [], []
    for layer in range(c.n_layers):
        W = weights[layer] if weights is not None else layer_weights(c, layer)
        h, kn, vn = encoder_layer_forward(c, W, h, k_caches[layer], v_caches[layer], router_bias)
        k_out.append(np.concatenate([np.asarray(k_caches[layer], np.float64), kn], axis=2))
        v_out.append(np.concatenate([np.asarray(v_caches[layer], np.float64), vn], axis=2))
    return k_out, v_out


def generate(cfg: OracleConfig, prompt: np.ndarray, n_blocks: int, n_steps: int,
             router_bias=None, weights=None, block_tokens=None, history: Optional[list] = None):
    """Block-autoregressive generation (G2): encode the prompt, then per block denoise
    an all-mask canvas for n_steps fixed passes against the cache and encode the
    finished block onto it [HO How Different; G4 How Text Diffusion Actually Works].

    prompt int [B, P].  ``block_tokens`` (optional, [B, n_blocks * Tc]) replaces each
    finished block by the given tokens before it is encoded, so that a test can feed
    another implementation's blocks and compare the next one.  Returns (tokens
    [B, n_blocks * Tc], k_caches, v_caches).
    """
    c = cfg
    prompt = np.asarray(prompt)
    B = prompt.shape[0]
    kc, vc = empty_cache(c, B)
    kc, vc = encode(c, prompt, kc, vc, router_bias, weights)
    out = []
    for blk in range(n_blocks):
        canvas = np.full((B, c.canvas_len), c.mask_id, dtype=np.int32)
        canvas = denoise_block(c, canvas, kc, vc, n_steps, router_bias, weights)
        out.append(canvas)
        if history is not None:
            history.append(dict(block=canvas.copy(), P=kc[0].shape[2]))
        fed = canvas if block_tokens is None else \
            np.asarray(block_tokens)[:, blk * c.canvas_len:(blk + 1) * c.canvas_len]
        kc, vc = encode(c, fed, kc, vc, router_bias, weights)
    return np.concatenate(out, axis=1), kc, vc
