"""The canvas denoising step, restated plainly in numpy float64 (test infrastructure only).

Page citations (title, then section):

[HO]  "Hands-On with Diffusion Gemma: Another Gemma with a Diffusion Mechanism",
      sections "How Is This Different from Previous Models?" and "Detailed Specs".
[EF]  "DiffusionGemma: The Diffusion Era Begins with 4x Faster Text Generation",
      sections "What is Diffusion and Why is it Coming to Text Generation Now?",
      "DiffusionGemma's Technical Architecture", "Recommended Inference Settings".
[G4]  "DiffusionGemma: Google's Experimental Diffusion LLM",
      section "How Text Diffusion Actually Works".

What the pages fix: a 256-slot canvas that starts all-mask [HO How Different;
EF What is Diffusion; G4]; bidirectional attention inside the block plus
cross-attention into the prompt's cached KV [EF Technical Architecture];
30 blocks as (5 local sliding-window + 1 global) x 5, window 1024, GQA on the
global layers, RoPE on local layers and p-RoPE on global ones [HO Detailed
Specs; EF Technical Architecture]; a 128-expert MoE with 8 active + 1 shared
expert and a router [EF Technical Architecture; HO Detailed Specs]; the
tied embedding / lm_head [HO Detailed Specs]; confident tokens locked in over
several passes [HO How Different; EF What is Diffusion; G4].

Readings taken where the pages are silent (each one is a parameter or a
documented choice; the full list is kept with the design notes):
 R1  one joint softmax per layer over {visible prompt keys} U {all canvas keys},
     using the layer's single q/k/v/o projections;
 R2  a local layer sees the last min(window, P) prompt keys, a global layer all P;
 R3  layer l (0-based) is global iff (l + 1) % global_every == 0;
 R4  canvas row i sits at position P + i; prompt keys arrive already rotated;
     RoPE pairs (x_j, x_{j+dh/2}) with frequency theta^(-2j/dh); local layers
     rotate every pair, global layers only the first ceil(p * dh / 2) pairs
     (the highest frequencies);
 R5  attention scale 1/sqrt(dh), no soft-cap, no QK-norm;
 R6  RMSNorm x * w / sqrt(mean(x^2) + eps) with w = 1;
 R7  h += post_attn_norm(Attn(input_norm(h))); h += MoE(pre_ff_norm(h));
 R8  router: top-k by logit (equivalently by softmax probability), equal
     logits broken toward the lower expert index, weights = softmax over the
     chosen logits (the renormalised probabilities); per_expert_scale = 1;
 R9  one shared expert of width F, weight 1, on every row;
 R10 activation silu(gate) * up;
 R11 the mask-id logit is excluded from max, argmax and the softmax sum;
 R12 confidence = the largest softmax probability = 1 / sum_v exp(l_v - max);
 R13 each step commits k = ceil(r / steps_left) of the r still-masked rows,
     highest confidence first, equal confidences toward the lower row;
 R14 no timestep embedding; steps_left only sets k.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

from .rng import EMBED_TID, layer_tid, weight_tensor


@dataclass
class OracleConfig:
    n_layers: int
    d_model: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    n_experts: int
    top_k: int
    n_shared: int
    d_ff: int
    vocab: int
    canvas_len: int
    window: int = 1024
    global_every: int = 6
    mask_id: int = 0
    rms_eps: float = 1e-6
    rope_theta: float = 10000.0
    prope_fraction: float = 0.25
    rope_enabled: bool = True
    weight_std: float = 0.02
    bf16_weights: bool = True
    expert_fp8: bool = False     # FP8 E4M3 expert weights, one scale per row (oracle.quant)
    seed: int = 0

    @staticmethod
    def from_dict(d: dict) -> "OracleConfig":
        names = OracleConfig.__dataclass_fields__.keys()
        return OracleConfig(**{k: v for k, v in d.items() if k in names})


def is_global_layer(cfg: OracleConfig, layer: int) -> bool:
    """R3: (5 local + 1 global) x 5 [HO Detailed Specs] -> every 6th layer is global."""
    return (layer + 1) % cfg.global_every == 0


# ----------------------------------------------------------------------------- weights

class LayerWeights:
    """Weights of one decoder layer, drawn from the seed on first use (float64).

    Projection weights are stored (out_features, in_features): y = x @ W.T.
    Expert tensors are drawn one expert at a time so that host memory holds
    one layer's dense weights plus a single expert.
    """

    def __init__(self, cfg: OracleConfig, layer: int):
        self.cfg, self.layer = cfg, layer
        self._cache = {}

    def _draw(self, kind, shape, start=0):
        c = self.cfg
        w = weight_tensor(c.seed, layer_tid(self.layer, kind), shape, c.weight_std,
                          c.bf16_weights, start=start)
        return w.astype(np.float64)

    def get(self, kind):
        if kind not in self._cache:
            c = self.cfg
            dq, dkv = c.n_q_heads * c.head_dim, c.n_kv_heads * c.head_dim
            shape = {"wq": (dq, c.d_model), "wk": (dkv, c.d_model), "wv": (dkv, c.d_model),
                     "wo": (c.d_model, dq), "wr": (c.n_experts, c.d_model),
                     "sg": (c.d_ff, c.d_model), "su": (c.d_ff, c.d_model),
                     "sd": (c.d_model, c.d_ff)}[kind]
            self._cache[kind] = self._draw(kind, shape)
        return self._cache[kind]

    def expert(self, e: int):
        """(gate [F,d], up [F,d], down [d,F]) of routed expert e."""
        c = self.cfg
        n = c.d_ff * c.d_model
        return self._lowp((self._draw("wg", (c.d_ff, c.d_model), start=e * n),
                           self._draw("wu", (c.d_ff, c.d_model), start=e * n),
                           self._draw("wd", (c.d_model, c.d_ff), start=e * n)))

    def shared(self):
        return self._lowp((self.get("sg"), self.get("su"), self.get("sd")))

    def _lowp(self, mats):
        """The expert weights the layer computes with: as drawn, or (expert_fp8)
        quantised to FP8 E4M3 with a scale per output row and dequantised."""
        if not self.cfg.expert_fp8:
            return mats
        from .quant import dequantized
        return tuple(dequantized(m.astype(np.float32)) for m in mats)

    # Norm scales are ones under R6.
    def norm(self, _name):
        return np.ones(self.cfg.d_model)


def layer_weights(cfg: OracleConfig, layer: int) -> LayerWeights:
    return LayerWeights(cfg, layer)


def embedding_rows(cfg: OracleConfig, rows: np.ndarray) -> np.ndarray:
    """Rows of the tied embedding / lm_head [HO Detailed Specs, weight sharing]."""
    out = np.empty((len(rows), cfg.d_model))
    for i, r in enumerate(np.asarray(rows).ravel()):
        out[i] = weight_tensor(cfg.seed, EMBED_TID, (cfg.d_model,), cfg.weight_std,
                               cfg.bf16_weights, start=int(r) * cfg.d_model)
    return out


def embedding_block(cfg: OracleConfig, v0: int, v1: int) -> np.ndarray:
    return weight_tensor(cfg.seed, EMBED_TID, (v1 - v0, cfg.d_model), cfg.weight_std,
                         cfg.bf16_weights, start=v0 * cfg.d_model).astype(np.float64)


# ----------------------------------------------------------------------------- pieces

def rmsnorm(x: np.ndarray, w: np.ndarray, eps: float) -> np.ndarray:
    """R6, the norms listed in [HO Detailed Specs] (input, post-attention, pre-FFN, final)."""
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * w


def rope_pairs_rotated(cfg: OracleConfig, layer: int) -> int:
    """R4: RoPE on local layers, p-RoPE (first ceil(p*dh/2) pairs) on global ones [HO Detailed Specs]."""
    if not cfg.rope_enabled:
        return 0
    half = cfg.head_dim // 2
    if is_global_layer(cfg, layer):
        return int(math.ceil(cfg.prope_fraction * half))
    return half


def rope_rotate(x: np.ndarray, positions: np.ndarray, theta: float, n_rot: int) -> np.ndarray:
    """Rotate pairs (x_j, x_{j+dh/2}), j < n_rot, by angle pos * theta^(-2j/dh).

    x: [T, H, dh]; positions: [T].  Pairs j >= n_rot pass through unchanged.
    """
    x = np.asarray(x, dtype=np.float64)
    out = x.copy()
    dh = x.shape[-1]
    half = dh // 2
    if n_rot == 0:
        return out
    j = np.arange(n_rot, dtype=np.float64)
    inv_freq = theta ** (-2.0 * j / dh)
    ang = np.asarray(positions, dtype=np.float64)[:, None] * inv_freq[None, :]   # [T, n_rot]
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    a, b = x[..., :n_rot], x[..., half:half + n_rot]
    out[..., :n_rot] = a * c - b * s
    out[..., half:half + n_rot] = a * s + b * c
    return out


def _softmax_rows(s: np.ndarray) -> np.ndarray:
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=-1, keepdims=True)


def attention(q, k_canvas, v_canvas, k_prompt, v_prompt, n_visible: int) -> np.ndarray:
    """R1/R2/R5: one softmax over the visible prompt keys and all canvas keys.

    Bidirectional over the canvas [EF Technical Architecture; HO Detailed
    Specs], cross-attention into the cached prompt KV [EF Technical
    Architecture], grouped-query heads [HO Detailed Specs].
    q [Tc, Hq, dh]; k_canvas, v_canvas [Tc, Hkv, dh]; k_prompt, v_prompt
    [Hkv, P, dh]; the visible prompt keys are the last ``n_visible``.
    Returns o [Tc, Hq, dh].
    """
    Tc, Hq, dh = q.shape
    Hkv, P = k_prompt.shape[0], k_prompt.shape[1]
    group = Hq // Hkv
    out = np.empty((Tc, Hq, dh))
    for h in range(Hq):
        g = h // group
        keys = np.concatenate([k_prompt[g, P - n_visible:], k_canvas[:, g]], axis=0)
        vals = np.concatenate([v_prompt[g, P - n_visible:], v_canvas[:, g]], axis=0)
        p = _softmax_rows(q[:, h] @ keys.T / math.sqrt(dh))
        out[:, h] = p @ vals
    return out


def attention_split_kv(q, keys, vals, chunks) -> np.ndarray:
    """Same softmax-attention computed over key chunks and merged by log-sum-exp.

    q [Tq, dh]; keys, vals [Nk, dh]; ``chunks`` is a list of (start, stop).
    Each chunk gives (O_c, m_c, l_c) = (sum_j e^{s_j - m_c} v_j, max_j s_j,
    sum_j e^{s_j - m_c}); the merge rescales by e^{m_c - M}.  Used to show the
    split-KV decomposition the GPU uses is exact.
    """
    dh = q.shape[-1]
    parts = []
    for a, b in chunks:
        s = q @ keys[a:b].T / math.sqrt(dh)
        m = s.max(axis=-1)
        e = np.exp(s - m[:, None])
        parts.append((e @ vals[a:b], m, e.sum(axis=-1)))
    M = np.max(np.stack([p[1] for p in parts]), axis=0)
    num = sum(o * np.exp(m - M)[:, None] for o, m, _ in parts)
    den = sum(l * np.exp(m - M) for _, m, l in parts)
    return num / den[:, None]


def router_topk(logits: np.ndarray, k: int):
    """R8: top-k experts per row [EF Technical Architecture: 8 of 128 active; HO: router].

    Selection orders experts by (-logit, index); weights are the softmax over
    the k chosen logits (= the full softmax probabilities renormalised over
    the chosen experts).  Returns idx int32 [N, k] (best first), w float64 [N, k].
    """
    logits = np.asarray(logits)
    N, E = logits.shape
    idx = np.empty((N, k), dtype=np.int32)
    w = np.empty((N, k))
    for t in range(N):
        order = sorted(range(E), key=lambda e: (-float(logits[t, e]), e))[:k]
        idx[t] = order
        sel = np.array([float(logits[t, e]) for e in order])
        ex = np.exp(sel - sel.max())
        w[t] = ex / ex.sum()
    return idx, w


def router_permutation(idx: np.ndarray, n_experts: int):
    """Counting sort of (row, slot) assignments by expert, stable in row order.

    Returns offsets int32 [E+1] and perm int32 [N*k] where
    perm[offsets[e] + r] = t * k + j for the r-th assignment (t, j) to expert e
    in increasing t.  This is the grouping the expert FFN consumes.
    """
    N, k = idx.shape
    buckets = [[] for _ in range(n_experts)]
    for t in range(N):
        for j in range(k):
            buckets[int(idx[t, j])].append(t * k + j)
    offsets = np.zeros(n_experts + 1, dtype=np.int32)
    for e in range(n_experts):
        offsets[e + 1] = offsets[e] + len(buckets[e])
    perm = np.array([a for b in buckets for a in b], dtype=np.int32)
    return offsets, perm


def silu(x):
    return x / (1.0 + np.exp(-x))


def expert_mlp(x, wg, wu, wd):
    """R10 gated MLP (gate/up/down [HO Detailed Specs]): (silu(x Wg^T) * (x Wu^T)) Wd^T."""
    return (silu(x @ wg.T) * (x @ wu.T)) @ wd.T


def moe_ffn(cfg: OracleConfig, W: LayerWeights, x: np.ndarray, router_bias=None,
            forced_idx: Optional[np.ndarray] = None):
    """MoE FFN: router -> top-k routed experts + shared expert (R8, R9).

    x [N, d].  ``forced_idx`` replaces the selection (used when a near-tie in
    the router is decided differently by the device; the weights then are the
    softmax over the forced experts' logits).  Returns (y, logits, idx, w).
    """
    logits = x @ W.get("wr").T
    if router_bias is not None:
        logits = logits + np.asarray(router_bias, dtype=np.float64)[None, :]
    if forced_idx is None:
        idx, w = router_topk(logits, cfg.top_k)
    else:
        idx = np.asarray(forced_idx, dtype=np.int32)
        sel = np.take_along_axis(logits, idx.astype(np.int64), axis=1)
        ex = np.exp(sel - sel.max(axis=1, keepdims=True))
        w = ex / ex.sum(axis=1, keepdims=True)
    y = np.zeros_like(x)
    for e in np.unique(idx):
        rows, slots = np.nonzero(idx == e)
        wg, wu, wd = W.expert(int(e))
        y[rows] += w[rows, slots][:, None] * expert_mlp(x[rows], wg, wu, wd)
    if cfg.n_shared:
        y += expert_mlp(x, *W.shared())
    return y, logits, idx, w


def layer_forward(cfg: OracleConfig, W: LayerWeights, h: np.ndarray, k_prompt, v_prompt,
                  router_bias=None, forced_idx=None, trace: Optional[dict] = None):
    """One decoder block on the hidden states of B canvases (R7).

    h [B, Tc, d]; k_prompt, v_prompt [B, Hkv, P, dh] (already rotated).
    Returns the new h [B, Tc, d].  ``trace`` (a dict) receives intermediates.
    """
    c = cfg
    B, Tc, d = h.shape
    P = k_prompt.shape[2]
    layer = W.layer
    dh, Hq, Hkv = c.head_dim, c.n_q_heads, c.n_kv_heads
    n_rot = rope_pairs_rotated(c, layer)
    n_vis = P if is_global_layer(c, layer) else min(c.window, P)
    pos = P + np.arange(Tc)
    h = np.asarray(h, dtype=np.float64)

    x = rmsnorm(h, W.norm("input"), c.rms_eps)
    q = (x @ W.get("wq").T).reshape(B, Tc, Hq, dh)
    k = (x @ W.get("wk").T).reshape(B, Tc, Hkv, dh)
    v = (x @ W.get("wv").T).reshape(B, Tc, Hkv, dh)
    o = np.empty((B, Tc, Hq, dh))
    for b in range(B):
        qb = rope_rotate(q[b], pos, c.rope_theta, n_rot)
        kb = rope_rotate(k[b], pos, c.rope_theta, n_rot)
        o[b] = attention(qb, kb, v[b], np.asarray(k_prompt[b], np.float64),
                         np.asarray(v_prompt[b], np.float64), n_vis)
    attn = o.reshape(B, Tc, Hq * dh) @ W.get("wo").T
    h1 = h + rmsnorm(attn, W.norm("post_attn"), c.rms_eps)
    x2 = rmsnorm(h1, W.norm("pre_ff"), c.rms_eps)
    fidx = None if forced_idx is None else np.asarray(forced_idx).reshape(B * Tc, -1)
    y, logits, idx, w = moe_ffn(c, W, x2.reshape(B * Tc, d), router_bias, fidx)
    h2 = h1 + y.reshape(B, Tc, d)
    if trace is not None:
        trace.update(x=x, q=q, k=k, v=v, attn_o=o, attn=attn, h1=h1, x2=x2,
                     router_logits=logits, idx=idx, w=w, moe=y.reshape(B, Tc, d), out=h2)
    return h2


def head_reduce(cfg: OracleConfig, hn: np.ndarray, vocab_block: int = 8192):
    """Tied vocab head and the per-row statistics the commit uses (R11, R12).

    hn [N, d] are final-normed hidden states.  logits = hn E^T over the whole
    vocabulary [EF: vocab 262K; HO: embed_tokens shared with lm_head].  With
    the mask id excluded: m = max logit, a = argmax (lowest index on ties),
    s = sum exp(l - m), conf = 1 / s.  Returns (conf, a, m, s).
    """
    N = hn.shape[0]
    logits = np.empty((N, cfg.vocab))
    for v0 in range(0, cfg.vocab, vocab_block):
        v1 = min(cfg.vocab, v0 + vocab_block)
        logits[:, v0:v1] = hn @ embedding_block(cfg, v0, v1).T
    return logit_stats(logits, cfg.mask_id)


def logit_stats(logits: np.ndarray, mask_id: int):
    """(conf, argmax, max, sum) of each row of full logits, mask id excluded (R11, R12)."""
    logits = np.array(logits, dtype=np.float64, copy=True)
    N = logits.shape[0]
    logits[:, mask_id] = -np.inf
    a = np.argmax(logits, axis=1).astype(np.int32)      # first maximal index
    m = logits[np.arange(N), a]
    s = np.exp(logits - m[:, None]).sum(axis=1)
    return 1.0 / s, a, m, s


def commit_count(n_masked: int, steps_left: int) -> int:
    """R13: k = ceil(r / steps_left) [HO How Different / Detailed Specs: confident tokens locked in]."""
    if steps_left < 1:
        raise ValueError("steps_left must be >= 1")
    return -(-n_masked // steps_left)


def commit(canvas: np.ndarray, conf: np.ndarray, tok: np.ndarray, steps_left: int, mask_id: int):
    """R13: lock in the k most confident still-masked rows of each canvas.

    canvas, tok int [B, Tc]; conf [B, Tc].  Rows already committed keep their
    token.  Returns (new_canvas, committed bool [B, Tc]).
    """
    canvas = np.array(canvas, dtype=np.int32, copy=True)
    committed = np.zeros(canvas.shape, dtype=bool)
    for b in range(canvas.shape[0]):
        masked = [i for i in range(canvas.shape[1]) if canvas[b, i] == mask_id]
        k = commit_count(len(masked), steps_left)
        order = sorted(masked, key=lambda i: (-float(conf[b, i]), i))[:k]
        for i in order:
            canvas[b, i] = tok[b, i]
            committed[b, i] = True
    return canvas, committed


def final_hidden(cfg: OracleConfig, canvas: np.ndarray, k_prompt_layers, v_prompt_layers,
                 router_bias=None, weights=None) -> np.ndarray:
    """The states the vocab head reads: embedding of the canvas tokens, every block,
    then the final norm [HO Detailed Specs].  Returns hn [B * Tc, d]."""
    c = cfg
    B, Tc = canvas.shape
    h = embedding_rows(c, canvas.reshape(-1)).reshape(B, Tc, c.d_model)
    for layer in range(c.n_layers):
        W = weights[layer] if weights is not None else layer_weights(c, layer)
        h = layer_forward(c, W, h, k_prompt_layers[layer], v_prompt_layers[layer], router_bias)
    return rmsnorm(h, np.ones(c.d_model), c.rms_eps).reshape(B * Tc, c.d_model)


def canvas_step(cfg: OracleConfig, canvas: np.ndarray, k_prompt_layers, v_prompt_layers,
                steps_left: int, router_bias=None, weights=None):
    """One denoising pass over the canvas, then the commit (R1-R14).

    canvas int [B, Tc]; k_prompt_layers[l], v_prompt_layers[l] are
    [B, Hkv, P, dh].  ``weights`` optionally supplies LayerWeights per layer.
    Returns (new_canvas, conf, tok, committed).
    """
    c = cfg
    B, Tc = canvas.shape
    hn = final_hidden(c, canvas, k_prompt_layers, v_prompt_layers, router_bias, weights)
    conf, tok, _, _ = head_reduce(c, hn)
    conf, tok = conf.reshape(B, Tc), tok.reshape(B, Tc)
    new_canvas, committed = commit(canvas, conf, tok, steps_left, c.mask_id)
    return new_canvas, conf, tok, committed


def denoise_block(cfg: OracleConfig, canvas, k_prompt_layers, v_prompt_layers, n_steps: int,
                  router_bias=None, weights=None, history: Optional[list] = None):
    """Fixed-step denoising of one canvas block: step s runs with steps_left = n_steps - s.

    [HO How Different: passes repeat until every token is final; G4: a small,
    fixed number of passes per 256-token block].
    """
    canvas = np.array(canvas, dtype=np.int32, copy=True)
    for s in range(n_steps):
        canvas, conf, tok, committed = canvas_step(cfg, canvas, k_prompt_layers, v_prompt_layers,
                                                   n_steps - s, router_bias, weights)
        if history is not None:
            history.append(dict(canvas=canvas.copy(), conf=conf, tok=tok, committed=committed))
    return canvas
