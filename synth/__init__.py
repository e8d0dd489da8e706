"""Seeded synthetic inputs and workload shapes for the canvas denoising step.

This module holds no arithmetic of the method.  It only fixes the shapes of
the workloads and draws the seeded inputs that both the CUDA path and the CPU
oracle consume: the prompt K/V cache of every layer, hidden states for the
single-layer workload, the initial all-mask canvas, and the Zipf-skewed
router bias of the batched workload.  Weights are not drawn here: each side
draws them itself from the seed with the same published counter-based
generator.

Seeds: weights 0, prompt K/V 1, hidden states 2, Zipf expert permutation 3.
"""

from __future__ import annotations

import copy

import numpy as np
import torch

WEIGHT_SEED = 0
PROMPT_SEED = 1
HIDDEN_SEED = 2
ZIPF_SEED = 3

_MODEL = dict(window=1024, global_every=6, mask_id=0, rms_eps=1e-6, rope_theta=10000.0,
              prope_fraction=0.25, rope_enabled=True, weight_std=0.02, seed=WEIGHT_SEED)

# Workload shapes.  "layer", "stack", "longctx" and "batched" use the model
# dimensions of the pages (hidden 2816, 30 layers as (5 local + 1 global) x 5,
# window 1024, 128 experts top-8 + 1 shared, canvas 256, vocab 262144).
CONFIGS = {
    # Tiny reference: 2 layers, d=256, 4q/2kv x 64, canvas 16, P=32, 8 experts
    # top-2 + 1 shared, F=512, vocab 1024, 4 denoising steps, mask id 0.
    "tiny": dict(_MODEL, n_layers=2, d_model=256, n_q_heads=4, n_kv_heads=2, head_dim=64,
                 n_experts=8, top_k=2, n_shared=1, d_ff=512, vocab=1024, canvas_len=16,
                 batch=1, prompt_len=32, steps=4, bf16_weights=False),
    # One global 2816-wide layer, canvas 256, prompt 2048, hidden states N(0,1), no head.
    "layer": dict(_MODEL, n_layers=1, d_model=2816, n_q_heads=16, n_kv_heads=8, head_dim=256,
                  n_experts=128, top_k=8, n_shared=1, d_ff=704, vocab=262144, canvas_len=256,
                  batch=1, prompt_len=2048, steps=1, global_every=1, bf16_weights=True),
    # Full 30-layer stack, prompt 4096, tied vocab 262144, 8 steps, batch 1.
    "stack": dict(_MODEL, n_layers=30, d_model=2816, n_q_heads=16, n_kv_heads=8, head_dim=256,
                  n_experts=128, top_k=8, n_shared=1, d_ff=704, vocab=262144, canvas_len=256,
                  batch=1, prompt_len=4096, steps=8, bf16_weights=True),
    # Long-context cross-attention: the stack with a 65536-token prompt.
    "longctx": dict(_MODEL, n_layers=30, d_model=2816, n_q_heads=16, n_kv_heads=8, head_dim=256,
                    n_experts=128, top_k=8, n_shared=1, d_ff=704, vocab=262144, canvas_len=256,
                    batch=1, prompt_len=65536, steps=8, bf16_weights=True),
    # 8 canvases, prompt 8192 each, Zipf(1.1) expert popularity.
    "batched": dict(_MODEL, n_layers=30, d_model=2816, n_q_heads=16, n_kv_heads=8, head_dim=256,
                    n_experts=128, top_k=8, n_shared=1, d_ff=704, vocab=262144, canvas_len=256,
                    batch=8, prompt_len=8192, steps=8, bf16_weights=True, zipf_s=1.1),
    # Test shape: several tiles per GEMM with ragged tails everywhere (F=192,
    # vocab 3000, canvas 48, prompt 300 with a 128 window), one local and one
    # global layer, batch 2.
    "ragged": dict(_MODEL, n_layers=2, d_model=512, n_q_heads=4, n_kv_heads=2, head_dim=256,
                   n_experts=16, top_k=4, n_shared=1, d_ff=192, vocab=3000, canvas_len=48,
                   batch=2, prompt_len=300, steps=4, window=128, global_every=2,
                   bf16_weights=True),
}


def config(name: str, **overrides) -> dict:
    c = copy.deepcopy(CONFIGS[name])
    c.update(overrides)
    c["name"] = name
    return c


def _normal_bf16(shape, seed_seq) -> torch.Tensor:
    g = np.random.default_rng(seed_seq)
    x = g.standard_normal(size=shape, dtype=np.float32)
    return torch.from_numpy(x).to(torch.bfloat16)


def prompt_kv(cfg: dict, layer: int, seed: int = PROMPT_SEED):
    """Prompt K and V of one layer, bf16 [B, Hkv, P, dh], N(0,1), treated as already rotated."""
    shape = (cfg["batch"], cfg["n_kv_heads"], cfg["prompt_len"], cfg["head_dim"])
    return (_normal_bf16(shape, [seed, layer, 0]), _normal_bf16(shape, [seed, layer, 1]))


def hidden_states(cfg: dict, seed: int = HIDDEN_SEED) -> torch.Tensor:
    """Hidden states bf16 [B * canvas_len, d_model], N(0,1)."""
    return _normal_bf16((cfg["batch"] * cfg["canvas_len"], cfg["d_model"]), [seed])


def initial_canvas(cfg: dict) -> torch.Tensor:
    """int32 [B, canvas_len], every slot the mask id."""
    return torch.full((cfg["batch"], cfg["canvas_len"]), cfg["mask_id"], dtype=torch.int32)


def zipf_router_bias(n_experts: int, s: float, seed: int = ZIPF_SEED) -> torch.Tensor:
    """float32 [E]: b_e = ln p_rank(e), p_r proportional to r^-s over ranks 1..E,
    ranks assigned by a seeded random permutation of the experts."""
    g = np.random.default_rng([seed])
    rank = g.permutation(n_experts)                        # rank[e] in 0..E-1
    p = np.arange(1, n_experts + 1, dtype=np.float64) ** (-s)
    p /= p.sum()
    return torch.from_numpy(np.log(p[rank]).astype(np.float32))
