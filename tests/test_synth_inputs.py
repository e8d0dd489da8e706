"""The seeded input recipe (shared by the tests, the bench and the smoke run):
reproducible, with the distributions and the Zipf routing skew it states."""

import numpy as np
import pytest
import torch

import synth


def test_prompt_kv_is_seeded_per_layer_and_standard_normal():
    cfg = synth.config("ragged")
    k0, v0 = synth.prompt_kv(cfg, 0)
    k0b, _ = synth.prompt_kv(cfg, 0)
    k1, _ = synth.prompt_kv(cfg, 1)
    assert k0.dtype == torch.bfloat16
    assert k0.shape == (cfg["batch"], cfg["n_kv_heads"], cfg["prompt_len"], cfg["head_dim"])
    assert torch.equal(k0, k0b)                       # same seed, same values
    assert not torch.equal(k0, k1)                    # layers are independent
    assert not torch.equal(k0, v0)
    x = k0.float().numpy().ravel()
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01


def test_initial_canvas_is_all_mask():
    cfg = synth.config("tiny")
    c = synth.initial_canvas(cfg)
    assert c.dtype == torch.int32 and c.shape == (cfg["batch"], cfg["canvas_len"])
    assert bool((c == cfg["mask_id"]).all())


def test_zipf_bias_masses():
    b = synth.zipf_router_bias(128, 1.1).double().numpy()
    p = np.sort(np.exp(b))[::-1]
    assert p.sum() == pytest.approx(1.0, abs=1e-6)
    assert p[0] == pytest.approx(0.226, abs=0.002)      # rank 1
    assert p[:8].sum() == pytest.approx(0.57, abs=0.01)  # top 8 ranks
    assert p[-1] == pytest.approx(0.0011, abs=0.0002)   # rank 128
    # a seeded permutation: the same experts get the same ranks every time
    assert torch.equal(synth.zipf_router_bias(128, 1.1), synth.zipf_router_bias(128, 1.1))
