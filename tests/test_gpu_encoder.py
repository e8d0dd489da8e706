"""Parity of the causal encoder (dg_encode) and block-autoregressive generation
(dg_generate) with the oracle (oracle/encoder.py), through the C ABI.

Tolerances as for the decoder: the cached keys and values of every layer within
relative L2 1e-2 of the oracle's (bf16 storage on the device); every pass of a
generation compared with the oracle's pass on the same canvas and the cache the
oracle builds from the prompt and the device's previous blocks, commits equal up
to near ties of the oracle's own logits."""

import numpy as np
import pytest
import torch

import synth
from oracle import encoder as oe
from oracle import model as om
from tests import test_gpu_parity as tp
from tests.gpu_helpers import Ctx, rel_l2

pytestmark = pytest.mark.gpu

TOL = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from libbuild import build_library as build
    build()
    torch.cuda.set_device(0)


def _prompt(cfg, n, seed=11):
    g = np.random.default_rng(seed)
    return g.integers(1, cfg["vocab"], size=(cfg["batch"], n)).astype(np.int32)


def _context_kv(c, layer, n):
    B, Hkv, dh = c.B, c.cfg["n_kv_heads"], c.cfg["head_dim"]
    k = torch.empty(B, Hkv, n, dh, dtype=torch.bfloat16, device="cuda")
    v = torch.empty_like(k)
    c.dg.dg_context_kv(c.ctx, layer, k.data_ptr(), v.data_ptr())
    return k.float().cpu().numpy(), v.float().cpu().numpy()


def _check_cache(c, kc_ref, vc_ref, n):
    assert c.dg.dg_context_length(c.ctx) == n
    errs = []
    for l in range(c.cfg["n_layers"]):
        k, v = _context_kv(c, l, n)
        ek, ev = rel_l2(k, kc_ref[l]), rel_l2(v, vc_ref[l])
        errs.append((ek, ev))
        assert ek < TOL and ev < TOL, (l, ek, ev)
    return errs


@pytest.mark.parametrize("name,n,split,max_batch", [
    ("tiny", 32, None, None), ("tiny", 32, 7, None), ("tiny", 40, None, 4),
    ("ragged", 300, None, None), ("ragged", 300, 100, None), ("ragged", 300, None, 5)])
def test_encode_matches_oracle(name, n, split, max_batch):
    """The prompt is encoded in chunks of max_batch * canvas_len / batch rows (tiny: 16,
    or 64 with room for 4 canvases; ragged: 48, or 120 with room for 5, so the ragged
    window of 128 reaches back over earlier chunks); one call or two."""
    cfg = synth.config(name, bf16_weights=True)
    c = Ctx(cfg, max_batch=max_batch, with_prompt=False, max_context=n)
    try:
        toks = _prompt(cfg, n)
        td = torch.from_numpy(toks).cuda()
        if split is None:
            c.dg.dg_encode(c.ctx, td.data_ptr(), c.B, n)
        else:
            a = td[:, :split].contiguous()
            b = td[:, split:].contiguous()
            c.dg.dg_encode(c.ctx, a.data_ptr(), c.B, split)
            c.dg.dg_encode(c.ctx, b.data_ptr(), c.B, n - split)
        k0, v0 = oe.empty_cache(c.oc, c.B)
        kr, vr = oe.encode(c.oc, toks, k0, v0)
        errs = _check_cache(c, kr, vr, n)
        print(name, n, split, "cache rel-L2 per layer", errs)
    finally:
        c.close()


@pytest.mark.parametrize("global_every", [2, 1])
def test_encode_full_width_layer_with_a_short_window(global_every):
    """One layer of the stack's width (2816, 16q/8kv x 256, 128 experts), local with a
    window of 128 or global, 300 prompt tokens in chunks of 256 and 44: the per-row
    window cuts both the cached keys and the chunk's own keys."""
    cfg = synth.config("stack", n_layers=1, window=128, global_every=global_every,
                       prompt_len=300)
    c = Ctx(cfg, with_prompt=False, max_context=300)
    try:
        toks = _prompt(cfg, 300, seed=3)
        td = torch.from_numpy(toks).cuda()
        c.dg.dg_encode(c.ctx, td.data_ptr(), c.B, 300)
        k0, v0 = oe.empty_cache(c.oc, c.B)
        kr, vr = oe.encode(c.oc, toks, k0, v0)
        errs = _check_cache(c, kr, vr, 300)
        print("full width, global_every", global_every, "cache rel-L2", errs)
    finally:
        c.close()


def test_generate_matches_oracle_pass_by_pass():
    """tiny: prompt 32, three blocks of 16 slots, 4 passes each.  dg_generate equals the
    same work done call by call (dg_encode, dg_canvas_step, dg_encode of the block),
    and every pass of that equals the oracle's pass on the same canvas and the cache
    the oracle builds from the prompt and the device's previous blocks, up to near
    ties of the oracle's own logits (as for the decoder's pass)."""
    cfg = synth.config("tiny", bf16_weights=True)
    n_blocks, steps, P = 3, 4, cfg["prompt_len"]
    Tc, mask = cfg["canvas_len"], cfg["mask_id"]
    c = Ctx(cfg, with_prompt=False, max_context=P + n_blocks * Tc)
    try:
        prompt = _prompt(cfg, P, seed=5)
        pd = torch.from_numpy(prompt).cuda()
        out = torch.zeros(c.B, n_blocks * Tc, dtype=torch.int32, device="cuda")
        c.dg.dg_generate(c.ctx, pd.data_ptr(), c.B, P, n_blocks, steps, out.data_ptr())
        gen = out.cpu().numpy()
        assert not np.any(gen == mask)
        assert c.dg.dg_context_length(c.ctx) == P + n_blocks * Tc

        c.dg.dg_reset_context(c.ctx)
        c.dg.dg_encode(c.ctx, pd.data_ptr(), c.B, P)
        kr, vr = oe.empty_cache(c.oc, c.B)
        kr, vr = oe.encode(c.oc, prompt, kr, vr)
        n_near = 0
        for blk in range(n_blocks):
            canvas = torch.full((c.B, Tc), mask, dtype=torch.int32, device="cuda")
            for s in range(steps):
                canvas0 = canvas.cpu().numpy()
                c.dg.dg_canvas_step(c.ctx, canvas.data_ptr(), c.B, steps - s, None, None)
                c.dg.dg_sync(c.ctx)
                o_logits = tp._oracle_pass_logits(c.oc, canvas0, list(zip(kr, vr)))
                n_near += tp._assert_commit_matches_up_to_near_ties(
                    canvas.cpu().numpy(), canvas0, o_logits, mask, steps - s, tp.LOGIT_TOL)
            block = canvas.cpu().numpy()
            assert np.array_equal(block, gen[:, blk * Tc:(blk + 1) * Tc]), blk
            c.dg.dg_encode(c.ctx, canvas.data_ptr(), c.B, Tc)
            kr, vr = oe.encode(c.oc, block, kr, vr)
        errs = _check_cache(c, kr, vr, P + n_blocks * Tc)
        print("generate: near-tie exemptions", n_near, "final cache rel-L2", errs)
    finally:
        c.close()


def test_context_errors():
    cfg = synth.config("tiny", bf16_weights=True)
    c = Ctx(cfg, with_prompt=False, max_context=20)
    try:
        import canvas_denoising_step_b200 as dg
        td = torch.ones(c.B, 16, dtype=torch.int32, device="cuda")
        c.dg.dg_encode(c.ctx, td.data_ptr(), c.B, 16)
        with pytest.raises(dg.DgError) as e:
            c.dg.dg_encode(c.ctx, td.data_ptr(), c.B, 16)      # 32 > max_context
        assert e.value.code == dg.DG_ERR_INVALID_ARG
        assert c.dg.dg_context_length(c.ctx) == 16
        c.dg.dg_reset_context(c.ctx)
        assert c.dg.dg_context_length(c.ctx) == 0
        with pytest.raises(dg.DgError) as e:
            c.dg.dg_context_kv(c.ctx, 0, td.data_ptr(), td.data_ptr())
        assert e.value.code == dg.DG_ERR_BAD_STATE
    finally:
        c.close()
    c = Ctx(cfg, with_prompt=False)          # no own cache
    try:
        import canvas_denoising_step_b200 as dg
        td = torch.ones(c.B, 4, dtype=torch.int32, device="cuda")
        with pytest.raises(dg.DgError) as e:
            c.dg.dg_encode(c.ctx, td.data_ptr(), c.B, 4)
        assert e.value.code == dg.DG_ERR_BAD_STATE
    finally:
        c.close()
