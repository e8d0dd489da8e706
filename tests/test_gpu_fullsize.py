"""Parity at the full workload sizes, in the launch configuration the bench
uses: the single 2816-wide layer, layers and the vocab head of the 30-layer
stack (sampled rows for the head), a global layer over a 65536-token prompt,
and 8 batched canvases with Zipf-skewed routing.  The oracle recomputes every
row of each checked layer; the head is checked on sampled rows."""

import numpy as np
import pytest
import torch

import synth
from oracle import model as om
from tests.gpu_helpers import Ctx, rel_l2
from tests.test_gpu_parity import LAYER_TOL, _layer_check

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from libbuild import build_library as build
    build()
    torch.cuda.set_device(0)


def test_single_layer_workload():
    """One global 2816-wide layer, canvas 256, prompt 2048, hidden states N(0,1)."""
    rep = _layer_check("layer", 0)
    assert rep["layer"] < LAYER_TOL


def _layer_on_big_ctx(c, layer, router_bias=None):
    cfg, oc = c.cfg, c.oc
    B, Tc, T, d = c.B, c.Tc, c.T, cfg["d_model"]
    k = cfg["top_k"]
    x_in = synth.hidden_states(cfg)
    xd = x_in.cuda()
    out = torch.empty_like(xd)
    c.dg.dg_layer_forward(c.ctx, layer, xd.data_ptr(), out.data_ptr(), T)
    c.dg.dg_sync(c.ctx)
    got = out.float().cpu().numpy().reshape(B, Tc, d)
    idx = c.fetch("idx", torch.int32, (T, k))
    kp, vp = c.kv_np(layer)
    tr = {}
    ref = om.layer_forward(oc, om.layer_weights(oc, layer),
                           x_in.float().numpy().astype(np.float64).reshape(B, Tc, d), kp, vp,
                           router_bias=router_bias, trace=tr)
    flips = int((tr["idx"] != idx).any(axis=1).sum())
    err = rel_l2(got, ref)
    # with the device's routing forced, the remaining difference is rounding only
    tr2 = {}
    ref2 = om.layer_forward(oc, om.layer_weights(oc, layer),
                            x_in.float().numpy().astype(np.float64).reshape(B, Tc, d), kp, vp,
                            router_bias=router_bias, forced_idx=idx, trace=tr2)
    err_forced = rel_l2(got, ref2)
    return err, err_forced, flips, idx


@pytest.fixture(scope="module")
def stack_ctx():
    cfg = synth.config("stack")
    c = Ctx(cfg)
    yield c
    c.close()


@pytest.mark.parametrize("layer", [0, 5])
def test_stack_layers(stack_ctx, layer):
    err, err_forced, flips, _ = _layer_on_big_ctx(stack_ctx, layer)
    print("stack layer", layer, "rel-L2", err, "forced", err_forced, "rows flipped", flips)
    assert err_forced < LAYER_TOL
    if flips == 0:
        assert err < LAYER_TOL


def test_stack_head_sampled_rows_and_commit(stack_ctx):
    c = stack_ctx
    cfg, oc, B, Tc, T = c.cfg, c.oc, c.B, c.Tc, c.T
    canvas0 = synth.initial_canvas(cfg).numpy()
    canvas = torch.from_numpy(canvas0).cuda()
    conf = torch.empty(B, Tc, device="cuda")
    com = torch.empty(B, Tc, dtype=torch.uint8, device="cuda")
    S = cfg["steps"]
    c.dg.dg_canvas_step(c.ctx, canvas.data_ptr(), B, S, conf.data_ptr(), com.data_ptr())
    c.dg.dg_sync(c.ctx)
    hn = c.fetch("hn", torch.bfloat16, (T, cfg["d_model"]))
    tok = c.fetch("tok", torch.int32, (T,))
    conf_np = conf.cpu().numpy().ravel()
    rows = np.array([0, 1, 77, 128, 200, 255])
    rconf, rtok, _, _ = om.head_reduce(oc, hn[rows].astype(np.float64), vocab_block=32768)
    assert np.allclose(conf_np[rows], rconf, rtol=1e-3)
    assert np.array_equal(tok[rows], rtok)
    ref_can, ref_com = om.commit(canvas0, conf_np.reshape(B, Tc), tok.reshape(B, Tc), S,
                                 cfg["mask_id"])
    assert np.array_equal(canvas.cpu().numpy(), ref_can)
    assert int(com.cpu().numpy().sum()) == 32
    assert np.array_equal(com.cpu().numpy().astype(bool), ref_com)


def test_long_context_global_layer():
    """A global layer over a 65536-token prompt (split-KV path with many chunks)."""
    cfg = synth.config("longctx", n_layers=6)
    c = Ctx(cfg)
    try:
        err, err_forced, flips, _ = _layer_on_big_ctx(c, 5)
        print("longctx global layer rel-L2", err, "forced", err_forced, "rows flipped", flips)
        assert err_forced < LAYER_TOL
        e0, f0, fl0, _ = _layer_on_big_ctx(c, 0)
        print("longctx local layer rel-L2", e0, "forced", f0, "rows flipped", fl0)
        assert f0 < LAYER_TOL
    finally:
        c.close()


def test_batched_zipf_layer():
    """8 canvases (2048 rows), prompt 8192 each, Zipf(1.1)-biased routing."""
    cfg = synth.config("batched", n_layers=1)
    c = Ctx(cfg)
    try:
        bias = synth.zipf_router_bias(cfg["n_experts"], cfg["zipf_s"])
        bd = bias.cuda()
        c.dg.dg_set_router_bias(c.ctx, bd.data_ptr())
        err, err_forced, flips, idx = _layer_on_big_ctx(c, 0, router_bias=bias.numpy())
        counts = np.bincount(idx.ravel(), minlength=cfg["n_experts"])
        print("batched layer rel-L2", err, "forced", err_forced, "rows flipped", flips,
              "max/min expert rows", counts.max(), counts.min())
        assert counts.max() > 1000          # the skew reaches the hot expert
        assert err_forced < LAYER_TOL
    finally:
        c.close()
