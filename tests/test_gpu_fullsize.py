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
from tests.gpu_helpers import Ctx, rel_l2, router_flips
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


def _layer_on_big_ctx(c, layer, router_bias=None, x_in=None):
    """One block on the device (dg_layer_forward) against the oracle fed the same bf16
    input.  The oracle runs with the device's expert selection forced (so the
    comparison is rounding only); its own selection, from its own logits, must
    equal the device's except on rows that are near-ties (router_flips).
    Returns (rel-L2 with the device's routing, rows flipped, device idx, device output)."""
    cfg, oc = c.cfg, c.oc
    B, Tc, T, d = c.B, c.Tc, c.T, cfg["d_model"]
    k = cfg["top_k"]
    if x_in is None:
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
                           router_bias=router_bias, forced_idx=idx, trace=tr)
    own_idx, _ = om.router_topk(tr["router_logits"], k)
    flipped = router_flips(tr["router_logits"], own_idx, idx)
    return rel_l2(got, ref), int(flipped.sum()), idx, out


@pytest.fixture(scope="module")
def stack_ctx():
    cfg = synth.config("stack")
    c = Ctx(cfg)
    yield c
    c.close()


@pytest.mark.parametrize("layer", [0, 5])
def test_stack_layers(stack_ctx, layer):
    err, flips, _, _ = _layer_on_big_ctx(stack_ctx, layer)
    print("stack layer", layer, "rel-L2", err, "near-tie rows", flips)
    assert err < LAYER_TOL


def test_stack_all_layers_on_the_all_mask_flow(stack_ctx):
    """The routing the benchmark sees: all 30 blocks chained from the embedded
    all-mask canvas (nearly identical rows, a few dozen experts per layer, several
    row chunks per expert), each block checked against the oracle fed the device's
    own bf16 input to that block."""
    c = stack_ctx
    cfg, oc = c.cfg, c.oc
    L = cfg["n_layers"]
    act0 = c.fetch("expert_active", torch.int32, (L,)).copy()
    x = torch.from_numpy(om.embedding_rows(oc, synth.initial_canvas(cfg).numpy().ravel())
                         .astype(np.float32)).to(torch.bfloat16)
    errs, flips = [], []
    for l in range(L):
        err, nf, _, out = _layer_on_big_ctx(c, l, x_in=x)
        errs.append(err)
        flips.append(nf)
        x = out.cpu()
    act = c.fetch("expert_active", torch.int32, (L,)) - act0
    print("all-mask flow rel-L2 per layer", [f"{e:.2e}" for e in errs])
    print("near-tie rows per layer", flips, "active experts per layer", act.tolist())
    assert max(errs) < LAYER_TOL
    assert act.mean() < 96           # the concentrated routing the bench runs


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
    mx = c.fetch("head_max", torch.float32, (T,))
    conf_np = conf.cpu().numpy().ravel()
    rows = np.array([0, 1, 77, 128, 200, 255])
    rconf, rtok, rm, _ = om.head_reduce(oc, hn[rows].astype(np.float64), vocab_block=32768)
    assert np.allclose(conf_np[rows], rconf, rtol=1e-3)
    assert np.array_equal(tok[rows], rtok)
    assert np.abs(mx[rows] - rm).max() < 1e-3
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
        err, flips, _, _ = _layer_on_big_ctx(c, 5)
        print("longctx global layer rel-L2", err, "near-tie rows", flips)
        assert err < LAYER_TOL
        e0, fl0, _, _ = _layer_on_big_ctx(c, 0)
        print("longctx local layer rel-L2", e0, "near-tie rows", fl0)
        assert e0 < LAYER_TOL
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
        err, flips, idx, _ = _layer_on_big_ctx(c, 0, router_bias=bias.numpy())
        counts = np.bincount(idx.ravel(), minlength=cfg["n_experts"])
        print("batched layer rel-L2", err, "near-tie rows", flips,
              "max/min expert rows", counts.max(), counts.min())
        assert counts.max() > 1000          # the skew reaches the hot expert
        assert err < LAYER_TOL
    finally:
        c.close()


def test_batched_pass_head_and_commit():
    """One full pass of the batched workload: 8 canvases of 256 slots through the 30
    blocks with Zipf(1.1)-biased routing, the vocab head over all 2048 rows and one
    commit per canvas.  The head is checked on sampled rows of every canvas against
    the oracle fed the device's final hidden states; the commit bit-exactly on the
    device's confidences."""
    cfg = synth.config("batched")
    c = Ctx(cfg)
    try:
        oc, B, Tc, T = c.oc, c.B, c.Tc, c.T
        bias = synth.zipf_router_bias(cfg["n_experts"], cfg["zipf_s"])
        bd = bias.cuda()
        c.dg.dg_set_router_bias(c.ctx, bd.data_ptr())
        canvas0 = synth.initial_canvas(cfg).numpy()
        canvas = torch.from_numpy(canvas0).cuda()
        conf = torch.empty(B, Tc, device="cuda")
        com = torch.empty(B, Tc, dtype=torch.uint8, device="cuda")
        S = cfg["steps"]
        c.dg.dg_canvas_step(c.ctx, canvas.data_ptr(), B, S, conf.data_ptr(), com.data_ptr())
        c.dg.dg_sync(c.ctx)
        hn = c.fetch("hn", torch.bfloat16, (T, cfg["d_model"]))
        tok = c.fetch("tok", torch.int32, (T,))
        mx = c.fetch("head_max", torch.float32, (T,))
        conf_np = conf.cpu().numpy().ravel()
        rows = np.array([b * Tc + i for b in range(B) for i in (b * 29 % Tc, Tc - 1 - b)])
        rconf, rtok, rm, _ = om.head_reduce(oc, hn[rows].astype(np.float64), vocab_block=32768)
        assert np.allclose(conf_np[rows], rconf, rtol=1e-3)
        assert np.array_equal(tok[rows], rtok)
        assert np.abs(mx[rows] - rm).max() < 1e-3
        ref_can, ref_com = om.commit(canvas0, conf_np.reshape(B, Tc), tok.reshape(B, Tc), S,
                                     cfg["mask_id"])
        assert np.array_equal(canvas.cpu().numpy(), ref_can)
        assert np.array_equal(com.cpu().numpy().astype(bool), ref_com)
        assert np.array_equal(com.cpu().numpy().sum(axis=1), np.full(B, Tc // S))
    finally:
        c.close()
