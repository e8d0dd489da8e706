"""Entropy-bounded denoising on the device against the CPU oracle.

Criteria: entropies within rtol 1e-3 of the oracle fed the device's own final
hidden states; the pass's decisions (stop, which slots commit, which token
each takes) bit-exact with the oracle's decisions on the device's entropies,
argmax and drawn tokens; each drawn token valid for the oracle's own
distribution: the slot's uniform lies in that token's interval of the oracle's
cumulative distribution, up to 1e-4.
"""

import numpy as np
import pytest
import torch

import synth
from oracle import eb_sampler as eb
from oracle import model as om
from tests.gpu_helpers import Ctx

pytestmark = pytest.mark.gpu

H_RTOL = 1e-3
CDF_TOL = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from libbuild import build_library as build
    build()
    torch.cuda.set_device(0)


def _dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def test_eb_commit_hook_bit_exact():
    cfg = synth.config("ragged")
    c = Ctx(cfg, with_prompt=False)
    try:
        B, Tc, mask = c.B, c.Tc, cfg["mask_id"]
        g = np.random.default_rng(5)
        cases = []
        # high entropies: one slot a pass; ties broken toward the lower slot
        H = g.uniform(5.0, 8.0, size=(B, Tc)).astype(np.float32)
        H[0, [3, 9, 20]] = 4.0
        cases.append(("high", H, None, False))
        # dyadic entropies whose running sums are exact in float and double:
        # canvas 0 in entropy order sums 0.00390625 + 0.0078125 + 0.03125 = 0.04296875
        # and passes the bound 0.1 with the next (0.10546875): 3 commits; canvas 1
        # takes its six 0.015625 slots (0.09375) and stops at the first 0.5
        H = np.full((B, Tc), 0.5, np.float32)
        H[0, [1, 5, 7, 11]] = [0.0625, 0.03125, 0.00390625, 0.0078125]
        H[1, :6] = 0.015625
        cases.append(("bound", H, None, False))
        # low entropies, argmax equal to the previous pass on canvas 0 only: it stops
        H = np.full((B, Tc), 0.001, np.float32)
        cases.append(("stop", H, "same0", False))
        # the last allowed pass
        cases.append(("last", g.uniform(1, 2, size=(B, Tc)).astype(np.float32), None, True))
        for name, H, prev_kind, last in cases:
            canvas = np.where(g.uniform(size=(B, Tc)) < 0.25, 17, mask).astype(np.int32)
            if name == "bound":
                canvas[0, [1, 5, 7, 11]] = mask
                canvas[1, :6] = mask
            a = g.integers(1, cfg["vocab"], size=(B, Tc)).astype(np.int32)
            drawn = g.integers(1, cfg["vocab"], size=(B, Tc)).astype(np.int32)
            prev = None
            if prev_kind == "same0":
                prev = a.copy()
                prev[1, 4] += 1
            dH, da, dd = _dev(H), _dev(a), _dev(drawn)
            dp = _dev(prev) if prev is not None else None
            dcan = _dev(canvas)
            com = torch.empty(B, Tc, dtype=torch.uint8, device="cuda")
            stop = torch.empty(B, dtype=torch.uint8, device="cuda")
            c.dg.dg_eb_commit(c.ctx, dH.data_ptr(), da.data_ptr(), dd.data_ptr(),
                              dp.data_ptr() if dp is not None else None, dcan.data_ptr(), B,
                              last, com.data_ptr(), stop.data_ptr())
            c.dg.dg_sync(c.ctx)
            ref_can, ref_com, ref_stop = eb.eb_commit_step(canvas, H.astype(np.float64), a, drawn,
                                                           prev, mask, last)
            assert np.array_equal(dcan.cpu().numpy(), ref_can), name
            assert np.array_equal(com.cpu().numpy().astype(bool), ref_com), name
            assert np.array_equal(stop.cpu().numpy().astype(bool), ref_stop), name
            if name == "stop":
                assert ref_stop.tolist() == [True, False]
            if name == "bound":
                assert ref_com[0].sum() == 3 and ref_com[1].sum() == 6
    finally:
        c.close()


def _oracle_logits(oc, hn, block=32768):
    out = np.empty((hn.shape[0], oc.vocab))
    for v0 in range(0, oc.vocab, block):
        v1 = min(oc.vocab, v0 + block)
        out[:, v0:v1] = hn @ om.embedding_block(oc, v0, v1).T
    return out


def _check_draws(p, u, drawn, rows):
    """Each drawn token's interval [c_{j-1}, c_j) of the oracle's CDF holds u (within tol)."""
    for r in rows:
        cdf = np.cumsum(p[r]) / p[r].sum()
        j = int(drawn[r])
        lo = cdf[j - 1] if j > 0 else 0.0
        assert p[r, j] > 0, (r, j)
        assert lo - CDF_TOL <= u[r] < cdf[j] + CDF_TOL, (r, j, lo, u[r], cdf[j])


def _pass_check(c, canvas_np, step, n_max, u, prev_argmax):
    """One dg_eb_step teacher-forced: the oracle head on the device's hn."""
    cfg, oc, B, Tc, T = c.cfg, c.oc, c.B, c.Tc, c.T
    canvas = _dev(canvas_np)
    du = _dev(u.astype(np.float32))
    ent = torch.empty(B, Tc, device="cuda")
    com = torch.empty(B, Tc, dtype=torch.uint8, device="cuda")
    stop = torch.empty(B, dtype=torch.uint8, device="cuda")
    c.dg.dg_eb_step(c.ctx, canvas.data_ptr(), B, step, n_max, du.data_ptr(), ent.data_ptr(),
                    com.data_ptr(), stop.data_ptr())
    c.dg.dg_sync(c.ctx)
    hn = c.fetch("hn", torch.bfloat16, (T, cfg["d_model"]))
    a = c.fetch("tok", torch.int32, (T,))
    drawn = c.fetch("eb_drawn", torch.int32, (T,))
    H = ent.cpu().numpy().ravel()
    temp = eb.eb_temperature(step, n_max)
    lg = _oracle_logits(oc, hn.astype(np.float64))
    oH, oa, op = eb.eb_row_stats(lg, cfg["mask_id"], temp)
    assert np.allclose(H, oH, rtol=H_RTOL, atol=1e-5), np.abs(H - oH).max()
    assert np.array_equal(a, oa)
    # the decisions on the device's own entropies / argmax / drawn tokens
    new = canvas.cpu().numpy()
    drawn = np.where(com.cpu().numpy().ravel() == 1, drawn, a)
    ref_can, ref_com, ref_stop = eb.eb_commit_step(
        canvas_np, H.reshape(B, Tc).astype(np.float64), a.reshape(B, Tc), drawn.reshape(B, Tc),
        prev_argmax, cfg["mask_id"], step == n_max - 1)
    assert np.array_equal(new, ref_can)
    assert np.array_equal(com.cpu().numpy().astype(bool), ref_com)
    assert np.array_equal(stop.cpu().numpy().astype(bool), ref_stop)
    # tokens that came from a draw are valid draws of the oracle's distribution
    drew = [r for r in range(T) if ref_com.ravel()[r] and not ref_stop[r // Tc] and
            step != n_max - 1]
    _check_draws(op, u.ravel(), new.ravel(), drew)
    return new, a.reshape(B, Tc), H.reshape(B, Tc), len(drew)


@pytest.mark.parametrize("name", ["tiny", "ragged"])
def test_eb_block_passes_teacher_forced(name):
    """Four passes of a block: every pass checked against the oracle on the device's
    hidden states; then the same block through dg_eb_denoise_block gives the same
    canvas."""
    cfg = synth.config(name, bf16_weights=True)
    c = Ctx(cfg)
    try:
        B, Tc = c.B, c.Tc
        n_max = 4
        g = np.random.default_rng(9)
        u = g.uniform(size=(n_max, B, Tc))
        canvas = synth.initial_canvas(cfg).numpy()
        prev = None
        n_drawn = 0
        for s in range(n_max):
            before = canvas
            canvas, prev, H, nd = _pass_check(c, canvas, s, n_max, u[s], prev)
            n_drawn += nd
            keep = before != cfg["mask_id"]
            assert np.array_equal(canvas[keep], before[keep])
        assert (canvas != cfg["mask_id"]).all()
        assert n_drawn >= B * (n_max - 1)           # at least one drawn slot per pass
        blk = synth.initial_canvas(cfg).cuda()
        du = _dev(u.astype(np.float32))
        passes = c.dg.dg_eb_denoise_block(c.ctx, blk.data_ptr(), B, n_max, du.data_ptr())
        assert passes == [n_max] * B
        assert np.array_equal(blk.cpu().numpy(), canvas)
    finally:
        c.close()


def test_eb_pass_on_the_stack_sampled_rows():
    """One entropy-bounded pass of the 30-layer stack (vocab 262144): entropies and
    argmax on sampled rows against the oracle head on the device's hn, decisions
    bit-exact on the device's entropies, the drawn token valid."""
    cfg = synth.config("stack")
    c = Ctx(cfg)
    try:
        oc, B, Tc, T = c.oc, c.B, c.Tc, c.T
        g = np.random.default_rng(4)
        u = g.uniform(size=(B, Tc))
        canvas0 = synth.initial_canvas(cfg).numpy()
        canvas = _dev(canvas0)
        du = _dev(u.astype(np.float32))
        ent = torch.empty(B, Tc, device="cuda")
        com = torch.empty(B, Tc, dtype=torch.uint8, device="cuda")
        c.dg.dg_eb_step(c.ctx, canvas.data_ptr(), B, 0, 48, du.data_ptr(), ent.data_ptr(),
                        com.data_ptr(), None)
        c.dg.dg_sync(c.ctx)
        hn = c.fetch("hn", torch.bfloat16, (T, cfg["d_model"]))
        a = c.fetch("tok", torch.int32, (T,))
        H = ent.cpu().numpy().ravel()
        new = canvas.cpu().numpy()
        committed = np.nonzero(com.cpu().numpy().ravel())[0]
        rows = np.unique(np.concatenate([[0, 100, 255], committed]))
        lg = _oracle_logits(oc, hn[rows].astype(np.float64))
        oH, oa, op = eb.eb_row_stats(lg, cfg["mask_id"], eb.eb_temperature(0, 48))
        assert np.allclose(H[rows], oH, rtol=H_RTOL, atol=1e-5)
        assert np.array_equal(a[rows], oa)
        drawn = np.where(com.cpu().numpy().ravel() == 1, new.ravel(), a)
        ref_can, ref_com, _ = eb.eb_commit_step(canvas0, H.reshape(B, Tc).astype(np.float64),
                                                a.reshape(B, Tc), drawn.reshape(B, Tc), None,
                                                cfg["mask_id"], False)
        assert np.array_equal(new, ref_can)
        assert np.array_equal(com.cpu().numpy().astype(bool), ref_com)
        where = {int(r): k for k, r in enumerate(rows)}
        _check_draws(op, np.array([u.ravel()[r] for r in rows]),
                     np.array([new.ravel()[r] for r in rows]), [where[int(r)] for r in committed])
        print("stack eb pass: committed", committed.tolist(), "entropy range",
              float(H.min()), float(H.max()))
    finally:
        c.close()
