"""dg_router_topk_static (the router grouping with its scratch in the library's
own device data, no allocation) against dg_router_topk of a context.

Kept in a file collected last, so that it also runs after every other GPU test
of the session; it passes alone in a fresh process as well.
"""

import numpy as np
import pytest
import torch

import synth
from oracle import model as om
from gpu_helpers import Ctx

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _library():
    from libbuild import build_library
    build_library()


def _logits(T, E, seed):
    g = np.random.default_rng(seed)
    x = g.standard_normal((T, E)).astype(np.float32)
    x[0, [3, 5, 9, 11, 12]] = 2.5                  # ties for the top slots
    x[1, :] = 0.25                                  # all equal
    x[2, [0, E - 1]] = 9.0
    return x


def _outputs(T, E, k):
    return (torch.empty(T, k, dtype=torch.int32, device="cuda"),
            torch.empty(T, k, device="cuda"),
            torch.empty(E + 1, dtype=torch.int32, device="cuda"),
            torch.empty(T * k, dtype=torch.int32, device="cuda"))


@pytest.mark.parametrize("experts,top_k,batch", [(16, 4, 2), (128, 8, 8)])
def test_static_router_matches_context_router_twice(experts, top_k, batch):
    cfg = synth.config("ragged", n_experts=experts, top_k=top_k, batch=batch)
    c = Ctx(cfg, with_prompt=False)
    try:
        T, E, k = c.T, experts, top_k
        # two calls in a row on fresh logits, the second on fewer rows, so that
        # scratch left by the first call would show in the second
        for call, rows in enumerate((T, T - 37)):
            logits = _logits(rows, E, 100 + call)
            dl = torch.from_numpy(logits).cuda()
            ref = _outputs(rows, E, k)
            got = _outputs(rows, E, k)
            c.dg.dg_router_topk(c.ctx, dl.data_ptr(), rows, *(t.data_ptr() for t in ref))
            c.dg.dg_router_topk_static(dl.data_ptr(), rows, E, k, *(t.data_ptr() for t in got),
                                       stream=c.stream)
            torch.cuda.synchronize()
            r_idx, r_w, r_off, r_perm = (t.cpu().numpy() for t in ref)
            g_idx, g_w, g_off, g_perm = (t.cpu().numpy() for t in got)
            assert np.array_equal(g_idx, r_idx), call
            assert np.array_equal(g_off, r_off), call
            assert np.array_equal(g_perm, r_perm), call
            assert np.allclose(g_w, r_w, rtol=2e-6, atol=1e-7), call
            # and the definition the two share
            o_idx, _ = om.router_topk(logits, k)
            o_off, o_perm = om.router_permutation(o_idx, E)
            assert np.array_equal(g_idx, o_idx) and np.array_equal(g_off, o_off)
            assert np.array_equal(g_perm, o_perm)
    finally:
        c.close()


def test_static_router_rejects_sizes_over_its_limits():
    import canvas_denoising_step_b200 as dg
    x = torch.zeros(4096 * 8, device="cuda")
    o = torch.zeros(4096 * 8 * 4, dtype=torch.int32, device="cuda")
    p = o.data_ptr()
    for rows, E, k in ((2049, 128, 8), (0, 128, 8), (16, 260, 8), (16, 130, 8), (16, 128, 9),
                       (16, 4, 5)):
        assert dg.raw_call("dg_router_topk_static", x.data_ptr(), rows, E, k, p, p, p, p,
                           None) == dg.DG_ERR_INVALID_ARG, (rows, E, k)
    assert dg.raw_call("dg_router_topk_static", x.data_ptr() + 4, 16, 128, 8, p, p, p, p,
                       None) == dg.DG_ERR_INVALID_ARG
