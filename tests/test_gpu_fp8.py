"""FP8 E4M3 expert weights (expert_dtype = DG_DTYPE_FP8_E4M3) against the CPU oracle
with the same quantisation (oracle.quant).

Criteria: the device's codes and row scales bit-exact with the oracle's
quantisation of the same bf16 weights; layer outputs within relative L2 1e-2 of
the oracle computing with the dequantised weights; the pass's head and commit as
in the bf16 tests."""

import numpy as np
import pytest
import torch

import synth
from oracle import quant
from oracle import rng as orng
from tests.gpu_helpers import Ctx
from tests.test_gpu_fullsize import _layer_on_big_ctx
from tests.test_gpu_parity import LAYER_TOL, _layer_check, canvas_step_check

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from libbuild import build_library as build
    build()
    torch.cuda.set_device(0)


def _codes_as_values(c, name, shape):
    need = c.dg.dg_debug_tensor(c.ctx, name, None, 0)
    t = torch.empty(need, dtype=torch.uint8, device="cuda")
    c.dg.dg_debug_tensor(c.ctx, name, t.data_ptr(), need)
    return t.cpu().view(torch.float8_e4m3fn).float().numpy().reshape(shape)


@pytest.mark.parametrize("name", ["tiny", "ragged"])
def test_fp8_codes_and_scales_bit_exact(name):
    cfg = synth.config(name, bf16_weights=True, expert_fp8=1)
    c = Ctx(cfg, with_prompt=False)
    try:
        d, F, E = cfg["d_model"], cfg["d_ff"], cfg["n_experts"]
        lt = orng.layer_tid
        for l in range(cfg["n_layers"]):
            q_gu = _codes_as_values(c, f"wgu8:{l}", (E + 1, 2 * F, d))
            s_gu = c.fetch(f"sgu:{l}", torch.float32, (E + 1, 2 * F))
            q_d = _codes_as_values(c, f"wd8:{l}", (E + 1, d, F))
            s_d = c.fetch(f"sd8:{l}", torch.float32, (E + 1, d))

            def draw(kind, shape, start=0):
                return orng.weight_tensor(cfg["seed"], lt(l, kind), shape, cfg["weight_std"], True,
                                          start=start)
            groups = [(draw("sg", (F, d)), draw("su", (F, d)), draw("sd", (d, F)))]
            for e in (0, 1, E - 1):
                groups.append((draw("wg", (F, d), e * F * d), draw("wu", (F, d), e * F * d),
                               draw("wd", (d, F), e * d * F)))
            for gi, (g_w, u_w, d_w) in zip([0, 1, 2, E], groups):
                for rows, phys in ((g_w, slice(0, None, 2)), (u_w, slice(1, None, 2))):
                    q, s = quant.e4m3_rowwise(rows)
                    assert np.array_equal(q_gu[gi, phys], q), (l, gi)
                    assert np.array_equal(s_gu[gi, phys], s), (l, gi)
                q, s = quant.e4m3_rowwise(d_w)
                assert np.array_equal(q_d[gi], q) and np.array_equal(s_d[gi], s), (l, gi)
    finally:
        c.close()


@pytest.mark.parametrize("name,layer", [("tiny", 0), ("tiny", 1), ("ragged", 0), ("ragged", 1)])
def test_fp8_layer_parity(name, layer):
    _layer_check(name, layer, expert_fp8=1)


@pytest.mark.parametrize("name", ["tiny", "ragged"])
def test_fp8_canvas_step(name):
    canvas_step_check(synth.config(name, bf16_weights=True, expert_fp8=1))


def test_fp8_stack_layers():
    """Full-size layers (d_model 2816, 128 experts, width 704): a local and a global layer."""
    cfg = synth.config("stack", n_layers=6, expert_fp8=1)
    c = Ctx(cfg)
    try:
        for layer in (0, 5):
            err, flips, _, _ = _layer_on_big_ctx(c, layer)
            print("fp8 stack layer", layer, "rel-L2", err, "near-tie rows", flips)
            assert err < LAYER_TOL
    finally:
        c.close()
