"""Parity of the two-SM (cta_group::2) GEMM path, which DG_CTA_PAIR=1 switches on
for the q/k/v and o projections and the bf16 expert GEMMs (it is off by
default: it measured slower than the one-SM engine).  The same layer and pass
checks as the default path, on contexts created with the variable set."""

import pytest
import torch

from tests import test_gpu_parity as tp

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _pair_env(monkeypatch):
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from libbuild import build_library as build
    build()
    torch.cuda.set_device(0)
    monkeypatch.setenv("DG_CTA_PAIR", "1")


@pytest.mark.parametrize("name,layer", [("tiny", 1), ("ragged", 0), ("ragged", 1)])
def test_layer_parity_two_sm(name, layer):
    tp._layer_check(name, layer)


@pytest.mark.parametrize("name", ["tiny", "ragged"])
def test_canvas_step_two_sm(name):
    tp.canvas_step_check(tp.gpu_cfg(name))
