"""Parity of the fused router (DG_FUSED_ROUTER=1: the logits GEMM split over a
cluster, summed through distributed shared memory, top-k and grouping in one
kernel; off by default, it measured slower than the two-kernel router).  The same
layer and pass checks as the default path, including the router's bit-exact
grouping and the batched workload's 2048 rows (eight clusters)."""

import pytest
import torch

from tests import test_gpu_parity as tp

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _fused_env(monkeypatch):
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from libbuild import build_library as build
    build()
    torch.cuda.set_device(0)
    monkeypatch.setenv("DG_FUSED_ROUTER", "1")


@pytest.mark.parametrize("name,layer", [("tiny", 0), ("ragged", 0), ("ragged", 1)])
def test_layer_parity_fused_router(name, layer):
    tp._layer_check(name, layer)


@pytest.mark.parametrize("name", ["tiny", "ragged"])
def test_canvas_step_fused_router(name):
    tp.canvas_step_check(tp.gpu_cfg(name))


def test_batched_layer_fused_router():
    from tests import test_gpu_fullsize as tf
    tf.test_batched_zipf_layer()
