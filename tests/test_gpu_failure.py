"""Failure detection on the device without a fault: a kernel's wait on an
mbarrier that nothing completes gives up after its limit, reports
DG_ERR_TIMEOUT to the host, and the device stays usable."""

import time

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _library():
    from libbuild import build_library
    build_library()


def test_bounded_wait_times_out_and_the_device_stays_usable():
    import canvas_denoising_step_b200 as dg
    from oracle import model as om
    t0 = time.time()
    assert dg.dg_selftest_bounded_wait(0) == dg.DG_ERR_TIMEOUT
    elapsed = time.time() - t0
    assert 1.5 < elapsed < 30.0, elapsed
    # the same process keeps using the device: a router grouping after the timeout
    T, E, k = 64, 16, 4
    logits = np.random.default_rng(5).standard_normal((T, E)).astype(np.float32)
    dl = torch.from_numpy(logits).cuda()
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, device="cuda")
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    dg.dg_router_topk_static(dl.data_ptr(), T, E, k, idx.data_ptr(), w.data_ptr(),
                             off.data_ptr(), perm.data_ptr())
    torch.cuda.synchronize()
    ref_idx, _ = om.router_topk(logits, k)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
