"""The attention's in-cluster merge against the separate merge kernel.

By default the attention writes its key ranges' partials to global memory and
the merge kernel (attn_merge.cu) combines them.  With DG_ATTN_CLUSTER_MERGE=1
the key ranges of one query tile run as one thread-block cluster and merge in
shared memory (attention_tc.cu).  Both take the same fp32 steps in the same
order, so the attention output must agree bit for bit, on cluster sizes 1 to 6,
ragged query tiles, local and global layers.  The default route's parity with
the oracle is what the layer, pass and full-size tests check."""

import numpy as np
import pytest
import torch

import synth
from tests.gpu_helpers import Ctx

pytestmark = pytest.mark.gpu

CASES = [
    ("tiny", {}, 0), ("tiny", {}, 1),                     # two key ranges
    ("ragged", {}, 0), ("ragged", {}, 1),                 # three and six; 96 of 128 query rows
    ("stack", dict(vocab=1024, n_layers=6), 0),           # four ranges over a 1024-key window
    ("stack", dict(vocab=1024, n_layers=6), 5),           # four ranges over 4096 keys
    ("batched", dict(vocab=1024, n_layers=1), 0),         # one range: a cluster of one CTA
]


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from libbuild import build_library as build
    build()
    torch.cuda.set_device(0)


def _attn_o(cfg, layer, cluster, monkeypatch):
    if cluster:
        monkeypatch.setenv("DG_ATTN_CLUSTER_MERGE", "1")
    else:
        monkeypatch.delenv("DG_ATTN_CLUSTER_MERGE", raising=False)
    c = Ctx(cfg)
    try:
        x = synth.hidden_states(cfg).cuda()
        out = torch.empty_like(x)
        c.dg.dg_profile_enable(c.ctx, 1)
        c.dg.dg_layer_forward(c.ctx, layer, x.data_ptr(), out.data_ptr(), c.T)
        _, merges = c.dg.dg_profile_read(c.ctx, "attn_merge")
        _, attns = c.dg.dg_profile_read(c.ctx, "attention")
        c.dg.dg_profile_enable(c.ctx, 0)
        bits = c.fetch_bits("attn_o")
    finally:
        c.close()
    return bits, merges, attns


@pytest.mark.parametrize("name,over,layer", CASES)
def test_cluster_merge_equals_merge_kernel(name, over, layer, monkeypatch):
    cfg = synth.config(name, **over)
    fused, m_f, a_f = _attn_o(cfg, layer, True, monkeypatch)
    sep, m_s, a_s = _attn_o(cfg, layer, False, monkeypatch)
    assert a_f == 1 and a_s == 1
    assert m_f == 0, "DG_ATTN_CLUSTER_MERGE=1 launched the merge kernel"
    assert m_s == 1, "the default route did not launch the merge kernel"
    assert fused.shape == sep.shape
    assert not np.all(fused == 0)
    diff = np.flatnonzero(fused != sep)
    assert diff.size == 0, f"{diff.size} of {fused.size} outputs differ, first at {diff[:8]}"
