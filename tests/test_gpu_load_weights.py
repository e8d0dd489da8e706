"""dg_load_weights copies a caller's weight tensor into the library's layout:
checked bit for bit by reading the fused q/k/v, the interleaved gate/up and
the grouped down weights back (no GPU kernel is involved, only copies)."""

import numpy as np
import pytest
import torch

import synth
from gpu_helpers import Ctx

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _library():
    from libbuild import build_library
    build_library()


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def test_loaded_tensors_land_in_the_library_layout():
    cfg = synth.config("ragged")
    c = Ctx(cfg, with_prompt=False)
    try:
        dg = c.dg
        d, F, E = cfg["d_model"], cfg["d_ff"], cfg["n_experts"]
        Hq, Hkv, dh = cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"]
        l = 1
        g = torch.Generator().manual_seed(11)
        def rnd(*shape):
            return torch.randn(*shape, generator=g).to(torch.bfloat16)
        src = {"wq": rnd(Hq * dh, d), "wk": rnd(Hkv * dh, d), "wv": rnd(Hkv * dh, d),
               "wg": rnd(E, F, d), "wu": rnd(E, F, d), "sg": rnd(F, d), "su": rnd(F, d),
               "wd": rnd(E, d, F), "sd": rnd(d, F)}
        for name, t in src.items():
            # device sources, except one host source (the copies accept either)
            s = t if name == "sg" else t.cuda()
            dg.dg_load_weights(c.ctx, f"{name}:{l}", s.data_ptr(), s.numel() * 2)
        torch.cuda.synchronize()
        qkv = c.fetch_bits(f"wqkv:{l}").reshape((Hq + 2 * Hkv) * dh, d)
        assert np.array_equal(qkv[:Hq * dh], _bits(src["wq"]))
        assert np.array_equal(qkv[Hq * dh:(Hq + Hkv) * dh], _bits(src["wk"]))
        assert np.array_equal(qkv[(Hq + Hkv) * dh:], _bits(src["wv"]))
        gu = c.fetch_bits(f"wgu:{l}").reshape(E + 1, 2 * F, d)
        assert np.array_equal(gu[0, 0::2], _bits(src["sg"]))
        assert np.array_equal(gu[0, 1::2], _bits(src["su"]))
        assert np.array_equal(gu[1:, 0::2], _bits(src["wg"]))
        assert np.array_equal(gu[1:, 1::2], _bits(src["wu"]))
        dn = c.fetch_bits(f"wd:{l}").reshape(E + 1, d, F)
        assert np.array_equal(dn[0], _bits(src["sd"]))
        assert np.array_equal(dn[1:], _bits(src["wd"]))
        # a wrong size or name is rejected and changes nothing
        before = c.fetch_bits(f"wgu:{l}")
        bad = src["wg"].cuda()
        with pytest.raises(dg.DgError):
            dg.dg_load_weights(c.ctx, f"wg:{l}", bad.data_ptr(), bad.numel() * 2 - 2)
        with pytest.raises(dg.DgError):
            dg.dg_load_weights(c.ctx, f"wz:{l}", bad.data_ptr(), bad.numel() * 2)
        with pytest.raises(dg.DgError):
            dg.dg_load_weights(c.ctx, f"wg:{cfg['n_layers']}", bad.data_ptr(), bad.numel() * 2)
        assert np.array_equal(c.fetch_bits(f"wgu:{l}"), before)
    finally:
        c.close()
