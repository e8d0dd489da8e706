"""Helpers for the GPU parity tests: contexts on seeded inputs, read-back of
internal tensors through the C ABI, and comparison metrics."""

from __future__ import annotations

import numpy as np
import torch

import synth
from oracle import model as om
from oracle import rng as orng


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


class Ctx:
    """A libdg context with seeded weights and the prompt K/V of every layer."""

    def __init__(self, cfg: dict, max_batch=None, max_prompt=None, with_prompt=True,
                 max_context=0):
        import canvas_denoising_step_b200 as dg
        self.dg, self.cfg = dg, cfg
        self.B, self.Tc, self.P = cfg["batch"], cfg["canvas_len"], cfg["prompt_len"]
        self.T = self.B * self.Tc
        # a dedicated stream (made current for torch too), so passes run from CUDA graphs
        self.torch_stream = torch.cuda.Stream()
        self.prev_stream = torch.cuda.current_stream()
        torch.cuda.set_stream(self.torch_stream)
        self.stream = self.torch_stream.cuda_stream
        self.ctx = dg.dg_create(dg.config_from_dict(cfg, max_batch, max_prompt,
                                                    max_context=max_context), self.stream)
        dg.dg_init_weights(self.ctx, cfg["seed"])
        self.kv_host, self.kv_dev = [], []
        if with_prompt:
            for l in range(cfg["n_layers"]):
                k, v = synth.prompt_kv(cfg, l)
                kd, vd = k.cuda(), v.cuda()
                self.kv_host.append((k, v))
                self.kv_dev.append((kd, vd))
                dg.dg_set_prompt_kv(self.ctx, l, kd.data_ptr(), vd.data_ptr(), self.B, self.P)
        self.oc = om.OracleConfig.from_dict(cfg)

    def kv_np(self, layer: int):
        """Prompt K, V of one layer as float64 numpy [B, Hkv, P, dh]."""
        k, v = self.kv_host[layer]
        return (k.float().numpy().astype(np.float64), v.float().numpy().astype(np.float64))

    def close(self):
        if self.ctx:
            self.dg.dg_destroy(self.ctx)
            self.ctx = None
            torch.cuda.synchronize()
            torch.cuda.set_stream(self.prev_stream)

    def fetch(self, name: str, dtype, shape) -> np.ndarray:
        need = self.dg.dg_debug_tensor(self.ctx, name, None, 0)
        t = torch.empty(need // torch.tensor([], dtype=dtype).element_size(), dtype=dtype,
                        device="cuda")
        self.dg.dg_debug_tensor(self.ctx, name, t.data_ptr(), need)
        arr = t.float().cpu().numpy() if dtype == torch.bfloat16 else t.cpu().numpy()
        return arr.reshape(shape)

    def fetch_bits(self, name: str) -> np.ndarray:
        """A bf16 tensor as raw uint16 bits."""
        need = self.dg.dg_debug_tensor(self.ctx, name, None, 0)
        t = torch.empty(need // 2, dtype=torch.int16, device="cuda")
        self.dg.dg_debug_tensor(self.ctx, name, t.data_ptr(), need)
        return t.cpu().numpy().view(np.uint16)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """uint16 bits of float32 values that are exactly bf16."""
    return (np.ascontiguousarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def oracle_weight_bits(cfg: dict, tid: int, shape, start=0) -> np.ndarray:
    return bf16_bits(orng.weight_tensor(cfg["seed"], tid, shape, cfg["weight_std"], True,
                                        start=start))


ROUTER_TIE_TOL = 2e-2   # logit units; the device's logits differ from the oracle's by ~1e-3


def router_flips(o_logits, o_idx, d_idx, tol=ROUTER_TIE_TOL) -> np.ndarray:
    """Rows whose device top-k set differs from the oracle's own.  Each such row must
    be a near-tie in the oracle's logits: every expert chosen by one side only lies
    within `tol` of the oracle's k-th largest logit (the selection boundary).
    Returns the boolean mask of flipped rows."""
    o_logits = np.asarray(o_logits, dtype=np.float64)
    k = o_idx.shape[1]
    flipped = np.zeros(o_idx.shape[0], dtype=bool)
    for t in range(o_idx.shape[0]):
        a, b = set(int(e) for e in o_idx[t]), set(int(e) for e in d_idx[t])
        if a == b:
            continue
        flipped[t] = True
        boundary = np.sort(o_logits[t])[::-1][k - 1]
        for e in a ^ b:
            assert abs(o_logits[t, e] - boundary) < tol, (t, e, o_logits[t, e], boundary)
    return flipped
