"""Python binding of libdg, the B200 canvas denoising step library.

Argument marshalling only: every function here forwards to the C function of
the same name in ``libdg.so`` (declared in ``include/dg.h``).  Pointers are
plain integers (``tensor.data_ptr()`` for torch tensors); torch is used by
callers only for device memory and streams.  Importing fails loudly when the
library has not been built (``python canvas_denoising_step_b200/build.py``).
"""

from __future__ import annotations

import ctypes
import os
from ctypes import (POINTER, c_char_p, c_double, c_float, c_int, c_int32, c_size_t, c_uint8,
                    c_uint64, c_void_p)

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdg.so")

DG_OK = 0
DG_ERR_INVALID_ARG = -1
DG_ERR_BAD_STATE = -2
DG_ERR_OOM = -3
DG_ERR_CUDA = -4
DG_ERR_TIMEOUT = -5
DG_ERR_DEVICE_FAULT = -6
DG_ERR_UNSUPPORTED = -7
DG_DTYPE_BF16 = 0
DG_DTYPE_FP8_E4M3 = 1


class DgConfig(ctypes.Structure):
    """Mirror of ``dg_config`` in include/dg.h (field order and types must match)."""

    _fields_ = [
        ("n_layers", c_int), ("d_model", c_int), ("n_q_heads", c_int), ("n_kv_heads", c_int),
        ("head_dim", c_int),
        ("n_experts", c_int), ("top_k", c_int), ("n_shared", c_int), ("d_ff", c_int),
        ("vocab", c_int), ("canvas_len", c_int), ("window", c_int), ("global_every", c_int),
        ("mask_id", c_int), ("max_batch", c_int), ("max_prompt", c_int),
        ("rms_eps", c_float), ("rope_theta", c_float), ("prope_fraction", c_float),
        ("rope_enabled", c_int),
        ("weight_std", c_double),
        ("alloc_limit_bytes", c_size_t),
        ("expert_dtype", c_int),
        ("max_context", c_int),
    ]


class DgError(RuntimeError):
    def __init__(self, code: int, func: str, msg: str):
        super().__init__(f"{func} failed ({code}): {msg}")
        self.code = code


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python canvas_denoising_step_b200/build.py` (nvcc, sm_100a)")

_lib = ctypes.CDLL(LIB_PATH)

_SIGS = {
    "dg_create": (c_int, [POINTER(DgConfig), c_void_p, POINTER(c_void_p)]),
    "dg_init_weights": (c_int, [c_void_p, c_uint64]),
    "dg_load_weights": (c_int, [c_void_p, c_char_p, c_void_p, c_size_t]),
    "dg_set_prompt_kv": (c_int, [c_void_p, c_int, c_void_p, c_void_p, c_int, c_int]),
    "dg_set_router_bias": (c_int, [c_void_p, c_void_p]),
    "dg_canvas_step": (c_int, [c_void_p, c_void_p, c_int, c_int, c_void_p, c_void_p]),
    "dg_canvas_step_host": (c_int, [c_void_p, c_void_p, c_int, c_int, c_void_p, c_void_p]),
    "dg_denoise_block": (c_int, [c_void_p, c_void_p, c_int, c_int]),
    "dg_encode": (c_int, [c_void_p, c_void_p, c_int, c_int]),
    "dg_reset_context": (c_int, [c_void_p]),
    "dg_context_length": (c_int, [c_void_p, POINTER(c_int)]),
    "dg_context_kv": (c_int, [c_void_p, c_int, c_void_p, c_void_p]),
    "dg_generate": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_void_p]),
    "dg_eb_step": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p,
                           c_void_p]),
    "dg_eb_denoise_block": (c_int, [c_void_p, c_void_p, c_int, c_int, c_void_p, c_void_p]),
    "dg_eb_commit": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int,
                             c_int, c_void_p, c_void_p]),
    "dg_layer_forward": (c_int, [c_void_p, c_int, c_void_p, c_void_p, c_int]),
    "dg_router_topk": (c_int, [c_void_p, c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p]),
    "dg_router_topk_static": (c_int, [c_void_p, c_int, c_int, c_int, c_void_p, c_void_p,
                                      c_void_p, c_void_p, c_void_p]),
    "dg_selftest_bounded_wait": (c_int, [c_void_p]),
    "dg_commit": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_void_p, c_void_p]),
    "dg_debug_tensor": (c_int, [c_void_p, c_char_p, c_void_p, c_size_t, POINTER(c_size_t)]),
    "dg_profile_enable": (c_int, [c_void_p, c_int]),
    "dg_profile_read": (c_int, [c_void_p, c_char_p, POINTER(c_double), POINTER(c_int)]),
    "dg_kernel_name": (c_char_p, [c_int]),
    "dg_sync": (c_int, [c_void_p]),
    "dg_last_error": (c_char_p, [c_void_p]),
    "dg_device_bytes": (c_size_t, [c_void_p]),
    "dg_last_launch_count": (c_int, [c_void_p]),
    "dg_destroy": (None, [c_void_p]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype, _f.argtypes = _res, _args


def _check(ctx, code: int, func: str):
    if code != DG_OK:
        msg = _lib.dg_last_error(ctx)
        raise DgError(code, func, msg.decode() if msg else "")


def config_from_dict(d: dict, max_batch: int | None = None, max_prompt: int | None = None,
                     alloc_limit_bytes: int = 0, max_context: int = 0) -> DgConfig:
    """A DgConfig from a workload description (the keys of synth.CONFIGS)."""
    return DgConfig(
        n_layers=d["n_layers"], d_model=d["d_model"], n_q_heads=d["n_q_heads"],
        n_kv_heads=d["n_kv_heads"], head_dim=d["head_dim"], n_experts=d["n_experts"],
        top_k=d["top_k"], n_shared=d["n_shared"], d_ff=d["d_ff"], vocab=d["vocab"],
        canvas_len=d["canvas_len"], window=d["window"], global_every=d["global_every"],
        mask_id=d["mask_id"], max_batch=max_batch or d["batch"],
        max_prompt=max_prompt or d["prompt_len"], rms_eps=d["rms_eps"],
        rope_theta=d["rope_theta"], prope_fraction=d["prope_fraction"],
        rope_enabled=int(d["rope_enabled"]), weight_std=d["weight_std"],
        alloc_limit_bytes=alloc_limit_bytes,
        expert_dtype=DG_DTYPE_FP8_E4M3 if d.get("expert_fp8") else DG_DTYPE_BF16,
        max_context=max_context)


# --------------------------------------------------------------------------- C names

def dg_create(cfg: DgConfig, stream: int = 0) -> int:
    out = c_void_p()
    _check(None, _lib.dg_create(ctypes.byref(cfg), c_void_p(stream), ctypes.byref(out)), "dg_create")
    return out.value


def dg_init_weights(ctx: int, seed: int) -> None:
    _check(ctx, _lib.dg_init_weights(ctx, seed), "dg_init_weights")


def dg_load_weights(ctx: int, name: str, src: int, nbytes: int) -> None:
    _check(ctx, _lib.dg_load_weights(ctx, name.encode(), src, nbytes), "dg_load_weights")


def dg_set_prompt_kv(ctx: int, layer: int, k: int, v: int, batch: int, n_prompt: int) -> None:
    _check(ctx, _lib.dg_set_prompt_kv(ctx, layer, k, v, batch, n_prompt), "dg_set_prompt_kv")


def dg_set_router_bias(ctx: int, bias: int | None) -> None:
    _check(ctx, _lib.dg_set_router_bias(ctx, bias), "dg_set_router_bias")


def dg_canvas_step(ctx: int, canvas: int, batch: int, steps_left: int, conf_out: int | None = None,
                   committed_out: int | None = None) -> None:
    _check(ctx, _lib.dg_canvas_step(ctx, canvas, batch, steps_left, conf_out, committed_out),
           "dg_canvas_step")


def dg_canvas_step_host(ctx: int, canvas_host: int, batch: int, steps_left: int,
                        conf_host: int | None = None, committed_host: int | None = None) -> None:
    _check(ctx, _lib.dg_canvas_step_host(ctx, canvas_host, batch, steps_left, conf_host,
                                         committed_host), "dg_canvas_step_host")


def dg_denoise_block(ctx: int, canvas: int, batch: int, n_steps: int) -> None:
    _check(ctx, _lib.dg_denoise_block(ctx, canvas, batch, n_steps), "dg_denoise_block")


def dg_encode(ctx: int, tokens: int, batch: int, n: int) -> None:
    _check(ctx, _lib.dg_encode(ctx, tokens, batch, n), "dg_encode")


def dg_reset_context(ctx: int) -> None:
    _check(ctx, _lib.dg_reset_context(ctx), "dg_reset_context")


def dg_context_length(ctx: int) -> int:
    n = c_int()
    _check(ctx, _lib.dg_context_length(ctx, ctypes.byref(n)), "dg_context_length")
    return n.value


def dg_context_kv(ctx: int, layer: int, k_out: int, v_out: int) -> None:
    _check(ctx, _lib.dg_context_kv(ctx, layer, k_out, v_out), "dg_context_kv")


def dg_generate(ctx: int, prompt: int, batch: int, n_prompt: int, n_blocks: int, n_steps: int,
                out: int) -> None:
    _check(ctx, _lib.dg_generate(ctx, prompt, batch, n_prompt, n_blocks, n_steps, out),
           "dg_generate")


def dg_eb_step(ctx: int, canvas: int, batch: int, step: int, n_max: int, u: int,
               entropy_out: int | None = None, committed_out: int | None = None,
               stopped_out: int | None = None) -> None:
    _check(ctx, _lib.dg_eb_step(ctx, canvas, batch, step, n_max, u, entropy_out, committed_out,
                                stopped_out), "dg_eb_step")


def dg_eb_denoise_block(ctx: int, canvas: int, batch: int, n_max: int, u: int) -> list[int]:
    """Runs the block; returns the passes each canvas took part in."""
    passes = (c_int * batch)()
    _check(ctx, _lib.dg_eb_denoise_block(ctx, canvas, batch, n_max, u, passes),
           "dg_eb_denoise_block")
    return list(passes)


def dg_eb_commit(ctx: int, entropy: int, argmax: int, drawn: int, prev_argmax: int | None,
                 canvas: int, batch: int, last: bool, committed_out: int | None = None,
                 stopped_out: int | None = None) -> None:
    _check(ctx, _lib.dg_eb_commit(ctx, entropy, argmax, drawn, prev_argmax, canvas, batch,
                                  int(last), committed_out, stopped_out), "dg_eb_commit")


def dg_layer_forward(ctx: int, layer: int, x_in: int, x_out: int, n_rows: int) -> None:
    _check(ctx, _lib.dg_layer_forward(ctx, layer, x_in, x_out, n_rows), "dg_layer_forward")


def dg_router_topk(ctx: int, logits: int, n_rows: int, idx: int, w: int, offsets: int,
                   perm: int) -> None:
    _check(ctx, _lib.dg_router_topk(ctx, logits, n_rows, idx, w, offsets, perm), "dg_router_topk")


def dg_router_topk_static(logits: int, n_rows: int, n_experts: int, top_k: int, idx: int, w: int,
                          offsets: int, perm: int, stream: int = 0) -> None:
    """Context-free router grouping that allocates no device memory (see dg.h)."""
    code = _lib.dg_router_topk_static(logits, n_rows, n_experts, top_k, idx, w, offsets, perm,
                                      stream)
    if code != DG_OK:
        raise DgError(code, "dg_router_topk_static", "rejected or failed")


def dg_selftest_bounded_wait(stream: int = 0) -> int:
    """Runs the bounded-wait self-test; returns its status (DG_ERR_TIMEOUT expected)."""
    return _lib.dg_selftest_bounded_wait(stream)


def dg_commit(ctx: int, conf: int, canvas: int, batch: int, steps_left: int, cand_tok: int,
              committed_out: int | None = None) -> None:
    _check(ctx, _lib.dg_commit(ctx, conf, canvas, batch, steps_left, cand_tok, committed_out),
           "dg_commit")


def dg_debug_tensor(ctx: int, name: str, dst: int | None, nbytes: int) -> int:
    need = c_size_t(0)
    _check(ctx, _lib.dg_debug_tensor(ctx, name.encode(), dst, nbytes, ctypes.byref(need)),
           "dg_debug_tensor")
    return need.value


def dg_profile_enable(ctx: int, on: bool) -> None:
    _check(ctx, _lib.dg_profile_enable(ctx, int(on)), "dg_profile_enable")


def dg_profile_read(ctx: int, kernel: str) -> tuple[float, int]:
    """(total device ms, launches) recorded for one kernel kind."""
    t, n = c_double(0.0), c_int(0)
    _check(ctx, _lib.dg_profile_read(ctx, kernel.encode(), ctypes.byref(t), ctypes.byref(n)),
           "dg_profile_read")
    return t.value, n.value


def dg_kernel_name(i: int) -> str | None:
    n = _lib.dg_kernel_name(i)
    return n.decode() if n else None


def dg_sync(ctx: int) -> None:
    _check(ctx, _lib.dg_sync(ctx), "dg_sync")


def dg_last_error(ctx: int | None) -> str:
    m = _lib.dg_last_error(ctx)
    return m.decode() if m else ""


def dg_device_bytes(ctx: int) -> int:
    return _lib.dg_device_bytes(ctx)


def dg_last_launch_count(ctx: int) -> int:
    return _lib.dg_last_launch_count(ctx)


def dg_destroy(ctx: int | None) -> None:
    _lib.dg_destroy(ctx)


def raw_call(name: str, *args) -> int:
    """Calls a C entry point and returns its raw status (for argument-check tests)."""
    return getattr(_lib, name)(*args)


library = _lib
