"""C-ABI checks that need no GPU: the library loads, exports every function
include/dg.h declares, its config struct matches the binding's mirror, and
argument / no-device errors come back as status codes."""

import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dg.h")


@pytest.fixture(scope="module")
def dg():
    from libbuild import build_library as build
    build()
    import canvas_denoising_step_b200 as m
    return m


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dg_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(dg):
    names = declared_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(dg.library, n), f"libdg.so does not export {n}"
    out = subprocess.run(["nm", "-D", "--defined-only", dg.LIB_PATH], capture_output=True,
                         text=True).stdout
    for n in names:
        assert re.search(rf"\bT {n}\b", out), f"{n} is not a defined text symbol"


def test_config_struct_layout_matches_header(dg, tmp_path):
    fields = [f for f, _ in dg.DgConfig._fields_]
    src = tmp_path / "layout.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "dg.h"\nint main(void){\n'
                   '  printf("%zu\\n", sizeof(dg_config));\n' +
                   "".join(f'  printf("%zu\\n", offsetof(dg_config, {f}));\n' for f in fields) +
                   "  return 0;\n}\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                   check=True)
    vals = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True,
                                           check=True).stdout.split()]
    assert vals[0] == ctypes.sizeof(dg.DgConfig)
    for f, off in zip(fields, vals[1:]):
        assert getattr(dg.DgConfig, f).offset == off, f


def test_invalid_configs_rejected_before_device_use(dg):
    import synth
    base = synth.config("tiny")
    bad = [dict(d_model=100), dict(head_dim=96), dict(n_q_heads=3), dict(top_k=9),
           dict(canvas_len=300), dict(mask_id=1024), dict(n_shared=2), dict(d_ff=100)]
    for b in bad:
        cfg = dg.config_from_dict(dict(base, **b))
        out = ctypes.c_void_p()
        rc = dg.raw_call("dg_create", ctypes.byref(cfg), None, ctypes.byref(out))
        assert rc == dg.DG_ERR_INVALID_ARG, b
        assert out.value is None
        assert dg.dg_last_error(None) != ""
    cfg = dg.config_from_dict(base, max_context=-1)
    out = ctypes.c_void_p()
    assert dg.raw_call("dg_create", ctypes.byref(cfg), None, ctypes.byref(out)) == \
        dg.DG_ERR_INVALID_ARG


def test_configs_whose_router_grouping_cannot_fit_are_rejected(dg):
    """4096 rows x 256 experts (264 KB) and x 200 experts (206 KB) of grouping state
    exceed the router's 200 KB of shared memory: dg_create refuses them up front;
    4096 rows x 128 experts (133 KB) is accepted by the checks (and then stops at
    the missing device)."""
    import synth
    base = synth.config("tiny", canvas_len=256)
    for E, want_reject in ((256, True), (200, True), (128, False)):
        cfg = dg.config_from_dict(dict(base, n_experts=E), max_batch=16)
        out = ctypes.c_void_p()
        rc = dg.raw_call("dg_create", ctypes.byref(cfg), None, ctypes.byref(out))
        msg = dg.dg_last_error(None)
        if want_reject:
            assert rc == dg.DG_ERR_INVALID_ARG and "router" in msg, (E, rc, msg)
        else:
            assert "router" not in msg, (E, msg)
        assert out.value is None


def test_null_arguments_and_no_device(dg):
    import synth
    cfg = dg.config_from_dict(synth.config("tiny"))
    assert dg.raw_call("dg_create", None, None, None) == dg.DG_ERR_INVALID_ARG
    out = ctypes.c_void_p()
    rc = dg.raw_call("dg_create", ctypes.byref(cfg), None, ctypes.byref(out))
    import torch
    if not torch.cuda.is_available():
        assert rc == dg.DG_ERR_CUDA and out.value is None
        assert "device" in dg.dg_last_error(None)
    else:
        assert rc == dg.DG_OK
        dg.dg_destroy(out.value)
    for name, args in [("dg_init_weights", (None, 0)), ("dg_sync", (None,)),
                       ("dg_canvas_step", (None, None, 1, 1, None, None)),
                       ("dg_denoise_block", (None, None, 1, 1)),
                       ("dg_layer_forward", (None, 0, None, None, 1)),
                       ("dg_set_prompt_kv", (None, 0, None, None, 1, 1)),
                       ("dg_router_topk", (None, None, 1, None, None, None, None)),
                       ("dg_commit", (None, None, None, 1, 1, None, None)),
                       ("dg_encode", (None, None, 1, 1)), ("dg_reset_context", (None,)),
                       ("dg_context_length", (None, None)),
                       ("dg_context_kv", (None, 0, None, None)),
                       ("dg_generate", (None, None, 1, 1, 1, 1, None))]:
        assert dg.raw_call(name, *args) == dg.DG_ERR_INVALID_ARG, name
    dg.dg_destroy(None)
    assert dg.dg_device_bytes(None) == 0


def test_static_router_limits_checked_before_device_use(dg):
    # argument errors are reported before any CUDA call, so no GPU is needed
    p = 0x10000   # 16-byte aligned, never dereferenced
    bad = [(0, 128, 8), (2049, 128, 8), (16, 2, 1), (16, 130, 8), (16, 260, 8), (16, 128, 0),
           (16, 128, 9), (16, 4, 5)]
    for rows, E, k in bad:
        assert dg.raw_call("dg_router_topk_static", p, rows, E, k, p, p, p, p, None) == \
            dg.DG_ERR_INVALID_ARG, (rows, E, k)
    assert dg.raw_call("dg_router_topk_static", p + 4, 16, 128, 8, p, p, p, p, None) == \
        dg.DG_ERR_INVALID_ARG
    assert dg.raw_call("dg_router_topk_static", None, 16, 128, 8, p, p, p, p, None) == \
        dg.DG_ERR_INVALID_ARG


def test_load_weights_needs_a_context(dg):
    assert dg.raw_call("dg_load_weights", None, b"wq:0", 0x10000, 16) == dg.DG_ERR_INVALID_ARG
