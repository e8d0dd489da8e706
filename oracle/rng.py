"""Seeded weight generator of the oracle (test infrastructure only).

The weights of the synthetic model are "drawn N(0, 0.02) from a seed".  The
CUDA library draws them on the device; the oracle draws the same numbers on
the host with its own implementation of one counter-based generator, written
here from its published definition:

* SplitMix64 (G. L. Steele, D. Lea, C. H. Flood, "Fast splittable
  pseudorandom number generators", OOPSLA 2014): the state advances by the
  odd constant GAMMA = 0x9E3779B97F4A7C15 and each output is the 64-bit
  finaliser ``mix64`` of the new state.  The i-th output (i = 0, 1, ...) of a
  generator seeded with ``key`` is therefore ``mix64(key + (i + 1) * GAMMA)``,
  which makes element i of a tensor independent of every other element.
* The per-tensor key is ``mix64(seed + tid * 0xD1B54A32D192ED03)`` where
  ``tid`` names the tensor (``64 * (layer + 1) + kind`` for a layer tensor,
  1 for the tied embedding).
* Normal deviates use the Irwin-Hall construction: the four 16-bit fields of
  one output are summed and centred, ``z = sum - 131070`` (an integer whose
  variance is (65536**2 - 1) / 3), and the weight is the single rounded
  float32 product ``float32(z) * float32(std * sqrt(3) / 65536)``.  Integer
  steps plus one correctly rounded multiply make the value bit-identical on
  any IEEE machine.  The deviate is a close, bounded (|x| <= 3.46 std)
  approximation of a normal with exactly the stated variance (up to 1 part in
  4e9).
* bf16 weights are the round-to-nearest-even bf16 of that float32.
"""

from __future__ import annotations

import math

import numpy as np

MASK64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
KEY_MULT = 0xD1B54A32D192ED03
MIX_M1 = 0xBF58476D1CE4E5B9
MIX_M2 = 0x94D049BB133111EB

# Logical tensors of one decoder layer, by kind index inside the layer's id block.
TENSOR_KIND = {
    "wq": 0,   # [Hq*dh, d]     query projection
    "wk": 1,   # [Hkv*dh, d]    key projection
    "wv": 2,   # [Hkv*dh, d]    value projection
    "wo": 3,   # [d, Hq*dh]     output projection
    "wr": 4,   # [E, d]         router
    "wg": 5,   # [E, F, d]      expert gate
    "wu": 6,   # [E, F, d]      expert up
    "wd": 7,   # [E, d, F]      expert down
    "sg": 8,   # [F, d]         shared-expert gate
    "su": 9,   # [F, d]         shared-expert up
    "sd": 10,  # [d, F]         shared-expert down
}
EMBED_TID = 1


def layer_tid(layer: int, kind: str) -> int:
    return 64 * (layer + 1) + TENSOR_KIND[kind]


def splitmix64_mix(z: int) -> int:
    """SplitMix64 output finaliser on a Python int (mod 2**64)."""
    z &= MASK64
    z = ((z ^ (z >> 30)) * MIX_M1) & MASK64
    z = ((z ^ (z >> 27)) * MIX_M2) & MASK64
    return z ^ (z >> 31)


def splitmix64_stream_key(seed: int, tid: int) -> int:
    return splitmix64_mix((seed + tid * KEY_MULT) & MASK64)


def _mix_np(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * np.uint64(MIX_M1)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(MIX_M2)
    return z ^ (z >> np.uint64(31))


def splitmix64_outputs(key: int, start: int, count: int) -> np.ndarray:
    """Outputs start .. start+count-1 of SplitMix64 seeded with ``key``."""
    i = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(key) + i * np.uint64(GAMMA)
        return _mix_np(z)


def irwin_hall_normal_f32(u: np.ndarray, std: float) -> np.ndarray:
    """float32 deviates of standard deviation ``std`` from 64-bit outputs."""
    m = np.uint64(0xFFFF)
    s = (u & m) + ((u >> np.uint64(16)) & m) + ((u >> np.uint64(32)) & m) + (u >> np.uint64(48))
    z = s.astype(np.int64) - 131070
    scale = np.float32(std * math.sqrt(3.0) / 65536.0)
    return z.astype(np.float32) * scale


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); returned as float32."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) & np.uint64(0xFFFF0000)
    return b.astype(np.uint32).view(np.float32)


def weight_tensor_numpy(seed: int, tid: int, shape, std: float, bf16: bool,
                        start: int = 0, chunk: int = 1 << 22) -> np.ndarray:
    """The logical tensor ``tid`` (row-major ``shape``) as float32 values.

    ``start`` offsets the element counter, so a slice of a larger logical
    tensor (one expert of a stacked expert tensor, a block of vocabulary rows)
    can be drawn alone: element (i0, ..., ik) of the full tensor is output
    ``start + flat_index`` of the tensor's stream.
    """
    n = int(np.prod(shape))
    key = splitmix64_stream_key(seed, tid)
    out = np.empty(n, dtype=np.float32)
    for c0 in range(0, n, chunk):
        c1 = min(n, c0 + chunk)
        out[c0:c1] = irwin_hall_normal_f32(splitmix64_outputs(key, start + c0, c1 - c0), std)
    if bf16:
        out = round_to_bf16(out)
    return out.reshape(shape)


_C_GEN = None


def _c_generator():
    """The C restatement of the same generator (oracle/csrc/weightgen.c), or None."""
    global _C_GEN
    if _C_GEN is None:
        import ctypes
        try:
            from .build_c import build
            lib = ctypes.CDLL(build())
            f = lib.oracle_weight_normal
            f.restype = None
            f.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64, ctypes.c_float,
                          ctypes.c_int, ctypes.c_void_p]
            _C_GEN = f
        except Exception:  # no compiler: the numpy path is used
            _C_GEN = False
    return _C_GEN or None


def weight_tensor(seed: int, tid: int, shape, std: float, bf16: bool, start: int = 0) -> np.ndarray:
    """As ``weight_tensor_numpy``; drawn by the C restatement when it is available
    (the two are tested bit-identical)."""
    f = _c_generator()
    if f is None:
        return weight_tensor_numpy(seed, tid, shape, std, bf16, start)
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float32)
    scale = np.float32(std * math.sqrt(3.0) / 65536.0)
    f(splitmix64_stream_key(seed, tid), start, n, float(scale), int(bf16), out.ctypes.data)
    return out.reshape(shape)
