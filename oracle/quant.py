"""Low-precision expert weights (test infrastructure only; nothing on the product
path imports this module).

"DiffusionGemma: The Diffusion Era Begins with 4x Faster Text Generation",
Comparison with Other Models and Approaches, names low-precision (NVFP4) kernels
for the model on Hopper and Blackwell, which cut the bytes of the expert weights
that dominate a pass.  The reading taken here: FP8 E4M3 expert weights with one fp32
scale per output row (per channel), activations kept in bf16.  For a weight row
w (the bf16 values of the seeded generator, read as float32):

    s   = float32(max_k |w_k|) / float32(448)          (float32 division, RN)
    q_k = e4m3(float32(w_k) / s)                       (float32 division, then
                                                        round to nearest even E4M3)
    w'_k = q_k * s                                     (the weight the layer uses)

448 is the largest finite E4M3 value, so |w_k / s| <= 448 and no code saturates.
E4M3 (the OCP "e4m3fn" format): 1 sign bit, 4 exponent bits (bias 7), 3 mantissa
bits; exponent field 0 holds the subnormals m * 2^-9; S.1111.111 is NaN (never
produced here).  A row of zeros gets s = 0 and q = 0.
"""

from __future__ import annotations

import numpy as np
import torch

E4M3_MAX = 448.0


def e4m3_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest E4M3 value (ties to even), as float32."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).to(torch.float32).numpy()


def e4m3_rowwise(w: np.ndarray):
    """Quantise each row of w (float32 values) as the module docstring states.
    Returns (q float32 [rows, cols] holding E4M3 values, s float32 [rows])."""
    w = np.asarray(w, dtype=np.float32)
    amax = np.max(np.abs(w), axis=-1).astype(np.float32)
    s = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    safe = np.where(s > 0, s, np.float32(1.0)).astype(np.float32)
    q = e4m3_round((w / safe[..., None]).astype(np.float32))
    q = np.where(s[..., None] > 0, q, np.float32(0.0)).astype(np.float32)
    return q, s


def dequantized(w: np.ndarray) -> np.ndarray:
    """The weights the low-precision layer computes with: q * s per row, float64."""
    q, s = e4m3_rowwise(w)
    return q.astype(np.float64) * s.astype(np.float64)[..., None]
