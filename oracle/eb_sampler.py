"""Entropy-bounded denoising (the next step after the fixed-step commit), CPU oracle.

TEST INFRASTRUCTURE ONLY (see the package header): nothing on the product path
imports this module.

The pages name the sampler and its settings but not its steps:
"DiffusionGemma: The Diffusion Era Begins with 4x Faster Text Generation"
(efeozkan.com.tr), section "Recommended Inference Settings" -- an entropy-bound
sampler, at most 48 denoising steps, a temperature that decays linearly from
0.8 to 0.4, an entropy bound of 0.1, and an adaptive stop once the average canvas
entropy is below 0.005 and the high-probability tokens have stayed the same for
2 consecutive steps; "DiffusionGemma: Exploring the Paradigm Shift in
Non-Autoregressive Language Modeling" (techsurvey.info), section "Serving in
Production", repeats the 0.005 halting threshold.  The readings taken (E1-E6)
are stated at each function.  Random draws are inputs (uniforms u in [0, 1)).
"""

from __future__ import annotations

import numpy as np

N_MAX_STEPS = 48
T_START, T_END = 0.8, 0.4
ENTROPY_BOUND = 0.1
STOP_ENTROPY = 0.005
STOP_STABLE_STEPS = 2


def eb_temperature(step: int, n_max: int = N_MAX_STEPS, t_start: float = T_START,
                   t_end: float = T_END) -> float:
    """E1: the temperature of step 0 .. n_max-1 falls linearly from t_start to t_end."""
    if not 0 <= step < n_max:
        raise ValueError("step out of range")
    if n_max == 1:
        return t_start
    return t_start + (t_end - t_start) * step / (n_max - 1)


def eb_row_stats(logits: np.ndarray, mask_id: int, temperature: float):
    """E2: per row, the distribution softmax(l / T) over the vocabulary without the
    mask id (as in the fixed-step head), its entropy H = -sum p ln p (nats), and
    the argmax token (lowest index on ties).  Returns (H, argmax, p)."""
    z = np.array(logits, dtype=np.float64, copy=True) / temperature
    z[:, mask_id] = -np.inf
    a = np.argmax(z, axis=1).astype(np.int32)
    z = z - z[np.arange(z.shape[0]), a][:, None]
    e = np.exp(z)
    s = e.sum(axis=1)
    p = e / s[:, None]
    zp = np.where(p > 0, z, 0.0) * p
    H = np.log(s) - zp.sum(axis=1)
    return H, a, p


def eb_sample(p: np.ndarray, u: np.ndarray) -> np.ndarray:
    """E3: token i of each row by inverse CDF: the first vocab index whose
    cumulative probability (in index order) exceeds u_i."""
    c = np.cumsum(p, axis=1)
    tok = np.empty(p.shape[0], dtype=np.int32)
    for r in range(p.shape[0]):
        j = 0
        while j < p.shape[1] - 1 and c[r, j] <= u[r] * c[r, -1]:
            j += 1
        while p[r, j] == 0 and j > 0:   # never land on a zero-probability token
            j -= 1
        tok[r] = j
    return tok


def eb_unmask(canvas: np.ndarray, H: np.ndarray, tok: np.ndarray, mask_id: int,
              bound: float = ENTROPY_BOUND):
    """E4: in each canvas, the masked slots in order of entropy (lowest first, then
    lowest slot) are committed while their summed entropy stays within the bound;
    at least one slot is committed while any is masked.  canvas, tok int [B, Tc];
    H [B, Tc].  Returns (new_canvas, committed bool [B, Tc])."""
    canvas = np.array(canvas, dtype=np.int32, copy=True)
    committed = np.zeros(canvas.shape, dtype=bool)
    for b in range(canvas.shape[0]):
        masked = [i for i in range(canvas.shape[1]) if canvas[b, i] == mask_id]
        order = sorted(masked, key=lambda i: (float(H[b, i]), i))
        total = 0.0
        for n, i in enumerate(order):
            total += float(H[b, i])
            if n > 0 and total > bound:
                break
            canvas[b, i] = tok[b, i]
            committed[b, i] = True
    return canvas, committed


def eb_should_stop(mean_entropy_history, argmax_history, threshold: float = STOP_ENTROPY,
                   stable: int = STOP_STABLE_STEPS) -> bool:
    """E5: stop once the canvas's mean entropy (over all its slots) at the latest step
    is below the threshold and the argmax tokens of every slot agree over the last
    `stable` consecutive steps (the latest `stable` argmax vectors are equal).

    The two pages word the stability test differently: "DiffusionGemma: The
    Diffusion Era Begins with 4x Faster Text Generation", Recommended Inference
    Settings, has the high-probability tokens stay the same for 2 consecutive
    steps; "DiffusionGemma: Exploring the Paradigm Shift in Non-Autoregressive
    Language Modeling", Serving in Production, halts a block once two consecutive
    passes reach consensus.  The reading that fits both: two consecutive passes
    (2 argmax vectors) agree, so a block can stop at the second pass."""
    if len(mean_entropy_history) == 0 or mean_entropy_history[-1] >= threshold:
        return False
    if len(argmax_history) < max(stable, 1):
        return False
    last = [np.asarray(a) for a in argmax_history[-stable:]]
    return all(np.array_equal(last[0], x) for x in last[1:])


def eb_commit_step(canvas: np.ndarray, H: np.ndarray, argmax: np.ndarray, drawn: np.ndarray,
                   prev_argmax, mask_id: int, last: bool, bound: float = ENTROPY_BOUND,
                   threshold: float = STOP_ENTROPY):
    """The decisions of one entropy-bounded pass, per canvas (E4, E5, E6).

    canvas, argmax, drawn int [B, Tc]; H [B, Tc] (the pass's entropies);
    prev_argmax int [B, Tc] or None (the previous pass's argmax tokens).
    E5: a canvas stops when its mean entropy over all slots (summed in slot
    order) is below the threshold and its argmax tokens equal the previous
    pass's.  E6: a canvas that stops, or reaches the last allowed pass,
    commits every still-masked slot with its argmax token; any other canvas
    commits by the entropy bound (E4) with the drawn tokens.
    Returns (new_canvas, committed bool [B, Tc], stopped bool [B])."""
    canvas = np.array(canvas, dtype=np.int32, copy=True)
    B, Tc = canvas.shape
    committed = np.zeros((B, Tc), dtype=bool)
    stopped = np.zeros(B, dtype=bool)
    for b in range(B):
        total = 0.0
        for i in range(Tc):
            total += float(H[b, i])
        hist = [argmax[b]] if prev_argmax is None else [prev_argmax[b], argmax[b]]
        stopped[b] = eb_should_stop([total / Tc], hist, threshold)
        if stopped[b] or last:
            for i in range(Tc):
                if canvas[b, i] == mask_id:
                    canvas[b, i] = argmax[b, i]
                    committed[b, i] = True
        else:
            nb, cb = eb_unmask(canvas[b:b + 1], H[b:b + 1], drawn[b:b + 1], mask_id, bound)
            canvas[b], committed[b] = nb[0], cb[0]
    return canvas, committed, stopped


def eb_denoise_block(cfg, canvas, k_prompt_layers, v_prompt_layers, u_steps,
                     n_max: int = N_MAX_STEPS, weights=None, router_bias=None,
                     history=None):
    """Entropy-bounded denoising of one block of B canvases (E1-E6): pass s runs at
    temperature eb_temperature(s, n_max), draws with the uniforms u_steps[s]
    ([B, Tc]), and commits by eb_commit_step; a canvas that has stopped, or has no
    masked slot left, is frozen while the others go on.  Ends when every canvas is
    frozen or after n_max passes.  Returns (canvas, passes run per canvas)."""
    from . import model as om
    canvas = np.array(canvas, dtype=np.int32, copy=True)
    B, Tc = canvas.shape
    done = np.zeros(B, dtype=bool)
    passes = np.zeros(B, dtype=np.int32)
    prev = None
    for s in range(n_max):
        if done.all():
            break
        T = eb_temperature(s, n_max)
        hn = om.final_hidden(cfg, canvas, k_prompt_layers, v_prompt_layers, router_bias, weights)
        logits = hn @ om.embedding_block(cfg, 0, cfg.vocab).T
        H, a, p = eb_row_stats(logits, cfg.mask_id, T)
        drawn = eb_sample(p, np.asarray(u_steps[s]).reshape(-1))
        H, a, drawn = H.reshape(B, Tc), a.reshape(B, Tc), drawn.reshape(B, Tc)
        new, com, stop = eb_commit_step(canvas, H, a, drawn, prev, cfg.mask_id, s == n_max - 1)
        for b in range(B):
            if done[b]:
                continue
            canvas[b] = new[b]
            passes[b] += 1
            if stop[b] or not (canvas[b] == cfg.mask_id).any():
                done[b] = True
        if history is not None:
            history.append(dict(canvas=canvas.copy(), H=H, argmax=a, drawn=drawn, committed=com,
                                stopped=stop, done=done.copy()))
        prev = a
    return canvas, passes
