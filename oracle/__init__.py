"""CPU oracle for the DiffusionGemma-style canvas denoising step.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import or run anything in this package.
The product path (``canvas_denoising_step_b200`` and its CUDA library) never
imports it and shares no code with it.

The oracle is a plain, slow, obviously-correct restatement of the method in
numpy float64.  Each function cites the passage of the pages it follows:

* "Hands-On with Diffusion Gemma: Another Gemma with a Diffusion Mechanism"
  (dev.to), sections "How Is This Different from Previous Models?" and
  "Detailed Specs";
* "DiffusionGemma: The Diffusion Era Begins with 4x Faster Text Generation"
  (efeozkan.com.tr), sections "What is Diffusion ..." and
  "DiffusionGemma's Technical Architecture";
* "DiffusionGemma: Google's Experimental Diffusion LLM" (gemma4all.com),
  section "How Text Diffusion Actually Works".

Where those pages are silent the reading taken is stated at the function.
``eb_sampler`` holds the entropy-bounded denoising rule and ``encoder`` the
causal encoder (prompt prefill, context building) with the block-autoregressive
outer loop (rows of the build after the step itself; their readings are stated
in those modules).
Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(brute force, closed forms, identities and invariants); the end-to-end values
of a whole step are pinned only through those parts, because the pages print
no worked example.
"""

from .rng import (  # noqa: F401
    splitmix64_mix,
    splitmix64_stream_key,
    splitmix64_outputs,
    irwin_hall_normal_f32,
    round_to_bf16,
    weight_tensor,
    TENSOR_KIND,
)
from .model import (  # noqa: F401
    OracleConfig,
    LayerWeights,
    layer_weights,
    rmsnorm,
    rope_rotate,
    rope_pairs_rotated,
    is_global_layer,
    attention,
    attention_split_kv,
    router_topk,
    router_permutation,
    silu,
    expert_mlp,
    moe_ffn,
    layer_forward,
    head_reduce,
    logit_stats,
    embedding_rows,
    embedding_block,
    commit,
    commit_count,
    canvas_step,
    denoise_block,
)
