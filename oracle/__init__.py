"""fp64 CPU oracle of the KaLM-Reranker-V1 FBNL scoring path.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may call it.  It shares no code with
the CUDA library (no kernels, headers, helpers or constant tables); the only
thing both sides use is the seeded input generator in ``synthetic/``.

What it computes is the plain definition of each step, in fp64, with values
rounded to bf16 (nearest, ties to even) exactly where the path stores bf16
tensors.  Sources, by page title and section:

* "KaLM-Reranker-V1-Nano - MLX (Apple Silicon)", section "What this is": the
  passage encoder output is chunk-pooled (chunk 4, masked mean per chunk) into
  cached document vectors; the decoder runs one scaled-dot-product attention
  over the concatenation of its self-attention K/V and cross-attention K/V
  computed from those cached vectors; the score is softmax([yes, no])[yes] at
  the decoder's final position.
* "KaLM-Reranker-V1-Large-Q8_0-GGUF" (ModelScope), "Frozen inference contract":
  right padding, masked mean pooling over consecutive groups of 4 tokens,
  score = sigmoid(yes_logit - no_logit).
* "KaLM-Reranker-V1-Small-Q4_K_M-GGUF", "Score a pair": margin = yes - no,
  score = sigmoid(margin), larger margins rank first.
* "KaLM-Reranker-V1-Nano - MLX (Apple Silicon)", "Derivation": rotary
  position parameters and inverse-frequency tables come from the model
  config; the rotation itself (pairing element i with i + D/2, angle
  position * theta^(-2i/D)) is the standard form, a reading the pages leave
  open, as is which segments are rotated (here: the decoder's self Q and K).

Readings taken where the pages are silent are listed with each function.
Parity is pinned by ``tests/test_oracle_pins.py`` (brute force, closed forms,
library special cases, invariants); nothing here is "parity unpinned".
"""
from .kalm_oracle import (  # noqa: F401
    bf16_round,
    rope_inv_freq,
    apply_rope,
    bf16_bits_to_f64,
    f64_to_bf16_bits,
    pooled_counts,
    chunk_pool,
    linear,
    merged_attention_doc,
    merged_attention,
    decoder_layer,
    yes_no_score,
    sigmoid,
    forward_doc,
    forward_query,
)
