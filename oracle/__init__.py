"""CPU oracle of the batch-1 decode step.  TEST INFRASTRUCTURE ONLY.

This package is the slow, plain, float64 statement of what the persistent
decode kernel computes.  Only the tests, the smoke check and the benchmark's
CPU-baseline leg may import it; the product path never does, and it shares
no code with the CUDA library (the seeded input generator in ``synth`` is the
only module both sides use).

What it computes (Kog Inference Engine write-ups: the monokernel bullet runs
"the entire decode path" as one persistent kernel; "prefill, decode, LM-head
sampling" in the "Software versus silicon" section; FP16, batch 1, greedy,
"no quantisation, no speculative decoding, no pruning" in the "Laneformer 2B"
results table).  The pages give no model definition, so the decoder is the
textbook pre-norm one: RMSNorm, rotate-half RoPE, grouped-query attention over
a KV cache, SwiGLU MLP, untied embedding and LM head, greedy argmax.  The lane
variant follows the lane-structured transformer and Delayed Tensor
Parallelism bullets (8 lanes, cross-lane sum delayed by delta = 2 layers).

Pins: every function here is checked by ``tests/test_oracle_*.py`` against
library routines (numpy/torch conversions, ``torch.nn.functional``, the
``transformers`` Llama decoder in float64), closed forms, invariants and a
pure-Python no-cache brute force; none is "parity unpinned".
"""
from .numerics import round_to_storage, storage_to_f64  # noqa: F401
from .decoder import Oracle, argmax_lowest, rmsnorm, rope, silu, top2_margin  # noqa: F401
from .sampling import sample_token, sampling_margins  # noqa: F401
