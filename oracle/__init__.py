"""fp64 CPU oracle for the fused chunked top-K KL distillation loss.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, links or runs
this package: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may.  It shares no code with the CUDA library (no kernels,
headers, helpers, tables or pre/post-processing); it receives the exact bytes
the GPU consumed and recomputes everything from the definitions.

Sources (cited by page title and section throughout):

* [DD] developersdigest.tech, "Distilling an LLM on One GPU: Offline Top-K
  Logits and a Fused Chunked KL Loss" -- sections "Why distillation recovery is
  expensive", "The two changes", "What this changes in practice".
* [GX] goaixin.org, "Breaking the Memory Barrier: How New Research Makes Large
  Language Model Knowledge Distillation Practical on a Single GPU" -- sections
  "Detailed Chronology and Technical Evolution", "Supporting Context and
  Metrics".
* [ST] scitechpulse.com, "New distillation trick cuts training memory below
  single-GPU limit for large language models" (no section headings).
* [AS] andresseo.expert, "The $250GB Memory Spike That Killed Distillation
  Projects Is Now Optional" -- sections "Offline Top-K: Compute the Teacher
  Once, Then Discard It", "Fused Chunked KL: The Loss That Never Builds the Full
  Grid", "What a Single H200 GPU Can Now Do That Once Required Four Nodes".

Pins: every function here is checked by ``tests/test_oracle_pins.py`` against
something other than itself (closed forms, library routines on special cases,
brute force, finite differences, hand-derived fixtures).  No function is
"parity unpinned".
"""

from .kd_oracle import (  # noqa: F401
    bf16_bits_to_f64,
    topk_rows,
    teacher_distribution,
    forward,
    forward_rows,
    backward,
    backward_dH_rows,
    backward_dW_rows,
    dense_bruteforce_loss,
)
