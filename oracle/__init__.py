"""fp64 CPU oracle for the masked WIDE layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the benchmark's CPU-baseline leg (and its ``--impl reference`` arm) may import
it.  It shares no code with the CUDA path (``token_level_dynamic_b200``) and
neither imports the other; the seeded inputs come from ``synth``.

Source: "WIDE: Boosting Adaptive LLM Inference via Token-level Dynamic Width
Pruning" (abstract; technical summary sections 1, 2.A, 2.B and 2.C).

Contents
  ffn.ffn_masked        masked SwiGLU FFN, definition form (numpy float64)
  ffn.ffn_token_loop    the same, per-token loop over kept groups (C, fp64)
  ffn.reorder           canonical mask reordering (C)
  attention.*           RMSNorm, RoPE, masked GQA attention, whole layer
  router.*              bottleneck router -> packed group masks (section 2.A)

Parity pins live in tests/test_oracle_*.py.  Nothing here is "parity
unpinned".
"""
from . import ffn, attention, router  # noqa: F401
from ._clib import build  # noqa: F401
