"""Exact attention forward oracle (fp64, CPU).

TEST INFRASTRUCTURE ONLY.  The tests, the package smoke check and the
benchmark's CPU-baseline / reference leg are the only callers; the product
path (the CUDA library and its Python binding) never imports this package.
Nothing here shares code with the CUDA path.

Two independent implementations of the same plain definition
(FlashAttention: Fast and Memory-Efficient Exact Attention with IO-Awareness,
wiki notes, section "Problem setting": O = softmax(Q K^T) V, with the scores
and probabilities materialised as in the "standard attention" row of the
section "IO complexity analysis"):

* ``attn_oracle.c``   -- plain C, fp64, OpenMP over query rows (the oracle the
  parity tests and the CPU baseline use);
* ``attn_oracle_np``  -- NumPy fp64 twin that materialises the whole N x N
  matrix (used to cross-check the C oracle on small cases).

The backward (exact dQ, dK, dV for an upstream dO; wiki notes, section
"Recomputation") has the same pair: ``attn_bwd_oracle.c`` and
``attention_bwd_full`` in the NumPy twin.

Parity status: pinned (see tests/test_oracle_pins.py).
"""
from .oracle_c import attention_bwd_rows, attention_rows, build, library_path, max_threads
from .attn_oracle_np import attention_bwd_full, attention_full

__all__ = ["attention_rows", "attention_full", "attention_bwd_rows", "attention_bwd_full", "build",
           "library_path", "max_threads"]
