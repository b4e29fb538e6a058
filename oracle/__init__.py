"""fp64 CPU oracle for the fused attention forward pass — TEST INFRASTRUCTURE ONLY.

What it computes is the plain definition of scaled-dot-product attention with the
FlexAttention variants, written out in numpy float64: materialise the scores, apply the
score modification and the mask, run a two-pass softmax, multiply by V, and report the
per-row log-sum-exp.  It is deliberately slow and shares no code, header, table or
constant with the CUDA path under ``tiled_attention_14_b200/``; neither imports the
other.  Only the test suite, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import it.  The product path never calls
it and has no CPU fallback.

Modules
-------
``attention``  the attention forward (scores, score_mod, mask, softmax, O, LSE), with
               grouped-query heads and packed variable-length sequences.
``attention_bwd``  the gradients dQ, dK, dV of that forward (the chain rule, step by step).
``e4m3``       the FP8 e4m3 code book, encoder and per-128-row block quantiser.
``fp4``        the FP4 e2m1 code book and encoder, the MX (32-element, power-of-two scale)
               block quantiser, and the Direct-P attention forward that maps scores
               straight to FP4 codes.
``tile_map``   the block-sparse tile classification (EMPTY / PARTIAL / FULL), by brute force.

Every function is pinned by the ``-m "not gpu"`` tests in ``tests/test_oracle_*.py``
against closed forms, invariants, brute force on tiny inputs and library routines
(torch's CPU fp64 SDPA, torch's e4m3 cast, ml_dtypes' e2m1 type).  No function is left "parity unpinned".
"""
