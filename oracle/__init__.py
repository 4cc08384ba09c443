"""fp64 CPU oracle for the dictionary-compressed projection (TEST INFRASTRUCTURE).

This package is a plain, slow, obviously-correct restatement of what the
DictLLM hot path computes (arXiv 2611.08082, "DictLLM: Post-training
Compression of Large Language Model with Dictionary Kernels"; technical review
"DictLLM: Shared Dictionaries for Post-Training Compression", Eq. (1)):

    W_l ~= D_g C_l,   Z_l = X_l D_g,   Y_l ~= Z_l C_l

with D_g and C_l stored in NVFP4 (4-bit E2M1 values, one 8-bit E4M3 scale per
block of sixteen values, one fp32 per-tensor scale; review section "From
retained values to measured decoding").

It is test infrastructure only.  Only ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import
it.  It shares no code with the CUDA library (no kernels, headers, helpers,
tables or constant generators); the only common code is the seeded input
generator module ``synth``, which holds none of the method's arithmetic.

Modules
  nvfp4       E2M1 / E4M3 decode tables written from the public format
              definitions; round-to-nearest-even encoders; block quantiser.
  pack        the packed byte layouts of D_g and C_l (bit-exact contract).
  forward     decode of packed factors, dense W = D C, X W, the factored
              (X D) C path and a brute-force triple loop.
  accounting  Eq. (2), Eq. (3), the multiply-add count, NVFP4 bits per value,
              Eq. (12) break-even, and the algorithmic bytes per call.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
against values the pages print, closed forms, library routines or brute
force. The pages print no input/output pair for the end-to-end quantised
forward; it is pinned by the special case where quantisation is exact (factors
whose NVFP4 blocks each hold an entry of magnitude 6 x 448 and otherwise values
of the scaled E2M1 grid), where pack, decode and forward must reproduce the
integer product of the original factors exactly, for every index layout.
"""
