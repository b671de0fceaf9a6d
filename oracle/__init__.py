"""Plain, slow, fp64 CPU statement of the Codec-Gauge cache-coordinate codec.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and
its Python binding) imports, links or executes anything in this package; only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg do.

Source: "Codec-Gauge: Learning Compression-Friendly Gauges for Transformer KV
Caches" (arXiv 2607.20538), the Chinese translation (problem statement) and the
English method / experimental-setup text.  Every display equation of the method
was stripped from the pages; where a formula is missing, the function that
implements it says which reading it takes.

Modules:
  fpround   -- IEEE fp32 / fp16 / bf16 rounding and an exact fp32 FMA
  gauge     -- G = exp(A - A^T), group-wise application y = G x and its inverse
  quant     -- block-uniform and KIVI-style min/max quantizers, LE bit packing
  codec     -- encode / decode of a whole [L][2][B][H][T][d] cache
  spectral  -- 2-D orthonormal DCT-II statistics L_freq, L_rate and gradients
  metrics   -- NRMSE, bits/value

Parity status (each function's docstring repeats it):
  * spectral.l_freq / l_rate / objective: pinned to the stated formulas
    (closed forms, Parseval, brute force).  Whether those formulas equal the
    pages' elided equations is "parity unpinned": the equations are missing.
"""
