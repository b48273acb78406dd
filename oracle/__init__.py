"""CPU oracle for the QSVD joint-QKV latent decode path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and
its Python binding) imports, calls or links anything here; only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of
``bench.py`` use it.  It shares no code with the CUDA path: the one common
dependency is the seeded input module ``synthetic``, which holds no arithmetic
of the method.

Everything is plain NumPy in float64, except the latent quantiser, which the
pages fix to a low-precision integer grid and which is written with float32
semantics so that it can be compared bit for bit (``quant_ref``).

Sources (web pages on the method; cited by title and section):

* "QSVD: Efficient Low-Rank Approximation for Unified Query-Key-Value Weight
  Compression" -- paper notes (Paper-Notes, NeurIPS 2025), sections
  方法详解 / 关键设计 (joint SVD, beta split, rotations H1/H2).
* "QSVD ... in Low-Precision Vision-Language Models" -- paper digest,
  sections Problem, Method (Steps 1-3), Key Contributions.
* "WSVD: Weighted Low-Rank Approximation ..." -- paper digest, sections
  Problem and Method (fused flash-decoding kernel, section 3.4).
* "SVDQuant 低秩残差量化算法" glossary entry, section 2.3 数学描述
  (Eckart-Young statement).

Parity pins: every function here is checked in ``tests/test_oracle_*.py``
against closed forms, invariants, library routines or brute force.  The only
unpinned items are the synthetic constants of the input recipe (kappa, the
3x3 DCT factor, the outlier channel picks), which the pages do not fix; both
sides consume the same stored inputs, so parity does not depend on them.
"""
