"""Plain, slow, fp64 CPU oracle for the OrbitQuant hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute anything in this package: only ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline / reference legs of ``bench.py`` use it.  It shares no
code, tables or constants with the CUDA library; the two meet only through the
seeded synthetic inputs, which hold none of the method's arithmetic.

Sources (the web pages this method is taken from):

* [OQ]  "OrbitQuant: Data-Agnostic Quantization for Image and Video Diffusion
  Transformers" (picx.dev structured summary of arXiv 2607.02461).  This is
  the authority on what is computed.
* [TQ]  "TurboQuant: Online Vector Quantization with Near-optimal Distortion
  Rate" (Docswell slide deck, slides numbered by its "Page. N" markers).
  Source of the sphere marginal f_d, the Lloyd-Max construction and the
  distortion bounds that OrbitQuant inherits.
* [RHT] "Quantizing With Randomized Hadamard Transforms: Efficient Heuristic
  Now Proven" (gist.science explainer).  Related theory only.

Module map:

* ``splitmix64``  -- the counter-based generator that draws the permutation
  and the Rademacher signs (the pages fix no generator; see ``rpbh``).
* ``rpbh``        -- the RPBH rotation Pi_d by definition (dense Hadamard,
  explicit permutation and sign matrices).
* ``codebook``    -- f_d and the Lloyd-Max codebook by numerical integration.
* ``quantize``    -- norm, normalise, brute-force nearest centroid, packing.
* ``linear``      -- the quantized linear layer as an fp64 sum.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
against closed forms, printed values or brute force, except the pages'
"Proposition 1" (its statement is not printed), which is not implemented.
"""
