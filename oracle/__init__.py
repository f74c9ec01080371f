"""CPU reference ("oracle") for Radial Attention's block-sparse masked attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this package: only the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference arm of ``bench.py`` use it.  It shares no code with
the CUDA path (no kernels, headers, helpers, tables or constant generators);
the two only meet on inputs drawn by the seeded generator module
``block_sparse_attention_csr_b200.inputs``, which holds none of the method's
arithmetic, and that module is never imported from here either: callers pass
arrays in.

Everything is plain NumPy in float64 (the pages fix no precision for the
reference computation).

Sources (web pages about the method; cited by title and section):

* [review]   "Paper review: Radial Attention: O(n log n) Sparse Attention with
             Energy Decay for Long Video Generation" (jaehun.me) -- §3 (Eq.1,
             Eq.2), §4.2 (Fig.5, Eq.4, flattening, attention sink / App. A.1
             Eq.8, 128x128 blocks), §4.2 Eq.6, and the worked toy example
             ("Walking Through a Toy Example", cases A-D).
* [rebuttal] "Radial Attention: O(n log n) Sparse Attention for Long Video
             Generation" -- authors' responses (paperhub.cn): central band
             width, width scale between bands, diagonal-frequency reduction,
             constant sparsity across resolutions.

Modules:

* :mod:`oracle.mask`      -- the token-level mask, its block-level CSR.
* :mod:`oracle.attention` -- masked softmax attention forward and backward.
* :mod:`oracle.lora`      -- LoRA-wrapped Q/K/V/O projections around it ([review] §4.3).

Parity status per function is stated in each module header.
"""

from . import mask, attention  # noqa: F401
