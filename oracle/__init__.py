"""CPU fp64 oracle for block-sparse attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import anything from this package.  The product (the CUDA
library and its Python binding) never imports it, and this package imports
nothing from the product: the two share no code.  The only shared module is
``workloads`` (seeded input generation, no attention arithmetic).

What it computes, and where the pages define it:

* ``masks``      -- the three mask rules of the FlexAttention how-to
  (dreaming.press, "Mask 1: causal", "Mask 2: sliding-window causal",
  "Mask 3: document-packed"); True means the pair is used, the SDPA
  convention (qiita GeneLab_999 SDPA tutorial, section 4 "罠1").
* ``attention``  -- the attention definition softmax(Q K^T / sqrt(E) + B) V
  (SDPA tutorial, section 1) with B = 0 / -inf from the mask and the optional
  tanh softcap score_mod (how-to, "Bonus: a score_mod for soft-capping"),
  evaluated densely in fp64, row chunk by row chunk, never skipping a block.
* ``online``     -- the same quantity by the tiled running-max / running-sum
  recurrence the FlashAttention pages describe; an independent derivation
  used only to cross-check ``attention``.
* ``blockmask``  -- 128x128 block classification (empty / full / partial) by
  evaluating the mask on every pair (FlexAttention vs SDPA on M1 Max,
  "役割とデータの流れ": BlockMask groups the work in 128x128 token blocks).
* ``bruteforce`` -- pure-Python triple loops for tiny shapes.

Readings where the pages are silent (each pinned by a test under tests/):
score_mod acts on the already scaled score; LSE is the natural log of the
softmax denominator; a row with no live key yields out = 0 and LSE = -inf;
L != S uses absolute (upper-left aligned) indices; positions past L or S are
never live, so a block that holds them is never FULL.
"""
from . import masks, attention, online, blockmask, bruteforce  # noqa: F401
