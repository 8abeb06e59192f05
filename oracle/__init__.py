"""Plain fp64 CPU oracle for decode-time latent attention in looped Transformers.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (the CUDA library and its Python binding) never
imports, calls or falls back to anything here, and nothing here imports the
product path.  The two share no code; only the seeded input generators in
``synth`` feed both.

What is computed, and where the pages define it
------------------------------------------------
Two web pages define the method:

* "Looped Latent Attention: Cross-Loop Key-Value Compression For Looped
  Transformers" (ICLR 2027 submission page, Abstract) -- called the *LLA
  abstract* below.  It defines the per-head LLA codec that "reconstructs
  loop-specific vectors only when attention reads them", the LLA-2D variant
  that folds heads into one latent, and the absorbed LLA-D variant that
  "reads latents without reconstruction".
* The Hybrid Latent Attention summary page (picx.dev), sections
  "Methodology / Latent Writer" (eq. 2), "Methodology / Latent Reader"
  (eqs. 3 and 4) and "Methodology / Rotary Embedding Alignment" -- called the
  *HLA summary* below.

Modules:

* ``rope``     -- the rotary operator R at any even dimension, with the
                  frequency-aligned pairing of latent dimensions.
* ``rounding`` -- IEEE round-to-nearest-even to bf16 / fp32 storage.
* ``quant``    -- fp8 (e4m3) latent rows with per-token, per-part scales.
* ``hla``      -- HLA latent writer (eq. 2) and absorbed read (eqs. 3-4), plus
                  the reconstruct-then-attend form used by invariants.
* ``lla``      -- LLA per-head / LLA-2D writers, LLA reconstruct-on-read, and
                  the absorbed LLA-D read.
* ``exact``    -- exact per-loop RoPE attention (the teacher's per-loop cache).
* ``codec``    -- full-rank SVD codecs used only to state the exactness
                  invariant (full rank latent attention == exact attention).

Each function's docstring states how it reads the points the pages leave
open (sum ranges, window extent, where the rotation of the key latent is
applied, the pairing of latent dimensions to rotary frequencies).

Parity status: every function here is pinned by a ``-m "not gpu"`` test in
``tests/test_oracle_*.py`` against a closed form, a special case that reduces
to textbook attention or a library routine, or an invariant that the pages
state (full rank is exact, absorbed equals reconstruct, rotation commutes
with same-frequency pair combinations, a window covering the context is exact
attention).  No function is "parity unpinned".
"""

from . import rope, rounding, quant, hla, lla, exact, codec  # noqa: F401
