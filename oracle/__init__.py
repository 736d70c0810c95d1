"""CPU oracle for top-p block-sparse self-attention (TEST INFRASTRUCTURE ONLY).

This package is the plain, slow, obviously-correct statement of what the GPU
path computes.  It exists to check the CUDA library and is used only by
``tests/``, by ``__graft_entry__.smoke()`` and by the CPU-baseline leg of
``bench.py``.  Nothing in the product package imports it, and it imports
nothing from the product package: it shares no code, tables or helpers with
the CUDA path.  Inputs arrive as numpy arrays; random draws are made by the
caller.

Sources (cited by page title and section in every function):

* "RECAP: Reciprocal Sparse Attention and Hierarchical Caching for Efficient
  Video Diffusion" -- full text, sections 1, 3.2, 3.4 (block means, cached
  dense refinement that corrects the sparse estimate, dense refreshes; the
  coarse tail of the omitted blocks and its reconstruction, section 3.2).
* the head-wise adaptive top-p abstract (Temporal Mask Reuse / Error-guided
  Budgeted Calibration) and the GSRS abstract ("Top-p selection for adaptive
  sparsity control") -- online top-p block selection with per-head p.
* "Ride the Wave: Precision-Allocated Sparse Attention for Smooth Video
  Generation" (DFSAttn) abstract -- Hilbert-curve token reordering, block
  scoring.
* CalibAtt (calibrated sparse attention), abstract and Fig. 5 -- threshold the
  top key blocks per query block, skip the unselected blocks.
* CalibAtt appendix, Fig. S9, Fig. S10 and Table S3 -- skip lists of
  interval pairs per query block, per-layer trimming, merging outlier rows.
* the GSRS abstract -- exact attention weights evaluated inside the
  FlashAttention computation (the kept share of the attention mass).

Modules:
  hilbert     -- 3-D Hilbert order of the latent grid, perm / inv
  scoring     -- block mean pooling and per-query-block softmax of block logits
  topp        -- cumulative top-p block selection, mask and kept lists
  attention   -- masked softmax attention over the kept blocks (O, LSE)
  correction  -- dense-minus-sparse refinement and the alpha-scaled correction
  refresh     -- the outputs of a single-pass dense refresh (dense and sparse
                 attention, refinement, exact kept attention mass)
  reuse       -- query-key drift of the block means, and scoring / selection
                 restricted to an earlier candidate set
  tail        -- coarse estimate of the omitted attention tail (block means
                 with the key-variance and value-key covariance corrections)
                 and its reconstruction with a cached refinement
  intervals   -- interval (skip-list) encoding of the kept blocks, merging of
                 outlier rows to a width, the width for a merge percentage
  fp8         -- E4M3 quantization of Q and K per token block (the FP8 path)

Every function carries a "Pinned by" note naming the tests (in
``tests/test_oracle.py`` unless stated) that tie it to something other than
itself.
"""

from . import hilbert, scoring, topp, attention, correction, refresh, reuse, intervals, tail, fp8  # noqa: F401
