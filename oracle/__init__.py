"""CPU oracle for Log-linear Sparse Attention (LLSA).

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the tests, the smoke check in
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
or run anything in this package.  The CUDA library never calls it, and it
shares no code with the CUDA library: the only thing both sides take from a
common module is the seeded input generator, which holds none of the method's
arithmetic.

Every function follows "Trainable Log-linear Sparse Attention for Efficient
Diffusion Transformers" (howistudyai explainer, Steps 1-4 and Building Blocks)
in plain numpy, step by step, with no blocking or fusion.  Floating point
results are fp64, except where a float decides an integer (the Top-K scores):
there the decision is taken in fp32, in one stated summation order, which is
the precision and order of the CUDA kernels.

Parity status of each function (what pins it, in tests/test_oracle_*.py):
  pool             pinned: constant input, Z-order ramp centroids, fp64 mean
                   within the summation error bound.
  select_level     pinned: exhaustive flat Top-K on integer inputs, planted
  select_all       winners, tie-break order, the factor-2 descent example.
  attn_fwd         pinned: dense masked attention, full softmax attention,
                   the weight-as-duplication invariant.
  index_transpose  pinned: dense block-mask transpose, pair-count invariants,
                   the 100-query x 8-key example (800 pairs).
  attn_bwd         pinned: central finite differences of <dO, O>.
  zorder_index     pinned: the 4x4 grid written out by hand, a decoded
  reorder          token, 4x4-tile runs, round trips.
  enriched_top     pinned: dense masked attention over levels 2..Lc,
                   padded index lists, finite differences.
  level_topk       pinned: flat exhaustive Top-K_1 under all-keeping upper
                   levels, a planted descent that turns on K_2, padding.
"""

from .llsa_oracle import (  # noqa: F401
    pool,
    enriched_top,
    reorder,
    zorder_index,
    select_level,
    select_all,
    level_topk,
    candidates_for_level,
    key_sets,
    attn_fwd,
    index_transpose,
    attn_bwd,
    run_forward,
    default_scale,
)
