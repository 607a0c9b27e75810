"""CPU oracle for Re-ttention's statistically reshaped static block-sparse attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls, links or
executes anything in this package: only ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` do.  The
oracle shares no code with the CUDA path (no kernels, headers, helpers, tables
or pre/post-processing); the two meet only in the seeded input generators.

Contents
--------
``reference``  NumPy float64 definitions of every step of the path: full
               attention, the calibration statistics (rho, residual R), the
               ramped reshaping of the sparse step, the DiTFastAttn contrast and
               the CSR block index.
``brute.c``    An independent scalar triple-loop float64 brute force in plain C
               (token-level keep mask), used to pin ``reference`` on tiny inputs.
               ``oracle.brute`` compiles and loads it.

Sources (Re-ttention: Ultra Sparse Visual Generation via Attention Statistical
Reshape):
- OpenReview discussion, authors' reply to W1 (first reviewer) and to W1 of the
  third reviewer: the worked 4-key example, rho as the ratio of the sparse to
  the full softmax denominator, the residual as the attention contribution of
  the masked tokens only.
- OpenReview discussion, reply to Q2: rho is per attention head and per token.
- OpenReview discussion, reply to Pwod W1: the ramp-up hyperparameter lambda
  that raises rho with the steps since calibration (formula not given; see
  ``reference.ramp_ref``; that function's arithmetic is "parity unpinned").
- Summary page, "Approach": cache the denominator ratio from a full-attention
  step, rescale sparse probabilities by it (with a ramp-up), add the cached
  residual of the masked tokens.
"""

from .reference import (  # noqa: F401
    RAMP_MUL_LINEAR,
    RAMP_ADD_LINEAR,
    RAMP_GEOMETRIC,
    token_keep_mask,
    full_attention_ref,
    calibrate_ref,
    ramp_ref,
    sparse_step_ref,
    build_block_index_ref,
    ditfastattn_residual_ref,
    calibrate_rows_ref,
    sparse_step_rows_ref,
)
