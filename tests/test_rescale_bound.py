"""The lazy-rescale check of the d > 64 kernels, in float32 on the host.

The kernels compute each row block's p_c = 2^(x_c), x_c = fma(s_c, c_log2, -m),
sum the p_c in float32 (four partial sums of pairs, then combined) and take the
exact largest x only when some row sum exceeds 255: p_c <= the row sum for
non-negative p_c, and x_c > 8 gives p_c > 255.  These tests emulate that
float32 arithmetic (with the exponential perturbed by more than the hardware
approximation's relative error) and check that no block with an x above 8 can
pass the check unflagged, and that the largest x equals the fma of the largest
logit (the fma is monotone in s_c for c_log2 > 0).
"""

import numpy as np

RESCALE_LOG2 = 8.0
RESCALE_SUM = np.float32(255.0)
EX2_REL_ERR = 2.0 ** -20           # larger than the hardware ex2.approx error bound


def _fma32(a, b, c):
    """float32 fma: the exact a*b + c (float64 holds the float32 product
    exactly) rounded once to float32."""
    return (a.astype(np.float64) * np.float64(b) + np.float64(c)).astype(np.float32)


def _row_sums32(p):
    """Row sums in the kernels' order: pairs accumulated into four partial sums
    (element pair c goes to partial c % 4), then ((s0 + s1) + (s2 + s3)), then
    the two halves of the pair added."""
    rows, n = p.shape
    lo = np.zeros((rows, 4), np.float32)
    hi = np.zeros((rows, 4), np.float32)
    for c in range(n // 2):
        lo[:, c % 4] = lo[:, c % 4] + p[:, 2 * c]
        hi[:, c % 4] = hi[:, c % 4] + p[:, 2 * c + 1]
    tlo = (lo[:, 0] + lo[:, 1]) + (lo[:, 2] + lo[:, 3])
    thi = (hi[:, 0] + hi[:, 1]) + (hi[:, 2] + hi[:, 3])
    return (tlo + thi).astype(np.float32)


def _blocks(rng, rows, scale, shift):
    s = (rng.standard_normal((rows, 128)) * scale).astype(np.float32)
    c_log2 = np.float32(1.4426950408889634 / np.sqrt(128.0))
    # the running max of an earlier block: the row max of this block minus a
    # random shift, so that x ranges from well below to well above 8
    m = (s.max(axis=1).astype(np.float64) * c_log2 - shift).astype(np.float32)
    return s, c_log2, m


def test_a_block_with_x_above_8_always_has_a_row_sum_above_255():
    rng = np.random.default_rng(0)
    flagged_needed = 0
    for scale in (1.0, 4.0, 16.0):
        for shift in (0.0, 7.9, 8.0, 8.05, 9.0, 20.0):
            s, c_log2, m = _blocks(rng, 4096, scale, shift)
            x = _fma32(s, c_log2, -m[:, None])
            for sign in (-1.0, 1.0):
                p = (np.exp2(x.astype(np.float64)) * (1.0 + sign * EX2_REL_ERR)).astype(np.float32)
                sums = _row_sums32(p)
                needs = (x > RESCALE_LOG2).any(axis=1)
                flagged = sums > RESCALE_SUM
                assert not np.any(needs & ~flagged), (scale, shift, sign)
                flagged_needed += int(needs.sum())
    assert flagged_needed > 0             # the cases above do reach the rescale


def test_largest_x_is_the_fma_of_the_largest_logit():
    rng = np.random.default_rng(1)
    for scale in (1.0, 8.0, 100.0):
        s, c_log2, m = _blocks(rng, 4096, scale, 3.0)
        x = _fma32(s, c_log2, -m[:, None])
        direct = x.max(axis=1)
        via_max = _fma32(s.max(axis=1), c_log2, -m)
        np.testing.assert_array_equal(direct, via_max)


def test_masked_keys_do_not_flag():
    # keys past the sequence end are -inf logits: p = 0, so they add nothing
    s, c_log2, m = _blocks(np.random.default_rng(2), 256, 1.0, 0.0)
    s[:, 100:] = -np.inf
    x = _fma32(s, c_log2, -m[:, None])
    p = np.exp2(x.astype(np.float64)).astype(np.float32)
    assert np.all(p[:, 100:] == 0.0)
    assert np.all(_row_sums32(p) <= RESCALE_SUM)
