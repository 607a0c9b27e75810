"""Head sharding of one attention problem across ranks.

rho and the residual are per head and per token, and the block mask is
static, so the heads of one problem are independent: rank r of N runs the
calibration and the sparse steps on its own contiguous range of heads, on
strided views of the full [B, H, L, d] tensors, with no collective in the
data path.  These helpers give the range and the matching slice of a
per-head mask; the kernels themselves take the views through their strides.
"""

from __future__ import annotations

import numpy as np


def head_range(H: int, world: int, rank: int) -> tuple[int, int]:
    """[h0, h1) of rank `rank` of `world`: contiguous, sizes differ by at most 1."""
    if H < 1 or world < 1 or not 0 <= rank < world:
        raise ValueError("need H >= 1, world >= 1 and 0 <= rank < world")
    base, extra = divmod(H, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def shard_mask(mask: np.ndarray, h0: int, h1: int) -> np.ndarray:
    """The block mask [Hm, nqb, nkb] for heads [h0, h1): a mask shared by all
    heads (Hm == 1) is kept whole, a per-head mask is sliced."""
    if mask.shape[0] == 1:
        return mask
    return np.ascontiguousarray(mask[h0:h1])


def shard_heads(t, h0: int, h1: int):
    """View of heads [h0, h1) of a [B, H, L, ...] tensor (no copy)."""
    return t[:, h0:h1]
