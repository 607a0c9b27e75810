"""Seeded synthetic inputs shaped like the self-attention layers Re-ttention is
evaluated on (PixArt, Hunyuan-DiT, CogVideoX-2B) plus the tiny and long-video
cases.  This module holds none of the method's arithmetic: it only draws
Q/K/V, drifts them from one denoising step to the next, and lays out the
static block masks.  Both the CUDA path and the CPU oracle consume what it
makes.

Recipe
------
* Q, K, V ~ N(0, 1) in float32, rounded to bf16, layout [B, H, L, d]
  contiguous.  Each (batch, head) slab is drawn from its own generator,
  ``torch.Generator(device).manual_seed(stream_seed(seed, 0, b, h))``, in the
  order Q, K, V, so that a rank that owns a range of heads draws exactly those
  heads' values and nothing else.
* Next denoising step: X_{s+1} = bf16(X_s + 0.05 N(0, 1)), the noise of slab
  (b, h) drawn from a generator seeded with stream_seed(seed, s + 1, b, h),
  again in the order Q, K, V.
* Text tokens (MM-DiT "unified self-attention", Re-ttention OpenReview reply
  to Q5) come first in the sequence, visual tokens follow in row-major
  (frame, y, x) order.
* Static block mask (Re-ttention OpenReview reply to W2: static, spatially or
  temporally local windows): a key block is kept for a query block when it
  holds any text token, or when it is among the nearest key blocks by the
  Euclidean distance between the blocks' centroids (mean (f, y, x) of their
  visual tokens; ties to the lower index), the query block itself first, until
  ``kept`` blocks are kept.  A query block with no visual token keeps the text
  blocks and then the lowest-index other blocks.  The tiny case keeps the
  diagonal block only.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional, Tuple

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    L: int
    d: int
    block: int
    kept: int                   # kept key blocks per query block
    n_sparse_steps: int         # sparse steps after each calibration
    seed: int
    n_text: int = 0             # text tokens, placed first
    grid: Optional[Tuple[int, int, int]] = None   # (frames, rows, cols) of visual tokens
    lam: float = 0.04
    diagonal: bool = False      # tiny case: keep only the diagonal block

    @property
    def nqb(self) -> int:
        return -(-self.L // self.block)

    @property
    def nkb(self) -> int:
        return self.nqb


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 256, 64, 64, kept=1, n_sparse_steps=1, seed=0, diagonal=True),
    "pixart": Workload("pixart", 2, 16, 4096, 72, 128, kept=2, n_sparse_steps=4, seed=1,
                       grid=(1, 64, 64)),
    "hunyuan": Workload("hunyuan", 2, 16, 4352, 88, 128, kept=3, n_sparse_steps=4, seed=2,
                        n_text=256, grid=(1, 64, 64)),
    "cogvideox": Workload("cogvideox", 1, 30, 17776, 64, 128, kept=4, n_sparse_steps=9, seed=3,
                          n_text=226, grid=(13, 30, 45)),
}
# long-video sweep: density 25 / 12.5 / 6.25 / 3.1 % of 900 key blocks
for _dens, _tag in ((0.25, "25"), (0.125, "12.5"), (0.0625, "6.25"), (0.03125, "3.1")):
    WORKLOADS[f"longvideo-{_tag}"] = Workload(
        f"longvideo-{_tag}", 1, 24, 115200, 128, 128, kept=int(math.floor(900 * _dens + 0.5)),
        n_sparse_steps=1, seed=4, grid=(32, 45, 80))


# ---------------------------------------------------------------------------
# static block masks
# ---------------------------------------------------------------------------

def token_coords(w: Workload, perm=None) -> np.ndarray:
    """(f, y, x) grid coordinates of the token at each position [L, 3]; NaN for
    text tokens.  perm (optional, [L]): position i holds raster token perm[i]
    (raster = text tokens, then the grid with x fastest)."""
    raster = np.arange(w.L) if perm is None else np.asarray(perm, dtype=np.int64)
    out = np.full((w.L, 3), np.nan)
    if w.grid is not None:
        F, Y, X = w.grid
        vis = raster >= w.n_text
        r = raster[vis] - w.n_text
        out[vis] = np.stack([r // (Y * X), (r // X) % Y, r % X], axis=1)
    return out


def block_centroids(w: Workload, perm=None):
    """Mean (f, y, x) of each block's visual tokens; NaN rows for text-only blocks.
    Also returns the boolean 'holds a text token' per block.  perm as in
    token_coords (text tokens stay first, so the text blocks do not move)."""
    nb = w.nqb
    tok = np.arange(w.L)
    blk = tok // w.block
    has_text = np.zeros(nb, dtype=bool)
    if w.n_text:
        has_text[np.unique(blk[: w.n_text])] = True
    cent = np.full((nb, 3), np.nan)
    if w.grid is not None:
        coords_all = token_coords(w, perm)
        f, y, x = (coords_all[w.n_text:, k] for k in range(3))
        coords = np.stack([f, y, x], axis=1).astype(np.float64)
        vb = blk[w.n_text:]
        sums = np.zeros((nb, 3))
        np.add.at(sums, vb, coords)
        cnt = np.bincount(vb, minlength=nb)
        ok = cnt > 0
        cent[ok] = sums[ok] / cnt[ok, None]
    return cent, has_text


def block_mask(w: Workload, perm=None) -> np.ndarray:
    """uint8 [1, nqb, nkb] static block mask shared by every batch and head,
    built on the token order perm (see token_coords; default raster)."""
    nb = w.nqb
    m = np.zeros((nb, nb), dtype=np.uint8)
    if w.diagonal:
        np.fill_diagonal(m, 1)
        return m[None]
    cent, has_text = block_centroids(w, perm)
    text_blocks = np.nonzero(has_text)[0]
    visual = ~np.isnan(cent[:, 0])
    for qb in range(nb):
        row = set(int(t) for t in text_blocks)
        if visual[qb]:
            dist = np.linalg.norm(cent - cent[qb], axis=1)
            dist[~visual] = np.inf
            order = np.lexsort((np.arange(nb), dist))   # by distance, then index
        else:
            order = np.arange(nb)
        for kb in order:
            if len(row) >= w.kept:
                break
            if np.isfinite(cent[kb, 0]) or not visual[qb]:
                row.add(int(kb))
        m[qb, sorted(row)] = 1
    return m[None]


# ---------------------------------------------------------------------------
# Q / K / V
# ---------------------------------------------------------------------------

def _randn(shape, gen, device):
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32)


def stream_seed(seed: int, step: int, b: int, h: int) -> int:
    """Seed of the generator that draws slab (b, h) at denoising step `step`
    (0 = the initial values, s + 1 = the drift from step s to s + 1)."""
    return ((seed * 1009 + step) * 65537 + b) * 65537 + h


def _head_range(w: Workload, heads):
    h0, h1 = (0, w.H) if heads is None else heads
    if not 0 <= h0 < h1 <= w.H:
        raise ValueError(f"head range {heads} outside 0..{w.H}")
    return h0, h1


def initial_qkv(w: Workload, device="cpu", heads=None):
    """Step-0 Q, K, V: bf16 [B, H, L, d] from N(0, 1).  heads = (h0, h1)
    draws only heads h0..h1-1 (a [B, h1-h0, L, d] slice with the values the
    whole problem has there)."""
    h0, h1 = _head_range(w, heads)
    out = [torch.empty((w.B, h1 - h0, w.L, w.d), dtype=torch.bfloat16, device=device) for _ in range(3)]
    for b in range(w.B):
        for h in range(h0, h1):
            gen = torch.Generator(device=device).manual_seed(stream_seed(w.seed, 0, b, h))
            for x in out:
                x[b, h - h0] = _randn((w.L, w.d), gen, device).to(torch.bfloat16)
    return tuple(out)


def drift_qkv(w: Workload, qkv, s: int, heads=None):
    """Step s+1 from step s: X + 0.05 N(0, 1), rounded to bf16.  heads as in
    initial_qkv (qkv then holds that head range)."""
    h0, h1 = _head_range(w, heads)
    device = qkv[0].device
    out = [torch.empty_like(x) for x in qkv]
    for b in range(w.B):
        for h in range(h0, h1):
            gen = torch.Generator(device=device).manual_seed(stream_seed(w.seed, s + 1, b, h))
            for x, y in zip(qkv, out):
                n = _randn((w.L, w.d), gen, device)
                y[b, h - h0] = (x[b, h - h0].float() + 0.05 * n).to(torch.bfloat16)
    return tuple(out)


def qkv_steps(w: Workload, n_steps: int, device="cpu", heads=None):
    """List of (Q, K, V) for steps 0 .. n_steps-1 of one calibration cycle
    (heads = (h0, h1) for one rank's head range)."""
    steps = [initial_qkv(w, device, heads)]
    for s in range(n_steps - 1):
        steps.append(drift_qkv(w, steps[-1], s, heads))
    return steps


def random_qkv(B, H, L, d, seed, device="cpu"):
    """Free-shape N(0, 1) bf16 inputs for edge-case tests."""
    gen = torch.Generator(device=device).manual_seed(seed)
    return tuple(_randn((B, H, L, d), gen, device).to(torch.bfloat16) for _ in range(3))


def random_block_mask(Hm, nqb, nkb, density, seed, ensure_nonempty=False):
    """Bernoulli(density) uint8 [Hm, nqb, nkb] block mask for edge-case tests."""
    rng = np.random.default_rng(seed)
    m = (rng.random((Hm, nqb, nkb)) < density).astype(np.uint8)
    if ensure_nonempty:
        for h in range(Hm):
            for qb in range(nqb):
                if not m[h, qb].any():
                    m[h, qb, rng.integers(nkb)] = 1
    return m
