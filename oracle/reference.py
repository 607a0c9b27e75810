"""Plain float64 NumPy definitions of Re-ttention's reshaped block-sparse attention.

TEST INFRASTRUCTURE ONLY (see the package docstring): the product path never
imports this module.

Notation (per batch b, head h; query row i, key j; all float64):

    s_ij   = c * <q_i, k_j>,    c = 1/sqrt(d) with the true head dimension d
    V(i)   = all valid keys j < L
    M(i)   = keys whose key block is kept for i's query block (static mask)
    m_i    = max_{j in V(i)} s_ij                      (calibration step)
    Z_full = sum_{j in V(i)}        exp(s_ij - m_i)
    Z_sp   = sum_{j in M(i)}        exp(s_ij - m_i)
    rho_i  = Z_sp / Z_full                                   "Eq. 8"
    R_i    = sum_{j in V(i) \\ M(i)} exp(s_ij - m_i) v_j / Z_full
    O_i    = sum_{j in V(i)}        exp(s_ij - m_i) v_j / Z_full   (full attention)

and, at a later step with drifted inputs (primes) and step distance k,

    O'_i = ramp(rho_i, lambda, k) * softmax_{M(i)}(s'_i) . v'  +  R_i
    O'_i = R_i                              if M(i) is empty.

Where the pages fix these (Re-ttention OpenReview discussion):
- reply to W1 of the first reviewer and W1 of the third reviewer: the worked
  4-key example: full row [0.1,0.4,0.4,0.1], window {1,2}: the reshaped sparse
  row is [0,0.4,0.4,0] (so rho = 0.8), the residual is [0.1,0,0,0.1] (only the
  masked tokens' attention); next step full row [0.1,0.3,0.5,0.1] gives sparse
  [0,0.375,0.625,0], reshaped [0,0.3,0.5,0], plus the residual = the full row.
- reply to Q2: rho is local, per attention head and per token, not averaged.
- reply to Q4: the residual has the shape of the attention output.
- reply to the third reviewer's W1 and to Pwod's W1: the cached rho is raised
  by a ramp-up hyperparameter lambda because rho grows over denoising.

Every function takes the inputs the GPU receives, widened exactly from bf16 to
float64, and computes each quantity by its definition: scores as a matrix
product, a row max, then the sums (two passes), materialised one query block at
a time.  There is no online softmax, no fusion and no reordering.
"""

from __future__ import annotations

import math

import numpy as np

RAMP_MUL_LINEAR = 0
RAMP_ADD_LINEAR = 1
RAMP_GEOMETRIC = 2

# sparse-step epilogues: Re-ttention's, and the two ablations the pages compare
EPI_RESHAPED = 0      # rho_hat * attn + R
EPI_NO_RHO = 1        # attn + R   (with R = O_full - O_sparse: DiTFastAttn's reconstruction)
EPI_NO_R = 2          # rho_hat * attn

# residual kept by a calibration step
RES_MASKED = 0        # Re-ttention: the masked tokens' part of the full output
RES_SUBTRACTIVE = 1   # DiTFastAttn: O_full - O_sparse


# ---------------------------------------------------------------------------
# masks
# ---------------------------------------------------------------------------

def _key_keep(block_mask_row: np.ndarray, block: int, L: int) -> np.ndarray:
    """Token-level kept keys M(i) for one query block: key j kept iff its key
    block j // block is kept.  Keys j >= L do not exist."""
    return np.repeat(np.asarray(block_mask_row, dtype=bool), block)[:L]


def token_keep_mask(block_mask_2d: np.ndarray, block: int, L: int) -> np.ndarray:
    """[L, L] boolean matrix whose row i is M(i).  Small L only."""
    bm = np.asarray(block_mask_2d, dtype=bool)
    qb = np.arange(L) // block
    return bm[qb][:, qb]


def _head_mask(block_mask: np.ndarray, h: int) -> np.ndarray:
    """The static mask is shared by all heads (Hm == 1) or given per head."""
    bm = np.asarray(block_mask)
    return bm[0] if bm.shape[0] == 1 else bm[h]


def _scale(d: int, scale):
    return (1.0 / math.sqrt(d)) if (scale is None or scale == 0) else float(scale)


# ---------------------------------------------------------------------------
# per-row definitions
# ---------------------------------------------------------------------------

def _full_rows(q_rows, k, v, c):
    s = c * (q_rows @ k.T)                      # [n, L]
    m = s.max(axis=1, keepdims=True)            # pass 1: row max over V(i)
    e = np.exp(s - m)                           # pass 2: exponentials and sums
    return (e @ v) / e.sum(axis=1, keepdims=True)


def _calibrate_rows(q_rows, k, v, keep, c):
    """keep: bool [n, L] (M(i) per row).  Returns O [n,d], rho [n], R [n,d]."""
    s = c * (q_rows @ k.T)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    e_in = np.where(keep, e, 0.0)
    e_out = np.where(keep, 0.0, e)
    z_full = e.sum(axis=1)
    z_sp = e_in.sum(axis=1)
    o = (e @ v) / z_full[:, None]
    r = (e_out @ v) / z_full[:, None]
    return o, z_sp / z_full, r


def _sparse_rows(q_rows, k, v, keep, rho_hat, r, c):
    """Reshaped sparse step for n rows: rho_hat * softmax over M(i) . v + R."""
    s = c * (q_rows @ k.T)
    has = keep.any(axis=1)
    s_in = np.where(keep, s, -np.inf)
    m = np.where(has, s_in.max(axis=1, initial=-np.inf), 0.0)
    e = np.where(keep, np.exp(s - m[:, None]), 0.0)
    z = e.sum(axis=1)
    attn = np.zeros_like(r)
    if has.any():
        attn[has] = (e[has] @ v) / z[has, None]
    return rho_hat[:, None] * attn + r


# ---------------------------------------------------------------------------
# public definitions
# ---------------------------------------------------------------------------

def full_attention_ref(q, k, v, scale=None):
    """Plain softmax attention over all L keys.  q, k, v: float64 [B,H,L,d]."""
    B, H, L, d = q.shape
    c = _scale(d, scale)
    out = np.empty_like(q)
    for b in range(B):
        for h in range(H):
            for i0 in range(0, L, 128):
                out[b, h, i0:i0 + 128] = _full_rows(q[b, h, i0:i0 + 128], k[b, h], v[b, h], c)
    return out


def calibrate_ref(q, k, v, block_mask, block, scale=None):
    """Calibration (full-attention) step.

    q, k, v: float64 [B,H,L,d]; block_mask: [Hm, nqb, nkb] with Hm in {1, H}.
    Returns (O [B,H,L,d], rho [B,H,L], R [B,H,L,d]).
    """
    B, H, L, d = q.shape
    c = _scale(d, scale)
    nqb = -(-L // block)
    o = np.empty_like(q)
    r = np.empty_like(q)
    rho = np.empty(q.shape[:3])
    for b in range(B):
        for h in range(H):
            bm = _head_mask(block_mask, h)
            for qb in range(nqb):
                i0, i1 = qb * block, min(L, (qb + 1) * block)
                keep = np.broadcast_to(_key_keep(bm[qb], block, L), (i1 - i0, L))
                o[b, h, i0:i1], rho[b, h, i0:i1], r[b, h, i0:i1] = _calibrate_rows(
                    q[b, h, i0:i1], k[b, h], v[b, h], keep, c)
    return o, rho, r


def ramp_ref(rho, lam, k, mode=RAMP_MUL_LINEAR):
    """Ramped denominator ratio rho_hat(rho, lambda, k), k = steps since calibration.

    The pages say only that the cached rho is used "plus" a ramp-up
    hyperparameter lambda because rho increases over the denoising steps; the
    formula itself is not on the pages.  Readings offered (all equal rho at
    lambda = 0 or k = 0, all increase with k, all clamp at 1 because a sub-sum
    ratio cannot exceed 1):
      RAMP_MUL_LINEAR  min(1, rho * (1 + lambda k))     (default)
      RAMP_ADD_LINEAR  min(1, rho + lambda k)
      RAMP_GEOMETRIC   min(1, rho * (1 + lambda)^k)
    Parity unpinned beyond lambda = 0 / k = 0.
    """
    rho = np.asarray(rho, dtype=np.float64)
    if mode == RAMP_MUL_LINEAR:
        x = rho * (1.0 + lam * k)
    elif mode == RAMP_ADD_LINEAR:
        x = rho + lam * k
    elif mode == RAMP_GEOMETRIC:
        x = rho * (1.0 + lam) ** k
    else:
        raise ValueError(f"unknown ramp mode {mode}")
    return np.minimum(1.0, x)


def sparse_step_ref(q, k, v, block_mask, block, rho, r, lam, kdist,
                    mode=RAMP_MUL_LINEAR, scale=None):
    """Reshaped sparse step: O' = ramp(rho) * softmax_{M(i)}(s') v' + R."""
    B, H, L, d = q.shape
    c = _scale(d, scale)
    nqb = -(-L // block)
    out = np.empty_like(q)
    for b in range(B):
        for h in range(H):
            bm = _head_mask(block_mask, h)
            rho_hat = ramp_ref(rho[b, h], lam, kdist, mode)
            for qb in range(nqb):
                i0, i1 = qb * block, min(L, (qb + 1) * block)
                keep = np.broadcast_to(_key_keep(bm[qb], block, L), (i1 - i0, L))
                out[b, h, i0:i1] = _sparse_rows(q[b, h, i0:i1], k[b, h], v[b, h], keep,
                                                rho_hat[i0:i1], r[b, h, i0:i1], c)
    return out


def ditfastattn_residual_ref(q, k, v, block_mask, block, scale=None):
    """DiTFastAttn's subtractive residual R_sub = O_full - O_sparse (the contrast
    the Re-ttention reply to W1 works through).  Reconstruction at a later step is
    sparse_step_ref(..., rho=ones, r=R_sub, lam=0): the sparse output, not
    reshaped, plus R_sub."""
    B, H, L, d = q.shape
    o_full = full_attention_ref(q, k, v, scale)
    ones = np.ones((B, H, L))
    zero = np.zeros_like(q)
    o_sp = sparse_step_ref(q, k, v, block_mask, block, ones, zero, 0.0, 0, RAMP_MUL_LINEAR, scale)
    return o_full - o_sp


def sparse_step_epilogue_ref(q, k, v, block_mask, block, rho, r, lam, kdist, epilogue=EPI_RESHAPED,
                             mode=RAMP_MUL_LINEAR, scale=None):
    """Sparse step with one of the epilogues the replies to W1 and the
    ablation table set side by side.  attn is the softmax over the kept keys
    (0 for a row with none):
      EPI_RESHAPED  ramp(rho) * attn + R      (Re-ttention)
      EPI_NO_RHO    attn + R                  (no statistical reshape; with
                                               DiTFastAttn's R_sub this is its
                                               reconstruction)
      EPI_NO_R      ramp(rho) * attn          (no residual)
    rho is not used by EPI_NO_RHO, r not by EPI_NO_R (either may be None)."""
    B, H, L, d = q.shape
    if epilogue == EPI_RESHAPED:
        return sparse_step_ref(q, k, v, block_mask, block, rho, r, lam, kdist, mode, scale)
    if epilogue == EPI_NO_RHO:
        return sparse_step_ref(q, k, v, block_mask, block, np.ones((B, H, L)), r, 0.0, 0, mode, scale)
    if epilogue == EPI_NO_R:
        return sparse_step_ref(q, k, v, block_mask, block, rho, np.zeros_like(q), lam, kdist, mode, scale)
    raise ValueError(f"unknown epilogue {epilogue}")


def schedule_ref(steps, block_mask, block, period, lam, mode=RAMP_MUL_LINEAR, epilogue=EPI_RESHAPED,
                 residual=RES_MASKED, scale=None):
    """Outputs of a denoising schedule: steps[t] = (q, k, v) of step t.  Step t
    is a calibration (full attention; it refreshes the cached rho and
    residual) when t % period == 0, else the sparse step at distance
    t % period with the cached statistics, as the pages run Re-ttention
    between periodic full-attention steps."""
    outs = []
    rho = r = None
    for t, (q, k, v) in enumerate(steps):
        kd = t % period
        if kd == 0:
            o, rho, r = calibrate_ref(q, k, v, block_mask, block, scale)
            if residual == RES_SUBTRACTIVE:
                r = ditfastattn_residual_ref(q, k, v, block_mask, block, scale)
            outs.append(o)
        else:
            outs.append(sparse_step_epilogue_ref(q, k, v, block_mask, block, rho, r, lam, kd, epilogue, mode,
                                                 scale))
    return outs


def hilbert_order_ref(n_text, F, Y, X):
    """Token order of the reordering row: text tokens first (unchanged), then
    the F x Y x X grid (raster index n_text + (f*Y + y)*X + x) sorted by the
    Hilbert index, over the axes longer than 1, within the smallest cube of
    side 2^b that holds the grid.  The index follows Skilling's transpose
    method ("Programming the Hilbert curve", 2004), evaluated here for all
    grid points at once.  Returns perm (int64 [L]): position i holds raster
    token perm[i]."""
    ext = [F, Y, X]
    bits = 0
    while (1 << bits) < max(ext):
        bits += 1
    f, y, x = np.meshgrid(np.arange(F), np.arange(Y), np.arange(X), indexing="ij")
    axes = [c.ravel().astype(np.int64) for c, e in zip((f, y, x), ext) if e > 1]
    n = len(axes)
    if n == 0:
        return np.arange(n_text + 1)
    a = [c.copy() for c in axes]
    q = 1 << (bits - 1) if bits > 0 else 0
    while q > 1:
        low = q - 1
        for i in range(n):
            hit = (a[i] & q) != 0
            swap = (a[0] ^ a[i]) & low
            a0_new = np.where(hit, a[0] ^ low, a[0] ^ swap)
            ai_new = np.where(hit, a[i], a[i] ^ swap) if i > 0 else a0_new
            a[0] = a0_new
            if i > 0:
                a[i] = ai_new
        q >>= 1
    for i in range(1, n):
        a[i] = a[i] ^ a[i - 1]
    t = np.zeros_like(a[0])
    q = 1 << (bits - 1) if bits > 0 else 0
    while q > 1:
        t = np.where((a[n - 1] & q) != 0, t ^ (q - 1), t)
        q >>= 1
    a = [c ^ t for c in a]
    key = np.zeros_like(a[0])
    for j in range(bits - 1, -1, -1):
        for i in range(n):
            key = (key << 1) | ((a[i] >> j) & 1)
    order = np.argsort(key, kind="stable")
    return np.concatenate([np.arange(n_text), n_text + order]).astype(np.int64)


def permute_tokens_ref(x, perm, inverse=False):
    """Rows of x [B, H, L, d] reordered: out[:, :, i] = x[:, :, perm[i]], or
    out[:, :, perm[i]] = x[:, :, i] with inverse."""
    perm = np.asarray(perm)
    if not inverse:
        return x[:, :, perm]
    out = np.empty_like(x)
    out[:, :, perm] = x
    return out


def build_block_index_ref(block_mask):
    """CSR of a dense block mask [Hm, nqb, nkb]: rows are (h, qb) flattened
    h-major; row_ptr has Hm*nqb+1 entries (exclusive prefix sum of the row
    counts); col_idx lists each row's kept key blocks in ascending order."""
    bm = np.asarray(block_mask) != 0
    Hm, nqb, nkb = bm.shape
    flat = bm.reshape(Hm * nqb, nkb)
    rows, cols = np.nonzero(flat)               # row-major order => ascending cols
    counts = np.bincount(rows, minlength=Hm * nqb)
    row_ptr = np.zeros(Hm * nqb + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum(counts)
    return row_ptr.astype(np.int32), cols.astype(np.int32)


# ---------------------------------------------------------------------------
# sampled rows (for sizes where the whole problem is too slow on the CPU)
# ---------------------------------------------------------------------------

def calibrate_rows_ref(q_bh, k_bh, v_bh, block_mask_h, block, rows, scale=None):
    """calibrate_ref restricted to query rows ``rows`` of one (b, h).
    q_bh, k_bh, v_bh: float64 [L, d]; block_mask_h: [nqb, nkb]."""
    L, d = k_bh.shape
    rows = np.asarray(rows)
    keep = np.stack([_key_keep(block_mask_h[i // block], block, L) for i in rows])
    return _calibrate_rows(q_bh[rows], k_bh, v_bh, keep, _scale(d, scale))


def sparse_step_rows_ref(q_bh, k_bh, v_bh, block_mask_h, block, rows, rho_rows, r_rows,
                         lam, kdist, mode=RAMP_MUL_LINEAR, scale=None):
    """sparse_step_ref restricted to query rows ``rows`` of one (b, h);
    rho_rows [n] and r_rows [n, d] are those rows' cached statistics."""
    L, d = k_bh.shape
    rows = np.asarray(rows)
    keep = np.stack([_key_keep(block_mask_h[i // block], block, L) for i in rows])
    rho_hat = ramp_ref(rho_rows, lam, kdist, mode)
    return _sparse_rows(q_bh[rows], k_bh, v_bh, keep, rho_hat, np.asarray(r_rows, np.float64),
                        _scale(d, scale))
