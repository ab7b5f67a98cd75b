"""fp64 restatement of the rotated-sparse linear path (test infrastructure).

Only the test suite, the smoke check and the benchmark's CPU-baseline leg may
use this module.  It must never be imported by the library.

All arithmetic is fp64.  Inputs may be given in any real floating dtype; they
are widened to fp64 (exact for fp32 and bf16 values).  Shapes: activations
are [M, d] (a single row may be passed as [d]), weights are row-major
[d_in, d_out], rotations are [d, d].
"""
from __future__ import annotations

import numpy as np


def _rows(a) -> tuple[np.ndarray, bool]:
    a = np.asarray(a, dtype=np.float64)
    if a.ndim == 1:
        return a[None, :], True
    if a.ndim != 2:
        raise ValueError("expected a vector or a [M, d] matrix")
    return a, False


def rotate(x, Q) -> np.ndarray:
    """x_rot = x . Q for every activation row.

    La RoSA summary, 方法详解 / 技术框架: in the rotation stage each layer's
    input activation is multiplied by that layer's orthogonal matrix.
    x_rot[m, j] = sum_i x[m, i] * Q[i, j].
    """
    xr, single = _rows(x)
    Q = np.asarray(Q, dtype=np.float64)
    if Q.shape != (xr.shape[1], xr.shape[1]):
        raise ValueError("Q must be d x d")
    out = xr @ Q
    return out[0] if single else out


def topk(x_rot, K: int) -> tuple[np.ndarray, np.ndarray]:
    """Exact per-row Top-K by magnitude.

    La RoSA summary, 方法详解 / 技术框架 (sparsification stage): keep the K
    entries of largest magnitude of each rotated activation vector, set the
    others to zero; abstract: Top-K gives the same sparsity on every token.

    Order of preference: larger |x| first, and among equal magnitudes the
    lower index first (+0 and -0 are equal).  The first K in that order are
    kept.  Returns (idx, val): idx [M, K] int64 in ascending index order and
    val [M, K] the kept entries with their signs.
    """
    xr, single = _rows(x_rot)
    M, d = xr.shape
    if not (0 <= K <= d):
        raise ValueError("K must satisfy 0 <= K <= d")
    if not np.all(np.isfinite(xr)):
        raise ValueError("Top-K is defined here for finite inputs only")
    idx = np.empty((M, K), dtype=np.int64)
    val = np.empty((M, K), dtype=np.float64)
    positions = np.arange(d)
    for m in range(M):
        mag = np.abs(xr[m])
        # np.lexsort sorts by the last key first: primary key -|x| ascending
        # (largest magnitude first), secondary key the index ascending.
        preference = np.lexsort((positions, -mag))
        kept = np.sort(preference[:K])
        idx[m] = kept
        val[m] = xr[m, kept]
    if single:
        return idx[0], val[0]
    return idx, val


def sparse_linear(idx, val, W_rot) -> np.ndarray:
    """y = sparse(x_rot) . W_rot, summing only over the kept rows.

    y[m, j] = sum_k val[m, k] * W_rot[idx[m, k], j].  Only the K selected rows
    of the counter-rotated weight take part (abstract: activation sparsity
    reduces memory transfers).
    """
    W = np.asarray(W_rot, dtype=np.float64)
    idx = np.asarray(idx)
    val = np.asarray(val, dtype=np.float64)
    single = idx.ndim == 1
    if single:
        idx, val = idx[None, :], val[None, :]
    if idx.shape != val.shape:
        raise ValueError("idx and val must have the same shape")
    y = np.empty((idx.shape[0], W.shape[1]), dtype=np.float64)
    for m in range(idx.shape[0]):
        y[m] = val[m] @ W[idx[m]]
    return y[0] if single else y


def dense_linear(x, W) -> np.ndarray:
    """y = x . W, the dense projection (row-major [d_in, d_out] weight)."""
    xr, single = _rows(x)
    W = np.asarray(W, dtype=np.float64)
    y = xr @ W
    return y[0] if single else y


def prepare_weights(Q, W) -> np.ndarray:
    """W_rot = Q^T . W (offline counter-rotation of the weight).

    The pages do not print it; since Q Q^T = I, x . W = (x . Q) . (Q^T . W),
    so rotating the input by Q requires the weight rows to be rotated by Q^T.
    W_rot[i, j] = sum_k Q[k, i] * W[k, j].
    """
    Q = np.asarray(Q, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    if Q.shape[0] != Q.shape[1] or Q.shape[0] != W.shape[0]:
        raise ValueError("Q must be d_in x d_in and W d_in x d_out")
    return Q.T @ W


def fold_rotation(Q, Wt_prev) -> np.ndarray:
    """The producer's weight with the rotation folded into it.

    Reading (the pages leave open where Q is applied): a layer whose input x
    is produced by a linear map x = h . Wt_prev^T (Wt_prev [d, d_prev] in
    torch.nn.Linear layout, one row per output channel) can receive x . Q
    directly from a producer with weight Wt_fold = Q^T . Wt_prev, because
    h . Wt_fold^T = h . Wt_prev^T . Q.  Returns Wt_fold [d, d_prev]:
    Wt_fold[i, j] = sum_k Q[k, i] * Wt_prev[k, j].
    """
    Q = np.asarray(Q, dtype=np.float64)
    Wt = np.asarray(Wt_prev, dtype=np.float64)
    if Q.shape[0] != Q.shape[1] or Q.shape[0] != Wt.shape[0]:
        raise ValueError("Q must be d x d and Wt_prev d x d_prev")
    return Q.T @ Wt


def rotate_topk_linear(x, Q, W_rot, K: int):
    """The three steps in the pages' order: rotate, keep the Top-K, multiply.

    Returns (y, idx, val, x_rot).
    """
    x_rot = rotate(x, Q)
    idx, val = topk(x_rot, K)
    y = sparse_linear(idx, val, W_rot)
    return y, idx, val, x_rot


_BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127
_BF16_MIN_NORMAL = 2.0 ** -126


def round_to_bf16(a) -> np.ndarray:
    """Round each value to the nearest bfloat16, ties to even; fp64 result.

    bfloat16 keeps 8 significant bits and fp32's exponent range.  A normal
    value a = m * 2^e (0.5 <= |m| < 1) rounds to rint(m * 2^8) * 2^(e-8); below
    the smallest normal the spacing is fixed at 2^-133; beyond the largest
    finite value the result is +-inf.
    """
    a = np.asarray(a, dtype=np.float64)
    m, e = np.frexp(a)
    out = np.ldexp(np.rint(m * 256.0), e - 8)
    tiny = np.abs(a) < _BF16_MIN_NORMAL
    if np.any(tiny):
        out = np.where(tiny, np.rint(a * 2.0 ** 133) * 2.0 ** -133, out)
    over = np.abs(out) > _BF16_MAX
    if np.any(over):
        out = np.where(over, np.copysign(np.inf, a), out)
    return out


def threshold_select(x, t: float) -> list[tuple[np.ndarray, np.ndarray]]:
    """Threshold sparsification: keep the entries with |x_j| >= t.

    R-Sparse report, 研究流程与方法 / R-Sparse框架设计 (input activation
    sparsification through a threshold function set from the sparsity
    budget).  The count kept varies per row, so one (idx, val) pair per row
    is returned, idx ascending.
    """
    xr, _ = _rows(x)
    out = []
    for m in range(xr.shape[0]):
        kept = np.nonzero(np.abs(xr[m]) >= t)[0]
        out.append((kept.astype(np.int64), xr[m, kept]))
    return out


def lowrank_factors(W, r: int) -> tuple[np.ndarray, np.ndarray]:
    """Rank-r factors of W from its SVD: A_r = U_r S_r^1/2, B_r = S_r^1/2 V_r^T.

    R-Sparse report, 研究流程与方法 / R-Sparse框架设计 (low-rank compensation
    module).  W is row-major [d_in, d_out] here, so A_r is [d_in, r], B_r is
    [r, d_out] and A_r . B_r is the best rank-r approximation of W.
    """
    W = np.asarray(W, dtype=np.float64)
    U, S, Vt = np.linalg.svd(W, full_matrices=False)
    root = np.sqrt(S[:r])
    return U[:, :r] * root[None, :], root[:, None] * Vt[:r, :]


def sparse_lowrank_linear(x, W, A_r, B_r, idx) -> np.ndarray:
    """Hybrid output y = y_s + y_r of one row.

    y_s multiplies the kept entries by their weight rows; y_r sends the
    dropped part (x - sigma(x)) through the low-rank factors, y_r =
    (x - sigma(x)) . A_r . B_r (R-Sparse report, R-Sparse框架设计, hybrid
    computation).
    """
    x = np.asarray(x, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    idx = np.asarray(idx)
    kept = np.zeros_like(x)
    kept[idx] = x[idx]
    dropped = x - kept
    y_s = kept[idx] @ W[idx]
    y_r = (dropped @ np.asarray(A_r, dtype=np.float64)) @ np.asarray(B_r, dtype=np.float64)
    return y_s + y_r
