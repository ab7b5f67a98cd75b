"""The oracle against its pins, and planted mistakes against the same pins.

Runs on the CPU only.  A planted mistake is a broken copy of one oracle
function defined here; each must fail at least one pin.
"""
import numpy as np
import pytest

import oracle
from tests import pins


def test_rotate_pins():
    pins.check_rotate(oracle.rotate)


def test_topk_pins():
    pins.check_topk(oracle.topk)


def test_sparse_linear_pins():
    pins.check_sparse_linear(oracle.sparse_linear)


def test_dense_linear_pins():
    pins.check_dense_linear(oracle.dense_linear)


def test_prepare_weights_pins():
    pins.check_prepare_weights(oracle.prepare_weights, oracle.rotate)


def test_fold_rotation_pins():
    pins.check_fold_rotation(oracle.fold_rotation, oracle.rotate)


def test_round_to_bf16_pins():
    pins.check_round_to_bf16(oracle.round_to_bf16)


def test_threshold_select_pins():
    pins.check_threshold_select(oracle.threshold_select, oracle.topk)


def test_lowrank_pins():
    pins.check_lowrank(oracle.lowrank_factors, oracle.sparse_lowrank_linear)


def test_generator_rotation_is_orthogonal():
    from synthdata import orthogonal
    for d, seed in ((8, 1), (64, 2), (256, 3)):
        Q = orthogonal(d, seed).numpy()
        assert np.max(np.abs(Q.T @ Q - np.eye(d))) < 1e-10
        assert np.max(np.abs(Q @ Q.T - np.eye(d))) < 1e-10


def test_composed_path_dense_equivalence_and_identity_rotation():
    from synthdata import orthogonal
    rng = np.random.default_rng(17)
    d, n = 64, 40
    Q = orthogonal(d, 4).numpy()
    W = rng.standard_normal((d, n))
    x = rng.standard_normal((2, d))
    W_rot = oracle.prepare_weights(Q, W)
    y, idx, val, x_rot = oracle.rotate_topk_linear(x, Q, W_rot, d)
    np.testing.assert_allclose(y, x @ W, rtol=0, atol=1e-10 * np.max(np.abs(x @ W)))
    # Q = I is the unrotated fixed-count selection (TEAL-style magnitude Top-K)
    y, idx, val, _ = oracle.rotate_topk_linear(x, np.eye(d), W, 25)
    for m in range(2):
        want = pins.brute_force_topk(x[m, :9], 4)  # spot-check the selection rule
        i9, _ = oracle.topk(x[m, :9], 4)
        assert tuple(i9) == want
        dense = np.zeros(d)
        dense[idx[m]] = x[m, idx[m]]
        np.testing.assert_allclose(y[m], dense @ W, rtol=1e-13, atol=1e-13)
        assert np.sum(dense != 0) == 25


def test_k_for_sparsity_rule():
    from synthdata import k_for_sparsity
    assert k_for_sparsity(256, 40) == 154
    assert k_for_sparsity(4096, 40) == 2458
    assert k_for_sparsity(11008, 40) == 6605
    assert k_for_sparsity(4096, 0) == 4096 and k_for_sparsity(4096, 100) == 0
    for d in (256, 4096, 5120, 8192, 11008, 13824, 28672):
        for s in (0, 25, 40, 50):
            K = k_for_sparsity(d, s)
            assert (d - K) / d <= s / 100 + 1e-12 and (d - K + 1) / d > s / 100


# ------------------------------------------------------------ planted mistakes

def _rotate_transposed(x, Q):
    return oracle.rotate(x, np.asarray(Q).T)


def _rotate_dropped_term(x, Q):
    Q = np.array(Q, dtype=np.float64)
    Q[-1, :] = 0.0
    return oracle.rotate(x, Q)


def _topk_signed(x, K):
    x = np.asarray(x, dtype=np.float64)
    single = x.ndim == 1
    X = x[None] if single else x
    idx = np.stack([np.sort(np.lexsort((np.arange(X.shape[1]), -row))[:K]) for row in X])
    val = np.take_along_axis(X, idx, axis=1)
    return (idx[0], val[0]) if single else (idx, val)


def _topk_high_index_wins(x, K):
    x = np.asarray(x, dtype=np.float64)
    single = x.ndim == 1
    X = x[None] if single else x
    d = X.shape[1]
    idx = np.stack([np.sort(np.lexsort((-np.arange(d), -np.abs(row)))[:K]) for row in X])
    val = np.take_along_axis(X, idx, axis=1)
    return (idx[0], val[0]) if single else (idx, val)


def _topk_magnitude_order(x, K):
    x = np.asarray(x, dtype=np.float64)
    single = x.ndim == 1
    X = x[None] if single else x
    d = X.shape[1]
    idx = np.stack([np.lexsort((np.arange(d), -np.abs(row)))[:K] for row in X])
    val = np.take_along_axis(X, idx, axis=1)
    return (idx[0], val[0]) if single else (idx, val)


def _topk_abs_values(x, K):
    idx, val = oracle.topk(x, K)
    return idx, np.abs(val)


def _sparse_linear_off_by_one(idx, val, W):
    W = np.asarray(W, dtype=np.float64)
    return oracle.sparse_linear(np.minimum(np.asarray(idx) + 1, W.shape[0] - 1), val, W)


def _sparse_linear_drops_last(idx, val, W):
    idx, val = np.asarray(idx), np.asarray(val, dtype=np.float64).copy()
    val[..., -1:] = 0.0
    return oracle.sparse_linear(idx, val, W)


def _prepare_untransposed(Q, W):
    return np.asarray(Q, dtype=np.float64) @ np.asarray(W, dtype=np.float64)


def _fold_untransposed(Q, Wt):
    return np.asarray(Q, dtype=np.float64) @ np.asarray(Wt, dtype=np.float64)


def _round_truncating(a):
    a = np.asarray(a, dtype=np.float64)
    m, e = np.frexp(a)
    return np.ldexp(np.trunc(m * 256.0), e - 8)


def _dense_drops_last_input(x, W):
    x = np.asarray(x, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    return x[..., :-1] @ W[:-1]


def _threshold_strict(x, t):
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    return [(np.nonzero(np.abs(r) > t)[0], r[np.abs(r) > t]) for r in x]


def _threshold_signed(x, t):
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    return [(np.nonzero(r >= t)[0], r[r >= t]) for r in x]


def _lowrank_full_spectrum(W, r):
    U, S, Vt = np.linalg.svd(np.asarray(W, dtype=np.float64), full_matrices=False)
    return U[:, :r] * S[None, :r], Vt[:r, :]


def _lowrank_subtracts(x, W, A_r, B_r, idx):
    x = np.asarray(x, dtype=np.float64)
    kept = np.zeros_like(x)
    kept[idx] = x[idx]
    return kept @ W - (x - kept) @ A_r @ B_r


def _lowrank_whole_input(x, W, A_r, B_r, idx):
    x = np.asarray(x, dtype=np.float64)
    kept = np.zeros_like(x)
    kept[idx] = x[idx]
    return kept @ W + x @ A_r @ B_r


@pytest.mark.parametrize("check, broken", [
    (pins.check_rotate, _rotate_transposed),
    (pins.check_rotate, _rotate_dropped_term),
    (pins.check_topk, _topk_signed),
    (pins.check_topk, _topk_high_index_wins),
    (pins.check_topk, _topk_magnitude_order),
    (pins.check_topk, _topk_abs_values),
    (pins.check_sparse_linear, _sparse_linear_off_by_one),
    (pins.check_sparse_linear, _sparse_linear_drops_last),
    (lambda f: pins.check_prepare_weights(f, oracle.rotate), _prepare_untransposed),
    (pins.check_round_to_bf16, _round_truncating),
    (lambda f: pins.check_fold_rotation(f, oracle.rotate), _fold_untransposed),
    (pins.check_dense_linear, _dense_drops_last_input),
    (lambda f: pins.check_threshold_select(f, oracle.topk), _threshold_strict),
    (lambda f: pins.check_threshold_select(f, oracle.topk), _threshold_signed),
    (lambda f: pins.check_lowrank(f, oracle.sparse_lowrank_linear), _lowrank_full_spectrum),
    (lambda f: pins.check_lowrank(oracle.lowrank_factors, f), _lowrank_subtracts),
    (lambda f: pins.check_lowrank(oracle.lowrank_factors, f), _lowrank_whole_input),
])
def test_planted_mistake_is_caught(check, broken):
    with pytest.raises(AssertionError):
        check(broken)
