"""Pins of the fp64 oracle: checks against facts fixed outside the oracle.

Each ``check_*`` function takes the oracle function it pins as an argument and
raises AssertionError when the function disagrees with a closed form, an
invariant, a library routine in a special case, a hand-derived example or a
brute-force enumeration.  ``test_oracle_pins.py`` runs them on the real
oracle, and also on deliberately broken copies to show that each plausible
mistake (a transposed operand, a dropped term, a wrong sign, a wrong index,
the wrong tie-break) trips at least one of them.
"""
from __future__ import annotations

import itertools
import json
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def golden(name: str) -> dict:
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def haar(d: int, seed: int) -> np.ndarray:
    from synthdata import orthogonal
    return orthogonal(d, seed).numpy()


# ----------------------------------------------------------------- rotation

def check_rotate(rotate) -> None:
    g = golden("hadamard4.json")
    np.testing.assert_allclose(rotate(np.array(g["x"]), np.array(g["Q"])), g["x_rot"], rtol=0, atol=1e-15)
    gv = golden("givens2.json")
    got = rotate(np.array(gv["x"]), np.array(gv["Q"]))
    np.testing.assert_allclose(got, gv["x_rot"], rtol=0, atol=1e-14)
    assert not np.allclose(got, gv["x_rot_if_transposed"])
    # permutation matrix: Q[p[j], j] = 1 moves x[p[j]] to position j exactly
    rng = np.random.default_rng(11)
    d = 17
    p = rng.permutation(d)
    P = np.zeros((d, d))
    P[p, np.arange(d)] = 1.0
    x = rng.standard_normal((3, d))
    assert np.array_equal(rotate(x, P), x[:, p])
    # identity
    assert np.array_equal(rotate(x, np.eye(d)), x)
    # norm preservation and inverse rotation by Q^T, Haar Q of width 64
    Q = haar(64, 5)
    x = rng.standard_normal((4, 64)) * 3.0
    xr = rotate(x, Q)
    np.testing.assert_allclose(np.linalg.norm(xr, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    np.testing.assert_allclose(rotate(xr, Q.T), x, rtol=0, atol=1e-12)
    # batch rows are rotated independently
    for m in range(x.shape[0]):
        np.testing.assert_allclose(rotate(x[m], Q), xr[m], rtol=0, atol=1e-13)


# ----------------------------------------------------------------- Top-K

def _dominates(mag: np.ndarray, S: tuple[int, ...]) -> bool:
    inside = set(S)
    for i in S:
        for j in range(len(mag)):
            if j in inside:
                continue
            if not (mag[i] > mag[j] or (mag[i] == mag[j] and i < j)):
                return False
    return True


def brute_force_topk(x: np.ndarray, K: int) -> tuple[int, ...]:
    """The unique K-subset S with every kept entry preferred to every dropped one."""
    mag = np.abs(x)
    found = [S for S in itertools.combinations(range(len(x)), K) if _dominates(mag, S)]
    assert len(found) == 1, "preference order must single out exactly one subset"
    return found[0]


def check_topk(topk) -> None:
    g = golden("hadamard4.json")
    for k, want in g["topk"].items():
        idx, val = topk(np.array(g["x_rot"]), int(k))
        assert list(idx) == want["idx"] and list(val) == want["val"], (k, idx, val)
    t = g["tie"]
    idx, val = topk(np.array(t["x_rot"]), t["K"])
    assert list(idx) == t["idx"] and list(val) == t["val"]
    rng = np.random.default_rng(3)
    # brute force on tiny vectors with forced ties, signed zeros and negatives
    for trial in range(60):
        d = int(rng.integers(1, 10))
        x = rng.integers(-3, 4, size=d).astype(np.float64)
        if trial % 3 == 0:
            x = rng.standard_normal(d)
        if trial % 5 == 0 and d > 1:
            x[rng.integers(0, d)] = -0.0
        for K in range(0, d + 1):
            idx, val = topk(x, K)
            want = brute_force_topk(x, K)
            assert tuple(int(i) for i in idx) == want, (x, K, idx, want)
            assert np.array_equal(val, x[list(want)])
    # all equal magnitudes with mixed signs: the lowest indices win
    x = np.array([-2.0, 2.0, -2.0, 2.0, 2.0, -2.0])
    idx, val = topk(x, 4)
    assert list(idx) == [0, 1, 2, 3] and list(val) == [-2.0, 2.0, -2.0, 2.0]
    # +0 and -0 tie; 1-ulp neighbours are not ties; subnormals are ordered
    x = np.array([0.0, -0.0, 0.0, 1.0])
    assert list(topk(x, 2)[0]) == [0, 3]
    one = 1.0
    up = np.nextafter(one, 2.0)
    x = np.array([one, -up, one, up])
    assert list(topk(x, 2)[0]) == [1, 3]
    tiny = np.array([5e-324, 1e-323, -5e-324, 0.0])
    assert list(topk(tiny, 2)[0]) == [0, 1]
    # per-row independence, exact count, ascending order, sign kept
    X = rng.standard_normal((5, 40))
    idx, val = topk(X, 13)
    for m in range(5):
        i1, v1 = topk(X[m], 13)
        assert np.array_equal(idx[m], i1) and np.array_equal(val[m], v1)
        assert len(set(idx[m].tolist())) == 13 and np.all(np.diff(idx[m]) > 0)
        assert np.array_equal(val[m], X[m, idx[m]])
    # scaling by a power of two keeps the set and scales the values exactly
    i2, v2 = topk(X * 2.0 ** 7, 13)
    assert np.array_equal(i2, idx) and np.array_equal(v2, val * 2.0 ** 7)
    # dropped mass equals the sum of the d-K smallest squares
    x = rng.standard_normal(50)
    idx, _ = topk(x, 20)
    keep = np.zeros(50, dtype=bool)
    keep[idx] = True
    np.testing.assert_allclose(np.sum(x[~keep] ** 2), np.sum(np.sort(x ** 2)[:30]), rtol=1e-14)
    # the extreme counts
    assert topk(x, 0)[0].shape == (0,)
    assert np.array_equal(topk(x, 50)[0], np.arange(50))


# ----------------------------------------------------------------- linear

def check_sparse_linear(sparse_linear) -> None:
    g = golden("hadamard4.json")
    for k, want in g["topk"].items():
        y = sparse_linear(np.array(want["idx"]), np.array(want["val"]), np.array(g["W_rot"]))
        np.testing.assert_allclose(y, want["y"], rtol=0, atol=1e-14)
    gv = golden("givens2.json")
    y = sparse_linear(np.array(gv["top1"]["idx"]), np.array(gv["top1"]["val"]), np.array(gv["W_rot"]))
    np.testing.assert_allclose(y, gv["top1"]["y"], rtol=0, atol=1e-13)
    rng = np.random.default_rng(8)
    d, n = 37, 23
    W = rng.standard_normal((d, n))
    x = rng.standard_normal(d)
    # K = d with every index: the plain matrix-vector product (library matmul)
    np.testing.assert_allclose(sparse_linear(np.arange(d), x, W), np.matmul(x, W), rtol=1e-13, atol=1e-13)
    # a subset equals the product of the zero-filled vector with W
    idx = np.sort(rng.choice(d, 11, replace=False))
    dense = np.zeros(d)
    dense[idx] = x[idx]
    np.testing.assert_allclose(sparse_linear(idx, x[idx], W), np.matmul(dense, W), rtol=1e-13, atol=1e-13)
    # each output column only sees the kept rows: one-hot rows of W
    E = np.zeros((d, d))
    E[np.arange(d), np.arange(d)] = 1.0
    np.testing.assert_array_equal(sparse_linear(idx, x[idx], E), dense)
    # empty selection gives zero; rows of a batch are independent
    assert np.array_equal(sparse_linear(np.zeros(0, dtype=np.int64), np.zeros(0), W), np.zeros(n))
    I2 = np.stack([idx, np.sort(rng.choice(d, 11, replace=False))])
    V2 = rng.standard_normal((2, 11))
    Y2 = sparse_linear(I2, V2, W)
    for m in range(2):
        np.testing.assert_allclose(Y2[m], sparse_linear(I2[m], V2[m], W), rtol=0, atol=0)


def check_dense_linear(dense_linear) -> None:
    g = golden("hadamard4.json")
    np.testing.assert_allclose(dense_linear(np.array(g["x"]), np.array(g["W"])), g["y_dense"], rtol=0, atol=0)
    gv = golden("givens2.json")
    np.testing.assert_allclose(dense_linear(np.array(gv["x"]), np.array(gv["W"])), gv["y_dense"], rtol=0, atol=0)
    rng = np.random.default_rng(9)
    W = rng.standard_normal((6, 5))
    e3 = np.zeros(6)
    e3[3] = 1.0
    assert np.array_equal(dense_linear(e3, W), W[3])


def check_prepare_weights(prepare_weights, rotate) -> None:
    g = golden("hadamard4.json")
    np.testing.assert_allclose(prepare_weights(np.array(g["Q"]), np.array(g["W"])), g["W_rot"], rtol=0, atol=1e-15)
    gv = golden("givens2.json")
    np.testing.assert_allclose(prepare_weights(np.array(gv["Q"]), np.array(gv["W"])), gv["W_rot"], rtol=0, atol=1e-14)
    rng = np.random.default_rng(12)
    d, n = 19, 7
    p = rng.permutation(d)
    P = np.zeros((d, d))
    P[p, np.arange(d)] = 1.0
    W = rng.standard_normal((d, n))
    # Q[p[i], i] = 1, so row i of Q^T W is row p[i] of W
    assert np.array_equal(prepare_weights(P, W), W[p])
    # dense equivalence: (x Q)(Q^T W) = x W for a Haar rotation
    Q = haar(48, 21)
    W = rng.standard_normal((48, 30))
    x = rng.standard_normal((3, 48))
    np.testing.assert_allclose(rotate(x, Q) @ prepare_weights(Q, W), x @ W, rtol=0, atol=1e-12)


def check_fold_rotation(fold_rotation, rotate) -> None:
    rng = np.random.default_rng(16)
    d, d_prev = 24, 10
    Wt = rng.standard_normal((d, d_prev))
    # the identity rotation leaves the producer unchanged
    assert np.array_equal(fold_rotation(np.eye(d), Wt), Wt)
    # a permutation Q[p[i], i] = 1 moves output channel p[i] to position i
    p = rng.permutation(d)
    P = np.zeros((d, d))
    P[p, np.arange(d)] = 1.0
    assert np.array_equal(fold_rotation(P, Wt), Wt[p])
    # the folded producer delivers the rotated input: h Wt_fold^T = (h Wt^T) Q
    Q = haar(d, 22)
    h = rng.standard_normal((3, d_prev))
    np.testing.assert_allclose(h @ fold_rotation(Q, Wt).T, rotate(h @ Wt.T, Q), rtol=0, atol=1e-12)
    # a 2 x 2 Givens rotation by hand: Q = [[c, -s], [s, c]] gives rows
    # (c w0 + s w1, -s w0 + c w1)
    c, sn = 0.6, 0.8
    G = np.array([[c, -sn], [sn, c]])
    w = np.array([[1.0, 2.0], [3.0, -1.0]])
    np.testing.assert_allclose(fold_rotation(G, w), [[c * 1 + sn * 3, c * 2 + sn * -1],
                                                      [-sn * 1 + c * 3, -sn * 2 + c * -1]], rtol=0, atol=1e-15)


def check_round_to_bf16(round_to_bf16) -> None:
    import torch
    rng = np.random.default_rng(4)
    a = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(2000) * 1e-39).astype(np.float32),
        (rng.standard_normal(2000) * 1e36).astype(np.float32),
        np.array([0.0, -0.0, 1.0, -1.0, 3.3895314e38, 1e-45], dtype=np.float32),
    ])
    # values exactly halfway between two bfloat16 neighbours
    halves = (np.arange(128, 256, dtype=np.float64) + 0.5) / 128.0
    a = np.concatenate([a, halves.astype(np.float32), -halves.astype(np.float32)])
    want = torch.from_numpy(a).to(torch.bfloat16).to(torch.float64).numpy()
    got = round_to_bf16(a.astype(np.float64))
    assert np.array_equal(got, want)
    # closed forms: 1 + 2^-8 is halfway between 1 and 1 + 2^-7, ties to even (1)
    assert round_to_bf16(np.array([1.0 + 2.0 ** -8]))[0] == 1.0
    assert round_to_bf16(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 1.0 + 2.0 ** -6
    assert round_to_bf16(np.array([1.0 + 2.0 ** -8 + 2.0 ** -30]))[0] == 1.0 + 2.0 ** -7


# ------------------------------------------------------------ R-Sparse parts

def check_threshold_select(threshold_select, topk) -> None:
    rng = np.random.default_rng(14)
    x = rng.standard_normal((3, 30))
    for (idx, val), row in zip(threshold_select(x, 0.0), x):
        assert np.array_equal(idx, np.arange(30)) and np.array_equal(val, row)
    for (idx, _), row in zip(threshold_select(x, 1e9), x):
        assert idx.size == 0
    # with distinct magnitudes, t = the K-th largest magnitude keeps the Top-K set
    for row in x:
        K = 12
        t = np.sort(np.abs(row))[::-1][K - 1]
        (idx, val), = threshold_select(row, t)
        ti, tv = topk(row, K)
        assert np.array_equal(idx, ti) and np.array_equal(val, tv)
    # the boundary is inclusive
    (idx, _), = threshold_select(np.array([0.5, -1.0, 2.0]), 1.0)
    assert list(idx) == [1, 2]


def check_lowrank(lowrank_factors, sparse_lowrank_linear) -> None:
    rng = np.random.default_rng(15)
    W = rng.standard_normal((20, 12))
    A, B = lowrank_factors(W, 12)
    np.testing.assert_allclose(A @ B, W, rtol=0, atol=1e-12)
    S = np.linalg.svd(W, compute_uv=False)
    for r in (1, 4, 9):
        A, B = lowrank_factors(W, r)
        assert A.shape == (20, r) and B.shape == (r, 12)
        # Eckart-Young: the Frobenius error is the energy of the dropped spectrum
        np.testing.assert_allclose(np.linalg.norm(W - A @ B) ** 2, np.sum(S[r:] ** 2), rtol=1e-10)
        # both factors carry the square root of the spectrum
        np.testing.assert_allclose(np.linalg.norm(A, axis=0), np.sqrt(S[:r]), rtol=1e-12)
    x = rng.standard_normal(20)
    idx = np.sort(rng.choice(20, 8, replace=False))
    A, B = lowrank_factors(W, 12)
    # full rank: the compensation restores the dense product
    np.testing.assert_allclose(sparse_lowrank_linear(x, W, A, B, idx), x @ W, rtol=0, atol=1e-12)
    # rank 0: only the sparse part
    A0, B0 = np.zeros((20, 0)), np.zeros((0, 12))
    dense = np.zeros(20)
    dense[idx] = x[idx]
    np.testing.assert_allclose(sparse_lowrank_linear(x, W, A0, B0, idx), dense @ W, rtol=0, atol=1e-12)
