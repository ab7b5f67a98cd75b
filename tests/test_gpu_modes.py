"""Parity of the comparison modes with the fp64 oracle, through the C ABI:

* threshold selection |x| >= t (R-Sparse report, R-Sparse框架设计): the kept
  lists and counts bit-exact on given fp32 rows, including ties at t, +-0,
  subnormals, t <= 0 and t = +Inf;
* the fused rotate -> threshold -> sparse linear call (one token: the
  cooperative kernel in threshold mode; several tokens: the composed path);
* the identity rotation (no Q): fixed-K and threshold selection on x itself,
  where the selection is exact because x_rot = x.

Bars as in test_gpu_parity: x_rot within the fp32 summation bound of the
exact rotation, the kept set exactly the selection of the path's own fp32
x_rot and valid against the exact rotation outside a band of the bound's
width around t, y within 2e-3 of the oracle's product on that set.
"""
import numpy as np
import pytest
import torch

import oracle
import synthdata as sd
from tests.test_gpu_parity import U, Y_TOL, check_selection, f64, rel_inf, status

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    from activation_sparsity_b200 import build_lib
    build_lib.build()
    import activation_sparsity_b200 as L
    torch.cuda.init()
    return L


def f32(v: float) -> float:
    return float(np.float32(v))


# ---------------------------------------------------------------- threshold selection

SIZES = [(1, 1), (3, 7), (2, 256), (4, 1000), (1, 4096), (2, 11008), (1, 32768), (16, 512)]


def thresholds(x: np.ndarray) -> list[float]:
    mag = np.abs(x[0])
    srt = np.sort(mag)
    mid = srt[len(srt) // 2]  # an exact magnitude of the row: a tie at t
    return sorted({0.0, -1.0, f32(mid), f32(srt[-1]), f32(mid * 1.0000001), float("inf"), 1e-40, 1e30})


@pytest.mark.parametrize("kind", sd.ADVERSARIAL_KINDS)
@pytest.mark.parametrize("M,d", SIZES)
def test_threshold_bit_exact(L, kind, M, d):
    x = sd.adversarial_rows(kind, M, d, 700 + d)
    xd = x.cuda()
    xn = x.double().numpy()
    for t in thresholds(xn):
        st = status()
        idx, val, nnz = L.larosa_threshold(xd, t, dev_status=st)
        assert L.larosa_check(st) == 0
        want = oracle.threshold_select(xn, f32(t))
        n = nnz.cpu().numpy()
        gi = idx.cpu().numpy()
        gv = val.cpu().numpy()
        for m in range(M):
            wi, wv = want[m]
            assert n[m] == len(wi), (kind, d, t)
            assert np.array_equal(gi[m, :n[m]], wi), (kind, d, t)
            assert np.array_equal(gv[m, :n[m]].view(np.uint32), wv.astype(np.float32).view(np.uint32))


def test_threshold_reports_nonfinite(L):
    x = sd.adversarial_rows("gaussian", 2, 300, 5)
    x[1, 17] = float("nan")
    st = status()
    _, _, nnz = L.larosa_threshold(x.cuda(), 0.5, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & 0x1
    assert 0 <= int(nnz[1].item()) <= 300


# ---------------------------------------------------------------- fused threshold path

def threshold_outputs(L, x, Qt, W, t):
    M, d_in = x.shape
    d_out = W.shape[1]
    ws = L.Workspace()
    buf = ws.get(M, d_in, d_out, d_in)
    st = status()
    y = L.larosa_rotate_threshold_linear(x, Qt, W, t, ws=ws, dev_status=st)
    assert L.larosa_check(st) == 0
    o_x, o_i, o_v = L.larosa_workspace_layout(M, d_in, d_out, d_in)
    o_n = L.larosa_workspace_nnz_offset(M, d_in, d_out, d_in)
    x_rot = buf[o_x:o_x + M * d_in * 4].view(torch.float32).view(M, d_in)
    idx = buf[o_i:o_i + M * d_in * 4].view(torch.int32).view(M, d_in)
    val = buf[o_v:o_v + M * d_in * 4].view(torch.float32).view(M, d_in)
    nnz = buf[o_n:o_n + M * 4].view(torch.int32)
    return (f64(y), f64(x_rot), idx.cpu().numpy().astype(np.int64), val.cpu().numpy(),
            nnz.cpu().numpy().astype(np.int64))


def check_threshold_path(x_rot, x_rot_ref, gamma, idx, val, nnz, t):
    M, d = x_rot.shape
    for m in range(M):
        # exactly the threshold selection of the path's own fp32 x_rot
        (wi, wv), = oracle.threshold_select(x_rot[m], t)
        assert nnz[m] == len(wi)
        assert np.array_equal(idx[m, :nnz[m]], wi)
        assert np.array_equal(val[m, :nnz[m]], wv.astype(np.float32))
        # against the exact rotation: only entries within the bound of t may differ
        kept = np.zeros(d, dtype=bool)
        kept[wi] = True
        mag = np.abs(x_rot_ref[m])
        assert np.all(kept[mag >= t + gamma[m] + 1e-30])
        assert not np.any(kept[mag < t - gamma[m] - 1e-30])


@pytest.mark.parametrize("dtype,M,d_in,d_out,drop", [
    (torch.float32, 1, 256, 512, 40),
    (torch.bfloat16, 1, 1024, 1032, 40),
    (torch.bfloat16, 1, 4096, 4096, 40),
    (torch.bfloat16, 1, 11008, 4096, 50),
    (torch.bfloat16, 1, 200, 24, 50),
    (torch.bfloat16, 4, 1024, 1032, 40),
    (torch.bfloat16, 16, 512, 256, 25),
    (torch.bfloat16, 1, 1024, 1032, 0),
    (torch.bfloat16, 1, 1024, 1032, 100),
    # several bf16 tokens: the tensor-core product with the threshold
    # kernel's coefficient rows (everything kept, nothing kept, the 7B shape)
    (torch.bfloat16, 2, 1024, 1032, 0),
    (torch.bfloat16, 4, 1024, 1032, 100),
    (torch.bfloat16, 8, 4096, 4096, 40),
    # several fp32 tokens: the union of the kept rows, row-streamed
    (torch.float32, 4, 256, 512, 50),
])
def test_fused_threshold(L, dtype, M, d_in, d_out, drop):
    Q = sd.orthogonal(d_in, 801, device="cuda" if d_in > 4096 else "cpu").to(dtype).cpu()
    W = sd.weights(d_in, d_out, 0.02 if dtype == torch.bfloat16 else 1 / 16, 802, dtype)
    x = sd.activations(M, d_in, 803, dtype)
    Qt = Q.t().contiguous().cuda()
    W_rot = L.larosa_prepare_weights(Qt, W.cuda())
    xq, qq = f64(x), f64(Q)
    x_rot_ref = oracle.rotate(xq, qq)
    gamma = (d_in + 2) * U * (np.abs(xq) @ np.abs(qq))
    # t drops about drop % of the first token's exact magnitudes (0: t = 0, 100: t = +Inf)
    mag = np.sort(np.abs(x_rot_ref[0]))
    t = 0.0 if drop == 0 else float("inf") if drop == 100 else f32(mag[int(len(mag) * drop / 100)])
    y, x_rot, idx, val, nnz = threshold_outputs(L, x.cuda(), Qt, W_rot, t)
    assert np.all(np.abs(x_rot - x_rot_ref) <= gamma + 1e-30)
    check_threshold_path(x_rot, x_rot_ref, gamma, idx, val, nnz, t)
    W_rot_ref = oracle.prepare_weights(qq, f64(W))
    if dtype == torch.bfloat16:
        W_rot_ref = oracle.round_to_bf16(W_rot_ref)
    ref = np.stack([oracle.sparse_linear(idx[m, :nnz[m]], x_rot_ref[m, idx[m, :nnz[m]]], W_rot_ref)
                    for m in range(M)])
    if drop == 100:
        assert np.all(y == 0.0) and np.all(nnz == 0)
    else:
        assert rel_inf(y, ref) <= Y_TOL


# ---------------------------------------------------------------- the identity rotation

@pytest.mark.parametrize("dtype,M,d_in,d_out,sparsity", [
    (torch.float32, 1, 256, 512, 40),
    (torch.bfloat16, 1, 200, 24, 50),
    (torch.bfloat16, 1, 4096, 4096, 40),
    (torch.bfloat16, 1, 11008, 4096, 40),
    (torch.bfloat16, 4, 1024, 1032, 40),
])
def test_fused_identity_topk(L, dtype, M, d_in, d_out, sparsity):
    K = sd.k_for_sparsity(d_in, sparsity)
    W = sd.weights(d_in, d_out, 0.02 if dtype == torch.bfloat16 else 1 / 16, 902, dtype)
    x = sd.activations(M, d_in, 903, dtype)
    ws = L.Workspace()
    buf = ws.get(M, d_in, d_out, K)
    st = status()
    y = L.larosa_rotate_topk_linear(x.cuda(), None, W.cuda(), K, ws=ws, dev_status=st)
    assert L.larosa_check(st) == 0
    o_x, o_i, o_v = L.larosa_workspace_layout(M, d_in, d_out, K)
    x_rot = f64(buf[o_x:o_x + M * d_in * 4].view(torch.float32).view(M, d_in))
    idx = buf[o_i:o_i + M * K * 4].view(torch.int32).view(M, K).cpu().numpy().astype(np.int64)
    xq = f64(x)
    # the identity rotation: x_rot is x itself, so the selection is exact
    assert np.array_equal(x_rot, xq)
    want_i, want_v = oracle.topk(xq, K)
    assert np.array_equal(idx, want_i.reshape(M, K))
    ref = np.stack([oracle.sparse_linear(want_i.reshape(M, K)[m], want_v.reshape(M, K)[m], f64(W))
                    for m in range(M)])
    assert rel_inf(f64(y), ref) <= Y_TOL


def crowded_row(d: int, n_high: int, n_bin: int, width: float, seed: int, dtype) -> np.ndarray:
    """One row whose Top-K boundary falls inside a crowded 12-bit key bin.

    n_high magnitudes in [2, 4) (certainly kept), n_bin in [1, 1 + width)
    (one bin of bits 30..19 when width <= 1/16), the rest in [0, 0.5); random
    signs and positions.  Rounded to ``dtype``, so bf16 rows carry ties.
    """
    rng = np.random.default_rng(seed)
    mag = rng.uniform(0.0, 0.5, d)
    pos = rng.permutation(d)
    mag[pos[:n_high]] = rng.uniform(2.0, 4.0, n_high)
    mag[pos[n_high:n_high + n_bin]] = 1.0 + rng.uniform(0.0, width, n_bin)
    x = mag * rng.choice([-1.0, 1.0], d)
    return torch.from_numpy(x[None, :]).to(dtype)


@pytest.mark.parametrize("dtype,d,n_high,n_bin,width", [
    (torch.float32, 4096, 500, 2000, 1 / 16),       # B holds 2000 keys: one sub-bin of ~8 is ranked
    (torch.float32, 4096, 300, 1500, 1 / 4096),     # 1500 keys within one sub-bin: the bisection decides
    (torch.bfloat16, 8192, 1000, 2400, 1 / 16),     # bf16: 8 distinct keys in B, hundreds of ties each
    (torch.bfloat16, 28672, 2000, 3600, 1 / 16),    # the 70B down-projection width
])
def test_fused_identity_crowded_boundary_bin(L, dtype, d, n_high, n_bin, width):
    """The selector where the boundary bin holds more keys than its candidate slots."""
    d_out = 512
    W = sd.weights(d, d_out, 0.02 if dtype == torch.bfloat16 else 1 / 16, 922, dtype)
    x = crowded_row(d, n_high, n_bin, width, 923, dtype)
    xq = f64(x)
    for K in (n_high + 1, n_high + n_bin // 3, n_high + n_bin - 1):
        ws = L.Workspace()
        buf = ws.get(1, d, d_out, K)
        st = status()
        y = L.larosa_rotate_topk_linear(x.cuda(), None, W.cuda(), K, ws=ws, dev_status=st)
        assert L.larosa_check(st) == 0
        o_x, o_i, _ = L.larosa_workspace_layout(1, d, d_out, K)
        assert np.array_equal(f64(buf[o_x:o_x + d * 4].view(torch.float32).view(1, d)), xq)
        idx = buf[o_i:o_i + K * 4].view(torch.int32).cpu().numpy().astype(np.int64)
        want_i, want_v = oracle.topk(xq, K)
        assert np.array_equal(idx, want_i.reshape(K)), K
        ref = oracle.sparse_linear(want_i.reshape(K), want_v.reshape(K), f64(W))
        assert rel_inf(f64(y)[0], ref) <= Y_TOL


@pytest.mark.parametrize("dtype,M,d_in,d_out", [
    (torch.bfloat16, 1, 4096, 4096),
    (torch.bfloat16, 1, 11008, 4096),
    (torch.bfloat16, 4, 1024, 1032),
])
def test_fused_identity_threshold(L, dtype, M, d_in, d_out):
    W = sd.weights(d_in, d_out, 0.02, 912, dtype)
    x = sd.activations(M, d_in, 913, dtype)
    xq = f64(x)
    t = f32(np.sort(np.abs(xq[0]))[int(0.4 * d_in)])
    y, x_rot, idx, val, nnz = threshold_outputs(L, x.cuda(), None, W.cuda(), t)
    assert np.array_equal(x_rot, xq)
    want = oracle.threshold_select(xq, t)
    for m in range(M):
        wi, wv = want[m]
        assert nnz[m] == len(wi) and np.array_equal(idx[m, :nnz[m]], wi)
    ref = np.stack([oracle.sparse_linear(want[m][0], want[m][1], f64(W)) for m in range(M)])
    assert rel_inf(y, ref) <= Y_TOL


def test_identity_topk_matches_rotated_path_with_identity_q(L):
    """Qt = NULL and an explicit identity Qt select the same set and give the same y."""
    d_in, d_out, K = 1024, 1032, 600
    W = sd.weights(d_in, d_out, 0.02, 922, torch.bfloat16).cuda()
    x = sd.activations(1, d_in, 923, torch.bfloat16).cuda()
    eye = torch.eye(d_in, dtype=torch.bfloat16, device="cuda")
    y0 = L.larosa_rotate_topk_linear(x, None, W, K)
    y1 = L.larosa_rotate_topk_linear(x, eye, L.larosa_prepare_weights(eye, W), K)
    assert rel_inf(f64(y0), f64(y1)) <= 1e-6


# ---------------------------------------------------------------- folded rotation

@pytest.mark.parametrize("d_prev,d,d_out", [(1024, 4096, 4096), (4096, 11008, 4096)])
def test_folded_rotation_path(L, d_prev, d, d_out):
    """Q folded into the producing layer; the consumer runs with the identity rotation."""
    from tests.test_gpu_parity import check_bf16_rounding
    K = sd.k_for_sparsity(d, 40.0)
    Q = sd.orthogonal(d, 951, device="cuda" if d > 4096 else "cpu").to(torch.bfloat16).cpu()
    Qt = Q.t().contiguous().cuda()
    Wt_prev = sd.weights(d, d_prev, 0.02, 952, torch.bfloat16)  # producer, nn.Linear layout [d, d_prev]
    W = sd.weights(d, d_out, 0.02, 953, torch.bfloat16)
    h = sd.activations(1, d_prev, 954, torch.bfloat16)
    # offline: fold Q into the producer, counter-rotate the consumer
    Wt_fold = L.larosa_fold_rotation(Qt, Wt_prev.cuda())
    W_rot = L.larosa_prepare_weights(Qt, W.cuda())
    qq, wp = f64(Q), f64(Wt_prev)
    exact_fold = oracle.fold_rotation(qq, wp)
    cols = np.random.default_rng(955).choice(d_prev, size=32, replace=False)
    check_bf16_rounding(f64(Wt_fold)[:, cols], exact_fold[:, cols],
                        (d + 2) * U * (np.abs(qq).T @ np.abs(wp[:, cols])))
    # per token: the producer emits x . Q (rounded to bf16, as a layer output)
    x_rot = L.larosa_dense_linear(h.cuda(), Wt_fold).to(torch.bfloat16)
    ws = L.Workspace()
    buf = ws.get(1, d, d_out, K)
    st = status()
    y = L.larosa_rotate_topk_linear(x_rot, None, W_rot, K, ws=ws, dev_status=st)
    assert L.larosa_check(st) == 0
    _, o_i, _ = L.larosa_workspace_layout(1, d, d_out, K)
    idx = buf[o_i:o_i + K * 4].view(torch.int32).cpu().numpy().astype(np.int64)
    xr = f64(x_rot)[0]
    want_i, want_v = oracle.topk(xr, K)
    assert np.array_equal(idx, want_i)
    W_rot_ref = oracle.round_to_bf16(oracle.prepare_weights(qq, f64(W)))
    assert rel_inf(f64(y)[0], oracle.sparse_linear(want_i, want_v, W_rot_ref)) <= Y_TOL
    # the unfolded path on the exact values keeps nearly the same rows: only
    # entries within the rounding of the fold and of the bf16 output differ
    x_exact = oracle.rotate(f64(h) @ wp.T, qq)[0]
    exact_i, _ = oracle.topk(x_exact, K)
    assert len(np.intersect1d(idx, exact_i)) >= 0.95 * K


# ---------------------------------------------------------------- sparse + low rank

@pytest.mark.parametrize("dtype,M,d_in,d_out,r,sparsity", [
    (torch.float32, 1, 256, 512, 32, 40),
    (torch.bfloat16, 1, 512, 256, 64, 40),
    (torch.bfloat16, 4, 1024, 1032, 128, 50),
    (torch.bfloat16, 16, 512, 256, 64, 40),
    (torch.bfloat16, 1, 4096, 4096, 256, 40),
    (torch.bfloat16, 2, 200, 24, 16, 0),
    # several bf16 tokens with both factor products on the tensor cores
    (torch.bfloat16, 8, 2048, 2048, 256, 40),
    (torch.bfloat16, 3, 2048, 1032, 64, 50),
    (torch.bfloat16, 4, 1024, 1032, 128, 100),
    # one token, one launch: every entry dropped, none dropped, ranks that are
    # not powers of two, the down projection's width, a width over 16384 (a
    # factor CTA covers at most 4096 entries of x), every entry of the down
    # width dropped (the factor CTAs at their cap of 64), the largest rank of
    # the one-launch kernel in both weight types
    (torch.bfloat16, 1, 1024, 1032, 40, 100),
    (torch.bfloat16, 1, 1024, 1032, 40, 0),
    (torch.float32, 1, 1000, 264, 72, 50),
    (torch.bfloat16, 1, 11008, 4096, 256, 40),
    (torch.bfloat16, 1, 4096, 12288, 8, 40),
    (torch.bfloat16, 1, 20000, 264, 64, 40),
    (torch.bfloat16, 1, 11008, 1024, 256, 100),
    (torch.bfloat16, 1, 2048, 2048, 2048, 40),
    (torch.float32, 1, 2048, 2048, 2048, 50),
])
def test_sparse_lowrank_linear(L, dtype, M, d_in, d_out, r, sparsity):
    """y = y_s + (x - sigma(x)) A_r B_r against the oracle on the same factors."""
    K = sd.k_for_sparsity(d_in, sparsity)
    W = sd.weights(d_in, d_out, 0.02 if dtype == torch.bfloat16 else 1 / 16, 1002, dtype)
    A64, B64 = oracle.lowrank_factors(f64(W), r)
    A = torch.from_numpy(A64).to(dtype)
    B = torch.from_numpy(B64).to(dtype)
    x = sd.activations(M, d_in, 1003, torch.float32)
    xq = f64(x)
    idx, val = oracle.topk(xq, K)
    idx, val = idx.reshape(M, K), val.reshape(M, K)
    st = status()
    y = L.larosa_sparse_lowrank_linear(x.cuda(), torch.from_numpy(idx.astype(np.int32)).cuda(),
                                       torch.from_numpy(val.astype(np.float32)).cuda(), W.cuda(),
                                       A.cuda(), B.cuda(), dev_status=st)
    assert L.larosa_check(st) == 0
    ref = np.stack([oracle.sparse_lowrank_linear(xq[m], f64(W), f64(A), f64(B), idx[m]) for m in range(M)])
    assert rel_inf(f64(y), ref) <= Y_TOL


def test_sparse_lowrank_one_launch_repeats_on_one_workspace(L):
    """The one-token kernel leaves its counters at zero: calls with different
    kept lists on one workspace each match the oracle, and repeat bit for bit."""
    d_in, d_out, r = 4096, 4096, 256
    K = sd.k_for_sparsity(d_in, 40)
    W = sd.weights(d_in, d_out, 0.02, 1012, torch.bfloat16)
    A64, B64 = oracle.lowrank_factors(f64(W), r)
    A, B = torch.from_numpy(A64).to(torch.bfloat16).cuda(), torch.from_numpy(B64).to(torch.bfloat16).cuda()
    Wd = W.cuda()
    ws = torch.zeros(L.larosa_lowrank_workspace_bytes(1, d_in, d_out, K, r), dtype=torch.uint8, device="cuda")
    st = status()
    first = None
    for call in range(3):
        x = sd.activations(1, d_in, 1013 + (call % 2), torch.float32)
        xq = f64(x)
        idx, val = oracle.topk(xq, K)
        y = L.larosa_sparse_lowrank_linear(x.cuda(), torch.from_numpy(idx.reshape(1, K).astype(np.int32)).cuda(),
                                           torch.from_numpy(val.reshape(1, K).astype(np.float32)).cuda(), Wd,
                                           A, B, ws=ws, dev_status=st)
        assert L.larosa_check(st) == 0
        ref = oracle.sparse_lowrank_linear(xq[0], f64(W), f64(A), f64(B), idx.reshape(K))
        assert rel_inf(f64(y)[0], ref) <= Y_TOL, call
        if call == 0:
            first = y.clone()
        elif call == 2:
            assert torch.equal(y, first)  # same inputs as call 0
