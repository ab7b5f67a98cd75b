"""Parity of every C-ABI entry point with the fp64 oracle, on a CUDA device.

Inputs come from the seeded generators in ``synthdata``; the oracle sees the
same values widened to fp64.  Bars:

* Top-K on given fp32 rows: indices and values bit-exact.
* Sparse / dense linear, rotation: within the fp32 summation bound
  (n + 2) * 2^-24 * sum_i |a_i b_i| per output, and y within 2e-3 of
  max |y_ref| (the stated tolerance for bf16 weights with fp32 accumulation).
* Weight counter-rotation: >= 99.9 % of bf16 outputs identical to the
  round-to-nearest-even of the exact fp64 product, each within the fp32
  summation bound plus half a bf16 ulp of it.
* Fused path: its intermediate x_rot within the summation bound of the exact
  rotation; its kept set a valid Top-K of the exact rotation up to twice that
  bound (rows whose magnitudes differ by less are interchangeable); y within
  2e-3 of the oracle's product on that set.
"""
import numpy as np
import pytest
import torch

import oracle
import synthdata as sd

pytestmark = pytest.mark.gpu

U = 2.0 ** -24
Y_TOL = 2e-3


@pytest.fixture(scope="module")
def L():
    from activation_sparsity_b200 import build_lib
    build_lib.build()
    import activation_sparsity_b200 as L
    torch.cuda.init()
    return L


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().double().numpy()


def rel_inf(got, ref) -> float:
    scale = np.max(np.abs(ref))
    return float(np.max(np.abs(got - ref)) / scale) if scale > 0 else float(np.max(np.abs(got)))


def status():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    _, e = np.frexp(np.abs(v))
    return np.ldexp(1.0, e - 8)


def check_bf16_rounding(got: np.ndarray, exact: np.ndarray, gamma: np.ndarray,
                        min_same: float = 0.999) -> None:
    """got is the bf16 rounding of an fp32-accumulated value within gamma of exact.

    Every element must lie within gamma plus half a bf16 ulp of the exact
    product.  At least min_same of them must equal its round-to-nearest-even
    (a wrong rounding mode would miss about half): the fp32 sum lands on the
    other side of a bf16 rounding midpoint only when the exact value lies
    within the accumulation error of one, which grows with the length of the
    sum.
    """
    want = oracle.round_to_bf16(exact)
    same = got == want
    assert same.mean() >= min_same, same.mean()
    assert np.all(np.abs(got - exact) <= gamma + 0.5 * bf16_ulp(got) + 1e-30)


# ---------------------------------------------------------------- prepare

@pytest.mark.parametrize("dtype,d,n", [
    (torch.float32, 256, 512),
    (torch.bfloat16, 256, 1032),
    (torch.bfloat16, 1000, 264),
    (torch.bfloat16, 130, 8),
])
def test_prepare_weights(L, dtype, d, n):
    Q = sd.orthogonal(d, 101).to(dtype)
    W = sd.weights(d, n, 0.02, 102, dtype)
    W_rot = L.larosa_prepare_weights(Q.t().contiguous().cuda(), W.cuda())
    torch.cuda.synchronize()
    exact = oracle.prepare_weights(f64(Q), f64(W))
    got = f64(W_rot)
    if dtype == torch.float32:
        bound = (d + 2) * U * (np.abs(f64(Q)).T @ np.abs(f64(W)))
        assert np.all(np.abs(got - exact) <= bound)
    else:
        check_bf16_rounding(got, exact, (d + 2) * U * (np.abs(f64(Q)).T @ np.abs(f64(W))))


# ---------------------------------------------------------------- rotate

@pytest.mark.parametrize("dtype,M,d", [
    (torch.float32, 1, 256),
    (torch.bfloat16, 1, 256),
    (torch.bfloat16, 3, 1000),
    (torch.bfloat16, 16, 512),
    (torch.float32, 5, 1024),
    (torch.bfloat16, 8, 2048),
    (torch.bfloat16, 1, 4096),
    (torch.bfloat16, 2, 11008),
    (torch.bfloat16, 16, 4096),   # activations too large for shared memory
    (torch.float32, 16, 2048),
    (torch.bfloat16, 1, 28672),
    (torch.bfloat16, 1, 8),
])
def test_rotate(L, dtype, M, d):
    if d > 4096:
        Q = sd.orthogonal(d, 201, device="cuda").to(dtype)
    else:
        Q = sd.orthogonal(d, 201).to(dtype).cuda()
    x = sd.activations(M, d, 202, dtype)
    got = f64(L.larosa_rotate(x.cuda(), Q.t().contiguous()))
    xq, qq = f64(x), f64(Q)
    ref = oracle.rotate(xq, qq)
    bound = (d + 2) * U * (np.abs(xq) @ np.abs(qq))
    assert np.all(np.abs(got - ref) <= bound + 1e-30)


# ---------------------------------------------------------------- Top-K

TOPK_SIZES = [(1, 1), (3, 7), (2, 256), (4, 1000), (1, 4096), (2, 11008), (1, 32768), (16, 512)]


@pytest.mark.parametrize("kind", sd.ADVERSARIAL_KINDS)
@pytest.mark.parametrize("M,d", TOPK_SIZES)
def test_topk_bit_exact(L, kind, M, d):
    x = sd.adversarial_rows(kind, M, d, 300 + d)
    xd = x.cuda()
    for K in sorted({0, 1, max(0, d // 3), d - 1, d, sd.k_for_sparsity(d, 40)}):
        if K < 0:
            continue
        st = status()
        idx, val = L.larosa_topk(xd, K, dev_status=st)
        assert L.larosa_check(st) == 0
        want_i, want_v = oracle.topk(x.double().numpy(), K)
        got_i = idx.cpu().numpy().astype(np.int64)
        assert np.array_equal(got_i, want_i.reshape(M, K)), (kind, d, K)
        got_v = val.cpu().numpy()
        want_v32 = want_v.reshape(M, K).astype(np.float32)
        assert np.array_equal(got_v.view(np.uint32), want_v32.view(np.uint32)), (kind, d, K)


def test_topk_reports_nonfinite(L):
    x = sd.adversarial_rows("gaussian", 2, 512, 7)
    x[1, 100] = float("nan")
    x[1, 5] = float("inf")
    st = status()
    idx, _ = L.larosa_topk(x.cuda(), 200, dev_status=st)
    flags = int(st.item())
    assert flags & 0x1
    i = idx.cpu().numpy()
    assert np.all((i >= 0) & (i < 512))
    # the finite row is still exact
    want_i, _ = oracle.topk(x[0].double().numpy(), 200)
    assert np.array_equal(i[0], want_i)


# ---------------------------------------------------------------- linear

SPARSE_CASES = [
    (torch.float32, 1, 256, 512, 154),
    (torch.float32, 1, 256, 512, 256),
    (torch.bfloat16, 1, 64, 8, 0),
    (torch.bfloat16, 1, 64, 8, 64),
    (torch.bfloat16, 1, 1000, 1032, 600),
    (torch.bfloat16, 1, 4096, 4096, 2458),
    (torch.bfloat16, 1, 4096, 12288, 2458),
    (torch.bfloat16, 1, 11008, 4096, 6605),
    (torch.bfloat16, 2, 512, 520, 300),
    (torch.bfloat16, 4, 1024, 2048, 400),
    (torch.bfloat16, 8, 512, 1024, 100),
    (torch.bfloat16, 16, 512, 256, 300),
    (torch.float32, 3, 300, 100, 50),
    # few rows kept per token: two and four tokens stream the union of their
    # kept rows instead of the dense product; eight and sixteen stay dense
    (torch.bfloat16, 2, 4096, 2048, 205),
    (torch.bfloat16, 4, 4096, 1032, 123),
    (torch.bfloat16, 8, 4096, 1024, 205),
    (torch.bfloat16, 16, 2048, 512, 41),
    # one-token stream-K edge shapes: fewer units than SMs, one tile, ragged tiles
    (torch.bfloat16, 1, 64, 8, 1),
    (torch.bfloat16, 1, 300, 40, 7),
    (torch.bfloat16, 1, 4096, 8200, 100),
    (torch.bfloat16, 1, 28672, 2048, 17204),
    (torch.float32, 1, 1000, 1028, 999),
]


@pytest.mark.parametrize("dtype,M,d_in,d_out,K", SPARSE_CASES)
def test_sparse_linear(L, dtype, M, d_in, d_out, K):
    idx, val = sd.index_values(M, d_in, K, 400 + K)
    W = sd.weights(d_in, d_out, 0.02, 401, dtype)
    st = status()
    y = L.larosa_sparse_linear(idx.cuda(), val.cuda(), W.cuda(), dev_status=st)
    assert L.larosa_check(st) == 0
    got = f64(y)
    Wd = f64(W)
    ref = oracle.sparse_linear(idx.numpy().astype(np.int64), f64(val), Wd)
    ref = ref.reshape(M, d_out)
    if K == 0:
        assert np.array_equal(got, np.zeros_like(got))
        return
    absum = np.stack([np.abs(f64(val)[m]) @ np.abs(Wd[idx[m].numpy()]) for m in range(M)])
    # the tensor-core paths of several bf16 tokens multiply each coefficient
    # as a bf16 head and tail, within 2^-16 of its value
    rep = 2.0 ** -16 if (M >= 2 and dtype == torch.bfloat16) else 0.0
    assert np.all(np.abs(got - ref) <= ((K + 2) * U + rep) * absum + 1e-30)
    assert rel_inf(got, ref) <= Y_TOL


def test_sparse_linear_reports_bad_index(L):
    idx, val = sd.index_values(1, 256, 10, 5)
    idx[0, 3] = 999
    W = sd.weights(256, 64, 0.02, 6, torch.bfloat16)
    st = status()
    y = L.larosa_sparse_linear(idx.cuda(), val.cuda(), W.cuda(), dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & 0x4
    keep = np.array([k for k in range(10) if k != 3])
    ref = oracle.sparse_linear(idx.numpy()[0, keep].astype(np.int64), f64(val)[0, keep], f64(W))
    assert rel_inf(f64(y)[0], ref) <= Y_TOL


@pytest.mark.parametrize("dtype,M,d_in,d_out", [
    (torch.float32, 1, 256, 512),
    (torch.bfloat16, 1, 4096, 4096),
    (torch.bfloat16, 3, 1000, 1032),
    (torch.bfloat16, 16, 512, 512),
    (torch.bfloat16, 1, 16, 8),
    (torch.bfloat16, 1, 11008, 4096),
    (torch.float32, 1, 336, 44),
    (torch.bfloat16, 4, 4096, 12288),
])
def test_dense_linear(L, dtype, M, d_in, d_out):
    x = sd.activations(M, d_in, 501, dtype)
    W = sd.weights(d_in, d_out, 0.02, 502, dtype)
    got = f64(L.larosa_dense_linear(x.cuda(), W.t().contiguous().cuda()))
    xd, Wd = f64(x), f64(W)
    ref = oracle.dense_linear(xd, Wd)
    assert np.all(np.abs(got - ref) <= (d_in + 2) * U * (np.abs(xd) @ np.abs(Wd)) + 1e-30)


# ---------------------------------------------------------------- fused

def fused_outputs(L, x, Qt, W_rot, K):
    """Runs the fused call; returns y and the workspace copies of x_rot, idx, val."""
    M, d_in = x.shape
    d_out = W_rot.shape[1]
    ws = L.Workspace()
    buf = ws.get(M, d_in, d_out, K)
    st = status()
    y = L.larosa_rotate_topk_linear(x, Qt, W_rot, K, ws=ws, dev_status=st)
    assert L.larosa_check(st) == 0
    o_x, o_i, o_v = L.larosa_workspace_layout(M, d_in, d_out, K)
    x_rot = buf[o_x:o_x + M * d_in * 4].view(torch.float32).view(M, d_in)
    idx = buf[o_i:o_i + M * K * 4].view(torch.int32).view(M, K)
    val = buf[o_v:o_v + M * K * 4].view(torch.float32).view(M, K)
    return f64(y), f64(x_rot), idx.cpu().numpy().astype(np.int64), val.cpu().numpy()


def check_selection(x_rot_ref, gamma, idx, K):
    """idx is a valid Top-K of x_rot_ref up to 2*gamma; returns nothing."""
    M, d = x_rot_ref.shape
    for m in range(M):
        s = idx[m]
        assert len(s) == K and np.all(np.diff(s) > 0) and (K == 0 or (s[0] >= 0 and s[-1] < d))
        if K in (0, d):
            continue
        mag = np.abs(x_rot_ref[m])
        inside = np.zeros(d, dtype=bool)
        inside[s] = True
        g2 = 2 * np.max(gamma[m])
        assert mag[inside].min() >= mag[~inside].max() - g2
        # the unique part matches the exact selection
        want, _ = oracle.topk(x_rot_ref[m], K)
        wanted = np.zeros(d, dtype=bool)
        wanted[want] = True
        differ = inside != wanted
        thr = np.sort(mag)[::-1][K - 1]
        assert np.all(np.abs(mag[differ] - thr) <= 2 * g2)


@pytest.mark.parametrize("dtype,M,d_in,d_out,sparsity", [
    (torch.float32, 1, 256, 512, 40),
    (torch.float32, 1, 256, 512, 0),
    (torch.bfloat16, 1, 1024, 1032, 40),
    (torch.bfloat16, 4, 1024, 1032, 40),
    (torch.bfloat16, 1, 4096, 4096, 50),
    (torch.bfloat16, 16, 512, 256, 25),
    (torch.bfloat16, 1, 64, 8, 90),
    (torch.bfloat16, 1, 200, 24, 50),
    (torch.bfloat16, 1, 11008, 4096, 40),
])
def test_fused(L, dtype, M, d_in, d_out, sparsity):
    K = sd.k_for_sparsity(d_in, sparsity)
    Q = sd.orthogonal(d_in, 601, device="cuda" if d_in > 4096 else "cpu").to(dtype).cpu()
    W = sd.weights(d_in, d_out, 0.02 if dtype == torch.bfloat16 else 1 / 16, 602, dtype)
    x = sd.activations(M, d_in, 603, dtype)
    Qt = Q.t().contiguous().cuda()
    W_rot = L.larosa_prepare_weights(Qt, W.cuda())
    y, x_rot, idx, val = fused_outputs(L, x.cuda(), Qt, W_rot, K)
    xq, qq = f64(x), f64(Q)
    x_rot_ref = oracle.rotate(xq, qq)
    gamma = (d_in + 2) * U * (np.abs(xq) @ np.abs(qq))
    assert np.all(np.abs(x_rot - x_rot_ref) <= gamma + 1e-30)
    check_selection(x_rot_ref, gamma, idx, K)
    for m in range(M):
        # exactly the oracle's Top-K of the path's own fp32 x_rot
        want, _ = oracle.topk(x_rot[m], K)
        assert np.array_equal(idx[m], want)
        assert np.array_equal(val[m], x_rot[m, idx[m]].astype(np.float32))
    W_rot_ref = oracle.prepare_weights(qq, f64(W))
    if dtype == torch.bfloat16:
        W_rot_ref = oracle.round_to_bf16(W_rot_ref)
    ref = np.stack([oracle.sparse_linear(idx[m], x_rot_ref[m, idx[m]], W_rot_ref) for m in range(M)])
    assert rel_inf(y, ref) <= Y_TOL


@pytest.mark.parametrize("dtype,tol", [(torch.float32, 1e-5), (torch.bfloat16, 1e-2)])
def test_fused_dense_equivalence_at_full_k(L, dtype, tol):
    """K = d: rotating and counter-rotating returns the dense layer."""
    d_in, d_out = 256, 512
    Q = sd.orthogonal(d_in, 701).to(dtype)
    W = sd.weights(d_in, d_out, 1 / 16, 702, dtype)
    x = sd.activations(1, d_in, 703, dtype)
    Qt = Q.t().contiguous().cuda()
    W_rot = L.larosa_prepare_weights(Qt, W.cuda())
    y = f64(L.larosa_rotate_topk_linear(x.cuda(), Qt, W_rot, d_in))
    ref = oracle.dense_linear(f64(x), f64(W))
    assert rel_inf(y, ref) <= tol


def test_fused_is_deterministic(L):
    d_in, d_out, K = 4096, 4096, 2458
    Qt = sd.orthogonal(d_in, 801, device="cuda").to(torch.bfloat16).t().contiguous()
    W = sd.weights(d_in, d_out, 0.02, 802, torch.bfloat16, device="cuda")
    x = sd.activations(1, d_in, 803, torch.bfloat16).cuda()
    W_rot = L.larosa_prepare_weights(Qt, W)
    y1 = L.larosa_rotate_topk_linear(x, Qt, W_rot, K).clone()
    y2 = L.larosa_rotate_topk_linear(x, Qt, W_rot, K).clone()
    assert torch.equal(y1, y2)


@pytest.mark.parametrize("kind", sd.ADVERSARIAL_KINDS)
@pytest.mark.parametrize("d", [8, 200, 1024, 4096, 11008])
def test_fused_selection_bit_exact_under_identity_rotation(L, kind, d):
    """Q = I is orthogonal and makes the fused rotation exact (x_rot = x), so the
    selection inside the fused kernel can be compared bit for bit with the
    oracle's Top-K of x on rows full of ties, signed zeros and subnormals."""
    d_out = 72
    x = sd.adversarial_rows(kind, 1, d, 900 + d)
    Qt = torch.eye(d, dtype=torch.float32, device="cuda")
    W_rot = sd.weights(d, d_out, 1 / 16, 901, torch.float32).cuda()
    xd = f64(x)
    for K in sorted({1, max(1, d // 3), sd.k_for_sparsity(d, 40), d - 1}):
        y, x_rot, idx, val = fused_outputs(L, x.cuda(), Qt, W_rot, K)
        # x_rot equals x up to the sign of zero
        assert np.array_equal(np.abs(x_rot), np.abs(xd)), (kind, d, K)
        want_i, want_v = oracle.topk(xd, K)
        assert np.array_equal(idx.reshape(-1), want_i.reshape(-1)), (kind, d, K)
        assert np.array_equal(np.abs(val.reshape(-1)), np.abs(want_v.reshape(-1)).astype(np.float32))
        ref = oracle.sparse_linear(want_i.reshape(-1), xd[0, want_i.reshape(-1)], f64(W_rot))
        got, bound = y.reshape(-1), (K + 2) * U * (np.abs(xd[0, want_i.reshape(-1)]) @ np.abs(f64(W_rot)[want_i.reshape(-1)]))
        assert np.all(np.abs(got - ref) <= bound + 1e-37), (kind, d, K)


@pytest.mark.parametrize("dtype,d,sparsity", [
    (torch.float32, 256, 40), (torch.bfloat16, 1024, 40), (torch.bfloat16, 4096, 40),
    (torch.bfloat16, 11008, 40), (torch.bfloat16, 4096, 0), (torch.bfloat16, 4096, 100),
    (torch.bfloat16, 8, 50), (torch.bfloat16, 32768, 50),
])
def test_rotate_topk(L, dtype, d, sparsity):
    """Rotation and Top-K in one kernel: x_rot within the summation bound, the
    kept set a valid Top-K of the exact rotation, and (idx, val) exactly the
    Top-K of the kernel's own fp32 x_rot."""
    K = sd.k_for_sparsity(d, sparsity)
    Q = sd.orthogonal(d, 1001 + d, device="cuda" if d > 4096 else "cpu").to(dtype).cpu()
    x = sd.activations(1, d, 1002 + d, dtype)
    st = status()
    x_rot, idx, val = L.larosa_rotate_topk(x.cuda(), Q.t().contiguous().cuda(), K, dev_status=st)
    assert L.larosa_check(st) == 0
    xq, qq = f64(x), f64(Q)
    x_rot_ref = oracle.rotate(xq, qq)
    gamma = (d + 2) * U * (np.abs(xq) @ np.abs(qq))
    got = f64(x_rot)
    assert np.all(np.abs(got - x_rot_ref) <= gamma + 1e-30)
    idx = idx.cpu().numpy().astype(np.int64)
    check_selection(x_rot_ref, gamma, idx, K)
    # selection rule on the kernel's fp32 values: every kept magnitude is
    # >= every dropped one, and equal magnitudes favour the lower index
    mags = np.abs(got[0]).astype(np.float32)
    kept = np.zeros(d, dtype=bool)
    kept[idx[0]] = True
    if 0 < K < d:
        thr = mags[kept].min()
        assert np.all(mags[~kept] <= thr)
        tied_out = np.nonzero(~kept & (mags == thr))[0]
        tied_in = np.nonzero(kept & (mags == thr))[0]
        assert len(tied_out) == 0 or tied_in.max() < tied_out.min()
    want, _ = oracle.topk(got[0], K)
    assert np.array_equal(idx[0], want)
    assert np.array_equal(f64(val)[0], got[0, idx[0]])


def test_one_workspace_serves_calls_of_every_size(L):
    """The one-token fused call keeps a call number and alternating counters
    in the workspace from call to call; calls of other sizes (several tokens,
    the threshold layout) on the same workspace must leave them intact.  A
    one-token call after each of them returns exactly what it returns on a
    workspace of its own, without a device error."""
    d_in, d_out = 1024, 2048
    K = sd.k_for_sparsity(d_in, 40)
    dev = torch.device("cuda")
    Qt = sd.orthogonal(d_in, 1301).to(torch.bfloat16).t().contiguous().to(dev)
    W_rot = L.larosa_prepare_weights(Qt, sd.weights(d_in, d_out, 0.02, 1302, torch.bfloat16, device=dev))
    x1 = sd.activations(1, d_in, 1303, torch.bfloat16).to(dev)
    st = status()
    y_alone = L.larosa_rotate_topk_linear(x1, Qt, W_rot, K, ws=L.Workspace(), dev_status=st).clone()
    ws = L.Workspace()
    for M in (1, 4, 16):
        ws.get(M, d_in, d_out, d_in)
        ws.get(M, d_in, d_out, K)
    for M in (4, 16, 2):
        xM = sd.activations(M, d_in, 1310 + M, torch.bfloat16).to(dev)
        L.larosa_rotate_topk_linear(xM, Qt, W_rot, K, ws=ws, dev_status=st)
        L.larosa_rotate_threshold_linear(xM, Qt, W_rot, 0.05, ws=ws, dev_status=st)
        for _ in range(2):  # the call number alternates the counters' slots
            y1 = L.larosa_rotate_topk_linear(x1, Qt, W_rot, K, ws=ws, dev_status=st)
            assert L.larosa_check(st) == 0, M
            assert torch.equal(y1, y_alone), M
