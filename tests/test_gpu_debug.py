"""The library's debug checks of kept lists and the split override of the
tensor-core batch kernels, through the C ABI on the GPU.

Debug checks (larosa_set_debug): a call that takes kept lists checks them
before its compute, a call that writes them checks what it wrote; a list
that repeats an index (or, where the library wrote it, is out of order)
reports LAROSA_DEV_LIST, an index out of range LAROSA_DEV_INDEX, a non-finite
value LAROSA_DEV_NONFINITE.  The results themselves do not change.

Split override (larosa_set_split_k): the tensor-core kernels of 2 to 16 bf16
tokens split their reduction over a forced number of CTAs; every split stays
within the fp32 summation bound of the oracle's product, a fixed split
repeats bit for bit, and 0 restores the choice per shape.
"""
import numpy as np
import pytest
import torch

import oracle
import synthdata as sd
from tests.test_gpu_parity import U, Y_TOL, f64, rel_inf, status

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    from activation_sparsity_b200 import build_lib
    build_lib.build()
    import activation_sparsity_b200 as L
    torch.cuda.init()
    return L


@pytest.fixture
def debug_on(L):
    prev = L.larosa_set_debug(True)
    yield
    L.larosa_set_debug(prev)


@pytest.fixture
def split_restore(L):
    prev = L.larosa_set_split_k(0)
    yield
    L.larosa_set_split_k(prev)


def flags(L, st) -> int:
    torch.cuda.synchronize()
    return int(st.item())


@pytest.mark.parametrize("M", [1, 4, 16])
def test_valid_lists_pass_and_results_do_not_change(L, M):
    d_in, d_out, K = 1024, 2048, 400
    idx, val = sd.index_values(M, d_in, K, 1500 + M)
    W = sd.weights(d_in, d_out, 0.02, 1501, torch.bfloat16, device="cuda")
    idx, val = idx.cuda(), val.cuda()
    plain = L.larosa_sparse_linear(idx, val, W).clone()
    prev = L.larosa_set_debug(True)
    try:
        st = status()
        y = L.larosa_sparse_linear(idx, val, W, dev_status=st)
        assert flags(L, st) == 0
        assert torch.equal(y, plain)
        # lists in descending order are valid input (order does not matter)
        st = status()
        L.larosa_sparse_linear(idx.flip(-1).contiguous(), val.flip(-1).contiguous(), W, dev_status=st)
        assert flags(L, st) == 0
    finally:
        L.larosa_set_debug(prev)


@pytest.mark.parametrize("M", [1, 4])
def test_repeated_index_is_reported(L, debug_on, M):
    d_in, d_out, K = 512, 256, 100
    idx, val = sd.index_values(M, d_in, K, 1510 + M)
    idx[M - 1, 7] = idx[M - 1, 3]  # one row names an index twice
    W = sd.weights(d_in, d_out, 0.02, 1511, torch.bfloat16, device="cuda")
    st = status()
    L.larosa_sparse_linear(idx.cuda(), val.cuda(), W, dev_status=st)
    assert flags(L, st) & L.LAROSA_DEV_LIST
    with pytest.raises(L.LarosaError) as err:
        L.larosa_check(st)
    assert err.value.status == L.LAROSA_ERR_LIST
    st = status()
    L.larosa_sparse_linear_noalloc(idx.cuda(), val.cuda(), W, dev_status=st)
    assert flags(L, st) & L.LAROSA_DEV_LIST


def test_out_of_range_and_nonfinite_are_reported(L, debug_on):
    d_in, d_out, K = 512, 256, 100
    idx, val = sd.index_values(1, d_in, K, 1520)
    W = sd.weights(d_in, d_out, 0.02, 1521, torch.bfloat16, device="cuda")
    bad = idx.clone()
    bad[0, 5] = d_in
    st = status()
    L.larosa_sparse_linear(bad.cuda(), val.cuda(), W, dev_status=st)
    assert flags(L, st) & L.LAROSA_DEV_INDEX
    nan = val.clone()
    nan[0, 9] = float("nan")
    st = status()
    L.larosa_sparse_linear(idx.cuda(), nan.cuda(), W, dev_status=st)
    assert flags(L, st) & L.LAROSA_DEV_NONFINITE


def test_sparse_lowrank_lists_are_checked(L, debug_on):
    d_in, d_out, r = 512, 256, 32
    K = sd.k_for_sparsity(d_in, 40)
    W = sd.weights(d_in, d_out, 0.02, 1530, torch.bfloat16)
    A64, B64 = oracle.lowrank_factors(f64(W), r)
    A, B = torch.from_numpy(A64).to(torch.bfloat16).cuda(), torch.from_numpy(B64).to(torch.bfloat16).cuda()
    x = sd.activations(1, d_in, 1531, torch.float32)
    i, v = oracle.topk(f64(x)[0], K)
    idx = torch.from_numpy(i.reshape(1, K).astype(np.int32))
    val = torch.from_numpy(v.reshape(1, K).astype(np.float32))
    st = status()
    L.larosa_sparse_lowrank_linear(x.cuda(), idx.cuda(), val.cuda(), W.cuda(), A, B, dev_status=st)
    assert flags(L, st) == 0
    idx[0, 1] = idx[0, 0]
    st = status()
    L.larosa_sparse_lowrank_linear(x.cuda(), idx.cuda(), val.cuda(), W.cuda(), A, B, dev_status=st)
    assert flags(L, st) & L.LAROSA_DEV_LIST


@pytest.mark.parametrize("M", [1, 2, 8])
def test_lists_the_library_writes_pass(L, debug_on, M):
    d_in, d_out = 4096, 1024
    K = sd.k_for_sparsity(d_in, 40)
    Q = sd.orthogonal(d_in, 1540).to(torch.bfloat16)
    Qt = Q.t().contiguous().cuda()
    W = sd.weights(d_in, d_out, 0.02, 1541, torch.bfloat16, device="cuda")
    x = sd.activations(M, d_in, 1542, torch.bfloat16).cuda()
    st = status()
    L.larosa_rotate_topk_linear(x, Qt, W, K, dev_status=st)
    L.larosa_rotate_topk_linear(x, None, W, K, dev_status=st)
    x_rot = L.larosa_rotate(x, Qt)
    L.larosa_topk(x_rot, K, dev_status=st)
    L.larosa_topk_linear(x_rot, W, K, dev_status=st)
    if M == 1:
        L.larosa_rotate_topk(x, Qt, K, dev_status=st)
    assert flags(L, st) == 0


@pytest.mark.parametrize("M", [2, 16])
def test_forced_splits_stay_within_the_bound(L, split_restore, M):
    d_in, d_out, K = 4096, 2048, 2458
    idx, val = sd.index_values(M, d_in, K, 1550 + M)
    W = sd.weights(d_in, d_out, 0.02, 1551, torch.bfloat16)
    Wc, ic, vc = W.cuda(), idx.cuda(), val.cuda()
    Q = sd.orthogonal(1024, 1552).to(torch.bfloat16)
    Qt = Q.t().contiguous().cuda()
    x = sd.activations(M, 1024, 1553, torch.bfloat16)
    Wd, xd, qd = f64(W), f64(x), f64(Q)
    i64, v64 = idx.numpy().astype(np.int64), val.double().numpy()
    ref = np.stack([oracle.sparse_linear(i64[m], v64[m], Wd) for m in range(M)])
    absum = np.stack([np.abs(v64[m]) @ np.abs(Wd[i64[m]]) for m in range(M)])
    rot_ref = oracle.rotate(xd, qd)
    rot_bound = (1024 + 2) * U * (np.abs(xd) @ np.abs(qd))
    auto_y = L.larosa_sparse_linear(ic, vc, Wc).clone()
    for R in (1, 2, 3, 8):
        L.larosa_set_split_k(R)
        st = status()
        y1 = L.larosa_sparse_linear(ic, vc, Wc, dev_status=st).clone()
        y2 = L.larosa_sparse_linear(ic, vc, Wc, dev_status=st).clone()
        assert flags(L, st) == 0
        assert torch.equal(y1, y2), R
        got = f64(y1)
        assert np.all(np.abs(got - ref) <= ((K + 2) * U + 2.0 ** -16) * absum + 1e-30), R
        assert rel_inf(got, ref) <= Y_TOL, R
        xr = f64(L.larosa_rotate(x.cuda(), Qt))
        assert np.all(np.abs(xr - rot_ref) <= rot_bound + 1e-30), R
    L.larosa_set_split_k(0)
    assert torch.equal(L.larosa_sparse_linear(ic, vc, Wc), auto_y)
