"""larosa_topk_linear: the exact Top-K of an already rotated fp32 vector and the
sparse linear over the kept rows, against the fp64 oracle through the C ABI.

The call runs the Top-K kernel and the sparse linear on its kept lists (from
8 bf16 tokens on the tcgen05 product, with the coefficient rows written by the
Top-K kernel).  The input is the selection vector itself, so the kept list must
equal the oracle's Top-K of it bit for bit (ties to the lower index, +0 and
-0 equal), on the adversarial families as on Gaussian rows; y must lie within
the fp32 summation bound of the oracle's product on that list, and within the
2e-3 bar.
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


def run(L, x_rot, W, K):
    """y and the workspace copies of idx/val ([M, K] each)."""
    M, d_in = x_rot.shape
    d_out = W.shape[1]
    ws = L.Workspace()
    buf = ws.get(M, d_in, d_out, K)
    st = status()
    y = L.larosa_topk_linear(x_rot, W, K, ws=ws, dev_status=st)
    assert L.larosa_check(st) == 0
    _, o_i, o_v = L.larosa_workspace_layout(M, d_in, d_out, K)
    idx = buf[o_i:o_i + M * K * 4].view(torch.int32).view(M, K).cpu().numpy().astype(np.int64)
    val = buf[o_v:o_v + M * K * 4].view(torch.float32).view(M, K).cpu().numpy()
    return f64(y), idx, val


def check(y, idx, val, x, W, K, rep=0.0):
    """Kept list bit-exact against the oracle's Top-K of x; y within the bound."""
    xd, Wd = f64(x), f64(W)
    M = xd.shape[0]
    for m in range(M):
        want_i, want_v = oracle.topk(xd[m], K)
        assert np.array_equal(idx[m], want_i), m
        assert np.array_equal(np.abs(val[m]), np.abs(want_v).astype(np.float32)), m
        ref = oracle.sparse_linear(want_i, want_v, Wd)
        bound = ((K + 2) * U + rep) * (np.abs(want_v) @ np.abs(Wd[want_i])) if K else np.zeros_like(ref)
        assert np.all(np.abs(y[m] - ref) <= bound + 1e-37), m


@pytest.mark.parametrize("kind", sd.ADVERSARIAL_KINDS)
@pytest.mark.parametrize("d", [8, 200, 1024, 4096, 11008, 16384, 20000])
def test_topk_linear_one_token_bit_exact_selection(L, kind, d):
    d_out = 72
    x = sd.adversarial_rows(kind, 1, d, 1400 + d).cuda()
    W = sd.weights(d, d_out, 1 / 16, 1401, torch.float32).cuda()
    for K in sorted({0, 1, max(1, d // 3), sd.k_for_sparsity(d, 40), d - 1, d}):
        y, idx, val = run(L, x, W, K)
        check(y, idx, val, x, W, K)


@pytest.mark.parametrize("d_in,d_out,sparsity", [
    (4096, 12288, 40),    # LLaMA2-7B q|k|v
    (4096, 4096, 50),     # o
    (11008, 4096, 40),    # down
    (13824, 5120, 40),    # LLaMA2-13B down
    (1000, 1032, 25),     # ragged column tiles
])
def test_topk_linear_bf16_weights(L, d_in, d_out, sparsity):
    K = sd.k_for_sparsity(d_in, sparsity)
    x = sd.activations(1, d_in, 1410, torch.float32).cuda()
    W = sd.weights(d_in, d_out, 0.02, 1411, torch.bfloat16, device="cuda")
    y, idx, val = run(L, x, W, K)
    check(y, idx, val, x, W, K)
    want_i, want_v = oracle.topk(f64(x)[0], K)
    assert rel_inf(y[0], oracle.sparse_linear(want_i, want_v, f64(W))) <= Y_TOL


@pytest.mark.parametrize("M,sparsity", [(2, 40), (4, 40), (8, 40), (16, 40),
                                        # few rows per token: two and four tokens stream the union
                                        (2, 95), (4, 97)])
def test_topk_linear_several_tokens(L, M, sparsity):
    d_in, d_out = 1024, 2048
    K = sd.k_for_sparsity(d_in, sparsity)
    x = sd.activations(M, d_in, 1420 + M, torch.float32).cuda()
    W = sd.weights(d_in, d_out, 0.02, 1421, torch.bfloat16, device="cuda")
    y, idx, val = run(L, x, W, K)
    # from 2 bf16 tokens on the tensor cores multiply each coefficient as a
    # bf16 head and tail, within 2^-16 of its value
    check(y, idx, val, x, W, K, rep=2.0 ** -16)


def test_topk_linear_is_deterministic_and_matches_the_two_calls(L):
    d_in, d_out = 4096, 4096
    K = sd.k_for_sparsity(d_in, 40)
    x = sd.activations(1, d_in, 1430, torch.float32).cuda()
    W = sd.weights(d_in, d_out, 0.02, 1431, torch.bfloat16, device="cuda")
    y1 = L.larosa_topk_linear(x, W, K).clone()
    y2 = L.larosa_topk_linear(x, W, K).clone()
    assert torch.equal(y1, y2)
    idx, val = L.larosa_topk(x, K)
    y3 = L.larosa_sparse_linear(idx, val, W)
    assert rel_inf(f64(y1), f64(y3)) <= 1e-6


def test_topk_linear_reports_nonfinite(L):
    d_in, d_out, K = 1024, 64, 300
    x = sd.activations(1, d_in, 1440, torch.float32)
    x[0, 17] = float("nan")
    W = sd.weights(d_in, d_out, 0.02, 1441, torch.bfloat16, device="cuda")
    st = status()
    L.larosa_topk_linear(x.cuda(), W, K, dev_status=st)
    with pytest.raises(L.LarosaError) as err:
        L.larosa_check(st)
    assert err.value.status == 7  # LAROSA_ERR_NONFINITE
