"""The tcgen05 kernels for 2 to 16 tokens against the fp64 oracle, smallest
cases first: the rotation / dense row-dot product (128 output rows x 16 token
slots per CTA, split over a cluster) and the sparse linear as a dense product
with the tokens' coefficients (256 output columns per CTA).  Bars as in test_gpu_parity: the fp32 summation bound
per element; for the sparse linear also the coefficients' bf16 head + tail
representation (2^-16 of each coefficient) and the 2e-3 norm bar.
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


@pytest.mark.parametrize("M,d", [(16, 64), (8, 128), (12, 256), (2, 512), (4, 1024), (5, 192), (16, 1024),
                                 (16, 4096), (8, 11008), (3, 11008)])
def test_rotate_tcgen05(L, M, d):
    Q = sd.orthogonal(d, 211, device="cuda" if d > 4096 else "cpu").to(torch.bfloat16)
    x = sd.activations(M, d, 212, torch.bfloat16)
    got = f64(L.larosa_rotate(x.cuda(), Q.cuda().t().contiguous()))
    xq, qq = f64(x), f64(Q)
    ref = oracle.rotate(xq, qq)
    bound = (d + 2) * U * (np.abs(xq) @ np.abs(qq))
    assert np.all(np.abs(got - ref) <= bound + 1e-30)


@pytest.mark.parametrize("M,d_in,d_out", [(16, 64, 8), (8, 128, 136), (16, 512, 1000), (2, 4096, 4096),
                                         (16, 4096, 4096)])
def test_dense_tcgen05(L, M, d_in, d_out):
    x = sd.activations(M, d_in, 221, torch.bfloat16)
    W = sd.weights(d_in, d_out, 0.02, 222, torch.bfloat16)
    got = f64(L.larosa_dense_linear(x.cuda(), W.t().contiguous().cuda()))
    xd, Wd = f64(x), f64(W)
    ref = oracle.dense_linear(xd, Wd)
    assert np.all(np.abs(got - ref) <= (d_in + 2) * U * (np.abs(xd) @ np.abs(Wd)) + 1e-30)


@pytest.mark.parametrize("M,d_in,d_out,K", [(8, 64, 128, 20), (16, 512, 1032, 300), (16, 4096, 4096, 2458),
                                            (12, 11008, 4096, 6605), (2, 512, 264, 300), (4, 4096, 4096, 2458),
                                            (7, 1000, 2056, 400)])
def test_sparse_tcgen05(L, M, d_in, d_out, K):
    idx, val = sd.index_values(M, d_in, K, 230 + K)
    W = sd.weights(d_in, d_out, 0.02, 231, torch.bfloat16)
    st = status()
    y = L.larosa_sparse_linear(idx.cuda(), val.cuda(), W.cuda(), dev_status=st)
    assert L.larosa_check(st) == 0
    got, Wd = f64(y), f64(W)
    ref = oracle.sparse_linear(idx.numpy().astype(np.int64), f64(val), Wd).reshape(M, d_out)
    absum = np.stack([np.abs(f64(val)[m]) @ np.abs(Wd[idx[m].numpy()]) for m in range(M)])
    assert np.all(np.abs(got - ref) <= ((K + 2) * U + 2.0 ** -16) * absum + 1e-30)
    assert rel_inf(got, ref) <= Y_TOL
    # the row bitmap in the workspace header is left at zero: a second call
    # through the row-streaming path (M = 4) on the same default workspace
    # still matches
    idx4, val4 = sd.index_values(4, d_in, K, 240 + K)
    y4 = L.larosa_sparse_linear(idx4.cuda(), val4.cuda(), W.cuda(), dev_status=st)
    assert L.larosa_check(st) == 0
    ref4 = oracle.sparse_linear(idx4.numpy().astype(np.int64), f64(val4), Wd).reshape(4, d_out)
    assert rel_inf(f64(y4), ref4) <= Y_TOL
