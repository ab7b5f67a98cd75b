"""larosa_sparse_linear_noalloc against larosa_sparse_linear, through the C ABI.

The no-allocation variant serves callers that cannot give the library a
workspace (an operator slot that passes only inputs and outputs, or a loop in
which cudaMalloc/cudaFree are not allowed).  It must return what the
workspace entry point returns, on consecutive calls that reuse its fixed
device scratch, and refuse sizes whose scratch would not fit.

This file is collected last on purpose.  It must pass both alone in a fresh
process and after the rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

import synthdata as sd

pytestmark = pytest.mark.gpu

Y_TOL = 2e-3  # the tolerance the parity tests use for y


@pytest.fixture(scope="module")
def lib():
    from activation_sparsity_b200 import build_lib
    build_lib.build()
    from activation_sparsity_b200 import larosa
    return larosa.raw_library()


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _call_noalloc(lib, idx, val, W, y, st):
    M, K = idx.shape
    d_in, d_out = W.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.larosa_sparse_linear_noalloc(_p(idx), _p(val), M, K, _p(W), d_in, d_out, _p(y),
                                            1 if W.dtype == torch.bfloat16 else 0, _p(st), stream)


def _rel_inf(got, ref):
    return float((got - ref).abs().max() / ref.abs().max())


@pytest.mark.parametrize("M,d_in,d_out,K", [
    (1, 4096, 12288, 2458),   # LLaMA2-7B q|k|v at 40 % sparsity
    (1, 11008, 4096, 6605),   # LLaMA2-7B down at 40 % sparsity
    (4, 1024, 2048, 400),     # several tokens sharing streamed rows
])
def test_noalloc_matches_workspace_entry_point_on_two_calls(lib, M, d_in, d_out, K):
    import activation_sparsity_b200 as L
    idx, val = sd.index_values(M, d_in, K, 900 + M)
    W = sd.weights(d_in, d_out, 0.02, 901, torch.bfloat16, device="cuda")
    idx, val = idx.cuda(), val.cuda()
    ref = L.larosa_sparse_linear(idx, val, W)
    torch.cuda.synchronize()
    for call in range(2):
        y = torch.full((M, d_out), float("nan"), dtype=torch.float32, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        rc = _call_noalloc(lib, idx, val, W, y, st)
        assert rc == 0, (call, rc)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        assert torch.isfinite(y).all()
        assert _rel_inf(y, ref) <= Y_TOL, call


def test_noalloc_refuses_sizes_beyond_its_scratch(lib):
    M, d_in, d_out, K = 16, 32768, 4096, 100   # dense per-token coefficients alone take 2 MiB
    idx = torch.zeros((M, K), dtype=torch.int32, device="cuda")
    val = torch.zeros((M, K), dtype=torch.float32, device="cuda")
    W = torch.zeros((d_in, d_out), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((M, d_out), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert _call_noalloc(lib, idx, val, W, y, st) == 6  # LAROSA_ERR_WORKSPACE
    lib.larosa_last_error_string.restype = ctypes.c_char_p
    msg = lib.larosa_last_error_string().decode()
    assert "scratch" in msg and str(2 << 20) in msg
    torch.cuda.synchronize()
    assert np.all(y.cpu().numpy() == 0)  # nothing was enqueued
