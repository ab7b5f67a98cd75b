"""larosa_sparse_linear_noalloc through the C ABI, against the fp64 oracle and
against larosa_sparse_linear.

The no-allocation variant serves callers that cannot give the library a
workspace (an operator slot that passes only inputs and outputs, or a loop in
which cudaMalloc/cudaFree are not allowed).  It runs the same kernels with the
same launch geometry as the workspace entry point, so its output must equal
that entry point's bit for bit, and both must lie within the fp32 summation
bound of the oracle's exact sum.  Two consecutive calls use different index
sets, so a value left behind in the shared static scratch by the first call
(coefficient rows, the row bitmap, the union list, split-K tickets) would
change the second call's result.  Sizes whose scratch would not fit are
refused, and larosa_sparse_linear_noalloc_bytes says so in advance.

This file is collected last on purpose.  It must pass both alone in a fresh
process and after the rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synthdata as sd

pytestmark = pytest.mark.gpu

Y_TOL = 2e-3  # the tolerance the parity tests use for y
U = 2.0 ** -24  # unit roundoff of fp32
SCRATCH = 2 << 20  # LAROSA_NOALLOC_SCRATCH_BYTES


@pytest.fixture(scope="module")
def lib():
    from activation_sparsity_b200 import build_lib
    build_lib.build()
    from activation_sparsity_b200 import larosa
    lib = larosa.raw_library()
    lib.larosa_last_error_string.restype = ctypes.c_char_p
    return lib


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _call_noalloc(lib, idx, val, W, y, st):
    M, K = idx.shape
    d_in, d_out = W.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.larosa_sparse_linear_noalloc(_p(idx), _p(val), M, K, _p(W), d_in, d_out, _p(y),
                                            1 if W.dtype == torch.bfloat16 else 0, _p(st), stream)


def _check_against_oracle(y, idx, val, W):
    got = y.double().cpu().numpy()
    Wd = W.double().cpu().numpy()
    i64 = idx.cpu().numpy().astype(np.int64)
    v64 = val.double().cpu().numpy()
    M, K = i64.shape
    # from 2 bf16 tokens on the tensor cores multiply each coefficient as a
    # bf16 head and tail, which keep it to within 2^-16 of its value
    rep = 2.0 ** -16 if (M >= 2 and W.dtype == torch.bfloat16) else 0.0
    for m in range(M):
        ref = oracle.sparse_linear(i64[m], v64[m], Wd)
        bound = ((K + 2) * U + rep) * (np.abs(v64[m]) @ np.abs(Wd[i64[m]]))
        assert np.all(np.abs(got[m] - ref) <= bound + 1e-30), m
        assert np.max(np.abs(got[m] - ref)) <= Y_TOL * np.max(np.abs(ref)), m


@pytest.mark.parametrize("M,d_in,d_out,K", [
    (1, 4096, 12288, 2458),   # LLaMA2-7B q|k|v at 40 % sparsity
    (1, 11008, 4096, 6605),   # LLaMA2-7B down at 40 % sparsity
    (4, 1024, 2048, 400),     # several tokens sharing streamed rows
    (8, 2048, 1024, 1229),    # eight tokens: the scratch holds coefficient rows of all of them
    (2, 4096, 1024, 100),     # few rows per token: the union of the kept rows is streamed
])
def test_noalloc_matches_oracle_and_workspace_entry_point_on_two_calls(lib, M, d_in, d_out, K):
    import activation_sparsity_b200 as L
    W = sd.weights(d_in, d_out, 0.02, 901, torch.bfloat16, device="cuda")
    need = L.larosa_sparse_linear_noalloc_bytes(M, d_in, d_out, K)
    assert need <= SCRATCH
    if M == 1:
        assert need == 0  # the one-token cluster gather uses no scratch on this GPU
    for call in range(2):
        # a different index set on each call: few rows shared between them
        idx, val = sd.index_values(M, d_in, K, 900 + 17 * call + M)
        idx, val = idx.cuda(), val.cuda()
        ref = L.larosa_sparse_linear(idx, val, W)
        y = torch.full((M, d_out), float("nan"), dtype=torch.float32, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        rc = _call_noalloc(lib, idx, val, W, y, st)
        assert rc == 0, (call, rc)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        # same kernels, same geometry: the same sums in the same order
        assert torch.equal(y, ref), call
        _check_against_oracle(y, idx, val, W)


def test_noalloc_refuses_sizes_beyond_its_scratch(lib):
    import activation_sparsity_b200 as L
    # 16 fp32 tokens at d_in = 32768: their dense fp32 coefficient rows alone take 2 MiB
    M, d_in, d_out, K = 16, 32768, 1024, 100
    assert L.larosa_sparse_linear_noalloc_bytes(M, d_in, d_out, K, torch.float32) > SCRATCH
    # the same sizes in bf16 take the tensor-core path, whose head and tail rows just fit
    assert L.larosa_sparse_linear_noalloc_bytes(M, d_in, d_out, K) == SCRATCH
    idx = torch.zeros((M, K), dtype=torch.int32, device="cuda")
    val = torch.zeros((M, K), dtype=torch.float32, device="cuda")
    W = torch.zeros((d_in, d_out), dtype=torch.float32, device="cuda")
    y = torch.zeros((M, d_out), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert _call_noalloc(lib, idx, val, W, y, st) == 6  # LAROSA_ERR_WORKSPACE
    msg = lib.larosa_last_error_string().decode()
    assert "scratch" in msg and str(SCRATCH) in msg
    torch.cuda.synchronize()
    assert np.all(y.cpu().numpy() == 0)  # nothing was enqueued


def test_noalloc_one_token_needs_no_scratch_at_the_largest_sizes(lib):
    """One token never reaches the scratch-using fallback on this GPU: the
    cluster gather plan fits every accepted size, up to d_in = K = 32768."""
    import activation_sparsity_b200 as L
    for d_in, d_out, K in [(32768, 8192, 32768), (32768, 65536, 16384), (8, 8, 1), (4096, 8, 0)]:
        assert L.larosa_sparse_linear_noalloc_bytes(1, d_in, d_out, K) == 0, (d_in, d_out, K)
