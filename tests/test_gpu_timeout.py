"""The bounded waits inside the one-token fused kernel, made to run out on
purpose without faulting or hanging the GPU.

Every wait of a kernel gives up after the wait limit (larosa_set_wait_limit_ns)
and reports LAROSA_DEV_TIMEOUT.  The fused kernel's CTAs wait for the exact
arrival count of their call; a workspace whose arrival counter does not start
at zero (as after a call that gave up) can never show that count, so every
wait on it runs out.  The test sets the limit to 1 ms, plants such a counter,
and checks that the call returns quickly with the timeout reported, that no
CTA streamed a row (y is zero), and that after the workspace is zeroed again
the next call matches the oracle.
"""
import time

import numpy as np
import pytest
import torch

import oracle
import synthdata as sd
from tests.test_gpu_parity import U, Y_TOL, check_selection, f64, fused_outputs, rel_inf, status

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    from activation_sparsity_b200 import build_lib
    build_lib.build()
    import activation_sparsity_b200 as L
    torch.cuda.init()
    return L


def test_wait_limit_setter_validates_and_restores(L):
    prev = L.larosa_set_wait_limit_ns(5_000_000)
    assert prev == 2_000_000_000
    assert L.larosa_set_wait_limit_ns(0) == 5_000_000  # 0 restores the default
    for bad in (1, 999, 60_000_000_001):
        with pytest.raises(L.LarosaError):
            L.larosa_set_wait_limit_ns(bad)
    assert L.larosa_set_wait_limit_ns(0) == 2_000_000_000  # unchanged by the refusals


@pytest.mark.parametrize("threshold", [False, True])
def test_fused_wait_times_out_and_recovers(L, threshold):
    d_in, d_out = 4096, 4096
    K = sd.k_for_sparsity(d_in, 40)
    t = 0.01  # the threshold mode's t (it keeps most of the rotated entries)
    dev = torch.device("cuda")
    Qt = sd.orthogonal(d_in, 1201, device=dev).to(torch.bfloat16).t().contiguous()
    W = sd.weights(d_in, d_out, 0.02, 1202, torch.bfloat16, device=dev)
    W_rot = L.larosa_prepare_weights(Qt, W)
    x = sd.activations(1, d_in, 1203, torch.bfloat16).to(dev)

    def call(ws, st, y=None):
        if threshold:
            return L.larosa_rotate_threshold_linear(x, Qt, W_rot, t, y=y, ws=ws, dev_status=st)
        return L.larosa_rotate_topk_linear(x, Qt, W_rot, K, y=y, ws=ws, dev_status=st)

    # the same call on a workspace that never failed (also loads and plans everything)
    st = status()
    y_fresh = call(L.Workspace(), st).clone()
    assert L.larosa_check(st) == 0

    # the threshold call lays its workspace out for K = d_in
    K_ws = d_in if threshold else K
    ws = L.Workspace()
    buf = ws.get(1, d_in, d_out, K_ws)
    sync = L.larosa_workspace_sync_offset(1, d_in, d_out, K_ws)
    # a fresh workspace: the call is number 1 and counts its arrivals in word 1
    words = buf[sync:sync + 32].view(torch.int32)
    assert int(words.abs().sum()) == 0
    words[1] = 1 << 30
    y = torch.full((1, d_out), float("nan"), dtype=torch.float32, device=dev)
    torch.cuda.synchronize()
    prev = L.larosa_set_wait_limit_ns(1_000_000)
    try:
        t0 = time.perf_counter()
        call(ws, st, y)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
    finally:
        L.larosa_set_wait_limit_ns(prev)
    assert elapsed < 1.0, elapsed
    with pytest.raises(L.LarosaError) as err:
        L.larosa_check(st)
    assert err.value.status == 8  # LAROSA_ERR_TIMEOUT
    assert torch.equal(y, torch.zeros_like(y))  # every CTA gave up before streaming a row

    # recovery: zero the workspace and the status word; the call then returns
    # exactly what it returns on a workspace that never failed
    ws.reset()
    st.zero_()
    y2 = call(ws, st)
    assert L.larosa_check(st) == 0
    assert torch.equal(y2, y_fresh)
    if not threshold:
        # and that result is the oracle's
        _, x_rot, idx, _ = fused_outputs(L, x, Qt, W_rot, K)
        xq, qq = f64(x), f64(Qt).T
        x_rot_ref = oracle.rotate(xq, qq)
        gamma = (d_in + 2) * U * (np.abs(xq) @ np.abs(qq))
        check_selection(x_rot_ref, gamma, idx, K)
        want, _ = oracle.topk(x_rot[0], K)
        assert np.array_equal(idx[0], want)
        W_rot_ref = oracle.round_to_bf16(oracle.prepare_weights(qq, f64(W)))
        ref = oracle.sparse_linear(idx[0], x_rot_ref[0, idx[0]], W_rot_ref)
        assert rel_inf(f64(y2)[0], ref) <= Y_TOL
