"""Full-size parity on the LLaMA2-7B decoder layer, batch 1, 40 % sparsity,
in the launch configuration the benchmark times (default workspace, same
shapes).  The oracle recomputes the exact rotation, checks the kept set and
evaluates sampled output columns one by one.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.test_gpu_parity import (U, Y_TOL, check_bf16_rounding, check_selection, f64,
                                   fused_outputs, rel_inf)

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def layer():
    from activation_sparsity_b200 import build_lib
    build_lib.build()
    from activation_sparsity_b200.workload import build_layer
    return build_layer(4096, 11008, 4096, 40.0, workload_id=1, layer=0, device=torch.device("cuda"))


@pytest.mark.parametrize("gi", [0, 1, 2, 3])
def test_llama2_7b_layer_group(layer, gi):
    import activation_sparsity_b200 as L
    g = layer.groups[gi]
    y, x_rot, idx, val = fused_outputs(L, g.x, g.Qt, g.W_rot, g.K)
    xq, qq = f64(g.x), f64(g.Qt).T
    x_rot_ref = oracle.rotate(xq, qq)
    gamma = (g.d_in + 2) * U * (np.abs(xq) @ np.abs(qq))
    assert np.all(np.abs(x_rot - x_rot_ref) <= gamma + 1e-30)
    check_selection(x_rot_ref, gamma, idx, g.K)
    # the kept set is exactly the oracle's Top-K of the kernel's own fp32 x_rot
    # (checked against the exact rotation just above), ties to the lower index
    want, _ = oracle.topk(x_rot[0], g.K)
    assert np.array_equal(idx[0], want)
    assert np.array_equal(val[0], x_rot[0, idx[0]].astype(np.float32))
    rng = np.random.default_rng(1000 + gi)
    cols = np.sort(rng.choice(g.d_out, size=96, replace=False))
    Wc = f64(g.W[:, torch.from_numpy(cols).cuda()])
    exact = oracle.prepare_weights(qq, Wc)
    W_rot_ref = oracle.round_to_bf16(exact)
    got_w = f64(g.W_rot[:, torch.from_numpy(cols).cuda()])
    check_bf16_rounding(got_w, exact, (g.d_in + 2) * U * (np.abs(qq).T @ np.abs(Wc)))
    ref = oracle.sparse_linear(idx[0], x_rot_ref[0, idx[0]], W_rot_ref)
    assert rel_inf(y[0, cols], ref) <= Y_TOL
