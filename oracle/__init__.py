"""fp64 CPU oracle of the LaRoSA rotated-sparse linear path.

TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the benchmark's
CPU-baseline leg import this package; the library never calls it and shares
no code with it.  Every function is a plain restatement in numpy fp64 of what
the pages define, with a library primitive (a matrix product, a sort) as a
step where it serves, and no blocking, fusion or reordering beyond that.

Functions and the passages they follow (page title, section):

* ``rotate``            La RoSA summary, 方法详解 / 技术框架 (rotation stage);
                        abstract ("layerwise orthogonal rotations to transform
                        input activations").
* ``topk``              La RoSA summary, 方法详解 / 技术框架 (sparsification
                        stage: keep the K largest-magnitude entries, zero the
                        rest); abstract ("Top-K selection ... consistent
                        model-level sparsity").
* ``sparse_linear``     the product of the sparsified rotated vector with the
                        counter-rotated weight, restricted to its nonzeros;
                        abstract ("reduce ... memory transfers").
* ``prepare_weights``   W_rot = Q^T W: not printed on the pages; it follows
                        from Q being orthogonal (x W = (x Q)(Q^T W)).
* ``dense_linear``      y = x W, the dense layer the method replaces.
* ``rotate_topk_linear`` the three steps above in the pages' order.
* ``fold_rotation``     the rotation moved into the producing linear layer
                        (x . Q delivered by the producer): a reading, since
                        the pages do not say where Q is applied.
* ``round_to_bf16``     round-to-nearest-even onto bfloat16 (storage format of
                        the prepared weights; not a step of the method).
* ``threshold_select``  R-Sparse report, 研究流程与方法 / R-Sparse框架设计
                        (keep inputs with |x_j| >= t).
* ``lowrank_factors``, ``sparse_lowrank_linear``  same section (low-rank
                        compensation A_r = U_r S_r^1/2, B_r = S_r^1/2 V_r^T and
                        the hybrid output y ~ y_s + y_r).

Readings where the pages are silent:

* orientation: activations are row vectors, x_rot = x . Q, so the weight is
  counter-rotated as Q^T . W (row-major [d_in x d_out]);
* tie-break of equal magnitudes: the lower index wins; +0 and -0 are equal;
* Top-K is per token (per activation row), never per batch;
* the selected entries are returned in ascending index order;
* inputs must be finite (the pages do not define Top-K over NaN).

Every function is pinned by tests against closed forms, invariants, library
routines in special cases or brute force; none is "parity unpinned".
"""
from .larosa_ref import (  # noqa: F401
    rotate,
    topk,
    sparse_linear,
    dense_linear,
    prepare_weights,
    rotate_topk_linear,
    fold_rotation,
    round_to_bf16,
    threshold_select,
    lowrank_factors,
    sparse_lowrank_linear,
)
