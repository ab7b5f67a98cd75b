"""B200-native (sm_100a) LaRoSA rotated-sparse linear.

For each token entering a linear layer: rotate the activation by the layer's
orthogonal Q, keep its K largest-magnitude entries, and multiply by the
counter-rotated weight W_rot = Q^T W, reading only the K kept rows
("La RoSA: Enhancing LLM Efficiency via Layerwise Rotated Sparse
Activation", method and abstract).  The same path also runs with the
identity rotation (no Q: fixed-K magnitude sparsity) and with a threshold
|x_rot| >= t in place of the Top-K (the threshold function of the R-Sparse
report).

The compute lives in liblarosa.so (C ABI, include/larosa.h); the submodule
``larosa`` is its thin Python binding and is loaded on first use of any name
below.  Loading fails loudly if the library is not built: there is no
fallback path.  (``build_lib`` builds the library without loading it.)
"""
_EXPORTS = (
    "LarosaError", "Workspace", "larosa_check", "larosa_dense_linear", "larosa_prepare_weights",
    "larosa_rotate", "larosa_rotate_topk", "larosa_rotate_topk_linear", "larosa_sparse_linear",
    "larosa_topk_linear",
    "larosa_sparse_linear_noalloc", "larosa_topk", "larosa_version", "larosa_workspace_bytes",
    "larosa_workspace_layout", "larosa_workspace_nnz_offset", "larosa_threshold",
    "larosa_rotate_threshold_linear", "larosa_fold_rotation",
    "larosa_sparse_lowrank_linear", "larosa_lowrank_workspace_bytes", "larosa_sparse_linear_noalloc_bytes",
    "larosa_workspace_sync_offset", "larosa_set_wait_limit_ns", "larosa_set_debug", "larosa_set_split_k",
    "LAROSA_OK", "LAROSA_ERR_NONFINITE", "LAROSA_ERR_TIMEOUT", "LAROSA_ERR_INDEX", "LAROSA_ERR_LIST",
    "LAROSA_DEV_NONFINITE", "LAROSA_DEV_TIMEOUT", "LAROSA_DEV_INDEX", "LAROSA_DEV_LIST", "LAROSA_MAX_SPLIT_K",
    "LAROSA_NOALLOC_SCRATCH_BYTES", "LAROSA_F32", "LAROSA_BF16", "LAROSA_MAX_D", "LAROSA_MAX_M",
    "LIB_PATH",
)
__all__ = list(_EXPORTS)


def __getattr__(name):
    if name in _EXPORTS:
        from . import larosa
        return getattr(larosa, name)
    raise AttributeError(f"module {__name__!r} has no attribute {name!r}")
