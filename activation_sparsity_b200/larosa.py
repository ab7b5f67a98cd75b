"""Python binding of liblarosa.so: argument marshalling only.

Every function here has the name of the C entry point it calls, takes torch
tensors that live on a CUDA device, passes their data pointers, sizes and the
current CUDA stream to the library, and raises LarosaError on a nonzero
status.  All arithmetic happens in the library's CUDA kernels; there is no
CPU or PyTorch fallback, and importing this module fails if the library has
not been built.

Tensors must be contiguous.  Output tensors and the workspace may be passed
in; when omitted they are allocated with torch (the only thing PyTorch does
here besides providing the stream).
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblarosa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m activation_sparsity_b200.build_lib` "
        "(there is no fallback implementation)")

_lib = ctypes.CDLL(LIB_PATH)

_c = ctypes
_vp, _i, _sz = _c.c_void_p, _c.c_int, _c.c_size_t

_SIGNATURES = {
    "larosa_status_string": ([_i], _c.c_char_p),
    "larosa_version": ([], _i),
    "larosa_last_error_string": ([], _c.c_char_p),
    "larosa_prepare_weights": ([_vp, _vp, _vp, _i, _i, _i, _vp], _i),
    "larosa_fold_rotation": ([_vp, _vp, _vp, _i, _i, _i, _vp], _i),
    "larosa_rotate": ([_vp, _vp, _vp, _i, _i, _i, _vp], _i),
    "larosa_topk": ([_vp, _i, _i, _i, _vp, _vp, _vp, _vp], _i),
    "larosa_rotate_topk": ([_vp, _vp, _vp, _vp, _vp, _i, _i, _vp, _sz, _vp, _i, _vp], _i),
    "larosa_sparse_linear": ([_vp, _vp, _i, _i, _vp, _i, _i, _vp, _vp, _sz, _i, _vp, _vp], _i),
    "larosa_rotate_topk_linear": ([_vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _sz, _vp, _i, _vp], _i),
    "larosa_topk_linear": ([_vp, _vp, _i, _i, _i, _i, _vp, _vp, _sz, _vp, _i, _vp], _i),
    "larosa_threshold": ([_vp, _i, _i, _c.c_float, _vp, _vp, _vp, _vp, _vp], _i),
    "larosa_rotate_threshold_linear": ([_vp, _vp, _vp, _i, _i, _i, _c.c_float, _vp, _vp, _sz, _vp, _i,
                                        _vp], _i),
    "larosa_dense_linear": ([_vp, _vp, _i, _i, _i, _vp, _i, _vp], _i),
    "larosa_sparse_lowrank_linear": ([_vp, _vp, _vp, _i, _i, _vp, _vp, _vp, _i, _i, _i, _vp, _vp, _sz, _i, _vp,
                                      _vp], _i),
    "larosa_lowrank_workspace_bytes": ([_i, _i, _i, _i, _i], _sz),
    "larosa_sparse_linear_noalloc": ([_vp, _vp, _i, _i, _vp, _i, _i, _vp, _i, _vp, _vp], _i),
    "larosa_sparse_linear_noalloc_bytes": ([_i, _i, _i, _i, _i], _sz),
    "larosa_workspace_sync_offset": ([_i, _i, _i, _i, _c.POINTER(_sz)], _i),
    "larosa_set_wait_limit_ns": ([_c.c_uint64, _c.POINTER(_c.c_uint64)], _i),
    "larosa_set_debug": ([_i, _c.POINTER(_i)], _i),
    "larosa_set_split_k": ([_i, _c.POINTER(_i)], _i),
    "larosa_workspace_bytes": ([_i, _i, _i, _i], _sz),
    "larosa_workspace_layout": ([_i, _i, _i, _i, _c.POINTER(_sz), _c.POINTER(_sz), _c.POINTER(_sz)], _i),
    "larosa_workspace_nnz_offset": ([_i, _i, _i, _i, _c.POINTER(_sz)], _i),
    "larosa_check": ([_vp, _vp, _c.POINTER(_i)], _i),
}
for _name, (_args, _ret) in _SIGNATURES.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = _ret

LAROSA_F32 = 0
LAROSA_BF16 = 1
LAROSA_OK = 0
LAROSA_ERR_NONFINITE = 7
LAROSA_ERR_TIMEOUT = 8
LAROSA_ERR_INDEX = 9
LAROSA_ERR_LIST = 10
LAROSA_DEV_NONFINITE = 0x1
LAROSA_DEV_TIMEOUT = 0x2
LAROSA_DEV_INDEX = 0x4
LAROSA_DEV_LIST = 0x8
LAROSA_MAX_SPLIT_K = 8
LAROSA_MAX_M = 16
LAROSA_MAX_D = 32768
LAROSA_NOALLOC_SCRATCH_BYTES = 2 << 20


class LarosaError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = _lib.larosa_status_string(status).decode()
        detail = _lib.larosa_last_error_string().decode()
        super().__init__(f"{where}: {msg}" + (f" ({detail})" if detail and status == 5 else ""))
        self.status = status


def _check(status: int, where: str) -> None:
    if status != LAROSA_OK:
        raise LarosaError(status, where)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _as2d(t: torch.Tensor) -> torch.Tensor:
    return t if t.dim() == 2 else t.reshape(1, -1)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return LAROSA_BF16
    if t.dtype == torch.float32:
        return LAROSA_F32
    raise TypeError(f"unsupported dtype {t.dtype}: bfloat16 or float32")


def _need(t: torch.Tensor, name: str, dtype=None) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


# ------------------------------------------------------------------ workspace

class Workspace:
    """A zero-initialised scratch buffer for one stream, grown on demand.

    The library leaves the counter words it uses at zero after every call, so
    the buffer is reused without clearing.  A buffer serves one stream at a
    time; calls on different streams that may overlap need their own.
    """

    def __init__(self, device=None):
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None \
            else torch.device(device)
        self.buf = torch.zeros(0, dtype=torch.uint8, device=self.device)
        self._need: dict[tuple[int, int, int, int], int] = {}

    def get(self, M: int, d_in: int, d_out: int, K: int) -> torch.Tensor:
        key = (M, d_in, d_out, K)
        need = self._need.get(key)
        if need is None:
            with torch.cuda.device(self.device):
                need = int(_lib.larosa_workspace_bytes(M, d_in, d_out, K))
            if need == 0:
                raise LarosaError(2, "larosa_workspace_bytes")
            self._need[key] = need
        if self.buf.numel() < need:
            self.buf = torch.zeros(need, dtype=torch.uint8, device=self.device)
        return self.buf

    def reset(self) -> None:
        """Zero the buffer again (needed after a device-side error)."""
        self.buf.zero_()


_ws_lock = threading.Lock()
_ws_cache: dict[tuple[int, int], Workspace] = {}
_status_cache: dict[int, torch.Tensor] = {}


def default_workspace(device: torch.device) -> Workspace:
    key = (device.index, torch.cuda.current_stream(device).cuda_stream)
    with _ws_lock:
        ws = _ws_cache.get(key)
        if ws is None:
            ws = _ws_cache[key] = Workspace(device)
        return ws


def default_status(device: torch.device) -> torch.Tensor:
    """The per-device status word used when none is passed (see larosa_check)."""
    with _ws_lock:
        st = _status_cache.get(device.index)
        if st is None:
            st = _status_cache[device.index] = torch.zeros(1, dtype=torch.int32, device=device)
        return st


def _ws_args(ws, device, M, d_in, d_out, K):
    if ws is None:
        ws = default_workspace(device)
    buf = ws.get(M, d_in, d_out, K) if isinstance(ws, Workspace) else ws
    return ctypes.c_void_p(buf.data_ptr()), ctypes.c_size_t(buf.numel() * buf.element_size())


def _status_ptr(dev_status, device):
    return _ptr(default_status(device) if dev_status is None else dev_status)


# ------------------------------------------------------------------ entry points

def larosa_version() -> int:
    return int(_lib.larosa_version())


def larosa_workspace_bytes(M: int, d_in: int, d_out: int, K: int) -> int:
    return int(_lib.larosa_workspace_bytes(M, d_in, d_out, K))


def larosa_lowrank_workspace_bytes(M: int, d_in: int, d_out: int, K: int, r: int) -> int:
    return int(_lib.larosa_lowrank_workspace_bytes(M, d_in, d_out, K, r))


def larosa_workspace_layout(M: int, d_in: int, d_out: int, K: int) -> tuple[int, int, int]:
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(_lib.larosa_workspace_layout(M, d_in, d_out, K, ctypes.byref(a), ctypes.byref(b),
                                        ctypes.byref(c)), "larosa_workspace_layout")
    return a.value, b.value, c.value


def larosa_workspace_nnz_offset(M: int, d_in: int, d_out: int, K: int) -> int:
    a = ctypes.c_size_t()
    _check(_lib.larosa_workspace_nnz_offset(M, d_in, d_out, K, ctypes.byref(a)),
           "larosa_workspace_nnz_offset")
    return a.value


def larosa_workspace_sync_offset(M: int, d_in: int, d_out: int, K: int) -> int:
    a = ctypes.c_size_t()
    _check(_lib.larosa_workspace_sync_offset(M, d_in, d_out, K, ctypes.byref(a)),
           "larosa_workspace_sync_offset")
    return a.value


def larosa_set_wait_limit_ns(limit_ns: int) -> int:
    """Sets the in-kernel wait limit for later launches (0: the default);
    returns the previous limit."""
    prev = ctypes.c_uint64(0)
    _check(_lib.larosa_set_wait_limit_ns(int(limit_ns), ctypes.byref(prev)), "larosa_set_wait_limit_ns")
    return prev.value


def larosa_set_debug(on: bool) -> bool:
    """Turns the library's debug checks of kept lists on or off for later
    calls; returns the previous setting (see larosa_set_debug in the header)."""
    prev = ctypes.c_int(0)
    _check(_lib.larosa_set_debug(1 if on else 0, ctypes.byref(prev)), "larosa_set_debug")
    return bool(prev.value)


def larosa_set_split_k(splits: int) -> int:
    """Forces the reduction split of the tensor-core kernels of 2 to 16 tokens
    (0: chosen per shape); returns the previous setting."""
    prev = ctypes.c_int(0)
    _check(_lib.larosa_set_split_k(int(splits), ctypes.byref(prev)), "larosa_set_split_k")
    return prev.value


def larosa_sparse_linear_noalloc_bytes(M: int, d_in: int, d_out: int, K: int,
                                       dtype: torch.dtype = torch.bfloat16) -> int:
    code = LAROSA_BF16 if dtype == torch.bfloat16 else LAROSA_F32
    return int(_lib.larosa_sparse_linear_noalloc_bytes(M, d_in, d_out, K, code))


def larosa_prepare_weights(Qt: torch.Tensor, W: torch.Tensor, W_rot: torch.Tensor | None = None
                           ) -> torch.Tensor:
    """W_rot = Q^T . W = Qt . W (offline counter-rotation), same dtype as W.

    Qt is the rotation stored transposed (Qt = Q.T.contiguous() for x_rot = x @ Q).
    """
    _need(Qt, "Qt")
    _need(W, "W", Qt.dtype)
    d_in, d_out = W.shape
    if W_rot is None:
        W_rot = torch.empty_like(W)
    _need(W_rot, "W_rot", W.dtype)
    _check(_lib.larosa_prepare_weights(_ptr(Qt), _ptr(W), _ptr(W_rot), d_in, d_out, _dtype_code(W),
                                       _stream(W.device)), "larosa_prepare_weights")
    return W_rot


def larosa_fold_rotation(Qt: torch.Tensor, Wt_prev: torch.Tensor, out: torch.Tensor | None = None
                         ) -> torch.Tensor:
    """Q^T . Wt_prev: the producer's nn.Linear weight [d, d_prev] after folding the
    rotation into it, so that the producer outputs x . Q."""
    _need(Qt, "Qt")
    _need(Wt_prev, "Wt_prev", Qt.dtype)
    d, d_prev = Wt_prev.shape
    if out is None:
        out = torch.empty_like(Wt_prev)
    _need(out, "out", Wt_prev.dtype)
    _check(_lib.larosa_fold_rotation(_ptr(Qt), _ptr(Wt_prev), _ptr(out), d, d_prev, _dtype_code(Wt_prev),
                                     _stream(Wt_prev.device)), "larosa_fold_rotation")
    return out


def larosa_rotate(x: torch.Tensor, Qt: torch.Tensor, x_rot: torch.Tensor | None = None
                  ) -> torch.Tensor:
    """x_rot = x . Q with Qt = Q^T, fp32 output [M, d]."""
    _need(x, "x")
    _need(Qt, "Qt", x.dtype)
    x2 = _as2d(x)
    M, d = x2.shape
    if x_rot is None:
        x_rot = torch.empty((M, d), dtype=torch.float32, device=x.device)
    _need(x_rot, "x_rot", torch.float32)
    _check(_lib.larosa_rotate(_ptr(x2), _ptr(Qt), _ptr(x_rot), M, d, _dtype_code(x),
                              _stream(x.device)), "larosa_rotate")
    return x_rot


def larosa_topk(x_rot: torch.Tensor, K: int, idx: torch.Tensor | None = None,
                val: torch.Tensor | None = None, dev_status: torch.Tensor | None = None
                ) -> tuple[torch.Tensor, torch.Tensor]:
    """Per-row Top-K by magnitude: (idx int32 [M, K] ascending, val fp32 [M, K])."""
    _need(x_rot, "x_rot", torch.float32)
    x2 = _as2d(x_rot)
    M, d = x2.shape
    if idx is None:
        idx = torch.empty((M, K), dtype=torch.int32, device=x_rot.device)
    if val is None:
        val = torch.empty((M, K), dtype=torch.float32, device=x_rot.device)
    _need(idx, "idx", torch.int32)
    _need(val, "val", torch.float32)
    _check(_lib.larosa_topk(_ptr(x2), M, d, K, _ptr(idx), _ptr(val),
                            _status_ptr(dev_status, x_rot.device), _stream(x_rot.device)),
           "larosa_topk")
    return idx, val


def larosa_rotate_topk(x: torch.Tensor, Qt: torch.Tensor, K: int, x_rot: torch.Tensor | None = None,
                       idx: torch.Tensor | None = None, val: torch.Tensor | None = None, ws=None,
                       dev_status: torch.Tensor | None = None
                       ) -> tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """One token: x_rot = x @ Q (Qt = Q^T) and its Top-K by magnitude in one
    kernel; returns (x_rot fp32 [1, d], idx int32 [1, K] ascending, val fp32 [1, K])."""
    _need(x, "x")
    _need(Qt, "Qt", x.dtype)
    x2 = _as2d(x)
    M, d = x2.shape
    if M != 1:
        raise LarosaError(2, "larosa_rotate_topk: one token only")
    if x_rot is None:
        x_rot = torch.empty((1, d), dtype=torch.float32, device=x.device)
    if idx is None:
        idx = torch.empty((1, K), dtype=torch.int32, device=x.device)
    if val is None:
        val = torch.empty((1, K), dtype=torch.float32, device=x.device)
    _need(x_rot, "x_rot", torch.float32)
    _need(idx, "idx", torch.int32)
    _need(val, "val", torch.float32)
    p, n = _ws_args(ws, x.device, 1, d, 1, K)
    _check(_lib.larosa_rotate_topk(_ptr(x2), _ptr(Qt), _ptr(x_rot), _ptr(idx), _ptr(val), d, K, p, n,
                                   _status_ptr(dev_status, x.device), _dtype_code(x),
                                   _stream(x.device)), "larosa_rotate_topk")
    return x_rot, idx, val


def larosa_sparse_linear(idx: torch.Tensor, val: torch.Tensor, W_rot: torch.Tensor,
                         y: torch.Tensor | None = None, ws=None,
                         dev_status: torch.Tensor | None = None) -> torch.Tensor:
    """y = sum_k val[:, k] * W_rot[idx[:, k]], fp32 [M, d_out]."""
    _need(idx, "idx", torch.int32)
    _need(val, "val", torch.float32)
    _need(W_rot, "W_rot")
    i2 = _as2d(idx)
    val = _as2d(val)
    M, K = i2.shape
    d_in, d_out = W_rot.shape
    if y is None:
        y = torch.empty((M, d_out), dtype=torch.float32, device=W_rot.device)
    _need(y, "y", torch.float32)
    p, n = _ws_args(ws, W_rot.device, M, d_in, d_out, K)
    _check(_lib.larosa_sparse_linear(_ptr(i2), _ptr(val), M, K, _ptr(W_rot), d_in, d_out, _ptr(y),
                                     p, n, _dtype_code(W_rot), _status_ptr(dev_status, W_rot.device),
                                     _stream(W_rot.device)), "larosa_sparse_linear")
    return y


def larosa_sparse_linear_noalloc(idx: torch.Tensor, val: torch.Tensor, W_rot: torch.Tensor,
                                 y: torch.Tensor | None = None,
                                 dev_status: torch.Tensor | None = None) -> torch.Tensor:
    """larosa_sparse_linear with the library's fixed device scratch instead of a
    workspace (for callers that cannot allocate); calls on one device must not
    overlap."""
    _need(idx, "idx", torch.int32)
    _need(val, "val", torch.float32)
    _need(W_rot, "W_rot")
    i2 = _as2d(idx)
    val = _as2d(val)
    M, K = i2.shape
    d_in, d_out = W_rot.shape
    if y is None:
        y = torch.empty((M, d_out), dtype=torch.float32, device=W_rot.device)
    _need(y, "y", torch.float32)
    status = _lib.larosa_sparse_linear_noalloc(_ptr(i2), _ptr(val), M, K, _ptr(W_rot), d_in, d_out,
                                               _ptr(y), _dtype_code(W_rot),
                                               _status_ptr(dev_status, W_rot.device),
                                               _stream(W_rot.device))
    if status != LAROSA_OK:
        raise LarosaError(status, "larosa_sparse_linear_noalloc: "
                          + _lib.larosa_last_error_string().decode())
    return y


def larosa_rotate_topk_linear(x: torch.Tensor, Qt: torch.Tensor | None, W_rot: torch.Tensor, K: int,
                              y: torch.Tensor | None = None, ws=None,
                              dev_status: torch.Tensor | None = None) -> torch.Tensor:
    """Fused rotate -> Top-K -> sparse linear (Qt = Q^T), fp32 output [M, d_out].

    Qt = None is the identity rotation (the unrotated fixed-K mode)."""
    _need(x, "x")
    if Qt is not None:
        _need(Qt, "Qt", x.dtype)
    _need(W_rot, "W_rot", x.dtype)
    x2 = _as2d(x)
    M, d_in = x2.shape
    d_out = W_rot.shape[1]
    if y is None:
        y = torch.empty((M, d_out), dtype=torch.float32, device=x.device)
    _need(y, "y", torch.float32)
    p, n = _ws_args(ws, x.device, M, d_in, d_out, K)
    _check(_lib.larosa_rotate_topk_linear(_ptr(x2), _ptr(Qt), _ptr(W_rot), M, d_in, d_out, K, _ptr(y),
                                          p, n, _status_ptr(dev_status, x.device), _dtype_code(x),
                                          _stream(x.device)), "larosa_rotate_topk_linear")
    return y


def larosa_topk_linear(x_rot: torch.Tensor, W_rot: torch.Tensor, K: int, y: torch.Tensor | None = None,
                       ws=None, dev_status: torch.Tensor | None = None) -> torch.Tensor:
    """Top-K of an already rotated fp32 vector and the sparse linear over the kept
    rows of W_rot, fp32 output [M, d_out] (the kept list stays in the workspace)."""
    _need(x_rot, "x_rot", torch.float32)
    _need(W_rot, "W_rot")
    x2 = _as2d(x_rot)
    M, d_in = x2.shape
    d_out = W_rot.shape[1]
    if W_rot.shape[0] != d_in:
        raise ValueError("W_rot must be [d_in, d_out]")
    if y is None:
        y = torch.empty((M, d_out), dtype=torch.float32, device=x_rot.device)
    _need(y, "y", torch.float32)
    p, n = _ws_args(ws, x_rot.device, M, d_in, d_out, K)
    _check(_lib.larosa_topk_linear(_ptr(x2), _ptr(W_rot), M, d_in, d_out, K, _ptr(y), p, n,
                                   _status_ptr(dev_status, x_rot.device), _dtype_code(W_rot),
                                   _stream(x_rot.device)), "larosa_topk_linear")
    return y


def larosa_threshold(x_rot: torch.Tensor, t: float, idx: torch.Tensor | None = None,
                     val: torch.Tensor | None = None, nnz: torch.Tensor | None = None,
                     dev_status: torch.Tensor | None = None
                     ) -> tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Per-row threshold selection |x_rot| >= t: (idx int32 [M, d], val fp32 [M, d],
    nnz int32 [M]); row m's first nnz[m] entries are the kept ones, ascending."""
    _need(x_rot, "x_rot", torch.float32)
    x2 = _as2d(x_rot)
    M, d = x2.shape
    dev = x_rot.device
    if idx is None:
        idx = torch.empty((M, d), dtype=torch.int32, device=dev)
    if val is None:
        val = torch.empty((M, d), dtype=torch.float32, device=dev)
    if nnz is None:
        nnz = torch.empty((M,), dtype=torch.int32, device=dev)
    _need(idx, "idx", torch.int32)
    _need(val, "val", torch.float32)
    _need(nnz, "nnz", torch.int32)
    _check(_lib.larosa_threshold(_ptr(x2), M, d, float(t), _ptr(idx), _ptr(val), _ptr(nnz),
                                 _status_ptr(dev_status, dev), _stream(dev)), "larosa_threshold")
    return idx, val, nnz


def larosa_rotate_threshold_linear(x: torch.Tensor, Qt: torch.Tensor | None, W_rot: torch.Tensor,
                                   t: float, y: torch.Tensor | None = None, ws=None,
                                   dev_status: torch.Tensor | None = None) -> torch.Tensor:
    """Fused rotate -> threshold |x_rot| >= t -> sparse linear, fp32 output [M, d_out].

    Qt = None is the identity rotation.  The kept lists and counts stay in the
    workspace (larosa_workspace_layout / larosa_workspace_nnz_offset with K = d_in)."""
    _need(x, "x")
    if Qt is not None:
        _need(Qt, "Qt", x.dtype)
    _need(W_rot, "W_rot", x.dtype)
    x2 = _as2d(x)
    M, d_in = x2.shape
    d_out = W_rot.shape[1]
    if y is None:
        y = torch.empty((M, d_out), dtype=torch.float32, device=x.device)
    _need(y, "y", torch.float32)
    p, n = _ws_args(ws, x.device, M, d_in, d_out, d_in)
    _check(_lib.larosa_rotate_threshold_linear(_ptr(x2), _ptr(Qt), _ptr(W_rot), M, d_in, d_out, float(t),
                                               _ptr(y), p, n, _status_ptr(dev_status, x.device),
                                               _dtype_code(x), _stream(x.device)),
           "larosa_rotate_threshold_linear")
    return y


def larosa_sparse_lowrank_linear(x: torch.Tensor, idx: torch.Tensor, val: torch.Tensor, W: torch.Tensor,
                                 A_r: torch.Tensor, B_r: torch.Tensor, y: torch.Tensor | None = None,
                                 ws: torch.Tensor | None = None, dev_status: torch.Tensor | None = None
                                 ) -> torch.Tensor:
    """y = sparse(x) . W + ((x - sparse(x)) . A_r) . B_r for the kept lists idx/val of x (fp32)."""
    _need(x, "x", torch.float32)
    _need(W, "W")
    _need(A_r, "A_r", W.dtype)
    _need(B_r, "B_r", W.dtype)
    x2 = _as2d(x)
    M, d_in = x2.shape
    d_out, r = W.shape[1], A_r.shape[1]
    idx2, val2 = _as2d(idx), _as2d(val)
    K = idx2.shape[1]
    _need(idx2, "idx", torch.int32)
    _need(val2, "val", torch.float32)
    if y is None:
        y = torch.empty((M, d_out), dtype=torch.float32, device=x.device)
    _need(y, "y", torch.float32)
    nb = int(_lib.larosa_lowrank_workspace_bytes(M, d_in, d_out, K, r))
    if nb == 0:
        raise LarosaError(2, "larosa_lowrank_workspace_bytes")
    if ws is None or ws.numel() * ws.element_size() < nb:
        ws = torch.zeros(nb, dtype=torch.uint8, device=x.device)
    _check(_lib.larosa_sparse_lowrank_linear(_ptr(x2), _ptr(idx2), _ptr(val2), M, K, _ptr(W), _ptr(A_r),
                                             _ptr(B_r), d_in, d_out, r, _ptr(y), _ptr(ws),
                                             ws.numel() * ws.element_size(), _dtype_code(W),
                                             _status_ptr(dev_status, x.device), _stream(x.device)),
           "larosa_sparse_lowrank_linear")
    return y


def larosa_dense_linear(x: torch.Tensor, Wt: torch.Tensor, y: torch.Tensor | None = None
                        ) -> torch.Tensor:
    """Dense baseline y = x . W with Wt = W^T in torch.nn.Linear layout [d_out, d_in]."""
    _need(x, "x")
    _need(Wt, "Wt", x.dtype)
    x2 = _as2d(x)
    M, d_in = x2.shape
    d_out = Wt.shape[0]
    if Wt.shape[1] != d_in:
        raise ValueError("Wt must be [d_out, d_in]")
    if y is None:
        y = torch.empty((M, d_out), dtype=torch.float32, device=x.device)
    _need(y, "y", torch.float32)
    _check(_lib.larosa_dense_linear(_ptr(x2), _ptr(Wt), M, d_in, d_out, _ptr(y), _dtype_code(x),
                                    _stream(x.device)), "larosa_dense_linear")
    return y


def larosa_check(dev_status: torch.Tensor | None = None, device=None) -> int:
    """Synchronises the current stream and returns the raw device status bits.

    Raises LarosaError for a nonzero word (the status of its lowest bit).
    """
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    st = default_status(device) if dev_status is None else dev_status
    flags = ctypes.c_int(0)
    status = _lib.larosa_check(_ptr(st), _stream(st.device), ctypes.byref(flags))
    _check(status, "larosa_check")
    return flags.value


def raw_library() -> ctypes.CDLL:
    """The loaded ctypes library (for tests of the C ABI itself)."""
    return _lib
