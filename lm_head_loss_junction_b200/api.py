"""Torch-tensor front end of libmls.

Each function checks tensor shapes/dtypes, allocates outputs with torch when
the caller does not pass them, and forwards raw pointers to the C ABI of the
same name (``mls_*``).  Every step of the computation runs in the library's
CUDA kernels; nothing here computes.
"""
from __future__ import annotations

import ctypes
from typing import List, Optional, Sequence, Tuple

import torch

from . import _lib
from ._lib import MLS_BF16, MLS_F32, check, i64_array, lib, ptr_array


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return MLS_BF16
    if t.dtype == torch.float32:
        return MLS_F32
    raise TypeError(f"unsupported dtype {t.dtype}; expected bfloat16 or float32")


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _need(t: torch.Tensor, name: str, dtype=None, ndim=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims")


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


# ---------------------------------------------------------------- junction
def junction_fwd(x: torch.Tensor, o: torch.Tensor, E: torch.Tensor, *, out=None, scale_out=None,
                 variant: int = 0, status=None, stream=None) -> torch.Tensor:
    """y = [ (||E[x]|| / ||o||) o ; E[x] ] per token (see mls_junction_fwd; `variant`
    selects an ablation, see mls_junction_fwd_variant)."""
    _need(x, "x", torch.int32, 1)
    _need(o, "o", ndim=2)
    _need(E, "E", o.dtype, 2)
    T, D = o.shape
    V, delta = E.shape
    if x.shape[0] != T:
        raise ValueError("x and o disagree on T")
    y = out if out is not None else torch.empty((T, D + delta), dtype=o.dtype, device=o.device)
    _need(y, "out", o.dtype, 2)
    if scale_out is not None:
        _need(scale_out, "scale_out", torch.float32, 1)
    if variant:
        code = lib().mls_junction_fwd_variant(x.data_ptr(), T, o.data_ptr(), D, E.data_ptr(), V, delta,
                                              y.data_ptr(), _ptr(scale_out), int(variant), _dtype_code(o),
                                              _ptr(status), _stream_ptr(stream))
    else:
        code = lib().mls_junction_fwd(x.data_ptr(), T, o.data_ptr(), D, E.data_ptr(), V, delta, y.data_ptr(),
                                      _ptr(scale_out), _dtype_code(o), _ptr(status), _stream_ptr(stream))
    check("mls_junction_fwd", code)
    return y


def junction_bwd_workspace(T: int, V: int) -> int:
    n = ctypes.c_size_t()
    check("mls_junction_bwd_workspace", lib().mls_junction_bwd_workspace(T, V, ctypes.byref(n)))
    return n.value


def junction_bwd(x: torch.Tensor, o: torch.Tensor, E: torch.Tensor, dy: torch.Tensor, *,
                 want_de_rows: bool = True, dE: Optional[torch.Tensor] = None, accumulate_dE: bool = False,
                 do_out=None, de_out=None, workspace=None, variant: int = 0, status=None, stream=None):
    """Returns (do, de_rows or None, dE or None) (see mls_junction_bwd)."""
    _need(x, "x", torch.int32, 1)
    _need(o, "o", ndim=2)
    _need(E, "E", o.dtype, 2)
    _need(dy, "dy", o.dtype, 2)
    T, D = o.shape
    V, delta = E.shape
    if tuple(dy.shape) != (T, D + delta):
        raise ValueError("dy must be [T, D + delta]")
    do = do_out if do_out is not None else torch.empty_like(o)
    de = de_out
    if de is None and want_de_rows:
        de = torch.empty((T, delta), dtype=o.dtype, device=o.device)
    ws_bytes = 0
    if dE is not None:
        _need(dE, "dE", torch.float32, 2)
        ws_bytes = junction_bwd_workspace(T, V)
        if workspace is None:
            workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=o.device)
        ws_bytes = workspace.numel() * workspace.element_size()
    if variant:
        code = lib().mls_junction_bwd_variant(x.data_ptr(), T, o.data_ptr(), D, E.data_ptr(), V, delta,
                                              dy.data_ptr(), do.data_ptr(), _ptr(de), _ptr(dE),
                                              int(bool(accumulate_dE)), _ptr(workspace), ws_bytes, int(variant),
                                              _dtype_code(o), _ptr(status), _stream_ptr(stream))
    else:
        code = lib().mls_junction_bwd(x.data_ptr(), T, o.data_ptr(), D, E.data_ptr(), V, delta, dy.data_ptr(),
                                      do.data_ptr(), _ptr(de), _ptr(dE), int(bool(accumulate_dE)),
                                      _ptr(workspace), ws_bytes, _dtype_code(o), _ptr(status),
                                      _stream_ptr(stream))
    check("mls_junction_bwd", code)
    return do, de, dE


def junction_fwd_multi(x: torch.Tensor, o: Sequence[torch.Tensor], E: Sequence[torch.Tensor], *, out=None,
                       scale_out=None, status=None, stream=None) -> List[torch.Tensor]:
    """Every junction of a suite in one call: y[k] = junction(o[k], E[k]) (see mls_junction_fwd_multi)."""
    J = len(o)
    if len(E) != J or J < 1:
        raise ValueError("o and E must be non-empty lists of the same length")
    _need(x, "x", torch.int32, 1)
    T = x.shape[0]
    V = E[0].shape[0]
    D = [o[0].shape[1]]
    for k in range(J):
        _need(o[k], f"o[{k}]", o[0].dtype, 2)
        _need(E[k], f"E[{k}]", o[0].dtype, 2)
        if o[k].shape[0] != T or E[k].shape[0] != V or o[k].shape[1] != D[k]:
            raise ValueError(f"junction {k}: o must be [T, D_k] (D_k the previous junction's output width)")
        D.append(D[k] + E[k].shape[1])
    y = out if out is not None else [torch.empty((T, D[k + 1]), dtype=o[0].dtype, device=x.device)
                                     for k in range(J)]
    for k in range(J):
        _need(y[k], f"out[{k}]", o[0].dtype, 2)
    sc = None
    if scale_out is not None:
        sc = ptr_array([_ptr(t) for t in scale_out])
    code = lib().mls_junction_fwd_multi(x.data_ptr(), T, V, J, i64_array(D), ptr_array([t.data_ptr() for t in o]),
                                        ptr_array([t.data_ptr() for t in E]), ptr_array([t.data_ptr() for t in y]),
                                        sc, _dtype_code(o[0]), _ptr(status), _stream_ptr(stream))
    check("mls_junction_fwd_multi", code)
    return y


def junction_bwd_multi_workspace(T: int, V: int, J: int) -> int:
    n = ctypes.c_size_t()
    check("mls_junction_bwd_multi_workspace", lib().mls_junction_bwd_multi_workspace(T, V, J, ctypes.byref(n)))
    return n.value


def junction_bwd_multi(x: torch.Tensor, o: Sequence[torch.Tensor], E: Sequence[torch.Tensor],
                       dy: Sequence[torch.Tensor], *, do_out=None, de_out=None, dE=None, accumulate_dE=False,
                       workspace=None, status=None, stream=None):
    """Backward of every junction of a suite in one call (see mls_junction_bwd_multi).
    de_out / dE: lists (entries may be None) or None.  Returns (do list, de list, dE list)."""
    J = len(o)
    _need(x, "x", torch.int32, 1)
    T = x.shape[0]
    V = E[0].shape[0]
    D = [o[0].shape[1]] + [o[0].shape[1]] * J
    for k in range(J):
        D[k + 1] = D[k] + E[k].shape[1]
        if tuple(dy[k].shape) != (T, D[k + 1]):
            raise ValueError(f"dy[{k}] must be [T, D_k+1]")
    do = do_out if do_out is not None else [torch.empty_like(t) for t in o]
    de = de_out if de_out is not None else [None] * J
    tables = dE if dE is not None else [None] * J
    ws_bytes = 0
    if any(t is not None for t in tables):
        ws_bytes = junction_bwd_multi_workspace(T, V, J)
        if workspace is None:
            workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=x.device)
        ws_bytes = workspace.numel() * workspace.element_size()
    code = lib().mls_junction_bwd_multi(x.data_ptr(), T, V, J, i64_array(D), ptr_array([t.data_ptr() for t in o]),
                                        ptr_array([t.data_ptr() for t in E]), ptr_array([t.data_ptr() for t in dy]),
                                        ptr_array([t.data_ptr() for t in do]), ptr_array([_ptr(t) for t in de]),
                                        ptr_array([_ptr(t) for t in tables]), int(bool(accumulate_dE)),
                                        _ptr(workspace), ws_bytes, _dtype_code(o[0]), _ptr(status),
                                        _stream_ptr(stream))
    check("mls_junction_bwd_multi", code)
    return do, de, tables


# ---------------------------------------------------------------- multi-exit loss
def multiexit_loss_workspace(T: int, D: Sequence[int], V: int, dtype: torch.dtype) -> Tuple[int, int]:
    f = ctypes.c_size_t()
    b = ctypes.c_size_t()
    code = lib().mls_multiexit_loss_workspace(len(D), T, i64_array(D), V,
                                              MLS_BF16 if dtype == torch.bfloat16 else MLS_F32,
                                              ctypes.byref(f), ctypes.byref(b))
    check("mls_multiexit_loss_workspace", code)
    return f.value, b.value


def multiexit_loss_bwd_plan(T: int, D: Sequence[int], V: int, dtype: torch.dtype, ws_bytes: int):
    """(Tb, Vc, min_bytes): how the backward call splits its work for a workspace of ws_bytes
    (see mls_multiexit_loss_bwd_plan)."""
    tb = ctypes.c_int64()
    vc = ctypes.c_int64()
    mn = ctypes.c_size_t()
    code = lib().mls_multiexit_loss_bwd_plan(len(D), T, i64_array(D), V,
                                             MLS_BF16 if dtype == torch.bfloat16 else MLS_F32, int(ws_bytes),
                                             ctypes.byref(tb), ctypes.byref(vc), ctypes.byref(mn))
    check("mls_multiexit_loss_bwd_plan", code)
    return tb.value, vc.value, mn.value


def _loss_common(y, h, W):
    M = len(h)
    if len(W) != M or M < 1:
        raise ValueError("h and W must be non-empty lists of the same length")
    _need(y, "y", torch.int32, 1)
    T = y.shape[0]
    V = W[0].shape[0]
    dt = h[0].dtype
    D = []
    for m in range(M):
        _need(h[m], f"h[{m}]", dt, 2)
        _need(W[m], f"W[{m}]", dt, 2)
        if h[m].shape[0] != T or W[m].shape[0] != V or h[m].shape[1] != W[m].shape[1]:
            raise ValueError(f"exit {m}: h must be [T, D_m] and W [V, D_m]")
        D.append(h[m].shape[1])
    return M, T, V, D, dt


def _workspace(ws, nbytes, device):
    if ws is None:
        ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=device)
    return ws, ws.numel() * ws.element_size()


def multiexit_loss_fwd(y: torch.Tensor, h: List[torch.Tensor], W: List[torch.Tensor], alpha_d: float = 0.3, *,
                       losses=None, stats=None, workspace=None, exit_weights=None, distill="ce",
                       teacher_grad: bool = False, status=None, stream=None):
    """Returns (losses [2M], stats [3M-1, T], or [4M-2, T] for Jensen-Shannon or acceptance
    with the teacher gradient) (see mls_multiexit_loss_fwd; any option uses mls_multiexit_loss_fwd_opts)."""
    M, T, V, D, dt = _loss_common(y, h, W)
    dev = y.device
    if losses is None:
        losses = torch.empty(2 * M, dtype=torch.float32, device=dev)
    rows = 4 * M - 2 if (distill in ("js", "accept") and teacher_grad and M > 1) else 3 * M - 1
    if stats is None:
        stats = torch.empty((rows, T), dtype=torch.float32, device=dev)
    elif stats.shape[0] < rows:
        raise ValueError(f"stats needs {rows} rows")
    fwd_b, _ = multiexit_loss_workspace(T, D, V, dt)
    workspace, ws_bytes = _workspace(workspace, fwd_b, dev)
    args = (M, T, V, i64_array(D), y.data_ptr(), ptr_array([t.data_ptr() for t in h]),
            ptr_array([t.data_ptr() for t in W]), float(alpha_d), _dtype_code(h[0]), losses.data_ptr(),
            stats.data_ptr(), workspace.data_ptr(), ws_bytes)
    opts = _lib.loss_options(exit_weights, distill, teacher_grad)
    if opts is None:
        code = lib().mls_multiexit_loss_fwd(*args, _ptr(status), _stream_ptr(stream))
    else:
        code = lib().mls_multiexit_loss_fwd_opts(*args, ctypes.byref(opts), _ptr(status), _stream_ptr(stream))
    check("mls_multiexit_loss_fwd", code)
    return losses, stats


def multiexit_loss_bwd(y: torch.Tensor, h: List[torch.Tensor], W: List[torch.Tensor], stats: torch.Tensor,
                       alpha_d: float = 0.3, grad_scale: float = 1.0, *, dh=None, dW=None,
                       accumulate_dW: bool = False, workspace=None, exit_weights=None, distill="ce",
                       teacher_grad: bool = False, status=None, stream=None):
    """Returns (dh list, dW list) (see mls_multiexit_loss_bwd)."""
    M, T, V, D, dt = _loss_common(y, h, W)
    dev = y.device
    _need(stats, "stats", torch.float32, 2)
    if dh is None:
        dh = [torch.empty_like(t) for t in h]
    if dW is None:
        dW = [torch.empty((V, d), dtype=torch.float32, device=dev) for d in D]
    _, bwd_b = multiexit_loss_workspace(T, D, V, dt)
    workspace, ws_bytes = _workspace(workspace, bwd_b, dev)
    args = (M, T, V, i64_array(D), y.data_ptr(), ptr_array([t.data_ptr() for t in h]),
            ptr_array([t.data_ptr() for t in W]), float(alpha_d), _dtype_code(h[0]), stats.data_ptr(),
            float(grad_scale), ptr_array([t.data_ptr() for t in dh]), ptr_array([t.data_ptr() for t in dW]),
            int(bool(accumulate_dW)), workspace.data_ptr(), ws_bytes)
    opts = _lib.loss_options(exit_weights, distill, teacher_grad)
    if opts is None:
        code = lib().mls_multiexit_loss_bwd(*args, _ptr(status), _stream_ptr(stream))
    else:
        code = lib().mls_multiexit_loss_bwd_opts(*args, ctypes.byref(opts), _ptr(status), _stream_ptr(stream))
    check("mls_multiexit_loss_bwd", code)
    return dh, dW


def exit_agreement(h: List[torch.Tensor], W: List[torch.Tensor], stats: torch.Tensor, *, per_token=False,
                   want_top1=False, workspace=None, status=None, stream=None):
    """Agreement of every smaller exit with the largest (see mls_exit_agreement).

    Returns (metrics [3(M-1)] = mean beta, mean KL, mean top-1 agreement per
    smaller exit, per-token rows [3(M-1), T] or None, top-1 ids [M, T] or None).
    """
    M = len(h)
    if len(W) != M or M < 2:
        raise ValueError("need at least two exits")
    T, V, dt = h[0].shape[0], W[0].shape[0], h[0].dtype
    D = []
    for m in range(M):
        _need(h[m], f"h[{m}]", dt, 2)
        _need(W[m], f"W[{m}]", dt, 2)
        D.append(h[m].shape[1])
    _need(stats, "stats", torch.float32, 2)
    dev = h[0].device
    metrics = torch.empty(3 * (M - 1), dtype=torch.float32, device=dev)
    rows = torch.empty((3 * (M - 1), T), dtype=torch.float32, device=dev) if per_token else None
    top1 = torch.empty((M, T), dtype=torch.int32, device=dev) if want_top1 else None
    n = ctypes.c_size_t()
    check("mls_exit_agreement_workspace",
          lib().mls_exit_agreement_workspace(M, T, i64_array(D), V, _dtype_code(h[0]), ctypes.byref(n)))
    workspace, ws_bytes = _workspace(workspace, n.value, dev)
    code = lib().mls_exit_agreement(M, T, V, i64_array(D), ptr_array([t.data_ptr() for t in h]),
                                    ptr_array([t.data_ptr() for t in W]), _dtype_code(h[0]), stats.data_ptr(),
                                    metrics.data_ptr(), _ptr(rows), _ptr(top1), workspace.data_ptr(), ws_bytes,
                                    _ptr(status), _stream_ptr(stream))
    check("mls_exit_agreement", code)
    return metrics, rows, top1


def status_read(status: torch.Tensor, stream=None) -> Tuple[int, int]:
    """Synchronises, returns (status code, raw flag word) and clears the word."""
    out = ctypes.c_int32()
    code = lib().mls_status_read(status.data_ptr(), _stream_ptr(stream), ctypes.byref(out))
    return code, out.value


def new_status(device="cuda") -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device)
