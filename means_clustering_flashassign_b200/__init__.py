"""Exact Lloyd K-Means on B200 (sm_100a): FlashAssign + Sort-Inverse Update.

Thin Python binding of ``libkm.so`` (C ABI in ``include/km.h``).  This module
only marshals arguments: it checks shapes, allocates outputs and workspace with
torch (device memory and streams are the only things torch provides) and calls
the C entry points, which run every step of the computation in CUDA kernels.
There is no CPU or PyTorch fallback: if the library is missing or the GPU is
not an sm_100 part, calls raise.

Method: "Flash-KMeans: Fast and Memory-Efficient Exact K-Means", §2.1
FlashAssign (fused distance tiles + online argmin, no N x K matrix in device
memory), §2.2 Sort-Inverse Update (argsort of the assignment vector +
segmented on-chip reduction), §2.3 Chunked Stream Overlap (host-resident points
streamed in chunks).
"""

from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

from . import build as _build

__all__ = ["KMError", "library", "library_path", "workspace_size", "assign", "update", "fit", "fit_host",
           "workspace_status", "selftest_timeout", "argsort", "fit_profile", "launch_count", "assign_static",
           "ablation_assign_materialized", "ablation_update_atomic", "plan", "update_accumulate",
           "finalize_sums", "fit_data_parallel", "pack_layout", "exchange_packed", "fit_source", "FitGraph",
           "OP_ASSIGN", "OP_UPDATE", "OP_FIT", "OP_FIT_HOST",
           "OP_ARGSORT",
           "F32", "BF16", "EXPORTS"]

OP_ASSIGN, OP_UPDATE, OP_FIT, OP_FIT_HOST, OP_ARGSORT = 0, 1, 2, 3, 4
F32, BF16 = 0, 1
STATUS = {0: "KM_OK", 1: "KM_ERR_INVALID_ARG", 2: "KM_ERR_UNSUPPORTED", 3: "KM_ERR_CUDA",
          4: "KM_ERR_WORKSPACE", 5: "KM_ERR_TIMEOUT", 6: "KM_ERR_INJECTED"}
EXPORTS = ["km_version", "km_status_string", "km_last_error", "km_workspace_size", "km_workspace_status",
           "km_assign", "km_update", "km_argsort", "km_fit", "km_fit_profile", "km_fit_timed", "km_fit_host", "km_selftest_timeout",
           "km_launch_count", "km_assign_static", "km_ablation_workspace_size", "km_ablation_assign_materialized",
           "km_ablation_update_atomic", "km_plan_describe", "km_update_accumulate", "km_finalize_sums",
           "km_fit_source", "km_fit_graph_create", "km_fit_graph_launch", "km_fit_graph_elapsed",
           "km_fit_graph_destroy"]

_lock = threading.Lock()
_lib = None

# km_chunk_source: const void* (*)(void* user, int64_t row0, int64_t rows, int slot)
CHUNK_SOURCE = ctypes.CFUNCTYPE(ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int)


class KMError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status
        self.message = message


def library_path() -> str:
    return _build.LIB


def library() -> ctypes.CDLL:
    """Load libkm.so (building it first if the sources are newer)."""
    global _lib
    with _lock:
        if _lib is None:
            path = _build.LIB
            if not _build.up_to_date():
                path = _build.build()
            if not os.path.exists(path):
                raise RuntimeError(f"libkm.so not found at {path}; run means_clustering_flashassign_b200.build")
            L = ctypes.CDLL(path)
            P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
            L.km_version.restype = I
            L.km_status_string.argtypes = [I]
            L.km_status_string.restype = ctypes.c_char_p
            L.km_last_error.restype = ctypes.c_char_p
            L.km_workspace_size.argtypes = [I, I, I64, I, I, I, I64]
            L.km_workspace_size.restype = SZ
            L.km_workspace_status.argtypes = [P, P]
            L.km_assign.argtypes = [P, P, I, I64, I, I, I, P, P, P, P, SZ, P]
            L.km_update.argtypes = [P, P, I, I64, I, I, I, P, P, P, SZ, P]
            L.km_fit.argtypes = [P, P, I, I64, I, I, I, I, P, P, P, P, P, SZ, P]
            L.km_fit_host.argtypes = [P, P, I64, I, I, I, I, I64, P, P, P, P, P, SZ, P]
            L.km_selftest_timeout.argtypes = [P, SZ, I64, P]
            L.km_argsort.argtypes = [P, I64, I, P, P, P, SZ, P]
            L.km_plan_describe.argtypes = [I, I, I64, I, I, I, I64, P]
            L.km_update_accumulate.argtypes = [P, P, I64, I, I, I, P, P, I, P, SZ, P]
            L.km_finalize_sums.argtypes = [P, P, I, I, I, P, P, P, P]
            L.km_ablation_workspace_size.argtypes = [I, I64, I, I, I, I64]
            L.km_ablation_workspace_size.restype = SZ
            L.km_ablation_assign_materialized.argtypes = [P, P, I64, I, I, I, I64, P, P, P, SZ, P]
            L.km_ablation_update_atomic.argtypes = [P, P, I64, I, I, I, P, P, P, SZ, P]
            L.km_fit_profile.argtypes = [P, P, I, I64, I, I, I, I, P, P, P, P, P, SZ, P, P]
            L.km_fit_timed.argtypes = [P, P, I, I64, I, I, I, I, P, P, P, P, P, SZ, P, P]
            L.km_launch_count.restype = ctypes.c_uint64
            L.km_assign_static.argtypes = [P, P, I, I64, I, I, I, P, P, P, P]
            L.km_fit_source.argtypes = [CHUNK_SOURCE, P, P, I64, I, I, I, I, I64, P, P, P, P, P, SZ, P]
            L.km_fit_graph_create.argtypes = [P, P, P, I, I64, I, I, I, I, P, P, P, P, P, SZ, I]
            L.km_fit_graph_launch.argtypes = [P, P]
            L.km_fit_graph_elapsed.argtypes = [P, P]
            L.km_fit_graph_destroy.argtypes = [P]
            for f in EXPORTS:
                getattr(L, f).restype = getattr(L, f).restype or I
            _lib = L
    return _lib


def _check(status: int) -> None:
    if status != 0:
        msg = library().km_last_error().decode(errors="replace")
        raise KMError(status, msg)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"points must be bfloat16 or float32, got {t.dtype}")


def _shape3(X: torch.Tensor, name: str):
    if X.dim() == 2:
        return 1, X.shape[0], X.shape[1], False
    if X.dim() == 3:
        return X.shape[0], X.shape[1], X.shape[2], True
    raise ValueError(f"{name} must be (N, D) or (B, N, D)")


def workspace_size(op: int, B: int, N: int, D: int, K: int, dtype: int, chunk_rows: int = 0) -> int:
    n = library().km_workspace_size(op, B, N, D, K, dtype, chunk_rows)
    if n == 0:
        raise KMError(2, library().km_last_error().decode(errors="replace"))
    return int(n)


def _workspace(op, B, N, D, K, dtype, device, workspace=None, chunk_rows=0):
    need = workspace_size(op, B, N, D, K, dtype, chunk_rows)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    if workspace.numel() < need:
        raise ValueError(f"workspace has {workspace.numel()} bytes, needs {need}")
    return workspace


def _contig_cuda(t: torch.Tensor, name: str) -> torch.Tensor:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _check_tensor(t: torch.Tensor, name: str, device: torch.device, dtype=None, shape=None) -> torch.Tensor:
    """Reject a tensor the kernels would read or write out of place: on
    another device than the points, of another dtype or shape than the call
    writes, or not contiguous (the kernels index it as a dense array)."""
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, the points are on {device}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _check_stream(stream, device: torch.device) -> None:
    if stream is not None and stream.device != device:
        raise ValueError(f"the stream is on {stream.device}, the points are on {device}")


def assign(X: torch.Tensor, C: torch.Tensor, *, idx=None, mindist=None, want_mindist: bool = True,
           want_objective: bool = True, workspace=None, stream=None):
    """FlashAssign: nearest centroid of every point (lowest index on ties).

    X: (N, D) or (B, N, D) bf16/f32 CUDA tensor; C: (K, D) or (B, K, D), same dtype.
    Returns (idx int32, mindist float32 or None, objective float64 [B] or None).
    """
    B, N, D, K, dt, shp = _assign_args(X, C, idx, mindist, stream)
    with torch.cuda.device(X.device):
        idx = torch.empty(shp, dtype=torch.int32, device=X.device) if idx is None else idx
        if mindist is None and want_mindist:
            mindist = torch.empty(shp, dtype=torch.float32, device=X.device)
        obj = torch.empty(B, dtype=torch.float64, device=X.device) if want_objective else None
        ws = _workspace(OP_ASSIGN, B, N, D, K, dt, X.device, workspace)
        _check_tensor(ws, "workspace", X.device, torch.uint8)
        _check(library().km_assign(_ptr(X), _ptr(C), B, N, D, K, dt, _ptr(idx), _ptr(mindist), _ptr(obj),
                                   _ptr(ws), ws.numel(), _stream(stream)))
    return idx, mindist, obj


def _assign_args(X, C, idx, mindist, stream):
    """Shapes of an assignment call, with every tensor checked against X."""
    _contig_cuda(X, "X"), _contig_cuda(C, "C")
    B, N, D, batched = _shape3(X, "X")
    Bc, K, Dc, _ = _shape3(C, "C")
    if Bc != B or Dc != D or C.dtype != X.dtype:
        raise ValueError("C must match X in batch, D and dtype")
    dt = _dtype_code(X)
    shp = (B, N) if batched else (N,)
    _check_tensor(C, "C", X.device)
    if idx is not None:
        _check_tensor(idx, "idx", X.device, torch.int32, shp)
    if mindist is not None:
        _check_tensor(mindist, "mindist", X.device, torch.float32, shp)
    _check_stream(stream, X.device)
    return B, N, D, K, dt, shp


def assign_static(X: torch.Tensor, C: torch.Tensor, *, idx=None, mindist=None, want_mindist: bool = True,
                  want_objective: bool = True, stream=None):
    """assign() without a workspace: scratch comes from the library's fixed
    16 MiB static device area (for callers that cannot allocate; shapes that
    need more are refused).  Same results as assign()."""
    B, N, D, K, dt, shp = _assign_args(X, C, idx, mindist, stream)
    with torch.cuda.device(X.device):
        idx = torch.empty(shp, dtype=torch.int32, device=X.device) if idx is None else idx
        if mindist is None and want_mindist:
            mindist = torch.empty(shp, dtype=torch.float32, device=X.device)
        obj = torch.empty(B, dtype=torch.float64, device=X.device) if want_objective else None
        _check(library().km_assign_static(_ptr(X), _ptr(C), B, N, D, K, dt, _ptr(idx), _ptr(mindist), _ptr(obj),
                                          _stream(stream)))
    return idx, mindist, obj


def update(X: torch.Tensor, idx: torch.Tensor, C: torch.Tensor, *, counts=None, want_counts: bool = True,
           workspace=None, stream=None):
    """Sort-Inverse Update: C (float32, in: previous, out: new) <- member means.

    Returns (C, counts int32 or None).  C is updated in place.
    """
    _contig_cuda(X, "X"), _contig_cuda(idx, "idx"), _contig_cuda(C, "C")
    B, N, D, batched = _shape3(X, "X")
    Bc, K, Dc, _ = _shape3(C, "C")
    if Bc != B or Dc != D or C.dtype != torch.float32 or idx.dtype != torch.int32:
        raise ValueError("C must be float32 (B, K, D) matching X; idx int32")
    dt = _dtype_code(X)
    _check_tensor(idx, "idx", X.device, torch.int32, (B, N) if batched else (N,))
    _check_tensor(C, "C", X.device)
    kshape = (B, K) if batched else (K,)
    if counts is not None:
        _check_tensor(counts, "counts", X.device, torch.int32, kshape)
    _check_stream(stream, X.device)
    with torch.cuda.device(X.device):
        if counts is None and want_counts:
            counts = torch.empty(kshape, dtype=torch.int32, device=X.device)
        ws = _workspace(OP_UPDATE, B, N, D, K, dt, X.device, workspace)
        _check_tensor(ws, "workspace", X.device, torch.uint8)
        _check(library().km_update(_ptr(X), _ptr(idx), B, N, D, K, dt, _ptr(C), _ptr(counts), _ptr(ws),
                                   ws.numel(), _stream(stream)))
    return C, counts


def argsort(idx: torch.Tensor, K: int, *, workspace=None, stream=None):
    """Stable argsort of an assignment vector by cluster id on the device.

    Returns (perm int32 [N], start int32 [K+1]).
    """
    _contig_cuda(idx, "idx")
    if idx.dtype != torch.int32 or idx.dim() != 1:
        raise ValueError("idx must be a 1-D int32 tensor")
    N = idx.shape[0]
    _check_stream(stream, idx.device)
    with torch.cuda.device(idx.device):
        perm = torch.empty(N, dtype=torch.int32, device=idx.device)
        start = torch.empty(K + 1, dtype=torch.int32, device=idx.device)
        ws = _workspace(OP_ARGSORT, 1, N, 0, K, 0, idx.device, workspace)
        _check_tensor(ws, "workspace", idx.device, torch.uint8)
        _check(library().km_argsort(_ptr(idx), N, K, _ptr(perm), _ptr(start), _ptr(ws), ws.numel(),
                                    _stream(stream)))
    return perm, start


def update_accumulate(X: torch.Tensor, idx: torch.Tensor, sums: torch.Tensor, counts: torch.Tensor, *,
                      zero_first: bool = True, workspace=None, stream=None) -> None:
    """Sort-Inverse Update of one shard added into float64 sums [K, D] and
    float64 counts [K] (zeroed first by default).  sums and counts may be
    views into one buffer (see pack_layout)."""
    _contig_cuda(X, "X"), _contig_cuda(idx, "idx"), _contig_cuda(sums, "sums"), _contig_cuda(counts, "counts")
    if X.dim() != 2 or sums.dim() != 2:
        raise ValueError("X must be [N, D] and sums [K, D]")
    N, D = X.shape
    K = sums.shape[0]
    _check_tensor(idx, "idx", X.device, torch.int32, (N,))
    _check_tensor(sums, "sums", X.device, torch.float64, (K, D))
    _check_tensor(counts, "counts", X.device, torch.float64, (K,))
    _check_stream(stream, X.device)
    dt = _dtype_code(X)
    with torch.cuda.device(X.device):
        ws = _workspace(OP_UPDATE, 1, N, D, K, dt, X.device, workspace)
        _check_tensor(ws, "workspace", X.device, torch.uint8)
        _check(library().km_update_accumulate(_ptr(X), _ptr(idx), N, D, K, dt, _ptr(sums), _ptr(counts),
                                              1 if zero_first else 0, _ptr(ws), ws.numel(), _stream(stream)))


def finalize_sums(sums: torch.Tensor, counts: torch.Tensor, C: torch.Tensor, C_lp: Optional[torch.Tensor] = None,
                  counts_out: Optional[torch.Tensor] = None, *, stream=None) -> None:
    """C = sums / counts where counts > 0 (else kept), in place; C_lp gets the
    dtype copy for the next assign; counts_out the int32 counts.  sums
    float64 [K, D], counts float64 [K], C float32 [K, D]."""
    _contig_cuda(C, "C")
    if C.dim() != 2:
        raise ValueError("C must be [K, D]")
    K, D = C.shape
    dev = C.device
    _check_tensor(C, "C", dev, torch.float32)
    _check_tensor(sums, "sums", dev, torch.float64, (K, D))
    _check_tensor(counts, "counts", dev, torch.float64, (K,))
    if C_lp is not None:
        _check_tensor(C_lp, "C_lp", dev, shape=(K, D))
    if counts_out is not None:
        _check_tensor(counts_out, "counts_out", dev, torch.int32, (K,))
    _check_stream(stream, dev)
    dt = _dtype_code(C_lp) if C_lp is not None else F32
    with torch.cuda.device(dev):
        _check(library().km_finalize_sums(_ptr(sums), _ptr(counts), K, D, dt, _ptr(C), _ptr(C_lp),
                                          _ptr(counts_out), _stream(stream)))


def pack_layout(K: int, D: int) -> dict:
    """Layout of the one float64 buffer a data-parallel iteration exchanges:
    the per-cluster sums [K*D], the counts [K] (exact integers in float64)
    and the objective [1], in that order, so that one all-reduce (sum) adds
    all three across the ranks.  Returns slices into a flat buffer."""
    kd = K * D
    return {"sums": slice(0, kd), "counts": slice(kd, kd + K), "objective": slice(kd + K, kd + K + 1),
            "size": kd + K + 1}


def exchange_packed(buf: torch.Tensor, *, group=None) -> None:
    """Add a packed buffer (pack_layout) across the ranks of `group` in
    place: one all-reduce.  NCCL reduces device tensors directly; a gloo
    group goes through a host copy."""
    import torch.distributed as dist
    if buf.dtype != torch.float64 or buf.dim() != 1 or not buf.is_contiguous():
        raise ValueError("the exchange buffer must be a contiguous 1-D float64 tensor")
    if buf.is_cuda and dist.get_backend(group) == "gloo":
        h = buf.cpu()
        dist.all_reduce(h, group=group)
        buf.copy_(h)
    else:
        dist.all_reduce(buf, group=group)


def fit_data_parallel(X: torch.Tensor, C0: torch.Tensor, iters: int, *, group=None, sync_objective: bool = True):
    """Lloyd iterations over a point set sharded by rows across the ranks of a
    torch.distributed process group: every rank passes its own rows X and the
    same C0.  Per iteration each rank assigns its rows and sums them per
    cluster (float64, deterministic) into one packed buffer (sums, counts,
    objective); one all-reduce adds the ranks' buffers; every rank finalises
    the same sums, so C is the same on all ranks.  The objective history stays
    on the device until the end (no host synchronisation per iteration).
    Returns dict(C float32 [K, D], idx (this rank's rows), counts int32 [K],
    objective float64 [iters]: the whole point set's J_t, on the host when
    sync_objective, else on the device)."""
    _contig_cuda(X, "X"), _contig_cuda(C0, "C0")
    if X.dim() != 2 or C0.dim() != 2 or C0.shape[1] != X.shape[1] or C0.dtype != X.dtype:
        raise ValueError("X [N, D] and C0 [K, D] of one dtype")
    _check_tensor(C0, "C0", X.device)
    N, D = X.shape
    K = C0.shape[0]
    dev = X.device
    lay = pack_layout(K, D)
    with torch.cuda.device(dev):
        C = C0.float().contiguous().clone()
        C_lp = C0.clone()
        buf = torch.empty(lay["size"], dtype=torch.float64, device=dev)
        sums = buf[lay["sums"]].view(K, D)
        cnt = buf[lay["counts"]]
        obj = buf[lay["objective"]]
        counts = torch.empty(K, dtype=torch.int32, device=dev)
        idx = torch.empty(N, dtype=torch.int32, device=dev)
        dt = _dtype_code(X)
        ws_a = _workspace(OP_ASSIGN, 1, N, D, K, dt, dev)
        ws_u = _workspace(OP_UPDATE, 1, N, D, K, dt, dev)
        J = torch.empty(iters, dtype=torch.float64, device=dev)
        L = library()
        s = _stream(None)
        for t in range(iters):
            _check(L.km_assign(_ptr(X), _ptr(C_lp), 1, N, D, K, dt, _ptr(idx), None, _ptr(obj), _ptr(ws_a),
                               ws_a.numel(), s))
            _check(L.km_update_accumulate(_ptr(X), _ptr(idx), N, D, K, dt, _ptr(sums), _ptr(cnt), 1, _ptr(ws_u),
                                          ws_u.numel(), s))
            exchange_packed(buf, group=group)
            _check(L.km_finalize_sums(_ptr(sums), _ptr(cnt), K, D, dt, _ptr(C), _ptr(C_lp), _ptr(counts), s))
            J[t:t + 1].copy_(obj)
    return dict(C=C, idx=idx, counts=counts, objective=J.cpu() if sync_objective else J)


def plan(op: int, B: int, N: int, D: int, K: int, dtype: int, chunk_rows: int = 0) -> dict:
    """The tiling the library would use for this shape (host-only query)."""
    out = (ctypes.c_int64 * 9)()
    _check(library().km_plan_describe(op, B, N, D, K, dtype, chunk_rows, ctypes.cast(out, ctypes.c_void_p)))
    keys = ("pair", "BN", "XB", "CS", "smem", "Kp", "sort_passes", "sort_block", "update_form")
    return {k: int(v) for k, v in zip(keys, out)}


def ablation_assign_materialized(X: torch.Tensor, C: torch.Tensor, *, chunk_rows: Optional[int] = None,
                                 mindist: bool = True, stream=None):
    """Baseline (not the method): the N x K distance matrix through device
    memory -- a library GEMM writes the scores, an argmin kernel reads them.
    One instance.  Returns (idx int32 [N], mindist float32 [N] or None)."""
    _contig_cuda(X, "X"), _contig_cuda(C, "C")
    if X.dim() != 2 or C.dim() != 2 or C.shape[1] != X.shape[1] or C.dtype != X.dtype:
        raise ValueError("X [N, D] and C [K, D] of one dtype")
    N, D = X.shape
    K = C.shape[0]
    dt = _dtype_code(X)
    _check_tensor(C, "C", X.device)
    _check_stream(stream, X.device)
    cr = N if chunk_rows is None else int(chunk_rows)
    with torch.cuda.device(X.device):
        idx = torch.empty(N, dtype=torch.int32, device=X.device)
        md = torch.empty(N, dtype=torch.float32, device=X.device) if mindist else None
        wsb = int(library().km_ablation_workspace_size(0, N, D, K, dt, cr))
        ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device=X.device)
        _check(library().km_ablation_assign_materialized(_ptr(X), _ptr(C), N, D, K, dt, cr, _ptr(idx), _ptr(md),
                                                         _ptr(ws), ws.numel(), _stream(stream)))
    return idx, md


def ablation_update_atomic(X: torch.Tensor, idx: torch.Tensor, C: torch.Tensor, *, stream=None):
    """Baseline (not the method): every point added to its cluster's sum with
    float atomics, then C = sum / count (empty clusters keep C).  C float32
    [K, D] is updated in place.  Returns counts int32 [K]."""
    _contig_cuda(X, "X"), _contig_cuda(idx, "idx"), _contig_cuda(C, "C")
    if X.dim() != 2 or C.dim() != 2 or C.shape[1] != X.shape[1] or C.dtype != torch.float32:
        raise ValueError("X [N, D] and float32 C [K, D]")
    if idx.dtype != torch.int32 or idx.shape != (X.shape[0],):
        raise ValueError("idx must be int32 [N]")
    N, D = X.shape
    K = C.shape[0]
    dt = _dtype_code(X)
    _check_tensor(idx, "idx", X.device, torch.int32, (N,))
    _check_tensor(C, "C", X.device, torch.float32)
    _check_stream(stream, X.device)
    with torch.cuda.device(X.device):
        counts = torch.empty(K, dtype=torch.int32, device=X.device)
        wsb = int(library().km_ablation_workspace_size(1, N, D, K, dt, 0))
        ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device=X.device)
        _check(library().km_ablation_update_atomic(_ptr(X), _ptr(idx), N, D, K, dt, _ptr(C), _ptr(counts),
                                                   _ptr(ws), ws.numel(), _stream(stream)))
    return counts


def _fit_outputs(X, C0, iters, C_out, idx_out, counts_out, objective, want_idx, stream):
    """Checked shapes and outputs of a fit call (allocated on X's device)."""
    _contig_cuda(X, "X"), _contig_cuda(C0, "C0")
    B, N, D, batched = _shape3(X, "X")
    Bc, K, Dc, _ = _shape3(C0, "C0")
    if Bc != B or Dc != D or C0.dtype != X.dtype:
        raise ValueError("C0 must match X in batch, D and dtype")
    if iters < 0:
        raise ValueError("iters must be >= 0")
    dev = X.device
    _check_tensor(C0, "C0", dev)
    _check_stream(stream, dev)
    cshape, ishape, kshape = ((B, K, D), (B, N), (B, K)) if batched else ((K, D), (N,), (K,))
    oshape = (B, iters) if batched else (iters,)
    if C_out is None:
        C_out = torch.empty(cshape, dtype=torch.float32, device=dev)
    _check_tensor(C_out, "C_out", dev, torch.float32, cshape)
    if idx_out is None and want_idx:
        idx_out = torch.empty(ishape, dtype=torch.int32, device=dev)
    if idx_out is not None:
        _check_tensor(idx_out, "idx_out", dev, torch.int32, ishape)
    if counts_out is None:
        counts_out = torch.empty(kshape, dtype=torch.int32, device=dev)
    _check_tensor(counts_out, "counts_out", dev, torch.int32, kshape)
    if objective is None:
        objective = torch.empty(oshape, dtype=torch.float64, device=dev)
    _check_tensor(objective, "objective", dev, torch.float64, oshape)
    return B, N, D, K, _dtype_code(X), C_out, idx_out, counts_out, objective


def fit(X: torch.Tensor, C0: torch.Tensor, iters: int, *, C_out=None, idx_out=None, counts_out=None,
        objective=None, want_idx: bool = True, workspace=None, stream=None):
    """`iters` exact Lloyd iterations from C0 on the device.

    Returns dict(C float32, idx int32 or None, counts int32, objective float64 [B, iters] or [iters]).
    """
    _contig_cuda(X, "X")
    with torch.cuda.device(X.device):
        B, N, D, K, dt, C_out, idx_out, counts_out, objective = _fit_outputs(
            X, C0, iters, C_out, idx_out, counts_out, objective, want_idx, stream)
        ws = _workspace(OP_FIT, B, N, D, K, dt, X.device, workspace)
        _check_tensor(ws, "workspace", X.device, torch.uint8)
        _check(library().km_fit(_ptr(X), _ptr(C0), B, N, D, K, dt, iters, _ptr(C_out), _ptr(idx_out),
                                _ptr(counts_out), _ptr(objective), _ptr(ws), ws.numel(), _stream(stream)))
    return dict(C=C_out, idx=idx_out, counts=counts_out, objective=objective)


def fit_profile(X: torch.Tensor, C0: torch.Tensor, iters: int, *, C_out=None, idx_out=None, counts_out=None,
                objective=None, workspace=None, stream=None):
    """fit() with CUDA-event timing of each iteration's assignment and update.

    Synchronous.  Returns the fit() dict plus "phase_ms": float32 [iters, 2]
    (assignment kernel ms, update ms) and "iters_ms": device time of the
    iterations (first assignment start to last update end).
    """
    _contig_cuda(X, "X")
    with torch.cuda.device(X.device):
        B, N, D, K, dt, C_out, idx_out, counts_out, objective = _fit_outputs(
            X, C0, iters, C_out, idx_out, counts_out, objective, False, stream)
        phase = torch.zeros(2 * iters + 1, dtype=torch.float32)
        ws = _workspace(OP_FIT, B, N, D, K, dt, X.device, workspace)
        _check_tensor(ws, "workspace", X.device, torch.uint8)
        _check(library().km_fit_profile(_ptr(X), _ptr(C0), B, N, D, K, dt, iters, _ptr(C_out), _ptr(idx_out),
                                        _ptr(counts_out), _ptr(objective), _ptr(ws), ws.numel(), _stream(stream),
                                        _ptr(phase)))
    return dict(C=C_out, idx=idx_out, counts=counts_out, objective=objective,
                phase_ms=phase[:2 * iters].reshape(iters, 2), iters_ms=float(phase[2 * iters]))


def fit_timed(X: torch.Tensor, C0: torch.Tensor, iters: int, *, C_out=None, idx_out=None, counts_out=None,
              objective=None, workspace=None, stream=None):
    """fit() with the device time of its iterations, events around the loop only.

    Synchronous.  Returns the fit() dict plus "iters_ms": device time from
    the first assignment's start to the last update's end.  Unlike
    fit_profile, no event sits between the kernels, so they chain as in fit().
    """
    _contig_cuda(X, "X")
    with torch.cuda.device(X.device):
        B, N, D, K, dt, C_out, idx_out, counts_out, objective = _fit_outputs(
            X, C0, iters, C_out, idx_out, counts_out, objective, False, stream)
        ms = ctypes.c_float(0.0)
        ws = _workspace(OP_FIT, B, N, D, K, dt, X.device, workspace)
        _check_tensor(ws, "workspace", X.device, torch.uint8)
        _check(library().km_fit_timed(_ptr(X), _ptr(C0), B, N, D, K, dt, iters, _ptr(C_out), _ptr(idx_out),
                                      _ptr(counts_out), _ptr(objective), _ptr(ws), ws.numel(), _stream(stream),
                                      ctypes.byref(ms)))
    return dict(C=C_out, idx=idx_out, counts=counts_out, objective=objective, iters_ms=float(ms.value))


class FitGraph:
    """fit() captured once as a CUDA graph (km_fit_graph_create); every
    launch() enqueues one complete fit from C0 into the same output tensors.

    The graph holds pointers: this object keeps X, C0, the outputs and the
    workspace alive, and the caller may refill X / C0 in place between
    launches.  With timed=True, iters_ms() gives the device time of the last
    launch's iterations.  close() (or garbage collection) releases it.
    """

    def __init__(self, X: torch.Tensor, C0: torch.Tensor, iters: int, *, C_out=None, idx_out=None,
                 counts_out=None, objective=None, want_idx: bool = True, workspace=None, timed: bool = False):
        self._h = None
        _contig_cuda(X, "X")
        with torch.cuda.device(X.device):
            B, N, D, K, dt, C_out, idx_out, counts_out, objective = _fit_outputs(
                X, C0, iters, C_out, idx_out, counts_out, objective, want_idx, None)
            ws = _workspace(OP_FIT, B, N, D, K, dt, X.device, workspace)
            _check_tensor(ws, "workspace", X.device, torch.uint8)
            h = ctypes.c_void_p()
            _check(library().km_fit_graph_create(ctypes.byref(h), _ptr(X), _ptr(C0), B, N, D, K, dt, iters,
                                                 _ptr(C_out), _ptr(idx_out), _ptr(counts_out), _ptr(objective),
                                                 _ptr(ws), ws.numel(), 1 if timed else 0))
        self._h = h
        self.device = X.device
        self.X, self.C0, self.workspace = X, C0, ws
        self.result = dict(C=C_out, idx=idx_out, counts=counts_out, objective=objective)

    def launch(self, stream=None) -> dict:
        """Enqueue one fit (asynchronous); returns the output tensors."""
        if self._h is None:
            raise RuntimeError("the graph was closed")
        _check_stream(stream, self.device)
        with torch.cuda.device(self.device):
            _check(library().km_fit_graph_launch(self._h, _stream(stream)))
        return self.result

    def iters_ms(self) -> float:
        """Waits for the last launch; milliseconds of its iterations."""
        ms = ctypes.c_float(0.0)
        _check(library().km_fit_graph_elapsed(self._h, ctypes.byref(ms)))
        return float(ms.value)

    def close(self) -> None:
        if self._h is not None:
            torch.cuda.synchronize(self.device)
            library().km_fit_graph_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def launch_count() -> int:
    """Kernels this library has enqueued in this process so far."""
    return int(library().km_launch_count())


def fit_host(X_host: torch.Tensor, C0: torch.Tensor, iters: int, chunk_rows: int, *, C_out=None, idx_out=None,
             want_idx: bool = False, counts_out=None, workspace=None, stream=None):
    """Out-of-core Lloyd: X_host is a pinned CPU tensor (N, D), streamed per iteration in chunks.

    Synchronous.  Returns dict(C, idx or None, counts, objective (CPU float64 [iters])).
    """
    if X_host.is_cuda or not X_host.is_pinned():
        raise ValueError("X_host must be a pinned CPU tensor")
    if not X_host.is_contiguous():
        raise ValueError("X_host must be contiguous")
    _contig_cuda(C0, "C0")
    if X_host.dim() != 2 or C0.dim() != 2 or C0.shape[1] != X_host.shape[1] or C0.dtype != X_host.dtype:
        raise ValueError("X_host [N, D] and C0 [K, D] of one dtype")
    N, D = X_host.shape
    K = C0.shape[0]
    dt = _dtype_code(X_host)
    dev = C0.device
    _check_stream(stream, dev)
    with torch.cuda.device(dev):
        C_out = torch.empty((K, D), dtype=torch.float32, device=dev) if C_out is None else C_out
        _check_tensor(C_out, "C_out", dev, torch.float32, (K, D))
        if idx_out is None and want_idx:
            idx_out = torch.empty(N, dtype=torch.int32, device=dev)
        if idx_out is not None:
            _check_tensor(idx_out, "idx_out", dev, torch.int32, (N,))
        counts_out = torch.empty(K, dtype=torch.int32, device=dev) if counts_out is None else counts_out
        _check_tensor(counts_out, "counts_out", dev, torch.int32, (K,))
        obj = torch.empty(iters, dtype=torch.float64)
        ws = _workspace(OP_FIT_HOST, 1, N, D, K, dt, dev, workspace, chunk_rows)
        _check_tensor(ws, "workspace", dev, torch.uint8)
        _check(library().km_fit_host(_ptr(X_host), _ptr(C0), N, D, K, dt, iters, chunk_rows, _ptr(C_out),
                                     _ptr(idx_out), _ptr(counts_out), _ptr(obj), _ptr(ws), ws.numel(),
                                     _stream(stream)))
    return dict(C=C_out, idx=idx_out, counts=counts_out, objective=obj)


def fit_source(source, N: int, C0: torch.Tensor, iters: int, chunk_rows: int, *, dtype=torch.bfloat16,
               C_out=None, idx_out=None, want_idx: bool = False, counts_out=None, workspace=None, stream=None):
    """Out-of-core Lloyd over a point set that is never held whole: every
    iteration, source(row0, rows, slot) returns a pinned CPU tensor holding
    rows [row0, row0 + rows) (shape (rows, D), the given dtype).  The tensor
    returned for a slot (0 or 1) is kept alive and unchanged until that slot
    is asked for again.  Same results as fit_host on the concatenated rows.

    Synchronous.  Returns dict(C, idx or None, counts, objective (CPU float64 [iters])).
    """
    _contig_cuda(C0, "C0")
    if C0.dim() != 2 or C0.dtype != dtype:
        raise ValueError("C0 must be [K, D] of the points' dtype")
    K, D = C0.shape
    dt = _dtype_code(C0)
    dev = C0.device
    _check_stream(stream, dev)
    held = [None, None]      # the tensors behind the two slots
    errors = []
    es = C0.element_size()

    def trampoline(_user, row0, rows, slot):
        try:
            t = source(int(row0), int(rows), int(slot))
            if (t.is_cuda or not t.is_pinned() or not t.is_contiguous() or t.dtype != dtype
                    or tuple(t.shape) != (rows, D)):
                raise ValueError(f"the source must return a pinned contiguous {dtype} tensor of shape ({rows}, {D})")
            held[slot] = t
            return t.data_ptr()
        except BaseException as e:  # the library sees NULL and stops
            errors.append(e)
            return None

    cb = CHUNK_SOURCE(trampoline)
    with torch.cuda.device(dev):
        C_out = torch.empty((K, D), dtype=torch.float32, device=dev) if C_out is None else C_out
        _check_tensor(C_out, "C_out", dev, torch.float32, (K, D))
        if idx_out is None and want_idx:
            idx_out = torch.empty(N, dtype=torch.int32, device=dev)
        if idx_out is not None:
            _check_tensor(idx_out, "idx_out", dev, torch.int32, (N,))
        counts_out = torch.empty(K, dtype=torch.int32, device=dev) if counts_out is None else counts_out
        _check_tensor(counts_out, "counts_out", dev, torch.int32, (K,))
        obj = torch.empty(iters, dtype=torch.float64)
        ws = _workspace(OP_FIT_HOST, 1, N, D, K, dt, dev, workspace, chunk_rows)
        _check_tensor(ws, "workspace", dev, torch.uint8)
        st = library().km_fit_source(cb, None, _ptr(C0), N, D, K, dt, iters, chunk_rows, _ptr(C_out),
                                     _ptr(idx_out), _ptr(counts_out), _ptr(obj), _ptr(ws), ws.numel(),
                                     _stream(stream))
    if errors:
        raise errors[0]
    _check(st)
    del es
    return dict(C=C_out, idx=idx_out, counts=counts_out, objective=obj)


def workspace_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise and read/clear the workspace status word (0 or KM_ERR_TIMEOUT)."""
    return int(library().km_workspace_status(_ptr(workspace), _stream(stream)))


def selftest_timeout(limit_ns: int = 1_000_000, device="cuda") -> int:
    """Run the bounded-wait self-test kernel; returns the status it reports."""
    ws = torch.zeros(256, dtype=torch.uint8, device=device)
    return int(library().km_selftest_timeout(_ptr(ws), ws.numel(), int(limit_ns), _stream(None)))
