"""CPU oracle for exact Lloyd K-Means (float64, plain C + OpenMP).

TEST INFRASTRUCTURE ONLY: imported by the tests, ``__graft_entry__.smoke()`` and
the bench's CPU-baseline leg, never by the library.  It shares no code with the
CUDA path.  The arithmetic lives in ``km_oracle.c``; this module only compiles
it with gcc (``-O2``, no fast-math) and marshals numpy arrays.

Every function follows "Flash-KMeans: Fast and Memory-Efficient Exact K-Means",
§2 (Methodology: unchanged Lloyd mathematics, no approximation):
  assign   -- argmin of squared Euclidean distance, lowest index on ties;
  update   -- per-cluster mean, empty clusters keep their centroid;
  argsort  -- stable ordering of point indices by cluster id (§2.2's inverse map);
  fit      -- T assign/update rounds, objective recorded under the centroids used;
  objective_assigned_bf16 -- the objective of a given assignment of bfloat16 points.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "km_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_SO = os.path.join(_BUILD, "libkmoracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile km_oracle.c into a shared library (gcc, OpenMP)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def compile_source(src_text: str, out_path: str) -> str:
    """Compile C source text with the oracle's flags (used for planted-mistake tests)."""
    c_path = out_path + ".c"
    with open(c_path, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                           "-fno-fast-math", "-o", out_path, c_path, "-lm"])
    return out_path


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


def _configure(L):
    P = ctypes.c_void_p
    i64, i32 = ctypes.c_int64, ctypes.c_int
    L.kmo_assign.argtypes = [P, P, i64, i32, i32, P, P, P]
    L.kmo_update.argtypes = [P, P, i64, i32, i32, P, P]
    L.kmo_objective.argtypes = [P, i64]
    L.kmo_objective.restype = ctypes.c_double
    L.kmo_objective_assigned_bf16.argtypes = [P, P, P, i64, i32]
    L.kmo_objective_assigned_bf16.restype = ctypes.c_double
    L.kmo_round_bf16.argtypes = [P, P, i64]
    L.kmo_round_f32.argtypes = [P, P, i64]
    L.kmo_round_bf16_one.argtypes = [ctypes.c_double]
    L.kmo_round_bf16_one.restype = ctypes.c_double
    L.kmo_argsort.argtypes = [P, i64, i32, P, P]
    L.kmo_fit.argtypes = [P, i64, i32, i32, i32, i32, P, P, P, P]
    L.kmo_num_threads.restype = ctypes.c_int
    L.kmo_set_num_threads.argtypes = [ctypes.c_int]
    return L


def load_library(path: str):
    """Load a compiled copy of km_oracle.c (the tests load planted-mistake
    variants this way to show that the pins catch them)."""
    return _configure(ctypes.CDLL(path))


def swap_library(L):
    """Make the module functions use library L; returns the previous one."""
    global _lib
    with _lock:
        old, _lib = _lib, L
    return old


def lib():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _configure(ctypes.CDLL(build()))
    return _lib


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # torch tensor: exact widening to float64 on the CPU
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _i32(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").numpy()
    return np.ascontiguousarray(a, dtype=np.int32)


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return lib().kmo_num_threads()


def set_num_threads(n: int) -> None:
    lib().kmo_set_num_threads(int(n))


def assign(X, C):
    """Return (idx int32[N], d1 float64[N], d2 float64[N]) -- exact argmin,
    best and second-best squared distances (d2 = inf when K == 1)."""
    X, C = _f64(X), _f64(C)
    N, D = X.shape
    K = C.shape[0]
    assert C.shape[1] == D
    idx = np.empty(N, np.int32)
    d1 = np.empty(N, np.float64)
    d2 = np.empty(N, np.float64)
    lib().kmo_assign(_p(X), _p(C), N, D, K, _p(idx), _p(d1), _p(d2))
    return idx, d1, d2


def update(X, idx, C_prev):
    """Return (C_new float64[K,D], counts int64[K]); empty clusters keep C_prev."""
    X, idx = _f64(X), _i32(idx)
    C = _f64(C_prev).copy()
    N, D = X.shape
    K = C.shape[0]
    counts = np.empty(K, np.int64)
    lib().kmo_update(_p(X), _p(idx), N, D, K, _p(C), _p(counts))
    return C, counts


def objective(d1) -> float:
    d1 = _f64(d1)
    return float(lib().kmo_objective(_p(d1), d1.shape[0]))


def objective_assigned_bf16(X, C, idx) -> float:
    """sum_i ||x_i - c_{idx[i]}||^2 in float64 (direct form) for bfloat16
    points X (a torch bfloat16 tensor on the CPU, or its raw uint16 bits as a
    numpy array), float64-widened centroids C and an assignment idx."""
    if hasattr(X, "detach"):
        import torch
        X = X.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)
    Xb = np.ascontiguousarray(X, dtype=np.uint16)
    Cd, ii = _f64(C), _i32(idx)
    N, D = Xb.shape
    assert Cd.shape[1] == D and ii.shape[0] == N
    return float(lib().kmo_objective_assigned_bf16(_p(Xb), _p(Cd), _p(ii), N, D))


def round_bf16(a) -> np.ndarray:
    a = _f64(a)
    out = np.empty_like(a)
    lib().kmo_round_bf16(_p(a), _p(out), a.size)
    return out


def round_f32(a) -> np.ndarray:
    a = _f64(a)
    out = np.empty_like(a)
    lib().kmo_round_f32(_p(a), _p(out), a.size)
    return out


def argsort(idx, K: int):
    """Stable argsort by cluster id: (perm int32[N], start int64[K+1])."""
    idx = _i32(idx)
    perm = np.empty(idx.shape[0], np.int32)
    start = np.empty(K + 1, np.int64)
    lib().kmo_argsort(_p(idx), idx.shape[0], K, _p(perm), _p(start))
    return perm, start


MIRROR = {"exact": 0, "bf16": 1, "f32": 2}


def fit(X, C0, iters: int, mirror: str = "exact"):
    """T Lloyd iterations.  Returns dict(C, idx, counts, J)."""
    X, C = _f64(X), _f64(C0).copy()
    N, D = X.shape
    K = C.shape[0]
    idx = np.empty(N, np.int32)
    counts = np.empty(K, np.int64)
    J = np.empty(iters, np.float64)
    lib().kmo_fit(_p(X), N, D, K, iters, MIRROR[mirror], _p(C), _p(idx), _p(counts), _p(J))
    return dict(C=C, idx=idx, counts=counts, J=J)
