"""SOCKET oracle: plain fp64 CPU reference of the decode hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
CUDA library never calls it, and nothing in ``soft_lsh_top_b200`` imports it.

The arithmetic lives in ``socket_oracle.c`` (plain C, double precision, one
function per step of the method, each citing the page section it follows).
This module only compiles that file with gcc, loads it with ctypes and
marshals numpy / torch CPU arrays into it.

Every function here is pinned by ``tests/test_oracle_pins.py`` against closed
forms, invariants and brute force; see that file for what pins what.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "socket_oracle.c")
_LIB = os.path.join(_HERE, "libsocket_oracle.so")
_lock = threading.Lock()
_lib = None

F32, BF16, F64 = 0, 1, 2

_c_i64 = ctypes.c_int64
_c_int = ctypes.c_int
_c_dbl = ctypes.c_double
_vp = ctypes.c_void_p


def compile_oracle(src: str = _SRC, out: str = _LIB, extra_flags=()) -> str:
    """Compile the oracle C file into a shared library (plain -O2, no fast-math)."""
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-Wall", "-Wextra",
           *extra_flags, src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return out


def build(force: bool = False) -> str:
    """Build ``libsocket_oracle.so`` next to its source if missing or stale."""
    with _lock:
        stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
        if force or stale:
            tmp = _LIB + f".tmp{os.getpid()}"
            compile_oracle(_SRC, tmp)
            os.replace(tmp, _LIB)
    return _LIB


def _declare(lib):
    lib.oracle_set_num_threads.argtypes = [_c_int]
    lib.oracle_set_num_threads.restype = None
    lib.oracle_get_max_threads.argtypes = []
    lib.oracle_get_max_threads.restype = _c_int
    lib.oracle_hash.argtypes = [_vp, _vp, _c_int, _c_i64, _c_int, _vp, _c_int, _c_int, _vp, _vp, _vp]
    lib.oracle_hash.restype = None
    lib.oracle_soft_assign.argtypes = [_vp, _c_int, _c_int, _vp, _c_int, _c_int, _c_dbl, _vp]
    lib.oracle_soft_assign.restype = None
    lib.oracle_score.argtypes = [_vp, _vp, _c_i64, _c_int, _c_int, _vp, _c_int, _vp]
    lib.oracle_score.restype = None
    lib.oracle_topk.argtypes = [_vp, _c_i64, _c_int, _vp]
    lib.oracle_topk.restype = None
    lib.oracle_attention.argtypes = [_vp, _c_int, _c_int, _vp, _vp, _c_int, _c_int, _vp, _c_int, _vp]
    lib.oracle_attention.restype = None
    lib.oracle_decode_unit.argtypes = [_vp, _c_int, _c_int, _c_int, _vp, _c_int, _c_int, _c_dbl,
                                       _vp, _vp, _c_i64, _c_i64, _vp, _vp, _c_int, _c_int,
                                       _vp, _vp, _vp, _vp]
    lib.oracle_decode_unit.restype = None
    lib.oracle_decode.argtypes = [_vp, _c_int, _c_i64, _c_int, _c_int, _vp, _c_int, _c_int, _c_dbl,
                                  _vp, _vp, _c_i64, _c_i64, _vp, _vp, _c_int, _c_int,
                                  _vp, _vp, _vp]
    lib.oracle_decode.restype = None
    return lib


def load(path: str | None = None):
    """Load the oracle library (building it first if needed).

    ``path`` loads another build of the same source (the pin tests use this to
    load deliberately broken copies and check that the pins catch them).
    """
    global _lib
    if path is not None:
        return _declare(ctypes.CDLL(path))
    if _lib is None:
        build()
        _lib = _declare(ctypes.CDLL(_LIB))
    return _lib


def set_num_threads(n: int) -> None:
    load().oracle_set_num_threads(int(n))


def max_threads() -> int:
    return int(load().oracle_get_max_threads())


# ----------------------------------------------------------------------------
# marshalling helpers
# ----------------------------------------------------------------------------

def _stored(x):
    """Return (contiguous numpy array holding the stored bits, dtype code)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), BF16
            if x.dtype == torch.float32:
                return x.numpy(), F32
            if x.dtype == torch.float64:
                return x.numpy(), F64
            raise TypeError(f"unsupported tensor dtype {x.dtype}")
    except ImportError:  # pragma: no cover - torch is always present here
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.float64:
        return x, F64
    if x.dtype == np.uint16:  # raw bf16 bits
        return x, BF16
    raise TypeError(f"unsupported array dtype {x.dtype}")


def _f64(x) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return np.ascontiguousarray(x.detach().cpu().to(torch.float64).numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


# ----------------------------------------------------------------------------
# the steps of the method
# ----------------------------------------------------------------------------

def hash_keys(K, V, W, L: int, P: int, lib=None):
    """Step 1.  K, V: [n, d]; W: [L, P, d].  Returns (ids [L, n] uint8,
    vnorm [n] float64, margin [n] float64 = min |W_lp k| / ||k||)."""
    lib = lib or load()
    Ks, kdt = _stored(K)
    Vs, vdt = _stored(V)
    if kdt != vdt:
        raise TypeError("K and V must share a dtype")
    n, d = Ks.shape
    Wd = _f64(W).reshape(L, P, d)
    ids = np.zeros((L, n), dtype=np.uint8)
    vnorm = np.zeros(n, dtype=np.float64)
    margin = np.zeros(n, dtype=np.float64)
    lib.oracle_hash(_ptr(Ks), _ptr(Vs), kdt, n, d, _ptr(Wd), L, P, _ptr(ids), _ptr(vnorm), _ptr(margin))
    return ids, vnorm, margin


def soft_assign(q, W, L: int, P: int, tau: float, lib=None) -> np.ndarray:
    """Step 2 for one query head.  q: [d].  Returns p [L, 2^P] float64."""
    lib = lib or load()
    qs, qdt = _stored(q)
    d = qs.shape[-1]
    Wd = _f64(W).reshape(L, P, d)
    prob = np.zeros((L, 1 << P), dtype=np.float64)
    lib.oracle_soft_assign(_ptr(qs), qdt, d, _ptr(Wd), L, P, float(tau), _ptr(prob))
    return prob


def score(ids, vnorm_f32, prob, lib=None) -> np.ndarray:
    """Step 3.  ids: [L, n] uint8; vnorm_f32: [n] float32; prob: [G, L, 2^P]."""
    lib = lib or load()
    ids = np.ascontiguousarray(ids, dtype=np.uint8)
    vn = np.ascontiguousarray(vnorm_f32, dtype=np.float32)
    prob = np.ascontiguousarray(prob, dtype=np.float64)
    if prob.ndim == 2:
        prob = prob[None]
    G, L, nb = prob.shape
    P = int(nb).bit_length() - 1
    n = ids.shape[1]
    out = np.zeros(n, dtype=np.float64)
    lib.oracle_score(_ptr(ids), _ptr(vn), n, L, P, _ptr(prob), G, _ptr(out))
    return out


def topk(scores, k: int, lib=None) -> np.ndarray:
    """Step 4 selection.  Returns the k chosen indices, ascending, int32."""
    lib = lib or load()
    s = np.ascontiguousarray(scores, dtype=np.float64)
    idx = np.zeros(k, dtype=np.int32)
    lib.oracle_topk(_ptr(s), s.shape[0], int(k), _ptr(idx))
    return idx


def attention(q, K, V, idx, lib=None) -> np.ndarray:
    """Step 4 attention.  q: [G, d]; K, V: [n, d]; idx: [k].  Returns [G, d]."""
    lib = lib or load()
    qs, qdt = _stored(q)
    if qs.ndim == 1:
        qs = qs[None]
    Ks, kdt = _stored(K)
    Vs, vdt = _stored(V)
    G, d = qs.shape
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    out = np.zeros((G, d), dtype=np.float64)
    lib.oracle_attention(_ptr(qs), qdt, G, _ptr(Ks), _ptr(Vs), kdt, d, _ptr(idx), idx.shape[0], _ptr(out))
    return out


def decode_unit(q, W, L: int, P: int, tau: float, ids, vnorm_f32, K, V, n: int, k: int, lib=None):
    """Steps 2-4 for one (batch, kv-head) unit.

    q: [G, d]; ids: [L, ncap]; vnorm_f32: [ncap]; K, V: [ncap, d].
    Returns (idx [k] int32, out [G, d], scores [n], prob [G, L, 2^P]).
    """
    lib = lib or load()
    qs, qdt = _stored(q)
    Ks, kdt = _stored(K)
    Vs, _ = _stored(V)
    G, d = qs.shape
    ids = np.ascontiguousarray(ids, dtype=np.uint8)
    ncap = ids.shape[1]
    vn = np.ascontiguousarray(vnorm_f32, dtype=np.float32)
    Wd = _f64(W).reshape(L, P, d)
    idx = np.zeros(k, dtype=np.int32)
    out = np.zeros((G, d), dtype=np.float64)
    sc = np.zeros(n, dtype=np.float64)
    prob = np.zeros((G, L, 1 << P), dtype=np.float64)
    lib.oracle_decode_unit(_ptr(qs), qdt, G, d, _ptr(Wd), L, P, float(tau), _ptr(ids), _ptr(vn),
                           ncap, n, _ptr(Ks), _ptr(Vs), kdt, int(k), _ptr(idx), _ptr(out), _ptr(sc),
                           _ptr(prob))
    return idx, out, sc, prob


def decode(q, W, L: int, P: int, tau: float, ids, vnorm_f32, K, V, n: int, k: int,
           want_scores: bool = True, lib=None):
    """Steps 2-4 for U independent units, in parallel.

    q: [U, G, d]; ids: [U, L, ncap]; vnorm_f32: [U, ncap]; K, V: [U, ncap, d].
    Returns (idx [U, k], out [U, G, d], scores [U, n] or None).
    """
    lib = lib or load()
    qs, qdt = _stored(q)
    Ks, kdt = _stored(K)
    Vs, _ = _stored(V)
    U, G, d = qs.shape
    ids = np.ascontiguousarray(ids, dtype=np.uint8)
    ncap = ids.shape[2]
    vn = np.ascontiguousarray(vnorm_f32, dtype=np.float32)
    Wd = _f64(W).reshape(L, P, d)
    idx = np.zeros((U, k), dtype=np.int32)
    out = np.zeros((U, G, d), dtype=np.float64)
    sc = np.zeros((U, n), dtype=np.float64) if want_scores else None
    lib.oracle_decode(_ptr(qs), qdt, U, G, d, _ptr(Wd), L, P, float(tau), _ptr(ids), _ptr(vn),
                      ncap, n, _ptr(Ks), _ptr(Vs), kdt, int(k), _ptr(idx), _ptr(out),
                      _ptr(sc) if sc is not None else None)
    return idx, out, sc


def decode_per_head(q, W, L: int, P: int, tau: float, ids, vnorm_f32, K, V, n: int, k: int,
                    want_scores: bool = True, lib=None):
    """Steps 2-4 with one selection per query head: the method as the pages
    state it for a single query ([ES] "Mecanismo Central: LSH Suave" steps
    2-4 -- each new query induces its own bucket distribution, scores and
    top-k).  Head g of unit u is run as a unit of its own, with the one query
    row q[u, g] over u's ids, norms, keys and values; no arithmetic is added.

    q: [U, G, d]; ids: [U, L, ncap]; vnorm_f32: [U, ncap]; K, V: [U, ncap, d].
    Returns (idx [U, G, k], out [U, G, d], scores [U, G, n] or None).
    """
    qs, _ = _stored(q)
    Ks, _ = _stored(K)
    Vs, _ = _stored(V)
    U, G, d = qs.shape
    rep = lambda a: np.repeat(np.asarray(a), G, axis=0)  # unit u -> units u G .. u G + G - 1
    idx, out, sc = decode(qs.reshape(U * G, 1, d), W, L, P, tau, rep(ids), rep(vnorm_f32), rep(Ks), rep(Vs),
                          n, k, want_scores=want_scores, lib=lib)
    return idx.reshape(U, G, k), out.reshape(U, G, d), (sc.reshape(U, G, n) if sc is not None else None)
