"""SOCKET decode hot path on B200: Python binding of ``libsocket_attn.so``.

The functions here only marshal arguments into the C ABI declared in
``include/socket_attn.h`` (same names): they check that torch tensors have the
shapes, dtypes, devices and layouts the C side assumes, pass raw pointers and
sizes, and turn a non-zero status into ``SocketError``.  Every step of the
method runs in the library's CUDA kernels; there is no Python or CPU
implementation to fall back on, and importing a call fails loudly when the
library has not been built (``python -m soft_lsh_top_b200._build``).

PyTorch provides device memory and streams only.  Calls are asynchronous on
the current torch stream unless ``stream`` (a ``torch.cuda.Stream``) is given.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "SocketError", "socket_hash_keys", "socket_decode", "socket_decode_static", "socket_decode_workspace_size",
    "socket_decode_per_head", "socket_decode_per_head_workspace_size", "socket_hash_check", "socket_decode_append",
    "socket_last_error", "socket_version", "socket_ids_row_bytes", "ids_shape", "socket_set_step_events",
    "socket_set_wait_limit", "socket_set_selection_path", "socket_last_decode_path", "socket_shard_select", "socket_shard_merge", "socket_shard_attend",
    "socket_shard_attend_workspace_size", "socket_shard_combine", "library_path", "load_library",
    "alloc_cache_index", "alloc_decode_buffers",
]

SOCKET_OK, SOCKET_EINVAL, SOCKET_EUNSUPPORTED, SOCKET_ECUDA, SOCKET_EWORKSPACE = range(5)
SOCKET_F32, SOCKET_BF16 = 0, 1
HEAD_DIM = 128
WS_ERROR_OFFSET = 0

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libsocket_attn.so")
_lib = None

_i64, _int, _dbl, _vp, _sz = ctypes.c_int64, ctypes.c_int, ctypes.c_double, ctypes.c_void_p, ctypes.c_size_t

_STATUS = {1: "EINVAL", 2: "EUNSUPPORTED", 3: "ECUDA", 4: "EWORKSPACE"}


class SocketError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"SOCKET_{_STATUS.get(status, status)}: {message}")
        self.status = status


def library_path() -> str:
    return _LIB_PATH


def load_library(path: str | None = None):
    """Load the CUDA library (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or _LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"SOCKET CUDA library missing at {p}; build it with "
                           "`python -m soft_lsh_top_b200._build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(p)
    lib.socket_hash_keys.argtypes = [_vp, _vp, _int, _i64, _i64, _i64, _i64, _i64, _i64, _vp, _int, _int, _vp, _vp, _vp]
    lib.socket_hash_keys.restype = _int
    lib.socket_hash_check.argtypes = [_vp]
    lib.socket_hash_check.restype = _int
    lib.socket_decode_workspace_size.argtypes = [_i64, _i64, _i64, _i64, _i64, _int, _int, _int]
    lib.socket_decode_workspace_size.restype = _sz
    lib.socket_decode.argtypes = [_vp, _int, _vp, _vp, _vp, _vp, _vp, _int, _i64, _i64, _i64, _i64, _i64, _i64,
                                  _int, _int, _dbl, _int, _vp, _sz, _vp, _vp, _vp, _vp]
    lib.socket_decode.restype = _int
    lib.socket_decode_per_head_workspace_size.argtypes = [_i64, _i64, _i64, _i64, _i64, _int, _int, _int]
    lib.socket_decode_per_head_workspace_size.restype = _sz
    lib.socket_decode_per_head.argtypes = lib.socket_decode.argtypes
    lib.socket_decode_append.argtypes = [_vp, _int, _vp, _vp, _vp, _vp, _vp, _int, _i64, _i64, _i64, _i64, _i64,
                                         _i64, _int, _int, _dbl, _int, _i64, _vp, _sz, _vp, _vp, _vp, _vp]
    lib.socket_decode_append.restype = _int
    lib.socket_decode_per_head.restype = _int
    lib.socket_decode_static.argtypes = [_vp, _int, _vp, _vp, _vp, _vp, _vp, _int, _i64, _i64, _i64, _i64, _i64,
                                         _i64, _int, _int, _dbl, _int, _vp, _vp, _vp, _vp]
    lib.socket_decode_static.restype = _int
    lib.socket_last_error.argtypes = []
    lib.socket_last_error.restype = ctypes.c_char_p
    lib.socket_set_step_events.argtypes = [ctypes.POINTER(ctypes.c_void_p), _int]
    lib.socket_set_step_events.restype = _int
    lib.socket_shard_select.argtypes = [_vp, _int, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _i64, _int, _int,
                                        _dbl, _int, _i64, _vp, _sz, _vp, _vp, _vp]
    lib.socket_shard_select.restype = _int
    lib.socket_shard_merge.argtypes = [_vp, _vp, _int, _i64, _i64, _int, _i64, _i64, _vp, _vp, _vp, _vp]
    lib.socket_shard_merge.restype = _int
    lib.socket_shard_attend_workspace_size.argtypes = [_i64, _i64, _i64, _i64, _i64, _int]
    lib.socket_shard_attend_workspace_size.restype = _sz
    lib.socket_shard_attend.argtypes = [_vp, _int, _vp, _vp, _int, _i64, _i64, _i64, _i64, _i64, _int, _vp, _vp,
                                        _vp, _sz, _vp, _vp, _vp]
    lib.socket_shard_attend.restype = _int
    lib.socket_shard_combine.argtypes = [_vp, _vp, _int, _i64, _i64, _i64, _vp, _vp]
    lib.socket_shard_combine.restype = _int
    lib.socket_set_wait_limit.argtypes = [ctypes.c_uint32]
    lib.socket_set_wait_limit.restype = ctypes.c_uint32
    lib.socket_set_selection_path.argtypes = [_int]
    lib.socket_set_selection_path.restype = _int
    lib.socket_last_decode_path.argtypes = []
    lib.socket_last_decode_path.restype = _int
    lib.socket_ids_row_bytes.argtypes = [_int]
    lib.socket_ids_row_bytes.restype = _int
    lib.socket_version.argtypes = []
    lib.socket_version.restype = _int
    if path is None:
        _lib = lib
    return lib


def socket_last_error() -> str:
    return load_library().socket_last_error().decode()


def socket_version() -> int:
    return int(load_library().socket_version())


# ----------------------------------------------------------------------------
# marshalling helpers
# ----------------------------------------------------------------------------

def _code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SOCKET_BF16
    if t.dtype == torch.float32:
        return SOCKET_F32
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def _check(t: torch.Tensor, name: str, shape, dtype=None, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def _stream_handle(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _raise(status: int):
    if status != SOCKET_OK:
        raise SocketError(status, socket_last_error())


# ----------------------------------------------------------------------------
# the C ABI
# ----------------------------------------------------------------------------

def socket_hash_keys(K: torch.Tensor, V: torch.Tensor, W: torch.Tensor, ids: torch.Tensor,
                     vnorm: torch.Tensor, n_begin: int = 0, n_end: int | None = None, stream=None) -> None:
    """Hash keys [n_begin, n_end) of every unit into ``ids`` and ``vnorm``.

    K, V: [B, Hkv, Ncap, 128] (float32 or bfloat16); W: [L, P, 128] bfloat16;
    ids: [B, Hkv, Ncap/32, Lr/16, 32, 16] uint8, Lr = socket_ids_row_bytes(L) (see the header); vnorm: [B, Hkv, Ncap] float32.
    """
    lib = load_library()
    B, Hkv, Ncap, d = K.shape
    L, P, _ = W.shape
    dev = K.device
    _check(K, "K", (B, Hkv, Ncap, d), device=dev)
    _check(V, "V", (B, Hkv, Ncap, d), dtype=K.dtype, device=dev)
    _check(W, "W", (L, P, d), dtype=torch.bfloat16, device=dev)
    _check(ids, "ids", ids_shape(B, Hkv, Ncap, L), dtype=torch.uint8, device=dev)
    _check(vnorm, "vnorm", (B, Hkv, Ncap), dtype=torch.float32, device=dev)
    n_end = Ncap if n_end is None else int(n_end)
    with torch.cuda.device(dev):
        _raise(lib.socket_hash_keys(K.data_ptr(), V.data_ptr(), _code(K), B, Hkv, Ncap, int(n_begin), n_end, d,
                                    W.data_ptr(), L, P, ids.data_ptr(), vnorm.data_ptr(), _stream_handle(stream)))


def socket_hash_check(stream=None) -> None:
    """Wait for the stream; raise SocketError if a hashing kernel gave up on a
    bounded wait since the last check (the record is then cleared)."""
    _raise(load_library().socket_hash_check(_stream_handle(stream)))


def socket_ids_row_bytes(L: int) -> int:
    """Bytes of one key's id row for L tables (32 per started block of 32)."""
    n = int(load_library().socket_ids_row_bytes(int(L)))
    if n == 0:
        raise SocketError(1, f"L={L} outside 1..128")
    return n


def ids_shape(B: int, Hkv: int, Ncap: int, L: int) -> tuple:
    """Shape of the bucket-id array: [B, Hkv, Ncap/32, Lr/16, 32, 16]."""
    return (B, Hkv, Ncap // 32, socket_ids_row_bytes(L) // 16, 32, 16)


def socket_decode_workspace_size(B: int, Hq: int, Hkv: int, Ncap: int, d: int, L: int, P: int, k: int) -> int:
    n = int(load_library().socket_decode_workspace_size(B, Hq, Hkv, Ncap, d, L, P, k))
    if n == 0:
        raise ValueError("invalid sizes for socket_decode")
    return n


def socket_decode_per_head_workspace_size(B: int, Hq: int, Hkv: int, Ncap: int, d: int, L: int, P: int,
                                          k: int) -> int:
    n = int(load_library().socket_decode_per_head_workspace_size(B, Hq, Hkv, Ncap, d, L, P, k))
    if n == 0:
        raise ValueError("invalid sizes for socket_decode_per_head")
    return n


def _decode(per_head: bool, q, W, ids, vnorm, K, V, N, tau, k, workspace, idx_out, out, scores_out, stream,
            n_new: int = 0):
    lib = load_library()
    B, Hq, d = q.shape
    _, Hkv, Ncap, _ = K.shape
    L, P, _ = W.shape
    dev = q.device
    sel = Hq if per_head else Hkv  # selections per batch row
    _check(q, "q", (B, Hq, d), device=dev)
    _check(W, "W", (L, P, d), dtype=torch.bfloat16, device=dev)
    _check(ids, "ids", ids_shape(B, Hkv, Ncap, L), dtype=torch.uint8, device=dev)
    _check(vnorm, "vnorm", (B, Hkv, Ncap), dtype=torch.float32, device=dev)
    _check(K, "K", (B, Hkv, Ncap, d), device=dev)
    _check(V, "V", (B, Hkv, Ncap, d), dtype=K.dtype, device=dev)
    _check(idx_out, "idx_out", (B, sel, k), dtype=torch.int32, device=dev)
    _check(out, "out", (B, Hq, d), dtype=torch.float32, device=dev)
    if workspace.dtype != torch.uint8 or workspace.dim() != 1 or not workspace.is_cuda or workspace.device != dev:
        raise ValueError("workspace must be a 1-D uint8 CUDA tensor on the inputs' device")
    if scores_out is not None:
        _check(scores_out, "scores_out", (B, sel, Ncap), dtype=torch.float32, device=dev)
    head = (q.data_ptr(), _code(q), W.data_ptr(), ids.data_ptr(), vnorm.data_ptr(), K.data_ptr(), V.data_ptr(),
            _code(K), B, Hq, Hkv, Ncap, int(N), d, L, P, float(tau), int(k))
    tail = (workspace.data_ptr(), workspace.numel(), idx_out.data_ptr(), out.data_ptr(),
            scores_out.data_ptr() if scores_out is not None else None, _stream_handle(stream))
    with torch.cuda.device(dev):
        if n_new:
            _raise(lib.socket_decode_append(*head, int(n_new), *tail))
        elif per_head:
            _raise(lib.socket_decode_per_head(*head, *tail))
        else:
            _raise(lib.socket_decode(*head, *tail))


def socket_decode(q: torch.Tensor, W: torch.Tensor, ids: torch.Tensor, vnorm: torch.Tensor,
                  K: torch.Tensor, V: torch.Tensor, N: int, tau: float, k: int,
                  workspace: torch.Tensor, idx_out: torch.Tensor, out: torch.Tensor,
                  scores_out: torch.Tensor | None = None, stream=None) -> None:
    """One decode step (soft assignment, scoring, top-k, sparse attention),
    one selection per kv head.

    q: [B, Hq, 128]; W: [L, P, 128] bfloat16; ids: [B, Hkv, Ncap/32, Lr/16, 32, 16] uint8, Lr = socket_ids_row_bytes(L) (see the header);
    vnorm: [B, Hkv, Ncap] float32; K, V: [B, Hkv, Ncap, 128];
    workspace: uint8 tensor of >= socket_decode_workspace_size() bytes;
    idx_out: [B, Hkv, k] int32; out: [B, Hq, 128] float32;
    scores_out: optional [B, Hkv, Ncap] float32.
    """
    _decode(False, q, W, ids, vnorm, K, V, N, tau, k, workspace, idx_out, out, scores_out, stream)


def socket_decode_append(q: torch.Tensor, W: torch.Tensor, ids: torch.Tensor, vnorm: torch.Tensor,
                         K: torch.Tensor, V: torch.Tensor, N: int, tau: float, k: int, n_new: int,
                         workspace: torch.Tensor, idx_out: torch.Tensor, out: torch.Tensor,
                         scores_out: torch.Tensor | None = None, stream=None) -> None:
    """socket_decode after appending keys N - n_new .. N - 1 to K and V: the
    step also hashes those keys (writing their ids and vnorm).  Shapes as
    socket_decode; 1 <= n_new <= 64."""
    if int(n_new) < 1:
        raise ValueError("n_new must be >= 1")
    _decode(False, q, W, ids, vnorm, K, V, N, tau, k, workspace, idx_out, out, scores_out, stream, n_new=int(n_new))


def socket_decode_per_head(q: torch.Tensor, W: torch.Tensor, ids: torch.Tensor, vnorm: torch.Tensor,
                           K: torch.Tensor, V: torch.Tensor, N: int, tau: float, k: int,
                           workspace: torch.Tensor, idx_out: torch.Tensor, out: torch.Tensor,
                           scores_out: torch.Tensor | None = None, stream=None) -> None:
    """socket_decode with one selection per query head: idx_out [B, Hq, k],
    scores_out optional [B, Hq, Ncap], workspace of
    >= socket_decode_per_head_workspace_size() bytes; the rest as socket_decode."""
    _decode(True, q, W, ids, vnorm, K, V, N, tau, k, workspace, idx_out, out, scores_out, stream)


def socket_decode_static(q: torch.Tensor, W: torch.Tensor, ids: torch.Tensor, vnorm: torch.Tensor,
                         K: torch.Tensor, V: torch.Tensor, N: int, tau: float, k: int,
                         idx_out: torch.Tensor, out: torch.Tensor, scores_out: torch.Tensor | None = None,
                         stream=None) -> None:
    """socket_decode without a caller workspace, for callers that cannot
    allocate device memory: the library's own fixed 64 MiB device scratch is
    used instead (see include/socket_attn.h).  Calls that overlap on the GPU
    share that scratch and must be serialised by the caller."""
    lib = load_library()
    B, Hq, d = q.shape
    _, Hkv, Ncap, _ = K.shape
    L, P, _ = W.shape
    dev = q.device
    _check(q, "q", (B, Hq, d), device=dev)
    _check(W, "W", (L, P, d), dtype=torch.bfloat16, device=dev)
    _check(ids, "ids", ids_shape(B, Hkv, Ncap, L), dtype=torch.uint8, device=dev)
    _check(vnorm, "vnorm", (B, Hkv, Ncap), dtype=torch.float32, device=dev)
    _check(K, "K", (B, Hkv, Ncap, d), device=dev)
    _check(V, "V", (B, Hkv, Ncap, d), dtype=K.dtype, device=dev)
    _check(idx_out, "idx_out", (B, Hkv, k), dtype=torch.int32, device=dev)
    _check(out, "out", (B, Hq, d), dtype=torch.float32, device=dev)
    if scores_out is not None:
        _check(scores_out, "scores_out", (B, Hkv, Ncap), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        _raise(lib.socket_decode_static(q.data_ptr(), _code(q), W.data_ptr(), ids.data_ptr(), vnorm.data_ptr(),
                                        K.data_ptr(), V.data_ptr(), _code(K), B, Hq, Hkv, Ncap, int(N), d, L, P,
                                        float(tau), int(k), idx_out.data_ptr(), out.data_ptr(),
                                        scores_out.data_ptr() if scores_out is not None else None,
                                        _stream_handle(stream)))


def socket_set_step_events(events) -> None:
    """Register torch.cuda.Event objects (created with enable_timing=True) that
    every later socket_decode on this thread records around its kernels;
    an empty list turns the recording off."""
    lib = load_library()
    n = len(events)
    arr = (ctypes.c_void_p * max(n, 1))(*[ctypes.c_void_p(int(e.cuda_event)) for e in events])
    _raise(lib.socket_set_step_events(arr, n))


def _check_workspace(workspace: torch.Tensor, dev):
    if workspace.dtype != torch.uint8 or workspace.dim() != 1 or not workspace.is_cuda or workspace.device != dev:
        raise ValueError("workspace must be a 1-D uint8 CUDA tensor on the inputs' device")


def socket_shard_select(q: torch.Tensor, W: torch.Tensor, ids: torch.Tensor, vnorm: torch.Tensor, N: int,
                        tau: float, k: int, n_offset: int, workspace: torch.Tensor, cand_score: torch.Tensor,
                        cand_index: torch.Tensor, stream=None) -> None:
    """This shard's own top-k as (score, global index) pairs (see the header).

    q: [B, Hq, 128]; W: [L, P, 128] bfloat16; ids, vnorm: this shard's cache
    index ([B, Hkv, ...] as for socket_decode, N keys); workspace of
    >= socket_decode_workspace_size(..., min(k, N)) bytes; cand_score: [B, Hkv, k]
    float32; cand_index: [B, Hkv, k] int32."""
    lib = load_library()
    B, Hq, d = q.shape
    L, P, _ = W.shape
    Hkv, Ncap = vnorm.shape[1], vnorm.shape[2]
    dev = q.device
    _check(q, "q", (B, Hq, d), device=dev)
    _check(W, "W", (L, P, d), dtype=torch.bfloat16, device=dev)
    _check(ids, "ids", ids_shape(B, Hkv, Ncap, L), dtype=torch.uint8, device=dev)
    _check(vnorm, "vnorm", (B, Hkv, Ncap), dtype=torch.float32, device=dev)
    _check(cand_score, "cand_score", (B, Hkv, k), dtype=torch.float32, device=dev)
    _check(cand_index, "cand_index", (B, Hkv, k), dtype=torch.int32, device=dev)
    _check_workspace(workspace, dev)
    with torch.cuda.device(dev):
        _raise(lib.socket_shard_select(q.data_ptr(), _code(q), W.data_ptr(), ids.data_ptr(), vnorm.data_ptr(), B, Hq,
                                       Hkv, Ncap, int(N), d, L, P, float(tau), int(k), int(n_offset),
                                       workspace.data_ptr(), workspace.numel(), cand_score.data_ptr(),
                                       cand_index.data_ptr(), _stream_handle(stream)))


def socket_shard_merge(cand_score: torch.Tensor, cand_index: torch.Tensor, n_offset: int, n_local: int,
                       idx_out: torch.Tensor, local_idx: torch.Tensor, local_count: torch.Tensor,
                       stream=None) -> None:
    """The global top-k from all shards' pairs, cand_score / cand_index
    [S, B, Hkv, k] in shard order: idx_out [B, Hkv, k] int32 (global),
    local_idx [B, Hkv, k] int32 and local_count [B, Hkv] int32 (this shard's
    keys [n_offset, n_offset + n_local) among them, as local indices)."""
    lib = load_library()
    S, B, Hkv, k = cand_score.shape
    dev = cand_score.device
    _check(cand_score, "cand_score", (S, B, Hkv, k), dtype=torch.float32, device=dev)
    _check(cand_index, "cand_index", (S, B, Hkv, k), dtype=torch.int32, device=dev)
    _check(idx_out, "idx_out", (B, Hkv, k), dtype=torch.int32, device=dev)
    _check(local_idx, "local_idx", (B, Hkv, k), dtype=torch.int32, device=dev)
    _check(local_count, "local_count", (B, Hkv), dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        _raise(lib.socket_shard_merge(cand_score.data_ptr(), cand_index.data_ptr(), S, B, Hkv, k, int(n_offset),
                                      int(n_local), idx_out.data_ptr(), local_idx.data_ptr(), local_count.data_ptr(),
                                      _stream_handle(stream)))


def socket_shard_attend_workspace_size(B: int, Hq: int, Hkv: int, Ncap: int, k: int) -> int:
    n = int(load_library().socket_shard_attend_workspace_size(B, Hq, Hkv, Ncap, HEAD_DIM, k))
    if n == 0:
        raise ValueError("invalid sizes for socket_shard_attend")
    return n


def socket_shard_attend(q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, k: int, local_idx: torch.Tensor,
                        local_count: torch.Tensor, workspace: torch.Tensor, out: torch.Tensor, ml: torch.Tensor,
                        stream=None) -> None:
    """Attention over this shard's share of the selection: out [B, Hq, 128]
    float32 (normalised over those keys) and ml [B, Hq, 2] float32 (largest
    logit, sum of weights)."""
    lib = load_library()
    B, Hq, d = q.shape
    _, Hkv, Ncap, _ = K.shape
    dev = q.device
    _check(q, "q", (B, Hq, d), device=dev)
    _check(K, "K", (B, Hkv, Ncap, d), device=dev)
    _check(V, "V", (B, Hkv, Ncap, d), dtype=K.dtype, device=dev)
    _check(local_idx, "local_idx", (B, Hkv, k), dtype=torch.int32, device=dev)
    _check(local_count, "local_count", (B, Hkv), dtype=torch.int32, device=dev)
    _check(out, "out", (B, Hq, d), dtype=torch.float32, device=dev)
    _check(ml, "ml", (B, Hq, 2), dtype=torch.float32, device=dev)
    _check_workspace(workspace, dev)
    with torch.cuda.device(dev):
        _raise(lib.socket_shard_attend(q.data_ptr(), _code(q), K.data_ptr(), V.data_ptr(), _code(K), B, Hq, Hkv, Ncap,
                                       d, int(k), local_idx.data_ptr(), local_count.data_ptr(), workspace.data_ptr(),
                                       workspace.numel(), out.data_ptr(), ml.data_ptr(), _stream_handle(stream)))


def socket_shard_combine(outs: torch.Tensor, mls: torch.Tensor, out: torch.Tensor, stream=None) -> None:
    """Log-sum-exp merge of the shards' partial results outs [S, B, Hq, 128]
    and mls [S, B, Hq, 2] into out [B, Hq, 128] float32."""
    lib = load_library()
    S, B, Hq, d = outs.shape
    dev = outs.device
    _check(outs, "outs", (S, B, Hq, d), dtype=torch.float32, device=dev)
    _check(mls, "mls", (S, B, Hq, 2), dtype=torch.float32, device=dev)
    _check(out, "out", (B, Hq, d), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        _raise(lib.socket_shard_combine(outs.data_ptr(), mls.data_ptr(), S, B, Hq, d, out.data_ptr(),
                                        _stream_handle(stream)))


def socket_set_wait_limit(polls: int) -> int:
    """Polls before a decode kernel's wait for requested data gives up (0: at
    once, for tests of the failure path; 0xffffffff: the default).  Returns
    the previous limit."""
    return int(load_library().socket_set_wait_limit(polls & 0xffffffff))


SOCKET_PATH_AUTO, SOCKET_PATH_SEPARATE = 0, 1


def socket_set_selection_path(path: int) -> int:
    """Kernels for selection and attention in later decode calls:
    SOCKET_PATH_AUTO (by shape) or SOCKET_PATH_SEPARATE (always top-k, then
    attention).  Returns the previous path; raises on another value."""
    prev = int(load_library().socket_set_selection_path(int(path)))
    if prev < 0:
        raise SocketError(SOCKET_EINVAL, f"unknown selection path {path}")
    return prev


SOCKET_STEP_SEPARATE, SOCKET_STEP_FUSED, SOCKET_STEP_ONE_KERNEL = 0, 1, 2


def socket_last_decode_path() -> int:
    """Kernels of this thread's last decode call: SOCKET_STEP_SEPARATE (soft
    tables, scoring, top-k, attention), SOCKET_STEP_FUSED (soft tables,
    scoring, fused selection + attention) or SOCKET_STEP_ONE_KERNEL; -1 if
    there was none, or it failed before launching."""
    return int(load_library().socket_last_decode_path())


# ----------------------------------------------------------------------------
# allocation helpers (torch owns the memory)
# ----------------------------------------------------------------------------

def alloc_cache_index(B: int, Hkv: int, Ncap: int, L: int, device) -> tuple[torch.Tensor, torch.Tensor]:
    """Bucket-id and value-norm buffers for a cache of Ncap keys per unit."""
    ids = torch.empty(ids_shape(B, Hkv, Ncap, L), dtype=torch.uint8, device=device)
    vnorm = torch.empty(B, Hkv, Ncap, dtype=torch.float32, device=device)
    return ids, vnorm


def alloc_decode_buffers(B: int, Hq: int, Hkv: int, Ncap: int, L: int, P: int, k: int, device,
                         per_head: bool = False):
    """(workspace, idx_out, out) for socket_decode (per_head: socket_decode_per_head) at these sizes."""
    size = socket_decode_per_head_workspace_size if per_head else socket_decode_workspace_size
    ws = torch.empty(size(B, Hq, Hkv, Ncap, HEAD_DIM, L, P, k), dtype=torch.uint8, device=device)
    idx = torch.empty(B, Hq if per_head else Hkv, k, dtype=torch.int32, device=device)
    out = torch.empty(B, Hq, HEAD_DIM, dtype=torch.float32, device=device)
    return ws, idx, out


def read_device_error(workspace: torch.Tensor) -> int:
    """The device error word of a decode workspace (synchronises the stream)."""
    return int(workspace[WS_ERROR_OFFSET:WS_ERROR_OFFSET + 4].view(torch.int32).item())
