"""The C ABI library loads, exports what include/*.h declares, and rejects bad
arguments on the host before any launch (CPU only: no call here reaches a
kernel launch)."""
import ctypes
import glob
import os
import re

import numpy as np

import pytest

from soft_lsh_top_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

OK, EINVAL, EUNSUP, ECUDA, EWS = 0, 1, 2, 3, 4


@pytest.fixture(scope="module")
def lib():
    path = _build.build()
    import soft_lsh_top_b200 as s
    return s.load_library(path)


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(socket_\w+)\s*\(", text, flags=re.M))
    return sorted(names)


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ("socket_hash_keys", "socket_hash_check", "socket_decode", "socket_decode_workspace_size",
                 "socket_decode_per_head", "socket_decode_per_head_workspace_size", "socket_decode_append",
                 "socket_shard_select", "socket_shard_merge", "socket_shard_attend",
                 "socket_shard_attend_workspace_size", "socket_shard_combine", "socket_last_error"):
        assert want in names


def test_every_declared_symbol_is_exported(lib):
    raw = ctypes.CDLL(_build.LIB)
    for name in declared_functions():
        assert hasattr(raw, name), name


def test_version(lib):
    assert lib.socket_version() == 200


def test_wait_limit_diagnostic_round_trips(lib):
    """socket_set_wait_limit returns the previous limit; 0xffffffff restores
    the default (host state only, nothing launched)."""
    default = lib.socket_set_wait_limit(7)
    assert default == 1 << 22
    assert lib.socket_set_wait_limit(0xFFFFFFFF) == 7
    assert lib.socket_set_wait_limit(0xFFFFFFFF) == default


def test_selection_path_diagnostic_round_trips(lib):
    """socket_set_selection_path returns the previous path and refuses other
    values without changing the current one (host state only)."""
    assert lib.socket_set_selection_path(1) == 0
    assert lib.socket_set_selection_path(7) == -1
    assert lib.socket_set_selection_path(0) == 1
    assert lib.socket_set_selection_path(0) == 0


# Fake, aligned, never-dereferenced device addresses: every call below fails
# validation before it could touch them.
P16 = 0x10000


def decode(lib, entry="socket_decode", **kw):
    a = dict(q=P16, q_dtype=1, W=P16, ids=P16, vnorm=P16, K=P16, V=P16, kv_dtype=1, B=1, Hq=4, Hkv=1, Ncap=64,
             N=64, d=128, L=4, P=8, tau=0.5, k=8, ws=P16, ws_bytes=1 << 30, idx=P16, out=P16, scores=None,
             stream=None)
    a.update(kw)
    return getattr(lib, entry)(a["q"], a["q_dtype"], a["W"], a["ids"], a["vnorm"], a["K"], a["V"], a["kv_dtype"],
                             a["B"], a["Hq"], a["Hkv"], a["Ncap"], a["N"], a["d"], a["L"], a["P"], a["tau"],
                             a["k"], a["ws"], a["ws_bytes"], a["idx"], a["out"], a["scores"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(d=64), EUNSUP),
    (dict(P=9), EUNSUP),
    (dict(P=0), EUNSUP),
    (dict(L=0), EUNSUP),
    (dict(L=129), EUNSUP),
    (dict(Hq=5, Hkv=2), EINVAL),
    (dict(Hq=34, Hkv=2), EUNSUP),
    (dict(k=0), EINVAL),
    (dict(k=65), EINVAL),
    (dict(N=80), EINVAL),
    (dict(Ncap=70, N=64), EINVAL),
    (dict(Ncap=48, N=48), EINVAL),
    (dict(tau=-1.0), EINVAL),
    (dict(tau=float("nan")), EINVAL),
    (dict(tau=float("inf")), EINVAL),
    (dict(q_dtype=7), EINVAL),
    (dict(K=P16 + 8), EINVAL),
    (dict(ids=P16 + 4), EINVAL),
    (dict(out=P16 + 4), EINVAL),
    (dict(scores=P16 + 4), EINVAL),
    (dict(idx=P16 + 2), EINVAL),
    (dict(K=None), EINVAL),
    (dict(ws=P16 + 16), EWS),
    (dict(ws_bytes=16), EWS),
])
@pytest.mark.parametrize("entry", ["socket_decode", "socket_decode_per_head"])
def test_decode_rejects(lib, entry, kw, status):
    assert decode(lib, entry, **kw) == status
    assert lib.socket_last_error().decode() != ""
    assert lib.socket_last_decode_path() == -1  # nothing launched


@pytest.mark.parametrize("n_new", [0, -1, 65, 9])
def test_decode_append_rejects_n_new(lib, n_new):
    # N = 8 keys: n_new may not exceed N, nor 64, nor be below 1.
    assert lib.socket_decode_append(P16, 1, P16, P16, P16, P16, P16, 1, 1, 4, 1, 64, 8, 128, 4, 8, 0.5, 8, n_new,
                                    P16, 1 << 30, P16, P16, None, None) == EINVAL
    assert "n_new" in lib.socket_last_error().decode()


def test_per_head_rejects_too_many_query_heads(lib):
    # 4096 x 32 query-head units exceed the limit; 4096 x 2 kv units would not.
    assert decode(lib, "socket_decode_per_head", B=4096, Hq=32, Hkv=2) == EUNSUP
    assert "B*Hq" in lib.socket_last_error().decode()


def hash_call(lib, **kw):
    a = dict(K=P16, V=P16, kv_dtype=1, B=2, Hkv=2, Ncap=64, n_begin=0, n_end=64, d=128, W=P16, L=4, P=8,
             ids=P16, vnorm=P16, stream=None)
    a.update(kw)
    return lib.socket_hash_keys(a["K"], a["V"], a["kv_dtype"], a["B"], a["Hkv"], a["Ncap"], a["n_begin"],
                                a["n_end"], a["d"], a["W"], a["L"], a["P"], a["ids"], a["vnorm"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(d=96), EUNSUP),
    (dict(P=9), EUNSUP),
    (dict(n_begin=10, n_end=5), EINVAL),
    (dict(n_end=65), EINVAL),
    (dict(n_begin=-1), EINVAL),
    (dict(Ncap=60, n_end=60), EINVAL),
    (dict(Ncap=48, n_end=48), EINVAL),
    (dict(kv_dtype=3), EINVAL),
    (dict(vnorm=P16 + 4), EINVAL),
    (dict(W=None), EINVAL),
    (dict(B=0), EINVAL),
])
def test_hash_rejects(lib, kw, status):
    assert hash_call(lib, **kw) == status


def test_empty_hash_range_is_a_no_op(lib):
    assert hash_call(lib, n_begin=16, n_end=16) == OK


def test_workspace_size(lib):
    f = lib.socket_decode_workspace_size
    small = f(1, 4, 1, 64, 128, 4, 8, 8)
    big = f(8, 32, 8, 131072, 128, 32, 8, 2048)
    assert 0 < small < big
    # scores (4 B per key) and the soft tables dominate; partials grow with k.
    assert big >= 64 * 131072 * 4 + 64 * 32 * 256 * 4
    assert f(8, 32, 8, 131072, 128, 32, 8, 4096) > big
    assert f(1, 4, 1, 64, 64, 4, 8, 8) == 0          # d != 128
    assert f(1, 4, 1, 64, 128, 4, 8, 100) == 0       # k > Ncap
    assert f(1, 3, 2, 64, 128, 4, 8, 8) == 0         # Hq % Hkv != 0


def test_per_head_workspace_size(lib):
    f, g = lib.socket_decode_workspace_size, lib.socket_decode_per_head_workspace_size
    # one head per kv head: the same step, the same workspace
    assert g(2, 4, 4, 4096, 128, 32, 8, 256) == f(2, 4, 4, 4096, 128, 32, 8, 256)
    # four heads per kv head: a table set, a score row and a selection per head
    grouped, per_head = f(8, 32, 8, 131072, 128, 32, 8, 2048), g(8, 32, 8, 131072, 128, 32, 8, 2048)
    assert per_head >= 256 * 131072 * 4 + 256 * 32 * 256 * 4 > grouped
    assert g(4096, 32, 2, 64, 128, 4, 8, 8) == 0     # B*Hq above 65535
    assert g(1, 3, 2, 64, 128, 4, 8, 8) == 0         # Hq % Hkv != 0


def test_python_binding_checks_shapes_before_the_library():
    import torch
    import soft_lsh_top_b200 as s
    with pytest.raises((ValueError, TypeError)):
        s.socket_hash_keys(torch.zeros(1, 1, 16, 128), torch.zeros(1, 1, 16, 128),
                           torch.zeros(4, 8, 128, dtype=torch.bfloat16),
                           torch.zeros(1, 1, 4, 16, dtype=torch.uint8), torch.zeros(1, 1, 16))
    with pytest.raises((ValueError, TypeError)):   # ids in the unchunked [.., Ncap, Lr] shape
        s.socket_hash_keys(torch.zeros(1, 1, 32, 128), torch.zeros(1, 1, 32, 128),
                           torch.zeros(4, 8, 128, dtype=torch.bfloat16),
                           torch.zeros(1, 1, 32, 32, dtype=torch.uint8), torch.zeros(1, 1, 32))


def test_ids_row_bytes(lib):
    f = lib.socket_ids_row_bytes
    assert [f(L) for L in (1, 12, 32, 33, 60, 64, 65, 128)] == [32, 32, 32, 64, 64, 64, 96, 128]
    assert f(0) == 0 and f(129) == 0 and f(-3) == 0


@pytest.mark.parametrize("L", [1, 7, 32, 33, 60, 128])
def test_rotated_id_rows(L):
    """The documented id layout: a bijection between tables and used bytes;
    in every slot the 32 keys 32m .. 32m + 31 name 32 different tables, the one
    periodic column lane + r of the expanded soft table holds; and piece p of
    the chunk's 32 keys is one contiguous 512-byte run."""
    from parity import ids_to_rows, padding_bytes, row_slots, rows_to_ids
    ncap = 96
    slot = row_slots(L, ncap)                                       # [L, ncap]
    for n in range(ncap):
        assert len(set(slot[:, n])) == L
    Lr = 32 * ((L + 31) // 32)
    table_of = np.full((ncap, Lr), -1)
    for l in range(L):
        table_of[np.arange(ncap), slot[l]] = l
    for s in range(Lr):
        c, r = divmod(s, 32)
        for m in range(ncap // 32):
            keys = np.arange(32 * m, 32 * m + 32)
            t = table_of[keys, s]
            lane = keys % 32
            want = 32 * c + (lane + r) % 32                         # column lane + r of block c
            live = want < L
            assert np.array_equal(t[live], want[live]) and np.all(t[~live] == -1)
    rng = np.random.default_rng(5)
    ids = rng.integers(1, 256, size=(3, L, ncap), dtype=np.uint8)
    rows = ids_to_rows(ids, L)
    assert rows.shape == (3, ncap // 32, Lr // 16, 32, 16)
    assert np.array_equal(rows_to_ids(rows, L), ids)
    # key n's row, read back piece by piece, is table_of's row
    for n in (0, 5, 31, 32, 95):
        row = rows[0, n // 32, :, n % 32, :].reshape(-1)
        for s in range(Lr):
            assert row[s] == (ids[0, table_of[n, s], n] if table_of[n, s] >= 0 else 0)
    assert padding_bytes(L, ncap).sum() == ncap * (Lr - L)


def test_python_append_rejects_no_new_keys():
    import torch
    import soft_lsh_top_b200 as s
    z = torch.zeros(1)
    with pytest.raises(ValueError, match="n_new"):
        s.socket_decode_append(z, z, z, z, z, z, 8, 0.5, 4, 0, z, z, z)


def test_sharded_calls_reject_bad_arguments_on_the_host(lib):
    """The sequence-sharded entry points validate before any launch (the
    pointers are never dereferenced)."""
    f = P16
    # a shard holds at least one key
    assert lib.socket_shard_select(f, 1, f, f, f, 1, 4, 1, 64, 0, 128, 8, 8, 0.5, 8, 0, f, 1 << 30, f, f, None) == EINVAL
    # global indices must stay below 2^31
    assert lib.socket_shard_select(f, 1, f, f, f, 1, 4, 1, 64, 64, 128, 8, 8, 0.5, 8, (1 << 31) - 10, f, 1 << 30, f, f,
                                   None) == EINVAL
    assert lib.socket_shard_merge(f, f, 0, 1, 1, 8, 0, 64, f, f, f, None) == EINVAL
    assert lib.socket_shard_merge(f, f, 2, 1, 1, 8, -1, 64, f, f, f, None) == EINVAL
    assert lib.socket_shard_attend_workspace_size(1, 4, 1, 64, 128, 0) == 0
    assert lib.socket_shard_attend_workspace_size(1, 4, 1, 64, 128, 8) > 0
    assert lib.socket_shard_attend(f, 1, f, f, 1, 1, 4, 1, 64, 128, 8, f, f, f, 16, f, f, None) == EWS
    assert lib.socket_shard_combine(f, f, 2, 1, 4, 64, f, None) == EUNSUP
    assert lib.socket_shard_combine(f, f, 0, 1, 4, 128, f, None) == EINVAL


@pytest.mark.parametrize("L, expect", [(16, 36 / 512), (32, 36 / 512), (60, 68 / 512), (80, 100 / 512)])
def test_index_memory_overhead(L, expect):
    """The cached index (id rows of socket_ids_row_bytes(L) bytes plus a
    float32 value norm per key) against the bf16 key and value rows it sits
    beside: (Lr + 4) / (2 d 2).  The pages report about 15 % over the KV
    cache ([ES] "Resultados Experimentales", "Sobrecarga de Memoria"; [DE]
    "Experimentelle Ergebnisse", "Speicher-Overhead") without naming L; the
    workloads here (L = 32 and 60) come to 7.0 % and 13.3 %."""
    import soft_lsh_top_b200 as sk

    B, Hkv, Ncap = 2, 3, 4096
    ids, vnorm = sk.alloc_cache_index(B, Hkv, Ncap, L, "cpu")
    index_bytes = ids.numel() * ids.element_size() + vnorm.numel() * vnorm.element_size()
    kv_bytes = 2 * B * Hkv * Ncap * sk.HEAD_DIM * 2
    assert index_bytes / kv_bytes == pytest.approx(expect, rel=1e-12)
    if L in (32, 60):
        assert index_bytes / kv_bytes < 0.15
