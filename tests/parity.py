"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and compare it with the oracle under the matching rules.

Matching rules (floating point decides the selection, so the selection is
compared in the kernel's precision and, separately, against fp64):
  * bucket ids bit-exact, except keys whose smallest |<W_lp, k>| is below
    1e-4 ||k|| (the oracle reports that margin);
  * value norms within 1e-6 relative (float32 sum of squares of 128 terms);
  * scores within 1e-5 relative, with an absolute floor of 1e-5 x the unit's
    largest score (near-underflow temperatures make tiny scores meaningless
    in relative terms);
  * the selected set bit-exact against the oracle's selection applied to the
    kernel's own float32 scores, and differing from the fp64 selection only at
    keys whose fp64 score is within 1e-6 relative of the fp64 k-th score;
  * attention output within 2e-3 max-abs of fp64 attention on the same set.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import soft_lsh_top_b200 as sk

ID_MARGIN = 1e-4
VNORM_RTOL = 1e-6
SCORE_RTOL = 1e-5
SCORE_FLOOR = 1e-5
SET_BAND = 1e-6
OUT_ATOL = 2e-3


def row_slots(L, ncap):
    """Slot of table l in key n's id row, [L, ncap]: 32 (l // 32) + (l - n) mod 32
    (the rotation documented for socket_hash_keys)."""
    l = np.arange(L)[:, None]
    n = np.arange(ncap)[None, :]
    return 32 * (l // 32) + (l % 32 - n) % 32


def _chunked_index(L, ncap):
    """For table l and key n, the flat byte offset of its id inside a unit's
    chunked array [ncap/32][Lr/16][32][16]: chunk n // 32, piece s // 16,
    lane n % 32, byte s % 16 with s = row_slots(L, ncap)."""
    Lr = 32 * ((L + 31) // 32)
    s = row_slots(L, ncap)
    n = np.arange(ncap)[None, :]
    return (((n // 32) * (Lr // 16) + s // 16) * 32 + n % 32) * 16 + s % 16


def ids_to_rows(tab_ids, L):
    """Table-major ids [..., L, ncap] -> chunked rows [..., ncap/32, Lr/16, 32, 16] (padding 0)."""
    ncap = tab_ids.shape[-1]
    Lr = 32 * ((L + 31) // 32)
    flat = np.zeros(tab_ids.shape[:-2] + (ncap * Lr,), dtype=np.uint8)
    flat[..., _chunked_index(L, ncap)] = tab_ids
    return flat.reshape(tab_ids.shape[:-2] + (ncap // 32, Lr // 16, 32, 16))


def rows_to_ids(rows, L):
    """Chunked rows [..., ncap/32, Lr/16, 32, 16] -> table-major ids [..., L, ncap]."""
    ncap = rows.shape[-4] * 32
    flat = rows.reshape(rows.shape[:-4] + (-1,))
    return flat[..., _chunked_index(L, ncap)]


def padding_bytes(L, ncap):
    """Mask [ncap * Lr] of the chunked array's bytes that hold no table's id."""
    Lr = 32 * ((L + 31) // 32)
    used = np.zeros(ncap * Lr, dtype=bool)
    used[_chunked_index(L, ncap)] = True
    return ~used


def gpu_hash(inp, w, n_begin=0, n_end=None):
    dev = inp["K"].device
    ids, vnorm = sk.alloc_cache_index(inp["K"].shape[0], w.Hkv, w.ncap, w.L, dev)
    ids.zero_()
    vnorm.zero_()
    sk.socket_hash_keys(inp["K"], inp["V"], inp["W"], ids, vnorm, n_begin, w.N if n_end is None else n_end)
    sk.socket_hash_check()
    return ids, vnorm


def gpu_decode(inp, w, ids, vnorm, N=None, tau=None, k=None, q=None, per_head=False):
    """socket_decode (per_head: socket_decode_per_head) with the scores kept."""
    dev = inp["K"].device
    B = inp["K"].shape[0]
    N = w.N if N is None else N
    k = w.k if k is None else k
    q = inp["q"] if q is None else q
    ws, idx, out = sk.alloc_decode_buffers(B, w.Hq, w.Hkv, w.ncap, w.L, w.P, k, dev, per_head=per_head)
    scores = torch.full((B, w.Hq if per_head else w.Hkv, w.ncap), float("nan"), dtype=torch.float32, device=dev)
    fn = sk.socket_decode_per_head if per_head else sk.socket_decode
    fn(q, inp["W"], ids, vnorm, inp["K"], inp["V"], N, w.tau if tau is None else tau, k, ws, idx, out,
       scores_out=scores)
    torch.cuda.synchronize()
    assert sk.read_device_error(ws) == 0
    return idx, out, scores


def oracle_hash_units(inp, w, units, n_begin=0, n_end=None):
    """Oracle ids [len(units), L, ncap] (zeros outside the range), fp64 vnorm, margin."""
    n_end = w.N if n_end is None else n_end
    ids = np.zeros((len(units), w.L, w.ncap), dtype=np.uint8)
    vn = np.zeros((len(units), w.ncap), dtype=np.float64)
    mg = np.full((len(units), w.ncap), np.inf)
    for i, u in enumerate(units):
        b, h = divmod(u, w.Hkv)
        K = inp["K"][b, h, n_begin:n_end].cpu()
        V = inp["V"][b, h, n_begin:n_end].cpu()
        a, v, m = oracle.hash_keys(K, V, inp["W"].cpu(), w.L, w.P)
        ids[i, :, n_begin:n_end] = a
        vn[i, n_begin:n_end] = v
        mg[i, n_begin:n_end] = m
    return ids, vn, mg


def check_hash(gpu_rows, gpu_vn, orc_ids, orc_vn, margin, n_begin, n_end):
    """gpu_rows [U, ncap/32, Lr/16, 32, 16], gpu_vn [U, ncap]: numpy for the same
    units as the oracle arrays.  Bytes of tables >= L must hold 0 for the
    hashed keys."""
    L = orc_ids.shape[1]
    ncap = gpu_rows.shape[1] * 32
    Lr = gpu_rows.shape[2] * 16
    pad = padding_bytes(L, ncap).reshape(ncap // 32, Lr // 16, 32, 16)
    keys = np.zeros((ncap // 32, 1, 32, 1), dtype=bool)
    keys.reshape(-1)[n_begin:n_end] = True
    flat = gpu_rows.reshape(gpu_rows.shape[0], -1)
    assert not np.any(flat[:, (pad & keys).reshape(-1)]), "padding slots not zero"
    gpu_ids = rows_to_ids(gpu_rows, L)
    g = gpu_ids[..., n_begin:n_end]
    o = orc_ids[..., n_begin:n_end]
    exempt = margin[:, n_begin:n_end] < ID_MARGIN                    # [U, n]
    diff = np.any(g != o, axis=1)                                    # [U, n]
    assert not np.any(diff & ~exempt), f"{int(np.sum(diff & ~exempt))} non-exempt id mismatches"
    gv = gpu_vn[:, n_begin:n_end].astype(np.float64)
    ov = orc_vn[:, n_begin:n_end]
    assert np.all(np.abs(gv - ov) <= VNORM_RTOL * ov + 1e-30)
    return int(np.sum(diff)), int(np.sum(exempt))


def check_unit(q_u, W, L, P, tau, ids_u, vn_u, K_u, V_u, N, k, g_idx, g_out, g_sc):
    """Compare one unit's GPU results with the oracle decode on the same ids/norms."""
    o_idx, o_out, o_sc, _ = oracle.decode_unit(q_u, W, L, P, tau, ids_u, vn_u, K_u, V_u, N, k)
    g_sc = np.asarray(g_sc[:N], dtype=np.float64)
    floor = SCORE_FLOOR * o_sc.max()
    bad = np.abs(g_sc - o_sc) > SCORE_RTOL * np.abs(o_sc) + floor
    assert not bad.any(), f"{int(bad.sum())} scores off, worst rel {np.max(np.abs(g_sc - o_sc) / (o_sc + floor)):.3g}"
    g_idx = np.asarray(g_idx)
    assert np.array_equal(g_idx, oracle.topk(g_sc, k)), "selection differs from the oracle's on the kernel's scores"
    kth = np.sort(o_sc)[-k]
    swapped = np.setxor1d(g_idx, o_idx)
    far = swapped[np.abs(o_sc[swapped] - kth) > SET_BAND * kth]
    assert far.size == 0, f"selected set differs away from the k-th score: {far[:10]}"
    same = oracle.attention(q_u, K_u, V_u, g_idx)
    err = np.max(np.abs(np.asarray(g_out, dtype=np.float64) - same))
    assert err <= OUT_ATOL, f"attention max-abs error {err}"
    if swapped.size == 0:
        assert np.max(np.abs(np.asarray(g_out, dtype=np.float64) - o_out)) <= OUT_ATOL
    return {"swapped": int(swapped.size), "out_err": float(err)}


def check_decode(inp, w, orc_ids, orc_vn32, units, g_idx, g_out, g_sc, N=None, tau=None, k=None, q=None,
                 per_head=False):
    """Compare sampled kv units.  per_head: the results of
    socket_decode_per_head, each query head checked as a unit of one query
    row over its kv head's ids, norms, keys and values."""
    N = w.N if N is None else N
    k = w.k if k is None else k
    tau = w.tau if tau is None else tau
    q = inp["q"] if q is None else q
    Wc = inp["W"].cpu()
    stats = []
    for i, u in enumerate(units):
        b, h = divmod(u, w.Hkv)
        q_u = q[b, h * w.G:(h + 1) * w.G].cpu()
        K_u = inp["K"][b, h].cpu()
        V_u = inp["V"][b, h].cpu()
        if per_head:
            for g in range(w.G):
                r = h * w.G + g
                stats.append(check_unit(q_u[g:g + 1], Wc, w.L, w.P, tau, orc_ids[i], orc_vn32[i], K_u, V_u, N, k,
                                        g_idx[b, r].cpu().numpy(), g_out[b, r:r + 1].cpu().numpy(),
                                        g_sc[b, r].cpu().numpy()))
            continue
        stats.append(check_unit(q_u, Wc, w.L, w.P, tau, orc_ids[i], orc_vn32[i], K_u, V_u, N, k,
                                g_idx[b, h].cpu().numpy(), g_out[b, h * w.G:(h + 1) * w.G].cpu().numpy(),
                                g_sc[b, h].cpu().numpy()))
    return stats


def substitute_units(ids, vnorm, w, units, orc_ids, orc_vn32):
    """Copy the oracle's ids / norms of `units` into the device index tensors."""
    for i, u in enumerate(units):
        b, h = divmod(u, w.Hkv)
        ids[b, h].copy_(torch.from_numpy(ids_to_rows(orc_ids[i], w.L)))
        vnorm[b, h].copy_(torch.from_numpy(orc_vn32[i]))
