"""One decode step over a sequence split by position across ranks.

Each rank holds a contiguous range of the sequence's keys (its own cache
arrays, hashed with socket_hash_keys as usual) and runs the same step: it
selects its own top-k (socket_shard_select), the ranks all-gather their
(score, global index) pairs, every rank re-selects the global top-k from
them (socket_shard_merge), attends over the selected keys it holds
(socket_shard_attend), and the ranks all-gather their partial softmax
states, which every rank merges (socket_shard_combine).  The result equals
socket_decode over the whole cache: the same selection, and the same
output up to float32 rounding.  The kernels are the library's; this module
only moves tensors between ranks with torch.distributed (NCCL over NVLink on
GPUs) and allocates the buffers.

The steps are injectable (``ops``) so the exchange itself can be exercised
by processes without a GPU.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist

from . import (HEAD_DIM, socket_decode_workspace_size, socket_shard_attend, socket_shard_attend_workspace_size,
               socket_shard_combine, socket_shard_merge, socket_shard_select)


@dataclass
class Shard:
    """This rank's keys: global positions [n_offset, n_offset + N)."""
    ids: torch.Tensor     # [B, Hkv, Ncap/32, Lr/16, 32, 16] uint8
    vnorm: torch.Tensor   # [B, Hkv, Ncap] float32
    K: torch.Tensor       # [B, Hkv, Ncap, 128]
    V: torch.Tensor       # [B, Hkv, Ncap, 128]
    N: int
    n_offset: int


class KernelOps:
    """The step's kernels on this rank's GPU (workspaces cached by shape)."""

    def __init__(self):
        self._ws = {}

    def _workspace(self, key, nbytes: int, device) -> torch.Tensor:
        ws = self._ws.get(key)
        if ws is None or ws.numel() < nbytes or ws.device != device:
            ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
            self._ws[key] = ws
        return ws

    def select(self, q, W, shard: Shard, tau: float, k: int):
        B, Hq, _ = q.shape
        _, Hkv, Ncap = shard.vnorm.shape
        L, P, _ = W.shape
        k_eff = min(k, shard.N)  # a shard with fewer than k keys selects them all
        ws = self._workspace("select", socket_decode_workspace_size(B, Hq, Hkv, Ncap, HEAD_DIM, L, P, k_eff),
                             q.device)
        score = torch.empty(B, Hkv, k, dtype=torch.float32, device=q.device)
        index = torch.empty(B, Hkv, k, dtype=torch.int32, device=q.device)
        socket_shard_select(q, W, shard.ids, shard.vnorm, shard.N, tau, k, shard.n_offset, ws, score, index)
        return score, index

    def merge(self, scores, indices, shard: Shard, k: int):
        _, B, Hkv, _ = scores.shape
        idx = torch.empty(B, Hkv, k, dtype=torch.int32, device=scores.device)
        local_idx = torch.empty_like(idx)
        local_count = torch.empty(B, Hkv, dtype=torch.int32, device=scores.device)
        socket_shard_merge(scores, indices, shard.n_offset, shard.N, idx, local_idx, local_count)
        return idx, local_idx, local_count

    def attend(self, q, shard: Shard, k: int, local_idx, local_count):
        B, Hq, d = q.shape
        _, Hkv, Ncap, _ = shard.K.shape
        ws = self._workspace("attend", socket_shard_attend_workspace_size(B, Hq, Hkv, Ncap, k), q.device)
        out = torch.empty(B, Hq, d, dtype=torch.float32, device=q.device)
        ml = torch.empty(B, Hq, 2, dtype=torch.float32, device=q.device)
        socket_shard_attend(q, shard.K, shard.V, k, local_idx, local_count, ws, out, ml)
        return out, ml

    def combine(self, outs, mls):
        _, B, Hq, d = outs.shape
        out = torch.empty(B, Hq, d, dtype=torch.float32, device=outs.device)
        socket_shard_combine(outs, mls, out)
        return out


def all_gather_stacked(x: torch.Tensor, group=None) -> torch.Tensor:
    """[world, *x.shape]: every rank's x, in rank order."""
    world = dist.get_world_size(group)
    parts = [torch.empty_like(x) for _ in range(world)]
    dist.all_gather(parts, x.contiguous(), group=group)
    return torch.stack(parts)


def check_layout(shard: Shard, group=None) -> None:
    """The ranks' key ranges must tile the sequence in rank order."""
    me = torch.tensor([shard.n_offset, shard.N], dtype=torch.int64, device=shard.vnorm.device)
    ranges = all_gather_stacked(me, group).cpu().tolist()
    pos = 0
    for r, (off, n) in enumerate(ranges):
        if off != pos or n < 1:
            raise ValueError(f"rank {r} holds keys [{off}, {off + n}); expected a range starting at {pos}")
        pos = off + n


def decode_step(q: torch.Tensor, W: torch.Tensor, shard: Shard, tau: float, k: int, group=None, ops=None,
                gather=None):
    """One sharded decode step on this rank.  Returns (idx [B, Hkv, k] int32,
    global indices ascending; out [B, Hq, 128] float32), the same on every
    rank.  Every rank must call it with the same q, W, tau and k."""
    ops = ops if ops is not None else KernelOps()
    gather = gather if gather is not None else (lambda t: all_gather_stacked(t, group))
    score, index = ops.select(q, W, shard, tau, k)
    scores, indices = gather(score), gather(index)
    idx, local_idx, local_count = ops.merge(scores, indices, shard, k)
    out, ml = ops.attend(q, shard, k, local_idx, local_count)
    return idx, ops.combine(gather(out), gather(ml))
