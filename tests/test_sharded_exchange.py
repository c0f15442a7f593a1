"""The sequence-sharded decode step's exchange, on CPU: gloo ranks.

soft_lsh_top_b200.sharded.decode_step splits one step into per-rank steps
(select on the rank's keys, merge the gathered pairs, attend on the rank's
share, merge the softmax states) joined by two all-gathers.  Here each rank
runs those steps with oracle arithmetic (fp64, test-side stand-ins for the
kernels, which the GPU tests check) over gloo, and the result must equal
the oracle's decode of the whole sequence: the same k indices, the same
output to fp64 rounding.  What this pins is the exchange: pairs gathered in
rank order with global indices, each rank's share of the selection, and the
log-sum-exp merge of the shards' states.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

W_CASE = dict(name="sharded_cpu", B=1, Hq=4, Hkv=2, N=2600, L=6, P=6, tau=0.4, k=150, seed=7300)


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleOps:
    """The step's four operations in fp64 on CPU, from the oracle's hash,
    scores and selection."""

    def __init__(self, oracle, W, L, P):
        self.o, self.W, self.L, self.P = oracle, W, L, P

    def select(self, q, W, shard, tau, k):
        B, Hq, _ = q.shape
        Hkv = shard.K.shape[1]
        G = Hq // Hkv
        k_eff = min(k, shard.N)
        score = torch.full((B, Hkv, k), -1.0, dtype=torch.float64)
        index = torch.full((B, Hkv, k), -1, dtype=torch.int32)
        for b in range(B):
            for h in range(Hkv):
                K = shard.K[b, h, :shard.N]
                V = shard.V[b, h, :shard.N]
                ids, vn, _ = self.o.hash_keys(K, V, W, self.L, self.P)
                _, _, sc, _ = self.o.decode_unit(q[b, h * G:(h + 1) * G], W, self.L, self.P, tau, ids,
                                                 vn.astype(np.float32), K, V, shard.N, k_eff)
                sel = self.o.topk(sc, k_eff)
                score[b, h, :k_eff] = torch.from_numpy(sc[sel])
                index[b, h, :k_eff] = torch.from_numpy(sel.astype(np.int32) + shard.n_offset)
        return score, index

    def merge(self, scores, indices, shard, k):
        S, B, Hkv, _ = scores.shape
        idx = torch.full((B, Hkv, k), -1, dtype=torch.int32)
        local_idx = torch.zeros((B, Hkv, k), dtype=torch.int32)
        local_count = torch.zeros((B, Hkv), dtype=torch.int32)
        for b in range(B):
            for h in range(Hkv):
                sc = scores[:, b, h].reshape(-1).numpy()
                ix = indices[:, b, h].reshape(-1).numpy()
                ok = ix >= 0
                sc, ix = sc[ok], ix[ok]
                order = np.lexsort((ix, -sc))[:k]  # score descending, index ascending
                chosen = np.sort(ix[order])
                idx[b, h, :chosen.size] = torch.from_numpy(chosen.astype(np.int32))
                mine = chosen[(chosen >= shard.n_offset) & (chosen < shard.n_offset + shard.N)] - shard.n_offset
                local_idx[b, h, :mine.size] = torch.from_numpy(mine.astype(np.int32))
                local_count[b, h] = mine.size
        return idx, local_idx, local_count

    def attend(self, q, shard, k, local_idx, local_count):
        B, Hq, d = q.shape
        Hkv = shard.K.shape[1]
        G = Hq // Hkv
        out = torch.zeros((B, Hq, d), dtype=torch.float64)
        ml = torch.zeros((B, Hq, 2), dtype=torch.float64)
        for b in range(B):
            for h in range(Hkv):
                rows = local_idx[b, h, :int(local_count[b, h])].long()
                Kr = shard.K[b, h, rows].double()
                Vr = shard.V[b, h, rows].double()
                for g in range(G):
                    r = h * G + g
                    if rows.numel() == 0:
                        ml[b, r] = torch.tensor([float("-inf"), 0.0], dtype=torch.float64)
                        continue
                    logits = Kr @ q[b, r].double() / np.sqrt(d)
                    m = logits.max()
                    w = torch.exp(logits - m)
                    out[b, r] = (w[:, None] * Vr).sum(0) / w.sum()
                    ml[b, r] = torch.stack([m, w.sum()])
        return out, ml

    def combine(self, outs, mls):
        m = mls[..., 0]
        l = mls[..., 1]
        has = l > 0
        M = torch.where(has, m, torch.full_like(m, float("-inf"))).max(dim=0).values
        w = torch.where(has, torch.exp(m - M) * l, torch.zeros_like(l))
        return (w[..., None] * outs).sum(0) / w.sum(0)[..., None]


def _rank_main(rank: int, world: int, port: int, cuts, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch.distributed as dist

    import oracle
    import workloads as wl
    from soft_lsh_top_b200 import sharded

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = wl.Workload(**W_CASE)
        inp = wl.make_inputs(w)
        a, b = cuts[rank], cuts[rank + 1]
        shard = sharded.Shard(ids=None, vnorm=torch.zeros(1), K=inp["K"][:, :, a:b], V=inp["V"][:, :, a:b],
                              N=b - a, n_offset=a)
        sharded.check_layout(shard)
        ops = OracleOps(oracle, inp["W"], w.L, w.P)
        idx, out = sharded.decode_step(inp["q"], inp["W"], shard, w.tau, w.k, ops=ops)
        results.put((rank, idx.numpy(), out.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("cuts", [[0, 1400, 2600], [0, 100, 1700, 2600]])
def test_sharded_step_over_gloo_equals_the_whole_sequence(cuts):
    """Two and three ranks (one holding fewer keys than k): every rank ends
    with the whole sequence's selection and output."""
    sys.path.insert(0, ROOT)
    import oracle
    import workloads as wl

    world = len(cuts) - 1
    ctx = mp.get_context("spawn")
    results = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, cuts, results)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted((results.get(timeout=300) for _ in procs), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0

    w = wl.Workload(**W_CASE)
    inp = wl.make_inputs(w)
    for b in range(w.B):
        for h in range(w.Hkv):
            K = inp["K"][b, h, :w.N]
            V = inp["V"][b, h, :w.N]
            ids, vn, _ = oracle.hash_keys(K, V, inp["W"], w.L, w.P)
            want_idx, want_out, _, _ = oracle.decode_unit(inp["q"][b, h * w.G:(h + 1) * w.G], inp["W"], w.L, w.P,
                                                          w.tau, ids, vn.astype(np.float32), K, V, w.N, w.k)
            for _, idx, out in got:
                assert np.array_equal(idx[b, h], want_idx)
                np.testing.assert_allclose(out[b, h * w.G:(h + 1) * w.G], want_out, rtol=0, atol=1e-10)
