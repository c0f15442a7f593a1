"""Sequence-sharded decode kernels on one GPU: the shards emulated in one
process, the all-gathers replaced by stacking the shards' results in shard
order.  The merged selection must equal socket_decode's over the whole cache
bit for bit (every shard computes the same float32 scores for its keys), and
the combined output must match socket_decode's to float32 rounding and the
fp64 oracle's attention on that selection within the usual 2e-3."""
import numpy as np
import pytest
import torch

import oracle
import soft_lsh_top_b200 as sk
import workloads as wl
from parity import gpu_decode, gpu_hash
from soft_lsh_top_b200 import sharded

pytestmark = pytest.mark.gpu

DEV = "cuda:0"

CASES = {
    # bf16 (tensor-core attention), a shard starting off a 32-key boundary
    "bf16_two_shards": (wl.Workload(name="sh2", B=2, Hq=8, Hkv=2, N=9001, L=12, P=8, tau=0.3, k=400, seed=7401),
                        [0, 4111, 9001]),
    # four shards, one smaller than k (its pairs are padded)
    "bf16_four_shards": (wl.Workload(name="sh4", B=1, Hq=4, Hkv=2, N=6000, L=8, P=7, tau=0.5, k=500, seed=7402),
                         [0, 300, 2900, 4500, 6000]),
    # float32 keys (CUDA-core attention), groups of three
    "f32_three_shards": (wl.Workload(name="sh3", B=1, Hq=6, Hkv=2, N=3000, L=9, P=6, tau=0.25, k=120, dtype="f32",
                                     seed=7403), [0, 1000, 2001, 3000]),
}


def _shard_of(inp, w, a, b):
    n = b - a
    ncap = (n + 31) // 32 * 32
    B = inp["K"].shape[0]
    K = torch.zeros(B, w.Hkv, ncap, 128, dtype=inp["K"].dtype, device=DEV)
    V = torch.zeros_like(K)
    K[:, :, :n] = inp["K"][:, :, a:b]
    V[:, :, :n] = inp["V"][:, :, a:b]
    ids, vnorm = sk.alloc_cache_index(B, w.Hkv, ncap, w.L, DEV)
    sk.socket_hash_keys(K, V, inp["W"], ids, vnorm, 0, n)
    return sharded.Shard(ids=ids, vnorm=vnorm, K=K, V=V, N=n, n_offset=a)


@pytest.mark.parametrize("case", sorted(CASES))
def test_sharded_kernels_equal_the_unsharded_decode(case):
    w, cuts = CASES[case]
    inp = wl.make_inputs(w, DEV)
    ids, vnorm = gpu_hash(inp, w)
    want_idx, want_out, _ = gpu_decode(inp, w, ids, vnorm)

    shards = [_shard_of(inp, w, a, b) for a, b in zip(cuts[:-1], cuts[1:])]
    ops = sharded.KernelOps()
    pairs = [ops.select(inp["q"], inp["W"], sh, w.tau, w.k) for sh in shards]
    scores = torch.stack([p[0] for p in pairs])
    indices = torch.stack([p[1] for p in pairs])
    merged = [ops.merge(scores, indices, sh, w.k) for sh in shards]
    parts = [ops.attend(inp["q"], sh, w.k, m[1], m[2]) for sh, m in zip(shards, merged)]
    out = ops.combine(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]))
    torch.cuda.synchronize()

    for idx, local_idx, local_count in merged:
        assert torch.equal(idx, want_idx)
    # each shard's share is exactly its part of the selection, in local indices
    for sh, (_, local_idx, local_count) in zip(shards, merged):
        for b in range(w.B):
            for h in range(w.Hkv):
                g = want_idx[b, h]
                mine = g[(g >= sh.n_offset) & (g < sh.n_offset + sh.N)] - sh.n_offset
                assert int(local_count[b, h]) == mine.numel()
                assert torch.equal(local_idx[b, h, :mine.numel()], mine)
    torch.testing.assert_close(out, want_out, rtol=1e-5, atol=1e-5)
    Wc = inp["W"].cpu()
    for b in range(w.B):
        for h in range(w.Hkv):
            ref = oracle.attention(inp["q"][b, h * w.G:(h + 1) * w.G].cpu(), inp["K"][b, h].cpu(),
                                   inp["V"][b, h].cpu(), want_idx[b, h].cpu().numpy())
            err = np.max(np.abs(out[b, h * w.G:(h + 1) * w.G].double().cpu().numpy() - ref))
            assert err <= 2e-3, err


def test_a_shard_with_no_selected_keys_contributes_nothing():
    """A shard none of whose keys is selected gets count 0, a zero output and
    l = 0, and the combine ignores it."""
    w = wl.Workload(name="sh_empty", B=1, Hq=4, Hkv=1, N=3000, L=6, P=8, tau=0.3, k=64, seed=7404)
    inp = wl.make_inputs(w, DEV)
    # keys 2000.. get tiny values, so their scores (value norm times the soft
    # collision mass) cannot reach the top 64
    inp["V"][:, :, 2000:w.N] *= 1e-6
    ids, vnorm = gpu_hash(inp, w)
    want_idx, want_out, _ = gpu_decode(inp, w, ids, vnorm)
    assert int(want_idx.max()) < 2000
    shards = [_shard_of(inp, w, 0, 2000), _shard_of(inp, w, 2000, w.N)]
    ops = sharded.KernelOps()
    pairs = [ops.select(inp["q"], inp["W"], sh, w.tau, w.k) for sh in shards]
    scores = torch.stack([p[0] for p in pairs])
    indices = torch.stack([p[1] for p in pairs])
    merged = [ops.merge(scores, indices, sh, w.k) for sh in shards]
    assert int(merged[1][2].sum()) == 0
    parts = [ops.attend(inp["q"], sh, w.k, m[1], m[2]) for sh, m in zip(shards, merged)]
    torch.cuda.synchronize()
    assert torch.all(parts[1][0] == 0)
    assert torch.all(parts[1][1][..., 1] == 0)
    out = ops.combine(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]))
    assert torch.equal(merged[0][0], want_idx)
    torch.testing.assert_close(out, want_out, rtol=1e-5, atol=1e-5)
