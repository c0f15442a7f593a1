"""CUDA path vs oracle, element by element, through the C ABI (needs a GPU).

Small and ragged cases are compared on every unit and key; the full-size
workloads (batch-8 128K, one million tokens, batch-32 16K with appends) are
compared on sampled units, in the same launch configuration the benchmark
times.  Matching rules are in parity.py.
"""
import numpy as np
import pytest
import torch

import oracle
import soft_lsh_top_b200 as sk
import workloads as wl
from parity import (check_decode, check_hash, gpu_decode, gpu_hash, ids_to_rows, oracle_hash_units, rows_to_ids,
                    substitute_units)

pytestmark = pytest.mark.gpu

DEV = "cuda:0"

SMALL = {
    "tiny_f32_4k": wl.TINY,
    "llama_32k": wl.LLAMA_32K,
    "ragged_multitile": wl.LLAMA_32K.scaled(name="ragged", B=2, Hq=8, Hkv=2, N=70001, L=12, k=700, tau=0.4,
                                            seed=7001),
    "odd_group3_p5": wl.Workload(name="odd", B=2, Hq=6, Hkv=2, N=3001, L=7, P=5, tau=0.7, k=77, seed=7002),
    "f32_group2_p6": wl.Workload(name="f32g2", B=1, Hq=4, Hkv=2, N=2500, L=9, P=6, tau=0.25, k=100, dtype="f32",
                                 seed=7003),
    # bfloat16 at the group sizes that bound the attention kernels: one head,
    # eight heads (the widest tensor-core tile) and sixteen (the CUDA-core path).
    "bf16_single_head": wl.Workload(name="g1", B=2, Hq=2, Hkv=2, N=4099, L=8, P=8, tau=0.3, k=200, seed=7005),
    "bf16_group8_p7": wl.Workload(name="g8", B=1, Hq=16, Hkv=2, N=5000, L=10, P=7, tau=0.5, k=300, seed=7006),
    "bf16_group16": wl.Workload(name="g16", B=1, Hq=16, Hkv=1, N=3000, L=6, P=8, tau=0.4, k=129, seed=7007),
    # more than 64 tables: the scoring runs in two launches that pass partial
    # sums through the score buffer (three and four 32-table blocks).
    "bf16_l80_p7": wl.Workload(name="l80", B=1, Hq=4, Hkv=2, N=2500, L=80, P=7, tau=0.4, k=150, seed=7008),
    "f32_l128_group2": wl.Workload(name="l128", B=1, Hq=4, Hkv=2, N=1800, L=128, P=5, tau=0.6, k=90, dtype="f32",
                                   seed=7009),
}


@pytest.fixture(scope="module", params=sorted(SMALL))
def small(request):
    w = SMALL[request.param]
    inp = wl.make_inputs(w, DEV)
    units = list(range(w.U))
    orc_ids, orc_vn, margin = oracle_hash_units(inp, w, units)
    return w, inp, units, orc_ids, orc_vn, margin


def test_hash_matches_oracle(small):
    w, inp, units, orc_ids, orc_vn, margin = small
    ids, vnorm = gpu_hash(inp, w)
    torch.cuda.synchronize()
    g_ids = ids.reshape(w.U, w.ncap // 32, -1, 32, 16).cpu().numpy()
    g_vn = vnorm.reshape(w.U, w.ncap).cpu().numpy()
    check_hash(g_ids, g_vn, orc_ids, orc_vn, margin, 0, w.N)


def _decode_on_oracle_index(small, **kw):
    """Decode on the oracle's ids and norms (so that scores compare key by key)."""
    w, inp, units, orc_ids, orc_vn, _ = small
    orc_vn32 = orc_vn.astype(np.float32)
    ids = torch.from_numpy(ids_to_rows(orc_ids, w.L)).reshape(inp["K"].shape[0], w.Hkv, w.ncap // 32, -1, 32,
                                                               16).to(DEV)
    vn = torch.from_numpy(orc_vn32).reshape(inp["K"].shape[0], w.Hkv, w.ncap).to(DEV)
    idx, out, sc = gpu_decode(inp, w, ids, vn, **kw)
    return check_decode(inp, w, orc_ids, orc_vn32, units, idx, out, sc, **kw)


@pytest.mark.parametrize("case", ["bf16_single_head", "odd_group3_p5", "bf16_l80_p7"])
def test_hash_in_ranges_matches_oracle(case):
    """The cache hashed piecewise -- a long range from an unaligned start, single
    appended keys, a range inside one 32-key chunk, the rest -- equals the
    oracle's hash of every key (tensor-core tiles that start anywhere and end
    ragged; the last case has more hyperplanes than one tensor-core
    accumulator holds and runs in two passes over 32-table blocks)."""
    w = SMALL[case]
    inp = wl.make_inputs(w, DEV)
    ids, vnorm = sk.alloc_cache_index(inp["K"].shape[0], w.Hkv, w.ncap, w.L, DEV)
    ids.zero_()
    vnorm.zero_()
    cuts = sorted({0, 37, 38, 39, 70, 1000, 1001, w.N - 1, w.N})
    for a, b in zip(cuts[:-1], cuts[1:]):
        sk.socket_hash_keys(inp["K"], inp["V"], inp["W"], ids, vnorm, a, b)
    sk.socket_hash_check()
    units = list(range(w.U))
    orc_ids, orc_vn, margin = oracle_hash_units(inp, w, units)
    check_hash(ids.reshape(w.U, w.ncap // 32, -1, 32, 16).cpu().numpy(), vnorm.reshape(w.U, w.ncap).cpu().numpy(),
               orc_ids, orc_vn, margin, 0, w.N)


# Many units with more appended keys than one projection pass holds.
APPEND_EXTRA = {
    "many_units_l32": wl.Workload(name="append_many", B=80, Hq=2, Hkv=1, N=2100, L=32, P=8, tau=0.3, k=64,
                                  seed=7401),
}


@pytest.mark.parametrize("case", ["bf16_single_head", "odd_group3_p5", "f32_group2_p6", "bf16_l80_p7",
                                  "bf16_group16", "many_units_l32"])
def test_decode_append_hashes_and_decodes(case):
    """socket_decode_append: the step hashes the keys just appended (1, 5, then
    33 keys, so chunk boundaries are crossed) and decodes over them.  The ids
    and norms of every key match the oracle's hash (within the float32
    exemption band), and each step's scores, selection and output match the
    oracle run on the index the step saw."""
    w = SMALL[case] if case in SMALL else APPEND_EXTRA[case]
    inp = wl.make_inputs(w, DEV)
    B = inp["K"].shape[0]
    ids, vnorm = sk.alloc_cache_index(B, w.Hkv, w.ncap, w.L, DEV)
    ids.zero_()
    vnorm.zero_()
    n = w.N - 39
    sk.socket_hash_keys(inp["K"], inp["V"], inp["W"], ids, vnorm, 0, n)
    sk.socket_hash_check()
    ws, idx, out = sk.alloc_decode_buffers(B, w.Hq, w.Hkv, w.ncap, w.L, w.P, w.k, DEV)
    units = list(range(w.U))
    for n_new in (1, 5, 33):
        n += n_new
        scores = torch.full((B, w.Hkv, w.ncap), float("nan"), dtype=torch.float32, device=DEV)
        sk.socket_decode_append(inp["q"], inp["W"], ids, vnorm, inp["K"], inp["V"], n, w.tau, w.k, n_new, ws, idx,
                                out, scores_out=scores)
        torch.cuda.synchronize()
        assert sk.read_device_error(ws) == 0
        # Keys appended in the call are hashed by the soft-table kernel, so such
        # a step never runs as the one-kernel step.
        assert sk.socket_last_decode_path() in (sk.SOCKET_STEP_SEPARATE, sk.SOCKET_STEP_FUSED)
        g_ids = rows_to_ids(ids.reshape(w.U, w.ncap // 32, -1, 32, 16).cpu().numpy(), w.L)
        g_vn = vnorm.reshape(w.U, w.ncap).cpu().numpy()
        check_decode(inp, w, g_ids, g_vn, units, idx, out, scores, N=n)
    orc_ids, orc_vn, margin = oracle_hash_units(inp, w, units, 0, n)
    check_hash(ids.reshape(w.U, w.ncap // 32, -1, 32, 16).cpu().numpy(), vnorm.reshape(w.U, w.ncap).cpu().numpy(),
               orc_ids, orc_vn, margin, 0, n)


def test_decode_matches_oracle(small):
    _decode_on_oracle_index(small)


def test_decode_per_head_matches_oracle(small):
    """One selection per query head: every head's scores, selection and
    output against the oracle run on that head alone."""
    _decode_on_oracle_index(small, per_head=True)


def test_per_head_with_one_head_per_kv_head_is_the_grouped_decode():
    """With Hq == Hkv both entry points compute the same thing, bit for bit."""
    w = SMALL["bf16_single_head"]
    inp = wl.make_inputs(w, DEV)
    ids, vnorm = gpu_hash(inp, w)
    idx_a, out_a, sc_a = gpu_decode(inp, w, ids, vnorm)
    idx_b, out_b, sc_b = gpu_decode(inp, w, ids, vnorm, per_head=True)
    assert torch.equal(idx_a, idx_b)
    assert torch.equal(out_a, out_b)
    assert torch.equal(sc_a[..., :w.N], sc_b[..., :w.N])


@pytest.mark.parametrize("variant", ["k1", "k_eq_n", "tau_0.01", "tau_5", "tau_0_hard", "n_not_ncap",
                                     "per_head_k1", "per_head_tau_0_hard", "per_head_n_not_ncap"])
def test_decode_edge_cases(small, variant):
    w = small[0]
    kw = {}
    if variant.startswith("per_head_"):
        variant = variant[len("per_head_"):]
        kw["per_head"] = True
    if variant == "k1":
        _decode_on_oracle_index(small, k=1, **kw)
    elif variant == "k_eq_n":
        _decode_on_oracle_index(small, k=w.N, **kw)
    elif variant == "tau_0.01":
        _decode_on_oracle_index(small, tau=0.01, **kw)
    elif variant == "tau_5":
        _decode_on_oracle_index(small, tau=5.0, **kw)
    elif variant == "tau_0_hard":
        _decode_on_oracle_index(small, tau=0.0, **kw)
    else:
        n = w.N - 13
        _decode_on_oracle_index(small, N=n, k=min(w.k, n), **kw)


def test_all_ties_select_lowest_indices():
    """Zero queries give every bucket 2^-P and equal value norms give every key
    the same score: the selection must be keys 0..k-1."""
    w = wl.Workload(name="ties", B=1, Hq=4, Hkv=2, N=9000, L=5, P=8, tau=0.3, k=333, seed=7004)
    inp = wl.make_inputs(w, DEV)
    inp["q"].zero_()
    inp["V"].fill_(1.0)
    ids, vnorm = gpu_hash(inp, w)
    idx, out, sc = gpu_decode(inp, w, ids, vnorm)
    want = torch.arange(w.k, dtype=torch.int32, device=DEV)
    for b in range(w.B):
        for h in range(w.Hkv):
            assert torch.equal(idx[b, h], want)
    assert torch.all(sc[..., : w.N] == sc[0, 0, 0])
    torch.testing.assert_close(out, torch.ones_like(out), atol=1e-6, rtol=0)


def test_all_ties_candidate_path():
    """All scores equal with the unit's keys within the candidate capacity:
    the threshold bin holds every key and the ties are ranked by index."""
    w = wl.Workload(name="ties_small", B=1, Hq=4, Hkv=2, N=3000, L=5, P=8, tau=0.3, k=333, seed=7010)
    inp = wl.make_inputs(w, DEV)
    inp["q"].zero_()
    inp["V"].fill_(1.0)
    ids, vnorm = gpu_hash(inp, w)
    idx, out, sc = gpu_decode(inp, w, ids, vnorm)
    want = torch.arange(w.k, dtype=torch.int32, device=DEV)
    for b in range(w.B):
        for h in range(w.Hkv):
            assert torch.equal(idx[b, h], want)


def test_all_ties_above_candidate_capacity():
    """All scores equal with more keys than the candidate list holds: the
    last top-k CTA of each unit selects over all of the unit's scores and
    compacts from them -- still keys 0..k-1."""
    w = wl.Workload(name="ties_wide", B=1, Hq=2, Hkv=1, N=40000, L=4, P=8, tau=0.3, k=1000, seed=7012)
    inp = wl.make_inputs(w, DEV)
    inp["q"].zero_()
    inp["V"].fill_(1.0)
    ids, vnorm = gpu_hash(inp, w)
    idx, out, sc = gpu_decode(inp, w, ids, vnorm)
    assert torch.equal(idx[0, 0], torch.arange(w.k, dtype=torch.int32, device=DEV))
    torch.testing.assert_close(out, torch.ones_like(out), atol=1e-6, rtol=0)


def test_decode_in_a_cuda_graph_matches_direct_calls():
    """A decode captured in a CUDA graph (the kernels' dependent launches become
    graph edges) reproduces a direct call bit for bit."""
    w = SMALL["llama_32k"]
    inp = wl.make_inputs(w, DEV)
    ids, vnorm = gpu_hash(inp, w)
    ws, idx, out = sk.alloc_decode_buffers(w.B, w.Hq, w.Hkv, w.ncap, w.L, w.P, w.k, DEV)
    run = lambda: sk.socket_decode(inp["q"], inp["W"], ids, vnorm, inp["K"], inp["V"], w.N, w.tau, w.k, ws, idx, out)
    run()
    torch.cuda.synchronize()
    want_idx, want_out = idx.clone(), out.clone()
    idx.fill_(-1)
    out.fill_(float("nan"))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert sk.read_device_error(ws) == 0
    assert torch.equal(idx, want_idx)
    assert torch.equal(out.view(torch.int32), want_out.view(torch.int32))


def test_decode_is_deterministic():
    w = SMALL["ragged_multitile"]
    inp = wl.make_inputs(w, DEV)
    ids, vnorm = gpu_hash(inp, w)
    a = gpu_decode(inp, w, ids, vnorm)
    b = gpu_decode(inp, w, ids, vnorm)
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.int32) if x.dtype == torch.float32 else x,
                           y.view(torch.int32) if y.dtype == torch.float32 else y)


# ----------------------------------------------------------------------------
# full-size workloads, sampled units
# ----------------------------------------------------------------------------

def _full_size(w, sample_units):
    torch.cuda.empty_cache()
    inp = wl.make_inputs(w, DEV)
    ids, vnorm = gpu_hash(inp, w)
    torch.cuda.synchronize()
    orc_ids, orc_vn, margin = oracle_hash_units(inp, w, sample_units)
    g_ids = torch.stack([ids[u // w.Hkv, u % w.Hkv] for u in sample_units]).cpu().numpy()
    g_vn = torch.stack([vnorm[u // w.Hkv, u % w.Hkv] for u in sample_units]).cpu().numpy()
    check_hash(g_ids, g_vn, orc_ids, orc_vn, margin, 0, w.N)
    return inp, ids, vnorm, orc_ids, orc_vn.astype(np.float32)


def test_topk_slices_above_bitmap_capacity():
    """N above 16 x 65536: each top-k CTA's slice exceeds the bitmap, so the
    selection is written by the compaction pass over the scores."""
    w = wl.Workload(name="wide", B=1, Hq=4, Hkv=1, N=1_100_000, L=8, P=6, tau=0.5, k=512, seed=7011)
    inp, ids, vnorm, orc_ids, orc_vn32 = _full_size(w, [0])
    substitute_units(ids, vnorm, w, [0], orc_ids, orc_vn32)
    idx, out, sc = gpu_decode(inp, w, ids, vnorm)
    check_decode(inp, w, orc_ids, orc_vn32, [0], idx, out, sc)


def test_batch8_128k_sampled_units_and_needles():
    """Planted needles: on sampled units the kernels select exactly the needles
    the oracle selects (some needles genuinely rank below k in fp64: a needle
    planted for one query head competes with keys the group's other heads
    favour); over all 64 units, recall stays at or above 99 %."""
    w = wl.BATCH8_128K
    units = [0, 11, 27, 63]
    inp, ids, vnorm, orc_ids, orc_vn32 = _full_size(w, units)
    idx, _, _ = gpu_decode(inp, w, ids, vnorm)
    assert sk.socket_last_decode_path() == sk.SOCKET_STEP_SEPARATE  # 64 units: the four kernels
    needles = inp["needles"]
    found = sum(int(torch.isin(needles[b, h].to(torch.int32), idx[b, h]).sum())
                for b in range(w.B) for h in range(w.Hkv))
    recall = found / needles.numel()
    assert recall >= 0.99, recall
    substitute_units(ids, vnorm, w, units, orc_ids, orc_vn32)
    idx, out, sc = gpu_decode(inp, w, ids, vnorm)
    check_decode(inp, w, orc_ids, orc_vn32, units, idx, out, sc)
    for i, u in enumerate(units):
        b, h = divmod(u, w.Hkv)
        q_u = inp["q"][b, h * w.G:(h + 1) * w.G].cpu()
        o_idx = oracle.decode_unit(q_u, inp["W"].cpu(), w.L, w.P, w.tau, orc_ids[i], orc_vn32[i],
                                   inp["K"][b, h].cpu(), inp["V"][b, h].cpu(), w.N, w.k)[0]
        nd = needles[b, h].cpu().numpy()
        assert np.array_equal(np.isin(nd, idx[b, h].cpu().numpy()), np.isin(nd, o_idx)), u
    del inp
    torch.cuda.empty_cache()


def test_batch8_128k_per_head_sampled_units_and_needles():
    """One selection per query head at full size: sampled kv units checked
    head by head against the oracle, and every head finds all 16 of its own
    needles (cosine 0.9 to its query; no competition from the group's other
    heads, unlike the grouped selection)."""
    w = wl.BATCH8_128K
    units = [5, 40]
    inp, ids, vnorm, orc_ids, orc_vn32 = _full_size(w, units)
    idx, _, _ = gpu_decode(inp, w, ids, vnorm, per_head=True)
    needles, m = inp["needles"], w.needles_per_head
    found = sum(int(torch.isin(needles[b, kvh, g * m:(g + 1) * m].to(torch.int32), idx[b, kvh * w.G + g]).sum())
                for b in range(w.B) for kvh in range(w.Hkv) for g in range(w.G))
    assert found == needles.numel(), found / needles.numel()
    substitute_units(ids, vnorm, w, units, orc_ids, orc_vn32)
    idx, out, sc = gpu_decode(inp, w, ids, vnorm, per_head=True)
    check_decode(inp, w, orc_ids, orc_vn32, units, idx, out, sc, per_head=True)
    del inp
    torch.cuda.empty_cache()


def test_per_head_many_kv_units_sampled():
    """Per-head selection over enough kv units that the soft-table kernel
    takes eight tables per CTA (each CTA writes its kv unit's four heads'
    tables, two hyperplane rows per thread): sampled kv units, head by head,
    against the oracle."""
    w = wl.Workload(name="ph_many", B=80, Hq=4, Hkv=1, N=2100, L=32, P=8, tau=0.3, k=64, seed=7402)
    units = [0, 37, 79]
    inp, ids, vnorm, orc_ids, orc_vn32 = _full_size(w, units)
    substitute_units(ids, vnorm, w, units, orc_ids, orc_vn32)
    idx, out, sc = gpu_decode(inp, w, ids, vnorm, per_head=True)
    check_decode(inp, w, orc_ids, orc_vn32, units, idx, out, sc, per_head=True)


def test_million_token_sampled_units():
    w = wl.MILLION
    units = [2, 7]
    inp, ids, vnorm, orc_ids, orc_vn32 = _full_size(w, units)
    substitute_units(ids, vnorm, w, units, orc_ids, orc_vn32)
    idx, out, sc = gpu_decode(inp, w, ids, vnorm)
    check_decode(inp, w, orc_ids, orc_vn32, units, idx, out, sc)
    del inp
    torch.cuda.empty_cache()


def test_append_mix_sampled_units():
    """Prefill hash of 16384 keys, then 64 steps that each hash one appended
    key at offset N+t and decode over N+t+1 keys; then the temperature sweep."""
    w = wl.APPEND_MIX
    units = [0, 131, 255]
    torch.cuda.empty_cache()
    inp = wl.make_inputs(w, DEV)
    ids, vnorm = gpu_hash(inp, w)                      # keys [0, N)
    for t in range(w.appends):
        sk.socket_hash_keys(inp["K"], inp["V"], inp["W"], ids, vnorm, w.N + t, w.N + t + 1)
        gpu_decode(inp, w, ids, vnorm, N=w.N + t + 1, q=inp["q_steps"][t])
    sk.socket_hash_check()
    n_all = w.N + w.appends
    orc_ids, orc_vn, margin = oracle_hash_units(inp, w, units, 0, n_all)
    g_ids = torch.stack([ids[u // w.Hkv, u % w.Hkv] for u in units]).cpu().numpy()
    g_vn = torch.stack([vnorm[u // w.Hkv, u % w.Hkv] for u in units]).cpu().numpy()
    check_hash(g_ids, g_vn, orc_ids, orc_vn, margin, 0, n_all)
    orc_vn32 = orc_vn.astype(np.float32)
    substitute_units(ids, vnorm, w, units, orc_ids, orc_vn32)
    for t in (0, 31, 63):
        idx, out, sc = gpu_decode(inp, w, ids, vnorm, N=w.N + t + 1, q=inp["q_steps"][t])
        check_decode(inp, w, orc_ids, orc_vn32, units, idx, out, sc, N=w.N + t + 1, q=inp["q_steps"][t])
    for tau in w.tau_sweep:
        idx, out, sc = gpu_decode(inp, w, ids, vnorm, N=n_all, tau=tau, q=inp["q_steps"][-1])
        check_decode(inp, w, orc_ids, orc_vn32, units, idx, out, sc, N=n_all, tau=tau, q=inp["q_steps"][-1])
    del inp
    torch.cuda.empty_cache()
