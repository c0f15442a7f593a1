"""socket_decode_static, the decode entry point that allocates nothing.

It serves callers that cannot call cudaMalloc and get no scratch from anyone
(for example code embedded in a serving runtime that has reserved the GPU's
memory for its own pool).  It runs the same kernels as socket_decode on the
same inputs, only with its scratch in a fixed device array, so its results
must equal socket_decode's bit for bit, on consecutive calls that share that
scratch; it must not allocate device memory; and it must refuse sizes that
do not fit the scratch.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import pytest
import torch

import soft_lsh_top_b200 as sk
import workloads as wl
from soft_lsh_top_b200 import _build

EWORKSPACE = 4


def test_static_decode_rejects_sizes_beyond_its_scratch():
    """Sizes whose workspace exceeds the static scratch are refused before any
    device work (the pointers below are never dereferenced)."""
    lib = sk.load_library(_build.build())
    fake = 0x10000
    B, Hq, Hkv, Ncap, d, L, P, k = 64, 32, 8, 1 << 20, 128, 32, 8, 2048
    assert lib.socket_decode_workspace_size(B, Hq, Hkv, Ncap, d, L, P, k) > (64 << 20)
    st = lib.socket_decode_static(fake, 1, fake, fake, fake, fake, fake, 1, B, Hq, Hkv, Ncap, Ncap, d, L, P, 0.3, k,
                                  fake, fake, None, None)
    assert st == EWORKSPACE
    assert "static scratch" in lib.socket_last_error().decode()


def _bits(t):
    return t.view(torch.int32) if t.dtype == torch.float32 else t


@pytest.mark.gpu
def test_static_decode_matches_workspace_decode_on_consecutive_calls():
    dev = torch.device("cuda:0")
    w = wl.LLAMA_32K.scaled(name="no_alloc", B=2, Hq=8, Hkv=2, N=40001, L=24, k=900, seed=9101)
    inp = wl.make_inputs(w, dev)
    ids, vnorm = sk.alloc_cache_index(w.B, w.Hkv, w.ncap, w.L, dev)
    sk.socket_hash_keys(inp["K"], inp["V"], inp["W"], ids, vnorm, 0, w.N)
    ws, _, _ = sk.alloc_decode_buffers(w.B, w.Hq, w.Hkv, w.ncap, w.L, w.P, w.k, dev)
    queries = [inp["q"], torch.randn(inp["q"].shape, generator=torch.Generator(dev).manual_seed(5),
                                     device=dev).to(inp["q"].dtype)]
    results = []
    for q in queries:
        ref_idx = torch.empty(w.B, w.Hkv, w.k, dtype=torch.int32, device=dev)
        ref_out = torch.empty(w.B, w.Hq, 128, dtype=torch.float32, device=dev)
        ref_sc = torch.empty(w.B, w.Hkv, w.ncap, dtype=torch.float32, device=dev)
        sk.socket_decode(q, inp["W"], ids, vnorm, inp["K"], inp["V"], w.N, w.tau, w.k, ws, ref_idx, ref_out,
                         scores_out=ref_sc)
        out_bufs = (torch.full_like(ref_idx, -1), torch.full_like(ref_out, float("nan")),
                    torch.full_like(ref_sc, float("nan")))
        results.append(((ref_idx, ref_out, ref_sc), out_bufs))
    torch.cuda.synchronize()

    # The first call on the device looks up the scratch's address (and may
    # load the module that holds it); measure memory from after that call on.
    _, (idx0, out0, sc0) = results[0]
    sk.socket_decode_static(queries[0], inp["W"], ids, vnorm, inp["K"], inp["V"], w.N, w.tau, w.k, idx0, out0,
                            scores_out=sc0)
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info(dev)
    torch_before = torch.cuda.memory_allocated(dev)
    for q, (_, (idx, out, sc)) in zip(queries, results):
        # two calls in a row; the second sees the first call's leftover scratch
        idx.fill_(-1)
        out.fill_(float("nan"))
        sc.fill_(float("nan"))
        sk.socket_decode_static(q, inp["W"], ids, vnorm, inp["K"], inp["V"], w.N, w.tau, w.k, idx, out,
                                scores_out=sc)
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info(dev)
    assert free_after == free_before, (free_before, free_after)
    assert torch.cuda.memory_allocated(dev) == torch_before
    for (ref_idx, ref_out, ref_sc), (idx, out, sc) in results:
        # the same kernels on the same inputs: bit-identical results
        assert torch.equal(idx, ref_idx)
        assert torch.equal(_bits(sc[..., : w.N]), _bits(ref_sc[..., : w.N]))
        assert torch.equal(_bits(out), _bits(ref_out))
