"""The seeded input recipe (workloads.py), checked on CPU at reduced sizes.

The full-size workloads share these generators; here each stated property is
checked on a small copy of the workload.  The properties: determinism per
seed, a cache capacity rounded to 32, outlier channels, lognormal value norms,
planted needles at the stated cosine, the mean drift per block, and one query
per append step.
"""
import math

import pytest
import torch

import workloads as wl


def small(w, **kw):
    base = dict(B=2, N=4096, seed=w.seed)
    base.update(kw)
    return w.scaled(**base)


def test_same_seed_same_tensors_and_rows_restrict_without_changing_values():
    w = small(wl.BATCH8_128K, B=3, N=600)
    a = wl.make_inputs(w)
    b = wl.make_inputs(w)
    for key in ("W", "q", "K", "V", "needles"):
        assert torch.equal(a[key], b[key]), key
    part = wl.make_inputs(w, batches=[1])
    assert torch.equal(part["K"][0], a["K"][1])
    assert torch.equal(part["V"][0], a["V"][1])
    other = wl.make_inputs(w.scaled(seed=w.seed + 1))
    assert not torch.equal(other["K"], a["K"])


@pytest.mark.parametrize("N, appends, ncap", [(4096, 0, 4096), (4097, 0, 4128), (16384, 64, 16448), (70001, 0, 70016)])
def test_cache_capacity_rounds_up_to_32(N, appends, ncap):
    w = wl.TINY.scaled(N=N, appends=appends)
    assert w.ncap == ncap and w.ncap % 32 == 0


def test_shapes_and_dtypes():
    for w in (small(wl.LLAMA_32K, N=256), small(wl.TINY, N=256)):
        x = wl.make_inputs(w)
        assert x["W"].shape == (w.L, w.P, w.d) and x["W"].dtype == torch.bfloat16
        assert x["q"].shape == (w.B, w.Hq, w.d) and x["q"].dtype == w.torch_dtype
        assert x["K"].shape == (w.B, w.Hkv, w.ncap, w.d) and x["K"].dtype == w.torch_dtype
        assert x["V"].shape == x["K"].shape


def test_outlier_channels_are_scaled():
    w = small(wl.LLAMA_32K, N=8192, needles_per_head=0, value_lognormal_sigma=0.0)
    x = wl.make_inputs(w)
    K = x["K"].float()
    std = K.reshape(-1, w.d).std(dim=0)
    ch = list(w.outlier_channels)
    rest = [c for c in range(w.d) if c not in ch]
    ratio = std[ch].mean() / std[rest].mean()
    assert abs(ratio - w.outlier_scale) < 0.05 * w.outlier_scale


def test_value_rows_carry_a_lognormal_factor():
    w = small(wl.LLAMA_32K, N=16384, outlier_channels=(), needles_per_head=0)
    x = wl.make_inputs(w)
    norms = x["V"].float().norm(dim=-1).reshape(-1)
    # ||v|| = e^(sigma g) * chi_128: log ||v|| has variance sigma^2 + var(log chi_128).
    var_chi = 1.0 / (2 * w.d)  # var(log chi_d) ~ 1 / (2d) for large d
    var = torch.log(norms).var().item()
    assert abs(var - (w.value_lognormal_sigma ** 2 + var_chi)) < 0.02


def test_needles_sit_at_the_stated_cosine_to_their_query_head():
    w = small(wl.BATCH8_128K, N=4096)
    x = wl.make_inputs(w)
    m = w.needles_per_head
    q = x["q"].float()
    for b in range(w.B):
        for kvh in range(w.Hkv):
            where = x["needles"][b, kvh]
            assert where.numel() == w.G * m and len(set(where.tolist())) == w.G * m
            keys = x["K"][b, kvh, where].float()
            heads = kvh * w.G + torch.arange(w.G * m) // m
            cos = torch.nn.functional.cosine_similarity(keys, q[b, heads], dim=-1)
            # bf16 storage of the key moves the cosine by well under 1e-2
            assert torch.all((cos - w.needle_cosine).abs() < 1e-2), cos


def test_drift_shifts_the_mean_by_the_stated_step_per_block():
    w = wl.MILLION.scaled(B=1, Hq=4, Hkv=1, N=3 * 4096, drift_block=4096, needles_per_head=0,
                          value_lognormal_sigma=0.0, outlier_channels=())
    x = wl.make_inputs(w)
    K = x["K"][0, 0].float()
    means = [K[i * 4096:(i + 1) * 4096].mean().item() for i in range(3)]
    for i in range(3):
        assert abs(means[i] - w.drift_per_block * i) < 0.01, means


def test_one_query_per_append_step():
    w = small(wl.APPEND_MIX, N=512)
    x = wl.make_inputs(w)
    assert x["q_steps"].shape == (w.appends, w.B, w.Hq, w.d)
    assert w.ncap >= w.N + w.appends


def test_step_bytes_counts_ids_norms_and_gathered_rows():
    w = wl.BATCH8_128K
    assert w.step_bytes() == w.U * (w.N * w.L + 4 * w.N + 2 * w.k * w.d * 2)
    assert w.step_bytes() == 369_098_752
    assert math.isclose(w.U * w.N * (w.L + 4), 301_989_888)
