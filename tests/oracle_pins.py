"""Pins that tie the oracle to facts other than itself.

Each ``pin_*`` function takes a loaded oracle library (``oracle.load()`` or a
deliberately broken build of it) and raises ``AssertionError`` when the
library disagrees with a closed form, an invariant of the method, a worked
example printed on the pages, a textbook identity, a library routine that
computes the same quantity another way, or brute force on tiny inputs.

Sources: the SOCKET summaries "Resumen Técnico: SOCKET - Estimador de Núcleo
de Colisión Suave para Atención Escasa" (gist.science/es/paper/2602.06283) and
"SOCKET: SOft Collision Kernel EsTimator for Sparse Attention"
(gist.science/de/paper/2602.06283).  Section names are given per pin.
"""
from __future__ import annotations

import itertools
import math
import os

import numpy as np
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _sigmoid(x):
    x = np.asarray(x, dtype=np.float64)
    return np.where(x >= 0, 1.0 / (1.0 + np.exp(-np.abs(x))), np.exp(-np.abs(x)) / (1.0 + np.exp(-np.abs(x))))


def _signs(P):
    """s[b, p] = +1 if bit p of b is set else -1."""
    b = np.arange(1 << P)[:, None]
    return np.where((b >> np.arange(P)[None, :]) & 1, 1.0, -1.0)


def _z(W, q):
    W = np.asarray(W, dtype=np.float64)
    q = np.asarray(q, dtype=np.float64)
    return W @ q / np.linalg.norm(q)


# ----------------------------------------------------------------------------
# step 2: soft assignment
# ----------------------------------------------------------------------------

def pin_probabilities_sum_to_one(lib):
    """A softmax over the 2^P buckets is a distribution (closed form: sum = 1)."""
    rng = np.random.default_rng(11)
    for P in (1, 4, 8):
        for tau in (1.0, 0.5, 0.3, 0.2, 0.1, 0.01, 1e-3):
            W = rng.standard_normal((3, P, 24))
            q = rng.standard_normal(24)
            p = oracle.soft_assign(q, W, 3, P, tau, lib=lib)
            assert np.all(p >= 0.0)
            assert np.max(np.abs(p.sum(axis=1) - 1.0)) < 1e-12, (P, tau)


def pin_factorised_product_of_sigmoids(lib):
    """The softmax over sign patterns factorises: exp(s z/t) / (exp(z/t) + exp(-z/t))
    = sigmoid(2 s z / t) per plane, so p(b) = prod_p sigmoid(2 s_bp z_p / t).
    Algebraic identity; the oracle evaluates the unfactorised softmax."""
    rng = np.random.default_rng(12)
    for P in (2, 4, 8):
        for tau in (1.0, 0.5, 0.3):
            W = rng.standard_normal((2, P, 16))
            q = rng.standard_normal(16)
            z = _z(W, q)                                     # [L, P]
            s = _signs(P)                                    # [2^P, P]
            want = np.prod(_sigmoid(2.0 * s[None, :, :] * z[:, None, :] / tau), axis=-1)
            got = oracle.soft_assign(q, W, 2, P, tau, lib=lib)
            assert np.allclose(got, want, rtol=1e-11, atol=1e-300), (P, tau)


def pin_basis_planes_closed_form(lib):
    """With unit hyperplanes e_0, e_1 and q = (3, 4): z = (0.6, 0.8), and with
    tau = 1 the four buckets get sigmoid(+-1.2) * sigmoid(+-1.6), bucket b
    taking the + sign of plane p when bit p of b is set (bit 0 <-> plane 0)."""
    W = np.zeros((1, 2, 4))
    W[0, 0, 0] = 1.0
    W[0, 1, 1] = 1.0
    q = np.array([3.0, 4.0, 0.0, 0.0])
    sg = lambda x: 1.0 / (1.0 + math.exp(-x))
    want = [sg(-1.2) * sg(-1.6), sg(1.2) * sg(-1.6), sg(-1.2) * sg(1.6), sg(1.2) * sg(1.6)]
    got = oracle.soft_assign(q, W, 1, 2, 1.0, lib=lib)[0]
    assert np.allclose(got, want, rtol=1e-13, atol=0), got


def pin_golden_lay_example(lib):
    """The 70 % / 30 % bucket example of the German page's lay explanation, and
    its hard limit (fixture tests/golden/lay_example_p1.txt)."""
    W = np.array([[[1.0, 0.0]]])
    with open(os.path.join(GOLDEN, "lay_example_p1.txt")) as f:
        rows = [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]
    assert rows
    for tau, q0, q1, p0, p1, tol in rows:
        p = oracle.soft_assign(np.array([float(q0), float(q1)]), W, 1, 1, float(tau), lib=lib)[0]
        assert abs(p[0] - float(p0)) <= float(tol) and abs(p[1] - float(p1)) <= float(tol), (tau, p)


def pin_hard_limit_theorem3(lib):
    """Theorem 3 ("Fundamento Teórico" / "Theoretische Grundlage"): the
    soft-bucketing bias vanishes as tau -> 0.  Per table, the deviation from
    the one-hot of the query's own hard bucket is bounded by the union bound
    sum_p sigmoid(-2 |z_p| / tau), and it shrinks as tau falls.  The hard
    bucket comes from hashing q as if it were a key."""
    rng = np.random.default_rng(13)
    L, P, d = 8, 8, 16
    W = rng.standard_normal((L, P, d))
    q = rng.standard_normal(d)
    z = _z(W, q)
    hard = oracle.hash_keys(q[None, :], q[None, :], W, L, P, lib=lib)[0][:, 0]
    onehot = np.zeros((L, 1 << P))
    onehot[np.arange(L), hard] = 1.0
    last = np.inf
    for tau in (1.0, 0.1, 0.01, 1e-3):
        p = oracle.soft_assign(q, W, L, P, tau, lib=lib)
        dev = np.max(np.abs(p - onehot), axis=1)
        bound = np.sum(_sigmoid(-2.0 * np.abs(z) / tau), axis=1)
        assert np.all(dev <= bound + 1e-12), (tau, dev, bound)
        assert dev.max() <= last + 1e-15
        last = dev.max()
    clear = np.min(np.abs(z), axis=1) >= 0.02      # tables with no plane near the query
    assert clear.sum() >= 4 and np.all(dev[clear] < 1e-8)


def pin_small_signal_lemma4(lib):
    """Lemma 4: for small signals (large tau) the soft score is linear in the
    projected coordinates: p(b) = 2^-P (1 + <s_b, z> / tau) + O(tau^-2).  The
    residual must fall by ~4x each time tau doubles."""
    rng = np.random.default_rng(14)
    L, P, d = 2, 8, 16
    W = rng.standard_normal((L, P, d))
    q = rng.standard_normal(d)
    z = _z(W, q)
    s = _signs(P)
    res = []
    for tau in (20.0, 40.0, 80.0, 160.0):
        lin = (1.0 + (z @ s.T) / tau) / (1 << P)             # [L, 2^P]
        res.append(np.max(np.abs(oracle.soft_assign(q, W, L, P, tau, lib=lib) - lin)))
    for a, b in zip(res, res[1:]):
        assert 3.5 <= a / b <= 4.5, res


# ----------------------------------------------------------------------------
# step 1: hashing
# ----------------------------------------------------------------------------

def pin_hash_unit_planes(lib):
    """With hyperplane (l, p) equal to the unit vector e_{c(l,p)}, the bucket
    id is sum_p [k_{c(l,p)} > 0] 2^p, the margin is min |k_c| / ||k||.  Every
    (l, p) uses a different channel, so a swapped table/plane index, a flipped
    sign or a reversed bit order all change the ids."""
    rng = np.random.default_rng(15)
    L, P, d = 3, 5, 32
    chan = rng.permutation(d)[: L * P].reshape(L, P)
    W = np.zeros((L, P, d))
    for l in range(L):
        for p in range(P):
            W[l, p, chan[l, p]] = 1.0
    K = rng.standard_normal((40, d))
    V = rng.standard_normal((40, d))
    ids, vnorm, margin = oracle.hash_keys(K, V, W, L, P, lib=lib)
    for l in range(L):
        want = sum(((K[:, chan[l, p]] > 0).astype(np.int64) << p) for p in range(P))
        assert np.array_equal(ids[l].astype(np.int64), want), l
    want_margin = np.min(np.abs(K[:, chan.ravel()]), axis=1) / np.linalg.norm(K, axis=1)
    assert np.allclose(margin, want_margin, rtol=1e-14)


def pin_hash_symmetries(lib):
    """Sign-random-projection symmetries: id(-k) = (2^P - 1) - id(k) and
    id(c k) = id(k) for c > 0; value norms: ||(3, 4, 0, ...)|| = 5,
    ||(1, ..., 1)|| = sqrt(d), and ||c v|| = |c| ||v||."""
    rng = np.random.default_rng(16)
    L, P, d = 4, 8, 16
    W = rng.standard_normal((L, P, d))
    K = rng.standard_normal((64, d))
    V = np.zeros((64, d))
    V[:, 0], V[:, 1] = 3.0, 4.0
    V[32:] = 1.0
    V[48:] *= -2.5
    ids, vn, _ = oracle.hash_keys(K, V, W, L, P, lib=lib)
    ids_neg, _, _ = oracle.hash_keys(-K, V, W, L, P, lib=lib)
    ids_scaled, _, _ = oracle.hash_keys(3.7 * K, V, W, L, P, lib=lib)
    assert np.array_equal(ids_neg.astype(int), (1 << P) - 1 - ids.astype(int))
    assert np.array_equal(ids_scaled, ids)
    assert np.allclose(vn[:32], 5.0, rtol=1e-15)
    assert np.allclose(vn[32:48], math.sqrt(d), rtol=1e-15)
    assert np.allclose(vn[48:], 2.5 * math.sqrt(d), rtol=1e-15)


def pin_angular_collision_rate(lib):
    """Random-hyperplane hashing (SimHash): two vectors at angle theta share a
    sign on one Gaussian plane with probability 1 - theta/pi, so they share a
    P-plane bucket with probability (1 - theta/pi)^P -- the angular kernel the
    pages say SOCKET's scores approximate ("Fundamento Teórico").  Checked
    over 50000 independent tables within a 4-sigma binomial band."""
    rng = np.random.default_rng(17)
    d, M = 8, 50000
    for P in (4, 8):
        W = rng.standard_normal((M, P, d))
        for theta in (0.3, 0.8, 1.5):
            q = np.zeros(d)
            q[0] = 1.0
            k = np.zeros(d)
            k[0], k[1] = math.cos(theta), math.sin(theta)
            X = np.stack([q, k])
            ids, _, _ = oracle.hash_keys(X, X, W, M, P, lib=lib)
            rate = np.mean(ids[:, 0] == ids[:, 1])
            e = (1.0 - theta / math.pi) ** P
            assert abs(rate - e) <= 4.0 * math.sqrt(e * (1 - e) / M), (P, theta, rate, e)


# ----------------------------------------------------------------------------
# step 3: scoring (through the full unit decode, so the wiring is pinned too)
# ----------------------------------------------------------------------------

def _unit_case(rng, G, n, d, L, P):
    W = rng.standard_normal((L, P, d))
    q = rng.standard_normal((G, d))
    K = rng.standard_normal((n, d))
    V = rng.standard_normal((n, d)) * rng.uniform(0.2, 3.0, size=(n, 1))
    return W, q, K, V


def pin_score_hard_collision_count(lib):
    """As tau -> 0 the score becomes ||v|| times the hard-LSH collision count
    (Theorem 3 limit); checked with one head, within ||v|| times the summed
    per-table union bounds."""
    rng = np.random.default_rng(18)
    L, P, d, n = 6, 8, 16, 200
    W, q, K, V = _unit_case(rng, 1, n, d, L, P)
    ids, vn, _ = oracle.hash_keys(K, V, W, L, P, lib=lib)
    vn32 = vn.astype(np.float32)
    hard = oracle.hash_keys(q, q, W, L, P, lib=lib)[0][:, 0]
    count = np.sum(ids == hard[:, None], axis=0)
    tau = 1e-3
    bound = np.sum(_sigmoid(-2.0 * np.abs(_z(W, q[0])) / tau))
    _, _, sc, _ = oracle.decode_unit(q, W, L, P, tau, ids, vn32, K, V, n, 5, lib=lib)
    want = vn32.astype(np.float64) * count
    assert np.all(np.abs(sc - want) <= vn32 * bound + 1e-12)
    assert count.max() >= 1


def pin_hard_mode_is_collision_count(lib):
    """tau = 0, hard LSH ([ES] "Enunciado del Problema": binary collision
    signals; [DE] "Der alte Weg (Harte LSH)"): each head's query is hashed like
    a key, p is one-hot on that bucket, and the score is ||v|| times the number
    of (head, table) pairs where key and query collide -- counted here by brute
    force from the hash of the keys and of the queries."""
    rng = np.random.default_rng(19)
    L, P, d, n, G = 7, 5, 16, 300, 3
    W, q, K, V = _unit_case(rng, G, n, d, L, P)
    ids, vn, _ = oracle.hash_keys(K, V, W, L, P, lib=lib)
    vn32 = vn.astype(np.float32)
    qids = oracle.hash_keys(q, q, W, L, P, lib=lib)[0]            # [L, G]
    for h in range(G):
        prob = oracle.soft_assign(q[h], W, L, P, 0.0, lib=lib)
        want = np.zeros_like(prob)
        want[np.arange(L), qids[:, h]] = 1.0
        assert np.array_equal(prob, want)
    count = sum(np.sum(ids == qids[:, h][:, None], axis=0) for h in range(G))
    _, _, sc, _ = oracle.decode_unit(q, W, L, P, 0.0, ids, vn32, K, V, n, 5, lib=lib)
    assert np.array_equal(sc, vn32.astype(np.float64) * count)
    assert count.max() >= 1


def pin_score_heads_add(lib):
    """Grouped heads share one selection and their scores add: the score of a
    2-head group equals the sum of each head's score alone."""
    rng = np.random.default_rng(19)
    L, P, d, n = 5, 6, 16, 300
    W, q, K, V = _unit_case(rng, 2, n, d, L, P)
    ids, vn, _ = oracle.hash_keys(K, V, W, L, P, lib=lib)
    vn32 = vn.astype(np.float32)
    tau = 0.7
    s2 = oracle.decode_unit(q, W, L, P, tau, ids, vn32, K, V, n, 3, lib=lib)[2]
    s0 = oracle.decode_unit(q[:1], W, L, P, tau, ids, vn32, K, V, n, 3, lib=lib)[2]
    s1 = oracle.decode_unit(q[1:], W, L, P, tau, ids, vn32, K, V, n, 3, lib=lib)[2]
    assert np.allclose(s2, s0 + s1, rtol=1e-13)
    assert not np.allclose(s0, s1)


def pin_per_head_selection(lib):
    """One selection per query head: head g's scores split the grouped score
    by head (they add up to it), its k keys are the k largest of its own
    scores with ties to the lower index (a stable sort here), and its output
    is softmax attention over them (numpy, fp64)."""
    rng = np.random.default_rng(21)
    L, P, d, n, G, U, k = 6, 5, 16, 257, 3, 2, 9
    W = rng.standard_normal((L, P, d))
    q = rng.standard_normal((U, G, d))
    K = rng.standard_normal((U, n, d))
    V = rng.standard_normal((U, n, d))
    hashed = [oracle.hash_keys(K[u], V[u], W, L, P, lib=lib) for u in range(U)]
    ids = np.stack([h[0] for h in hashed])
    vn32 = np.stack([h[1].astype(np.float32) for h in hashed])
    tau = 0.4
    idx, out, sc = oracle.decode_per_head(q, W, L, P, tau, ids, vn32, K, V, n, k, lib=lib)
    _, _, gsc = oracle.decode(q, W, L, P, tau, ids, vn32, K, V, n, k, lib=lib)
    assert np.allclose(sc.sum(axis=1), gsc, rtol=1e-13)
    for u in range(U):
        for g in range(G):
            order = np.argsort(-sc[u, g], kind="stable")
            assert np.array_equal(idx[u, g], np.sort(order[:k]))
            sel = idx[u, g]
            logits = K[u, sel] @ q[u, g] / np.sqrt(d)
            w = np.exp(logits - logits.max())
            w /= w.sum()
            assert np.allclose(out[u, g], w @ V[u, sel], rtol=1e-12, atol=1e-13)
    assert any(not np.array_equal(idx[u, 0], idx[u, g]) for u in range(U) for g in range(1, G))


def pin_score_uniform_query(lib):
    """A zero query puts probability 2^-P on every bucket, so every key scores
    G * L * 2^-P * ||v|| whatever its bucket ids."""
    rng = np.random.default_rng(20)
    L, P, d, n, G = 7, 4, 16, 50, 3
    W, _, K, V = _unit_case(rng, G, n, d, L, P)
    q = np.zeros((G, d))
    ids, vn, _ = oracle.hash_keys(K, V, W, L, P, lib=lib)
    vn32 = vn.astype(np.float32)
    sc = oracle.decode_unit(q, W, L, P, 0.3, ids, vn32, K, V, n, 4, lib=lib)[2]
    assert np.allclose(sc, G * L * vn32.astype(np.float64) / (1 << P), rtol=1e-14)


# ----------------------------------------------------------------------------
# step 4: selection
# ----------------------------------------------------------------------------

def pin_topk_brute_force(lib):
    """Deterministic top-k ("Selección" / "Auswahl"), ties to the lower index:
    equals, on tiny inputs with many ties, the brute-force choice among all
    k-subsets of the one with the largest score sum, and among those the
    lexicographically smallest sorted index tuple."""
    rng = np.random.default_rng(21)
    for _ in range(40):
        n = int(rng.integers(1, 9))
        s = rng.integers(0, 3, n).astype(np.float64)
        for k in range(1, n + 1):
            best = max(itertools.combinations(range(n), k),
                       key=lambda c: (sum(s[list(c)]), tuple(-i for i in c)))
            got = oracle.topk(s, k, lib=lib)
            assert list(got) == list(best), (s, k, got, best)


def pin_topk_against_lexsort(lib):
    """On 5000 scores with planted ties, the selection equals numpy's stable
    lexicographic sort by (score descending, index ascending)."""
    rng = np.random.default_rng(22)
    s = np.round(rng.standard_normal(5000), 2)
    for k in (1, 17, 999, 5000):
        want = np.sort(np.lexsort((np.arange(s.size), -s))[:k])
        assert np.array_equal(oracle.topk(s, k, lib=lib), want), k


# ----------------------------------------------------------------------------
# step 4: exact attention over the subset
# ----------------------------------------------------------------------------

def pin_attention_small_subsets(lib):
    """One selected key: the output is that key's value row.  Two keys a, b:
    weight sigmoid((q.K_a - q.K_b)/sqrt(d)) on V_a, the rest on V_b."""
    rng = np.random.default_rng(23)
    n, d, G = 50, 16, 3
    q = rng.standard_normal((G, d))
    K = rng.standard_normal((n, d))
    V = rng.standard_normal((n, d))
    out = oracle.attention(q, K, V, np.array([7], dtype=np.int32), lib=lib)
    assert np.array_equal(out, np.repeat(V[7][None], G, axis=0))
    out = oracle.attention(q, K, V, np.array([3, 11], dtype=np.int32), lib=lib)
    wa = 1.0 / (1.0 + np.exp(-(q @ K[3] - q @ K[11]) / math.sqrt(d)))
    want = wa[:, None] * V[3][None] + (1 - wa)[:, None] * V[11][None]
    assert np.allclose(out, want, rtol=1e-13, atol=1e-15)


def pin_full_selection_is_dense_attention(lib):
    """With k = n the method attends over every key, so a unit decode equals
    dense softmax attention (torch scaled_dot_product_attention in fp64)."""
    rng = np.random.default_rng(24)
    L, P, d, n, G = 4, 8, 32, 120, 4
    W, q, K, V = _unit_case(rng, G, n, d, L, P)
    ids, vn, _ = oracle.hash_keys(K, V, W, L, P, lib=lib)
    _, out, _, _ = oracle.decode_unit(q, W, L, P, 0.3, ids, vn.astype(np.float32), K, V, n, n, lib=lib)
    qt = torch.from_numpy(q)[None, :, None, :]                       # [1, G, 1, d]
    Kt = torch.from_numpy(K)[None, None].expand(1, G, n, d)
    Vt = torch.from_numpy(V)[None, None].expand(1, G, n, d)
    want = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt)[0, :, 0].numpy()
    assert np.allclose(out, want, rtol=1e-12, atol=1e-13)


def pin_batched_decode_matches_units(lib):
    """The batched entry point runs the same per-unit computation for every
    (batch, kv-head) unit, on the right slices of every input."""
    rng = np.random.default_rng(25)
    U, G, L, P, d, ncap, n, k = 3, 2, 4, 6, 16, 48, 45, 9
    W = rng.standard_normal((L, P, d))
    q = rng.standard_normal((U, G, d))
    K = rng.standard_normal((U, ncap, d))
    V = rng.standard_normal((U, ncap, d))
    ids = rng.integers(0, 1 << P, size=(U, L, ncap), dtype=np.uint8)
    vn = rng.uniform(0.5, 2.0, size=(U, ncap)).astype(np.float32)
    idx, out, sc = oracle.decode(q, W, L, P, 0.4, ids, vn, K, V, n, k, lib=lib)
    for u in range(U):
        i1, o1, s1, _ = oracle.decode_unit(q[u], W, L, P, 0.4, ids[u], vn[u], K[u], V[u], n, k, lib=lib)
        assert np.array_equal(idx[u], i1) and np.array_equal(out[u], o1) and np.array_equal(sc[u], s1)


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_") and callable(v)]
