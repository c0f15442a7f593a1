"""Plant plausible mistakes in copies of the oracle and check the pins notice.

Each mutant is a one-site textual change to ``oracle/socket_oracle.c`` (a
flipped sign, a dropped term, a swapped index, a reversed order).  Every
mutant is compiled into its own library and must fail at least one pin; the
untouched source must pass them all.  Mistakes are only ever planted in the
oracle, on the CPU.
"""
import os

import pytest

import oracle
from oracle_pins import ALL_PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "socket_oracle.c")

MUTANTS = {
    "hash_sign_flipped": ("if (y > 0.0) id |= 1u << p;", "if (y < 0.0) id |= 1u << p;"),
    "hash_bit_order_reversed": ("if (y > 0.0) id |= 1u << p;", "if (y > 0.0) id |= 1u << (P - 1 - p);"),
    "hash_table_plane_swapped": ("const double* w = W + ((int64_t)l * P + p) * d;\n                double y = 0.0;\n                for (int j = 0; j < d; ++j) y += w[j] * load_elem(K",
                                 "const double* w = W + ((int64_t)p * L + l) * d;\n                double y = 0.0;\n                for (int j = 0; j < d; ++j) y += w[j] * load_elem(K"),
    "vnorm_without_sqrt": ("vnorm[i] = sqrt(vv);", "vnorm[i] = vv;"),
    "soft_sign_pattern_flipped": ("(((b >> p) & 1) ? 1.0 : -1.0)", "(((b >> p) & 1) ? -1.0 : 1.0)"),
    "soft_missing_temperature": ("logit[b] = s / tau;", "logit[b] = s;"),
    "soft_temperature_doubled": ("logit[b] = s / tau;", "logit[b] = s / (2.0 * tau);"),
    "soft_query_not_normalised": ("z[p] = qnorm > 0.0 ? y / qnorm : 0.0;", "z[p] = y;"),
    "score_without_value_norm": ("s += (double)vnorm[i] * mass;", "s += mass;"),
    "score_first_head_only": ("for (int h = 0; h < G; ++h) {\n            double mass", "for (int h = 0; h < 1; ++h) {\n            double mass"),
    "topk_ties_to_higher_index": ("return (x->index > y->index) - (x->index < y->index);", "return (x->index < y->index) - (x->index > y->index);"),
    "topk_smallest_scores": ("if (x->score > y->score) return -1;\n    if (x->score < y->score) return 1;",
                             "if (x->score > y->score) return 1;\n    if (x->score < y->score) return -1;"),
    "attention_unscaled_logits": ("const double scale = 1.0 / sqrt((double)d);", "const double scale = 1.0;"),
    "attention_unnormalised_weights": ("double w = exp(logit[i] - mx) / total;", "double w = exp(logit[i] - mx);"),
    "attention_values_from_keys": ("out[(int64_t)h * d + j] += w * load_elem(V,", "out[(int64_t)h * d + j] += w * load_elem(K,"),
    "decode_every_head_uses_head0": ("oracle_soft_assign((const char*)q + (size_t)h * d", "oracle_soft_assign((const char*)q + (size_t)0 * d"),
    "hard_query_sign_flipped": ("if (y > 0.0) hb |= 1 << p;", "if (y < 0.0) hb |= 1 << p;"),
    "hard_bit_order_reversed": ("if (y > 0.0) hb |= 1 << p;", "if (y > 0.0) hb |= 1 << (P - 1 - p);"),
    "hard_mass_off_the_bucket": ("prob[(int64_t)l * nb + b] = b == hb ? 1.0 : 0.0;", "prob[(int64_t)l * nb + b] = b == hb ? 0.0 : 1.0;"),
}


def _failures(lib):
    failed = []
    for pin in ALL_PINS:
        try:
            pin(lib)
        except AssertionError:
            failed.append(pin.__name__)
    return failed


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    so = oracle.compile_oracle(str(path), str(tmp_path / f"lib_{name}.so"))
    assert _failures(oracle.load(so)), f"no pin caught mutant {name}"


def test_unmutated_passes_every_pin():
    assert _failures(oracle.load()) == []


def test_per_head_pin_catches_heads_on_the_wrong_kv_unit(monkeypatch):
    """The per-head decode is a composition in Python; plant the plausible
    mistake there (units repeated as a tile, so head g of unit u reads another
    unit's keys) and check its pin notices."""
    import numpy as np

    import oracle_pins

    def mutant(q, W, L, P, tau, ids, vnorm_f32, K, V, n, k, want_scores=True, lib=None):
        qs = np.asarray(q)
        U, G, d = qs.shape
        rep = lambda a: np.tile(np.asarray(a), (G,) + (1,) * (np.asarray(a).ndim - 1))
        idx, out, sc = oracle.decode(qs.reshape(U * G, 1, d), W, L, P, tau, rep(ids), rep(vnorm_f32), rep(K),
                                     rep(V), n, k, want_scores=want_scores, lib=lib)
        return idx.reshape(U, G, k), out.reshape(U, G, d), (sc.reshape(U, G, n) if sc is not None else None)

    lib = oracle.load()
    oracle_pins.pin_per_head_selection(lib)
    monkeypatch.setattr(oracle, "decode_per_head", mutant)
    with pytest.raises(AssertionError):
        oracle_pins.pin_per_head_selection(lib)
