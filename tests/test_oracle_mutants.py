"""Planted mistakes: each mutant of the oracle's C source (one plausible slip:
a dropped term, a wrong sign or index, a transposed operand) is compiled on the
CPU and must fail at least one of the pins.  This checks that the pins, not
just the oracle, are strong enough."""
import ctypes
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins
from tests import test_golden as golden

SRC = os.path.join(os.path.dirname(oracle.__file__), "bsattn_oracle.c")

MUTANTS = {
    "no_scale": [("acc *= scale;", "acc *= 1.0;")],
    "gqa_mod_instead_of_div": [("const int kvh = h / g;", "const int kvh = h % Hkv;")],
    "causal_off_by_one": [("(causal && key > qpos[r])", "(causal && key >= qpos[r])")],
    "any_row_instead_of_all": [("double dmax = -INFINITY;", "double dmax = INFINITY;"),
                               ("if (dr > dmax)", "if (dr < dmax)")],
    "skip_sign_flipped": [("skip = dmax < ln_lambda;", "skip = dmax > ln_lambda;")],
    "no_normalisation": [("out[(size_t)r * d + x] /= z[r];", "(void)0;")],
    "split_never_resets": [("starts[t] = (t % chunk) == 0;", "starts[t] = t == 0;")],
    "k_used_as_v": [("const uint16_t *vrow = vbase + (k0 + c) * d;",
                     "const uint16_t *vrow = kbase + (k0 + c) * d;")],
    "lse_without_log_sum": [("lse[r] = mprev[r] + log(z[r]);", "lse[r] = mprev[r];")],
    "index_causal_off_by_one": [("> (int64_t)(i + 1) * q_block - 1)", "> (int64_t)(i + 1) * q_block)")],
    "mask_ignored": [("if (mask && !mask[((int64_t)mh * nq + i) * nk + j])", "if (0)")],
    "running_max_not_updated": [("if (mt > mprev[r])\n                mprev[r] = mt;", "(void)mt;")],
    "reverse_ignored": [("        if (reverse)\n", "        if (0)\n")],
    "seed_ignored": [("if (seed_tile >= 0 && tiles[t] != seed_tile)", "if (0)")],
    "seed_from_split_first_tile": [("SCORE_TILE(seed_tile);", "SCORE_TILE(tiles[t]);")],
    "padding_keys_not_masked": [("query_tile(qrows, qpos, nrows, kb, vb, len, d,",
                                 "query_tile(qrows, qpos, nrows, kb, vb, N, d,")],
    "decode_splits_cut_full_cache": [("const int chunk = Tp > 0 ? (Tp + num_splits - 1) / num_splits : 1;",
                                      "const int chunk = (T + num_splits - 1) / num_splits;")],
}

CHECKS = [
    lambda: pins.test_lambda0_all_ones_equals_dense(2, 4, 2, 200, 64, 64, True),
    pins.test_static_mask_equals_brute_force_element_mask,
    pins.test_static_mask_causal_per_head_mask_gqa,
    pins.test_closed_form_skip,
    pins.test_closed_form_keep,
    pins.test_closed_form_one_row_disagrees_keeps_tile,
    pins.test_closed_form_order_matters,
    pins.test_closed_form_reverse_order,
    pins.test_decode_sink_seed_closed_form,
    lambda: pins.test_varlen_prefill_equals_each_sequence_alone(False, True, 1e-2),
    pins.test_varlen_decode_equals_each_cache_alone,
    pins.test_decode_split_resets_running_max,
    pins.test_decode_gqa_group_vote,
    pins.test_index_matches_definition_and_causal,
    golden.test_causal_dense_count,
]


def _build_mutant(tmp_path, name, edits):
    src = open(SRC).read()
    for old, new in edits:
        assert src.count(old) == 1, f"{name}: pattern {old!r} not unique"
        src = src.replace(old, new)
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"{name}.so"
    c.write_text(src)
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c11", str(c),
                           "-o", str(so), "-lm"])
    return oracle.bind(ctypes.CDLL(str(so)))


def test_unmutated_oracle_passes_checks():
    for chk in CHECKS:
        chk()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path, monkeypatch):
    lib = _build_mutant(tmp_path, name, MUTANTS[name])
    monkeypatch.setattr(oracle, "_lib", lib)
    caught = []
    for chk in CHECKS:
        try:
            chk()
        except (AssertionError, oracle.OracleError):
            caught.append(chk)
    assert caught, f"mutant {name} passed every pin"
