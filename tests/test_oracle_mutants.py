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
from tests import test_oracle_bwd_pins as bwd

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
    # backward
    "bwd_drops_row_term": [("const double ds = p[a] * (dp[a] - D);", "const double ds = p[a] * dp[a];")],
    "bwd_dk_from_keys": [("dkb[c * d + x] += scale * ds * qr[x];",
                          "dkb[c * d + x] += scale * ds * kb[c * d + x];")],
    "bwd_dv_from_ds": [("dvb[c * d + x] += p[a] * dor[x];", "dvb[c * d + x] += ds * dor[x];")],
    "bwd_dq_unscaled": [("dqr[x] += scale * ds * kb[c * d + x];", "dqr[x] += ds * kb[c * d + x];")],
    "bwd_skipped_tiles_get_gradient": [("if (st[j] != 2)", "if (st[j] == 0)")],
    "bwd_causal_ignored": [("if (c < len && !(causal && c > t))", "if (c < len)")],
    "bwd_unnormalised_p": [("p[a] /= z;", "(void)z;")],
    "bwd_group_by_modulo": [("for (int h = kvh * g; h < (kvh + 1) * g; ++h)",
                             "for (int h = kvh; h < Hq; h += Hkv)")],
    "bwd_padding_keys_kept": [("if (c < len && !(causal && c > t))", "if (c < N && !(causal && c > t))")],
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
    lambda: bwd.test_bwd_dense_equals_autograd(2, 4, 2, 200, 64, 64, True),
    bwd.test_bwd_blasst_equals_autograd_over_executed_tiles,
    lambda: bwd.test_bwd_central_differences_with_skips("k"),
    bwd.test_bwd_never_executed_keys_get_no_gradient,
    bwd.test_bwd_gqa_equals_group_sum_of_mha,
    lambda: bwd.test_bwd_varlen_equals_each_sequence_alone(False),
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
