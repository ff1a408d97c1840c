"""Plant plausible mistakes in a copy of the oracle (on the CPU) and check that the pins
catch every one of them.  Each mutant is the oracle source with one textual change,
compiled to a temporary shared object and swapped in for the duration of the check."""
import os
import subprocess
import tempfile

import pytest

import oracle
from oracle import build as oracle_build
from oracle import oracle as oracle_mod
from tests import test_oracle_pins as pins

MUTANTS = {
    "visible entries off by one": ("int64_t a = t - W + 1;", "int64_t a = t - W;"),
    "window one key too long": ("int64_t lo = t - W + 1 < 0 ? 0 : t - W + 1;", "int64_t lo = t - W < 0 ? 0 : t - W;"),
    "compressed segment dropped": ("for (int64_t j = 0; j < nc; ++j, ++n) {\n                    for (int64_t c = 0; c < d; ++c) keys[n * d + c] = bf(kc[",
                                   "for (int64_t j = 0; j < 0; ++j, ++n) {\n                    for (int64_t c = 0; c < d; ++c) keys[n * d + c] = bf(kc["),
    "softmax sign flipped": ("double p = exp(z[i] - m);", "double p = exp(m - z[i]);"),
    "pooling weights not normalised": ("for (int64_t i = 0; i < blk; ++i) alpha[i] /= s;", ""),
    "pooling block offset": ("int64_t pos = blk * j + i;", "int64_t pos = blk * j + i + (i + 1 < blk);"),
    "rms uses the sum": ("double inv = 1.0 / sqrt(ss / (double)d + eps);", "double inv = 1.0 / sqrt(ss + eps);"),
    "gate sign": ("o[c] *= 1.0 / (1.0 + exp(-bf(gate[", "o[c] *= 1.0 / (1.0 + exp(bf(gate["),
    "lse misses the max": ("if (lse) *lse = m + log(l);", "if (lse) *lse = log(l);"),
    "paged offset": ("row = pg * page_size + j % page_size;", "row = pg * page_size + (j + 1) % page_size;"),
    "window slot shifted": ("if (L - W + i < 0) continue;", "if (L - W + i <= 0) continue;"),
    "kv head of group 0": ("keys[n * d + c] = bf(k[((b * T + u) * Hkv + g) * d + c]);",
                           "keys[n * d + c] = bf(k[((b * T + u) * Hkv + 0) * d + c]);"),
    "query not normalised": ("if (gq) rmsnorm(qv, d, gq, eps);", ""),
    "scale dropped": ("z[i] = scale * s;", "z[i] = s;"),
}

CHECKS = [
    pins.test_compress_zero_weights_is_mean,
    pins.test_compress_cache_ratio_and_partial_tail_unused,
    pins.test_compress_two_row_closed_form,
    pins.test_compress_matches_numpy_pooling,
    pins.test_compress_dominant_weight_selects_row,
    pins.test_window_covers_everything_is_full_causal_attention,
    lambda: pins.test_block_one_zero_weights_is_full_causal_attention(3),
    lambda: pins.test_matches_dense_bruteforce(300, 40, 16, 4, 2),
    pins.test_hand_worked_example,
    lambda: pins.test_decode_equals_last_prefill_row(700, 256),
    pins.test_paged_equals_contiguous,
    pins.test_qk_norm_scale_invariance,
    pins.test_qk_norm_two_key_closed_form,
    pins.test_gate_limits,
    pins.test_decode_lse_matches_bruteforce,
]


def _caught(lib):
    saved = oracle_mod._lib
    oracle_mod._lib = lib
    try:
        for check in CHECKS:
            try:
                check()
            except (AssertionError, ValueError):
                return True
        return False
    finally:
        oracle_mod._lib = saved


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name):
    src = open(oracle_build.SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, "mutation anchor not found: " + name
    with tempfile.TemporaryDirectory() as tmp:
        c = os.path.join(tmp, "mutant.c")
        so = os.path.join(tmp, "mutant.so")
        with open(c, "w") as f:
            f.write(src.replace(old, new))
        subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", c, "-o", so, "-lm"], check=True)
        lib = oracle_mod._bind(so)
        assert _caught(lib), "no pin caught the planted mistake: " + name


def test_unmutated_oracle_passes_all_checks():
    assert not _caught(oracle_mod._load())


# ---- the backward oracle (oracle/backward.py, numpy): same idea, one textual change per
# mutant, the mutated module swapped in for the backward pins

BACKWARD_MUTANTS = {
    "dS misses rowsum(dO*O)": ("ds = p * (dp - (do * o).sum(axis=1, keepdims=True))", "ds = p * dp"),
    "pooling path of dK dropped": ("return dq, dk_raw + dk_pool, dv_raw + dv_pool, dw",
                                   "return dq, dk_raw, dv_raw + dv_pool, dw"),
    "weight softmax Jacobian dropped": ("dwb = a * (dal - (a * dal).sum(axis=2, keepdims=True))", "dwb = a * dal"),
    "entry boundary moved by one": ("n_c = np.maximum(0, (t - W + 1) // blk)", "n_c = np.maximum(0, (t - W + 2) // blk)"),
    "dq without the scale": ("dq[b, :, h] = scale * (ds @ keys)", "dq[b, :, h] = ds @ keys"),
    "gradient to the wrong kv head": ("            g = h * Hkv // Hq\n            keys, vals = _keys(k, v, kc, vc, b, g)",
                                      "            g = h % Hkv\n            keys, vals = _keys(k, v, kc, vc, b, g)"),
    "dV from dS": ("dvals = p.T @ do", "dvals = ds.T @ do"),
}


def _backward_checks(tb):
    return [
        lambda: tb.test_backward_matches_finite_differences(11, 2, 1, 2, 3),
        lambda: tb.test_backward_matches_finite_differences(13, 4, 2, 3, 4),
        tb.test_pool_backward_matches_finite_differences,
        lambda: tb.test_one_token_blocks_are_causal_attention(4, 2),
        tb.test_window_covering_the_sequence_is_causal_attention,
        tb.test_weight_gradients_sum_to_zero_per_block,
        tb.test_value_gradients_sum_to_output_gradients,
        tb.test_query_with_only_itself_has_zero_gradient,
        tb.test_dense_forward_matches_c_oracle,
    ]


def _backward_caught(module):
    from tests import test_oracle_backward as tb
    saved = tb.ob
    tb.ob = module
    try:
        for check in _backward_checks(tb):
            try:
                check()
            except AssertionError:
                return True
        return False
    finally:
        tb.ob = saved


@pytest.mark.parametrize("name", sorted(BACKWARD_MUTANTS))
def test_backward_pins_catch_mutant(name):
    import types
    from oracle import backward
    src = open(backward.__file__).read()
    old, new = BACKWARD_MUTANTS[name]
    assert src.count(old) == 1, "mutation anchor not found: " + name
    mutant = types.ModuleType("backward_mutant")
    exec(compile(src.replace(old, new), "backward_mutant.py", "exec"), mutant.__dict__)
    assert _backward_caught(mutant), "no pin caught the planted mistake: " + name


def test_unmutated_backward_passes_all_checks():
    from oracle import backward
    assert not _backward_caught(backward)


# ---- the VHA oracle (numpy): the function's source with one change, swapped in for its pins

VHA_MUTANTS = {
    "identity skip dropped": ('return o + np.einsum("hk,nkc->nhc", U, t)', 'return np.einsum("hk,nkc->nhc", U, t)'),
    "factors swapped": ('t = np.einsum("hk,nhc->nkc", V, o)', 't = np.einsum("hk,nhc->nkc", U, o)'),
    "mixing matrix transposed": ('t = np.einsum("hk,nhc->nkc", V, o)\n    return o + np.einsum("hk,nkc->nhc", U, t)',
                                 't = np.einsum("hk,nhc->nkc", U, o)\n    return o + np.einsum("hk,nkc->nhc", V, t)'),
}


def _vha_caught(fn):
    saved = oracle.vha
    oracle.vha = fn
    try:
        for check in (pins.test_vha_zero_factor_is_identity, pins.test_vha_rank_one_closed_form,
                      pins.test_vha_factor_gauge_invariance, pins.test_vha_equals_dense_mixing_matrix):
            try:
                check()
            except AssertionError:
                return True
        return False
    finally:
        oracle.vha = saved


@pytest.mark.parametrize("name", sorted(VHA_MUTANTS))
def test_vha_pins_catch_mutant(name):
    import inspect
    import textwrap
    import numpy as np
    src = textwrap.dedent(inspect.getsource(oracle_mod.vha))
    old, new = VHA_MUTANTS[name]
    assert src.count(old) == 1, "mutation anchor not found: " + name
    ns = {"np": np}
    exec(compile(src.replace(old, new), "vha_mutant.py", "exec"), ns)
    assert _vha_caught(ns["vha"]), "no pin caught the planted mistake: " + name


def test_unmutated_vha_passes_all_checks():
    assert not _vha_caught(oracle_mod.vha)
