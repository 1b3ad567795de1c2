"""The pins must catch plausible mistakes in the oracle.

Each case plants one mistake in a private copy of the oracle's C source (a
dropped term, a wrong sign or index, a wrong mask alignment, a wrong GQA map),
compiles it on the CPU, swaps it in, and checks that the pin suite fails.
The real oracle is restored afterwards.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
from tests import test_oracle as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "sdpa_oracle.c")

MUTATIONS = {
    "drop_scale": ("for (int j = 0; j < Sk; ++j) scores[j] *= a->scale;", ""),
    "strict_top_left": ("if (causal == 1) return j <= i;", "if (causal == 1) return j < i;"),
    "bottom_right_offset_sign": ("return j <= i + (Sk - Sq);", "return j <= i + (Sq - Sk);"),
    "gqa_modulo_map": ("const int hk = hq / group;\n    const double *qrow",
                       "const int hk = hq % a->Hkv;\n    const double *qrow"),
    "no_normalisation": ("for (int j = 0; j < Sk; ++j) scores[j] /= sum;", ""),
    "lse_without_max": ("*lse_out = mx + log(sum);", "*lse_out = log(sum);"),
    "reversed_v_rows": ("const double *vrow = vbase + (size_t)j * d;",
                        "const double *vrow = vbase + (size_t)(Sk - 1 - j) * d;"),
    "combine_drops_local_sum": ("const double w = ls * exp(part_m[r * ns + s] - M);",
                                "const double w = exp(part_m[r * ns + s] - M);"),
    "partials_not_local_max": ("const double p = exp(x[j] - mx);", "const double p = exp(x[j]);"),
    "bias_subtracted": ("for (int j = 0; j < Sk; ++j) scores[j] += brow[j];",
                        "for (int j = 0; j < Sk; ++j) scores[j] -= brow[j];"),
    "bias_scaled": ("for (int j = 0; j < Sk; ++j) scores[j] += brow[j];",
                    "for (int j = 0; j < Sk; ++j) scores[j] += a->scale * brow[j];"),
    "bias_broadcast_swapped": ("const int bb = a->bias_b == 1 ? 0 : b, bh = a->bias_h == 1 ? 0 : hq;",
                               "const int bb = a->bias_h == 1 ? 0 : b, bh = a->bias_b == 1 ? 0 : hq;"),
    "bias_row_index": ("* a->Sq + i) * (size_t)Sk;", "* a->Sq + (a->Sq - 1 - i)) * (size_t)Sk;"),
    "bwd_no_jacobian_mean": ("const double dx = pj * (dprob[j] - D);", "const double dx = pj * dprob[j];"),
    "bwd_dk_unscaled": ("dkrow[c] += a->scale * dx * qrow[c];", "dkrow[c] += dx * qrow[c];"),
    "bwd_dv_from_dx": ("dvrow[c] += pj * grow[c];", "dvrow[c] += dx * grow[c];"),
    "bwd_dq_from_v": ("dqrow[c] += a->scale * dx * krow[c];",
                      "dqrow[c] += a->scale * dx * vbase[(size_t)j * d + c];"),
}


def _pin_suite(mod):
    """Run the pins that need no pytest parametrisation machinery."""
    import json
    for case in json.load(open(pins.GOLDEN))["cases"]:
        pins.test_hand_worked_examples(mod, case)
    pins.test_brute_force_every_tiny_shape(mod)
    for causal in (0, 1, 2):
        pins.test_gqa_equals_explicit_expansion(mod, causal)
    for ns in (2, 3):
        for causal in (0, 2):
            pins.test_split_combine_equals_unsplit(mod, ns, causal)
    pins.test_split_with_masked_and_empty_splits(mod)
    pins.test_partials_are_locally_normalised(mod)
    for dims in ((1, 1), (2, 1), (1, 4), (2, 4)):
        pins.test_bias_brute_force_every_broadcast(mod, dims, 1)
    pins.test_bias_of_log_weights_with_zero_query_is_weighted_mean(mod)
    pins.test_bwd_matches_finite_differences(mod, 2, 2, 1, 4, 3, 2, 2)
    pins.test_bwd_single_key_closed_form(mod)
    pins.test_bwd_two_key_closed_form(mod)


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(tmp_path, monkeypatch, name):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-shared", "-fPIC", "-pthread", str(mutated),
                    "-o", str(so), "-lm"], check=True)
    monkeypatch.setattr(oracle, "_lib", oracle.bind(ctypes.CDLL(str(so))))
    with pytest.raises(AssertionError):
        _pin_suite(oracle)


def test_unmutated_oracle_passes_suite():
    oracle._lib = None
    _pin_suite(oracle)


# ------------------------------------------------- rotary + KV append (numpy)
# Each case plants one mistake in a private copy of the source of
# oracle.rope_append, executes it in a copy of the oracle module's namespace,
# and checks that the rotary pins fail.

ROPE_MUTATIONS = {
    "rotation_sign": ("out[i] = vec[i] * c - vec[i + half] * s", "out[i] = vec[i] * c + vec[i + half] * s"),
    "cos_sin_swapped": ("c, s = cos[pos, i], sin[pos, i]", "c, s = sin[pos, i], cos[pos, i]"),
    "position_ignores_past": ("pos = past[b] + s", "pos = s"),
    "k_from_v_slot": ("kc[b, h, pos] = rotate(row[(Hq + h) * d:(Hq + h + 1) * d], pos)",
                      "kc[b, h, pos] = rotate(row[(Hq + Hkv + h) * d:(Hq + Hkv + h + 1) * d], pos)"),
    "v_rotated": ("vc[b, h, pos] = row[(Hq + Hkv + h) * d:(Hq + Hkv + h + 1) * d]",
                  "vc[b, h, pos] = rotate(row[(Hq + Hkv + h) * d:(Hq + Hkv + h + 1) * d], pos)"),
    "adjacent_pairs": ("""            out[i] = vec[i] * c - vec[i + half] * s
            out[i + half] = vec[i + half] * c + vec[i] * s""",
                       """            out[2 * i] = vec[2 * i] * c - vec[2 * i + 1] * s
            out[2 * i + 1] = vec[2 * i + 1] * c + vec[2 * i] * s"""),
    "total_off_by_one": ("[p + S_new for p in past]", "[p + S_new - 1 for p in past]"),
}


def _rope_pin_suite(mod):
    pins.test_rope_relative_position_property(mod)
    pins.test_rope_append_positions_norms_and_untouched_rows(mod)
    pins.test_rope_quarter_turn_closed_form(mod)


@pytest.mark.parametrize("name", sorted(ROPE_MUTATIONS))
def test_rope_pins_catch_planted_mistake(name):
    import inspect
    import textwrap
    import types
    old, new = ROPE_MUTATIONS[name]
    src = textwrap.dedent(inspect.getsource(oracle.rope_append))
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    namespace = dict(vars(oracle))
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), namespace)
    with pytest.raises(AssertionError):
        _rope_pin_suite(types.SimpleNamespace(rope_append=namespace["rope_append"]))


def test_unmutated_rope_oracle_passes_suite():
    _rope_pin_suite(oracle)
