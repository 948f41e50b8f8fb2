"""Plant plausible mistakes in a copy of the oracle (on the CPU) and check
that the pins catch every one of them."""

import os
import shutil

import pytest

import oracle
import _oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

# (name, exact text in oracle.c, replacement)
MUTANTS = [
    ("drop_scale", "s[j] = J->scale * dot;", "s[j] = dot;"),
    ("causal_off_by_one", "if (J->causal && (long)j > (long)i", "if (J->causal && (long)j >= (long)i"),
    ("causal_top_left", "(long)i + (long)J->Nk - (long)J->Nq", "(long)i"),
    ("gqa_modulo", "const int hk = hq / group;", "const int hk = hq % J->Hkv;"),
    ("no_max_in_lse", "*lse_out = m + log(l);", "*lse_out = log(l);"),
    ("no_division", "orow[c] /= l;", "orow[c] /= 1.0;"),
    ("v_from_k", "const uint16_t *vrow = J->v +", "const uint16_t *vrow = J->k +"),
    ("max_not_subtracted_in_weights", "s[j] = exp(s[j] - m);", "s[j] = exp(s[j] - m * 0.5);"),
    ("ignore_key_range", "if (j < J->k_begin || j >= J->k_end)", "if (0)"),
    ("q_row_index", "(((size_t)b * J->Nq + i) * J->Hq + hq) * d;", "(((size_t)b * J->Nq + ri) * J->Hq + hq) * d;"),
    ("window_left_off_by_one", "(long)j < g - (long)J->window_left", "(long)j <= g - (long)J->window_left"),
    ("window_right_ignored", "if (J->window_right >= 0 && (long)j > g + (long)J->window_right)", "if (0)"),
    ("window_from_row_index", "const long g = (long)J->Nk - (long)J->Nq + (long)i;", "const long g = (long)i;"),
    ("drop_one_key_term", "for (int c = 0; c < d; ++c)\n            dot += qd[c]", "for (int c = 1; c < d; ++c)\n            dot += qd[c]"),
]


# mistakes in the backward pass, caught by the backward pins
BWD_MUTANTS = [
    ("bwd_dq_without_scale", "dqrow[c] += J->scale * ds * bf16_to_double(krow[c]);",
     "dqrow[c] += ds * bf16_to_double(krow[c]);"),
    ("bwd_ds_without_row_term", "const double ds = p[j] * (dp[j] - pdp);", "const double ds = p[j] * dp[j];"),
    ("bwd_dk_from_k", "dkrow[c] += J->scale * ds * bf16_to_double(qrow[c]);",
     "dkrow[c] += J->scale * ds * bf16_to_double(krow[c]);"),
    ("bwd_dv_unnormalised", "                p[j] /= l;\n", "                p[j] /= 1.0;\n"),
    ("bwd_dv_uses_ds", "dvrow[c] += p[j] * bf16_to_double(gorow[c]);", "dvrow[c] += dp[j] * bf16_to_double(gorow[c]);"),
    ("bwd_dp_from_q", "g += bf16_to_double(gorow[c]) * bf16_to_double(vj[c]);",
     "g += bf16_to_double(gorow[c]) * bf16_to_double(qrow[c]);"),
    ("bwd_one_head_per_group", "for (int hq = hk * group; hq < (hk + 1) * group; ++hq) {",
     "for (int hq = hk * group; hq < hk * group + 1; ++hq) {"),
]


def _mutant_fails_some_pin(tmp_path, name, old, new, pin_list):
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation site for {name} not found exactly once"
    src = tmp_path / "oracle_mut.c"
    src.write_text(text.replace(old, new))
    so = oracle.build(force=True, src=str(src), out=str(tmp_path / "liboracle_mut.so"))
    orc = oracle.Oracle(so)
    failed = []
    for pin in pin_list:
        try:
            pin(orc)
        except AssertionError:
            failed.append(pin.__name__)
    return failed


@pytest.mark.parametrize("name,old,new", BWD_MUTANTS, ids=[m[0] for m in BWD_MUTANTS])
def test_backward_pins_catch_mutant(tmp_path, name, old, new):
    assert _mutant_fails_some_pin(tmp_path, name, old, new, pins.BWD_PINS), \
        f"mutant {name} passed every backward pin"


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, old, new):
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation site for {name} not found exactly once"
    src = tmp_path / "oracle_mut.c"
    src.write_text(text.replace(old, new))
    so = oracle.build(force=True, src=str(src), out=str(tmp_path / "liboracle_mut.so"))
    orc = oracle.Oracle(so)
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"
