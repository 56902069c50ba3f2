"""Planted mistakes in the oracle (on the CPU): each mutated copy must fail a pin.

A copy of the oracle source gets one plausible slip (a flipped sign, a
transposed operand, reversed conv taps, a dropped term or clamp, the read
placed before the write), is compiled to a temporary library, and the pins of
``test_oracle_pins`` are run against it.  At least one pin has to fail for
every mutation; otherwise the pins would not be constraining that part.
"""

import os
import subprocess
import tempfile

import pytest

from oracle import oracle
from tests import test_golden as golden
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "kda_oracle.c")

MUTATIONS = {
    "delta_sign": ("dl[j] = (vt[j] - p[j]) * beta", "dl[j] = (p[j] - vt[j]) * beta"),
    "delta_sign_rec": ("dl[j] = (vt[j] - p[j]) * bt", "dl[j] = (p[j] - vt[j]) * bt"),
    "predict_transposed": ("acc += kt[i] * S[i * D + j];", "acc += kt[i] * S[j * D + i];"),
    "read_transposed": ("acc += qt[i] * S[i * D + j];", "acc += qt[i] * S[j * D + i];"),
    "conv_taps_reversed": ("J->conv_w[c * KCONV + j] *", "J->conv_w[c * KCONV + (KCONV - 1 - j)] *"),
    "no_lower_bound": ("gt[i] = g < J->lower_bound ? J->lower_bound : g;", "gt[i] = g;"),
    "no_dt_bias": (" + J->dt_bias[h * D + i];", ";"),
    "no_silu": ("dst[i] = silu(acc);", "dst[i] = acc;"),
    "write_without_k": ("S[i * D + j] += kt[i] * dl[j];", "S[i * D + j] += dl[j];"),
    "decay_exp_of_neg": ("double e = exp(gt[i]);", "double e = exp(-gt[i]);"),
    "eps_outside_root": ("1.0 / sqrt(sq + J->eps)", "1.0 / (sqrt(sq) + J->eps)"),
    "conv_history_shift": ("raw_at(J, n, t - (KCONV - 1) + j, c)", "raw_at(J, n, t - KCONV + j, c)"),
    "beta_not_sigmoid": ("const double beta = (J->beta2 ? 2.0 : 1.0) * sigmoid(J->b[row * H + h]);",
                         "const double beta = (J->beta2 ? 2.0 : 1.0) * J->b[row * H + h];"),
    "beta2_ignored": ("(J->beta2 ? 2.0 : 1.0) * sigmoid", "1.0 * sigmoid"),
    "beta2_squared": ("(J->beta2 ? 2.0 : 1.0) * sigmoid", "(J->beta2 ? 4.0 : 1.0) * sigmoid"),
    "onorm_sum_not_mean": ("sqrt(ms / (double)D + J->oeps)", "sqrt(ms + J->oeps)"),
    "onorm_eps_outside_root": ("1.0 / sqrt(ms / (double)D + J->oeps)", "1.0 / (sqrt(ms / (double)D) + J->oeps)"),
    "onorm_no_weight": ("ot[j] * r * J->onw[j] * sigmoid", "ot[j] * r * sigmoid"),
    "ogate_not_sigmoid": ("* sigmoid(J->ogate[(row * H + h) * D + j])", "* exp(J->ogate[(row * H + h) * D + j])"),
    "ogate_channel_shift": ("J->ogate[(row * H + h) * D + j]", "J->ogate[(row * H + h) * D + (j + 1) % D]"),
}


def _order_mutations(ind: str, out_lhs: str, beta: str):
    """The loop's order changed: the output read before the write, or the prediction taken
    before the decay (``ind``: the loop body's indentation; the forward pass and the
    recurrence entry spell the output store and beta differently)."""
    decay = (ind + "for (int64_t i = 0; i < D; ++i) {\n" + ind + "    double e = exp(gt[i]);\n" + ind +
             "    for (int64_t j = 0; j < D; ++j) S[i * D + j] *= e;\n" + ind + "}\n")
    predict = (ind + "for (int64_t j = 0; j < D; ++j) {\n" + ind + "    double acc = 0.0;\n" + ind +
               "    for (int64_t i = 0; i < D; ++i) acc += kt[i] * S[i * D + j];\n" + ind +
               "    p[j] = acc;\n" + ind + "}\n")
    write = (ind + "for (int64_t i = 0; i < D; ++i)\n" + ind +
             "    for (int64_t j = 0; j < D; ++j) S[i * D + j] += kt[i] * dl[j];\n")
    read = (ind + "for (int64_t j = 0; j < D; ++j) {\n" + ind + "    double acc = 0.0;\n" + ind +
            "    for (int64_t i = 0; i < D; ++i) acc += qt[i] * S[i * D + j];\n" + ind +
            "    " + out_lhs + "\n" + ind + "}\n")
    correct = ind + "for (int64_t j = 0; j < D; ++j) dl[j] = (vt[j] - p[j]) * " + beta + ";\n"
    return (decay + predict + correct, predict + decay + correct), (write + read, read + write)


_fw = _order_mutations(" " * 8, "ot[j] = J->scale * acc;", "beta")
_rc = _order_mutations(" " * 16, "o[(row * H + h) * D + j] = scale * acc;", "bt")
MUTATIONS["predict_before_decay"] = _fw[0]   # (_fw[1] does not apply: see below)
MUTATIONS["predict_before_decay_rec"] = _rc[0]
MUTATIONS["read_before_write_rec"] = _rc[1]
# in the forward pass the output pointer is declared between the write and the read
_WRITE = ("        for (int64_t i = 0; i < D; ++i)\n"
          "            for (int64_t j = 0; j < D; ++j) S[i * D + j] += kt[i] * dl[j];\n")
_READ = ("        double *ot = J->o + (row * H + h) * D;\n"
         "        for (int64_t j = 0; j < D; ++j) {\n"
         "            double acc = 0.0;\n"
         "            for (int64_t i = 0; i < D; ++i) acc += qt[i] * S[i * D + j];\n"
         "            ot[j] = J->scale * acc;\n"
         "        }\n")
MUTATIONS["read_before_write"] = (_WRITE + _READ, _READ + _WRITE)


PIN_TESTS = [
    lambda: [pins.test_recurrence_matches_unrolled_product(T, D, s)
             for T, D, s in [(1, 2, 0), (3, 3, 1), (8, 4, 2)]],
    pins.test_delta_rule_retrieval_identity,
    pins.test_beta_zero_only_decays,
    pins.test_prologue_matches_torch_conv1d_and_scipy,
    pins.test_gate_closed_forms,
    pins.test_lower_bound_decay_closed_form,
    pins.test_forward_equals_prologue_then_recurrence,
    lambda: [pins.test_prefill_then_decode_equals_long_prefill(a, b) for a, b in [(7, 5), (1, 4)]],
    pins.test_negative_eigenvalues_beta_is_twice_sigmoid,
    pins.test_negative_eigenvalues_write_is_a_householder_reflection,
    pins.test_negative_eigenvalues_equal_plain_run_with_rescaled_b,
    pins.test_output_gate_unit_rms_and_direction,
    pins.test_output_gate_is_a_sigmoid,
    pins.test_output_gate_acts_channel_by_channel,
    pins.test_output_gate_weight_is_per_channel,
    pins.test_output_gate_eps_inside_the_mean_square,
    golden.test_hand_worked_recurrence,
    golden.test_gate_and_beta_closed_forms,
]


def _build_mutant(old, new, tmpdir):
    src = open(SRC).read()
    assert old in src, "mutation anchor not found: %r" % old
    path_c = os.path.join(tmpdir, "mut.c")
    path_so = os.path.join(tmpdir, "libmut.so")
    open(path_c, "w").write(src.replace(old, new))
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                           "-o", path_so, path_c, "-lm"])
    return path_so


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name):
    old, new = MUTATIONS[name]
    with tempfile.TemporaryDirectory() as d:
        so = _build_mutant(old, new, d)
        prev = oracle.swap_library(so)
        caught = []
        try:
            for pin in PIN_TESTS:
                try:
                    pin()
                except AssertionError:
                    caught.append(pin)
        finally:
            oracle.swap_library(None)
            oracle._lib = prev
    assert caught, "no pin failed for planted mistake %r" % name
