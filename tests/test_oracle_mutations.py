"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's C source (on the CPU,
in a temporary directory), builds it, binds it in place of the real oracle
library, and runs the pin tests that should notice: at least one of them must
fail.  The mistakes are the ones an implementation of the method could make:
a wrong chunk mean, W_L applied transposed, the query's own chunk among its
candidates, a group score from one head, bf16 rounding with ties away from
zero, ties between chunks broken the wrong way, the router's comparison reversed,
uniform fusion weights, the in-chunk softmax without its 1/sqrt(d), and in
the backward a dropped softmax term, a missing landmark share, a missing e
term and a sign error; in the selection variants a refiner without its
1/sqrt(d), without its residual or with W_k transposed, and a Quest score
that takes the smaller product, starts the channel minimum at 0 or reads one
head of the group.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_backward_pins as bw
from tests import test_oracle_pins as pins
from tests import test_oracle_variant_pins as vp

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "hsa_oracle.c")

MUTANTS = {
    "chunk mean over S-1 keys": (
        "for (int e = 0; e < d; ++e) mean[e] /= (double)S;",
        "for (int e = 0; e < d; ++e) mean[e] /= (double)(S - 1);",
        [pins.test_landmarks_identity_projection_is_chunk_mean]),
    "W_L applied transposed": (
        "acc += mean[e] * load(W, (size_t)e * d + f, dt);",
        "acc += mean[e] * load(W, (size_t)f * d + e, dt);",
        [pins.test_landmarks_projection_orientation]),
    "own chunk among the candidates": (
        "long long ncand = row_p[r] / S;",
        "long long ncand = row_p[r] / S + 1;",
        [pins.test_decode_position_sees_all_complete_chunks,
         lambda: pins.test_select_matches_exact_integer_brute_force(0.0)]),
    "group score from one head": (
        "                for (int h = j * G; h < (j + 1) * G; ++h) {\n                    double dot = 0.0;",
        "                for (int h = j * G; h < j * G + 1; ++h) {\n                    double dot = 0.0;",
        [pins.test_select_group_sum_decides]),
    "bf16 rounding ties away from zero": (
        "double r = nearbyint(x / ulp) * ulp;",
        "double r = round(x / ulp) * ulp;",
        [pins.test_round_bf16_ties_to_even]),
    "ties to the higher chunk": (
        "return (x->c > y->c) - (x->c < y->c);",
        "return (x->c < y->c) - (x->c > y->c);",
        [lambda: pins.test_select_matches_exact_integer_brute_force(0.0)]),
    "router comparison reversed": (
        "if (sk - sk1 < tau * fabs(sk)) ke = ncand < 2 * k ? ncand : 2 * k;",
        "if (sk - sk1 > tau * fabs(sk)) ke = ncand < 2 * k ? ncand : 2 * k;",
        [pins.test_router_threshold_hand_cases]),
    "uniform fusion weights": (
        "for (int i = 0; i < ke; ++i) { w[i] = exp(score[so + i] - m); z += w[i]; }",
        "for (int i = 0; i < ke; ++i) { w[i] = 1.0; z += w[i]; }",
        [pins.test_two_chunk_fusion_is_sigmoid_of_score_gap]),
    "no 1/sqrt(d) in the chunk softmax": (
        "a[u] = dot * scale;",
        "a[u] = dot;",
        [pins.test_attention_scale_closed_form_single_aligned_key]),
    "backward: weighted mean left out of ds": (
        "double ds = w[i] * (dw[i] - wdw);",
        "double ds = w[i] * dw[i];",
        [lambda: bw.test_backward_matches_central_finite_differences(2, 0.0, 1)]),
    "backward: landmark share of dK dropped": (
        "dm[x] = acc / (double)S;",
        "dm[x] = 0.0 * acc;",
        [lambda: bw.test_gradient_sums_closed_forms(0.0)]),
    "backward: e left out of dz": (
        "double dz = ai[u] * (gv - go) * scale;",
        "double dz = ai[u] * gv * scale;",
        [bw.test_single_slot_rows_match_sdpa_autograd]),
    "backward: sign of dL": (
        "dLc[x] += ds * load(Qr, qh + x, dt);",
        "dLc[x] -= ds * load(Qr, qh + x, dt);",
        [lambda: bw.test_backward_matches_central_finite_differences(2, 0.0, 1)]),
    "refiner: no 1/sqrt(d)": (
        "logit[u] = dot * scale;",
        "logit[u] = dot;",
        [lambda: vp.test_refiner_matches_sdpa(vp.torch.float32, 16, 8)]),
    "refiner: residual dropped": (
        "for (int f = 0; f < d; ++f) out[f] = l0[f] + acc[f];",
        "for (int f = 0; f < d; ++f) out[f] = acc[f];",
        [vp.test_refiner_without_value_path_is_the_plain_landmark]),
    "refiner: W_k transposed": (
        "s += load(K, row0 + u * rstride + e, dt) * load(Wk, (size_t)e * d + f, dt);",
        "s += load(K, row0 + u * rstride + e, dt) * load(Wk, (size_t)f * d + e, dt);",
        [lambda: vp.test_refiner_matches_sdpa(vp.torch.float32, 16, 8)]),
    "quest: smaller product taken": (
        "bound += hi > lo ? hi : lo;",
        "bound += hi < lo ? hi : lo;",
        [vp.test_quest_score_bounds_every_key]),
    "quest: channel minimum starts at 0": (
        "for (int e = 0; e < d; ++e) { out[e] = -INFINITY; out[d + e] = INFINITY; }",
        "for (int e = 0; e < d; ++e) { out[e] = -INFINITY; out[d + e] = 0.0; }",
        [vp.test_quest_summaries_are_channel_max_and_min]),
    "quest: one head of the group": (
        "                for (int h = j * G; h < (j + 1) * G; ++h) {\n                    double bound = 0.0;",
        "                for (int h = j * G; h < j * G + 1; ++h) {\n                    double bound = 0.0;",
        [lambda: vp.test_quest_score_is_exact_when_the_chunk_has_one_key_value("single_key")]),
}


def _build_mutant(tmp_path, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique: {old}"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", str(lib), str(path), "-lm"],
                   check=True)
    return oracle._bind(ctypes.CDLL(str(lib)))


@pytest.mark.parametrize("name", list(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path, monkeypatch):
    old, new, checks = MUTANTS[name]
    monkeypatch.setattr(oracle, "_lib", _build_mutant(tmp_path, old, new))
    caught = 0
    for check in checks:
        try:
            check()
        except AssertionError:
            caught += 1
    assert caught > 0, f"no pin notices the planted mistake: {name}"


def test_unmutated_oracle_passes_the_same_checks():
    """The same checks pass on the real oracle, so a failure above is the mutation's."""
    for _, _, checks in MUTANTS.values():
        for check in checks:
            check()
