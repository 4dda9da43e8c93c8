"""The oracle's pins reject plausible mistakes (CPU only).

Each case copies the C oracle source, plants one mistake (a dropped term, a
wrong sign, a wrong index or operand, a wrong order), builds the copy with gcc
in a temporary directory and runs the pins of test_oracle_pins.py against it:
at least one pin must fail. The product oracle is never modified.
"""
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "deltalog_oracle.c")

MUTATIONS = {
    # eager step
    "eager_drops_decay": ("row[j] = row[j] * avec[j];", "row[j] = row[j];"),
    "eager_wrong_sign": ("beta * (v[i] - u) : v[i];", "beta * (v[i] + u) : v[i];"),
    "eager_writes_q": ("row[j] = row[j] + coef * k[j];", "row[j] = row[j] + coef * q[j];"),
    "eager_output_reads_k": ("acc += row[j] * q[j];", "acc += row[j] * k[j];"),
    "head_decay_wrong_head": ("return a[(long)t * NH + h];", "return a[(long)t * NH];"),
    "channel_decay_reversed": ("return a[((long)t * NH + h) * dk + j];",
                               "return a[((long)t * NH + h) * dk + (dk - 1 - j)];"),
    # deferred read
    "read_drops_decay": ("x[j] = ai[j] * (x[j] - s[i] * ki[j]);", "x[j] = (x[j] - s[i] * ki[j]);"),
    "read_wrong_order": ("for (int i = lg->n - 1; i >= 0; --i) {", "for (int i = 0; i < lg->n; ++i) {"),
    "read_value_weight": ("acc += s[i] * lg->v[(long)i * dv + r];",
                          "acc += lg->beta[i] * lg->v[(long)i * dv + r];"),
    # merge
    "merge_drops_base_decay": ("newrow[c] = row[c] * gn[c];", "newrow[c] = row[c];"),
    "merge_wrong_sign": ("u += C[i * (n + 1) + j] * delta[j];", "u -= C[i * (n + 1) + j] * delta[j];"),
    "merge_read_undecayed": ("G += row[c] * gi[c] * ki[c];", "G += row[c] * ki[c];"),
    "merge_write_undecayed": ("newrow[c] += delta[j] * kj[c] * dnj[c];", "newrow[c] += delta[j] * kj[c];"),
    "merge_decay_product": ("cur[c] = prev[c] * ai[c];", "cur[c] = prev[c];"),
    "no_final_flush": ("        deferred_merge(Sbar, &lg);\n        free(s);", "        free(s);"),
    # RWKV6
    "rwkv6_scales_value_by_beta": ("beta * (v[i] - u) : v[i];", "beta * (v[i] - u) : beta * v[i];"),
    "rwkv6_eager_corrects": ("double coef = delta ?", "double coef = 1 ?"),
    "rwkv6_read_subtracts": ("x[j] = ai[j] * x[j];", "x[j] = ai[j] * (x[j] - s[i] * ki[j]);"),
    "rwkv6_read_drops_decay": ("x[j] = ai[j] * x[j];", "x[j] = x[j];"),
    "rwkv6_merge_decays_own_value": ("delta[i] = lg->v[(long)(i - 1) * dv + r];",
                                     "delta[i] = lg->v[(long)(i - 1) * dv + r] * lg->a[(long)(i - 1) * dk];"),
    # int8 base
    "i8_rounds_half_away": ("code = nearbyintf((float)row[c] / scale);", "code = roundf((float)row[c] / scale);"),
    "i8_scale_128": ("const float scale = m / 127.0f;", "const float scale = m / 128.0f;"),
    "i8_decided_in_fp64": ("code = nearbyintf((float)row[c] / scale);", "code = (float)nearbyint(row[c] / scale);"),
    "i8_start_unrounded": ("        quantize_rows_i8(Sbar, dv, dk);\n        for (int t = 0; t < T; ++t) {",
                           "        for (int t = 0; t < T; ++t) {"),
    "i8_no_rounding_at_merges": ("                deferred_merge(Sbar, &lg);\n                quantize_rows_i8(Sbar, dv, dk);",
                                 "                deferred_merge(Sbar, &lg);"),
}

CHECKS = {
    "p0": lambda impl: [pins.run_golden(f, impl) for f in ("eager", "deferred1", "deferred2", "deferred3")],
    "p1": pins.check_p1,
    "p2": pins.check_p2,
    "p3": pins.check_p3,
    "p4": pins.check_p4,
    "p5": pins.check_p5,
    "p6": pins.check_p6,
    "p7": pins.check_p7,
    "p9": pins.check_p9,
    "p10": pins.check_p10,
    "p12": pins.check_p12,
}


def build_mutant(tmp_path, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique/present: {old!r}"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-std=c99", "-O1", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
                    "-w", "-o", str(so), str(path), "-lm"], check=True)
    return oracle.CLib(str(so))


def test_clean_oracle_passes_every_pin(oracle_mod):
    impl = oracle._load()
    for name, check in CHECKS.items():
        check(impl)


@pytest.mark.parametrize("mutation", sorted(MUTATIONS))
def test_planted_mistake_fails_a_pin(mutation, tmp_path):
    old, new = MUTATIONS[mutation]
    impl = build_mutant(tmp_path, old, new)
    caught = []
    for name, check in CHECKS.items():
        try:
            check(impl)
        except AssertionError:
            caught.append(name)
    assert caught, f"no pin rejects the planted mistake {mutation}"
