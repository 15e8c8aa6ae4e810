"""The oracle's pins must catch plausible mistakes.

Each case copies ``oracle/sfa_oracle.c`` to a temporary directory, plants one
mistake by a textual substitution, compiles the copy and runs the pin suite
against it in a child process.  The suite must fail for every mutant.  The
committed oracle is never modified.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "sfa_oracle.c")

MUTANTS = {
    "score_scale_1_over_d": [("1.0 / sqrt((double)d)", "1.0 / (double)d")],
    "window_one_too_long": [("(t - K + 1 > 0) ? t - K + 1 : 0", "(t - K > 0) ? t - K : 0")],
    "gqa_modulo_mapping": [("const int g = h / group;", "const int g = h % nkv;")],
    "ewma_weights_swapped": [("p->gamma_far * (*Sg) + (1.0 - p->gamma_far) * evicted",
                              "(1.0 - p->gamma_far) * (*Sg) + p->gamma_far * evicted")],
    "eviction_one_step_late": [("if (t >= K) {", "if (t > K) {")],
    "ring_mean_over_filled_slots": [("ring_mean /= (double)R;",
                                     "ring_mean /= (double)((t + 1 < R) ? t + 1 : R);")],
    "field_weight_dropped": [("0.5 * st->field[i]", "st->field[i]")],
    "temperature_dropped": [("/ p->temperature;", ";")],
    "slot_norm_dropped": [("fmax(slot_norm[j], SFA_ORACLE_NORM_FLOOR)", "1.0")],
    "pool_mixes_unit_slots": [("sem += w[j] * (double)slots[(size_t)j * H + i];",
                               "sem += w[j] * (double)slots[(size_t)j * H + i] / slot_norm[j];")],
    "scale_then_clip": [("double u = ring_mean + 0.5 * st->field[i] + 0.5 * sem;",
                         "double u = alpha_layer * (ring_mean + 0.5 * st->field[i] + 0.5 * sem);"),
                        ("out[i] = x[i] + alpha_layer * u;", "out[i] = x[i] + u;")],
    "layer_decay_off_by_one": [("pow(cross_decay, (double)layer)",
                                "pow(cross_decay, (double)(layer + 1))")],
    "far_term_dropped": [("o / denom + p->alpha_far * st->S[(size_t)g * d + i]", "o / denom")],
    "field_decay_swapped": [("p->ema_gamma * st->field[i] + (1.0 - p->ema_gamma) * x[i]",
                             "(1.0 - p->ema_gamma) * st->field[i] + p->ema_gamma * x[i]")],
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    src = open(SRC).read()
    for old, new in MUTANTS[name]:
        assert src.count(old) == 1, f"mutation anchor not unique: {old!r}"
        src = src.replace(old, new)
    shutil.copy(os.path.join(ROOT, "oracle", "sfa_oracle.h"), tmp_path)
    c = tmp_path / "sfa_oracle.c"
    c.write_text(src)
    so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-std=c99", "-O2", "-fno-fast-math", "-ffp-contract=off",
                    "-fopenmp", "-shared", "-fPIC", "-o", str(so), str(c), "-lm"], check=True)
    env = dict(os.environ, SFA_ORACLE_LIB=str(so))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"pins did not catch mutant {name}:\n{r.stdout[-2000:]}"
