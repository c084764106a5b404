"""Plant plausible mistakes in a copy of the oracle and check that the pins catch them.

Each mutant is a one-line change to a copy of ``oracle/la_oracle.c`` (a dropped term,
a wrong sign, a swapped operand, a read before the update).  The copy is compiled on
the CPU into a temporary library and the pin suite is run against it in a child
process; the pins must FAIL for every mutant.  The real oracle is never modified.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "la_oracle.c")

MUTANTS = {
    # mode 0
    "phi_drops_plus_one": ("x > 0.0 ? x + 1.0 : exp(x)", "x > 0.0 ? x : exp(x)"),
    "mode0_state_uses_query_feature": ("row[j] += v[i] * fk[j];", "row[j] += v[i] * fq[j];"),
    "mode0_denominator_before_update": ("            z[j] += fk[j];\n            den += z[j] * fq[j];",
                                        "            den += z[j] * fq[j];\n            z[j] += fk[j];"),
    # mode 1
    "mode1_drops_gate": ("row[j] = a * row[j] + v[i] * k[j];", "row[j] = row[j] + v[i] * k[j];"),
    "mode1_reads_with_key": ("                row[j] = a * row[j] + v[i] * k[j];\n                acc += row[j] * q[j];",
                             "                row[j] = a * row[j] + v[i] * k[j];\n                acc += row[j] * k[j];"),
    # mode 2
    "mode2_wrong_sign": ("row[j] = a * (row[j] - beta * sk[i] * k[j])", "row[j] = a * (row[j] + beta * sk[i] * k[j])"),
    "mode2_correction_not_decayed": ("row[j] = a * (row[j] - beta * sk[i] * k[j]) + beta * v[i] * k[j];",
                                     "row[j] = a * row[j] - beta * sk[i] * k[j] + beta * v[i] * k[j];"),
    "mode2_write_drops_beta": ("- beta * sk[i] * k[j]) + beta * v[i] * k[j];", "- beta * sk[i] * k[j]) + v[i] * k[j];"),
    "mode2_reads_old_state": ("                row[j] = a * (row[j] - beta * sk[i] * k[j]) + beta * v[i] * k[j];\n                acc += row[j] * q[j];",
                              "                acc += row[j] * q[j];\n                row[j] = a * (row[j] - beta * sk[i] * k[j]) + beta * v[i] * k[j];"),
    "mode2_correction_uses_query": ("acc += row[j] * k[j];\n            sk[i] = acc;", "acc += row[j] * q[j];\n            sk[i] = acc;"),
    # mode 3
    "mode3_correction_not_decayed": ("acc += row[j] * (av ? av[j] : 1.0) * k[j];", "acc += row[j] * k[j];"),
    "mode3_drops_channel_decay": ("row[j] = row[j] * (av ? av[j] : 1.0) - beta * sk[i] * k[j]",
                                  "row[j] = row[j] - beta * sk[i] * k[j]"),
    "mode3_reads_old_state": ("                row[j] = row[j] * (av ? av[j] : 1.0) - beta * sk[i] * k[j] + beta * v[i] * k[j];\n                acc += row[j] * q[j];",
                              "                acc += row[j] * q[j];\n                row[j] = row[j] * (av ? av[j] : 1.0) - beta * sk[i] * k[j] + beta * v[i] * k[j];"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistakes(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    mutant_c = tmp_path / "mutant.c"
    mutant_c.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", str(mutant_c), "-o", str(lib), "-lm"],
                   check=True)
    env = dict(os.environ, LA_ORACLE_LIB_OVERRIDE=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"planted mistake {name} passed every pin:\n{r.stdout[-2000:]}"
    assert "failed" in r.stdout or "error" in r.stdout.lower()


CONV_SRC = os.path.join(ROOT, "oracle", "conv.py")
CONV_MUTANTS = {
    "conv_taps_reversed": ("u += w[:, i] * full[:, i:i + T, :]",
                           "u += w[:, width - 1 - i] * full[:, i:i + T, :]"),
    "conv_window_not_carried": ("return y, full[:, T:, :].copy()", "return y, full[:, -(width - 1):, :].copy() * 0"),
    "conv_silu_sign": ("u = u / (1.0 + np.exp(-u))", "u = u / (1.0 + np.exp(u))"),
    "conv_norm_over_heads": ("r = u.reshape(B, T, H, C // H)", "r = u.reshape(B, T, C // H, H)"),
    "conv_head_layout": ("y = y.reshape(B, T, H, d).transpose(0, 2, 1, 3).copy()",
                         "y = y.reshape(B, H, T, d).copy()"),
}


@pytest.mark.parametrize("name", sorted(CONV_MUTANTS))
def test_conv_pins_catch_planted_mistakes(name, tmp_path):
    old, new = CONV_MUTANTS[name]
    src = open(CONV_SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    mutant = tmp_path / "conv_mutant.py"
    mutant.write_text(src.replace(old, new))
    env = dict(os.environ, LA_ORACLE_CONV_OVERRIDE=str(mutant))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_conv_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"planted mistake {name} passed every pin:\n{r.stdout[-2000:]}"
    assert "failed" in r.stdout or "error" in r.stdout.lower()


BWD_SRC = os.path.join(ROOT, "oracle", "backward.py")
BWD_MUTANTS = {
    "bwd_gate_after_write": ("        S = S if a is None else a[:, :, t, None, None] * S\n        S = S + v[:, :, t, :, None] * k[:, :, t, None, :]",
                             "        S = S + v[:, :, t, :, None] * k[:, :, t, None, :]\n        S = S if a is None else a[:, :, t, None, None] * S"),
    "bwd_reads_before_write": ("        S = S + v[:, :, t, :, None] * k[:, :, t, None, :]\n        outs.append(torch.einsum(\"bhij,bhj->bhi\", S, q[:, :, t]))",
                               "        outs.append(torch.einsum(\"bhij,bhj->bhi\", S, q[:, :, t]))\n        S = S + v[:, :, t, :, None] * k[:, :, t, None, :]"),
    "bwd_drops_final_state_term": ("        L = L + (ST * _t(dS_T)).sum()", "        L = L + 0.0 * (ST * _t(dS_T)).sum()"),
}


@pytest.mark.parametrize("name", sorted(BWD_MUTANTS))
def test_backward_pins_catch_planted_mistakes(name, tmp_path):
    old, new = BWD_MUTANTS[name]
    src = open(BWD_SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    mutant = tmp_path / "backward_mutant.py"
    mutant.write_text(src.replace(old, new))
    env = dict(os.environ, LA_ORACLE_BACKWARD_OVERRIDE=str(mutant))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_backward_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"planted mistake {name} passed every pin:\n{r.stdout[-2000:]}"
    assert "failed" in r.stdout or "error" in r.stdout.lower()


DELTA_BWD_MUTANTS = {
    "delta_correction_sign": ("S = S - b * Sk[..., :, None] * kt[..., None, :]",
                              "S = S + b * Sk[..., :, None] * kt[..., None, :]"),
    "delta_correction_uses_query": ('Sk = torch.einsum("bhij,bhj->bhi", S, kt)',
                                    'Sk = torch.einsum("bhij,bhj->bhi", S, q[:, :, t])'),
    "delta_write_drops_rate": ("+ b * v[:, :, t, :, None] * kt[..., None, :]",
                               "+ v[:, :, t, :, None] * kt[..., None, :]"),
    "kda_decays_rows": ("a[:, :, t, None, :] if mode == MODE_KDA", "a[:, :, t, None, :1] if mode == MODE_KDA"),
    "delta_drops_final_state_term": ("L = L + (_t(dS_T) * ST).sum()", "L = L + 0.0 * (_t(dS_T) * ST).sum()"),
    "delta_rate_gradient_misrouted": ("dq, dk, dv, db = (x.detach().numpy() for x in grads[:4])",
                                      "dq, dk, db, dv = (x.detach().numpy() for x in grads[:4])"),
}


@pytest.mark.parametrize("name", sorted(DELTA_BWD_MUTANTS))
def test_delta_backward_pins_catch_planted_mistakes(name, tmp_path):
    old, new = DELTA_BWD_MUTANTS[name]
    src = open(BWD_SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    mutant = tmp_path / "backward_mutant.py"
    mutant.write_text(src.replace(old, new))
    env = dict(os.environ, LA_ORACLE_BACKWARD_OVERRIDE=str(mutant))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_delta_backward_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"planted mistake {name} passed every pin:\n{r.stdout[-2000:]}"
    assert "failed" in r.stdout or "error" in r.stdout.lower()
