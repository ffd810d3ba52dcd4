"""Each plausible slip planted in a temporary copy of the oracle must fail at
least one pin.  The copies are compiled into a temporary directory and run in
a subprocess (a broken copy may also crash); the committed oracle is never
modified.  CPU only."""
import subprocess
import sys
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parents[1]
SRC = ROOT / "oracle" / "oracle.c"

# (name, exact text in oracle.c, replacement)
MUTANTS = [
    ("residual without clamp at zero",
     "w[v] = r > 0.0 ? r : 0.0;", "w[v] = r;"),
    ("acceptance ratio inverted",
     "double a = p[i] / q[i];", "double a = q[i] / p[i];"),
    ("accept when u equals a",
     "if (u[i] < a) {", "if (u[i] <= a) {"),
    ("final draw reuses the rejected position's uniform",
     "inverse_cdf_draw(w, V, u[k_max], &flags)", "inverse_cdf_draw(w, V, u[j], &flags)"),
    ("temperature dropped",
     "ell[v] = load_logit(row, dtype, v) / T;", "ell[v] = load_logit(row, dtype, v);"),
    ("log-sum-exp without the max",
     "return M + log(S);", "return log(S);"),
    ("inverse CDF with >=",
     "if (C > target) {", "if (C >= target) {"),
    ("final draw on the previous row",
     "(void)row_log_sum_exp(TROW(j), dtype, V, T, ell_t);",
     "(void)row_log_sum_exp(TROW(j > 0 ? j - 1 : 0), dtype, V, T, ell_t);"),
    ("scan does not stop at the first rejection",
     "            j = i;\n            break;\n        }\n    }\n\n    /* Step 3",
     "            if (j == L) j = i;\n        }\n    }\n\n    /* Step 3"),
    ("greedy tie goes to the highest index",
     "if (z > best_val) {", "if (z >= best_val) {"),
    ("residual sign flipped",
     "double r = w[v] - exp(ell_d[v] - lse_d_row[j]);",
     "double r = exp(ell_d[v] - lse_d_row[j]) - w[v];"),
    ("one-hot residual keeps the drafted token",
     "double r = w[x[j]] - 1.0;", "double r = w[x[j]];"),
    ("gather at the wrong id",
     "p[i] = exp(ell_t[x[i]] - lse_t_row[i]);",
     "p[i] = exp(ell_t[x[i] > 0 ? x[i] - 1 : 1] - lse_t_row[i]);"),
    ("first term dropped from the sum",
     "    for (int64_t v = 0; v < V; ++v)\n        S += exp(ell[v] - M);",
     "    for (int64_t v = 1; v < V; ++v)\n        S += exp(ell[v] - M);"),
    ("bonus drawn without the all-accepted row",
     "    /* else j == L: bonus draw from p_L [NG-PIPE]; w already holds p_L. */",
     "    else { (void)row_log_sum_exp(TROW(0), dtype, V, T, ell_t);\n"
     "      for (int64_t v = 0; v < V; ++v) w[v] = exp(ell_t[v] - lse_t_row[0]); }"),
    ("expected length counts the reach before the position",
     "            reach *= a[m - 1];\n            e += reach;", "            e += reach;\n            reach *= a[m - 1];"),
    ("simulated acceptance accepts on u == a",
     "if (!(uniforms[b * (k_max + 1) + i] < a[i])) {", "if (!(uniforms[b * (k_max + 1) + i] <= a[i])) {"),
    ("decay starts at the first position",
     "(i <= j ? 1.0 : pow(decay, (double)(i - j)))", "pow(decay, (double)i)"),
    ("acceptance probability not clamped at one",
     "                a[i] = r > 1.0 ? 1.0 : r;", "                a[i] = r;"),
    ("acceptance tie band 1e-3",
     "if (fabs(u[i] - a) < ORACLE_TIE_BAND)", "if (fabs(u[i] - a) < 1e-3)"),
    ("acceptance tie band 1e-7",
     "if (fabs(u[i] - a) < ORACLE_TIE_BAND)", "if (fabs(u[i] - a) < 1e-7)"),
    ("draw tie band 1e-3 of W",
     "fabs(C - target) < ORACLE_TIE_BAND * W)", "fabs(C - target) < 1e-3 * W)"),
    ("draw tie band 1e-7 of W",
     "            if (fabs(target - C_prev) < ORACLE_TIE_BAND * W ||\n                fabs(C - target) < ORACLE_TIE_BAND * W)",
     "            if (fabs(target - C_prev) < 1e-7 * W ||\n                fabs(C - target) < 1e-7 * W)"),
    ("draw tie band absolute instead of relative to W",
     "            if (fabs(target - C_prev) < ORACLE_TIE_BAND * W ||\n                fabs(C - target) < ORACLE_TIE_BAND * W)",
     "            if (fabs(target - C_prev) < ORACLE_TIE_BAND ||\n                fabs(C - target) < ORACLE_TIE_BAND)"),
    ("fallback takes the first positive weight",
     "    for (int64_t t = V - 1; t >= 0; --t)\n        if (w[t] > 0.0)",
     "    for (int64_t t = 0; t < V; ++t)\n        if (w[t] > 0.0)"),
    ("zero residual mass keeps the zero weights",
     "            for (int64_t v = 0; v < V; ++v)\n                w[v] = exp(ell_t[v] - lse_t_row[j]);\n        }",
     "        }"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    src = SRC.read_text()
    assert src.count(old) == 1, f"mutation site not unique / missing: {name}"
    mutant_src = tmp_path / "oracle_mutant.c"
    mutant_src.write_text(src.replace(old, new))
    lib = tmp_path / "liboracle_mutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", str(lib),
                    str(mutant_src), "-lm"], check=True)
    proc = subprocess.run([sys.executable, str(ROOT / "tests" / "pins.py"), str(lib)],
                          capture_output=True, text=True, timeout=600)
    assert proc.returncode != 0, f"mutant '{name}' passed every pin:\n{proc.stdout}\n{proc.stderr}"
