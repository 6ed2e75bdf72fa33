"""Plants plausible mistakes in a copy of the oracle and checks that the pins catch
every one (each mutant must fail at least one test of test_oracle_pins.py).

The mistakes are planted on the CPU in a temporary copy of the oracle source; the
committed oracle is never modified.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "sa_oracle.cpp")

MUTANTS = {
    "drop_1_over_sqrt_d": ("    s *= inv_sqrt_d;\n    A[j] = s;", "    A[j] = s;"),
    "W_k_transposed": ("K[e] += x * wk[e]; V[e] += x * wv[e];",
                       "K[e] += x * Wk[(int64_t)e * d + c]; V[e] += x * wv[e];"),
    "W_v_transposed": ("K[e] += x * wk[e]; V[e] += x * wv[e];",
                       "K[e] += x * wk[e]; V[e] += x * Wv[(int64_t)e * d + c];"),
    "sum_instead_of_mean": ("tav[(int64_t)j * d + e] / mj : 0.0", "tav[(int64_t)j * d + e] : 0.0"),
    "lse_missing_log_Z": ("return m + std::log(Z);", "return m;"),
    "mass_of_squares": ("acc_mass[j] += aj;", "acc_mass[j] += aj * aj;"),
    "dmass_sign": ("dmass[j] = -dot +", "dmass[j] = dot +"),
    "dmass_ignores_Gm": ("dmass[j] = -dot + (Gm ? Gm[(int64_t)u * k + j] : 0.0);", "dmass[j] = -dot;"),
    "softmax_backward_drops_D": ("const double dS = A[j] * (dA[j] - D);", "const double dS = A[j] * dA[j];"),
    "dX_drops_value_path": ("s += dK[e] * wk[e] + dV[e] * wv[e];", "s += dK[e] * wk[e];"),
    "dW_k_transposed": ("rk[e] += Xt[c2] * dK[e];", "rk[e] += Xt[e] * dK[c2];"),
    "dP_drops_scale": ("dpj[e] += dS * K[e] * inv_sqrt_d;", "dpj[e] += dS * K[e];"),
    "dV_drops_A": ("dV[e] += A[j] * g[e];", "dV[e] += g[e];"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found once"
    mut = tmp_path / "mutant.cpp"
    mut.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["g++", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c++17", "-o", str(lib),
                    str(mut)], check=True)
    env = dict(os.environ, SA_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutant {name} passed every pin:\n{r.stdout[-2000:]}"
