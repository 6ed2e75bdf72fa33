"""Plants plausible mistakes in a copy of the oracle and checks that the pins catch
every one (each Sketch Attention mutant must fail at least one test of
test_oracle_pins.py, each cross-attention mutant one of test_oracle_stca_pins.py).

The mistakes are planted on the CPU in a temporary copy of the oracle source; the
committed oracle is never modified.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "sa_oracle.cpp")
STCA_SRC = os.path.join(ROOT, "oracle", "stca_oracle.cpp")

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


STCA_MUTANTS = {
    "drop_1_over_sqrt_d": ("    z *= inv_sqrt_d;\n", ""),
    "lse_missing_log_Z": ("return m + std::log(Z);", "return m;"),
    "keys_projected_by_W_V": ("row_times(Su + (int64_t)j * d, WK, d, K + (int64_t)j * d);",
                              "row_times(Su + (int64_t)j * d, WV, d, K + (int64_t)j * d);"),
    "softmax_not_normalised": ("for (int j = 0; j < k; ++j) a[j] /= Z;", ""),
    "softmax_backward_drops_D": ("const double dz = a[j] * (da[j] - D);",
                                 "const double dz = a[j] * da[j];"),
    "dV_drops_weights": ("dvj[e] += a[j] * g[e];", "dvj[e] += g[e];"),
    "dS_drops_value_path": ("s += dkj[e] * wk[e] + dvj[e] * wv[e];", "s += dkj[e] * wk[e];"),
    "dK_drops_scale": ("dkj[e] += dz * q[e] * inv_sqrt_d;", "dkj[e] += dz * q[e];"),
    "dQ_W_q_not_transposed": ("for (int e = 0; e < d; ++e) s += dq[e] * w[e];",
                              "for (int e = 0; e < d; ++e) s += dq[e] * Wq[(int64_t)e * d + r];"),
    "dW_K_transposed": ("gk[e] += sj[r] * dkj[e];", "gk[e] += sj[e] * dkj[r];"),
    "dW_q_transposed": ("wq[e] += Qc[r] * dq[e];", "wq[e] += Qc[e] * dq[r];"),
}


def _mutant_fails_pins(src_path, old, new, env_var, pins, tmp_path):
    src = open(src_path).read()
    assert src.count(old) == 1, "mutation site not found exactly once"
    mut = tmp_path / "mutant.cpp"
    mut.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["g++", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c++17", "-o", str(lib),
                    str(mut)], check=True)
    env = dict(os.environ, **{env_var: str(lib)})
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", pins)],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode != 0, r.stdout[-2000:]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    failed, out = _mutant_fails_pins(SRC, *MUTANTS[name], "SA_ORACLE_LIB",
                                     "test_oracle_pins.py", tmp_path)
    assert failed, f"mutant {name} passed every pin:\n{out}"


@pytest.mark.parametrize("name", sorted(STCA_MUTANTS))
def test_cross_attention_pins_catch_mutant(name, tmp_path):
    failed, out = _mutant_fails_pins(STCA_SRC, *STCA_MUTANTS[name], "STCA_ORACLE_LIB",
                                     "test_oracle_stca_pins.py", tmp_path)
    assert failed, f"cross-attention mutant {name} passed every pin:\n{out}"
