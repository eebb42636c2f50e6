"""The oracle's pins must catch plausible mistakes.

Each case copies ``oracle/ssm_oracle.c``, plants ONE mistake in the copy by a
textual substitution (a dropped term, a wrong sign or index, a swapped
operand, the wrong discretisation), compiles it on the CPU into a temporary
library, and runs ``tests/test_oracle_pins.py`` against it in a subprocess.
The pin suite must FAIL for every mutant.  The real oracle is not modified.
"""
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "ssm_oracle.c")

MUTANTS = {
    # [Minimal-scan] §3.2 Euler-B replaced by full ZOH-B
    "zoh_B": ("const double deltaB_u = dt * B[row * N + n] * ui;",
              "const double deltaB_u = (exp(dt * A[d * N + n]) - 1.0) / A[d * N + n]"
              " * B[row * N + n] * ui;"),
    # B and C swapped in the scan
    "swap_B_C": ("yi += x[n] * C[row * N + n];", "yi += x[n] * B[row * N + n];"),
    # §5 D-skip dropped
    "drop_D": ("yi += ui * D[d];", "yi += 0.0 * D[d];"),
    # sign of the exponent flipped (exp(-delta A))
    "A_sign": ("const double deltaA = exp(dt * A[d * N + n]);",
               "const double deltaA = exp(-dt * A[d * N + n]);"),
    # A read transposed, (N, d_in) instead of (d_in, N)
    "A_transposed": ("const double deltaA = exp(dt * A[d * N + n]);",
                     "const double deltaA = exp(dt * A[n * d_in + d]);"),
    # dt_bias not added
    "drop_bias": ("dt += dt_bias[d];", "dt += 0.0 * dt_bias[d];"),
    # softplus not applied
    "drop_softplus": ("dt = oracle_softplus(dt);", "dt = dt;"),
    # gate not applied
    "drop_gate": ("yi *= oracle_silu(z[row * d_in + d]);", "yi *= 1.0;"),
    # readout with the state BEFORE the update (y_t = C h_{t-1})
    "readout_before_update": (
        "x[n] = deltaA * x[n] + deltaB_u;\n            }\n            /* §4",
        "x[n] = x[n];\n                (void)deltaA; (void)deltaB_u;\n            }\n            /* §4"),
    # h0 ignored
    "ignore_h0": ("x[n] = h0 ? h0[(ib * d_in + d) * N + n] : 0.0;", "x[n] = 0.0;"),
    # step: decay dropped
    "step_no_decay": ("*s = *s * dA + x[bd] * dB;", "*s = *s + x[bd] * dB;"),
    # step: bias dropped
    "step_drop_bias": ("delta += dt_bias[d];", "delta += 0.0 * dt_bias[d];"),
    # SS2D: direction k3 not reversed
    "ss2d_k3_not_reversed": ("if (k >= 2)\n        l = L - 1 - l;", "if (k == 2)\n        l = L - 1 - l;"),
    # SS2D: column-major index computed with W instead of H (square grids only agree)
    "ss2d_colmajor_wrong": ("int64_t h = l % H;           /* column-major: l = w H + h */\n"
                            "        const int64_t w = l / H;",
                            "int64_t h = l / W;           /* column-major: l = w H + h */\n"
                            "        const int64_t w = l % W;"),
    # conv step: window not rolled (the newest value overwrites the last tap only)
    "conv_no_roll": ("for (int64_t j = 0; j + 1 < d_conv; ++j)  /* roll left by one */",
                     "for (int64_t j = 0; j + 1 < 0; ++j)  /* roll left by one */"),
    # conv step: weight taps reversed
    "conv_taps_reversed": ("acc += cs[j] * weight[d * d_conv + j];",
                           "acc += cs[j] * weight[d * d_conv + d_conv - 1 - j];"),
    # SS2D snake: odd rows not flipped
    "ss2d_snake_rows_unflipped": ("if (order == 1 && h % 2 == 1)", "if (order == 1 && h % 2 == 7)"),
    # SS2D snake: even columns flipped instead of odd ones
    "ss2d_snake_cols_wrong_parity": ("if (order == 1 && w % 2 == 1)", "if (order == 1 && w % 2 == 0)"),
    # backward: the adjoint is not decayed on its way to the previous step
    "bwd_lam_no_decay": ("lam[n] *= a;", "lam[n] *= 1.0;"),
    # backward: dB misses the step size
    "bwd_dB_no_delta": ("dB[row * N + n] += lam[n] * dts[t] * ut;", "dB[row * N + n] += lam[n] * ut;"),
    # backward: softplus derivative dropped from the delta gradient
    "bwd_no_softplus_grad": ("ddt *= oracle_softplus_grad(pre[t]);", "ddt *= 1.0;"),
    # backward: the decay gradient uses h_t instead of h_{t-1}
    "bwd_hprev_off_by_one": ("const double hprev = hs[t * N + n];",
                             "const double hprev = hs[(t + 1) * N + n];"),
    # backward: wrong sign inside the SiLU derivative
    "bwd_silu_grad_sign": ("s * (1.0 + zt * (1.0 - s))", "s * (1.0 - zt * (1.0 - s))"),
    # backward: dC takes dout past the gate without the silu(z) factor
    "bwd_C_grad_ungated": ("dC[row * N + n] += g * hs[(t + 1) * N + n];",
                           "dC[row * N + n] += dout[at] * hs[(t + 1) * N + n];"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name):
    old, new = MUTANTS[name]
    src = open(SRC, encoding="utf-8").read()
    assert src.count(old) >= 1, f"mutant {name}: anchor text not found in the oracle"
    mutated = src.replace(old, new, 1)
    with tempfile.TemporaryDirectory() as tmp:
        csrc = os.path.join(tmp, "mutant.c")
        lib = os.path.join(tmp, "libmutant.so")
        open(csrc, "w", encoding="utf-8").write(mutated)
        subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-fopenmp", csrc, "-o", lib,
                        "-lm"], check=True)
        env = dict(os.environ, SSM_ORACLE_LIB_OVERRIDE=lib, OMP_NUM_THREADS="2")
        r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                            os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                           cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutant {name} survived the pins:\n{r.stdout[-2000:]}"
