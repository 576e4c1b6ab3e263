"""The pins must catch plausible mistakes in the oracle.

Each case copies the oracle's C source, plants one mistake (a dropped term, a
wrong sign, index or operand), builds the copy on the CPU and runs every pin of
test_oracle_pins against it: at least one pin must fail.  The oracle itself is
never modified.
"""
import functools
import inspect
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle
from oracle import oracle as _oracle_mod
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "gdn_oracle.c")

MUTANTS = {
    "decay_not_on_erase": ("beta * (v[i] - alpha * x[i])", "beta * (v[i] - x[i])"),
    "decay_not_on_state": ("alpha * S[(int64_t)i * dk + j] + u * k[j]", "S[(int64_t)i * dk + j] + u * k[j]"),
    "write_sign": ("double u = beta * (v[i] - alpha * x[i]);", "double u = beta * (v[i] + alpha * x[i]);"),
    "key_head_modulo": ("const int g = h / grp;\n        if (seq_mask", "const int g = h % Hqk;\n        if (seq_mask"),
    "softplus_branch": ("return x + log1p(exp(-x));", "return x + log1p(exp(x));"),
    "beta_sign": ("return 1.0 / (1.0 + exp(-b));", "return 1.0 / (1.0 + exp(b));"),
    "gate_rate_not_exp": ("return -exp(A_log) * softplus(a + dt_bias);", "return -A_log * softplus(a + dt_bias);"),
    "output_unscaled": ("o[i] = scale * acc;", "o[i] = acc;"),
    "conv_taps_reversed": ("acc += (double)w[c * 4 + j] * xv;", "acc += (double)w[c * 4 + (3 - j)] * xv;"),
    "l2_no_eps": ("1.0 / sqrt(ss + 1e-6)", "1.0 / sqrt(ss)"),
    "silu_sign": ("acc / (1.0 + exp(-acc))", "acc / (1.0 + exp(acc))"),
    "chunk_u_sign": ("Up[(int64_t)i * dv + e] - acc;", "Up[(int64_t)i * dv + e] + acc;"),
    "chunk_no_decay_in_A": ("val = be[i] * exp(G[i] - G[j]) * kk;", "val = be[i] * kk;"),
    "chunk_W_no_gamma": ("acc += Tm[i * C + j] * be[j] * exp(G[j]) * K[(int64_t)j * dk + e];",
                         "acc += Tm[i * C + j] * be[j] * K[(int64_t)j * dk + e];"),
    "chunk_state_no_decay": ("double acc = exp(GL) * S[(int64_t)e * dk + f];",
                             "double acc = S[(int64_t)e * dk + f];"),
    "chunk_inter_no_gamma": ("dst[e] = scale * (exp(G[i]) * inter + intra);",
                             "dst[e] = scale * (inter + intra);"),
    "chunk_substitution_sign": ("val -= A[i * C + m] * Tm[m * C + j];", "val += A[i * C + m] * Tm[m * C + j];"),
    "norm_sum_not_mean": ("1.0 / sqrt(ss / d + eps)", "1.0 / sqrt(ss + eps)"),
    "bw_dk_one_sided": ("-alpha * beta * (sg + gs) + beta * gv", "-alpha * beta * (2.0 * sg) + beta * gv"),
    "bw_dalpha_no_erase": ("const double dalpha = GS - beta * Skg;", "const double dalpha = GS;"),
    "bw_state_no_decay": ("G[(int64_t)i * dk + e] = alpha * (G[(int64_t)i * dk + e] - beta * g[i] * kt[e]);",
                          "G[(int64_t)i * dk + e] = G[(int64_t)i * dk + e] - beta * g[i] * kt[e];"),
    "bw_output_from_old_state": ("acc += St[(int64_t)i * dk + e] * dot[i];", "acc += S[(int64_t)i * dk + e] * dot[i];"),
    "bw_gate_sign": ("const double dat = dla * (-exp(A_log[h]) * sig);", "const double dat = dla * (exp(A_log[h]) * sig);"),
    "norm_no_eps": ("1.0 / sqrt(ss / d + eps)", "1.0 / sqrt(ss / d)"),
    "gate_sigmoid_only": ("const double g = z[row + e] / (1.0 + exp(-z[row + e]));",
                          "const double g = 1.0 / (1.0 + exp(-z[row + e]));"),
    "norm_weight_wrong_layer": ("const double* wl = w + (int64_t)(t % layers) * d;", "const double* wl = w;"),
    "norm_over_heads": ("const int64_t row = (t * Hv + h) * (int64_t)d;\n            double ss = 0.0;\n            for (int e = 0; e < d; ++e) ss += o[row + e] * o[row + e];",
                        "const int64_t row = (t * Hv + h) * (int64_t)d;\n            double ss = 0.0;\n            for (int e = 0; e < d; ++e) ss += o[t * Hv * (int64_t)d + e] * o[t * Hv * (int64_t)d + e];"),
    "cbw_inverse_sign": ("dA[i * C + j] = j < i ? -acc : 0.0;", "dA[i * C + j] = j < i ? acc : 0.0;"),
    "cbw_inverse_transposed": ("acc += Tm[m * C + i] * dT[m * C + j];", "acc += Tm[i * C + m] * dT[m * C + j];"),
    "cbw_kk_one_sided": ("dK[(int64_t)j * dk + f] += E * K[(int64_t)i * dk + f];",
                         "dK[(int64_t)j * dk + f] += 0.0 * E;"),
    "cbw_no_kappa_sum": ("dG[L - 1] += kk_sum;", "dG[L - 1] += 0.0 * kk_sum;"),
    "cbw_no_W_gamma_grad": ("dgam[j] += be[j] * sk;", "dgam[j] += 0.0 * sk;"),
    "cbw_carry_no_decay": ("dS[i] += gam[L - 1] * dSn[i];", "dS[i] += dSn[i];"),
    "fbw_no_norm_projection": ("const double da = normed ? (dout[e] - av[e] / nrm * dot) / nrm : dout[e];",
                               "const double da = normed ? dout[e] / nrm : dout[e];"),
    "fbw_silu_derivative": ("const double dy = da * sg * (1.0 + yv[e] * (1.0 - sg));",
                            "const double dy = da * sg * (1.0 + yv[e] * sg);"),
    "fbw_weight_tap_reversed": ("dw[c * 4 + j] += dy * gdn_oracle_front_x(x, conv_state_in, Ctot, n, bos, tau, c);",
                                "dw[c * 4 + (3 - j)] += dy * gdn_oracle_front_x(x, conv_state_in, Ctot, n, bos, tau, c);"),
    "fbw_history_slot": ("else if (dconv_state) dconv_state[((int64_t)n * Ctot + c) * 3 + (3 - (bos - tau))] += w[c * 4 + j] * dy;",
                         "else if (dconv_state) dconv_state[((int64_t)n * Ctot + c) * 3 + (bos - tau - 1)] += w[c * 4 + j] * dy;"),
    "f64_front_history_slot": ("return cs ? cs[((int64_t)n * Ctot + c) * 3 + (3 - m)] : 0.0;",
                               "return cs ? cs[((int64_t)n * Ctot + c) * 3 + (m - 1)] : 0.0;"),
    "f64_front_norm_on_v": ("const double inv = hh < 2 * Hqk ? 1.0 / sqrt(ss + 1e-6) : 1.0;",
                            "const double inv = 1.0 / sqrt(ss + 1e-6);"),
    "nbw_no_norm_term": ("d_o[row + e] = r * u - r * r * r / d * o[row + e] * ou;", "d_o[row + e] = r * u;"),
    "nbw_silu_derivative": ("dz[row + e] = dy[row + e] * wl[e] * r * o[row + e] * sg * (1.0 + z[row + e] * (1.0 - sg));",
                            "dz[row + e] = dy[row + e] * wl[e] * r * o[row + e] * sg;"),
    "nbw_weight_one_layer": ("dw[(int64_t)l * d + e] += dy[row + e] * r * o[row + e] * g;",
                             "dw[e] += dy[row + e] * r * o[row + e] * g;"),
}


class _Bound:
    """The oracle module's functions bound to another build of the library."""

    def __init__(self, lib):
        self._lib = lib

    def __getattr__(self, name):
        return functools.partial(getattr(_oracle_mod, name), lib=self._lib)


def _pin_functions():
    out = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_"):
            continue
        params = inspect.signature(fn).parameters
        if "C" in params:
            for C in (1, 16):
                out.append((f"{name}[{C}]", functools.partial(fn, C=C)))
        else:
            out.append((name, fn))
    return out


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mutated = src.replace(old, new, 1)
    csrc = tmp_path / "mut.c"
    csrc.write_text(mutated)
    lib_path = str(tmp_path / "libmut.so")
    subprocess.run(["gcc", "-O1", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", lib_path,
                    str(csrc), "-lm"], check=True)
    bound = _Bound(oracle.build(path=lib_path))
    failed = []
    for pin_name, fn in _pin_functions():
        try:
            with np.errstate(all="ignore"):
                fn(bound)
        except (AssertionError, ValueError):
            failed.append(pin_name)
    assert failed, f"no pin catches the planted mistake {name}"
