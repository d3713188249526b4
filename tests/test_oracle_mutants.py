"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's C++ source (a dropped
term, a wrong sign or index, a transposed operand, a reversed tap order, ...),
builds it in a temporary directory, and runs the pin suites against it: at
least one pin must fail. The real oracle is never modified.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "gdn_oracle.cpp")

MUTANTS = {
    "dropped_gate": ("S[e] *= gt;", "S[e] *= 1.0;"),
    "erase_sign": ("-= bt * Sk[i] * kt[j];", "+= bt * Sk[i] * kt[j];"),
    "transposed_state_read": ("acc += S[(size_t)i * d + j] * kt[j];",
                              "acc += S[(size_t)j * d + i] * kt[j];"),
    "transposed_write": ("+= bt * vt[i] * kt[j];", "+= bt * vt[j] * kt[i];"),
    "query_is_key": ("acc += S[(size_t)i * d + j] * qt[j];",
                     "acc += S[(size_t)i * d + j] * kt[j];"),
    "interleaved_gqa": ("const int kh = h / group;", "const int kh = h % H_k;"),
    "unscaled_output": ("ot[i] = scale * acc;", "ot[i] = acc;"),
    "reversed_taps": ("acc += w[c * 4 + j] * xh(p - 3 + j, c);",
                      "acc += w[c * 4 + j] * xh(p - j, c);"),
    "state_out_off_by_one": ("= xh(len - 3 + r, c);", "= xh(len - 4 + r, c);"),
    "l2_missing_root": ("1.0 / std::sqrt(ss + l2_eps);", "1.0 / (ss + l2_eps);"),
    "rms_sum_not_mean": ("std::sqrt(ss / dim + eps);", "std::sqrt(ss + eps);"),
    "gate_without_silu": ("* w[c] * silu(zr[c]);", "* w[c] * zr[c];"),
    "bias_dropped": ("double acc = bias ? bias[c] : 0.0;", "double acc = 0.0;"),
    "rope_turns_backwards": ("y[i + R / 2] = b * c + a * s;", "y[i + R / 2] = b * c - a * s;"),
    "rope_half_frequency": ("std::pow(base, -2.0 * i / R);", "std::pow(base, -1.0 * i / R);"),
    "rope_one_axis": ("(double)p[i % 3] * std::pow", "(double)p[0] * std::pow"),
    "qk_norm_sum_not_mean": ("1.0 / std::sqrt(ss / D + eps);", "1.0 / std::sqrt(ss + eps);"),
    "qk_norm_weight_dropped": ("y[d] = x[d] * inv * w[d];", "y[d] = x[d] * inv;"),
    "attention_interleaved_gqa": ("g = h / group;", "g = h % Hkv;"),
    "softmax_unshifted_sum": ("l += std::exp(sc[j - s0] - m);", "l += std::exp(sc[j - s0]);"),
    "gate_sign": ("o[d] / (1.0 + std::exp(-gt[d]));", "o[d] / (1.0 + std::exp(gt[d]));"),
    "mask_drops_diagonal": ("const double pj = std::exp(sc[j - s0] - m) / l;",
                            "const double pj = j == t && t > s0 ? 0.0 : std::exp(sc[j - s0] - m) / l;"),
}

PIN_FILES = ["tests/test_oracle_recurrence.py", "tests/test_oracle_conv_norm.py",
             "tests/test_oracle_chunked.py", "tests/test_oracle_attention.py"]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_detect_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    mpath = tmp_path / "mutant.cpp"
    mpath.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["g++", "-O1", "-std=c++17", "-fPIC", "-shared", "-pthread",
                    str(mpath), "-o", str(lib)], check=True)
    env = dict(os.environ, GDN_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q",
                        "-p", "no:cacheprovider", *PIN_FILES],
                       cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode != 0, f"mutant {name} survived the pins:\n{r.stdout[-2000:]}"
