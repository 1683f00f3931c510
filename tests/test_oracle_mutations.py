"""The pins must be able to fail: each planted slip in a copy of the oracle
(built into a temporary directory) has to make the pin suite fail.

This guards against pins that would pass whatever the oracle computed.
"""

import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "moe_oracle.cpp")

MUTANTS = {
    "nibble_order": ("return (k % 2 == 0) ? (byte & 0x0f) : (byte >> 4);",
                     "return (k % 2 == 1) ? (byte & 0x0f) : (byte >> 4);"),
    "gate_up_swapped": ("h[i] = static_cast<float>(silu(gu[i]) * gu[I + i]);",
                        "h[i] = static_cast<float>(silu(gu[I + i]) * gu[i]);"),
    "bias_dropped": ("out[r * m->K + k] = sq + b;", "out[r * m->K + k] = sq;"),
    "group_index": ("const int64_t g = k / group;", "const int64_t g = k % ngroups;"),
    "softmax_sign": ("p[e] = std::exp(logits[e] - mx);", "p[e] = std::exp(mx - logits[e]);"),
    "tie_rule": ("return a < b;\n  });\n  double sel", "return a > b;\n  });\n  double sel"),
    "sigmoid_sign": ("return 1.0 / (1.0 + std::exp(-z)); }", "return 1.0 / (1.0 + std::exp(z)); }"),
    "shared_ungated": ("if (has_shared) acc += gate * outs[nsel][r];",
                       "if (has_shared) acc += outs[nsel][r];"),
    "router_transposed": ("static_cast<double>(bf16_to_f32(wr[e * H + h]));",
                          "static_cast<double>(bf16_to_f32(wr[h * E + e]));"),
    "down_transposed": ("acc += static_cast<double>(wd[r * I + i]) * h[i];",
                        "acc += static_cast<double>(wd[i * H + r]) * h[i];"),
    "no_renorm": ("w[j] = renorm ? p[order[j]] / sel : p[order[j]];", "w[j] = p[order[j]];"),
    "rms_no_mean": ("1.0 / std::sqrt(ss / static_cast<double>(H) + eps);", "1.0 / std::sqrt(ss + eps);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_slip(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found once"
    mut = tmp_path / "mut.cpp"
    mut.write_text(src.replace(old, new))
    so = tmp_path / "libmut.so"
    subprocess.run(["g++", "-O1", "-std=c++17", "-ffp-contract=off", "-fPIC", "-shared", "-pthread",
                    str(mut), "-o", str(so)], check=True)
    env = dict(os.environ, MOE_ORACLE_LIB=str(so))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"pins passed with planted slip {name}:\n{r.stdout[-2000:]}"
