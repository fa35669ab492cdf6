"""Each planted mistake in a copy of the oracle must make at least one pin fail.

The mistakes are the plausible ones: a wrong scale or head index, a dropped
ReLU or merge term, a flipped order or tie-break, a wrong rounding rule, a
transposed operand, an off-by-one causal horizon.  The copies are built on the
CPU from the oracle's own source with one text substitution each.
"""
import ctypes
import os
import subprocess
import tempfile

import pytest

import oracle
from oracle import build as obuild
from tests import pins

MUTANTS = {
    "k_scale_index": ("half_to_double(c.ks[(cell * kHKV + g) * kNG + d / kGroup])",
                      "half_to_double(c.ks[(cell * kHKV + g) * kNG + d % kNG])"),
    "v_scale_from_k": ("half_to_double(c.vs[(cell * kHKV + g) * kNG + d / kGroup])",
                       "half_to_double(c.ks[(cell * kHKV + g) * kNG + d / kGroup])"),
    "gqa_mapping": ("h / kQPerKV", "h % kHKV"),
    "no_relu": ("std::max(0.0, dot)", "dot"),
    "order_sign": ("return s[a] > s[b];", "return s[a] < s[b];"),
    "tie_break": ("    return a < b;\n  }", "    return a > b;\n  }"),
    "softmax_sign": ("const double p = std::exp(s[j] - m);\n    l += p;\n    for (int d = 0; d < kD; ++d) out[d]",
                     "const double p = std::exp(m - s[j]);\n    l += p;\n    for (int d = 0; d < kD; ++d) out[d]"),
    "merge_drop_weight": ("L += l[j] * e;", "L += l[j];"),
    "quant_divisor": ("amax / 127.0f", "amax / 128.0f"),
    "quant_rounding": ("std::nearbyint(x[i] / sf)", "std::round(x[i] / sf)"),
    "iq_transposed": ("half_to_double(iq[h * kDI + d])", "half_to_double(iq[d * kHI + h])"),
    "weight_index": ("static_cast<double>(iw[h]) * std::max", "static_cast<double>(iw[0]) * std::max"),
    "causal_off_by_one": ("row(c, vis0 + r, ", "row(c, vis0 + r + 1, "),
    # the same slip made in all three softmax routines (attention, partials, brute force):
    # every closed form and invariant still holds; only the hand-worked weights catch it
    "softmax_exp2": [("std::exp(s[j] - m)", "std::exp2(s[j] - m)"), ("std::exp(s[c] - m)", "std::exp2(s[c] - m)")],
    "logit_divided_by_scale": [("s.push_back(scale * dot);", "s.push_back(dot / scale);"),
                               ("s[c] = scale * dot;", "s[c] = dot / scale;")],
    "temperature_after_max": [("std::exp(s[j] - m)", "std::exp(0.5 * (s[j] - m))"),
                              ("std::exp(s[c] - m)", "std::exp(0.5 * (s[c] - m))")],
    "gate_sign": ("std::exp(-static_cast<double>(gate[i]))", "std::exp(static_cast<double>(gate[i]))"),
    "gate_linear": ("out[i] *= 1.0 / (1.0 + std::exp(-static_cast<double>(gate[i])));",
                    "out[i] *= static_cast<double>(gate[i]);"),
    "scale_dropped": ("s.push_back(scale * dot);\n    cells.push_back(ids[i]);\n  }\n  for (int d = 0; d < kD; ++d) out[d] = 0.0;",
                      "s.push_back(dot);\n    cells.push_back(ids[i]);\n  }\n  for (int d = 0; d < kD; ++d) out[d] = 0.0;"),
}


# mutants the hand-worked softmax weights must catch (the closed forms cannot)
SOFTMAX_ONLY = {"softmax_exp2", "temperature_after_max", "logit_divided_by_scale"}


def _build_mutant(name, edits, tmp):
    src = open(obuild.SRC).read()
    for old, new in edits:
        assert src.count(old) >= 1, f"mutation site for {name} not found: {old!r}"
        src = src.replace(old, new)
    path = os.path.join(tmp, f"{name}.cpp")
    with open(path, "w") as f:
        f.write(src)
    lib = os.path.join(tmp, f"lib{name}.so")
    subprocess.run(["g++", "-std=c++17", "-O1", "-fPIC", "-shared", "-fopenmp", path, "-o", lib],
                   check=True)
    return lib


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    edits = MUTANTS[name]
    if isinstance(edits, tuple):
        edits = [edits]
    saved = oracle.lib()
    with tempfile.TemporaryDirectory() as tmp:
        path = _build_mutant(name, edits, tmp)
        oracle._lib = oracle.configure(ctypes.CDLL(path))
        failed = []
        try:
            for check in pins.ALL_CHECKS:
                try:
                    check()
                except AssertionError:
                    failed.append(check.__name__)
        finally:
            oracle._lib = saved
    assert failed, f"no pin caught mutant {name}"
    if name in SOFTMAX_ONLY:
        assert "check_attn_softmax_golden" in failed, failed
