"""The pins must catch a wrong oracle.

Each case below plants one plausible mistake in a copy of the oracle's C++
source (a dropped term, a wrong sign, index or rounding, a transposed
operand, a misread rule), builds it, and runs the pin suite
(tests/test_oracle_pins.py) against it through ``MOE_ORACLE_LIB``.  Every
mutant must fail at least one pin; the unmodified oracle passes the same
suite in the regular run.  CPU only.
"""
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

import pytest

from conftest import ROOT

SRC = os.path.join(ROOT, "oracle", "moe_oracle.cpp")

# name -> [(exact text in moe_oracle.cpp, replacement), ...]
MUTANTS = {
    "tie_to_higher_index": [(
        "[&](int32_t a, int32_t b) { return h[a] > h[b]; }",
        "[&](int32_t a, int32_t b) { return h[a] > h[b] || (h[a] == h[b] && a > b); }")],
    "gate_without_max_shift": [(
        "gate[t * k + j] = static_cast<float>(std::exp(static_cast<double>(h[e]) - m) / z);",
        "gate[t * k + j] = static_cast<float>(std::exp(static_cast<double>(h[e])) / z);")],
    "gate_renormalised_over_topk": [(
        "gate[t * k + j] = static_cast<float>(std::exp(static_cast<double>(h[e]) - m) / z);",
        "double zk = 0.0; for (int32_t i = 0; i < k; ++i) "
        "zk += std::exp(static_cast<double>(h[order[i]]) - m); "
        "gate[t * k + j] = static_cast<float>(std::exp(static_cast<double>(h[e]) - m) / zk);")],
    "capacity_ceil": [(
        "std::floor(static_cast<double>(T) / E * capacity_factor)",
        "std::ceil(static_cast<double>(T) / E * capacity_factor)")],
    "kept_off_by_one": [(
        "kept[t * k + j] = s < C ? 1 : 0;", "kept[t * k + j] = s <= C ? 1 : 0;")],
    "slots_from_one": [("int32_t s = arrivals[e]++;", "int32_t s = ++arrivals[e];")],
    "router_drops_bias": [(
        "if (bias) s += static_cast<double>(bias[e]);", "(void)bias;")],
    "router_transposed_weight": [(
        "s += load(x, t * d + c, dtype) * load(Wr, static_cast<int64_t>(e) * d + c, dtype);",
        "s += load(x, t * d + c, dtype) * load(Wr, static_cast<int64_t>(c) * E + e, dtype);")],
    "no_relu": [(
        "H[n] = store(hdst, n, dtype, a > 0.0 ? a : 0.0);", "H[n] = store(hdst, n, dtype, a);")],
    "hidden_not_rounded": [(
        "H[n] = store(hdst, n, dtype, a > 0.0 ? a : 0.0);",
        "store(hdst, n, dtype, a > 0.0 ? a : 0.0); H[n] = a > 0.0 ? a : 0.0;")],
    "ffn_uses_expert_0_W2": [(
        "                      static_cast<const char*>(W2) + e * d * f * es,",
        "                      static_cast<const char*>(W2),")],
    "dispatch_first_row_only": [(
        "int64_t t = tok_of_row[static_cast<int64_t>(e) * C + r];",
        "int64_t t = tok_of_row[static_cast<int64_t>(e) * C];")],
    "combine_without_gate": [(
        "s += static_cast<double>(gate[t * k + j]) * load(ye, row * d + c, dtype);",
        "s += load(ye, row * d + c, dtype);")],
    "combine_keeps_dropped": [(
        "        if (!kept[t * k + j]) continue;\n"
        "        int64_t row = static_cast<int64_t>(expert_idx[t * k + j]) * C + slot[t * k + j];",
        "        if (C == 0) continue;\n"
        "        int64_t row = static_cast<int64_t>(expert_idx[t * k + j]) * C +"
        " std::min(slot[t * k + j], C - 1);")],
    "splitmix_counter_from_zero": [(
        "uint64_t z = seed + (t + 1) * 0x9E3779B97F4A7C15ULL;",
        "uint64_t z = seed + t * 0x9E3779B97F4A7C15ULL;")],
    "rre_groups_interleaved": [(
        "expert_idx[t] = domain[t] * per + static_cast<int32_t>(r % static_cast<uint64_t>(per));",
        "expert_idx[t] = domain[t] + G * static_cast<int32_t>(r % static_cast<uint64_t>(per));")],
    "bf16_truncates": [(
        "double r = std::nearbyint(scaled);", "double r = std::trunc(scaled);")],
    "sparseclip_kappa_not_squared": [(
        "return std::sqrt(sd + kappa * kappa * ss);", "return std::sqrt(sd + kappa * ss);")],
    "sparseclip_scales_up": [(
        "const double coef = norm > max_norm ? max_norm / norm : 1.0;",
        "const double coef = max_norm / norm;")],
    "aux_without_expert_count": [(
        "out[0] = alpha * E * dot;", "out[0] = alpha * dot;")],
    "aux_tie_to_higher_index": [(
        "if (h[e] > h[best]) best = e;", "if (h[e] >= h[best]) best = e;")],
    "entropy_in_bits": [(
        "if (p[e] > 0.0) ht -= p[e] * std::log(p[e]);",
        "if (p[e] > 0.0) ht -= p[e] * std::log2(p[e]);")],
    "geglu_gate_and_linear_swapped": [
        ("g += xv * load(W1, static_cast<int64_t>(2 * i) * d + c, dtype);",
         "g += xv * load(W1, static_cast<int64_t>(2 * i + 1) * d + c, dtype);"),
        ("l += xv * load(W1, static_cast<int64_t>(2 * i + 1) * d + c, dtype);",
         "l += xv * load(W1, static_cast<int64_t>(2 * i) * d + c, dtype);")],
    "gelu_tanh_approximation": [(
        "const double gelu = 0.5 * g * (1.0 + std::erf(g / std::sqrt(2.0)));",
        "const double gelu = 0.5 * g * (1.0 + std::tanh(0.7978845608028654 * "
        "(g + 0.044715 * g * g * g)));")],
}


def _run_mutant(name, edits, tmp):
    src = open(SRC).read()
    for old, new in edits:
        assert src.count(old) == 1, f"{name}: the text to replace must occur once: {old!r}"
        src = src.replace(old, new)
    d = os.path.join(tmp, name)
    os.makedirs(d)
    cpp, so = os.path.join(d, "m.cpp"), os.path.join(d, "libm.so")
    open(cpp, "w").write(src)
    subprocess.run(["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-shared", "-fPIC",
                    "-pthread", cpp, "-o", so], check=True, capture_output=True)
    env = dict(os.environ, MOE_ORACLE_LIB=so)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode, r.stdout[-2000:]


def test_every_planted_mistake_fails_a_pin():
    tmp = os.path.join(ROOT, "_build", "oracle_mutants")  # a build folder, kept out of git
    shutil.rmtree(tmp, ignore_errors=True)
    os.makedirs(tmp)
    workers = max(1, min(8, (os.cpu_count() or 2) // 2))
    with cf.ThreadPoolExecutor(workers) as ex:
        futs = {n: ex.submit(_run_mutant, n, e, tmp) for n, e in MUTANTS.items()}
        results = {n: f.result() for n, f in futs.items()}
    shutil.rmtree(tmp, ignore_errors=True)
    survivors = {n: out for n, (rc, out) in results.items() if rc == 0}
    assert not survivors, "mutants that pass every pin:\n" + "\n".join(
        f"--- {n}\n{out}" for n, out in survivors.items())
    # a failure must be a failed pin, not a crash of the harness
    for n, (rc, out) in results.items():
        assert rc == 1, f"{n}: pytest exit {rc}\n{out}"


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutation_text_is_present(name):
    src = open(SRC).read()
    for old, _ in MUTANTS[name]:
        assert src.count(old) == 1, (name, old)
