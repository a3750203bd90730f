"""Mutation check of the oracle's pins (CPU only).

Each case plants one plausible mistake in a copy of ``oracle/moe_oracle.cpp``
(a swapped operand, a dropped rounding, a wrong sign, a broken tie-break or
sort order, an off-by-one, a missing weight), compiles the copy and runs the
oracle pins against it through ``MOE_ORACLE_LIB``: at least one pin must fail.
The planted mistakes live only in the temporary copies."""

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "moe_oracle.cpp")
PINS = ["tests/test_oracle_mlp.py", "tests/test_oracle_formats.py", "tests/test_oracle_route_align.py",
        "tests/test_oracle_expert_parallel.py"]

# (name, text in the oracle, planted replacement)
MUTANTS = [
    ("gate_up_swapped", "double gate = s.h[i];\n    double up = s.h[I + i];",
     "double gate = s.h[I + i];\n    double up = s.h[i];"),
    ("silu_not_rounded", "const double act = round_bf16(gate / (1.0 + std::exp(-gate)));",
     "const double act = gate / (1.0 + std::exp(-gate));"),
    ("silu_sign", "const double act = round_bf16(gate / (1.0 + std::exp(-gate)));",
     "const double act = round_bf16(gate / (1.0 + std::exp(gate)));"),
    ("product_not_rounded", "s.p[i] = round_bf16(act * up);", "s.p[i] = act * up;"),
    ("gemm2_reads_unquantised", "y[n] = dot_row(w2, n, s.p_hat.data());", "y[n] = dot_row(w2, n, s.p.data());"),
    ("h_not_rounded", "s.h[n] = round_bf16(dot_row(w13, n, x_hat));", "s.h[n] = dot_row(w13, n, x_hat);"),
    ("tie_to_higher_index", "(best < 0 || l[e] > l[best])", "(best < 0 || l[e] >= l[best])"),
    ("no_renormalisation", "renormalize ? w / chosen_sum : w", "w"),
    ("align_descending_order", "for (int64_t f = 0; f < n; ++f)                        // ascending flat order",
     "for (int64_t f = n - 1; f >= 0; --f)"),
    ("align_padding_off_by_one", "(counts[e] + block_m - 1) / block_m * block_m;",
     "(counts[e] + block_m - 2) / block_m * block_m;"),
    ("combine_unweighted", "const double w = router_weight_on_input ? 1.0 : static_cast<double>(wts[t * topk + j]);",
     "const double w = 1.0;"),
    ("act_scale_not_pow2", "  return pow2_ceil(static_cast<double>(raw));", "  return static_cast<double>(raw);"),
    ("e4m3_ties_away", "  double r = std::ldexp(std::nearbyint(std::ldexp(x, -q)), q);",
     "  double r = std::ldexp(std::round(std::ldexp(x, -q)), q);"),
    ("weight_scale_448_off", "std::max(static_cast<float>(bmax), static_cast<float>(1e-10)) / 448.0f;",
     "std::max(static_cast<float>(bmax), static_cast<float>(1e-10)) / 440.0f;"),
    ("weight_scale_one_k_block", "acc += (kE4m3.v[r[k]] * static_cast<double>(s[k / 128])) * v[k];",
     "acc += (kE4m3.v[r[k]] * static_cast<double>(s[0])) * v[k];"),
    ("e8m0_bias", "constexpr int kE8m0Bias = 127;", "constexpr int kE8m0Bias = 126;"),
    ("x_not_quantised", "for (int j = 0; j < group; ++j) xh[g * group + j] = kE4m3.v[codes[j]] * scale;",
     "for (int j = 0; j < group; ++j) xh[g * group + j] = row[g * group + j];"),
    ("router_weight_on_input_ignored",
     "row[k] = round_bf16(static_cast<double>(static_cast<float>(row[k]) * w));   // one fp32 product",
     "row[k] = row[k] + 0.0 * w;"),
    ("shard_split_rounded_up", "first[r] = static_cast<int32_t>((static_cast<int64_t>(r) * E) / world);",
     "first[r] = static_cast<int32_t>((static_cast<int64_t>(r) * E + world - 1) / world);"),
]


def _cxx():
    for c in (shutil.which("g++"), os.environ.get("CXX"), "/usr/bin/g++"):
        if c and os.path.exists(c):
            return c
    return None


def _run_mutant(cxx, workdir, name, old, new):
    """Build the copy with one planted mistake and run the pins against it: (exit code, output tail)."""
    src = open(SRC).read()
    if src.count(old) != 1:
        return -100, f"{name}: the text to mutate must occur exactly once"
    d = os.path.join(workdir, name)
    os.makedirs(d, exist_ok=True)
    mutated = os.path.join(d, "moe_oracle.cpp")
    with open(mutated, "w") as f:
        f.write(src.replace(old, new))
    lib = os.path.join(d, "libmoe_oracle_mutant.so")
    res = subprocess.run([cxx, "-O1", "-std=c++17", "-fPIC", "-shared", "-ffp-contract=off", mutated, "-o", lib],
                         capture_output=True, text=True)
    if res.returncode != 0:
        return -101, res.stderr[-2000:]
    env = dict(os.environ, MOE_ORACLE_LIB=lib, OMP_NUM_THREADS="2")
    run = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-m", "not gpu", "-p", "no:cacheprovider",
                          *PINS], cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    return run.returncode, run.stdout[-2000:]


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    cxx = _cxx()
    if cxx is None:
        pytest.skip("no C++ compiler")
    work = str(tmp_path_factory.mktemp("mutants"))
    with cf.ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as ex:
        futs = {m[0]: ex.submit(_run_mutant, cxx, work, *m) for m in MUTANTS}
        return {k: f.result() for k, f in futs.items()}


@pytest.mark.parametrize("name", [m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(outcomes, name):
    rc, tail = outcomes[name]
    assert rc == 1, f"mutant {name}: pins exit code {rc} (1 = a pin failed):\n{tail}"
