"""Mutation check of the oracle's pins (CPU only).

Each case plants one plausible mistake in a private copy of the oracle's C
source (a flipped sign, a transposed or dropped index, a wrong tie rule, a
missing gate, an unstable sort, the wrong rounding), builds it with gcc, and
runs the pin tests against that build.  The pins must fail for every mutant;
the product code is never involved.
"""
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "adafuse_oracle.c")

MUTANTS = {
    "merge_gate_sign": (r"acc \+= g\[s\] \* d;", "acc -= g[s] * d;"),
    "merge_A_transposed": (r"A\[e \* a_es \+ \(int64_t\)j \* d_in \+ i\]\);\n                acc \+= g",
                           "A[e * a_es + (int64_t)i * r + j]);\n                acc += g"),
    "merge_drop_last_rank_term": (r"for \(int32_t j = 0; j < r; \+\+j\)\n                    d \+= orc_bf16_to_double\(B\[e \* b_es \+ o \* r \+ j\]\) \*\n                         orc_bf16_to_double\(A",
                                  "for (int32_t j = 0; j < r - 1; ++j)\n                    d += orc_bf16_to_double(B[e * b_es + o * r + j]) *\n                         orc_bf16_to_double(A"),
    "topk_tie_to_higher_index": (r"    return a < b;\n}", "    return a > b;\n}"),
    "router_bias_dropped": (r"            if \(br\) acc = acc \+ br\[e\];\n            z\[t \* E \+ e\] = acc;",
                            "            z[t * E + e] = acc;"),
    "softmax_always_renormalised": (r"if \(renorm\) for", "if (1) for"),
    "apply_gate_missing": (r"acc \+= gate\[t \* k \+ s\] \* d;", "acc += d;"),
    "apply_uses_W_transposed": (r"orc_bf16_to_double\(W\[o \* d_in \+ i\]\);",
                                "orc_bf16_to_double(W[(i % d_out) * d_in + (o % d_in)]);"),
    "segments_unstable": (r"    for \(int64_t p = 0; p < P; \+\+p\) \{\n        int32_t e = idx\[p\];\n        if \(e < 0 \|\| e >= E\) continue;",
                          "    for (int64_t p = P - 1; p >= 0; --p) {\n        int32_t e = idx[p];\n        if (e < 0 || e >= E) continue;"),
    "bf16_ties_away_from_zero": (r"double n = nearbyint\(a / q\);", "double n = round(a / q);"),
    "router_fused_multiply_add": (r"                float p = xj \* Wr\[\(int64_t\)e \* H \+ j\];\n                acc = acc \+ p;",
                                  "                acc = fmaf(xj, Wr[(int64_t)e * H + j], acc);"),
    "router_bias_added_first": [(r"            float acc = 0\.0f;\n            for \(int32_t j = 0; j < H; \+\+j\) \{\n                float xj",
                                 "            float acc = br ? br[e] : 0.0f;\n            for (int32_t j = 0; j < H; ++j) {\n                float xj"),
                                (r"            if \(br\) acc = acc \+ br\[e\];\n            z\[t \* E \+ e\] = acc;",
                                 "            z[t * E + e] = acc;")],
    "softmax_without_max_shift": (r"double m = -INFINITY;\n        for \(int e = 0; e < E; \+\+e\) if \(!isnan\(zt\[e\]\) && \(double\)zt\[e\] > m\) m = \(double\)zt\[e\];",
                                  "double m = 0.0;"),
    "topk_nan_ranks_first": (r"    if \(na\) return 0;\n    if \(nb\) return 1;", "    if (na) return 1;\n    if (nb) return 0;"),
    "pool_mean_divides_by_T_minus_1": (r"xbar\[j\] = acc / \(float\)T;", "xbar[j] = acc / (float)(T > 1 ? T - 1 : 1);"),
    "merge_gate_squared": (r"acc \+= g\[s\] \* d;", "acc += g[s] * g[s] * d;"),
    "apply_base_term_dropped": (r"            for \(int64_t i = 0; i < d_in; \+\+i\)\n                acc \+= orc_bf16_to_double\(x\[t \* d_in \+ i\]\) \* orc_bf16_to_double\(W\[o \* d_in \+ i\]\);",
                                "            (void)W;"),
    "apply_shrink_reads_token_0": (r"\* d_in \+ i\]\) \*\n                               orc_bf16_to_double\(x\[t \* d_in \+ i\]\);",
                                   "* d_in + i]) *\n                               orc_bf16_to_double(x[i]);"),
    "segments_count_shifted": (r"offsets\[e \+ 1\] \+= 1;", "offsets[e] += 1;"),
    "bf16_negative_zero_to_positive": (r"if \(signbit\(v\)\) f = -f;", "if (v < 0) f = -f;"),
    "apply_f64_partial_rounded": (r"if \(y64\) y64\[\(t - t0\) \* d_out \+ o\] = acc;",
                                  "if (y64) y64[(t - t0) * d_out + o] = orc_bf16_to_double(orc_bf16_from_double(acc));"),
}


def _apply(name):
    sites = MUTANTS[name]
    if isinstance(sites, tuple):
        sites = [sites]
    with open(SRC) as f:
        mutated = f.read()
    for pat, rep in sites:
        mutated, n = re.subn(pat, lambda m: rep, mutated, count=1)
        if n != 1:
            return None
    return mutated


def _run_pins_on(name, workdir):
    """Build the mutant oracle and run the pin tests against it: (applied,
    pytest return code, end of its output)."""
    mutated = _apply(name)
    if mutated is None:
        return False, None, ""
    d = workdir / name
    d.mkdir()
    csrc = d / "mutant.c"
    csrc.write_text(mutated)
    lib = d / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                           "-ffp-contract=off", "-o", str(lib), str(csrc), "-lm"])
    env = dict(os.environ, ADAFUSE_ORACLE_LIB=str(lib), OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return True, r.returncode, r.stdout[-2000:]


@pytest.fixture(scope="module")
def mutant_runs(tmp_path_factory):
    """Every mutant's pin run, several at a time (each is an independent
    process on its own copy of the oracle)."""
    from concurrent.futures import ThreadPoolExecutor
    work = tmp_path_factory.mktemp("mutants")
    names = sorted(MUTANTS)
    with ThreadPoolExecutor(max_workers=max(1, min(8, (os.cpu_count() or 2) // 2))) as ex:
        return dict(zip(names, ex.map(lambda n: _run_pins_on(n, work), names)))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, mutant_runs):
    applied, rc, out = mutant_runs[name]
    assert applied, f"mutation {name} did not apply"
    assert rc != 0, f"pins did not catch mutant {name}:\n{out}"
