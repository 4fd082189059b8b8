"""The pins are strong enough to catch plausible mistakes in the oracle.

Each mutant below is one plausible slip in ``oracle/spec_verify_oracle.c``: a
transposed or non-strict comparison, a flipped sign, a wrong index, a dropped
step, a processor applied in the wrong order.  The test applies it to a copy
of the source, builds the copy with gcc, and runs the pin files against it
(through ``SV_ORACLE_LIB``).  At least one pin must fail for every mutant; the
unaltered copy must pass.  Left out are slips that would read out of bounds
(undefined behaviour proves nothing) and slips that change nothing a float32
input can reach:
  * the max subtracted before the exponential (exact arithmetic is unchanged);
  * drawing from the draft row instead of the target row when the residual
    max(0, p - q) has no mass: then p <= q everywhere and both sum to 1, so
    p = q and the two draws agree;
  * the nucleus reaching top_p with ">" instead of ">=": the two differ only
    when an fp64 running sum of exponentials equals a float32 top_p exactly,
    which no float32 logit row gives dependably;
  * the tree residual's mass taken as the sum of max(0, q - R) instead of
    max(0, R - q): R and q both sum to 1, so the two sums are equal.
"""
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "spec_verify_oracle.c")
PIN_FILES = ["tests/test_oracle.py", "tests/test_oracle_processors.py", "tests/test_oracle_tree.py",
             "tests/test_oracle_head.py"]

# (name, text, replacement, which occurrence of text)
MUTANTS = [
    # acceptance rule R1, in the plain and in the processor variant
    ("accept_transposed", "(double)u[i] * q < p", "(double)u[i] * p < q", 0),
    ("accept_transposed_procs", "(double)u[i] * q < p", "(double)u[i] * p < q", 1),
    ("accept_non_strict", "(double)u[i] * q < p", "(double)u[i] * q <= p", 0),
    ("accept_non_strict_procs", "(double)u[i] * q < p", "(double)u[i] * q <= p", 1),
    # residual max(0, p - q)
    ("residual_sign", "double r = pt[(size_t)j * V + v] - pd[(size_t)j * V + v];",
     "double r = pd[(size_t)j * V + v] - pt[(size_t)j * V + v];", 0),
    ("residual_sign_procs", "double r = pt[(size_t)j * V + v] - pd[(size_t)j * V + v];",
     "double r = pd[(size_t)j * V + v] - pt[(size_t)j * V + v];", 1),
    ("residual_absolute", "w[v] = r > 0.0 ? r : 0.0;", "w[v] = r > 0.0 ? r : -r;", 0),
    ("residual_absolute_procs", "w[v] = r > 0.0 ? r : 0.0;", "w[v] = r > 0.0 ? r : -r;", 1),
    # R2: the final draw takes u_k
    ("residual_uniform_index", "oracle_inverse_cdf(w, V, (double)u[k]", "oracle_inverse_cdf(w, V, (double)u[j]", 0),
    ("residual_uniform_index_procs", "oracle_inverse_cdf(w, V, (double)u[k]",
     "oracle_inverse_cdf(w, V, (double)u[j]", 1),
    ("bonus_uniform_index", "oracle_inverse_cdf(pt + (size_t)k * V, V, (double)u[k]",
     "oracle_inverse_cdf(pt + (size_t)k * V, V, (double)u[0]", 0),
    ("bonus_uniform_index_procs", "oracle_inverse_cdf(pt + (size_t)k * V, V, (double)u[k]",
     "oracle_inverse_cdf(pt + (size_t)k * V, V, (double)u[0]", 1),
    # R4: top-k threshold and ties
    ("top_k_off_by_one", "tau = work[top_k - 1];", "tau = work[top_k];", 0),
    ("top_k_off_by_one_procs", "tau = work[top_k - 1];", "tau = work[top_k];", 1),
    ("top_k_drops_ties", "prob[v] = (z >= tau) ?", "prob[v] = (z > tau) ?", 0),
    ("top_k_drops_ties_procs", "prob[v] = (z >= tau) ?", "prob[v] = (z > tau) ?", 1),
    # R5: temperature divides
    ("temperature_multiplies", "exp(z / T - m)", "exp(z * T - m)", 0),
    ("temperature_multiplies_procs", "exp(z / T - m)", "exp(z * T - m)", 1),
    # R6: greedy
    ("argmax_highest_index", "if (z > bv) {", "if (z >= bv) {", 0),
    ("greedy_last_mismatch", "} else if (i < k && j == k && d[i] != g) {", "} else if (i < k && d[i] != g) {", 0),
    ("greedy_bonus_overrides", "} else if (i == k && j == k) {", "} else if (i == k) {", 0),
    # R3: inverse CDF
    ("inverse_cdf_non_strict", "if (C > x) {", "if (C >= x) {", 0),
    ("inverse_cdf_lo_point", "*cdf_lo = prev / W;", "*cdf_lo = C / W;", 0),
    ("sampler_reflected_uniform", "oracle_inverse_cdf(prob, V, (double)u[r],", "oracle_inverse_cdf(prob, V, 1.0 - (double)u[r],", 0),
    # R7: row errors
    ("inf_logit_accepted", "if (isnan(z) || z == INFINITY) return 1;", "if (isnan(z)) return 1;", 0),
    ("uniform_one_accepted", "if (!(u[i] >= 0.0f && u[i] < 1.0f)) err = 1;",
     "if (!(u[i] >= 0.0f && u[i] <= 1.0f)) err = 1;", 0),
    ("uniform_one_accepted_procs", "if (!(u[i] >= 0.0f && u[i] < 1.0f)) err = 1;",
     "if (!(u[i] >= 0.0f && u[i] <= 1.0f)) err = 1;", 1),
    # outputs and layout
    ("out_p_is_q", "if (out_p) out_p[(size_t)b * k + i] = p;", "if (out_p) out_p[(size_t)b * k + i] = q;", 0),
    ("f32_row_stride", "size_t elt = dtype == OR_DTYPE_BF16 ? 2 : (dtype == OR_DTYPE_F64 ? 8 : 4);",
     "size_t elt = dtype == OR_DTYPE_BF16 ? 2 : (dtype == OR_DTYPE_F64 ? 8 : 2);", 0),
    ("f64_row_stride", "size_t elt = dtype == OR_DTYPE_BF16 ? 2 : (dtype == OR_DTYPE_F64 ? 8 : 4);",
     "size_t elt = dtype == OR_DTYPE_BF16 ? 2 : 4;", 0),
    # R13 repetition penalty
    ("penalty_ignores_sign", "z = z > 0.0 ? (double)(float)(z / pr->rep_penalty) : (double)(float)(z * pr->rep_penalty);",
     "z = (double)(float)(z / pr->rep_penalty);", 0),
    ("penalty_not_rounded", "z = z > 0.0 ? (double)(float)(z / pr->rep_penalty) : (double)(float)(z * pr->rep_penalty);",
     "z = z > 0.0 ? z / pr->rep_penalty : z * pr->rep_penalty;", 0),
    ("penalty_infinite_accepted", "!(pr->rep_penalty > 0.0) || isinf(pr->rep_penalty)", "!(pr->rep_penalty > 0.0)", 0),
    ("penalty_per_listing", "break; /* each id once */", "/* every listing */", 0),
    ("penalty_ids_of_first_sequence", "pr.rep_ids = rep_ids ? rep_ids + (size_t)b * n_rep : NULL;",
     "pr.rep_ids = rep_ids;", 0),
    # R14 vocabulary mask
    ("mask_bit_order", "(pr->mask[v / 32] >> (v % 32)) & 1u", "(pr->mask[v / 32] >> (31 - v % 32)) & 1u", 0),
    ("mask_of_first_sequence", "pr.mask = mask ? mask + (size_t)b * words : NULL;", "pr.mask = mask;", 0),
    # R12 order: processors before top-k
    ("top_k_before_processors", "work[v] = or_logit_procs(row, dtype, v, pr);", "work[v] = z0;", 0),
    # R15 nucleus
    ("nucleus_drops_ties", "if (!(prob[v] >= cut)) prob[v] = 0.0;", "if (!(prob[v] > cut)) prob[v] = 0.0;", 0),
    ("nucleus_no_renormalise", "for (v = 0; v < V; ++v) prob[v] /= K2;", "(void)K2;", 0),
    ("nucleus_one_past", "cut = pv[i].p;", "cut = pv[i + 1 < n ? i + 1 : i].p;", 0),
    ("top_p_of_first_sequence", "pr.top_p = top_p ? (double)top_p[b] : 1.0;", "pr.top_p = top_p ? (double)top_p[0] : 1.0;", 0),
    ("proposer_processors_of_first_sequence", "const int s = r / rows_per_seq;", "const int s = 0 * rows_per_seq;", 0),
    # R18 tree verification
    ("tree_accept_transposed", "if ((double)u[c - 1] * q < r) {", "if ((double)u[c - 1] * r < q) {", 0),
    ("tree_accept_non_strict", "if ((double)u[c - 1] * q < r) {", "if ((double)u[c - 1] * q <= r) {", 0),
    ("tree_child_uniform_index", "if ((double)u[c - 1] * q < r) {", "if ((double)u[c] * q < r) {", 0),
    ("tree_residual_not_renormalised", "R[v] = (R[v] > Q[v]) ? (R[v] - Q[v]) / W : 0.0;",
     "R[v] = (R[v] > Q[v]) ? (R[v] - Q[v]) : 0.0;", 0),
    ("tree_residual_never_taken", "if (W > 0.0)\n", "if (W < 0.0)\n", 0),
    ("tree_children_last_first", "for (c = a + 1; c <= N && !next; ++c) {\n                    double r, q, W = 0.0;",
     "for (c = N; c > a && !next; --c) {\n                    double r, q, W = 0.0;", 0),
    ("tree_final_uniform_index", "oracle_inverse_cdf(R, V, (double)u[N], &y, &lo, &hi);",
     "oracle_inverse_cdf(R, V, (double)u[0], &y, &lo, &hi);", 0),
    ("tree_rows_of_the_parent", "const long row = (long)b * (N + 1) + a;",
     "const long row = (long)b * (N + 1) + (a > 0 ? par[a - 1] : 0);", 0),
    ("tree_greedy_any_child", "if (par[c - 1] == a && t[c - 1] == g) next = c;", "if (par[c - 1] == a) next = c;", 0),
    ("tree_parent_not_checked", "|| par[i] < 0 || par[i] > i) err = 1;", "|| par[i] < 0 || par[i] > i + 1) err = 1;", 0),
    ("tree_out_p_is_q", "if (out_p) out_p[(size_t)b * N + c - 1] = r;", "if (out_p) out_p[(size_t)b * N + c - 1] = q;", 0),
    # the output projection and the fp64 rows it feeds to greedy verification
    ("head_skips_last_term", "for (j = 0; j < H; ++j) {\n                double t",
     "for (j = 0; j + 1 < H; ++j) {\n                double t", 0),
    ("head_weight_row_stride", "const void* w = weight + (size_t)v * (size_t)H;",
     "const void* w = weight + (size_t)v * (size_t)(H - 1);", 0),
    ("head_hidden_row_stride", "const void* h = hidden + (size_t)r * (size_t)H;",
     "const void* h = hidden + (size_t)r * (size_t)(H - 1);", 0),
    ("head_abs_signed", "a += fabs(t);", "a += t;", 0),
    ("head_columns_reversed", "out_z[(size_t)(r - row0) * (size_t)V + v] = z;",
     "out_z[(size_t)(r - row0) * (size_t)V + (V - 1 - v)] = z;", 0),
    ("f64_rows_read_as_float", "if (dtype == OR_DTYPE_F64) return ((const double*)row)[v];",
     "if (dtype == OR_DTYPE_F64) return (double)((const float*)row)[2 * v];", 0),
]


def _mutate(src: str, text: str, repl: str, which: int) -> str:
    pos = -1
    for _ in range(which + 1):
        pos = src.find(text, pos + 1)
        assert pos >= 0, f"mutation site {text!r} #{which} not found in the oracle source"
    return src[:pos] + repl + src[pos + len(text):]


def _build(src: str, out_dir: str, name: str) -> str:
    c = os.path.join(out_dir, name + ".c")
    so = os.path.join(out_dir, name + ".so")
    with open(c, "w") as f:
        f.write(src)
    # the flags of the oracle's own build
    subprocess.run(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
                    "-o", so, c, "-lm"], check=True, capture_output=True)
    return so


def _run_pins(so: str) -> int:
    env = dict(os.environ, SV_ORACLE_LIB=so, PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-m", "pytest", *PIN_FILES, "-x", "-q", "-m", "not gpu",
                        "-p", "no:cacheprovider"], cwd=ROOT, env=env, capture_output=True, timeout=600)
    return r.returncode


def test_every_mutant_is_caught_by_a_pin(tmp_path):
    if shutil.which("gcc") is None:
        pytest.fail("gcc is needed to build the oracle")
    src = open(SRC).read()
    jobs = {"unaltered": _build(src, str(tmp_path), "unaltered")}
    names = [m[0] for m in MUTANTS]
    assert len(set(names)) == len(names)
    for name, text, repl, which in MUTANTS:
        jobs[name] = _build(_mutate(src, text, repl, which), str(tmp_path), name)
    with ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as pool:
        codes = dict(zip(jobs, pool.map(_run_pins, jobs.values())))
    assert codes.pop("unaltered") == 0, "the pins fail on an unaltered copy of the oracle"
    survivors = sorted(n for n, rc in codes.items() if rc == 0)
    assert not survivors, f"no pin fails for these mutants: {survivors}"
