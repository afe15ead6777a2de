"""Mutation tests of the oracle's pins.

Each case plants one plausible slip in a copy of the oracle's C sources (a dropped
rounding, a rounding taken another way, a wrong sign, index, group size, offset or
operand), builds the copy with the oracle's own compiler flags, and runs the pin
files (tests/test_oracle_pins*.py) against it in a
fresh process (the oracle package loads
the library named by SAGE_ORACLE_LIB).  The pins must fail on every mutant, and
pass on an unmodified copy built the same way (the control case), so a pin that
cannot tell a slip from the reading it pins shows up here.

The readings pinned are those of the SageAttention summary page (Summary bullets
1-2: INT8 Q.K^T after smoothing K, P.V in fp16; idea I1: the K shift) and of the
SageAttention2 abstract for the FP8 P.V variant (E4M3 P~ and V, V smoothing) and of
the SpargeAttn abstract for the block-sparse variant (predicted map, softmax-aware skip) and
of the SageAttention3 abstract for the microscaling FP4 variant (E2M1 codes, UE4M3 scales).
"""
import concurrent.futures
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRCS = {f: os.path.join(ROOT, "oracle", f) for f in ("sage_oracle.c", "sage_oracle_sa2.c", "sage_oracle_sparse.c",
                                                        "sage_oracle_sa3.c")}
PINS = [os.path.join(ROOT, "tests", f) for f in ("test_oracle_pins.py", "test_oracle_pins_fp8.py",
                                                 "test_oracle_pins_sparse.py", "test_oracle_pins_fp4.py")]

# (name, text in sage_oracle.c, replacement, expected number of occurrences)
BASE_MUTATIONS = [
    ("p_unrounded", "const double pt = h2d(d2h(e));", "const double pt = e;", 1),
    ("p_rounded_via_fp32", "const double pt = h2d(d2h(e));", "const double pt = h2d(d2h((double)(float)e));", 1),
    ("row_sum_of_rounded_p", "l += e;\n        const double pt = h2d(d2h(e));",
     "const double pt = h2d(d2h(e));\n        l += pt;", 1),
    ("scale_by_reciprocal", "*s = a / 127.0f;", "*s = a * (1.0f / 127.0f);", 1),
    ("inverse_of_scale", "*inv = 127.0f / a;", "*inv = 1.0f / (a / 127.0f);", 1),
    ("codes_ties_away", "float r = nearbyintf(y);", "float r = roundf(y);", 1),
    ("codes_truncated", "float r = nearbyintf(y);", "float r = truncf(y);", 1),
    ("smoothing_sign", "if (mu) x = x - mu[bh * d + c];", "if (mu) x = x + mu[bh * d + c];", 2),
    ("k_mean_over_n_minus_1", "float mean32 = sum32 / (float)N;", "float mean32 = sum32 / (float)(N - 1);", 1),
    ("k_mean_fp32_accumulator", "int64_t s = 0;", "float s = 0;", 1),
    ("causal_off_by_one", "causal ? i + 1 : N;\n    const int8_t* qi", "causal ? i : N;\n    const int8_t* qi", 1),
    ("sm_scale_dropped", "s[j] = (double)dot * sqi * (double)skh[j / gk] * sm_scale;",
     "s[j] = (double)dot * sqi * (double)skh[j / gk];", 1),
    ("key_scale_group_of_q", "(double)skh[j / gk]", "(double)skh[j / gq]", 1),
    ("query_scale_per_key", "const double sqi = (double)sqh[i / gq];", "const double sqi = (double)sqh[0];", 1),
    ("no_max_subtraction", "const double e = exp(s[j] - m);", "const double e = exp(s[j]);", 1),
    ("qk_uses_q_twice", "const int8_t* kj = k8 + (bh * N + j) * d;", "const int8_t* kj = q8 + (bh * N + j) * d;", 1),
    ("qk_int_transposed", "S[(bh * N + i) * N + j] = acc;", "S[(bh * N + j) * N + i] = acc;", 1),
    ("output_via_fp32", "if (o16) o16[i * d + c] = d2h(o);", "if (o16) o16[i * d + c] = d2h((double)(float)o);", 1),
    ("fp64_attention_no_scale", "s[j] = dot * sm_scale;", "s[j] = dot;", 1),
    ("fp64_attention_causal_off_by_one", "const int64_t jend = causal ? i + 1 : N;\n                    double m",
     "const int64_t jend = causal ? i + 2 : N;\n                    double m", 1),
]

# (name, text in sage_oracle_sa2.c, replacement, expected number of occurrences)
FP8_MUTATIONS = [
    ("fp8_p_unrounded", "const double pt = oracle_e4m3_decode(oracle_e4m3_encode(p));", "const double pt = p;", 1),
    ("fp8_p_as_fp16", "const double pt = oracle_e4m3_decode(oracle_e4m3_encode(p));",
     "const double pt = (double)(_Float16)p;", 1),
    ("fp8_offset_exact_max", "const double M = ceil(umax);", "const double M = umax;", 1),
    ("fp8_offset_floor", "const double M = ceil(umax);", "const double M = floor(umax);", 1),
    ("fp8_row_sum_of_rounded", "l += p;\n        const double pt = oracle_e4m3_decode(oracle_e4m3_encode(p));",
     "const double pt = oracle_e4m3_decode(oracle_e4m3_encode(p));\n        l += pt;", 1),
    ("fp8_v_int8_range", "s = a / 448.0f;\n                inv = 448.0f / a;",
     "s = a / 127.0f;\n                inv = 127.0f / a;", 1),
    ("fp8_v_mean_not_added", "+ (vmh ? (double)vmh[c] : 0.0)", "", 1),
    ("fp8_v_smoothing_sign", "(float)h2d_sa2(vh[t * d + c]) - mean;", "(float)h2d_sa2(vh[t * d + c]) + mean;", 2),
    ("fp8_v_scale_not_applied", "acc[c] * (double)svh[c] / l", "acc[c] / l", 1),
    ("e4m3_ties_away", "double m = nearbyint(ldexp(a, 3 - eb));", "double m = round(ldexp(a, 3 - eb));", 1),
    ("e4m3_subnormal_step", "nearbyint(ldexp(a, 9))", "nearbyint(ldexp(a, 10))", 1),
    ("e4m3_nan_not_saturated", "return sign | 0x7E; /* 448", "return sign | 0x7F; /* 448", 1),
    ("e4m3_decode_bias", "ldexp(1.0 + F / 8.0, E - 7)", "ldexp(1.0 + F / 8.0, E - 8)", 1),
]

# (name, text in sage_oracle_sparse.c, replacement, expected number of occurrences)
SPARSE_MUTATIONS = [
    ("sparse_sort_ascending", "(p[order[b - 1]] < p[a] ||", "(p[order[b - 1]] > p[a] ||", 1),
    ("sparse_no_causal_diagonal", "if (causal && (j + 1) * BK > i * BQ) mrow[j] = 1;", "", 1),
    ("sparse_similarity_override_inverted", "if (!q_alike || ks[j] < theta) mrow[j] = 1;",
     "if (!q_alike || ks[j] > theta) mrow[j] = 1;", 1),
    ("sparse_similarity_over_n", "return s2 / ((double)n * (double)n);", "return s2 / (double)n;", 1),
    ("sparse_sum_not_mean", "mean[c] /= (double)n;", "", 1),
    ("sparse_cut_one_short", "while (cut < nvis && cum < tau)", "while (cut < nvis && cum + p[order[cut]] < tau)", 1),
    ("sparse_last_visible_block_dropped", "const int64_t nvis = causal ? last_q / BK + 1 : NKB;",
     "const int64_t nvis = causal ? last_q / BK : NKB;", 1),
    ("stage2_lambda_sign", "if (!(m < mrun[i - r0] - lambda)) skip = 0;", "if (!(m < mrun[i - r0] + lambda)) skip = 0;", 1),
    ("stage2_running_max_starts_at_zero", "mrun[i - r0] = -INFINITY;", "mrun[i - r0] = 0.0;", 1),
    ("stage2_running_max_frozen", "if (bmax[i - r0] > mrun[i - r0]) mrun[i - r0] = bmax[i - r0];", ";", 1),
    ("stage2_skipped_keys_still_used", "            continue;\n        }\n        used[b] = 1;",
     "        }\n        used[b] = 1;", 1),
]

# (name, text in sage_oracle_sa3.c, replacement, expected number of occurrences)
FP4_MUTATIONS = [
    ("fp4_ties_to_odd", "(dk == db && (k & 1) == 0)", "(dk == db && (k & 1) == 1)", 1),
    ("fp4_negative_zero_unsigned", "const uint8_t sign = signbit(x) ? 8 : 0;", "const uint8_t sign = x < 0 ? 8 : 0;", 1),
    ("fp4_group_scale_over_4", "const float t = gm / 6.0f;", "const float t = gm / 4.0f;", 1),
    ("fp4_group_max_signed", "if (fabsf(z[i]) > gm) gm = fabsf(z[i]);", "if (z[i] > gm) gm = z[i];", 1),
    ("fp4_range_448", "#define FP4_RANGE 2688.0f", "#define FP4_RANGE 448.0f", 1),
    ("fp4_k_not_smoothed", "(km ? km[bh * d + c] : 0.0f)", "0.0f", 2),
    ("fp4_v_mean_added", "- mean) * r;", "+ mean) * r;", 1),
    ("fp4_p_shift_12", "#define P_SHIFT 10.0", "#define P_SHIFT 12.0", 1),
    ("fp4_frame_frozen", "if (mt > m) {", "if (m == -INFINITY) {", 1),
    ("fp4_row_sum_fp16_terms", "l += p[k];", "l += (double)(_Float16)p[k];", 1),
    ("fp4_channel_scale_dropped", "const double o = acc[c] * gvc / l", "const double o = acc[c] / l", 1),
    ("fp4_mean_not_added", "+ (h->vm ? (double)h->vm[c] : 0.0);", "+ 0.0;", 1),
    ("fp4_key_tile_scale_of_query", "(double)h->gk[j / FP4_TILE]", "(double)h->gk[i / FP4_TILE]", 1),
    ("fp4_causal_off_by_one", "const int64_t jend = h->causal ? i + 1 : N;", "const int64_t jend = h->causal ? i : N;", 1),
    ("fp4_envelope_dropped", "b = 2.0 * sd;  /* at most", "b = 0.0;  /* at most", 1),
    ("fp4_unsure_never", "if (fabs(tmax - nearbyint(tmax)) <= 1e-4) unsure = 1;", ";", 1),
]

MUTATIONS = ([("sage_oracle.c",) + m for m in BASE_MUTATIONS] + [("sage_oracle_sa2.c",) + m for m in FP8_MUTATIONS]
             + [("sage_oracle_sparse.c",) + m for m in SPARSE_MUTATIONS]
             + [("sage_oracle_sa3.c",) + m for m in FP4_MUTATIONS])

CFLAGS = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared"]


def _build_and_run_pins(fname, name, old, new, count, tmpdir):
    os.makedirs(os.path.join(tmpdir, name), exist_ok=True)
    c_paths = []
    for f, path in SRCS.items():
        src = open(path).read()
        if f == fname and old:  # the control case builds the unmodified texts
            assert src.count(old) == count, f"{name}: expected {count} occurrence(s) of the mutated text"
            src = src.replace(old, new)
        c_paths.append(os.path.join(tmpdir, name, f))
        with open(c_paths[-1], "w") as fh:
            fh.write(src)
    so_path = os.path.join(tmpdir, name, "lib_oracle.so")
    subprocess.run(CFLAGS + ["-o", so_path, *c_paths, "-lm"], check=True, capture_output=True)
    env = dict(os.environ, SAGE_ORACLE_LIB=so_path, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", *PINS, "-x", "-q", "-p", "no:cacheprovider"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode, r.stdout[-2000:] + r.stderr[-2000:]


def test_pins_fail_on_every_mutant_and_pass_on_the_control(tmp_path):
    jobs = [("sage_oracle.c", "control", "", "", 0)] + MUTATIONS
    with concurrent.futures.ThreadPoolExecutor(max_workers=max(2, min(8, os.cpu_count() or 2))) as ex:
        futs = {name: ex.submit(_build_and_run_pins, f, name, old, new, cnt, str(tmp_path))
                for f, name, old, new, cnt in jobs}
        results = {name: fu.result() for name, fu in futs.items()}
    rc, out = results.pop("control")
    assert rc == 0, f"the unmodified oracle must pass its pins:\n{out}"
    survivors = {name: out for name, (rc, out) in results.items() if rc != 1}
    # pytest exits 1 when a test failed; anything else (0 = all passed, a crash) is a survivor
    assert not survivors, "mutants the pins did not catch: " + ", ".join(
        f"{n} (exit {results[n][0]})" for n in survivors)


@pytest.mark.parametrize("fname,name,old,new,count", MUTATIONS, ids=[m[1] for m in MUTATIONS])
def test_mutation_targets_exist(fname, name, old, new, count):
    # the planted slips refer to the oracle's current text (a refactor must update them)
    assert open(SRCS[fname]).read().count(old) == count
