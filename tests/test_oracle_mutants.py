"""Plant plausible mistakes in a copy of the oracle and check the pins catch them.

Each mutant is the oracle's C source with one textual slip (a dropped term, a
wrong sign, corner or index, a missing normalisation), compiled into a
throw-away library.  Every pin file of the oracle (PIN_FILES: the forward, the
split-KV order, and the next-row oracles) is then run against it in a fresh
interpreter and must fail.  The committed oracle itself is never modified.
"""
import concurrent.futures
import os
import subprocess
import sys
import textwrap

import pytest

from oracle import build as obuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = {
    "dropped_scale": [("? scale * dot_qk(q, k, b, h, i, j, H, Nq, Nk, d)\n                                    : -INFINITY;\n        for (long i = 0; i < Nq; ++i) {",
                       "? dot_qk(q, k, b, h, i, j, H, Nq, Nk, d)\n                                    : -INFINITY;\n        for (long i = 0; i < Nq; ++i) {")],
    "top_left_mask": [("if (causal && j > i + (Nk - Nq)) return 0;", "if (causal && j > i) return 0;")],
    "flipped_mask": [("if (causal && j > i + (Nk - Nq)) return 0;", "if (causal && j < i + (Nk - Nq)) return 0;")],
    "no_max_in_exp": [("Si[j] = (Si[j] == -INFINITY) ? 0.0 : exp(Si[j] - m);   /* Si now holds p_ij */",
                       "Si[j] = (Si[j] == -INFINITY) ? 0.0 : exp(Si[j]);   /* Si now holds p_ij */")],
    "lse_without_max": [("lse[((long)b * H + h) * Nq + i] = m + log(l);\n        }\n        free(S);",
                         "lse[((long)b * H + h) * Nq + i] = log(l);\n        }\n        free(S);")],
    "v_column_index": [("acc += Si[j] * v[IDX4(b, j, h, t, Nk, H, d)];",
                        "acc += Si[j] * v[IDX4(b, j, h, 0, Nk, H, d)];")],
    "key_head_index": [("const double* kj = k + IDX4(b, j, h, 0, Nk, H, d);",
                        "const double* kj = k + IDX4(b, j, 0, 0, Nk, H, d);")],
    "missing_normalisation": [("oi[t] = acc / l;", "oi[t] = acc;")],
    "blocked_l_not_rescaled": [("l[r] = alpha * l[r] + bsum;", "l[r] = l[r] + bsum;")],
    "blocked_acc_not_rescaled": [("for (int t = 0; t < d; ++t) acc[r * d + t] *= alpha;",
                                  "for (int t = 0; t < d; ++t) acc[r * d + t] *= 1.0;")],
    # the relative-position term of oracle_attn_fwd_relpos_f64
    "relpos_term_unscaled": [("S[i * Nk + j] = scale * (dot_qk(q, k, b, h, i, j, H, Nq, Nk, d) + rel);",
                              "S[i * Nk + j] = scale * dot_qk(q, k, b, h, i, j, H, Nq, Nk, d) + rel;")],
    "relpos_dist_transposed": [("const double* e = emb + (long)dist[i * Nk + j] * d;",
                                "const double* e = emb + (long)dist[(j % Nq) * Nk + (i % Nk)] * d;")],
    "relpos_term_uses_key": [("for (int t = 0; t < d; ++t) rel += qi[t] * e[t];",
                              "for (int t = 0; t < d; ++t) rel += k[IDX4(b, j, h, t, Nk, H, d)] * e[t];")],
    "relpos_term_dropped": [("S[i * Nk + j] = scale * (dot_qk(q, k, b, h, i, j, H, Nq, Nk, d) + rel);",
                             "S[i * Nk + j] = scale * (dot_qk(q, k, b, h, i, j, H, Nq, Nk, d) + 0.0 * rel);")],
    # the backward oracle
    "bwd_no_delta": [("const double ds = P[i * Nk + j] * (dP[i * Nk + j] - delta);",
                      "const double ds = P[i * Nk + j] * dP[i * Nk + j];")],
    "bwd_dq_unscaled": [("dqi[t] += scale * ds * krow[t];", "dqi[t] += ds * krow[t];")],
    "bwd_dk_uses_key": [("dkj[t] += scale * ds * qi[t];", "dkj[t] += scale * ds * krow[t];")],
    "bwd_dv_transposed": [("dvj[t] += pij * doi[t];", "dvj[t] += pij * vj[t];")],
    # the split-KV (decode) ordering
    "splitkv_l_not_rescaled": [("if (part_m[sp] != -INFINITY) big_l += part_l[sp] * exp(part_m[sp] - big_m);",
                                "if (part_m[sp] != -INFINITY) big_l += part_l[sp];")],
    "splitkv_o_not_rescaled": [("num += part_o[(long)sp * d + t] * exp(part_m[sp] - big_m);",
                                "num += part_o[(long)sp * d + t];")],
    "splitkv_lse_without_max": [("*lse_row = big_m + log(big_l);", "*lse_row = log(big_l);")],
    "splitkv_range_end_short": [("const long j_hi = (j_lo + span < Nk) ? j_lo + span : Nk;",
                                 "const long j_hi = (j_lo + span < Nk) ? j_lo + span - 1 : Nk;")],
    # the paged-cache, multi-query oracle
    "paged_top_left": [("if (causal && j > i + (L - Lq)) {", "if (causal && j > i) {")],
    "paged_row_in_page_dropped": [("const long slot = page * page_size + j % page_size;\n                const double* krow",
                                   "const long slot = page * page_size;\n                const double* krow")],
    "paged_head_offset_dropped": [("const double* krow = k_cache + (slot * H + h) * d;",
                                   "const double* krow = k_cache + (slot * H) * d;")],
    "paged_values_from_keys": [("sum_wv += w[j] * v_cache[(slot * H + h) * d + t];",
                                "sum_wv += w[j] * k_cache[(slot * H + h) * d + t];")],
    "paged_lse_without_max": [("*lse_bhi = top + log(total);", "*lse_bhi = log(total);")],
    # the lightning-indexer score and top-k
    "indexer_relu_dropped": [("const double relu = dotp > 0.0 ? dotp : 0.0;", "const double relu = dotp;")],
    "indexer_relu_after_sum": [("const double relu = dotp > 0.0 ? dotp : 0.0;", "const double relu = dotp;"),
                               ("if (mask) acc += mask[(b * T + t) * P + p];",
                                "if (acc < 0.0) acc = 0.0;\n            if (mask) acc += mask[(b * T + t) * P + p];")],
    "indexer_weight_transposed": [("acc += w[(b * T + t) * H + h] * relu;",
                                   "acc += w[(b * H + h) * T + t] * relu;")],
    "indexer_mask_dropped": [("if (mask) acc += mask[(b * T + t) * P + p];", "if (!mask) acc += 0.0;")],
    "indexer_key_batch": [("const double* key = kp + (b * P + p) * d;", "const double* key = kp + p * d;")],
    "topk_ties_last": [("if (best < 0 || srow[j] > srow[best]) best = j;",
                        "if (best < 0 || srow[j] >= srow[best]) best = j;")],
    "topk_keeps_neg_inf": [("if (taken[j] || !(srow[j] > -INFINITY)) continue;  /* skips -inf and NaN */",
                            "if (taken[j]) continue;")],
}

PIN_FILES = [os.path.join(ROOT, "tests", "test_oracle.py"),
             os.path.join(ROOT, "tests", "test_oracle_relpos.py"),
             os.path.join(ROOT, "tests", "test_oracle_bwd.py"),
             os.path.join(ROOT, "tests", "test_oracle_indexer.py"),
             os.path.join(ROOT, "tests", "test_oracle_paged.py"),
             os.path.join(ROOT, "tests", "test_oracle_splitkv.py")]

PIN_FIRST = {"relpos": "test_oracle_relpos.py", "bwd": "test_oracle_bwd.py",
             "indexer": "test_oracle_indexer.py", "topk": "test_oracle_indexer.py",
             "paged": "test_oracle_paged.py", "splitkv": "test_oracle_splitkv.py"}

RUNNER = textwrap.dedent("""
    import sys
    sys.path.insert(0, {root!r})
    import oracle
    from oracle import build
    lib = oracle.load({lib!r})
    oracle._lib, oracle._lib_path = lib, build.LIB
    import pytest
    sys.exit(pytest.main(["-x", "-q", "-p", "no:cacheprovider"] + {tests!r}))
""")


def _run_pins(lib, tests, cwd):
    env = dict(os.environ, OMP_NUM_THREADS="1")
    code = RUNNER.format(root=ROOT, lib=lib, tests=tests)
    return subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                          cwd=str(cwd), timeout=600, env=env)


def _run_mutant(name, workdir):
    """Build mutant `name` and run every pin file against it; returns (error, result)."""
    src = open(obuild.SRC).read()
    for old, new in MUTANTS[name]:
        if src.count(old) != 1:
            return f"mutation anchor for {name} not unique/present", None
        src = src.replace(old, new)
    mpath = workdir / f"{name}.c"
    mpath.write_text(src)
    lib = obuild.build(src=str(mpath), out=str(workdir / f"lib{name}.so"))
    # the pin file written for the mutated function goes first, so that the run (which
    # stops at the first failure) ends early
    first = [f for f in PIN_FILES if os.path.basename(f) == PIN_FIRST.get(name.split("_")[0])]
    return None, _run_pins(lib, first + [f for f in PIN_FILES if f not in first], workdir)


@pytest.fixture(scope="module")
def mutant_results(tmp_path_factory):
    """All mutants, built and run against the pins a few at a time (each run is a fresh
    interpreter, so most of its time is start-up)."""
    workdir = tmp_path_factory.mktemp("mutants")
    workers = max(1, min(6, os.cpu_count() or 1))
    with concurrent.futures.ThreadPoolExecutor(max_workers=workers) as pool:
        futures = {name: pool.submit(_run_mutant, name, workdir) for name in MUTANTS}
        return {name: f.result() for name, f in futures.items()}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, mutant_results):
    err, res = mutant_results[name]
    assert err is None, err
    assert res.returncode != 0, f"mutant {name} survived the pin suite:\n{res.stdout[-2000:]}"


def test_unmutated_copy_passes(tmp_path):
    """Control: the same harness on an unmodified copy passes."""
    lib = obuild.build(src=obuild.SRC, out=str(tmp_path / "libcopy.so"))
    res = _run_pins(lib, PIN_FILES, tmp_path)
    assert res.returncode == 0, res.stdout[-3000:] + res.stderr[-2000:]
