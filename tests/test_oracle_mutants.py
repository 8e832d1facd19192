"""The oracle pins must catch plausible mistakes.

Each case copies the oracle (oracle/veda_oracle.c, or the Python package that
composes its steps, oracle/__init__.py), plants one mistake (a dropped term, a
wrong index, a reversed comparison, a swapped operand, ...), builds the copy on
the CPU and runs the pin suite against it: the suite has to fail.  The
committed oracle is never modified.  The selected cases run concurrently
(each is its own build and pytest process); each test reports its own case.
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "veda_oracle.c")
PY = os.path.join(ROOT, "oracle", "__init__.py")

MUTANTS = {
    "score_drops_last_component": ("for (int64_t c = 0; c < r; ++c) acc += q[c] * k[c];",
                                   "for (int64_t c = 0; c < r - 1; ++c) acc += q[c] * k[c];"),
    "score_components_misaligned": ("for (int64_t c = 0; c < r; ++c) acc += q[c] * k[c];",
                                    "for (int64_t c = 0; c < r; ++c) acc += q[c] * k[(c + 1) % r];"),
    "attend_lse_without_max": ("if (lse) lse[u * T + tt] = mx + log(z);", "if (lse) lse[u * T + tt] = log(z);"),
    "pool_divides_by_T": ("o[e] = o[e] / (double)c;", "o[e] = o[e] / (double)T;"),
    "pool_tile_end_off_by_one": ("int64_t t1 = min64(N, t0 + T);", "int64_t t1 = min64(N, t0 + T - 1);"),
    "project_transposed_weight": ("(h * d + e) * r + c)", "(h * r + c) * d + e)"),
    "project_ignores_head": ("(h * d + e) * r + c)", "(e) * r + c)"),
    "score_uses_query_twice": ("acc += q[c] * k[c];", "acc += q[c] * q[c];"),
    "score_keys_of_head_zero": ("const double* k = khat + ((b * H + h) * nk + j) * r;",
                                "const double* k = khat + ((b * H + 0) * nk + j) * r;"),
    "select_kth_score_one_rank_early": ("if (kth) kth[rid] = row[k - 1].s;",
                                        "if (kth) kth[rid] = row[k > 1 ? k - 2 : 0].s;"),
    "score_keys_of_batch_zero": ("const double* k = khat + ((b * H + h) * nk + j) * r;",
                                 "const double* k = khat + ((0 * H + h) * nk + j) * r;"),
    "pool_reads_head_zero": ("o[e] += elem(x, dtype, b * sb + t * st + h * sh + e);",
                             "o[e] += elem(x, dtype, b * sb + t * st + e);"),
    "attend_values_of_head_zero": ("o[e] += w * elem(s->v, p->dtype, base + e);",
                                   "o[e] += w * elem(s->v, p->dtype, base - h * s->sh + e);"),
    "select_next_equals_kth": ("if (next) next[rid] = (k < nk) ? row[k].s : NAN;",
                               "if (next) next[rid] = (k < nk) ? row[k - 1].s : NAN;"),
    "attend_lse_base_two": ("if (lse) lse[u * T + tt] = mx + log(z);",
                            "if (lse) lse[u * T + tt] = mx + log2(z);"),
    "pool_token_and_head_strides_swapped": ("o[e] += elem(x, dtype, b * sb + t * st + h * sh + e);",
                                            "o[e] += elem(x, dtype, b * sb + t * sh + h * st + e);"),
    "select_keeps_lowest_scores": ("if (a->s > b->s) return -1;\n    if (a->s < b->s) return 1;",
                                   "if (a->s < b->s) return -1;\n    if (a->s > b->s) return 1;"),
    "select_ties_to_highest_index": ("return (a->j > b->j) - (a->j < b->j);",
                                     "return (a->j < b->j) - (a->j > b->j);"),
    "select_output_not_ascending": ("qsort(dst, (size_t)k, sizeof(int32_t), int32_ascending);", ""),
    "attend_drops_dense_keys": ("for (int64_t t = 0; t < p->dense.n; ++t) {",
                                "for (int64_t t = 0; t < 0; ++t) {"),
    "attend_reference_uses_video_index": ("int64_t j = idx_r[rid * k_r + m];",
                                          "int64_t j = idx_v[rid * k_v + m];"),
    "attend_forgets_scale": ("logit[a] = p->scale * dot;", "logit[a] = dot;"),
    "attend_logits_against_values": ("dot += qrow[e] * elem(s->k, p->dtype, base + e);",
                                     "dot += qrow[e] * elem(s->v, p->dtype, base + e);"),
    "attend_no_max_subtraction": ("const double w = exp(logit[a] - mx);", "const double w = exp(logit[a]);"),
    "attend_unnormalised": ("for (int64_t e = 0; e < d; ++e) o[e] = o[e] / z;", ""),
    "attend_query_tiles_from_video_length": ("const int64_t nq = (p->nq_tok + T - 1) / T;",
                                             "const int64_t nq = (p->video.n + T - 1) / T;"),
}


def _run_pins(env):
    return subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                           os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)


def _c_mutant(name, tmp_path):
    """Build the C oracle with mistake `name` and run the pins against it."""
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    mutant = tmp_path / "mutant.c"
    mutant.write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
                    "-o", str(so), str(mutant), "-lm"], check=True)
    env = dict(os.environ, VEDA_ORACLE_LIB=str(so), OMP_NUM_THREADS="1")
    return _run_pins(env)


# Mistakes in the Python composition of the steps (oracle/__init__.py).
PY_MUTANTS = {
    "select_tiles_reference_projected_with_wq": (
        'khat_r = project(pool(inp["k_ref"], T), inp["w_k"])',
        'khat_r = project(pool(inp["k_ref"], T), inp["w_q"])'),
    "select_tiles_reference_against_video_khat": (
        'select(qhat, khat_r, budget_ref)', 'select(qhat, khat, budget_ref)'),
    "select_tiles_reference_with_video_budget": (
        'select(qhat, khat_r, budget_ref)', 'select(qhat, khat_r, budget_video)'),
    "select_tiles_video_keys_projected_with_wq": (
        'khat = project(pool(inp["k"], T), inp["w_k"])', 'khat = project(pool(inp["k"], T), inp["w_q"])'),
    "select_tiles_queries_projected_with_wk": (
        'qhat = project(pool(inp["q"], T), inp["w_q"])', 'qhat = project(pool(inp["q"], T), inp["w_k"])'),
    "attend_units_reference_keys_and_values_swapped": (
        'ref = (inp["k_ref"], inp["v_ref"]) if ("k_ref" in inp and idx_r is not None) else None',
        'ref = (inp["v_ref"], inp["k_ref"]) if ("k_ref" in inp and idx_r is not None) else None'),
    "pool_wrapper_token_and_head_strides_swapped": (
        "lib().oracle_pool(x.data_ptr(), _code(x), B, N, H, d, sb, st, sh, T, _ptr(out))",
        "lib().oracle_pool(x.data_ptr(), _code(x), B, N, H, d, sb, sh, st, T, _ptr(out))"),
    "attend_default_scale_one_over_d": (
        "p.scale = (1.0 / math.sqrt(d)) if scale is None else float(scale)",
        "p.scale = (1.0 / d) if scale is None else float(scale)"),
    "attend_query_strides_from_video_keys": (
        "p.qsb, p.qst, p.qsh, _ = q.stride()", "p.qsb, p.qst, p.qsh, _ = _cpu(video[0]).stride()"),
    "attend_dense_queries_skip_reference": (
        '    ref, idx_r = None, None\n    if "k_ref" in inp:', '    ref, idx_r = None, None\n    if False:'),
    "attend_units_dense_keys_and_values_swapped": (
        'dense = (inp["k_dense"], inp["v_dense"]) if "k_dense" in inp else None\n    return attend(inp["q"]',
        'dense = (inp["v_dense"], inp["k_dense"]) if "k_dense" in inp else None\n    return attend(inp["q"]'),
}


def _py_mutant(name, tmp_path):
    """A copy of the oracle package with mistake `name` in its Python
    composition, ahead of the repository's on sys.path; the pins run on it."""
    old, new = PY_MUTANTS[name]
    src = open(PY).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    pkg = tmp_path / "oracle"
    pkg.mkdir()
    (pkg / "__init__.py").write_text(src.replace(old, new))
    (pkg / "veda_oracle.c").write_text(open(SRC).read())
    # tests/conftest.py puts VEDA_ORACLE_DIR ahead of the repository on sys.path
    env = dict(os.environ, VEDA_ORACLE_DIR=str(tmp_path), OMP_NUM_THREADS="1")
    env.pop("VEDA_ORACLE_LIB", None)
    probe = subprocess.run([sys.executable, "-c", "import sys; sys.path.insert(0, %r); "
                            "sys.path.insert(0, %r); import oracle; print(oracle.__file__)" % (ROOT, str(tmp_path))],
                           cwd=ROOT, env=env, capture_output=True, text=True, check=True)
    assert probe.stdout.strip().startswith(str(tmp_path)), probe.stdout
    return _run_pins(env)


C_TEST = "test_pins_catch_planted_mistake"
PY_TEST = "test_pins_catch_planted_mistake_in_composition"


@pytest.fixture(scope="module")
def mutant_runs(request, tmp_path_factory):
    """Every selected mutant of this module, run concurrently (each is an
    independent build and pytest process); results keyed by (test, name)."""
    jobs = [(item.originalname, item.callspec.params["name"]) for item in request.session.items
            if item.module is request.module and hasattr(item, "callspec")]
    run = {C_TEST: _c_mutant, PY_TEST: _py_mutant}
    # folders made here, one after another (mktemp is not safe across threads)
    dirs = [tmp_path_factory.mktemp(name) for _, name in jobs]

    def one(job_dir):
        (test, name), d = job_dir
        try:
            return run[test](name, d)
        except Exception as e:          # reported by the test that owns the job
            return e

    with ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as ex:
        return dict(zip(jobs, ex.map(one, zip(jobs, dirs))))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, mutant_runs):
    res = mutant_runs[(C_TEST, name)]
    if isinstance(res, Exception):
        raise res
    assert res.returncode != 0, f"pins did not catch mutant {name}:\n{res.stdout[-2000:]}"


@pytest.mark.parametrize("name", sorted(PY_MUTANTS))
def test_pins_catch_planted_mistake_in_composition(name, mutant_runs):
    res = mutant_runs[(PY_TEST, name)]
    if isinstance(res, Exception):
        raise res
    assert res.returncode != 0, f"pins did not catch mutant {name}:\n{res.stdout[-2000:]}"
