"""The oracle's pins catch plausible mistakes in the oracle itself.

Each case plants one mistake in a copy of oracle/msa_oracle.c (a sign, a dropped term, a wrong
index, a wrong position, a reversed tie order, an off-by-one causal mask, ...), builds it with
the oracle's own compiler flags, points the oracle package at the mutant and runs every pin of
test_oracle_pins.py.  At least one pin must fail for every mutant; the unmutated build passes
them all (that file's own run).  Everything here runs on the CPU.
"""
import os
import shutil
import subprocess
import tempfile

import pytest

import oracle
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "msa_oracle.c")

# (name, [(original text, mutated text), ...]); each original text occurs exactly once in the
# forward part of the source (everything before the gradients, which the pins here do not call;
# tests/test_oracle_backward.py pins those by finite differences)
BACKWARD_START = "\nvoid msa_oracle_route_backward("
MUTANTS = [
    ("rope_rotation_sign", [("    x[i] = a * c - b * s;", "    x[i] = a * c + b * s;")]),
    ("rope_adjacent_pairs", [("    double a = x[i], b = x[i + half];",
                              "    double a = x[i], b = x[(i + 1) % dim];")]),
    ("rope_frequency", [("    double freq = pow(theta, -2.0 * (double)i / (double)dim);",
                         "    double freq = pow(theta, -(double)i / (double)dim);")]),
    ("rope_global_not_document_position", [(
        "          rope_vec(rot + (int64_t)h * D, D, (double)(t - s_d), theta);",
        "          rope_vec(rot + (int64_t)h * D, D, (double)t, theta);")]),
    ("pool_divides_by_chunk_length", [("      const double n = (double)(t1 - t0);",
                                       "      const double n = (double)L;")]),
    ("chunk_count_off_by_one", [("    doc_chunk_off[d + 1] = doc_chunk_off[d] + (len + L - 1) / L;",
                                 "    doc_chunk_off[d + 1] = doc_chunk_off[d] + len / L + 1;")]),
    ("sum_not_mean_over_router_heads", [("  return s / (double)H_r;", "  return s;")]),
    ("key_norm_dropped", [("  return dot / (nq * nk);", "  return dot / nq;")]),
    ("running_state_overwritten", [(
        "      double best = doc_score[(int64_t)b * n_docs + d];",
        "      double best = -INFINITY;")]),
    ("min_not_max_over_chunks", [("          if (s > best) best = s;",
                                  "          if (s < best || best == -INFINITY) best = s;")]),
    ("ties_go_to_higher_id", [("  return (a->id > b->id) - (a->id < b->id);",
                               "  return (a->id < b->id) - (a->id > b->id);")]),
    ("softmax_scale_one_over_d", [("  const double scale = 1.0 / sqrt((double)D);",
                                   "  const double scale = 1.0 / (double)D;")]),
    ("gqa_heads_interleaved", [("        const int32_t g = h / group;",
                                "        const int32_t g = h % H_kv;")]),
    ("query_without_global_offset", [("        rope_vec(q, D, (double)(pos_offset + j), theta);",
                                      "        rope_vec(q, D, (double)j, theta);")]),
    ("new_token_cannot_see_itself", [
        ("      const int64_t n_ctx = n_mem + (int64_t)j + 1;",
         "      const int64_t n_ctx = n_mem + (int64_t)j + (j == 0);"),
        ("        for (int32_t l = 0; l <= j; ++l) {\n          memcpy(key",
         "        for (int32_t l = 0; l < j + (j == 0); ++l) {\n          memcpy(key"),
        ("        for (int32_t l = 0; l <= j; ++l) {\n          const double *vr",
         "        for (int32_t l = 0; l < j + (j == 0); ++l) {\n          const double *vr"),
    ]),
    ("memory_values_read_from_keys", [(
        "            const double *vr = Vbar + (c * H_kv + g) * (int64_t)D;",
        "            const double *vr = Kbar + (c * H_kv + g) * (int64_t)D;")]),
]

PINS = [getattr(pins, n) for n in sorted(dir(pins)) if n.startswith("test_")]


@pytest.fixture(scope="module")
def workdir():
    d = tempfile.mkdtemp(prefix="oracle_mutants_")
    yield d
    shutil.rmtree(d, ignore_errors=True)


def _build_mutant(workdir, name, edits):
    src = open(SRC).read()
    cut = src.index(BACKWARD_START)
    fwd, bwd = src[:cut], src[cut:]
    for old, new in edits:
        assert fwd.count(old) == 1, f"{name}: pattern must occur once: {old!r}"
        fwd = fwd.replace(old, new)
    src = fwd + bwd
    c_path = os.path.join(workdir, f"{name}.c")
    so_path = os.path.join(workdir, f"{name}.so")
    with open(c_path, "w") as f:
        f.write(src)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                           "-fopenmp", "-shared", "-fPIC", c_path, "-o", so_path, "-lm"])
    return so_path


def _failing_pins(so_path):
    saved_lib, saved_build = oracle._lib, oracle.build
    oracle._lib = None
    oracle.build = lambda force=False: so_path
    try:
        oracle._load()
        failed = []
        for pin in PINS:
            try:
                pin()
            except Exception:  # an assertion, or a mutant that breaks an invariant outright
                failed.append(pin.__name__)
        return failed
    finally:
        oracle.build = saved_build
        oracle._lib = saved_lib


@pytest.mark.parametrize("name,edits", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(workdir, name, edits):
    failed = _failing_pins(_build_mutant(workdir, name, edits))
    assert failed, f"no pin caught the planted mistake {name}"


# Mistakes planted in the oracle's Python interleave (the adaptive stop rule and the exclusion
# padding live there, out of reach of the C mutants above).
PY_MUTANTS = [
    ("stop_on_equal_score", "active &= top[:, 0] >= stop_score",
     "active &= top[:, 0] > stop_score"),
    ("stopped_round_kept", "ids[~active] = -1", "pass"),
    ("rounds_counted_for_stopped_queries", "n_rounds += active", "n_rounds += 1"),
    ("taken_documents_listed_again", "ids[excluded] = -1", "pass"),
]
PY_PINS = [getattr(pins, n) for n in sorted(dir(pins))
           if n.startswith("test_") and ("interleave" in n)]


@pytest.mark.parametrize("name,old,new", PY_MUTANTS, ids=[m[0] for m in PY_MUTANTS])
def test_pins_catch_planted_mistake_in_the_interleave(name, old, new, monkeypatch):
    import inspect
    src = inspect.getsource(oracle.interleave)
    assert src.count(old) == 1, f"{name}: pattern must occur once"
    ns = dict(vars(oracle))
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), ns)
    monkeypatch.setattr(oracle, "interleave", ns["interleave"])
    failed = []
    for pin in PY_PINS:
        try:
            pin()
        except Exception:
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {name}"
