"""The oracle's pins catch plausible mistakes: each mutant below plants one in
a copy of oracle/zr_oracle.c (a dropped term, a wrong sign, a swapped
constant, an off-by-one, a wrong order or tie-break), and the pin files
named beside it must fail against that copy.  The mistakes are planted in
the oracle, on the CPU; nothing here touches the library or a GPU."""
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys
import tempfile

import pytest

from conftest import ROOT

MUTANTS = [
    # name, original text, mutated text, pin files that must catch it
    ("drop_replica", "for (int32_t w = 1; w < world_size; ++w)", "for (int32_t w = 2; w < world_size; ++w)",
     ["test_oracle_reduce.py"]),
    ("reciprocal_not_division", "g_out[i] = s / (float)world_size;", "g_out[i] = s * (1.0f / (float)world_size);",
     ["test_oracle_reduce.py"]),
    ("fold_from_positive_zero", "float s = oracle_bf16_to_f32(grads[0][i]);\n        for (int32_t w = 1;",
     "float s = 0.0f;\n        for (int32_t w = 0;", ["test_oracle_reduce.py"]),
    ("decay_sign", "out->decay = (float)(1.0 - lr * (double)hp->weight_decay);",
     "out->decay = (float)(1.0 + lr * (double)hp->weight_decay);", ["test_oracle_adamw.py"]),
    ("eps_inside_root", "float denom = sqrtf(v_new) / s->bc2_sqrt + s->eps;",
     "float denom = sqrtf(v_new + s->eps) / s->bc2_sqrt;", ["test_oracle_adamw.py"]),
    ("no_second_bias_correction", "out->bc2_sqrt = (float)sqrt(bias2);", "out->bc2_sqrt = 1.0f;",
     ["test_oracle_adamw.py"]),
    ("first_moment_uses_beta2", "float m_new = s->beta1 * *m + s->one_minus_beta1 * g;",
     "float m_new = s->beta2 * *m + s->one_minus_beta2 * g;", ["test_oracle_adamw.py"]),
    ("update_sign", "p_new = p_new - update;", "p_new = p_new + update;", ["test_oracle_adamw.py"]),
    ("decay_after_update", "float p_new = *p * s->decay;", "float p_new = *p;",
     ["test_oracle_adamw.py"]),
    ("bf16_ties_away", "else if (rest == half && (kept & 1u)) round_up = 1;", "else if (rest == half) round_up = 1;",
     ["test_oracle_bf16.py"]),
    ("bf16_truncate", "return (uint16_t)(kept + (uint32_t)round_up);", "return (uint16_t)kept;",
     ["test_oracle_bf16.py"]),
    ("buckets_forward", "for (int32_t t = n_tensors - 1; t >= 0; --t) {\n        uint64_t bytes",
     "for (int32_t t = 0; t < n_tensors; ++t) {\n        uint64_t bytes", ["test_oracle_plan.py"]),
    ("bucket_cap_inclusive", "(holds_any && fill_bytes + bytes > cap_bytes)",
     "(holds_any && fill_bytes + bytes >= cap_bytes)", ["test_oracle_plan.py"]),
    ("groups_merged", "(holds_any && groups[t] != groups[t + 1])", "(holds_any && groups[t] > groups[t + 1])",
     ["test_oracle_plan.py"]),
    ("lpt_tie_to_highest_rank", "if (owned_numel[r] < owned_numel[best]) best = r;",
     "if (owned_numel[r] <= owned_numel[best]) best = r;", ["test_oracle_plan.py"]),
    ("flat_chunk_floor", "C = (N + world_size - 1) / world_size;", "C = N / world_size + 1;",
     ["test_oracle_plan.py"]),
    ("clip_without_eps", "double c = (double)max_norm / (sqrt(sumsq) + 1e-6);",
     "double c = (double)max_norm / sqrt(sumsq);", ["test_oracle_clip.py"]),
    ("sumsq_uncompensated", "return sum + correction;", "return sum;", ["test_oracle_clip.py"]),
    ("clip_applied_after_adam", "if (use_clip) oracle_scale(g_scratch, n_owned, clip_coef);\n    oracle_adamw(&s, g_scratch, n_owned, master, m, v);",
     "oracle_adamw(&s, g_scratch, n_owned, master, m, v);", ["test_oracle_invariants.py"]),
    ("cast_wrong_segment_offset", "param_out[segs[k].global_offset + j] =", "param_out[segs[k].owned_offset + j] =",
     ["test_oracle_invariants.py"]),
]


def _run_mutant(name, old, new, files):
    tmp = tempfile.mkdtemp(prefix=f"zr_mutant_{name}_")
    try:
        for d in ("oracle", "synth", "tests"):
            shutil.copytree(os.path.join(ROOT, d), os.path.join(tmp, d),
                            ignore=shutil.ignore_patterns("*.so", "__pycache__", "test_oracle_mutants.py"))
        src = os.path.join(tmp, "oracle", "zr_oracle.c")
        text = open(src).read()
        assert text.count(old) >= 1, f"{name}: text to mutate not found"
        open(src, "w").write(text.replace(old, new, 1))
        r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                            *[os.path.join("tests", f) for f in files]],
                           cwd=tmp, capture_output=True, text=True, timeout=600)
        return name, r.returncode, r.stdout[-400:]
    finally:
        shutil.rmtree(tmp, ignore_errors=True)


@pytest.mark.slow
def test_every_planted_mistake_fails_a_pin():
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(lambda m: _run_mutant(*m), MUTANTS))
    survivors = [(n, out) for n, rc, out in results if rc == 0]
    assert not survivors, f"mutants not caught by any pin: {survivors}"
    # and a clean copy passes the same pins (the harness itself is sound)
    name, rc, out = _run_mutant("none", "#include <math.h>", "#include <math.h>",
                                ["test_oracle_reduce.py", "test_oracle_adamw.py"])
    assert rc == 0, out
