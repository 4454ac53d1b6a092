"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of oracle/oracle.c, on the CPU. The
mistakes are a wrong index, a dropped term, a flipped order or a wrong
operand. The copy is built as a separate library, and the oracle's pin tests
(tests/test_oracle_*.py) run against it in a subprocess; at least one pin
must fail. The unaltered source, built the same way, must pass them all.
The checked-in oracle.c and liboracle.so are never touched.
"""
import concurrent.futures as cf
import os
import subprocess
import sys

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = ["tests/test_oracle_score.py", "tests/test_oracle_select.py", "tests/test_oracle_layout.py",
        "tests/test_oracle_attention.py", "tests/test_oracle_error.py", "tests/test_oracle_budget.py",
        "tests/test_oracle_memory.py"]

# name: (text in oracle.c, replacement)
MUTATIONS = {
    # score: age t - i off by one
    "age_off_by_one": ("float age = (float)(t - pos);", "float age = (float)(t - pos - 1);"),
    # score: -0 left as -0 (it must rank equal to +0)
    "negative_zero_kept": ("if (s == 0.0f) s = 0.0f;", ""),
    # order: lower scores first
    "score_ascending": ("(const orc_entry *)pb;\n    if (a->s > b->s) return -1;\n    if (a->s < b->s) return 1;",
                        "(const orc_entry *)pb;\n    if (a->s < b->s) return -1;\n    if (a->s > b->s) return 1;"),
    # ties: later positions first
    "ties_descending_position": ("return a->h < b->h ? -1 : 1;\n    if (a->i != b->i) return a->i < b->i ? -1 : 1;",
                                 "return a->h < b->h ? -1 : 1;\n    if (a->i != b->i) return a->i > b->i ? -1 : 1;"),
    # ties: head before layer
    "ties_head_before_layer": ("if (a->l != b->l) return a->l < b->l ? -1 : 1;\n"
                               "    if (a->h != b->h) return a->h < b->h ? -1 : 1;",
                               "if (a->h != b->h) return a->h < b->h ? -1 : 1;\n"
                               "    if (a->l != b->l) return a->l < b->l ? -1 : 1;"),
    # select: one entry over the budget
    "budget_plus_one": ("for (int64_t r = 0; r < m; r++) {\n            keep[e[r].c",
                        "for (int64_t r = 0; r < m + (m < n); r++) {\n            keep[e[r].c"),
    # attention: logits without the scale
    "no_scale": ("z[k] = (double)scale * dot;", "z[k] = dot;"),
    # attention: query of the wrong head in a GQA group
    "gqa_wrong_query": ("return q + (c * G + g) * D;", "return q + ((c * G + g) % G) * D;"),
    # attention: values read from the K pool
    "values_from_keys": ("acc[d] += p * kv_elem(cc, cc->v_pool, row, d);",
                         "acc[d] += p * kv_elem(cc, cc->k_pool, row, d);"),
    # attention: log-sum-exp without its max
    "lse_without_max": ("m_k + log(zk)", "log(zk)"),
    # dropped mass: the kept set's mass instead of the evicted set's
    "dropped_mass_of_kept": ("if (keep && !keep[c * slots_per_head + k]) z_ev += p;",
                             "if (keep && keep[c * slots_per_head + k]) z_ev += p;"),
    # dropped mass: relative to the kept mass, not the dense total
    "dropped_mass_over_kept": ("z_ev / z_all", "z_ev / (z_all - z_ev)"),
    # eviction error: squared distance (no square root)
    "error_no_sqrt": ("err[c * G + g] = (float)sqrt(sq);", "err[c * G + g] = (float)sq;"),
    # eviction error: dense output built from the keys
    "error_dense_from_keys": ("for (int32_t d = 0; d < D; d++) mu[d] += p * kv_elem(cc, cc->v_pool, row, d);",
                              "for (int32_t d = 0; d < D; d++) mu[d] += p * kv_elem(cc, cc->k_pool, row, d);"),
    # eviction error: dense normaliser over the kept entries only
    "error_dense_sum_over_kept": ("            s_all += p;\n",
                                  "            if (!keep || keep[c * slots_per_head + k]) s_all += p;\n"),
    # eviction error: kept output not normalised
    "error_kept_unnormalised": ("ma[d] = n_kept > 0 ? ma[d] / s_k : 0.0;", "ma[d] = n_kept > 0 ? ma[d] : 0.0;"),
    # per-head budget: one entry over the budget
    "per_head_budget_plus_one": ("for (int32_t r = 0; r < m; r++) keep[c * slots_per_head + e[r].slot] = 1;",
                                 "for (int32_t r = 0; r < m + (m < n); r++) keep[c * slots_per_head + e[r].slot] = 1;"),
    # per-head budget: ties by descending position
    "per_head_ties_descending": ("if (a->i != b->i) return a->i < b->i ? -1 : 1;\n    return 0;\n}\n\nstatic int cmp_recent",
                                 "if (a->i != b->i) return a->i > b->i ? -1 : 1;\n    return 0;\n}\n\nstatic int cmp_recent"),
    # ContourKV: the floor holds the oldest entries
    "floor_oldest": ("if (a->i != b->i) return a->i > b->i ? -1 : 1;", "if (a->i != b->i) return a->i < b->i ? -1 : 1;"),
    # ContourKV: a head at the threshold counts as flat
    "flat_not_strict": ("const int flat = mean > tau;", "const int flat = mean >= tau;"),
    # ContourKV: the global part ignores what the floors and flat heads took
    "m_rest_ignores_forced": ("int64_t m = m_global[b] - forced;", "int64_t m = m_global[b];"),
    # latent memory: no decay of the state
    "memory_no_decay": ("        for (int64_t e = 0; e < (int64_t)D * D; e++) Mc[e] *= decay;\n", ""),
    # latent memory: elu without the +1 (features may vanish or turn negative)
    "memory_phi_without_one": ("return y > 0.0 ? y + 1.0 : exp(y);", "return y > 0.0 ? y : exp(y) - 1.0;"),
    # latent memory: read not normalised by phi(q)^T b
    "memory_read_unnormalised": ("gate * num / den", "gate * num"),
    # latent memory: kept rows folded in instead of the evicted ones
    "memory_kept_rows": ("if (keep[c * slots_per_head + s]) continue;", "if (!keep[c * slots_per_head + s]) continue;"),
    # latent memory: gate without its bias
    "memory_gate_no_bias": ("double den = 0.0, z = (double)gate_b[hq];", "double den = 0.0, z = 0.0;"),
    # compaction: freed pages pushed in descending table order
    "pushes_descending": ("for (int32_t pi = keep_pages; pi < old_pages; pi++) {",
                          "for (int32_t pi = old_pages - 1; pi >= keep_pages; pi--) {"),
    # compaction: a moved row keeps the hole's log-retention
    "move_drops_log_retention": ("    cc->lb_pool[dst] = cc->lb_pool[src];\n", ""),
    # append: pops from the bottom of the free stack
    "pop_from_bottom": ("cc->block_table[c * cc->max_pages + k / cc->P] = cc->free_stack[--(*cc->free_top)];",
                        "cc->block_table[c * cc->max_pages + k / cc->P] = cc->free_stack[0]; --(*cc->free_top);"),
    # append: the new token's position one too small
    "append_position_minus_one": ("cc->pos_pool[row] = t[b];", "cc->pos_pool[row] = t[b] - 1;"),
    # append: every head takes head 0's log-retention
    "append_first_head_log_retention": ("cc->lb_pool[row] = lb_new[c];", "cc->lb_pool[row] = lb_new[0];"),
}


def _run_pins(tmpdir: str, name: str, src: str):
    c_path = os.path.join(tmpdir, f"{name}.c")
    so_path = os.path.join(tmpdir, f"lib{name}.so")
    with open(c_path, "w") as fh:
        fh.write(src)
    subprocess.check_call(["gcc", *oracle.GCC_FLAGS, c_path, "-o", so_path, "-lm"])
    env = dict(os.environ, RKV_ORACLE_LIB=so_path)
    r = subprocess.run([sys.executable, "-m", "pytest", *PINS, "-x", "-q", "-p", "no:cacheprovider"], cwd=ROOT,
                       env=env, capture_output=True, text=True, timeout=900)
    return r.returncode, (r.stdout + r.stderr)[-3000:]


def test_pins_catch_planted_mistakes(tmp_path):
    with open(os.path.join(ROOT, "oracle", "oracle.c")) as fh:
        src = fh.read()
    jobs = {"unaltered": src}
    for name, (text, repl) in MUTATIONS.items():
        assert src.count(text) == 1, f"{name}: the text to alter is not in oracle.c exactly once"
        jobs[name] = src.replace(text, repl)
    with cf.ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as ex:
        futs = {name: ex.submit(_run_pins, str(tmp_path), name, s) for name, s in jobs.items()}
        res = {name: f.result() for name, f in futs.items()}
    rc, log = res["unaltered"]
    assert rc == 0, f"the pins fail on the unaltered oracle:\n{log}"
    missed = [name for name in MUTATIONS if res[name][0] == 0]
    assert not missed, f"no pin fails for: {missed}"
