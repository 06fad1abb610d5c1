"""Planted mistakes in the oracle must trip at least one pin.

Each mutant is a copy of oracle/oracle.c with one plausible mistake (a dropped
term, a wrong sign or index, a transposed operand, a skipped step), compiled
into a temporary library on the CPU.  The pins of oracle_pins.py run against
it in a child process; the test passes when some pin fails.  Nothing here
touches a GPU.
"""
import os
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = {
    "sigmoid_sign": ("s[e] = 1.0 / (1.0 + exp(-(double)l[e]));",
                     "s[e] = 1.0 / (1.0 + exp((double)l[e]));"),
    "softplus_no_sqrt": ("s[e] = sqrt(softplus((double)l[e]));", "s[e] = softplus((double)l[e]);"),
    "softplus_wrong_branch": ("fmax(l, 0.0) + log1p(exp(-fabs(l)))", "fmax(l, 0.0) + log1p(exp(-l))"),
    "softmax_unnormalised": ("s[e] = exp((double)l[e] - m) / z;", "s[e] = exp((double)l[e] - m);"),
    "bias_in_weights": ("row_weights(l, s, row_ids,", "row_weights(l, key, row_ids,"),
    "bias_ignored": ("key[e] = s[e] + (bias ? (double)bias[e] : 0.0);", "key[e] = s[e];"),
    "tie_higher_id": ("return (a->id > b->id) - (a->id < b->id);",
                      "return (a->id < b->id) - (a->id > b->id);"),
    "nan_ranks_first": ("if (an != bn) return an ? 1 : -1;", "if (an != bn) return an ? -1 : 1;"),
    "group_score_amax_only": ("for (int32_t i = 0; i < group_topn; ++i) gs += cand[i].key;",
                              "gs = cand[0].key;"),
    "group_keep_worst": ("kept[grp[i].id] = 1;", "kept[grp[n_groups - 1 - i].id] = 1;"),
    "group_keep_one_less": ("for (int32_t i = 0; i < topk_groups; ++i) kept[grp[i].id] = 1;",
                            "for (int32_t i = 0; i + 1 < topk_groups; ++i) kept[grp[i].id] = 1;"),
    "no_renormalise": ("    if (renormalize) {\n        double sum", "    if (0) {\n        double sum"),
    "weights_for_ids_row_offset": (
        "        row_scores(logits + t * E, E, score, s);\n        row_weights(logits + t * E, s, ids + t * k_max,",
        "        row_scores(logits + t * k_max, E, score, s);\n        row_weights(logits + t * E, s, ids + t * k_max,"),
    "weights_for_ids_ids_row": ("row_weights(logits + t * E, s, ids + t * k_max, k_max,",
                                "row_weights(logits + t * E, s, ids + t, k_max,"),
    "weights_for_ids_no_renormalise": ("ids + t * k_max, k_max, score, renormalize, route_scale,",
                                       "ids + t * k_max, k_max, score, 0, route_scale,"),
    "route_scale_ignored": ("if (ids[j] >= 0) w[j] *= route_scale;", "if (ids[j] >= 0) w[j] *= 1.0;"),
    "gptoss_softmax_all": ("    if (score == ORACLE_TOPK_SOFTMAX) {\n        double m",
                           "    if (0) {\n        double m"),
    "k_per_token_ignored": ("int32_t kt = k_per_token ? k_per_token[t] : k_max;",
                            "int32_t kt = k_max;"),
    "gate_transposed": ("oracle_bf16_to_double(xr[i]) * oracle_bf16_to_double(we[i]);",
                        "oracle_bf16_to_double(xr[i]) * oracle_bf16_to_double(w[(int64_t)i * E + e]);"),
    "gate_drops_last": ("            for (int32_t i = 0; i < d; ++i)\n                acc +=",
                        "            for (int32_t i = 0; i + 1 < d; ++i)\n                acc +="),
    "hash_table_transposed": ("table[(int64_t)v * k + j]", "table[(int64_t)j * vocab + v]"),
    "hash_uniform_unscaled": ("rw[j] = route_scale / (double)k;", "rw[j] = 1.0 / (double)k;"),
    "dispatch_unstable": ("int32_t pos = offsets[e] + seen[e];",
                          "int32_t pos = offsets[e + 1] - 1 - seen[e];"),
    "offsets_off_by_one": ("offsets[e + 1] = offsets[e] + counts[e];",
                           "offsets[e + 1] = offsets[e] + counts[e] - (e == E - 1);"),
    "capacity_keeps_last": ("if (capacity > 0 && rank >= capacity) continue;",
                            "if (capacity > 0 && counts[e] - 1 - rank >= capacity) continue;"),
    "capacity_block_unpadded": ("int32_t block = (kept + pad - 1) / pad * pad;",
                                "int32_t block = kept / pad * pad + (kept % pad ? 1 : 0);"),
    "capacity_demand_clipped": ("            *dropped += kept - capacity;\n            kept = capacity;",
                                "            *dropped += kept - capacity;\n            kept = capacity;\n            counts[e] = capacity;"),
    "grouped_candidates_worst": ("cand[nc++] = grp[i];", "cand[nc++] = grp[gsz - 1 - i];"),
    "grouped_no_final_sort": ("        qsort(cand, (size_t)nc, sizeof(ranked), by_key_desc);\n        int32_t *sel = ids + t * k_max;",
                              "        int32_t *sel = ids + t * k_max;"),
    "oai_no_alpha": ("gc * (1.0 / (1.0 + exp(-ORACLE_OAI_ALPHA * gc))) * (uc + 1.0)",
                     "gc * (1.0 / (1.0 + exp(-gc))) * (uc + 1.0)"),
    "oai_no_plus_one": ("exp(-ORACLE_OAI_ALPHA * gc))) * (uc + 1.0)", "exp(-ORACLE_OAI_ALPHA * gc))) * uc"),
    "swiglu_gate_up_swapped": ("    return g * (1.0 / (1.0 + exp(-g))) * u;", "    return u * (1.0 / (1.0 + exp(-u))) * g;"),
    "down_transposed": ("const uint16_t *wr = w2 + ((int64_t)e * d + c) * F;",
                        "const uint16_t *wr = w2 + ((int64_t)e * F + (c % F)) * d;"),
    "ffn_wrong_expert": ("        if (offsets[e] <= r && r < offsets[e + 1]) return e;",
                         "        if (offsets[e] <= r && r < offsets[e + 1]) return (e + 1) % E;"),
    "ep_owner_modulo": ("const int32_t d = e / el;", "const int32_t d = e % G;"),
    "ep_sources_reversed": ("if (ids_all[(int64_t)r * n + a] == e) {",
                            "if (ids_all[(int64_t)(G - 1 - r) * n + a] == e) {"),
    "permute_wrong_row": ("memcpy(xs + (int64_t)pos * d, x + t * (int64_t)d,",
                          "memcpy(xs + (int64_t)pos * d, x + ((t + 1) % T) * (int64_t)d,"),
    "combine_drops_shared": ("acc += sv;", "acc += 0.0 * sv;"),
    "combine_ignores_weight": ("double term = (double)w[t * k_max + j] *", "double term = 1.0 *"),
}


def _run_pins(lib_path: str) -> subprocess.CompletedProcess:
    code = (
        "import sys; sys.path[:0] = [%r, %r]\n"
        "import oracle, oracle_pins\n"
        "with oracle.using_library(%r):\n"
        "    failed = oracle_pins.run_all(stop_at_first=True)\n"
        "print('FAILED:' + ';'.join(failed))\n" % (ROOT, os.path.join(ROOT, "tests"), lib_path))
    return subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                          timeout=600)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    with open(os.path.join(ROOT, "oracle", "oracle.c")) as f:
        src = f.read()
    assert src.count(old) == 1, f"mutation site for {name} not unique / not found"
    mutant_c = tmp_path / f"{name}.c"
    mutant_c.write_text(src.replace(old, new))
    lib = oracle.compile_c(str(mutant_c), str(tmp_path / f"lib{name}.so"))
    res = _run_pins(lib)
    # a crash of the child (e.g. a mutant reading out of bounds) also counts as caught
    caught = res.returncode != 0 or ("FAILED:" in res.stdout and
                                     res.stdout.strip().split("FAILED:")[-1] != "")
    assert caught, f"mutant {name} survived every pin:\n{res.stdout}\n{res.stderr}"
