"""Each plausible mistake planted in a copy of the oracle must fail a pin.

The copies are built from the committed C source with one textual change and
compiled into a temporary directory; the committed oracle is never modified.
CPU only.
"""
from pathlib import Path

import pytest

import oracle
from _pins import ALL_PINS

SRC = Path(oracle.__file__).resolve().parent / "gsa_oracle.c"

# (name, original text, planted text) -- each original must occur exactly once
MUTANTS = [
    ("tie_break_reversed", "return (a->m < b->m) ? -1 : (a->m > b->m);", "return (a->m > b->m) ? -1 : (a->m < b->m);"),
    ("lowest_scores_selected", "if (a->s > b->s) return -1;\n  if (a->s < b->s) return 1;",
     "if (a->s < b->s) return -1;\n  if (a->s > b->s) return 1;"),
    ("logit_scale_dropped", "z[u] = scale * dot(", "z[u] = dot("),
    ("max_subtraction_sign", "z[u] = exp(z[u] - Z);", "z[u] = exp(Z - z[u]);"),
    ("lse_missing_max", "if (lse) *lse = Z + log(denom);", "if (lse) *lse = log(denom);"),
    ("value_reads_key", "out[i] += w * elem(S->tok[u].vb,", "out[i] += w * elem(S->tok[u].kb,"),
    ("gqa_modulo_mapping", "const int b = row / a->hq, h = row % a->hq, kvh = h / (a->hq / a->hkv);\n  const int d = a->d, c = a->chunk, dt = a->dtype;\n  const double scale = resolve_scale(a->scale, d);\n  const int32_t N = a->n_gists[b], own = a->own_len[b];\n  const size_t qo",
     "const int b = row / a->hq, h = row % a->hq, kvh = h % a->hkv;\n  const int d = a->d, c = a->chunk, dt = a->dtype;\n  const double scale = resolve_scale(a->scale, d);\n  const int32_t N = a->n_gists[b], own = a->own_len[b];\n  const size_t qo"),
    ("decode_raw_row_off_by_one", "st = push(S, raw_k, raw_v, (rbase + (size_t)m * c + j) * d, TOK_RAW, m * c + j);",
     "st = push(S, raw_k, raw_v, (rbase + (size_t)m * c + j + 1) * d, TOK_RAW, m * c + j);"),
    ("decode_selected_gist_dropped", "      if (!st) st = push(S, gist_k, gist_v, (gbase + m) * d, TOK_GIST, m);\n    } else if (!exclude) {",
     "    } else if (!exclude) {"),
    ("decode_unselected_gists_dropped", "    } else if (!exclude) {\n      st = push(S, gist_k, gist_v,",
     "    } else if (exclude) {\n      st = push(S, gist_k, gist_v,"),
    ("decode_first_own_row_dropped", "for (int32_t j = 0; j < own && !st; ++j)\n    st = push(S, raw_k, raw_v,",
     "for (int32_t j = 1; j < own && !st; ++j)\n    st = push(S, raw_k, raw_v,"),
    ("hgsa_trailing_group_ignored", "if (grp >= M || meta_chosen[grp])", "if (grp < M && meta_chosen[grp])"),
    ("hgsa_unselected_meta_dropped", "if (!meta_chosen[j]) st = push(&S, a->meta_k", "if (meta_chosen[j]) st = push(&S, a->meta_k"),
    ("hgsa_meta_uses_gist_keys", "ms[j] = scale * dot(a->q, qo, a->meta_k,", "ms[j] = scale * dot(a->q, qo, a->gist_k,"),
    ("prefill_own_prefix_excludes_self", "for (int32_t r = 0; r <= j && !st; ++r)", "for (int32_t r = 0; r < j && !st; ++r)"),
    ("prefill_gist_query_excludes_itself", "for (int32_t t = 0; t <= m && !st; ++t)", "for (int32_t t = 0; t < m && !st; ++t)"),
    ("prefill_chunk_of_position_off_by_one", "const int32_t m = (int32_t)(pos / c), j = (int32_t)(pos % c);",
     "const int32_t m = (int32_t)((pos + 1) / c), j = (int32_t)((pos + 1) % c);"),
    ("backward_drops_mean_term", "const double dz = w[u] * (gv[u] - go);", "const double dz = w[u] * gv[u];"),
    ("backward_key_grad_from_key", "dk[i] += scale * dz * elem(a->q, qo + i, dt);",
     "dk[i] += scale * dz * elem(S.tok[u].kb, S.tok[u].off + i, dt);"),
    ("hgsa2_noncandidate_level1_attended", "if (cand1[j] && !chosen1[j]) st = push(&S, a->meta_k",
     "if (!chosen1[j]) st = push(&S, a->meta_k"),
    ("hgsa2_chosen_level2_attended", "if (!chosen2[i]) st = push(&S, a->meta2_k", "if (1) st = push(&S, a->meta2_k"),
    ("hgsa2_level0_under_level2_groups", "const int32_t n0 = select_level(a->q, qo, a->gist_k, gbase, d, dt, scale, N, a->group1, M1, chosen1,",
     "const int32_t n0 = select_level(a->q, qo, a->gist_k, gbase, d, dt, scale, N, a->group1 * a->group2, M2, chosen2,"),
    ("topp_output_descending", "return (a->m > b->m) - (a->m < b->m);", "return (a->m < b->m) - (a->m > b->m);"),
    ("topp_strict_mass_test", "if (mass >= top_p) break;", "if (mass > top_p) break;"),
    ("topp_unshifted_exponent", "for (int32_t m = 0; m < n; ++m) z += exp(cand[m].s - cand[0].s);",
     "for (int32_t m = 0; m < n; ++m) z += exp(cand[m].s);"),
    ("topk_output_in_rank_order", "while (j > 0 && out[j - 1] > cand[i].m) {", "while (0) {"),
    ("gist_step_self_dropped", "if (!st) st = push(&S, a->k_new, a->v_new,", "if (0) st = push(&S, a->k_new, a->v_new,"),
    ("gist_step_own_rows_of_previous_chunk",
     "(rbase + (size_t)N * c + j) * d, TOK_RAW, N * c + j);\n  if (!st) st = push(&S, a->k_new",
     "(rbase + (size_t)(N > 0 ? N - 1 : 0) * c + j) * d, TOK_RAW, N * c + j);\n  if (!st) st = push(&S, a->k_new"),
    ("gist_step_last_gist_dropped", "for (int32_t m = 0; m < N && !st; ++m) st = push(&S, a->gist_k,",
     "for (int32_t m = 0; m + 1 < N && !st; ++m) st = push(&S, a->gist_k,"),
    ("prefill_ignores_exclude", "} else if (!a->exclude) {\n        st = push(&S, a->k_gist", "} else {\n        st = push(&S, a->k_gist"),
]


@pytest.mark.parametrize("name,orig,planted", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, orig, planted):
    text = SRC.read_text()
    assert text.count(orig) == 1, f"mutation site for {name} not unique"
    mutant_src = tmp_path / "mutant.c"
    mutant_src.write_text(text.replace(orig, planted))
    lib = oracle.build(src=mutant_src, out=tmp_path / "libmutant.so")
    orc = oracle.Oracle(lib)
    caught = []
    for pin in ALL_PINS:
        try:
            pin(orc)
        except (AssertionError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"planted mistake {name} passed every pin"
