"""The oracle's pins catch plausible mistakes: each mutant below plants one mistake
in an oracle function (on the CPU, in a copy of the function's source) and at
least one pin of ``test_oracle.py`` must then fail.

A mutant is (function, text, replacement): the text must occur exactly once in
the function's source.  The mutated function is compiled against the oracle
module's globals and patched into the module and the package for the duration
of one test, so the oracle's own internal calls see it too.
"""
import inspect
import textwrap

import pytest

import oracle
import oracle.msa_oracle as MO
import test_oracle as T

# every pin of test_oracle.py (parametrised ones at representative arguments)
PINS = {
    "bf16": T.test_bf16_widening_exact,
    "chunk_layout": lambda: T.test_chunk_layout_brute_force([1, 63, 64, 65, 127, 128, 129, 200]),
    "rope_theta": T.test_rope_theta_endpoints,
    "rope_complex": T.test_rope_matches_complex_multiplication,
    "rope_invariants": T.test_rope_invariants,
    "encode_membership": T.test_encode_pooling_matches_membership_matrix,
    "encode_doc_positions": T.test_encode_k_uses_document_positions,
    "encode_single_token": T.test_encode_single_token_doc_is_unrotated_projection,
    "encode_doc_order": T.test_encode_doc_order_invariance,
    "route_golden": T.test_route_hand_derived_golden,
    "router_query": T.test_router_query_one_hot_rows_and_head_columns,
    "cosine": T.test_cosine_closed_forms_and_range,
    "planted": T.test_planted_equal_key_scores_one_and_is_selected,
    "head_mean": T.test_head_mean_not_head_max,
    "token_max": T.test_max_over_query_tokens,
    "max_vs_mean": T.test_max_vs_mean_aggregation_discriminates,
    "route_by_hand": T.test_route_topk_per_query_and_aggregation_by_hand,
    "topk_sort": lambda: [T.test_topk_matches_pure_python_sort(s) for s in (0, 1, 2)],
    "attention_closed": T.test_attention_closed_forms,
    "gqa": T.test_attend_gqa_head_mapping,
    "local_positions": T.test_attend_local_positions_are_relative_to_query,
    "pooled_logit": T.test_attend_pooled_key_logit_uses_only_query_rotation,
    "explicit_concat": T.test_attend_topk_order_irrelevant_and_matches_explicit_concat,
    "prefill_decodes": T.test_attend_tokens_prefill_equals_sequence_of_decodes,
    "prefill_first_token": T.test_attend_tokens_first_token_sees_chunk_and_first_local_key,
    "prefill_chunks_only": T.test_attend_tokens_before_local_context_see_only_chunks,
    "aux_golden": T.test_aux_loss_hand_derived_golden,
    "aux_fd": T.test_aux_loss_gradients_match_finite_differences,
    "aux_batch": T.test_aux_loss_indistinguishable_negatives_and_batch_mean,
}

# (name, oracle function, text, replacement)
MUTANTS = [
    ("bf16 widening shift", "bf16_to_f64", "<< 16", "<< 15"),
    ("last chunk not clipped", "chunk_layout", "length.append(min(chunk, end - t))", "length.append(chunk)"),
    ("RoPE frequency exponent halved", "rope_theta", "-2.0 * i / head_dim", "-1.0 * i / head_dim"),
    ("RoPE rotation sign", "rope", "[x1 * c - x2 * s, x2 * c + x1 * s]", "[x1 * c + x2 * s, x2 * c - x1 * s]"),
    ("RoPE interleaved pairs", "rope", "x[..., :half], x[..., half:]", "x[..., 0::2], x[..., 1::2]"),
    ("encode: global instead of document positions", "encode_memory", "pos = np.arange(b - a)",
     "pos = np.arange(a, b)"),
    ("encode: K without RoPE", "encode_memory", "K = rope(K, pos[:, None], rope_base)", "K = K"),
    ("encode: V pooled over a full chunk", "encode_memory", "Vb.append(V[t:e].mean(axis=0))",
     "Vb.append(V[t:e].sum(axis=0) / chunk)"),
    ("encode: K^R max-pooled", "encode_memory", "KRb.append(KR[t:e].mean(axis=0))", "KRb.append(KR[t:e].max(axis=0))"),
    ("router query: transposed W^QR", "router_query", "Hq @ bf16_to_f64(W_QR)", "Hq @ bf16_to_f64(W_QR).T"),
    ("cosine: one norm dropped", "cosine", "/ (na * nb)", "/ (na * na)"),
    ("chunk score: head max", "chunk_scores", "cos_h.mean(axis=1)", "cos_h.max(axis=1)"),
    ("chunk score: mean over query tokens", "chunk_scores", "np.max(np.stack(per_t), axis=0)",
     "np.mean(np.stack(per_t), axis=0)"),
    ("document score: always the mean", "doc_scores", 'seg.max(axis=1) if agg == "max" else seg.mean(axis=1)',
     "seg.mean(axis=1)"),
    ("document score: segment runs one chunk long", "doc_scores", "chunk_off[i]:chunk_off[i + 1]]",
     "chunk_off[i]:chunk_off[i + 1] + 1]"),
    ("top-k: ties to the higher id", "topk", "np.lexsort((np.arange(len(s)), -s))",
     "np.lexsort((-np.arange(len(s)), -s))"),
    ("routing: aggregation argument ignored", "route_topk", "doc_scores(S, chunk_off, agg)", "doc_scores(S, chunk_off)"),
    ("routing: every query takes query 0's selection", "route_topk", "topk(s[b], k)", "topk(s[0], k)"),
    ("context: local keys without the offset", "sparse_context", "(pos_offset + np.arange(L))[:, None]",
     "np.arange(L)[:, None]"),
    ("context: pooled keys rotated again", "sparse_context", "ks.append(Kb[a:b])",
     "ks.append(rope(Kb[a:b], pos_offset, rope_base))"),
    ("context: last local token dropped", "sparse_context", "Kl = bf16_to_f64(K_loc_b[:L])\n    Vl = bf16_to_f64(V_loc_b[:L])",
     "Kl = bf16_to_f64(K_loc_b[:L - 1])\n    Vl = bf16_to_f64(V_loc_b[:L - 1])\n    L = L - 1"),
    ("attention: no softmax scale", "attention", "logits = (K @ q) * scale", "logits = (K @ q)"),
    ("attention: no normalisation", "attention", "/ p.sum()", ""),
    ("decode: query one position late", "sparse_attend", "pos_offset + L - 1", "pos_offset + L"),
    ("decode: GQA heads interleaved", "sparse_attend", "h = g // G", "h = g % n_kv"),
    ("prefill: a token does not see itself", "sparse_attend_tokens", "(local_j <= own)", "(local_j < own)"),
    ("prefill: GQA heads interleaved", "sparse_attend_tokens", "h = g // G", "h = g % n_kv"),
    ("prefill: token positions one early", "sparse_attend_tokens", "own = L - M + t ", "own = L - M + t - 1 "),
    ("L_aux: no temperature", "aux_loss", "z = s / tau", "z = s"),
    ("L_aux: sum instead of mean over positives", "aux_loss", "math.log(w.sum())) / P", "math.log(w.sum()))"),
    ("L_aux: positive gradient sign", "aux_loss", "g[0] = -(1.0 - p[0])", "g[0] = (1.0 - p[0])"),
    ("L_aux: query gradient without the norm term", "aux_loss",
     "dq = dq - cos[j, h] * Q[i, h] / (nq[h] ** 2)", "dq = dq"),
    ("L_aux: key gradient without the norm term", "aux_loss",
     "dk = dk - cos[j, h] * keys[j, h] / (nk[j, h] ** 2)", "dk = dk"),
    ("L_aux: gradient not through the head mean", "aux_loss", "gc = g[j] / n_r", "gc = g[j]"),
]


def _patch(monkeypatch, fn_name, old, new):
    src = textwrap.dedent(inspect.getsource(getattr(MO, fn_name)))
    assert src.count(old) == 1, f"{fn_name}: {old!r} occurs {src.count(old)} times"
    ns = {}
    exec(compile(src.replace(old, new), f"<mutant of {fn_name}>", "exec"), MO.__dict__, ns)
    monkeypatch.setattr(MO, fn_name, ns[fn_name])
    if hasattr(oracle, fn_name):
        monkeypatch.setattr(oracle, fn_name, ns[fn_name])


def _failing_pins():
    failed = []
    for name, pin in PINS.items():
        try:
            pin()
        except Exception:  # an assertion, or an error the mistake provokes
            failed.append(name)
    return failed


def test_every_pin_passes_on_the_oracle_as_written():
    assert _failing_pins() == []


@pytest.mark.parametrize("name,fn,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(monkeypatch, name, fn, old, new):
    _patch(monkeypatch, fn, old, new)
    assert _failing_pins(), f"no pin catches the mutant '{name}'"


def test_mutants_cover_every_oracle_function():
    # every function of the oracle's arithmetic has at least one mutant
    funcs = {n for n, f in vars(MO).items() if inspect.isfunction(f) and f.__module__ == MO.__name__
             and not n.startswith("_")}
    assert funcs <= {m[1] for m in MUTANTS}, funcs - {m[1] for m in MUTANTS}
