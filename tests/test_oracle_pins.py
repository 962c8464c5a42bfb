"""The oracle against its pins, and planted mistakes against the same pins.

Each planted mistake is a deliberately broken copy of one oracle function (a
dropped term, a wrong sign or index, a swapped operand); the test asserts that
at least one pin rejects it.  Mistakes are planted only in oracle copies, on
the CPU.
"""
import math

import numpy as np
import pytest

import oracle as O
import oracle_pins as P


# ------------------------------------------------------------------ real oracle
def test_metadata_bruteforce():
    assert P.check_metadata_bruteforce(O.page_metadata, O.fixed_pages)


def test_metadata_incremental():
    assert P.check_metadata_incremental(O.page_metadata, O.fixed_pages)


def test_envelope_golden():
    assert P.check_envelope_golden(O.envelope_scores, O.centroid_scores, O.page_metadata)


def test_envelope_upper_bound():
    assert P.check_envelope_upper_bound(O.envelope_scores, O.page_metadata, O.fixed_pages)


def test_centroid_linearity():
    assert P.check_centroid_linearity(O.centroid_scores, O.page_metadata, O.fixed_pages)


def test_group_max():
    assert P.check_group_max(O.group_reduce)


def test_rank_order():
    assert P.check_rank_order(O.rank_order)


def test_topk_bruteforce():
    assert P.check_topk_bruteforce(O.select_topk)


def test_ratio_golden():
    assert P.check_ratio_golden(O.ratio_budget_pages)


def test_ratio_bruteforce():
    assert P.check_ratio_bruteforce(O.select_ratio, O.ratio_budget_pages)


def test_token_budget_bruteforce():
    assert P.check_token_budget_bruteforce(O.select_token_budget, O.rank_order)


def test_attention_sdpa():
    assert P.check_attention_sdpa(O.attend)


def test_full_budget_is_dense():
    assert P.check_full_budget_is_dense(O.decode_unit, O.attend)


def test_sigma_golden():
    assert P.check_sigma_golden(O.sigma_margin)


def test_sigma_range():
    assert P.check_sigma_range(O.sigma_margin)


def test_quantile():
    assert P.check_quantile(O.quantile_linear)


def test_tile_max_bruteforce():
    assert P.check_tile_max_bruteforce(O.tile_block_scores, O.envelope_scores,
                                       O.centroid_scores, O.page_metadata, O.fixed_pages)


def test_router_invariants():
    assert P.check_router_invariants(O.route, O.page_metadata, O.fixed_pages)


def test_route_decode():
    assert P.check_route_decode(O.route_decode, O.route, O.page_metadata, O.fixed_pages, O.head_scores,
                                O.group_reduce)


def test_tile_attention_sdpa():
    assert P.check_tile_attention_sdpa(O.tile_attention)


def test_fast_scores():
    assert P.check_fast_scores(O.envelope_scores_matmul, O.tile_block_scores, O.envelope_scores,
                               O.centroid_scores, O.page_metadata, O.fixed_pages)


def test_budget_scale_fact():
    """'The comparison': a 4096-token budget at ~29.5k context reads about a
    seventh of it, and the budget is page_size x top_k tokens."""
    assert round(29504 / 4096) == 7
    assert 16 * 256 == 4096 and 16 * 512 == 8192


# ------------------------------------------------------------------ planted mistakes
def _env_min(Q, kmin, kmax):          # max -> min
    Q = O.f64(Q)
    return np.stack([np.minimum(Q[h] * kmin, Q[h] * kmax).sum(1) for h in range(Q.shape[0])])


def _env_drop_last(Q, kmin, kmax):    # dropped term (last dimension)
    Q = O.f64(Q)
    return np.stack([np.maximum(Q[h] * kmin, Q[h] * kmax)[:, :-1].sum(1) for h in range(Q.shape[0])])


def _env_swapped_sign(Q, kmin, kmax):  # q+ paired with kmin
    Q = O.f64(Q)
    qp, qn = np.maximum(Q, 0), np.minimum(Q, 0)
    return qp @ O.f64(kmin).T + qn @ O.f64(kmax).T


def _meta_fixed_len(K, starts, ends):  # mean divides by the nominal page size
    kmin, kmax, kmean = O.page_metadata(K, starts, ends)
    ps = int(ends[0] - starts[0])
    for p in range(len(starts)):
        kmean[p] = O.f64(K)[starts[p]:ends[p]].sum(0) / ps
    return kmin, kmax, kmean


def _meta_swapped(K, starts, ends):
    kmin, kmax, kmean = O.page_metadata(K, starts, ends)
    return kmax, kmin, kmean


def _meta_off_by_one(K, starts, ends):
    return O.page_metadata(K, starts, np.maximum(starts + 1, ends - 1))


def _pages_floor(N, ps):               # drops the partial last page
    n = N // ps
    s = np.arange(n) * ps
    return s, s + ps


def _topk_high_index(S, k):            # ties broken toward the higher index
    S = O.f64(S) + 0.0
    idx = np.arange(len(S))
    order = np.lexsort((-idx, -S))
    return np.sort(order[:min(k, len(S))])


def _topk_signed_zero(S, k):           # -0.0 sorted below +0.0
    S = O.f64(S)
    keys = [(-(s), -math.copysign(1, s), i) for i, s in enumerate(S)]
    order = [i for _, _, i in sorted(keys)]
    return np.sort(np.array(order[:min(k, len(S))]))


def _ratio_ceil(P, ratio, topk_val, bos, eos):
    return min(P, max(topk_val + bos + eos, int(math.ceil(P * ratio))))


def _ratio_no_cap(P, ratio, topk_val, bos, eos):
    return max(topk_val + bos + eos, int(math.floor(P * ratio)))


def _select_ratio_bos_at_end(S, ratio, topk_val, bos, eos):  # forced pages at the wrong end
    return O.select_ratio(S, ratio, topk_val, eos, bos)


def _tokens_skip(S, lens, budget):
    return O.select_token_budget(S, lens, budget, skip=True)


def _attend_wrong_scale(Q, K, V, toks, scale):
    return O.attend(Q, K, V, toks, scale * scale)


def _attend_drop_first(Q, K, V, toks, scale):
    return O.attend(Q, K, V, toks[1:], scale)


def _sigma_off_index(S, k):
    S = O.f64(S)
    if len(S) <= k + 1:
        return 1.0
    d = S[0] - S[k + 1]
    return 0.0 if d == 0 else float((S[k - 1] - S[k + 1]) / d)


def _sigma_flipped(S, k):
    S = O.f64(S)
    if len(S) <= k:
        return 1.0
    d = S[0] - S[k]
    return 0.0 if d == 0 else float((S[0] - S[k - 1]) / d)


def _quantile_lower(v, q):
    return float(np.quantile(v, q, method="lower"))


def _tile_mean(Qtile, meta, rule, rows_per_batch=8):
    Qtile = O.f64(Qtile)
    flat = Qtile.reshape(-1, Qtile.shape[-1])
    return O.head_scores(flat, meta, rule).mean(axis=0)


def _route_le(Q, metas, rule, **kw):
    r = O.route(Q, metas, rule, **kw)
    trig = r.sigma_bar <= r.tau
    W = kw["rho"] * kw["k"]
    for t in range(len(trig)):
        for g in range(r.kv_idx.shape[1]):
            if trig[t] and not r.triggered[t]:
                E = int(np.isfinite(r.scores[t, g]).sum())
                order = O.rank_order(r.scores[t, g, :E])
                n = min(W, E)
                r.kv_idx[t, g, :n] = order[:n]
    r.triggered = trig
    return r


def _route_decode_page_order(unit_scores, **kw):   # lists in page order instead of rank order
    r = O.route_decode(unit_scores, **kw)
    for b in range(r.kv_idx.shape[0]):
        for g in range(r.kv_idx.shape[1]):
            n = int(r.kv_count[b, g])
            r.kv_idx[b, g, :n] = np.sort(r.kv_idx[b, g, :n])
    return r


def _route_decode_sigma_max(unit_scores, **kw):   # sigma_bar as the max over KV heads
    r = O.route_decode(unit_scores, **kw)
    r.sigma_bar = r.sigma.max(axis=1)
    return r


def _tile_attn_noncausal(Q, K, V, kv_idx, *, q_pos0, tile_rows, block_size, n_tokens, scale):
    return O.tile_attention(Q, K, V, kv_idx, q_pos0=q_pos0 + 10 ** 9, tile_rows=tile_rows,
                            block_size=block_size, n_tokens=n_tokens, scale=scale)


def _env_fast_swapped(Q, kmin, kmax):   # q+ paired with kmin in the matrix form
    Q = O.f64(Q)
    return np.maximum(Q, 0) @ O.f64(kmin).T + np.minimum(Q, 0) @ O.f64(kmax).T


MISTAKES = [
    ("envelope min instead of max", lambda: P.check_envelope_upper_bound(_env_min, O.page_metadata, O.fixed_pages)
     and P.check_envelope_golden(_env_min, O.centroid_scores, O.page_metadata)),
    ("envelope dropped dimension", lambda: P.check_envelope_upper_bound(_env_drop_last, O.page_metadata, O.fixed_pages)
     and P.check_envelope_golden(_env_drop_last, O.centroid_scores, O.page_metadata)),
    ("envelope q+/q- swapped", lambda: P.check_envelope_upper_bound(_env_swapped_sign, O.page_metadata, O.fixed_pages)
     and P.check_envelope_golden(_env_swapped_sign, O.centroid_scores, O.page_metadata)),
    ("centroid divides by nominal page size", lambda: P.check_centroid_linearity(O.centroid_scores, _meta_fixed_len, O.fixed_pages)
     and P.check_metadata_bruteforce(_meta_fixed_len, O.fixed_pages)),
    ("metadata min/max swapped", lambda: P.check_metadata_bruteforce(_meta_swapped, O.fixed_pages)
     and P.check_envelope_upper_bound(O.envelope_scores, _meta_swapped, O.fixed_pages)),
    ("metadata page end off by one", lambda: P.check_metadata_bruteforce(_meta_off_by_one, O.fixed_pages)),
    ("partial last page dropped", lambda: P.check_metadata_bruteforce(O.page_metadata, _pages_floor)),
    ("tie to higher index", lambda: P.check_topk_bruteforce(_topk_high_index)),
    ("-0.0 below +0.0", lambda: P.check_topk_bruteforce(_topk_signed_zero)),
    ("ratio ceil instead of floor", lambda: P.check_ratio_bruteforce(O.select_ratio, _ratio_ceil)
     and P.check_ratio_golden(_ratio_ceil)),
    ("ratio not capped at P", lambda: P.check_ratio_golden(_ratio_no_cap)),
    ("bos/eos at the wrong end", lambda: P.check_ratio_bruteforce(_select_ratio_bos_at_end, O.ratio_budget_pages)),
    ("token budget skips instead of stopping", lambda: P.check_token_budget_bruteforce(_tokens_skip, O.rank_order)),
    ("attention wrong scale", lambda: P.check_attention_sdpa(_attend_wrong_scale)),
    ("attention drops a token", lambda: P.check_attention_sdpa(_attend_drop_first)),
    ("sigma uses s_(k+1)", lambda: P.check_sigma_golden(_sigma_off_index)),
    ("sigma numerator flipped", lambda: P.check_sigma_golden(_sigma_flipped)),
    ("quantile lower instead of linear", lambda: P.check_quantile(_quantile_lower)),
    ("tile score mean instead of max", lambda: P.check_tile_max_bruteforce(
        _tile_mean, O.envelope_scores, O.centroid_scores, O.page_metadata, O.fixed_pages)),
    ("trigger on <= instead of <", lambda: P.check_router_invariants(_route_le, O.page_metadata, O.fixed_pages)),
    ("matrix-form envelope q+/q- swapped", lambda: P.check_fast_scores(
        _env_fast_swapped, O.tile_block_scores, O.envelope_scores, O.centroid_scores,
        O.page_metadata, O.fixed_pages)),
    ("tile attention not causal", lambda: P.check_tile_attention_sdpa(_tile_attn_noncausal)),
    ("decode router lists in page order", lambda: P.check_route_decode(
        _route_decode_page_order, O.route, O.page_metadata, O.fixed_pages, O.head_scores, O.group_reduce)),
    ("decode router sigma_bar as max", lambda: P.check_route_decode(
        _route_decode_sigma_max, O.route, O.page_metadata, O.fixed_pages, O.head_scores, O.group_reduce)),
]


@pytest.mark.parametrize("name,run", MISTAKES, ids=[m[0] for m in MISTAKES])
def test_planted_mistake_is_caught(name, run):
    assert not run(), f"planted mistake '{name}' passed every pin"
