"""The selection certificate (tests/certify.py) and the per-unit check
(tests/unit_check.py) on the CPU: certified near-ties are accepted, and
planted wrong sets -- a skipped high-scoring chunk, a short fill, an
over-budget fill, a wrong count, a page from below the band -- are rejected.
The oracle's own selections serve as the right answers."""
import math

import numpy as np
import pytest

import oracle as O
from certify import certify_selection, certify_token_budget, tie_delta
import unit_check


def _rejects(fn, *a, **k):
    with pytest.raises(AssertionError):
        fn(*a, **k)


# ------------------------------------------------------------------ token budgets
def _tsa_case():
    # chunk scores with a near-tie between chunks 3 and 5 at the greedy stop
    S = np.array([9.0, 8.0, 7.5, 5.0, 1.0, 5.0 - 2e-6, 6.0, 0.5])
    lens = np.array([40, 30, 20, 25, 16, 16, 10, 50])
    # rank order: 0 (40 tokens), 1 (30), 2 (20), 6 (10) -> 100 tokens; then 3 (25), 5 (16)
    return S, lens


def test_token_budget_oracle_set_accepted():
    S, lens = _tsa_case()
    for budget in (40, 99, 100, 115, 116, 125, 200, 1000):
        o = set(int(p) for p in O.select_token_budget(S, lens, budget))
        assert certify_token_budget(S, lens, budget, o) is False


def test_token_budget_near_tie_alternative_accepted():
    S, lens = _tsa_case()
    # budget 116: the oracle takes 3 next (25 tokens) -> does not fit, stops at
    # {0,1,6,2}; the fp32 order may put 5 (16 tokens, within the tie band)
    # first, which fits: {0,1,6,2,5}, then 3 does not fit
    o = set(int(p) for p in O.select_token_budget(S, lens, 116))
    assert o == {0, 1, 6, 2}
    assert certify_token_budget(S, lens, 116, {0, 1, 6, 2, 5}) is True


def test_token_budget_planted_wrong_sets_rejected():
    S, lens = _tsa_case()
    budget = 116
    # skips a high-scoring chunk (1) and takes lower ones instead
    _rejects(certify_token_budget, S, lens, budget, {0, 6, 2, 3, 5})
    # stops early: chunk 6 (10 tokens) would still fit after {0, 1, 2}
    _rejects(certify_token_budget, S, lens, budget, {0, 1, 2})
    # a high-scoring chunk dropped although it fits
    _rejects(certify_token_budget, S, lens, budget, {0, 1, 6})
    # a short fill at a larger budget: after {0,1,6,2} both 3 and 5 still fit
    _rejects(certify_token_budget, S, lens, 200, {0, 1, 6, 2})
    # over budget
    _rejects(certify_token_budget, S, lens, 99, {0, 1, 6, 2})
    # a chunk from far below the band
    _rejects(certify_token_budget, S, lens, budget, {0, 1, 6, 2, 4})
    # every chunk kept although they do not all fit
    _rejects(certify_token_budget, S, lens, 200, set(range(8)))
    # out-of-range index
    _rejects(certify_token_budget, S, lens, budget, {0, 1, 6, 2, 99})


def test_token_budget_no_tie_requires_exact_set():
    S = np.array([9.0, 8.0, 7.0, 6.0, 5.0])
    lens = np.array([10, 10, 10, 10, 10])
    # with decisive gaps, only the oracle's set passes
    assert certify_token_budget(S, lens, 35, {0, 1, 2}) is False
    _rejects(certify_token_budget, S, lens, 35, {0, 1, 3})
    _rejects(certify_token_budget, S, lens, 35, {0, 1})


def test_token_budget_random_alternatives():
    """Random scores with planted near-ties: every set the certificate
    accepts is a greedy prefix of some near-tie-respecting order, checked by
    brute force over the orders of the tied groups."""
    import itertools
    rng = np.random.default_rng(7)
    for trial in range(100):
        P = 6
        S = np.round(rng.normal(size=P), 1)
        tie = rng.choice(P, 2, replace=False)
        S[tie[1]] = S[tie[0]] - 3e-6
        lens = rng.integers(16, 64, size=P)
        budget = int(rng.integers(16, lens.sum()))
        # every permutation that respects the order outside the band
        ok_sets = set()
        for perm in itertools.permutations(range(P)):
            good = all(not (S[perm[j]] > S[perm[i]] + tie_delta(S[perm[i]], S[perm[j]]))
                       for i in range(P) for j in range(i + 1, P))
            if not good:
                continue
            used, kept = 0, []
            for p in perm:
                if used + lens[p] > budget:
                    break
                kept.append(p)
                used += lens[p]
            ok_sets.add(frozenset(kept))
        for mask in range(1 << P):
            g = {p for p in range(P) if mask >> p & 1}
            try:
                certify_token_budget(S, lens, budget, g)
                accepted = True
            except AssertionError:
                accepted = False
            assert accepted == (frozenset(g) in ok_sets), (trial, S, lens, budget, g)


# ------------------------------------------------------------------ count cuts
def test_topk_certificate():
    S = np.array([5.0, 4.0, 3.0 + 1e-6, 3.0, 1.0])
    assert certify_selection(S, {0, 1, 2}, {"kind": "topk", "k": 3}) is False
    assert certify_selection(S, {0, 1, 3}, {"kind": "topk", "k": 3}) is True   # near-tie swap
    _rejects(certify_selection, S, {0, 2, 3}, {"kind": "topk", "k": 3})        # dropped 1
    _rejects(certify_selection, S, {0, 1, 4}, {"kind": "topk", "k": 3})        # below band
    _rejects(certify_selection, S, {0, 1}, {"kind": "topk", "k": 3})           # short
    S2 = np.array([5.0, 4.0, 3.0, 2.0])
    _rejects(certify_selection, S2, {0, 1, 3}, {"kind": "topk", "k": 3})       # decisive cut


def test_ratio_certificate_forced_pages():
    P = 40
    S = np.linspace(10, 0, P)
    bd = {"kind": "ratio", "ratio": 0.125, "bos": 1, "eos": 1}
    o = set(int(p) for p in O.select_ratio(S, 0.125, 1, 1, 1))
    assert certify_selection(S, o, bd) is False
    _rejects(certify_selection, S, (o - {P - 1}) | {5}, bd)  # forced last page missing


# ------------------------------------------------------------------ per-unit check
def _fake_run(Q, K, V, starts, ends, rule, budget, scale, *, sel=None, out_bias=0.0):
    meta = O.page_metadata(K, starts, ends)
    P = len(starts)
    if rule == "envelope":
        lo = meta[0].astype(np.float32).view(np.uint32) >> 16
        hi = meta[1].astype(np.float32).view(np.uint32) >> 16
        m = np.concatenate([lo, hi], axis=1).astype(np.uint16).view(np.uint8)
    else:
        m = meta[2].astype(np.float32).view(np.uint8)
    S = O.group_reduce(O.head_scores(Q, meta, rule))
    if sel is None:
        sel = O.select_topk(S, budget["k"])
    toks = O.tokens_of(sel, starts, ends)
    o, l = O.attend(Q, K, V, toks, scale)
    return dict(rule=rule, budget=budget, meta=m.reshape(P, 512), scores=S.astype(np.float32),
                sel=np.asarray(sel), out=(o + out_bias).astype(np.float32), lse=l.astype(np.float32))


@pytest.mark.parametrize("rule", ["envelope", "centroid"])
def test_unit_check_accepts_oracle_and_rejects_planted(rule):
    import torch
    g = torch.Generator().manual_seed(3)
    N = 300
    Q = torch.randn(8, 128, generator=g).bfloat16().float().numpy()
    K = torch.randn(N, 128, generator=g).bfloat16().float().numpy()
    V = torch.randn(N, 128, generator=g).bfloat16().float().numpy()
    starts, ends = O.fixed_pages(N, 16)
    host = dict(Q=Q, K=K, V=V, starts=starts, ends=ends, chunks=False)
    bd = {"kind": "topk", "k": 5}
    sc = 1 / math.sqrt(128)
    good = _fake_run(Q, K, V, starts, ends, rule, bd, sc)
    st = unit_check.check_unit(host, [good], scale=sc)
    assert st[0]["max_out_err"] < 1e-6
    # outputs off by more than the tolerance
    _rejects(unit_check.check_unit, host, [_fake_run(Q, K, V, starts, ends, rule, bd, sc, out_bias=3e-3)], scale=sc)
    # a wrong page set (the sixth-best page instead of the fifth)
    order = O.rank_order(good["scores"].astype(np.float64))
    wrong = np.sort(np.r_[order[:4], order[5]])
    _rejects(unit_check.check_unit, host, [_fake_run(Q, K, V, starts, ends, rule, bd, sc, sel=wrong)], scale=sc)
    # corrupted metadata
    bad = dict(good)
    bad["meta"] = good["meta"].copy()
    bad["meta"][3, 7] ^= 1
    _rejects(unit_check.check_unit, host, [bad], scale=sc)


def test_parallel_unit_check_harness():
    """The pooled check (spawned workers) on a small CPU-generated layer whose
    'GPU' results are the oracle's own: accepted; then one planted output
    error in one unit is reported."""
    import torch

    import datagen as DG
    import gpu_runner as R
    lay = DG.make_decode_layer(B=2, Hq=16, Hkv=2, seq_lens=[200, 131], seed=11, device="cpu")
    sc = 1 / math.sqrt(128)
    runs = []
    for rule, k in (("envelope", 4), ("centroid", 6)):
        B, Hkv = 2, 2
        P = 13
        sel = torch.full((B, Hkv, k), -1, dtype=torch.int32)
        cnt = torch.zeros((B, Hkv), dtype=torch.int32)
        out = torch.zeros((B, 16, 128))
        lse = torch.zeros((B, 16))
        meta = torch.zeros((B, Hkv, P, 512), dtype=torch.uint8)
        for b in range(B):
            N = int(lay.seq_len[b])
            s, e = O.fixed_pages(N, 16)
            for g in range(Hkv):
                K = lay.k[b, g, :N].float().numpy()
                V = lay.v[b, g, :N].float().numpy()
                Q = lay.q[b, 8 * g:8 * g + 8].float().numpy()
                fr = _fake_run(Q, K, V, s, e, rule, {"kind": "topk", "k": k}, sc)
                meta[b, g, :len(s)] = torch.from_numpy(fr["meta"])
                sel[b, g, :len(fr["sel"])] = torch.from_numpy(fr["sel"].astype(np.int32))
                cnt[b, g] = len(fr["sel"])
                out[b, 8 * g:8 * g + 8] = torch.from_numpy(fr["out"])
                lse[b, 8 * g:8 * g + 8] = torch.from_numpy(fr["lse"])
        runs.append((dict(sel_idx=sel, sel_count=cnt, out=out, lse=lse, meta=meta, scores=None),
                     rule, {"kind": "topk", "k": k}))
    st = R.check_units_parallel(lay, runs, page_size=16, scale=sc, batch_units=3)
    assert [s["units"] for s in st] == [4, 4]
    runs[1][0]["out"][1, 12, 5] += 0.01
    _rejects(R.check_units_parallel, lay, runs, page_size=16, scale=sc)
