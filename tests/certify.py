"""Selection certificates: is a page (or chunk) set that the GPU kept one of
the sets the method allows, given the oracle's float64 scores?

The GPU scores pages in fp32 (tensor-core sums), so where two oracle scores
differ by less than the near-tie tolerance their GPU order may flip.  The
rule (the near-tie reading of the method's "score, keep the best" step): the
GPU set must equal the oracle's, except that chunks whose oracle scores lie
within delta = 1e-5 * max(|s_a|, |s_b|, 1) of each other may trade places.

Fixed top-k and ratio budgets cut the order at a count, so the certificate is
a band around the cut.  A token budget cuts the greedy prefix of the order at
the first chunk that overflows, so the certificate requires, for the GPU set
K (kept) and D (dropped):
  (a) order: every kept chunk scores at least every dropped chunk - delta;
  (b) prefix: K is a prefix of one order that agrees with the oracle order
      outside the delta band -- given (a), K first then D in oracle order is
      such an order, and the dropped chunk that comes next in it may be any
      dropped chunk within delta of the best dropped score;
  (c) greedy stop: the kept weight fits the budget and that next chunk
      would overflow it (unless every chunk is kept).
Only numpy and the oracle's order are used here (no GPU, no product code).
"""
from __future__ import annotations

import numpy as np

import oracle as O

TIE_REL = 1e-5


def tie_delta(a: float, b: float) -> float:
    return TIE_REL * max(abs(a), abs(b), 1.0)


def certify_cut(S, order, n_keep, gset, where=""):
    """Count cut of `order` after n_keep entries.  Exact set equality unless
    the cut is a near-tie; then pages above the band must be kept, pages
    below it dropped, and the count must match.  Returns True when a
    certified near-tie allowed a difference."""
    oset = set(int(p) for p in order[:n_keep])
    if n_keep == 0 or n_keep >= len(order):
        assert gset == oset, f"{where}: set differs with no cut ({len(gset)} vs {len(oset)})"
        return False
    a, b = S[order[n_keep - 1]], S[order[n_keep]]
    delta = tie_delta(a, b)
    if a - b >= delta:
        assert gset == oset, f"{where}: set differs at a decisive cut (gap {a - b:.3g})"
        return False
    assert len(gset) == len(oset), f"{where}: count {len(gset)} vs {len(oset)}"
    assert gset <= set(int(x) for x in order), f"{where}: kept page outside the candidates"
    for p in (int(x) for x in order):
        if S[p] > a + delta:
            assert p in gset, f"{where}: page {p} above the tie band dropped"
        if S[p] < b - delta:
            assert p not in gset, f"{where}: page {p} below the tie band kept"
    return gset != oset


def certify_token_budget(S, lens, budget: int, gset: set, where=""):
    """Greedy token budget over chunks (longest prefix of the rank order that
    fits; stop at the first chunk that does not).  Checks (a)-(c) of the
    module docstring.  Returns True when the set differs from the oracle's
    (a certified near-tie)."""
    S = np.asarray(S, dtype=np.float64)
    lens = np.asarray(lens, dtype=np.int64)
    P = len(S)
    assert all(0 <= p < P for p in gset), f"{where}: chunk index out of range"
    oset = set(int(p) for p in O.select_token_budget(S, lens, budget))
    if gset == oset:
        return False
    used = int(sum(int(lens[p]) for p in gset))
    assert used <= budget, f"{where}: kept {used} tokens > budget {budget}"
    dropped = [p for p in range(P) if p not in gset]
    if not dropped:
        # every chunk kept: only right if they all fit, and then the oracle
        # keeps them all too (handled above)
        raise AssertionError(f"{where}: every chunk kept but the oracle keeps {len(oset)}")
    kept = sorted(gset)
    y_max = max(dropped, key=lambda p: (S[p], -p))
    # (a) order across the cut
    if kept:
        x_min = min(kept, key=lambda p: (S[p], -p))
        assert S[x_min] >= S[y_max] - tie_delta(S[x_min], S[y_max]), (
            f"{where}: kept chunk {x_min} (score {S[x_min]:.9g}) below dropped chunk {y_max} "
            f"(score {S[y_max]:.9g}) beyond the tie band")
    # (b) + (c): some dropped chunk that may come next must overflow
    nxt = [p for p in dropped if S[p] >= S[y_max] - tie_delta(S[p], S[y_max])]
    assert any(used + int(lens[p]) > budget for p in nxt), (
        f"{where}: greedy fill stopped early: {used} tokens kept, and the next chunk "
        f"(one of {nxt[:4]}...) would still fit the budget {budget}")
    return True


def certify_selection(S, gset: set, budget: dict, lens=None, where=""):
    """Returns True when a certified near-tie allowed a difference."""
    S = np.asarray(S, dtype=np.float64)
    P = len(S)
    order = O.rank_order(S)
    kind = budget["kind"]
    if kind == "topk":
        return certify_cut(S, order, min(budget["k"], P), gset, where)
    if kind == "ratio":
        K = O.ratio_budget_pages(P, budget["ratio"], budget.get("topk_val", 1), budget["bos"], budget["eos"])
        forced = set(int(x) for x in O.forced_pages(P, budget["bos"], budget["eos"]))
        assert forced <= gset, f"{where}: forced pages missing"
        rest = np.array([p for p in order if int(p) not in forced], dtype=np.int64)
        return certify_cut(S, rest, K - len(forced), gset - forced, where)
    return certify_token_budget(S, lens, budget["budget"], gset, where)
