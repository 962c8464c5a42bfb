"""Pins for the float64 oracle: each checker takes the oracle function under
test as an argument and returns True when it agrees with something other than
itself (brute force, an invariant, a closed form, a library routine or a
hand-worked fixture).  tests/test_oracle_pins.py runs them on the real oracle
and on deliberately broken copies, so every plausible mistake is shown to
fail at least one pin.

Sources, by page title and section:
* "Sparse Attention for Web Agents -- Offline Replay Records", "The comparison"
  (chunking, envelope and centroid scoring, budget = page_size x top_k) and
  "Headline results" (TSA at a 16384 budget reproduces full attention).
* "WebArena 0-99 Sparse-Attention Method Comparison", "Method configurations at
  a glance" (ratio budget, topk_val, bos/eos).
* "Onzekerheidsgestuurde Selectie voor Blok-schaarse Aandacht", "Methodologie"
  steps 2-5 (tile max, sigma, quantile trigger, rho-expansion, sentinels).
"""
from __future__ import annotations

import itertools
import json
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rng(seed=0):
    return np.random.default_rng(seed)


def _bf16_round(x):
    """Round float64 values to bf16 (through torch) so test inputs are exact
    bf16 numbers, as the kernels see them."""
    return torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).to(torch.float64).numpy()


# ---------------------------------------------------------------- metadata
def check_metadata_bruteforce(page_metadata, fixed_pages) -> bool:
    """Pure-Python min/max/mean per page and dimension (sorted(), math.fsum)
    on a ragged partition, against the oracle."""
    rng = _rng(1)
    for N, ps in [(1, 16), (5, 2), (17, 16), (33, 16), (7, 7)]:
        K = rng.integers(-8, 9, size=(N, 4)).astype(np.float64) / 4.0
        starts, ends = fixed_pages(N, ps)
        if len(starts) != -(-N // ps):
            return False
        cover = np.concatenate([np.arange(s, e) for s, e in zip(starts, ends)])
        if not np.array_equal(cover, np.arange(N)):
            return False
        kmin, kmax, kmean = page_metadata(K, starts, ends)
        for p, (s, e) in enumerate(zip(starts, ends)):
            for d in range(K.shape[1]):
                col = sorted(float(K[t, d]) for t in range(s, e))
                if kmin[p, d] != col[0] or kmax[p, d] != col[-1]:
                    return False
                if abs(kmean[p, d] - math.fsum(col) / len(col)) > 1e-15:
                    return False
    return True


def check_metadata_incremental(page_metadata, fixed_pages) -> bool:
    """Growing the cache one token at a time changes only the page that holds
    the new token; all earlier pages keep their metadata."""
    rng = _rng(2)
    K = rng.standard_normal((70, 8))
    prev = None
    for N in range(1, 71):
        s, e = fixed_pages(N, 16)
        cur = page_metadata(K[:N], s, e)
        if prev is not None:
            P_prev = prev[0].shape[0]
            open_page = (N - 1) // 16
            for a, b in zip(prev, cur):
                if not np.array_equal(a[:min(P_prev, open_page)], b[:min(P_prev, open_page)]):
                    return False
        prev = cur
    return True


# ---------------------------------------------------------------- scores
def check_envelope_golden(envelope_scores, centroid_scores, page_metadata) -> bool:
    g = golden("envelope_example.json")
    K = np.array(g["keys"])
    q = np.array(g["q"])[None, :]
    starts = np.array([0, 2])
    ends = np.array([2, 3])
    kmin, kmax, kmean = page_metadata(K, starts, ends)
    if not (np.array_equal(kmin, g["kmin"]) and np.array_equal(kmax, g["kmax"])
            and np.allclose(kmean, g["kmean"], rtol=0, atol=1e-15)):
        return False
    env = envelope_scores(q, kmin, kmax)[0]
    cen = centroid_scores(q, kmean)[0]
    return (np.allclose(env, g["envelope"], rtol=0, atol=1e-12)
            and np.allclose(cen, g["centroid"], rtol=0, atol=1e-12))


def check_envelope_upper_bound(envelope_scores, page_metadata, fixed_pages) -> bool:
    """The envelope is an upper bound on q.k for every key of the page, with
    equality when the page holds one key (or identical keys), and it equals
    q+ . kmax + q- . kmin (positive/negative parts of q)."""
    rng = _rng(3)
    for trial in range(6):
        N, D, H = 53, 16, 3
        K = _bf16_round(rng.standard_normal((N, D)) * (1 + trial))
        Q = _bf16_round(rng.standard_normal((H, D)))
        s, e = fixed_pages(N, 4 + trial)
        kmin, kmax, kmean = page_metadata(K, s, e)
        env = envelope_scores(Q, kmin, kmax)
        for h in range(H):
            for p in range(len(s)):
                dots = [math.fsum(Q[h, d] * K[t, d] for d in range(D)) for t in range(s[p], e[p])]
                if env[h, p] < max(dots) - 1e-9:
                    return False
                if e[p] - s[p] == 1 and abs(env[h, p] - dots[0]) > 1e-9:
                    return False
                qp = np.maximum(Q[h], 0.0)
                qn = np.minimum(Q[h], 0.0)
                alt = math.fsum(qp * kmax[p]) + math.fsum(qn * kmin[p])
                if abs(env[h, p] - alt) > 1e-9:
                    return False
        # identical keys: bound is tight
        Kc = np.repeat(K[:1], 8, axis=0)
        mc = page_metadata(Kc, np.array([0]), np.array([8]))
        ec = envelope_scores(Q, mc[0], mc[1])
        for h in range(H):
            if abs(ec[h, 0] - math.fsum(Q[h] * K[0])) > 1e-9:
                return False
    return True


def check_centroid_linearity(centroid_scores, page_metadata, fixed_pages) -> bool:
    """q . mean(K) = mean over the page's keys of q . k (linearity)."""
    rng = _rng(4)
    N, D, H = 45, 12, 4
    K = _bf16_round(rng.standard_normal((N, D)))
    Q = _bf16_round(rng.standard_normal((H, D)))
    s, e = fixed_pages(N, 16)
    kmin, kmax, kmean = page_metadata(K, s, e)
    cen = centroid_scores(Q, kmean)
    for h in range(H):
        for p in range(len(s)):
            dots = [math.fsum(Q[h, d] * K[t, d] for d in range(D)) for t in range(s[p], e[p])]
            if abs(cen[h, p] - math.fsum(dots) / len(dots)) > 1e-12:
                return False
    return True


def check_group_max(group_reduce) -> bool:
    rng = _rng(5)
    s = rng.standard_normal((8, 13))
    r = group_reduce(s, "max")
    return all(r[p] == max(s[h, p] for h in range(8)) for p in range(13))


# ---------------------------------------------------------------- selection
def _bruteforce_topk(S, k):
    """Among all size-k subsets, the one with the largest score sum; among
    equal sums, the lexicographically smallest sorted index tuple."""
    P = len(S)
    k = min(k, P)
    best = None
    for sub in itertools.combinations(range(P), k):
        tot = math.fsum(S[i] for i in sub)
        key = (-tot, sub)
        if best is None or key < best:
            best = key
    return list(best[1])


def check_topk_bruteforce(select_topk) -> bool:
    """Integer-valued scores force many exact ties (lowest index must win)."""
    rng = _rng(6)
    for trial in range(60):
        P = int(rng.integers(1, 11))
        k = int(rng.integers(1, 6))
        S = rng.integers(-3, 4, size=P).astype(np.float64)
        if trial % 7 == 0:
            S[:] = 1.0
        if list(select_topk(S, k)) != _bruteforce_topk(S, k):
            return False
    # -0.0 and +0.0 are the same score: the lower index wins
    if list(select_topk(np.array([0.0, -0.0, 0.0]), 1)) != [0]:
        return False
    if list(select_topk(np.array([-0.0, 0.0]), 1)) != [0]:
        return False
    return True


def check_rank_order(rank_order) -> bool:
    S = np.array([3.0, 5.0, 3.0, -1.0, 5.0, 0.0])
    return list(rank_order(S)) == [1, 4, 0, 2, 5, 3]


def check_ratio_golden(ratio_budget_pages) -> bool:
    g = golden("ratio_budget.json")
    return all(ratio_budget_pages(c["P"], c["ratio"], c["topk_val"], c["bos"], c["eos"]) == c["K"]
               for c in g["cases"])


def check_ratio_bruteforce(select_ratio, ratio_budget_pages) -> bool:
    """Forced first-bos / last-eos pages plus the best of the rest, checked by
    brute force over subsets that contain the forced pages."""
    rng = _rng(7)
    for trial in range(40):
        P = int(rng.integers(1, 11))
        bos, eos = [(1, 1), (0, 1), (1, 0), (0, 0), (2, 1)][trial % 5]
        ratio = [0.5, 0.25, 0.0625, 0.375][trial % 4]
        S = rng.integers(-3, 4, size=P).astype(np.float64)
        K = ratio_budget_pages(P, ratio, 1, bos, eos)
        forced = sorted(set(range(min(bos, P))) | set(range(max(0, P - eos), P)))
        rest = [p for p in range(P) if p not in forced]
        take = max(0, K - len(forced))
        sub = _bruteforce_topk(S[rest], take) if take > 0 and rest else []
        expect = sorted(forced + [rest[i] for i in sub])
        got = list(select_ratio(S, ratio, 1, bos, eos))
        if got != expect:
            return False
        if K != min(P, max(1 + bos + eos, int(P * ratio))):
            return False
    return True


def check_token_budget_bruteforce(select_token_budget, rank_order) -> bool:
    """Longest prefix of the rank order whose token count fits the budget
    (prefixes enumerated directly); a budget >= all tokens keeps every chunk."""
    rng = _rng(8)
    for trial in range(60):
        C = int(rng.integers(1, 9))
        lens = rng.integers(1, 30, size=C)
        S = rng.integers(-2, 3, size=C).astype(np.float64)
        budget = int(rng.integers(0, 120))
        order = list(rank_order(S))
        best = []
        for r in range(C + 1):
            if sum(int(lens[p]) for p in order[:r]) <= budget:
                best = order[:r]
        if list(select_token_budget(S, lens, budget)) != sorted(best):
            return False
        if list(select_token_budget(S, lens, int(lens.sum()))) != list(range(C)):
            return False
    return True


# ---------------------------------------------------------------- attention
def _sdpa(Q, K, V, mask, scale):
    q = torch.tensor(Q, dtype=torch.float64)[None, :, None, :]       # [1,H,1,D]
    k = torch.tensor(K, dtype=torch.float64)[None, None].expand(1, Q.shape[0], -1, -1)
    v = torch.tensor(V, dtype=torch.float64)[None, None].expand(1, Q.shape[0], -1, -1)
    m = torch.tensor(mask, dtype=torch.bool)[None, None, None, :]
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=m, scale=scale)
    z = (torch.tensor(K, dtype=torch.float64) @ torch.tensor(Q, dtype=torch.float64).T) * scale
    z = z.masked_fill(~torch.tensor(mask)[:, None], float("-inf"))
    lse = torch.logsumexp(z, dim=0)
    return o[0, :, 0, :].numpy(), lse.numpy()


def check_attention_sdpa(attend) -> bool:
    """Masked softmax attention in float64 by torch's scaled_dot_product_attention."""
    rng = _rng(9)
    for trial in range(5):
        N, D, H = 50 + 13 * trial, 16, 4
        Q = rng.standard_normal((H, D))
        K = rng.standard_normal((N, D)) * 2
        V = rng.standard_normal((N, D))
        toks = np.sort(rng.choice(N, size=int(rng.integers(1, N)), replace=False))
        mask = np.zeros(N, dtype=bool)
        mask[toks] = True
        scale = 1 / math.sqrt(D)
        o, l = attend(Q, K, V, toks, scale)
        o2, l2 = _sdpa(Q, K, V, mask, scale)
        if not (np.allclose(o, o2, rtol=0, atol=1e-12) and np.allclose(l, l2, rtol=0, atol=1e-12)):
            return False
    return True


def check_full_budget_is_dense(decode_unit, attend) -> bool:
    """A budget covering the whole cache keeps every page, so the result is
    dense attention ('Headline results': TSA at 16384 reproduces full
    attention), for top-k, ratio and token budgets."""
    rng = _rng(10)
    N, D, G = 77, 16, 4
    Q = _bf16_round(rng.standard_normal((G, D)))
    K = _bf16_round(rng.standard_normal((N, D)))
    V = _bf16_round(rng.standard_normal((N, D)))
    dense, dl = attend(Q, K, V, np.arange(N), 0.25)
    lens = [10, 20, 7, 40]
    off = np.concatenate([[0], np.cumsum(lens)])
    for rule in ("envelope", "centroid"):
        for budget, kw in [({"kind": "topk", "k": 5}, {}),
                           ({"kind": "ratio", "ratio": 1.0, "bos": 1, "eos": 1}, {}),
                           ({"kind": "tokens", "budget": N}, {"chunk_off": off})]:
            r = decode_unit(Q, K, V, N, rule=rule, page_size=16, budget=budget, scale=0.25, **kw)
            if r.n_tokens != N:
                return False
            if not (np.allclose(r.out, dense, rtol=0, atol=1e-13) and np.allclose(r.lse, dl, rtol=0, atol=1e-13)):
                return False
    return True


# ---------------------------------------------------------------- router
def check_sigma_golden(sigma_margin) -> bool:
    g = golden("sigma_examples.json")
    for c in g["cases"]:
        s = sorted(c["scores"], reverse=True)
        if abs(sigma_margin(np.array(s, dtype=np.float64), c["k"]) - c["sigma"]) > 1e-15:
            return False
    return True


def check_sigma_range(sigma_margin) -> bool:
    rng = _rng(11)
    for _ in range(200):
        E = int(rng.integers(1, 20))
        k = int(rng.integers(1, 8))
        s = np.sort(rng.integers(-5, 6, size=E).astype(np.float64))[::-1]
        v = sigma_margin(s, k)
        if not (0.0 <= v <= 1.0):
            return False
        if E > k and s[k - 1] == s[k] and v != 0.0:
            return False
    return True


def check_quantile(quantile_linear) -> bool:
    rng = _rng(12)
    for _ in range(30):
        x = rng.standard_normal(int(rng.integers(1, 40)))
        q = float(rng.random())
        if abs(quantile_linear(x, q) - float(np.quantile(x, q, method="linear"))) > 1e-12:
            return False
    return True


def _tiny_router_problem(seed=13):
    rng = _rng(seed)
    Hq, Hkv, D, bs, N, rows = 6, 2, 8, 4, 64, 16
    Q = _bf16_round(rng.standard_normal((rows, Hq, D)))
    K = [_bf16_round(rng.standard_normal((N, D))) for _ in range(Hkv)]
    V = [_bf16_round(rng.standard_normal((N, D))) for _ in range(Hkv)]
    return Q, K, V, dict(Hq=Hq, Hkv=Hkv, D=D, bs=bs, N=N, rows=rows, q_pos0=N - rows)


def check_tile_max_bruteforce(tile_block_scores, envelope_scores, centroid_scores,
                              page_metadata, fixed_pages) -> bool:
    """Tile score = max over the tile's rows and the group's heads of the
    per-row block score (step 2), by explicit loops."""
    Q, K, V, c = _tiny_router_problem()
    s, e = fixed_pages(c["N"], c["bs"])
    meta = page_metadata(K[0], s, e)
    G = c["Hq"] // c["Hkv"]
    Qt = Q[0:4, 0:G]
    for rule, fn in (("envelope", lambda q: envelope_scores(q, meta[0], meta[1])),
                     ("centroid", lambda q: centroid_scores(q, meta[2]))):
        got = tile_block_scores(Qt, meta, rule)
        for b in range(len(s)):
            m = max(fn(Qt[r, h][None, :])[0, b] for r in range(4) for h in range(G))
            if got[b] != m:
                return False
    return True


def check_router_invariants(route, page_metadata, fixed_pages) -> bool:
    Q, K, V, c = _tiny_router_problem()
    s, e = fixed_pages(c["N"], c["bs"])
    metas = [page_metadata(K[g], s, e) for g in range(c["Hkv"])]
    nb = len(s)
    common = dict(q_pos0=c["q_pos0"], tile_rows=4, block_size=c["bs"], n_blocks=nb)
    for rule in ("envelope", "centroid"):
        base = route(Q, metas, rule, k=3, rho=1, quantile=0.5, **common)
        # rho = 1: every list is the plain top-k prefix, whatever triggers
        for t in range(base.kv_idx.shape[0]):
            for g in range(c["Hkv"]):
                E = min(nb, (c["q_pos0"] + min(c["rows"], (t + 1) * 4) - 1) // c["bs"] + 1)
                S = base.scores[t, g, :E]
                order = sorted(range(E), key=lambda i: (-S[i], i))
                if list(base.kv_idx[t, g]) != order[:3]:
                    return False
        exp = route(Q, metas, rule, k=3, rho=2, quantile=0.5, **common)
        # top-k is a prefix of top-rho*k; untriggered lists carry rho*k-k sentinels
        for t in range(exp.kv_idx.shape[0]):
            for g in range(c["Hkv"]):
                row = list(exp.kv_idx[t, g])
                if row[:3] != list(base.kv_idx[t, g]):
                    return False
                if not exp.triggered[t] and row[3:] != [-1, -1, -1]:
                    return False
                if exp.triggered[t] and -1 in row:
                    return False
        # sigma_bar is the mean over KV heads
        if not np.allclose(exp.sigma_bar, exp.sigma.mean(axis=1), rtol=0, atol=0):
            return False
        # quantile 0 triggers nothing; quantile 1 triggers all but the maximal tiles
        r0 = route(Q, metas, rule, k=3, rho=2, quantile=0.0, **common)
        if r0.triggered.any():
            return False
        r1 = route(Q, metas, rule, k=3, rho=2, quantile=1.0, **common)
        if list(r1.triggered) != list(r1.sigma_bar < r1.sigma_bar.max()):
            return False
    return True


def check_route_decode(route_decode, route, page_metadata, fixed_pages, head_scores, group_reduce) -> bool:
    """The decode router equals route() when the batch has one sequence (its
    query row is a one-row tile at the newest position, every block
    eligible), and over a batch it keeps the router's invariants: rho = 1
    gives the plain top-k prefix, top-k is a prefix of top-rho*k, sentinels
    pad untriggered lists, quantile 0 triggers nothing."""
    rng = _rng(41)
    bs, Hkv, G, D = 4, 2, 3, 8
    lens = [37, 29, 41, 16]
    metas, Qs = [], []
    for N in lens:
        K = _bf16_round(rng.normal(size=(Hkv, N, D)))
        s_, e_ = fixed_pages(N, bs)
        metas.append([page_metadata(K[g], s_, e_) for g in range(Hkv)])
        Qs.append(_bf16_round(rng.normal(size=(Hkv * G, D))))
    for rule in ("envelope", "centroid"):
        unit = [[group_reduce(head_scores(Qs[b][g * G:(g + 1) * G], metas[b][g], rule)) for g in range(Hkv)]
                for b in range(len(lens))]
        # one sequence: the same as route() with one one-row tile at position N - 1
        N0 = lens[0]
        one = route_decode(unit[:1], k=3, rho=2, quantile=0.5)
        ref = route(Qs[0][None], metas[0], rule, q_pos0=N0 - 1, tile_rows=1, block_size=bs,
                    n_blocks=len(fixed_pages(N0, bs)[0]), k=3, rho=2, quantile=0.5)
        if not (np.array_equal(one.kv_idx, ref.kv_idx) and np.array_equal(one.kv_count, ref.kv_count)
                and np.allclose(one.sigma, ref.sigma, rtol=0, atol=1e-12)):
            return False
        base = route_decode(unit, k=3, rho=1, quantile=0.5)
        exp = route_decode(unit, k=3, rho=2, quantile=0.5)
        for b in range(len(lens)):
            for g in range(Hkv):
                S = unit[b][g]
                order = sorted(range(len(S)), key=lambda i: (-S[i], i))
                if list(base.kv_idx[b, g]) != order[:3]:
                    return False
                row = list(exp.kv_idx[b, g])
                if row[:3] != order[:3]:
                    return False
                if not exp.triggered[b] and row[3:] != [-1, -1, -1]:
                    return False
        if not np.allclose(exp.sigma_bar, exp.sigma.mean(axis=1), rtol=0, atol=0):
            return False
        if route_decode(unit, k=3, rho=2, quantile=0.0).triggered.any():
            return False
    return True


def check_tile_attention_sdpa(tile_attention) -> bool:
    """Causal attention over the tile's selected blocks, against torch SDPA
    with an explicit boolean mask built row by row."""
    Q, K, V, c = _tiny_router_problem()
    rows, Hq, D = Q.shape
    G = Hq // c["Hkv"]
    rng = _rng(14)
    T = rows // 4
    kv_idx = np.full((T, c["Hkv"], 4), -1)
    for t in range(T):
        for g in range(c["Hkv"]):
            n = int(rng.integers(1, 5))
            kv_idx[t, g, :n] = rng.choice(c["N"] // c["bs"], size=n, replace=False)
    out, lse = tile_attention(Q, K, V, kv_idx, q_pos0=c["q_pos0"], tile_rows=4,
                              block_size=c["bs"], n_tokens=c["N"], scale=0.3)
    for r in range(rows):
        t = r // 4
        pos = c["q_pos0"] + r
        for h in range(Hq):
            g = h // G
            mask = np.zeros(c["N"], dtype=bool)
            for b in kv_idx[t, g]:
                if b >= 0:
                    mask[b * c["bs"]:(b + 1) * c["bs"]] = True
            mask[pos + 1:] = False
            if not mask.any():
                if not (np.all(out[r, h] == 0) and lse[r, h] == -np.inf):
                    return False
                continue
            o2, l2 = _sdpa(Q[r, h][None, :], K[g], V[g], mask, 0.3)
            if not (np.allclose(out[r, h], o2[0], atol=1e-12, rtol=0) and abs(lse[r, h] - l2[0]) < 1e-12):
                return False
    return True


def check_fast_scores(envelope_fast, tile_block_scores, envelope_scores, centroid_scores,
                      page_metadata, fixed_pages) -> bool:
    """The matrix-product envelope (q+ . kmax + q- . kmin) and the fast tile
    scores agree with the literal per-dimension definitions."""
    rng = _rng(15)
    K = _bf16_round(rng.standard_normal((300, 16)) * 2)
    Q = _bf16_round(rng.standard_normal((9, 16)))
    s, e = fixed_pages(300, 16)
    meta = page_metadata(K, s, e)
    a = envelope_fast(Q, meta[0], meta[1])
    b = envelope_scores(Q, meta[0], meta[1])
    if not np.allclose(a, b, rtol=1e-12, atol=1e-12):
        return False
    Qt = Q.reshape(3, 3, 16)
    for rule in ("envelope", "centroid"):
        f = tile_block_scores(Qt, meta, rule, fast=True)
        sl = tile_block_scores(Qt, meta, rule, fast=False)
        if not np.allclose(f, sl, rtol=1e-12, atol=1e-12):
            return False
    return True
