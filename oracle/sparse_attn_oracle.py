"""Plain float64 CPU oracle for query-aware block-sparse GQA decode attention
and for the uncertainty router over query tiles.

TEST INFRASTRUCTURE ONLY.  This module is imported by ``tests/``, by
``__graft_entry__.smoke()`` and by the CPU-baseline / reference legs of
``bench.py``.  The product path (the CUDA library and its Python binding)
never imports, calls or links anything here, and this module imports nothing
from the product path.  It shares no code with the CUDA kernels: only the
seeded input generators in ``datagen/`` feed both sides.

Sources (web pages; cited by title and section):

* [OFFLINE] "Sparse Attention for Web Agents -- Offline Replay Records"
  (dataset card shiqihe/WebVoyager-GAIA-SparseAttention-Offline-Qwen3-VL-30B-A3B),
  section "The comparison": the method table (chunking x scoring) and the
  paragraph defining the budget as page_size x top_k.
* [WEBARENA] "WebArena 0-99 Sparse-Attention Method Comparison"
  (dataset card Sean1999/webarena), section "Method configurations at a
  glance": the ratio budget with forced bos/eos pages and topk_val.
* [ROUTER] "Technische Samenvatting: Onzekerheidsgestuurde Selectie voor
  Blok-schaarse Aandacht", section "Methodologie", steps 1-5: block scoring,
  per-tile selection, the normalised cut-off margin sigma, head averaging with
  a per-layer quantile trigger, and rho-expansion with sentinel padding.

Every array here is float64 (inputs are exact bf16 values, upcast), except
index arrays (int64).  Nothing is blocked, fused or reordered beyond what the
definitions state; numpy reductions serve as plain library steps.

Parity status per function (pins live in tests/test_oracle_*.py):
all functions below are pinned (brute force, invariants, closed forms,
library routines or hand-worked fixtures under tests/golden/).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

NEG_INF = float("-inf")


def f64(x) -> np.ndarray:
    """Upcast an array of exact bf16 (or float32) values to float64."""
    return np.asarray(x, dtype=np.float64)


# --------------------------------------------------------------------------
# 1. Partition of the cache into pages / chunks.
# [OFFLINE] "The comparison": Quest and BlockSparse use fixed 16-token pages,
# TSA uses variable chunks of 16-256 tokens aligned to document structure.
# --------------------------------------------------------------------------

def fixed_pages(n_tokens: int, page_size: int) -> tuple[np.ndarray, np.ndarray]:
    """Token ranges [start, end) of consecutive fixed-size pages covering
    tokens 0..n_tokens-1.  The last page may be partial."""
    n_pages = -(-n_tokens // page_size)
    starts = np.arange(n_pages, dtype=np.int64) * page_size
    ends = np.minimum(starts + page_size, n_tokens)
    return starts, ends


def chunk_pages(chunk_off) -> tuple[np.ndarray, np.ndarray]:
    """Token ranges of variable chunks given CSR offsets off[0..C]:
    chunk c covers [off[c], off[c+1])."""
    off = np.asarray(chunk_off, dtype=np.int64)
    return off[:-1].copy(), off[1:].copy()


# --------------------------------------------------------------------------
# 2. Per-page metadata: per-dimension key min / max (envelope) and key mean
# (centroid).  [OFFLINE] "The comparison", scoring column.
# --------------------------------------------------------------------------

def page_metadata(K, starts, ends):
    """K: [N, D] keys of one (sequence, KV head).  Returns (kmin, kmax, kmean),
    each [P, D]: the per-dimension minimum, maximum and mean of the keys of
    each page."""
    K = f64(K)
    P = len(starts)
    D = K.shape[1]
    kmin = np.empty((P, D))
    kmax = np.empty((P, D))
    kmean = np.empty((P, D))
    for p in range(P):
        blk = K[starts[p]:ends[p]]
        kmin[p] = blk.min(axis=0)
        kmax[p] = blk.max(axis=0)
        kmean[p] = blk.sum(axis=0) / blk.shape[0]
    return kmin, kmax, kmean


# --------------------------------------------------------------------------
# 3. Per-head page scores.
# Envelope: sum over dimensions of the larger of q_d*kmin_d and q_d*kmax_d,
# an upper bound on q.k for every key in the page ([OFFLINE] "The
# comparison"; [ROUTER] step 1, coordinate-wise upper bounds).
# Centroid: inner product of q with the mean key of the page ([OFFLINE] "The
# comparison"; [ROUTER] step 1, mean-pooled inner product).
# --------------------------------------------------------------------------

def envelope_scores(Q, kmin, kmax) -> np.ndarray:
    """Q: [H, D] query heads; kmin/kmax: [P, D].  Returns s[H, P]."""
    Q = f64(Q)
    kmin = f64(kmin)
    kmax = f64(kmax)
    H = Q.shape[0]
    P = kmin.shape[0]
    s = np.empty((H, P))
    for h in range(H):
        a = Q[h][None, :] * kmin
        b = Q[h][None, :] * kmax
        s[h] = np.maximum(a, b).sum(axis=1)
    return s


def envelope_scores_matmul(Q, kmin, kmax) -> np.ndarray:
    """The same envelope score written with the positive and negative parts of
    q: max(q_d kmin_d, q_d kmax_d) = q+_d kmax_d + q-_d kmin_d because
    kmax_d >= kmin_d; summed over d this is two matrix products.  Used for
    large router workloads; pinned against envelope_scores."""
    Q = f64(Q)
    qp = np.maximum(Q, 0.0)
    qn = np.minimum(Q, 0.0)
    return qp @ f64(kmax).T + qn @ f64(kmin).T


def centroid_scores(Q, kmean) -> np.ndarray:
    """Q: [H, D]; kmean: [P, D].  Returns s[H, P] = q_h . kmean_p."""
    Q = f64(Q)
    kmean = f64(kmean)
    H = Q.shape[0]
    s = np.empty((H, kmean.shape[0]))
    for h in range(H):
        s[h] = (Q[h][None, :] * kmean).sum(axis=1)
    return s


def head_scores(Q, meta, rule: str, fast: bool = False) -> np.ndarray:
    kmin, kmax, kmean = meta
    if rule == "envelope":
        return envelope_scores_matmul(Q, kmin, kmax) if fast else envelope_scores(Q, kmin, kmax)
    if rule == "centroid":
        return f64(Q) @ f64(kmean).T if fast else centroid_scores(Q, kmean)
    raise ValueError(rule)


def group_reduce(s_heads, reduce: str = "max") -> np.ndarray:
    """Combine the per-query-head scores of one GQA group into one score per
    page.  'max' is the reading used everywhere (the group shares one page
    set, as the tile shares one set in [ROUTER] step 2); 'sum' is kept only
    as an alternative reading for comparison."""
    s = f64(s_heads)
    if reduce == "max":
        return s.max(axis=0)
    if reduce == "sum":
        return s.sum(axis=0)
    raise ValueError(reduce)


# --------------------------------------------------------------------------
# 4. Deterministic order and budgets.
# --------------------------------------------------------------------------

def rank_order(S) -> np.ndarray:
    """Page indices sorted by score descending, lower index first on ties.
    -0.0 and +0.0 compare equal."""
    S = f64(S) + 0.0  # maps -0.0 to +0.0
    idx = np.arange(len(S))
    return np.lexsort((idx, -S)).astype(np.int64)


def select_topk(S, k: int) -> np.ndarray:
    """Fixed top-k ([OFFLINE] "The comparison": budget = page_size x top_k
    tokens).  Returns the selected page indices, ascending."""
    order = rank_order(S)
    return np.sort(order[:min(k, len(order))])


def ratio_budget_pages(P: int, ratio: float, topk_val: int, bos: int, eos: int) -> int:
    """[WEBARENA] "Method configurations at a glance": the number of kept
    blocks is max(topk_val + bos + eos, int(cached_block_len * topk_ratio)),
    with cached_block_len read as the number of pages P and int() as floor
    (ratio > 0).  Capped at P."""
    k = max(topk_val + bos + eos, int(math.floor(P * ratio)))
    return min(P, k)


def forced_pages(P: int, bos: int, eos: int) -> np.ndarray:
    """The first `bos` pages and the last `eos` pages (the last one holds the
    newest token), deduplicated, ascending."""
    f = set(range(min(bos, P))) | set(range(max(0, P - eos), P))
    return np.array(sorted(f), dtype=np.int64)


def select_ratio(S, ratio: float, topk_val: int, bos: int, eos: int) -> np.ndarray:
    """Ratio budget with forced bos/eos pages: the forced pages, then the best
    of the remaining pages in rank order until the budget is reached."""
    P = len(S)
    K = ratio_budget_pages(P, ratio, topk_val, bos, eos)
    forced = forced_pages(P, bos, eos)
    fset = set(int(x) for x in forced)
    rest = [int(p) for p in rank_order(S) if int(p) not in fset]
    take = max(0, K - len(forced))
    return np.array(sorted(list(fset) + rest[:take]), dtype=np.int64)


def select_token_budget(S, lens, budget: int, skip: bool = False) -> np.ndarray:
    """Token budget over variable chunks ([OFFLINE] "Headline results": TSA at
    budgets 4096/8192/16384).  Greedy by score: walk the rank order and take
    chunks while the running token count stays within the budget; stop at the
    first chunk that does not fit (skip=False, the reading used), or skip it
    and continue (skip=True, alternative reading)."""
    lens = np.asarray(lens, dtype=np.int64)
    taken = []
    used = 0
    for p in rank_order(S):
        L = int(lens[p])
        if used + L <= budget:
            taken.append(int(p))
            used += L
        elif not skip:
            break
    return np.array(sorted(taken), dtype=np.int64)


# --------------------------------------------------------------------------
# 5. Exact softmax attention over the selected tokens only.
# [OFFLINE] "The comparison": attend only to the kept chunks.
# --------------------------------------------------------------------------

def tokens_of(sel, starts, ends) -> np.ndarray:
    """Ascending token indices covered by the selected pages."""
    if len(sel) == 0:
        return np.zeros(0, dtype=np.int64)
    toks = np.concatenate([np.arange(starts[p], ends[p]) for p in np.sort(sel)])
    return toks.astype(np.int64)


def attend(Q, K, V, toks, scale: float):
    """Q: [H, D]; K, V: [N, D]; toks: attended token indices.
    Returns out[H, D] and lse[H] (natural log of the softmax denominator of
    the scaled logits).  An empty token set gives out = 0, lse = -inf."""
    Q = f64(Q)
    H, D = Q.shape
    if len(toks) == 0:
        return np.zeros((H, D)), np.full(H, NEG_INF)
    Ks = f64(K)[toks]
    Vs = f64(V)[toks]
    out = np.empty((H, D))
    lse = np.empty(H)
    for h in range(H):
        z = scale * (Ks @ Q[h])
        m = z.max()
        e = np.exp(z - m)
        l = e.sum()
        out[h] = (e @ Vs) / l
        lse[h] = m + math.log(l)
    return out, lse


@dataclass
class UnitResult:
    scores: np.ndarray      # [P] group score per page
    head_scores: np.ndarray  # [G, P]
    selected: np.ndarray    # ascending page indices
    out: np.ndarray         # [G, D]
    lse: np.ndarray         # [G]
    n_tokens: int           # tokens attended


def decode_unit(Qg, K, V, n_tokens: int, *, rule: str, page_size: int = 16,
                chunk_off=None, budget: dict, scale: float,
                reduce: str = "max", meta=None) -> UnitResult:
    """One (sequence, KV head) decode step: partition, metadata, per-head
    scores, group reduce, budgeted selection, attention over the selected
    tokens for every query head of the group.

    budget: {'kind': 'topk', 'k': k} | {'kind': 'ratio', 'ratio', 'topk_val',
    'bos', 'eos'} | {'kind': 'tokens', 'budget': B}."""
    if chunk_off is not None:
        starts, ends = chunk_pages(chunk_off)
    else:
        starts, ends = fixed_pages(n_tokens, page_size)
    Kn = f64(K)[:n_tokens]
    Vn = f64(V)[:n_tokens]
    if meta is None:
        meta = page_metadata(Kn, starts, ends)
    sh = head_scores(Qg, meta, rule)
    S = group_reduce(sh, reduce)
    kind = budget["kind"]
    if kind == "topk":
        sel = select_topk(S, budget["k"])
    elif kind == "ratio":
        sel = select_ratio(S, budget["ratio"], budget.get("topk_val", 1),
                           budget["bos"], budget["eos"])
    elif kind == "tokens":
        sel = select_token_budget(S, ends - starts, budget["budget"],
                                  budget.get("skip", False))
    else:
        raise ValueError(kind)
    toks = tokens_of(sel, starts, ends)
    out, lse = attend(Qg, Kn, Vn, toks, scale)
    return UnitResult(S, sh, sel, out, lse, len(toks))


# --------------------------------------------------------------------------
# 6. Uncertainty router over query tiles ([ROUTER] "Methodologie").
# --------------------------------------------------------------------------

def tile_block_scores(Qtile, meta, rule: str, rows_per_batch: int = 8, fast: bool = False) -> np.ndarray:
    """Step 2: the tile score of a block is the maximum, over the tile's rows
    (and, under GQA, the query heads that share the KV head), of the per-row
    block score.  Qtile: [R, G, D] -> scores [P].  fast=True evaluates the
    per-row scores as matrix products (envelope_scores_matmul)."""
    Qtile = f64(Qtile)
    R, G, D = Qtile.shape
    flat = Qtile.reshape(R * G, D)
    if fast:
        return head_scores(flat, meta, rule, fast=True).max(axis=0)
    best = None
    for i in range(0, flat.shape[0], rows_per_batch):
        s = head_scores(flat[i:i + rows_per_batch], meta, rule)  # [r, P]
        m = s.max(axis=0)
        best = m if best is None else np.maximum(best, m)
    return best


def sigma_margin(S_sorted, k: int) -> float:
    """Step 3: normalised cut-off margin on the descending block scores
    s_(0) >= s_(1) >= ...:  sigma = (s_(k-1) - s_(k)) / (s_(0) - s_(k)).
    With no block beyond the first k there is no cut and sigma = 1; if
    s_(0) = s_(k) every kept score ties the first dropped one and sigma = 0."""
    S_sorted = f64(S_sorted)
    E = len(S_sorted)
    if E <= k:
        return 1.0
    s0, skm1, sk = S_sorted[0], S_sorted[k - 1], S_sorted[k]
    den = s0 - sk
    if den == 0.0:
        return 0.0
    return float((skm1 - sk) / den)


def quantile_linear(values, q: float) -> float:
    """Per-layer empirical quantile (linear interpolation between order
    statistics at h = (T-1) q)."""
    v = np.sort(f64(values))
    T = len(v)
    h = (T - 1) * q
    lo = int(math.floor(h))
    hi = min(lo + 1, T - 1)
    return float(v[lo] + (h - lo) * (v[hi] - v[lo]))


@dataclass
class RouteResult:
    kv_idx: np.ndarray     # [T, Hkv, rho*k] int64, -1 = sentinel
    kv_count: np.ndarray   # [T, Hkv]
    sigma: np.ndarray      # [T, Hkv]
    sigma_bar: np.ndarray  # [T]
    tau: float
    triggered: np.ndarray  # [T] bool
    scores: np.ndarray     # [T, Hkv, P] tile scores (-inf for ineligible)


def route(Q, metas, rule: str, *, q_pos0: int, tile_rows: int, block_size: int,
          n_blocks: int, k: int, rho: int, quantile: float, tau=None,
          score_fn=None, fast: bool = False) -> RouteResult:
    """Steps 2-5 over all tiles of one layer.

    Q: [rows, Hq, D] query rows at positions q_pos0 .. q_pos0+rows-1.
    metas[g] = (kmin, kmax, kmean) of KV head g, each [n_blocks, D].
    A block is eligible for a tile when its first token is not after the
    tile's last row (causality).  Lists are in rank order, padded with -1 to
    rho*k entries; non-triggered tiles keep only the first k."""
    Q = f64(Q)
    rows, Hq, D = Q.shape
    Hkv = len(metas)
    G = Hq // Hkv
    T = -(-rows // tile_rows)
    W = rho * k
    kv_idx = np.full((T, Hkv, W), -1, dtype=np.int64)
    kv_count = np.zeros((T, Hkv), dtype=np.int64)
    sigma = np.zeros((T, Hkv))
    scores = np.full((T, Hkv, n_blocks), NEG_INF)
    orders = {}
    for t in range(T):
        r0 = t * tile_rows
        r1 = min(rows, r0 + tile_rows)
        last_pos = q_pos0 + r1 - 1
        E = min(n_blocks, last_pos // block_size + 1)
        for g in range(Hkv):
            Qt = Q[r0:r1, g * G:(g + 1) * G, :]
            if score_fn is not None:
                S = score_fn(t, g)
            else:
                S = tile_block_scores(Qt, metas[g], rule, fast=fast)
            S = S[:E]
            scores[t, g, :E] = S
            order = rank_order(S)
            orders[(t, g)] = order
            sigma[t, g] = sigma_margin(S[order], k)
    sigma_bar = sigma.mean(axis=1)
    if tau is None:
        tau = quantile_linear(sigma_bar, quantile)
    triggered = sigma_bar < tau
    for t in range(T):
        for g in range(Hkv):
            order = orders[(t, g)]
            n = min(W if triggered[t] else k, len(order))
            kv_idx[t, g, :n] = order[:n]
            kv_count[t, g] = n
    return RouteResult(kv_idx, kv_count, sigma, sigma_bar, float(tau), triggered, scores)


def route_decode(unit_scores, *, k: int, rho: int, quantile: float, tau=None) -> RouteResult:
    """Steps 3-5 with tiles of one query row: in a decode batch, sequence b is
    a tile whose only row is its newest token, so every page of the sequence
    is eligible, and its block scores for KV head g are the decode group
    scores S(p) (group_reduce of head_scores).  unit_scores[b][g]: those
    scores, [P_b].  sigma per (b, g) on the descending scores, sigma_bar the
    mean over KV heads, tau the linear quantile of sigma_bar over the batch's
    sequences (or the given tau), trigger iff sigma_bar < tau; lists in rank
    order, the first rho*k (triggered) or k pages, padded with -1."""
    B = len(unit_scores)
    Hkv = len(unit_scores[0])
    W = rho * k
    Pmax = max(len(unit_scores[b][g]) for b in range(B) for g in range(Hkv))
    kv_idx = np.full((B, Hkv, W), -1, dtype=np.int64)
    kv_count = np.zeros((B, Hkv), dtype=np.int64)
    sigma = np.zeros((B, Hkv))
    scores = np.full((B, Hkv, Pmax), NEG_INF)
    orders = {}
    for b in range(B):
        for g in range(Hkv):
            S = f64(unit_scores[b][g])
            scores[b, g, :len(S)] = S
            order = rank_order(S)
            orders[(b, g)] = order
            sigma[b, g] = sigma_margin(S[order], k)
    sigma_bar = sigma.mean(axis=1)
    if tau is None:
        tau = quantile_linear(sigma_bar, quantile)
    triggered = sigma_bar < tau
    for b in range(B):
        for g in range(Hkv):
            order = orders[(b, g)]
            n = min(W if triggered[b] else k, len(order))
            kv_idx[b, g, :n] = order[:n]
            kv_count[b, g] = n
    return RouteResult(kv_idx, kv_count, sigma, sigma_bar, float(tau), triggered, scores)


def tile_attention(Q, K, V, kv_idx, *, q_pos0: int, tile_rows: int,
                   block_size: int, n_tokens: int, scale: float):
    """Causal softmax attention of every query row over the tokens of its
    tile's selected blocks (sentinels skipped).  Row r (position q_pos0 + r),
    query head h of KV group g attends to the tokens t <= position of the
    blocks in kv_idx[tile, g].  A row that sees no token gets out = 0 and
    lse = -inf.

    Q: [rows, Hq, D]; K, V: [Hkv][N, D] lists; returns out [rows, Hq, D],
    lse [rows, Hq]."""
    Q = f64(Q)
    rows, Hq, D = Q.shape
    Hkv = len(K)
    G = Hq // Hkv
    T = -(-rows // tile_rows)
    out = np.zeros((rows, Hq, D))
    lse = np.full((rows, Hq), NEG_INF)
    for g in range(Hkv):
        for t in range(T):
            blocks = sorted(int(b) for b in kv_idx[t, g] if b >= 0)
            toks = [np.arange(b * block_size, min((b + 1) * block_size, n_tokens))
                    for b in blocks]
            toks = np.concatenate(toks) if toks else np.zeros(0, dtype=np.int64)
            Kt = f64(K[g][toks]) if len(toks) else None
            Vt = f64(V[g][toks]) if len(toks) else None
            for r in range(t * tile_rows, min(rows, (t + 1) * tile_rows)):
                pos = q_pos0 + r
                vis = np.nonzero(toks <= pos)[0]
                for j in range(G):
                    h = g * G + j
                    o, l = attend(Q[r, h][None, :], Kt, Vt, vis, scale)
                    out[r, h] = o[0]
                    lse[r, h] = l[0]
    return out, lse
