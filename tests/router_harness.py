"""Router parity harness: run sparse_attn_route through the C ABI and compare
with the float64 oracle ("Onzekerheidsgestuurde Selectie voor Blok-schaarse
Aandacht", "Methodologie" steps 2-5).

Checks, per (tile, KV head):
* the kept set equals the oracle's, except where a near-tie at the cut is
  certified (|s_(n-1) - s_(n)| < 1e-5 * max(|s|, 1), as for page selection);
* the list is in rank order: oracle scores non-increasing up to that same
  tolerance, lower index first on equal scores; entries past the count are -1;
* sigma within 1e-4 of the oracle's; sigma_bar and tau within 1e-4;
* triggers equal, except tiles whose oracle sigma_bar is within 1e-4 of tau
  (a decision that rounding may flip).
"""
from __future__ import annotations

import math

import numpy as np
import torch

import block_sparse_kv_page_b200 as sa
import oracle as O

TIE_REL = 1e-5
SIG_TOL = 1e-4


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def run_route_gpu(k_cache, q, *, rule, block, q_pos0, tile_rows, k, rho, quantile, tau=None):
    """k_cache: bf16 [1, Hkv, N, 128]; q: bf16 [rows, Hq, 128]."""
    dev = k_cache.device
    _, Hkv, N, D = k_cache.shape
    rows, Hq, _ = q.shape
    P = -(-N // block)
    sl = torch.tensor([N], dtype=torch.int32, device=dev)
    kv = sa.KvCache(k_cache, k_cache, sl, page_size=block, max_pages=P)
    meta = kv.meta_buffer()
    sa.sparse_attn_build_meta(kv, rule, 0, meta)
    T = -(-rows // tile_rows)
    W = rho * k
    ws = sa.make_workspace(kv, Hq, rows, W)
    kv_idx = torch.full((T, Hkv, W), -7, dtype=torch.int32, device=dev)
    kv_count = torch.full((T, Hkv), -7, dtype=torch.int32, device=dev)
    sigma = torch.full((T, Hkv), float("nan"), dtype=torch.float32, device=dev)
    sbar = torch.full((T,), float("nan"), dtype=torch.float32, device=dev)
    trig = torch.full((T,), 7, dtype=torch.uint8, device=dev)
    tau_out = torch.full((1,), float("nan"), dtype=torch.float32, device=dev)
    tau_t = None if tau is None else torch.tensor([tau], dtype=torch.float32, device=dev)
    sa.sparse_attn_route(kv, meta, rule, q, rows, q_pos0, tile_rows, k, rho, quantile, tau_t,
                         kv_idx, kv_count, sigma, sbar, trig, tau_out, ws)
    torch.cuda.synchronize()
    status = sa.sparse_attn_get_device_status(ws)
    return dict(kv_idx=kv_idx.cpu().numpy(), kv_count=kv_count.cpu().numpy(),
                sigma=sigma.cpu().numpy().astype(np.float64), sigma_bar=sbar.cpu().numpy().astype(np.float64),
                triggered=trig.cpu().numpy().astype(bool), tau=float(tau_out.item()), status=status,
                meta=meta, kv=kv, ws=ws)


def run_route_oracle(k_cache, q, *, rule, block, q_pos0, tile_rows, k, rho, quantile, tau=None):
    _, Hkv, N, D = k_cache.shape
    s, e = O.fixed_pages(N, block)
    metas = [O.page_metadata(to_np(k_cache[0, g]), s, e) for g in range(Hkv)]
    return O.route(to_np(q), metas, rule, q_pos0=q_pos0, tile_rows=tile_rows, block_size=block,
                   n_blocks=len(s), k=k, rho=rho, quantile=quantile, tau=tau, fast=True)


def compare(gpu, ref, *, k, rho):
    T, Hkv = ref.kv_count.shape
    W = rho * k
    stats = dict(ties=0, trig_exempt=0, max_sigma_err=0.0)
    assert gpu["status"] == 0, f"device status {gpu['status']}"
    assert abs(gpu["tau"] - ref.tau) <= SIG_TOL, f"tau {gpu['tau']} vs {ref.tau}"
    assert np.all(np.abs(gpu["sigma_bar"] - ref.sigma_bar) <= SIG_TOL), "sigma_bar"
    err = np.abs(gpu["sigma"] - ref.sigma)
    stats["max_sigma_err"] = float(err.max())
    assert err.max() <= SIG_TOL, f"sigma err {err.max()}"
    for t in range(T):
        exempt = abs(ref.sigma_bar[t] - ref.tau) < SIG_TOL
        if gpu["triggered"][t] != ref.triggered[t]:
            assert exempt, f"tile {t}: trigger differs away from tau"
            stats["trig_exempt"] += 1
        for g in range(Hkv):
            S = ref.scores[t, g]
            E = int(np.isfinite(S).sum())
            S = S[:E]
            n = int(gpu["kv_count"][t, g])
            row = gpu["kv_idx"][t, g]
            assert np.all(row[n:] == -1) and np.all(row[:n] >= 0), f"({t},{g}) sentinels"
            n_ref = int(ref.kv_count[t, g])
            if gpu["triggered"][t] == ref.triggered[t]:
                assert n == n_ref, f"({t},{g}) count {n} vs {n_ref}"
            lst = [int(x) for x in row[:n]]
            assert len(set(lst)) == n and all(x < E for x in lst), f"({t},{g}) invalid entries"
            order = O.rank_order(S)
            oset = set(int(x) for x in order[:n])
            if set(lst) != oset:
                a, b = S[order[n - 1]], S[order[n]]
                delta = TIE_REL * max(abs(a), abs(b), 1.0)
                assert a - b < delta, f"({t},{g}) set differs at a decisive cut"
                for p in order:
                    p = int(p)
                    if S[p] > a + delta:
                        assert p in lst, f"({t},{g}) block {p} above the tie band missing"
                    if S[p] < b - delta:
                        assert p not in lst, f"({t},{g}) block {p} below the tie band kept"
                stats["ties"] += 1
            for i in range(n - 1):
                x, y = S[lst[i]], S[lst[i + 1]]
                d = TIE_REL * max(abs(x), abs(y), 1.0)
                assert x >= y - d, f"({t},{g}) rank order broken at {i}"
                if x == y:
                    assert lst[i] < lst[i + 1], f"({t},{g}) tie not lowest-index first"
    return stats
