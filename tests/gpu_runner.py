"""Parity harness: run the CUDA path through the C ABI, run the float64 oracle
on host copies of the same bf16 tensors, and compare.

Selection parity (the near-tie certificate): the GPU page set must equal the
oracle's, except when the oracle's last kept score and first dropped score
differ by less than delta = 1e-5 * max(|s_(K-1)|, |s_(K)|, 1).  In that case
pages scoring above the band must be kept, pages below it dropped, and the
count must match.  Attention parity is checked on the set the GPU actually
chose (the oracle attends over the same pages), max-abs error <= 2e-3 on
unit-scale inputs (the tolerance the method's specification states; the
measured errors are far below it).
"""
from __future__ import annotations

import math

import numpy as np
import torch

import block_sparse_kv_page_b200 as sa
import oracle as O
from certify import TIE_REL, certify_selection  # noqa: F401

OUT_TOL = 2e-3


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def budget_struct(bd: dict):
    if bd["kind"] == "topk":
        return sa.budget_topk(bd["k"])
    if bd["kind"] == "ratio":
        return sa.budget_ratio(bd["ratio"], topk_val=bd.get("topk_val", 1), bos=bd["bos"], eos=bd["eos"])
    return sa.budget_tokens(bd["budget"])


def default_max_sel(bd: dict, max_pages: int) -> int:
    if bd["kind"] == "topk":
        return bd["k"]
    if bd["kind"] == "ratio":
        return O.ratio_budget_pages(max_pages, bd["ratio"], bd.get("topk_val", 1), bd["bos"], bd["eos"])
    return max_pages


def run_gpu(layer, *, page_size: int, rule: str, budget: dict, scale: float,
            max_pages: int | None = None, max_sel: int | None = None, ws=None, repeat: int = 1,
            per_head: bool = False):
    """build_meta + select + decode through the C ABI.  per_head: one page set
    per query head (the *_per_head calls); selection rows are then [B, Hq]."""
    B, Hkv, cap, D = layer.k.shape
    Hq = layer.q.shape[1]
    if max_pages is None:
        max_pages = -(-cap // page_size) if page_size else layer.chunk_off.shape[1] - 1
    if max_sel is None:
        max_sel = default_max_sel(budget, max_pages)
    kv = sa.KvCache(layer.k, layer.v, layer.seq_len, page_size=page_size, max_pages=max_pages,
                    chunk_off=layer.chunk_off, n_chunks=layer.n_chunks)
    dev = layer.k.device
    meta = kv.meta_buffer()
    if ws is None:
        ws = (sa.make_workspace_per_head(kv, Hq, max_sel) if per_head
              else sa.make_workspace(kv, Hq, B, max_sel))
    sa.sparse_attn_build_meta(kv, rule, 0, meta)
    U = Hq if per_head else Hkv
    results = []
    for _ in range(repeat):
        sel_idx = torch.full((B, U, max_sel), -7, dtype=torch.int32, device=dev)
        sel_count = torch.full((B, U), -7, dtype=torch.int32, device=dev)
        scores = torch.full((B, U, max_pages), float("nan"), dtype=torch.float32, device=dev)
        out = torch.full((B, Hq, 128), float("nan"), dtype=torch.float32, device=dev)
        lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device=dev)
        if per_head:
            sa.sparse_attn_select_per_head(kv, meta, rule, layer.q, budget_struct(budget), max_sel,
                                           sel_idx, sel_count, scores, ws)
            sa.sparse_attn_decode_per_head(kv, layer.q, scale, sel_idx, sel_count, max_sel, out, lse, ws)
        else:
            sa.sparse_attn_select(kv, meta, rule, layer.q, budget_struct(budget), max_sel,
                                  sel_idx, sel_count, scores, ws)
            sa.sparse_attn_decode(kv, layer.q, B, 0, 1, scale, sel_idx, sel_count, max_sel, out, lse, ws)
        torch.cuda.synchronize()
        results.append(dict(sel_idx=sel_idx.cpu(), sel_count=sel_count.cpu(), scores=scores.cpu(),
                            out=out.cpu(), lse=lse.cpu()))
    status = sa.sparse_attn_get_device_status(ws)
    r = results[0]
    r.update(meta=meta, kv=kv, ws=ws, status=status, max_sel=max_sel, max_pages=max_pages,
             runs=results)
    return r


def run_step(layer, *, page_size: int, rule: str, budget: dict, scale: float,
             max_pages: int | None = None, max_sel: int | None = None, ws=None, repeat: int = 1,
             stale: bool = True, append=None, out_dtype=torch.float32, per_head: bool = False):
    """One-launch decode step through the C ABI.  With `stale`, the metadata is
    first built for the cache as it stood before its newest token (seq_len - 1;
    pages never built hold a fill pattern), so the step's own refresh of the
    newest page is what makes the metadata current.  append = (k_new, v_new):
    run the step that stores the newest token's key and value itself.
    per_head: the step with one page set per query head (rows [B, Hq])."""
    B, Hkv, cap, D = layer.k.shape
    Hq = layer.q.shape[1]
    if max_pages is None:
        max_pages = -(-cap // page_size) if page_size else layer.chunk_off.shape[1] - 1
    if max_sel is None:
        max_sel = default_max_sel(budget, max_pages)
    kv = sa.KvCache(layer.k, layer.v, layer.seq_len, page_size=page_size, max_pages=max_pages,
                    chunk_off=layer.chunk_off, n_chunks=layer.n_chunks)
    dev = layer.k.device
    meta = kv.meta_buffer().fill_(0x5A)
    if stale:
        prev = (layer.seq_len - 1).clamp(min=1).to(torch.int32)
        kv_prev = sa.KvCache(layer.k, layer.v, prev, page_size=page_size, max_pages=max_pages,
                             chunk_off=layer.chunk_off, n_chunks=layer.n_chunks)
        sa.sparse_attn_build_meta(kv_prev, rule, 0, meta)
        # a one-token cache had nothing before its token: forget what was built
        for b in range(B):
            if int(layer.seq_len[b]) == 1:
                meta[b].fill_(0x5A)
    else:
        sa.sparse_attn_build_meta(kv, rule, 0, meta)
    if ws is None:
        ws = sa.make_workspace_per_head(kv, Hq, max_sel) if per_head else sa.make_workspace(kv, Hq, B, max_sel)
    U = Hq if per_head else Hkv
    results = []
    for _ in range(repeat):
        sel_idx = torch.full((B, U, max_sel), -7, dtype=torch.int32, device=dev)
        sel_count = torch.full((B, U), -7, dtype=torch.int32, device=dev)
        out = torch.full((B, Hq, 128), float("nan"), dtype=out_dtype, device=dev)
        lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device=dev)
        if per_head:
            sa.sparse_attn_decode_step_per_head(kv, meta, rule, layer.q, budget_struct(budget), max_sel,
                                                scale, sel_idx, sel_count, out, lse, ws)
        elif append is None:
            sa.sparse_attn_decode_step(kv, meta, rule, layer.q, budget_struct(budget), max_sel, scale,
                                       sel_idx, sel_count, out, lse, ws)
        else:
            sa.sparse_attn_decode_step_append(kv, meta, rule, layer.q, append[0], append[1],
                                              budget_struct(budget), max_sel, scale, sel_idx, sel_count,
                                              out, lse, ws)
        torch.cuda.synchronize()
        results.append(dict(sel_idx=sel_idx.cpu(), sel_count=sel_count.cpu(), out=out.cpu(),
                            lse=lse.cpu()))
    status = sa.sparse_attn_get_device_status(ws)
    r = dict(results[0])
    r.update(scores=None, meta=meta, kv=kv, ws=ws, status=status, max_sel=max_sel,
             max_pages=max_pages, runs=results)
    return r


def check_layer(layer, gpu, *, page_size: int, rule: str, budget: dict, scale: float,
                units=None, score_rel: float = 2e-6, out_tol: float = OUT_TOL, per_head: bool = False,
                host_cache: dict | None = None):
    """Compare every (b, g) unit (or the given subset) with the oracle.
    per_head: units are (b, query head h), each with its own page set; the
    oracle is the same one applied to the single head h (its group is {h}).
    host_cache: a dict that keeps the last unit's host copies of K, V and its
    oracle metadata, so that several runs over the same cache checked unit by
    unit compute them once.
    Returns a dict of statistics (max errors, tie exemptions)."""
    B, Hkv = layer.k.shape[:2]
    Hq = layer.q.shape[1]
    G = Hq // Hkv
    stats = dict(max_out_err=0.0, max_lse_err=0.0, max_score_err=0.0, ties=0, units=0)
    if units is None:
        units = [(b, x) for b in range(B) for x in range(Hq if per_head else Hkv)]
    for b, x in units:
        # x: the unit's row in the selection outputs; g: its KV head; heads [h0, h1)
        g, h0, h1 = (x // G, x, x + 1) if per_head else (x, x * G, (x + 1) * G)
        N = int(layer.seq_len[b])
        where = f"unit(b={b},{'h' if per_head else 'g'}={x})"
        Qg = to_np(layer.q[b, h0:h1])
        key = (id(layer), b, g, N)
        if host_cache is not None and host_cache.get("key") == key:
            K, V, starts, ends, meta = host_cache["val"]
        else:
            K = to_np(layer.k[b, g, :N])
            V = to_np(layer.v[b, g, :N])
            if page_size:
                starts, ends = O.fixed_pages(N, page_size)
            else:
                C = int(layer.n_chunks[b])
                off = layer.chunk_off[b, :C + 1].cpu().numpy().astype(np.int64)
                starts, ends = O.chunk_pages(off)
            meta = O.page_metadata(K, starts, ends)
            if host_cache is not None:
                host_cache["key"] = key
                host_cache["val"] = (K, V, starts, ends, meta)
        P = len(starts)
        # metadata parity
        gm = gpu["meta"][b, g, :P]
        if rule == "envelope":
            gmin = to_np(gm[:, :256].contiguous().view(torch.bfloat16))
            gmax = to_np(gm[:, 256:].contiguous().view(torch.bfloat16))
            assert np.array_equal(gmin, meta[0]) and np.array_equal(gmax, meta[1]), f"{where}: envelope metadata"
        else:
            gmean = gm.contiguous().view(torch.float32).cpu().numpy().astype(np.float64)
            ref32 = meta[2].astype(np.float32).astype(np.float64)
            ulp = np.spacing(np.abs(ref32).astype(np.float32)).astype(np.float64)
            assert np.all(np.abs(gmean - ref32) <= ulp), f"{where}: centroid metadata"
        # scores (when the call under test reports them)
        S = O.group_reduce(O.head_scores(Qg, meta, rule))
        if gpu.get("scores") is not None:
            gs = gpu["scores"][b, x, :P].numpy().astype(np.float64)
            err = np.abs(gs - S) / np.maximum(np.abs(S), 1.0)
            stats["max_score_err"] = max(stats["max_score_err"], float(err.max()))
            assert err.max() <= score_rel, f"{where}: score rel err {err.max():.3g}"
        # selection
        cnt = int(gpu["sel_count"][b, x])
        gl = gpu["sel_idx"][b, x, :cnt].numpy().astype(np.int64)
        assert np.all(np.diff(gl) > 0), f"{where}: selection not strictly ascending"
        gset = set(int(x) for x in gl)
        lens = (ends - starts) if not page_size else None
        if certify_selection(S, gset, budget, lens, where):
            stats["ties"] += 1
        # attention over the pages the GPU kept
        toks = O.tokens_of(gl, starts, ends)
        o_ref, l_ref = O.attend(Qg, K, V, toks, scale)
        o_gpu = gpu["out"][b, h0:h1].numpy().astype(np.float64)
        l_gpu = gpu["lse"][b, h0:h1].numpy().astype(np.float64)
        if len(toks) == 0:
            assert np.all(o_gpu == 0) and np.all(np.isneginf(l_gpu)), f"{where}: empty selection"
        else:
            e = float(np.abs(o_gpu - o_ref).max())
            le = float(np.abs(l_gpu - l_ref).max())
            stats["max_out_err"] = max(stats["max_out_err"], e)
            stats["max_lse_err"] = max(stats["max_lse_err"], le)
            assert e <= out_tol, f"{where}: out max-abs err {e:.3g}"
            assert le <= 1e-3 * max(1.0, float(np.abs(l_ref).max())), f"{where}: lse err {le:.3g}"
        stats["units"] += 1
    return stats


# ---------------------------------------------------------------------------
# Unit checks in spawned worker processes (full-size workloads).
_POOL = None


def oracle_pool():
    """A process pool for the oracle side of the checks.  Spawned (never
    forked: this process holds a CUDA context), one BLAS thread per worker."""
    global _POOL
    if _POOL is None:
        import atexit
        import multiprocessing as mp
        import os
        n = max(1, min(32, len(os.sched_getaffinity(0))))
        keep = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
        for k in keep:
            os.environ[k] = "1"
        try:
            _POOL = mp.get_context("spawn").Pool(n)
        finally:
            for k, v in keep.items():
                if v is None:
                    os.environ.pop(k, None)
                else:
                    os.environ[k] = v
        atexit.register(_POOL.terminate)
    return _POOL


def _host_f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def check_units_parallel(layer, runs, *, page_size: int, scale: float, units=None,
                         score_rel: float = 2e-6, out_tol: float = OUT_TOL, per_head: bool = False,
                         batch_units: int | None = None):
    """Check the given units (default: all) of every run against the oracle,
    several units at a time in the oracle pool.  runs: list of (gpu, rule,
    budget) over the same cache, gpu as returned by run_gpu / run_step.
    Returns aggregate statistics per run (max errors, certified ties)."""
    import unit_check
    B, Hkv = layer.k.shape[:2]
    Hq = layer.q.shape[1]
    G = Hq // Hkv
    if units is None:
        units = [(b, x) for b in range(B) for x in range(Hq if per_head else Hkv)]
    pool = oracle_pool()
    if batch_units is None:
        batch_units = 2 * pool._processes
    agg = [dict(max_out_err=0.0, max_lse_err=0.0, max_score_err=0.0, ties=0, units=0) for _ in runs]
    kw = dict(scale=scale, score_rel=score_rel, out_tol=out_tol)

    def task(b, x):
        g, h0, h1 = (x // G, x, x + 1) if per_head else (x, x * G, (x + 1) * G)
        N = int(layer.seq_len[b])
        if page_size:
            starts, ends = O.fixed_pages(N, page_size)
        else:
            C = int(layer.n_chunks[b])
            off = layer.chunk_off[b, :C + 1].cpu().numpy().astype(np.int64)
            starts, ends = O.chunk_pages(off)
        P = len(starts)
        host = dict(Q=_host_f32(layer.q[b, h0:h1]), K=_host_f32(layer.k[b, g, :N]),
                    V=_host_f32(layer.v[b, g, :N]), starts=starts, ends=ends, chunks=not page_size)
        rr = []
        for gpu, rule, budget in runs:
            cnt = int(gpu["sel_count"][b, x])
            sc = gpu.get("scores")
            rr.append(dict(rule=rule, budget=budget,
                           meta=gpu["meta"][b, g, :P].cpu().numpy(),
                           scores=None if sc is None else sc[b, x, :P].numpy(),
                           sel=gpu["sel_idx"][b, x, :cnt].numpy().astype(np.int64),
                           out=gpu["out"][b, h0:h1].float().numpy(),
                           lse=gpu["lse"][b, h0:h1].numpy()))
        return host, rr, dict(kw, where=f"unit(b={b},{'h' if per_head else 'g'}={x})")

    for i in range(0, len(units), batch_units):
        tasks = [task(b, x) for b, x in units[i:i + batch_units]]
        for ok, val in pool.map(unit_check.check_unit_task, tasks, chunksize=1):
            assert ok, val
            for a, s in zip(agg, val):
                a["max_out_err"] = max(a["max_out_err"], s["max_out_err"])
                a["max_lse_err"] = max(a["max_lse_err"], s["max_lse_err"])
                a["max_score_err"] = max(a["max_score_err"], s["max_score_err"])
                a["ties"] += int(s["tie"])
                a["units"] += 1
    return agg
