"""Per-unit parity check of one (sequence, KV head) -- or (sequence, query
head) -- unit against the float64 oracle, on host arrays only (numpy; no
torch, no CUDA, no product code), so that it can run in spawned worker
processes as well as in the test process.

A unit's host data: its query heads Q [G, 128], keys and values [N, 128]
(exact bf16 values as float32), and its page or chunk ranges.  Each run of
the CUDA path over the same cache contributes its metadata row (raw bytes),
optional group scores, kept pages (ascending) and outputs for the unit's
query heads.  For every run the oracle's metadata, scores, selection
certificate (tests/certify.py) and attention over the pages the GPU kept are
compared; the oracle's metadata is computed once per unit.
"""
from __future__ import annotations

import numpy as np

import oracle as O
from certify import certify_selection

OUT_TOL = 2e-3


def check_unit(host: dict, runs: list, *, scale: float, score_rel: float = 2e-6,
               out_tol: float = OUT_TOL, where: str = "") -> list:
    """host: dict(Q, K, V, starts, ends, chunks: bool).
    runs: list of dict(rule, budget, meta (uint8 [P, 512]), scores ([P] or
    None), sel (int64 ascending), out [G, 128], lse [G]).
    Returns one stats dict per run; raises AssertionError on a mismatch."""
    Q = np.asarray(host["Q"], dtype=np.float64)
    K = np.asarray(host["K"], dtype=np.float64)
    V = np.asarray(host["V"], dtype=np.float64)
    starts, ends = host["starts"], host["ends"]
    meta = O.page_metadata(K, starts, ends)
    P = len(starts)
    lens = (ends - starts) if host["chunks"] else None
    res = []
    for r in runs:
        rule, budget = r["rule"], r["budget"]
        w = f"{where} [{rule} {budget}]"
        st = dict(max_out_err=0.0, max_lse_err=0.0, max_score_err=0.0, tie=False)
        gm = np.ascontiguousarray(r["meta"][:P])
        if rule == "envelope":
            mm = gm.view(np.uint16).astype(np.uint32) << 16  # bf16 -> fp32 bit patterns
            mm = mm.view(np.float32).astype(np.float64)
            gmin, gmax = mm[:, :128], mm[:, 128:]
            assert np.array_equal(gmin, meta[0]) and np.array_equal(gmax, meta[1]), f"{w}: envelope metadata"
        else:
            gmean = gm.view(np.float32).astype(np.float64)
            ref32 = meta[2].astype(np.float32).astype(np.float64)
            ulp = np.spacing(np.abs(ref32).astype(np.float32)).astype(np.float64)
            assert np.all(np.abs(gmean - ref32) <= ulp), f"{w}: centroid metadata"
        S = O.group_reduce(O.head_scores(Q, meta, rule))
        if r.get("scores") is not None:
            gs = np.asarray(r["scores"][:P], dtype=np.float64)
            err = np.abs(gs - S) / np.maximum(np.abs(S), 1.0)
            st["max_score_err"] = float(err.max())
            assert err.max() <= score_rel, f"{w}: score rel err {err.max():.3g}"
        gl = np.asarray(r["sel"], dtype=np.int64)
        assert np.all(np.diff(gl) > 0), f"{w}: selection not strictly ascending"
        gset = set(int(x) for x in gl)
        st["tie"] = bool(certify_selection(S, gset, budget, lens, w))
        toks = O.tokens_of(gl, starts, ends)
        o_ref, l_ref = O.attend(Q, K, V, toks, scale)
        o_gpu = np.asarray(r["out"], dtype=np.float64)
        l_gpu = np.asarray(r["lse"], dtype=np.float64)
        if len(toks) == 0:
            assert np.all(o_gpu == 0) and np.all(np.isneginf(l_gpu)), f"{w}: empty selection"
        else:
            e = float(np.abs(o_gpu - o_ref).max())
            le = float(np.abs(l_gpu - l_ref).max())
            st["max_out_err"], st["max_lse_err"] = e, le
            assert e <= out_tol, f"{w}: out max-abs err {e:.3g}"
            assert le <= 1e-3 * max(1.0, float(np.abs(l_ref).max())), f"{w}: lse err {le:.3g}"
        res.append(st)
    return res


def check_unit_task(task):
    """Pool entry: (host, runs, kwargs) -> (ok, stats or message)."""
    host, runs, kw = task
    try:
        return True, check_unit(host, runs, **kw)
    except AssertionError as e:
        return False, str(e)


# ---------------------------------------------------------------------------
# Tile attention (the router's multi-row tiles) in worker processes: K and V
# of every KV head are read from .npy files (memory-mapped, loaded once per
# worker), so a task carries only its tile's rows and lists.
_KV_CACHE = {}


def _kv_arrays(npy_dir: str, Hkv: int):
    if _KV_CACHE.get("dir") != npy_dir:
        import os
        _KV_CACHE.clear()
        _KV_CACHE["dir"] = npy_dir
        _KV_CACHE["K"] = [np.load(os.path.join(npy_dir, f"k{g}.npy"), mmap_mode="r") for g in range(Hkv)]
        _KV_CACHE["V"] = [np.load(os.path.join(npy_dir, f"v{g}.npy"), mmap_mode="r") for g in range(Hkv)]
    return _KV_CACHE["K"], _KV_CACHE["V"]


def check_tile_task(task):
    """task: dict(npy_dir, Hkv, t, Q [rows_t, Hq, D], idx [1, Hkv, W], out, lse,
    q_pos0 (of the tile's first row), tile_rows, block_size, n_tokens, scale,
    out_tol).  Returns (ok, max-abs error or message)."""
    try:
        K, V = _kv_arrays(task["npy_dir"], task["Hkv"])
        o_ref, l_ref = O.tile_attention(task["Q"], K, V, task["idx"], q_pos0=task["q_pos0"],
                                        tile_rows=task["tile_rows"], block_size=task["block_size"],
                                        n_tokens=task["n_tokens"], scale=task["scale"])
        o = np.asarray(task["out"], dtype=np.float64)
        l = np.asarray(task["lse"], dtype=np.float64)
        t = task["t"]
        dead = np.isneginf(l_ref)
        assert np.array_equal(np.isneginf(l), dead), f"tile {t}: rows without visible keys differ"
        assert np.all(o[dead] == 0), f"tile {t}: rows without visible keys are not zero"
        e = float(np.abs(o - o_ref).max())
        assert e <= task["out_tol"], f"tile {t}: max-abs err {e}"
        le = float(np.abs(l[~dead] - l_ref[~dead]).max()) if (~dead).any() else 0.0
        assert le <= 1e-3, f"tile {t}: lse err {le}"
        return True, e
    except AssertionError as ex:
        return False, str(ex)
