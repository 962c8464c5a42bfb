"""Near-tie block pairs for the router workload, placed with the oracle.

For a seeded 30% of (tile, KV head) cells: take the block ranked k-1 (the
last kept one) for that cell and overwrite a low-ranked block with its keys
plus N(0, eps^2) noise, redrawing eps until the oracle's tile-score gap
between the two blocks is in [1e-4, 1e-2) relative -- a near-tie that still
sits above the 1e-5 parity tolerance.  Test infrastructure: uses the oracle.
"""
from __future__ import annotations

import numpy as np
import torch

import datagen as DG
import oracle as O


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def plant_near_ties(lay, *, rule, block, tile_rows, k, frac=0.3, seed=5999, max_tries=24):
    """Modifies lay.k in place.  Returns the list of planted (tile, head, a, b)."""
    q = lay.q
    rows, Hq, D = q.shape
    Hkv = lay.k.shape[1]
    G = Hq // Hkv
    N = lay.N
    T = -(-rows // tile_rows)
    rng = np.random.default_rng(seed)
    gen = torch.Generator(device=lay.k.device)
    gen.manual_seed(seed)
    cells = [(t, g) for t in range(T) for g in range(Hkv)]
    chosen = [cells[i] for i in sorted(rng.choice(len(cells), int(round(frac * len(cells))), replace=False))]
    s, e = O.fixed_pages(N, block)
    planted = []
    Qn = _np(q)
    for g in sorted(set(c[1] for c in chosen)):
        Kg = _np(lay.k[0, g])
        meta = O.page_metadata(Kg, s, e)
        used = set()
        for (t, gg) in chosen:
            if gg != g:
                continue
            r0 = t * tile_rows
            Qt = Qn[r0:r0 + tile_rows, g * G:(g + 1) * G]
            last_pos = lay.q_pos0 + min(rows, r0 + tile_rows) - 1
            E = min(len(s), last_pos // block + 1)
            S = O.tile_block_scores(Qt, meta, rule, fast=True)[:E]
            order = O.rank_order(S)
            a = int(order[k - 1])
            cands = [int(x) for x in order[E // 2:] if int(x) not in used and int(x) != a]
            if not cands:
                continue
            b = cands[int(rng.integers(len(cands)))]
            eps = 1e-2
            for _ in range(max_tries):
                DG.duplicate_block(lay.k, g, a, b, block, eps, gen)
                Kb = _np(lay.k[0, g, b * block:(b + 1) * block])
                mb = O.page_metadata(Kb, np.array([0]), np.array([block]))
                sb = O.tile_block_scores(Qt, mb, rule, fast=True)[0]
                rel = abs(S[a] - sb) / max(abs(S[a]), 1.0)
                if 1e-4 <= rel < 1e-2:
                    break
                eps = eps * 0.5 if rel >= 1e-2 else eps * 2.0
            used.update((a, b))
            Kg[b * block:(b + 1) * block] = _np(lay.k[0, g, b * block:(b + 1) * block])
            meta = O.page_metadata(Kg, s, e)
            planted.append((t, g, a, b))
    return planted
