"""GPU parity of multi-row tile attention (sparse_attn_decode with
tile_rows > 1) against the float64 oracle's causal tile attention, on the
lists the router produced (so both sides attend over the same blocks)."""
import math

import numpy as np
import pytest
import torch

import datagen as DG
import oracle as O

pytestmark = pytest.mark.gpu

OUT_TOL = 2e-3
SCALE = 1.0 / math.sqrt(128)


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _tile_attn_gpu(lay, kv_idx, kv_count, *, tile_rows, ws=None):
    import block_sparse_kv_page_b200 as sa
    dev = lay.k.device
    rows, Hq, D = lay.q.shape
    sl = torch.tensor([lay.N], dtype=torch.int32, device=dev)
    kv = sa.KvCache(lay.k, lay.v, sl, page_size=64, max_pages=-(-lay.N // 64))
    if ws is None:
        ws = sa.make_workspace(kv, Hq, rows, kv_idx.shape[-1])
    out = torch.full((rows, Hq, D), float("nan"), dtype=torch.float32, device=dev)
    lse = torch.full((rows, Hq), float("nan"), dtype=torch.float32, device=dev)
    sa.sparse_attn_decode(kv, lay.q, rows, lay.q_pos0, tile_rows, SCALE, kv_idx, kv_count,
                          kv_idx.shape[-1], out, lse, ws)
    torch.cuda.synchronize()
    return out.cpu().numpy(), lse.cpu().numpy(), sa.sparse_attn_get_device_status(ws)


def _check(lay, out, lse, kv_idx, *, tile_rows, tiles=None):
    rows, Hq, D = lay.q.shape
    Hkv = lay.k.shape[1]
    K = [_np(lay.k[0, g]) for g in range(Hkv)]
    V = [_np(lay.v[0, g]) for g in range(Hkv)]
    Q = _np(lay.q)
    idx = kv_idx.cpu().numpy()
    T = idx.shape[0]
    worst = 0.0
    for t in (range(T) if tiles is None else tiles):
        r0, r1 = t * tile_rows, min(rows, (t + 1) * tile_rows)
        o_ref, l_ref = O.tile_attention(Q[r0:r1], K, V, idx[t:t + 1], q_pos0=lay.q_pos0 + r0,
                                        tile_rows=tile_rows, block_size=64, n_tokens=lay.N, scale=SCALE)
        o, l = out[r0:r1].astype(np.float64), lse[r0:r1].astype(np.float64)
        dead = np.isneginf(l_ref)
        assert np.array_equal(np.isneginf(l), dead), f"tile {t}: rows without visible keys differ"
        assert np.all(o[dead] == 0)
        e = float(np.abs(o - o_ref).max())
        worst = max(worst, e)
        assert e <= OUT_TOL, f"tile {t}: max-abs err {e}"
        le = np.abs(l[~dead] - l_ref[~dead]).max() if (~dead).any() else 0.0
        assert le <= 1e-3, f"tile {t}: lse err {le}"
    return worst


@pytest.mark.parametrize("rule", ["envelope", "centroid"])
def test_tile_attention_on_routed_lists(cuda_dev, rule):
    import router_harness as H
    lay = DG.make_router_layer(Hq=28, Hkv=4, N=4096, rows=256, seed=7300, device=cuda_dev)
    g = H.run_route_gpu(lay.k, lay.q, rule=rule, block=64, q_pos0=lay.q_pos0, tile_rows=64,
                        k=8, rho=2, quantile=0.25)
    kv_idx = torch.from_numpy(g["kv_idx"]).to(cuda_dev)
    kv_count = torch.from_numpy(g["kv_count"]).to(cuda_dev)
    out, lse, status = _tile_attn_gpu(lay, kv_idx, kv_count, tile_rows=64)
    assert status == 0
    assert _check(lay, out, lse, kv_idx, tile_rows=64) < 1e-4


@pytest.mark.parametrize("tile_rows", [32, 128])
def test_tile_attention_other_tile_heights(cuda_dev, tile_rows):
    """Tiles of 32 rows (224 query vectors: one CTA, its second Q tile partly
    empty) and 128 rows (896 vectors: four CTAs) on router lists."""
    import router_harness as H
    lay = DG.make_router_layer(Hq=28, Hkv=4, N=4096, rows=256, seed=7600 + tile_rows, device=cuda_dev)
    g = H.run_route_gpu(lay.k, lay.q, rule="envelope", block=64, q_pos0=lay.q_pos0, tile_rows=tile_rows,
                        k=8, rho=2, quantile=0.25)
    kv_idx = torch.from_numpy(g["kv_idx"]).to(cuda_dev)
    kv_count = torch.from_numpy(g["kv_count"]).to(cuda_dev)
    out, lse, status = _tile_attn_gpu(lay, kv_idx, kv_count, tile_rows=tile_rows)
    assert status == 0
    assert _check(lay, out, lse, kv_idx, tile_rows=tile_rows) < 1e-4


def test_tile_attention_ragged_and_sentinels(cuda_dev):
    """Partial last block (N = 4000), a ragged last tile (200 rows, tiles of
    64), lists with sentinels in the middle, an empty list, and the diagonal
    block so that causality matters."""
    lay = DG.make_router_layer(Hq=28, Hkv=4, N=4000, rows=200, seed=7400, device=cuda_dev)
    T, Hkv, W = 4, 4, 6
    P = -(-lay.N // 64)
    rng = np.random.default_rng(3)
    idx = np.full((T, Hkv, W), -1, dtype=np.int32)
    cnt = np.zeros((T, Hkv), dtype=np.int32)
    for t in range(T):
        last_pos = lay.q_pos0 + min(200, (t + 1) * 64) - 1
        diag = last_pos // 64
        for g in range(Hkv):
            if (t, g) == (1, 2):
                continue  # empty list: every row gets out = 0, lse = -inf
            blocks = [diag] + list(rng.choice(diag, size=3, replace=False))
            if t == T - 1:
                blocks.append(P - 1)  # the partial block
            row = blocks[:2] + [-1] + blocks[2:]
            idx[t, g, :len(row)] = row
            cnt[t, g] = len(row)
    kv_idx = torch.from_numpy(idx).to(cuda_dev)
    kv_count = torch.from_numpy(cnt).to(cuda_dev)
    out, lse, status = _tile_attn_gpu(lay, kv_idx, kv_count, tile_rows=64)
    assert status == 0
    assert _check(lay, out, lse, kv_idx, tile_rows=64) < 1e-4
    assert np.all(out[64:128, 14:21] == 0) and np.all(np.isneginf(lse[64:128, 14:21]))


def test_tile_attention_flags_out_of_range_block(cuda_dev):
    import block_sparse_kv_page_b200 as sa
    lay = DG.make_router_layer(Hq=28, Hkv=4, N=1024, rows=64, seed=7500, device=cuda_dev)
    idx = np.array([[[0, 5, 999]] * 4], dtype=np.int32)
    cnt = np.full((1, 4), 3, dtype=np.int32)
    kv_idx = torch.from_numpy(idx).to(cuda_dev)
    out, lse, status = _tile_attn_gpu(lay, kv_idx, torch.from_numpy(cnt).to(cuda_dev), tile_rows=64)
    assert status == sa.SA_ERR_DEVICE_CHECK
    idx[:, :, 2] = -1
    assert _check(lay, out, lse, torch.from_numpy(idx), tile_rows=64) < 1e-4


def _check_all_tiles_parallel(lay, out, lse, kv_idx, *, tile_rows):
    """Every tile x KV head of a full-size run against the oracle, one tile per
    task in the oracle's worker pool (K and V handed over as .npy files)."""
    import os
    import shutil
    import tempfile

    import gpu_runner
    import unit_check
    rows, Hq, D = lay.q.shape
    Hkv = lay.k.shape[1]
    idx = kv_idx.cpu().numpy()
    T = idx.shape[0]
    Q = lay.q.float().cpu().numpy()
    d = tempfile.mkdtemp(prefix="tile_attn_kv_")
    try:
        for g in range(Hkv):
            np.save(os.path.join(d, f"k{g}.npy"), lay.k[0, g].float().cpu().numpy())
            np.save(os.path.join(d, f"v{g}.npy"), lay.v[0, g].float().cpu().numpy())
        tasks = []
        for t in range(T):
            r0, r1 = t * tile_rows, min(rows, (t + 1) * tile_rows)
            tasks.append(dict(npy_dir=d, Hkv=Hkv, t=t, Q=Q[r0:r1], idx=idx[t:t + 1], out=out[r0:r1],
                              lse=lse[r0:r1], q_pos0=lay.q_pos0 + r0, tile_rows=tile_rows, block_size=64,
                              n_tokens=lay.N, scale=SCALE, out_tol=OUT_TOL))
        worst = 0.0
        for ok, val in gpu_runner.oracle_pool().map(unit_check.check_tile_task, tasks, chunksize=1):
            assert ok, val
            worst = max(worst, val)
        return worst
    finally:
        shutil.rmtree(d, ignore_errors=True)


@pytest.mark.parametrize("rule", ["envelope", "centroid"])
def test_tile_attention_full_128k(cuda_dev, rule):
    """The full router workload: route, then tile attention over the 32
    tiles' lists; every tile and KV head (all 2048 rows x 28 heads) is checked
    against the oracle."""
    import router_harness as H
    lay = DG.make_router_layer(device=cuda_dev)
    g = H.run_route_gpu(lay.k, lay.q, rule=rule, block=64, q_pos0=lay.q_pos0, tile_rows=64,
                        k=32, rho=2, quantile=0.25)
    kv_idx = torch.from_numpy(g["kv_idx"]).to(cuda_dev)
    kv_count = torch.from_numpy(g["kv_count"]).to(cuda_dev)
    out, lse, status = _tile_attn_gpu(lay, kv_idx, kv_count, tile_rows=64)
    assert status == 0
    worst = _check_all_tiles_parallel(lay, out, lse, kv_idx, tile_rows=64)
    print(f"\n{rule}: 32 tiles x 4 KV heads, max-abs error {worst:.3g}")
    assert worst < 1e-4
