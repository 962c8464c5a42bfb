"""GPU parity of the decode path (metadata -> score + budgeted top-k ->
split-K attention + combine) against the float64 oracle, through the C ABI.

Sizes span several 16-page tiles, several splits and ragged tails; edge cases
cover one-token caches, a single partial page, budgets above the page count,
an empty token budget, exact duplicate pages and a bad page index.
"""
import math

import numpy as np
import pytest
import torch

import datagen as DG
import oracle as O

pytestmark = pytest.mark.gpu

SCALE = 1.0 / math.sqrt(128)


@pytest.fixture(scope="module")
def R():
    import gpu_runner
    return gpu_runner


def _layer(dev, B, Hq, Hkv, seq_lens, seed, **kw):
    return DG.make_decode_layer(B=B, Hq=Hq, Hkv=Hkv, seq_lens=seq_lens, seed=seed, device=dev, **kw)


@pytest.mark.parametrize("rule", ["envelope", "centroid"])
@pytest.mark.parametrize("Hq,Hkv", [(32, 4), (28, 4), (8, 8), (64, 8)])
@pytest.mark.parametrize("ps,k", [(16, 24), (64, 6)])
def test_topk_small(cuda_dev, R, rule, Hq, Hkv, ps, k):
    lay = _layer(cuda_dev, 2, Hq, Hkv, [1000, 777], seed=11 + Hq + ps, cap=1024, key_scale="channel")
    g = R.run_gpu(lay, page_size=ps, rule=rule, budget={"kind": "topk", "k": k}, scale=SCALE)
    assert g["status"] == 0
    st = R.check_layer(lay, g, page_size=ps, rule=rule, budget={"kind": "topk", "k": k}, scale=SCALE)
    assert st["units"] == 2 * Hkv
    assert st["max_out_err"] < 1e-4


@pytest.mark.parametrize("rule,bos,eos", [("centroid", 1, 1), ("envelope", 0, 1), ("envelope", 2, 3)])
@pytest.mark.parametrize("ratio", [0.25, 0.0625, 0.015625])
def test_ratio_small(cuda_dev, R, rule, bos, eos, ratio):
    lay = _layer(cuda_dev, 3, 64, 8, [2048, 1999, 40], seed=21)
    bd = {"kind": "ratio", "ratio": ratio, "bos": bos, "eos": eos}
    g = R.run_gpu(lay, page_size=16, rule=rule, budget=bd, scale=SCALE)
    assert g["status"] == 0
    R.check_layer(lay, g, page_size=16, rule=rule, budget=bd, scale=SCALE)


@pytest.mark.parametrize("budget", [0, 100, 512, 1024, 100000])
def test_token_budget_small(cuda_dev, R, budget):
    lens = DG.workload3_chunks(2, 3000, seed_offset=1)
    lens[1] = DG.chunk_lengths(np.random.default_rng(5), 1234)
    lay = _layer(cuda_dev, 2, 32, 4, [3000, 1234], seed=31, cap=3000, chunk_lens=lens, chunk_offset_std=0.5)
    bd = {"kind": "tokens", "budget": budget}
    g = R.run_gpu(lay, page_size=0, rule="envelope", budget=bd, scale=SCALE)
    assert g["status"] == 0
    R.check_layer(lay, g, page_size=0, rule="envelope", budget=bd, scale=SCALE)


@pytest.mark.parametrize("rule", ["envelope", "centroid"])
@pytest.mark.parametrize("N", [1, 15, 16, 17, 31])
def test_tiny_caches(cuda_dev, R, rule, N):
    lay = _layer(cuda_dev, 1, 32, 4, [N], seed=41 + N, cap=64)
    for k in (1, 2, 5):
        bd = {"kind": "topk", "k": k}
        g = R.run_gpu(lay, page_size=16, rule=rule, budget=bd, scale=SCALE)
        assert g["status"] == 0
        R.check_layer(lay, g, page_size=16, rule=rule, budget=bd, scale=SCALE)
        P = -(-N // 16)
        assert int(g["sel_count"].min()) == min(k, P)


@pytest.mark.parametrize("rule", ["envelope", "centroid"])
@pytest.mark.parametrize("case", ["topk", "ratio", "tokens"])
def test_per_query_head_selection(cuda_dev, R, rule, case):
    """One page set per query head: each (sequence, query head) is checked
    against the oracle run on that head alone (its group is the head itself)."""
    if case == "tokens":
        lens = DG.workload3_chunks(2, 2000, seed_offset=9)
        lay = _layer(cuda_dev, 2, 32, 4, [2000, 2000], seed=91, cap=2000, chunk_lens=lens,
                     chunk_offset_std=0.5)
        ps, bd = 0, {"kind": "tokens", "budget": 700}
    elif case == "ratio":
        lay = _layer(cuda_dev, 2, 28, 4, [1500, 999], seed=92, cap=1504)
        ps, bd = 16, {"kind": "ratio", "ratio": 0.0625, "bos": 1, "eos": 1}
    else:
        lay = _layer(cuda_dev, 3, 32, 4, [1000, 777, 17], seed=93, cap=1024, key_scale="channel")
        ps, bd = 16, {"kind": "topk", "k": 20}
    g = R.run_gpu(lay, page_size=ps, rule=rule, budget=bd, scale=SCALE, per_head=True)
    assert g["status"] == 0
    st = R.check_layer(lay, g, page_size=ps, rule=rule, budget=bd, scale=SCALE, per_head=True)
    assert st["units"] == lay.k.shape[0] * lay.q.shape[1]
    assert st["max_out_err"] < 1e-4
    # heads of one group pick different pages (else the variant would be moot)
    sel = g["sel_idx"]
    assert not torch.equal(sel[0, 0, :8], sel[0, 1, :8]) or not torch.equal(sel[0, 0, :8], sel[0, 2, :8])


def test_exact_duplicate_pages_lowest_index(cuda_dev, R):
    """Identical pages have identical scores; the lower index must win."""
    lay = _layer(cuda_dev, 1, 32, 4, [512], seed=51, cap=512)
    src = lay.k[0, :, 0:16].clone()
    for p in (5, 9, 20, 31):
        lay.k[0, :, 16 * p:16 * p + 16] = src
        lay.v[0, :, 16 * p:16 * p + 16] = lay.v[0, :, 0:16]
    # make the duplicated content win clearly: scale page 0 and copies up
    for p in (0, 5, 9, 20, 31):
        lay.k[0, :, 16 * p:16 * p + 16] = (src.float() * 3).to(torch.bfloat16)
    for rule in ("envelope", "centroid"):
        for k in (2, 3, 4):
            bd = {"kind": "topk", "k": k}
            g = R.run_gpu(lay, page_size=16, rule=rule, budget=bd, scale=SCALE)
            R.check_layer(lay, g, page_size=16, rule=rule, budget=bd, scale=SCALE)


def test_full_budget_equals_dense(cuda_dev, R):
    """A budget covering the cache keeps every page: the output is dense
    attention (the oracle's dense pin, now for the GPU)."""
    lay = _layer(cuda_dev, 2, 32, 4, [700, 333], seed=61, cap=704)
    g = R.run_gpu(lay, page_size=16, rule="envelope", budget={"kind": "topk", "k": 44}, scale=SCALE)
    for b, N in ((0, 700), (1, 333)):
        for gg in range(4):
            assert int(g["sel_count"][b, gg]) == -(-N // 16)
            Q = R.to_np(lay.q[b, 8 * gg:8 * gg + 8])
            o, l = O.attend(Q, R.to_np(lay.k[b, gg, :N]), R.to_np(lay.v[b, gg, :N]), np.arange(N), SCALE)
            assert np.abs(g["out"][b, 8 * gg:8 * gg + 8].numpy() - o).max() < 1e-4


def test_incremental_meta_equals_full(cuda_dev, R):
    import block_sparse_kv_page_b200 as sa
    for ps, lens in ((16, None), (64, None), (0, DG.workload3_chunks(2, 900, seed_offset=7))):
        lay = _layer(cuda_dev, 2, 32, 4, [900, 900], seed=71, cap=912,
                     chunk_lens=lens, chunk_offset_std=0.5 if lens else 0.0)
        mp = 57 if ps == 16 else (15 if ps == 64 else lay.chunk_off.shape[1] - 1)
        for rule in ("envelope", "centroid"):
            full = None
            for n in (899, 900):
                sl = torch.tensor([n, n], dtype=torch.int32, device=cuda_dev)
                kv = sa.KvCache(lay.k, lay.v, sl, page_size=ps, max_pages=mp,
                                chunk_off=lay.chunk_off, n_chunks=lay.n_chunks)
                if n == 899:
                    inc = kv.meta_buffer().zero_()
                    # chunk tables describe 900 tokens; clip the last chunk by seq_len
                    sa.sparse_attn_build_meta(kv, rule, 0, inc)
                else:
                    sa.sparse_attn_build_meta(kv, rule, -1, inc)
                    full = kv.meta_buffer().zero_()
                    sa.sparse_attn_build_meta(kv, rule, 0, full)
            torch.cuda.synchronize()
            assert torch.equal(inc, full), f"ps={ps} rule={rule}"


def test_deterministic(cuda_dev, R):
    lay = _layer(cuda_dev, 2, 32, 4, [3000, 2500], seed=81, cap=3008, key_scale="channel")
    for rule in ("envelope", "centroid"):
        g = R.run_gpu(lay, page_size=16, rule=rule, budget={"kind": "topk", "k": 64},
                      scale=SCALE, repeat=3)
        r0 = g["runs"][0]
        for r in g["runs"][1:]:
            for key in ("sel_idx", "sel_count", "scores", "out", "lse"):
                a, b = r0[key], r[key]
                assert torch.equal(torch.nan_to_num(a), torch.nan_to_num(b)), key


def test_bad_index_flags_and_skips(cuda_dev, R):
    import block_sparse_kv_page_b200 as sa
    lay = _layer(cuda_dev, 1, 32, 4, [256], seed=91, cap=256)
    kv = sa.KvCache(lay.k, lay.v, lay.seq_len, page_size=16, max_pages=16)
    ws = sa.make_workspace(kv, 32, 1, 4)
    idx = torch.tensor([[[0, 3, 99, 5]] * 4], dtype=torch.int32, device=cuda_dev)
    cnt = torch.full((1, 4), 4, dtype=torch.int32, device=cuda_dev)
    out = torch.empty((1, 32, 128), dtype=torch.float32, device=cuda_dev)
    sa.sparse_attn_decode(kv, lay.q, 1, 0, 1, SCALE, idx, cnt, 4, out, None, ws)
    assert sa.sparse_attn_get_device_status(ws) == sa.SA_ERR_DEVICE_CHECK
    # the valid pages were still attended
    toks = np.concatenate([np.arange(16 * p, 16 * p + 16) for p in (0, 3, 5)])
    Q = R.to_np(lay.q[0, 0:8])
    o, _ = O.attend(Q, R.to_np(lay.k[0, 0]), R.to_np(lay.v[0, 0]), toks, SCALE)
    assert np.abs(out[0, 0:8].cpu().numpy() - o).max() < 1e-4
    assert sa.sparse_attn_get_device_status(ws) == 0  # reading clears it
