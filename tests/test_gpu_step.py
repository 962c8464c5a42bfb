"""GPU parity of the one-launch decode step (sparse_attn_decode_step): newest
page metadata refresh + scoring + budgeted top-k + split-K attention in one
persistent launch.

Each case checks the step two ways:
* against the float64 oracle on every unit (metadata of every page, the
  selected set under the near-tie certificate, attention over the kept
  tokens), after building the metadata for the cache as it stood BEFORE its
  newest token, so only the step's own refresh makes it current;
* against the separate calls (build_meta, select, decode) on the same
  inputs: the page sets, outputs and log-sum-exps must be bit-identical,
  since the step runs the same item code with the same splits (under a token
  budget the step splits the attention by the budget: outputs then agree to
  1e-5, page sets still exactly).

Cases span fixed pages of 16 and 64 tokens, G = 7 and 8, ratio budgets with
forced pages, TSA chunks with a token budget and with a chunk-count budget
(both scoring rules), newest tokens that open a new page, one-token caches,
and hundreds of units; the cluster_* cases have few units with at least 16
decode splits each, which the step runs as one thread-block cluster per unit
(one and two decode splits per CTA).
"""
import math

import numpy as np
import pytest
import torch

import datagen as DG

pytestmark = pytest.mark.gpu

SCALE = 1.0 / math.sqrt(128)


@pytest.fixture(scope="module")
def R():
    import gpu_runner
    return gpu_runner


def _case(dev, name):
    """(layer, page_size, budget) of a named case."""
    if name == "ps16_topk":
        lay = DG.make_decode_layer(B=2, Hq=32, Hkv=4, seq_lens=[1000, 777], seed=301, device=dev,
                                   cap=1024, key_scale="channel")
        return lay, 16, {"kind": "topk", "k": 24}
    if name == "ps16_new_page":
        # the newest token opens page 64, page 1 and page 0 respectively
        lay = DG.make_decode_layer(B=3, Hq=32, Hkv=4, seq_lens=[1025, 17, 1], seed=302, device=dev,
                                   cap=1040)
        return lay, 16, {"kind": "topk", "k": 8}
    if name == "ps64_g7":
        lay = DG.make_decode_layer(B=2, Hq=28, Hkv=4, seq_lens=[3000, 2100], seed=303, device=dev,
                                   cap=3008)
        return lay, 64, {"kind": "topk", "k": 6}
    if name == "ratio_bos_eos":
        lay = DG.make_decode_layer(B=3, Hq=64, Hkv=8, seq_lens=[2048, 1999, 40], seed=304, device=dev)
        return lay, 16, {"kind": "ratio", "ratio": 0.0625, "bos": 1, "eos": 1}
    if name == "chunks_tokens":
        lens = DG.workload3_chunks(2, 3000, seed_offset=3)
        lens[1] = DG.chunk_lengths(np.random.default_rng(6), 1234)
        lay = DG.make_decode_layer(B=2, Hq=32, Hkv=4, seq_lens=[3000, 1234], seed=305, device=dev,
                                   cap=3000, chunk_lens=lens, chunk_offset_std=0.5)
        return lay, 0, {"kind": "tokens", "budget": 1024}
    if name == "chunks_topk":
        # TSA with a chunk-count budget (top 64 / top 32 chunks)
        rng = np.random.default_rng(8)
        lens = [DG.chunk_lengths(rng, n) for n in (4000, 3900, 2500)]
        lay = DG.make_decode_layer(B=3, Hq=32, Hkv=4, seq_lens=[4000, 3900, 2500], seed=307, device=dev,
                                   cap=4000, chunk_lens=lens, chunk_offset_std=0.5)
        return lay, 0, {"kind": "topk", "k": 32}
    # few units with at least 16 decode splits each: the one-cluster-per-unit launch
    if name == "cluster_ps16":
        lay = DG.make_decode_layer(B=1, Hq=32, Hkv=4, seq_lens=[8000], seed=311, device=dev,
                                   key_scale="channel")
        return lay, 16, {"kind": "topk", "k": 256}
    if name == "cluster_two_rounds":
        # 32 decode splits per unit: each CTA of a cluster runs two
        lay = DG.make_decode_layer(B=2, Hq=32, Hkv=4, seq_lens=[8192, 6001], seed=312, device=dev, cap=8192)
        return lay, 16, {"kind": "topk", "k": 512}
    if name == "cluster_chunks_tokens":
        lens = DG.workload3_chunks(1, 12000, seed_offset=5)
        lay = DG.make_decode_layer(B=1, Hq=32, Hkv=4, seq_lens=[12000], seed=313, device=dev,
                                   chunk_lens=lens, chunk_offset_std=0.5)
        return lay, 0, {"kind": "tokens", "budget": 4096}
    if name == "cluster_ratio":
        lay = DG.make_decode_layer(B=1, Hq=64, Hkv=8, seq_lens=[32768], seed=314, device=dev)
        return lay, 16, {"kind": "ratio", "ratio": 0.25, "bos": 1, "eos": 1}
    if name == "cluster_ps64_g7":
        lay = DG.make_decode_layer(B=1, Hq=28, Hkv=4, seq_lens=[20001], seed=315, device=dev, cap=20032)
        return lay, 64, {"kind": "topk", "k": 64}
    if name == "many_units":
        rng = np.random.default_rng(7)
        lens = [int(x) for x in rng.integers(1, 2048, size=64)]
        lay = DG.make_decode_layer(B=64, Hq=16, Hkv=8, seq_lens=lens, seed=306, device=dev, cap=2048)
        return lay, 16, {"kind": "topk", "k": 16}
    raise KeyError(name)


CASES = ["ps16_topk", "ps16_new_page", "ps64_g7", "ratio_bos_eos", "chunks_tokens", "chunks_topk",
         "many_units", "cluster_ps16", "cluster_two_rounds", "cluster_chunks_tokens", "cluster_ratio",
         "cluster_ps64_g7"]


def _pages(lay, b, ps):
    N = int(lay.seq_len[b])
    return -(-N // ps) if ps else int(lay.n_chunks[b])


def _assert_same(s, c, lay, ps, where, exact=True):
    """Page sets and metadata bit-identical; outputs too unless `exact` is
    False (a token budget: the step splits the attention by the budget, the
    separate decode call by max_sel, so the split merge rounds differently)."""
    for key in ("sel_idx", "sel_count", "out", "lse"):
        a, b = torch.nan_to_num(s[key], nan=7.0), torch.nan_to_num(c[key], nan=7.0)
        if exact or key in ("sel_idx", "sel_count"):
            assert torch.equal(a, b), f"{where}: {key}"
        else:
            assert torch.equal(torch.isinf(a), torch.isinf(b)), f"{where}: {key}"
            fa, fb = torch.nan_to_num(a, posinf=0.0, neginf=0.0), torch.nan_to_num(b, posinf=0.0, neginf=0.0)
            assert float((fa - fb).abs().max()) < 1e-5, f"{where}: {key}"
    for b in range(lay.k.shape[0]):
        P = _pages(lay, b, ps)
        assert torch.equal(s["meta"][b, :, :P], c["meta"][b, :, :P]), f"{where}: meta of sequence {b}"


@pytest.mark.parametrize("rule", ["envelope", "centroid"])
@pytest.mark.parametrize("name", CASES)
def test_step_parity(cuda_dev, R, rule, name):
    lay, ps, bd = _case(cuda_dev, name)
    s = R.run_step(lay, page_size=ps, rule=rule, budget=bd, scale=SCALE, stale=True)
    assert s["status"] == 0
    st = R.check_layer(lay, s, page_size=ps, rule=rule, budget=bd, scale=SCALE)
    assert st["units"] == lay.k.shape[0] * lay.k.shape[1]
    assert st["max_out_err"] < 1e-4
    c = R.run_gpu(lay, page_size=ps, rule=rule, budget=bd, scale=SCALE)
    assert c["status"] == 0
    _assert_same(s, c, lay, ps, f"{name}/{rule}", exact=bd["kind"] != "tokens")


@pytest.mark.parametrize("rule", ["envelope", "centroid"])
@pytest.mark.parametrize("name", ["ps16_topk", "ps16_new_page", "ps64_g7", "ratio_bos_eos", "chunks_tokens",
                                  "many_units"])
def test_step_per_head_parity(cuda_dev, R, rule, name):
    """The per-query-head step: every (sequence, query head) against the
    oracle run on that head alone, and against the separate per-head calls
    (the same page sets bit for bit; outputs within 1e-5: the step decodes
    each KV head's union of page sets once with per-head masks, the separate
    call each head's own set)."""
    lay, ps, bd = _case(cuda_dev, name)
    s = R.run_step(lay, page_size=ps, rule=rule, budget=bd, scale=SCALE, stale=True, per_head=True)
    assert s["status"] == 0
    st = R.check_layer(lay, s, page_size=ps, rule=rule, budget=bd, scale=SCALE, per_head=True)
    assert st["units"] == lay.k.shape[0] * lay.q.shape[1]
    assert st["max_out_err"] < 1e-4
    c = R.run_gpu(lay, page_size=ps, rule=rule, budget=bd, scale=SCALE, per_head=True)
    assert c["status"] == 0
    _assert_same(s, c, lay, ps, f"{name}/{rule}/per-head", exact=False)


@pytest.mark.parametrize("rule", ["envelope", "centroid"])
@pytest.mark.parametrize("name", ["ps16_topk", "ps16_new_page", "ps64_g7", "chunks_topk", "chunks_tokens",
                                  "cluster_ps16", "cluster_chunks_tokens"])
def test_step_append(cuda_dev, R, rule, name):
    """The step that stores the newest token's key and value itself equals
    storing them first and running the step, bit for bit, and leaves the same
    cache behind.  Before the call the cache's newest rows hold large values
    that would change the metadata and the attention if they were read."""
    import dataclasses
    lay, ps, bd = _case(cuda_dev, name)
    ref = R.run_step(lay, page_size=ps, rule=rule, budget=bd, scale=SCALE, stale=True)
    assert ref["status"] == 0
    B = lay.k.shape[0]
    bi = torch.arange(B, device=cuda_dev)
    n = lay.seq_len.long() - 1
    k_new = lay.k[bi, :, n].contiguous()  # [B, Hkv, 128]
    v_new = lay.v[bi, :, n].contiguous()
    lay2 = dataclasses.replace(lay, k=lay.k.clone(), v=lay.v.clone())
    lay2.k[bi, :, n] = 1000.0
    lay2.v[bi, :, n] = -1000.0
    app = R.run_step(lay2, page_size=ps, rule=rule, budget=bd, scale=SCALE, stale=True,
                     append=(k_new, v_new), repeat=2)
    assert app["status"] == 0
    _assert_same(app, ref, lay, ps, f"append {name}/{rule}")
    for r in app["runs"][1:]:
        for key in ("sel_idx", "sel_count", "out", "lse"):
            assert torch.equal(r[key], app["runs"][0][key]), key
    assert torch.equal(lay2.k, lay.k) and torch.equal(lay2.v, lay.v)
    # bf16 output: the same fp32 results rounded to nearest even
    bf = R.run_step(lay2, page_size=ps, rule=rule, budget=bd, scale=SCALE, stale=True,
                    append=(k_new, v_new), out_dtype=torch.bfloat16)
    assert bf["status"] == 0 and bf["out"].dtype == torch.bfloat16
    assert torch.equal(bf["out"], ref["out"].to(torch.bfloat16)), f"bf16 output {name}/{rule}"
    assert torch.equal(bf["lse"], ref["lse"]) and torch.equal(bf["sel_idx"], ref["sel_idx"])


def test_step_output_to_pinned_host_memory(cuda_dev, R):
    """The step may write its result straight into pinned host memory (which
    the device reaches under unified addressing): the same bits as a device
    output, with the device status clear."""
    import block_sparse_kv_page_b200 as sa
    lay, ps, bd = _case(cuda_dev, "ps16_topk")
    ref = R.run_step(lay, page_size=ps, rule="envelope", budget=bd, scale=SCALE, stale=True)
    assert ref["status"] == 0
    B, Hkv = lay.k.shape[:2]
    Hq = lay.q.shape[1]
    sel = torch.full((B, Hkv, ref["max_sel"]), -7, dtype=torch.int32, device=cuda_dev)
    cnt = torch.full((B, Hkv), -7, dtype=torch.int32, device=cuda_dev)
    out_h = torch.full((B, Hq, 128), float("nan"), dtype=torch.float32).pin_memory()
    sa.sparse_attn_decode_step(ref["kv"], ref["meta"], "envelope", lay.q, R.budget_struct(bd), ref["max_sel"],
                               SCALE, sel, cnt, out_h, None, ref["ws"])
    torch.cuda.synchronize()
    assert sa.sparse_attn_get_device_status(ref["ws"]) == 0
    assert torch.equal(out_h, ref["out"])
    assert torch.equal(sel.cpu(), ref["sel_idx"]) and torch.equal(cnt.cpu(), ref["sel_count"])


def test_step_repeat_and_interleave(cuda_dev, R):
    """Calls in a row on one workspace: the step leaves its flags, counters
    and queue cleared, also around the other calls."""
    import block_sparse_kv_page_b200 as sa
    lay, ps, bd = _case(cuda_dev, "ps16_topk")
    s = R.run_step(lay, page_size=ps, rule="envelope", budget=bd, scale=SCALE, repeat=3)
    assert s["status"] == 0
    for r in s["runs"][1:]:
        for key in ("sel_idx", "sel_count", "out", "lse"):
            assert torch.equal(r[key], s["runs"][0][key]), key
    # the same workspace through select + decode, then the step again
    c = R.run_gpu(lay, page_size=ps, rule="envelope", budget=bd, scale=SCALE, ws=s["ws"])
    assert c["status"] == 0
    again = R.run_step(lay, page_size=ps, rule="envelope", budget=bd, scale=SCALE, ws=s["ws"])
    assert again["status"] == 0
    _assert_same(again, c, lay, ps, "after interleave")
    assert sa.sparse_attn_get_device_status(s["ws"]) == 0


def test_step_refresh_matches_build(cuda_dev, R):
    """The metadata the step leaves behind equals a full build of the grown
    cache (every page, both rules, pages and chunks)."""
    import block_sparse_kv_page_b200 as sa
    for name in ("ps16_new_page", "ps64_g7", "chunks_tokens"):
        lay, ps, bd = _case(cuda_dev, name)
        for rule in ("envelope", "centroid"):
            s = R.run_step(lay, page_size=ps, rule=rule, budget=bd, scale=SCALE)
            full = s["kv"].meta_buffer().fill_(0x5A)
            sa.sparse_attn_build_meta(s["kv"], rule, 0, full)
            torch.cuda.synchronize()
            for b in range(lay.k.shape[0]):
                P = _pages(lay, b, ps)
                assert torch.equal(s["meta"][b, :, :P], full[b, :, :P]), f"{name}/{rule}/b{b}"


def test_step_rejects_bad_arguments(cuda_dev, R):
    import block_sparse_kv_page_b200 as sa
    lay, ps, bd = _case(cuda_dev, "ps16_topk")
    kv = sa.KvCache(lay.k, lay.v, lay.seq_len, page_size=16, max_pages=64)
    meta = kv.meta_buffer()
    ws = sa.make_workspace(kv, 32, 2, 24)
    sel = torch.empty((2, 4, 24), dtype=torch.int32, device=cuda_dev)
    cnt = torch.empty((2, 4), dtype=torch.int32, device=cuda_dev)
    out = torch.empty((2, 32, 128), dtype=torch.float32, device=cuda_dev)
    with pytest.raises(sa.SparseAttnError) as e:  # budget above max_sel
        sa.sparse_attn_decode_step(kv, meta, "envelope", lay.q, sa.budget_topk(25), 24, SCALE,
                                   sel, cnt, out, None, ws)
    assert e.value.status == sa.SA_ERR_INVALID
    with pytest.raises(sa.SparseAttnError) as e:  # workspace too small
        sa.sparse_attn_decode_step(kv, meta, "envelope", lay.q, sa.budget_topk(24), 24, SCALE,
                                   sel, cnt, out, None, ws[:1024])
    assert e.value.status == sa.SA_ERR_WORKSPACE
    with pytest.raises(sa.SparseAttnError) as e:  # non-finite scale
        sa.sparse_attn_decode_step(kv, meta, "envelope", lay.q, sa.budget_topk(24), 24, float("nan"),
                                   sel, cnt, out, None, ws)
    assert e.value.status == sa.SA_ERR_INVALID


def test_step_sequence_in_cuda_graph(cuda_dev, R):
    """Per-layer steps launched back to back (programmatic dependent launches
    on one stream) and captured in a CUDA graph give bit-identical results to
    the same calls with a synchronisation after each; the graph replays
    deterministically and leaves the workspace clean."""
    import block_sparse_kv_page_b200 as sa
    layers = [DG.make_decode_layer(B=2, Hq=32, Hkv=4, seq_lens=[1500, 900], seed=900 + l, device=cuda_dev,
                                   cap=1504, key_scale="channel") for l in range(4)]
    bd = sa.budget_topk(24)
    kvs = [sa.KvCache(lay.k, lay.v, lay.seq_len, page_size=16, max_pages=94) for lay in layers]
    metas = []
    for kv in kvs:
        m = kv.meta_buffer()
        sa.sparse_attn_build_meta(kv, "envelope", 0, m)
        metas.append(m)
    ws = sa.make_workspace(kvs[0], 32, 2, 24)
    outs = [dict(sel=torch.zeros((2, 4, 24), dtype=torch.int32, device=cuda_dev),
                 cnt=torch.zeros((2, 4), dtype=torch.int32, device=cuda_dev),
                 out=torch.zeros((2, 32, 128), dtype=torch.float32, device=cuda_dev),
                 lse=torch.zeros((2, 32), dtype=torch.float32, device=cuda_dev)) for _ in layers]

    def run_all(sync_each):
        for l, lay in enumerate(layers):
            o = outs[l]
            sa.sparse_attn_decode_step(kvs[l], metas[l], "envelope", lay.q, bd, 24, SCALE, o["sel"], o["cnt"],
                                       o["out"], o["lse"], ws)
            if sync_each:
                torch.cuda.synchronize()

    run_all(True)
    ref = [{k: v.clone() for k, v in o.items()} for o in outs]
    for o in outs:
        for v in o.values():
            v.zero_()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        run_all(False)  # warm outside capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run_all(False)
    for _ in range(3):
        for o in outs:
            for v in o.values():
                v.zero_()
        g.replay()
        torch.cuda.synchronize()
        for l in range(len(layers)):
            for key in ("sel", "cnt", "out", "lse"):
                assert torch.equal(outs[l][key], ref[l][key]), f"layer {l}: {key}"
    assert sa.sparse_attn_get_device_status(ws) == 0
    del g
