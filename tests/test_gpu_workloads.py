"""Parity at the full sizes of the decode workloads, in the launch shape the
benchmark uses (independent layers stacked along the batch axis, one launch
per stage), checked against the oracle on sampled (layer, sequence, KV head)
units.

* 48-layer Qwen3-VL-30B-A3B-shaped decode at 29,504 tokens: envelope and
  centroid, budgets 4096 and 8192 tokens (top-256 / top-512 pages).
* TSA variable chunks at 29,504 tokens, batch 4: greedy token budgets 4096,
  8192, 16384; and 16,384 tokens at budget 16,384 (= dense attention).
* 64-layer Qwen3-32B-shaped ratio budgets at 32,768 tokens, batch 8, 64:8:
  all seven ratios, centroid with bos=eos=1 and envelope with bos=0, eos=1.
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


def _stack(layers):
    """Stack independent layers along the batch axis (the benchmark's layout)."""
    st = DG.DecodeLayer(
        q=torch.cat([l.q for l in layers]), k=torch.cat([l.k for l in layers]),
        v=torch.cat([l.v for l in layers]), seq_len=torch.cat([l.seq_len for l in layers]))
    if layers[0].chunk_off is not None:
        w = max(l.chunk_off.shape[1] for l in layers)
        offs = []
        for l in layers:
            o = l.chunk_off
            if o.shape[1] < w:
                pad = o[:, -1:].expand(-1, w - o.shape[1])
                o = torch.cat([o, pad], dim=1)
            offs.append(o)
        st.chunk_off = torch.cat(offs).contiguous()
        st.n_chunks = torch.cat([l.n_chunks for l in layers])
    return st


@pytest.fixture(scope="module")
def qwen3vl_stack(cuda_dev):
    layers = [DG.workload2_layer(l, cuda_dev) for l in range(48)]
    st = _stack(layers)
    del layers
    return st


@pytest.mark.parametrize("rule", ["envelope", "centroid"])
@pytest.mark.parametrize("budget", [4096, 8192])
def test_qwen3vl_48_layers_full(cuda_dev, R, qwen3vl_stack, rule, budget):
    lay = qwen3vl_stack
    bd = {"kind": "topk", "k": budget // 16}
    g = R.run_gpu(lay, page_size=16, rule=rule, budget=bd, scale=SCALE)
    assert g["status"] == 0
    assert (g["sel_count"] == budget // 16).all()
    units = [(b, h) for b in (0, 17, 31, 47) for h in range(4)]
    st = R.check_layer(lay, g, page_size=16, rule=rule, budget=bd, scale=SCALE, units=units)
    assert st["max_out_err"] < 1e-4
    print(f"\n{rule}@{budget}: {st}")


@pytest.mark.parametrize("budget", [4096, 8192, 16384])
def test_tsa_chunks_full(cuda_dev, R, budget):
    layers = [DG.workload3_layer(l, cuda_dev) for l in (0, 47)]
    lay = _stack(layers)
    bd = {"kind": "tokens", "budget": budget}
    g = R.run_gpu(lay, page_size=0, rule="envelope", budget=bd, scale=SCALE)
    assert g["status"] == 0
    st = R.check_layer(lay, g, page_size=0, rule="envelope", budget=bd, scale=SCALE)
    assert st["units"] == 8 * 4
    print(f"\ntokens@{budget}: {st}")


@pytest.mark.parametrize("rule,k", [("envelope", 64), ("centroid", 64), ("centroid", 32)])
def test_tsa_chunk_count_full(cuda_dev, R, rule, k):
    """TSA with a chunk-count budget (top 64 / top 32 chunks), min/max and
    centroid scoring, on the full 29,504-token batch-4 workload."""
    layers = [DG.workload3_layer(l, cuda_dev) for l in (0, 47)]
    lay = _stack(layers)
    bd = {"kind": "topk", "k": k}
    g = R.run_gpu(lay, page_size=0, rule=rule, budget=bd, scale=SCALE)
    assert g["status"] == 0
    assert (g["sel_count"] == k).all()
    st = R.check_layer(lay, g, page_size=0, rule=rule, budget=bd, scale=SCALE)
    assert st["units"] == 8 * 4
    assert st["max_out_err"] < 1e-4
    print(f"\n{rule} top-{k} chunks: {st}")


def test_tsa_centroid_tokens_full(cuda_dev, R):
    layers = [DG.workload3_layer(l, cuda_dev) for l in (3,)]
    lay = _stack(layers)
    bd = {"kind": "tokens", "budget": 4096}
    g = R.run_gpu(lay, page_size=0, rule="centroid", budget=bd, scale=SCALE)
    assert g["status"] == 0
    st = R.check_layer(lay, g, page_size=0, rule="centroid", budget=bd, scale=SCALE)
    assert st["units"] == 4 * 4


def test_tsa_full_budget_equals_dense(cuda_dev, R):
    lay = DG.workload3_layer(5, cuda_dev, N=16384)
    bd = {"kind": "tokens", "budget": 16384}
    g = R.run_gpu(lay, page_size=0, rule="envelope", budget=bd, scale=SCALE)
    for b in range(4):
        for h in range(4):
            assert int(g["sel_count"][b, h]) == int(lay.n_chunks[b])
    units = [(b, h) for b in range(4) for h in range(4)]
    R.check_layer(lay, g, page_size=0, rule="envelope", budget=bd, scale=SCALE, units=units)
    Q = R.to_np(lay.q[0, 0:8])
    o, _ = O.attend(Q, R.to_np(lay.k[0, 0]), R.to_np(lay.v[0, 0]), np.arange(16384), SCALE)
    assert np.abs(g["out"][0, 0:8].numpy() - o).max() < 1e-4


@pytest.mark.parametrize("layer", [0, 31, 63])
def test_qwen3_32b_ratio_full(cuda_dev, R, layer):
    lay = DG.workload4_layer(layer, cuda_dev)
    ratios = DG.WORKLOAD4_RATIOS if layer == 0 else (0.5, 0.015625)
    rng = np.random.default_rng(layer)
    for rule, bos, eos in (("centroid", 1, 1), ("envelope", 0, 1)):
        for ratio in ratios:
            bd = {"kind": "ratio", "ratio": ratio, "bos": bos, "eos": eos}
            g = R.run_gpu(lay, page_size=16, rule=rule, budget=bd, scale=SCALE)
            assert g["status"] == 0
            K = O.ratio_budget_pages(2048, ratio, 1, bos, eos)
            assert (g["sel_count"] == K).all()
            picks = rng.choice(64, size=6, replace=False)
            units = [(int(u) // 8, int(u) % 8) for u in picks]
            R.check_layer(lay, g, page_size=16, rule=rule, budget=bd, scale=SCALE, units=units)
