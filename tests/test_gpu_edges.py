"""GPU parity at the edges of the selection's two code paths and of the head
layouts, against the float64 oracle through the C ABI.

* More than 2048 pages per (sequence, KV head): the selection keeps its keys
  in shared memory instead of registers (2049 pages: the first size past the
  register path; 2500 pages; 2300 variable chunks under a token budget).
* Exactly 2048 pages: the largest unit the register path takes.
* A single KV head (G = 8) and G = 1 (every query head its own KV head).
* The largest sizes the calls take: 16,384 pages in one unit, 32,768 units in
  one decode step.
Each case runs the separate calls and the one-launch step (which must agree
with them bit for bit).
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


def _check_both(R, lay, ps, rule, bd):
    g = R.run_gpu(lay, page_size=ps, rule=rule, budget=bd, scale=SCALE)
    assert g["status"] == 0
    st = R.check_layer(lay, g, page_size=ps, rule=rule, budget=bd, scale=SCALE)
    assert st["max_out_err"] < 1e-4
    s = R.run_step(lay, page_size=ps, rule=rule, budget=bd, scale=SCALE, stale=True)
    assert s["status"] == 0
    for key in ("sel_idx", "sel_count"):
        assert (s[key] == g[key]).all(), key
    if bd["kind"] != "tokens":  # a token budget splits the step's attention differently (rounding)
        assert (s["out"] == g["out"]).all()
    else:
        assert float((s["out"] - g["out"]).abs().max()) < 1e-5
    return g


@pytest.mark.parametrize("rule", ["envelope", "centroid"])
@pytest.mark.parametrize("N,bd", [
    (32769, {"kind": "topk", "k": 300}),                                    # 2049 pages
    (40000, {"kind": "topk", "k": 257}),                                    # 2500 pages
    (40000, {"kind": "ratio", "ratio": 0.0625, "bos": 1, "eos": 1}),
    (32768, {"kind": "topk", "k": 512}),                                    # 2048 pages: register path
])
def test_many_pages_single_kv_head(cuda_dev, R, rule, N, bd):
    lay = DG.make_decode_layer(B=1, Hq=8, Hkv=1, seq_lens=[N], seed=701 + N % 97, device=cuda_dev,
                               key_scale="channel")
    _check_both(R, lay, 16, rule, bd)


@pytest.mark.parametrize("rule", ["envelope", "centroid"])
def test_many_chunks_token_budget(cuda_dev, R, rule):
    rng = np.random.default_rng(17)
    lens = [DG.chunk_lengths(rng, 40000, lo=16, hi=19), DG.chunk_lengths(rng, 9000)]
    assert len(lens[0]) > 2048
    lay = DG.make_decode_layer(B=2, Hq=16, Hkv=2, seq_lens=[40000, 9000], seed=711, device=cuda_dev,
                               cap=40000, chunk_lens=lens, chunk_offset_std=0.5)
    _check_both(R, lay, 0, rule, {"kind": "tokens", "budget": 5000})


@pytest.mark.parametrize("rule", ["envelope", "centroid"])
def test_group_of_one(cuda_dev, R, rule):
    lay = DG.make_decode_layer(B=2, Hq=4, Hkv=4, seq_lens=[3000, 1200], seed=721, device=cuda_dev)
    _check_both(R, lay, 16, rule, {"kind": "topk", "k": 33})


@pytest.mark.parametrize("rule", ["envelope", "centroid"])
def test_max_pages_per_unit(cuda_dev, R, rule):
    """16,384 pages in one (sequence, KV head), the largest page axis the
    selection takes (its keys fill 128 KiB of shared memory in the step)."""
    N = 16384 * 16
    lay = DG.make_decode_layer(B=1, Hq=8, Hkv=1, seq_lens=[N], seed=731, device=cuda_dev)
    _check_both(R, lay, 16, rule, {"kind": "topk", "k": 1000})


def test_max_units_in_one_step(cuda_dev, R):
    """32,768 (sequence, KV head) units in one decode step (its limit: unit
    flags and split counters share the workspace header), short ragged
    caches; a seeded sample of units is checked against the oracle and all of
    them against the separate calls."""
    rng = np.random.default_rng(741)
    B, Hkv = 8192, 4
    lens = [int(x) for x in rng.integers(1, 200, size=B)]
    lay = DG.make_decode_layer(B=B, Hq=16, Hkv=Hkv, seq_lens=lens, seed=741, device=cuda_dev, cap=200)
    bd = {"kind": "topk", "k": 4}
    s = R.run_step(lay, page_size=16, rule="envelope", budget=bd, scale=SCALE, stale=True)
    assert s["status"] == 0
    picks = rng.choice(B * Hkv, size=48, replace=False)
    units = [(int(u) // Hkv, int(u) % Hkv) for u in picks]
    st = R.check_layer(lay, s, page_size=16, rule="envelope", budget=bd, scale=SCALE, units=units)
    assert st["max_out_err"] < 1e-4
    g = R.run_gpu(lay, page_size=16, rule="envelope", budget=bd, scale=SCALE)
    assert g["status"] == 0
    for key in ("sel_idx", "sel_count", "out", "lse"):
        a_, b_ = torch.nan_to_num(s[key], nan=7.0), torch.nan_to_num(g[key], nan=7.0)
        assert torch.equal(a_, b_), key
