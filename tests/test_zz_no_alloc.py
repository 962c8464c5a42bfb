"""The workspace-free decode entry point, checked against the regular one.

sparse_attn_decode_static serves callers that cannot allocate device memory
where they run the attention (a plugin handed only its input/output pointers
at enqueue time, or a decode loop that must not pay cudaMalloc's device-wide
synchronisation).  Its scratch is an array built into the library, so two
calls in a row must both give the same result as sparse_attn_decode with a
caller-provided workspace, within the output tolerance the parity tests use.

This file is collected last on purpose; it passes alone in a fresh process
(the first call looks up the array's address) and after the other tests.
"""
import ctypes as C
import math

import pytest
import torch

import datagen as DG

pytestmark = pytest.mark.gpu

OUT_TOL = 2e-3


def _problem(dev):
    import block_sparse_kv_page_b200 as sa
    lay = DG.make_decode_layer(B=2, Hq=32, Hkv=4, seq_lens=[3000, 2222], cap=3008, seed=4242,
                               device=dev, key_scale="channel")
    kv = sa.KvCache(lay.k, lay.v, lay.seq_len, page_size=16, max_pages=188)
    k = 64
    meta = kv.meta_buffer()
    ws = sa.make_workspace(kv, 32, 2, k)
    sel = torch.empty((2, 4, k), dtype=torch.int32, device=dev)
    cnt = torch.empty((2, 4), dtype=torch.int32, device=dev)
    sa.sparse_attn_build_meta(kv, "envelope", 0, meta)
    sa.sparse_attn_select(kv, meta, "envelope", lay.q, sa.budget_topk(k), k, sel, cnt, None, ws)
    return sa, lay, kv, ws, sel, cnt, k


def test_static_scratch_matches_workspace_decode(cuda_dev):
    sa, lay, kv, ws, sel, cnt, k = _problem(cuda_dev)
    scale = 1.0 / math.sqrt(128)
    ref = torch.empty((2, 32, 128), dtype=torch.float32, device=cuda_dev)
    ref_lse = torch.empty((2, 32), dtype=torch.float32, device=cuda_dev)
    sa.sparse_attn_decode(kv, lay.q, 2, 0, 1, scale, sel, cnt, k, ref, ref_lse, ws)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_dev)
    for call in range(2):
        out = torch.full_like(ref, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        sa.sparse_attn_decode_static(kv, lay.q, 2, 0, 1, scale, sel, cnt, k, out, lse, status)
        torch.cuda.synchronize()
        assert torch.isfinite(out).all(), f"call {call}: non-finite output"
        err = (out - ref).abs().max().item()
        assert err <= OUT_TOL, f"call {call}: max-abs difference {err}"
        assert (lse - ref_lse).abs().max().item() <= 1e-3, f"call {call}: lse differs"
    assert int(status.item()) == 0


def test_static_scratch_rejects_calls_beyond_its_size(cuda_dev):
    """More than 4096 (row, KV head) units do not fit the built-in scratch:
    the call is refused on the host with SA_ERR_WORKSPACE, nothing launched.
    (Real, correctly sized buffers are passed all the same.)"""
    import block_sparse_kv_page_b200 as sa
    B = 1025
    k = torch.zeros((B, 4, 16, 128), dtype=torch.bfloat16, device=cuda_dev)
    v = torch.zeros_like(k)
    sl = torch.full((B,), 16, dtype=torch.int32, device=cuda_dev)
    kv = sa.KvCache(k, v, sl, page_size=16, max_pages=1)
    q = torch.zeros((B, 32, 128), dtype=torch.bfloat16, device=cuda_dev)
    idx = torch.zeros((B, 4, 1), dtype=torch.int32, device=cuda_dev)
    cnt = torch.ones((B, 4), dtype=torch.int32, device=cuda_dev)
    out = torch.zeros((B, 32, 128), dtype=torch.float32, device=cuda_dev)
    r = sa.lib.sparse_attn_decode_static(C.byref(kv.desc), q.data_ptr(), 32, B, 0, 1, 0.088,
                                         idx.data_ptr(), cnt.data_ptr(), 1, out.data_ptr(), None,
                                         None, torch.cuda.current_stream().cuda_stream)
    assert r == sa.SA_ERR_WORKSPACE
