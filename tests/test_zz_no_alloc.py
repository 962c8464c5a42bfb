"""The workspace-free decode entry point, checked against the regular one.

sparse_attn_decode_static serves callers that cannot allocate device memory
where they run the attention (a plugin handed only its input/output pointers
at enqueue time, or a decode loop that must not pay cudaMalloc's device-wide
synchronisation).  Its scratch is an array built into the library.  It runs
the same kernel with the same work split as sparse_attn_decode, so two calls
in a row must both reproduce sparse_attn_decode's output bit for bit, and
the calls must leave the device's free memory unchanged.

This file is collected last on purpose; it passes alone in a fresh process
(the first call looks up the array's address) and after the other tests.
"""
import ctypes as C
import math

import pytest
import torch

import datagen as DG

pytestmark = pytest.mark.gpu


def _problem(dev, B, seq_lens, k, seed):
    import block_sparse_kv_page_b200 as sa
    cap = max(seq_lens)
    lay = DG.make_decode_layer(B=B, Hq=32, Hkv=4, seq_lens=seq_lens, cap=cap, seed=seed, device=dev,
                               key_scale="channel")
    P = -(-cap // 16)
    kv = sa.KvCache(lay.k, lay.v, lay.seq_len, page_size=16, max_pages=P)
    meta = kv.meta_buffer()
    ws = sa.make_workspace(kv, 32, B, k)
    sel = torch.empty((B, 4, k), dtype=torch.int32, device=dev)
    cnt = torch.empty((B, 4), dtype=torch.int32, device=dev)
    sa.sparse_attn_build_meta(kv, "envelope", 0, meta)
    sa.sparse_attn_select(kv, meta, "envelope", lay.q, sa.budget_topk(k), k, sel, cnt, None, ws)
    return sa, lay, kv, ws, sel, cnt


@pytest.mark.parametrize("B,seq_lens,k", [(2, [3000, 2222], 64), (4, [8192, 5000, 7777, 16], 256)])
def test_static_scratch_matches_workspace_decode(cuda_dev, B, seq_lens, k):
    sa, lay, kv, ws, sel, cnt = _problem(cuda_dev, B, seq_lens, k, seed=4242 + B)
    # the work is split, so the split partials in the built-in array are used:
    # at most 2 x SMs units' worth of items makes every unit take >= 2 splits
    # when its page budget allows (>= 32 pages, i.e. two 16-tile items)
    sms = torch.cuda.get_device_properties(cuda_dev).multi_processor_count
    units = B * 4
    assert (2 * sms + units - 1) // units >= 2 and (k + 15) // 16 >= 2
    scale = 1.0 / math.sqrt(128)
    ref = torch.empty((B, 32, 128), dtype=torch.float32, device=cuda_dev)
    ref_lse = torch.empty((B, 32), dtype=torch.float32, device=cuda_dev)
    sa.sparse_attn_decode(kv, lay.q, B, 0, 1, scale, sel, cnt, k, ref, ref_lse, ws)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_dev)
    outs = [torch.full_like(ref, float("nan")) for _ in range(3)]
    lses = [torch.full_like(ref_lse, float("nan")) for _ in range(3)]
    # first call: on a fresh process it looks up the array's address
    sa.sparse_attn_decode_static(kv, lay.q, B, 0, 1, scale, sel, cnt, k, outs[0], lses[0], status)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info(cuda_dev)[0]
    for call in (1, 2):  # two calls in a row
        sa.sparse_attn_decode_static(kv, lay.q, B, 0, 1, scale, sel, cnt, k, outs[call], lses[call], status)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info(cuda_dev)[0] == free0, "the calls changed the device's free memory"
    for call in range(3):
        assert torch.equal(outs[call], ref), f"call {call}: output differs from sparse_attn_decode"
        assert torch.equal(lses[call], ref_lse), f"call {call}: lse differs from sparse_attn_decode"
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
