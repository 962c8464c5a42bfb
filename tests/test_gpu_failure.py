"""Failure detection on the GPU without a GPU fault: the decode step's only
inter-CTA wait (a decode item waiting for its unit's selection flag) is made
to run out by withholding one unit's flag (sparse_attn_decode_step_wait_test,
a short poll limit).  The launch must end on its own, report SA_ERR_TIMEOUT
through the workspace status word, and leave the workspace clean: the next
regular step on the same workspace is oracle-correct with status OK.  Only
the unit-flag wait is exercised this way -- never an mbarrier wait with TMA
copies in flight."""
import math
import time

import pytest
import torch

import datagen as DG

pytestmark = pytest.mark.gpu

SCALE = 1.0 / math.sqrt(128)


@pytest.mark.parametrize("held_unit,spin", [(5, 1024), (0, 64)])
def test_step_flag_wait_times_out_then_next_step_is_clean(cuda_dev, held_unit, spin):
    import block_sparse_kv_page_b200 as sa
    import gpu_runner as R
    lay = DG.make_decode_layer(B=2, Hq=32, Hkv=4, seq_lens=[3000, 2500], cap=3008, seed=901,
                               device=cuda_dev, key_scale="channel")
    bd = {"kind": "topk", "k": 48}
    kv = sa.KvCache(lay.k, lay.v, lay.seq_len, page_size=16, max_pages=188)
    meta = kv.meta_buffer()
    sa.sparse_attn_build_meta(kv, "envelope", 0, meta)
    ws = sa.make_workspace(kv, 32, 2, 48)
    sel = torch.zeros((2, 4, 48), dtype=torch.int32, device=cuda_dev)
    cnt = torch.zeros((2, 4), dtype=torch.int32, device=cuda_dev)
    out = torch.zeros((2, 32, 128), dtype=torch.float32, device=cuda_dev)
    lse = torch.zeros((2, 32), dtype=torch.float32, device=cuda_dev)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    sa.sparse_attn_decode_step_wait_test(kv, meta, "envelope", lay.q, sa.budget_topk(48), 48, SCALE, sel, cnt,
                                         out, lse, held_unit, spin, ws)
    torch.cuda.synchronize()  # the launch ended by itself
    dt = time.perf_counter() - t0
    assert dt < 5.0, f"the launch took {dt:.2f} s"
    assert sa.sparse_attn_get_device_status(ws) == sa.SA_ERR_TIMEOUT
    # reading the status cleared it; the same workspace serves the next step
    g = R.run_step(lay, page_size=16, rule="envelope", budget=bd, scale=SCALE, ws=ws)
    assert g["status"] == 0
    st = R.check_layer(lay, g, page_size=16, rule="envelope", budget=bd, scale=SCALE)
    assert st["units"] == 8
    # and a re-initialised workspace too
    sa.sparse_attn_workspace_init(ws)
    g2 = R.run_step(lay, page_size=16, rule="envelope", budget=bd, scale=SCALE, ws=ws)
    assert g2["status"] == 0
    assert torch.equal(g2["out"], g["out"]) and torch.equal(g2["sel_idx"], g["sel_idx"])
