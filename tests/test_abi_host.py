"""C-ABI library: loads, exports every function include/sparse_attn.h declares,
and rejects bad arguments on the host before any launch (CPU only: the
pointers below are never dereferenced because validation fails first)."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sparse_attn.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sparse_attn_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def abi():
    from block_sparse_kv_page_b200 import _abi
    return _abi


@pytest.fixture(scope="module")
def lib(abi):
    return abi.load()


def test_header_declares_the_four_calls():
    names = _declared()
    for n in ("sparse_attn_build_meta", "sparse_attn_select", "sparse_attn_decode", "sparse_attn_route"):
        assert n in names


def test_every_declared_symbol_is_exported(lib, abi):
    names = _declared()
    assert names, "no declarations parsed"
    for n in names:
        assert hasattr(lib, n), f"{n} not exported"
    assert sorted(abi.PROTOTYPES) == names, "binding prototypes differ from the header"


def test_package_import_uses_in_tree_library():
    import block_sparse_kv_page_b200 as sa
    assert os.path.dirname(sa._abi.LIB_PATH) == os.path.join(ROOT, "block_sparse_kv_page_b200")
    assert os.path.exists(sa._abi.LIB_PATH)


def test_status_strings(lib):
    for code in range(7):
        s = lib.sparse_attn_status_string(code)
        assert s and s != b"unknown status"
    assert lib.sparse_attn_status_string(99) == b"unknown status"


def _desc(abi, **kw):
    d = dict(batch=1, n_kv_heads=4, head_dim=128, page_size=16, cap_tokens=1024,
             k=0x10000, v=0x20000, seq_len=0x30000, chunk_off=None, n_chunks=None, max_pages=64)
    d.update(kw)
    return abi.sa_kv_desc(d["batch"], d["n_kv_heads"], d["head_dim"], d["page_size"], d["cap_tokens"],
                          d["k"], d["v"], d["seq_len"], d["chunk_off"], d["n_chunks"], d["max_pages"])


def _select(lib, abi, desc, *, hq=32, budget=None, max_sel=16, ws=0x100000, ws_bytes=1 << 30,
            meta=0x40000, q=0x50000, sel=0x60000, cnt=0x70000):
    if budget is None:
        budget = abi.sa_budget(abi.SA_BUDGET_TOPK, 8, 0.0, 0, 0, 0, 0)
    return lib.sparse_attn_select(C.byref(desc) if desc is not None else None, meta, 0, q, hq,
                                  C.byref(budget), max_sel, sel, cnt, None, ws, ws_bytes, None)


def test_select_validation(lib, abi):
    ok = _desc(abi)
    assert _select(lib, abi, None) == abi.SA_ERR_INVALID
    assert _select(lib, abi, _desc(abi, head_dim=64)) == abi.SA_ERR_UNSUPPORTED
    assert _select(lib, abi, _desc(abi, page_size=8)) == abi.SA_ERR_UNSUPPORTED
    assert _select(lib, abi, _desc(abi, k=0x10001)) == abi.SA_ERR_INVALID      # misaligned K
    assert _select(lib, abi, _desc(abi, batch=0)) == abi.SA_ERR_INVALID
    assert _select(lib, abi, ok, hq=30) == abi.SA_ERR_INVALID                  # Hq % Hkv
    assert _select(lib, abi, ok, hq=64) == abi.SA_ERR_UNSUPPORTED              # G = 16
    assert _select(lib, abi, ok, q=0x50002) == abi.SA_ERR_INVALID              # misaligned q
    assert _select(lib, abi, ok, meta=0) == abi.SA_ERR_INVALID
    assert _select(lib, abi, ok, max_sel=4) == abi.SA_ERR_INVALID              # top_k > max_sel
    assert _select(lib, abi, ok, ws=0) == abi.SA_ERR_WORKSPACE
    assert _select(lib, abi, ok, ws=0x100010) == abi.SA_ERR_WORKSPACE          # not 256-aligned
    assert _select(lib, abi, ok, ws_bytes=1024) == abi.SA_ERR_WORKSPACE
    bad_ratio = abi.sa_budget(abi.SA_BUDGET_RATIO, 0, 1.5, 1, 1, 1, 0)
    assert _select(lib, abi, ok, budget=bad_ratio) == abi.SA_ERR_INVALID
    big_ratio = abi.sa_budget(abi.SA_BUDGET_RATIO, 0, 0.5, 1, 1, 1, 0)       # K = 32 > max_sel
    assert _select(lib, abi, ok, budget=big_ratio) == abi.SA_ERR_INVALID
    tokens = abi.sa_budget(abi.SA_BUDGET_TOKENS, 0, 0.0, 0, 0, 0, 4096)
    assert _select(lib, abi, ok, budget=tokens) == abi.SA_ERR_UNSUPPORTED      # fixed pages
    chunked = _desc(abi, page_size=0)                                          # no chunk table
    assert _select(lib, abi, chunked, budget=tokens) == abi.SA_ERR_INVALID


def test_decode_validation(lib, abi):
    ok = _desc(abi)

    def call(desc=ok, hq=32, rows=1, tile=1, scale=0.088, out=0x80000, ws_bytes=1 << 30):
        return lib.sparse_attn_decode(C.byref(desc), 0x50000, hq, rows, 0, tile, scale, 0x60000,
                                      0x70000, 16, out, None, 0x100000, ws_bytes, None)
    assert call(rows=2) == abi.SA_ERR_INVALID          # decode rows must equal batch
    assert call(out=0x80004) == abi.SA_ERR_INVALID     # out not 16-byte aligned
    assert call(scale=float("nan")) == abi.SA_ERR_INVALID
    assert call(tile=0) == abi.SA_ERR_INVALID
    assert call(ws_bytes=256) == abi.SA_ERR_WORKSPACE
    assert call(desc=_desc(abi, head_dim=256)) == abi.SA_ERR_UNSUPPORTED


def test_decode_step_validation(lib, abi):
    ok = _desc(abi)
    topk = abi.sa_budget(abi.SA_BUDGET_TOPK, 8, 0.0, 0, 0, 0, 0)

    def call(desc=ok, hq=32, budget=topk, max_sel=16, scale=0.088, meta=0x40000, out=0x80000,
             ws=0x100000, ws_bytes=1 << 30):
        return lib.sparse_attn_decode_step(C.byref(desc), meta, 0, 0x50000, hq, C.byref(budget),
                                           max_sel, scale, 0x60000, 0x70000, out, None, ws,
                                           ws_bytes, None)
    assert call(meta=0) == abi.SA_ERR_INVALID
    assert call(meta=0x40008) == abi.SA_ERR_INVALID       # metadata not 16-byte aligned
    assert call(max_sel=4) == abi.SA_ERR_INVALID          # top_k > max_sel
    assert call(out=0x80004) == abi.SA_ERR_INVALID
    assert call(scale=float("inf")) == abi.SA_ERR_INVALID
    assert call(hq=64) == abi.SA_ERR_UNSUPPORTED          # G = 16
    assert call(ws_bytes=4096) == abi.SA_ERR_WORKSPACE
    assert call(ws=0x100010) == abi.SA_ERR_WORKSPACE
    assert call(desc=_desc(abi, batch=8193)) == abi.SA_ERR_UNSUPPORTED  # 2 x units > 65536
    tokens = abi.sa_budget(abi.SA_BUDGET_TOKENS, 0, 0.0, 0, 0, 0, 512)
    assert call(budget=tokens) == abi.SA_ERR_UNSUPPORTED  # token budgets need chunks


def test_decode_step_per_head_validation(lib, abi):
    """The per-query-head step takes the per-head workspace, which holds the
    per-head scores and the decode partials at once; its units are
    (sequence, query head), so the unit bound is reached 8x sooner."""
    ok = _desc(abi)
    topk = abi.sa_budget(abi.SA_BUDGET_TOPK, 8, 0.0, 0, 0, 0, 0)
    need = lib.sparse_attn_workspace_size_per_head(C.byref(ok), 32, 16)
    assert need > 0

    def call(desc=ok, max_sel=16, ws_bytes=need):
        return lib.sparse_attn_decode_step_per_head(C.byref(desc), 0x40000, 0, 0x50000, 32, C.byref(topk),
                                                    max_sel, 0.088, 0x60000, 0x70000, 0x80000, None,
                                                    0x100000, ws_bytes, None)
    assert call(ws_bytes=need - 256) == abi.SA_ERR_WORKSPACE
    assert call(max_sel=4) == abi.SA_ERR_INVALID          # top_k > max_sel
    assert call(desc=_desc(abi, batch=1025)) == abi.SA_ERR_UNSUPPORTED  # 2 x 1025 x 32 > 65536


def test_decode_step_append_validation(lib, abi):
    ok = _desc(abi)
    topk = abi.sa_budget(abi.SA_BUDGET_TOPK, 8, 0.0, 0, 0, 0, 0)

    def call(k_new=0x90000, v_new=0xa0000, max_sel=16, ws_bytes=1 << 30, out_dtype=abi.SA_OUT_F32):
        return lib.sparse_attn_decode_step_append(C.byref(ok), 0x40000, 0, 0x50000, 32, k_new, v_new,
                                                  C.byref(topk), max_sel, 0.088, 0x60000, 0x70000,
                                                  0x80000, out_dtype, None, 0x100000, ws_bytes, None)
    assert call(out_dtype=2) == abi.SA_ERR_INVALID
    assert call(k_new=0) == abi.SA_ERR_INVALID
    assert call(v_new=0) == abi.SA_ERR_INVALID
    assert call(k_new=0x90004) == abi.SA_ERR_INVALID      # not 8-byte aligned
    assert call(max_sel=4) == abi.SA_ERR_INVALID          # the step's own checks still apply
    assert call(ws_bytes=4096) == abi.SA_ERR_WORKSPACE


def test_build_meta_validation(lib, abi):
    ok = _desc(abi)
    assert lib.sparse_attn_build_meta(C.byref(ok), 7, 0, 0x40000, None) == abi.SA_ERR_INVALID
    assert lib.sparse_attn_build_meta(C.byref(ok), 0, 0, 0x40008, None) == abi.SA_ERR_INVALID
    assert lib.sparse_attn_build_meta(None, 0, 0, 0x40000, None) == abi.SA_ERR_INVALID


def test_route_validation(lib, abi):
    ok = _desc(abi, page_size=64)

    def call(desc=ok, k=32, rho=2, quantile=0.25, rows=128, tile=64):
        return lib.sparse_attn_route(C.byref(desc), 0x40000, 0, 0x50000, 28, rows, 0, tile, k, rho,
                                     quantile, None, 0x60000, 0x70000, 0x80000, 0x90000, 0xa0000,
                                     None, 0x100000, 1 << 30, None)
    assert call(desc=_desc(abi, page_size=64, batch=2)) == abi.SA_ERR_INVALID
    assert call(quantile=1.5) == abi.SA_ERR_INVALID
    assert call(k=0) == abi.SA_ERR_INVALID
    assert call(rho=0) == abi.SA_ERR_INVALID


def test_workspace_size(lib, abi):
    ok = _desc(abi)
    n = lib.sparse_attn_workspace_size(C.byref(ok), 32, 1, 16)
    assert n >= 256 + 4 * 65536 + 4 * 64 * 4
    assert lib.sparse_attn_workspace_size(C.byref(ok), 30, 1, 16) == 0
    assert lib.sparse_attn_workspace_size(C.byref(_desc(abi, head_dim=64)), 32, 1, 16) == 0
    assert lib.sparse_attn_workspace_init(None, 1 << 20, None) == abi.SA_ERR_WORKSPACE


def test_decode_static_rejects_tile_attention(lib, abi):
    """The workspace-free decode serves one-row decode only: multi-row tiles
    (tile_rows > 1) are refused on the host, before any CUDA call."""
    d = _desc(abi, batch=1)
    r = lib.sparse_attn_decode_static(C.byref(d), 0x50000, 32, 64, 0, 64, 0.088, 0x60000, 0x70000, 16,
                                      0x80000, None, None, None)
    assert r == abi.SA_ERR_UNSUPPORTED
    # and a one-row call with a bad row count is invalid, also before any launch
    r = lib.sparse_attn_decode_static(C.byref(d), 0x50000, 32, 3, 0, 1, 0.088, 0x60000, 0x70000, 16,
                                      0x80000, None, None, None)
    assert r == abi.SA_ERR_INVALID


def test_route_decode_step_validation(lib, abi):
    """The one-launch decode router validates on the host like the separate
    router call: chunks unsupported, quantile in [0, 1], rho*k bounded, a
    workspace that holds the scores, router tables and both windows' partials."""
    ok = _desc(abi)

    def call(desc=ok, k=8, rho=2, quantile=0.25, scale=0.088, ws_bytes=1 << 30, out=0x80000):
        return lib.sparse_attn_route_decode_step(C.byref(desc), 0x40000, 0, 0x50000, 32, k, rho, quantile, None,
                                                 scale, 0x60000, 0x70000, 0x90000, 0xa0000, 0xb0000, None, out,
                                                 None, 0x100000, ws_bytes, None)
    assert call(desc=_desc(abi, page_size=0, chunk_off=0x30000, n_chunks=0x30100)) == abi.SA_ERR_UNSUPPORTED
    assert call(quantile=1.5) == abi.SA_ERR_INVALID
    assert call(k=0) == abi.SA_ERR_INVALID
    assert call(k=512, rho=2) == abi.SA_ERR_UNSUPPORTED           # rho * k > 1023
    assert call(scale=float("nan")) == abi.SA_ERR_INVALID
    assert call(out=0x80004) == abi.SA_ERR_INVALID                # misaligned output
    need = lib.sparse_attn_workspace_size(C.byref(ok), 32, 1, 16)
    assert need > 0
    assert call(ws_bytes=need - 256) == abi.SA_ERR_WORKSPACE
