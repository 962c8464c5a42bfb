"""Python binding of libsparse_attn.so: the C-ABI calls under the same names,
taking torch tensors (device memory) and the current torch stream.

Argument marshalling only: every step of the path runs in the CUDA kernels
behind the C ABI.  Errors from the library raise SparseAttnError.
"""
from __future__ import annotations

import ctypes as C

import torch

from . import _abi
from ._abi import (SA_BUDGET_RATIO, SA_BUDGET_TOKENS, SA_BUDGET_TOPK, SA_SCORE_CENTROID,
                   SA_SCORE_ENVELOPE, sa_budget, sa_kv_desc)

lib = _abi.load()

RULES = {"envelope": SA_SCORE_ENVELOPE, "centroid": SA_SCORE_CENTROID}


class SparseAttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        msg = lib.sparse_attn_status_string(int(status)).decode()
        super().__init__(f"{where}: status {status} ({msg})")


def _check(st: int, where: str) -> None:
    if st != 0:
        raise SparseAttnError(st, where)


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _rule(rule) -> int:
    return RULES[rule] if isinstance(rule, str) else int(rule)


class KvCache:
    """A cache view: K, V bf16 [B, Hkv, cap, 128] plus sequence lengths and,
    for variable chunks, the CSR chunk table.  Holds references to the
    tensors so the pointers in `desc` stay valid."""

    def __init__(self, k: torch.Tensor, v: torch.Tensor, seq_len: torch.Tensor, *,
                 page_size: int, max_pages: int, chunk_off: torch.Tensor | None = None,
                 n_chunks: torch.Tensor | None = None):
        for name, t in (("k", k), ("v", v)):
            if t.dtype != torch.bfloat16 or t.dim() != 4 or not t.is_contiguous():
                raise ValueError(f"{name} must be a contiguous bf16 [B, Hkv, cap, D] tensor")
        if seq_len.dtype != torch.int32:
            raise ValueError("seq_len must be int32")
        if chunk_off is not None and (chunk_off.dtype != torch.int32 or not chunk_off.is_contiguous()):
            raise ValueError("chunk_off must be contiguous int32 [B, max_pages + 1]")
        self.k, self.v, self.seq_len = k, v, seq_len
        self.chunk_off, self.n_chunks = chunk_off, n_chunks
        B, Hkv, cap, D = k.shape
        self.page_size, self.max_pages = int(page_size), int(max_pages)
        self.desc = sa_kv_desc(B, Hkv, D, int(page_size), cap, k.data_ptr(), v.data_ptr(),
                               seq_len.data_ptr(), _ptr(chunk_off), _ptr(n_chunks), int(max_pages))

    @property
    def batch(self) -> int:
        return self.desc.batch

    @property
    def n_kv_heads(self) -> int:
        return self.desc.n_kv_heads

    def meta_buffer(self) -> torch.Tensor:
        return torch.empty((self.batch, self.n_kv_heads, self.max_pages, 512),
                           dtype=torch.uint8, device=self.k.device)


def budget_topk(k: int) -> sa_budget:
    return sa_budget(SA_BUDGET_TOPK, int(k), 0.0, 0, 0, 0, 0)


def budget_ratio(ratio: float, *, topk_val: int = 1, bos: int = 0, eos: int = 1) -> sa_budget:
    return sa_budget(SA_BUDGET_RATIO, 0, float(ratio), int(topk_val), int(bos), int(eos), 0)


def budget_tokens(n: int) -> sa_budget:
    return sa_budget(SA_BUDGET_TOKENS, 0, 0.0, 0, 0, 0, int(n))


def sparse_attn_workspace_size(kv: KvCache, n_q_heads: int, n_q_rows: int, max_sel: int) -> int:
    return int(lib.sparse_attn_workspace_size(C.byref(kv.desc), n_q_heads, n_q_rows, max_sel))


def sparse_attn_workspace_init(ws: torch.Tensor, stream=None) -> None:
    _check(lib.sparse_attn_workspace_init(ws.data_ptr(), ws.numel() * ws.element_size(),
                                          _stream(stream)), "sparse_attn_workspace_init")


def make_workspace(kv: KvCache, n_q_heads: int, n_q_rows: int, max_sel: int, stream=None) -> torch.Tensor:
    n = sparse_attn_workspace_size(kv, n_q_heads, n_q_rows, max_sel)
    if n == 0:
        raise SparseAttnError(_abi.SA_ERR_INVALID, "sparse_attn_workspace_size")
    ws = torch.empty(n, dtype=torch.uint8, device=kv.k.device)
    sparse_attn_workspace_init(ws, stream)
    return ws


def sparse_attn_workspace_size_per_head(kv: KvCache, n_q_heads: int, max_sel: int) -> int:
    return int(lib.sparse_attn_workspace_size_per_head(C.byref(kv.desc), int(n_q_heads), int(max_sel)))


def make_workspace_per_head(kv: KvCache, n_q_heads: int, max_sel: int, stream=None) -> torch.Tensor:
    """Workspace for sparse_attn_select_per_head / sparse_attn_decode_per_head /
    sparse_attn_decode_step_per_head."""
    n = sparse_attn_workspace_size_per_head(kv, n_q_heads, max_sel)
    if n == 0:
        raise SparseAttnError(_abi.SA_ERR_INVALID, "sparse_attn_workspace_size_per_head")
    ws = torch.empty(n, dtype=torch.uint8, device=kv.k.device)
    sparse_attn_workspace_init(ws, stream)
    return ws


def sparse_attn_build_meta(kv: KvCache, rule, first_token: int, meta: torch.Tensor, stream=None) -> None:
    _check(lib.sparse_attn_build_meta(C.byref(kv.desc), _rule(rule), int(first_token),
                                      meta.data_ptr(), _stream(stream)), "sparse_attn_build_meta")


def sparse_attn_select(kv: KvCache, meta: torch.Tensor, rule, q: torch.Tensor, budget: sa_budget,
                       max_sel: int, sel_idx: torch.Tensor, sel_count: torch.Tensor,
                       scores_out: torch.Tensor | None, ws: torch.Tensor, stream=None) -> None:
    if q.dtype != torch.bfloat16 or not q.is_contiguous():
        raise ValueError("q must be contiguous bf16 [B, Hq, 128]")
    _check(lib.sparse_attn_select(C.byref(kv.desc), meta.data_ptr(), _rule(rule), q.data_ptr(),
                                  q.shape[-2], C.byref(budget), int(max_sel), sel_idx.data_ptr(),
                                  sel_count.data_ptr(), _ptr(scores_out), ws.data_ptr(),
                                  ws.numel() * ws.element_size(), _stream(stream)),
           "sparse_attn_select")


def sparse_attn_select_per_head(kv: KvCache, meta: torch.Tensor, rule, q: torch.Tensor, budget: sa_budget,
                                max_sel: int, sel_idx: torch.Tensor, sel_count: torch.Tensor,
                                scores_out: torch.Tensor | None, ws: torch.Tensor, stream=None) -> None:
    """One page set per query head: sel_idx [B, Hq, max_sel], sel_count [B, Hq]."""
    if q.dtype != torch.bfloat16 or not q.is_contiguous():
        raise ValueError("q must be contiguous bf16 [B, Hq, 128]")
    _check(lib.sparse_attn_select_per_head(C.byref(kv.desc), meta.data_ptr(), _rule(rule), q.data_ptr(),
                                           q.shape[-2], C.byref(budget), int(max_sel), sel_idx.data_ptr(),
                                           sel_count.data_ptr(), _ptr(scores_out), ws.data_ptr(),
                                           ws.numel() * ws.element_size(), _stream(stream)),
           "sparse_attn_select_per_head")


def sparse_attn_decode_per_head(kv: KvCache, q: torch.Tensor, scale: float, idx: torch.Tensor,
                                count: torch.Tensor, max_sel: int, out: torch.Tensor,
                                lse: torch.Tensor | None, ws: torch.Tensor, stream=None) -> None:
    """Decode where query head h attends its own page list idx[b, h]."""
    if q.dtype != torch.bfloat16 or not q.is_contiguous():
        raise ValueError("q must be contiguous bf16 [B, Hq, 128]")
    if out.dtype != torch.float32 or not out.is_contiguous():
        raise ValueError("out must be contiguous fp32")
    _check(lib.sparse_attn_decode_per_head(C.byref(kv.desc), q.data_ptr(), q.shape[-2], float(scale),
                                           idx.data_ptr(), count.data_ptr(), int(max_sel), out.data_ptr(),
                                           _ptr(lse), ws.data_ptr(), ws.numel() * ws.element_size(),
                                           _stream(stream)),
           "sparse_attn_decode_per_head")


def sparse_attn_decode(kv: KvCache, q: torch.Tensor, n_q_rows: int, q_pos0: int, tile_rows: int,
                       scale: float, idx: torch.Tensor, count: torch.Tensor, max_sel: int,
                       out: torch.Tensor, lse: torch.Tensor | None, ws: torch.Tensor,
                       stream=None) -> None:
    if q.dtype != torch.bfloat16 or not q.is_contiguous():
        raise ValueError("q must be contiguous bf16")
    if out.dtype != torch.float32 or not out.is_contiguous():
        raise ValueError("out must be contiguous fp32")
    _check(lib.sparse_attn_decode(C.byref(kv.desc), q.data_ptr(), q.shape[-2], int(n_q_rows),
                                  int(q_pos0), int(tile_rows), float(scale), idx.data_ptr(),
                                  count.data_ptr(), int(max_sel), out.data_ptr(), _ptr(lse),
                                  ws.data_ptr(), ws.numel() * ws.element_size(), _stream(stream)),
           "sparse_attn_decode")


def sparse_attn_decode_step(kv: KvCache, meta: torch.Tensor, rule, q: torch.Tensor, budget: sa_budget,
                            max_sel: int, scale: float, sel_idx: torch.Tensor, sel_count: torch.Tensor,
                            out: torch.Tensor, lse: torch.Tensor | None, ws: torch.Tensor,
                            stream=None) -> None:
    if q.dtype != torch.bfloat16 or not q.is_contiguous():
        raise ValueError("q must be contiguous bf16 [B, Hq, 128]")
    if out.dtype != torch.float32 or not out.is_contiguous():
        raise ValueError("out must be contiguous fp32")
    _check(lib.sparse_attn_decode_step(C.byref(kv.desc), meta.data_ptr(), _rule(rule), q.data_ptr(),
                                       q.shape[-2], C.byref(budget), int(max_sel), float(scale),
                                       sel_idx.data_ptr(), sel_count.data_ptr(), out.data_ptr(),
                                       _ptr(lse), ws.data_ptr(), ws.numel() * ws.element_size(),
                                       _stream(stream)),
           "sparse_attn_decode_step")


def sparse_attn_decode_step_wait_test(kv: KvCache, meta: torch.Tensor, rule, q: torch.Tensor,
                                      budget: sa_budget, max_sel: int, scale: float, sel_idx: torch.Tensor,
                                      sel_count: torch.Tensor, out: torch.Tensor, lse: torch.Tensor | None,
                                      held_unit: int, flag_spin_limit: int, ws: torch.Tensor,
                                      stream=None) -> None:
    """The decode step with unit `held_unit`'s selection never published, so
    that its decode items run their bounded wait out (SA_ERR_TIMEOUT in the
    workspace status word).  A test of the error path; outputs unspecified."""
    if q.dtype != torch.bfloat16 or not q.is_contiguous():
        raise ValueError("q must be contiguous bf16 [B, Hq, 128]")
    if out.dtype != torch.float32 or not out.is_contiguous():
        raise ValueError("out must be contiguous fp32")
    _check(lib.sparse_attn_decode_step_wait_test(C.byref(kv.desc), meta.data_ptr(), _rule(rule), q.data_ptr(),
                                                 q.shape[-2], C.byref(budget), int(max_sel), float(scale),
                                                 sel_idx.data_ptr(), sel_count.data_ptr(), out.data_ptr(),
                                                 _ptr(lse), int(held_unit), int(flag_spin_limit),
                                                 ws.data_ptr(), ws.numel() * ws.element_size(),
                                                 _stream(stream)),
           "sparse_attn_decode_step_wait_test")


def sparse_attn_decode_step_per_head(kv: KvCache, meta: torch.Tensor, rule, q: torch.Tensor,
                                     budget: sa_budget, max_sel: int, scale: float, sel_idx: torch.Tensor,
                                     sel_count: torch.Tensor, out: torch.Tensor, lse: torch.Tensor | None,
                                     ws: torch.Tensor, stream=None) -> None:
    """The decode step with one page set per query head: sel_idx [B, Hq, max_sel],
    sel_count [B, Hq]; ws from make_workspace_per_head."""
    if q.dtype != torch.bfloat16 or not q.is_contiguous():
        raise ValueError("q must be contiguous bf16 [B, Hq, 128]")
    if out.dtype != torch.float32 or not out.is_contiguous():
        raise ValueError("out must be contiguous fp32")
    _check(lib.sparse_attn_decode_step_per_head(C.byref(kv.desc), meta.data_ptr(), _rule(rule), q.data_ptr(),
                                                q.shape[-2], C.byref(budget), int(max_sel), float(scale),
                                                sel_idx.data_ptr(), sel_count.data_ptr(), out.data_ptr(),
                                                _ptr(lse), ws.data_ptr(), ws.numel() * ws.element_size(),
                                                _stream(stream)),
           "sparse_attn_decode_step_per_head")


def sparse_attn_decode_step_append(kv: KvCache, meta: torch.Tensor, rule, q: torch.Tensor,
                                   k_new: torch.Tensor, v_new: torch.Tensor, budget: sa_budget,
                                   max_sel: int, scale: float, sel_idx: torch.Tensor,
                                   sel_count: torch.Tensor, out: torch.Tensor, lse: torch.Tensor | None,
                                   ws: torch.Tensor, stream=None) -> None:
    """The decode step with the newest token's key and value (bf16 [B, Hkv, 128])
    stored into the cache at row seq_len - 1 inside the same launch.  out is
    fp32 or bf16 [B, Hq, 128] (bf16: the fp32 result rounded to nearest even)."""
    if q.dtype != torch.bfloat16 or not q.is_contiguous():
        raise ValueError("q must be contiguous bf16 [B, Hq, 128]")
    for name, t in (("k_new", k_new), ("v_new", v_new)):
        if t.dtype != torch.bfloat16 or not t.is_contiguous() or tuple(t.shape) != (kv.batch, kv.k.shape[1], 128):
            raise ValueError(f"{name} must be contiguous bf16 [B, Hkv, 128]")
    if out.dtype not in (torch.float32, torch.bfloat16) or not out.is_contiguous():
        raise ValueError("out must be contiguous fp32 or bf16")
    out_dtype = _abi.SA_OUT_BF16 if out.dtype == torch.bfloat16 else _abi.SA_OUT_F32
    _check(lib.sparse_attn_decode_step_append(C.byref(kv.desc), meta.data_ptr(), _rule(rule), q.data_ptr(),
                                              q.shape[-2], k_new.data_ptr(), v_new.data_ptr(),
                                              C.byref(budget), int(max_sel), float(scale),
                                              sel_idx.data_ptr(), sel_count.data_ptr(), out.data_ptr(),
                                              out_dtype, _ptr(lse), ws.data_ptr(),
                                              ws.numel() * ws.element_size(), _stream(stream)),
           "sparse_attn_decode_step_append")


def sparse_attn_decode_static(kv: KvCache, q: torch.Tensor, n_q_rows: int, q_pos0: int,
                              tile_rows: int, scale: float, idx: torch.Tensor, count: torch.Tensor,
                              max_sel: int, out: torch.Tensor, lse: torch.Tensor | None,
                              device_status: torch.Tensor | None = None, stream=None) -> None:
    """sparse_attn_decode without a workspace, for callers that cannot
    allocate device memory where they run it: the scratch is an 8 MiB array
    inside the library, shared by every call, so calls must not overlap on
    the GPU.  One-row decode only (tile_rows == 1).  device_status: optional
    zeroed int32 device tensor that receives the first device-side error
    code; without it, device-side errors of the call are not reported."""
    if q.dtype != torch.bfloat16 or not q.is_contiguous():
        raise ValueError("q must be contiguous bf16")
    if out.dtype != torch.float32 or not out.is_contiguous():
        raise ValueError("out must be contiguous fp32")
    _check(lib.sparse_attn_decode_static(C.byref(kv.desc), q.data_ptr(), q.shape[-2], int(n_q_rows),
                                         int(q_pos0), int(tile_rows), float(scale), idx.data_ptr(),
                                         count.data_ptr(), int(max_sel), out.data_ptr(), _ptr(lse),
                                         _ptr(device_status), _stream(stream)),
           "sparse_attn_decode_static")


def sparse_attn_route_decode(kv: KvCache, meta: torch.Tensor, rule, q: torch.Tensor, k: int, rho: int,
                             quantile: float, tau: torch.Tensor | None, kv_idx: torch.Tensor,
                             kv_count: torch.Tensor, sigma: torch.Tensor, sigma_bar: torch.Tensor,
                             triggered: torch.Tensor, tau_out: torch.Tensor | None, ws: torch.Tensor,
                             stream=None) -> None:
    """The router with one-row tiles: every sequence's decode query is a tile.
    kv_idx [B, Hkv, rho*k] rank-ordered, -1 padded; kv_count [B, Hkv];
    sigma [B, Hkv]; sigma_bar [B]; triggered [B] uint8."""
    if q.dtype != torch.bfloat16 or not q.is_contiguous():
        raise ValueError("q must be contiguous bf16 [B, Hq, 128]")
    _check(lib.sparse_attn_route_decode(C.byref(kv.desc), meta.data_ptr(), _rule(rule), q.data_ptr(),
                                        q.shape[-2], int(k), int(rho), float(quantile), _ptr(tau),
                                        kv_idx.data_ptr(), kv_count.data_ptr(), sigma.data_ptr(),
                                        sigma_bar.data_ptr(), triggered.data_ptr(), _ptr(tau_out),
                                        ws.data_ptr(), ws.numel() * ws.element_size(), _stream(stream)),
           "sparse_attn_route_decode")


def sparse_attn_route_decode_step(kv: KvCache, meta: torch.Tensor, rule, q: torch.Tensor, k: int, rho: int,
                                  quantile: float, tau: torch.Tensor | None, scale: float, kv_idx: torch.Tensor,
                                  kv_count: torch.Tensor, sigma: torch.Tensor, sigma_bar: torch.Tensor,
                                  triggered: torch.Tensor, tau_out: torch.Tensor | None, out: torch.Tensor,
                                  lse: torch.Tensor | None, ws: torch.Tensor, stream=None) -> None:
    """The router on the decode batch and the decode over its lists in one
    launch (newest-page metadata refresh included): the outputs of
    sparse_attn_route_decode plus out [B, Hq, 128] fp32 and lse [B, Hq]."""
    if q.dtype != torch.bfloat16 or not q.is_contiguous():
        raise ValueError("q must be contiguous bf16 [B, Hq, 128]")
    if out.dtype != torch.float32 or not out.is_contiguous():
        raise ValueError("out must be contiguous fp32")
    _check(lib.sparse_attn_route_decode_step(C.byref(kv.desc), meta.data_ptr(), _rule(rule), q.data_ptr(),
                                             q.shape[-2], int(k), int(rho), float(quantile), _ptr(tau),
                                             float(scale), kv_idx.data_ptr(), kv_count.data_ptr(),
                                             sigma.data_ptr(), sigma_bar.data_ptr(), triggered.data_ptr(),
                                             _ptr(tau_out), out.data_ptr(), _ptr(lse), ws.data_ptr(),
                                             ws.numel() * ws.element_size(), _stream(stream)),
           "sparse_attn_route_decode_step")


def sparse_attn_route(kv: KvCache, meta: torch.Tensor, rule, q: torch.Tensor, n_q_rows: int,
                      q_pos0: int, tile_rows: int, k: int, rho: int, quantile: float,
                      tau: torch.Tensor | None, kv_idx: torch.Tensor, kv_count: torch.Tensor,
                      sigma: torch.Tensor, sigma_bar: torch.Tensor, triggered: torch.Tensor,
                      tau_out: torch.Tensor | None, ws: torch.Tensor, stream=None) -> None:
    if q.dtype != torch.bfloat16 or not q.is_contiguous():
        raise ValueError("q must be contiguous bf16 [rows, Hq, 128]")
    _check(lib.sparse_attn_route(C.byref(kv.desc), meta.data_ptr(), _rule(rule), q.data_ptr(),
                                 q.shape[-2], int(n_q_rows), int(q_pos0), int(tile_rows), int(k),
                                 int(rho), float(quantile), _ptr(tau), kv_idx.data_ptr(),
                                 kv_count.data_ptr(), sigma.data_ptr(), sigma_bar.data_ptr(),
                                 triggered.data_ptr(), _ptr(tau_out), ws.data_ptr(),
                                 ws.numel() * ws.element_size(), _stream(stream)),
           "sparse_attn_route")


def sparse_attn_get_device_status(ws: torch.Tensor, stream=None) -> int:
    out = C.c_int(0)
    _check(lib.sparse_attn_get_device_status(ws.data_ptr(), C.byref(out), _stream(stream)),
           "sparse_attn_get_device_status")
    return int(out.value)


def sparse_attn_status_string(code: int) -> str:
    return lib.sparse_attn_status_string(int(code)).decode()
