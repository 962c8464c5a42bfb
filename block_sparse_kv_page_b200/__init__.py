"""Query-aware block-sparse GQA decode attention and the uncertainty router,
hand-written CUDA for sm_100a behind a C ABI (include/sparse_attn.h).

The Python side only marshals arguments to libsparse_attn.so; importing the
package fails if the library has not been built (no CPU fallback).
"""
from .ops import (KvCache, SparseAttnError, budget_ratio, budget_tokens, budget_topk,  # noqa: F401
                  lib, make_workspace, make_workspace_per_head, sparse_attn_build_meta,
                  sparse_attn_decode, sparse_attn_decode_per_head, sparse_attn_select_per_head,
                  sparse_attn_workspace_size_per_head,
                  sparse_attn_decode_static, sparse_attn_decode_step,
                  sparse_attn_decode_step_append, sparse_attn_decode_step_per_head,
                  sparse_attn_decode_step_wait_test,
                  sparse_attn_get_device_status, sparse_attn_route, sparse_attn_route_decode,
                  sparse_attn_route_decode_step,
                  sparse_attn_select,
                  sparse_attn_status_string, sparse_attn_workspace_init,
                  sparse_attn_workspace_size)
from ._abi import (SA_BUDGET_RATIO, SA_BUDGET_TOKENS, SA_BUDGET_TOPK, SA_ERR_CUDA,  # noqa: F401
                   SA_ERR_DEVICE_CHECK, SA_ERR_INVALID, SA_ERR_TIMEOUT, SA_ERR_UNSUPPORTED,
                   SA_ERR_WORKSPACE, SA_OK, SA_OUT_BF16, SA_OUT_F32, SA_SCORE_CENTROID,
                   SA_SCORE_ENVELOPE)
