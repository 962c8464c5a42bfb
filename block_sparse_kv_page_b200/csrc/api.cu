// C-ABI entry points: host-side argument validation, workspace layout and
// kernel launches.  Nothing here computes results; every step of the path
// runs in the kernels of meta.cu, select.cu, decode.cu, step.cu, route.cu and
// tile_attn_tc.cu.
//
// Workspace layout (byte offsets from ws, which must be 256-byte aligned):
//   [0, 256)                 status word (int32) at 0; item-queue counters of
//                            the persistent kernels at 64 (select), 72
//                            (decode), 80 (router), 88 (decode step), 96
//                            (routed decode step's counters); each kernel
//                            leaves its queue rewound to zero
//   [256, 256 + 4*kMaxUnits) last-CTA counters, shared by every call; each
//                            call uses counters [0, its units) and leaves
//                            them zero, so calls issued in order on one
//                            stream can share one workspace
//   [kScratch, ...)          per-call scratch (scores of select, split
//                            partials of decode -- after the scores in the
//                            decode step --, router tables), not preserved
//                            between calls
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "common.cuh"
#include "internal.h"

namespace sa {

constexpr int kMaxUnits = 65536;
constexpr size_t kQueueSelect = 64;
constexpr size_t kQueueDecode = 72;
constexpr size_t kQueueRoute = 80;
constexpr size_t kQueueStep = 88;
constexpr size_t kQueueRouteStep = 96;  // routed decode step: units selected, triggers-published flag
constexpr int kMaxRouteTiles = 1024;
constexpr int kMaxRouteList = 1023;
constexpr size_t kScratch = 256 + 4 * (size_t)kMaxUnits;
constexpr int kMaxSelectPages = 16384;
constexpr int kMaxChunkSel = 8192;

size_t select_smem_bytes(int max_pages);

namespace {

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

sa_status check_kv(const sa_kv_desc* kv) {
  if (!kv) return SA_ERR_INVALID;
  if (kv->batch < 1 || kv->n_kv_heads < 1 || kv->max_pages < 1 || kv->cap_tokens < 1)
    return SA_ERR_INVALID;
  if (kv->head_dim != kHeadDim) return SA_ERR_UNSUPPORTED;
  if (kv->page_size != 0 && (kv->page_size % 16 != 0 || kv->page_size < 16 || kv->page_size > 256))
    return SA_ERR_UNSUPPORTED;
  if (kv->cap_tokens > 0x7fffffffLL) return SA_ERR_UNSUPPORTED;
  if (!kv->k || !kv->v || !aligned(kv->k, 16) || !aligned(kv->v, 16)) return SA_ERR_INVALID;
  if (!kv->seq_len || !aligned(kv->seq_len, 4)) return SA_ERR_INVALID;
  if (kv->page_size == 0) {
    if (!kv->chunk_off || !kv->n_chunks || !aligned(kv->chunk_off, 4) || !aligned(kv->n_chunks, 4))
      return SA_ERR_INVALID;
  }
  return SA_OK;
}

KvView view(const sa_kv_desc* kv) {
  KvView v;
  v.B = kv->batch;
  v.Hkv = kv->n_kv_heads;
  v.page_size = kv->page_size;
  v.cap = kv->cap_tokens;
  v.k = kv->k;
  v.v = kv->v;
  v.seq_len = kv->seq_len;
  v.chunk_off = kv->chunk_off;
  v.n_chunks = kv->n_chunks;
  v.max_pages = kv->max_pages;
  return v;
}

sa_status check_group(const sa_kv_desc* kv, int n_q_heads, int* G) {
  if (n_q_heads < 1 || n_q_heads % kv->n_kv_heads != 0) return SA_ERR_INVALID;
  *G = n_q_heads / kv->n_kv_heads;
  if (*G > kMaxGroup) return SA_ERR_UNSUPPORTED;
  return SA_OK;
}

sa_status check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (!ws || !aligned(ws, 256)) return SA_ERR_WORKSPACE;
  if (ws_bytes < need) return SA_ERR_WORKSPACE;
  return SA_OK;
}

sa_status launched(cudaError_t e) {
  if (e != cudaSuccess) {
    cudaGetLastError();
    return SA_ERR_CUDA;
  }
  return SA_OK;
}

// Tiles a unit is expected to hold under a token budget: the budget in 16-token
// tiles plus an eighth for the ragged last tiles of the kept chunks.  It only
// sizes the work split of the decode step (any actual count is handled).
int token_budget_tiles(int token_budget) {
  const long long t = ((long long)token_budget + 15) / 16;
  const long long e = t + (t + 7) / 8;
  return e < 1 ? 1 : (e > 0x3fffffff ? 0x3fffffff : (int)e);
}

int max_tiles_per_unit(const sa_kv_desc* kv, int max_sel) {
  const long long t = kv->page_size > 0 ? (long long)max_sel * (kv->page_size / 16)
                                        : (long long)max_sel * 16;
  return t > 0x3fffffff ? 0x3fffffff : (int)t;
}

// Group scores, one row of max_pages rounded up to 4 floats per unit, so the
// selecting CTA can read a row with 16-byte loads.
int score_stride(const sa_kv_desc* kv) { return (kv->max_pages + 3) & ~3; }

// Decode router scratch after the scores: sigma (double) and eligible
// counts per unit, and (routed decode step) the triggered units' list.
size_t route_decode_ws_bytes(long long units) {
  return align256((size_t)units * 8) + align256((size_t)units * 4) + align256((size_t)units * 16);
}

size_t select_scratch(const sa_kv_desc* kv, bool per_head = false, int n_q_heads = 0) {
  const size_t units = (size_t)kv->batch * (per_head ? n_q_heads : kv->n_kv_heads);
  return align256(units * score_stride(kv) * sizeof(float));
}

// Per-head decode step: the union of each KV head's G page sets, entries
// int32 [B * Hkv][max_pages], head masks uint8 [B * Hkv][max_pages], counts
// int32 [B * Hkv].
size_t union_mask_off(const sa_kv_desc* kv) {
  return align256((size_t)kv->batch * kv->n_kv_heads * kv->max_pages * 4);
}
size_t union_count_off(const sa_kv_desc* kv) {
  return union_mask_off(kv) + align256((size_t)kv->batch * kv->n_kv_heads * kv->max_pages);
}
size_t union_scratch(const sa_kv_desc* kv) {
  return union_count_off(kv) + align256((size_t)kv->batch * kv->n_kv_heads * 4);
}

// Split partials: one slot per work item (none when no unit is split).
size_t decode_scratch(const DecodePlan& p) {
  if (p.splits <= 1 && p.splits_fine <= 1) return 0;
  return align256((size_t)p.items * kMaxGroup * (kHeadDim + 4) * sizeof(float));
}

}  // namespace

namespace {
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else
      cudaGetLastError();
  }
  return fn;
}
}  // namespace

bool encode_tmap_2d(CUtensorMap* map, const void* base, unsigned long long rows, int row_bytes,
                    CUtensorMapDataType dt, int elem_bytes, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)(row_bytes / elem_bytes), (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  const cuuint32_t box[2] = {(cuuint32_t)(128 / elem_bytes), (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t set_smem_attr(const void* func, size_t bytes) {
  struct Entry {
    const void* f;
    int dev;
    size_t bytes;
  };
  static Entry cache[64];
  static int n = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaGetLastError();
  for (int i = 0; i < n; ++i)
    if (cache[i].f == func && cache[i].dev == dev && cache[i].bytes >= bytes) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  for (int i = 0; i < n; ++i)
    if (cache[i].f == func && cache[i].dev == dev) {
      cache[i].bytes = bytes;
      return cudaSuccess;
    }
  if (n < 64) cache[n++] = Entry{func, dev, bytes};
  return cudaSuccess;
}

int device_sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return 148;
  }
  if (dev >= 0 && dev < 64 && cache[dev] > 0) return cache[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return 148;
  }
  if (dev >= 0 && dev < 64) cache[dev] = n;
  return n;
}

namespace {
// Multi-row tiles (router output): causal attention of each tile over its
// listed 64-token blocks.  Needs only the status word of the workspace.
sa_status tile_attention(const sa_kv_desc* kv, const void* q, int n_q_heads, int G, int n_q_rows,
                         int q_pos0, int tile_rows, float scale, const int32_t* idx,
                         const int32_t* count, int max_sel, float* out, float* lse, int* status,
                         void* ws, size_t ws_bytes, void* stream) {
  if (kv->page_size != 64) return SA_ERR_UNSUPPORTED;
  if (q_pos0 < 0 || max_sel > kMaxRouteList + 1) return SA_ERR_UNSUPPORTED;
  const long long T = ((long long)n_q_rows + tile_rows - 1) / tile_rows;
  if (T * kv->n_kv_heads > kMaxUnits) return SA_ERR_UNSUPPORTED;
  if (ws) {
    if (!aligned(ws, 256) || ws_bytes < 256) return SA_ERR_WORKSPACE;
  } else if (status) {
    return SA_ERR_WORKSPACE;
  }
  const unsigned long long kv_rows = (unsigned long long)kv->n_kv_heads * kv->cap_tokens;
  if (kv_rows > 0x7fffffffULL) return SA_ERR_UNSUPPORTED;
  TileAttnArgs a{};  // every field zero unless set below
  if (!encode_tmap_2d(&a.tmap_k, kv->k, kv_rows, kHeadDim * 2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 64) ||
      !encode_tmap_2d(&a.tmap_v, kv->v, kv_rows, kHeadDim * 2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 64))
    return SA_ERR_CUDA;
  a.kv = view(kv);
  a.q = q;
  a.Hq = n_q_heads;
  a.G = G;
  a.n_rows = n_q_rows;
  a.q_pos0 = q_pos0;
  a.tile_rows = tile_rows;
  a.n_tiles = (int)T;
  a.n_mchunks = tile_attn_tc_mchunks(tile_rows * G);
  a.scale_log2 = scale * kLog2e;
  a.idx = idx;
  a.count = count;
  a.max_sel = max_sel;
  a.out = out;
  a.lse = lse;
  a.status = status;
  return launched(launch_tile_attn_tc(a, (cudaStream_t)stream));
}

// Argument checks of a selection (sparse_attn_select and sparse_attn_decode_step).
sa_status check_select(const sa_kv_desc* kv, const void* meta, sa_score_rule rule, const void* q,
                       int n_q_heads, const sa_budget* budget, int max_sel, const int32_t* sel_idx,
                       const int32_t* sel_count, const float* scores_out, int* G) {
  sa_status s = check_kv(kv);
  if (s != SA_OK) return s;
  if ((s = check_group(kv, n_q_heads, G)) != SA_OK) return s;
  if (rule != SA_SCORE_ENVELOPE && rule != SA_SCORE_CENTROID) return SA_ERR_INVALID;
  if (!meta || !aligned(meta, 16) || !q || !aligned(q, 16)) return SA_ERR_INVALID;
  if (!budget || !sel_idx || !sel_count || max_sel < 1) return SA_ERR_INVALID;
  if (!aligned(sel_idx, 4) || !aligned(sel_count, 4) || (scores_out && !aligned(scores_out, 4)))
    return SA_ERR_INVALID;
  if (kv->max_pages > kMaxSelectPages) return SA_ERR_UNSUPPORTED;
  const long long units = (long long)kv->batch * kv->n_kv_heads;
  if (units > kMaxUnits) return SA_ERR_UNSUPPORTED;
  switch (budget->kind) {
    case SA_BUDGET_TOPK:
      if (budget->top_k < 1 || budget->top_k > max_sel) return SA_ERR_INVALID;
      break;
    case SA_BUDGET_RATIO: {
      if (!(budget->topk_ratio > 0.0 && budget->topk_ratio <= 1.0)) return SA_ERR_INVALID;
      if (budget->topk_val < 0 || budget->bos < 0 || budget->eos < 0) return SA_ERR_INVALID;
      const long long fl = (long long)std::floor((double)kv->max_pages * budget->topk_ratio);
      long long K = (long long)budget->topk_val + budget->bos + budget->eos;
      if (fl > K) K = fl;
      if (K > kv->max_pages) K = kv->max_pages;
      if (K > max_sel) return SA_ERR_INVALID;
      break;
    }
    case SA_BUDGET_TOKENS:
      if (kv->page_size != 0) return SA_ERR_UNSUPPORTED;  // token budgets are for variable chunks
      if (budget->token_budget < 0) return SA_ERR_INVALID;
      break;
    default:
      return SA_ERR_INVALID;
  }
  const unsigned long long meta_rows = (unsigned long long)units * kv->max_pages;
  if (meta_rows > 0x7fffffffULL) return SA_ERR_UNSUPPORTED;  // TMA row coordinates are int32
  return SA_OK;
}

// Selection arguments (scores in the scratch, unit counters after the
// header); false if the metadata tensor map cannot be encoded.
bool fill_select(SelectArgs* a, const sa_kv_desc* kv, const void* meta, sa_score_rule rule,
                 const void* q, int n_q_heads, int G, const sa_budget* budget, int max_sel,
                 int32_t* sel_idx, int32_t* sel_count, float* scores_out, void* ws) {
  const unsigned long long meta_rows = (unsigned long long)kv->batch * kv->n_kv_heads * kv->max_pages;
  const bool env = rule == SA_SCORE_ENVELOPE;
  if (!encode_tmap_2d(&a->tmap_meta, meta, meta_rows, kMetaBytes,
                      env ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                      env ? 2 : 4, 16))
    return false;
  a->kv = view(kv);
  a->meta = meta;
  a->rule = (int)rule;
  a->q = q;
  a->Hq = n_q_heads;
  a->G = G;
  a->budget_kind = (int)budget->kind;
  a->top_k = budget->top_k;
  a->topk_val = budget->topk_val;
  a->bos = budget->bos;
  a->eos = budget->eos;
  a->token_budget = budget->token_budget;
  a->ratio = budget->topk_ratio;
  a->max_sel = max_sel;
  a->sel_idx = sel_idx;
  a->sel_count = sel_count;
  a->scores_out = scores_out;
  a->ws_scores = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + kScratch);
  a->ws_stride = score_stride(kv);
  a->ws_count = reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(ws) + 256);
  a->ws_queue = nullptr;
  a->status = reinterpret_cast<int*>(ws);
  a->splits = select_splits(kv->batch * kv->n_kv_heads, kv->max_pages, device_sm_count());
  a->meta_refresh = nullptr;
  a->per_head = 0;
  a->score_only = 0;
  a->k_new = a->v_new = nullptr;
  a->k_dst = a->v_dst = nullptr;
  return true;
}

// Decode arguments for one query row per sequence (tile_rows = 1); false if
// the K/V tensor maps cannot be encoded.
bool fill_decode(DecodeArgs* a, const sa_kv_desc* kv, const void* q, int n_q_heads, int G,
                 float scale, const int32_t* idx, const int32_t* count, int max_sel, float* out,
                 float* lse, float* ws_part, uint32_t* ws_count, int* status,
                 const DecodePlan& plan) {
  const unsigned long long kv_rows = (unsigned long long)kv->batch * kv->n_kv_heads * kv->cap_tokens;
  if (!encode_tmap_2d(&a->tmap_k, kv->k, kv_rows, kHeadDim * 2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 16) ||
      !encode_tmap_2d(&a->tmap_v, kv->v, kv_rows, kHeadDim * 2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 16))
    return false;
  a->kv = view(kv);
  a->q = q;
  a->Hq = n_q_heads;
  a->G = G;
  a->n_rows = kv->batch;
  a->q_pos0 = 0;
  a->tile_rows = 1;
  a->scale_log2 = scale * kLog2e;
  a->idx = idx;
  a->count = count;
  a->max_sel = max_sel;
  a->out = out;
  a->out_bf16 = nullptr;
  a->per_head = 0;
  a->lse = lse;
  a->ws_part = ws_part;
  a->ws_count = ws_count;
  a->ws_queue = nullptr;
  a->status = status;
  a->splits = plan.splits;
  a->fine_unit0 = plan.fine_unit0;
  a->splits_fine = plan.splits_fine;
  a->n_items = (int)plan.items;
  return true;
}

}  // namespace

}  // namespace sa

using namespace sa;

extern "C" {

size_t sparse_attn_workspace_size(const sa_kv_desc* kv, int32_t n_q_heads, int32_t n_q_rows,
                                  int32_t max_sel) {
  if (check_kv(kv) != SA_OK || max_sel < 1 || n_q_rows < 0) return 0;
  int G;
  if (check_group(kv, n_q_heads, &G) != SA_OK) return 0;
  const int sm = device_sm_count();
  const int rows = n_q_rows > kv->batch ? n_q_rows : kv->batch;
  const long long units = (long long)rows * kv->n_kv_heads;
  if (units > kMaxUnits) return 0;
  // selection scores + decode partials (both live during sparse_attn_decode_step)
  const DecodePlan plan = decode_plan((int)units, max_tiles_per_unit(kv, max_sel), sm);
  size_t tail = select_scratch(kv) + decode_scratch(plan);
  const int route_tiles = rows < kMaxRouteTiles ? rows : kMaxRouteTiles;  // tiles <= query rows
  const size_t rt = route_ws_bytes(route_tiles, kv->n_kv_heads, kv->max_pages, max_sel);
  if (rt > tail) tail = rt;
  if (kv->batch <= kMaxRouteTiles && kv->page_size > 0) {  // decode router: scores + router scratch
    const long long ru = (long long)kv->batch * kv->n_kv_heads;
    size_t rd = select_scratch(kv) + route_decode_ws_bytes(ru);
    // the routed decode step adds split partials of its top-k windows (at
    // most the splits of a plain decode over max_sel), of its expansion
    // windows (planned for as few as one row's units) and one merged top-k
    // partial per unit
    const DecodePlan rp = decode_plan((int)ru, max_tiles_per_unit(kv, max_sel), sm);
    const DecodePlan ep = decode_plan(kv->n_kv_heads, max_tiles_per_unit(kv, max_sel), sm);
    const int rs = rp.splits + ep.splits;
    rd += decode_scratch(DecodePlan{rs, (int)ru, rs, ru * (rs + 1)});
    if (rd > tail) tail = rd;
  }
  return kScratch + tail;
}

size_t sparse_attn_workspace_size_per_head(const sa_kv_desc* kv, int32_t n_q_heads, int32_t max_sel) {
  if (check_kv(kv) != SA_OK || max_sel < 1) return 0;
  int G;
  if (check_group(kv, n_q_heads, &G) != SA_OK) return 0;
  const long long units = (long long)kv->batch * n_q_heads;
  if (units > kMaxUnits) return 0;
  const int sm = device_sm_count();
  // the separate per-head decode: partials per (sequence, query head)
  const DecodePlan plan = decode_plan((int)units, max_tiles_per_unit(kv, max_sel), sm);
  const size_t calls = decode_scratch(plan);
  // the fused per-head step keeps the scores, the KV heads' unions and the
  // split partials of the union decode at once
  const long long kv_units = (long long)kv->batch * kv->n_kv_heads;
  const int dec_sel = (int)std::min<long long>((long long)G * max_sel, kv->max_pages);
  const DecodePlan up = decode_plan((int)kv_units, max_tiles_per_unit(kv, dec_sel), sm);
  const size_t step = union_scratch(kv) + decode_scratch(up);
  return kScratch + select_scratch(kv, true, n_q_heads) + (step > calls ? step : calls);
}

sa_status sparse_attn_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || !aligned(ws, 256) || ws_bytes < kScratch) return SA_ERR_WORKSPACE;
  return launched(cudaMemsetAsync(ws, 0, ws_bytes, (cudaStream_t)stream));
}

sa_status sparse_attn_build_meta(const sa_kv_desc* kv, sa_score_rule rule, int32_t first_token,
                                 void* meta, void* stream) {
  sa_status s = check_kv(kv);
  if (s != SA_OK) return s;
  if (rule != SA_SCORE_ENVELOPE && rule != SA_SCORE_CENTROID) return SA_ERR_INVALID;
  if (!meta || !aligned(meta, 16)) return SA_ERR_INVALID;
  return launched(launch_build_meta(view(kv), (int)rule, first_token, meta, nullptr,
                                    (cudaStream_t)stream));
}

// Selection per (sequence, KV head), or per (sequence, query head).
static sa_status select_impl(const sa_kv_desc* kv, const void* meta, sa_score_rule rule,
                             const void* q, int32_t n_q_heads, const sa_budget* budget,
                             int32_t max_sel, int32_t* sel_idx, int32_t* sel_count,
                             float* scores_out, bool per_head, void* ws, size_t ws_bytes,
                             void* stream) {
  int G;
  sa_status s = check_select(kv, meta, rule, q, n_q_heads, budget, max_sel, sel_idx, sel_count,
                             scores_out, &G);
  if (s != SA_OK) return s;
  if (per_head && (long long)kv->batch * n_q_heads > kMaxUnits) return SA_ERR_UNSUPPORTED;
  const size_t need = kScratch + select_scratch(kv, per_head, n_q_heads);
  if ((s = check_ws(ws, ws_bytes, need)) != SA_OK) return s;
  SelectArgs a{};  // every field zero unless set below
  if (!fill_select(&a, kv, meta, rule, q, n_q_heads, G, budget, max_sel, sel_idx, sel_count,
                   scores_out, ws))
    return SA_ERR_CUDA;
  if (per_head) {
    a.per_head = 1;
    a.splits = select_splits(kv->batch * n_q_heads, kv->max_pages, device_sm_count());
  }
  a.ws_queue = reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(ws) + kQueueSelect);
  return launched(launch_select(a, (cudaStream_t)stream));
}

sa_status sparse_attn_select(const sa_kv_desc* kv, const void* meta, sa_score_rule rule,
                             const void* q, int32_t n_q_heads, const sa_budget* budget,
                             int32_t max_sel, int32_t* sel_idx, int32_t* sel_count,
                             float* scores_out, void* ws, size_t ws_bytes, void* stream) {
  return select_impl(kv, meta, rule, q, n_q_heads, budget, max_sel, sel_idx, sel_count, scores_out,
                     false, ws, ws_bytes, stream);
}

sa_status sparse_attn_select_per_head(const sa_kv_desc* kv, const void* meta, sa_score_rule rule,
                                      const void* q, int32_t n_q_heads, const sa_budget* budget,
                                      int32_t max_sel, int32_t* sel_idx, int32_t* sel_count,
                                      float* scores_out, void* ws, size_t ws_bytes, void* stream) {
  return select_impl(kv, meta, rule, q, n_q_heads, budget, max_sel, sel_idx, sel_count, scores_out,
                     true, ws, ws_bytes, stream);
}

// Decode of one query row per sequence (validated arguments), per KV head or
// per query head.
static sa_status decode_rows(const sa_kv_desc* kv, const void* q, int32_t n_q_heads, int G,
                             float scale, const int32_t* idx, const int32_t* count, int32_t max_sel,
                             float* out, float* lse, bool per_head, void* ws, size_t ws_bytes,
                             void* stream) {
  if (kv->page_size == 0 && max_sel > kMaxChunkSel) return SA_ERR_UNSUPPORTED;
  const long long units = (long long)kv->batch * (per_head ? n_q_heads : kv->n_kv_heads);
  if (units > kMaxUnits) return SA_ERR_UNSUPPORTED;
  const unsigned long long kv_rows = (unsigned long long)kv->batch * kv->n_kv_heads * kv->cap_tokens;
  if (kv_rows > 0x7fffffffULL) return SA_ERR_UNSUPPORTED;  // TMA row coordinates are int32
  const DecodePlan plan = decode_plan((int)units, max_tiles_per_unit(kv, max_sel), device_sm_count());
  if (plan.items > 0x7fffffffLL) return SA_ERR_UNSUPPORTED;
  const size_t need = kScratch + decode_scratch(plan);
  sa_status s;
  if ((s = check_ws(ws, ws_bytes, need)) != SA_OK) return s;

  DecodeArgs a{};  // every field zero unless set below
  char* w = reinterpret_cast<char*>(ws);
  if (!fill_decode(&a, kv, q, n_q_heads, G, scale, idx, count, max_sel, out, lse,
                   reinterpret_cast<float*>(w + kScratch), reinterpret_cast<uint32_t*>(w + 256),
                   reinterpret_cast<int*>(ws), plan))
    return SA_ERR_CUDA;
  a.per_head = per_head ? 1 : 0;
  a.ws_queue = reinterpret_cast<uint32_t*>(w + kQueueDecode);
  return launched(launch_decode(a, (cudaStream_t)stream));
}

sa_status sparse_attn_decode(const sa_kv_desc* kv, const void* q, int32_t n_q_heads,
                             int32_t n_q_rows, int32_t q_pos0, int32_t tile_rows, float scale,
                             const int32_t* idx, const int32_t* count, int32_t max_sel,
                             float* out, float* lse, void* ws, size_t ws_bytes, void* stream) {
  sa_status s = check_kv(kv);
  if (s != SA_OK) return s;
  int G;
  if ((s = check_group(kv, n_q_heads, &G)) != SA_OK) return s;
  if (!q || !aligned(q, 16) || !idx || !count || !aligned(idx, 4) || !aligned(count, 4))
    return SA_ERR_INVALID;
  if (!out || !aligned(out, 16) || (lse && !aligned(lse, 4))) return SA_ERR_INVALID;
  if (max_sel < 1 || tile_rows < 1 || n_q_rows < 1) return SA_ERR_INVALID;
  if (!std::isfinite(scale)) return SA_ERR_INVALID;
  if (tile_rows == 1) {
    if (n_q_rows != kv->batch) return SA_ERR_INVALID;
  } else {
    if (kv->batch != 1 || kv->page_size == 0) return SA_ERR_INVALID;
    return tile_attention(kv, q, n_q_heads, G, n_q_rows, q_pos0, tile_rows, scale, idx, count,
                          max_sel, out, lse, reinterpret_cast<int*>(ws), ws, ws_bytes, stream);
  }
  return decode_rows(kv, q, n_q_heads, G, scale, idx, count, max_sel, out, lse, false, ws, ws_bytes,
                     stream);
}

sa_status sparse_attn_decode_per_head(const sa_kv_desc* kv, const void* q, int32_t n_q_heads,
                                      float scale, const int32_t* idx, const int32_t* count,
                                      int32_t max_sel, float* out, float* lse, void* ws,
                                      size_t ws_bytes, void* stream) {
  sa_status s = check_kv(kv);
  if (s != SA_OK) return s;
  int G;
  if ((s = check_group(kv, n_q_heads, &G)) != SA_OK) return s;
  if (!q || !aligned(q, 16) || !idx || !count || !aligned(idx, 4) || !aligned(count, 4))
    return SA_ERR_INVALID;
  if (!out || !aligned(out, 16) || (lse && !aligned(lse, 4))) return SA_ERR_INVALID;
  if (max_sel < 1) return SA_ERR_INVALID;
  if (!std::isfinite(scale)) return SA_ERR_INVALID;
  return decode_rows(kv, q, n_q_heads, G, scale, idx, count, max_sel, out, lse, true, ws, ws_bytes,
                     stream);
}

// The decode step with or without the append of the newest token's K/V.
static sa_status decode_step(const sa_kv_desc* kv, void* meta, sa_score_rule rule,
                             const void* q, int32_t n_q_heads, const void* k_new,
                             const void* v_new, const sa_budget* budget, int32_t max_sel,
                             float scale, int32_t* sel_idx, int32_t* sel_count, void* out,
                             bool out_bf16, float* lse, bool per_head, void* ws, size_t ws_bytes,
                             void* stream, int hold_flag_of = 0, uint32_t flag_spin_limit = 0) {
  int G;
  sa_status s = check_select(kv, meta, rule, q, n_q_heads, budget, max_sel, sel_idx, sel_count,
                             nullptr, &G);
  if (s != SA_OK) return s;
  if (!out || !aligned(out, 16) || (lse && !aligned(lse, 4))) return SA_ERR_INVALID;
  if (!std::isfinite(scale)) return SA_ERR_INVALID;
  if (kv->page_size == 0 && max_sel > kMaxChunkSel) return SA_ERR_UNSUPPORTED;
  const long long units = (long long)kv->batch * (per_head ? n_q_heads : kv->n_kv_heads);
  const long long kv_units = (long long)kv->batch * kv->n_kv_heads;
  // unit flags + split counters (+ per-head step: scoring and selection counts per KV head)
  if (2 * units + (per_head ? 2 * kv_units : 0) > kMaxUnits) return SA_ERR_UNSUPPORTED;
  const unsigned long long kv_rows = (unsigned long long)kv->batch * kv->n_kv_heads * kv->cap_tokens;
  if (kv_rows > 0x7fffffffULL) return SA_ERR_UNSUPPORTED;  // TMA row coordinates are int32
  const int sm = device_sm_count();
  // per-head: the decode runs per (sequence, KV head) over the union of the
  // G heads' sets (at most G * max_sel entries, and at most max_pages)
  const int dec_sel = per_head ? (int)std::min<long long>((long long)G * max_sel, kv->max_pages) : max_sel;
  int plan_tiles = max_tiles_per_unit(kv, dec_sel);
  if (budget->kind == SA_BUDGET_TOKENS) {  // the budget, not max_sel, bounds what is attended
    const long long t = (long long)token_budget_tiles(budget->token_budget) * (per_head ? G : 1);
    if (t < plan_tiles) plan_tiles = (int)t;
  }
  const DecodePlan plan = decode_plan((int)kv_units, plan_tiles, sm);
  const size_t sel_bytes = select_scratch(kv, per_head, n_q_heads);
  const size_t union_bytes = per_head ? union_scratch(kv) : 0;
  const size_t need = kScratch + sel_bytes + union_bytes + decode_scratch(plan);
  if ((s = check_ws(ws, ws_bytes, need)) != SA_OK) return s;
  if (step_smem_bytes(kv->max_pages, per_head ? kv->max_pages : max_sel, kv->page_size == 0) > 227 * 1024)
    return SA_ERR_UNSUPPORTED;

  StepArgs a{};  // every field zero unless set below
  char* w = reinterpret_cast<char*>(ws);
  // unit flags and split counters at w + 256, one per (sequence, KV head)
  // (the per-head step flags the KV heads' unions, not the query heads)
  uint32_t* flags = reinterpret_cast<uint32_t*>(w + 256);
  char* union_base = w + kScratch + sel_bytes;
  if (!fill_select(&a.sel, kv, meta, rule, q, n_q_heads, G, budget, max_sel, sel_idx, sel_count,
                   nullptr, ws) ||
      !fill_decode(&a.dec, kv, q, n_q_heads, G, scale,
                   per_head ? reinterpret_cast<int32_t*>(union_base) : sel_idx,
                   per_head ? reinterpret_cast<int32_t*>(union_base + union_count_off(kv)) : sel_count,
                   dec_sel, out_bf16 ? nullptr : static_cast<float*>(out), lse,
                   reinterpret_cast<float*>(union_base + union_bytes), flags + kv_units,
                   reinterpret_cast<int*>(ws), plan))
    return SA_ERR_CUDA;
  if (out_bf16) a.dec.out_bf16 = static_cast<__nv_bfloat16*>(out);
  if (per_head) {
    // scoring items per (sequence, KV head) write the G heads' rows; then one
    // selection item per (sequence, query head); the decode per (sequence,
    // KV head) over the union of its heads' sets, each head masked to its own
    a.sel.per_head = 1;
    a.sel.kv_scored = flags + 2 * kv_units;
    a.sel.kv_selected = flags + 3 * kv_units;
    a.sel.union_idx = reinterpret_cast<int32_t*>(union_base);
    a.sel.union_mask = reinterpret_cast<uint8_t*>(union_base + union_mask_off(kv));
    a.sel.union_count = reinterpret_cast<int32_t*>(union_base + union_count_off(kv));
    a.dec.mask = a.sel.union_mask;
    a.dec.per_head = 0;
    a.dec.max_sel = kv->max_pages;  // the union rows' stride
    a.n_sel = (int)units;
  }
  a.sel.meta_refresh = static_cast<unsigned char*>(meta);
  if (k_new) {
    a.sel.k_new = k_new;
    a.sel.v_new = v_new;
    a.sel.k_dst = const_cast<void*>(kv->k);
    a.sel.v_dst = const_cast<void*>(kv->v);
  }
  a.queue = reinterpret_cast<uint32_t*>(w + kQueueStep);
  a.sel.hold_flag_of = hold_flag_of;
  a.flag_spin_limit = flag_spin_limit;
  // few units (one layer at batch 1, say): one thread-block cluster per unit;
  // the flag-wait test needs the persistent kernel (it exercises its flags)
  const int C = (per_head || hold_flag_of) ? 0 : step_cluster_size((int)units, plan.splits, sm);
  if (C > 0 && plan.fine_unit0 == units) {
    StepArgs c = a;
    c.sel.splits = C;
    c.n_score = (int)(units * C);
    c.n_dec = (int)plan.items;
    if (launch_step_cluster(c, C, (cudaStream_t)stream) == cudaSuccess) return SA_OK;
    cudaGetLastError();  // the cluster shape could not be launched here: use the persistent kernel
  }
  const long long n_score = kv_units * a.sel.splits, n_dec = plan.items;
  if (n_score + a.n_sel + n_dec > 0x7fffffffLL) return SA_ERR_UNSUPPORTED;
  a.n_score = (int)n_score;
  a.n_dec = (int)n_dec;
  return launched(launch_step(a, (cudaStream_t)stream));
}

sa_status sparse_attn_decode_step(const sa_kv_desc* kv, void* meta, sa_score_rule rule,
                                  const void* q, int32_t n_q_heads, const sa_budget* budget,
                                  int32_t max_sel, float scale, int32_t* sel_idx,
                                  int32_t* sel_count, float* out, float* lse, void* ws,
                                  size_t ws_bytes, void* stream) {
  return decode_step(kv, meta, rule, q, n_q_heads, nullptr, nullptr, budget, max_sel, scale, sel_idx,
                     sel_count, out, false, lse, false, ws, ws_bytes, stream);
}

sa_status sparse_attn_decode_step_per_head(const sa_kv_desc* kv, void* meta, sa_score_rule rule,
                                           const void* q, int32_t n_q_heads, const sa_budget* budget,
                                           int32_t max_sel, float scale, int32_t* sel_idx,
                                           int32_t* sel_count, float* out, float* lse, void* ws,
                                           size_t ws_bytes, void* stream) {
  return decode_step(kv, meta, rule, q, n_q_heads, nullptr, nullptr, budget, max_sel, scale, sel_idx,
                     sel_count, out, false, lse, true, ws, ws_bytes, stream);
}

sa_status sparse_attn_decode_step_append(const sa_kv_desc* kv, void* meta, sa_score_rule rule,
                                         const void* q, int32_t n_q_heads, const void* k_new,
                                         const void* v_new, const sa_budget* budget,
                                         int32_t max_sel, float scale, int32_t* sel_idx,
                                         int32_t* sel_count, void* out, sa_out_dtype out_dtype,
                                         float* lse, void* ws, size_t ws_bytes, void* stream) {
  if (!k_new || !v_new || !aligned(k_new, 8) || !aligned(v_new, 8)) return SA_ERR_INVALID;
  if (out_dtype != SA_OUT_F32 && out_dtype != SA_OUT_BF16) return SA_ERR_INVALID;
  return decode_step(kv, meta, rule, q, n_q_heads, k_new, v_new, budget, max_sel, scale, sel_idx,
                     sel_count, out, out_dtype == SA_OUT_BF16, lse, false, ws, ws_bytes, stream);
}

sa_status sparse_attn_decode_step_wait_test(const sa_kv_desc* kv, void* meta, sa_score_rule rule,
                                            const void* q, int32_t n_q_heads, const sa_budget* budget,
                                            int32_t max_sel, float scale, int32_t* sel_idx,
                                            int32_t* sel_count, float* out, float* lse,
                                            int32_t held_unit, uint32_t flag_spin_limit, void* ws,
                                            size_t ws_bytes, void* stream) {
  const long long units = kv ? (long long)kv->batch * kv->n_kv_heads : 0;
  if (held_unit < 0 || held_unit >= units || flag_spin_limit < 1) return SA_ERR_INVALID;
  return decode_step(kv, meta, rule, q, n_q_heads, nullptr, nullptr, budget, max_sel, scale, sel_idx,
                     sel_count, out, false, lse, false, ws, ws_bytes, stream, held_unit + 1,
                     flag_spin_limit);
}

sa_status sparse_attn_route(const sa_kv_desc* kv, const void* meta, sa_score_rule rule,
                            const void* q, int32_t n_q_heads, int32_t n_q_rows, int32_t q_pos0,
                            int32_t tile_rows, int32_t k, int32_t rho, float quantile,
                            const float* tau, int32_t* kv_idx, int32_t* kv_count, float* sigma,
                            float* sigma_bar, uint8_t* triggered, float* tau_out, void* ws,
                            size_t ws_bytes, void* stream) {
  sa_status s = check_kv(kv);
  if (s != SA_OK) return s;
  int G;
  if ((s = check_group(kv, n_q_heads, &G)) != SA_OK) return s;
  if (rule != SA_SCORE_ENVELOPE && rule != SA_SCORE_CENTROID) return SA_ERR_INVALID;
  if (!meta || !aligned(meta, 16) || !q || !aligned(q, 16)) return SA_ERR_INVALID;
  if (!kv_idx || !kv_count || !sigma || !sigma_bar || !triggered) return SA_ERR_INVALID;
  if (kv->batch != 1 || kv->page_size == 0) return SA_ERR_INVALID;
  if (n_q_rows < 1 || tile_rows < 1 || k < 1 || rho < 1 || q_pos0 < 0) return SA_ERR_INVALID;
  if (!(quantile >= 0.f && quantile <= 1.f)) return SA_ERR_INVALID;
  if (!aligned(kv_idx, 4) || !aligned(kv_count, 4) || !aligned(sigma, 4) || !aligned(sigma_bar, 4) ||
      (tau && !aligned(tau, 4)) || (tau_out && !aligned(tau_out, 4)))
    return SA_ERR_INVALID;
  const long long T = ((long long)n_q_rows + tile_rows - 1) / tile_rows;
  const long long W = (long long)rho * k;
  if (T > kMaxRouteTiles || W > kMaxRouteList || (long long)k + 1 > kMaxRouteList + 1)
    return SA_ERR_UNSUPPORTED;
  if (kv->max_pages > kMaxSelectPages) return SA_ERR_UNSUPPORTED;
  const long long units = T * kv->n_kv_heads;
  if (units > kMaxUnits) return SA_ERR_UNSUPPORTED;
  const unsigned long long meta_rows = (unsigned long long)kv->n_kv_heads * kv->max_pages;
  if (meta_rows > 0x7fffffffULL) return SA_ERR_UNSUPPORTED;
  const size_t need = kScratch + route_ws_bytes((int)T, kv->n_kv_heads, kv->max_pages, (int)W);
  if ((s = check_ws(ws, ws_bytes, need)) != SA_OK) return s;

  RouteArgs a{};  // every field zero unless set below
  const bool env = rule == SA_SCORE_ENVELOPE;
  if (!encode_tmap_2d(&a.tmap_meta, meta, meta_rows, kMetaBytes,
                      env ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                      env ? 2 : 4, 16))
    return SA_ERR_CUDA;
  if (!encode_tmap_2d(&a.tmap_meta_tc, meta, meta_rows, kMetaBytes,
                      env ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                      env ? 2 : 4, 128))
    return SA_ERR_CUDA;
  a.kv = view(kv);
  a.rule = (int)rule;
  a.q = q;
  a.Hq = n_q_heads;
  a.G = G;
  a.n_rows = n_q_rows;
  a.q_pos0 = q_pos0;
  a.tile_rows = tile_rows;
  a.n_tiles = (int)T;
  a.k = k;
  a.rho = rho;
  a.W = (int)W;
  a.nsplit = route_splits(tile_rows * G);
  a.quantile = quantile;
  a.tau_in = tau;
  a.kv_idx = kv_idx;
  a.kv_count = kv_count;
  a.sigma = sigma;
  a.sigma_bar = sigma_bar;
  a.triggered = triggered;
  a.tau_out = tau_out;
  char* scratch = reinterpret_cast<char*>(ws) + kScratch;
  const size_t tg = (size_t)units;
  const size_t keys_bytes = align256(tg * kv->max_pages * 4);
  a.ws_keys = reinterpret_cast<uint32_t*>(scratch);
  a.dec_scores = nullptr;  // query tiles: the keys above, not decode group scores
  a.dec_stride = 0;
  a.ws_sigma = reinterpret_cast<double*>(scratch + keys_bytes);
  a.ws_elig = reinterpret_cast<int32_t*>(scratch + keys_bytes + align256(tg * 8));
  a.ws_count = reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(ws) + 256);
  a.ws_final = reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(ws) + kQueueRoute);
  a.status = reinterpret_cast<int*>(ws);
  // tile-score keys start at 0 (below every score) for the atomicMax merge
  if (cudaMemsetAsync(a.ws_keys, 0, tg * kv->max_pages * 4, (cudaStream_t)stream) != cudaSuccess) {
    cudaGetLastError();
    return SA_ERR_CUDA;
  }
  return launched(launch_route(a, (cudaStream_t)stream));
}

sa_status sparse_attn_route_decode(const sa_kv_desc* kv, const void* meta, sa_score_rule rule,
                                   const void* q, int32_t n_q_heads, int32_t k, int32_t rho,
                                   float quantile, const float* tau, int32_t* kv_idx,
                                   int32_t* kv_count, float* sigma, float* sigma_bar,
                                   uint8_t* triggered, float* tau_out, void* ws, size_t ws_bytes,
                                   void* stream) {
  if (!kv || kv->page_size <= 0) return kv ? SA_ERR_UNSUPPORTED : SA_ERR_INVALID;
  if (k < 1 || rho < 1) return SA_ERR_INVALID;
  if (!(quantile >= 0.f && quantile <= 1.f)) return SA_ERR_INVALID;
  if (!kv_idx || !kv_count || !sigma || !sigma_bar || !triggered) return SA_ERR_INVALID;
  if (!aligned(sigma, 4) || !aligned(sigma_bar, 4) || (tau && !aligned(tau, 4)) ||
      (tau_out && !aligned(tau_out, 4)))
    return SA_ERR_INVALID;
  const long long W = (long long)rho * k;
  if (W > kMaxRouteList || (long long)k + 1 > kMaxRouteList + 1) return SA_ERR_UNSUPPORTED;
  if (kv->batch > kMaxRouteTiles) return SA_ERR_UNSUPPORTED;
  // the scores: the decode scoring items in score-only mode
  int G;
  const sa_budget dummy{SA_BUDGET_TOPK, 1, 0.f, 0, 0, 0, 0};
  sa_status s = check_select(kv, meta, rule, q, n_q_heads, &dummy, (int)W, kv_idx, kv_count, nullptr, &G);
  if (s != SA_OK) return s;
  const long long units = (long long)kv->batch * kv->n_kv_heads;
  const size_t sel_bytes = select_scratch(kv);
  const size_t need = kScratch + sel_bytes + route_decode_ws_bytes(units);
  if ((s = check_ws(ws, ws_bytes, need)) != SA_OK) return s;
  if (route_decode_smem_bytes(kv->max_pages, (int)W, k, kv->batch, kv->n_kv_heads) > 227 * 1024) return SA_ERR_UNSUPPORTED;
  SelectArgs sa_{};  // every field zero unless set below
  if (!fill_select(&sa_, kv, meta, rule, q, n_q_heads, G, &dummy, (int)W, kv_idx, kv_count, nullptr, ws))
    return SA_ERR_CUDA;
  sa_.score_only = 1;
  sa_.ws_queue = reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(ws) + kQueueSelect);
  if ((s = launched(launch_select(sa_, (cudaStream_t)stream))) != SA_OK) return s;

  // the router's selection, sigma, quantile, triggers and lists over those scores
  RouteArgs a{};  // every field zero unless set below
  a.kv = view(kv);
  a.rule = (int)rule;
  a.q = q;
  a.Hq = n_q_heads;
  a.G = G;
  a.n_rows = kv->batch;
  a.q_pos0 = 0;
  a.tile_rows = 1;
  a.n_tiles = kv->batch;
  a.k = k;
  a.rho = rho;
  a.W = (int)W;
  a.nsplit = 1;
  a.quantile = quantile;
  a.tau_in = tau;
  a.kv_idx = kv_idx;
  a.kv_count = kv_count;
  a.sigma = sigma;
  a.sigma_bar = sigma_bar;
  a.triggered = triggered;
  a.tau_out = tau_out;
  a.ws_keys = nullptr;
  a.dec_scores = sa_.ws_scores;
  a.dec_stride = score_stride(kv);
  char* rbase = reinterpret_cast<char*>(ws) + kScratch + sel_bytes;
  a.ws_sigma = reinterpret_cast<double*>(rbase);
  a.ws_elig = reinterpret_cast<int32_t*>(rbase + align256((size_t)units * 8));
  a.ws_count = reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(ws) + 256);
  a.ws_final = reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(ws) + kQueueRoute);
  a.status = reinterpret_cast<int*>(ws);
  return launched(launch_route_decode(a, (cudaStream_t)stream));
}

sa_status sparse_attn_route_decode_step(const sa_kv_desc* kv, void* meta, sa_score_rule rule,
                                        const void* q, int32_t n_q_heads, int32_t k, int32_t rho,
                                        float quantile, const float* tau, float scale, int32_t* kv_idx,
                                        int32_t* kv_count, float* sigma, float* sigma_bar,
                                        uint8_t* triggered, float* tau_out, float* out, float* lse,
                                        void* ws, size_t ws_bytes, void* stream) {
  if (!kv || kv->page_size <= 0) return kv ? SA_ERR_UNSUPPORTED : SA_ERR_INVALID;
  if (k < 1 || rho < 1) return SA_ERR_INVALID;
  if (!(quantile >= 0.f && quantile <= 1.f)) return SA_ERR_INVALID;
  if (!kv_idx || !kv_count || !sigma || !sigma_bar || !triggered) return SA_ERR_INVALID;
  if (!aligned(sigma, 4) || !aligned(sigma_bar, 4) || (tau && !aligned(tau, 4)) ||
      (tau_out && !aligned(tau_out, 4)))
    return SA_ERR_INVALID;
  if (!out || !aligned(out, 16) || (lse && !aligned(lse, 4))) return SA_ERR_INVALID;
  if (!std::isfinite(scale)) return SA_ERR_INVALID;
  const long long W = (long long)rho * k;
  if (W > kMaxRouteList || (long long)k + 1 > kMaxRouteList + 1) return SA_ERR_UNSUPPORTED;
  if (kv->batch > kMaxRouteTiles) return SA_ERR_UNSUPPORTED;
  int G;
  const sa_budget dummy{SA_BUDGET_TOPK, 1, 0.f, 0, 0, 0, 0};
  sa_status s = check_select(kv, meta, rule, q, n_q_heads, &dummy, (int)W, kv_idx, kv_count, nullptr, &G);
  if (s != SA_OK) return s;
  const long long units = (long long)kv->batch * kv->n_kv_heads;
  if (2 * units > kMaxUnits) return SA_ERR_UNSUPPORTED;  // unit flags + split counters
  const unsigned long long kv_rows = (unsigned long long)kv->batch * kv->n_kv_heads * kv->cap_tokens;
  if (kv_rows > 0x7fffffffULL) return SA_ERR_UNSUPPORTED;
  if (route_decode_smem_bytes(kv->max_pages, (int)W, k, kv->batch, kv->n_kv_heads) >
      (size_t)(kv->max_pages * 8 > 65536 ? kv->max_pages * 8 : 65536))
    return SA_ERR_UNSUPPORTED;  // the selection's keys and candidates live in the step's ring
  if (step_smem_bytes(kv->max_pages, (int)W, false) > 227 * 1024) return SA_ERR_UNSUPPORTED;
  // the top-k windows and the expansion windows get their own splits
  const int sm = device_sm_count();
  const int sub = kv->page_size / 16;
  const int sb = decode_plan((int)units, k * sub, sm).splits;
  // expansion windows: split for the units expected to trigger (the rows
  // below the q-quantile; every unit when the threshold is given), so the
  // last items of the launch stay short
  long long trig_units = units;
  if (tau == nullptr) {
    const long long rows = (long long)std::ceil((double)quantile * kv->batch);
    trig_units = (rows < 1 ? 1 : rows) * kv->n_kv_heads;
    if (trig_units > units) trig_units = units;
  }
  const int se = W > k ? decode_plan((int)trig_units, (int)(W - k) * sub, sm).splits : 0;
  DecodePlan plan{sb + se, (int)units, sb + se, units * (sb + se)};
  const size_t sel_bytes = select_scratch(kv);
  const size_t rt_bytes = route_decode_ws_bytes(units);
  // partial slots: sb + se per unit and the unit's merged top-k window
  const size_t need = kScratch + sel_bytes + rt_bytes +
                      decode_scratch(DecodePlan{sb + se, (int)units, sb + se, units * (sb + se + 1)});
  if ((s = check_ws(ws, ws_bytes, need)) != SA_OK) return s;

  RouteStepArgs ra{};  // every field zero unless set below
  StepArgs& a = ra.st;
  char* w = reinterpret_cast<char*>(ws);
  if (!fill_select(&a.sel, kv, meta, rule, q, n_q_heads, G, &dummy, (int)W, kv_idx, kv_count, nullptr, ws) ||
      !fill_decode(&a.dec, kv, q, n_q_heads, G, scale, kv_idx, kv_count, (int)W, out, lse,
                   reinterpret_cast<float*>(w + kScratch + sel_bytes + rt_bytes),
                   reinterpret_cast<uint32_t*>(w + 256) + units, reinterpret_cast<int*>(ws), plan))
    return SA_ERR_CUDA;
  a.sel.meta_refresh = static_cast<unsigned char*>(meta);
  a.dec.route_k = k;
  a.dec.route_w = (int)W;
  a.dec.route_base_splits = sb;
  a.queue = reinterpret_cast<uint32_t*>(w + kQueueStep);
  RouteArgs& r = ra.route;
  r.kv = view(kv);
  r.rule = (int)rule;
  r.q = q;
  r.Hq = n_q_heads;
  r.G = G;
  r.n_rows = kv->batch;
  r.q_pos0 = 0;
  r.tile_rows = 1;
  r.n_tiles = kv->batch;
  r.k = k;
  r.rho = rho;
  r.W = (int)W;
  r.nsplit = 1;
  r.quantile = quantile;
  r.tau_in = tau;
  r.kv_idx = kv_idx;
  r.kv_count = kv_count;
  r.sigma = sigma;
  r.sigma_bar = sigma_bar;
  r.triggered = triggered;
  r.tau_out = tau_out;
  r.ws_keys = nullptr;
  r.dec_scores = a.sel.ws_scores;
  r.dec_stride = score_stride(kv);
  char* rbase = w + kScratch + sel_bytes;
  r.ws_sigma = reinterpret_cast<double*>(rbase);
  r.ws_elig = reinterpret_cast<int32_t*>(rbase + align256((size_t)units * 8));
  r.trig_list = reinterpret_cast<int4*>(rbase + align256((size_t)units * 8) + align256((size_t)units * 4));
  r.status = reinterpret_cast<int*>(ws);
  ra.routed = reinterpret_cast<uint32_t*>(w + kQueueRouteStep);
  const long long n_score = units * a.sel.splits;
  if (n_score + plan.items > 0x7fffffffLL) return SA_ERR_UNSUPPORTED;
  a.n_score = (int)n_score;
  a.n_dec = (int)plan.items;
  ra.n_base = (int)(units * sb);
  return launched(launch_route_step(ra, (cudaStream_t)stream));
}

sa_status sparse_attn_get_device_status(void* ws, sa_status* host_out, void* stream) {
  if (!ws || !host_out || !aligned(ws, 256)) return SA_ERR_INVALID;
  int v = 0;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaMemcpyAsync(&v, ws, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess) {
    cudaGetLastError();
    return SA_ERR_CUDA;
  }
  if (cudaStreamSynchronize(st) != cudaSuccess) {
    cudaGetLastError();
    return SA_ERR_CUDA;
  }
  if (cudaMemsetAsync(ws, 0, sizeof(int), st) != cudaSuccess) {
    cudaGetLastError();
    return SA_ERR_CUDA;
  }
  *host_out = (sa_status)v;
  return SA_OK;
}

const char* sparse_attn_status_string(sa_status s) {
  switch (s) {
    case SA_OK: return "ok";
    case SA_ERR_INVALID: return "invalid argument";
    case SA_ERR_UNSUPPORTED: return "unsupported shape or option";
    case SA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case SA_ERR_CUDA: return "CUDA launch or runtime error";
    case SA_ERR_TIMEOUT: return "bounded device wait timed out";
    case SA_ERR_DEVICE_CHECK: return "device-side range check failed";
  }
  return "unknown status";
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode with library-owned scratch, for callers that cannot allocate device
// memory where they call us (see sparse_attn_decode_static in sparse_attn.h).
// The scratch is this file's device array; host code only ever uses the
// address that cudaGetSymbolAddress returns for the current device.
namespace sa {
namespace {
constexpr size_t kStaticScratchBytes = (size_t)8 << 20;
constexpr int kStaticMaxUnits = 4096;
constexpr size_t kStaticPartOff = 256 + 4 * (size_t)kStaticMaxUnits;  // after status/queues/counters
static_assert(kStaticPartOff % 256 == 0, "partials must stay 256-byte aligned");
}  // namespace
}  // namespace sa

static __device__ __align__(256) unsigned char g_decode_scratch[sa::kStaticScratchBytes];

namespace sa {
namespace {
// Device address of g_decode_scratch on the current device, looked up once
// per device.  Host threads may race on a device's first call: each slot is
// atomic, and every racer stores the same address.
sa_status static_scratch(unsigned char** out) {
  static std::atomic<unsigned char*> addr[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return SA_ERR_CUDA;
  }
  unsigned char* a = addr[dev].load(std::memory_order_acquire);
  if (!a) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return SA_ERR_CUDA;
    }
    a = static_cast<unsigned char*>(p);
    addr[dev].store(a, std::memory_order_release);
  }
  *out = a;
  return SA_OK;
}
}  // namespace
}  // namespace sa

extern "C" sa_status sparse_attn_decode_static(const sa_kv_desc* kv, const void* q, int32_t n_q_heads,
                                               int32_t n_q_rows, int32_t q_pos0, int32_t tile_rows,
                                               float scale, const int32_t* idx, const int32_t* count,
                                               int32_t max_sel, float* out, float* lse,
                                               int32_t* device_status, void* stream) {
  sa_status s = check_kv(kv);
  if (s != SA_OK) return s;
  int G;
  if ((s = check_group(kv, n_q_heads, &G)) != SA_OK) return s;
  if (!q || !aligned(q, 16) || !idx || !count || !aligned(idx, 4) || !aligned(count, 4))
    return SA_ERR_INVALID;
  if (!out || !aligned(out, 16) || (lse && !aligned(lse, 4))) return SA_ERR_INVALID;
  if (device_status && !aligned(device_status, 4)) return SA_ERR_INVALID;
  if (max_sel < 1 || tile_rows < 1 || n_q_rows < 1) return SA_ERR_INVALID;
  if (!std::isfinite(scale)) return SA_ERR_INVALID;
  if (tile_rows == 1) {
    if (n_q_rows != kv->batch) return SA_ERR_INVALID;
  } else {
    if (kv->batch != 1 || kv->page_size == 0) return SA_ERR_INVALID;
    return SA_ERR_UNSUPPORTED;
  }
  if (kv->page_size == 0 && max_sel > kMaxChunkSel) return SA_ERR_UNSUPPORTED;
  const long long units = (long long)n_q_rows * kv->n_kv_heads;
  if (units > kStaticMaxUnits) return SA_ERR_WORKSPACE;  // beyond the built-in scratch
  const unsigned long long kv_rows = (unsigned long long)kv->batch * kv->n_kv_heads * kv->cap_tokens;
  if (kv_rows > 0x7fffffffULL) return SA_ERR_UNSUPPORTED;
  const DecodePlan plan = decode_plan((int)units, max_tiles_per_unit(kv, max_sel), device_sm_count());
  if (kStaticPartOff + decode_scratch(plan) > kStaticScratchBytes) return SA_ERR_WORKSPACE;

  unsigned char* scratch = nullptr;
  if ((s = static_scratch(&scratch)) != SA_OK) return s;
  DecodeArgs a{};  // every field zero unless set below
  if (!encode_tmap_2d(&a.tmap_k, kv->k, kv_rows, kHeadDim * 2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 16) ||
      !encode_tmap_2d(&a.tmap_v, kv->v, kv_rows, kHeadDim * 2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 16))
    return SA_ERR_CUDA;
  // status word, queue and the counters of this call's units start at zero
  if (cudaMemsetAsync(scratch, 0, 256 + 4 * (size_t)units, (cudaStream_t)stream) != cudaSuccess) {
    cudaGetLastError();
    return SA_ERR_CUDA;
  }
  a.kv = view(kv);
  a.q = q;
  a.Hq = n_q_heads;
  a.G = G;
  a.n_rows = n_q_rows;
  a.q_pos0 = q_pos0;
  a.tile_rows = tile_rows;
  a.scale_log2 = scale * kLog2e;
  a.idx = idx;
  a.count = count;
  a.max_sel = max_sel;
  a.out = out;
  a.out_bf16 = nullptr;
  a.per_head = 0;
  a.lse = lse;
  a.ws_part = reinterpret_cast<float*>(scratch + kStaticPartOff);
  a.ws_count = reinterpret_cast<uint32_t*>(scratch + 256);
  a.ws_queue = reinterpret_cast<uint32_t*>(scratch + kQueueDecode);
  a.status = device_status ? reinterpret_cast<int*>(device_status) : reinterpret_cast<int*>(scratch);
  a.splits = plan.splits;
  a.fine_unit0 = plan.fine_unit0;
  a.splits_fine = plan.splits_fine;
  a.n_items = (int)plan.items;
  return launched(launch_decode(a, (cudaStream_t)stream));
}
