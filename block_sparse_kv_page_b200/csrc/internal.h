// Internal launch interface between the C-ABI entry points (api.cu) and the
// kernel files.  Host-only declarations; not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "sparse_attn.h"

namespace sa {

// Plain copy of the cache view, passed to kernels by value.
struct KvView {
  int B, Hkv, page_size;      // page_size 0 = variable chunks
  long long cap;
  const void* k;
  const void* v;
  const int32_t* seq_len;
  const int32_t* chunk_off;   // [B][max_pages + 1]
  const int32_t* n_chunks;
  int max_pages;
};

// Workspace regions (byte offsets from ws, each 256-aligned).
struct WsLayout {
  size_t status;        // int32 status word
  size_t sel_count;     // uint32 [units] last-CTA counters of select
  size_t dec_count;     // uint32 [rows * Hkv] last-CTA counters of decode
  size_t sel_scores;    // float [units][max_pages] group scores
  size_t dec_part;      // float partials [slots][G][kHeadDim + 2]
  size_t route;         // router scratch
  size_t total;
  int dec_slots;        // partial slots available (units * splits bound)
};

int device_sm_count();
// Encode a 2D tiled tensor map: `rows` rows of `row_bytes` bytes at `base`,
// element type `dt` of `elem_bytes`, box = box_rows x 128 bytes, 128B swizzle.
bool encode_tmap_2d(CUtensorMap* map, const void* base, unsigned long long rows, int row_bytes,
                    CUtensorMapDataType dt, int elem_bytes, int box_rows);
// Opt a kernel into `bytes` of dynamic shared memory on the current device
// (cached per device and kernel, so repeated launches skip the driver call).
cudaError_t set_smem_attr(const void* func, size_t bytes);

// Launch with programmatic stream serialisation (programmatic dependent
// launch): the grid may be scheduled while the previous kernel of the stream
// drains.  Every kernel launched this way calls grid_dep_wait() before its
// first global access and grid_dep_trigger() once it has no work left.
template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kernel)(Params...), unsigned grid, unsigned block, size_t smem,
                       cudaStream_t st, const Args&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}
int select_splits(int units, int max_pages, int sm_count);
WsLayout workspace_layout(const sa_kv_desc* kv, int n_q_heads, int n_q_rows, int max_sel,
                          int sm_count);

cudaError_t launch_build_meta(const KvView& kv, int rule, int first_token, void* meta,
                              int* status, cudaStream_t st);

// Work unit u of a selection or decode: sequence b, KV head g (its K/V and
// metadata rows belong to kv unit b * Hkv + g), and the query heads
// [h0, h0 + n_heads) that share the unit's page set: the G heads of KV head g,
// or a single query head when every query head selects its own pages.
struct UnitMap {
  int b, g, kvu, h0, n_heads;
};
// PER_HEAD is a compile-time choice: the shared-selection kernels keep their
// plain (sequence, KV head) indexing.
template <bool PER_HEAD>
__host__ __device__ inline UnitMap unit_map(int u, int Hkv, int Hq, int G) {
  UnitMap m;
  if (PER_HEAD) {
    m.b = u / Hq;
    m.h0 = u - m.b * Hq;
    m.g = m.h0 / G;
    m.n_heads = 1;
  } else {
    m.b = u / Hkv;
    m.g = u - m.b * Hkv;
    m.h0 = m.g * G;
    m.n_heads = G;
  }
  m.kvu = m.b * Hkv + m.g;
  return m;
}

struct SelectArgs {
  CUtensorMap tmap_meta;      // metadata rows [B*Hkv*max_pages][512 B], boxes 16 x 128 B, 128B swizzle
  KvView kv;
  const void* meta;
  int rule;
  const void* q;
  int Hq, G;
  int budget_kind, top_k, topk_val, bos, eos, token_budget;
  double ratio;
  int per_head;               // 1: one unit per (sequence, query head), else per (sequence, KV head)
  int score_only;             // 1: group scores to ws_scores only (no selection, sel_* unused)
  int max_sel;
  int32_t* sel_idx;
  int32_t* sel_count;
  float* scores_out;
  float* ws_scores;           // [units][ws_stride] group scores
  int ws_stride;              // max_pages rounded up to a multiple of 4 (16-byte rows)
  uint32_t* ws_count;
  uint32_t* ws_queue;         // [2] persistent-grid item queue (head, finished CTAs)
  int* status;
  int splits;
  unsigned char* meta_refresh;  // decode step: writable metadata (same array as meta)
  // decode step with append (all null otherwise): the newest token's key and
  // value, bf16 [B][Hkv][128], stored into the cache (k_dst / v_dst = the
  // cache arrays) at row seq_len[b] - 1
  const void* k_new;
  const void* v_new;
  void* k_dst;
  void* v_dst;
  // decode step, test of the bounded wait only: 1 + the unit whose selection
  // flag is never published (its decode items run their wait out and report
  // SA_ERR_TIMEOUT); 0 = none
  int hold_flag_of;
  // per-query-head decode step: scoring items per (sequence, KV head) count
  // their completions here [B * Hkv]; the per-head selection items wait for
  // the count to reach `splits`, then count themselves in kv_selected; the
  // last of a KV head's G builds the union of their page sets (union_idx /
  // union_mask [B * Hkv][max_pages], union_count) for its decode items
  uint32_t* kv_scored;
  uint32_t* kv_selected;
  int32_t* union_idx;
  uint8_t* union_mask;
  int32_t* union_count;
};
cudaError_t launch_select(const SelectArgs& a, cudaStream_t st);

struct DecodeArgs {
  CUtensorMap tmap_k;         // K rows [B*Hkv*cap][128 bf16], boxes 16 x 64, 128B swizzle
  CUtensorMap tmap_v;         // V, same geometry
  KvView kv;
  const void* q;
  int Hq, G;
  int per_head;               // 1: one unit per (row, query head), else per (row, KV head)
  int n_rows, q_pos0, tile_rows;
  float scale_log2;           // scale * log2(e)
  const int32_t* idx;
  const int32_t* count;
  const uint8_t* mask;        // nullable [units][max_sel]: bit j = query head h0 + j attends the entry
  int max_sel;
  float* out;
  __nv_bfloat16* out_bf16;    // non-null: the output goes here, rounded to bf16, instead of `out`
  float* lse;
  float* ws_part;
  uint32_t* ws_count;
  uint32_t* ws_queue;
  int* status;
  int splits;                 // splits of units [0, fine_unit0)
  int fine_unit0;             // units from here on (the end of the queue) use splits_fine
  int splits_fine;
  int n_items;                // fine_unit0 * splits + (units - fine_unit0) * splits_fine
  // routed decode step (0 = off): the units' lists are in rank order; splits
  // [0, route_base_splits) cover list entries [0, route_k) (the top k, decoded
  // as soon as the unit is selected), the others entries [route_k, route_w)
  // (the expansion, decoded once the trigger is known); each clipped to the
  // unit's count
  int route_k, route_w, route_base_splits;
};
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st);

// Split plan of a decode launch: `splits` ranges per unit, except that the
// units at the end of the item queue get `splits_fine` (finer) ranges so the
// last wave of items is short and the launch drains quickly.
struct DecodePlan {
  int splits, fine_unit0, splits_fine;
  long long items;            // work items = partial slots
};
DecodePlan decode_plan(int units, int max_tiles, int sm_count);

struct RouteArgs {
  CUtensorMap tmap_meta;      // block metadata rows [Hkv*max_pages][512 B], boxes 16 x 128 B, 128B swizzle
  CUtensorMap tmap_meta_tc;   // the same rows, boxes 128 x 128 B (tensor-core M tiles)
  KvView kv;
  int rule;
  const void* q;              // bf16 [n_rows][Hq][128]
  int Hq, G;
  int n_rows, q_pos0, tile_rows, n_tiles;
  int k, rho, W;              // W = rho * k: list width
  int nsplit;                 // query-vector splits per (tile, KV head)
  float quantile;
  const float* tau_in;
  int32_t* kv_idx;
  int32_t* kv_count;
  float* sigma;
  float* sigma_bar;
  uint8_t* triggered;
  float* tau_out;
  uint32_t* ws_keys;          // [n_tiles][Hkv][max_pages] tile-score keys (zeroed before launch)
  const float* dec_scores;    // decode router: group scores [B*Hkv][dec_stride] (the tiles are
  int dec_stride;             // the sequences, one query row each); null for query tiles
  double* ws_sigma;           // [n_tiles][Hkv]
  int32_t* ws_elig;           // [n_tiles][Hkv] eligible block counts
  uint32_t* ws_count;         // [n_tiles * Hkv] split counters (left zero)
  uint32_t* ws_final;         // [1] finalize counter (left zero)
  int4* trig_list;            // routed decode step: the triggered (tile, KV head) pairs
                              // {tile x Hkv + head, list count, sequence length, 0}; else null
  int* status;
};
// One decode step in one launch: newest-page metadata refresh, scoring,
// selection and decode.  Scoring items come first in the queue; decode item j
// of unit u waits (bounded) for u's selection flag.
struct StepArgs {
  SelectArgs sel;             // meta_refresh set, ws_count = unit flags [units]
  DecodeArgs dec;             // idx/count = sel outputs, ws_count = split counters [units]
  uint32_t* queue;            // [2] item queue (head, finished CTAs)
  int n_score, n_dec;         // items of each kind
  int n_sel;                  // per-query-head step: selection items (one per (sequence, query head))
  uint32_t flag_spin_limit;   // polls of a unit-flag wait before SA_ERR_TIMEOUT; 0 = default (~1 s)
};
cudaError_t launch_step(const StepArgs& a, cudaStream_t st);

// The router applied to decode, in one launch: scoring items, each unit's
// rank-order selection and sigma (the last scoring CTA of the unit), the
// batch's quantile and triggers (the last unit), and the decode of every
// unit's top k (as soon as the unit is selected) and of the expansion of the
// triggered units (once the triggers are known).
struct RouteStepArgs {
  StepArgs st;                // sel: score-only scoring; dec: route_k/w set, idx/count = the lists
  RouteArgs route;            // dec_scores = the group scores; tiles = the sequences
  uint32_t* routed;           // [2]: units selected so far; 1 + the triggered units, once published
  int n_base;                 // decode items of the top-k windows (unit order), then the
                              // expansion windows of the triggered units (route.trig_list order)
};
cudaError_t launch_route_step(const RouteStepArgs& a, cudaStream_t st);
// Few units: one cluster of C CTAs per unit (sel.splits must be C).
int step_cluster_size(int units, int dec_splits, int sm_count);
cudaError_t launch_step_cluster(const StepArgs& a, int C, cudaStream_t st);
size_t step_smem_bytes(int max_pages, int max_sel, bool chunks);

struct TileAttnArgs {
  CUtensorMap tmap_k;         // K rows [Hkv*cap][128 bf16], boxes 64 x 64, 128B swizzle
  CUtensorMap tmap_v;         // V, same geometry (read MN-major by the PV MMA)
  KvView kv;                  // batch 1, 64-token blocks
  const void* q;              // bf16 [n_rows][Hq][128]
  int Hq, G;
  int n_rows, q_pos0, tile_rows, n_tiles, n_mchunks;
  float scale_log2;
  const int32_t* idx;         // [n_tiles][Hkv][max_sel], -1 = sentinel
  const int32_t* count;       // [n_tiles][Hkv]
  int max_sel;
  float* out;
  float* lse;
  int* status;
};
// Tile attention on tcgen05 (CTA = 128 query vectors of a (tile, KV head)).
cudaError_t launch_tile_attn_tc(const TileAttnArgs& a, cudaStream_t st);
int tile_attn_tc_mchunks(int vectors_per_tile);

cudaError_t launch_route(const RouteArgs& a, cudaStream_t st);
// Decode router tail: one CTA per (sequence, KV head) over dec_scores.
cudaError_t launch_route_decode(const RouteArgs& a, cudaStream_t st);
size_t route_decode_smem_bytes(int max_pages, int W, int k, int n_tiles, int Hkv);
// Router scratch: keys, lists, sigma and eligible counts for n_tiles x Hkv.
size_t route_ws_bytes(int n_tiles, int Hkv, int max_pages, int W);
int route_splits(int vectors_per_tile);

}  // namespace sa
