// One decode step in one launch: newest-page metadata refresh, page scoring,
// budgeted top-k selection and sparse paged flash-decode.
//
// "Sparse Attention for Web Agents -- Offline Replay Records", section "The
// comparison": chunk the cache, score the chunks against the current query,
// keep the best ones and attend only to them.  The three stages are the work
// items of select_item.cuh and decode_item.cuh; this kernel only schedules
// them.
//
// Schedule.  A persistent grid pulls item ids from one atomic counter.  Ids
// [0, n_score) are scoring items (unit, tile range), in unit order; the CTA
// that finishes a unit's last scoring item selects its pages and publishes
// the unit's flag (release).  Ids [n_score, n_score + n_dec) are decode items
// (unit, tile range), also in unit order; the CTA that takes one waits
// (bounded, acquire) for its unit's flag.  Every scoring item has been taken
// by a running CTA before any decode id is handed out and scoring never
// waits, so every flag is eventually published whatever the residency: the
// waits cannot deadlock.  In practice the decode of the first units overlaps
// the scoring of the last ones, which hides the selection tail and the gap
// between launches.
//
// All item kinds share one per-warp TMA ring (same stage count and tile size),
// so one WarpState carries the ring position from item to item.  The last CTA
// out clears the unit flags and split counters and rewinds the queue.
#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.h"
#include "decode_item.cuh"
#include "route_select.cuh"
#include "select_item.cuh"

namespace cg = cooperative_groups;

#ifndef SA_STEP_CTAS_PER_SM
#define SA_STEP_CTAS_PER_SM 3
#endif
// CTAs per cluster of the small-unit decode step (16 needs the non-portable
// cluster size; 8 is portable)
#ifndef SA_STEP_CLUSTER
#define SA_STEP_CLUSTER 16
#endif

namespace sa {
namespace {

static_assert(sel::kWarps == dec::kWarps, "one CTA shape for both item kinds");
static_assert(sel::kStages == dec::kStages && sel::kTileBytes == dec::kTileBytes,
              "both item kinds use the same per-warp ring");

static_assert(sel::kCandOffset + 16 * sel::kWarps * 32 * 8 <= sel::kRingBytes,
              "the routed step's candidates (and their bitonic fallback) fit the ring");
constexpr int kWarps = sel::kWarps;
constexpr int kThreads = kWarps * 32;
constexpr int kStages = sel::kStages;
constexpr int kBarBytes = kWarps * kStages * 8;
constexpr int kTileRefBytes = dec::kMaxItemTiles * (int)sizeof(dec::TileRef);
constexpr uint32_t kFlagSpinLimit = 1u << 22;  // x (load + <= 256 ns sleep): about a second
constexpr size_t kClusterMinSmem = 116 * 1024;  // more than half an SM's shared memory

// Ring, or the selection keys/weights when those are larger.
__host__ __device__ int body_bytes(int max_pages) {
  const int kb = (sel::keys_bytes(max_pages) + 1023) & ~1023;
  return kb > sel::kRingBytes ? kb : sel::kRingBytes;
}

// Wait until a unit's selection is published and return its kept count (the
// flag's low bits); -1 (and SA_ERR_TIMEOUT) after `limit` polls.
SA_DEV int wait_selected(const uint32_t* flag, int* status, uint32_t limit) {
  uint32_t ns = 32;
  for (uint32_t i = 0; i < limit; ++i) {
    const uint32_t v = ld_acquire_u32(flag);
    if (v & sel::kUnitSelected) return (int)(v & ~sel::kUnitSelected);
    __nanosleep(ns);
    if (ns < 256) ns <<= 1;
  }
  flag_status(status, SA_ERR_TIMEOUT);
  return -1;
}

// Wait until *flag is nonzero (acquire) and return it; 0 (and
// SA_ERR_TIMEOUT) after `limit` polls.
SA_DEV uint32_t wait_nonzero(const uint32_t* flag, int* status, uint32_t limit) {
  uint32_t ns = 32;
  for (uint32_t i = 0; i < limit; ++i) {
    const uint32_t v = ld_acquire_u32(flag);
    if (v != 0u) return v;
    __nanosleep(ns);
    if (ns < 256) ns <<= 1;
  }
  flag_status(status, SA_ERR_TIMEOUT);
  return 0u;
}

// Wait until *count reaches `target` (acquire); false (and SA_ERR_TIMEOUT)
// after `limit` polls.
SA_DEV bool wait_count(const uint32_t* count, uint32_t target, int* status, uint32_t limit) {
  uint32_t ns = 32;
  for (uint32_t i = 0; i < limit; ++i) {
    if (ld_acquire_u32(count) >= target) return true;
    __nanosleep(ns);
    if (ns < 256) ns <<= 1;
  }
  flag_status(status, SA_ERR_TIMEOUT);
  return false;
}

// PER_HEAD: units are (sequence, query head), each selecting its own pages.
// Their scores still come from one scoring pass per (sequence, KV head)
// (items [0, n_score) write the G heads' own score rows); items
// [n_score, n_score + n_sel) are the per-head selections, each waiting
// (bounded) until its KV head's scoring items are all done; the last of a KV
// head's G selections builds the union of their page sets with a head mask
// per page and publishes the KV head's flag.  The decode items follow, one
// set per (sequence, KV head) over the union (a page is streamed once for
// every head that kept it; each head attends only its own pages).  Every
// wait is on items handed out earlier that never wait on later ones, so none
// can deadlock.
template <int RULE, bool PER_HEAD>
__global__ void __launch_bounds__(kThreads, SA_STEP_CTAS_PER_SM)
    step_kernel(const __grid_constant__ StepArgs a) {
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint32_t s_hist[512];
  __shared__ uint32_t s_scan[32];
  __shared__ uint32_t s_bc[8];
  __shared__ int s_last, s_item, s_ntiles, s_count, s_ntok;
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int body = body_bytes(a.sel.kv.max_pages);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + body);
  const sel::SelSmem S{base, bars, s_hist, s_scan, s_bc, &s_last};
  const dec::Smem D{base, bars, reinterpret_cast<dec::TileRef*>(base + body + kBarBytes),
                    reinterpret_cast<int*>(base + body + kBarBytes + kTileRefBytes), s_scan, &s_last,
                    &s_ntiles};
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(bars + warp * kStages + s, 1);
    fence_barrier_init();
  }
  if (threadIdx.x == 0) {
    prefetch_tmap(&a.sel.tmap_meta);
    prefetch_tmap(&a.dec.tmap_k);
    prefetch_tmap(&a.dec.tmap_v);
  }
  __syncthreads();
  grid_dep_wait();  // the previous kernel of the stream has completed (no global access before)
  WarpState ws{0u, true, 0u, 0u};
  const int n_pre = a.n_score + a.n_sel;  // items before the decode items
  const int n_items = n_pre + a.n_dec;
  const uint32_t limit = a.flag_spin_limit ? a.flag_spin_limit : kFlagSpinLimit;
  for (;;) {
    if (threadIdx.x == 0) {
      int item = (int)atomicAdd(&a.queue[0], 1u);
      if (PER_HEAD && item >= a.n_score && item < n_pre) {
        const int u = item - a.n_score, b = u / a.sel.Hq;
        const int kvu = b * a.sel.kv.Hkv + (u - b * a.sel.Hq) / a.sel.G;
        if (!wait_count(a.sel.kv_scored + kvu, (uint32_t)a.sel.splits, a.sel.status, limit))
          item = n_items;  // gave up: this CTA stops taking work
      } else if (item >= n_pre && item < n_items) {
        int u, split;
        dec::item_unit(a.dec, item - n_pre, u, split);
        // the sequence length is an input of the launch: its load (kept in a
        // register until after the wait) overlaps the acquire
        const int ntok = a.dec.kv.seq_len[u / a.dec.kv.Hkv];  // decode units: (sequence, KV head)
        const int cnt = wait_selected(a.sel.ws_count + u, a.sel.status, limit);  // acquire
        s_count = cnt;
        s_ntok = ntok;
        if (cnt < 0) item = n_items;  // gave up: this CTA stops taking work
      }
      s_item = item;
    }
    __syncthreads();
    const int item = s_item;
    if (item >= n_items) {
      grid_dep_trigger();  // no work left here: the next kernel may start launching
      break;
    }
    if (item < a.n_score) {
      if (PER_HEAD)  // the G heads' score rows of one (sequence, KV head)
        sel::select_item<RULE, true, false, true, true>(a.sel, item / a.sel.splits, item % a.sel.splits, S, ws);
      else
        sel::select_item<RULE, true, false>(a.sel, item / a.sel.splits, item % a.sel.splits, S, ws);
    } else if (PER_HEAD && item < n_pre) {
      // one query head's selection from its score row; the KV head's last
      // one builds the union of the G heads' sets and publishes its flag
      const int u = item - a.n_score, b = u / a.sel.Hq;
      const int kvu = b * a.sel.kv.Hkv + (u - b * a.sel.Hq) / a.sel.G;
      sel::select_unit_of(a.sel, u, S, nullptr, a.sel.Hq);
      __syncthreads();
      if (threadIdx.x == 0)
        s_last = atom_add_acq_rel_u32(&a.sel.kv_selected[kvu], 1u) == (uint32_t)(a.sel.G - 1);
      __syncthreads();
      if (s_last) {
        int N, P;
        sel::unit_geometry(a.sel, b, N, P);
        fence_proxy_async();  // the ring becomes the union's mask words
        const int n = sel::build_union(a.sel, kvu, P, reinterpret_cast<uint32_t*>(base), s_scan);
        __syncthreads();
        if (threadIdx.x == 0) st_release_u32(&a.sel.ws_count[kvu], sel::kUnitSelected | (uint32_t)n);
      }
    } else {
      int u, split;
      dec::item_unit(a.dec, item - n_pre, u, split);
      if (a.sel.k_new != nullptr && lane == 0) fence_proxy_async_global();  // appended rows, then TMA
      dec::decode_item<false>(a.dec, u, split, D, ws, s_count, s_ntok);  // count from the unit's flag
    }
    fence_proxy_async();  // generic writes to the ring (keys, merge) before the next TMA writes
    __syncthreads();
  }
  if (!ws.alive && lane == 0) {  // a wait timed out: let the copies in flight land (bounded)
    uint64_t* wb = bars + warp * kStages;
    for (uint32_t g = ws.drain_lo; g < ws.drain_hi; ++g)
      mbar_wait(wb + g % kStages, (g / kStages) & 1u, nullptr);
  }
  // the last CTA out clears the unit flags and split counters, rewinds the queue
  if (threadIdx.x == 0) {
    __threadfence();
    s_last = atomicAdd(&a.queue[1], 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (s_last) {
    __threadfence();
    // unit flags and split counters: one per (sequence, KV head) (per-head
    // steps flag the KV heads' unions)
    const int units = a.sel.kv.B * a.sel.kv.Hkv;
    for (int i = threadIdx.x; i < units; i += blockDim.x) {
      a.sel.ws_count[i] = 0;
      a.dec.ws_count[i] = 0;
    }
    if (PER_HEAD)
      for (int i = threadIdx.x; i < a.sel.kv.B * a.sel.kv.Hkv; i += blockDim.x) {
        a.sel.kv_scored[i] = 0;
        a.sel.kv_selected[i] = 0;
      }
    if (threadIdx.x == 0) {
      a.queue[0] = 0;
      a.queue[1] = 0;
    }
  }
}

// The decode step for few units (a single layer at batch 1, say): one
// thread-block cluster of C CTAs per unit (sequence, KV head), one CTA per
// SM, so the handoffs between stages are cluster barriers and distributed
// shared memory instead of global item claims, flag polls and L2 round trips:
//  1. CTA r scores tile range r of C (the one holding the newest page also
//     refreshes it) and writes the group scores straight into the leader's
//     (rank 0) shared memory -- after a cluster barrier that every CTA
//     arrives on once its set-up is done and waits on only before its first
//     such store, so the leader is known to run and the wait overlaps the
//     first metadata load;
//  2. cluster barrier; the leader selects the unit's pages from its shared
//     memory and writes them out;
//  3. cluster barrier; CTA r runs decode splits r, r + C, ... with a deeper
//     TMA ring (kClStages per warp: a split's tiles are all in flight at
//     once).  With exactly C splits each CTA writes its partial into the
//     leader's shared memory and, after a last barrier, the leader merges
//     them; with more, the splits merge through the workspace as in the
//     persistent kernel.
// The same item code and splits as the separate calls and the same merge
// arithmetic, so results are identical to them.
constexpr int kClStages = 4;  // decode ring depth per warp in the cluster kernel

struct ClusterLayout {
  int ring, bars_sel, bars_dec, tiles, pre, scores, parts, total;
};
__host__ __device__ inline ClusterLayout cluster_layout(int max_pages, int max_sel, bool chunks, int C,
                                                        bool local_merge) {
  ClusterLayout L;
  const int dec_ring = dec::kWarps * kClStages * dec::kTileBytes;
  const int sel_body = body_bytes(max_pages);
  L.ring = 0;
  L.bars_sel = sel_body > dec_ring ? sel_body : dec_ring;
  L.bars_dec = L.bars_sel + kBarBytes;
  L.tiles = L.bars_dec + dec::kWarps * kClStages * 8;
  L.pre = L.tiles + kTileRefBytes;
  L.scores = (L.pre + (chunks ? (max_sel + 1) * 4 : 0) + 15) & ~15;
  L.parts = (L.scores + ((max_pages + 3) & ~3) * 4 + 15) & ~15;
  L.total = L.parts + (local_merge ? C * dec::kPartStride * 4 : 0);
  return L;
}

template <int RULE>
__global__ void __launch_bounds__(kThreads, 1) step_cluster_kernel(const __grid_constant__ StepArgs a) {
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint32_t s_hist[512];
  __shared__ uint32_t s_scan[32];
  __shared__ uint32_t s_bc[8];
  __shared__ int s_last, s_ntiles;
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int r = (int)cluster_ctarank(), C = (int)cluster_nctarank();
  const int u = (int)cluster_id_x();
  const bool local_merge = a.dec.splits == C;
  const ClusterLayout Lo = cluster_layout(a.sel.kv.max_pages, a.dec.max_sel, a.sel.kv.page_size == 0, C,
                                          local_merge);
  uint64_t* bars_sel = reinterpret_cast<uint64_t*>(base + Lo.bars_sel);
  uint64_t* bars_dec = reinterpret_cast<uint64_t*>(base + Lo.bars_dec);
  float* my_scores = reinterpret_cast<float*>(base + Lo.scores);
  float* my_parts = reinterpret_cast<float*>(base + Lo.parts);
  const sel::SelSmem S{base, bars_sel, s_hist, s_scan, s_bc, &s_last};
  const dec::Smem D{base, bars_dec, reinterpret_cast<dec::TileRef*>(base + Lo.tiles),
                    reinterpret_cast<int*>(base + Lo.pre), s_scan, &s_last, &s_ntiles};
  cg::cluster_group cl = cg::this_cluster();
  float* lead_scores = cl.map_shared_rank(my_scores, 0);
  float* lead_parts = cl.map_shared_rank(my_parts, 0);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(bars_sel + warp * kStages + s, 1);
    for (int s = 0; s < kClStages; ++s) mbar_init(bars_dec + warp * kClStages + s, 1);
    fence_barrier_init();
  }
  if (threadIdx.x == 0) {
    prefetch_tmap(&a.sel.tmap_meta);
    prefetch_tmap(&a.dec.tmap_k);
    prefetch_tmap(&a.dec.tmap_v);
  }
  __syncthreads();
  cluster_arrive_relaxed();  // this CTA runs (waited for before the first store to the leader)
  grid_dep_wait();           // the previous kernel of the stream has completed (no global access before)
  grid_dep_trigger();        // the next kernel may be scheduled now; it waits for this one to complete
  WarpState ws{0u, true, 0u, 0u};
  // 1. scoring of tile range r of C (a.sel.splits == C), scores to the leader
  sel::select_item<RULE, true, false, true, false, true>(a.sel, u, r, S, ws, lead_scores);
  if (!ws.alive && lane == 0) {  // a wait timed out: let the copies in flight land (bounded)
    for (uint32_t g = ws.drain_lo; g < ws.drain_hi; ++g)
      mbar_wait(bars_sel + warp * kStages + g % kStages, (g / kStages) & 1u, nullptr);
  }
  fence_proxy_async();  // generic writes to the ring (the refresh patch) before it is reused
  __syncthreads();
  cluster_sync();       // every range's scores are in the leader's shared memory
  // 2. the leader selects
  if (r == 0) sel::select_unit_of(a.sel, u, S, my_scores, a.sel.kv.Hkv);
  fence_proxy_async();  // the ring held the keys: generic writes before the decode TMA writes
  __syncthreads();
  cluster_sync();       // the selection is visible to every CTA of the cluster
  // 3. decode splits r, r + C, ... (each reads the kept count and pages)
  if (a.sel.k_new != nullptr && lane == 0) fence_proxy_async_global();  // appended rows, then TMA
  WarpState wd{0u, ws.alive, 0u, 0u};
  for (int split = r; split < a.dec.splits; split += C) {
    dec::decode_item<false, kClStages>(a.dec, u, split, D, wd, -1, -1, local_merge ? lead_parts : nullptr);
    fence_proxy_async();
    __syncthreads();
  }
  if (!wd.alive && ws.alive && lane == 0) {  // a wait timed out: let the copies in flight land (bounded)
    for (uint32_t g = wd.drain_lo; g < wd.drain_hi; ++g)
      mbar_wait(bars_dec + warp * kClStages + g % kClStages, (g / kClStages) & 1u, nullptr);
  }
  if (local_merge) {
    cluster_sync();  // every split's partial is in the leader's shared memory
    const int h = threadIdx.x / dec::kThreadsPerHead;
    const int d0 = (threadIdx.x % dec::kThreadsPerHead) * dec::kDimsPerThread;
    if (r == 0 && h < a.dec.G) {
      const int b = u / a.dec.kv.Hkv, g = u - b * a.dec.kv.Hkv;
      dec::merge_splits<true>(a.dec, my_parts + h * dec::kPartHead, C,
                              (size_t)b * a.dec.Hq + (size_t)g * a.dec.G + h, d0);
    }
  }
}

// The router applied to decode in one launch (see RouteStepArgs).  Queue:
// [0, n_score) scoring items (newest-page refresh, group scores to the
// workspace); the CTA finishing a unit's last one selects the unit's top
// max(rho k, k + 1) pages in rank order with sigma (the router's selection)
// and publishes the unit's flag (with its list count); the CTA finishing the
// last unit computes sigma_bar, the quantile threshold and the triggers,
// trims the untriggered lists to k, lists the triggered units and publishes
// the `routed` flag (1 + their number).  Then [n_score, n_score + n_base)
// the top-k windows of the units' lists, unit by unit (each waits for its
// unit's flag), then the expansion windows of the triggered units only (they
// wait for the routed flag; the first item past them ends the CTA's work).
// A unit's top-k windows merge when the last of them is done; a triggered
// unit's expansion windows then merge onto that (decode_item.cuh,
// kRouteExp).  Waits only ever point to items handed out earlier that never
// wait, so none can deadlock.
template <int RULE>
__global__ void __launch_bounds__(kThreads, SA_STEP_CTAS_PER_SM)
    route_step_kernel(const __grid_constant__ RouteStepArgs ra) {
  const StepArgs& a = ra.st;
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint32_t s_hist[512];
  __shared__ uint32_t s_scan[32];
  __shared__ uint32_t s_bc[8];
  __shared__ int s_last, s_item, s_ntiles, s_count, s_ntok, s_flag, s_unit, s_split;
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int body = body_bytes(a.sel.kv.max_pages);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + body);
  const sel::SelSmem S{base, bars, s_hist, s_scan, s_bc, &s_last};
  const dec::Smem D{base, bars, reinterpret_cast<dec::TileRef*>(base + body + kBarBytes),
                    reinterpret_cast<int*>(base + body + kBarBytes + kTileRefBytes), s_scan, &s_last,
                    &s_ntiles};
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(bars + warp * kStages + s, 1);
    fence_barrier_init();
  }
  if (threadIdx.x == 0) {
    prefetch_tmap(&a.sel.tmap_meta);
    prefetch_tmap(&a.dec.tmap_k);
    prefetch_tmap(&a.dec.tmap_v);
  }
  __syncthreads();
  grid_dep_wait();  // the previous kernel of the stream has completed (no global access before)
  WarpState ws{0u, true, 0u, 0u};
  const int units = a.sel.kv.B * a.sel.kv.Hkv;
  const int n_pre = a.n_score + ra.n_base;
  const int n_items = a.n_score + a.n_dec;
  const uint32_t limit = a.flag_spin_limit ? a.flag_spin_limit : kFlagSpinLimit;
  for (;;) {
    if (threadIdx.x == 0) {
      int item = (int)atomicAdd(&a.queue[0], 1u);
      if (item >= a.n_score && item < n_pre) {  // top-k window: once the unit's list is written
        const int sb = a.dec.route_base_splits;
        const int u = (item - a.n_score) / sb;
        const int ntok = a.dec.kv.seq_len[u / a.dec.kv.Hkv];  // overlaps the acquire
        int cnt = wait_selected(a.sel.ws_count + u, a.sel.status, limit);
        if (cnt > ra.route.k) cnt = ra.route.k;
        s_unit = u;
        s_split = item - a.n_score - u * sb;
        s_count = cnt;
        s_ntok = ntok;
        if (cnt < 0) item = n_items;  // gave up: this CTA stops taking work
      } else if (item >= n_pre && item < n_items) {  // expansion window of the q-th triggered unit
        const int sb = a.dec.route_base_splits, se = a.dec.splits - sb;
        const int x = item - n_pre, q = x / se;
        const uint32_t v = wait_nonzero(ra.routed + 1, a.sel.status, limit);  // 1 + triggered units
        if (v == 0u || q >= (int)v - 1) {
          item = n_items;  // timed out, or past the last triggered unit: no more work here
        } else {
          const int4 e = __ldcg(ra.route.trig_list + q);
          s_unit = e.x;
          s_split = sb + (x - q * se);
          s_count = e.y;
          s_ntok = e.z;
        }
      }
      s_item = item;
    }
    __syncthreads();
    const int item = s_item;
    if (item >= n_items) {
      grid_dep_trigger();
      break;
    }
    if (item < a.n_score) {
      const int u = item / a.sel.splits;
      sel::select_item<RULE, true, false, true>(a.sel, u, item % a.sel.splits, S, ws);
      __syncthreads();
      if (threadIdx.x == 0) {
        const uint32_t prev = atom_add_acq_rel_u32(&a.sel.ws_count[u], 1u);
        s_flag = prev == (uint32_t)(a.sel.splits - 1);
      }
      __syncthreads();
      if (s_flag) {  // the unit's last scoring item: the router's selection
        const int b = u / a.sel.kv.Hkv, g = u - b * a.sel.kv.Hkv;
        int N, P;
        sel::unit_geometry(a.sel, b, N, P);
        fence_proxy_async();  // the ring becomes the selection's keys
        if (P <= 16 * kThreads) {
          // the plain step's register selection finds the candidates (keys
          // above the cut, then equal keys in page order), the router's code
          // ranks them and computes sigma
          const int cap = min(max(ra.route.W, ra.route.k + 1), P);
          auto* cand = reinterpret_cast<unsigned long long*>(base + sel::kCandOffset);
          sel::select_unit_regs<16, false>(a.sel, u, N, P, (uint32_t)cap, 0, P, nullptr, S, nullptr, cand);
          rsel::route_select_finish(ra.route, u, P, cand, cap);
        } else {
          rsel::route_select_tile(ra.route, b, g, P, base, s_hist, s_bc, s_scan);
        }
        __syncthreads();
        if (threadIdx.x == 0) {
          // one fence publishes the list, count and sigma through both signals
          fence_acq_rel_gpu();
          st_relaxed_u32(&a.sel.ws_count[u], sel::kUnitSelected | (uint32_t)ra.route.kv_count[u]);
          s_flag = atom_add_relaxed_u32(ra.routed, 1u) == (uint32_t)(units - 1);
          if (s_flag) fence_acq_rel_gpu();  // the last unit: acquire every unit's sigma and count
        }
        __syncthreads();
        if (s_flag) {  // every unit selected: quantile, triggers, the triggered units
          double tau;
          const int n_trig = rsel::route_triggers(ra.route, base, tau);
          if (threadIdx.x == 0) st_release_u32(ra.routed + 1, 1u + (uint32_t)n_trig);
          rsel::route_outputs(ra.route, base, tau);  // read by no decode item
        }
      }
    } else {
      dec::decode_item<false>(a.dec, s_unit, s_split, D, ws, s_count, s_ntok);
    }
    fence_proxy_async();  // generic writes to the ring (keys, merge) before the next TMA writes
    __syncthreads();
  }
  if (!ws.alive && lane == 0) {  // a wait timed out: let the copies in flight land (bounded)
    uint64_t* wb = bars + warp * kStages;
    for (uint32_t g = ws.drain_lo; g < ws.drain_hi; ++g)
      mbar_wait(wb + g % kStages, (g / kStages) & 1u, nullptr);
  }
  // the last CTA out clears the unit flags, split counters and routed counters
  if (threadIdx.x == 0) {
    __threadfence();
    s_last = atomicAdd(&a.queue[1], 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (s_last) {
    __threadfence();
    for (int i = threadIdx.x; i < units; i += blockDim.x) {
      a.sel.ws_count[i] = 0;
      a.dec.ws_count[i] = 0;
    }
    if (threadIdx.x == 0) {
      ra.routed[0] = 0;
      ra.routed[1] = 0;
      a.queue[0] = 0;
      a.queue[1] = 0;
    }
  }
}

// Resident CTAs per SM of a step kernel for a shared-memory size (cached).
int step_occupancy(const void* fn, size_t smem) {
  struct Entry {
    const void* f;
    int dev;
    size_t smem;
    int occ;
  };
  static Entry cache[32];
  static int n = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  for (int i = 0; i < n; ++i)
    if (cache[i].f == fn && cache[i].dev == dev && cache[i].smem == smem) return cache[i].occ;
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, kThreads, smem) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  if (n < 32) cache[n++] = Entry{fn, dev, smem, occ};
  return occ;
}

}  // namespace

size_t step_smem_bytes(int max_pages, int max_sel, bool chunks) {
  size_t s = 1024 + (size_t)body_bytes(max_pages) + kBarBytes + kTileRefBytes;
  if (chunks) s += (size_t)(max_sel + 1) * 4;  // decode: tile prefix of the kept chunks
  return s;
}

// Cluster size of the small-unit decode step: C CTAs per unit, one CTA per
// SM, when all units' clusters fit the GPU at once and the unit's decode
// splits fill them; 0 = use the persistent kernel.
int step_cluster_size(int units, int dec_splits, int sm_count) {
  if (units < 1 || dec_splits < SA_STEP_CLUSTER) return 0;
  if ((long long)units * SA_STEP_CLUSTER > sm_count) return 0;
  return SA_STEP_CLUSTER;
}

cudaError_t launch_step_cluster(const StepArgs& a, int C, cudaStream_t st) {
  const ClusterLayout Lo = cluster_layout(a.sel.kv.max_pages, a.dec.max_sel, a.sel.kv.page_size == 0, C,
                                          a.dec.splits == C);
  size_t smem = 1024 + (size_t)Lo.total;
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  if (smem < kClusterMinSmem) smem = kClusterMinSmem;  // one CTA per SM
  const int units = a.sel.kv.B * a.sel.kv.Hkv;
  const void* fn = a.sel.rule == 0 ? (const void*)step_cluster_kernel<0> : (const void*)step_cluster_kernel<1>;
  cudaError_t e = set_smem_attr(fn, smem);
  if (e != cudaSuccess) return e;
  if (C > 8) {
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(units * C));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = (unsigned)C;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (a.sel.rule == 0) return cudaLaunchKernelEx(&cfg, step_cluster_kernel<0>, a);
  return cudaLaunchKernelEx(&cfg, step_cluster_kernel<1>, a);
}

cudaError_t launch_route_step(const RouteStepArgs& a, cudaStream_t st) {
  const size_t smem = step_smem_bytes(a.st.sel.kv.max_pages, a.st.dec.max_sel, false);
  const long long items = (long long)a.st.n_score + a.st.n_dec;
  if (items > 0x7fffffffLL) return cudaErrorInvalidValue;
  using Fn = void (*)(const RouteStepArgs);
  const Fn f = a.st.sel.rule == 0 ? route_step_kernel<0> : route_step_kernel<1>;
  cudaError_t e = set_smem_attr((const void*)f, smem);
  if (e != cudaSuccess) return e;
  int occ = step_occupancy((const void*)f, smem);
  if (occ < 1) return cudaErrorInvalidConfiguration;
  if (occ > SA_STEP_CTAS_PER_SM) occ = SA_STEP_CTAS_PER_SM;
  long long grid = (long long)device_sm_count() * occ;
  if (grid > items) grid = items;
  return launch_pdl(f, (unsigned)grid, kThreads, smem, st, a);
}

cudaError_t launch_step(const StepArgs& a, cudaStream_t st) {
  const size_t smem = step_smem_bytes(a.sel.kv.max_pages, a.dec.max_sel, a.sel.kv.page_size == 0);
  const long long items = (long long)a.n_score + a.n_sel + a.n_dec;
  if (items > 0x7fffffffLL) return cudaErrorInvalidValue;
  using Fn = void (*)(const StepArgs);
  const Fn fns[2][2] = {{step_kernel<0, false>, step_kernel<0, true>}, {step_kernel<1, false>, step_kernel<1, true>}};
  const Fn f = fns[a.sel.rule == 0 ? 0 : 1][a.sel.per_head ? 1 : 0];
  const void* fn = (const void*)f;
  cudaError_t e = set_smem_attr(fn, smem);
  if (e != cudaSuccess) return e;
  int occ = step_occupancy(fn, smem);
  if (occ < 1) return cudaErrorInvalidConfiguration;
  if (occ > SA_STEP_CTAS_PER_SM) occ = SA_STEP_CTAS_PER_SM;
  long long grid = (long long)device_sm_count() * occ;
  if (grid > items) grid = items;
  return launch_pdl(f, (unsigned)grid, kThreads, smem, st, a);
}

}  // namespace sa
