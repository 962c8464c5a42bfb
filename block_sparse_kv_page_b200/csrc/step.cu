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
#include "common.cuh"
#include "internal.h"
#include "decode_item.cuh"
#include "select_item.cuh"

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

// PER_HEAD: units are (sequence, query head), each selecting its own pages.
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
  const int n_items = a.n_score + a.n_dec;
  for (;;) {
    if (threadIdx.x == 0) {
      int item = (int)atomicAdd(&a.queue[0], 1u);
      if (item >= a.n_score && item < n_items) {
        int u, split;
        dec::item_unit(a.dec, item - a.n_score, u, split);
        // the sequence length is an input of the launch: its load (kept in a
        // register until after the wait) overlaps the acquire
        const int ntok = a.dec.kv.seq_len[unit_map<PER_HEAD>(u, a.dec.kv.Hkv, a.dec.Hq, a.dec.G).b];
        const int cnt = wait_selected(a.sel.ws_count + u, a.sel.status,
                                      a.flag_spin_limit ? a.flag_spin_limit : kFlagSpinLimit);  // acquire
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
      sel::select_item<RULE, true, PER_HEAD>(a.sel, item / a.sel.splits, item % a.sel.splits, S, ws);
    } else {
      int u, split;
      dec::item_unit(a.dec, item - a.n_score, u, split);
      if (a.sel.k_new != nullptr && lane == 0) fence_proxy_async_global();  // appended rows, then TMA
      dec::decode_item<PER_HEAD>(a.dec, u, split, D, ws, s_count, s_ntok);  // count from the unit's flag
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
    const int units = a.sel.kv.B * (a.sel.per_head ? a.sel.Hq : a.sel.kv.Hkv);
    for (int i = threadIdx.x; i < units; i += blockDim.x) {
      a.sel.ws_count[i] = 0;
      a.dec.ws_count[i] = 0;
    }
    if (threadIdx.x == 0) {
      a.queue[0] = 0;
      a.queue[1] = 0;
    }
  }
}

// The decode step for few units (a single layer at batch 1, say): one
// thread-block cluster of C CTAs per unit (sequence, KV head), so the
// handoffs between stages are hardware cluster barriers instead of global
// item claims and flag polls.  CTA r of the cluster scores tile range r of C
// (the one holding the newest page also refreshes it); after a cluster
// barrier the leader (rank 0) selects the unit's pages; after another, CTA r
// runs decode splits r, r + C, ... of the unit, merged by the last of them
// as in the persistent kernel.  The same item code with the same splits as
// the separate calls, so results are identical to them.
template <int RULE>
__global__ void __launch_bounds__(kThreads, 1) step_cluster_kernel(const __grid_constant__ StepArgs a) {
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint32_t s_hist[512];
  __shared__ uint32_t s_scan[32];
  __shared__ uint32_t s_bc[8];
  __shared__ int s_last, s_ntiles;
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
  grid_dep_wait();     // the previous kernel of the stream has completed (no global access before)
  grid_dep_trigger();  // the next kernel may be scheduled now; it waits for this one to complete
  const int r = (int)cluster_ctarank(), C = (int)cluster_nctarank();
  const int u = (int)cluster_id_x();
  WarpState ws{0u, true, 0u, 0u};
  // 1. scoring of tile range r of C (a.sel.splits == C)
  sel::select_item<RULE, true, false, true>(a.sel, u, r, S, ws);
  fence_proxy_async();  // generic writes to the ring (the refresh patch) before its next TMA writes
  __syncthreads();
  cluster_sync();       // every range's scores are visible to the leader
  // 2. the leader selects
  if (r == 0) sel::select_unit_of(a.sel, u, S);
  fence_proxy_async();  // the ring held the keys
  __syncthreads();
  cluster_sync();       // the selection is visible to every CTA of the cluster
  // 3. decode splits r, r + C, ... (each reads the kept count and pages)
  if (a.sel.k_new != nullptr && lane == 0) fence_proxy_async_global();  // appended rows, then TMA
  for (int split = r; split < a.dec.splits; split += C) {
    dec::decode_item<false>(a.dec, u, split, D, ws);
    fence_proxy_async();
    __syncthreads();
  }
  if (!ws.alive && lane == 0) {  // a wait timed out: let the copies in flight land (bounded)
    uint64_t* wb = bars + warp * kStages;
    for (uint32_t g = ws.drain_lo; g < ws.drain_hi; ++g)
      mbar_wait(wb + g % kStages, (g / kStages) & 1u, nullptr);
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
  size_t smem = step_smem_bytes(a.sel.kv.max_pages, a.dec.max_sel, a.sel.kv.page_size == 0);
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

cudaError_t launch_step(const StepArgs& a, cudaStream_t st) {
  const size_t smem = step_smem_bytes(a.sel.kv.max_pages, a.dec.max_sel, a.sel.kv.page_size == 0);
  const long long items = (long long)a.n_score + a.n_dec;
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
