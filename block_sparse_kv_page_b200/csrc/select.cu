// Standalone page scoring + budgeted top-k selection kernel: a persistent
// grid pulls (unit, tile range) items from an atomic queue and runs
// sel::select_item on each (select_item.cuh: TMA-staged metadata, tensor-core
// scores, last-CTA radix selection with the lowest-index tie rule).
#include "common.cuh"
#include "internal.h"
#include "select_item.cuh"

namespace sa {
namespace {

using namespace sel;

// MODE 0: one page set per (sequence, KV head); 1: per (sequence, query head);
// 2: group scores only.
template <int RULE, int MODE>
__global__ void __launch_bounds__(kThreads, SA_SEL_CTAS_PER_SM) select_kernel(const __grid_constant__ SelectArgs a) {
  constexpr bool PER_HEAD = MODE == 1;
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint32_t s_hist[512];
  __shared__ uint32_t s_scan[32];
  __shared__ uint32_t s_bc[8];
  __shared__ int s_last, s_item;
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  // barriers sit after the ring, or after the keys/weights area when that is larger
  const int kb = keys_bytes(a.kv.max_pages);
  const int bar_off = kb > kRingBytes ? ((kb + 1023) & ~1023) : kRingBytes;
  const SelSmem S{base, reinterpret_cast<uint64_t*>(base + bar_off), s_hist, s_scan, s_bc, &s_last};
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(S.bars + warp * kStages + s, 1);
    fence_barrier_init();
  }
  if (threadIdx.x == 0) prefetch_tmap(&a.tmap_meta);
  __syncthreads();
  grid_dep_wait();  // the previous kernel of the stream has completed (no global access before)
  WarpState ws{0u, true, 0u, 0u};
  const int n_items = a.kv.B * (PER_HEAD ? a.Hq : a.kv.Hkv) * a.splits;
  for (;;) {
    if (threadIdx.x == 0) s_item = (int)atomicAdd(&a.ws_queue[0], 1u);
    __syncthreads();
    const int item = s_item;
    if (item >= n_items) {
      grid_dep_trigger();  // no work left here: the next kernel may start launching
      break;
    }
    select_item<RULE, false, PER_HEAD, MODE == 2>(a, item / a.splits, item % a.splits, S, ws);
    fence_proxy_async();  // generic writes to the ring (keys) before the next TMA writes
    __syncthreads();
  }
  if (!ws.alive && lane == 0) {  // a wait timed out: let the copies in flight land (bounded)
    uint64_t* bars = S.bars + warp * kStages;
    for (uint32_t gg = ws.drain_lo; gg < ws.drain_hi; ++gg)
      mbar_wait(bars + gg % kStages, (gg / kStages) & 1u, nullptr);
  }
  // the last CTA out rewinds the queue for the next launch
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(&a.ws_queue[1], 1u) == gridDim.x - 1) {
      a.ws_queue[0] = 0;
      a.ws_queue[1] = 0;
    }
  }
}

}  // namespace

// Splits per unit: items of about SA_SEL_ITEM_PAGES pages, but at least two
// items per SM when there are few units, and at least
// SA_SEL_MIN_ITEM_TILES_PER_WARP tiles per warp.
int select_splits(int units, int max_pages, int sm_count) {
  int s = (max_pages + SA_SEL_ITEM_PAGES - 1) / SA_SEL_ITEM_PAGES;
  const int fill = (2 * sm_count + units - 1) / units;
  if (fill > s) s = fill;
  const int min_pages = 16 * kWarps * SA_SEL_MIN_ITEM_TILES_PER_WARP;
  const int cap = (max_pages + min_pages - 1) / min_pages;
  if (s > cap) s = cap;
  if (s > 256) s = 256;
  if (s < 1) s = 1;
  return s;
}

size_t select_smem_bytes(int max_pages) {
  const size_t keys = ((size_t)keys_bytes(max_pages) + 1023) & ~(size_t)1023;
  const size_t body = keys > (size_t)kRingBytes ? keys : (size_t)kRingBytes;
  return 1024 + body + kWarps * kStages * 8;
}

cudaError_t launch_select(const SelectArgs& a, cudaStream_t st) {
  const size_t smem = select_smem_bytes(a.kv.max_pages);
  const long long items = (long long)a.kv.B * (a.per_head ? a.Hq : a.kv.Hkv) * a.splits;
  if (items > 0x7fffffffLL) return cudaErrorInvalidValue;
  long long grid = (long long)device_sm_count() * SA_SEL_CTAS_PER_SM;
  if (grid > items) grid = items;
  const int mode = a.score_only ? 2 : (a.per_head ? 1 : 0);
  void (*const fns[2][3])(SelectArgs) = {{select_kernel<0, 0>, select_kernel<0, 1>, select_kernel<0, 2>},
                                         {select_kernel<1, 0>, select_kernel<1, 1>, select_kernel<1, 2>}};
  auto fn = fns[a.rule == 0 ? 0 : 1][mode];
  const cudaError_t e = set_smem_attr((const void*)fn, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(fn, (unsigned)grid, kThreads, smem, st, a);
}

}  // namespace sa
