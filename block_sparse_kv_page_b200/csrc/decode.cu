// Standalone sparse paged flash-decode kernel: a persistent grid pulls
// (unit, tile range) items from an atomic queue and runs dec::decode_item on
// each (decode_item.cuh: TMA-streamed K/V tiles of the selected pages,
// tensor-core QK and PV, online softmax, last-CTA split combine).
#include "common.cuh"
#include "internal.h"
#include "decode_item.cuh"

namespace sa {
namespace {

using namespace dec;

template <bool PER_HEAD>
__global__ void __launch_bounds__(kThreads, SA_DEC_CTAS_PER_SM) decode_kernel(const __grid_constant__ DecodeArgs a) {
  extern __shared__ unsigned char smem_raw[];
  __shared__ int s_item, s_last, s_ntiles;
  __shared__ uint32_t s_scan[kWarps];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const Smem sm{base, reinterpret_cast<uint64_t*>(base + kOffBars), reinterpret_cast<TileRef*>(base + kOffTiles),
                reinterpret_cast<int*>(base + kOffPre), s_scan, &s_last, &s_ntiles};
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(sm.bars + warp * kStages + s, 1);
    fence_barrier_init();
  }
  if (threadIdx.x == 0) {
    prefetch_tmap(&a.tmap_k);
    prefetch_tmap(&a.tmap_v);
  }
  __syncthreads();
  grid_dep_wait();  // the previous kernel of the stream has completed (no global access before)
  WarpState ws{0u, true, 0u, 0u};
  for (;;) {
    if (threadIdx.x == 0) s_item = (int)atomicAdd(&a.ws_queue[0], 1u);
    __syncthreads();
    const int item = s_item;
    if (item >= a.n_items) {
      grid_dep_trigger();  // no work left here: the next kernel may start launching
      break;
    }
    int u, split;
    item_unit(a, item, u, split);
    decode_item<PER_HEAD>(a, u, split, sm, ws);
    fence_proxy_async();  // generic writes to the ring (merge) before the next TMA writes
    __syncthreads();
  }
  if (!ws.alive && lane == 0) {  // a wait timed out: let the copies in flight land (bounded)
    uint64_t* bars = sm.bars + warp * kStages;
    for (uint32_t g = ws.drain_lo; g < ws.drain_hi; ++g)
      mbar_wait(bars + g % kStages, (g / kStages) & 1u, nullptr);
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

// Splits per unit: items of about SA_DEC_ITEM_TILES tiles, but at least two
// items per SM when there are few units, and at least SA_DEC_MIN_ITEM_TILES
// tiles per item (each item pays a fixed setup and combine cost).  The
// units of the last wave of items (one item per resident CTA) may get
// SA_DEC_TAIL_FINE times finer splits, so the launch does not end on a few
// long items.  Off by default: on the 48-layer decode step a factor of 2 or 4
// costs more in per-item overhead (about 9 us of claim, setup, pipeline fill
// and combine per item) than it saves in the tail.
DecodePlan decode_plan(int units, int max_tiles, int sm_count) {
  int s = (max_tiles + SA_DEC_ITEM_TILES - 1) / SA_DEC_ITEM_TILES;
  const int fill = (2 * sm_count + units - 1) / units;
  if (fill > s) s = fill;
  const int cap = (max_tiles + SA_DEC_MIN_ITEM_TILES - 1) / SA_DEC_MIN_ITEM_TILES;
  if (s > cap) s = cap;
  if (s > 256) s = 256;
  if (s < 1) s = 1;
  int fine = SA_DEC_TAIL_FINE * s;
  if (fine > cap) fine = cap;
  if (fine > 256) fine = 256;
  DecodePlan p{s, units, s, 0};
  if (fine > s) {
    const int wave = sm_count * SA_DEC_CTAS_PER_SM;
    const int fine_units = (wave + fine - 1) / fine;
    p.fine_unit0 = units > fine_units ? units - fine_units : 0;
    p.splits_fine = fine;
  }
  p.items = (long long)p.fine_unit0 * p.splits + (long long)(units - p.fine_unit0) * p.splits_fine;
  return p;
}

size_t decode_smem_bytes(int max_sel, bool chunks) {
  size_t s = 1024 + kOffPre;  // alignment slack + ring + barriers + tile refs
  if (chunks) s += (size_t)(max_sel + 1) * 4;
  return s;
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st) {
  const size_t smem = decode_smem_bytes(a.max_sel, a.kv.page_size == 0);
  const long long items = a.n_items;
  long long grid = (long long)device_sm_count() * SA_DEC_CTAS_PER_SM;
  if (grid > items) grid = items;
  const void* fn = a.per_head ? (const void*)decode_kernel<true> : (const void*)decode_kernel<false>;
  const cudaError_t e = set_smem_attr(fn, smem);
  if (e != cudaSuccess) return e;
  return a.per_head ? launch_pdl(decode_kernel<true>, (unsigned)grid, kThreads, smem, st, a)
                    : launch_pdl(decode_kernel<false>, (unsigned)grid, kThreads, smem, st, a);
}

}  // namespace sa
