// One work item of page scoring + budgeted top-k selection: the scoring of a
// range of 16-page tiles of one unit (sequence, KV head), and, for the CTA
// that finishes the unit's last range, the selection.  Called by the
// standalone selection kernel and by the fused decode step.
//
// "Sparse Attention for Web Agents -- Offline Replay Records", section "The
// comparison": each chunk is scored against the current query (envelope =
// per-dimension min/max upper bound; centroid = mean key) and the best ones
// are kept, the budget being page_size x top_k attended tokens; TSA fills a
// token budget over variable chunks.  "WebArena 0-99 Sparse-Attention Method
// Comparison", section "Method configurations at a glance": ratio budget
// max(topk_val + bos + eos, int(blocks * ratio)) with forced bos/eos blocks.
//
// Scoring.  The metadata of a tile (16 pages x 512 B) arrives by TMA as four
// 16 x 128-byte boxes, 128B-swizzled, into a per-warp mbarrier ring; lane 0
// of each warp keeps several tiles in flight.  All G grouped query heads are
// scored on tensor cores:
//   envelope: S^T[16 pages x 8 heads] = [kmin | kmax] (16 x 256, bf16)
//             x [q- | q+]^T (256 x 8, bf16), m16n8k16 via ldmatrix, exact
//             products, fp32 accumulation;
//   centroid: S^T = kmean (16 x 128, fp32) x q^T (128 x 8, bf16) on the FP64
//             tensor cores (m8n8k4): exact products and sums, one rounding to
//             fp32, so near-ties are resolved as in float64.
// The group score (max over the G heads) goes to the workspace.  In the fused
// step (FUSED), the warp that owns the tile holding the page of the
// newest token (N - 1) first rebuilds that page's metadata from K, stores it
// to the metadata array and patches the staged tile, so the step scores the
// cache as it stands after the append.
//
// Selection.  The CTA that finishes a unit's last item (atomic counter;
// nobody waits) loads the unit's scores and runs a weighted MSB-first radix
// select on order-preserving 32-bit keys: it finds the cut key T and the
// capacity left for keys equal to T; equal keys are then taken in ascending
// page order (the lowest-index tie rule), so the result is exactly "the
// longest prefix of the (score desc, index asc) order within the budget".
// Weight 1 per page gives top-k / ratio; weight = chunk length gives the token
// budget.  Output is the kept set in ascending page order.  In the fused step
// the unit's counter is left at kUnitSelected | kept count (release) once the
// output is written, for consumers in the same launch.
#pragma once

#include "common.cuh"
#include "internal.h"
#include "page_meta.cuh"
#include "radix.cuh"

// Scoring item size in pages.  At 29.5K-token contexts (1844 pages per unit)
// 384 gives five items per unit; on the 48-layer decode step 4, 5, 6, 7 and 8
// items per unit measured 104.8, 103.0, 106.0, 105.9 and 106.3 us.
#ifndef SA_SEL_ITEM_PAGES
#define SA_SEL_ITEM_PAGES 384
#endif
#ifndef SA_SEL_STAGES
#define SA_SEL_STAGES 2
#endif
#ifndef SA_SEL_CTAS_PER_SM
#define SA_SEL_CTAS_PER_SM 3
#endif
#ifndef SA_SEL_WARPS
#define SA_SEL_WARPS 4
#endif
#ifndef SA_SEL_MIN_ITEM_TILES_PER_WARP
#define SA_SEL_MIN_ITEM_TILES_PER_WARP 2
#endif

namespace sa {
namespace sel {

constexpr int kWarps = SA_SEL_WARPS;
constexpr int kThreads = kWarps * 32;
constexpr int kStages = SA_SEL_STAGES;
constexpr int kTileBytes = 8192;          // 16 pages x 512 B = four 2 KiB boxes
constexpr int kBoxBytes = 2048;
constexpr int kRingBytes = kWarps * kStages * kTileBytes;
constexpr uint32_t kUnitSelected = 0x80000000u;
constexpr int kSelBatch = 4;              // 16-byte score loads in flight per thread

// Selection-phase shared memory: keys and weights, 4 B each per page.
__host__ __device__ constexpr int keys_bytes(int max_pages) { return 8 * max_pages; }

struct SelSmem {
  unsigned char* ring;   // [warp][stage][kTileBytes]; reused for keys/weights in selection
  uint64_t* bars;        // [warp][stage]
  uint32_t* hist;        // 512 (two 256-bin buffers)
  uint32_t* scan;        // 32
  uint32_t* bc;          // 8
  int* last;
};

// Selection from keys staged in shared memory (any P up to max_pages).
SA_DEV void select_unit_smem(const SelectArgs& a, const int u, const int N, const int P,
                             const uint32_t cap, const int forced_lo, const int forced_hi,
                             const int32_t* off, const SelSmem& S, const float* sc_local) {
  const int tid = threadIdx.x;
  uint32_t* keys = reinterpret_cast<uint32_t*>(S.ring);
  uint32_t* wts = keys + a.kv.max_pages;
  const float* sc_u = sc_local ? sc_local : a.ws_scores + (size_t)u * a.ws_stride;
  const bool weighted = off != nullptr;
  // Keys (and chunk weights) into shared memory.  Every thread issues all its
  // loads of a batch before using any: under full HBM load each dependent
  // round trip to L2 costs about a microsecond.
  uint32_t wall_local = 0;
  const int P4 = (P + 3) >> 2;  // 16-byte groups of 4 pages (rows are padded to 4)
  for (int base4 = 0; base4 < P4; base4 += kSelBatch * (int)blockDim.x) {
    float4 v[kSelBatch];
    int o[kSelBatch][5];
#pragma unroll
    for (int j = 0; j < kSelBatch; ++j) {
      const int i4 = base4 + j * (int)blockDim.x + tid;
      const float4* src = reinterpret_cast<const float4*>(sc_u) + i4;
      v[j] = i4 < P4 ? (sc_local ? *src : __ldcg(src)) : make_float4(0.f, 0.f, 0.f, 0.f);
      if (weighted) {
#pragma unroll
        for (int e = 0; e < 5; ++e) o[j][e] = (i4 < P4 && 4 * i4 + e <= P) ? off[4 * i4 + e] : 0;
      }
    }
#pragma unroll
    for (int j = 0; j < kSelBatch; ++j) {
      const int i4 = base4 + j * (int)blockDim.x + tid;
      const float sv[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int p = 4 * i4 + e;
        if (i4 < P4 && p < P) {
          uint32_t key = order_key(sv[e]);
          if (p < forced_lo || p >= forced_hi) key = 0xffffffffu;
          keys[p] = key;
          if (weighted) {
            const int L = max(min(o[j][e + 1], N) - o[j][e], 0);
            wts[p] = (uint32_t)L;
            wall_local += (uint32_t)L;
          } else {
            wall_local += 1u;
          }
        }
      }
    }
  }
  uint32_t wall;
  block_excl_scan(wall_local, S.scan, wall);  // includes a __syncthreads

  int32_t* sel_u = a.sel_idx + (size_t)u * a.max_sel;
  if (wall <= cap) {  // everything fits
    for (int p = tid; p < P; p += blockDim.x)
      if (p < a.max_sel) sel_u[p] = p;
    if (tid == 0) {
      if (P > a.max_sel) flag_status(a.status, SA_ERR_DEVICE_CHECK);
      a.sel_count[u] = min(P, a.max_sel);
    }
    return;
  }
  const RadixCut cut = radix_cut(keys, weighted ? wts : nullptr, P, cap, S.hist, S.bc);

  const int per = (P + blockDim.x - 1) / blockDim.x;
  const int i0 = min(P, tid * per), i1 = min(P, i0 + per);
  uint32_t eqw = 0;
  for (int i = i0; i < i1; ++i)
    if (keys[i] == cut.T) eqw += weighted ? wts[i] : 1u;
  uint32_t dummy;
  const uint32_t eq0 = block_excl_scan(eqw, S.scan, dummy);
  uint32_t cnt = 0, eq = eq0;
  for (int i = i0; i < i1; ++i) {
    const uint32_t k = keys[i];
    bool sel = k > cut.T;
    if (k == cut.T) {
      eq += weighted ? wts[i] : 1u;
      sel = eq <= cut.rem;
    }
    cnt += sel ? 1u : 0u;
  }
  uint32_t total;
  uint32_t pos = block_excl_scan(cnt, S.scan, total);
  eq = eq0;
  for (int i = i0; i < i1; ++i) {
    const uint32_t k = keys[i];
    bool sel = k > cut.T;
    if (k == cut.T) {
      eq += weighted ? wts[i] : 1u;
      sel = eq <= cut.rem;
    }
    if (sel) {
      if (pos < (uint32_t)a.max_sel) sel_u[pos] = i;
      ++pos;
    }
  }
  if (tid == 0) {
    if (total > (uint32_t)a.max_sel) flag_status(a.status, SA_ERR_DEVICE_CHECK);
    a.sel_count[u] = (int32_t)min(total, (uint32_t)a.max_sel);
  }
}

// Selection with the keys in registers, for P <= KPT * 128 (four warps):
// thread t holds pages [KPT t, KPT t + KPT), so thread order is page order.
// WEIGHTED: chunk lengths (token budget), else every page weighs 1.
//
// The cut T (weight(keys > T) <= cap < weight(keys >= T)) comes from an
// MSB-first radix search over 12-bit windows of the keys, histogrammed with
// shared-memory reductions only (the keys are never re-read from memory):
//  - all-ones keys (forced pages) are settled first: if they overflow the
//    budget they are the cut, else their weight is spent up front;
//  - the first window starts at the highest bit where the other keys differ
//    (the scores of one unit often share sign and exponent), so it spreads
//    them over up to 4096 bins; the second usually isolates the cut; with unit
//    weights the search stops as soon as the budget is met exactly at a bin
//    edge (nothing of the cut bin is taken);
//  - a pass costs two barriers: thread t sums bin row 127 - t (32 bins, rows
//    in descending order) and publishes the sum; then every warp, on its own,
//    scans the 128 row sums, picks the row holding the cut and scans its 32
//    bins, so the cut needs no broadcast.  Bin rows are 16-byte-chunk XOR
//    swizzled so that the row sums are conflict-free vector loads.
// Keys above T are kept, keys equal to T in page order while the weight fits;
// block scans give each thread its first output slot (one packed scan with
// unit weights).  The bins live in the ring area, idle during selection.
SA_DEV uint32_t bin_slot(uint32_t b) {  // physical word of bin b in a 4096-bin buffer
  const uint32_t r = b >> 5, w = b & 31u;
  return (r << 5) | ((((w >> 2) ^ (r & 7u)) << 2) | (w & 3u));
}

// cand (non-null, shared memory past the first 36 KiB of S.ring): instead of
// sel_idx and sel_count, the kept pages go to cand[0 .. kept) in page order
// as composite keys (score key << 32 | ~page, the router's rank-order key).
constexpr int kCandOffset = 36 * 1024;
static_assert(2 * 4096 * 4 + 128 * 4 + 16 * 4 <= kCandOffset, "bins, row sums and warp totals stay below cand");
SA_DEV unsigned long long cand_key(uint32_t key, int p) {
  return ((unsigned long long)key << 32) | (0xffffffffu - (uint32_t)p);
}
template <int KPT, bool WEIGHTED>
SA_DEV void select_unit_regs(const SelectArgs& a, const int u, const int N, const int P,
                             const uint32_t cap, const int forced_lo, const int forced_hi,
                             const int32_t* off, const SelSmem& S, const float* sc_local,
                             unsigned long long* cand = nullptr) {
  static_assert(KPT % 4 == 0 && KPT <= 32, "pages per thread");
  static_assert(kThreads == 128, "the register path maps 4096 bins onto 128 threads");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* sc_u = sc_local ? sc_local : a.ws_scores + (size_t)u * a.ws_stride;
  const int p0 = tid * KPT;
  uint32_t* H0 = reinterpret_cast<uint32_t*>(S.ring);  // [2][4096] bins
  uint32_t* tsum = H0 + 2 * 4096;                       // [128] row sums
  uint32_t* wred = tsum + 128;                          // [4 warps][4]
  uint32_t key[KPT], wt[WEIGHTED ? KPT : 1], valid = 0u;
  {
    // every load issued before any is used (one round trip to L2)
    float4 v[KPT / 4];
#pragma unroll
    for (int q = 0; q < KPT / 4; ++q) {
      const float4* src = reinterpret_cast<const float4*>(sc_u + p0) + q;
      v[q] = p0 + 4 * q < P ? (sc_local ? *src : __ldcg(src)) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    int o[WEIGHTED ? KPT + 1 : 1];
    if (WEIGHTED) {
#pragma unroll
      for (int i = 0; i <= KPT; ++i) o[i] = p0 + i <= P ? off[p0 + i] : 0;
    }
#pragma unroll
    for (int q = 0; q < KPT / 4; ++q) {
      const float sv[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = 4 * q + e, p = p0 + i;
        uint32_t k = order_key(sv[e]);
        if (p < forced_lo || p >= forced_hi) k = 0xffffffffu;
        key[i] = k;
        if (WEIGHTED) wt[i] = (uint32_t)max(min(o[i + 1], N) - o[i], 0);
        if (p < P) valid |= 1u << i;
      }
    }
  }
  auto W = [&](int i) -> uint32_t { return WEIGHTED ? wt[i] : 1u; };
  // range of the keys below all-ones, weight of the all-ones keys, total weight
  uint32_t kmn = 0xffffffffu, kmx = 0u, wsum = 0u, wtop = 0u;
#pragma unroll
  for (int i = 0; i < KPT; ++i)
    if (valid >> i & 1u) {
      wsum += W(i);
      if (key[i] == 0xffffffffu) {
        wtop += W(i);
      } else {
        kmn = min(kmn, key[i]);
        kmx = max(kmx, key[i]);
      }
    }
  kmn = __reduce_min_sync(0xffffffffu, kmn);
  kmx = __reduce_max_sync(0xffffffffu, kmx);
  wsum = __reduce_add_sync(0xffffffffu, wsum);
  wtop = __reduce_add_sync(0xffffffffu, wtop);
  if (lane == 0) *reinterpret_cast<uint4*>(wred + 4 * warp) = make_uint4(kmn, kmx, wsum, wtop);
#pragma unroll
  for (int x = 0; x < 8; ++x)  // first pass's bins
    reinterpret_cast<uint4*>(H0)[tid + 128 * x] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();
  uint32_t gmin = 0xffffffffu, gmax = 0u, wall = 0u, wtop_all = 0u;
#pragma unroll
  for (int x = 0; x < kWarps; ++x) {
    const uint4 r = *reinterpret_cast<const uint4*>(wred + 4 * x);
    gmin = min(gmin, r.x);
    gmax = max(gmax, r.y);
    wall += r.z;
    wtop_all += r.w;
  }
  int32_t* sel_u = a.sel_idx + (size_t)u * a.max_sel;
  if (wall <= cap) {  // everything fits
    if (cand != nullptr) {
#pragma unroll
      for (int i = 0; i < KPT; ++i)
        if (valid >> i & 1u) cand[p0 + i] = cand_key(key[i], p0 + i);
      return;
    }
#pragma unroll
    for (int i = 0; i < KPT; ++i)
      if ((valid >> i & 1u) && p0 + i < a.max_sel) sel_u[p0 + i] = p0 + i;
    if (tid == 0) {
      if (P > a.max_sel) flag_status(a.status, SA_ERR_DEVICE_CHECK);
      a.sel_count[u] = min(P, a.max_sel);
    }
    return;
  }
  // ---- the cut
  uint32_t T, rem;
  if (wtop_all > cap) {
    T = 0xffffffffu;
    rem = cap;
  } else if (gmin == gmax || (!WEIGHTED && cap == wtop_all)) {
    T = gmax;  // with nothing left to spend, no key <= gmax is taken
    rem = cap - wtop_all;
  } else {
    rem = cap - wtop_all;
    int hi = 32 - __clz(gmin ^ gmax);  // bits [hi, 32) are common to [gmin, gmax]
    uint32_t prefix = hi == 32 ? 0u : (gmin >> hi) << hi;
    for (int pass = 0; hi > 0; ++pass) {
      // window = key bits [hi - 12, hi), or [0, hi) left-aligned in 12 bits
      const int sr = hi >= 12 ? hi - 12 : 0, sl = hi >= 12 ? 0 : 12 - hi;
      uint32_t* H = H0 + 4096 * (pass & 1);
      uint32_t* Hn = H0 + 4096 * ((pass & 1) ^ 1);
#pragma unroll
      for (int x = 0; x < KPT; ++x) {
        const bool in = (valid >> x & 1u) && (!WEIGHTED || W(x) != 0u) && key[x] != 0xffffffffu &&
                        (hi == 32 || ((key[x] ^ prefix) >> hi) == 0u);
        if (in) atomicAdd(&H[bin_slot(((key[x] >> sr) << sl) & 4095u)], W(x));
      }
      __syncthreads();
      {
        // row 127 - tid: its 8 chunks in an order that spreads a quarter-warp over the banks
        const uint4* row = reinterpret_cast<const uint4*>(H + 32 * (127 - tid));
        uint32_t sum = 0u;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 v = row[c ^ (tid & 7)];
          sum += v.x + v.y + v.z + v.w;
        }
        tsum[tid] = sum;
#pragma unroll
        for (int x = 0; x < 8; ++x)  // next pass's bins (last read a pass ago)
          reinterpret_cast<uint4*>(Hn)[tid + 128 * x] = make_uint4(0u, 0u, 0u, 0u);
      }
      __syncthreads();
      // every warp: the thread (row) holding the cut, then the bin inside it
      const uint4 t4 = *reinterpret_cast<const uint4*>(tsum + 4 * lane);  // threads 4l .. 4l+3
      const uint32_t s4 = t4.x + t4.y + t4.z + t4.w;
      uint32_t inc = s4;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
      }
      const int L = __ffs(__ballot_sync(0xffffffffu, inc > rem)) - 1;
      uint32_t above = __shfl_sync(0xffffffffu, inc - s4, L);
      const uint32_t tv[4] = {__shfl_sync(0xffffffffu, t4.x, L), __shfl_sync(0xffffffffu, t4.y, L),
                              __shfl_sync(0xffffffffu, t4.z, L), __shfl_sync(0xffffffffu, t4.w, L)};
      int tt = 4 * L + 3;
#pragma unroll
      for (int x = 0; x < 3; ++x) {
        if (above + tv[x] > rem) { tt = 4 * L + x; break; }
        above += tv[x];
      }
      const uint32_t bin = 32u * (uint32_t)(127 - tt) + (uint32_t)(31 - lane);  // descending
      const uint32_t hv = H[bin_slot(bin)];
      uint32_t binc = hv;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, binc, o);
        if (lane >= o) binc += y;
      }
      const int J = __ffs(__ballot_sync(0xffffffffu, above + binc > rem)) - 1;
      const uint32_t run = above + __shfl_sync(0xffffffffu, binc - hv, J);
      const uint32_t cb = 32u * (uint32_t)(127 - tt) + (uint32_t)(31 - J);
      rem -= run;
      if (hi >= 12) {
        prefix |= cb << sr;
        hi = sr;
      } else {
        prefix |= cb >> sl;
        hi = 0;
      }
      if (!WEIGHTED && rem == 0u && hi > 0 && (prefix | ((1u << hi) - 1u)) != 0xffffffffu) {
        prefix |= (1u << hi) - 1u;  // every key of the cut bin is below this T
        break;
      }
    }
    T = prefix;
  }
  // ---- kept pages: keys above T, keys equal to T in page order while the weight fits
  uint32_t keep = 0u, total, pos;
  if (!WEIGHTED) {
    uint32_t gt = 0u, eqc = 0u;
#pragma unroll
    for (int i = 0; i < KPT; ++i)
      if (valid >> i & 1u) {
        gt += key[i] > T ? 1u : 0u;
        eqc += key[i] == T ? 1u : 0u;
      }
    uint32_t tot2;
    const uint32_t ex = block_excl_scan((gt << 16) | eqc, S.scan, tot2);  // both < 2^16
    uint32_t eq = ex & 0xffffu;
#pragma unroll
    for (int i = 0; i < KPT; ++i) {
      if (!(valid >> i & 1u)) continue;
      bool k = key[i] > T;
      if (key[i] == T) k = ++eq <= rem;
      if (k) keep |= 1u << i;
    }
    pos = (ex >> 16) + min(ex & 0xffffu, rem);
    total = (tot2 >> 16) + min(tot2 & 0xffffu, rem);
  } else {
    uint32_t eqw = 0u;
#pragma unroll
    for (int i = 0; i < KPT; ++i)
      if ((valid >> i & 1u) && key[i] == T) eqw += W(i);
    uint32_t dummy;
    uint32_t eq = block_excl_scan(eqw, S.scan, dummy);
#pragma unroll
    for (int i = 0; i < KPT; ++i) {
      if (!(valid >> i & 1u)) continue;
      bool k = key[i] > T;
      if (key[i] == T) {
        eq += W(i);
        k = eq <= rem;
      }
      if (k) keep |= 1u << i;
    }
    pos = block_excl_scan((uint32_t)__popc(keep), S.scan, total);
  }
  if (cand != nullptr) {
#pragma unroll
    for (int i = 0; i < KPT; ++i)
      if (keep >> i & 1u) cand[pos++] = cand_key(key[i], p0 + i);
    return;
  }
#pragma unroll
  for (int i = 0; i < KPT; ++i)
    if (keep >> i & 1u) {
      if (pos < (uint32_t)a.max_sel) sel_u[pos] = p0 + i;
      ++pos;
    }
  if (tid == 0) {
    if (total > (uint32_t)a.max_sel) flag_status(a.status, SA_ERR_DEVICE_CHECK);
    a.sel_count[u] = (int32_t)min(total, (uint32_t)a.max_sel);
  }
}

// Selection of unit u from its scores -- in the workspace, or at sc_local in
// this CTA's shared memory (16-byte aligned, rows padded to 4): writes
// sel_idx (ascending page order) and sel_count.  All threads of the CTA call it.
SA_DEV void select_unit(const SelectArgs& a, const int u, const int b, const int N, const int P,
                        const SelSmem& S, const float* sc_local = nullptr) {
  const bool weighted = a.budget_kind == SA_BUDGET_TOKENS;
  const int32_t* off = weighted ? a.kv.chunk_off + (size_t)b * (a.kv.max_pages + 1) : nullptr;
  int forced_lo = 0, forced_hi = P;  // pages < forced_lo or >= forced_hi are forced (ratio)
  uint32_t cap;
  if (a.budget_kind == SA_BUDGET_TOPK) {
    cap = (uint32_t)min(a.top_k, P);
  } else if (a.budget_kind == SA_BUDGET_RATIO) {
    const long long fl = (long long)floor((double)P * a.ratio);
    long long K = (long long)a.topk_val + a.bos + a.eos;
    if (fl > K) K = fl;
    if (K > P) K = P;
    cap = (uint32_t)K;
    forced_lo = min(a.bos, P);
    forced_hi = max(0, P - a.eos);
  } else {
    cap = (uint32_t)max(a.token_budget, 0);
  }
  if (P <= 16 * kThreads) {
    if (weighted)
      select_unit_regs<16, true>(a, u, N, P, cap, forced_lo, forced_hi, off, S, sc_local);
    else
      select_unit_regs<16, false>(a, u, N, P, cap, forced_lo, forced_hi, off, S, sc_local);
  } else
    select_unit_smem(a, u, N, P, cap, forced_lo, forced_hi, off, S, sc_local);
}

// Tokens N and pages (or chunks) P of sequence b; false (and P = 0) when
// they are out of range.
SA_DEV bool unit_geometry(const SelectArgs& a, const int b, int& N, int& P) {
  N = a.kv.seq_len[b];
  bool bad = (N < 1 || N > a.kv.cap);
  if (a.kv.page_size > 0) {
    P = bad ? 0 : (N + a.kv.page_size - 1) / a.kv.page_size;
  } else {
    P = a.kv.n_chunks[b];
    bad = bad || P < 1;
  }
  if (P > a.kv.max_pages) bad = true;
  if (bad) P = 0;
  return !bad;
}

// Selection of unit u (sequence, KV head) from the group scores its scoring
// items wrote (at sc_local in shared memory, or in the workspace); the caller
// has made them visible to this CTA.
// units_per_seq: units of one sequence (Hkv, or Hq for per-query-head units).
SA_DEV void select_unit_of(const SelectArgs& a, const int u, const SelSmem& S, const float* sc_local,
                           const int units_per_seq) {
  const int b = u / units_per_seq;
  int N, P;
  unit_geometry(a, b, N, P);  // a bad geometry was flagged by the scoring
  select_unit(a, u, b, N, P, S, sc_local);
}

// The union of the page sets that the G query heads of KV unit kvu selected
// (rows b * Hq + g * G + j of sel_idx / sel_count, written earlier in the
// launch and made visible to this CTA), with bit j of an entry's mask set
// when head j kept the page: written to union_idx / union_mask in ascending
// page order; returns the entry count (also stored in union_count).  Every
// page is then streamed once for all the heads that kept it.  All threads
// call it; `words` holds ceil(P / 4) words of shared memory.
SA_DEV int build_union(const SelectArgs& a, const int kvu, const int P, uint32_t* words, uint32_t* scan) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int b = kvu / a.kv.Hkv, g = kvu - b * a.kv.Hkv;
  const int nw = (P + 3) >> 2;
  for (int i = tid; i < nw; i += nt) words[i] = 0u;
  __syncthreads();
  for (int j = 0; j < a.G; ++j) {
    const int u = b * a.Hq + g * a.G + j;
    const int n = min(__ldcg(a.sel_count + u), a.max_sel);
    const int32_t* lst = a.sel_idx + (size_t)u * a.max_sel;
    for (int e = tid; e < n; e += nt) {
      const int p = __ldcg(lst + e);
      if (p >= 0 && p < P) atomicOr(&words[p >> 2], (1u << j) << (8 * (p & 3)));
    }
  }
  __syncthreads();
  // compaction in page order: thread t takes pages [t per, (t + 1) per)
  const int per = (P + nt - 1) / nt;
  const int p0 = min(P, tid * per), p1 = min(P, p0 + per);
  const uint8_t* m8 = reinterpret_cast<const uint8_t*>(words);
  uint32_t cnt = 0;
  for (int p = p0; p < p1; ++p) cnt += m8[p] ? 1u : 0u;
  uint32_t total;
  uint32_t pos = block_excl_scan(cnt, scan, total);
  int32_t* uidx = a.union_idx + (size_t)kvu * a.kv.max_pages;
  uint8_t* umask = a.union_mask + (size_t)kvu * a.kv.max_pages;
  for (int p = p0; p < p1; ++p)
    if (m8[p]) {
      uidx[pos] = p;
      umask[pos] = m8[p];
      ++pos;
    }
  if (tid == 0) a.union_count[kvu] = (int)total;
  return (int)total;
}

// FUSED (the decode step): refresh the newest page while scoring and publish
// the unit's flag after selecting.
// SCORE_ONLY: write the group scores and stop (no selection; the unit
// counters are not touched).
// score_dst (non-null): where the unit's group scores go, indexed by page
// (another CTA's shared memory, say), instead of the workspace.
// HEAD_ROWS (with SCORE_ONLY, per (sequence, KV head) units): the G query
// heads' own scores go to their rows b * Hq + h of the workspace (no group
// max), and the item then counts itself done in a.kv_scored[u] (release).
// CL_WAIT (a cluster launch whose CTAs arrived on the cluster barrier after
// setting up): each thread waits on that barrier before its first store to
// score_dst (another CTA's shared memory, which must be running), or at the
// end if it stores none -- once the first tile is scored, so the wait
// overlaps the first metadata load.
template <int RULE, bool FUSED, bool PER_HEAD = false, bool SCORE_ONLY = false, bool HEAD_ROWS = false,
          bool CL_WAIT = false>
SA_DEV void select_item(const SelectArgs& a, const int u, const int split, const SelSmem& S,
                        WarpState& ws, float* score_dst = nullptr) {
  static_assert(!HEAD_ROWS || (SCORE_ONLY && !PER_HEAD), "head rows: score-only items of KV units");
  static_assert(!CL_WAIT || (SCORE_ONLY && !HEAD_ROWS), "cluster wait: score-only items");
  bool cl_waited = !CL_WAIT;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, c = lane & 3;
  const int Hkv = a.kv.Hkv;
  const UnitMap um = unit_map<PER_HEAD>(u, Hkv, a.Hq, a.G);
  const int b = um.b, kvu = um.kvu;
  // per-query-head units share their KV head's metadata, cache rows and the
  // newest-page refresh: one of them (the first head of the group) stores
  // what is shared, every one patches its own staged copy
  const bool kv_owner = !PER_HEAD || um.h0 % a.G == 0;

  // ---- unit geometry (every CTA of the unit computes the same values)
  int N, P;
  if (!unit_geometry(a, b, N, P) && tid == 0 && split == 0) flag_status(a.status, SA_ERR_DEVICE_CHECK);
  const int TP = (P + 15) >> 4;
  const int t_begin = (int)(((long long)TP * split) / a.splits);
  const int t_end = (int)(((long long)TP * (split + 1)) / a.splits);

  // ---- B fragments: the unit's query heads (columns >= n_heads are zero)
  const bool head_ok = gq < um.n_heads;
  const __nv_bfloat16* qrow = reinterpret_cast<const __nv_bfloat16*>(a.q) +
                              ((size_t)b * a.Hq + (size_t)um.h0 + (head_ok ? gq : 0)) * kHeadDim;
  uint32_t bq[RULE == 0 ? 32 : 1];
  double bd[RULE == 0 ? 1 : 32];
  if (RULE == 0) {
    // k-step ks covers row elements 16ks .. 16ks + 15 of [kmin | kmax];
    // the paired query vector is [q- | q+] (natural order)
#pragma unroll
    for (int ks = 0; ks < 16; ++ks) {
      const int e = 16 * (ks & 7) + 2 * c;
      uint32_t lo = head_ok ? __ldg(reinterpret_cast<const uint32_t*>(qrow + e)) : 0u;
      uint32_t hi = head_ok ? __ldg(reinterpret_cast<const uint32_t*>(qrow + e + 8)) : 0u;
      if (ks < 8) { lo = bf16x2_neg_part(lo); hi = bf16x2_neg_part(hi); }
      else        { lo = bf16x2_pos_part(lo); hi = bf16x2_pos_part(hi); }
      bq[2 * ks] = lo;
      bq[2 * ks + 1] = hi;
    }
  } else {
    // k-step (box bx, chunk j): lane c holds dimension 32 bx + 4 j + c
#pragma unroll
    for (int bx = 0; bx < 4; ++bx)
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int e = 32 * bx + 4 * j + c;
        bd[8 * bx + j] = head_ok ? (double)__bfloat162float(qrow[e]) : 0.0;
      }
  }

  // ---- scoring: warp w takes tiles t_begin + w, + 4, ...
  float* sc_u = score_dst ? score_dst : a.ws_scores + (size_t)u * a.ws_stride;
  float* out_u = a.scores_out ? a.scores_out + (size_t)u * a.kv.max_pages : nullptr;
  unsigned char* ring = S.ring + warp * (kStages * kTileBytes);
  uint64_t* bars = S.bars + warp * kStages;
  const int row_base = kvu * a.kv.max_pages;
  const int lrow = (lane & 7) + 8 * ((lane >> 3) & 1);  // ldmatrix: rows 0-7 / 8-15
  const int lchk = lane >> 4;                            //            chunk +0 / +1
  const int nt = t_end - t_begin;
  const int n_it = max(0, (nt - warp + kWarps - 1) / kWarps);

  auto issue = [&](int it) {  // lane 0 only
    const uint32_t g_it = ws.gi + (uint32_t)it;
    uint64_t* bar = bars + g_it % kStages;
    unsigned char* st = ring + (g_it % kStages) * kTileBytes;
    const int y = row_base + 16 * (t_begin + warp + it * kWarps);
    mbar_arrive_expect_tx(bar, kTileBytes);
    const int xs = RULE == 0 ? 64 : 32;  // elements per 128-byte box row
#pragma unroll
    for (int bx = 0; bx < 4; ++bx) tma_load_2d(st + bx * kBoxBytes, &a.tmap_meta, bx * xs, y, bar);
  };

  int issued = 0;
  if (ws.alive) {
    issued = min(n_it, kStages - 1);
    if (lane == 0)
      for (int it = 0; it < issued; ++it) issue(it);
  }

  // ---- page of the newest token, when this call refreshes it: rows [r_s, r_e)
  int p_new = -1, r_s = 0, r_e = 0;
  if (FUSED && P > 0) {
    if (a.kv.page_size > 0) {
      p_new = P - 1;
      r_s = p_new * a.kv.page_size;
      r_e = min(r_s + a.kv.page_size, N);
    } else {
      const int32_t* off = a.kv.chunk_off + (size_t)b * (a.kv.max_pages + 1);
      p_new = off[P - 1] <= N - 1 ? P - 1 : chunk_containing(off, P, N - 1);
      r_s = off[p_new];
      const int e_raw = off[p_new + 1];
      if (r_s < 0 || e_raw < r_s) {
        if (tid == 0 && split == 0) flag_status(a.status, SA_ERR_DEVICE_CHECK);
        p_new = -1;
      } else {
        r_e = min(e_raw, N);  // a chunk table may run ahead of the cache: clip to N
        if (r_s >= r_e) p_new = -1;
      }
    }
  }
  const int t_new = p_new >= 0 ? (p_new >> 4) : -1;
  if (t_new >= t_begin && t_new < t_end && (t_new - t_begin) % kWarps == warp && ws.alive) {
    // the warp that will refresh the newest page starts pulling its key rows
    // into L2 while the metadata tiles land (with few units the refresh is on
    // the critical path of the launch)
    const char* k0 = static_cast<const char*>(a.kv.k) + ((size_t)kvu * a.kv.cap + (size_t)r_s) * (2 * kHeadDim);
    for (int i = lane; i < 2 * (r_e - r_s); i += 32) prefetch_l2(k0 + (size_t)i * 128);
  }

  for (int it = 0; it < n_it && ws.alive; ++it) {
    __syncwarp();
    if (it + kStages - 1 < n_it) {
      if (lane == 0) issue(it + kStages - 1);
      issued = it + kStages;
    }
    const uint32_t g_it = ws.gi + (uint32_t)it;
    if (!mbar_wait(bars + g_it % kStages, (g_it / kStages) & 1u, a.status)) {
      ws.alive = false;
      ws.drain_lo = g_it;
      ws.drain_hi = ws.gi + (uint32_t)issued;
      break;
    }
    unsigned char* st = ring + (g_it % kStages) * kTileBytes;
    const int t = t_begin + warp + it * kWarps;
    if (t == t_new) {
      // with append: store the newest key and value at row N - 1 (lane l
      // owns elements 4l .. 4l + 3), and use the key without reading it back
      const bool app = a.k_new != nullptr;
      uint2 knew = make_uint2(0u, 0u);
      if (app) {
        const size_t src = (size_t)kvu * kHeadDim + lane * 4;
        knew = __ldg(reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(a.k_new) + src));
        if (kv_owner) {
          const size_t dst = ((size_t)kvu * a.kv.cap + (size_t)(N - 1)) * kHeadDim + lane * 4;
          const uint2 vnew = __ldg(reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(a.v_new) + src));
          *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.k_dst) + dst) = knew;
          *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.v_dst) + dst) = vnew;
          fence_proxy_async_global();  // the decode items read the row with TMA
        }
      }
      // rebuild the newest page's metadata, store it, patch the staged row
      const __nv_bfloat16* k_lane = reinterpret_cast<const __nv_bfloat16*>(a.kv.k) +
                                    ((size_t)kvu * a.kv.cap) * kHeadDim + lane * 4;
      const PageMetaLane m = page_meta_lane<RULE>(k_lane, r_s, r_e, app, knew);
      if (kv_owner)
        store_page_meta<RULE>(a.meta_refresh + ((size_t)kvu * a.kv.max_pages + p_new) * kMetaBytes, m, lane);
      const int r = p_new & 15;
      if (RULE == 0) {
        const uint32_t o = swz128(r, (lane & 15) >> 1) + 8 * (lane & 1);
        *reinterpret_cast<uint2*>(st + (lane >> 4) * kBoxBytes + o) = m.lo;
        *reinterpret_cast<uint2*>(st + (2 + (lane >> 4)) * kBoxBytes + o) = m.hi;
      } else {
        *reinterpret_cast<float4*>(st + (lane >> 3) * kBoxBytes + swz128(r, lane & 7)) = m.mean;
      }
      fence_proxy_async();  // generic writes to the stage before its next TMA refill
      __syncwarp();
    }
    float acc[4];
    if (RULE == 0) {
      float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < 16; ++ks) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(a0, a1, a2, a3, st + (ks >> 2) * kBoxBytes + swz128(lrow, 2 * (ks & 3) + lchk));
        if (ks & 1) mma_bf16(s1, a0, a1, a2, a3, bq[2 * ks], bq[2 * ks + 1]);
        else        mma_bf16(s0, a0, a1, a2, a3, bq[2 * ks], bq[2 * ks + 1]);
      }
#pragma unroll
      for (int x = 0; x < 4; ++x) acc[x] = s0[x] + s1[x];
    } else {
      // FP64 tensor cores: exact products and sums, one final rounding
      double c00 = 0.0, c01 = 0.0, c10 = 0.0, c11 = 0.0;  // pages gq / gq + 8
#pragma unroll
      for (int bx = 0; bx < 4; ++bx)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float x0 = *reinterpret_cast<const float*>(st + bx * kBoxBytes + swz128(gq, j) + 4 * c);
          const float x1 = *reinterpret_cast<const float*>(st + bx * kBoxBytes + swz128(gq + 8, j) + 4 * c);
          const double bv = bd[8 * bx + j];
          mma_f64(c00, c01, (double)x0, bv);
          mma_f64(c10, c11, (double)x1, bv);
        }
      acc[0] = (float)c00; acc[1] = (float)c01; acc[2] = (float)c10; acc[3] = (float)c11;
    }
    const float ninf = -__int_as_float(0x7f800000);
    const bool c0 = 2 * c < um.n_heads, c1 = 2 * c + 1 < um.n_heads;
    if (HEAD_ROWS) {
      // lane (gq, c) holds heads 2c, 2c + 1 of pages gq and gq + 8
      const int pg0 = t * 16 + gq, pg1 = pg0 + 8;
      float* row = a.ws_scores + ((size_t)b * a.Hq + (size_t)um.h0 + 2 * c) * a.ws_stride;
      if (c0) {
        if (pg0 < P) row[pg0] = acc[0];
        if (pg1 < P) row[pg1] = acc[2];
      }
      if (c1) {
        if (pg0 < P) row[a.ws_stride + pg0] = acc[1];
        if (pg1 < P) row[a.ws_stride + pg1] = acc[3];
      }
      continue;
    }
    float mlo = fmaxf(c0 ? acc[0] : ninf, c1 ? acc[1] : ninf);
    float mhi = fmaxf(c0 ? acc[2] : ninf, c1 ? acc[3] : ninf);
    mlo = fmaxf(mlo, __shfl_xor_sync(0xffffffffu, mlo, 1));
    mlo = fmaxf(mlo, __shfl_xor_sync(0xffffffffu, mlo, 2));
    mhi = fmaxf(mhi, __shfl_xor_sync(0xffffffffu, mhi, 1));
    mhi = fmaxf(mhi, __shfl_xor_sync(0xffffffffu, mhi, 2));
    if (!cl_waited) {
      cluster_wait();
      cl_waited = true;
    }
    if (c < 2) {
      const int page = t * 16 + gq + 8 * c;
      const float s = c == 0 ? mlo : mhi;
      if (page < P) {
        sc_u[page] = s;
        if (out_u) out_u[page] = s;
      }
    }
  }
  ws.gi += (uint32_t)n_it;
  if (!cl_waited) cluster_wait();
  if (HEAD_ROWS) {
    __syncthreads();  // then one acq_rel increment publishes the CTA's score rows
    if (tid == 0) atom_add_acq_rel_u32(&a.kv_scored[u], 1u);
  }
  if (SCORE_ONLY) return;

  // ---- the last CTA of the unit selects (its counter increment is acq_rel:
  // it publishes this CTA's scores and acquires those of the other splits)
  __syncthreads();
  if (a.splits > 1) {
    if (tid == 0) {
      const uint32_t prev = atom_add_acq_rel_u32(&a.ws_count[u], 1u);
      *S.last = (prev == (uint32_t)(a.splits - 1));
    }
    __syncthreads();
    if (!*S.last) return;
  }
  if (tid == 0 && a.splits > 1 && !FUSED) a.ws_count[u] = 0;  // ready for the next call
  select_unit(a, u, b, N, P, S);
  if (FUSED) {
    __syncthreads();
    // the flag carries the kept count too (thread 0 wrote it), so a decode
    // item reads both with its one acquire
    if (tid == 0 && a.hold_flag_of != u + 1)
      st_release_u32(&a.ws_count[u], kUnitSelected | (uint32_t)a.sel_count[u]);
  }
}

}  // namespace sel
}  // namespace sa
