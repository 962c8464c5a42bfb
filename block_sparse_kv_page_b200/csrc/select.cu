// Fused page scoring + budgeted top-k selection for GQA decode.
//
// "Sparse Attention for Web Agents -- Offline Replay Records", section "The
// comparison": each chunk is scored against the current query (envelope =
// per-dimension min/max upper bound; centroid = mean key) and the best ones
// are kept, the budget being page_size x top_k attended tokens; TSA fills a
// token budget over variable chunks.  "WebArena 0-99 Sparse-Attention Method
// Comparison", section "Method configurations at a glance": ratio budget
// max(topk_val + bos + eos, int(blocks * ratio)) with forced bos/eos blocks.
//
// Work split.  A unit is one (sequence, KV head).  Its pages are cut into
// `splits` contiguous ranges of 16-page tiles; an item is one (unit, range).
// A persistent grid pulls items from an atomic queue.  Each of a CTA's 4
// warps streams its tiles of 16 metadata rows (512 B each) through a private
// 3-stage cp.async ring (every load instruction covers whole 32-byte sectors)
// and scores them for all G grouped query heads with tensor-core products:
//   envelope: S^T[16 pages x 8 heads] = [kmin | kmax] (16 x 256, bf16)
//             x [q- | q+]^T (256 x 8, bf16), m16n8k16, exact products;
//   centroid: S^T = kmean (16 x 128, fp32) x q^T (128 x 8, bf16), on the
//             FP64 tensor cores (m8n8k4): exact products and sums, one final
//             rounding to fp32, so near-ties are resolved as in float64.
// The group score (max over the G heads) goes to the workspace.  The CTA that
// finishes a unit last (atomic counter; nobody waits) loads the unit's scores
// and selects: a weighted MSB-first radix select on order-preserving 32-bit
// keys finds the cut key T and the capacity left for keys equal to T; equal
// keys are then taken in ascending page order (the lowest-index tie rule), so
// the result is exactly "the longest prefix of the (score desc, index asc)
// order within the budget".  Weight 1 per page gives top-k / ratio; weight =
// chunk length gives the token budget.  Output is the kept set in ascending
// page order.
#include "common.cuh"
#include "internal.h"

namespace sa {
namespace {

#ifndef SA_SEL_ITEM_PAGES
#define SA_SEL_ITEM_PAGES 256
#endif
#ifndef SA_SEL_CTAS_PER_SM
#define SA_SEL_CTAS_PER_SM 2
#endif

constexpr int kSelWarps = 4;
constexpr int kSelThreads = kSelWarps * 32;
constexpr int kSelStages = 3;
constexpr int kSlotBytes = 32 * 16;              // one 16-byte chunk per lane
constexpr int kStageBytes = 16 * kSlotBytes;     // 16 chunks per lane = 16 rows x 512 B
constexpr int kRingBytes = kSelWarps * kSelStages * kStageBytes;

// Byte offset, inside a 512-byte metadata row, of the j-th chunk lane c loads.
template <int RULE>
SA_DEV int chunk_byte(int j, int c) {
  if (RULE == 0) return 16 * (4 * j + c);                 // bf16: elements 32j + 8c .. +8
  return 16 * (8 * (j >> 1) + 4 * (j & 1) + c);          // fp32: floats 32(j/2) + 16(j&1) + 4c .. +4
}

struct RadixCut {
  uint32_t T;
  uint32_t rem;
};

// Weighted radix select on keys[0..P): the key T such that the total weight of
// keys > T is <= cap < total weight of keys >= T, and rem = cap - weight(> T).
// Requires total weight > cap.
SA_DEV RadixCut radix_cut(const uint32_t* keys, const uint32_t* wts, int P, uint32_t cap,
                          uint32_t* hist, uint32_t* bc) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nt = blockDim.x;
  uint32_t prefix = 0, mask = 0, rem = cap;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = tid; i < 256; i += nt) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < P; i += nt) {
      const uint32_t k = keys[i];
      if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], wts ? wts[i] : 1u);
    }
    __syncthreads();
    if (warp == 0) {
      uint32_t h[8], ls = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        h[q] = hist[255 - 8 * lane - q];
        ls += h[q];
      }
      uint32_t inc = ls;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
      }
      const unsigned ball = __ballot_sync(0xffffffffu, inc > rem);
      const int L = __ffs(ball) - 1;
      if (lane == L) {
        uint32_t run = inc - ls;
        int d = 255 - 8 * lane - 7;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (run + h[q] > rem) {
            d = 255 - 8 * lane - q;
            break;
          }
          run += h[q];
        }
        bc[0] = (uint32_t)d;
        bc[1] = run;
      }
    }
    __syncthreads();
    const uint32_t d = bc[0];
    rem -= bc[1];
    prefix |= d << shift;
    mask |= 0xffu << shift;
    __syncthreads();
  }
  return {prefix, rem};
}

struct SelSmem {
  unsigned char* smem;   // max(ring, 8 * max_pages) bytes
  uint32_t* hist;        // 256
  uint32_t* scan;        // 32
  uint32_t* bc;          // 4
  int* last;
};

template <int RULE>
SA_DEV void select_item(const SelectArgs& a, const int u, const int split, const SelSmem& S) {
  unsigned char* smem = S.smem;
  uint32_t* s_hist = S.hist;
  uint32_t* s_scan = S.scan;
  uint32_t* s_bc = S.bc;
  int& s_last = *S.last;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, c = lane & 3;
  const int Hkv = a.kv.Hkv;
  const int b = u / Hkv, g = u % Hkv;

  // ---- unit geometry (every CTA of the unit computes the same values)
  const int N = a.kv.seq_len[b];
  int P;
  bool bad = (N < 1 || N > a.kv.cap);
  if (a.kv.page_size > 0) {
    P = bad ? 0 : (N + a.kv.page_size - 1) / a.kv.page_size;
  } else {
    P = a.kv.n_chunks[b];
    bad = bad || P < 1;
  }
  if (P > a.kv.max_pages) bad = true;
  if (bad) {
    P = 0;
    if (tid == 0 && split == 0) flag_status(a.status, SA_ERR_DEVICE_CHECK);
  }
  const int TP = (P + 15) >> 4;
  const int t_begin = (int)(((long long)TP * split) / a.splits);
  const int t_end = (int)(((long long)TP * (split + 1)) / a.splits);

  // ---- B fragments: the G query heads of this KV group (columns >= G are zero)
  const bool head_ok = gq < a.G;
  const __nv_bfloat16* qrow = reinterpret_cast<const __nv_bfloat16*>(a.q) +
                              ((size_t)b * a.Hq + (size_t)g * a.G + (head_ok ? gq : 0)) * kHeadDim;
  uint32_t bq[RULE == 0 ? 32 : 1];
  double bd[RULE == 0 ? 1 : 32];
  if (RULE == 0) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint4 v = head_ok ? ldg_nc128(qrow + 32 * (j & 3) + 8 * c) : make_uint4(0, 0, 0, 0);
      if (j < 4) {  // paired with kmin: q-
        v.x = bf16x2_neg_part(v.x); v.y = bf16x2_neg_part(v.y);
        v.z = bf16x2_neg_part(v.z); v.w = bf16x2_neg_part(v.w);
      } else {      // paired with kmax: q+
        v.x = bf16x2_pos_part(v.x); v.y = bf16x2_pos_part(v.y);
        v.z = bf16x2_pos_part(v.z); v.w = bf16x2_pos_part(v.w);
      }
      bq[4 * j + 0] = v.x; bq[4 * j + 1] = v.y; bq[4 * j + 2] = v.z; bq[4 * j + 3] = v.w;
    }
  } else {
    // bd[8i + 4h + r] = q[head][32i + 16h + 4c + r] as fp64: the same dimensions
    // as the metadata chunk (i, h) this lane loads (k-step (2i + h, r))
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint2 v = make_uint2(0, 0);
        if (head_ok) v = __ldg(reinterpret_cast<const uint2*>(qrow + 32 * i + 16 * hh + 4 * c));
        bd[8 * i + 4 * hh + 0] = (double)bf16_lo(v.x);
        bd[8 * i + 4 * hh + 1] = (double)bf16_hi(v.x);
        bd[8 * i + 4 * hh + 2] = (double)bf16_lo(v.y);
        bd[8 * i + 4 * hh + 3] = (double)bf16_hi(v.y);
      }
    }
  }

  // ---- scoring: warp w takes tiles t_begin + w, + 4, ...
  unsigned char* ring = smem + warp * (kSelStages * kStageBytes);
  const unsigned char* meta_u =
      reinterpret_cast<const unsigned char*>(a.meta) + (size_t)u * a.kv.max_pages * kMetaBytes;
  float* sc_u = a.ws_scores + (size_t)u * a.kv.max_pages;
  float* out_u = a.scores_out ? a.scores_out + (size_t)u * a.kv.max_pages : nullptr;

  auto issue = [&](int it) {
    const int t = t_begin + warp + it * kSelWarps;
    if (t < t_end) {
      unsigned char* st = ring + (it % kSelStages) * kStageBytes;
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int page = t * 16 + gq + 8 * r;
        const bool ok = page < P;
        const unsigned char* src = meta_u + (size_t)(ok ? page : 0) * kMetaBytes;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          cp_async16(st + (r * 8 + j) * kSlotBytes + lane * 16, src + chunk_byte<RULE>(j, c), ok);
      }
    }
    cp_async_commit();
  };

  const int n_it = (t_end - t_begin - warp + kSelWarps - 1) / kSelWarps;
#pragma unroll
  for (int it = 0; it < kSelStages - 1; ++it) issue(it);
  for (int it = 0; it < n_it; ++it) {
    cp_async_wait<kSelStages - 2>();
    issue(it + kSelStages - 1);
    const unsigned char* st = ring + (it % kSelStages) * kStageBytes + lane * 16;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (RULE == 0) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint4 lo = lds128(st + j * kSlotBytes);
        const uint4 hi = lds128(st + (8 + j) * kSlotBytes);
        mma_bf16(acc, lo.x, hi.x, lo.y, hi.y, bq[4 * j + 0], bq[4 * j + 1]);
        mma_bf16(acc, lo.z, hi.z, lo.w, hi.w, bq[4 * j + 2], bq[4 * j + 3]);
      }
    } else {
      // Centroid on the FP64 tensor cores: fp32 kmean and bf16 q are exact in
      // fp64, so the only rounding left is the final fp64 -> fp32 of the score.
      double c00 = 0.0, c01 = 0.0, c10 = 0.0, c11 = 0.0;  // pages gq / gq + 8
#pragma unroll
      for (int j = 0; j < 8; ++j) {  // chunk j = floats 32(j/2) + 16(j&1) + 4c .. +4
        const uint4 r0 = lds128(st + j * kSlotBytes);
        const uint4 r1 = lds128(st + (8 + j) * kSlotBytes);
        const uint32_t a0[4] = {r0.x, r0.y, r0.z, r0.w}, a1[4] = {r1.x, r1.y, r1.z, r1.w};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const double b = bd[8 * (j >> 1) + 4 * (j & 1) + r];
          mma_f64(c00, c01, (double)__uint_as_float(a0[r]), b);
          mma_f64(c10, c11, (double)__uint_as_float(a1[r]), b);
        }
      }
      acc[0] = (float)c00; acc[1] = (float)c01; acc[2] = (float)c10; acc[3] = (float)c11;
    }
    const float ninf = -__int_as_float(0x7f800000);
    const bool c0 = 2 * c < a.G, c1 = 2 * c + 1 < a.G;
    float mlo = fmaxf(c0 ? acc[0] : ninf, c1 ? acc[1] : ninf);
    float mhi = fmaxf(c0 ? acc[2] : ninf, c1 ? acc[3] : ninf);
    mlo = fmaxf(mlo, __shfl_xor_sync(0xffffffffu, mlo, 1));
    mlo = fmaxf(mlo, __shfl_xor_sync(0xffffffffu, mlo, 2));
    mhi = fmaxf(mhi, __shfl_xor_sync(0xffffffffu, mhi, 1));
    mhi = fmaxf(mhi, __shfl_xor_sync(0xffffffffu, mhi, 2));
    const int t = t_begin + warp + it * kSelWarps;
    if (c < 2) {
      const int page = t * 16 + gq + 8 * c;
      const float s = c == 0 ? mlo : mhi;
      if (page < P) {
        sc_u[page] = s;
        if (out_u) out_u[page] = s;
      }
    }
  }
  cp_async_wait<0>();

  // ---- the last CTA of the unit selects
  __syncthreads();
  if (a.splits > 1) {
    __threadfence();
    if (tid == 0) {
      const uint32_t prev = atomicAdd(&a.ws_count[u], 1u);
      s_last = (prev == (uint32_t)(a.splits - 1));
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
  }
  if (tid == 0 && a.splits > 1) a.ws_count[u] = 0;  // ready for the next call

  uint32_t* keys = reinterpret_cast<uint32_t*>(smem);
  uint32_t* wts = keys + a.kv.max_pages;
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
  uint32_t wall_local = 0;
  for (int p = tid; p < P; p += blockDim.x) {
    const float s = __ldcg(sc_u + p);
    uint32_t key = order_key(s);
    if (p < forced_lo || p >= forced_hi) key = 0xffffffffu;
    keys[p] = key;
    if (weighted) {
      const int L = min(off[p + 1], N) - off[p];
      wts[p] = (uint32_t)max(L, 0);
      wall_local += (uint32_t)max(L, 0);
    } else {
      wall_local += 1u;
    }
  }
  uint32_t wall;
  block_excl_scan(wall_local, s_scan, wall);  // includes a __syncthreads

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
  const RadixCut cut = radix_cut(keys, weighted ? wts : nullptr, P, cap, s_hist, s_bc);

  const int per = (P + blockDim.x - 1) / blockDim.x;
  const int i0 = min(P, tid * per), i1 = min(P, i0 + per);
  uint32_t eqw = 0;
  for (int i = i0; i < i1; ++i)
    if (keys[i] == cut.T) eqw += weighted ? wts[i] : 1u;
  uint32_t dummy;
  const uint32_t eq0 = block_excl_scan(eqw, s_scan, dummy);
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
  uint32_t pos = block_excl_scan(cnt, s_scan, total);
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

template <int RULE>
__global__ void __launch_bounds__(kSelThreads) select_kernel(SelectArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ uint32_t s_hist[256];
  __shared__ uint32_t s_scan[32];
  __shared__ uint32_t s_bc[4];
  __shared__ int s_last, s_item;
  const SelSmem S{smem, s_hist, s_scan, s_bc, &s_last};
  const int n_items = a.kv.B * a.kv.Hkv * a.splits;
  for (;;) {
    if (threadIdx.x == 0) s_item = (int)atomicAdd(&a.ws_queue[0], 1u);
    __syncthreads();
    const int item = s_item;
    if (item >= n_items) break;
    select_item<RULE>(a, item / a.splits, item % a.splits, S);
    __syncthreads();
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
// items per SM when there are few units, and at least one tile per warp.
int select_splits(int units, int max_pages, int sm_count) {
  int s = (max_pages + SA_SEL_ITEM_PAGES - 1) / SA_SEL_ITEM_PAGES;
  const int fill = (2 * sm_count + units - 1) / units;
  if (fill > s) s = fill;
  const int cap = (max_pages + 16 * kSelWarps - 1) / (16 * kSelWarps);
  if (s > cap) s = cap;
  if (s > 256) s = 256;
  if (s < 1) s = 1;
  return s;
}

size_t select_smem_bytes(int max_pages) {
  const size_t keys = (size_t)max_pages * 8;
  return keys > (size_t)kRingBytes ? keys : (size_t)kRingBytes;
}

cudaError_t launch_select(const SelectArgs& a, cudaStream_t st) {
  const size_t smem = select_smem_bytes(a.kv.max_pages);
  const long long items = (long long)a.kv.B * a.kv.Hkv * a.splits;
  if (items > 0x7fffffffLL) return cudaErrorInvalidValue;
  const int ctas_per_sm = smem <= (size_t)kRingBytes ? SA_SEL_CTAS_PER_SM : 1;
  long long grid = (long long)device_sm_count() * ctas_per_sm;
  if (grid > items) grid = items;
  cudaError_t e;
  if (a.rule == 0) {
    e = set_smem_attr((const void*)select_kernel<0>, smem);
    if (e != cudaSuccess) return e;
    select_kernel<0><<<(unsigned)grid, kSelThreads, smem, st>>>(a);
  } else {
    e = set_smem_attr((const void*)select_kernel<1>, smem);
    if (e != cudaSuccess) return e;
    select_kernel<1><<<(unsigned)grid, kSelThreads, smem, st>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace sa
