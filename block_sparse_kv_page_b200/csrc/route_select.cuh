// The router's per-(tile, KV head) selection and its finalize, shared by the
// router kernels (route.cu) and the routed decode step (step.cu).
//
// "Technische Samenvatting: Onzekerheidsgestuurde Selectie voor Blok-schaarse
// Aandacht", section "Methodologie": step 2 (the top blocks of a tile in rank
// order), step 3 (sigma = (s_(k-1) - s_(k)) / (s_(0) - s_(k))), step 4 (sigma_bar
// = mean over the heads; a tile triggers below the layer's quantile) and
// step 5 (the top rho*k blocks for a triggered tile, else the top k, padded
// with -1 sentinels).
#pragma once

#include "common.cuh"
#include "internal.h"
#include "radix.cuh"

namespace sa {
namespace rsel {

// Inverse of order_key.
SA_DEV float key_to_float(uint32_t k) {
  const uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
  return __uint_as_float(u);
}

struct RouteGeom {
  int E;        // eligible blocks of the tile
  int V;        // query vectors of the tile
  int row0;     // first query row of the tile
};

SA_DEV RouteGeom route_geom(const RouteArgs& a, int t, int N) {
  RouteGeom r;
  r.row0 = t * a.tile_rows;
  const int rows = min(a.tile_rows, a.n_rows - r.row0);
  r.V = rows * a.G;
  const int P = (N + a.kv.page_size - 1) / a.kv.page_size;
  const long long last_pos = (long long)a.q_pos0 + r.row0 + rows - 1;
  const long long e = last_pos / a.kv.page_size + 1;
  r.E = (int)(e < P ? e : P);
  return r;
}

// ---------------------------------------------------------------- rank order
// Sorts cand[0 .. n) (unique nonzero 64-bit keys) into descending order in
// place, when n <= (warps of the CTA) x 32 x kRunKeys; false (nothing done)
// otherwise.  Warp r sorts the run cand[r R .. (r + 1) R), R = 32 kRunKeys
// (zero-padded past n, and the padding, smaller than every key, never
// stored), in registers -- a bitonic network, lane l holding keys
// l kRunKeys .. + kRunKeys - 1, exchanges within a lane in registers and
// across lanes by shuffles, no barrier -- and writes it back; each key's
// final position is then its position in its run plus, for every other run,
// the number of its keys that are larger (a binary search: the run is
// descending).  Touches cand[0 .. n) only.  All threads of the CTA call it.
constexpr int kRunKeys = 4;
constexpr int kRunLen = 32 * kRunKeys;

SA_DEV bool rank_sort_desc(unsigned long long* cand, const int n) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (int)blockDim.x >> 5;
  const int runs = (n + kRunLen - 1) / kRunLen;
  if (runs > nw) return false;
  unsigned long long x[kRunKeys];
  const int p0 = lane * kRunKeys;  // this lane's first position in its run
  if (warp < runs) {
#pragma unroll
    for (int j = 0; j < kRunKeys; ++j) {
      const int i = warp * kRunLen + p0 + j;
      x[j] = i < n ? cand[i] : 0ull;
    }
    // bitonic network over the run, descending: the pair (e, e ^ d) of
    // block `size` keeps the larger key at the lower position when
    // (e & size) == 0, else at the higher one.  The stages run as a loop
    // (compact code: this runs once per unit, with the instruction cache
    // cold and every miss a slow round trip); only the in-lane distances 1
    // and 2 need their own register code.
    static_assert(kRunKeys == 4, "in-lane stages written for 4 keys a lane");
#pragma unroll 1
    for (int size = 2; size <= kRunLen; size <<= 1) {
#pragma unroll 1
      for (int d = size >> 1; d > 0; d >>= 1) {
        if (d >= kRunKeys) {
#pragma unroll
          for (int j = 0; j < kRunKeys; ++j) {
            const int e = p0 + j;
            const unsigned long long w = __shfl_xor_sync(0xffffffffu, x[j], d / kRunKeys);
            const bool keep_max = ((e & d) == 0) == ((e & size) == 0);
            x[j] = keep_max ? (x[j] > w ? x[j] : w) : (x[j] < w ? x[j] : w);
          }
        } else {  // in-lane pairs: (0,1),(2,3) for d = 1; (0,2),(1,3) for d = 2
          auto cx = [&](unsigned long long& lo, unsigned long long& hi, int e) {
            const bool desc = (e & size) == 0;
            const bool swap = desc ? lo < hi : lo > hi;
            const unsigned long long t = lo;
            lo = swap ? hi : lo;
            hi = swap ? t : hi;
          };
          if (d == 1) {
            cx(x[0], x[1], p0);
            cx(x[2], x[3], p0 + 2);
          } else {
            cx(x[0], x[2], p0);
            cx(x[1], x[3], p0 + 1);
          }
        }
      }
    }
  }
  __syncthreads();  // every key of cand is in registers
  if (warp < runs) {
#pragma unroll
    for (int j = 0; j < kRunKeys; ++j) {
      const int i = warp * kRunLen + p0 + j;
      if (i < n) cand[i] = x[j];
    }
  }
  __syncthreads();  // the sorted runs
  int rank[kRunKeys];
  if (warp < runs) {
#pragma unroll
    for (int j = 0; j < kRunKeys; ++j) rank[j] = p0 + j;
    for (int r = 0; r < runs; ++r) {
      if (r == warp) continue;
      const unsigned long long* run = cand + r * kRunLen;
      const int len = min(kRunLen, n - r * kRunLen);  // positions past it hold the padding
      int lo[kRunKeys], hi[kRunKeys];
#pragma unroll
      for (int j = 0; j < kRunKeys; ++j) { lo[j] = 0; hi[j] = kRunLen; }
#pragma unroll 1
      for (int step = kRunLen; step > 1; step >>= 1) {  // log2(kRunLen) halvings
#pragma unroll
        for (int j = 0; j < kRunKeys; ++j) {
          const int mid = (lo[j] + hi[j]) >> 1;
          if (mid < len && run[mid] > x[j]) lo[j] = mid + 1; else hi[j] = mid;
        }
      }
#pragma unroll
      for (int j = 0; j < kRunKeys; ++j) {
        // one last probe closes a range of one left by the halvings
        if (lo[j] < hi[j] && lo[j] < len && run[lo[j]] > x[j]) ++lo[j];
        rank[j] += lo[j];
      }
    }
  }
  __syncthreads();  // every search is done before the runs are overwritten
  if (warp < runs) {
#pragma unroll
    for (int j = 0; j < kRunKeys; ++j)
      if (x[j] != 0ull) cand[rank[j]] = x[j];
  }
  __syncthreads();
  return true;
}

// Bitonic sort of cand[0 .. n) into descending order in place (for lists
// longer than rank_sort_desc takes).  All threads of the CTA call it.
SA_DEV void bitonic_sort_desc(unsigned long long* cand, const int n_sel) {
  const int tid = threadIdx.x;
  int n2 = 1;
  while (n2 < n_sel) n2 <<= 1;
  for (int i = n_sel + tid; i < n2; i += blockDim.x) cand[i] = 0ull;
  __syncthreads();
  // Strides of 32 and up pair elements of different warps (shared memory, a
  // barrier each); the strides below 32 of one size run in registers, a warp
  // per 32 consecutive elements exchanging by shuffles, then one barrier.
  const int lane = tid & 31, nw = (int)blockDim.x >> 5;
  for (int size = 2; size <= n2; size <<= 1) {
    int stride = size >> 1;
    for (; stride >= 32; stride >>= 1) {
      for (int i = tid; i < n2; i += blockDim.x) {
        const int j = i ^ stride;
        if (j > i) {
          const bool desc = (i & size) == 0;
          const unsigned long long x = cand[i], y = cand[j];
          if (desc ? (x < y) : (x > y)) {
            cand[i] = y;
            cand[j] = x;
          }
        }
      }
      __syncthreads();
    }
    for (int r = tid >> 5; 32 * r < n2; r += nw) {
      const int e = 32 * r + lane;
      unsigned long long v = e < n2 ? cand[e] : 0ull;
      const bool desc = (e & size) == 0;
      for (int st = stride; st > 0; st >>= 1) {
        const unsigned long long w = __shfl_xor_sync(0xffffffffu, v, st);
        // the lower index of a pair keeps the larger value when descending
        v = (((e & st) == 0) == desc) ? (v > w ? v : w) : (v < w ? v : w);
      }
      if (e < n2) cand[e] = v;
    }
    __syncthreads();
  }
}

SA_DEV void route_select_finish(const RouteArgs& a, const int tg, const int E, unsigned long long* cand,
                                const int n_sel);

// ---------------------------------------------------------------- selection for one (t, g)
SA_DEV void route_select_tile(const RouteArgs& a, int t, int g, int E, unsigned char* smem,
                              uint32_t* hist, uint32_t* bc, uint32_t* scan) {
  const int tid = threadIdx.x;
  const int Hkv = a.kv.Hkv;
  const int tg = t * Hkv + g;
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem);                         // [E]
  unsigned long long* cand = reinterpret_cast<unsigned long long*>(smem + ((E * 4 + 15) & ~15));
  uint32_t* kp = a.ws_keys + (size_t)tg * a.kv.max_pages;
  const float* sp = a.dec_scores ? a.dec_scores + (size_t)tg * a.dec_stride : nullptr;
  // 16 loads in flight per thread: one round trip for a 2048-page unit on 128 threads
  for (int b = 0; b < E; b += 16 * (int)blockDim.x) {
    uint32_t v[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int i = b + j * (int)blockDim.x + tid;
      // tile-score keys, or (decode router) group scores turned into keys
      v[j] = i >= E ? 0u : (sp ? order_key(__ldcg(sp + i)) : __ldcg(kp + i));
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int i = b + j * (int)blockDim.x + tid;
      if (i < E) keys[i] = v[j];
    }
  }
  __syncthreads();
  const int want = max(a.W, a.k + 1);
  const int cap = min(want, E);
  int n_sel;
  if (E <= cap) {
    for (int i = tid; i < E; i += blockDim.x)
      cand[i] = ((unsigned long long)keys[i] << 32) | (0xffffffffu - (uint32_t)i);
    n_sel = E;
  } else {
    const RadixCut cut = radix_cut(keys, nullptr, E, (uint32_t)cap, hist, bc);
    // compaction in index order: keys > T, then the first `rem` keys == T
    const int per = (E + blockDim.x - 1) / blockDim.x;
    const int i0 = min(E, tid * per), i1 = min(E, i0 + per);
    uint32_t eqc = 0;
    for (int i = i0; i < i1; ++i) eqc += keys[i] == cut.T ? 1u : 0u;
    uint32_t dummy;
    const uint32_t eq0 = block_excl_scan(eqc, scan, dummy);
    uint32_t cnt = 0, eq = eq0;
    for (int i = i0; i < i1; ++i) {
      const uint32_t k = keys[i];
      const bool s = k > cut.T || (k == cut.T && ++eq <= cut.rem);
      cnt += s ? 1u : 0u;
    }
    uint32_t total;
    uint32_t pos = block_excl_scan(cnt, scan, total);
    eq = eq0;
    for (int i = i0; i < i1; ++i) {
      const uint32_t k = keys[i];
      const bool s = k > cut.T || (k == cut.T && ++eq <= cut.rem);
      if (s) cand[pos++] = ((unsigned long long)k << 32) | (0xffffffffu - (uint32_t)i);
    }
    n_sel = cap;
  }
  route_select_finish(a, tg, E, cand, n_sel);
}

// The rest of a (tile, KV head)'s selection, from its n_sel candidates in
// cand (composite keys, any order; the top max(rho k, k + 1) of its E
// eligible blocks): rank order, sigma, the list as if the tile triggered
// and its count.  All threads of the CTA call it.
SA_DEV void route_select_finish(const RouteArgs& a, const int tg, const int E, unsigned long long* cand,
                                const int n_sel) {
  const int tid = threadIdx.x;
  // rank order: descending composite key = (score key, ~index); sorted runs
  // merged by rank when they fit the CTA's warps, else a bitonic sort
  __syncthreads();
  if (!rank_sort_desc(cand, n_sel)) bitonic_sort_desc(cand, n_sel);
  if (tid == 0) {
    double sg;
    if (E <= a.k) {
      sg = 1.0;
    } else {
      const double s0 = key_to_float((uint32_t)(cand[0] >> 32));
      const double skm1 = key_to_float((uint32_t)(cand[a.k - 1] >> 32));
      const double sk = key_to_float((uint32_t)(cand[a.k] >> 32));
      sg = (s0 == sk) ? 0.0 : (skm1 - sk) / (s0 - sk);
    }
    a.ws_sigma[tg] = sg;
    a.sigma[tg] = (float)sg;
    a.ws_elig[tg] = E;
  }
  // the list as if the tile triggers (the top rho k, -1 past the eligible
  // blocks); the finalize trims the tiles that do not trigger to k
  int32_t* lst = a.kv_idx + (size_t)tg * a.W;
  for (int i = tid; i < a.W; i += blockDim.x)
    lst[i] = i < n_sel ? (int32_t)(0xffffffffu - (uint32_t)(cand[i] & 0xffffffffu)) : -1;
  if (tid == 0) a.kv_count[tg] = min(a.W, E);
}

// ---------------------------------------------------------------- finalize (one CTA)
// Shared memory it needs: T x 16 + T x Hkv x 12 bytes.
__host__ __device__ inline size_t finalize_smem_bytes(int n_tiles, int Hkv) {
  return (size_t)n_tiles * 16 + (size_t)n_tiles * Hkv * 12;
}

// Runs while the rest of the GPU streams at full bandwidth, when every
// global round trip is slow and one SM's stores drain slowly: all its loads
// are issued at once, up front, and it comes in two parts.
// route_triggers: sigma_bar, the quantile threshold and the triggers into
// shared memory, and (with a.trig_list) the triggered (tile, KV head) pairs
// in order as {tile x Hkv + head, list count, the tile's sequence length}
// (decode router: the tiles are the sequences); returns their number (every
// thread).  route_outputs, after it: sigma_bar, tau, the triggers and the
// lists of the tiles that did not trigger trimmed to k -- stores no decode
// item reads, so the routed decode step publishes the triggered units
// before it runs them.
struct FinalizeSmem {
  double* sbar;    // [T]
  double* sorted;  // [T]
  double* sig;     // [T x Hkv]
  int* elig;       // [T x Hkv]
};
SA_DEV FinalizeSmem finalize_smem(const RouteArgs& a, unsigned char* smem) {
  const int T = a.n_tiles, units = T * a.kv.Hkv;
  FinalizeSmem f;
  f.sbar = reinterpret_cast<double*>(smem);
  f.sorted = f.sbar + T;
  f.sig = f.sorted + T;
  f.elig = reinterpret_cast<int*>(f.sig + units);
  return f;
}

SA_DEV int route_triggers(const RouteArgs& a, unsigned char* smem, double& tau_out) {
  const int tid = threadIdx.x, nt = (int)blockDim.x;
  const int T = a.n_tiles, Hkv = a.kv.Hkv, units = T * Hkv;
  const FinalizeSmem f = finalize_smem(a, smem);
  __shared__ double s_tau;
  __shared__ int s_ntrig;
  __shared__ uint32_t scan[32];
  for (int i0 = tid; i0 < units; i0 += 4 * nt) {
    double sv[4];
    int ev[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int i = i0 + j * nt;
      sv[j] = i < units ? __ldcg(a.ws_sigma + i) : 0.0;
      ev[j] = i < units ? __ldcg(a.ws_elig + i) : 0;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int i = i0 + j * nt;
      if (i < units) {
        f.sig[i] = sv[j];
        f.elig[i] = ev[j];
      }
    }
  }
  __syncthreads();
  for (int t = tid; t < T; t += nt) {
    double s = 0.0;
    for (int g = 0; g < Hkv; ++g) s += f.sig[t * Hkv + g];
    f.sbar[t] = s / Hkv;
  }
  __syncthreads();
  for (int t = tid; t < T; t += nt) {  // rank by (value, index)
    int r = 0;
    const double v = f.sbar[t];
    for (int u = 0; u < T; ++u) r += (f.sbar[u] < v || (f.sbar[u] == v && u < t)) ? 1 : 0;
    f.sorted[r] = v;
  }
  __syncthreads();
  if (tid == 0) {
    double tau;
    if (a.tau_in) {
      tau = (double)*a.tau_in;
    } else {
      const double h = (T - 1) * (double)a.quantile;
      const int lo = (int)floor(h);
      const int hi = min(lo + 1, T - 1);
      tau = f.sorted[lo] + (h - lo) * (f.sorted[hi] - f.sorted[lo]);
    }
    s_tau = tau;
  }
  __syncthreads();
  const double tau = s_tau;
  tau_out = tau;
  if (a.trig_list == nullptr) return 0;
  // the triggered pairs in (tile, KV head) order: each thread a run of them
  const int per = (units + nt - 1) / nt;
  const int i0 = min(units, tid * per), i1 = min(units, i0 + per);
  uint32_t cnt = 0;
  for (int i = i0; i < i1; ++i) cnt += f.sbar[i / Hkv] < tau ? 1u : 0u;
  uint32_t total;
  uint32_t pos = block_excl_scan(cnt, scan, total);
  for (int i = i0; i < i1; ++i) {
    const int t = i / Hkv;
    if (f.sbar[t] < tau) a.trig_list[pos++] = make_int4(i, min(a.W, f.elig[i]), a.kv.seq_len[t], 0);
  }
  if (tid == 0) s_ntrig = (int)total;
  __syncthreads();
  return s_ntrig;
}

SA_DEV void route_outputs(const RouteArgs& a, unsigned char* smem, const double tau) {
  const int tid = threadIdx.x, nt = (int)blockDim.x;
  const int T = a.n_tiles, Hkv = a.kv.Hkv, units = T * Hkv;
  const FinalizeSmem f = finalize_smem(a, smem);
  if (tid == 0 && a.tau_out) *a.tau_out = (float)tau;
  for (int t = tid; t < T; t += nt) {
    a.sigma_bar[t] = (float)f.sbar[t];
    a.triggered[t] = f.sbar[t] < tau ? 1 : 0;
  }
  // the selecting CTAs wrote every list as if its tile triggered: trim the
  // others to their top k (entries k .. W - 1 become sentinels)
  if (a.W > a.k) {
    for (int tg = tid; tg < units; tg += nt)
      if (!(f.sbar[tg / Hkv] < tau)) a.kv_count[tg] = min(a.k, f.elig[tg]);
    const int lane = tid & 31, nw = nt >> 5;
    for (int tg = tid >> 5; tg < units; tg += nw) {  // sentinels: a warp per (tile, KV head)
      if (f.sbar[tg / Hkv] < tau) continue;
      int32_t* row = a.kv_idx + (size_t)tg * a.W;
      for (int i = a.k + lane; i < a.W; i += 32) row[i] = -1;
    }
  }
}

SA_DEV void route_finalize(const RouteArgs& a, unsigned char* smem) {
  double tau;
  route_triggers(a, smem, tau);
  route_outputs(a, smem, tau);
}

}  // namespace rsel
}  // namespace sa
