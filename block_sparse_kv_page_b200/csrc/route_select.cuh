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
  for (int b = 0; b < E; b += 8 * (int)blockDim.x) {  // 8 loads in flight per thread
    uint32_t v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = b + j * (int)blockDim.x + tid;
      // tile-score keys, or (decode router) group scores turned into keys
      v[j] = i >= E ? 0u : (sp ? order_key(__ldcg(sp + i)) : __ldcg(kp + i));
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
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
  // bitonic sort, descending composite key = (score key, ~index): rank order
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
SA_DEV void route_finalize(const RouteArgs& a, unsigned char* smem) {
  const int tid = threadIdx.x;
  const int T = a.n_tiles, Hkv = a.kv.Hkv;
  double* sbar = reinterpret_cast<double*>(smem);   // [T]
  double* sorted = sbar + T;                        // [T]
  __shared__ double s_tau;
  for (int t = tid; t < T; t += blockDim.x) {
    double s = 0.0;
    for (int g = 0; g < Hkv; ++g) s += __ldcg(a.ws_sigma + t * Hkv + g);
    sbar[t] = s / Hkv;
    a.sigma_bar[t] = (float)sbar[t];
  }
  __syncthreads();
  for (int t = tid; t < T; t += blockDim.x) {  // rank by (value, index)
    int r = 0;
    const double v = sbar[t];
    for (int u = 0; u < T; ++u) r += (sbar[u] < v || (sbar[u] == v && u < t)) ? 1 : 0;
    sorted[r] = v;
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
      tau = sorted[lo] + (h - lo) * (sorted[hi] - sorted[lo]);
    }
    s_tau = tau;
    if (a.tau_out) *a.tau_out = (float)tau;
  }
  __syncthreads();
  const double tau = s_tau;
  for (int t = tid; t < T; t += blockDim.x) a.triggered[t] = sbar[t] < tau ? 1 : 0;
  // the selecting CTAs wrote every list as if its tile triggered: trim the
  // others to their top k (entries k .. W - 1 become sentinels), a warp per
  // tile, lanes along the entries
  if (a.W > a.k) {
    const int lane = tid & 31, nw = blockDim.x >> 5;
    for (int t = tid >> 5; t < T; t += nw) {  // warp per tile
      if (sbar[t] < tau) continue;
      for (int g = 0; g < Hkv; ++g) {
        const int tg = t * Hkv + g;
        int32_t* row = a.kv_idx + (size_t)tg * a.W;
        for (int i = a.k + lane; i < a.W; i += 32) row[i] = -1;
        if (lane == 0) a.kv_count[tg] = min(a.k, __ldcg(a.ws_elig + tg));
      }
    }
  }
}

}  // namespace rsel
}  // namespace sa
