// Uncertainty router over query tiles.
//
// "Technische Samenvatting: Onzekerheidsgestuurde Selectie voor Blok-schaarse
// Aandacht", section "Methodologie":
//   step 1  blocks scored by a backbone (envelope = coordinate-wise upper bound
//           from per-block key min/max; centroid = mean-pooled inner product);
//   step 2  selection per query tile: the tile score of a block is the maximum
//           of the per-row scores over the tile's rows (and here over the G
//           query heads that share the KV head);
//   step 3  sigma = (s_(k-1) - s_(k)) / (s_(0) - s_(k)) per tile and head on the
//           descending block scores;
//   step 4  sigma_bar = mean of sigma over the heads; a tile triggers when
//           sigma_bar falls below the layer's empirical quantile q;
//   step 5  triggered tiles keep the top rho*k blocks, the others the top k,
//           padded with sentinels (-1) so every list has the same shape.
//
// One launch, no CTA waits on another:
//   * CTA (tile t, KV head g, split sp) scores every eligible block of head g
//     against its share (<= 224) of the tile's query vectors (row x head) on
//     tensor cores -- block metadata streamed by TMA (16 blocks x 512 B per
//     stage, 128B swizzle), query vectors resident in shared memory:
//       envelope: [kmin|kmax] (16 x 256 bf16) x [q-|q+]^T, m16n8k16, exact products;
//       centroid: kmean (16 x 128 fp32) x q^T on m16n8k8 tf32 with kmean split
//                 into a tf32 head and its exact remainder (products exact to
//                 about 2^-21);
//     and folds its per-block maxima into the tile-score keys with atomicMax
//     on order-preserving uint32 keys.
//   * The last split CTA of (t, g) (atomic counter) selects the top
//     max(rho*k, k+1) eligible blocks by radix select, sorts them to rank
//     order (score desc, index asc) and computes sigma in double.
//   * The last (t, g) CTA computes sigma_bar, the quantile threshold, the
//     triggers and writes the sentinel-padded lists.
#include "common.cuh"
#include "internal.h"
#include "radix.cuh"
#include "tcgen05.cuh"

namespace sa {
namespace {

constexpr int kRtWarps = 4;
constexpr int kRtThreads = 32 * kRtWarps;
constexpr int kRtNTilesPerWarp = 7;                         // n8 tiles of query vectors per warp
constexpr int kRtVecs = 8 * kRtNTilesPerWarp * kRtWarps;     // 224 query vectors per CTA
constexpr int kRtStages = 3;
constexpr int kTileBytes = 8192;                             // 16 blocks x 512 B
constexpr int kBoxBytes = 2048;
constexpr int kQsChunk = kRtVecs * 128;                      // one 128-byte K chunk of all vectors
constexpr int kQsBytes = 4 * kQsChunk;                       // 112 KiB
constexpr int kOffRing = kQsBytes;
constexpr int kOffBars = kOffRing + kRtStages * kTileBytes;
constexpr int kSmemBytes = kOffBars + kRtStages * 8;

SA_DEV void ldsm_x2(uint32_t& r0, uint32_t& r1, const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];\n"
               : "=r"(r0), "=r"(r1)
               : "r"(smem_addr(p)));
}

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
  for (int b = 0; b < E; b += 8 * (int)blockDim.x) {  // 8 loads in flight per thread
    uint32_t v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = b + j * (int)blockDim.x + tid;
      v[j] = i < E ? __ldcg(kp + i) : 0u;
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
  for (int size = 2; size <= n2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
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
  int32_t* lst = a.ws_list + (size_t)tg * a.W;
  for (int i = tid; i < a.W; i += blockDim.x)
    lst[i] = i < n_sel ? (int32_t)(0xffffffffu - (uint32_t)(cand[i] & 0xffffffffu)) : -1;
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
  for (int tg = tid; tg < T * Hkv; tg += blockDim.x) {
    const int t = tg / Hkv;
    const bool trig = sbar[t] < tau;
    if (tg % Hkv == 0) a.triggered[t] = trig ? 1 : 0;
    const int E = __ldcg(a.ws_elig + tg);
    a.kv_count[tg] = min(trig ? a.W : a.k, E);
  }
  // the lists, every (tile, head, entry) by its own thread: independent loads
  const int total = T * Hkv * a.W;
  for (int b = 0; b < total; b += 8 * (int)blockDim.x) {  // 8 loads in flight per thread
    int32_t v[8], ne[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int x = b + j * (int)blockDim.x + tid;
      v[j] = x < total ? __ldcg(a.ws_list + x) : -1;
      ne[j] = x < total ? __ldcg(a.ws_elig + x / a.W) : 0;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int x = b + j * (int)blockDim.x + tid;
      if (x >= total) continue;
      const int tg = x / a.W, i = x - tg * a.W;
      const int n = min(sbar[tg / Hkv] < tau ? a.W : a.k, ne[j]);
      a.kv_idx[x] = i < n ? v[j] : -1;
    }
  }
}

// ---------------------------------------------------------------- after scoring
// The last split CTA of (t, g) selects; the last (t, g) CTA finalizes.  The
// counter increments are acq_rel after a barrier: they publish this CTA's
// tile-score keys (or list) and acquire everyone else's.
SA_DEV void route_tail(const RouteArgs& a, int t, int g, int E, unsigned char* base, uint32_t* hist,
                       uint32_t* bc, uint32_t* scan, int* flag) {
  const int tid = threadIdx.x;
  const int tg = t * a.kv.Hkv + g;
  __syncthreads();
  if (tid == 0) {
    *flag = 1;
    if (a.nsplit > 1) *flag = atom_add_acq_rel_u32(a.ws_count + tg, 1u) == (uint32_t)(a.nsplit - 1);
  }
  __syncthreads();
  if (!*flag) return;
  if (tid == 0 && a.nsplit > 1) a.ws_count[tg] = 0;
  route_select_tile(a, t, g, E, base, hist, bc, scan);
  __syncthreads();
  if (tid == 0) *flag = atom_add_acq_rel_u32(a.ws_final, 1u) == (uint32_t)(a.n_tiles * a.kv.Hkv - 1);
  __syncthreads();
  if (!*flag) return;
  if (tid == 0) *a.ws_final = 0;
  route_finalize(a, base);
}

// ---------------------------------------------------------------- the kernel
template <int RULE>
__global__ void __launch_bounds__(kRtThreads) route_kernel(const __grid_constant__ RouteArgs a) {
  extern __shared__ unsigned char smem_raw[];
  __shared__ float s_wmax[2][kRtWarps][16];
  __shared__ uint32_t s_hist[256];
  __shared__ uint32_t s_scan[32];
  __shared__ uint32_t s_bc[4];
  __shared__ int s_flag;
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* qs = base;
  unsigned char* ring = base + kOffRing;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + kOffBars);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, c = lane & 3;
  const int Hkv = a.kv.Hkv;
  const int sp = blockIdx.x % a.nsplit;
  const int tg = blockIdx.x / a.nsplit;
  const int t = tg / Hkv, g = tg % Hkv;
  const int N = a.kv.seq_len[0];
  const RouteGeom geo = route_geom(a, t, N);
  const int v0 = sp * kRtVecs;

  if (tid == 0) {
    for (int s = 0; s < kRtStages; ++s) mbar_init(bars + s, 1);
    fence_barrier_init();
    prefetch_tmap(&a.tmap_meta);
  }

  // ---- query vectors of this split into shared memory (K-major, 128B-swizzled chunks)
  const __nv_bfloat16* Q = reinterpret_cast<const __nv_bfloat16*>(a.q);
  for (int x = tid; x < kRtVecs * 16; x += kRtThreads) {
    const int vi = x >> 4, d8 = x & 15;  // vector, 8-element chunk of the 128-dim query
    const int v = v0 + vi;
    uint4 raw = make_uint4(0u, 0u, 0u, 0u);
    if (v < geo.V) {
      const int r = v / a.G, j = v - (v / a.G) * a.G;
      raw = ldg_nc128(Q + ((size_t)(geo.row0 + r) * a.Hq + (size_t)g * a.G + j) * kHeadDim + 8 * d8);
    }
    if (RULE == 0) {  // [q- | q+]: element e of 256 -> chunk e/64, 16-byte piece (e%64)/8
      uint4 neg, pos;
      neg.x = bf16x2_neg_part(raw.x); neg.y = bf16x2_neg_part(raw.y);
      neg.z = bf16x2_neg_part(raw.z); neg.w = bf16x2_neg_part(raw.w);
      pos.x = bf16x2_pos_part(raw.x); pos.y = bf16x2_pos_part(raw.y);
      pos.z = bf16x2_pos_part(raw.z); pos.w = bf16x2_pos_part(raw.w);
      *reinterpret_cast<uint4*>(qs + (d8 >> 3) * kQsChunk + swz128(vi, d8 & 7)) = neg;
      *reinterpret_cast<uint4*>(qs + (2 + (d8 >> 3)) * kQsChunk + swz128(vi, d8 & 7)) = pos;
    } else {  // fp32 [128]: element d -> chunk d/32, piece (d%32)/4
      const float4 lo = make_float4(bf16_lo(raw.x), bf16_hi(raw.x), bf16_lo(raw.y), bf16_hi(raw.y));
      const float4 hi = make_float4(bf16_lo(raw.z), bf16_hi(raw.z), bf16_lo(raw.w), bf16_hi(raw.w));
      const int ch = d8 >> 2, pc = 2 * (d8 & 3);
      *reinterpret_cast<float4*>(qs + ch * kQsChunk + swz128(vi, pc)) = lo;
      *reinterpret_cast<float4*>(qs + ch * kQsChunk + swz128(vi, pc + 1)) = hi;
    }
  }
  __syncthreads();

  // ---- stream the eligible blocks of head g, 16 per stage
  const int TB = (geo.E + 15) >> 4;
  const int row_base = g * a.kv.max_pages;
  auto issue = [&](int tb) {
    uint64_t* bar = bars + tb % kRtStages;
    unsigned char* st = ring + (tb % kRtStages) * kTileBytes;
    mbar_arrive_expect_tx(bar, kTileBytes);
    const int xs = RULE == 0 ? 64 : 32;
#pragma unroll
    for (int bx = 0; bx < 4; ++bx) tma_load_2d(st + bx * kBoxBytes, &a.tmap_meta, bx * xs, row_base + 16 * tb, bar);
  };
  if (tid == 0)
    for (int tb = 0; tb < min(TB, kRtStages); ++tb) issue(tb);

  const float ninf = -__int_as_float(0x7f800000);
  const int lrow = (lane & 7) + 8 * ((lane >> 3) & 1);
  const int lchk = lane >> 4;
  const int brow = lane & 7, bchk = (lane >> 3) & 1;  // ldmatrix.x2 for B (lanes 0-15)
  uint32_t* keys_tg = a.ws_keys + (size_t)tg * a.kv.max_pages;
  int tb_fail = -1;  // first stage whose wait timed out (CTA-uniform)

  for (int tb = 0; tb < TB; ++tb) {
    const bool ok = mbar_wait(bars + tb % kRtStages, (tb / kRtStages) & 1u, a.status);
    if (!__syncthreads_and(ok)) {
      tb_fail = tb;
      break;
    }
    const bool alive = true;
    const unsigned char* st = ring + (tb % kRtStages) * kTileBytes;
    float acc[kRtNTilesPerWarp][4];
#pragma unroll
    for (int i = 0; i < kRtNTilesPerWarp; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    if (alive) {
      if (RULE == 0) {
#pragma unroll 4
        for (int ks = 0; ks < 16; ++ks) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4(a0, a1, a2, a3, st + (ks >> 2) * kBoxBytes + swz128(lrow, 2 * (ks & 3) + lchk));
#pragma unroll
          for (int i = 0; i < kRtNTilesPerWarp; ++i) {
            const int nt = warp * kRtNTilesPerWarp + i;
            uint32_t b0, b1;
            ldsm_x2(b0, b1, qs + (ks >> 2) * kQsChunk + swz128(8 * nt + brow, 2 * (ks & 3) + bchk));
            mma_bf16(acc[i], a0, a1, a2, a3, b0, b1);
          }
        }
      } else {
#pragma unroll 2
        for (int ks = 0; ks < 16; ++ks) {  // dims 8ks .. 8ks + 7
          const int bx = ks >> 2, ch = 2 * (ks & 3);
          const float x0 = *reinterpret_cast<const float*>(st + bx * kBoxBytes + swz128(gq, ch) + 4 * c);
          const float x1 = *reinterpret_cast<const float*>(st + bx * kBoxBytes + swz128(gq + 8, ch) + 4 * c);
          const float x2 = *reinterpret_cast<const float*>(st + bx * kBoxBytes + swz128(gq, ch + 1) + 4 * c);
          const float x3 = *reinterpret_cast<const float*>(st + bx * kBoxBytes + swz128(gq + 8, ch + 1) + 4 * c);
          const uint32_t h0 = __float_as_uint(x0) & 0xffffe000u, h1 = __float_as_uint(x1) & 0xffffe000u;
          const uint32_t h2 = __float_as_uint(x2) & 0xffffe000u, h3 = __float_as_uint(x3) & 0xffffe000u;
          const uint32_t l0 = __float_as_uint(x0 - __uint_as_float(h0));
          const uint32_t l1 = __float_as_uint(x1 - __uint_as_float(h1));
          const uint32_t l2 = __float_as_uint(x2 - __uint_as_float(h2));
          const uint32_t l3 = __float_as_uint(x3 - __uint_as_float(h3));
#pragma unroll
          for (int i = 0; i < kRtNTilesPerWarp; ++i) {
            const int v = 8 * (warp * kRtNTilesPerWarp + i) + gq;
            const uint32_t b0 = *reinterpret_cast<const uint32_t*>(qs + bx * kQsChunk + swz128(v, ch) + 4 * c);
            const uint32_t b1 = *reinterpret_cast<const uint32_t*>(qs + bx * kQsChunk + swz128(v, ch + 1) + 4 * c);
            mma_tf32(acc[i], h0, h1, h2, h3, b0, b1);
            mma_tf32(acc[i], l0, l1, l2, l3, b0, b1);
          }
        }
      }
    }
    // max over this warp's query vectors (C[block][vector]: c0,c1 block gq, c2,c3 block gq+8)
    float mlo = ninf, mhi = ninf;
#pragma unroll
    for (int i = 0; i < kRtNTilesPerWarp; ++i) {
      const int vcol = v0 + 8 * (warp * kRtNTilesPerWarp + i) + 2 * c;
      const bool ok0 = vcol < geo.V, ok1 = vcol + 1 < geo.V;
      mlo = fmaxf(mlo, fmaxf(ok0 ? acc[i][0] : ninf, ok1 ? acc[i][1] : ninf));
      mhi = fmaxf(mhi, fmaxf(ok0 ? acc[i][2] : ninf, ok1 ? acc[i][3] : ninf));
    }
    mlo = fmaxf(mlo, __shfl_xor_sync(0xffffffffu, mlo, 1));
    mlo = fmaxf(mlo, __shfl_xor_sync(0xffffffffu, mlo, 2));
    mhi = fmaxf(mhi, __shfl_xor_sync(0xffffffffu, mhi, 1));
    mhi = fmaxf(mhi, __shfl_xor_sync(0xffffffffu, mhi, 2));
    if (c == 0) {
      s_wmax[tb & 1][warp][gq] = mlo;
      s_wmax[tb & 1][warp][gq + 8] = mhi;
    }
    __syncthreads();  // stage tb consumed by every warp; wmax[tb & 1] complete
    if (tid == 0 && tb + kRtStages < TB) issue(tb + kRtStages);
    if (tid < 16) {
      const int blk = 16 * tb + tid;
      float m = s_wmax[tb & 1][0][tid];
#pragma unroll
      for (int w = 1; w < kRtWarps; ++w) m = fmaxf(m, s_wmax[tb & 1][w][tid]);
      if (blk < geo.E && m != ninf) atomicMax(keys_tg + blk, order_key(m));
    }
  }
  if (tb_fail >= 0 && tid == 0) {  // let the copies still in flight land (bounded) before leaving
    const int hi = min(TB, tb_fail + kRtStages);
    for (int tb = tb_fail; tb < hi; ++tb) mbar_wait(bars + tb % kRtStages, (tb / kRtStages) & 1u, nullptr);
  }

  route_tail(a, t, g, geo.E, base, s_hist, s_bc, s_scan, &s_flag);
}

// ---------------------------------------------------------------- tensor-core (tcgen05) envelope scoring
// CTA = (tile t, KV head g, split of <= 224 query vectors), one per SM.  The
// scores of 128 blocks against the split's vectors are one tcgen05 GEMM
//   D[128 blocks x 224 vectors] = [kmin|kmax] (128 x 256 bf16, K-major)
//                                 . [q-|q+]^T (224 x 256 bf16, K-major)
// accumulated in tensor memory (fp32).  Warp-specialised:
//   warp 4 (one thread)  copies metadata by TMA in 16 KiB K-chunks (128 blocks
//                        x 128 B) into a kTcStages ring;
//   warp 5 (one thread)  issues the MMAs (4 per chunk, 32 B of K each) and
//                        commits: a chunk's stage is freed when its MMAs are
//                        done, an accumulator is marked full after 4 chunks;
//   warps 0-3            epilogue: thread i owns block i of the M tile (TMEM
//                        lane i), takes the max over the vectors in registers
//                        and folds it into the tile-score keys (atomicMax).
// The two accumulators alternate, so the epilogue of one M tile overlaps the
// MMAs of the next; every wait is bounded.
constexpr int kTcEpiWarps = 4;
constexpr int kTcThreads = 32 * (kTcEpiWarps + 2);
constexpr int kTcProducerWarp = kTcEpiWarps;
constexpr int kTcMmaWarp = kTcEpiWarps + 1;
constexpr int kTcStages = 6;
constexpr int kTcChunkBytes = 128 * 128;
constexpr int kTcAccCols = 256;                               // one accumulator (224 used)
constexpr int kTcOffRing = kQsBytes;
constexpr int kTcOffBars = kTcOffRing + kTcStages * kTcChunkBytes;
constexpr int kTcNumBars = 2 * kTcStages + 4 + 1;             // full, empty, acc full x2, acc empty x2, drain
constexpr int kTcSmemBytes = kTcOffBars + kTcNumBars * 8 + 16;
static_assert(kRtVecs % 16 == 0 && kRtVecs <= kTcAccCols, "MMA N");
static_assert(1024 + kTcSmemBytes > 114 * 1024, "one CTA per SM: it allocates all 512 TMEM columns");

__global__ void __launch_bounds__(kTcThreads, 1) route_tc_kernel(const __grid_constant__ RouteArgs a) {
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint32_t s_hist[256];
  __shared__ uint32_t s_scan[32];
  __shared__ uint32_t s_bc[4];
  __shared__ int s_flag;
  __shared__ uint32_t s_tmem;
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* qs = base;
  unsigned char* ring = base + kTcOffRing;
  uint64_t* full = reinterpret_cast<uint64_t*>(base + kTcOffBars);
  uint64_t* empty = full + kTcStages;
  uint64_t* acc_full = empty + kTcStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Hkv = a.kv.Hkv;
  const int sp = blockIdx.x % a.nsplit;
  const int tg = blockIdx.x / a.nsplit;
  const int t = tg / Hkv, g = tg % Hkv;
  const int N = a.kv.seq_len[0];
  const RouteGeom geo = route_geom(a, t, N);
  const int v0 = sp * kRtVecs;

  if (tid == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_full + 1, 1);
    mbar_init(acc_empty, kTcEpiWarps);
    mbar_init(acc_empty + 1, kTcEpiWarps);
    mbar_init(drain, 1);
    fence_barrier_init();
    prefetch_tmap(&a.tmap_meta_tc);
  }
  if (warp == 0) {
    tc::tmem_alloc(&s_tmem, 2 * kTcAccCols);
    tc::tmem_relinquish();
  }
  __syncthreads();  // barriers initialised
  const int n_mt = (geo.E + 127) >> 7;  // M tiles of 128 blocks
  const int n_ch = 4 * n_mt;            // K-chunks
  const int row_base = g * a.kv.max_pages;
  // the first ring of metadata copies needs no wait: start it before the queries load
  const int n_pre = min(kTcStages, n_ch);
  if (warp == kTcProducerWarp && lane == 0)
    for (int j = 0; j < n_pre; ++j) {
      mbar_arrive_expect_tx(full + j, kTcChunkBytes);
      tma_load_2d(ring + j * kTcChunkBytes, &a.tmap_meta_tc, (j & 3) * 64, row_base + 128 * (j >> 2), full + j);
    }

  // ---- [q- | q+] of this split's vectors: K-major, 128B-swizzled chunks (the
  // MMA's B operand); kQBatch 16-byte loads per thread in flight at once
  constexpr int kQPieces = kRtVecs * 16;  // 16-byte pieces of the 224 x 128 bf16 queries
  constexpr int kQBatch = 8;
  const __nv_bfloat16* Q = reinterpret_cast<const __nv_bfloat16*>(a.q);
#pragma unroll 1
  for (int b0 = 0; b0 < kQPieces; b0 += kQBatch * kTcThreads) {
    uint4 rw[kQBatch];
#pragma unroll
    for (int i = 0; i < kQBatch; ++i) {
      const int x = b0 + i * kTcThreads + tid;
      const int vi = x >> 4, d8 = x & 15;
      const int v = v0 + vi;
      rw[i] = make_uint4(0u, 0u, 0u, 0u);
      if (x < kQPieces && v < geo.V) {
        const int r = v / a.G, j = v - r * a.G;
        rw[i] = ldg_nc128(Q + ((size_t)(geo.row0 + r) * a.Hq + (size_t)g * a.G + j) * kHeadDim + 8 * d8);
      }
    }
#pragma unroll
    for (int i = 0; i < kQBatch; ++i) {
      const int x = b0 + i * kTcThreads + tid;
      if (x >= kQPieces) continue;
      const int vi = x >> 4, d8 = x & 15;
      const uint4 raw = rw[i];
      uint4 neg, pos;
      neg.x = bf16x2_neg_part(raw.x); neg.y = bf16x2_neg_part(raw.y);
      neg.z = bf16x2_neg_part(raw.z); neg.w = bf16x2_neg_part(raw.w);
      pos.x = bf16x2_pos_part(raw.x); pos.y = bf16x2_pos_part(raw.y);
      pos.z = bf16x2_pos_part(raw.z); pos.w = bf16x2_pos_part(raw.w);
      *reinterpret_cast<uint4*>(qs + (d8 >> 3) * kQsChunk + swz128(vi, d8 & 7)) = neg;
      *reinterpret_cast<uint4*>(qs + (2 + (d8 >> 3)) * kQsChunk + swz128(vi, d8 & 7)) = pos;
    }
  }
  fence_proxy_async();  // generic writes of qs before the tensor cores read it
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = s_tmem;

  int fail = 0;                         // this thread saw a wait run out

  if (warp == kTcProducerWarp) {
    // ---- TMA producer: chunk j -> stage j % kTcStages
    if (lane == 0) {
      int issued = n_pre;
      for (int j = n_pre; j < n_ch; ++j) {
        const int s = j % kTcStages;
        if (j >= kTcStages && !mbar_wait(empty + s, ((j / kTcStages) - 1) & 1u, a.status)) {
          fail = 1;
          break;
        }
        mbar_arrive_expect_tx(full + s, kTcChunkBytes);
        tma_load_2d(ring + s * kTcChunkBytes, &a.tmap_meta_tc, (j & 3) * 64, row_base + 128 * (j >> 2), full + s);
        issued = j + 1;
      }
      // every copy issued has landed before the CTA moves on (bounded)
      for (int j = max(0, issued - kTcStages); j < issued; ++j)
        mbar_wait(full + (j % kTcStages), (j / kTcStages) & 1u, nullptr);
    }
  } else if (warp == kTcMmaWarp) {
    // ---- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_f32acc(tc::kFmtBF16, 128, kRtVecs);
      for (int m = 0; m < n_mt && !fail; ++m) {
        if (m >= 2 && !mbar_wait(acc_empty + (m & 1), ((m >> 1) - 1) & 1u, a.status)) {
          fail = 1;
          break;
        }
        tc::fence_after_sync();
        const uint32_t d = tmem + (uint32_t)((m & 1) * kTcAccCols);
        for (int c = 0; c < 4; ++c) {
          const int j = 4 * m + c, s = j % kTcStages;
          if (!mbar_wait(full + s, (j / kTcStages) & 1u, a.status)) {
            fail = 1;
            break;
          }
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc::mma_bf16_ss(d, tc::smem_desc_sw128(ring + s * kTcChunkBytes + 32 * k),
                            tc::smem_desc_sw128(qs + c * kQsChunk + 32 * k), idesc, (c | k) != 0);
          tc::commit(empty + s);
        }
        if (!fail) tc::commit(acc_full + (m & 1));
      }
      // every MMA issued has completed before TMEM is freed (bounded)
      tc::commit(drain);
      mbar_wait(drain, 0, nullptr);
    }
  } else {
    // ---- epilogue: thread tid owns block 128 e + tid of M tile e (TMEM lane tid)
    uint32_t* keys_tg = a.ws_keys + (size_t)tg * a.kv.max_pages;
    const float ninf = -__int_as_float(0x7f800000);
    const int nv = min(kRtVecs, geo.V - v0);
    for (int e = 0; e < n_mt; ++e) {
      const bool ok = mbar_wait(acc_full + (e & 1), (e >> 1) & 1u, a.status);
      if (!__all_sync(0xffffffffu, ok)) {
        fail = 1;
        break;
      }
      tc::fence_after_sync();
      const uint32_t ta = tmem + (uint32_t)((e & 1) * kTcAccCols) + ((uint32_t)(32 * warp) << 16);
      float mx = ninf;
#pragma unroll
      for (int cc = 0; cc < kRtVecs / 16; cc += 2) {
        uint32_t r0[16], r1[16];
        tc::ld_32x32b_x16(ta + 16 * cc, r0);
        tc::ld_32x32b_x16(ta + 16 * cc + 16, r1);
        tc::wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          if (16 * cc + i < nv) mx = fmaxf(mx, __uint_as_float(r0[i]));
          if (16 * cc + 16 + i < nv) mx = fmaxf(mx, __uint_as_float(r1[i]));
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty + (e & 1));
      const int blk = 128 * e + tid;
      if (blk < geo.E && mx != ninf) atomicMax(keys_tg + blk, order_key(mx));
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 0) tc::tmem_dealloc(tmem, 2 * kTcAccCols);
  route_tail(a, t, g, geo.E, base, s_hist, s_bc, s_scan, &s_flag);
}

}  // namespace

int route_splits(int vectors_per_tile) { return (vectors_per_tile + kRtVecs - 1) / kRtVecs; }

size_t route_ws_bytes(int n_tiles, int Hkv, int max_pages, int W) {
  auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const size_t tg = (size_t)n_tiles * Hkv;
  return al(tg * max_pages * 4) + al(tg * W * 4) + al(tg * 8) + al(tg * 4);
}

cudaError_t launch_route(const RouteArgs& a, cudaStream_t st) {
  const size_t smem = 1024 + kSmemBytes;
  const long long grid = (long long)a.n_tiles * a.kv.Hkv * a.nsplit;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
  cudaError_t e;
  if (a.rule == 0) {
    const size_t smem_tc = 1024 + kTcSmemBytes;
    e = set_smem_attr((const void*)route_tc_kernel, smem_tc);
    if (e != cudaSuccess) return e;
    route_tc_kernel<<<(unsigned)grid, kTcThreads, smem_tc, st>>>(a);
  } else {
    e = set_smem_attr((const void*)route_kernel<1>, smem);
    if (e != cudaSuccess) return e;
    route_kernel<1><<<(unsigned)grid, kRtThreads, smem, st>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace sa
