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
  for (int i = tid; i < E; i += blockDim.x) keys[i] = __ldcg(kp + i);
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
    const int n = min(trig ? a.W : a.k, E);
    const int32_t* lst = a.ws_list + (size_t)tg * a.W;
    int32_t* dst = a.kv_idx + (size_t)tg * a.W;
    for (int i = 0; i < a.W; ++i) dst[i] = i < n ? __ldcg(lst + i) : -1;
    a.kv_count[tg] = n;
  }
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

  // ---- the last split of (t, g) selects; the last (t, g) finalizes
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    s_flag = 1;
    if (a.nsplit > 1) s_flag = atomicAdd(a.ws_count + tg, 1u) == (uint32_t)(a.nsplit - 1);
  }
  __syncthreads();
  if (!s_flag) return;
  __threadfence();
  if (tid == 0 && a.nsplit > 1) a.ws_count[tg] = 0;
  route_select_tile(a, t, g, geo.E, base, s_hist, s_bc, s_scan);
  __threadfence();
  __syncthreads();
  if (tid == 0) s_flag = atomicAdd(a.ws_final, 1u) == (uint32_t)(a.n_tiles * Hkv - 1);
  __syncthreads();
  if (!s_flag) return;
  __threadfence();
  if (tid == 0) *a.ws_final = 0;
  route_finalize(a, base);
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
    e = set_smem_attr((const void*)route_kernel<0>, smem);
    if (e != cudaSuccess) return e;
    route_kernel<0><<<(unsigned)grid, kRtThreads, smem, st>>>(a);
  } else {
    e = set_smem_attr((const void*)route_kernel<1>, smem);
    if (e != cudaSuccess) return e;
    route_kernel<1><<<(unsigned)grid, kRtThreads, smem, st>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace sa
