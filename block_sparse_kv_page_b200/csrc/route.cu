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
//     the 5th-generation tensor cores (tcgen05, accumulators in tensor memory):
//       envelope: [kmin|kmax] (128 blocks x 256 bf16) . [q-|q+]^T, exact
//                 products, fp32 accumulation;
//       centroid: kmean (fp32) split into three bf16 parts hi + mid + lo,
//                 three bf16 GEMMs against the exact bf16 queries;
//     each block's max over the vectors is folded into the tile-score keys
//     with atomicMax on order-preserving uint32 keys.
//   * The last split CTA of (t, g) (atomic counter) selects the top
//     max(rho*k, k+1) eligible blocks by radix select, sorts them to rank
//     order (score desc, index asc) and computes sigma in double.
//   * The last (t, g) CTA computes sigma_bar, the quantile threshold, the
//     triggers and writes the sentinel-padded lists.
#include "common.cuh"
#include "internal.h"
#include "radix.cuh"
#include "route_select.cuh"
#include "tcgen05.cuh"

namespace sa {
namespace {

using namespace rsel;

constexpr int kRtVecs = 224;                                // query vectors per CTA (MMA N)
constexpr int kQsChunk = kRtVecs * 128;                      // one 128-byte K chunk of all vectors
constexpr int kQsBytes = 4 * kQsChunk;                       // 112 KiB ([q- | q+], 256 bf16)

// Max over the first nv (<= kRtVecs) fp32 columns of this thread's TMEM lane
// starting at ta: four loads in flight per wait, four independent max chains,
// no per-column test when every column is valid.
SA_DEV float acc_row_max(uint32_t ta, int nv) {
  const float ninf = -__int_as_float(0x7f800000);
  float m[4] = {ninf, ninf, ninf, ninf};
  constexpr int kChunks = kRtVecs / 16;  // 14
#pragma unroll
  for (int c0 = 0; c0 < kChunks; c0 += 4) {
    uint32_t r[4][16];
#pragma unroll
    for (int c = 0; c < 4; ++c)
      if (c0 + c < kChunks) tc::ld_32x32b_x16(ta + 16 * (c0 + c), r[c]);
    tc::wait_ld();
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if (c0 + c >= kChunks) continue;
      tc::reg_fence(r[c]);
      if (nv >= kRtVecs) {
#pragma unroll
        for (int i = 0; i < 16; ++i) m[i & 3] = fmaxf(m[i & 3], __uint_as_float(r[c][i]));
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (16 * (c0 + c) + i < nv) m[i & 3] = fmaxf(m[i & 3], __uint_as_float(r[c][i]));
      }
    }
  }
  return fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
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

// ---------------------------------------------------------------- decode router
// The router applied to decode: every sequence of the batch is a tile of one
// query row (position N_b - 1), so all of its pages are eligible and its
// block scores are the group scores the decode scoring wrote (max over the G
// heads).  CTA = (sequence, KV head): rank-order selection and sigma; the last
// CTA computes sigma_bar, the quantile threshold over the batch's sequences,
// the triggers and the sentinel-padded lists.  One wave of latency-bound
// selections: 512 threads a CTA shorten each one's loops (256: 6-8% slower).
constexpr int kRdThreads = 512;

__global__ void __launch_bounds__(kRdThreads) route_decode_kernel(const __grid_constant__ RouteArgs a) {
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint32_t s_hist[512];
  __shared__ uint32_t s_scan[32];
  __shared__ uint32_t s_bc[8];
  __shared__ int s_flag;
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 15) & ~static_cast<uintptr_t>(15));
  grid_dep_wait();  // the scores come from the previous kernel of the stream
  const int tg = blockIdx.x;
  const int b = tg / a.kv.Hkv, g = tg - b * a.kv.Hkv;
  const int N = a.kv.seq_len[b];
  int E = 0;
  if (N < 1 || N > a.kv.cap) {
    if (threadIdx.x == 0 && g == 0) flag_status(a.status, SA_ERR_DEVICE_CHECK);
  } else {
    E = (N + a.kv.page_size - 1) / a.kv.page_size;
    if (E > a.kv.max_pages) {
      if (threadIdx.x == 0 && g == 0) flag_status(a.status, SA_ERR_DEVICE_CHECK);
      E = 0;
    }
  }
  route_select_tile(a, b, g, E, base, s_hist, s_bc, s_scan);
  __syncthreads();
  if (threadIdx.x == 0) s_flag = atom_add_acq_rel_u32(a.ws_final, 1u) == (uint32_t)(gridDim.x - 1);
  __syncthreads();
  if (!s_flag) return;
  if (threadIdx.x == 0) *a.ws_final = 0;
  route_finalize(a, base);
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
// ring depth: 4 stages of one K-chunk each, so stage j % 4 always holds K-chunk
// j % 4 of its M tile (measured 0.094-0.095 ms against 0.098 with 5 or 6 stages,
// 0.099 with 3, 0.107 with 2)
constexpr int kTcStages = 4;
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
  // CTA -> (split, tile, KV head), split-major: the first wave holds the
  // first split of every (tile, KV head), so the selection that the last split
  // of a pair runs falls at the end of its SM's work, not in front of a
  // second-wave CTA
  const int n_tg = a.n_tiles * a.kv.Hkv;
  const int sp = blockIdx.x / n_tg;
  const int tg = blockIdx.x % n_tg;
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
      const float mx = acc_row_max(ta, nv);
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

// ---------------------------------------------------------------- tensor-core (tcgen05) centroid scoring
// The block means are fp32; the MMA takes bf16.  Each mean is split into
// three bf16 parts hi + mid + lo (each the round-to-nearest of what the
// previous parts left, so together they carry the fp32 mantissa), and the
// scores are three bf16 GEMMs against the exact bf16 queries accumulated in
// one fp32 accumulator: products exact, only the fp32 sums round.
//   warp 4 (one thread)  copies the fp32 means by TMA in half-chunks (128
//                        blocks x 64 dims = two 16 KiB boxes) into kCrRaw stages;
//   warps 0-3            split each half-chunk into the three bf16 parts
//                        (128B-swizzled K-major tiles, kCrConv stages), then
//                        run the max epilogue of the previous M tile;
//   warp 5 (one thread)  issues 3 parts x 4 MMAs per half-chunk.
constexpr int kCrRaw = 2;                                    // fp32 half-chunk stages (32 KiB)
constexpr int kCrConv = 2;                                   // bf16 stages (3 parts x 16 KiB)
constexpr int kCrQChunk = kRtVecs * 128;                     // 224 vectors x 64 bf16 dims
constexpr int kCrOffRaw = 2 * kCrQChunk;
constexpr int kCrOffConv = kCrOffRaw + kCrRaw * 2 * kTcChunkBytes;
constexpr int kCrOffBars = kCrOffConv + kCrConv * 3 * kTcChunkBytes;
constexpr int kCrNumBars = 4 * kCrRaw + 4 + 1;               // raw full/empty, conv full/empty, acc x4, drain
constexpr int kCrSmemBytes = kCrOffBars + kCrNumBars * 8 + 16;
static_assert(kCrQChunk % 1024 == 0 && kCrOffRaw % 1024 == 0 && kCrOffConv % 1024 == 0, "1 KiB atoms");
static_assert(1024 + kCrSmemBytes > 114 * 1024 && 1024 + kCrSmemBytes <= 227 * 1024, "one CTA per SM");

__global__ void __launch_bounds__(kTcThreads, 1) route_tc_centroid_kernel(const __grid_constant__ RouteArgs a) {
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint32_t s_hist[256];
  __shared__ uint32_t s_scan[32];
  __shared__ uint32_t s_bc[4];
  __shared__ int s_flag;
  __shared__ uint32_t s_tmem;
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* qs = base;
  unsigned char* raw = base + kCrOffRaw;
  unsigned char* conv = base + kCrOffConv;
  uint64_t* raw_full = reinterpret_cast<uint64_t*>(base + kCrOffBars);
  uint64_t* raw_empty = raw_full + kCrRaw;
  uint64_t* conv_full = raw_empty + kCrRaw;
  uint64_t* conv_empty = conv_full + kCrConv;
  uint64_t* acc_full = conv_empty + kCrConv;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Hkv = a.kv.Hkv;
  // CTA -> (split, tile, KV head), split-major: the first wave holds the
  // first split of every (tile, KV head), so the selection that the last split
  // of a pair runs falls at the end of its SM's work, not in front of a
  // second-wave CTA
  const int n_tg = a.n_tiles * a.kv.Hkv;
  const int sp = blockIdx.x / n_tg;
  const int tg = blockIdx.x % n_tg;
  const int t = tg / Hkv, g = tg % Hkv;
  const int N = a.kv.seq_len[0];
  const RouteGeom geo = route_geom(a, t, N);
  const int v0 = sp * kRtVecs;

  if (tid == 0) {
    for (int s = 0; s < kCrRaw; ++s) {
      mbar_init(raw_full + s, 1);
      mbar_init(raw_empty + s, kTcEpiWarps);
    }
    for (int s = 0; s < kCrConv; ++s) {
      mbar_init(conv_full + s, kTcEpiWarps);
      mbar_init(conv_empty + s, 1);
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
  const int n_hc = 2 * n_mt;            // half-chunks (64 dims each)
  const int row_base = g * a.kv.max_pages;
  auto load = [&](int j) {  // producer thread: fp32 dims [64 (j&1), +64) of M tile j >> 1
    const int s = j % kCrRaw;
    unsigned char* dst = raw + s * (2 * kTcChunkBytes);
    mbar_arrive_expect_tx(raw_full + s, 2 * kTcChunkBytes);
    tma_load_2d(dst, &a.tmap_meta_tc, 64 * (j & 1), row_base + 128 * (j >> 1), raw_full + s);
    tma_load_2d(dst + kTcChunkBytes, &a.tmap_meta_tc, 64 * (j & 1) + 32, row_base + 128 * (j >> 1), raw_full + s);
  };
  const int n_pre = min(kCrRaw, n_hc);
  if (warp == kTcProducerWarp && lane == 0)
    for (int j = 0; j < n_pre; ++j) load(j);

  // ---- the split's queries as bf16, K-major 128B-swizzled (the MMA's B operand)
  constexpr int kQPieces = kRtVecs * 16;
  const __nv_bfloat16* Q = reinterpret_cast<const __nv_bfloat16*>(a.q);
#pragma unroll 1
  for (int b0 = 0; b0 < kQPieces; b0 += 8 * kTcThreads) {
    uint4 rw[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int x = b0 + i * kTcThreads + tid;
      const int vi = x >> 4, d8 = x & 15, v = v0 + vi;
      rw[i] = make_uint4(0u, 0u, 0u, 0u);
      if (x < kQPieces && v < geo.V) {
        const int r = v / a.G, j = v - r * a.G;
        rw[i] = ldg_nc128(Q + ((size_t)(geo.row0 + r) * a.Hq + (size_t)g * a.G + j) * kHeadDim + 8 * d8);
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int x = b0 + i * kTcThreads + tid;
      if (x >= kQPieces) continue;
      const int vi = x >> 4, d8 = x & 15;
      *reinterpret_cast<uint4*>(qs + (d8 >> 3) * kCrQChunk + swz128(vi, d8 & 7)) = rw[i];
    }
  }
  fence_proxy_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = s_tmem;
  int fail = 0;

  if (warp == kTcProducerWarp) {
    if (lane == 0) {
      int issued = n_pre;
      for (int j = n_pre; j < n_hc; ++j) {
        const int s = j % kCrRaw;
        if (!mbar_wait(raw_empty + s, ((j / kCrRaw) - 1) & 1u, a.status)) {
          fail = 1;
          break;
        }
        load(j);
        issued = j + 1;
      }
      for (int j = max(0, issued - kCrRaw); j < issued; ++j)  // every copy has landed (bounded)
        mbar_wait(raw_full + (j % kCrRaw), (j / kCrRaw) & 1u, nullptr);
    }
  } else if (warp == kTcMmaWarp) {
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_f32acc(tc::kFmtBF16, 128, kRtVecs);
      for (int m = 0; m < n_mt && !fail; ++m) {
        if (m >= 2 && !mbar_wait(acc_empty + (m & 1), ((m >> 1) - 1) & 1u, a.status)) {
          fail = 1;
          break;
        }
        tc::fence_after_sync();
        const uint32_t d = tmem + (uint32_t)((m & 1) * kTcAccCols);
        for (int c = 0; c < 2; ++c) {
          const int j = 2 * m + c, s = j % kCrConv;
          if (!mbar_wait(conv_full + s, (j / kCrConv) & 1u, a.status)) {
            fail = 1;
            break;
          }
          const unsigned char* cs = conv + s * (3 * kTcChunkBytes);
#pragma unroll
          for (int part = 0; part < 3; ++part)
#pragma unroll
            for (int k = 0; k < 4; ++k)
              tc::mma_bf16_ss(d, tc::smem_desc_sw128(cs + part * kTcChunkBytes + 32 * k),
                              tc::smem_desc_sw128(qs + c * kCrQChunk + 32 * k), idesc, (c | part | k) != 0);
          tc::commit(conv_empty + s);
        }
        if (!fail) tc::commit(acc_full + (m & 1));
      }
      tc::commit(drain);
      mbar_wait(drain, 0, nullptr);
    }
  } else {
    // ---- warps 0-3: thread tid is block (row) tid of every M tile
    // split half-chunk j (fp32, two swizzled boxes) into three bf16 parts
    auto convert = [&](int j) -> bool {
      const int sr = j % kCrRaw, sc = j % kCrConv;
      bool ok = mbar_wait(raw_full + sr, (j / kCrRaw) & 1u, a.status);
      if (ok && j >= kCrConv) ok = mbar_wait(conv_empty + sc, ((j / kCrConv) - 1) & 1u, a.status);
      if (!__all_sync(0xffffffffu, ok)) return false;
      tc::fence_after_sync();
      const unsigned char* src = raw + sr * (2 * kTcChunkBytes);
      unsigned char* dst = conv + sc * (3 * kTcChunkBytes);
#pragma unroll 2
      for (int p8 = 0; p8 < 8; ++p8) {  // output piece p8: dims 8 p8 .. 8 p8 + 7 of the half-chunk
        const unsigned char* box = src + (p8 >> 2) * kTcChunkBytes;
        const uint4 xa = lds128(box + swz128(tid, 2 * (p8 & 3)));
        const uint4 xb = lds128(box + swz128(tid, 2 * (p8 & 3) + 1));
        const float x[8] = {__uint_as_float(xa.x), __uint_as_float(xa.y), __uint_as_float(xa.z),
                            __uint_as_float(xa.w), __uint_as_float(xb.x), __uint_as_float(xb.y),
                            __uint_as_float(xb.z), __uint_as_float(xb.w)};
        uint32_t hi[4], mid[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          hi[e] = pack_bf16(x[2 * e], x[2 * e + 1]);
          const float r0 = x[2 * e] - bf16_lo(hi[e]), r1 = x[2 * e + 1] - bf16_hi(hi[e]);
          mid[e] = pack_bf16(r0, r1);
          lo[e] = pack_bf16(r0 - bf16_lo(mid[e]), r1 - bf16_hi(mid[e]));
        }
        const uint32_t o = swz128(tid, p8);
        *reinterpret_cast<uint4*>(dst + o) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(dst + kTcChunkBytes + o) = make_uint4(mid[0], mid[1], mid[2], mid[3]);
        *reinterpret_cast<uint4*>(dst + 2 * kTcChunkBytes + o) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
      fence_proxy_async();  // generic accesses of both stages before the async proxy's next ones
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(conv_full + sc);
        mbar_arrive(raw_empty + sr);
      }
      return true;
    };
    uint32_t* keys_tg = a.ws_keys + (size_t)tg * a.kv.max_pages;
    const float ninf = -__int_as_float(0x7f800000);
    const int nv = min(kRtVecs, geo.V - v0);
    for (int j = 0; j < min(2, n_hc) && !fail; ++j)
      if (!convert(j)) fail = 1;
    for (int e = 0; e < n_mt && !fail; ++e) {
      for (int j = 2 * (e + 1); j < min(2 * (e + 2), n_hc); ++j)  // the next M tile's parts first
        if (!convert(j)) {
          fail = 1;
          break;
        }
      if (fail) break;
      const bool ok = mbar_wait(acc_full + (e & 1), (e >> 1) & 1u, a.status);
      if (!__all_sync(0xffffffffu, ok)) {
        fail = 1;
        break;
      }
      tc::fence_after_sync();
      const uint32_t ta = tmem + (uint32_t)((e & 1) * kTcAccCols) + ((uint32_t)(32 * warp) << 16);
      const float mx = acc_row_max(ta, nv);
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
  return al(tg * max_pages * 4) + al(tg * 8) + al(tg * 4);
}

size_t route_decode_smem_bytes(int max_pages, int W, int k, int n_tiles, int Hkv) {
  int cap = W > k + 1 ? W : k + 1;
  if (cap > max_pages) cap = max_pages;
  int n2 = 1;
  while (n2 < cap) n2 <<= 1;
  const size_t sel = (((size_t)max_pages * 4 + 15) & ~(size_t)15) + (size_t)n2 * 8;
  const size_t fin = finalize_smem_bytes(n_tiles, Hkv);
  return 16 + (sel > fin ? sel : fin);
}

cudaError_t launch_route_decode(const RouteArgs& a, cudaStream_t st) {
  const size_t smem = route_decode_smem_bytes(a.kv.max_pages, a.W, a.k, a.n_tiles, a.kv.Hkv);
  const cudaError_t e = set_smem_attr((const void*)route_decode_kernel, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(route_decode_kernel, (unsigned)(a.n_tiles * a.kv.Hkv), kRdThreads, smem, st, a);
}

cudaError_t launch_route(const RouteArgs& a, cudaStream_t st) {
  const long long grid = (long long)a.n_tiles * a.kv.Hkv * a.nsplit;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
  cudaError_t e;
  if (a.rule == 0) {
    const size_t smem_tc = 1024 + kTcSmemBytes;
    e = set_smem_attr((const void*)route_tc_kernel, smem_tc);
    if (e != cudaSuccess) return e;
    route_tc_kernel<<<(unsigned)grid, kTcThreads, smem_tc, st>>>(a);
  } else {
    const size_t smem_tc = 1024 + kCrSmemBytes;
    e = set_smem_attr((const void*)route_tc_centroid_kernel, smem_tc);
    if (e != cudaSuccess) return e;
    route_tc_centroid_kernel<<<(unsigned)grid, kTcThreads, smem_tc, st>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace sa
