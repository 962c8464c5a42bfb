// Causal attention of query tiles over their routed blocks, on tcgen05.
//
// "Technische Samenvatting: Onzekerheidsgestuurde Selectie voor Blok-schaarse
// Aandacht", "Methodologie" step 5: every tile attends to the blocks its list
// names (the top k, or the top rho*k when the tile triggered); sentinel (-1)
// entries are skipped.  Chunked-prefill rows attend causally: row r at
// position q_pos0 + r sees only keys at positions <= its own.
//
// CTA = (tile, KV head, 256 query vectors) = two Q tiles of 128 vectors that
// share every K/V block, one CTA per SM; a query vector is one (row, query
// head) pair of the tile and owns one TMEM lane in its Q tile's columns.
// Warp-specialised, all waits bounded:
//   warp 8 (one thread)  streams each kept block (64 keys) of K and V by TMA
//                        into a kStages ring (four 64-row x 128 B boxes);
//   warp 9 + t (one thread) issues, for Q tile t and block i in order,
//                        S = Q_t K_i^T (M = 128 vectors, N = 64 keys, K = 128
//                        dims; K-major operands) into one of the tile's two
//                        S/P buffers, then O_t += [P_hi | P_lo] . [V_{i-1} ;
//                        V_{i-1}] (A = P read from tensor memory, N = 128
//                        dims, K = 2 x 64 keys; V read MN-major) once
//                        P_{i-1} is written; the tensor pipe interleaves the
//                        two tiles' MMAs, so one tile's softmax and handoffs
//                        overlap the other tile's MMAs;
//   warps 0-3 / 4-7      the softmax of tile 0 / 1: thread = query vector
//                        (TMEM lane 32 (warp % 4) + lane), its whole row of
//                        64 keys: masks (causal, cache end) only on the
//                        diagonal and cache-end blocks, online softmax in the
//                        log2 domain against a reference max, P split into a
//                        bf16 hi + lo pair (error ~2^-17) stored over S in
//                        tensor memory as the PV MMA's A operand.
// O stays in tensor memory; it is rescaled in place only when a row's max
// grows past the reference by more than 2^8.  The MMAs of one issuing thread
// run in issue order, so the S/P buffer of block i + 2 is written only after
// the PV of block i has read it.  Accumulation order per vector is the block
// order of the list, so results do not depend on scheduling.
#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace sa {
namespace {

constexpr int kBlk = 64;                       // keys per block
constexpr int kTiles = 2;                      // Q tiles of 128 vectors per CTA
constexpr int kSmWarps = 4 * kTiles;           // softmax: one warp per TMEM lane quarter and tile
constexpr int kThreadsTc = 32 * (kSmWarps + 1 + kTiles);
constexpr int kProducerWarp = kSmWarps;
constexpr int kMmaWarp0 = kSmWarps + 1;        // warp kMmaWarp0 + t issues tile t's MMAs
#ifndef SA_TA_STAGES
#define SA_TA_STAGES 3
#endif
constexpr int kStages = SA_TA_STAGES;
constexpr int kBox = kBlk * 128;               // 64 rows x 128 B
constexpr int kStage = 4 * kBox;               // K lo | K hi | V lo | V hi = 32 KiB
constexpr int kQTile = 2 * 128 * 128;          // 128 vectors x 128 dims bf16, two K chunks
constexpr int kOffQ = 0;
constexpr int kOffRing = kOffQ + kTiles * kQTile;
constexpr int kOffBars = kOffRing + kStages * kStage;
// kv full/empty per stage; per tile and buffer: S full, P full, PV done; drain
constexpr int kNumBars = 2 * kStages + 3 * kTiles * 2 + 1;
constexpr int kOffList = kOffBars + kNumBars * 8 + 8;
// tensor memory: tile t's two S/P buffers at columns [128 t, 128 t + 128) (64
// fp32 columns each; P's bf16 hi | lo pairs overwrite them), its O
// accumulator at [256 + 128 t, 256 + 128 t + 128)
constexpr uint32_t kColSP = 0;
constexpr uint32_t kColO = 256;
static_assert(1024 + kOffList > 114 * 1024, "one CTA per SM: it allocates all 512 TMEM columns");

// 2^x by the hardware approximation (relative error about 2^-22; 2^-inf = +0).
SA_DEV float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// MN-major view of V (keys x dims, dims contiguous): 8-key atoms 1 KiB apart,
// the two 64-dim boxes 8 KiB apart.
SA_DEV uint64_t v_desc(const unsigned char* v) {
  const uint64_t d = tc::smem_desc_sw128(v);
  return (d & ~(0x3FFFull << 16)) | ((uint64_t)(kBox >> 4) << 16);
}

__global__ void __launch_bounds__(kThreadsTc, 1) tile_attn_tc_kernel(const __grid_constant__ TileAttnArgs a) {
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint32_t s_tmem;
  __shared__ uint32_t s_scan[32];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* qs = base + kOffQ;
  unsigned char* ring = base + kOffRing;
  uint64_t* kv_full = reinterpret_cast<uint64_t*>(base + kOffBars);
  uint64_t* kv_empty = kv_full + kStages;
  uint64_t* s_full = kv_empty + kStages;   // [tile][buffer]
  uint64_t* p_full = s_full + 2 * kTiles;  // [tile][buffer]
  uint64_t* o_full = p_full + 2 * kTiles;  // [tile][block parity]: PV of the block done
  uint64_t* drain = o_full + 2 * kTiles;
  int* blist = reinterpret_cast<int*>(base + kOffList);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Hkv = a.kv.Hkv, G = a.G;
  const int nmc = a.n_mchunks;
  const int mc = blockIdx.x % nmc;
  // (tile, KV head) of this CTA.  With few enough pairs the CTAs take them
  // longest list first (the hardware starts CTAs in index order, so the long
  // lists of triggered tiles start in the first wave instead of ending the
  // launch): every CTA ranks all pairs by (count desc, index asc) and takes
  // the pair of rank blockIdx.x / nmc.
  __shared__ int s_cnt[kThreadsTc];
  __shared__ int s_pair;
  const int n_pairs = a.n_tiles * Hkv;
  int tg = blockIdx.x / nmc;
  if (n_pairs <= kThreadsTc) {
    int mine = 0;
    if (tid < n_pairs) {
      mine = __ldg(a.count + tid);
      if (mine < 0 || mine > a.max_sel) mine = 0;
      s_cnt[tid] = mine;
    }
    __syncthreads();
    if (tid < n_pairs) {
      int rank = 0;
      for (int u = 0; u < n_pairs; ++u) {
        const int c = s_cnt[u];
        rank += (c > mine || (c == mine && u < tid)) ? 1 : 0;
      }
      if (rank == tg) s_pair = tid;
    }
    __syncthreads();
    tg = s_pair;
  }
  const int t = tg / Hkv, g = tg % Hkv;
  const int N = a.kv.seq_len[0];
  const int P = (N + kBlk - 1) / kBlk;
  const int row0 = t * a.tile_rows;
  const int rows_t = min(a.tile_rows, a.n_rows - row0);
  const int V = rows_t * G;
  const float ninf = -__int_as_float(0x7f800000);

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_empty + s, kTiles);  // each tile's MMA thread commits after its PV
    }
    for (int x = 0; x < 2 * kTiles; ++x) {
      mbar_init(s_full + x, 1);
      mbar_init(p_full + x, 4);  // the tile's four softmax warps
      mbar_init(o_full + x, 1);
    }
    mbar_init(drain, kTiles);
    fence_barrier_init();
    prefetch_tmap(&a.tmap_k);
    prefetch_tmap(&a.tmap_v);
  }
  if (warp == 0) {
    tc::tmem_alloc(&s_tmem, 512);
    tc::tmem_relinquish();
  }

  // ---- the kept blocks in list order: sentinels skipped, out-of-range flagged.
  // Thread i takes a contiguous range of the list; one scan places them.
  int n = __ldg(a.count + tg);
  if (n < 0 || n > a.max_sel) {
    if (tid == 0) flag_status(a.status, SA_ERR_DEVICE_CHECK);
    n = 0;
  }
  const int32_t* lst = a.idx + (size_t)tg * a.max_sel;
  const int per = (n + kThreadsTc - 1) / kThreadsTc;
  const int i0 = min(n, tid * per), i1 = min(n, i0 + per);
  uint32_t cnt = 0;
  for (int i = i0; i < i1; ++i) {
    const int blk = __ldg(lst + i);
    if (blk >= P) flag_status(a.status, SA_ERR_DEVICE_CHECK);
    cnt += (blk >= 0 && blk < P) ? 1u : 0u;
  }
  uint32_t nb_u;
  uint32_t pos = block_excl_scan(cnt, s_scan, nb_u);
  for (int i = i0; i < i1; ++i) {
    const int blk = __ldg(lst + i);
    if (blk >= 0 && blk < P) blist[pos++] = blk;
  }
  const int nb = (int)nb_u;

  // ---- the CTA's 256 query vectors: tile vi / 128, row vi % 128 of its
  // K-major, 128B-swizzled Q (rows past V zero); 8 loads in flight per thread
  const __nv_bfloat16* Q = reinterpret_cast<const __nv_bfloat16*>(a.q);
  const int v0 = mc * 128 * kTiles;
  constexpr int kQPieces = 128 * kTiles * 16;
#pragma unroll 1
  for (int b0 = 0; b0 < kQPieces; b0 += 8 * kThreadsTc) {
    uint4 rw[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int x = b0 + i * kThreadsTc + tid;
      const int vi = x >> 4, d8 = x & 15, v = v0 + vi;
      rw[i] = make_uint4(0u, 0u, 0u, 0u);
      if (x < kQPieces && v < V)
        rw[i] = ldg_nc128(Q + ((size_t)(row0 + v / G) * a.Hq + (size_t)g * G + v % G) * kHeadDim + 8 * d8);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int x = b0 + i * kThreadsTc + tid;
      if (x >= kQPieces) continue;
      const int vi = x >> 4, d8 = x & 15;
      *reinterpret_cast<uint4*>(qs + (vi >> 7) * kQTile + (d8 >> 3) * (128 * 128) + swz128(vi & 127, d8 & 7)) =
          rw[i];
    }
  }
  fence_proxy_async();  // generic writes (queries, list) before the async proxy reads them
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = s_tmem;
  int fail = 0;

  if (warp == kProducerWarp) {
    // ---- TMA producer: block i -> stage i % kStages (freed once both tiles' PV read it)
    if (lane == 0) {
      const long long rowbase = (long long)g * a.kv.cap;  // B == 1: unit = KV head
      int issued = 0;
      for (int i = 0; i < nb; ++i) {
        const int s = i % kStages;
        if (i >= kStages && !mbar_wait(kv_empty + s, ((i / kStages) - 1) & 1u, a.status)) {
          fail = 1;
          break;
        }
        unsigned char* st = ring + s * kStage;
        const int y = (int)(rowbase + (long long)blist[i] * kBlk);
        mbar_arrive_expect_tx(kv_full + s, kStage);
        tma_load_2d(st + 0 * kBox, &a.tmap_k, 0, y, kv_full + s);
        tma_load_2d(st + 1 * kBox, &a.tmap_k, 64, y, kv_full + s);
        tma_load_2d(st + 2 * kBox, &a.tmap_v, 0, y, kv_full + s);
        tma_load_2d(st + 3 * kBox, &a.tmap_v, 64, y, kv_full + s);
        issued = i + 1;
      }
      // every copy issued has landed before the CTA moves on (bounded)
      for (int i = max(0, issued - kStages); i < issued; ++i)
        mbar_wait(kv_full + (i % kStages), (i / kStages) & 1u, nullptr);
    }
  } else if (warp >= kMmaWarp0) {
    // ---- MMA issuer of tile tt, in order: QK of block i (its K/V stage
    // landed; its S/P buffer was last read by the PV of block i - 2, issued
    // before), then the PV of block i - 1 once P_{i-1} is written.  One thread
    // per tile: an MMA issue returns about when the tensor pipe has taken the
    // MMAs, so a single thread serving both tiles held each tile's PV behind
    // the other tile's QKs; the pipe interleaves the two threads' MMAs.  A K/V
    // stage is free once both tiles' PVs that read it are done.
    const int tt = warp - kMmaWarp0;
    if (lane == 0) {
      const uint32_t idesc_s = tc::idesc_f32acc(tc::kFmtBF16, 128, kBlk);
      const uint32_t idesc_o = tc::idesc_f32acc(tc::kFmtBF16, 128, kHeadDim) | (1u << 16);  // V MN-major
      const unsigned char* qt = qs + tt * kQTile;
      auto pv = [&](int i) -> bool {
        const int s = i % kStages, b = i & 1;
        if (!mbar_wait(p_full + 2 * tt + b, (i >> 1) & 1u, a.status)) return false;
        tc::fence_after_sync();
        const unsigned char* vb = ring + s * kStage + 2 * kBox;
#pragma unroll
        for (int j = 0; j < 8; ++j)  // K = [P_hi keys 0-63 | P_lo keys 0-63], 16 per step
          tc::mma_bf16_ts(tmem + kColO + 128u * tt, tmem + kColSP + 128u * tt + 64u * b + 8u * j,
                          v_desc(vb + 16 * 128 * (j & 3)), idesc_o, i > 0 || j != 0);
        tc::commit(o_full + 2 * tt + b);
        tc::commit(kv_empty + s);
        return true;
      };
      for (int i = 0; i < nb && !fail; ++i) {
        const int s = i % kStages, b = i & 1;
        if (!mbar_wait(kv_full + s, (i / kStages) & 1u, a.status)) {
          fail = 1;
          break;
        }
        tc::fence_after_sync();
        const unsigned char* kb = ring + s * kStage;
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc::mma_bf16_ss(tmem + kColSP + 128u * tt + 64u * b, tc::smem_desc_sw128(qt + c * (128 * 128) + 32 * k),
                            tc::smem_desc_sw128(kb + c * kBox + 32 * k), idesc_s, (c | k) != 0);
        tc::commit(s_full + 2 * tt + b);
        if (i > 0 && !pv(i - 1)) fail = 1;
      }
      if (!fail && nb > 0 && !pv(nb - 1)) fail = 1;
      // every MMA issued has completed before TMEM is freed (bounded)
      tc::commit(drain);
      mbar_wait(drain, 0, nullptr);
    }
  } else {
    // ---- softmax of tile tt: TMEM lane r = 32 (warp % 4) + lane is query
    // vector v0 + 128 tt + r; the thread owns that vector's whole row.
    const int tt = warp >> 2, quarter = warp & 3;
    const int r = 32 * quarter + lane;
    const int v = v0 + 128 * tt + r;
    const bool vok = v < V;
    const int qpos = vok ? a.q_pos0 + row0 + v / G : -1;
    const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
    const uint32_t sp_base = tmem + lane_off + kColSP + 128u * tt;
    const uint32_t to = tmem + lane_off + kColO + 128u * tt;
    uint64_t* s_full_t = s_full + 2 * tt;
    uint64_t* p_full_t = p_full + 2 * tt;
    uint64_t* o_full_t = o_full + 2 * tt;
    // PV of block j complete.  A tile's PV barrier for one block parity never
    // runs two phases ahead of a wait here: PV of block j + 2 needs P_{j+2},
    // which this thread writes later (or, after the loop, does not exist).
    auto wait_pv = [&](int j) -> bool {
      const bool ok = mbar_wait(o_full_t + (j & 1), (j >> 1) & 1u, a.status);
      return __all_sync(0xffffffffu, ok);
    };
    float mref = ninf, lh = 0.f;  // reference max (log2 units) and the row sum against it
    const float sl2 = a.scale_log2;
    for (int i = 0; i < nb; ++i) {
      const int b = i & 1;
      const bool ok = mbar_wait(s_full_t + b, (i >> 1) & 1u, a.status);
      if (!__all_sync(0xffffffffu, ok)) {
        fail = 1;
        break;
      }
      tc::fence_after_sync();
      const uint32_t ts = sp_base + 64u * b;
      uint32_t r0[16], r1[16], r2[16], r3[16];  // keys 0-15, 16-31, 32-47, 48-63
      tc::ld_32x32b_x16(ts, r0);
      tc::ld_32x32b_x16(ts + 16, r1);
      tc::ld_32x32b_x16(ts + 32, r2);
      tc::ld_32x32b_x16(ts + 48, r3);
      tc::wait_ld();
      tc::reg_fence(r0);
      tc::reg_fence(r1);
      tc::reg_fence(r2);
      tc::reg_fence(r3);
      const int kb0 = blist[i] * kBlk;
      // Blocks fully visible to every row of the warp (all but the diagonal and
      // the cache end) skip the masks, and with a positive scale the max is
      // taken on raw scores (scaling commutes with max); four max chains.
      const bool fast = sl2 > 0.f && __all_sync(0xffffffffu, kb0 + kBlk - 1 <= qpos && kb0 + kBlk <= N);
      float sv[64], mq[4] = {ninf, ninf, ninf, ninf}, mul;
#pragma unroll
      for (int x = 0; x < 16; ++x) {
        sv[x] = __uint_as_float(r0[x]);
        sv[16 + x] = __uint_as_float(r1[x]);
        sv[32 + x] = __uint_as_float(r2[x]);
        sv[48 + x] = __uint_as_float(r3[x]);
      }
      if (fast) {
#pragma unroll
        for (int x = 0; x < 64; ++x) mq[x & 3] = fmaxf(mq[x & 3], sv[x]);
        mul = sl2;
      } else {
#pragma unroll
        for (int x = 0; x < 64; ++x) {
          const int key = kb0 + x;
          sv[x] = (key <= qpos && key < N) ? sv[x] * sl2 : ninf;
          mq[x & 3] = fmaxf(mq[x & 3], sv[x]);
        }
        mul = 1.f;
      }
      float mx = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
      if (fast) mx *= sl2;
      // raise the reference max when the row's max passes it by more than 8
      const float mn = fmaxf(mref, mx);
      const bool upd = mn != ninf && (mref == ninf || mn > mref + 8.f);
      const float alpha = !upd ? 1.f : (mref == ninf ? 0.f : fast_exp2(mref - mn));
      if (upd) mref = mn;
      lh *= alpha;
      if (i > 0 && __any_sync(0xffffffffu, upd)) {
        // O holds blocks [0, i): once the last of them is in, scale this row in place
        if (!wait_pv(i - 1)) {
          fail = 1;
          break;
        }
        tc::fence_after_sync();
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t q[16];
          tc::ld_32x32b_x16(to + 16 * c, q);
          tc::wait_ld();
#pragma unroll
          for (int x = 0; x < 16; ++x) q[x] = __float_as_uint(__uint_as_float(q[x]) * alpha);
          tc::st_32x32b_x16(to + 16 * c, q);
        }
      }
      const float nmn = mref == ninf ? 0.f : -mref;  // all masked so far: every p is exp2(-inf) = 0
      // P = exp2(s - mref) as bf16 hi + lo pairs over S: hi pairs in columns
      // 0-31, lo pairs in 32-63 (S of this block was read above)
      float rq[4] = {0.f, 0.f, 0.f, 0.f};  // four independent partial row sums
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        uint32_t phi[16], plo[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float p0 = fast_exp2(fmaf(sv[32 * h2 + 2 * j], mul, nmn));
          const float p1 = fast_exp2(fmaf(sv[32 * h2 + 2 * j + 1], mul, nmn));
          rq[j & 3] += p0 + p1;
          phi[j] = pack_bf16(p0, p1);
          plo[j] = pack_bf16(p0 - bf16_lo(phi[j]), p1 - bf16_hi(phi[j]));
        }
        tc::st_32x32b_x16(ts + 16 * h2, phi);
        tc::st_32x32b_x16(ts + 32 + 16 * h2, plo);
      }
      lh += (rq[0] + rq[1]) + (rq[2] + rq[3]);
      // V rows past the cache end hold other data: zero them before PV reads
      // them (each tile's warps do it, as each tile's PV waits only for its own)
      if (kb0 + kBlk > N) {
        unsigned char* st = ring + (i % kStages) * kStage;
        for (int x = r; x < (kb0 + kBlk - N) * 16; x += 128) {
          const int row = (N - kb0) + (x >> 4), ch = x & 15;
          *reinterpret_cast<uint4*>(st + (2 + (ch >> 3)) * kBox + swz128(row, ch & 7)) = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async();  // the zeroed V rows before the tensor cores read them
      }
      tc::wait_st();
      tc::fence_before_sync();  // P and the rescaled O before PV_i reads them
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full_t + b);
    }
    // the row's output: PV of the last block (the earlier ones ran before it),
    // then O / l straight from tensor memory
    if (!fail && nb > 0 && !wait_pv(nb - 1)) fail = 1;
    if (!fail) {
      tc::fence_after_sync();
      const size_t orow = (size_t)(row0 + v / G) * a.Hq + (size_t)g * G + v % G;
      const float inv = lh > 0.f ? 1.f / lh : 0.f;
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t q[16];
        if (nb > 0) {
          tc::ld_32x32b_x16(to + 16 * c, q);
          tc::wait_ld();
        } else {
#pragma unroll
          for (int x = 0; x < 16; ++x) q[x] = 0u;
        }
        if (vok) {
          float* dst = a.out + orow * kHeadDim + 16 * c;
#pragma unroll
          for (int x = 0; x < 16; x += 4)
            *reinterpret_cast<float4*>(dst + x) =
                make_float4(__uint_as_float(q[x]) * inv, __uint_as_float(q[x + 1]) * inv,
                            __uint_as_float(q[x + 2]) * inv, __uint_as_float(q[x + 3]) * inv);
        }
      }
      if (vok && a.lse) a.lse[orow] = lh > 0.f ? mref * kLn2 + logf(lh) : ninf;
    }
  }
  tc::fence_before_sync();
  __syncthreads_and(!fail);
  tc::fence_after_sync();
  if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

}  // namespace

size_t tile_attn_tc_smem_bytes(int max_sel) { return 1024 + kOffList + (size_t)max_sel * 4; }

cudaError_t launch_tile_attn_tc(const TileAttnArgs& a, cudaStream_t st) {
  const size_t smem = tile_attn_tc_smem_bytes(a.max_sel);
  const long long grid = (long long)a.n_tiles * a.kv.Hkv * a.n_mchunks;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
  const cudaError_t e = set_smem_attr((const void*)tile_attn_tc_kernel, smem);
  if (e != cudaSuccess) return e;
  tile_attn_tc_kernel<<<(unsigned)grid, kThreadsTc, smem, st>>>(a);
  return cudaGetLastError();
}

// CTAs per (tile, KV head): 256 query vectors each.
int tile_attn_tc_mchunks(int vectors_per_tile) { return (vectors_per_tile + 128 * kTiles - 1) / (128 * kTiles); }

}  // namespace sa
