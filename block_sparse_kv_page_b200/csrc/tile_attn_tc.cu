// Causal attention of query tiles over their routed blocks, on tcgen05.
//
// "Technische Samenvatting: Onzekerheidsgestuurde Selectie voor Blok-schaarse
// Aandacht", "Methodologie" step 5: every tile attends to the blocks its list
// names (the top k, or the top rho*k when the tile triggered); sentinel (-1)
// entries are skipped.  Chunked-prefill rows attend causally: row r at
// position q_pos0 + r sees only keys at positions <= its own.
//
// CTA = (tile, KV head, 128 query vectors), one CTA per SM; a query vector is
// one (row, query head) pair of the tile and owns one TMEM lane.  The blocks
// of the list run through a pipeline kDepth blocks deep: kDepth K/V stages in
// shared memory and kDepth S/P buffers of 64 columns in tensor memory, with
// the O accumulator (128 columns) beside them.  Warp-specialised, all waits
// bounded:
//   warp 4 (one thread)  streams each kept block (64 keys) of K and V by TMA
//                        into stage i % kDepth (four 64-row x 128 B boxes),
//                        once the PV of block i - kDepth has freed it;
//   warp 5 (one thread)  issues S_i = Q K_i^T (M = 128 vectors, N = 64 keys,
//                        K = 128 dims; K-major operands) kDepth - 1 blocks
//                        ahead of the PVs, and O += [P_hi | P_lo] [V_i ; V_i]
//                        (A = P read from tensor memory, N = 128 dims, K =
//                        2 x 64 keys; V read MN-major) once P_i is written.
//                        The MMAs run in issue order, so the S of block
//                        i + kDepth - 1, written into the buffer of block
//                        i - 1, follows the PV that read P_{i-1};
//   warps 0-3            the softmax: thread = query vector (TMEM lane 32 w +
//                        lane), its whole row of 64 keys: masks (causal,
//                        cache end) only on the diagonal and cache-end blocks,
//                        online softmax in the log2 domain against a
//                        reference max, P split into a bf16 hi + lo pair
//                        (error ~2^-17) stored over S as the PV's A operand.
// With S computed kDepth - 1 blocks ahead, the softmax of block i + 1 starts
// as soon as that of block i ends, and the tensor pipe holds the next blocks'
// QKs and the PVs of the finished ones.  O stays in tensor memory; it is
// rescaled in place only when a row's max grows past the reference by more
// than 2^8.  Accumulation order per vector is the block order of the list, so
// results do not depend on scheduling.
#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace sa {
namespace {

constexpr int kBlk = 64;                       // keys per block
constexpr int kSmWarps = 4;                    // softmax: one warp per TMEM lane quarter
constexpr int kThreadsTc = 32 * (kSmWarps + 2);
constexpr int kProducerWarp = kSmWarps;
constexpr int kMmaWarp = kSmWarps + 1;
#ifndef SA_TA_DEPTH
#define SA_TA_DEPTH 5
#endif
constexpr int kDepth = SA_TA_DEPTH;            // blocks in flight: K/V stages and S/P buffers
constexpr int kBox = kBlk * 128;               // 64 rows x 128 B
constexpr int kStage = 4 * kBox;               // K lo | K hi | V lo | V hi = 32 KiB
constexpr int kQChunk = 128 * 128;             // 128 vectors x 64 dims bf16
constexpr int kQTile = 2 * kQChunk;            // 128 vectors x 128 dims bf16, two K chunks
constexpr int kOffQ = 0;
constexpr int kOffRing = kOffQ + kQTile;
constexpr int kOffBars = kOffRing + kDepth * kStage;
// per slot: kv full, kv empty, S full, P full, PV done; drain
constexpr int kNumBars = 5 * kDepth + 1;
constexpr int kOffList = kOffBars + kNumBars * 8 + 8;
// tensor memory: S/P buffer b at columns [64 b, 64 b + 64) (64 fp32 S
// columns; P's bf16 hi | lo pairs overwrite them), O at [384, 512)
constexpr uint32_t kColO = 384;
static_assert(64 * kDepth <= (int)kColO, "S/P buffers below the O accumulator");
static_assert(1024 + kOffList > 114 * 1024, "one CTA per SM: it allocates all 512 TMEM columns");
static_assert(1024 + kOffList + 4096 <= 227 * 1024, "shared memory, with a list of up to 1023 blocks");

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
  uint64_t* kv_empty = kv_full + kDepth;
  uint64_t* s_full = kv_empty + kDepth;
  uint64_t* p_full = s_full + kDepth;
  uint64_t* o_done = p_full + kDepth;  // the PV of the slot's block is done
  uint64_t* drain = o_done + kDepth;
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
    for (int s = 0; s < kDepth; ++s) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_empty + s, 1);  // the PV that read the stage commits
      mbar_init(s_full + s, 1);
      mbar_init(p_full + s, kSmWarps);
      mbar_init(o_done + s, 1);
    }
    mbar_init(drain, 1);
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

  // ---- the CTA's 128 query vectors: row vi of the K-major, 128B-swizzled Q
  // (rows past V zero); 8 loads in flight per thread
  const __nv_bfloat16* Q = reinterpret_cast<const __nv_bfloat16*>(a.q);
  const int v0 = mc * 128;
  constexpr int kQPieces = 128 * 16;
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
      *reinterpret_cast<uint4*>(qs + (d8 >> 3) * kQChunk + swz128(vi, d8 & 7)) = rw[i];
    }
  }
  fence_proxy_async();  // generic writes (queries, list) before the async proxy reads them
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = s_tmem;
  int fail = 0;

  if (warp == kProducerWarp) {
    // ---- TMA producer: block i -> stage i % kDepth (freed by the PV of block i - kDepth)
    if (lane == 0) {
      const long long rowbase = (long long)g * a.kv.cap;  // B == 1: unit = KV head
      int issued = 0;
      for (int i = 0; i < nb; ++i) {
        const int s = i % kDepth;
        if (i >= kDepth && !mbar_wait(kv_empty + s, ((i / kDepth) - 1) & 1u, a.status)) {
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
      for (int i = max(0, issued - kDepth); i < issued; ++i)
        mbar_wait(kv_full + (i % kDepth), (i / kDepth) & 1u, nullptr);
    }
  } else if (warp == kMmaWarp) {
    // ---- MMA issuer: the QKs of blocks 0 .. kDepth - 2 up front, then per
    // block i: its PV once P_i is written, then the QK of block i + kDepth - 1
    // (into the buffer of block i - 1, whose PV was issued before it)
    if (lane == 0) {
      const uint32_t idesc_s = tc::idesc_f32acc(tc::kFmtBF16, 128, kBlk);
      const uint32_t idesc_o = tc::idesc_f32acc(tc::kFmtBF16, 128, kHeadDim) | (1u << 16);  // V MN-major
      auto qk = [&](int j) -> bool {
        const int s = j % kDepth;
        if (!mbar_wait(kv_full + s, (j / kDepth) & 1u, a.status)) return false;
        tc::fence_after_sync();
        const unsigned char* kb = ring + s * kStage;
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc::mma_bf16_ss(tmem + 64u * s, tc::smem_desc_sw128(qs + c * kQChunk + 32 * k),
                            tc::smem_desc_sw128(kb + c * kBox + 32 * k), idesc_s, (c | k) != 0);
        tc::commit(s_full + s);
        return true;
      };
      auto pv = [&](int i) -> bool {
        const int s = i % kDepth;
        if (!mbar_wait(p_full + s, (i / kDepth) & 1u, a.status)) return false;
        tc::fence_after_sync();
        const unsigned char* vb = ring + s * kStage + 2 * kBox;
#pragma unroll
        for (int j = 0; j < 8; ++j)  // K = [P_hi keys 0-63 | P_lo keys 0-63], 16 per step
          tc::mma_bf16_ts(tmem + kColO, tmem + 64u * s + 8u * j, v_desc(vb + 16 * 128 * (j & 3)), idesc_o,
                          i > 0 || j != 0);
        tc::commit(o_done + s);
        tc::commit(kv_empty + s);
        return true;
      };
      for (int j = 0; j < min(nb, kDepth - 1) && !fail; ++j)
        if (!qk(j)) fail = 1;
      for (int i = 0; i < nb && !fail; ++i) {
        if (!pv(i)) {
          fail = 1;
          break;
        }
        const int j = i + kDepth - 1;
        if (j < nb && !qk(j)) fail = 1;
      }
      // every MMA issued has completed before TMEM is freed (bounded)
      tc::commit(drain);
      mbar_wait(drain, 0, nullptr);
    }
  } else {
    // ---- softmax: TMEM lane r = 32 warp + lane is query vector v0 + r; the
    // thread owns that vector's whole row
    const int r = 32 * warp + lane;
    const int v = v0 + r;
    const bool vok = v < V;
    const int qpos = vok ? a.q_pos0 + row0 + v / G : -1;
    const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
    const uint32_t sp_base = tmem + lane_off;
    const uint32_t to = tmem + lane_off + kColO;
    // PV of block j complete.  A slot's PV barrier never runs two phases
    // ahead of a wait here: the PV of block j + kDepth needs P_{j + kDepth},
    // which this thread writes later (or, after the loop, does not exist).
    auto wait_pv = [&](int j) -> bool {
      const bool ok = mbar_wait(o_done + (j % kDepth), (j / kDepth) & 1u, a.status);
      return __all_sync(0xffffffffu, ok);
    };
    float mref = ninf, lh = 0.f;  // reference max (log2 units) and the row sum against it
    const float sl2 = a.scale_log2;
    for (int i = 0; i < nb; ++i) {
      const int b = i % kDepth;
      const bool ok = mbar_wait(s_full + b, (i / kDepth) & 1u, a.status);
      if (!__all_sync(0xffffffffu, ok)) {
        fail = 1;
        break;
      }
      tc::fence_after_sync();
      const uint32_t ts = sp_base + 64u * b;  // S/P buffer of the block
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
      // V rows past the cache end hold other data: zero them before PV reads them
      if (kb0 + kBlk > N) {
        unsigned char* st = ring + b * kStage;
        for (int x = r; x < (kb0 + kBlk - N) * 16; x += 128) {
          const int row = (N - kb0) + (x >> 4), ch = x & 15;
          *reinterpret_cast<uint4*>(st + (2 + (ch >> 3)) * kBox + swz128(row, ch & 7)) = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async();  // the zeroed V rows before the tensor cores read them
      }
      tc::wait_st();
      tc::fence_before_sync();  // P and the rescaled O before PV_i reads them
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full + b);
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

// CTAs per (tile, KV head): 128 query vectors each.
int tile_attn_tc_mchunks(int vectors_per_tile) { return (vectors_per_tile + 127) / 128; }

}  // namespace sa
