// Causal attention of query tiles over their routed blocks, on tcgen05.
//
// "Technische Samenvatting: Onzekerheidsgestuurde Selectie voor Blok-schaarse
// Aandacht", "Methodologie" step 5: every tile attends to the blocks its list
// names (the top k, or the top rho*k when the tile triggered); sentinel (-1)
// entries are skipped.  Chunked-prefill rows attend causally: row r at
// position q_pos0 + r sees only keys at positions <= its own.
//
// CTA = (tile, KV head, 128 query vectors), one CTA per SM; a query vector is
// one (row, query head) pair of the tile and owns one lane of tensor memory.
// Warp-specialised, all waits bounded:
//   warp 8 (one thread)  streams each kept block (64 keys) of K and V by TMA
//                        into a kStages ring (four 64-row x 128 B boxes);
//   warp 9 (one thread)  issues, per block i, S_i = Q K_i^T (M = 128 vectors,
//                        N = 64 keys, K = 128 dims; K-major operands) into one
//                        of two S accumulators, and O += [P_hi | P_lo] .
//                        [V_i ; V_i] (A from tensor memory; N = 128 dims,
//                        K = 2 x 64 keys; V read MN-major) into the O
//                        accumulator; QK of the next
//                        block is issued before PV of this one, so the
//                        softmax overlaps the tensor cores;
//   warps 0-7            two per TMEM lane quarter (query vector): mask
//                        (causal, cache end), online softmax in the log2
//                        domain against a reference max, P split into a bf16
//                        hi + lo pair (error ~2^-17) stored to tensor memory
//                        as the next MMA's A operand; O stays in tensor
//                        memory and is rescaled in place only when a row's
//                        max grows by more than 2^8.
// Accumulation order per vector is the block order of the list, so results
// do not depend on scheduling.
#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace sa {
namespace {

constexpr int kBlk = 64;                       // keys per block
constexpr int kSmWarps = 8;                    // softmax warps: two per TMEM lane quarter
constexpr int kThreadsTc = 32 * (kSmWarps + 2);
constexpr int kProducerWarp = kSmWarps;
constexpr int kMmaWarp = kSmWarps + 1;
#ifndef SA_TA_STAGES
#define SA_TA_STAGES 3
#endif
constexpr int kStages = SA_TA_STAGES;
constexpr int kBox = kBlk * 128;               // 64 rows x 128 B
constexpr int kStage = 4 * kBox;               // K lo | K hi | V lo | V hi = 32 KiB
constexpr int kQBytes = 2 * 128 * 128;         // 128 vectors x 128 dims bf16, two K chunks
constexpr int kOffQ = 0;
constexpr int kOffRing = kOffQ + kQBytes;
constexpr int kOffBars = kOffRing + kStages * kStage;
// kv full/empty, s full/empty, p full, o full (PV of even / odd blocks), drain
constexpr int kNumBars = 2 * kStages + 2 * 2 + 2 + 2 + 1;
constexpr int kOffRed = kOffBars + kNumBars * 8 + 8;        // softmax row sums, 2 halves x 128 rows
constexpr int kOffList = kOffRed + 2 * 128 * 4;
constexpr uint32_t kColS = 0;                  // S accumulators: columns [0, 128)
constexpr uint32_t kColO = 128;                // O accumulator: columns [128, 256)
constexpr uint32_t kColP = 256;                // P_hi | P_lo (bf16 pairs), two buffers: [256, 384)
static_assert(1024 + kOffList > 114 * 1024, "one CTA per SM: it allocates all 512 TMEM columns");

// MN-major view of V (keys x dims, dims contiguous): 8-key atoms 1 KiB apart,
// the two 64-dim boxes 8 KiB apart.
// 2^x by the hardware approximation (relative error about 2^-22; 2^-inf = +0).
SA_DEV float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

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
  uint64_t* s_full = kv_empty + kStages;
  uint64_t* s_empty = s_full + 2;
  uint64_t* p_full = s_empty + 2;
  uint64_t* o_full = p_full + 2;
  uint64_t* drain = o_full + 2;
  int* blist = reinterpret_cast<int*>(base + kOffList);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Hkv = a.kv.Hkv, G = a.G;
  const int nmc = a.n_mchunks;
  const int mc = blockIdx.x % nmc;
  const int tg = blockIdx.x / nmc;
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
      mbar_init(kv_empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full + b, 1);
      mbar_init(s_empty + b, kSmWarps);
      mbar_init(p_full + b, kSmWarps);
      mbar_init(o_full + b, 1);
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

  // ---- the CTA's 128 query vectors (K-major, 128B-swizzled, rows past V zero);
  // 8 loads in flight per thread
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
      *reinterpret_cast<uint4*>(qs + (d8 >> 3) * (128 * 128) + swz128(vi, d8 & 7)) = rw[i];
    }
  }
  fence_proxy_async();  // generic writes (queries, list) before the async proxy reads them
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = s_tmem;
  int fail = 0;
  // softmax-warp state, used after the final barrier (other warps: unused)
  const int quarter = warp & 3, h = (warp >> 2) & 1;
  const int r = 32 * quarter + lane;
  const int v = v0 + r;
  const bool vok = v < V;
  const int qpos = vok ? a.q_pos0 + row0 + v / G : -1;
  float* red = reinterpret_cast<float*>(base + kOffRed);  // [2 halves][128 rows] row sums
  float mref = ninf, lh = 0.f;  // reference max (log2 units) and row sum against it
  float o[64];
#pragma unroll
  for (int d = 0; d < 64; ++d) o[d] = 0.f;

  if (warp == kProducerWarp) {
    // ---- TMA producer: block i -> stage i % kStages
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
  } else if (warp == kMmaWarp) {
    // ---- MMA issuer: qk(0), then per block i: qk(i + 1), pv(i)
    if (lane == 0) {
      const uint32_t idesc_s = tc::idesc_f32acc(tc::kFmtBF16, 128, kBlk);
      const uint32_t idesc_o = tc::idesc_f32acc(tc::kFmtBF16, 128, kHeadDim) | (1u << 16);  // V MN-major
      // Both queues are polled without blocking: QK of block i + 1 needs its
      // K/V stage and a free S buffer, PV of block i needs P_i; whichever is
      // ready goes first, so a late K/V stage never holds back a PV whose P is
      // written (and the stage it frees).  QK runs at most one block ahead.
      auto qk = [&](int i) {
        const int s = i % kStages, b = i & 1;
        const unsigned char* kb = ring + s * kStage;
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc::mma_bf16_ss(tmem + kColS + 64u * b, tc::smem_desc_sw128(qs + c * (128 * 128) + 32 * k),
                            tc::smem_desc_sw128(kb + c * kBox + 32 * k), idesc_s, (c | k) != 0);
        tc::commit(s_full + b);
      };
      auto pv = [&](int i) {
        const int s = i % kStages, b = i & 1;
        const unsigned char* vb = ring + s * kStage + 2 * kBox;
#pragma unroll
        for (int j = 0; j < 8; ++j)  // K = [P_hi keys 0-63 | P_lo keys 0-63], 16 per step
          tc::mma_bf16_ts(tmem + kColO, tmem + kColP + 64u * b + 8u * j, v_desc(vb + 16 * 128 * (j & 3)),
                          idesc_o, i > 0 || j != 0);
        tc::commit(o_full + b);
        tc::commit(kv_empty + s);
      };
      int nq = 0, npv = 0;
      uint32_t idle = 0;
      while (npv < nb) {
        bool progress = false;
        if (nq < nb && nq <= npv + 1 && mbar_test(kv_full + nq % kStages, (nq / kStages) & 1u) &&
            (nq < 2 || mbar_test(s_empty + (nq & 1), ((nq >> 1) - 1) & 1u))) {
          tc::fence_after_sync();
          qk(nq++);
          progress = true;
        }
        if (npv < nq && mbar_test(p_full + (npv & 1), (npv >> 1) & 1u)) {
          tc::fence_after_sync();
          pv(npv++);
          progress = true;
        }
        if (progress) {
          idle = 0;
        } else if (++idle >= kSpinLimit) {
          flag_status(a.status, SA_ERR_TIMEOUT);
          fail = 1;
          break;
        }
      }
      // every MMA issued has completed before TMEM is freed (bounded)
      tc::commit(drain);
      mbar_wait(drain, 0, nullptr);
    }
  } else {
    // ---- softmax: TMEM lane r = 32 (warp % 4) + lane is query vector v0 + r;
    // half h = warp / 4 exponentiates keys [32 h, 32 h + 32) of S and owns dims
    // [64 h, 64 h + 64) of O.  Both halves read the whole S row, so they hold the
    // same maxima without exchanging anything; their row sums are added after
    // the CTA's final barrier.  O accumulates in tensor memory over the blocks,
    // against a reference max mref that may lag the row's running max: P =
    // 2^(s - mref) stays below 2^8, and O and the row sum are rescaled in place
    // only when a row's max passes mref by more than 8 (log2 units), which with
    // bounded scores happens in the first blocks only.
    const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
    const uint32_t to = tmem + lane_off + kColO + 64u * h;
    int o_seen = 0;  // PV results waited for: blocks [0, o_seen)
    auto wait_pv = [&](int j) -> bool {  // PV of block j complete (phases in order)
      const bool ok = mbar_wait(o_full + (j & 1), (j >> 1) & 1u, a.status);
      return __all_sync(0xffffffffu, ok);
    };
    // S of block i in r0..r3 (own half: r0, r1; other half: r2, r3); the loads of
    // block i + 1 are issued before waiting for PV of block i - 1, so their
    // latency overlaps that wait
    uint32_t r0[16], r1[16], r2[16], r3[16];
    auto load_s = [&](int i) -> bool {
      const int b = i & 1;
      const bool ok = mbar_wait(s_full + b, (i >> 1) & 1u, a.status);
      if (!__all_sync(0xffffffffu, ok)) return false;
      tc::fence_after_sync();
      const uint32_t ts = tmem + lane_off + kColS + 64u * b;
      tc::ld_32x32b_x16(ts + 32u * h, r0);
      tc::ld_32x32b_x16(ts + 32u * h + 16, r1);
      tc::ld_32x32b_x16(ts + 32u * (h ^ 1), r2);
      tc::ld_32x32b_x16(ts + 32u * (h ^ 1) + 16, r3);
      return true;
    };
    if (nb > 0 && !load_s(0)) fail = 1;
    for (int i = 0; i < nb && !fail; ++i) {
      const int b = i & 1;
      tc::wait_ld();
      tc::reg_fence(r0);
      tc::reg_fence(r1);
      tc::reg_fence(r2);
      tc::reg_fence(r3);
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_empty + b);  // S_i read: the buffer may take S_{i+2}
      const int kb0 = blist[i] * kBlk;
      // scores in registers: this half's 32 keys in sv, the row max over all 64.
      // Blocks fully visible to every row of the warp (all but the diagonal and
      // the cache end) skip the masks, and with a positive scale the max is
      // taken on raw scores (scaling commutes with max).
      const float sl2 = a.scale_log2;
      const bool fast = sl2 > 0.f && __all_sync(0xffffffffu, kb0 + kBlk - 1 <= qpos && kb0 + kBlk <= N);
      // (four independent max chains: the reduction is latency-bound)
      float sv[32], mq[4] = {ninf, ninf, ninf, ninf}, mul;
      if (fast) {
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          sv[x] = __uint_as_float(r0[x]);
          sv[16 + x] = __uint_as_float(r1[x]);
          mq[x & 3] = fmaxf(mq[x & 3], fmaxf(fmaxf(sv[x], sv[16 + x]),
                                             fmaxf(__uint_as_float(r2[x]), __uint_as_float(r3[x]))));
        }
        mul = sl2;
      } else {
        const int kv0 = kb0 + 32 * h, kw0 = kb0 + 32 * (h ^ 1);
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          const int k0 = kv0 + x, k1 = k0 + 16, w0 = kw0 + x, w1 = w0 + 16;
          sv[x] = (k0 <= qpos && k0 < N) ? __uint_as_float(r0[x]) * sl2 : ninf;
          sv[16 + x] = (k1 <= qpos && k1 < N) ? __uint_as_float(r1[x]) * sl2 : ninf;
          const float u0 = (w0 <= qpos && w0 < N) ? __uint_as_float(r2[x]) * sl2 : ninf;
          const float u1 = (w1 <= qpos && w1 < N) ? __uint_as_float(r3[x]) * sl2 : ninf;
          mq[x & 3] = fmaxf(mq[x & 3], fmaxf(fmaxf(sv[x], sv[16 + x]), fmaxf(u0, u1)));
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
        // O holds blocks [0, i): once the last of them is in, scale this half in place
        if (o_seen < i) {
          if (!wait_pv(i - 1)) {
            fail = 1;
            break;
          }
          o_seen = i;
        }
        tc::fence_after_sync();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t q[16];
          tc::ld_32x32b_x16(to + 16 * c, q);
          tc::wait_ld();
#pragma unroll
          for (int x = 0; x < 16; ++x) q[x] = __float_as_uint(__uint_as_float(q[x]) * alpha);
          tc::st_32x32b_x16(to + 16 * c, q);
        }
        tc::wait_st();
      }
      const float nmn = mref == ninf ? 0.f : -mref;  // all masked so far: every p is exp2(-inf) = 0
      // P = exp2(s - mref) as a bf16 hi + lo pair into tensor memory, this
      // half's keys: hi pairs in columns 16 h .. 16 h + 15, lo pairs 32 further
      uint32_t phi[16], plo[16];
      float rq[4] = {0.f, 0.f, 0.f, 0.f};  // four independent partial row sums
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float p0 = fast_exp2(fmaf(sv[2 * j], mul, nmn));
        const float p1 = fast_exp2(fmaf(sv[2 * j + 1], mul, nmn));
        rq[j & 3] += p0 + p1;
        // hi = p truncated to bf16 (the upper halves, one byte permute); lo = the
        // exact remainder p - hi (< 2^-7 p) rounded to bf16: |p - hi - lo| < 2^-16 p
        phi[j] = pack_bf16(p0, p1);
        plo[j] = pack_bf16(p0 - bf16_lo(phi[j]), p1 - bf16_hi(phi[j]));
      }
      const uint32_t tp = tmem + lane_off + kColP + 64u * b + 16u * h;
      tc::st_32x32b_x16(tp, phi);
      tc::st_32x32b_x16(tp + 32, plo);
      lh += (rq[0] + rq[1]) + (rq[2] + rq[3]);
      // V rows past the cache end hold other data: zero them before PV reads them
      if (kb0 + kBlk > N) {
        unsigned char* st = ring + (i % kStages) * kStage;
        for (int x = 32 * warp + lane; x < (kb0 + kBlk - N) * 16; x += 32 * kSmWarps) {
          const int row = (N - kb0) + (x >> 4), ch = x & 15;
          *reinterpret_cast<uint4*>(st + (2 + (ch >> 3)) * kBox + swz128(row, ch & 7)) = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async();  // the zeroed V rows before the tensor cores read them
      }
      tc::wait_st();
      tc::fence_before_sync();  // P and the rescaled O before PV_i reads them
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full + b);
      if (i + 1 < nb && !load_s(i + 1)) {
        fail = 1;
        break;
      }
      // PV_{i-1} done before P_{i+1} overwrites its buffer
      if (i >= 1 && o_seen < i) {
        if (!wait_pv(i - 1)) {
          fail = 1;
          break;
        }
        o_seen = i;
      }
    }
    tc::wait_ld();  // no TMEM load of S left in flight (a failed wait may leave one)
    // the result: PV of the last block, then this half of O into registers
    for (int j = o_seen; j < nb && !fail; ++j)
      if (!wait_pv(j)) fail = 1;
    if (!fail && nb > 0) {
      tc::fence_after_sync();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t q[16];
        tc::ld_32x32b_x16(to + 16 * c, q);
        tc::wait_ld();
#pragma unroll
        for (int x = 0; x < 16; ++x) o[16 * c + x] = __uint_as_float(q[x]);
      }
    }
    red[h * 128 + r] = lh;  // added to the other half's after the final barrier
  }
  tc::fence_before_sync();
  const int all_ok = __syncthreads_and(!fail);
  tc::fence_after_sync();
  if (warp == 0) tc::tmem_dealloc(tmem, 512);
  // ---- softmax warps: row sum of both halves, this half's 64 dims of the output
  if (warp < kSmWarps && all_ok && vok) {
    const float l = lh + red[(h ^ 1) * 128 + r];
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const size_t orow = (size_t)(row0 + v / G) * a.Hq + (size_t)g * G + v % G;
    float* dst = a.out + orow * kHeadDim + 64 * h;
#pragma unroll
    for (int d = 0; d < 64; d += 4)
      *reinterpret_cast<float4*>(dst + d) = make_float4(o[d] * inv, o[d + 1] * inv, o[d + 2] * inv, o[d + 3] * inv);
    if (a.lse && h == 0) a.lse[orow] = l > 0.f ? mref * kLn2 + logf(l) : ninf;
  }
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

int tile_attn_tc_mchunks(int vectors_per_tile) { return (vectors_per_tile + 127) / 128; }

}  // namespace sa
