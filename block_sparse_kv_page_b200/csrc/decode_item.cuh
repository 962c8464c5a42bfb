// One work item of sparse paged flash-decode over the selected pages (split-K
// + combine).  Called by the standalone decode kernel and by the fused decode
// step.
//
// "Sparse Attention for Web Agents -- Offline Replay Records", section "The
// comparison": after choosing the best chunks the methods attend only to
// them; exact softmax attention over the selected tokens.
//
// Work split.  A unit is one (sequence, KV head) with its G <= 8 query heads.
// Its selected pages are cut into 16-token tiles (a 16-token page is one
// tile; larger pages and variable chunks give several, the last one ragged)
// and the tiles into `splits` contiguous ranges; an item is one (unit,
// range).  A persistent grid (one or two CTAs per SM) pulls items from an
// atomic queue, so the load balances whatever the unit count.
//
// Data movement.  K and V are streamed with TMA: a tile is four 2D boxes of
// 16 rows x 64 bf16 (K low/high dims, V low/high dims) landing 128B-swizzled
// in a per-warp ring of mbarrier-tracked stages.  Lane 0 of each warp issues
// the copies for the warp's tiles several stages ahead; fragments are read
// with ldmatrix (conflict-free under the swizzle).  Every barrier wait is
// bounded and reports SA_ERR_TIMEOUT instead of hanging.
//
// Math per tile and warp (tensor cores, fp32 accumulation):
//   QK:  S^T[16 tok x 8 heads] = K (16 x 128) . Q^T, m16n8k16 bf16;
//   P:   exp2 of the scaled scores, rounded to a bf16 hi + lo pair, moved
//        from the C layout to the B layout with movmatrix (8x8 transpose);
//   PV:  O^T[128 dims x 8 heads] += V^T (128 x 16 tok) . P^T (ldmatrix.trans).
// Each warp keeps its own online-softmax state; the warps merge in shared
// memory; with several splits the CTA writes its (max, sum, acc) partial to
// the workspace and the CTA that finishes the unit's last item (atomic
// counter, no waiting) merges the partials in split order, so results do not
// depend on scheduling.
#pragma once

#include "common.cuh"
#include "internal.h"

#ifndef SA_DEC_WARPS
#define SA_DEC_WARPS 4
#endif
#ifndef SA_DEC_STAGES
#define SA_DEC_STAGES 2
#endif
#ifndef SA_DEC_ITEM_TILES
#define SA_DEC_ITEM_TILES 64
#endif
#ifndef SA_DEC_CTAS_PER_SM
#define SA_DEC_CTAS_PER_SM 3
#endif
#ifndef SA_DEC_TAIL_FINE
#define SA_DEC_TAIL_FINE 1
#endif
#ifndef SA_DEC_MIN_ITEM_TILES
#define SA_DEC_MIN_ITEM_TILES 16
#endif

namespace sa {
namespace dec {

constexpr int kWarps = SA_DEC_WARPS;
constexpr int kThreads = kWarps * 32;
constexpr int kStages = SA_DEC_STAGES;
constexpr int kTileBytes = 8192;                 // K box lo | K box hi | V box lo | V box hi
constexpr int kBoxBytes = 2048;                  // 16 rows x 128 B
constexpr int kRingBytes = kWarps * kStages * kTileBytes;
constexpr int kMaxItemTiles = SA_DEC_ITEM_TILES; // tile refs resolved per round
constexpr int kPartHead = kHeadDim + 4;            // acc[128], m, l, 2 pad: 16-byte rows
constexpr int kPartStride = kMaxGroup * kPartHead;  // floats per partial slot
constexpr int kMergeBatch = 4;                     // split partials loaded per round trip
constexpr int kThreadsPerHead = kThreads / kMaxGroup;  // merge: threads per head
constexpr int kDimsPerThread = kHeadDim / kThreadsPerHead;
static_assert(kDimsPerThread % 4 == 0, "merge writes float4");

// Dynamic shared memory (offsets from a 1024-aligned base).
constexpr int kOffBars = kRingBytes;
struct TileRef {
  int row;     // first tile row in the [B*Hkv*cap] row space (u * cap + token)
  int n;       // valid tokens (0 = empty tile)
  int mask;    // the unit's query heads that attend the tile (bit j = head h0 + j)
};

constexpr int kOffTiles = kOffBars + kWarps * kStages * 8;
constexpr int kOffPre = kOffTiles + kMaxItemTiles * (int)sizeof(TileRef);

struct Smem {
  unsigned char* ring;   // [warp][stage][kTileBytes]
  uint64_t* bars;        // [warp][stage]
  TileRef* tiles;        // [kMaxItemTiles]
  int* pre;              // chunk mode: tile prefix [max_sel + 1]
  uint32_t* scan;        // kWarps words
  int* last;
  int* ntiles;
};

// Unit and split of decode item j (queue order: units ascending).
SA_DEV void item_unit(const DecodeArgs& a, const int j, int& u, int& split) {
  const int n0 = a.fine_unit0 * a.splits;
  if (j < n0) {
    u = j / a.splits;
    split = j - u * a.splits;
  } else {
    const int r = (j - n0) / a.splits_fine;
    u = a.fine_unit0 + r;
    split = j - n0 - r * a.splits_fine;
  }
}

// Output row `row`, dims d0 .. d0 + kDimsPerThread - 1 = A * inv, as fp32 or
// rounded to bf16 (round to nearest even).
SA_DEV void store_out(const DecodeArgs& a, size_t row, int d0, const float (&A)[kDimsPerThread],
                      float inv) {
  if (a.out_bf16) {
    __nv_bfloat16* o = a.out_bf16 + row * kHeadDim + d0;
#pragma unroll
    for (int x = 0; x < kDimsPerThread; x += 4)
      *reinterpret_cast<uint2*>(o + x) = make_uint2(pack_bf16(A[x] * inv, A[x + 1] * inv),
                                                    pack_bf16(A[x + 2] * inv, A[x + 3] * inv));
  } else {
    float* o = a.out + row * kHeadDim + d0;
#pragma unroll
    for (int x = 0; x < kDimsPerThread; x += 4)
      *reinterpret_cast<float4*>(o + x) = make_float4(A[x] * inv, A[x + 1] * inv, A[x + 2] * inv, A[x + 3] * inv);
  }
}

// Merge of a unit's split partials for head h, dims d0 .. d0 + 7, in split
// order, kMergeBatch partials per batch with every load of a batch issued
// before any is used (each dependent round trip to L2 costs about a
// microsecond under full HBM load).  base = slot 0 of the unit, head h;
// LOCAL: the partials are in (this CTA's) shared memory, else in global
// memory written earlier in the launch.  The same arithmetic either way.
// part_out (non-null, head h's row of a partial slot): the merged partial is
// stored there too, unnormalised, like a split's.
template <bool LOCAL>
SA_DEV void merge_splits(const DecodeArgs& a, const float* base, const int splits, const size_t out_row,
                         const int d0, float* part_out = nullptr) {
  const float ninf = -__int_as_float(0x7f800000);
  float MM = ninf, LL = 0.f, AA[kDimsPerThread];
#pragma unroll
  for (int x = 0; x < kDimsPerThread; ++x) AA[x] = 0.f;
  for (int sp0 = 0; sp0 < splits; sp0 += kMergeBatch) {
    float2 ml[kMergeBatch];
    float4 v[kMergeBatch][kDimsPerThread / 4];
#pragma unroll
    for (int j = 0; j < kMergeBatch; ++j) {
      const bool ok = sp0 + j < splits;
      const float* src = base + (size_t)(ok ? sp0 + j : 0) * kPartStride;
      const float2* pml = reinterpret_cast<const float2*>(src + kHeadDim);
      ml[j] = ok ? (LOCAL ? *pml : __ldcg(pml)) : make_float2(ninf, 0.f);
#pragma unroll
      for (int q4 = 0; q4 < kDimsPerThread / 4; ++q4) {
        const float4* pv = reinterpret_cast<const float4*>(src + d0) + q4;
        v[j][q4] = ok ? (LOCAL ? *pv : __ldcg(pv)) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    float nm = MM;
#pragma unroll
    for (int j = 0; j < kMergeBatch; ++j) nm = fmaxf(nm, ml[j].x);
    if (nm == ninf) continue;
    const float fo = exp2f(MM - nm);  // 0 while nothing has been merged
    LL *= fo;
#pragma unroll
    for (int x = 0; x < kDimsPerThread; ++x) AA[x] *= fo;
#pragma unroll
    for (int j = 0; j < kMergeBatch; ++j) {
      const float f = exp2f(ml[j].x - nm);
      LL += ml[j].y * f;
#pragma unroll
      for (int q4 = 0; q4 < kDimsPerThread / 4; ++q4) {
        AA[4 * q4 + 0] += v[j][q4].x * f;
        AA[4 * q4 + 1] += v[j][q4].y * f;
        AA[4 * q4 + 2] += v[j][q4].z * f;
        AA[4 * q4 + 3] += v[j][q4].w * f;
      }
    }
    MM = nm;
  }
  const float inv = LL > 0.f ? 1.f / LL : 0.f;
  store_out(a, out_row, d0, AA, inv);
  if (a.lse && d0 == 0) a.lse[out_row] = LL > 0.f ? MM * kLn2 + logf(LL) : ninf;
  if (part_out != nullptr) {
#pragma unroll
    for (int x = 0; x < kDimsPerThread; x += 4)
      *reinterpret_cast<float4*>(part_out + d0 + x) = make_float4(AA[x], AA[x + 1], AA[x + 2], AA[x + 3]);
    if (d0 == 0) *reinterpret_cast<float2*>(part_out + kHeadDim) = make_float2(MM, LL);
  }
}

// Routed lists (route_k > 0): a unit's top-k window runs in splits
// [0, sb) and its expansion window, decoded only for a unit whose tile
// triggered, in splits [sb, sb + se).  Partial slots per unit: sb + se + 1
// ([0, sb) top-k splits, [sb] their merge, [sb + 1, ..) expansion splits).
// One counter per unit: top-k splits add 1, expansion splits add 1 << 16,
// the top-k merge adds 1 << 30.  The last top-k split merges its window and
// writes the output (final unless the unit triggered) and the merged
// partial; the final merge of a triggered unit (the top-k merge and the
// expansion splits) falls to whichever of the last expansion split and the
// top-k merge comes second in the counter's order.
constexpr uint32_t kRouteExp = 1u << 16, kRouteBaseMerged = 1u << 30;
SA_DEV int route_exp_count(uint32_t v) { return (int)((v >> 16) & 0x3fffu); }

// Publish a routed split's partial and run the merges it falls to (see
// kRouteExp).  The counter increments are acq_rel after a barrier: they
// publish this CTA's partial and acquire the others'.
SA_DEV void route_publish(const DecodeArgs& a, const int u, const int split, const int splits,
                          const size_t slot0, const Smem& sm, const int h, const int G, const int d0,
                          const size_t out_row, const float (&A)[kDimsPerThread], const float M, const float L) {
  const int sb = a.route_base_splits, se = splits - sb;
  const bool base = split < sb;
  float* part = a.ws_part + (slot0 + (base ? split : split + 1)) * kPartStride;
  if (h < G) {
    float* dst = part + h * kPartHead;
#pragma unroll
    for (int x = 0; x < kDimsPerThread; x += 4)
      *reinterpret_cast<float4*>(dst + d0 + x) = make_float4(A[x], A[x + 1], A[x + 2], A[x + 3]);
    if (d0 == 0) *reinterpret_cast<float2*>(dst + kHeadDim) = make_float2(M, L);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t prev = atom_add_acq_rel_u32(&a.ws_count[u], base ? 1u : kRouteExp);
    // 1: merge the top-k window; 2: the final merge
    *sm.last = base ? ((prev & 0xffffu) == (uint32_t)(sb - 1) ? 1 : 0)
                    : (route_exp_count(prev) == se - 1 && (prev & kRouteBaseMerged) ? 2 : 0);
  }
  __syncthreads();
  int what = *sm.last;
  if (what == 1) {
    if (h < G)
      merge_splits<false>(a, a.ws_part + slot0 * kPartStride + h * kPartHead, sb, out_row, d0,
                          se > 0 ? a.ws_part + (slot0 + sb) * kPartStride + h * kPartHead : nullptr);
    if (se == 0) return;
    __syncthreads();
    if (threadIdx.x == 0) {
      const uint32_t prev = atom_add_acq_rel_u32(&a.ws_count[u], kRouteBaseMerged);
      *sm.last = route_exp_count(prev) == se ? 2 : 0;  // every expansion split already in
    }
    __syncthreads();
    what = *sm.last;
  }
  if (what == 2 && h < G)
    merge_splits<false>(a, a.ws_part + (slot0 + sb) * kPartStride + h * kPartHead, se + 1, out_row, d0);
}

// n_known >= 0: the unit's kept count, already read by the caller (the fused
// step takes it from the unit's selection flag); else it is loaded here.
// n_tok_known >= 0 likewise stands for the sequence length.
// STAGES: depth of the per-warp TMA ring (its barriers: sm.bars[warp][STAGES]).
// part_dst (several splits only): write the split's partial to part_dst +
// split * kPartStride (another CTA's shared memory, say) and return; the
// caller merges (merge_splits) once every split's partial is there.
template <bool PER_HEAD = false, int STAGES = kStages>
SA_DEV void decode_item(const DecodeArgs& a, const int u, const int split, const Smem& sm,
                        WarpState& ws, const int n_known = -1, const int n_tok_known = -1,
                        float* part_dst = nullptr) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, c = lane & 3;
  const UnitMap um = unit_map<PER_HEAD>(u, a.kv.Hkv, a.Hq, a.G);
  const int b = um.b;
  const int G = um.n_heads;  // query heads attending this unit's pages
  const float ninf = -__int_as_float(0x7f800000);

  // ---- geometry of the unit
  const int N = n_tok_known >= 0 ? n_tok_known : a.kv.seq_len[b];
  bool bad = (N < 1 || N > a.kv.cap);
  int n_ent = n_known >= 0 ? n_known : __ldcg(a.count + u);  // L2: may be written earlier in the launch
  if (n_ent < 0 || n_ent > a.max_sel) bad = true;
  if (bad) n_ent = 0;
  const int32_t* idx_u = a.idx + (size_t)u * a.max_sel;
  const int ps = a.kv.page_size;
  const int sub = ps > 0 ? ps / 16 : 0;
  int P = 0;
  const int32_t* off = nullptr;
  int* pre = sm.pre;
  if (ps > 0) {
    P = (N + ps - 1) / ps;
    if (tid == 0) *sm.ntiles = n_ent * sub;
  } else {
    off = a.kv.chunk_off + (size_t)b * (a.kv.max_pages + 1);
    P = a.kv.n_chunks[b];
    if (P < 1 || P > a.kv.max_pages) { bad = true; n_ent = 0; P = 0; }
    const int per = (n_ent + kThreads - 1) / kThreads;
    const int e0 = min(n_ent, tid * per), e1 = min(n_ent, e0 + per);
    uint32_t loc = 0;
    for (int e = e0; e < e1; ++e) {
      const int ch = __ldcg(idx_u + e);
      int nt = 0;
      if (ch >= 0 && ch < P && off[ch] >= 0) nt = (max(0, min(off[ch + 1], N) - off[ch]) + 15) >> 4;
      pre[e] = nt;
      loc += (uint32_t)nt;
    }
    uint32_t tot;
    uint32_t run = block_excl_scan(loc, sm.scan, tot);
    for (int e = e0; e < e1; ++e) {
      const int nt = pre[e];
      pre[e] = (int)run;
      run += (uint32_t)nt;
    }
    if (tid == 0) { pre[n_ent] = (int)tot; *sm.ntiles = (int)tot; }
  }
  if (bad && tid == 0 && split == 0) flag_status(a.status, SA_ERR_DEVICE_CHECK);
  __syncthreads();
  const int T = *sm.ntiles;
  // this unit's split count and first partial slot
  const bool coarse = u < a.fine_unit0;
  const int splits = coarse ? a.splits : a.splits_fine;
  const size_t slot0 = a.route_k > 0 ? (size_t)u * (a.splits + 1)
                       : coarse ? (size_t)u * a.splits
                                : (size_t)a.fine_unit0 * a.splits + (size_t)(u - a.fine_unit0) * a.splits_fine;
  int t_begin = (int)(((long long)T * split) / splits);
  int t_end = (int)(((long long)T * (split + 1)) / splits);
  if (a.route_k > 0) {  // routed lists: the top-k window, then the expansion window
    const int sb = a.route_base_splits, se = splits - sb;
    const long long kt = (long long)a.route_k * sub, wt = (long long)a.route_w * sub;
    if (split < sb) {
      t_begin = (int)(kt * split / sb);
      t_end = (int)(kt * (split + 1) / sb);
    } else {
      t_begin = (int)(kt + (wt - kt) * (split - sb) / se);
      t_end = (int)(kt + (wt - kt) * (split - sb + 1) / se);
    }
    t_begin = min(t_begin, T);
    t_end = min(t_end, T);
  }
  const long long row0 = (long long)um.kvu * a.kv.cap;

  // Token range of tile t of the unit (n = 0 for a skipped, invalid entry).
  const uint8_t* mask_u = a.mask ? a.mask + (size_t)u * a.max_sel : nullptr;
  auto tile_ref = [&](int t) -> TileRef {
    TileRef r{0, 0, 0xff};
    int start;
    if (ps > 0) {
      const int e = t / sub, part = t - e * sub;
      const int p = __ldcg(idx_u + e);
      if (mask_u) r.mask = __ldcg(mask_u + e);
      if (p < 0 || p >= P) {
        flag_status(a.status, SA_ERR_DEVICE_CHECK);
        r.n = 0;
        return r;
      }
      start = p * ps + part * 16;
      r.n = max(0, min(16, N - start));
    } else {
      int lo = 0, hi = n_ent - 1;  // last e with pre[e] <= t
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (pre[mid] <= t) lo = mid; else hi = mid - 1;
      }
      const int ch = __ldcg(idx_u + lo);
      if (mask_u) r.mask = __ldcg(mask_u + lo);
      if (ch < 0 || ch >= P || off[ch] < 0) {
        flag_status(a.status, SA_ERR_DEVICE_CHECK);
        return r;
      }
      start = off[ch] + (t - pre[lo]) * 16;
      r.n = max(0, min(16, min(off[ch + 1], N) - start));
    }
    r.row = (int)(row0 + start);
    return r;
  };

  // ---- Q fragments (B operand, natural k order): q[head][16s + 2c (+8)]
  const bool head_ok = gq < G;
  const __nv_bfloat16* qrow = reinterpret_cast<const __nv_bfloat16*>(a.q) +
                              ((size_t)b * a.Hq + (size_t)um.h0 + (head_ok ? gq : 0)) * kHeadDim;
  uint32_t bq[16];
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    bq[2 * s + 0] = head_ok ? __ldg(reinterpret_cast<const uint32_t*>(qrow + 16 * s + 2 * c)) : 0u;
    bq[2 * s + 1] = head_ok ? __ldg(reinterpret_cast<const uint32_t*>(qrow + 16 * s + 8 + 2 * c)) : 0u;
  }

  float m0 = ninf, m1 = ninf, l0 = 0.f, l1 = 0.f;
  float acc[8][4];
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;

  unsigned char* ring = sm.ring + warp * (STAGES * kTileBytes);
  uint64_t* bars = sm.bars + warp * STAGES;
  // ldmatrix lane addressing: matrix = lane / 8, row-in-matrix = lane % 8
  const int lrow_a = (lane & 7) + 8 * ((lane >> 3) & 1);  // K: rows 0-7 / 8-15
  const int lchk_a = lane >> 4;                            //    chunk +0 / +1
  const int lrow_v = (lane & 7) + 8 * (lane >> 4);         // V: tokens 0-7 / 8-15
  const int lchk_v = (lane >> 3) & 1;                      //    chunk +0 / +1

  for (int r0 = t_begin; r0 < t_end; r0 += kMaxItemTiles) {
    const int nt = min(kMaxItemTiles, t_end - r0);
    for (int i = tid; i < nt; i += kThreads) sm.tiles[i] = tile_ref(r0 + i);
    __syncthreads();

    const int n_it = max(0, (nt - warp + kWarps - 1) / kWarps);
    auto issue = [&](int it) {  // lane 0 only
      const int t = warp + it * kWarps;
      if (t >= nt) return;
      const uint32_t g_it = ws.gi + (uint32_t)it;
      uint64_t* bar = bars + g_it % STAGES;
      unsigned char* st = ring + (g_it % STAGES) * kTileBytes;
      const TileRef r = sm.tiles[t];
      if (r.n == 0) {
        mbar_arrive(bar);  // nothing to load: complete the phase
        return;
      }
      mbar_arrive_expect_tx(bar, kTileBytes);
      tma_load_2d(st + 0 * kBoxBytes, &a.tmap_k, 0, r.row, bar);
      tma_load_2d(st + 1 * kBoxBytes, &a.tmap_k, 64, r.row, bar);
      tma_load_2d(st + 2 * kBoxBytes, &a.tmap_v, 0, r.row, bar);
      tma_load_2d(st + 3 * kBoxBytes, &a.tmap_v, 64, r.row, bar);
    };
    int issued = 0;  // tiles of this round issued so far (identical on every lane)
    if (ws.alive) {
      issued = min(n_it, STAGES - 1);
      if (lane == 0)
        for (int it = 0; it < issued; ++it) issue(it);
    }

    for (int it = 0; it < n_it && ws.alive; ++it) {
      __syncwarp();  // every lane is done reading the stage about to be refilled
      if (it + STAGES - 1 < n_it) {
        if (lane == 0) issue(it + STAGES - 1);
        issued = it + STAGES;
      }
      const uint32_t g_it = ws.gi + (uint32_t)it;
      if (!mbar_wait(bars + g_it % STAGES, (g_it / STAGES) & 1u, a.status)) {
        ws.alive = false;
        ws.drain_lo = g_it;
        ws.drain_hi = ws.gi + (uint32_t)issued;
        break;
      }
      unsigned char* st = ring + (g_it % STAGES) * kTileBytes;
      const TileRef r = sm.tiles[warp + it * kWarps];
      if (r.n < 16) {  // zero V rows past the valid tokens (they may hold other data)
        for (int x = lane; x < (16 - r.n) * 16; x += 32) {
          const int row = r.n + (x >> 4), ch = x & 15;
          *reinterpret_cast<uint4*>(st + 2 * kBoxBytes + (ch >> 3) * kBoxBytes + swz128(row, ch & 7)) =
              make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async();
        __syncwarp();
      }

      // S^T = K . Q^T, two independent accumulation chains
      float s[4] = {0.f, 0.f, 0.f, 0.f}, s2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(a0, a1, a2, a3, st + (ks >> 2) * kBoxBytes + swz128(lrow_a, 2 * (ks & 3) + lchk_a));
        if (ks & 1) mma_bf16(s2, a0, a1, a2, a3, bq[2 * ks], bq[2 * ks + 1]);
        else        mma_bf16(s, a0, a1, a2, a3, bq[2 * ks], bq[2 * ks + 1]);
      }
      // tokens gq / gq + 8 of the tile, heads 2c / 2c + 1 (those the tile's mask keeps)
      const bool v0 = gq < r.n, v1 = gq + 8 < r.n;
      const bool k0 = (r.mask >> (2 * c)) & 1, k1 = (r.mask >> (2 * c + 1)) & 1;
      const float z0 = v0 && k0 ? (s[0] + s2[0]) * a.scale_log2 : ninf;
      const float z1 = v0 && k1 ? (s[1] + s2[1]) * a.scale_log2 : ninf;
      const float z2 = v1 && k0 ? (s[2] + s2[2]) * a.scale_log2 : ninf;
      const float z3 = v1 && k1 ? (s[3] + s2[3]) * a.scale_log2 : ninf;
      float mx0 = fmaxf(z0, z2), mx1 = fmaxf(z1, z3);
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
      }
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
      const float al0 = mn0 == ninf ? 1.f : exp2f(m0 - mn0);
      const float al1 = mn1 == ninf ? 1.f : exp2f(m1 - mn1);
      const float p0 = mn0 == ninf ? 0.f : exp2f(z0 - mn0);
      const float p2 = mn0 == ninf ? 0.f : exp2f(z2 - mn0);
      const float p1 = mn1 == ninf ? 0.f : exp2f(z1 - mn1);
      const float p3 = mn1 == ninf ? 0.f : exp2f(z3 - mn1);
      m0 = mn0; m1 = mn1;
      l0 = l0 * al0 + (p0 + p2);
      l1 = l1 * al1 + (p1 + p3);
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        acc[mt][0] *= al0; acc[mt][1] *= al1; acc[mt][2] *= al0; acc[mt][3] *= al1;
      }
      // P (C layout: [token][head]) -> bf16 hi/lo -> B layout ([head][token])
      const uint32_t hlo = pack_bf16(p0, p1), hhi = pack_bf16(p2, p3);
      const uint32_t llo = pack_bf16(p0 - bf16_lo(hlo), p1 - bf16_hi(hlo));
      const uint32_t lhi = pack_bf16(p2 - bf16_lo(hhi), p3 - bf16_hi(hhi));
      const uint32_t bh0 = movmatrix_t(hlo), bh1 = movmatrix_t(hhi);
      const uint32_t bl0 = movmatrix_t(llo), bl1 = movmatrix_t(lhi);

      // O^T += V^T . P^T: m-tile mt = dims 16mt .. 16mt + 15
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4_t(a0, a1, a2, a3,
                  st + (2 + (mt >> 2)) * kBoxBytes + swz128(lrow_v, 2 * (mt & 3) + lchk_v));
        mma_bf16(acc[mt], a0, a1, a2, a3, bh0, bh1);
        mma_bf16(acc[mt], a0, a1, a2, a3, bl0, bl1);
      }
    }
    ws.gi += (uint32_t)n_it;
    __syncthreads();  // tile refs of this round no longer read
  }

  // ---- merge the warps in shared memory
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
  }
  __syncthreads();  // ring no longer read
  float* w_acc = reinterpret_cast<float*>(sm.ring);                     // [warp][8][128]
  float* w_ml = w_acc + kWarps * kMaxGroup * kHeadDim;               // [warp][8][2]
  if (gq == 0) {
    w_ml[(warp * kMaxGroup + 2 * c) * 2 + 0] = m0;
    w_ml[(warp * kMaxGroup + 2 * c) * 2 + 1] = l0;
    w_ml[(warp * kMaxGroup + 2 * c + 1) * 2 + 0] = m1;
    w_ml[(warp * kMaxGroup + 2 * c + 1) * 2 + 1] = l1;
  }
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    float* h0 = w_acc + (warp * kMaxGroup + 2 * c) * kHeadDim + 16 * mt + gq;
    float* h1 = w_acc + (warp * kMaxGroup + 2 * c + 1) * kHeadDim + 16 * mt + gq;
    h0[0] = acc[mt][0];
    h1[0] = acc[mt][1];
    h0[8] = acc[mt][2];
    h1[8] = acc[mt][3];
  }
  __syncthreads();

  const int h = tid / kThreadsPerHead;               // head handled by this thread
  const int d0 = (tid % kThreadsPerHead) * kDimsPerThread;
  float M = ninf, L = 0.f, A[kDimsPerThread];
#pragma unroll
  for (int x = 0; x < kDimsPerThread; ++x) A[x] = 0.f;
  if (h < G) {
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, w_ml[(w * kMaxGroup + h) * 2]);
    if (M != ninf) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float f = exp2f(w_ml[(w * kMaxGroup + h) * 2] - M);
        L += w_ml[(w * kMaxGroup + h) * 2 + 1] * f;
        const float* src = w_acc + (w * kMaxGroup + h) * kHeadDim + d0;
#pragma unroll
        for (int x = 0; x < kDimsPerThread; ++x) A[x] += src[x] * f;
      }
    }
  }
  const size_t out_row = (size_t)b * a.Hq + (size_t)um.h0 + h;

  if (splits == 1) {
    if (h < G) {
      const float inv = L > 0.f ? 1.f / L : 0.f;
      store_out(a, out_row, d0, A, inv);
      if (a.lse && d0 == 0) a.lse[out_row] = L > 0.f ? M * kLn2 + logf(L) : ninf;
    }
    return;
  }

  // ---- several splits: publish the partial; the merge runs once all are in
  if (part_dst != nullptr) {
    if (h < G) {
      float* dst = part_dst + (size_t)split * kPartStride + h * kPartHead;
#pragma unroll
      for (int x = 0; x < kDimsPerThread; x += 4)
        *reinterpret_cast<float4*>(dst + d0 + x) = make_float4(A[x], A[x + 1], A[x + 2], A[x + 3]);
      if (d0 == 0) *reinterpret_cast<float2*>(dst + kHeadDim) = make_float2(M, L);
    }
    return;
  }
  if (a.route_k > 0) {
    route_publish(a, u, split, splits, slot0, sm, h, G, d0, out_row, A, M, L);
    return;
  }
  float* part = a.ws_part + (slot0 + split) * kPartStride;
  if (h < G) {
    float* dst = part + h * kPartHead;
#pragma unroll
    for (int x = 0; x < kDimsPerThread; x += 4)
      *reinterpret_cast<float4*>(dst + d0 + x) = make_float4(A[x], A[x + 1], A[x + 2], A[x + 3]);
    if (d0 == 0) *reinterpret_cast<float2*>(dst + kHeadDim) = make_float2(M, L);
  }
  // the counter increment is acq_rel: it publishes this CTA's partial and,
  // for the last CTA, acquires the other splits' partials
  __syncthreads();
  if (tid == 0) {
    const uint32_t prev = atom_add_acq_rel_u32(&a.ws_count[u], 1u);
    *sm.last = (prev == (uint32_t)(splits - 1));
  }
  __syncthreads();
  if (!*sm.last) return;
  if (tid == 0) a.ws_count[u] = 0;
  if (h >= G) return;
  merge_splits<false>(a, a.ws_part + slot0 * kPartStride + h * kPartHead, splits, out_row, d0);
}

}  // namespace dec
}  // namespace sa
