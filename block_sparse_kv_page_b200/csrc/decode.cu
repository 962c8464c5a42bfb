// Sparse paged flash-decode over the selected pages, split-K + combine.
//
// "Sparse Attention for Web Agents -- Offline Replay Records", section "The
// comparison": after choosing the best chunks the methods attend only to
// them; exact softmax attention over the selected tokens.
//
// Work split.  A unit is one (sequence, KV head) with its G <= 8 query heads.
// Its selected pages are cut into 16-token tiles (a 16-token page is one
// tile; larger pages and variable chunks give several, the last one ragged),
// the tiles into `splits` contiguous ranges, one CTA (4 warps) per range.
// Each warp streams its tiles through a private 3-stage cp.async ring (K and
// V tile = 8 KiB, one 16-byte chunk per lane and slot, fragment-major so the
// shared-memory reads are conflict-free) and keeps its own online-softmax
// state for the G heads:
//   QK:  S^T[16 tok x 8 heads] = K (16 x 128) . Q^T, m16n8k16 bf16, fp32 acc;
//   P:   exp2 of the scaled scores, rounded to a bf16 hi + lo pair, moved
//        from the C layout to the B layout with movmatrix (8x8 transpose);
//   PV:  O^T[128 dims x 8 heads] += V^T (128 x 16 tok) . P^T, m16n8k16, with
//        the output dimensions permuted so each lane loads 32 contiguous
//        bytes of every V row it needs.
// The four warps merge in shared memory; with several splits the CTA writes
// its (max, sum, acc) partial to the workspace and the CTA that finishes the
// unit last (atomic counter, no waiting) merges the partials in split order,
// so results do not depend on scheduling.
#include "common.cuh"
#include "internal.h"

namespace sa {
namespace {

constexpr int kDecWarps = 4;
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kDecStages = 3;
constexpr int kSlot = 32 * 16;                 // one 16-byte chunk per lane
constexpr int kDecStageBytes = 16 * kSlot;     // 8 K chunks + 8 V chunks per lane
constexpr int kDecRingBytes = kDecWarps * kDecStages * kDecStageBytes;
constexpr int kPartStride = kMaxGroup * (kHeadDim + 2);  // floats per partial slot

struct TileRef {
  int start;   // first token of the tile in the unit's cache
  int n;       // valid tokens (0 = empty tile)
};

__global__ void __launch_bounds__(kDecThreads) decode_kernel(DecodeArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_last;
  __shared__ int s_ntiles;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, c = lane & 3;
  const int u = blockIdx.x / a.splits;      // (row, kv head)
  const int split = blockIdx.x % a.splits;
  const int Hkv = a.kv.Hkv;
  const int b = u / Hkv, g = u % Hkv;
  const int G = a.G;
  const float ninf = -__int_as_float(0x7f800000);

  // ---- geometry of the unit
  const int N = a.kv.seq_len[b];
  bool bad = (N < 1 || N > a.kv.cap);
  int n_ent = a.count[u];
  if (n_ent < 0 || n_ent > a.max_sel) bad = true;
  if (bad) n_ent = 0;
  const int32_t* idx_u = a.idx + (size_t)u * a.max_sel;
  const int ps = a.kv.page_size;
  const int sub = ps > 0 ? ps / 16 : 0;
  int P = 0;
  const int32_t* off = nullptr;
  int* pre = reinterpret_cast<int*>(smem + kDecRingBytes);  // chunk mode: tile prefix [n_ent+1]
  if (ps > 0) {
    P = (N + ps - 1) / ps;
    if (tid == 0) s_ntiles = n_ent * sub;
  } else {
    off = a.kv.chunk_off + (size_t)b * (a.kv.max_pages + 1);
    P = a.kv.n_chunks[b];
    if (P < 1 || P > a.kv.max_pages) { bad = true; n_ent = 0; P = 0; }
    // tile count of every entry, exclusive prefix in shared memory
    const int per = (n_ent + kDecThreads - 1) / kDecThreads;
    const int e0 = min(n_ent, tid * per), e1 = min(n_ent, e0 + per);
    uint32_t loc = 0;
    for (int e = e0; e < e1; ++e) {
      const int ch = idx_u[e];
      int nt = 0;
      if (ch >= 0 && ch < P && off[ch] >= 0) nt = (max(0, min(off[ch + 1], N) - off[ch]) + 15) >> 4;
      pre[e] = nt;
      loc += (uint32_t)nt;
    }
    __shared__ uint32_t s_scan[kDecWarps];
    uint32_t tot;
    uint32_t run = block_excl_scan(loc, s_scan, tot);
    for (int e = e0; e < e1; ++e) {
      const int nt = pre[e];
      pre[e] = (int)run;
      run += (uint32_t)nt;
    }
    if (tid == 0) { pre[n_ent] = (int)tot; s_ntiles = (int)tot; }
  }
  if (bad && tid == 0 && split == 0) flag_status(a.status, SA_ERR_DEVICE_CHECK);
  __syncthreads();
  const int T = s_ntiles;
  const int t_begin = (int)(((long long)T * split) / a.splits);
  const int t_end = (int)(((long long)T * (split + 1)) / a.splits);

  auto tile_ref = [&](int t) -> TileRef {
    TileRef r{0, 0};
    if (ps > 0) {
      const int e = t / sub, part = t - e * sub;
      const int p = idx_u[e];
      if (p < 0 || p >= P) {
        if (lane == 0) flag_status(a.status, SA_ERR_DEVICE_CHECK);
        return r;
      }
      r.start = p * ps + part * 16;
      r.n = max(0, min(16, N - r.start));
    } else {
      int lo = 0, hi = n_ent - 1;  // last e with pre[e] <= t
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (pre[mid] <= t) lo = mid; else hi = mid - 1;
      }
      const int ch = idx_u[lo];
      if (ch < 0 || ch >= P || off[ch] < 0) {
        if (lane == 0) flag_status(a.status, SA_ERR_DEVICE_CHECK);
        return r;
      }
      r.start = off[ch] + (t - pre[lo]) * 16;
      r.n = max(0, min(16, min(off[ch + 1], N) - r.start));
    }
    return r;
  };

  // ---- Q fragments of this lane's head column (zero for heads >= G)
  const bool head_ok = gq < G;
  const __nv_bfloat16* qrow = reinterpret_cast<const __nv_bfloat16*>(a.q) +
                              ((size_t)b * a.Hq + (size_t)g * G + (head_ok ? gq : 0)) * kHeadDim;
  uint32_t bq[16];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 v = head_ok ? ldg_nc128(qrow + 32 * i + 8 * c) : make_uint4(0, 0, 0, 0);
    bq[4 * i + 0] = v.x; bq[4 * i + 1] = v.y; bq[4 * i + 2] = v.z; bq[4 * i + 3] = v.w;
  }

  const __nv_bfloat16* Kb = reinterpret_cast<const __nv_bfloat16*>(a.kv.k) + (size_t)u * a.kv.cap * kHeadDim;
  const __nv_bfloat16* Vb = reinterpret_cast<const __nv_bfloat16*>(a.kv.v) + (size_t)u * a.kv.cap * kHeadDim;
  unsigned char* ring = smem + warp * (kDecStages * kDecStageBytes);

  auto issue = [&](int it) {
    const int t = t_begin + warp + it * kDecWarps;
    if (t < t_end) {
      const TileRef r = tile_ref(t);
      unsigned char* st = ring + (it % kDecStages) * kDecStageBytes + lane * 16;
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {  // K rows gq, gq + 8: chunks 32i + 8c
        const int j = gq + 8 * rr;
        const bool ok = j < r.n;
        const __nv_bfloat16* src = Kb + (size_t)(ok ? r.start + j : 0) * kHeadDim + 8 * c;
#pragma unroll
        for (int i = 0; i < 4; ++i) cp_async16(st + (rr * 4 + i) * kSlot, src + 32 * i, ok);
      }
#pragma unroll
      for (int tk = 0; tk < 4; ++tk) {  // V rows 2c, 2c+1, 2c+8, 2c+9: dims 16gq .. +16
        const int j = 2 * c + (tk & 1) + 8 * (tk >> 1);
        const bool ok = j < r.n;
        const __nv_bfloat16* src = Vb + (size_t)(ok ? r.start + j : 0) * kHeadDim + 16 * gq;
        cp_async16(st + (8 + 2 * tk) * kSlot, src, ok);
        cp_async16(st + (9 + 2 * tk) * kSlot, src + 8, ok);
      }
    }
    cp_async_commit();
  };

  float m0 = ninf, m1 = ninf, l0 = 0.f, l1 = 0.f;
  float acc[8][4];
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;

  const int n_it = max(0, (t_end - t_begin - warp + kDecWarps - 1) / kDecWarps);
#pragma unroll
  for (int it = 0; it < kDecStages - 1; ++it) issue(it);
  for (int it = 0; it < n_it; ++it) {
    cp_async_wait<kDecStages - 2>();
    issue(it + kDecStages - 1);
    const int t = t_begin + warp + it * kDecWarps;
    const TileRef r = tile_ref(t);
    const unsigned char* st = ring + (it % kDecStages) * kDecStageBytes + lane * 16;

    // S^T = K . Q^T
    float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 k0 = lds128(st + i * kSlot);
      const uint4 k1 = lds128(st + (4 + i) * kSlot);
      mma_bf16(s, k0.x, k1.x, k0.y, k1.y, bq[4 * i + 0], bq[4 * i + 1]);
      mma_bf16(s, k0.z, k1.z, k0.w, k1.w, bq[4 * i + 2], bq[4 * i + 3]);
    }
    const bool v0 = gq < r.n, v1 = gq + 8 < r.n;
    const float z0 = v0 ? s[0] * a.scale_log2 : ninf;
    const float z1 = v0 ? s[1] * a.scale_log2 : ninf;
    const float z2 = v1 ? s[2] * a.scale_log2 : ninf;
    const float z3 = v1 ? s[3] * a.scale_log2 : ninf;
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
    // P (C layout: [token][head]) -> bf16 hi/lo -> B layout ([head][token]) by transpose
    const uint32_t hlo = pack_bf16(p0, p1), hhi = pack_bf16(p2, p3);
    const uint32_t llo = pack_bf16(p0 - bf16_lo(hlo), p1 - bf16_hi(hlo));
    const uint32_t lhi = pack_bf16(p2 - bf16_lo(hhi), p3 - bf16_hi(hhi));
    const uint32_t bh0 = movmatrix_t(hlo), bh1 = movmatrix_t(hhi);
    const uint32_t bl0 = movmatrix_t(llo), bl1 = movmatrix_t(lhi);

    const uint4 va = lds128(st + 8 * kSlot), vb = lds128(st + 9 * kSlot);    // token 2c
    const uint4 vc = lds128(st + 10 * kSlot), vd = lds128(st + 11 * kSlot);  // token 2c+1
    const uint4 ve = lds128(st + 12 * kSlot), vf = lds128(st + 13 * kSlot);  // token 2c+8
    const uint4 vg = lds128(st + 14 * kSlot), vh = lds128(st + 15 * kSlot);  // token 2c+9
    const uint32_t X0[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
    const uint32_t X1[8] = {vc.x, vc.y, vc.z, vc.w, vd.x, vd.y, vd.z, vd.w};
    const uint32_t X2[8] = {ve.x, ve.y, ve.z, ve.w, vf.x, vf.y, vf.z, vf.w};
    const uint32_t X3[8] = {vg.x, vg.y, vg.z, vg.w, vh.x, vh.y, vh.z, vh.w};
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      const uint32_t a0 = prmt(X0[mt], X1[mt], 0x5410), a1 = prmt(X0[mt], X1[mt], 0x7632);
      const uint32_t a2 = prmt(X2[mt], X3[mt], 0x5410), a3 = prmt(X2[mt], X3[mt], 0x7632);
      mma_bf16(acc[mt], a0, a1, a2, a3, bh0, bh1);
      mma_bf16(acc[mt], a0, a1, a2, a3, bl0, bl1);
    }
  }
  cp_async_wait<0>();

  // ---- merge the 4 warps in shared memory
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
  }
  __syncthreads();  // ring no longer read
  float* w_acc = reinterpret_cast<float*>(smem);                       // [warp][8][128]
  float* w_ml = w_acc + kDecWarps * kMaxGroup * kHeadDim;               // [warp][8][2]
  if (gq == 0) {
    w_ml[(warp * kMaxGroup + 2 * c) * 2 + 0] = m0;
    w_ml[(warp * kMaxGroup + 2 * c) * 2 + 1] = l0;
    w_ml[(warp * kMaxGroup + 2 * c + 1) * 2 + 0] = m1;
    w_ml[(warp * kMaxGroup + 2 * c + 1) * 2 + 1] = l1;
  }
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    const int d = 16 * gq + 2 * mt;
    *reinterpret_cast<float2*>(w_acc + (warp * kMaxGroup + 2 * c) * kHeadDim + d) =
        make_float2(acc[mt][0], acc[mt][2]);
    *reinterpret_cast<float2*>(w_acc + (warp * kMaxGroup + 2 * c + 1) * kHeadDim + d) =
        make_float2(acc[mt][1], acc[mt][3]);
  }
  __syncthreads();

  const int h = tid >> 4;            // head handled by this thread
  const int d0 = (tid & 15) * 8;     // 8 dimensions
  float M = ninf, L = 0.f, A[8];
#pragma unroll
  for (int x = 0; x < 8; ++x) A[x] = 0.f;
  if (h < G) {
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, w_ml[(w * kMaxGroup + h) * 2]);
    if (M != ninf) {
#pragma unroll
      for (int w = 0; w < kDecWarps; ++w) {
        const float f = exp2f(w_ml[(w * kMaxGroup + h) * 2] - M);
        L += w_ml[(w * kMaxGroup + h) * 2 + 1] * f;
        const float* src = w_acc + (w * kMaxGroup + h) * kHeadDim + d0;
#pragma unroll
        for (int x = 0; x < 8; ++x) A[x] += src[x] * f;
      }
    }
  }
  const size_t out_row = (size_t)b * a.Hq + (size_t)g * G + h;

  if (a.splits == 1) {
    if (h < G) {
      const float inv = L > 0.f ? 1.f / L : 0.f;
      float4* o = reinterpret_cast<float4*>(a.out + out_row * kHeadDim + d0);
      o[0] = make_float4(A[0] * inv, A[1] * inv, A[2] * inv, A[3] * inv);
      o[1] = make_float4(A[4] * inv, A[5] * inv, A[6] * inv, A[7] * inv);
      if (a.lse && d0 == 0) a.lse[out_row] = L > 0.f ? M * kLn2 + logf(L) : ninf;
    }
    return;
  }

  // ---- several splits: publish the partial; the last CTA of the unit merges
  float* part = a.ws_part + ((size_t)u * a.splits + split) * kPartStride;
  if (h < G) {
    float* dst = part + h * (kHeadDim + 2);
#pragma unroll
    for (int x = 0; x < 8; ++x) dst[d0 + x] = A[x];
    if (d0 == 0) { dst[kHeadDim] = M; dst[kHeadDim + 1] = L; }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const uint32_t prev = atomicAdd(&a.ws_count[u], 1u);
    s_last = (prev == (uint32_t)(a.splits - 1));
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (tid == 0) a.ws_count[u] = 0;
  if (h >= G) return;

  const float* base = a.ws_part + (size_t)u * a.splits * kPartStride + h * (kHeadDim + 2);
  float MM = ninf;
  for (int sp = 0; sp < a.splits; ++sp) MM = fmaxf(MM, __ldcg(base + (size_t)sp * kPartStride + kHeadDim));
  float LL = 0.f, AA[8];
#pragma unroll
  for (int x = 0; x < 8; ++x) AA[x] = 0.f;
  if (MM != ninf) {
    for (int sp = 0; sp < a.splits; ++sp) {
      const float* src = base + (size_t)sp * kPartStride;
      const float f = exp2f(__ldcg(src + kHeadDim) - MM);
      LL += __ldcg(src + kHeadDim + 1) * f;
#pragma unroll
      for (int x = 0; x < 8; ++x) AA[x] += __ldcg(src + d0 + x) * f;
    }
  }
  const float inv = LL > 0.f ? 1.f / LL : 0.f;
  float4* o = reinterpret_cast<float4*>(a.out + out_row * kHeadDim + d0);
  o[0] = make_float4(AA[0] * inv, AA[1] * inv, AA[2] * inv, AA[3] * inv);
  o[1] = make_float4(AA[4] * inv, AA[5] * inv, AA[6] * inv, AA[7] * inv);
  if (a.lse && d0 == 0) a.lse[out_row] = LL > 0.f ? MM * kLn2 + logf(LL) : ninf;
}

}  // namespace

int decode_splits(int units, int max_tiles, int sm_count) {
  const int target = 2 * sm_count;
  int s = (target + units - 1) / units;
  const int max_s = (max_tiles + 3) / 4;  // at least ~4 tiles per split
  if (s > max_s) s = max_s;
  if (s > 64) s = 64;
  if (s < 1) s = 1;
  return s;
}

size_t decode_smem_bytes(int max_sel, bool chunks) {
  size_t s = kDecRingBytes;
  if (chunks) s += (size_t)(max_sel + 1) * 4;
  return s;
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st) {
  const size_t smem = decode_smem_bytes(a.max_sel, a.kv.page_size == 0);
  const long long grid = (long long)a.n_rows * a.kv.Hkv * a.splits;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  decode_kernel<<<(unsigned)grid, kDecThreads, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace sa
