// Causal attention of query tiles over their routed blocks.
//
// "Technische Samenvatting: Onzekerheidsgestuurde Selectie voor Blok-schaarse
// Aandacht", "Methodologie" step 5: every tile attends to the blocks its list
// names (the top k, or the top rho*k when the tile triggered); sentinel (-1)
// entries are skipped.  Chunked-prefill rows attend causally: row r at
// position q_pos0 + r sees only keys at positions <= its own.
//
// Work split: CTA = (tile, KV head, 64 query vectors), a query vector being
// one (row, query head) pair of the tile, 16 per warp.  The kept blocks of the
// (tile, KV head) stream through a CTA-shared ring: each 64-token block is
// four TMA boxes (64 rows x 64 bf16, 128B swizzle) of K and V.  Per block and
// warp, on tensor cores (m16n8k16 bf16, fp32 accumulation):
//   S = Q K^T  (16 vectors x 64 keys; K fragments by ldmatrix),
//   online softmax per vector with the causal mask,
//   O += P V   (P reused from the S registers as the A operand, split into a
//               bf16 hi + lo pair; V fragments by ldmatrix.trans).
#include "common.cuh"
#include "internal.h"

namespace sa {
namespace {

constexpr int kTaWarps = 4;
constexpr int kTaThreads = 32 * kTaWarps;
constexpr int kTaVecs = 16 * kTaWarps;      // query vectors per CTA
constexpr int kTaStages = 3;
constexpr int kBlk = 64;                    // tokens per block (one TMA box of rows)
constexpr int kBox = kBlk * 128;            // 64 rows x 128 B
constexpr int kStage = 4 * kBox;            // K lo | K hi | V lo | V hi = 32 KiB
constexpr int kOffBars = kTaStages * kStage;
constexpr int kOffList = kOffBars + kTaStages * 8;

__global__ void __launch_bounds__(kTaThreads) tile_attn_kernel(const __grid_constant__ TileAttnArgs a) {
  extern __shared__ unsigned char smem_raw[];
  __shared__ int s_nb;
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + kOffBars);
  int* blist = reinterpret_cast<int*>(base + kOffList);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, c = lane & 3;
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
    for (int s = 0; s < kTaStages; ++s) mbar_init(bars + s, 1);
    fence_barrier_init();
    prefetch_tmap(&a.tmap_k);
    prefetch_tmap(&a.tmap_v);
    // the kept blocks, in list order (sentinels skipped; out-of-range flagged)
    int n = a.count[tg];
    if (n < 0 || n > a.max_sel) {
      flag_status(a.status, SA_ERR_DEVICE_CHECK);
      n = 0;
    }
    const int32_t* lst = a.idx + (size_t)tg * a.max_sel;
    int nb = 0;
    for (int i = 0; i < n; ++i) {
      const int blk = lst[i];
      if (blk < 0) continue;
      if (blk >= P) {
        flag_status(a.status, SA_ERR_DEVICE_CHECK);
        continue;
      }
      blist[nb++] = blk;
    }
    s_nb = nb;
  }
  __syncthreads();
  const int nb = s_nb;
  const long long rowbase = (long long)g * a.kv.cap;  // B == 1: unit u = g

  auto issue = [&](int i) {  // thread 0
    uint64_t* bar = bars + i % kTaStages;
    unsigned char* st = base + (i % kTaStages) * kStage;
    const int y = (int)(rowbase + (long long)blist[i] * kBlk);
    mbar_arrive_expect_tx(bar, kStage);
    tma_load_2d(st + 0 * kBox, &a.tmap_k, 0, y, bar);
    tma_load_2d(st + 1 * kBox, &a.tmap_k, 64, y, bar);
    tma_load_2d(st + 2 * kBox, &a.tmap_v, 0, y, bar);
    tma_load_2d(st + 3 * kBox, &a.tmap_v, 64, y, bar);
  };
  if (tid == 0)
    for (int i = 0; i < min(nb, kTaStages); ++i) issue(i);

  // ---- this lane's two query vectors (rows gq and gq + 8 of the warp's m-tile)
  const int va = mc * kTaVecs + 16 * warp + gq, vb = va + 8;
  const bool oka = va < V, okb = vb < V;
  const int pos_a = oka ? a.q_pos0 + row0 + va / G : -1;
  const int pos_b = okb ? a.q_pos0 + row0 + vb / G : -1;
  const __nv_bfloat16* Q = reinterpret_cast<const __nv_bfloat16*>(a.q);
  const __nv_bfloat16* qa = Q + ((size_t)(row0 + (oka ? va / G : 0)) * a.Hq + (size_t)g * G + (oka ? va % G : 0)) * kHeadDim;
  const __nv_bfloat16* qb = Q + ((size_t)(row0 + (okb ? vb / G : 0)) * a.Hq + (size_t)g * G + (okb ? vb % G : 0)) * kHeadDim;
  uint32_t qf[8][4];
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const int e = 16 * ks + 2 * c;
    qf[ks][0] = oka ? __ldg(reinterpret_cast<const uint32_t*>(qa + e)) : 0u;
    qf[ks][1] = okb ? __ldg(reinterpret_cast<const uint32_t*>(qb + e)) : 0u;
    qf[ks][2] = oka ? __ldg(reinterpret_cast<const uint32_t*>(qa + e + 8)) : 0u;
    qf[ks][3] = okb ? __ldg(reinterpret_cast<const uint32_t*>(qb + e + 8)) : 0u;
  }

  float m_a = ninf, m_b = ninf, l_a = 0.f, l_b = 0.f;
  float o[16][4];
#pragma unroll
  for (int dt = 0; dt < 16; ++dt) o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;

  int i_fail = -1;
  for (int i = 0; i < nb; ++i) {
    const bool ok = mbar_wait(bars + i % kTaStages, (i / kTaStages) & 1u, a.status);
    if (!__syncthreads_and(ok)) {
      i_fail = i;
      break;
    }
    unsigned char* st = base + (i % kTaStages) * kStage;
    const int blk = blist[i];
    const int kv0 = blk * kBlk;
    if (kv0 + kBlk > N) {  // zero V rows past the cache end (they may hold other data)
      for (int x = tid; x < (kv0 + kBlk - N) * 16; x += kTaThreads) {
        const int r = (N - kv0) + (x >> 4), ch = x & 15;
        *reinterpret_cast<uint4*>(st + (2 + (ch >> 3)) * kBox + swz128(r, ch & 7)) = make_uint4(0u, 0u, 0u, 0u);
      }
      fence_proxy_async();
      __syncthreads();
    }
    // S = Q K^T : 8 key n-tiles x 8 dim k-steps
    float s[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < 8; ks += 2) {
        const int ch = 2 * ks + (lane >> 3);  // 8-dim chunk 0..15
        uint32_t b0, b1, b2, b3;
        ldsm_x4(b0, b1, b2, b3, st + (ch >> 3) * kBox + swz128(8 * nt + (lane & 7), ch & 7));
        mma_bf16(s[nt], qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], b0, b1);
        mma_bf16(s[nt], qf[ks + 1][0], qf[ks + 1][1], qf[ks + 1][2], qf[ks + 1][3], b2, b3);
      }
    }
    // causal + cache-end mask, online softmax (log2 domain)
    float mx_a = ninf, mx_b = ninf;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const int p0 = kv0 + 8 * nt + 2 * c;
      s[nt][0] = (p0 <= pos_a && p0 < N) ? s[nt][0] * a.scale_log2 : ninf;
      s[nt][1] = (p0 + 1 <= pos_a && p0 + 1 < N) ? s[nt][1] * a.scale_log2 : ninf;
      s[nt][2] = (p0 <= pos_b && p0 < N) ? s[nt][2] * a.scale_log2 : ninf;
      s[nt][3] = (p0 + 1 <= pos_b && p0 + 1 < N) ? s[nt][3] * a.scale_log2 : ninf;
      mx_a = fmaxf(mx_a, fmaxf(s[nt][0], s[nt][1]));
      mx_b = fmaxf(mx_b, fmaxf(s[nt][2], s[nt][3]));
    }
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
    const float mn_a = fmaxf(m_a, mx_a), mn_b = fmaxf(m_b, mx_b);
    const float al_a = mn_a == ninf ? 1.f : exp2f(m_a - mn_a);
    const float al_b = mn_b == ninf ? 1.f : exp2f(m_b - mn_b);
    m_a = mn_a;
    m_b = mn_b;
    float rs_a = 0.f, rs_b = 0.f;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      s[nt][0] = mn_a == ninf ? 0.f : exp2f(s[nt][0] - mn_a);
      s[nt][1] = mn_a == ninf ? 0.f : exp2f(s[nt][1] - mn_a);
      s[nt][2] = mn_b == ninf ? 0.f : exp2f(s[nt][2] - mn_b);
      s[nt][3] = mn_b == ninf ? 0.f : exp2f(s[nt][3] - mn_b);
      rs_a += s[nt][0] + s[nt][1];
      rs_b += s[nt][2] + s[nt][3];
    }
    l_a = l_a * al_a + rs_a;
    l_b = l_b * al_b + rs_b;
#pragma unroll
    for (int dt = 0; dt < 16; ++dt) {
      o[dt][0] *= al_a; o[dt][1] *= al_a; o[dt][2] *= al_b; o[dt][3] *= al_b;
    }
    // O += P V : 4 key k-steps x 16 dim n-tiles; P as the A operand (hi + lo)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t ph[4], pl[4];
      ph[0] = pack_bf16(s[2 * j][0], s[2 * j][1]);
      ph[1] = pack_bf16(s[2 * j][2], s[2 * j][3]);
      ph[2] = pack_bf16(s[2 * j + 1][0], s[2 * j + 1][1]);
      ph[3] = pack_bf16(s[2 * j + 1][2], s[2 * j + 1][3]);
      pl[0] = pack_bf16(s[2 * j][0] - bf16_lo(ph[0]), s[2 * j][1] - bf16_hi(ph[0]));
      pl[1] = pack_bf16(s[2 * j][2] - bf16_lo(ph[1]), s[2 * j][3] - bf16_hi(ph[1]));
      pl[2] = pack_bf16(s[2 * j + 1][0] - bf16_lo(ph[2]), s[2 * j + 1][1] - bf16_hi(ph[2]));
      pl[3] = pack_bf16(s[2 * j + 1][2] - bf16_lo(ph[3]), s[2 * j + 1][3] - bf16_hi(ph[3]));
      const int key = 16 * j + (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
      for (int dt = 0; dt < 16; dt += 2) {
        const int ch = dt + (lane >> 4);  // 8-dim chunk
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(b0, b1, b2, b3, st + (2 + (ch >> 3)) * kBox + swz128(key, ch & 7));
        mma_bf16(o[dt], ph[0], ph[1], ph[2], ph[3], b0, b1);
        mma_bf16(o[dt], pl[0], pl[1], pl[2], pl[3], b0, b1);
        mma_bf16(o[dt + 1], ph[0], ph[1], ph[2], ph[3], b2, b3);
        mma_bf16(o[dt + 1], pl[0], pl[1], pl[2], pl[3], b2, b3);
      }
    }
    __syncthreads();  // stage i consumed by every warp
    if (tid == 0 && i + kTaStages < nb) issue(i + kTaStages);
  }
  if (i_fail >= 0 && tid == 0) {  // let the copies still in flight land (bounded)
    const int hi = min(nb, i_fail + kTaStages);
    for (int i = i_fail; i < hi; ++i) mbar_wait(bars + i % kTaStages, (i / kTaStages) & 1u, nullptr);
  }

  // ---- normalise and write
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
  const float inv_a = l_a > 0.f ? 1.f / l_a : 0.f, inv_b = l_b > 0.f ? 1.f / l_b : 0.f;
  if (oka) {
    const size_t orow = (size_t)(row0 + va / G) * a.Hq + (size_t)g * G + va % G;
    float* dst = a.out + orow * kHeadDim;
#pragma unroll
    for (int dt = 0; dt < 16; ++dt)
      *reinterpret_cast<float2*>(dst + 8 * dt + 2 * c) = make_float2(o[dt][0] * inv_a, o[dt][1] * inv_a);
    if (a.lse && c == 0) a.lse[orow] = l_a > 0.f ? m_a * kLn2 + logf(l_a) : ninf;
  }
  if (okb) {
    const size_t orow = (size_t)(row0 + vb / G) * a.Hq + (size_t)g * G + vb % G;
    float* dst = a.out + orow * kHeadDim;
#pragma unroll
    for (int dt = 0; dt < 16; ++dt)
      *reinterpret_cast<float2*>(dst + 8 * dt + 2 * c) = make_float2(o[dt][2] * inv_b, o[dt][3] * inv_b);
    if (a.lse && c == 0) a.lse[orow] = l_b > 0.f ? m_b * kLn2 + logf(l_b) : ninf;
  }
}

}  // namespace

size_t tile_attn_smem_bytes(int max_sel) { return 1024 + kOffList + (size_t)max_sel * 4; }

cudaError_t launch_tile_attn(const TileAttnArgs& a, cudaStream_t st) {
  const size_t smem = tile_attn_smem_bytes(a.max_sel);
  const long long grid = (long long)a.n_tiles * a.kv.Hkv * a.n_mchunks;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
  const cudaError_t e = set_smem_attr((const void*)tile_attn_kernel, smem);
  if (e != cudaSuccess) return e;
  tile_attn_kernel<<<(unsigned)grid, kTaThreads, smem, st>>>(a);
  return cudaGetLastError();
}

int tile_attn_mchunks(int vectors_per_tile) { return (vectors_per_tile + kTaVecs - 1) / kTaVecs; }

}  // namespace sa
