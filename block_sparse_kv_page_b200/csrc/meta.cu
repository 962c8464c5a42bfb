// Page metadata builder: per (sequence, KV head, page) the per-dimension key
// minimum and maximum (envelope scoring) or the key mean (centroid scoring).
// "Sparse Attention for Web Agents -- Offline Replay Records", section "The
// comparison" (scoring column: per-dimension min/max upper bound, mean of
// chunk keys).
//
// One warp per page; lane l owns dimensions 4l..4l+3 and walks the page's
// tokens with 8-byte loads (a warp reads each 256-byte key row coalesced).
// min/max are exact in bf16; the mean is accumulated in fp64 and rounded once
// to fp32.  Only pages overlapping [t0_b, N_b) are rewritten, so appending a
// token costs one page per (sequence, KV head).
#include "common.cuh"
#include "internal.h"

namespace sa {
namespace {

constexpr int kMetaWarps = 8;

struct MetaParams {
  KvView kv;
  int rule;          // 0 envelope, 1 centroid
  int first_token;
  int pages_per_unit;  // warps launched per (b, g)
  unsigned char* meta;
  int* status;
};

__device__ int chunk_containing(const int32_t* off, int n, int t) {
  // largest c in [0, n) with off[c] <= t
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <int RULE>
__global__ void __launch_bounds__(kMetaWarps * 32) build_meta_kernel(MetaParams p) {
  const int lane = threadIdx.x & 31;
  const long long wid = (long long)blockIdx.x * kMetaWarps + (threadIdx.x >> 5);
  const long long units = (long long)p.kv.B * p.kv.Hkv;
  if (wid >= units * p.pages_per_unit) return;
  const int u = (int)(wid / p.pages_per_unit);
  const int j = (int)(wid % p.pages_per_unit);
  const int b = u / p.kv.Hkv;
  const int N = p.kv.seq_len[b];
  if (N < 1 || N > p.kv.cap) {
    if (j == 0 && lane == 0) flag_status(p.status, SA_ERR_DEVICE_CHECK);
    return;
  }
  const int t0 = p.first_token >= 0 ? p.first_token : max(0, N + p.first_token);
  if (t0 >= N) return;

  int page, s, e;
  if (p.kv.page_size > 0) {
    const int ps = p.kv.page_size;
    const int P = (N + ps - 1) / ps;
    page = t0 / ps + j;
    if (page >= P) return;
    s = page * ps;
    e = min(s + ps, N);
  } else {
    const int32_t* off = p.kv.chunk_off + (size_t)b * (p.kv.max_pages + 1);
    const int C = p.kv.n_chunks[b];
    if (C < 1 || C > p.kv.max_pages) {
      if (j == 0 && lane == 0) flag_status(p.status, SA_ERR_DEVICE_CHECK);
      return;
    }
    page = chunk_containing(off, C, t0) + j;
    if (page >= C) return;
    s = off[page];
    e = off[page + 1];
    if (s < 0 || e < s) {
      if (lane == 0) flag_status(p.status, SA_ERR_DEVICE_CHECK);
      return;
    }
    e = min(e, N);  // a chunk table may run ahead of the cache: clip to N
    if (s >= e) return;
  }
  if (page >= p.kv.max_pages) {
    if (lane == 0) flag_status(p.status, SA_ERR_DEVICE_CHECK);
    return;
  }

  const __nv_bfloat16* K = reinterpret_cast<const __nv_bfloat16*>(p.kv.k) +
                           ((size_t)u * p.kv.cap) * kHeadDim + lane * 4;
  float mn[4], mx[4];
  double sm[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    mn[i] = __int_as_float(0x7f800000);
    mx[i] = -__int_as_float(0x7f800000);
    sm[i] = 0.0;
  }
  // 16 rows per batch, all loads issued before any is used
  for (int t = s; t < e; t += 16) {
    const int n = min(16, e - t);
    uint2 r[16];
#pragma unroll
    for (int x = 0; x < 16; ++x)
      r[x] = x < n ? __ldg(reinterpret_cast<const uint2*>(K + (size_t)(t + x) * kHeadDim))
                   : make_uint2(0u, 0u);
#pragma unroll
    for (int x = 0; x < 16; ++x) {
      if (x < n) {
        const float f[4] = {bf16_lo(r[x].x), bf16_hi(r[x].x), bf16_lo(r[x].y), bf16_hi(r[x].y)};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if (RULE == 0) {
            mn[i] = fminf(mn[i], f[i]);
            mx[i] = fmaxf(mx[i], f[i]);
          } else {
            sm[i] += (double)f[i];
          }
        }
      }
    }
  }

  unsigned char* dst = p.meta + ((size_t)u * p.kv.max_pages + page) * kMetaBytes;
  if (RULE == 0) {
    // bf16 values: min/max of bf16 inputs are bf16 inputs, so the casts are exact.
    uint2 lo, hi;
    lo.x = pack_bf16(mn[0], mn[1]);
    lo.y = pack_bf16(mn[2], mn[3]);
    hi.x = pack_bf16(mx[0], mx[1]);
    hi.y = pack_bf16(mx[2], mx[3]);
    reinterpret_cast<uint2*>(dst)[lane] = lo;
    reinterpret_cast<uint2*>(dst + 256)[lane] = hi;
  } else {
    const double inv = 1.0 / (double)(e - s);
    float4 m;
    m.x = (float)(sm[0] * inv);
    m.y = (float)(sm[1] * inv);
    m.z = (float)(sm[2] * inv);
    m.w = (float)(sm[3] * inv);
    reinterpret_cast<float4*>(dst)[lane] = m;
  }
}

}  // namespace

cudaError_t launch_build_meta(const KvView& kv, int rule, int first_token, void* meta,
                              int* status, cudaStream_t st) {
  MetaParams p;
  p.kv = kv;
  p.rule = rule;
  p.first_token = first_token;
  p.meta = reinterpret_cast<unsigned char*>(meta);
  p.status = status;
  int ppu;
  if (first_token >= 0) {
    ppu = kv.page_size > 0 ? kv.max_pages - first_token / kv.page_size : kv.max_pages;
  } else {
    const long long n = -(long long)first_token;
    // pages overlapping the last n tokens: ceil((n - 1) / ps) + 1 at most
    ppu = kv.page_size > 0 ? (int)((n - 1 + kv.page_size - 1) / kv.page_size + 1)
                           : (int)(n < kv.max_pages ? n : kv.max_pages);
  }
  if (ppu > kv.max_pages) ppu = kv.max_pages;
  if (ppu <= 0) return cudaSuccess;
  p.pages_per_unit = ppu;
  const long long warps = (long long)kv.B * kv.Hkv * ppu;
  const long long blocks = (warps + kMetaWarps - 1) / kMetaWarps;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  if (rule == 0)
    build_meta_kernel<0><<<(unsigned)blocks, kMetaWarps * 32, 0, st>>>(p);
  else
    build_meta_kernel<1><<<(unsigned)blocks, kMetaWarps * 32, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace sa
