// Page metadata builder: per (sequence, KV head, page) the per-dimension key
// minimum and maximum (envelope scoring) or the key mean (centroid scoring).
// "Sparse Attention for Web Agents -- Offline Replay Records", section "The
// comparison" (scoring column: per-dimension min/max upper bound, mean of
// chunk keys).
//
// One warp per page (page_meta.cuh: lane l owns dimensions 4l..4l+3; min/max
// exact in bf16, mean summed in fp64 and rounded once to fp32).  Only pages
// overlapping [t0_b, N_b) are rewritten, so appending a token costs one page
// per (sequence, KV head).
#include "common.cuh"
#include "internal.h"
#include "page_meta.cuh"

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

template <int RULE>
__global__ void __launch_bounds__(kMetaWarps * 32) build_meta_kernel(MetaParams p) {
  grid_dep_wait();     // the previous kernel of the stream has completed
  grid_dep_trigger();  // one short pass: the next kernel may start launching
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
  const PageMetaLane m = page_meta_lane<RULE>(K, s, e);
  store_page_meta<RULE>(p.meta + ((size_t)u * p.kv.max_pages + page) * kMetaBytes, m, lane);
}

}  // namespace

cudaError_t launch_build_meta(const KvView& kv, int rule, int first_token, void* meta,
                              int* status, cudaStream_t st) {
  MetaParams p{};
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
  if (rule == 0) return launch_pdl(build_meta_kernel<0>, (unsigned)blocks, kMetaWarps * 32, 0, st, p);
  return launch_pdl(build_meta_kernel<1>, (unsigned)blocks, kMetaWarps * 32, 0, st, p);
}

}  // namespace sa
