// Metadata of one page or chunk computed by one warp: per-dimension key
// minimum and maximum (envelope scoring) or key mean (centroid scoring).
// "Sparse Attention for Web Agents -- Offline Replay Records", section "The
// comparison" (scoring column: per-dimension min/max upper bound, mean of
// chunk keys).
//
// Lane l owns dimensions 4l..4l+3 and walks the rows with 8-byte loads, so a
// warp reads each 256-byte key row coalesced.  min/max are exact in bf16; the
// mean is summed in fp64 in row order and rounded once to fp32.  The metadata
// builder and the fused decode step both call this, so a page refreshed by
// either holds the same bytes.
#pragma once

#include "common.cuh"

namespace sa {

struct PageMetaLane {
  uint2 lo;      // envelope: kmin of dims 4l..4l+3 (bf16 x 4); bytes [8l, 8l + 8) of the row
  uint2 hi;      // envelope: kmax of dims 4l..4l+3; bytes [256 + 8l, 256 + 8l + 8)
  float4 mean;   // centroid: mean of dims 4l..4l+3; bytes [16l, 16l + 16)
};

// k_lane = first key row of the (sequence, KV head) + 4 * lane elements;
// the page covers rows [s, e), e > s.  With use_last, row e - 1 is taken from
// `last` (this lane's 4 elements) instead of memory: the fused step appends
// the newest key and folds it in without reading it back.
template <int RULE>
SA_DEV PageMetaLane page_meta_lane(const __nv_bfloat16* k_lane, int s, int e, bool use_last = false,
                                   uint2 last = make_uint2(0u, 0u)) {
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
      r[x] = x >= n                    ? make_uint2(0u, 0u)
             : use_last && t + x == e - 1 ? last
                                          : __ldg(reinterpret_cast<const uint2*>(k_lane + (size_t)(t + x) * kHeadDim));
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
  PageMetaLane m;
  if (RULE == 0) {
    // min/max of bf16 inputs are bf16 inputs, so the casts are exact
    m.lo = make_uint2(pack_bf16(mn[0], mn[1]), pack_bf16(mn[2], mn[3]));
    m.hi = make_uint2(pack_bf16(mx[0], mx[1]), pack_bf16(mx[2], mx[3]));
    m.mean = make_float4(0.f, 0.f, 0.f, 0.f);
  } else {
    const double inv = 1.0 / (double)(e - s);
    m.mean = make_float4((float)(sm[0] * inv), (float)(sm[1] * inv), (float)(sm[2] * inv),
                         (float)(sm[3] * inv));
    m.lo = m.hi = make_uint2(0u, 0u);
  }
  return m;
}

// Store the lane's part of the 512-byte metadata row at `dst` (global).
template <int RULE>
SA_DEV void store_page_meta(unsigned char* dst, const PageMetaLane& m, int lane) {
  if (RULE == 0) {
    reinterpret_cast<uint2*>(dst)[lane] = m.lo;
    reinterpret_cast<uint2*>(dst + 256)[lane] = m.hi;
  } else {
    reinterpret_cast<float4*>(dst)[lane] = m.mean;
  }
}

// Chunk holding token t: the largest c in [0, n) with off[c] <= t.
SA_DEV int chunk_containing(const int32_t* off, int n, int t) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

}  // namespace sa
