// Block-wide weighted radix select on order-preserving 32-bit keys, shared by
// the page selector and the router.
#pragma once

#include "common.cuh"


namespace sa {

struct RadixCut {
  uint32_t T;    // the cut key
  uint32_t rem;  // capacity left for keys equal to T
};

// Weighted MSB-first radix select on keys[0..P): the key T such that the total
// weight of keys > T is <= cap < total weight of keys >= T, and
// rem = cap - weight(keys > T).  Requires total weight > cap.  All threads of
// the block call it; hist holds 256 words, bc 4 words (shared memory).
// The leading bytes shared by every key (scores of one unit often share sign
// and exponent) are skipped.
SA_DEV RadixCut radix_cut(const uint32_t* keys, const uint32_t* wts, int P, uint32_t cap,
                          uint32_t* hist, uint32_t* bc) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nt = blockDim.x;
  // common prefix of all keys: bytes where min and max agree
  uint32_t kmn = 0xffffffffu, kmx = 0u;
  for (int i = tid; i < P; i += nt) {
    kmn = min(kmn, keys[i]);
    kmx = max(kmx, keys[i]);
  }
  kmn = __reduce_min_sync(0xffffffffu, kmn);
  kmx = __reduce_max_sync(0xffffffffu, kmx);
  if (tid < 4) bc[tid] = tid & 1 ? 0u : 0xffffffffu;
  __syncthreads();
  if (lane == 0) {
    atomicMin(&bc[0], kmn);
    atomicMax(&bc[1], kmx);
  }
  __syncthreads();
  const uint32_t gmin = bc[0], gmax = bc[1];
  __syncthreads();
  const int first_pass = (gmin == gmax) ? 4 : (__clz(gmin ^ gmax) >> 3);
  if (first_pass == 4) return {gmin, cap};  // all keys equal: index order decides
  uint32_t mask = first_pass == 0 ? 0u : (0xffffffffu << (32 - 8 * first_pass));
  uint32_t prefix = gmin & mask, rem = cap;
  for (int pass = first_pass; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = tid; i < 256; i += nt) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < P; i += nt) {
      const uint32_t k = keys[i];
      if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], wts ? wts[i] : 1u);
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns buckets 255-8l .. 248-8l (descending); find the bucket
      // where the running weight from the top first exceeds rem
      uint32_t h[8], ls = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        h[q] = hist[255 - 8 * lane - q];
        ls += h[q];
      }
      uint32_t inc = ls;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
      }
      const unsigned ball = __ballot_sync(0xffffffffu, inc > rem);
      const int L = __ffs(ball) - 1;
      if (lane == L) {
        uint32_t run = inc - ls;
        int d = 255 - 8 * lane - 7;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (run + h[q] > rem) {
            d = 255 - 8 * lane - q;
            break;
          }
          run += h[q];
        }
        bc[0] = (uint32_t)d;
        bc[1] = run;
      }
    }
    __syncthreads();
    const uint32_t d = bc[0];
    rem -= bc[1];
    prefix |= d << shift;
    mask |= 0xffu << shift;
    __syncthreads();
  }
  return {prefix, rem};
}

}  // namespace sa
