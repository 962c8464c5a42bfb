// Uncertainty router over query tiles (placeholder until the router kernels land).
#include "common.cuh"
#include "internal.h"

namespace sa {

size_t route_ws_bytes(int n_tiles, int Hkv, int max_pages) {
  (void)n_tiles; (void)Hkv; (void)max_pages;
  return 0;
}

cudaError_t launch_route(const RouteArgs& a, cudaStream_t st) {
  (void)a; (void)st;
  return cudaErrorNotSupported;
}

}  // namespace sa
