// Device helpers shared by the sparse-attention kernels (sm_100a).
//
// Fragment conventions (warp-level mma.sync, m16n8k16 bf16):
// lane = 4*g + c with g = lane / 4 (row group) and c = lane % 4.
//   A (16 x 16 bf16): reg0 = A[g][2c..2c+1], reg1 = A[g+8][2c..2c+1],
//                     reg2 = A[g][2c+8..2c+9], reg3 = A[g+8][2c+8..2c+9]
//   B (16 x 8 bf16):  reg0 = B[2c..2c+1][g], reg1 = B[2c+8..2c+9][g]
//   C (16 x 8 f32):   c0,c1 = C[g][2c..2c+1], c2,c3 = C[g+8][2c..2c+1]
// The reduction index k of a dot product may be permuted freely as long as
// A and B use the same permutation; the kernels pick the permutation that
// lets every lane fetch whole 16-byte chunks of a row, so global loads are
// fully coalesced and shared-memory reads are conflict-free.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "sparse_attn.h"

#define SA_DEV __device__ __forceinline__

namespace sa {

constexpr int kHeadDim = 128;
constexpr int kMetaBytes = 512;      // metadata bytes per (b, kv head, page)
constexpr int kMaxGroup = 8;         // query heads per KV head handled by one n8 MMA tile
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// ---------------------------------------------------------------- async copy
SA_DEV uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Record the first device-side error code in the workspace status word.
SA_DEV void flag_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

SA_DEV uint4 lds128(const void* p) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "r"(smem_addr(p)));
  return r;
}

SA_DEV uint4 ldg_nc128(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// ---------------------------------------------------------------- TMA + mbarrier
// 2D tiled bulk copies (no multicast) completing on a CTA-local mbarrier.
constexpr uint32_t kSpinLimit = 1u << 22;  // bounded waits: give up and flag SA_ERR_TIMEOUT

SA_DEV void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
SA_DEV void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}
SA_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}
SA_DEV bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Non-blocking test of phase `parity` of `bar` (for a thread that polls
// several barriers in turn).
SA_DEV bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Wait for phase `parity` of `bar`; after kSpinLimit polls give up, flag the
// status word and return false (the caller stops using the stage).
SA_DEV bool mbar_wait(uint64_t* bar, uint32_t parity, int* status) {
  for (uint32_t i = 0; i < kSpinLimit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  flag_status(status, SA_ERR_TIMEOUT);
  return false;
}
SA_DEV void tma_load_2d(void* dst, const void* tmap, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];\n" ::"r"(smem_addr(dst)),
      "l"(tmap), "r"(x), "r"(y), "r"(smem_addr(bar))
      : "memory");
}
SA_DEV void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_addr(bar)) : "memory");
}
SA_DEV void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }
// Orders this thread's generic-proxy global accesses with its async-proxy
// (TMA) ones: global data written with plain stores in the same launch and
// read by a later TMA copy takes one on each side of the handoff.
SA_DEV void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;\n" ::: "memory"); }
// Programmatic dependent launch: a kernel launched with programmatic stream
// serialisation may start while the previous kernel of the stream is still
// running; grid_dep_wait() returns once that kernel has completed and its
// memory operations are visible (at once when there is none), so it goes
// before the first global access.  grid_dep_trigger() lets the next such
// kernel begin launching (once every CTA of this grid has triggered or exited).
SA_DEV void grid_dep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
SA_DEV void grid_dep_trigger() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }
// Thread-block clusters: this CTA's rank in its cluster, the cluster's CTA
// count and its index in the grid (x).  cluster_sync(): every thread of every
// CTA of the cluster arrives (release at cluster scope) and waits (acquire),
// so each CTA's earlier writes, global or shared, are visible to the others.
SA_DEV uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
  return r;
}
SA_DEV uint32_t cluster_nctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;\n" : "=r"(r));
  return r;
}
SA_DEV uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;\n" : "=r"(r));
  return r;
}
SA_DEV void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}
// The two halves of cluster_sync, for work in between: a relaxed arrive
// (orders nothing; says "this CTA runs") and an acquire wait that the threads
// of a warp may reach at different points.
SA_DEV void cluster_arrive_relaxed() { asm volatile("barrier.cluster.arrive.relaxed.aligned;\n" ::: "memory"); }
SA_DEV void cluster_wait() { asm volatile("barrier.cluster.wait.acquire;\n" ::: "memory"); }
// Start moving the 128-byte line at p into L2 (no register written).
SA_DEV void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];\n" ::"l"(p)); }
SA_DEV void prefetch_tmap(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];\n" ::"l"(tmap) : "memory");
}

// Position of one warp in its private ring of mbarrier-tracked stages.  The
// ring outlives work items: stage = gi % stages, phase parity = (gi / stages) & 1.
struct WarpState {
  uint32_t gi;           // stages consumed so far by this warp
  bool alive;            // false after a barrier wait timed out
  uint32_t drain_lo;     // after a timeout: stages [drain_lo, drain_hi) may still be landing
  uint32_t drain_hi;
};

// CTA-to-CTA handoff.  After a __syncthreads, one thread's release (or
// acq_rel) operation at GPU scope publishes the writes of the whole CTA (the
// PTX memory model makes release cumulative over what the barrier ordered
// before it); the consumer's acquire makes them visible to its thread, and a
// __syncthreads passes that on to the rest of its CTA.
SA_DEV uint32_t atom_add_acq_rel_u32(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;\n" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// A GPU-scope fence, and the relaxed (strong) store and add that, after it,
// publish what the fence ordered before them -- two signals for the cost of
// one fence; the consumer of the add's count fences again to acquire.
SA_DEV void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;\n" ::: "memory"); }
SA_DEV void st_relaxed_u32(uint32_t* p, uint32_t v) {
  asm volatile("st.relaxed.gpu.global.u32 [%0], %1;\n" ::"l"(p), "r"(v) : "memory");
}
SA_DEV uint32_t atom_add_relaxed_u32(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.relaxed.gpu.global.add.u32 %0, [%1], %2;\n" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// GPU-scope acquire load / release store of a 32-bit flag in global memory.
SA_DEV uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];\n" : "=r"(v) : "l"(p) : "memory");
  return v;
}
SA_DEV void st_release_u32(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;\n" ::"l"(p), "r"(v) : "memory");
}

// Byte offset of 16-byte chunk j (0..7) of row r inside a 128B-swizzled box
// whose rows are 128 bytes (the TMA SWIZZLE_128B pattern: chunk j ^ (r & 7)).
SA_DEV uint32_t swz128(int r, int j) { return (uint32_t)(r * 128 + ((j ^ (r & 7)) << 4)); }

SA_DEV void ldsm_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3, const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_addr(p)));
}
SA_DEV void ldsm_x4_t(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3, const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_addr(p)));
}

// ---------------------------------------------------------------- tensor-core MMA
SA_DEV void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                     uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// FP64 tensor-core MMA m8n8k4: a = A[g][c], b = B[c][g], c0,c1 = C[g][2c..2c+1].
SA_DEV void mma_f64(double& c0, double& c1, double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};\n"
               : "+d"(c0), "+d"(c1)
               : "d"(a), "d"(b));
}

// Transpose an 8x8 b16 matrix held in the standard fragment layout.
SA_DEV uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}

SA_DEV uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;\n" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

SA_DEV uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
SA_DEV float bf16_lo(uint32_t x) { return __uint_as_float(x << 16); }
SA_DEV float bf16_hi(uint32_t x) { return __uint_as_float(x & 0xffff0000u); }

// Elementwise min(x, 0) / max(x, 0) of a packed bf16 pair (exact).
SA_DEV uint32_t bf16x2_neg_part(uint32_t x) {
  const uint32_t lo = (x & 0x8000u) ? (x & 0xffffu) : 0u;
  const uint32_t hi = (x & 0x80000000u) ? (x & 0xffff0000u) : 0u;
  return lo | hi;
}
SA_DEV uint32_t bf16x2_pos_part(uint32_t x) {
  const uint32_t lo = (x & 0x8000u) ? 0u : (x & 0xffffu);
  const uint32_t hi = (x & 0x80000000u) ? 0u : (x & 0xffff0000u);
  return lo | hi;
}

// ---------------------------------------------------------------- ordering keys
// Monotone map float -> uint32 (larger float -> larger key); -0.0 maps with +0.0.
SA_DEV uint32_t order_key(float s) {
  uint32_t u = __float_as_uint(s + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---------------------------------------------------------------- block scans
// Exclusive prefix sum over the block of one uint32 per thread; also returns
// the block total.  `scratch` holds at least (blockDim.x / 32) words.
SA_DEV uint32_t block_excl_scan(uint32_t v, uint32_t* scratch, uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[warp] = x;
  __syncthreads();
  uint32_t base = 0, tot = 0;
  for (int w = 0; w < nw; ++w) {
    const uint32_t s = scratch[w];
    if (w < warp) base += s;
    tot += s;
  }
  __syncthreads();
  total = tot;
  return base + x - v;
}

}  // namespace sa
