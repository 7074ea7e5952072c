// wq_common.cuh -- device helpers and the kernel-layout geometry shared by the
// library's CUDA sources (sm_100a only).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "wq.h"

namespace wq {

constexpr int kGroup = 128;           // group size along K
constexpr int kTileRows = 128;        // rows of one layout tile
constexpr int kSlabGroups = 4;        // groups in one K-slab
constexpr int kSlabK = kGroup * kSlabGroups;
constexpr int kCodeBytesPerGroupRow = kGroup / 2;   // 64 bytes of nibbles
constexpr int kCounterBytes = WQ_WORKSPACE_COUNTER_BYTES;
constexpr int kRowsPerCounter = 16;   // one completion counter per 16 output rows

// Device error word bits (see wq_last_device_status).
constexpr int kDevErrTimeout = 1;

// Geometry of layout WQ_LAYOUT_TILED for an N x K weight.
struct Geom {
  int N, K, NG, NS, NB, sym, meta;   // meta: metadata bytes per (row, group)
  long long full_tile;               // bytes of a tile with kSlabGroups groups
  long long total;                   // bytes of the whole layout
  int Npad;                          // NB * kTileRows
};

__host__ __device__ inline Geom make_geom(int N, int K, int sym) {
  Geom g;
  g.N = N;
  g.K = K;
  g.NG = K / kGroup;
  g.NS = (g.NG + kSlabGroups - 1) / kSlabGroups;
  g.NB = (N + kTileRows - 1) / kTileRows;
  g.sym = sym;
  g.meta = sym ? 2 : 4;
  g.full_tile = (long long)kTileRows * kSlabGroups * (kCodeBytesPerGroupRow + g.meta);
  int last = g.NG - kSlabGroups * (g.NS - 1);
  g.total = (long long)(g.NS - 1) * g.NB * g.full_tile +
            (long long)g.NB * kTileRows * last * (kCodeBytesPerGroupRow + g.meta);
  g.Npad = g.NB * kTileRows;
  return g;
}

__host__ __device__ inline int slab_groups(const Geom& g, int s) {
  int gs = g.NG - kSlabGroups * s;
  return gs < kSlabGroups ? gs : kSlabGroups;
}

__host__ __device__ inline long long tile_bytes(const Geom& g, int gs) {
  return (long long)kTileRows * gs * (kCodeBytesPerGroupRow + g.meta);
}

__host__ __device__ inline long long tile_offset(const Geom& g, int s, int b) {
  return (long long)s * g.NB * g.full_tile + (long long)b * tile_bytes(g, slab_groups(g, s));
}

// ------------------------------------------------------------------ PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbarrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
          smem_u32(bar)),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test of the same condition.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// As mbar_try_wait, but a thread whose phase has not completed is suspended
// (it issues nothing) until the phase completes or about `hint_ns`
// nanoseconds have passed.
__device__ __forceinline__ bool mbar_try_wait_suspend(uint64_t* bar, uint32_t parity,
                                                      uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Wait until the phase with the given parity of `bar` has completed, for at
// most `limit_ns` nanoseconds.  Returns false on timeout.  The waiting
// thread sleeps in the barrier instead of spinning, so waiting warps leave
// the issue slots to the working ones.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  uint64_t limit_ns) {
  if (limit_ns < 20000u) {
    // a short limit (the timeout test hook): poll with the non-blocking
    // test_wait (try_wait may itself wait for a while), so the limit holds
    const uint64_t t0 = global_timer_ns();
    while (true) {
      if (mbar_test_wait(bar, parity)) return true;
      if (global_timer_ns() - t0 > limit_ns) return false;
    }
  }
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait_suspend(bar, parity, 20000u)) return true;
    if (global_timer_ns() - t0 > limit_ns) return false;
  }
}

// 1-D bulk copy global -> shared (no multicast), completion counted in bytes
// on `bar`.  dst, src and bytes must be multiples of 16.
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes,
                                              uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Order this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (bulk copy) accesses.
__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void named_barrier_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Programmatic dependent launch (sm_90+): wait until the previous kernel of
// the stream has completed and its memory is visible (a no-op when this grid
// was not launched as a programmatic dependent), and allow the next kernel of
// the stream to start early.
__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Host: launch `fn` so that it may start while the previous kernel of the
// stream finishes (it must call griddep_wait before touching what that
// kernel writes).
cudaError_t launch_pdl(const void* fn, dim3 grid, dim3 block, void** args, size_t smem,
                       cudaStream_t stream);

// Host: C(i, j) = beta * C(i, j) + alpha * sum_k A(i, k) B(k, j) in fp64 on
// `stream`, with A(i, k) = A[i * a_i + k * a_k], B(k, j) = B[k * b_k + j * b_j]
// and C(i, j) = C[i * ldc + j]; with lower != 0 only the 64 x 64 tiles that
// touch the lower triangle are computed; beta == 0 never reads C.  A plain
// tiled CUDA-core kernel (fp64 has no tensor-core path on this GPU's tcgen05
// instructions), used by the offline calibrated quantizers.
struct GemmF64 {
  const double* A;
  long long a_i, a_k;
  const double* B;
  long long b_k, b_j;
  double* C;
  long long ldc;
  int M, N, K;
  double alpha, beta;
  int lower;
};
cudaError_t gemm_f64(const GemmF64& p, cudaStream_t stream);

// Host: once per (device, kernel, dynamic smem size), raise the kernel's
// dynamic shared-memory limit and query how many CTAs fit on one SM.  Later
// calls only read the cache, so launches issued during stream capture make no
// attribute or occupancy calls.
cudaError_t kernel_setup(const void* fn, size_t smem, int threads, int* ctas_per_sm);

}  // namespace wq
