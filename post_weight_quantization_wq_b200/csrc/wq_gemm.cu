// wq_gemm.cu -- W4A16 skinny GEMM for M = 16..64 activation rows on the 5th-
// generation tensor cores (tcgen05, sm_100a):
//
//   y[m][n] = sum_g s16[n][g] * sum_{k in g} x[m][k] * (q[n][k] - z[n][g])
//
// At 16..64 rows the product is a dense contraction, so the dequantized
// weights go through the tensor cores ("3.6 量化(Quantization)", section
// 仅权重 vs 权重 + 激活: the 4-bit weights are dequantized to 16-bit inside the
// matmul kernel; "大模型量化全景解析", section dtype、storage dtype、compute
// dtype: 16-bit compute, higher-precision accumulation).
//
// Per group of 128 inputs, the weight tile A (128 output rows x 128 inputs)
// holds the bf16 integers 128 + q (exact), x arrives as the bf16 tile B
// (Mpad rows x 128 inputs), and the tensor core accumulates D = A B^T in fp32
// in tensor memory.  The group's exact contribution is then
//   s16 * (D - (128 + z) * sum_k x[m][k])
// added in fp32 to each row's running sum; the zero point and the 128 bias
// never enter the bf16 operands, so any stored z is handled exactly.
//
// Warp roles of one CTA (persistent, one per SM, contiguous run of layout
// tiles u = b * NS + s like the GEMV):
//   warp 0     producer: 1-D bulk copy of each code tile (codes + metadata)
//              into a 2-stage ring, and per group two 2-D TMA loads of x
//              (SWIZZLE_128B, rows >= M zero-filled) into a 4-slot ring;
//   warp 1     allocates tensor memory; one lane issues 8 tcgen05.mma
//              (M=128, N=Mpad, K=16) per group into one of two accumulator
//              buffers and commits them to mbarriers;
//   warps 2-5  dequantize: 4 LOP3 + 3 shifts turn a code word into four
//              bf16 pairs (inputs 2t, 2t+1 of the interleaved word) stored
//              into the K-major SWIZZLE_128B A tile (double-buffered);
//   warps 6-9  epilogue: one thread per output row reads the group's
//              accumulator row with tcgen05.ld, folds in s16, z and sum(x),
//              and keeps the row's running sums; row tiles split between
//              CTAs are finished through the workspace as in the GEMV.
// Every wait is bounded; on timeout the kernel records the device error word
// and winds down (waiting, bounded, for its copies and MMAs in flight).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "wq_common.cuh"

namespace wq {

struct GemmParams {
  const uint8_t* packed;
  float* y;
  float* partials;         // fp32 [NS][64][Npad]
  unsigned* counters;
  int* err;
  Geom g;
  int M;
  long long tiles;
  unsigned long long wait_ns;
  unsigned long long drain_ns;
  uint32_t lop_mask_lo, lop_bf16_128;
};

constexpr int kGemmWarps = 10;
constexpr int kGemmThreads = kGemmWarps * 32;
constexpr int kCodeStages = 2;
constexpr int kBSlots = 4;
constexpr int kGemmPartialM = 64;           // workspace row stride (max M)

template <int MPAD>
struct GemmSmem {
  static constexpr int kA = kTileRows * kGroup * 2;          // 32 KB bf16 A tile
  static constexpr int kB = MPAD * kGroup * 2;               // bf16 B tile
  static constexpr int kAOff = 0;
  static constexpr int kBOff = kAOff + 2 * kA;
  static constexpr int kTileOff = kBOff + kBSlots * kB;
  static constexpr int kTileBytes = kTileRows * kSlabGroups * (kCodeBytesPerGroupRow + 4);
  // fp32 scratch for sum(x): totals [2][MPAD], partial sums [2][8][MPAD]
  static constexpr int kXsumOff = kTileOff + kCodeStages * kTileBytes;
  static constexpr int kXsumBytes = (2 * MPAD + 2 * 8 * MPAD) * 4;
  static constexpr int kBarOff = (kXsumOff + kXsumBytes + 15) / 16 * 16;
  static constexpr int kNumBars = 2 * kCodeStages + 2 * 2 + 2 * kBSlots + 2 * 2 + 2;
  // accumulator buffers in tensor memory: column stride and allocation
  static constexpr int kAccStride = MPAD <= 32 ? MPAD : 64;
  static constexpr uint32_t kTmemCols = 2 * kAccStride <= 32 ? 32 : 2 * kAccStride <= 64 ? 64 : 128;
  static constexpr int kBytes = kBarOff + kNumBars * 8 + 16;
  static constexpr int kAlloc = kBytes + 1024;                // slack for 1024-B alignment
};

// UMMA shared-memory descriptor: K-major, SWIZZLE_128B, 8-row atoms of
// 128-byte rows (stride 1024 B), sm_100 descriptor version 1.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t smem_addr) {
  return (uint64_t)((smem_addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) |
         ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor of kind::f16: bf16 A and B, fp32 D, both K-major,
// M = 128, N = MPAD.
template <int MPAD>
__host__ __device__ constexpr uint32_t umma_idesc_bf16() {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(MPAD >> 3) << 17) |
         ((uint32_t)(128 >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, "
      "{%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ uint32_t and_or3(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ int owner_of(long long u, long long T, int G) {
  return (int)(((u + 1) * G + T - 1) / T) - 1;
}

template <int MPAD>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_w4a16_tc_kernel(const GemmParams prm, const __grid_constant__ CUtensorMap xmap) {
  using SM = GemmSmem<MPAD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const Geom g = prm.g;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kBarOff);
  uint64_t* tfull = bars;                       // [2] code tile landed
  uint64_t* tempty = tfull + kCodeStages;       // [2] code tile consumed (4 dequant warps)
  uint64_t* afull = tempty + kCodeStages;       // [2] A tile written (4 dequant warps)
  uint64_t* aempty = afull + 2;                 // [2] A tile read by the MMAs (commit)
  uint64_t* bfull = aempty + 2;                 // [4] x tile landed (TMA)
  uint64_t* bempty = bfull + kBSlots;           // [4] x tile used by MMA (commit) + epilogue
  uint64_t* accfull = bempty + kBSlots;         // [2] accumulator ready (commit)
  uint64_t* accempty = accfull + 2;             // [2] accumulator read (4 epilogue warps)
  uint64_t* xp_bar = accempty + 2;              // partial sums of x written (4 epilogue warps)
  uint64_t* xs_bar = xp_bar + 1;                // totals of x written (warps holding et < MPAD)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(xs_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* xsum = reinterpret_cast<float*>(smem + SM::kXsumOff);       // [2][MPAD]
  float* xpart = xsum + 2 * MPAD;                                    // [2][8][MPAD]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const long long t0 = (long long)blockIdx.x * prm.tiles / G;
  const long long t1 = (long long)(blockIdx.x + 1) * prm.tiles / G;
  const int ntiles = (int)(t1 - t0);
  constexpr uint32_t kTmemCols = SM::kTmemCols;
  constexpr int kXsWarps = (MPAD + 31) / 32;    // epilogue warps that total sum(x)

  if (threadIdx.x == 0) {
    for (int i = 0; i < kCodeStages; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&afull[i], 4);
      mbar_init(&aempty[i], 1);
      mbar_init(&accfull[i], 1);
      mbar_init(&accempty[i], 4);
    }
    for (int i = 0; i < kBSlots; ++i) {
      mbar_init(&bfull[i], 1);
      mbar_init(&bempty[i], 2);
    }
    mbar_init(xp_bar, 4);
    mbar_init(xs_bar, kXsWarps);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  auto fail = [&]() {
    atomicOr(prm.err, kDevErrTimeout);
    *abort_flag = 1;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int b = (int)(t0 / g.NS), s = (int)(t0 % g.NS);
      int j = 0, issued_t = 0, issued_b = 0;
      bool ok = true;
      for (int i = 0; i < ntiles && ok; ++i) {
        const int st = i % kCodeStages;
        if (i >= kCodeStages)
          ok = mbar_wait_bounded(&tempty[st], ((i / kCodeStages) - 1) & 1, prm.wait_ns);
        if (!ok || *abort_flag) { ok = false; break; }
        const int gs = slab_groups(g, s);
        const uint32_t tbytes = (uint32_t)tile_bytes(g, gs);
        mbar_arrive_expect_tx(&tfull[st], tbytes);
        bulk_copy_g2s(smem + SM::kTileOff + st * SM::kTileBytes,
                      prm.packed + tile_offset(g, s, b), tbytes, &tfull[st]);
        issued_t = i + 1;
        for (int gg = 0; gg < gs; ++gg, ++j) {
          const int bs = j % kBSlots;
          if (j >= kBSlots)
            ok = mbar_wait_bounded(&bempty[bs], ((j / kBSlots) - 1) & 1, prm.wait_ns);
          if (!ok || *abort_flag) { ok = false; break; }
          uint8_t* bdst = smem + SM::kBOff + bs * SM::kB;
          mbar_arrive_expect_tx(&bfull[bs], 2 * MPAD * 128);
          const int k0 = s * kSlabK + gg * kGroup;
          tma_load_2d(bdst, &xmap, k0, 0, &bfull[bs]);
          tma_load_2d(bdst + MPAD * 128, &xmap, k0 + 64, 0, &bfull[bs]);
          issued_b = j + 1;
        }
        if (++s == g.NS) { s = 0; ++b; }
      }
      if (!ok) {
        fail();
        for (int st = 0; st < kCodeStages && st < issued_t; ++st)
          mbar_wait_bounded(&tfull[st], ((issued_t - 1 - st) / kCodeStages) & 1, prm.drain_ns);
        for (int bs = 0; bs < kBSlots && bs < issued_b; ++bs)
          mbar_wait_bounded(&bfull[bs], ((issued_b - 1 - bs) / kBSlots) & 1, prm.drain_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int s = (int)(t0 % g.NS);
      int j = 0;
      bool ok = true;
      constexpr uint32_t idesc = umma_idesc_bf16<MPAD>();
      const uint32_t a0 = smem_u32(smem + SM::kAOff), b0 = smem_u32(smem + SM::kBOff);
      for (int i = 0; i < ntiles && ok; ++i) {
        const int gs = slab_groups(g, s);
        for (int gg = 0; gg < gs; ++gg, ++j) {
          const int ab = j & 1, bs = j % kBSlots, acc = j & 1;
          ok = mbar_wait_bounded(&afull[ab], (j >> 1) & 1, prm.wait_ns) &&
               mbar_wait_bounded(&bfull[bs], (j / kBSlots) & 1, prm.wait_ns) &&
               (j < 2 || mbar_wait_bounded(&accempty[acc], ((j >> 1) - 1) & 1, prm.wait_ns));
          if (!ok || *abort_flag) { ok = false; break; }
          tc_fence_after();
          const uint32_t abase = a0 + ab * SM::kA, bbase = b0 + bs * SM::kB;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            // K = 16 slice kk: 64-input block kk / 4, 32-byte step inside its swizzled rows
            const uint32_t koff = (kk & 3) * 32;
            const uint64_t ad = umma_desc_sw128(abase + (kk >> 2) * (kTileRows * 128) + koff);
            const uint64_t bd = umma_desc_sw128(bbase + (kk >> 2) * (MPAD * 128) + koff);
            umma_bf16(tmem_base + acc * SM::kAccStride, ad, bd, idesc, kk > 0 ? 1u : 0u);
          }
          umma_commit(&aempty[ab]);
          umma_commit(&bempty[bs]);
          umma_commit(&accfull[acc]);
        }
        if (++s == g.NS) s = 0;
      }
      if (!ok) {
        fail();
        // let the MMAs already issued finish before the accumulator is freed
        if (j > 0) mbar_wait_bounded(&accfull[(j - 1) & 1], ((j - 1) >> 1) & 1, prm.drain_ns);
      }
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ dequantize
    const int dt = threadIdx.x - 64;          // 0..127
    const uint32_t mlo = prm.lop_mask_lo, b128 = prm.lop_bf16_128;
    int s = (int)(t0 % g.NS);
    int j = 0;
    bool ok = true;
    for (int i = 0; i < ntiles && ok; ++i) {
      const int st = i % kCodeStages;
      const int gs = slab_groups(g, s);
      bool w_ok = mbar_wait_bounded(&tfull[st], (i / kCodeStages) & 1, prm.wait_ns);
      if (!__all_sync(0xFFFFFFFFu, w_ok) || *abort_flag) { ok = false; break; }
      const uint8_t* tile = smem + SM::kTileOff + st * SM::kTileBytes;
      for (int gg = 0; gg < gs; ++gg, ++j) {
        const int ab = j & 1;
        if (j >= 2) w_ok = mbar_wait_bounded(&aempty[ab], ((j >> 1) - 1) & 1, prm.wait_ns);
        if (!__all_sync(0xFFFFFFFFu, w_ok) || *abort_flag) { ok = false; break; }
        uint8_t* A = smem + SM::kAOff + ab * SM::kA;
#pragma unroll
        for (int it = 0; it < 4; ++it) {
          const int item = it * 128 + dt;     // (row, 16-byte chunk of the group's 64 B)
          const int r = item >> 2, c = item & 3;
          const uint4 cw = *reinterpret_cast<const uint4*>(
              tile + r * gs * kCodeBytesPerGroupRow + gg * kCodeBytesPerGroupRow + c * 16);
          const uint32_t wds[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            // word q of chunk c covers inputs 32c + 8q .. +8 of the group
            const uint32_t w = wds[q];
            uint4 v;
            v.x = and_or3(w, mlo, b128);          // inputs 0, 1 -> 128 + q
            v.y = and_or3(w >> 4, mlo, b128);     // inputs 2, 3
            v.z = and_or3(w >> 8, mlo, b128);     // inputs 4, 5
            v.w = and_or3(w >> 12, mlo, b128);    // inputs 6, 7
            const int kc = 4 * c + q;             // 8-input chunk 0..15 of the group
            const int kb = kc >> 3, cc = kc & 7;
            *reinterpret_cast<uint4*>(A + kb * (kTileRows * 128) + r * 128 +
                                      ((cc ^ (r & 7)) << 4)) = v;
          }
        }
        fence_proxy_async_shared();               // make the tile visible to the tensor core
        __syncwarp();
        if (lane == 0) mbar_arrive(&afull[ab]);
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[st]);
      if (++s == g.NS) s = 0;
    }
    if (!ok && lane == 0) fail();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q4 = warp & 3;                  // TMEM lane quadrant of this warp
    const int et = (warp - 6) * 32 + lane;    // 0..127 among the epilogue threads
    const int row = q4 * 32 + lane;           // row of the tile (= TMEM lane)
    constexpr int kParts = 128 / MPAD;        // xsum partial sums per activation row
    constexpr int kPartK = kGroup / kParts;
    float run[MPAD];
#pragma unroll
    for (int m = 0; m < MPAD; ++m) run[m] = 0.0f;
    int b = (int)(t0 / g.NS), s = (int)(t0 % g.NS);
    int piece_s0 = -1;
    int j = 0;
    bool ok = true;
    for (int i = 0; i < ntiles; ++i) {
      const int gs = slab_groups(g, s);
      if (piece_s0 < 0) piece_s0 = s;
      const uint8_t* meta_g = prm.packed + tile_offset(g, s, b) +
                              (long long)kTileRows * gs * kCodeBytesPerGroupRow;
      for (int gg = 0; gg < gs && ok; ++gg, ++j) {
        const int bs = j % kBSlots, acc = j & 1;
        // this row's scale and zero for the group (L2-resident: the bulk copy
        // of the tile has just read them)
        float sc, cz;
        if (g.sym) {
          sc = __half2float(__ldg(reinterpret_cast<const __half*>(meta_g) + row * gs + gg));
          cz = 136.0f;                         // 128 + 8
        } else {
          const __half2 sz = __ldg(reinterpret_cast<const __half2*>(meta_g) + row * gs + gg);
          sc = __low2float(sz);
          cz = 128.0f + __high2float(sz);
        }
        // sum_k x[m][k] over the group, from the swizzled B tile
        bool w_ok = mbar_wait_bounded(&bfull[bs], (j / kBSlots) & 1, prm.wait_ns);
        if (!__all_sync(0xFFFFFFFFu, w_ok) || *abort_flag) { ok = false; break; }
        const uint8_t* B = smem + SM::kBOff + bs * SM::kB;
        float* xp = xpart + (j & 1) * 8 * MPAD;
        float* xt = xsum + (j & 1) * MPAD;
        if (et < kParts * MPAD) {
          const int m = et % MPAD, part = et / MPAD;
          float sum = 0.0f;
#pragma unroll
          for (int kc = 0; kc < kPartK / 8; ++kc) {
            const int k = part * kPartK + kc * 8;
            const int kb = k >> 6, cc = (k & 63) >> 3;
            const uint4 v = *reinterpret_cast<const uint4*>(B + kb * (MPAD * 128) + m * 128 +
                                                            ((cc ^ (m & 7)) << 4));
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int h = 0; h < 4; ++h)
              sum += __uint_as_float(w4[h] << 16) + __uint_as_float(w4[h] & 0xFFFF0000u);
          }
          xp[part * MPAD + m] = sum;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(xp_bar);
        w_ok = mbar_wait_bounded(xp_bar, j & 1, prm.wait_ns);
        if (!__all_sync(0xFFFFFFFFu, w_ok) || *abort_flag) { ok = false; break; }
        if (et == 0) mbar_arrive(&bempty[bs]);       // B no longer needed here
        if (warp - 6 < kXsWarps) {
          if (et < MPAD) {
            float tot = 0.0f;
#pragma unroll
            for (int pp = 0; pp < kParts; ++pp) tot += xp[pp * MPAD + et];
            xt[et] = tot;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(xs_bar);
        }
        w_ok = mbar_wait_bounded(xs_bar, j & 1, prm.wait_ns);
        if (!__all_sync(0xFFFFFFFFu, w_ok) || *abort_flag) { ok = false; break; }
        // the group's accumulator row
        w_ok = mbar_wait_bounded(&accfull[acc], (j >> 1) & 1, prm.wait_ns);
        if (!__all_sync(0xFFFFFFFFu, w_ok) || *abort_flag) { ok = false; break; }
        tc_fence_after();
        // 16 columns at a time: load, wait, fold (keeps few registers live)
#pragma unroll
        for (int c = 0; c < MPAD / 16; ++c) {
          float d[16];
          tmem_ld16(tmem_base + ((uint32_t)(q4 * 32) << 16) + acc * SM::kAccStride + c * 16, d);
          tmem_wait_ld();
#pragma unroll
          for (int m = 0; m < 16; ++m)
            run[16 * c + m] = fmaf(sc, fmaf(-cz, xt[16 * c + m], d[m]), run[16 * c + m]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&accempty[acc]);
      }
      if (!ok) break;
      // ---- end of this CTA's piece of row tile b: write y or a partial
      const bool piece_end = (s == g.NS - 1) || (i == ntiles - 1);
      if (piece_end) {
        const bool whole = (piece_s0 == 0) && (s == g.NS - 1);
        const int n = b * kTileRows + row;
        if (whole) {
          if (n < g.N) {
#pragma unroll
            for (int m = 0; m < MPAD; ++m)
              if (m < prm.M) prm.y[(size_t)m * g.N + n] = run[m];
          }
        } else {
#pragma unroll
          for (int m = 0; m < MPAD; ++m)
            if (m < prm.M)
              prm.partials[((size_t)piece_s0 * kGemmPartialM + m) * g.Npad + n] = run[m];
          __threadfence();
          __syncwarp();
          const long long ub = (long long)b * g.NS;
          const int c_first = owner_of(ub, prm.tiles, G);
          const int c_last = owner_of(ub + g.NS - 1, prm.tiles, G);
          unsigned prev = 0;
          unsigned* ctr = prm.counters + (size_t)b * (kTileRows / kRowsPerCounter) + q4;
          if (lane == 0) prev = atomicAdd(ctr, 1u);
          prev = __shfl_sync(0xFFFFFFFFu, prev, 0);
          if (prev == (unsigned)(c_last - c_first)) {
            __threadfence();
            if (n < g.N)
              for (int m = 0; m < prm.M; ++m) {
                float tot = 0.0f;
                for (int c2 = c_first; c2 <= c_last; ++c2) {
                  const long long tc = (long long)c2 * prm.tiles / G;
                  const int sa = (int)((tc > ub ? tc : ub) - ub);
                  tot += __ldcg(prm.partials + ((size_t)sa * kGemmPartialM + m) * g.Npad + n);
                }
                prm.y[(size_t)m * g.N + n] = tot;
              }
            if (lane == 0) *ctr = 0u;
          }
        }
#pragma unroll
        for (int m = 0; m < MPAD; ++m) run[m] = 0.0f;
        piece_s0 = -1;
      }
      if (++s == g.NS) { s = 0; ++b; }
    }
    if (!ok && lane == 0) fail();
  }

  // All roles meet here; then the allocating warp frees tensor memory.
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(kTmemCols)
                 : "memory");
  }
}

// ------------------------------------------------------------------ launcher

size_t gemm_workspace_bytes(int M, int N, int K) {
  (void)M;
  const Geom g = make_geom(N, K, 1);
  if (g.NS <= 1) return 0;
  return (size_t)kCounterBytes + (size_t)g.NS * kGemmPartialM * g.Npad * sizeof(float);
}

static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

template <int MPAD>
static cudaError_t launch_gemm_t(const GemmParams& prm, const void* x, int num_sms,
                                 cudaStream_t stream) {
  using SM = GemmSmem<MPAD>;
  auto enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  // x: bf16 [M][K]; box of 64 inputs x MPAD rows, 128-byte swizzle, rows >= M
  // (and any coordinate past the tensor) read as zero.
  CUtensorMap map;
  cuuint64_t dims[2] = {(cuuint64_t)prm.g.K, (cuuint64_t)prm.M};
  cuuint64_t strides[1] = {(cuuint64_t)prm.g.K * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)MPAD};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  const void* fn = reinterpret_cast<const void*>(&gemm_w4a16_tc_kernel<MPAD>);
  int per_sm = 0;
  cudaError_t e = kernel_setup(fn, SM::kAlloc, kGemmThreads, &per_sm);
  if (e != cudaSuccess) return e;
  long long grid = (long long)num_sms * per_sm;
  if (grid > prm.tiles) grid = prm.tiles;
  GemmParams p = prm;
  void* args[] = {&p, &map};
  return cudaLaunchKernel(fn, dim3((unsigned)grid), dim3(kGemmThreads), args, SM::kAlloc, stream);
}

cudaError_t launch_gemm(const void* x, const void* packed, int M, int N, int K, int sym,
                        float* y, void* workspace, int* err, int num_sms,
                        unsigned long long wait_ns, cudaStream_t stream) {
  GemmParams prm;
  prm.g = make_geom(N, K, sym);
  prm.packed = static_cast<const uint8_t*>(packed);
  prm.y = y;
  prm.counters = static_cast<unsigned*>(workspace);
  prm.partials = workspace ? reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kCounterBytes)
                           : nullptr;
  prm.err = err;
  prm.M = M;
  prm.tiles = (long long)prm.g.NS * prm.g.NB;
  prm.wait_ns = wait_ns;
  prm.drain_ns = 1000000000ull;
  prm.lop_mask_lo = 0x000F000Fu;
  prm.lop_bf16_128 = 0x43004300u;
  const int mpad = (M + 15) / 16 * 16;
  switch (mpad) {
    case 16: return launch_gemm_t<16>(prm, x, num_sms, stream);
    case 32: return launch_gemm_t<32>(prm, x, num_sms, stream);
    case 48: return launch_gemm_t<48>(prm, x, num_sms, stream);
    default: return launch_gemm_t<64>(prm, x, num_sms, stream);
  }
}

}  // namespace wq
