// wq_gemm.cu -- W4A16 skinny GEMM for M = 1..64 activation rows on the 5th-
// generation tensor cores (tcgen05, sm_100a):
//
//   y[m][n] = sum_g s16[n][g] * sum_{k in g} x[m][k] * (q[n][k] - z[n][g])
//
// With several rows of x the product is a dense contraction, so the
// dequantized weights go through the tensor cores ("3.6 量化(Quantization)",
// section 仅权重 vs 权重 + 激活: the 4-bit weights are dequantized to 16-bit
// inside the matmul kernel; "大模型量化全景解析", section dtype、storage dtype、
// compute dtype: 16-bit compute, higher-precision accumulation).  x is
// zero-padded by its tensor map to Mpad = 16, 32, 48 or 64 rows.
//
// Per group of 128 inputs, the weight tile A (128 output rows x 128 inputs)
// holds the bf16 integers 128 + q (exact), x arrives as the bf16 tile B
// (Mpad rows x 128 inputs), and the tensor core accumulates D = A B^T in fp32
// in tensor memory.  The group's exact contribution is then
//   s16 * (D - (128 + z) * sum_k x[m][k])
// added in fp32 to each row's running sum; the zero point and the 128 bias
// never enter the bf16 operands, so any stored z is handled exactly.
//
// Data flow of one CTA (persistent, one per SM, contiguous run of layout
// tiles u = b * NS + s like the GEMV).  The roles hand work to each other in
// stages of two consecutive groups of the CTA's group sequence (one mbarrier
// handoff per 256 inputs); per group:
//   codes   2-D TMA load of the group's 128 rows x 64 B of codes out of the
//           packed tile (SWIZZLE_64B, so that a warp reading 32 rows at one
//           column offset touches every bank once) into a ring of 6..8
//           stages; the tile's metadata by one bulk copy per tile;
//   A       the dequantizing warps turn each row's 16 code words into 64
//           bf16 pairs and store them into tensor memory (tcgen05.st): the
//           A operand never passes through shared memory;
//   x       2-D TMA loads of the bf16 activation tile (SWIZZLE_128B, rows >= M
//           zero-filled), and a bulk copy of the group's precomputed sum(x)
//           row;
//   MMA     one lane issues 8 tcgen05.mma (M=128, N=Mpad, K=16, A in tensor
//           memory, B in shared memory) into one of 4 accumulators;
//   fold    one thread per output row reads its accumulator row (tcgen05.ld)
//           and adds s16 * (D - (128 + z) * sum(x)) to the row's running sums;
//           row tiles split between CTAs are finished through the workspace
//           as in the GEMV.
// Warps: 0 code producer, 1 tensor-memory owner and MMA issuer, 2
// activation producer, 4-11 dequantize (inputs 0-63 and 64-127 of each
// group, one warp per lane quadrant), 12-19 fold (columns 0..Mpad/2-1 and
// Mpad/2..Mpad-1 of the accumulator, one warp per lane quadrant).  Every
// wait is bounded; on timeout the kernel records the device error word and
// winds down (waiting, bounded, for its copies and MMAs in flight).
#include <cuda.h>
#include <cstring>
#include <cudaTypedefs.h>

#include "wq_common.cuh"
#include "wq_tc.cuh"

namespace wq {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
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

struct GemmParams {
  const uint8_t* packed;
  const float* xsum;       // fp32 [NG][64]: sum of x over each group, per row of x
  float* y;
  float* partials;         // fp32 [NS][Mpad][Npad]
  unsigned* counters;
  int* err;
  Geom g;
  int M;
  int ns_full;             // slabs with kSlabGroups groups
  int tile_rows;           // 256-byte (full slab) or gs*64-byte rows per tile
  long long tiles;
  unsigned long long wait_ns;
  unsigned long long drain_ns;
  uint32_t lop_mask_lo, lop_bf16_128;
};

constexpr int kGemmWarps = 20;
constexpr int kGemmThreads = kGemmWarps * 32;
constexpr int kDqWarps = 8;
constexpr int kEpiWarps = 8;
// The pipeline moves stages of kGps consecutive groups (of this CTA's group
// sequence): one barrier handoff per stage between the roles.  Group j lives
// in buffer j % 4 (A operand, accumulator, x tile); stage q = j / 2 uses the
// barrier pair q % 2.
constexpr int kGps = 2;                     // groups per stage
constexpr int kPipe = 2;                    // stages in flight between roles
constexpr int kABufs = kGps * kPipe;        // A operands in tensor memory (4)
constexpr int kAccBufs = kABufs;            // accumulators in tensor memory
constexpr int kBSlots = kABufs;             // bf16 x tiles
constexpr int kXsStages = 4;                // stage slots of sum(x) rows
constexpr int kXsSlots = kXsStages * kGps;  // sum(x) rows
constexpr int kMetaSlots = 8;               // per-tile scales (and zeros)
constexpr int kMetaSlotBytes = kTileRows * kSlabGroups * 4;   // 2 KB
constexpr int kXsumRow = 64;                // floats per group in the sum(x) table
constexpr int kCodeGroupBytes = kTileRows * kCodeBytesPerGroupRow;   // 8 KB
constexpr uint32_t kTmemCols = 512;

template <int MPAD>
struct GemmSmem {
  static constexpr int kCodeStages = MPAD <= 32 ? 8 : 6;      // stage slots of codes
  static constexpr int kCodeSlots = kCodeStages * kGps;
  static constexpr int kB = MPAD * kGroup * 2;                // bf16 x tile
  static constexpr int kBOff = 0;
  static constexpr int kCodeOff = kBOff + kBSlots * kB;
  static constexpr int kXsOff = kCodeOff + kCodeSlots * kCodeGroupBytes;
  static constexpr int kXs = kXsumRow * 4;                     // one sum(x) row
  static constexpr int kMetaOff = kXsOff + kXsSlots * kXs;
  static constexpr int kBarOff = kMetaOff + kMetaSlots * kMetaSlotBytes;
  static constexpr int kNumBars = 2 * kCodeStages + 6 * kPipe + 2 * kXsStages + 2 * kMetaSlots;
  static constexpr int kBytes = kBarOff + kNumBars * 8 + 16;
  static constexpr int kAlloc = kBytes + 1024;                // slack for 1024-B alignment
  // tensor memory columns: A buffers (64 columns = 128 bf16 each), then
  // the accumulators
  static constexpr int kAccStride = MPAD <= 32 ? 32 : 64;
  static constexpr int kAccCol = kABufs * 64;
  static_assert(kAccCol + kAccBufs * kAccStride <= (int)kTmemCols, "tensor memory");
};

// Instruction descriptor of kind::f16: bf16 A and B, fp32 D, both K-major,
// M = 128, N = MPAD.
template <int MPAD>
__host__ __device__ constexpr uint32_t umma_idesc_bf16() {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(MPAD >> 3) << 17) |
         ((uint32_t)(128 >> 4) << 24);
}

// D (tensor memory) (+)= A (tensor memory, 128 rows x 16 bf16, two per
// column) * B (shared memory descriptor)^T
__device__ __forceinline__ void umma_bf16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate));
}


__device__ __forceinline__ int owner_of(long long u, long long T, int G) {
  return (int)(((u + 1) * G + T - 1) / T) - 1;
}

// Walks the groups of this CTA's run of tiles in order: group j is group gg
// of slab s of row tile b.
struct GroupCursor {
  int b, s, gg, gs;
  __device__ void init(const Geom& g, long long t0) {
    b = (int)(t0 / g.NS);
    s = (int)(t0 % g.NS);
    gg = 0;
    gs = slab_groups(g, s);
  }
  // returns true when the step crossed into the next tile
  __device__ bool next(const Geom& g) {
    if (++gg < gs) return false;
    gg = 0;
    if (++s == g.NS) { s = 0; ++b; }
    gs = slab_groups(g, s);
    return true;
  }
};

template <int MPAD>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_w4a16_tc_kernel(const GemmParams prm, const __grid_constant__ CUtensorMap xmap,
                         const __grid_constant__ CUtensorMap cmap_full,
                         const __grid_constant__ CUtensorMap cmap_tail) {
  using SM = GemmSmem<MPAD>;
  constexpr int NCS = SM::kCodeStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const Geom g = prm.g;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kBarOff);
  uint64_t* cfull = bars;                       // [NCS] codes of a stage landed (TMA)
  uint64_t* cempty = cfull + NCS;               // [NCS] codes read (8 dequant warps)
  uint64_t* afull = cempty + NCS;               // [2] A operands stored (8 dequant warps)
  uint64_t* aempty = afull + kPipe;             // [2] A operands read by the MMAs (commit)
  uint64_t* bfull = aempty + kPipe;             // [2] x tiles landed (TMA)
  uint64_t* bempty = bfull + kPipe;             // [2] x tiles read by the MMAs (commit)
  uint64_t* accfull = bempty + kPipe;           // [2] accumulators ready (commit)
  uint64_t* accempty = accfull + kPipe;         // [2] accumulators read (8 fold warps)
  uint64_t* xsfull = accempty + kPipe;          // [4] sum(x) rows landed
  uint64_t* xsempty = xsfull + kXsStages;       // [4] sum(x) rows read (8 fold warps)
  uint64_t* mfull = xsempty + kXsStages;        // [8] metadata of a tile landed
  uint64_t* mempty = mfull + kMetaSlots;        // [8] metadata read (8 fold warps)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mempty + kMetaSlots);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const long long t0 = (long long)blockIdx.x * prm.tiles / G;
  const long long t1 = (long long)(blockIdx.x + 1) * prm.tiles / G;
  // groups of this CTA's run of tiles, and stages of kGps of them
  int ngroups = 0;
  for (long long u = t0; u < t1; ++u) ngroups += slab_groups(g, (int)(u % g.NS));
  const int nstages = (ngroups + kGps - 1) / kGps;
  auto stage_groups = [&](int q) { return ngroups - kGps * q < kGps ? ngroups - kGps * q : kGps; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < NCS; ++i) {
      mbar_init(&cfull[i], 1);
      mbar_init(&cempty[i], kDqWarps);
    }
    for (int i = 0; i < kPipe; ++i) {
      mbar_init(&afull[i], kDqWarps);
      mbar_init(&aempty[i], 1);
      mbar_init(&bfull[i], 1);
      mbar_init(&bempty[i], 1);
      mbar_init(&accfull[i], 1);
      mbar_init(&accempty[i], kEpiWarps);
    }
    for (int i = 0; i < kXsStages; ++i) {
      mbar_init(&xsfull[i], 1);
      mbar_init(&xsempty[i], kEpiWarps);
    }
    for (int i = 0; i < kMetaSlots; ++i) {
      mbar_init(&mfull[i], 1);
      mbar_init(&mempty[i], kEpiWarps);
    }
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

  // The producer and MMA warps run their loops with all 32 lanes (so loop
  // state stays warp-uniform) and let one elected lane issue each copy or
  // MMA.
  if (warp == 0) {
    // ------------------------------------------------------------ code producer
    GroupCursor c;
    c.init(g, t0);
    int issued = 0, tile = 0, issued_m = 0;
    bool ok = true;
    for (int q = 0; q < nstages && ok; ++q) {
      const int cnt = stage_groups(q);
      const int cs = q % NCS;
      if (q >= NCS) ok = warp_wait(&cempty[cs], ((q / NCS) - 1) & 1, prm.wait_ns);
      if (!ok || *abort_flag) { ok = false; break; }
      if (elect_one()) mbar_arrive_expect_tx(&cfull[cs], cnt * kCodeGroupBytes);
      __syncwarp();
      for (int sub = 0; sub < cnt; ++sub, c.next(g)) {
        if (c.gg == 0) {
          // the tile's metadata block (128 rows x gs groups) into a meta slot
          const int ms = tile % kMetaSlots;
          if (tile >= kMetaSlots)
            ok = warp_wait(&mempty[ms], ((tile / kMetaSlots) - 1) & 1, prm.wait_ns);
          if (!ok || *abort_flag) { ok = false; break; }
          if (elect_one()) {
            const uint32_t mbytes = (uint32_t)(kTileRows * c.gs * g.meta);
            mbar_arrive_expect_tx(&mfull[ms], mbytes);
            bulk_copy_g2s(smem + SM::kMetaOff + ms * kMetaSlotBytes,
                          prm.packed + tile_offset(g, c.s, c.b) +
                              (long long)kTileRows * c.gs * kCodeBytesPerGroupRow,
                          mbytes, &mfull[ms]);
          }
          __syncwarp();
          issued_m = ++tile;
        }
        if (elect_one()) {
          uint8_t* dst = smem + SM::kCodeOff + (cs * kGps + sub) * kCodeGroupBytes;
          if (c.s < prm.ns_full)
            tma_load_2d(dst, &cmap_full, c.gg * kCodeBytesPerGroupRow,
                        (c.s * g.NB + c.b) * prm.tile_rows, &cfull[cs]);
          else
            tma_load_2d(dst, &cmap_tail, c.gg * kCodeBytesPerGroupRow, c.b * prm.tile_rows,
                        &cfull[cs]);
        }
        __syncwarp();
      }
      issued = q + 1;
    }
    if (!ok) {
      if (lane == 0) fail();
      // a stage whose expect_tx was posted but not all its copies issued
      // never completes; the bounded waits just run out for it
      for (int k = issued - NCS < 0 ? 0 : issued - NCS; k < issued; ++k)
        warp_wait(&cfull[k % NCS], (k / NCS) & 1, prm.drain_ns);
      for (int k = issued_m - kMetaSlots < 0 ? 0 : issued_m - kMetaSlots; k < issued_m; ++k)
        warp_wait(&mfull[k % kMetaSlots], (k / kMetaSlots) & 1, prm.drain_ns);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ activation producer
    GroupCursor c;
    c.init(g, t0);
    int issued_b = 0, issued_x = 0;
    bool ok = true;
    for (int q = 0; q < nstages; ++q) {
      const int cnt = stage_groups(q);
      const int ps = q % kPipe, xq = q % kXsStages;
      if (q >= kPipe) ok = warp_wait(&bempty[ps], ((q / kPipe) - 1) & 1, prm.wait_ns);
      if (ok && q >= kXsStages)
        ok = warp_wait(&xsempty[xq], ((q / kXsStages) - 1) & 1, prm.wait_ns);
      if (!ok || *abort_flag) { ok = false; break; }
      if (elect_one()) {
        mbar_arrive_expect_tx(&bfull[ps], cnt * 2 * MPAD * 128);
        mbar_arrive_expect_tx(&xsfull[xq], cnt * MPAD * 4);
        GroupCursor cc = c;
        for (int sub = 0; sub < cnt; ++sub, cc.next(g)) {
          const int j = kGps * q + sub;
          const int k0 = cc.s * kSlabK + cc.gg * kGroup;
          uint8_t* bdst = smem + SM::kBOff + (j % kBSlots) * SM::kB;
          tma_load_2d(bdst, &xmap, k0, 0, &bfull[ps]);
          tma_load_2d(bdst + MPAD * 128, &xmap, k0 + 64, 0, &bfull[ps]);
          bulk_copy_g2s(smem + SM::kXsOff + (xq * kGps + sub) * SM::kXs,
                        prm.xsum + (size_t)(cc.s * kSlabGroups + cc.gg) * kXsumRow, MPAD * 4,
                        &xsfull[xq]);
        }
      }
      __syncwarp();
      for (int sub = 0; sub < cnt; ++sub) c.next(g);
      issued_b = issued_x = q + 1;
    }
    if (!ok) {
      if (lane == 0) fail();
      for (int k = issued_b - kPipe < 0 ? 0 : issued_b - kPipe; k < issued_b; ++k)
        warp_wait(&bfull[k % kPipe], (k / kPipe) & 1, prm.drain_ns);
      for (int k = issued_x - kXsStages < 0 ? 0 : issued_x - kXsStages; k < issued_x; ++k)
        warp_wait(&xsfull[k % kXsStages], (k / kXsStages) & 1, prm.drain_ns);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    int q = 0;
    bool ok = true;
    constexpr uint32_t idesc = umma_idesc_bf16<MPAD>();
    const uint32_t b0 = smem_u32(smem + SM::kBOff);
    for (; q < nstages; ++q) {
      const int ps = q % kPipe;
      ok = warp_wait(&afull[ps], (q / kPipe) & 1, prm.wait_ns) &&
           warp_wait(&bfull[ps], (q / kPipe) & 1, prm.wait_ns) &&
           (q < kPipe || warp_wait(&accempty[ps], ((q / kPipe) - 1) & 1, prm.wait_ns));
      if (!ok || *abort_flag) { ok = false; break; }
      tc_fence_after();
      const int cnt = stage_groups(q);
      if (elect_one()) {
        for (int sub = 0; sub < cnt; ++sub) {
          const int bj = (kGps * q + sub) % kABufs;
          const uint32_t bbase = b0 + bj * SM::kB;
          const uint32_t ta = tmem_base + bj * 64;
          const uint32_t td = tmem_base + SM::kAccCol + bj * SM::kAccStride;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            // K = 16 slice kk: 8 columns of A; in B, 64-input block kk / 4 and
            // a 32-byte step inside its swizzled rows
            const uint64_t bd = umma_desc_sw128(bbase + (kk >> 2) * (MPAD * 128) + (kk & 3) * 32);
            umma_bf16_ts(td, ta + kk * 8, bd, idesc, kk > 0 ? 1u : 0u);
          }
        }
        umma_commit(&aempty[ps]);
        umma_commit(&bempty[ps]);
        umma_commit(&accfull[ps]);
      }
      __syncwarp();
    }
    if (!ok) {
      if (lane == 0) fail();
      // let the MMAs already issued finish before tensor memory is freed
      if (q > 0) warp_wait(&accfull[(q - 1) % kPipe], ((q - 1) / kPipe) & 1, prm.drain_ns);
    }
  } else if (warp >= 4 && warp < 4 + kDqWarps) {
    // ------------------------------------------------------------ dequantize
    const int quad = warp & 3;                // TMEM lane quadrant of this warp
    const int h = (warp - 4) >> 2;            // inputs 64h .. 64h+63 of each group
    const int r = quad * 32 + lane;           // row of the tile (= TMEM lane)
    const uint32_t mlo = prm.lop_mask_lo, b128 = prm.lop_bf16_128;
    const uint32_t lane_base = tmem_base + ((uint32_t)(quad * 32) << 16) + h * 32;
    // byte offsets of this row's two 16-byte chunks 2h, 2h+1 in a code slot
    // (64-byte swizzle: chunk index ^= address bits 7..8)
    const int sw = (r >> 1) & 3;
    const int off0 = r * 64 + (((2 * h) ^ sw) << 4);
    const int off1 = r * 64 + (((2 * h + 1) ^ sw) << 4);
    bool ok = true;
    for (int q = 0; q < nstages; ++q) {
      const int cs = q % NCS, ps = q % kPipe;
      bool w_ok = mbar_wait_bounded(&cfull[cs], (q / NCS) & 1, prm.wait_ns);
      if (w_ok && q >= kPipe)
        w_ok = mbar_wait_bounded(&aempty[ps], ((q / kPipe) - 1) & 1, prm.wait_ns);
      if (!__all_sync(0xFFFFFFFFu, w_ok) || *abort_flag) { ok = false; break; }
      tc_fence_after();
      const int cnt = stage_groups(q);
      for (int sub = 0; sub < cnt; ++sub) {
        const int bj = (kGps * q + sub) % kABufs;
        const uint8_t* slot = smem + SM::kCodeOff + (cs * kGps + sub) * kCodeGroupBytes;
        const uint4 c0 = *reinterpret_cast<const uint4*>(slot + off0);
        const uint4 c1 = *reinterpret_cast<const uint4*>(slot + off1);
        const uint32_t wds[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t v[16];
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {
            // word covers 8 inputs; slot t of the interleaved word holds input
            // 2t (t < 4) or 2(t-4)+1, so each LOP3 yields one bf16 pair
            // (128 + q_even, 128 + q_odd)
            const uint32_t w = wds[4 * half + qq];
            v[4 * qq + 0] = and_or3(w, mlo, b128);
            v[4 * qq + 1] = and_or3(w >> 4, mlo, b128);
            v[4 * qq + 2] = and_or3(w >> 8, mlo, b128);
            v[4 * qq + 3] = and_or3(w >> 12, mlo, b128);
          }
          tmem_st16(lane_base + bj * 64 + half * 16, v);
        }
      }
      __syncwarp();                           // every lane's codes are in registers
      if (lane == 0) mbar_arrive(&cempty[cs]);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[ps]);
    }
    if (!ok && lane == 0) fail();
  } else if (warp >= 12) {
    // ------------------------------------------------------------ fold
    constexpr int EC = MPAD / 2;              // accumulator columns of this thread
    const int q4 = warp & 3;                  // TMEM lane quadrant of this warp
    const int half = (warp - 12) >> 2;        // columns half*EC .. half*EC+EC-1
    const int m0 = half * EC;
    const int row = q4 * 32 + lane;           // row of the tile (= TMEM lane)
    float2 run[EC / 2];                       // running sums, columns in pairs
#pragma unroll
    for (int m = 0; m < EC / 2; ++m) run[m] = make_float2(0.0f, 0.0f);
    GroupCursor c;
    c.init(g, t0);
    int piece_s0 = -1;
    bool ok = true;
    float scs[kSlabGroups], czs[kSlabGroups];   // this row's (scale, 128 + zero) per group
    int tile = 0;
    for (int q = 0; q < nstages && ok; ++q) {
      const int ps = q % kPipe, xq = q % kXsStages;
      bool w_ok = mbar_wait_bounded(&xsfull[xq], (q / kXsStages) & 1, prm.wait_ns) &&
                  mbar_wait_bounded(&accfull[ps], (q / kPipe) & 1, prm.wait_ns);
      if (!__all_sync(0xFFFFFFFFu, w_ok) || *abort_flag) { ok = false; break; }
      tc_fence_after();
      const int cnt = stage_groups(q);
      for (int sub = 0; sub < cnt; ++sub) {
        const int j = kGps * q + sub;
        if (piece_s0 < 0) piece_s0 = c.s;
        if (c.gg == 0) {
          // the tile's scales (and zeros) for this row, then release the slot
          const int ms = tile % kMetaSlots;
          const bool m_ok = mbar_wait_bounded(&mfull[ms], (tile / kMetaSlots) & 1, prm.wait_ns);
          if (!__all_sync(0xFFFFFFFFu, m_ok) || *abort_flag) { ok = false; break; }
          const uint8_t* mb = smem + SM::kMetaOff + ms * kMetaSlotBytes;
#pragma unroll
          for (int qq = 0; qq < kSlabGroups; ++qq) {
            if (qq < c.gs) {
              if (g.sym) {
                scs[qq] = __half2float(reinterpret_cast<const __half*>(mb)[row * c.gs + qq]);
                czs[qq] = 136.0f;              // 128 + 8
              } else {
                const __half2 sz = reinterpret_cast<const __half2*>(mb)[row * c.gs + qq];
                scs[qq] = __low2float(sz);
                czs[qq] = 128.0f + __high2float(sz);
              }
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&mempty[ms]);
          ++tile;
        }
        float sc = scs[0], cz = czs[0];
#pragma unroll
        for (int qq = 1; qq < kSlabGroups; ++qq)
          if (c.gg == qq) { sc = scs[qq]; cz = czs[qq]; }
        GroupCursor nc = c;
        const bool tile_end = nc.next(g);
        const float* xt =
            reinterpret_cast<const float*>(smem + SM::kXsOff + (xq * kGps + sub) * SM::kXs) + m0;
        const uint32_t tacc = tmem_base + ((uint32_t)(q4 * 32) << 16) + SM::kAccCol +
                              (j % kAccBufs) * SM::kAccStride + m0;
        // batches of up to 16 columns: load, wait, fold (bounds live registers)
#pragma unroll
        for (int b0 = 0; b0 < EC; b0 += 16) {
          constexpr int kMaxB = EC < 16 ? EC : 16;
          float d[kMaxB];
#pragma unroll
          for (int cc = 0; cc < kMaxB / 8; ++cc)
            if (b0 + cc * 8 < EC) tmem_ld8(tacc + b0 + cc * 8, d + cc * 8);
          tmem_wait_ld();
          // run += s16 * (D - (128 + z) * sum(x)), two columns per FFMA2
          const float2 s2 = make_float2(sc, sc), ncz2 = make_float2(-cz, -cz);
#pragma unroll
          for (int m = 0; m < kMaxB; m += 4)
            if (b0 + m < EC) {
              const float4 x4 = *reinterpret_cast<const float4*>(xt + b0 + m);
              const float2 t0v =
                  __ffma2_rn(ncz2, make_float2(x4.x, x4.y), make_float2(d[m], d[m + 1]));
              const float2 t1v =
                  __ffma2_rn(ncz2, make_float2(x4.z, x4.w), make_float2(d[m + 2], d[m + 3]));
              run[(b0 + m) / 2] = __ffma2_rn(s2, t0v, run[(b0 + m) / 2]);
              run[(b0 + m) / 2 + 1] = __ffma2_rn(s2, t1v, run[(b0 + m) / 2 + 1]);
            }
        }
        if (!tile_end) { c = nc; continue; }
        // ---- last group of a tile: end of this CTA's piece of row tile b?
        const bool piece_end = (c.s == g.NS - 1) || (j == ngroups - 1);
        if (piece_end) {
          const int b = c.b;
          const bool whole = (piece_s0 == 0) && (c.s == g.NS - 1);
          const int n = b * kTileRows + row;
          if (whole) {
            if (n < g.N) {
#pragma unroll
              for (int m = 0; m < EC; ++m)
                if (m0 + m < prm.M)
                  prm.y[(size_t)(m0 + m) * g.N + n] = (m & 1) ? run[m / 2].y : run[m / 2].x;
            }
          } else {
#pragma unroll
            for (int m = 0; m < EC; ++m)
              if (m0 + m < prm.M)
                prm.partials[((size_t)piece_s0 * MPAD + m0 + m) * g.Npad + n] =
                    (m & 1) ? run[m / 2].y : run[m / 2].x;
            __threadfence();
            __syncwarp();
            const long long ub = (long long)b * g.NS;
            const int c_first = owner_of(ub, prm.tiles, G);
            const int c_last = owner_of(ub + g.NS - 1, prm.tiles, G);
            unsigned prev = 0;
            unsigned* ctr =
                prm.counters + (size_t)b * (kTileRows / kRowsPerCounter) + q4 + 4 * half;
            if (lane == 0) prev = atomicAdd(ctr, 1u);
            prev = __shfl_sync(0xFFFFFFFFu, prev, 0);
            if (prev == (unsigned)(c_last - c_first)) {
              __threadfence();
              const int m_end = prm.M < m0 + EC ? prm.M : m0 + EC;
              if (n < g.N) {
                // pieces in slab order; the loads of one piece for up to 16
                // rows of x are independent and go out together
                constexpr int kRB = EC < 16 ? EC : 16;
                for (int mb = m0; mb < m_end; mb += kRB) {
                  float tot[kRB];
#pragma unroll
                  for (int m = 0; m < kRB; ++m) tot[m] = 0.0f;
                  for (int c2 = c_first; c2 <= c_last; ++c2) {
                    const long long tc = (long long)c2 * prm.tiles / G;
                    const int sa = (int)((tc > ub ? tc : ub) - ub);
                    const float* src = prm.partials + ((size_t)sa * MPAD + mb) * g.Npad + n;
#pragma unroll
                    for (int m = 0; m < kRB; ++m)
                      if (mb + m < m_end) tot[m] += __ldcg(src + (size_t)m * g.Npad);
                  }
#pragma unroll
                  for (int m = 0; m < kRB; ++m)
                    if (mb + m < m_end) prm.y[(size_t)(mb + m) * g.N + n] = tot[m];
                }
              }
              if (lane == 0) *ctr = 0u;
            }
          }
#pragma unroll
          for (int m = 0; m < EC / 2; ++m) run[m] = make_float2(0.0f, 0.0f);
          piece_s0 = -1;
        }
        c = nc;
      }
      if (!ok) break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&accempty[ps]);
        mbar_arrive(&xsempty[xq]);
      }
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

// sum_{k in g} x[m][k] for every group g and row m of x, in fp32 (fixed
// order); rows m >= M are 0.  One warp per group, lane = row of x.
__global__ void __launch_bounds__(256) gemm_xsum_kernel(const uint16_t* __restrict__ x, int M,
                                                        int K, float* __restrict__ xsum) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int NG = K / kGroup;
  if (warp >= NG) return;
  for (int m = lane; m < kXsumRow; m += 32) {
    float acc = 0.0f;
    if (m < M) {
      const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)m * K + warp * kGroup);
#pragma unroll 4
      for (int c = 0; c < kGroup / 8; ++c) {
        const uint4 v = __ldg(src + c);
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int h = 0; h < 4; ++h)
          acc += __uint_as_float(w4[h] << 16) + __uint_as_float(w4[h] & 0xFFFF0000u);
      }
    }
    xsum[(size_t)warp * kXsumRow + m] = acc;
  }
}

// ------------------------------------------------------------------ launcher

static int gemm_mpad(int M) { return (M + 15) / 16 * 16; }

// split-K partial sums: fp32 [NS][Mpad][Npad]
static size_t gemm_partials_bytes(const Geom& g, int M) {
  return g.NS <= 1 ? 0 : (size_t)g.NS * gemm_mpad(M) * g.Npad * sizeof(float);
}

size_t gemm_fold_workspace_bytes(int M, int N, int K);
cudaError_t launch_gemm_fold(const void* x, const void* packed, int M, int N, int K, int sym,
                             float* y, void* workspace, int* err, unsigned long long wait_ns,
                             cudaStream_t stream);

// Test hook: run the many-row (fold) kernel for every M, so it can be
// compared with the skinny kernel on the same shapes.
static int g_force_fold = 0;
void gemm_force_fold(int on) { g_force_fold = on; }

static bool use_fold(int M) { return M > 64 || g_force_fold; }

bool gemm_tc_supported(int M, int K);
bool gemv_forced_cuda_cores();
size_t gemv_tc_workspace_bytes(int M, int N, int K);
cudaError_t launch_gemv_tc(const void* x, const float* inv_s, const void* packed, int M, int N,
                           int K, int sym, float* y, void* workspace, int* err, int num_sms,
                           unsigned long long wait_ns, cudaStream_t stream);

// M <= 16 with every slab full goes to the int8 tensor-core decode kernel
// (unless a test hook forces the bf16 kernels).
static bool use_int8(int M, int K) {
  return !g_force_fold && !gemv_forced_cuda_cores() && gemm_tc_supported(M, K);
}

// Large enough for every kernel the shape may take (the test hooks switch
// kernels at run time).
size_t gemm_workspace_bytes(int M, int N, int K) {
  if (M > 64) return gemm_fold_workspace_bytes(M, N, K);
  const size_t fold = gemm_fold_workspace_bytes(M, N, K);
  const Geom g = make_geom(N, K, 1);
  const size_t skinny = (size_t)kCounterBytes + gemm_partials_bytes(g, M) +
                        (size_t)g.NG * kXsumRow * sizeof(float);
  size_t need = skinny > fold ? skinny : fold;
  if (gemm_tc_supported(M, K)) {
    const size_t tc = gemv_tc_workspace_bytes(M, N, K);
    if (tc > need) need = tc;
  }
  return need;
}

template <int MPAD>
static cudaError_t launch_gemm_t(const GemmParams& prm, const void* x, int num_sms,
                                 cudaStream_t stream) {
  using SM = GemmSmem<MPAD>;
  auto enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const Geom& g = prm.g;
  // x: bf16 [M][K]; box of 64 inputs x MPAD rows, 128-byte swizzle, rows >= M
  // (and any coordinate past the tensor) read as zero.
  CUtensorMap xmap;
  {
    cuuint64_t dims[2] = {(cuuint64_t)g.K, (cuuint64_t)prm.M};
    cuuint64_t strides[1] = {(cuuint64_t)g.K * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)MPAD};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  }
  // Codes: a tile is tile_rows rows of gs * 64 bytes (128 rows of codes,
  // then the metadata), so the tiles of the full slabs form one 2-D byte
  // array of 256-byte rows and the tiles of a partial last slab another.
  // Box: one group (64 bytes) x 128 rows, 64-byte swizzle.
  CUtensorMap cfull, ctail;
  memset(&cfull, 0, sizeof(cfull));
  memset(&ctail, 0, sizeof(ctail));
  auto encode_codes = [&](CUtensorMap* m, const uint8_t* base, int row_bytes,
                          long long rows) -> bool {
    cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    cuuint32_t box[2] = {(cuuint32_t)kCodeBytesPerGroupRow, (cuuint32_t)kTileRows};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  };
  if (prm.ns_full > 0 &&
      !encode_codes(&cfull, prm.packed, kSlabGroups * kCodeBytesPerGroupRow,
                    (long long)prm.ns_full * g.NB * prm.tile_rows))
    return cudaErrorInvalidValue;
  if (prm.ns_full < g.NS) {
    const int gs = slab_groups(g, g.NS - 1);
    if (!encode_codes(&ctail, prm.packed + tile_offset(g, g.NS - 1, 0),
                      gs * kCodeBytesPerGroupRow, (long long)g.NB * prm.tile_rows))
      return cudaErrorInvalidValue;
  }
  const void* fn = reinterpret_cast<const void*>(&gemm_w4a16_tc_kernel<MPAD>);
  int per_sm = 0;
  cudaError_t e = kernel_setup(fn, SM::kAlloc, kGemmThreads, &per_sm);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  long long grid = (long long)num_sms;        // one CTA per SM (all of tensor memory)
  if (grid > prm.tiles) grid = prm.tiles;
  GemmParams p = prm;
  void* args[] = {&p, &xmap, &cfull, &ctail};
  return cudaLaunchKernel(fn, dim3((unsigned)grid), dim3(kGemmThreads), args, SM::kAlloc, stream);
}

cudaError_t launch_gemm(const void* x, const void* packed, int M, int N, int K, int sym,
                        float* y, void* workspace, int* err, int num_sms,
                        unsigned long long wait_ns, cudaStream_t stream) {
  if (use_int8(M, K))
    return launch_gemv_tc(x, nullptr, packed, M, N, K, sym, y, workspace, err, num_sms, wait_ns,
                          stream);
  if (use_fold(M))
    return launch_gemm_fold(x, packed, M, N, K, sym, y, workspace, err, wait_ns, stream);
  GemmParams prm;
  prm.g = make_geom(N, K, sym);
  prm.packed = static_cast<const uint8_t*>(packed);
  prm.y = y;
  prm.counters = static_cast<unsigned*>(workspace);
  prm.partials = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kCounterBytes);
  float* xsum = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kCounterBytes +
                                         gemm_partials_bytes(prm.g, M));
  prm.xsum = xsum;
  prm.err = err;
  prm.M = M;
  prm.tiles = (long long)prm.g.NS * prm.g.NB;
  prm.ns_full = prm.g.NG / kSlabGroups;
  // rows of gs * 64 bytes per tile: 128 of codes + 128 * gs * meta / (gs * 64)
  prm.tile_rows = kTileRows + kTileRows * prm.g.meta / kCodeBytesPerGroupRow;
  prm.wait_ns = wait_ns;
  prm.drain_ns = 1000000000ull;
  prm.lop_mask_lo = 0x000F000Fu;
  prm.lop_bf16_128 = 0x43004300u;
  {
    const int warps = prm.g.NG;
    gemm_xsum_kernel<<<(warps * 32 + 255) / 256, 256, 0, stream>>>(
        static_cast<const uint16_t*>(x), M, K, xsum);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  switch (gemm_mpad(M)) {
    case 16: return launch_gemm_t<16>(prm, x, num_sms, stream);
    case 32: return launch_gemm_t<32>(prm, x, num_sms, stream);
    case 48: return launch_gemm_t<48>(prm, x, num_sms, stream);
    default: return launch_gemm_t<64>(prm, x, num_sms, stream);
  }
}

}  // namespace wq
