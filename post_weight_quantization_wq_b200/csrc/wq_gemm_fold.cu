// wq_gemm_fold.cu -- W4A16 GEMM for many activation rows (prefill, large
// batches) on the 5th-generation tensor cores, where the product is compute-
// bound ("大模型量化全景解析", section 八: prefill and large batches are bound
// by compute, decode by the weight bytes; "3.6 量化(Quantization)", section
// 仅权重 vs 权重 + 激活: the 4-bit weights are dequantized to 16-bit inside
// the matmul kernel):
//
//   y[m][n] = sum_g s16[n][g] * sum_{k in g} x[m][k] * (q[n][k] - z[n][g])
//
// A CTA owns a unit of (128 weight rows, MT activation rows, a range of
// groups).  Per group of 128 inputs:
//   * TMA brings the group's codes (128 rows x 64 bytes) and the activation
//     tile (MT rows x 128 inputs, bf16, 128-byte swizzle);
//   * four dequantizing warps write the bf16 integers 128 + q (exact) into a
//     128-byte-swizzled, K-major A tile in shared memory;
//   * one lane issues 8 tcgen05.mma (M = 128, N = MT, K = 16, both operands
//     from shared-memory descriptors) into one of four fp32 accumulators in
//     tensor memory;
//   * eight fold warps (two per tensor-memory lane quadrant, MT / 2 columns
//     each) load their part of the accumulator with one wait, release it to
//     the MMA issuer, and add s16 * (D - (128 + z) * sum_k x) to running sums
//     held in registers.
// The zero point and the 128 bias never enter the bf16 operands, so every
// dequantized value is exact.  Units along K are summed by a second kernel in
// a fixed order.
#include <cstring>

#include "wq_common.cuh"
#include "wq_tc.cuh"

namespace wq {

struct FoldParams {
  const uint8_t* packed;
  const float* xsum;       // fp32 [NG][Mpad]: sum of x over each group, per row of x
  float* out;              // y [M][N] (KS == 1) or partials [KS][Mpad][Npad]
  int* err;
  Geom g;
  int M, Mpad, KS, MTC;    // rows of x, padded rows, K splits, activation tiles
  int ns_full, tile_rows;
  unsigned long long wait_ns, drain_ns;
  uint32_t lop_mask_lo, lop_bf16_128;
};

constexpr int kFoldThreads = 14 * 32;     // TMA, MMA, 4 dequant, 8 fold warps
constexpr int kFoldWarps = 8;
constexpr int kFoldAcc = 4;               // accumulators in tensor memory
constexpr uint32_t kFoldTmemCols = 512;
constexpr int kFoldMetaSlots = 2;
constexpr int kFoldMetaBytes = kTileRows * kSlabGroups * 4;   // 2 KB

template <int MT>
struct FoldSmem {
  static constexpr int kA = kTileRows * kGroup * 2;            // 32 KB: 2 atoms of 64 inputs
  static constexpr int kBAtom = MT * 128;                      // MT rows x 64 bf16
  static constexpr int kB = 2 * kBAtom;
  static constexpr int kCodes = kTileRows * kCodeBytesPerGroupRow;   // 8 KB
  static constexpr int kStage = kA + kB + kCodes;              // multiple of 1024
  static constexpr int kStages = MT >= 64 ? 3 : 4;
  static constexpr int kMeta = kStages * kStage;
  static constexpr int kBar = kMeta + kFoldMetaSlots * kFoldMetaBytes;
  static constexpr int kNumBars = 3 * kStages + 2 * kFoldAcc + 2 * kFoldMetaSlots;
  static constexpr int kBytes = kBar + kNumBars * 8 + 16;
  static constexpr int kAlloc = kBytes + 1024;
  static_assert(kFoldAcc * MT <= (int)kFoldTmemCols, "tensor memory");
};

template <int MT>
__host__ __device__ constexpr uint32_t fold_idesc() {
  // kind::f16: fp32 D, bf16 A and B, both K-major, M = 128, N = MT
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(MT >> 3) << 17) | ((128u >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16_ss(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 16 consecutive fp32 columns of this thread's lane (valid after tmem_wait_ld).
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

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// The unit of this CTA: row tile b, activation tile mt, K split ks (activation
// tiles of one row tile are adjacent, so they share its codes in L2).
struct FoldUnit {
  int b, mt, ks, g0, g1;
};

__device__ __forceinline__ FoldUnit fold_unit(const FoldParams& p) {
  FoldUnit u;
  int t = blockIdx.x;
  u.mt = t % p.MTC;
  t /= p.MTC;
  u.ks = t % p.KS;
  u.b = t / p.KS;
  u.g0 = (int)((long long)u.ks * p.g.NG / p.KS);
  u.g1 = (int)((long long)(u.ks + 1) * p.g.NG / p.KS);
  return u;
}

template <int MT>
__global__ void __launch_bounds__(kFoldThreads, 1)
    gemm_w4a16_fold_kernel(const FoldParams p, const __grid_constant__ CUtensorMap xmap,
                           const __grid_constant__ CUtensorMap cmap_full,
                           const __grid_constant__ CUtensorMap cmap_tail) {
  using SM = FoldSmem<MT>;
  constexpr int S = SM::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SM::kBar);   // [S] codes + x landed
  uint64_t* afull = full + S;                                       // [S] A tile written
  uint64_t* empty = afull + S;                                      // [S] MMAs done with the stage
  uint64_t* dfull = empty + S;                                      // accumulator ready
  uint64_t* dempty = dfull + kFoldAcc;                              // accumulator read
  uint64_t* mfull = dempty + kFoldAcc;                              // [meta] landed
  uint64_t* mempty = mfull + kFoldMetaSlots;                        // [meta] read
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mempty + kFoldMetaSlots);

  const Geom g = p.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const FoldUnit u = fold_unit(p);
  const int ngr = u.g1 - u.g0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&afull[i], 4);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < kFoldAcc; ++i) {
      mbar_init(&dfull[i], 1);
      mbar_init(&dempty[i], kFoldWarps);
    }
    for (int i = 0; i < kFoldMetaSlots; ++i) {
      mbar_init(&mfull[i], 1);
      mbar_init(&mempty[i], kFoldWarps);
    }
    fence_mbarrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kFoldTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    int issued = 0, metas = 0;
    bool ok = true;
    for (int j = 0; j < ngr && ok; ++j) {
      const int gidx = u.g0 + j, s = gidx / kSlabGroups, gg = gidx % kSlabGroups;
      const int st = j % S;
      if (j == 0 || gg == 0) {
        // the metadata (scales, zeros) of the slab's 128 rows
        const int ms = metas % kFoldMetaSlots;
        if (metas >= kFoldMetaSlots)
          ok = warp_wait(&mempty[ms], ((metas / kFoldMetaSlots) - 1) & 1, p.wait_ns);
        if (!ok) break;
        const int gs = slab_groups(g, s);
        if (elect_one()) {
          const uint32_t mbytes = (uint32_t)(kTileRows * gs * g.meta);
          mbar_arrive_expect_tx(&mfull[ms], mbytes);
          bulk_copy_g2s(smem + SM::kMeta + ms * kFoldMetaBytes,
                        p.packed + tile_offset(g, s, u.b) +
                            (long long)kTileRows * gs * kCodeBytesPerGroupRow,
                        mbytes, &mfull[ms]);
        }
        __syncwarp();
        ++metas;
      }
      if (j >= S) ok = warp_wait(&empty[st], ((j / S) - 1) & 1, p.wait_ns);
      if (!ok) break;
      if (elect_one()) {
        uint8_t* sb = smem + st * SM::kStage;
        mbar_arrive_expect_tx(&full[st], (uint32_t)(SM::kCodes + SM::kB));
        if (s < p.ns_full)
          tma_load_2d(sb + SM::kA + SM::kB, &cmap_full, gg * kCodeBytesPerGroupRow,
                      (s * g.NB + u.b) * p.tile_rows, &full[st]);
        else
          tma_load_2d(sb + SM::kA + SM::kB, &cmap_tail, gg * kCodeBytesPerGroupRow,
                      u.b * p.tile_rows, &full[st]);
        const int k0 = gidx * kGroup;
        tma_load_2d(sb + SM::kA, &xmap, k0, u.mt * MT, &full[st]);
        tma_load_2d(sb + SM::kA + SM::kBAtom, &xmap, k0 + 64, u.mt * MT, &full[st]);
      }
      __syncwarp();
      issued = j + 1;
    }
    if (!ok) {
      if (lane == 0) atomicOr(p.err, kDevErrTimeout);
      for (int k = issued - S < 0 ? 0 : issued - S; k < issued; ++k)
        warp_wait(&full[k % S], (k / S) & 1, p.drain_ns);
      for (int k = metas - kFoldMetaSlots < 0 ? 0 : metas - kFoldMetaSlots; k < metas; ++k)
        warp_wait(&mfull[k % kFoldMetaSlots], (k / kFoldMetaSlots) & 1, p.drain_ns);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc = fold_idesc<MT>();
    bool ok = true;
    int done = 0;
    for (int j = 0; j < ngr; ++j) {
      const int st = j % S, db = j % kFoldAcc;
      ok = warp_wait(&afull[st], (j / S) & 1, p.wait_ns) &&
           warp_wait(&full[st], (j / S) & 1, p.wait_ns) &&
           (j < kFoldAcc || warp_wait(&dempty[db], ((j / kFoldAcc) - 1) & 1, p.wait_ns));
      if (!ok) break;
      tc_fence_after();
      if (elect_one()) {
        const uint32_t sa = smem_u32(smem + st * SM::kStage);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t a = sa + (kk >> 2) * (kTileRows * 128) + (kk & 3) * 32;
          const uint32_t bb = sa + SM::kA + (kk >> 2) * SM::kBAtom + (kk & 3) * 32;
          umma_bf16_ss(tmem_base + db * MT, umma_desc_sw128(a), umma_desc_sw128(bb), idesc,
                       kk > 0 ? 1u : 0u);
        }
        umma_commit(&empty[st]);
        umma_commit(&dfull[db]);
      }
      __syncwarp();
      done = j + 1;
    }
    if (!ok) {
      if (lane == 0) atomicOr(p.err, kDevErrTimeout);
      if (done > 0)
        warp_wait(&dfull[(done - 1) % kFoldAcc], ((done - 1) / kFoldAcc) & 1, p.drain_ns);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ dequantize
    // thread r writes row r of the A tile: 16 code words -> 128 bf16 (128 + q)
    const int r = (warp - 2) * 32 + lane;
    const uint32_t mlo = p.lop_mask_lo, b128 = p.lop_bf16_128;
    const int sw64 = (r >> 1) & 3;           // 64-byte swizzle of the codes
    const int sw128 = r & 7;                 // 128-byte swizzle of the A tile
    for (int j = 0; j < ngr; ++j) {
      const int st = j % S;
      if (!warp_wait(&full[st], (j / S) & 1, p.wait_ns)) {
        if (lane == 0) atomicOr(p.err, kDevErrTimeout);
        break;
      }
      uint8_t* sb = smem + st * SM::kStage;
      const uint8_t* codes = sb + SM::kA + SM::kB + r * kCodeBytesPerGroupRow;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 cw = *reinterpret_cast<const uint4*>(codes + ((c ^ sw64) << 4));
        const uint32_t wds[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int wi = 4 * c + i;          // code word = 8 inputs = one 16-byte A chunk
          const uint32_t w = wds[i];
          uint4 v;
          v.x = and_or3(w, mlo, b128);
          v.y = and_or3(w >> 4, mlo, b128);
          v.z = and_or3(w >> 8, mlo, b128);
          v.w = and_or3(w >> 12, mlo, b128);
          uint8_t* dst = sb + (wi >> 3) * (kTileRows * 128) + (r >> 3) * 1024 + sw128 * 128 +
                         (((wi & 7) ^ sw128) << 4);
          *reinterpret_cast<uint4*>(dst) = v;
        }
      }
      fence_proxy_async_smem();              // generic writes -> tensor-core reads
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[st]);
    }
  } else {
    // ------------------------------------------------------------ fold
    constexpr int EC = MT / 2;               // accumulator columns of this warp
    const int q = warp & 3;                  // tensor-memory lane quadrant
    const int half = (warp - 6) >> 2;        // columns half * EC .. half * EC + EC - 1
    const int row = q * 32 + lane;           // row of the tile
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    float run[EC];
#pragma unroll
    for (int c = 0; c < EC; ++c) run[c] = 0.0f;
    float scs[kSlabGroups], czs[kSlabGroups];
    int metas = 0;
    bool ok = true;
    for (int j = 0; j < ngr && ok; ++j) {
      const int gidx = u.g0 + j, s = gidx / kSlabGroups, gg = gidx % kSlabGroups;
      if (j == 0 || gg == 0) {
        const int ms = metas % kFoldMetaSlots;
        ok = warp_wait(&mfull[ms], (metas / kFoldMetaSlots) & 1, p.wait_ns);
        if (!ok) break;
        const int gs = slab_groups(g, s);
        const uint8_t* mb = smem + SM::kMeta + ms * kFoldMetaBytes;
#pragma unroll
        for (int t = 0; t < kSlabGroups; ++t) {
          scs[t] = 0.0f;
          czs[t] = 0.0f;
          if (t < gs) {
            if (g.sym) {
              scs[t] = __half2float(reinterpret_cast<const __half*>(mb)[row * gs + t]);
              czs[t] = 136.0f;               // 128 + 8
            } else {
              const __half2 sz = reinterpret_cast<const __half2*>(mb)[row * gs + t];
              scs[t] = __low2float(sz);
              czs[t] = 128.0f + __high2float(sz);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&mempty[ms]);
        ++metas;
      }
      float sc = scs[0], cz = czs[0];
#pragma unroll
      for (int t = 1; t < kSlabGroups; ++t)
        if (gg == t) { sc = scs[t]; cz = czs[t]; }
      const int db = j % kFoldAcc;
      ok = warp_wait(&dfull[db], (j / kFoldAcc) & 1, p.wait_ns);
      if (!ok) break;
      tc_fence_after();
      // this warp's columns of the accumulator in parts of up to 32 columns
      // (one wait each); the accumulator goes back to the MMA issuer as soon
      // as the last part is in registers, before its arithmetic
      constexpr int kPart = EC < 32 ? EC : 32;
      const uint32_t dcol = tmem_base + lane_off + db * MT + half * EC;
      const float* xs = p.xsum + (size_t)gidx * p.Mpad + u.mt * MT + half * EC;
#pragma unroll
      for (int p0 = 0; p0 < EC; p0 += kPart) {
        float d[kPart];
#pragma unroll
        for (int c0 = 0; c0 < kPart; c0 += 16) {
          if constexpr (kPart >= 16) tmem_ld16(dcol + p0 + c0, d + c0);
          else tmem_ld8(dcol + p0 + c0, d + c0);
        }
        tmem_wait_ld();
        if (p0 + kPart == EC) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&dempty[db]);
        }
#pragma unroll
        for (int i = 0; i < kPart; i += 4) {
          const float4 x4 = __ldg(reinterpret_cast<const float4*>(xs + p0 + i));
          const float xv[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
          for (int t = 0; t < 4; ++t)
            run[p0 + i + t] = __fmaf_rn(sc, __fmaf_rn(-cz, xv[t], d[i + t]), run[p0 + i + t]);
        }
      }
    }
    if (!ok) {
      if (lane == 0) atomicOr(p.err, kDevErrTimeout);
    } else if (ngr > 0) {
      // the unit's sums: y (one K split) or a partial
      const int n = u.b * kTileRows + row;
#pragma unroll
      for (int i = 0; i < EC; ++i) {
        const int m = u.mt * MT + half * EC + i;
        if (p.KS == 1) {
          if (m < p.M && n < g.N) p.out[(size_t)m * g.N + n] = run[i];
        } else if (m < p.M) {
          p.out[((size_t)u.ks * p.Mpad + m) * g.Npad + n] = run[i];
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(kFoldTmemCols)
                 : "memory");
  }
}

// sum_{k in g} x[m][k] for every group g and row m < Mpad of x, fp32 in a
// fixed order (rows m >= M are 0).  One warp per (group, row): lane l adds
// inputs 4l .. 4l+3, then a fixed shuffle tree.
__global__ void __launch_bounds__(256) fold_xsum_kernel(const uint16_t* __restrict__ x, int M,
                                                        int Mpad, int K, float* __restrict__ xsum) {
  const long long wid = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int NG = K / kGroup;
  if (wid >= (long long)NG * Mpad) return;
  const int gidx = (int)(wid / Mpad), m = (int)(wid % Mpad);
  float acc = 0.0f;
  if (m < M) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(x + (size_t)m * K + gidx * kGroup) + lane);
    acc = (__uint_as_float(v.x << 16) + __uint_as_float(v.x & 0xFFFF0000u)) +
          (__uint_as_float(v.y << 16) + __uint_as_float(v.y & 0xFFFF0000u));
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
  if (lane == 0) xsum[(size_t)gidx * Mpad + m] = acc;
}

// y[m][n] = sum over the K splits of the partials, in split order.
__global__ void fold_finish_kernel(const float* __restrict__ partials, int KS, int Mpad, int Npad,
                                   int M, int N, float* __restrict__ y) {
  const long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (e >= (long long)M * N) return;
  const int m = (int)(e / N), n = (int)(e % N);
  float t = 0.0f;
  for (int k = 0; k < KS; ++k) t += partials[((size_t)k * Mpad + m) * Npad + n];
  y[e] = t;
}

static int fold_mt(int M) { return M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128; }

// K splits: at least about two waves of CTAs over 148 SMs (the split depends
// on the shape only), each split at least 4 groups.
static int fold_splits(int NB, int MTC, int NG) {
  int ks = 1;
  while ((long long)NB * MTC * ks < 2 * 148 && NG / (ks + 1) >= 4 && ks < 16) ++ks;
  return ks;
}

struct FoldLayout {
  int MT, MTC, Mpad, KS;
  size_t xsum_bytes, part_bytes;
};

static FoldLayout fold_layout(int M, int N, int K) {
  const Geom g = make_geom(N, K, 1);
  FoldLayout l;
  l.MT = fold_mt(M);
  l.MTC = (M + l.MT - 1) / l.MT;
  l.Mpad = l.MTC * l.MT;
  l.KS = fold_splits(g.NB, l.MTC, g.NG);
  l.xsum_bytes = ((size_t)g.NG * l.Mpad * 4 + 255) / 256 * 256;
  l.part_bytes = l.KS > 1 ? (size_t)l.KS * l.Mpad * g.Npad * 4 : 0;
  return l;
}

// The workspace's first kCounterBytes are the completion counters of the
// skinny kernel (a workspace is shared by all calls on a stream): they are
// left untouched (zero); the sums of x and the partials follow them.
size_t gemm_fold_workspace_bytes(int M, int N, int K) {
  const FoldLayout l = fold_layout(M, N, K);
  return (size_t)kCounterBytes + l.xsum_bytes + l.part_bytes;
}

template <int MT>
static cudaError_t launch_fold_t(const FoldParams& prm, const void* x, cudaStream_t stream) {
  using SM = FoldSmem<MT>;
  auto enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const Geom& g = prm.g;
  CUtensorMap xmap, cfull, ctail;
  memset(&xmap, 0, sizeof(xmap));
  memset(&cfull, 0, sizeof(cfull));
  memset(&ctail, 0, sizeof(ctail));
  {
    cuuint64_t dims[2] = {(cuuint64_t)g.K, (cuuint64_t)prm.M};
    cuuint64_t strides[1] = {(cuuint64_t)g.K * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)MT};
    cuuint32_t estr[2] = {1, 1};
    if (enc(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
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
  const void* fn = reinterpret_cast<const void*>(&gemm_w4a16_fold_kernel<MT>);
  int per_sm = 0;
  cudaError_t e = kernel_setup(fn, SM::kAlloc, kFoldThreads, &per_sm);
  if (e != cudaSuccess) return e;
  FoldParams pp = prm;
  void* args[] = {&pp, &xmap, &cfull, &ctail};
  const long long grid = (long long)g.NB * prm.KS * prm.MTC;
  return cudaLaunchKernel(fn, dim3((unsigned)grid), dim3(kFoldThreads), args, SM::kAlloc, stream);
}

cudaError_t launch_gemm_fold(const void* x, const void* packed, int M, int N, int K, int sym,
                             float* y, void* workspace, int* err, unsigned long long wait_ns,
                             cudaStream_t stream) {
  const FoldLayout l = fold_layout(M, N, K);
  FoldParams prm;
  prm.g = make_geom(N, K, sym);
  prm.packed = static_cast<const uint8_t*>(packed);
  uint8_t* base = static_cast<uint8_t*>(workspace) + kCounterBytes;
  float* xsum = reinterpret_cast<float*>(base);
  float* partials = reinterpret_cast<float*>(base + l.xsum_bytes);
  prm.xsum = xsum;
  prm.out = l.KS > 1 ? partials : y;
  prm.err = err;
  prm.M = M;
  prm.Mpad = l.Mpad;
  prm.KS = l.KS;
  prm.MTC = l.MTC;
  prm.ns_full = prm.g.NG / kSlabGroups;
  prm.tile_rows = kTileRows + kTileRows * prm.g.meta / kCodeBytesPerGroupRow;
  prm.wait_ns = wait_ns;
  prm.drain_ns = 1000000000ull;
  prm.lop_mask_lo = 0x000F000Fu;
  prm.lop_bf16_128 = 0x43004300u;
  {
    const long long warps = (long long)prm.g.NG * l.Mpad;
    fold_xsum_kernel<<<(unsigned)((warps * 32 + 255) / 256), 256, 0, stream>>>(
        static_cast<const uint16_t*>(x), M, l.Mpad, K, xsum);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  cudaError_t e;
  switch (l.MT) {
    case 16: e = launch_fold_t<16>(prm, x, stream); break;
    case 32: e = launch_fold_t<32>(prm, x, stream); break;
    case 64: e = launch_fold_t<64>(prm, x, stream); break;
    default: e = launch_fold_t<128>(prm, x, stream); break;
  }
  if (e != cudaSuccess || l.KS == 1) return e;
  const long long outs = (long long)M * N;
  fold_finish_kernel<<<(unsigned)((outs + 255) / 256), 256, 0, stream>>>(
      partials, l.KS, l.Mpad, prm.g.Npad, M, N, y);
  return cudaGetLastError();
}

}  // namespace wq
