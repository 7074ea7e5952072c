// wq_gemv_tc.cu -- W4A16 decode linear for M = 2..16 rows of x on the
// integer tensor cores (tcgen05.mma kind::i8, sm_100a):
//
//   y[m][n] = sum_g s16[n][g] * sum_{k in g} x[m][k] * (q[n][k] - z[n][g])
//
// The same arithmetic as the integer path of wq_gemv.cu, with the dot products
// moved from dp4a onto the tensor cores.  Weight-only 4-bit decode is bound by
// the bytes of the weights ("推理优化中“用精度换性能“的核心技术：量化", section
// 一; "3.6 量化(Quantization)", section 为什么重要); the CUDA-core inner loop
// spends six instructions per 8 weights on them, this kernel two, so the
// instruction issue no longer competes with the stream of weights.
//
// Activations: x' = x, or x' = fp32(x) * inv_act_scale (the AWQ fold, one
// rounded fp32 product); each 64-input chunk c of row m of x' becomes 16-bit
// integers x_i = rn(x' * 2^e) with e putting the chunk's largest |x'| in
// [2^14, 2^15) (exact for a bf16 x: 8 significant bits), split as
// x_i = 256 h + l into signed high bytes h and unsigned low bytes l (the same
// rounding as the CUDA-core integer path).
//
// Weights: w & 0x0F0F0F0F and (w >> 4) & 0x0F0F0F0F of a layout word are its
// 8 codes as unsigned bytes (the inputs 0, 4, 1, 5 and 2, 6, 3, 7 of the
// word: nibble slot t holds input 2t for t < 4 and 2(t - 4) + 1 otherwise).
// They are the A operand, 128 rows (the tile's output rows) x 512 bytes,
// stored straight into tensor memory (tcgen05.st) by the unpacking warps:
// bytes 8 j .. 8 j + 7 of a row are those of the row's word j, in that order.
//
// B (shared memory, SWIZZLE_128B, K-major, signed bytes, NB = 8, 16, 32 or
// 48 rows for Mpad = 2, 4, 8, 16): row 2m holds the high bytes h of row m of x and
// row 2m + 1 its low bytes as l' = l - 128, both in the input order of the A
// bytes; row 2 Mpad holds ones.  Per chunk c (64 bytes of K = two MMAs of
// K = 32), one accumulator of NB int32 columns:
//   D[2m] = sum q h,  D[2m+1] = sum q l',  D[2Mp] = sum q,
// so that exactly (l = l' + 128)
//   sum_{k in c} q x_i = 256 D[2m] + D[2m+1] + 128 D[2Mp]
// (every term fits in int32: 64 products of at most 15 * 128).  With
// u_c = 2^-e of chunk c and the group's P = sum_{c in group} u_c * sum_{k in c} x_i
// (the same for every weight row, prepared with the activation rows), a
// group of two chunks adds s16 * (sum_c u_c * t_c - z * P) to y in fp32
// (u_c * t_c is exact: u_c is a power of two).
//
// The planes depend on the slab of x only, not on the row tile, so a first
// small kernel prepares them once per slab into the workspace (already in
// the swizzled order of shared memory); the streaming kernel, launched as its
// programmatic dependent, starts loading weights while it runs.
//
// Data flow of one CTA of the streaming kernel (persistent, one per SM;
// contiguous run of the layout tiles u = b * NS + s like the CUDA-core
// kernel, so a CTA walks the slabs of one row tile after another), in
// half-tiles of 256 inputs between the tensor-memory roles:
//   warp 0      2-D TMA loads of each tile's codes (two boxes of 128 rows x
//               128 bytes, 128-byte swizzle: a warp reading one 16-byte chunk
//               of 32 rows touches every bank once per 8 lanes) into a ring
//               of code stages;
//   warp 3      a bulk copy of each tile's metadata into a ring of its own;
//   warp 2      bulk copies of each tile's prepared planes and chunk factors
//               into a ring of operand slots;
//   warps 4-11  unpack: one row (tensor-memory lane) and half the slab each;
//               the code stage is released as soon as the words are in
//               registers;
//   warp 1      tensor-memory owner and MMA issuer: 8 MMAs (M = 128, N = NB,
//               K = 32) per half-tile into one of the accumulator sets;
//   warps 12-19 epilogue: one row and one half-tile each, running sums over
//               the slabs of a row tile in registers; the two halves of a row
//               meet in shared memory at the end of the CTA's piece of a row
//               tile, which is written to y, or to the split-K workspace when
//               the row tile is shared with another CTA (the small finish
//               kernel of the CUDA-core path adds the pieces in slab order).
// Tensor memory (512 columns): four A buffers of 64 columns (two at
// Mpad = 16), then up to four accumulator sets of 4 NB columns (two at
// Mpad = 8 and 16), one half-tile each.  Every wait is bounded; on timeout the
// kernel records the device error word and winds down, waiting (bounded) for
// its copies and MMAs in flight.
#include <cuda.h>
#include <cstring>
#include <cudaTypedefs.h>

#include "wq_common.cuh"
#include "wq_tc.cuh"

namespace wq {

cudaError_t launch_gemv_finish(const float* partials, float* y, int N, int M, int MP, int NS,
                               int Npad, int G, long long tiles, cudaStream_t stream);

namespace {

constexpr int kTgWarps = 20;
constexpr int kTgThreads = kTgWarps * 32;
constexpr int kTgMetaSlots = 4;
constexpr uint32_t kTgTmemCols = 512;
constexpr int kTgCodeBytes = kTileRows * kSlabGroups * kCodeBytesPerGroupRow;   // 32 KB
constexpr int kTgMaxM = 16;
constexpr int kTgMeta = kTileRows * kSlabGroups * 4;

// Rows of the B operand (2 per row of x, one row of ones), the tensor-memory
// split between A buffers (64 columns each) and accumulator sets (one
// half-tile each), and the shared-memory rings.
template <int MP>
struct TgShape {
  static constexpr int kNB = MP == 2 ? 8 : MP == 4 ? 16 : MP == 8 ? 32 : 48;   // >= 2 MP + 1
  static constexpr int kDCols = 4 * kNB;
  static constexpr int kABufs = MP == 16 ? 2 : 4;
  static constexpr int kColD = kABufs * 64;
  static constexpr int kDFit = (512 - kColD) / kDCols;
  static constexpr int kDBufs = kDFit < 4 ? kDFit : 4;
  static constexpr int kStages = MP == 16 ? 4 : 5;                // code stages (one tile each)
  static constexpr int kBSlots = MP == 16 ? 2 : MP == 8 ? 3 : 4;
  static constexpr int kBSlot = kNB * kSlabK;                     // 4 K-blocks x NB rows x 128
  static constexpr int kRows = 2 * MP;                            // prepared rows per K-block
  static constexpr int kXinfo = MP * 8 * 8;                       // float2 [MP][8 chunks]
  static_assert(kDBufs >= 2 && kColD + kDBufs * kDCols <= 512, "tensor memory");
};

template <int MP>
struct TgSmem {
  using SH = TgShape<MP>;
  static constexpr int kCode = 0;
  static constexpr int kB = kCode + SH::kStages * kTgCodeBytes;
  static constexpr int kMeta = kB + SH::kBSlots * SH::kBSlot;
  static constexpr int kXinfo = kMeta + kTgMetaSlots * kTgMeta;
  static constexpr int kExch = kXinfo + SH::kBSlots * SH::kXinfo;    // float [4][32][MP]
  static constexpr int kBar = kExch + 4 * 32 * MP * 4;
  // cfull/cempty, mfull/mempty, bfull/bempty/xiempty, afull/aempty, dfull/dempty
  static constexpr int kNumBars = 2 * SH::kStages + 2 * kTgMetaSlots + 3 * SH::kBSlots +
                                  2 * SH::kABufs + 2 * SH::kDBufs;
  static constexpr int kBytes = kBar + kNumBars * 8 + 16;
  static constexpr int kAlloc = kBytes + 1024;
  static_assert(kB % 1024 == 0 && kBar % 8 == 0, "alignment");
  static_assert(kAlloc <= 232448, "shared memory");
};


struct TgParams {
  const uint8_t* packed;
  const uint8_t* planes;   // prepared B rows: [NS][4 K-blocks][2 MP rows][128 B]
  const float2* xinfo;     // [NS][MP][8 chunks] (2^-e of the chunk, P of its group)
  float* y;                // fp32 [M][N]
  float* partials;         // fp32 [NS][MP][Npad]
  int* err;
  Geom g;
  int M, MP;
  int tile_rows;           // rows of 256 bytes per tile in the 2-D view of the layout
  long long tiles;         // NB * NS
  unsigned long long wait_ns, drain_ns;
};

// Instruction descriptor of kind::i8: int32 D, unsigned A, signed B, both
// K-major, M = 128, N = NB.
__host__ __device__ constexpr uint32_t tg_idesc(int nb) {
  return (2u << 4) | (0u << 7) | (1u << 10) | ((uint32_t)(nb >> 3) << 17) |
         ((uint32_t)(128 >> 4) << 24);
}

// D (tensor memory, int32) (+)= A (tensor memory, 128 rows x 32 bytes) *
// B (shared memory descriptor, 8 rows x 32 bytes)^T
__device__ __forceinline__ void umma_i8_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// N consecutive 32-bit columns of this thread's lane (N a multiple of 8).
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, int* v) {
  static_assert(N % 8 == 0, "columns");
  if constexpr (N > 16) {
    tmem_ld_cols<16>(taddr, v);
    tmem_ld_cols<N - 16>(taddr + 16, v + 16);
  } else if constexpr (N == 16) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
          "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
  } else {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7])
        : "r"(taddr));
  }
}

// Byte offset of 16-byte chunk ck (bytes 16 ck .. 16 ck + 15 of K) of row r
// within a K-block of B (8-row atoms of 128-byte rows, 1024-byte aligned, the
// chunk index swizzled with the row within its atom: SWIZZLE_128B).
__device__ __forceinline__ int b_row_chunk(int r, int ck) {
  return r * 128 + (((ck & 7) ^ (r & 7)) << 4);
}

// Bytes of the prepared rows of one slab: 4 K-blocks x 2 MP rows x 128.
__host__ __device__ constexpr int tg_slab_plane_bytes(int MP) { return 4 * 2 * MP * 128; }

// One warp per (slab s, row m < MP of x): the fixed-point bytes of row m of
// the slab (of x' = x * inv_s when inv_s is given), in the shared-memory
// order of rows 2m and 2m + 1 of each K-block, and per chunk (2^-e, P of its
// group of two chunks).  Rows m >= M are zeros.
// planes: [NS][4 K-blocks][2 MP rows][128 B]; xinfo: [NS][MP][8].
__global__ void __launch_bounds__(32 * kTgMaxM) gemv_tc_prep_kernel(const uint16_t* __restrict__ x,
                                                                    const float* __restrict__ inv_s,
                                                                    int M, int MP, int K,
                                                                    uint8_t* __restrict__ planes,
                                                                    float2* __restrict__ xinfo) {
  griddep_launch_dependents();
  const int s = blockIdx.x, m = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // x may be written, and this workspace still read, by the previous kernel
  griddep_wait();
  if (m >= MP) return;
  uint8_t* ps = planes + (size_t)s * tg_slab_plane_bytes(MP);
  const int c = lane >> 2, sub = lane & 3;   // 64-input chunk and quarter of it
  const int ck = lane;                       // 16-byte chunk of K (words 2 lane, 2 lane + 1)
  const int kb = ck >> 3;                    // K-block of 128 bytes
  auto row_at = [&](int r) { return ps + kb * 2 * MP * 128 + b_row_chunk(r, ck); };
  if (m >= M) {
    const uint4 z4 = make_uint4(0, 0, 0, 0);
    *reinterpret_cast<uint4*>(row_at(2 * m)) = z4;
    *reinterpret_cast<uint4*>(row_at(2 * m + 1)) = z4;
    if (sub == 0) xinfo[((size_t)s * MP + m) * 8 + c] = make_float2(0.0f, 0.0f);
    return;
  }
  // lane l: inputs 16 l .. 16 l + 15 of the slab
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)m * K + (size_t)s * kSlabK + 16 * lane);
  const uint4 r0 = src[0], r1 = src[1];
  const uint32_t r[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
  float xf[16];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    xf[2 * q] = __uint_as_float(r[q] << 16);
    xf[2 * q + 1] = __uint_as_float(r[q] & 0xFFFF0000u);
  }
  if (inv_s) {
    const float4* iv = reinterpret_cast<const float4*>(inv_s + (size_t)s * kSlabK + 16 * lane);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 f = iv[q];
      xf[4 * q] = __fmul_rn(xf[4 * q], f.x);
      xf[4 * q + 1] = __fmul_rn(xf[4 * q + 1], f.y);
      xf[4 * q + 2] = __fmul_rn(xf[4 * q + 2], f.z);
      xf[4 * q + 3] = __fmul_rn(xf[4 * q + 3], f.w);
    }
  }
  bool bad = false;
#pragma unroll
  for (int q = 0; q < 16; ++q) bad |= !(fabsf(xf[q]) <= 3.402823466e38f);   // NaN or infinity
  float amax = 0.0f;
#pragma unroll
  for (int q = 0; q < 16; ++q) amax = fmaxf(amax, fabsf(xf[q]));
  amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
  bad = __shfl_xor_sync(0xFFFFFFFFu, (int)bad, 1) | bad;
  bad = __shfl_xor_sync(0xFFFFFFFFu, (int)bad, 2) | bad;
  // x_i = rn(x * 2^e), the chunk's largest |x| in [2^14, 2^15); a chunk with
  // a NaN or an infinity gives zeros and a NaN factor
  int e = 0;
  if (!bad && amax > 0.0f) {
    int eb = (int)(__float_as_uint(amax) >> 23), pre = 0;
    if (eb == 0) {                                 // subnormal: exponent of amax * 2^64
      eb = (int)(__float_as_uint(amax * 0x1p64f) >> 23);
      pre = 64;
    }
    e = 141 - eb + pre;                            // in [-113, 147]
  }
  const float unscale = bad ? __uint_as_float(0x7FC00000u)
                        : (e <= 126 ? __uint_as_float((uint32_t)(127 - e) << 23)
                                    : __uint_as_float(1u << (149 - e)));
  const int e1 = e > 127 ? 64 : e;
  const float f1 = __uint_as_float((uint32_t)(e1 + 127) << 23);
  const float f2 = __uint_as_float((uint32_t)(e - e1 + 127) << 23);
  int xi[16];
  int sx = 0;
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    xi[q] = bad ? 0 : __float2int_rn(__fmul_rn(__fmul_rn(xf[q], f1), f2));
    sx += xi[q];
  }
  // bytes of the two words in the A byte order: inputs 0, 4, 1, 5, then
  // 2, 6, 3, 7 of each word; l' = l - 128 is the low byte with its top bit
  // flipped
  auto hb = [](int a) { return (uint32_t)(a >> 8) & 0xFFu; };
  auto lb = [](int a) { return ((uint32_t)a & 0xFFu) ^ 0x80u; };
  uint32_t hw[4], lw[4];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int* v = xi + 8 * t;
    hw[2 * t] = hb(v[0]) | hb(v[4]) << 8 | hb(v[1]) << 16 | hb(v[5]) << 24;
    hw[2 * t + 1] = hb(v[2]) | hb(v[6]) << 8 | hb(v[3]) << 16 | hb(v[7]) << 24;
    lw[2 * t] = lb(v[0]) | lb(v[4]) << 8 | lb(v[1]) << 16 | lb(v[5]) << 24;
    lw[2 * t + 1] = lb(v[2]) | lb(v[6]) << 8 | lb(v[3]) << 16 | lb(v[7]) << 24;
  }
  *reinterpret_cast<uint4*>(row_at(2 * m)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
  *reinterpret_cast<uint4*>(row_at(2 * m + 1)) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
  sx += __shfl_xor_sync(0xFFFFFFFFu, sx, 1);
  sx += __shfl_xor_sync(0xFFFFFFFFu, sx, 2);
  // u * sum x_i is exact (|sum x_i| < 2^21, u a power of two); P adds the
  // group's two chunks (lane ^ 4 holds the other one), the same sum on both
  const float v = __fmul_rn(unscale, (float)sx);
  const float other = __shfl_xor_sync(0xFFFFFFFFu, v, 4);
  const float P = (c & 1) ? __fadd_rn(other, v) : __fadd_rn(v, other);
  if (sub == 0) xinfo[((size_t)s * MP + m) * 8 + c] = make_float2(unscale, P);
}

template <int MP>
__global__ void __launch_bounds__(kTgThreads, 1)
    gemv_w4a16_tc_kernel(const TgParams prm, const __grid_constant__ CUtensorMap cmap) {
  using SH = TgShape<MP>;
  using SM = TgSmem<MP>;
  constexpr int NB = SH::kNB, kBSlots = SH::kBSlots, kDBufs = SH::kDBufs;
  constexpr int kTgStages = SH::kStages, kTgABufs = SH::kABufs;
  constexpr uint32_t kTgColA = 0, kTgColD = SH::kColD;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kBar);
  uint64_t* cfull = bars;
  uint64_t* cempty = cfull + kTgStages;
  uint64_t* mfull = cempty + kTgStages;
  uint64_t* mempty = mfull + kTgMetaSlots;
  uint64_t* bfull = mempty + kTgMetaSlots;
  uint64_t* bempty = bfull + kBSlots;
  uint64_t* xiempty = bempty + kBSlots;
  uint64_t* afull = xiempty + kBSlots;
  uint64_t* aempty = afull + kTgABufs;
  uint64_t* dfull = aempty + kTgABufs;
  uint64_t* dempty = dfull + kDBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(dempty + kDBufs);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const Geom g = prm.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long t0 = (long long)blockIdx.x * prm.tiles / gridDim.x;
  const long long t1 = (long long)(blockIdx.x + 1) * prm.tiles / gridDim.x;
  const int ntiles = (int)(t1 - t0);
  auto fail = [&]() {
    atomicOr(prm.err, kDevErrTimeout);
    *abort_flag = 1;
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < kTgStages; ++i) {
      mbar_init(&cfull[i], 1);
      mbar_init(&cempty[i], 8);                // the 8 unpacking warps
    }
    for (int i = 0; i < kTgMetaSlots; ++i) {
      mbar_init(&mfull[i], 1);
      mbar_init(&mempty[i], 8);                // the 8 epilogue warps
    }
    for (int i = 0; i < kBSlots; ++i) {
      mbar_init(&bfull[i], 1);
      mbar_init(&bempty[i], 1);                // MMA commit
      mbar_init(&xiempty[i], 8);               // the 8 epilogue warps
    }
    for (int i = 0; i < kTgABufs; ++i) {
      mbar_init(&afull[i], 4);                 // the 4 unpacking warps of a half
      mbar_init(&aempty[i], 1);                // MMA commit
    }
    for (int i = 0; i < kDBufs; ++i) {
      mbar_init(&dfull[i], 1);                 // MMA commit
      mbar_init(&dempty[i], 4);                // the 4 epilogue warps of a half
    }
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  // Every activation slot once: row 2 Mpad of each K-block holds ones, the
  // rows past it zeros; the prepared rows 0 .. 2 Mpad - 1 are copied in per
  // tile.
  for (int i = threadIdx.x; i < kBSlots * SH::kBSlot / 16; i += kTgThreads) {
    const int r = (i / 8) % NB;                // 16-byte chunk i: row of its K-block
    const uint32_t one = 0x01010101u;
    reinterpret_cast<uint4*>(smem + SM::kB)[i] =
        r == 2 * MP ? make_uint4(one, one, one, one) : make_uint4(0, 0, 0, 0);
  }
  fence_proxy_async_shared();            // read by the tensor cores
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTgTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ codes (TMA)
    // Weights are never written by a kernel of this library: no wait for the
    // previous kernel of the stream.
    int issued = 0;
    bool ok = true;
    for (int i = 0; i < ntiles; ++i) {
      const long long u = t0 + i;
      const int b = (int)(u / g.NS), s = (int)(u % g.NS);
      const int st = i % kTgStages;
      if (i >= kTgStages) ok = warp_wait(&cempty[st], ((i / kTgStages) - 1) & 1, prm.wait_ns);
      if (!ok || *abort_flag) { ok = false; break; }
      if (elect_one()) {
        uint8_t* dst = smem + SM::kCode + st * kTgCodeBytes;
        const int row = (s * g.NB + b) * prm.tile_rows;
        mbar_arrive_expect_tx(&cfull[st], (uint32_t)kTgCodeBytes);
        tma_load_2d(dst, &cmap, 0, row, &cfull[st]);
        tma_load_2d(dst + kTgCodeBytes / 2, &cmap, 128, row, &cfull[st]);
      }
      __syncwarp();
      issued = i + 1;
    }
    if (!ok) {
      if (lane == 0) fail();
      for (int k = issued - kTgStages < 0 ? 0 : issued - kTgStages; k < issued; ++k)
        warp_wait(&cfull[k % kTgStages], (k / kTgStages) & 1, prm.drain_ns);
    }
  } else if (warp == 3) {
    // ------------------------------------------------------------ metadata
    const uint32_t mbytes = (uint32_t)(kTileRows * kSlabGroups * g.meta);
    int issued = 0;
    bool ok = true;
    for (int i = 0; i < ntiles; ++i) {
      const long long u = t0 + i;
      const int b = (int)(u / g.NS), s = (int)(u % g.NS);
      const int ms = i % kTgMetaSlots;
      if (i >= kTgMetaSlots)
        ok = warp_wait(&mempty[ms], ((i / kTgMetaSlots) - 1) & 1, prm.wait_ns);
      if (!ok || *abort_flag) { ok = false; break; }
      if (elect_one()) {
        mbar_arrive_expect_tx(&mfull[ms], mbytes);
        bulk_copy_g2s(smem + SM::kMeta + ms * kTgMeta,
                      prm.packed + tile_offset(g, s, b) + kTgCodeBytes, mbytes, &mfull[ms]);
      }
      __syncwarp();
      issued = i + 1;
    }
    if (!ok) {
      if (lane == 0) fail();
      for (int k = issued - kTgMetaSlots < 0 ? 0 : issued - kTgMetaSlots; k < issued; ++k)
        warp_wait(&mfull[k % kTgMetaSlots], (k / kTgMetaSlots) & 1, prm.drain_ns);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ activations
    // The prepared rows of the tile's slab: for each K-block, rows
    // 0 .. 2 Mpad - 1 are one contiguous run at the start of its row groups.
    constexpr uint32_t kRun = SH::kRows * 128;
    constexpr uint32_t kBytes = 4 * kRun + MP * 64;
    griddep_wait();                      // the planes come from the preparing kernel
    int issued = 0;
    bool ok = true;
    for (int i = 0; i < ntiles; ++i) {
      const int s = (int)((t0 + i) % g.NS);
      const int xs = i % kBSlots;
      if (i >= kBSlots)
        ok = warp_wait(&bempty[xs], ((i / kBSlots) - 1) & 1, prm.wait_ns) &&
             warp_wait(&xiempty[xs], ((i / kBSlots) - 1) & 1, prm.wait_ns);
      if (!ok || *abort_flag) { ok = false; break; }
      if (elect_one()) {
        uint8_t* bslot = smem + SM::kB + xs * SH::kBSlot;
        const uint8_t* src = prm.planes + (size_t)s * tg_slab_plane_bytes(MP);
        mbar_arrive_expect_tx(&bfull[xs], kBytes);
        for (int kb = 0; kb < 4; ++kb)
          bulk_copy_g2s(bslot + kb * (NB / 8) * 1024, src + kb * kRun, kRun, &bfull[xs]);
        bulk_copy_g2s(smem + SM::kXinfo + xs * SH::kXinfo, prm.xinfo + (size_t)s * MP * 8,
                      MP * 64, &bfull[xs]);
      }
      __syncwarp();
      issued = i + 1;
    }
    if (!ok) {
      if (lane == 0) fail();
      for (int k = issued - kBSlots < 0 ? 0 : issued - kBSlots; k < issued; ++k)
        warp_wait(&bfull[k % kBSlots], (k / kBSlots) & 1, prm.drain_ns);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc = tg_idesc(NB);
    bool ok = true;
    int committed = -1;                  // last half-tile whose MMAs were committed
    for (int i = 0; i < ntiles && ok; ++i) {
      const int xs = i % kBSlots;
      for (int h = 0; h < 2; ++h) {
        const int j = 2 * i + h, ja = j % kTgABufs, jd = j % kDBufs;
        ok = warp_wait(&afull[ja], (j / kTgABufs) & 1, prm.wait_ns);
        if (ok && h == 0) ok = warp_wait(&bfull[xs], (i / kBSlots) & 1, prm.wait_ns);
        if (ok && j >= kDBufs) ok = warp_wait(&dempty[jd], ((j / kDBufs) - 1) & 1, prm.wait_ns);
        if (!ok || *abort_flag) { ok = false; break; }
        tc_fence_after();
        if (elect_one()) {
          const uint32_t a0 = tmem_base + kTgColA + ja * 64;
          const uint32_t d0 = tmem_base + kTgColD + jd * SH::kDCols;
          const uint32_t bs = smem_u32(smem + SM::kB + xs * SH::kBSlot);
#pragma unroll
          for (int cc = 0; cc < 4; ++cc)
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
              const int kb = (4 * h + cc) * 64 + kk * 32;     // byte of K within the slab
              const uint64_t bdesc =
                  umma_desc_sw128(bs + (kb >> 7) * (NB / 8) * 1024 + (kb & 127));
              umma_i8_ts(d0 + cc * NB, a0 + cc * 16 + kk * 8, bdesc, idesc, kk);
            }
          umma_commit(&aempty[ja]);
          umma_commit(&dfull[jd]);
          if (h == 1) umma_commit(&bempty[xs]);
        }
        __syncwarp();
        committed = j;
      }
    }
    if (!ok) {
      if (lane == 0) fail();
      if (committed >= 0)
        warp_wait(&dfull[committed % kDBufs], (committed / kDBufs) & 1, prm.drain_ns);
    }
  } else if (warp >= 4 && warp < 12) {
    // ------------------------------------------------------------ unpack
    const int quad = warp & 3;                 // tensor-memory lane quadrant
    const int h = (warp - 4) >> 2;             // half-tile: code bytes 128 h .. 128 h + 127 of each row
    const int r = quad * 32 + lane;            // row of the tile (= lane)
    const uint32_t lane_base = tmem_base + ((uint32_t)(quad * 32) << 16) + kTgColA;
    bool ok = true;
    for (int i = 0; i < ntiles; ++i) {
      const int st = i % kTgStages;
      const int j = 2 * i + h, jb = j % kTgABufs;
      bool w_ok = mbar_wait_bounded(&cfull[st], (i / kTgStages) & 1, prm.wait_ns);
      if (w_ok && j >= kTgABufs)
        w_ok = mbar_wait_bounded(&aempty[jb], ((j / kTgABufs) - 1) & 1, prm.wait_ns);
      if (!__all_sync(0xFFFFFFFFu, w_ok) || *abort_flag) { ok = false; break; }
      tc_fence_after();
      const uint8_t* row = smem + SM::kCode + st * kTgCodeBytes + h * (kTgCodeBytes / 2) + r * 128;
      uint4 cw[8];
#pragma unroll
      for (int q = 0; q < 8; ++q)
        cw[q] = *reinterpret_cast<const uint4*>(row + ((q ^ (r & 7)) << 4));
      __syncwarp();                            // every lane has its words
      if (lane == 0) mbar_arrive(&cempty[st]);
#pragma unroll
      for (int j4 = 0; j4 < 4; ++j4) {
        uint32_t v[16];
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const uint4 w = cw[2 * j4 + jj];
          const uint32_t wd[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            v[8 * jj + 2 * t] = wd[t] & 0x0F0F0F0Fu;
            v[8 * jj + 2 * t + 1] = (wd[t] >> 4) & 0x0F0F0F0Fu;
          }
        }
        tmem_st16(lane_base + jb * 64 + j4 * 16, v);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[jb]);
    }
    if (!ok && lane == 0) fail();
  } else if (warp >= 12) {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;
    const int eh = (warp - 12) >> 2;           // half-tile: chunks 4 eh .. 4 eh + 3 (groups 2 eh, 2 eh + 1)
    const int r = quad * 32 + lane;
    const uint32_t lane_base = tmem_base + ((uint32_t)(quad * 32) << 16) + kTgColD;
    float* exch = reinterpret_cast<float*>(smem + SM::kExch) + (quad * 32 + lane) * MP;
    float run[MP];
#pragma unroll
    for (int m = 0; m < MP; ++m) run[m] = 0.0f;
    int piece_s0 = -1;
    bool ok = true;
    griddep_wait();                            // y and the workspace may belong to the previous kernel
    for (int i = 0; i < ntiles; ++i) {
      const long long u = t0 + i;
      const int b = (int)(u / g.NS), s = (int)(u % g.NS);
      const int j = 2 * i + eh, jd = j % kDBufs;
      const int ms = i % kTgMetaSlots, xs = i % kBSlots;
      if (piece_s0 < 0) piece_s0 = s;
      if (ok) {
        bool w_ok = mbar_wait_bounded(&dfull[jd], (j / kDBufs) & 1, prm.wait_ns) &&
                    mbar_wait_bounded(&bfull[xs], (i / kBSlots) & 1, prm.wait_ns) &&
                    mbar_wait_bounded(&mfull[ms], (i / kTgMetaSlots) & 1, prm.wait_ns);
        if (!__all_sync(0xFFFFFFFFu, w_ok) || *abort_flag) ok = false;
      }
      if (ok) {
        tc_fence_after();
        // this row's (scale, zero) of groups 2 eh and 2 eh + 1
        const uint8_t* mb = smem + SM::kMeta + ms * kTgMeta;
        float sc[2], zc[2];
#pragma unroll
        for (int gg = 0; gg < 2; ++gg) {
          const int grp = 2 * eh + gg;
          if (g.sym) {
            sc[gg] = __half2float(reinterpret_cast<const __half*>(mb)[r * kSlabGroups + grp]);
            zc[gg] = 8.0f;
          } else {
            const __half2 sz = reinterpret_cast<const __half2*>(mb)[r * kSlabGroups + grp];
            sc[gg] = __low2float(sz);
            zc[gg] = __high2float(sz);
          }
        }
        const float2* xinfo = reinterpret_cast<const float2*>(smem + SM::kXinfo + xs * SH::kXinfo);
        // per group of two chunks: acc = sum_c u_c t_c, then
        // run += s16 (acc - z P); the accumulators kCS chunks at a time
        constexpr int kCS = NB >= 32 ? 1 : 2;
        const uint32_t dbase = lane_base + jd * SH::kDCols;
#pragma unroll
        for (int gg = 0; gg < 2; ++gg) {
          float acc[MP];
#pragma unroll
          for (int m = 0; m < MP; ++m) acc[m] = 0.0f;
#pragma unroll
          for (int c2 = 2 * gg; c2 < 2 * gg + 2; c2 += kCS) {
            int dv[kCS][NB];
#pragma unroll
            for (int c1 = 0; c1 < kCS; ++c1) tmem_ld_cols<NB>(dbase + (c2 + c1) * NB, dv[c1]);
            tmem_wait_ld();
#pragma unroll
            for (int c1 = 0; c1 < kCS; ++c1) {
              const int cc = c2 + c1;
              const int* D = dv[c1];
              const int ones = 128 * D[2 * MP];
#pragma unroll
              for (int m = 0; m < MP; ++m) {
                const int t = 256 * D[2 * m] + D[2 * m + 1] + ones;
                acc[m] = fmaf(xinfo[m * 8 + 4 * eh + cc].x, (float)t, acc[m]);
              }
            }
          }
#pragma unroll
          for (int m = 0; m < MP; ++m)
            run[m] = fmaf(sc[gg], fmaf(-zc[gg], xinfo[m * 8 + 4 * eh + 2 * gg].y, acc[m]), run[m]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&dempty[jd]);
          mbar_arrive(&mempty[ms]);
          mbar_arrive(&xiempty[xs]);
        }
      }

      // ---- end of this CTA's piece of row tile b: the two halves of a row
      //      meet, then y or the split-K slot of the piece
      const bool piece_end = (s == g.NS - 1) || (i == ntiles - 1);
      if (piece_end) {
        if (eh == 1) {
#pragma unroll
          for (int m = 0; m < MP; ++m) exch[m] = run[m];
        }
        named_barrier_sync(1 + quad, 64);
        if (eh == 0 && ok) {
          const bool whole = (piece_s0 == 0) && (s == g.NS - 1);
          const int n = b * kTileRows + r;
#pragma unroll
          for (int m = 0; m < MP; ++m) {
            if (m >= prm.M) break;
            const float v = run[m] + exch[m];
            if (whole) {
              if (n < g.N) prm.y[(size_t)m * g.N + n] = v;
            } else {
              prm.partials[((size_t)piece_s0 * MP + m) * g.Npad + n] = v;
            }
          }
        }
        named_barrier_sync(1 + quad, 64);
#pragma unroll
        for (int m = 0; m < MP; ++m) run[m] = 0.0f;
        piece_s0 = -1;
      }
    }
    if (!ok && lane == 0) fail();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(kTgTmemCols)
                 : "memory");
  }
}

template <int MP>
cudaError_t launch_tc(const TgParams& prm, int grid, cudaStream_t stream) {
  auto enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  // The codes of the tiles form one 2-D byte array of 256-byte rows (every
  // slab is full): tile (s, b) starts at row (s NB + b) tile_rows.
  CUtensorMap cmap;
  memset(&cmap, 0, sizeof(cmap));
  const long long rows = (long long)prm.g.NS * prm.g.NB * prm.tile_rows;
  cuuint64_t dims[2] = {(cuuint64_t)(kSlabGroups * kCodeBytesPerGroupRow), (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(kSlabGroups * kCodeBytesPerGroupRow)};
  cuuint32_t box[2] = {128, (cuuint32_t)kTileRows};
  cuuint32_t estr[2] = {1, 1};
  if (enc(&cmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(prm.packed), dims, strides,
          box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const void* fn = reinterpret_cast<const void*>(&gemv_w4a16_tc_kernel<MP>);
  int per_sm = 0;
  cudaError_t e = kernel_setup(fn, TgSmem<MP>::kAlloc, kTgThreads, &per_sm);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  TgParams p = prm;
  void* args[] = {&p, &cmap};
  return launch_pdl(fn, dim3((unsigned)grid), dim3(kTgThreads), args, TgSmem<MP>::kAlloc, stream);
}

// Rows of x padded to the kernel's instances.
int tg_mpad(int M) { return M <= 2 ? 2 : M <= 4 ? 4 : M <= 8 ? 8 : 16; }

// Workspace of the tensor-core path: the split-K counters region (unused) and
// partial sums of the CUDA-core path, then the prepared planes and chunk
// factors of every slab.
struct TgWorkspace {
  size_t partials, planes, xinfo, total;
};

TgWorkspace tg_workspace(int M, int N, int K) {
  const Geom g = make_geom(N, K, 1);
  const int MP = tg_mpad(M);
  auto a256 = [](size_t v) { return (v + 255) / 256 * 256; };
  TgWorkspace w;
  w.partials = kCounterBytes;
  w.planes = w.partials + (g.NS > 1 ? a256((size_t)g.NS * MP * g.Npad * sizeof(float)) : 0);
  w.xinfo = w.planes + (size_t)g.NS * tg_slab_plane_bytes(MP);
  w.total = w.xinfo + a256((size_t)g.NS * MP * 8 * sizeof(float2));
  return w;
}

}  // namespace

// The tensor-core decode path takes M = 2..8 rows of x (with or without the
// AWQ activation factor) on weights whose every slab is full (K a multiple of
// 512).  At M = 1 the CUDA-core kernel is faster: each small MMA (N = 8) costs
// about as much as a large one, so one row of x does not fill the tensor
// cores.
bool gemv_tc_supported(int M, int K) { return M >= 2 && M <= 8 && K % kSlabK == 0; }

// The same kernel serves the tensor-core GEMM entry for M = 1..16.
bool gemm_tc_supported(int M, int K) { return M >= 1 && M <= kTgMaxM && K % kSlabK == 0; }

size_t gemv_tc_workspace_bytes(int M, int N, int K) { return tg_workspace(M, N, K).total; }

cudaError_t launch_gemv_tc(const void* x, const float* inv_s, const void* packed, int M, int N,
                           int K, int sym, float* y, void* workspace, int* err, int num_sms,
                           unsigned long long wait_ns, cudaStream_t stream) {
  const TgWorkspace wl = tg_workspace(M, N, K);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  TgParams prm;
  prm.g = make_geom(N, K, sym);
  prm.packed = static_cast<const uint8_t*>(packed);
  prm.planes = ws + wl.planes;
  prm.xinfo = reinterpret_cast<const float2*>(ws + wl.xinfo);
  prm.y = y;
  prm.partials = reinterpret_cast<float*>(ws + wl.partials);
  prm.err = err;
  prm.M = M;
  prm.MP = tg_mpad(M);
  prm.tile_rows = kTileRows + kTileRows * prm.g.meta / kCodeBytesPerGroupRow;
  prm.tiles = (long long)prm.g.NS * prm.g.NB;
  prm.wait_ns = wait_ns;
  prm.drain_ns = 1000000000ull;
  const int grid = (int)(prm.tiles < num_sms ? prm.tiles : num_sms);
  // the activation planes of every slab, once
  {
    const uint16_t* xp = static_cast<const uint16_t*>(x);
    uint8_t* planes = ws + wl.planes;
    float2* xinfo = reinterpret_cast<float2*>(ws + wl.xinfo);
    int Mv = M, MPv = prm.MP, Kv = K;
    void* args[] = {&xp, &inv_s, &Mv, &MPv, &Kv, &planes, &xinfo};
    cudaError_t e = launch_pdl(reinterpret_cast<const void*>(&gemv_tc_prep_kernel),
                               dim3((unsigned)prm.g.NS), dim3(32 * prm.MP), args, 0, stream);
    if (e != cudaSuccess) return e;
  }
  cudaError_t e;
  switch (prm.MP) {
    case 2: e = launch_tc<2>(prm, grid, stream); break;
    case 4: e = launch_tc<4>(prm, grid, stream); break;
    case 8: e = launch_tc<8>(prm, grid, stream); break;
    default: e = launch_tc<16>(prm, grid, stream); break;
  }
  if (e != cudaSuccess || prm.g.NS <= 1) return e;
  return launch_gemv_finish(prm.partials, y, N, M, prm.MP, prm.g.NS, prm.g.Npad, grid, prm.tiles,
                            stream);
}

}  // namespace wq
