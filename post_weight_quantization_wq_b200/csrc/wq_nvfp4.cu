// wq_nvfp4.cu -- NVFP4 block-scaled 4-bit floating point: E2M1 elements in
// blocks of 16 consecutive inputs, one FP8 E4M3 scale per block and one fp32
// scale per tensor ("3.6 量化(Quantization)", section 数值格式: E2M1 is
// 1 sign / 2 exponent / 1 mantissa bits with magnitudes 0, 0.5, 1, 1.5, 2, 3,
// 4, 6; E4M3 is 1 / 4 / 3 bits with largest value 448; NVFP4 shares one E4M3
// scale among 16 elements plus one fp32 scale per tensor; section 实例演算:
// 4 + 8/16 = 4.5 bits per element).
//
// Quantization of a bf16 matrix A [R][C] (weights or activations), each step
// one correctly rounded fp32 operation:
//   S    = max(amax(A), 1e-8) / (6 * 448)          (tensor scale; the largest
//                                                   block scale lands on 448)
//   sb   = E4M3(amax_block / fl(6 S))               (round to nearest even,
//                                                   saturating at 448; a scale
//                                                   that rounds to 0 becomes
//                                                   the smallest subnormal)
//   q    = E2M1(a / fl(E4M3(sb) S))                 (nearest magnitude, ties to
//                                                   the even code, saturating at
//                                                   6, sign kept)
//   a_hat = E2M1(q) * E4M3(sb) * S.
// Both encoders are written from the formats' definitions (exponent, mantissa
// and rounding rules) with integer and compare operations, so the codes do
// not depend on a hardware conversion's corner cases.
#include <cstring>

#include "wq_common.cuh"
#include "wq_tc.cuh"

namespace wq {

constexpr int kFp4Block = 16;

cudaError_t launch_nvfp4_quantize(const void* A, int R, int C, uint8_t* codes, uint8_t* scales,
                                  float* tensor_scale, int* d_status, int sf_atom,
                                  int num_sms, cudaStream_t stream);

// E2M1 code of v: nearest of the magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 (codes
// 0..7), ties to the even code, saturating at 6; bit 3 is the sign of v (so
// -0 and negative values that round to 0 give code 8).
__device__ __forceinline__ uint32_t e2m1_encode(float v) {
  const float a = fabsf(v);
  uint32_t c;
  if (a <= 0.25f) c = 0;           // tie 0.25 -> 0 (even)
  else if (a < 0.75f) c = 1;
  else if (a <= 1.25f) c = 2;      // ties 0.75 and 1.25 -> 2
  else if (a < 1.75f) c = 3;
  else if (a <= 2.5f) c = 4;       // ties 1.75 and 2.5 -> 4
  else if (a < 3.5f) c = 5;
  else if (a <= 5.0f) c = 6;       // ties 3.5 and 5 -> 6
  else c = 7;
  return c | ((__float_as_uint(v) >> 28) & 8u);
}

// E4M3 code of d >= 0: bias 7, 3 mantissa bits, round to nearest even,
// saturating at 448 (code 0x7E); below 2^-6 the subnormal codes m * 2^-9.
__device__ __forceinline__ uint32_t e4m3_encode(float d) {
  if (!(d < 448.0f)) return 0x7Eu;
  if (d < 0x1p-6f) return (uint32_t)__float2int_rn(d * 512.0f);   // exact scaling; 8 -> 2^-6
  const uint32_t bits = __float_as_uint(d);
  int e = (int)(bits >> 23) - 127;              // -6 .. 8
  uint32_t r = (bits >> 20) & 7u;
  const uint32_t rem = bits & 0xFFFFFu;
  if (rem > 0x80000u || (rem == 0x80000u && (r & 1u))) ++r;
  if (r == 8u) { r = 0; ++e; }
  const uint32_t code = ((uint32_t)(e + 7) << 3) | r;
  return code > 0x7Eu ? 0x7Eu : code;
}

__device__ __forceinline__ float e4m3_decode(uint32_t c) {
  const uint32_t e = (c >> 3) & 15u, m = c & 7u;
  return e == 0 ? (float)m * 0x1p-9f : __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// amax of the whole tensor into *amax_bits (fp32 bits; non-negative floats
// order like their bit patterns), and the count of non-finite elements.
__global__ void __launch_bounds__(256) nvfp4_amax_kernel(const uint16_t* __restrict__ A,
                                                         long long n,
                                                         unsigned* __restrict__ amax_bits,
                                                         int* __restrict__ d_status) {
  float m = 0.0f;
  int bad = 0;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const float v = fabsf(__uint_as_float((uint32_t)A[i] << 16));
    if (!isfinite(v)) ++bad;
    else m = fmaxf(m, v);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    bad += __shfl_xor_sync(0xFFFFFFFFu, bad, o);
  }
  if ((threadIdx.x & 31) == 0) {
    atomicMax(amax_bits, __float_as_uint(m));
    if (bad && d_status) atomicAdd(d_status, bad);
  }
}

// One thread per block of 16 elements: its E4M3 scale and 8 bytes of codes.
// `sf_atom`: write the block scales in the tensor-core scale layout (rows in
// groups of 128, 512-byte blocks per 64 inputs) instead of [R][C/16].
__global__ void __launch_bounds__(256) nvfp4_quantize_kernel(
    const uint16_t* __restrict__ A, int R, int C, const unsigned* __restrict__ amax_bits,
    uint8_t* __restrict__ codes, uint8_t* __restrict__ scales, int sf_atom) {
  const long long nblk = (long long)R * (C / kFp4Block);
  const float amax = __uint_as_float(*amax_bits);
  const float S = __fdiv_rn(fmaxf(amax, 1e-8f), 2688.0f);     // 6 * 448
  const float S6 = __fmul_rn(6.0f, S);
  for (long long bi = blockIdx.x * (long long)blockDim.x + threadIdx.x; bi < nblk;
       bi += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(bi / (C / kFp4Block)), cb = (int)(bi % (C / kFp4Block));
    const uint4* src = reinterpret_cast<const uint4*>(A + (size_t)r * C + (size_t)cb * kFp4Block);
    const uint4 u0 = src[0], u1 = src[1];
    const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
    float v[16];
    float am = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
      am = fmaxf(am, fmaxf(fabsf(v[2 * i]), fabsf(v[2 * i + 1])));
    }
    uint32_t sb = e4m3_encode(__fdiv_rn(am, S6));
    if (sb == 0) sb = 1;
    const float eff = __fmul_rn(e4m3_decode(sb), S);
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      lo |= e2m1_encode(__fdiv_rn(v[i], eff)) << (4 * i);
      hi |= e2m1_encode(__fdiv_rn(v[8 + i], eff)) << (4 * i);
    }
    reinterpret_cast<uint2*>(codes)[bi] = make_uint2(lo, hi);
    if (sf_atom) {
      // row r = 128 t + 32 m1 + m0, inputs 64 kb + 16 ks + ...:
      // byte (t * C/64 + kb) * 512 + m0 * 16 + m1 * 4 + ks
      const int t = r >> 7, m1 = (r >> 5) & 3, m0 = r & 31;
      const int kb = cb >> 2, ks = cb & 3;
      scales[((size_t)t * (C / 64) + kb) * 512 + m0 * 16 + m1 * 4 + ks] = (uint8_t)sb;
    } else {
      scales[bi] = (uint8_t)sb;
    }
  }
}

// amax bits -> S in place.
__global__ void nvfp4_finish_scale_kernel(unsigned* amax_bits) {
  const float amax = __uint_as_float(*amax_bits);
  *reinterpret_cast<float*>(amax_bits) = __fdiv_rn(fmaxf(amax, 1e-8f), 2688.0f);
}

// ---- activations of the W4A4 linear: the same quantizer in two kernels
// with no memset, launched as programmatic dependents so that the FP4 GEMM
// behind them can start loading weights while x is quantized.
constexpr int kActAmaxCtas = 148;            // CTAs of the amax pass (at most)

// Per-CTA largest finite |x| into partial[blockIdx.x] (non-finite values are
// left out, as in the tensor quantizer).
__global__ void __launch_bounds__(256) nvfp4_act_amax_kernel(const uint16_t* __restrict__ A,
                                                             long long n,
                                                             float* __restrict__ partial) {
  griddep_launch_dependents();
  griddep_wait();                              // x may come from the previous kernel
  __shared__ float red[8];
  float m = 0.0f;
  const long long n8 = n / 8;                  // n is a multiple of 16
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n8;
       i += (long long)gridDim.x * blockDim.x) {
    const uint4 u = reinterpret_cast<const uint4*>(A)[i];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float a = fabsf(__uint_as_float(w[q] << 16));
      const float b = fabsf(__uint_as_float(w[q] & 0xFFFF0000u));
      if (a <= 3.402823466e38f) m = fmaxf(m, a);
      if (b <= 3.402823466e38f) m = fmaxf(m, b);
    }
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = red[0];
    for (int w = 1; w < 8; ++w) t = fmaxf(t, red[w]);
    partial[blockIdx.x] = t;
  }
}

// Every CTA reduces the partial maxima to S (reading F3; CTA 0 stores it),
// then quantizes as nvfp4_quantize_kernel does with the block scales in the
// tensor-core layout, and writes zero scales for the padding rows [R, RP)
// of the activation tile (finite, so that 0-coded padding rows stay 0).
__global__ void __launch_bounds__(256) nvfp4_act_quantize_kernel(
    const uint16_t* __restrict__ A, int R, int RP, int C, const float* __restrict__ partial,
    int np, uint8_t* __restrict__ codes, uint8_t* __restrict__ scales, float* __restrict__ s_out) {
  griddep_launch_dependents();
  griddep_wait();                              // the partial maxima are complete
  __shared__ float red[8];
  float m = 0.0f;
  for (int i = threadIdx.x; i < np; i += blockDim.x) m = fmaxf(m, partial[i]);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  float amax = red[0];
  for (int w = 1; w < 8; ++w) amax = fmaxf(amax, red[w]);
  const float S = __fdiv_rn(fmaxf(amax, 1e-8f), 2688.0f);     // 6 * 448
  const float S6 = __fmul_rn(6.0f, S);
  if (blockIdx.x == 0 && threadIdx.x == 0) *s_out = S;
  const int CB = C / kFp4Block;
  const long long nblk = (long long)R * CB;
  const long long npad = (long long)(RP - R) * CB;
  for (long long bi = blockIdx.x * (long long)blockDim.x + threadIdx.x; bi < nblk + npad;
       bi += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(bi / CB), cb = (int)(bi % CB);
    uint32_t sb = 0;
    if (bi < nblk) {
      const uint4* src = reinterpret_cast<const uint4*>(A + (size_t)r * C + (size_t)cb * kFp4Block);
      const uint4 u0 = src[0], u1 = src[1];
      const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
      float v[16];
      float am = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        am = fmaxf(am, fmaxf(fabsf(v[2 * i]), fabsf(v[2 * i + 1])));
      }
      sb = e4m3_encode(__fdiv_rn(am, S6));
      if (sb == 0) sb = 1;
      const float eff = __fmul_rn(e4m3_decode(sb), S);
      uint32_t lo = 0, hi = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        lo |= e2m1_encode(__fdiv_rn(v[i], eff)) << (4 * i);
        hi |= e2m1_encode(__fdiv_rn(v[8 + i], eff)) << (4 * i);
      }
      reinterpret_cast<uint2*>(codes)[bi] = make_uint2(lo, hi);
    }
    const int t = r >> 7, m1 = (r >> 5) & 3, m0 = r & 31;
    const int kb = cb >> 2, ks = cb & 3;
    scales[((size_t)t * (C / 64) + kb) * 512 + m0 * 16 + m1 * 4 + ks] = (uint8_t)sb;
  }
}

// Canonical block scales [N][K/16] -> the tensor-core scale layout.
__global__ void nvfp4_sf_relayout_kernel(const uint8_t* __restrict__ sf, int N, int K,
                                         uint8_t* __restrict__ out) {
  const int NBt = (N + 127) / 128;
  const long long total = (long long)NBt * (K / 64) * 512;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int blk = (int)(e / 512), off = (int)(e % 512);
    const int t = blk / (K / 64), kb = blk % (K / 64);
    const int m0 = off / 16, m1 = (off / 4) & 3, ks = off & 3;
    const int r = t * 128 + m1 * 32 + m0;
    out[e] = r < N ? sf[(size_t)r * (K / 16) + kb * 4 + ks] : (uint8_t)0;
  }
}

// ------------------------------------------------------------------ W4A4 linear
// y = dequant(x) dequant(W)^T with both operands NVFP4, on the block-scaled
// FP4 tensor cores (tcgen05.mma kind::mxf4nvf4, 16-element blocks with E4M3
// scales): per 64 inputs one MMA of M = 128 weight rows x N = MPAD activation
// rows; the block scales of both operands are copied from shared memory into
// tensor memory (tcgen05.cp) next to the fp32 accumulator; the tensor scales
// S_w S_x are applied once at the end.  The work is the sequence of (128-row
// tile of W, 256-input stage) pairs, tile-major; G persistent CTAs each take
// one contiguous share of it (stream-K), so a CTA ends one tile's piece and
// starts the next without a new launch, and every SM gets the same number of
// stages.  The partial sums of the pieces of a tile are added in CTA order by
// a small second kernel.

struct Fp4GemmParams {
  const uint8_t* w_sf;     // weight scale blocks [ceil(N/128)][K/64][512]
  const uint8_t* x_sf;     // activation scale blocks [K/64][512]
  float* partials;         // fp32 [tiles][P][MPAD][128] raw sums (no tensor scales)
  int* err;
  int N, K, M, KT, G, P;   // KT stages per tile, G CTAs, P pieces per tile at most
  unsigned long long wait_ns, drain_ns;
};

constexpr int kFp4StageK = 256;             // inputs per stage: 128 bytes per row
constexpr int kFp4Threads = 6 * 32;         // TMA producer, MMA issuer, 4 epilogue warps
constexpr uint32_t kFp4TmemCols = 512;

template <int MPAD>
struct Fp4Smem {
  static constexpr int kStages = MPAD <= 32 ? 8 : (MPAD <= 64 ? 6 : 5);
  static constexpr int kA = 128 * 128;                  // codes of 128 weight rows
  static constexpr int kB = MPAD * 128;                 // codes of MPAD activation rows
  static constexpr int kSF = 4 * 512;                   // 4 scale blocks of 64 inputs
  static constexpr int kStage = kA + kB + 2 * kSF;      // multiple of 1024
  static constexpr int kBar = kStages * kStage;
  static constexpr int kBytes = kBar + (2 * kStages + 4) * 8 + 16;
  static constexpr int kAlloc = kBytes + 1024;
  static constexpr int kSfCol = 2 * MPAD;               // scale columns after the 2 accumulators
  static_assert(kSfCol + kStages * 32 <= (int)kFp4TmemCols, "tensor memory");
};

// Instruction descriptor of kind::mxf4nvf4: E2M1 A and B (K-major), UE4M3
// scales, M = 128, N = MPAD, dense K = 64.
template <int MPAD>
__host__ __device__ constexpr uint32_t fp4_idesc() {
  return (1u << 7) | (1u << 10) | ((uint32_t)(MPAD >> 3) << 17) | (0u << 23) | ((128u >> 4) << 24);
}

// Shared-memory descriptor of one 512-byte scale block: 32 rows of 16 bytes,
// no swizzle (8-row core matrices 128 bytes apart).
__device__ __forceinline__ uint64_t sf_block_desc(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)(16 >> 4) << 16) |
         ((uint64_t)(128 >> 4) << 32) | ((uint64_t)1 << 46);
}

// 32 rows x 128 bits of shared memory into tensor-memory lanes 0..31 (and, by
// the warpx4 broadcast, 32..63, 64..95, 96..127), 4 columns.
__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t desc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(desc)
               : "memory");
}

__device__ __forceinline__ void umma_fp4(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate, uint32_t tsfa,
                                         uint32_t tsfb) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], "
      "p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb)
      : "memory");
}

// Persistent: CTA c takes the units (row tile, K split) c, c + grid, ... in
// order; the TMA ring runs on across units, and the accumulator is double
// buffered in tensor memory so the epilogue of one unit overlaps the MMAs of
// the next.
template <int MPAD>
__global__ void __launch_bounds__(kFp4Threads, 1)
    nvfp4_gemm_kernel(const Fp4GemmParams p, const __grid_constant__ CUtensorMap wmap,
                      const __grid_constant__ CUtensorMap xmap) {
  using SM = Fp4Smem<MPAD>;
  constexpr int S = SM::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SM::kBar);
  uint64_t* empty = full + S;
  uint64_t* accfull = empty + S;        // [2]
  uint64_t* accempty = accfull + 2;     // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accempty + 2);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KB = p.K / 64;                    // scale blocks along K
  const long long T = (long long)((p.N + 127) / 128) * p.KT;   // stages in all
  const long long g0 = (long long)blockIdx.x * T / p.G;          // this CTA's share
  const long long g1 = (long long)(blockIdx.x + 1) * T / p.G;
  const int b_first = (int)(g0 / p.KT);
  const int b_end = (int)((g1 - 1) / p.KT) + 1;
  // stages [s0, s1) of tile b that fall in this CTA's share
  auto piece = [&](int b, int& s0, int& s1) {
    const long long lo = (long long)b * p.KT, hi = lo + p.KT;
    s0 = (int)((g0 > lo ? g0 : lo) - lo);
    s1 = (int)((g1 < hi ? g1 : hi) - lo);
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&accfull[i], 1);
      mbar_init(&accempty[i], 4);
    }
    fence_mbarrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kFp4TmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // Weights never come from an earlier kernel of the stream: the first S
    // stages' weight codes and scales are requested before waiting for the
    // kernel that quantizes the activations, their activation parts after.
    auto issue = [&](int st, int b, int sg, bool wpart, bool xpart) {
      const int kb0 = 4 * sg;
      const int nkb = KB - kb0 < 4 ? KB - kb0 : 4;
      if (elect_one()) {
        uint8_t* sa = smem + st * SM::kStage;
        const uint32_t sfb = (uint32_t)nkb * 512u;
        if (wpart) {
          mbar_arrive_expect_tx(&full[st], (uint32_t)(SM::kA + SM::kB) + 2u * sfb);
          tma_load_2d(sa, &wmap, sg * 128, b * 128, &full[st]);
          bulk_copy_g2s(sa + SM::kA + SM::kB, p.w_sf + ((size_t)b * KB + kb0) * 512, sfb,
                        &full[st]);
        }
        if (xpart) {
          tma_load_2d(sa + SM::kA, &xmap, sg * 128, 0, &full[st]);
          bulk_copy_g2s(sa + SM::kA + SM::kB + SM::kSF, p.x_sf + (size_t)kb0 * 512, sfb,
                        &full[st]);
        }
      }
      __syncwarp();
    };
    int npre = 0;
    {
      int b = b_first, s0 = 0, s1 = 0;
      if (b < b_end) piece(b, s0, s1);
      for (int sg = s0; npre < S && b < b_end; ++npre) {
        issue(npre, b, sg, true, false);
        if (++sg == s1 && ++b < b_end) {
          piece(b, s0, s1);
          sg = s0;
        }
      }
    }
    griddep_wait();                         // the activations' codes and scales are complete
    int i = 0;                              // stages issued by this CTA
    bool ok = true;
    for (int b = b_first; b < b_end && ok; ++b) {
      int s0, s1;
      piece(b, s0, s1);
      for (int sg = s0; sg < s1; ++sg, ++i) {
        const int st = i % S;
        if (i < npre) {
          issue(st, b, sg, false, true);
          continue;
        }
        ok = warp_wait(&empty[st], ((i / S) - 1) & 1, p.wait_ns);
        if (!ok) break;
        issue(st, b, sg, true, true);
      }
    }
    if (!ok) {
      if (lane == 0) atomicOr(p.err, kDevErrTimeout);
      for (int k = i - S < 0 ? 0 : i - S; k < i; ++k)
        warp_wait(&full[k % S], (k / S) & 1, p.drain_ns);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc = fp4_idesc<MPAD>();
    bool ok = true;
    int i = 0, lu = 0;
    for (int b = b_first; b < b_end && ok; ++b, ++lu) {
      int s0, s1;
      piece(b, s0, s1);
      const int db = lu & 1;
      if (lu >= 2) ok = warp_wait(&accempty[db], ((lu / 2) - 1) & 1, p.wait_ns);
      if (!ok) break;
      for (int sg = s0; sg < s1; ++sg, ++i) {
        const int st = i % S;
        ok = warp_wait(&full[st], (i / S) & 1, p.wait_ns);
        if (!ok) break;
        tc_fence_after();
        const int kb0 = 4 * sg;
        const int nkb = KB - kb0 < 4 ? KB - kb0 : 4;
        if (elect_one()) {
          const uint32_t sa = smem_u32(smem + st * SM::kStage);
          const uint32_t tsf = tmem_base + SM::kSfCol + st * 32;
          for (int kk = 0; kk < nkb; ++kk) {
            tmem_cp_sf(tsf + kk * 4, sf_block_desc(sa + SM::kA + SM::kB + kk * 512));
            tmem_cp_sf(tsf + 16 + kk * 4,
                       sf_block_desc(sa + SM::kA + SM::kB + SM::kSF + kk * 512));
          }
          for (int kk = 0; kk < nkb; ++kk)
            umma_fp4(tmem_base + db * MPAD, umma_desc_sw128(sa + kk * 32),
                     umma_desc_sw128(sa + SM::kA + kk * 32), idesc,
                     (sg > s0 || kk > 0) ? 1u : 0u, tsf + kk * 4, tsf + 16 + kk * 4);
          umma_commit(&empty[st]);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (elect_one()) umma_commit(&accfull[db]);
      __syncwarp();
    }
    if (!ok) {
      if (lane == 0) atomicOr(p.err, kDevErrTimeout);
      if (i > 0) warp_wait(&empty[(i - 1) % S], ((i - 1) / S) & 1, p.drain_ns);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                  // tensor-memory lane quadrant of this warp
    griddep_wait();                          // the partial sums may still be read by an earlier kernel
    int lu = 0;
    for (int b = b_first; b < b_end; ++b, ++lu) {
      const int db = lu & 1;
      // piece index: this CTA's rank among the CTAs that share tile b
      const long long s = (long long)b * p.KT;
      const int c_first = (int)(((s + 1) * p.G - 1) / T);
      float* out = p.partials +
                   ((size_t)b * p.P + (size_t)(blockIdx.x - c_first)) * MPAD * 128;
      if (!warp_wait(&accfull[db], (lu / 2) & 1, p.wait_ns)) {
        if (lane == 0) atomicOr(p.err, kDevErrTimeout);
        break;
      }
      tc_fence_after();
      const int nl = q * 32 + lane;
#pragma unroll
      for (int c = 0; c < MPAD; c += 8) {
        float v[8];
        tmem_ld8(tmem_base + ((uint32_t)(q * 32) << 16) + db * MPAD + c, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (c + j < p.M) out[(size_t)(c + j) * 128 + nl] = v[j];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[db]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(kFp4TmemCols)
                 : "memory");
  }
}

// y[m][n] = (sum of the pieces of tile n / 128, in CTA order) * S_w * S_x.
__global__ void nvfp4_finish_kernel(const float* __restrict__ partials, int KT, int G, int P,
                                    int MPAD, int M, int N, const float* __restrict__ s_w,
                                    const float* __restrict__ s_x, float* __restrict__ y) {
  griddep_launch_dependents();
  griddep_wait();                      // the GEMM's partial sums are complete
  const long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (e >= (long long)M * N) return;
  const int m = (int)(e / N), n = (int)(e % N);
  const int b = n / 128;
  const long long T = (long long)((N + 127) / 128) * KT;
  const long long s_lo = (long long)b * KT, s_hi = s_lo + KT - 1;
  const int c_first = (int)(((s_lo + 1) * G - 1) / T);
  const int c_last = (int)(((s_hi + 1) * G - 1) / T);
  const float* src = partials + ((size_t)b * P * MPAD + m) * 128 + (n & 127);
  // every piece's load before the additions (in CTA order): one L2 round trip
  // per batch of pieces
  constexpr int kBatch = 8;
  float t = 0.0f;
  for (int c0 = 0; c0 <= c_last - c_first; c0 += kBatch) {
    float v[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; ++j)
      v[j] = c0 + j <= c_last - c_first ? src[(size_t)(c0 + j) * MPAD * 128] : 0.0f;
#pragma unroll
    for (int j = 0; j < kBatch; ++j)
      if (c0 + j <= c_last - c_first) t += v[j];
  }
  y[e] = t * (*s_w * *s_x);
}

static int fp4_mpad(int M) { return M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128; }

// The stream-K share count G is that of a 148-SM GPU whatever the device, so
// the workspace size and the order of the final additions are functions of
// the shape alone (on a smaller GPU the extra CTAs wait for a free SM).
constexpr int kFp4SplitSms = 148;

struct Fp4Split {
  int G, P;
};

// G = min(148, stages); P = the largest number of CTAs whose shares meet one tile.
static Fp4Split fp4_split(int NBt, int KT) {
  const long long T = (long long)NBt * KT;
  Fp4Split sp;
  sp.G = (int)(T < kFp4SplitSms ? T : kFp4SplitSms);
  sp.P = 1;
  for (int b = 0; b < NBt; ++b) {
    const long long s_lo = (long long)b * KT, s_hi = s_lo + KT - 1;
    const int c_first = (int)(((s_lo + 1) * sp.G - 1) / T);
    const int c_last = (int)(((s_hi + 1) * sp.G - 1) / T);
    if (c_last - c_first + 1 > sp.P) sp.P = c_last - c_first + 1;
  }
  return sp;
}

size_t nvfp4_linear_workspace_bytes(int M, int N, int K) {
  const int NBt = (N + 127) / 128;
  const int KT = (K + kFp4StageK - 1) / kFp4StageK;
  const Fp4Split sp = fp4_split(NBt, KT);
  auto a256 = [](size_t v) { return (v + 255) / 256 * 256; };
  return a256((size_t)M * K / 2) + a256((size_t)(K / 64) * 512) + a256(16 + 4 * kActAmaxCtas) +
         a256((size_t)NBt * sp.P * fp4_mpad(M) * 128 * 4);
}

template <int MPAD>
static cudaError_t launch_fp4_gemm(const Fp4GemmParams& prm, const uint8_t* w_codes,
                                   const uint8_t* x_codes, cudaStream_t stream) {
  using SM = Fp4Smem<MPAD>;
  auto enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap wmap, xmap;
  memset(&wmap, 0, sizeof(wmap));
  memset(&xmap, 0, sizeof(xmap));
  {
    cuuint64_t dims[2] = {(cuuint64_t)prm.K / 2, (cuuint64_t)prm.N};
    cuuint64_t strides[1] = {(cuuint64_t)prm.K / 2};
    cuuint32_t box[2] = {128, 128};
    cuuint32_t estr[2] = {1, 1};
    if (enc(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(w_codes), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    cuuint64_t dims[2] = {(cuuint64_t)prm.K / 2, (cuuint64_t)prm.M};
    cuuint64_t strides[1] = {(cuuint64_t)prm.K / 2};
    cuuint32_t box[2] = {128, (cuuint32_t)MPAD};
    cuuint32_t estr[2] = {1, 1};
    if (enc(&xmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(x_codes), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const void* fn = reinterpret_cast<const void*>(&nvfp4_gemm_kernel<MPAD>);
  int per_sm = 0;
  cudaError_t e = kernel_setup(fn, SM::kAlloc, kFp4Threads, &per_sm);
  if (e != cudaSuccess) return e;
  Fp4GemmParams pp = prm;
  void* args[] = {&pp, &wmap, &xmap};
  return launch_pdl(fn, dim3((unsigned)prm.G), dim3(kFp4Threads), args, SM::kAlloc, stream);
}

cudaError_t launch_nvfp4_linear(const void* x, const uint8_t* packed, const float* w_scale, int M,
                                int N, int K, float* y, void* workspace, int* err, int num_sms,
                                unsigned long long wait_ns, cudaStream_t stream) {
  const int NBt = (N + 127) / 128;
  const int KT = (K + kFp4StageK - 1) / kFp4StageK;
  auto a256 = [](size_t v) { return (v + 255) / 256 * 256; };
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* x_codes = ws;
  uint8_t* x_sf = x_codes + a256((size_t)M * K / 2);
  float* s_x = reinterpret_cast<float*>(x_sf + a256((size_t)(K / 64) * 512));
  float* amax_part = s_x + 4;
  float* partials =
      reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(s_x) + a256(16 + 4 * kActAmaxCtas));
  // the activations in NVFP4 (their block scales in the tensor-core layout):
  // per-CTA maxima, then the quantizer; each a programmatic dependent of the
  // kernel before it
  cudaError_t e;
  {
    const uint16_t* xp = static_cast<const uint16_t*>(x);
    long long n = (long long)M * K;
    long long ga = (n / 8 + 255) / 256;
    if (ga > kActAmaxCtas) ga = kActAmaxCtas;
    void* args[] = {&xp, &n, &amax_part};
    if ((e = launch_pdl(reinterpret_cast<const void*>(&nvfp4_act_amax_kernel), dim3((unsigned)ga),
                        dim3(256), args, 0, stream)) != cudaSuccess)
      return e;
    int R = M, RP = fp4_mpad(M), C = K, np = (int)ga;
    const long long work = (long long)RP * (K / kFp4Block);
    long long gq = (work + 255) / 256;
    if (gq > (long long)num_sms * 4) gq = (long long)num_sms * 4;
    uint8_t* codes = x_codes;
    uint8_t* scales = x_sf;
    const float* partp = amax_part;
    float* sout = s_x;
    void* qargs[] = {&xp, &R, &RP, &C, &partp, &np, &codes, &scales, &sout};
    if ((e = launch_pdl(reinterpret_cast<const void*>(&nvfp4_act_quantize_kernel),
                        dim3((unsigned)gq), dim3(256), qargs, 0, stream)) != cudaSuccess)
      return e;
  }
  Fp4GemmParams prm;
  prm.w_sf = packed + (size_t)N * K / 2;
  prm.x_sf = x_sf;
  prm.partials = partials;
  prm.err = err;
  prm.N = N;
  prm.K = K;
  prm.M = M;
  prm.KT = KT;
  const Fp4Split sp = fp4_split(NBt, KT);
  prm.G = sp.G;
  prm.P = sp.P;
  prm.wait_ns = wait_ns;
  prm.drain_ns = 1000000000ull;
  switch (fp4_mpad(M)) {
    case 16: e = launch_fp4_gemm<16>(prm, packed, x_codes, stream); break;
    case 32: e = launch_fp4_gemm<32>(prm, packed, x_codes, stream); break;
    case 64: e = launch_fp4_gemm<64>(prm, packed, x_codes, stream); break;
    default: e = launch_fp4_gemm<128>(prm, packed, x_codes, stream); break;
  }
  if (e != cudaSuccess) return e;
  const long long outs = (long long)M * N;
  const float* pp = partials;
  int KTv = KT, Gv = prm.G, Pv = prm.P, MPv = fp4_mpad(M), Mv = M, Nv = N;
  const float* swp = w_scale;
  const float* sxp = s_x;
  void* fargs[] = {&pp, &KTv, &Gv, &Pv, &MPv, &Mv, &Nv, &swp, &sxp, &y};
  return launch_pdl(reinterpret_cast<const void*>(&nvfp4_finish_kernel),
                    dim3((unsigned)((outs + 255) / 256)), dim3(256), fargs, 0, stream);
}

cudaError_t launch_nvfp4_quantize(const void* A, int R, int C, uint8_t* codes, uint8_t* scales,
                                  float* tensor_scale, int* d_status, int sf_atom,
                                  int num_sms, cudaStream_t stream) {
  cudaError_t e;
  if ((e = cudaMemsetAsync(tensor_scale, 0, sizeof(float), stream)) != cudaSuccess) return e;
  if (d_status && (e = cudaMemsetAsync(d_status, 0, sizeof(int), stream)) != cudaSuccess) return e;
  if (sf_atom) {
    const size_t sfb = (size_t)((R + 127) / 128) * (C / 64) * 512;
    if ((e = cudaMemsetAsync(scales, 0, sfb, stream)) != cudaSuccess) return e;
  }
  const long long n = (long long)R * C;
  unsigned* amax = reinterpret_cast<unsigned*>(tensor_scale);
  long long g = (n + 255) / 256;
  if (g > (long long)num_sms * 8) g = (long long)num_sms * 8;
  nvfp4_amax_kernel<<<(unsigned)g, 256, 0, stream>>>(static_cast<const uint16_t*>(A), n, amax,
                                                     d_status);
  const long long nblk = n / kFp4Block;
  long long gq = (nblk + 255) / 256;
  if (gq > (long long)num_sms * 16) gq = (long long)num_sms * 16;
  nvfp4_quantize_kernel<<<(unsigned)gq, 256, 0, stream>>>(static_cast<const uint16_t*>(A), R, C,
                                                          amax, codes, scales, sf_atom);
  nvfp4_finish_scale_kernel<<<1, 1, 0, stream>>>(amax);
  return cudaGetLastError();
}

cudaError_t launch_nvfp4_sf_relayout(const uint8_t* sf, int N, int K, uint8_t* out,
                                     cudaStream_t stream) {
  nvfp4_sf_relayout_kernel<<<1024, 256, 0, stream>>>(sf, N, K, out);
  return cudaGetLastError();
}

}  // namespace wq
