// wq_gemv.cu -- W4A16 decode linear for M = 1..8 activation rows on the CUDA
// cores:  y[m][n] = sum_g s16[n][g] * sum_{k in g} x'[m][k] * (q[n][k] - z[n][g]).
// (wq_gemv_w4a16 runs it at M = 1, and at every M whose K is not a multiple of
// 512; the int8 tensor-core kernel of wq_gemv_tc.cu takes the other shapes.)
//
// Weight-only 4-bit decode is bound by the bytes of the weights ("推理优化中
// “用精度换性能“的核心技术：量化", section 一; "3.6 量化(Quantization)",
// section 为什么重要): the weights are dequantized in registers inside the
// matmul kernel and multiplied with 16-bit activations, accumulating in fp32
// ("3.6 量化(Quantization)", section 仅权重 vs 权重 + 激活; "大模型量化全景解析",
// section dtype、storage dtype、compute dtype).
//
// Design (B200, sm_100a):
//   * persistent grid of one CTA per SM holding 1..3 teams (a producer warp
//     and eight consumer warps each, with their own shared memory); team t
//     owns the contiguous run [t0, t1) of the tile sequence u = b * NS + s
//     (row tile b of 128 output rows, K-slab s of 512 inputs), so it walks
//     the slabs of one row tile after another and keeps each row's running
//     sum in registers;
//   * the producer streams every tile (32 KB of nibbles + its fp16 metadata,
//     contiguous in memory) into a ring of shared-memory stages with one 1-D
//     bulk async copy (cp.async.bulk) completing on an mbarrier, and prepares
//     the tile's activation slab once for the team: 16-bit fixed-point x
//     (split into high and low bytes) plus the sum of x per 64 inputs
//     (integer path), or fp32 x * (1/s) (packed path);
//   * programmatic dependent launch: the first weight tiles are requested
//     before the kernel waits for the previous kernel of the stream;
//   * dequantization in registers without conversion instructions.  Integer
//     path (M <= 4): the producer rounds each 64-input chunk of u = x (or
//     u = fp32(x) * (1/s) with the AWQ factor, a separate kernel instance) to
//     integers x_i = rn(u * 2^e), e putting the chunk's largest |u| in
//     [2^14, 2^15); two masks per code word leave the 8 codes in place
//     as bytes (q or 16 q), and four dp4a per word and row of x (unsigned code
//     bytes times signed high / unsigned low activation bytes, int32
//     accumulators) give sum q x_i exactly; each (row, chunk) sum then loses
//     z * sum x_i and is scaled by s16 * 2^-e in fp32.  Packed path
//     (M = 5..8): bf16 pairs 128 + q (mask into 0x43004300) are widened to
//     the fp32 code q - z by a mixed-precision add and packed fp32x2 FMAs
//     multiply them with the fp32 activations;
//   * 8 lanes share a row of a tile, lane p covering inputs 64p..64p+63 of
//     the slab; each lane accumulates its own partial sums over the tiles of
//     a piece, and the lanes of a row are combined once per piece with a
//     transposing shuffle reduction;
//   * a row tile whose slabs are split between teams (only at the ends of a
//     team's run) is finished through the workspace: each piece stores its
//     fp32 partial sums and moves on, and a small second kernel (launched as
//     a programmatic dependent, so it is resident before this one ends and
//     overlaps the next linear's first weight loads) adds the pieces in slab
//     order, so y does not depend on the order the GPU runs the teams in.
//     The streaming kernel itself never waits on another team: no fence,
//     counter or partial-sum load sits on its critical path;
//   * every wait is bounded (globaltimer): on timeout the kernel records the
//     device error word, stops issuing copies, waits (bounded) for its copies
//     in flight and returns.
#include <type_traits>

#include "wq_common.cuh"

namespace wq {

struct GemvParams {
  const uint8_t* packed;
  const uint16_t* x;       // bf16 [M][K]
  const float* inv_s;      // fp32 [K] or nullptr
  float* y;                // fp32 [M][N]
  float* partials;         // fp32 [NS][MP][Npad]
  int* err;                // device error word
  Geom g;
  int M;                   // rows of x / y (<= MP)
  long long tiles;         // NS * NB
  unsigned long long wait_ns;
  unsigned long long drain_ns;
  // Masks and exponent patterns of the code extraction, passed at run time so
  // that each extraction is one 3-register LOP3 instead of two immediate ops.
  uint32_t lop_mask_lo, lop_bf16_128;
};

constexpr int kConsumerWarps = 8;
// per team: 8 consumer warps, the activation producer, the weight producer
constexpr int kGemvThreads = (kConsumerWarps + 2) * 32;
constexpr int kMaxFullTile = kTileRows * kSlabGroups * (kCodeBytesPerGroupRow + 4);
constexpr int kLaneK = 64;                          // inputs of one row per lane
constexpr int kChunks = kSlabK / kLaneK;            // 8 lanes per row
constexpr int kXbChunk = kLaneK * 2 + 16;           // 2 activation bytes per input + pad (conflict-free)
constexpr int kXfChunk = kLaneK * 4 + 16;           // fp32 chunk + pad

// A weight stage holds one tile (codes + metadata, kMaxFullTile bytes); the
// prepared activations of a tile live in a slot of a separate ring, so a
// stage can be refilled as soon as the consumers have its codes in registers.
template <int MP, bool IDOT>
struct StageLayout {
  static constexpr int kBytes = kMaxFullTile;       // one weight stage
  static constexpr int kX = 0;                      // activations within an x slot
  static constexpr int kXRow = kChunks * (IDOT ? kXbChunk : kXfChunk);
  static constexpr int kXsum = kX + MP * kXRow;     // integer path: float4 [MP][8] chunk info
  static constexpr int kXSlot = kXsum + (IDOT ? MP * kChunks * 16 : 0);
  // raw activation slot: bf16 [MP][512], then fp32 [512] of the AWQ factor
  static constexpr int kRawInv = MP * kSlabK * 2;
  static constexpr int kRawBytes = kRawInv + (IDOT ? 0 : kSlabK * 4);
};

// Sum v[] over the L lanes (L = 8 or 16, lane index p) of a lane group.
// Afterwards, for V >= L a lane holds V/L sums, v[i] being the sum of index
// i + (V/L)*p; for V < L a lane holds one sum, of index p >> (log2 L - log2 V).
template <int V, int L>
__device__ __forceinline__ void group_transpose_reduce(float (&v)[V], int p) {
  int C = V;
#pragma unroll
  for (int mk = L / 2; mk >= 1; mk >>= 1) {
    if (C >= 2) {
      const bool upper = (p & mk) != 0;
#pragma unroll
      for (int i = 0; i < V / 2; ++i) {
        if (i < C / 2) {
          const float send = upper ? v[i] : v[i + C / 2];
          const float keep = upper ? v[i + C / 2] : v[i];
          v[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, mk);
        }
      }
      C >>= 1;
    } else {
      v[0] += __shfl_xor_sync(0xFFFFFFFFu, v[0], mk);
    }
  }
}

__host__ __device__ constexpr int ilog2c(int v) { return v <= 1 ? 0 : 1 + ilog2c(v / 2); }

template <int V, int L>
struct GroupMap {
  static constexpr int kPerLane = (V >= L) ? V / L : 1;
  static constexpr int kShift = (V >= L) ? 0 : ilog2c(L) - ilog2c(V);
  __device__ static bool writer(int p) { return V >= L || (p & ((1 << kShift) - 1)) == 0; }
  __device__ static int index(int i, int p) { return V >= L ? i + kPerLane * p : (p >> kShift); }
};

// (a & b) | c in one LOP3 with all three operands in registers.
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

struct LopConsts {
  uint32_t mlo, b128;   // 0x000F000F 0x43004300
};

// Two bf16 values 128 + q of the nibble slots at bits [4i, 4i+4) and
// [16+4i, 20+4i) of w, i.e. inputs 2i and 2i+1 of an interleaved word (exact:
// 128..143 are bf16 integers).
__device__ __forceinline__ uint32_t nib_pair(uint32_t w, int i, const LopConsts& k) {
  return and_or(w >> (4 * i), k.mlo, k.b128);
}

// Integer dot products of the 8 codes of one (interleaved) word with the
// 16-bit fixed-point activations of its inputs, four bytes at a time: the
// low nibbles masked in place are the codes of inputs 0, 4, 1, 5 as bytes,
// the high nibbles masked in place are 16 x the codes of inputs 2, 6, 3, 7.
// xw holds the matching activation bytes: (high bytes of inputs 0, 4, 1, 5),
// (high bytes of 2, 6, 3, 7), then the low bytes in the same two orders.
//   a[0] += sum q h (low nibbles), a[1] += 16 sum q h (high nibbles),
//   a[2] += sum q l, a[3] += 16 sum q l,
// so sum_k q_k x_k = 256 (a[0] + a[1] / 16) + a[2] + a[3] / 16, exactly.
__device__ __forceinline__ void dp4a_word(uint32_t w, const uint4& xw, int (&a)[4]) {
  const uint32_t lo = w & 0x0F0F0F0Fu;
  const uint32_t hi = w & 0xF0F0F0F0u;
  asm("dp4a.u32.s32 %0, %4, %6, %0;\n\t"
      "dp4a.u32.s32 %1, %5, %7, %1;\n\t"
      "dp4a.u32.u32 %2, %4, %8, %2;\n\t"
      "dp4a.u32.u32 %3, %5, %9, %3;"
      : "+r"(a[0]), "+r"(a[1]), "+r"(a[2]), "+r"(a[3])
      : "r"(lo), "r"(hi), "r"(xw.x), "r"(xw.y), "r"(xw.z), "r"(xw.w));
}

// The 8 codes of one (interleaved) word as exact fp32 (q - z) pairs, in input
// order: f32(128 + q) + cz with cz = -(128 + z), by the mixed-precision add.
// nib_pair(w, i) holds the adjacent inputs (2i, 2i+1).
__device__ __forceinline__ void widen_word(uint32_t w, float cz, float2& d01, float2& d23,
                                           float2& d45, float2& d67, const LopConsts& k) {
  const uint32_t v0 = nib_pair(w, 0, k), v1 = nib_pair(w, 1, k), v2 = nib_pair(w, 2, k),
                 v3 = nib_pair(w, 3, k);
  asm("{\n\t.reg .b16 q0, q1, q2, q3, q4, q5, q6, q7;\n\t"
      "mov.b32 {q0, q1}, %8;\n\tmov.b32 {q2, q3}, %9;\n\t"
      "mov.b32 {q4, q5}, %10;\n\tmov.b32 {q6, q7}, %11;\n\t"
      "add.rn.f32.bf16 %0, q0, %12;\n\tadd.rn.f32.bf16 %1, q1, %12;\n\t"
      "add.rn.f32.bf16 %2, q2, %12;\n\tadd.rn.f32.bf16 %3, q3, %12;\n\t"
      "add.rn.f32.bf16 %4, q4, %12;\n\tadd.rn.f32.bf16 %5, q5, %12;\n\t"
      "add.rn.f32.bf16 %6, q6, %12;\n\tadd.rn.f32.bf16 %7, q7, %12;\n\t}"
      : "=f"(d01.x), "=f"(d01.y), "=f"(d23.x), "=f"(d23.y), "=f"(d45.x), "=f"(d45.y),
        "=f"(d67.x), "=f"(d67.y)
      : "r"(v0), "r"(v1), "r"(v2), "r"(v3), "f"(cz));
}

__device__ __forceinline__ float bf16_lo(uint32_t p) { return __uint_as_float(p << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t p) { return __uint_as_float(p & 0xFFFF0000u); }

// CTA that owns tile u when T tiles are split evenly over G CTAs
// (t0(c) = floor(c*T/G)).
__device__ __forceinline__ int owner_cta(long long u, long long T, int G) {
  return (int)(((u + 1) * G + T - 1) / T) - 1;
}

// The producer lanes' share of one activation slab: lane l holds inputs
// 16l .. 16l+15 of the slab for every row of x (and of the AWQ factor).
template <int MP, bool IDOT>
struct XSlice {
  uint4 xb[MP][2];
  float4 inv[4];
};

// Read lane l's share (inputs 16l .. 16l+15 of the slab) from a raw slot.
template <int MP, bool IDOT>
__device__ __forceinline__ void read_x_slice(XSlice<MP, IDOT>& xs, const uint8_t* raw,
                                             const GemvParams& prm, int s, int lane) {
  using SL = StageLayout<MP, IDOT>;
  const bool ok = s * kSlabK + 16 * lane < prm.g.K;   // inside the slab's groups
#pragma unroll
  for (int m = 0; m < MP; ++m) {
    xs.xb[m][0] = make_uint4(0, 0, 0, 0);
    xs.xb[m][1] = make_uint4(0, 0, 0, 0);
    if (ok && m < prm.M) {
      const uint4* src = reinterpret_cast<const uint4*>(raw + m * kSlabK * 2 + 32 * lane);
      xs.xb[m][0] = src[0];
      xs.xb[m][1] = src[1];
    }
  }
  if constexpr (!IDOT) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      xs.inv[q] = make_float4(1.f, 1.f, 1.f, 1.f);
      if (ok && prm.inv_s)
        xs.inv[q] = reinterpret_cast<const float4*>(raw + SL::kRawInv + 64 * lane)[q];
    }
  }
}

// Integer path with the AWQ factor: lane l's 16 factors of slab s, read from
// global memory (the factor is small and stays in L2); issued before the
// producer's waits so that their latency overlaps them.
template <int MP, bool IDOT>
__device__ __forceinline__ void load_inv_slice(XSlice<MP, IDOT>& xs, const GemvParams& prm, int s,
                                               int lane) {
  const bool ok = s * kSlabK + 16 * lane < prm.g.K;
#pragma unroll
  for (int q = 0; q < 4; ++q)
    xs.inv[q] = (ok && prm.inv_s)
                    ? __ldg(reinterpret_cast<const float4*>(prm.inv_s + (size_t)s * kSlabK + 16 * lane) + q)
                    : make_float4(1.f, 1.f, 1.f, 1.f);
}

template <int MP, bool IDOT, bool AWQI>
__device__ __forceinline__ void store_x_slice(const XSlice<MP, IDOT>& xs, uint8_t* stage,
                                              const GemvParams& prm, int lane) {
  using SL = StageLayout<MP, IDOT>;
  const int c = lane >> 2, sub = lane & 3;      // 64-input chunk and quarter of it
#pragma unroll
  for (int m = 0; m < MP; ++m) {
    if (m >= prm.M) break;
    const uint32_t r[8] = {xs.xb[m][0].x, xs.xb[m][0].y, xs.xb[m][0].z, xs.xb[m][0].w,
                           xs.xb[m][1].x, xs.xb[m][1].y, xs.xb[m][1].z, xs.xb[m][1].w};
    if constexpr (IDOT) {
      // 16-bit fixed point per 64-input chunk: x_i = rn(x * 2^e) with e chosen
      // from the chunk's largest |x| so that it lands in [2^14, 2^15) (exact
      // there: bf16 has 8 significant bits), every other value within half a
      // step 2^-e.  x_i = 256 h + l is stored as signed high bytes h and
      // unsigned low bytes l, ordered like the code bytes of an interleaved
      // word (see dp4a_word).  With the AWQ factor the chunk holds
      // u = fp32(x) * inv (one rounding) instead of x.  A chunk holding a NaN
      // or an infinity stores zeros and a NaN factor, so the rows it meets
      // come out NaN.
      float xf[16];
      bool bad = false;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        xf[2 * q] = bf16_lo(r[q]);
        xf[2 * q + 1] = bf16_hi(r[q]);
        if constexpr (!AWQI)
          bad |= (r[q] & 0x7F80u) == 0x7F80u || (r[q] & 0x7F800000u) == 0x7F800000u;
      }
      if constexpr (AWQI) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          xf[4 * q] = __fmul_rn(xf[4 * q], xs.inv[q].x);
          xf[4 * q + 1] = __fmul_rn(xf[4 * q + 1], xs.inv[q].y);
          xf[4 * q + 2] = __fmul_rn(xf[4 * q + 2], xs.inv[q].z);
          xf[4 * q + 3] = __fmul_rn(xf[4 * q + 3], xs.inv[q].w);
        }
#pragma unroll
        for (int q = 0; q < 16; ++q) bad |= !(fabsf(xf[q]) <= 3.402823466e38f);   // NaN or infinity
      }
      float amax = 0.0f;
#pragma unroll
      for (int q = 0; q < 16; ++q) amax = fmaxf(amax, fabsf(xf[q]));
      amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
      bad = __shfl_xor_sync(0xFFFFFFFFu, (int)bad, 1) | bad;
      bad = __shfl_xor_sync(0xFFFFFFFFu, (int)bad, 2) | bad;
      int e = 0;
      if (!bad && amax > 0.0f) {
        int eb = (int)(__float_as_uint(amax) >> 23), pre = 0;
        if (eb == 0) {                               // subnormal: exponent of amax * 2^64
          eb = (int)(__float_as_uint(amax * 0x1p64f) >> 23);
          pre = 64;
        }
        e = 141 - eb + pre;                          // in [-113, 147]
      }
      // 2^-e as fp32 (subnormal above 126), and 2^e as two normal factors
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
      uint32_t wv[8];
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int* v = xi + 8 * t;
        // code byte order of an interleaved word: low nibbles hold inputs
        // 0, 4, 1, 5 and high nibbles inputs 2, 6, 3, 7
        auto hb = [](int a) { return (uint32_t)(a >> 8) & 0xFFu; };
        auto lb = [](int a) { return (uint32_t)a & 0xFFu; };
        wv[4 * t + 0] = hb(v[0]) | hb(v[4]) << 8 | hb(v[1]) << 16 | hb(v[5]) << 24;
        wv[4 * t + 1] = hb(v[2]) | hb(v[6]) << 8 | hb(v[3]) << 16 | hb(v[7]) << 24;
        wv[4 * t + 2] = lb(v[0]) | lb(v[4]) << 8 | lb(v[1]) << 16 | lb(v[5]) << 24;
        wv[4 * t + 3] = lb(v[2]) | lb(v[6]) << 8 | lb(v[3]) << 16 | lb(v[7]) << 24;
      }
      uint4* dst = reinterpret_cast<uint4*>(stage + SL::kX + m * SL::kXRow + c * kXbChunk + sub * 32);
      dst[0] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
      dst[1] = make_uint4(wv[4], wv[5], wv[6], wv[7]);
      sx += __shfl_xor_sync(0xFFFFFFFFu, sx, 1);
      sx += __shfl_xor_sync(0xFFFFFFFFu, sx, 2);
      if (sub == 0)
        reinterpret_cast<float4*>(stage + SL::kXsum)[m * kChunks + c] =
            make_float4((float)sx, unscale, 0.0f, 0.0f);
    } else {
      float4* dst = reinterpret_cast<float4*>(stage + SL::kX + m * SL::kXRow + c * kXfChunk + sub * 64);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 iv = xs.inv[q];
        dst[q] = make_float4(__fmul_rn(bf16_lo(r[2 * q]), iv.x), __fmul_rn(bf16_hi(r[2 * q]), iv.y),
                             __fmul_rn(bf16_lo(r[2 * q + 1]), iv.z),
                             __fmul_rn(bf16_hi(r[2 * q + 1]), iv.w));
      }
    }
  }
}

// The scales (and zeros) of rows r0 + 4 j (j < JQ) for this lane's group grp
// of the stage's tile (0 for lanes past a ragged slab's groups).
template <int JQ>
__device__ __forceinline__ void load_group_params(float (&sc)[JQ], float (&zc)[JQ],
                                                  const uint8_t* meta, int gs, int sym, int r0,
                                                  int grp, bool active) {
#pragma unroll
  for (int j = 0; j < JQ; ++j) {
    const int r = r0 + 4 * j;
    sc[j] = 0.0f;
    zc[j] = 0.0f;
    if (active) {
      if (sym) {
        sc[j] = __half2float(reinterpret_cast<const __half*>(meta)[r * gs + grp]);
        zc[j] = 8.0f;
      } else {
        const __half2 sz = reinterpret_cast<const __half2*>(meta)[r * gs + grp];
        sc[j] = __low2float(sz);
        zc[j] = __high2float(sz);
      }
    }
  }
}

// Half hf (16 bytes = 4 code words) of this lane's 64 inputs of rows r0 + 4 j.
template <int JQ>
__device__ __forceinline__ void load_codes(uint4 (&c)[JQ], const uint8_t* stage, int pitch, int r0,
                                           int p, int hf, bool active) {
#pragma unroll
  for (int j = 0; j < JQ; ++j)
    c[j] = active ? *reinterpret_cast<const uint4*>(stage + (r0 + 4 * j) * pitch + p * 32 + hf * 16)
                  : make_uint4(0, 0, 0, 0);
}

// Bytes of shared memory one team of the GEMV uses, rounded to 128.
template <int MP, int STAGES, int XR, int RAWS, bool IDOT>
__host__ __device__ constexpr size_t gemv_team_smem() {
  return ((size_t)STAGES * StageLayout<MP, IDOT>::kBytes +
          (size_t)XR * StageLayout<MP, IDOT>::kXSlot +
          (size_t)RAWS * StageLayout<MP, IDOT>::kRawBytes + (2 * STAGES + 2 * XR + RAWS) * 8 +
          16 + 127) /
         128 * 128;
}

// One CTA per SM runs VC independent teams ("virtual CTAs"), each a producer
// warp and kConsumerWarps consumer warps with its own shared memory and its
// own contiguous run of tiles.  The team of a warp is its warp index mod VC,
// so every team gets warps of every age: CTAs sharing an SM are not scheduled
// evenly (the older CTA's warps win the issue slots), teams inside one CTA
// are, and the SM's work then finishes at the same time.
//
// A team's rings: STAGES weight stages (full: the tile's bytes landed; empty:
// every consumer warp has this tile's codes and metadata in registers), XR
// activation slots (xfull: the producer prepared the tile's activations;
// xempty: every consumer warp is done with the tile) and RAWS raw activation
// slots (bulk copies of x and of the AWQ factor).  Releasing a weight stage
// before the arithmetic keeps it busy only for the copy and a register load,
// so more of the shared memory is in flight (EARLY; it needs registers for
// all of the lane's codes, so it is used where a lane covers one pass of
// rows; otherwise the stage is released after the arithmetic).
template <int MP, int JQ, int STAGES, int XR, int RAWS, int VC, bool IDOT, bool EARLY, bool AWQI>
__global__ void __launch_bounds__(kGemvThreads * VC, 1) gemv_w4a16_kernel(GemvParams prm) {
  using SL = StageLayout<MP, IDOT>;
  extern __shared__ __align__(128) uint8_t smem_all[];
  const int team = (threadIdx.x >> 5) % VC;
  uint8_t* smem = smem_all + team * gemv_team_smem<MP, STAGES, XR, RAWS, IDOT>();
  const Geom g = prm.g;
  uint8_t* x_ring = smem + STAGES * SL::kBytes;
  uint8_t* raw_ring = x_ring + XR * SL::kXSlot;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(raw_ring + RAWS * SL::kRawBytes);
  uint64_t* empty_bar = full_bar + STAGES;
  uint64_t* xfull_bar = empty_bar + STAGES;
  uint64_t* xempty_bar = xfull_bar + XR;
  uint64_t* raw_bar = xempty_bar + XR;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(raw_bar + RAWS);

  const int warp = (threadIdx.x >> 5) / VC;     // warp index within the team
  const int lane = threadIdx.x & 31;
  const int ltid = warp * 32 + lane;           // thread index within the team
  const int G = gridDim.x * VC;                // teams of the grid
  const int vb = blockIdx.x * VC + team;       // this team's index
  const long long t0 = (long long)vb * prm.tiles / G;
  const long long t1 = (long long)(vb + 1) * prm.tiles / G;
  const int ntiles = (int)(t1 - t0);

  if (ltid == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full_bar[i], 1);                // producer's expect_tx
      mbar_init(&empty_bar[i], kConsumerWarps);
    }
    for (int i = 0; i < XR; ++i) {
      mbar_init(&xfull_bar[i], 32);              // the producer's 32 lanes
      mbar_init(&xempty_bar[i], kConsumerWarps);
    }
    for (int i = 0; i < RAWS; ++i) mbar_init(&raw_bar[i], 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  // Rows of x beyond M are never written: zero every activation slot once.
  for (int i = ltid; i < XR * SL::kXSlot / 16; i += kGemvThreads)
    reinterpret_cast<uint4*>(x_ring)[i] = make_uint4(0, 0, 0, 0);
  __syncthreads();
  // Programmatic dependent launch: the next kernel in the stream may start
  // as soon as SMs free up (it waits for this grid before it touches
  // anything this grid writes).
  griddep_launch_dependents();

  if (warp == kConsumerWarps + 1) {
    // ---------------------------------------------------------- weight producer
    // Every weight tile goes out as soon as its stage is free.  The first
    // STAGES tiles do not depend on the previous kernel in the stream (no
    // kernel of this library writes weights): they go out at once, so they
    // stream in while that kernel finishes.
    int wb = (int)(t0 / g.NS), ws = (int)(t0 % g.NS);
    int issued = 0;
    bool ok = true;
    for (int i = 0; i < ntiles; ++i) {
      const int st = i % STAGES;
      if (i >= STAGES) {
        ok = mbar_wait_bounded(&empty_bar[st], ((i / STAGES) - 1) & 1, prm.wait_ns);
        ok = __all_sync(0xFFFFFFFFu, ok) && !*abort_flag;
        if (!ok) break;
      }
      if (lane == 0) {
        const uint32_t tbytes = (uint32_t)tile_bytes(g, slab_groups(g, ws));
        mbar_arrive_expect_tx(&full_bar[st], tbytes);
        bulk_copy_g2s(smem + st * SL::kBytes, prm.packed + tile_offset(g, ws, wb), tbytes,
                      &full_bar[st]);
      }
      issued = i + 1;
      if (++ws == g.NS) { ws = 0; ++wb; }
    }
    if (!ok && lane == 0) {
      atomicOr(prm.err, kDevErrTimeout);
      *abort_flag = 1;
    }
    if (lane == 0 && *abort_flag) {
      // Wait (bounded) for every copy still in flight before the CTA exits.
      for (int st = 0; st < STAGES && st < issued; ++st) {
        const int uses = (issued - 1 - st) / STAGES + 1;   // copies issued on stage st
        mbar_wait_bounded(&full_bar[st], (uses - 1) & 1, prm.drain_ns);
      }
    }
    return;
  }

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------ activation producer
    // The raw activation slab (and AWQ factor) of tile i is bulk-copied into
    // raw slot i % RAWS, RAWS tiles ahead of its use, so the slab is already
    // in shared memory when it is prepared in activation slot i % XR.
    int raw_issued = 0;
    int ps = (int)(t0 % g.NS), pf = ps;
    auto next_slab = [&](int v) { return v + 1 == g.NS ? 0 : v + 1; };
    auto issue_raw = [&](int slot, int slab) {       // lane 0 only
      uint8_t* dst = raw_ring + slot * SL::kRawBytes;
      const int gsx = slab_groups(g, slab);
      // the integer path reads its AWQ factors from global memory instead
      const uint32_t xb = gsx * kGroup * 2, ib = (prm.inv_s && !IDOT) ? gsx * kGroup * 4 : 0;
      mbar_arrive_expect_tx(&raw_bar[slot], prm.M * xb + ib);
      for (int m = 0; m < prm.M; ++m)
        bulk_copy_g2s(dst + m * kSlabK * 2, prm.x + (size_t)m * g.K + slab * kSlabK, xb,
                      &raw_bar[slot]);
      if (ib) bulk_copy_g2s(dst + SL::kRawInv, prm.inv_s + slab * kSlabK, ib, &raw_bar[slot]);
    };
    griddep_wait();                      // x may belong to the previous kernel
    if (lane == 0)
      for (int r = 0; r < RAWS && r < ntiles; ++r) {
        issue_raw(r, pf);
        pf = next_slab(pf);
      }
    raw_issued = ntiles < RAWS ? ntiles : RAWS;
    pf = __shfl_sync(0xFFFFFFFFu, pf, 0);
    for (int i = 0; i < ntiles; ++i) {
      const int xs = i % XR;
      const int rs = i % RAWS;
      XSlice<MP, IDOT> xsl;
      if constexpr (AWQI) load_inv_slice<MP, IDOT>(xsl, prm, ps, lane);
      bool ok = true;
      if (i >= XR) ok = mbar_wait_bounded(&xempty_bar[xs], ((i / XR) - 1) & 1, prm.wait_ns);
      ok = __all_sync(0xFFFFFFFFu, ok) && !*abort_flag;
      if (ok) {
        ok = mbar_wait_bounded(&raw_bar[rs], (i / RAWS) & 1, prm.wait_ns);
        ok = __all_sync(0xFFFFFFFFu, ok) && !*abort_flag;
      }
      if (!ok) {
        if (lane == 0) {
          atomicOr(prm.err, kDevErrTimeout);
          *abort_flag = 1;
        }
        break;
      }
      read_x_slice<MP, IDOT>(xsl, raw_ring + rs * SL::kRawBytes, prm, ps, lane);
      store_x_slice<MP, IDOT, AWQI>(xsl, x_ring + xs * SL::kXSlot, prm, lane);
      mbar_arrive(&xfull_bar[xs]);
      ps = next_slab(ps);
      __syncwarp();                      // every lane has read raw slot rs
      if (i + RAWS < ntiles) {
        if (lane == 0) {
          fence_proxy_async_shared();    // generic reads before the async overwrite
          issue_raw(rs, pf);
        }
        pf = next_slab(pf);
        ++raw_issued;
      }
    }
    if (lane == 0 && *abort_flag) {
      for (int r = 0; r < RAWS && r < raw_issued; ++r) {
        const int uses = (raw_issued - 1 - r) / RAWS + 1;
        mbar_wait_bounded(&raw_bar[r], (uses - 1) & 1, prm.drain_ns);
      }
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  griddep_wait();                      // y and the workspace may belong to the previous kernel
  const int rq = lane >> 3;         // row of the quad handled by this lane group
  const int p = lane & 7;           // 64-input chunk of the slab
  constexpr int V = JQ * MP;
  constexpr int kPasses = 4 / JQ;
  using GM = GroupMap<V, 8>;
  const LopConsts lk{prm.lop_mask_lo, prm.lop_bf16_128};

  // Each lane keeps its own partial sums (its 64-input chunk of every tile of
  // the current piece) of the V (row, x row) pairs of each pass; the lanes of
  // a row are combined once, at the end of the piece.
  float part[kPasses][V];
#pragma unroll
  for (int a = 0; a < kPasses; ++a)
#pragma unroll
    for (int i2 = 0; i2 < V; ++i2) part[a][i2] = 0.0f;
  int piece_s0 = -1;                // first slab of the current row tile in this CTA
  bool aborted = false;
  int b = (int)(t0 / g.NS), s = (int)(t0 % g.NS) - 1;

  for (int i = 0; i < ntiles; ++i) {
    if (++s == g.NS) { s = 0; ++b; }
    const int gs = slab_groups(g, s);
    const int st = i % STAGES;
    const int xs = i % XR;
    if (piece_s0 < 0) piece_s0 = s;

    if (!aborted) {
      bool ok = mbar_wait_bounded(&full_bar[st], (i / STAGES) & 1, prm.wait_ns);
      ok = __all_sync(0xFFFFFFFFu, ok);            // keep the warp's decision uniform
      if (!ok) {
        if (lane == 0) atomicOr(prm.err, kDevErrTimeout);
        *abort_flag = 1;
        aborted = true;
      }
    }

    if (!aborted) {
      const uint8_t* stage = smem + st * SL::kBytes;
      const uint8_t* meta = stage + kTileRows * gs * kCodeBytesPerGroupRow;
      const int pitch = gs * kCodeBytesPerGroupRow;
      const int grp = p >> 1;
      const bool active = p < 2 * gs;            // full slabs: always; a ragged last slab: its groups
      // 1. EARLY: this lane's codes and group parameters of the tile into
      //    registers, then the weight stage goes back to the producer
      constexpr int kPI = EARLY ? kPasses : 1;   // passes whose codes are held at once
      uint4 cw[kPI][2][JQ];
      float scv[kPI][JQ], zcv[kPI][JQ];
      if constexpr (EARLY) {
#pragma unroll
        for (int pass = 0; pass < kPasses; ++pass) {
          load_group_params<JQ>(scv[pass], zcv[pass], meta, gs, g.sym, warp * 16 + 4 * pass * JQ + rq,
                                grp, active);
#pragma unroll
          for (int hf = 0; hf < 2; ++hf)
            load_codes<JQ>(cw[pass][hf], stage, pitch, warp * 16 + 4 * pass * JQ + rq, p, hf,
                           active);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[st]);
      }
      // 2. the tile's prepared activations
      bool ok = mbar_wait_bounded(&xfull_bar[xs], (i / XR) & 1, prm.wait_ns);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) {
        if (lane == 0) atomicOr(prm.err, kDevErrTimeout);
        *abort_flag = 1;
        aborted = true;
      }
      if (!aborted) {
      const uint8_t* xslot = x_ring + xs * SL::kXSlot;
      [[maybe_unused]] float4 xinfo[IDOT ? MP : 1];   // integer path: (sum x_i, 2^-e, -, -) of this lane's chunk
      if constexpr (IDOT) {
#pragma unroll
        for (int m = 0; m < MP; ++m)
          xinfo[m] = reinterpret_cast<const float4*>(xslot + SL::kXsum)[m * kChunks + p];
      }

      constexpr int kPassUnroll = kPasses;
      // A lane's 64 inputs of a row are two 16-byte halves of 4 words each; for
      // several rows of x (release after the arithmetic) the passes and halves
      // run one after the other, which bounds the registers in flight.
      constexpr int kHalfUnroll = (MP == 1) ? 2 : 1;
#pragma unroll kPassUnroll
      for (int pass = 0; pass < kPasses; ++pass) {
        const int pi = EARLY ? pass : 0;
        if constexpr (!EARLY)
          load_group_params<JQ>(scv[0], zcv[0], meta, gs, g.sym, warp * 16 + 4 * pass * JQ + rq,
                                grp, active);
        float v[V];
        if constexpr (IDOT) {
          int acc[JQ][MP][4];
#pragma unroll
          for (int j = 0; j < JQ; ++j)
#pragma unroll
            for (int m = 0; m < MP; ++m)
#pragma unroll
              for (int t = 0; t < 4; ++t) acc[j][m][t] = 0;
#pragma unroll kHalfUnroll
          for (int hf = 0; hf < 2; ++hf) {
            uint4 c[JQ];
            if constexpr (EARLY) {
#pragma unroll
              for (int j = 0; j < JQ; ++j) c[j] = cw[pi][hf][j];
            } else {
              load_codes<JQ>(c, stage, pitch, warp * 16 + 4 * pass * JQ + rq, p, hf, active);
            }
#pragma unroll
            for (int wd = 0; wd < 4; ++wd) {
              uint4 xw[MP];
#pragma unroll
              for (int m = 0; m < MP; ++m)
                xw[m] = *reinterpret_cast<const uint4*>(xslot + SL::kX + m * SL::kXRow +
                                                        p * kXbChunk + 16 * (4 * hf + wd));
#pragma unroll
              for (int j = 0; j < JQ; ++j) {
                const uint32_t w = wd == 0 ? c[j].x : wd == 1 ? c[j].y : wd == 2 ? c[j].z : c[j].w;
#pragma unroll
                for (int m = 0; m < MP; ++m) dp4a_word(w, xw[m], acc[j][m]);
              }
            }
          }
          // partial of (row, m) over this lane's 64 inputs:
          //   s16 * 2^-e * (sum x_i q - z * sum x_i)
#pragma unroll
          for (int j = 0; j < JQ; ++j)
#pragma unroll
            for (int m = 0; m < MP; ++m) {
              const int* a = acc[j][m];
              const int t = 256 * (a[0] + (a[1] >> 4)) + a[2] + (int)((uint32_t)a[3] >> 4);
              v[j * MP + m] = active ? (scv[pi][j] * ((float)t - zcv[pi][j] * xinfo[m].x)) *
                                           xinfo[m].y
                                     : 0.0f;
            }
        } else {
          float2 acc[JQ][MP];
          float cz[JQ];
#pragma unroll
          for (int j = 0; j < JQ; ++j) {
            cz[j] = -(128.0f + zcv[pi][j]);
#pragma unroll
            for (int m = 0; m < MP; ++m) acc[j][m] = make_float2(0.0f, 0.0f);
          }
#pragma unroll kHalfUnroll
          for (int hf = 0; hf < 2; ++hf) {
            uint4 c[JQ];
            if constexpr (EARLY) {
#pragma unroll
              for (int j = 0; j < JQ; ++j) c[j] = cw[pi][hf][j];
            } else {
              load_codes<JQ>(c, stage, pitch, warp * 16 + 4 * pass * JQ + rq, p, hf, active);
            }
#pragma unroll
            for (int wd = 0; wd < 4; ++wd) {
              float2 xv[MP][4];
#pragma unroll
              for (int m = 0; m < MP; ++m) {
                const float4* xp = reinterpret_cast<const float4*>(
                    xslot + SL::kX + m * SL::kXRow + p * kXfChunk + 32 * (4 * hf + wd));
                const float4 lo = xp[0], hi = xp[1];
                xv[m][0] = make_float2(lo.x, lo.y);
                xv[m][1] = make_float2(lo.z, lo.w);
                xv[m][2] = make_float2(hi.x, hi.y);
                xv[m][3] = make_float2(hi.z, hi.w);
              }
#pragma unroll
              for (int j = 0; j < JQ; ++j) {
                const uint32_t w = wd == 0 ? c[j].x : wd == 1 ? c[j].y : wd == 2 ? c[j].z : c[j].w;
                float2 d01, d23, d45, d67;           // exact (q - z) for the word's 8 inputs
                widen_word(w, cz[j], d01, d23, d45, d67, lk);
#pragma unroll
                for (int m = 0; m < MP; ++m) {
                  float2 a = acc[j][m];
                  a = __ffma2_rn(d01, xv[m][0], a);
                  a = __ffma2_rn(d23, xv[m][1], a);
                  a = __ffma2_rn(d45, xv[m][2], a);
                  a = __ffma2_rn(d67, xv[m][3], a);
                  acc[j][m] = a;
                }
              }
            }
          }
          // partial of (row, m) over this lane's 64 inputs: s16 * sum x' (q - z)
#pragma unroll
          for (int j = 0; j < JQ; ++j)
#pragma unroll
            for (int m = 0; m < MP; ++m)
              v[j * MP + m] = active ? scv[pi][j] * (acc[j][m].x + acc[j][m].y) : 0.0f;
        }
#pragma unroll
        for (int i2 = 0; i2 < V; ++i2) part[pass][i2] += v[i2];
      }
      __syncwarp();
      if (lane == 0) {
        if constexpr (!EARLY) mbar_arrive(&empty_bar[st]);
        mbar_arrive(&xempty_bar[xs]);
      }
      }
    }

    // ---- end of this CTA's piece of row tile b: write y or a partial
    const bool piece_end = (s == g.NS - 1) || (i == ntiles - 1);
    if (piece_end) {
      const bool whole = (piece_s0 == 0) && (s == g.NS - 1);
      float run[kPasses][GM::kPerLane];
#pragma unroll
      for (int pass = 0; pass < kPasses; ++pass) {
        group_transpose_reduce<V, 8>(part[pass], p);
#pragma unroll
        for (int i2 = 0; i2 < GM::kPerLane; ++i2) run[pass][i2] = part[pass][i2];
      }
      if (!aborted && GM::writer(p)) {
#pragma unroll
        for (int pass = 0; pass < kPasses; ++pass)
#pragma unroll
          for (int i2 = 0; i2 < GM::kPerLane; ++i2) {
            const int idx = GM::index(i2, p);
            const int j = idx / MP, m = idx % MP;
            const int n = b * kTileRows + warp * 16 + 4 * (pass * JQ + j) + rq;
            if (m < prm.M) {
              if (whole) {
                if (n < g.N) prm.y[(size_t)m * g.N + n] = run[pass][i2];
              } else {
                // partial piece: its slot is its first slab
                prm.partials[((size_t)piece_s0 * MP + m) * g.Npad + n] = run[pass][i2];
              }
            }
          }
      }
#pragma unroll
      for (int a = 0; a < kPasses; ++a)
#pragma unroll
        for (int i2 = 0; i2 < V; ++i2) part[a][i2] = 0.0f;
      piece_s0 = -1;
    }
  }
}

// ------------------------------------------------------------------ finish

struct FinishParams {
  const float* partials;   // fp32 [NS][MP][Npad]
  float* y;
  int N, M, MP, NS, Npad, G;
  long long tiles;
};

// y[m][n] of every row tile whose slabs were split between teams: the sum of
// its pieces' partials in slab order (piece c of the row tile starts at slab
// max(t0(c), b NS) - b NS).  One thread per output.  Rows of row tiles held
// by one team were written by the streaming kernel and are left alone.
__global__ void __launch_bounds__(256) gemv_finish_kernel(const FinishParams f) {
  griddep_launch_dependents();
  const long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (e >= (long long)f.M * f.N) {
    griddep_wait();
    return;
  }
  const int m = (int)(e / f.N), n = (int)(e % f.N);
  const int b = n / kTileRows;
  const long long ub = (long long)b * f.NS;
  const int c_first = owner_cta(ub, f.tiles, f.G);
  const int c_last = owner_cta(ub + f.NS - 1, f.tiles, f.G);
  griddep_wait();                    // the streaming kernel's partials are complete
  if (c_first == c_last) return;
  // All pieces' loads are issued before the first addition (they are
  // independent), then added in slab order: one L2 round trip per batch of
  // kBatch pieces instead of one per piece.
  constexpr int kBatch = 8;
  float tot = 0.0f;
  for (int c0 = c_first; c0 <= c_last; c0 += kBatch) {
    float v[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int c2 = c0 + j;
      v[j] = 0.0f;
      if (c2 <= c_last) {
        const long long tc = (long long)c2 * f.tiles / f.G;
        const int sa = (int)((tc > ub ? tc : ub) - ub);
        v[j] = __ldcg(f.partials + ((size_t)sa * f.MP + m) * f.Npad + n);
      }
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j)
      if (c0 + j <= c_last) tot += v[j];
  }
  f.y[(size_t)m * f.N + n] = tot;
}

// ------------------------------------------------------------------ launcher

struct GemvConfig {
  const void* fn;
  size_t smem;
  int teams;               // virtual CTAs per CTA
};

template <int MP, int JQ, int STAGES, int XR, int RAWS, int VC, bool IDOT, bool EARLY,
          bool AWQI = false>
static GemvConfig gemv_config() {
  GemvConfig c;
  c.fn = reinterpret_cast<const void*>(
      &gemv_w4a16_kernel<MP, JQ, STAGES, XR, RAWS, VC, IDOT, EARLY, AWQI>);
  c.smem = VC * gemv_team_smem<MP, STAGES, XR, RAWS, IDOT>();
  c.teams = VC;
  return c;
}

static int padded_m(int M) { return M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : 8; }

// Integer (dp4a) path for M <= 4, with or without the AWQ factor (applied
// in fp32 before the fixed point); packed fp32 path for M > 4 (where one
// widening per code is shared by 8 rows).  Teams x (weight stages, activation slots, raw slots) fill the
// shared memory of one CTA per SM; two teams keep the registers for a tile's
// codes held between the stage release and the arithmetic.
static GemvConfig pick_gemv(int M, bool awq) {
  switch (padded_m(M)) {
    case 1: return awq ? gemv_config<1, 2, 3, 3, 2, 2, true, true, true>()
                       : gemv_config<1, 2, 3, 3, 2, 2, true, true>();
    case 2: return awq ? gemv_config<2, 2, 3, 2, 3, 2, true, false, true>()
                       : gemv_config<2, 2, 3, 2, 3, 2, true, false>();
    case 4: return awq ? gemv_config<4, 2, 5, 2, 3, 1, true, false, true>()
                       : gemv_config<4, 2, 5, 2, 3, 1, true, false>();
    default: return gemv_config<8, 2, 5, 2, 2, 1, false, false>();
  }
}

// CTAs of the persistent grid for `tiles` tiles with `teams` teams per CTA:
// at most `ctas_per_sm` per SM and no more than the tiles need.  At most one
// team may be left without tiles; it is then team 0, ahead of every row
// tile.  A team without tiles among a row tile's owners would never deliver
// its piece of the split-K sum, so the last piece would never see the count
// it waits for.  Pure host arithmetic.
long long gemv_grid(long long tiles, int teams, int num_sms, int ctas_per_sm) {
  long long grid = (long long)num_sms * ctas_per_sm;
  const long long need = (tiles + teams - 1) / teams;
  if (grid > need) grid = need;
  while (grid > 1 && grid * teams > tiles + 1) --grid;
  return grid < 1 ? 1 : grid;
}

int gemv_teams(int M, bool awq) { return pick_gemv(M, awq).teams; }

long long gemv_tiles(int N, int K) {
  const Geom g = make_geom(N, K, 1);
  return (long long)g.NS * g.NB;
}

bool gemv_tc_supported(int M, int K);
cudaError_t launch_gemv_tc(const void* x, const float* inv_s, const void* packed, int M, int N,
                           int K, int sym, float* y, void* workspace, int* err, int num_sms,
                           unsigned long long wait_ns, cudaStream_t stream);

// Test hook: route every GEMV to the CUDA-core kernel (0: the tensor-core
// decode kernel takes the shapes it supports).
static int g_force_cuda_cores = 0;
void gemv_force_cuda_cores(int on) { g_force_cuda_cores = on; }
bool gemv_forced_cuda_cores() { return g_force_cuda_cores != 0; }

// The split-K finish of a persistent GEMV whose G CTAs each own the
// contiguous run [floor(c T / G), floor((c + 1) T / G)) of the T tiles.
cudaError_t launch_gemv_finish(const float* partials, float* y, int N, int M, int MP, int NS,
                               int Npad, int G, long long tiles, cudaStream_t stream) {
  FinishParams f;
  f.partials = partials;
  f.y = y;
  f.N = N;
  f.M = M;
  f.MP = MP;
  f.NS = NS;
  f.Npad = Npad;
  f.G = G;
  f.tiles = tiles;
  void* fargs[] = {&f};
  const long long outs = (long long)M * N;
  return launch_pdl(reinterpret_cast<const void*>(&gemv_finish_kernel),
                    dim3((unsigned)((outs + 255) / 256)), dim3(256), fargs, 0, stream);
}

size_t gemv_tc_workspace_bytes(int M, int N, int K);

// Shapes the tensor-core decode kernel takes get its workspace, which holds
// the CUDA-core kernel's as a prefix.
size_t gemv_workspace_bytes(int M, int N, int K) {
  if (gemv_tc_supported(M, K)) return gemv_tc_workspace_bytes(M, N, K);
  const Geom g = make_geom(N, K, 1);
  if (g.NS <= 1) return 0;
  return (size_t)kCounterBytes + (size_t)g.NS * padded_m(M) * g.Npad * sizeof(float);
}

cudaError_t launch_gemv(const void* x, const float* inv_s, const void* packed, int M, int N,
                        int K, int sym, float* y, void* workspace, int* err, int num_sms,
                        unsigned long long wait_ns, cudaStream_t stream) {
  if (!g_force_cuda_cores && gemv_tc_supported(M, K))
    return launch_gemv_tc(x, inv_s, packed, M, N, K, sym, y, workspace, err, num_sms, wait_ns,
                          stream);
  GemvParams prm;
  prm.g = make_geom(N, K, sym);
  prm.packed = static_cast<const uint8_t*>(packed);
  prm.x = static_cast<const uint16_t*>(x);
  prm.inv_s = inv_s;
  prm.y = y;
  prm.partials = workspace ? reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kCounterBytes)
                           : nullptr;
  prm.err = err;
  prm.M = M;
  prm.tiles = (long long)prm.g.NS * prm.g.NB;
  prm.wait_ns = wait_ns;
  prm.drain_ns = 1000000000ull;
  prm.lop_mask_lo = 0x000F000Fu;
  prm.lop_bf16_128 = 0x43004300u;

  const GemvConfig c = pick_gemv(M, inv_s != nullptr);
  int per_sm = 0;
  cudaError_t e = kernel_setup(c.fn, c.smem, kGemvThreads * c.teams, &per_sm);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const long long grid = gemv_grid(prm.tiles, c.teams, num_sms, per_sm);
  void* args[] = {&prm};
  e = launch_pdl(c.fn, dim3((unsigned)grid), dim3(kGemvThreads * c.teams), args, c.smem, stream);
  if (e != cudaSuccess || prm.g.NS <= 1) return e;
  return launch_gemv_finish(prm.partials, y, N, M, padded_m(M), prm.g.NS, prm.g.Npad,
                            (int)(grid * c.teams), prm.tiles, stream);
}

}  // namespace wq
