// wq_quantize.cu -- per-group RTN 4-bit quantization with canonical uint4
// packing, and the permutation into the tiled kernel layout.
//
// Quantizer ("3.6 量化(Quantization)", section 对称与非对称量化; "后训练量化（PTQ,
// Post-Training Quantization）", section 基础量化公式; "量化" compendium, section
// 量化方程), per group of 128 consecutive inputs of one output row
// ("3.6 量化(Quantization)", section 粒度):
//   symmetric : s = max|w| / 7,          q = clamp(rne(w / s), -7, 7), stored q + 8
//   asymmetric: s = (max - min) / 15,    z = rne(-min / s),
//               q = clamp(rne(w / s) + z, 0, 15)
// The range is floored at 1e-8 before the division (the pages' code), the
// scale is rounded to fp16 (round to nearest even) and the codes are
// computed with that stored fp16 scale (and the stored fp16 zero), so the
// metadata reproduce w_hat = s16 (q - z16) exactly.  All arithmetic is IEEE
// fp32 with explicit round-to-nearest intrinsics, so the result is the same
// on every run and matches a correctly rounded CPU evaluation bit for bit.
#include "wq_common.cuh"

namespace wq {

struct QuantParams {
  const uint4* W;        // bf16 [N][K] viewed as 16-byte chunks
  const float* awq;      // fp32 [K] or nullptr
  uint32_t* qweight;     // uint32 [N][K/8]
  uint16_t* scales;      // fp16 bits [N][K/128]
  uint16_t* zeros;       // fp16 bits [N][K/128] or nullptr (symmetric)
  int* d_status;         // count of non-finite groups, or nullptr
  long long groups;      // N * K / 128
  int NG;                // groups per row
  int sym;
};

struct GroupResult {
  uint32_t word0, word1;   // this lane's two packed words
  uint16_t s16, z16;
  bool bad;
};

// Round-to-nearest-even of w / sf for one element, given r = RN(1 / sf).
// t = RN(w * r) is within |t| * 2^-23 (plus rounding) of the exact quotient,
// so when t is farther than |t| * 2^-20 + 2^-24 from the nearest half-integer
// the correctly rounded quotient RN(w / sf) rounds to the same integer as t;
// otherwise (rare: near a tie, or |t| >= 2^20) the IEEE division decides.
__device__ __forceinline__ float round_quotient(float w, float sf, float r) {
  const float t = __fmul_rn(w, r);
  const float fl = floorf(t);
  const float d = fabsf(__fsub_rn(__fsub_rn(t, fl), 0.5f));
  if (d > __fmaf_rn(fabsf(t), 0x1p-20f, 0x1p-24f)) return rintf(t);
  return rintf(__fdiv_rn(w, sf));
}

// Eight lanes (a quarter warp, `mask`) quantize one group; lane ql holds
// elements 16*ql .. 16*ql+15 of the group, so it produces two packed words.
__device__ __forceinline__ GroupResult quantize_group(const uint4 raw0, const uint4 raw1,
                                                      const float* awq_k, unsigned mask,
                                                      int sym) {
  float w[16];
  const uint32_t r32[8] = {raw0.x, raw0.y, raw0.z, raw0.w, raw1.x, raw1.y, raw1.z, raw1.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    w[2 * i] = __uint_as_float(r32[i] << 16);
    w[2 * i + 1] = __uint_as_float(r32[i] & 0xFFFF0000u);
  }
  if (awq_k) {
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const float4 a = __ldg(reinterpret_cast<const float4*>(awq_k) + v);
      w[4 * v + 0] = __fmul_rn(w[4 * v + 0], a.x);   // W' = W diag(s)
      w[4 * v + 1] = __fmul_rn(w[4 * v + 1], a.y);
      w[4 * v + 2] = __fmul_rn(w[4 * v + 2], a.z);
      w[4 * v + 3] = __fmul_rn(w[4 * v + 3], a.w);
    }
  }
  bool bad = false;
  float mn = w[0], mx = w[0];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    bad |= !isfinite(w[i]);
    mn = fminf(mn, w[i]);
    mx = fmaxf(mx, w[i]);
  }
  bad = __any_sync(mask, bad);
#pragma unroll
  for (int o = 4; o >= 1; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(mask, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(mask, mx, o));
  }

  GroupResult res;
  res.word0 = res.word1 = 0;
  res.s16 = 0;
  res.z16 = 0;
  float sf = 1.0f, zf = 0.0f;
  if (!bad) {
    // symmetric range max|w| = max(-min, max), exactly
    float range = sym ? fmaxf(-mn, mx) : __fsub_rn(mx, mn);
    if (range < 1e-8f) range = 1e-8f;
    const float s32 = __fdiv_rn(range, sym ? 7.0f : 15.0f);
    uint16_t hs = __half_as_ushort(__float2half_rn(s32));
    if (hs == 0) hs = 0x0001;                       // underflow -> 2^-24
    if ((hs & 0x7C00u) == 0x7C00u) bad = true;      // fp16 overflow
    res.s16 = hs;
    sf = __half2float(__ushort_as_half(hs));
  }
  if (!bad && !sym) {
    const float z = __fadd_rn(rintf(__fdiv_rn(-mn, sf)), 0.0f);   // -0 -> +0
    const uint16_t hz = __half_as_ushort(__float2half_rn(z));
    if ((hz & 0x7C00u) == 0x7C00u) bad = true;
    res.z16 = hz;
    zf = __half2float(__ushort_as_half(hz));
  }
  if (bad) {
    res.bad = true;
    res.s16 = 0x7E00;
    res.z16 = 0x7E00;
    return res;
  }
  const float r = __frcp_rn(sf);
  const float lo = sym ? -7.0f : 0.0f, hi = sym ? 7.0f : 15.0f;
  uint32_t word[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float t = __fadd_rn(round_quotient(w[i], sf, r), zf);
    t = fminf(fmaxf(t, lo), hi);
    const int code = static_cast<int>(t) + (sym ? 8 : 0);
    word[i >> 3] |= static_cast<uint32_t>(code & 0xF) << (4 * (i & 7));
  }
  res.word0 = word[0];
  res.word1 = word[1];
  res.bad = false;
  return res;
}

__global__ void __launch_bounds__(256) quantize_rtn_kernel(QuantParams p) {
  const int lane = threadIdx.x & 31;
  const int ql = lane & 7;
  const unsigned mask = 0xFFu << (lane & 24);      // this quarter warp
  const long long nq = (long long)gridDim.x * (blockDim.x / 8);
  long long gid = ((long long)blockIdx.x * blockDim.x + threadIdx.x) / 8;

  // Two groups per iteration so each lane keeps four 16-byte loads in flight.
  for (; gid < p.groups; gid += 2 * nq) {
    const long long gid2 = gid + nq;
    const bool has2 = gid2 < p.groups;
    const uint4 a0 = __ldcs(p.W + gid * 16 + 2 * ql);
    const uint4 a1 = __ldcs(p.W + gid * 16 + 2 * ql + 1);
    uint4 b0 = make_uint4(0, 0, 0, 0), b1 = b0;
    if (has2) {
      b0 = __ldcs(p.W + gid2 * 16 + 2 * ql);
      b1 = __ldcs(p.W + gid2 * 16 + 2 * ql + 1);
    }
    const float* s1 = p.awq ? p.awq + (gid % p.NG) * kGroup + 16 * ql : nullptr;
    const GroupResult r1 = quantize_group(a0, a1, s1, mask, p.sym);
    reinterpret_cast<uint2*>(p.qweight)[gid * 8 + ql] = make_uint2(r1.word0, r1.word1);
    if (ql == 0) {
      p.scales[gid] = r1.s16;
      if (!p.sym) p.zeros[gid] = r1.z16;
      if (r1.bad && p.d_status) atomicAdd(p.d_status, 1);
    }
    if (has2) {
      const float* s2 = p.awq ? p.awq + (gid2 % p.NG) * kGroup + 16 * ql : nullptr;
      const GroupResult r2 = quantize_group(b0, b1, s2, mask, p.sym);
      reinterpret_cast<uint2*>(p.qweight)[gid2 * 8 + ql] = make_uint2(r2.word0, r2.word1);
      if (ql == 0) {
        p.scales[gid2] = r2.s16;
        if (!p.sym) p.zeros[gid2] = r2.z16;
        if (r2.bad && p.d_status) atomicAdd(p.d_status, 1);
      }
    }
  }
}

// ------------------------------------------------------------------ relayout

struct LayoutParams {
  const uint32_t* qweight;
  const uint16_t* scales;
  const uint16_t* zeros;
  uint8_t* out;
  Geom g;
};

// Nibble interleave of one code word: even nibbles 0,2,4,6 -> slots 0..3, odd
// nibbles 1,3,5,7 -> slots 4..7.
__device__ __forceinline__ uint32_t interleave_word(uint32_t w) {
  uint32_t e = w & 0x0F0F0F0Fu, o = (w >> 4) & 0x0F0F0F0Fu;
  e = (e | (e >> 4)) & 0x00FF00FFu;
  e = (e | (e >> 8)) & 0x0000FFFFu;
  o = (o | (o >> 4)) & 0x00FF00FFu;
  o = (o | (o >> 8)) & 0x0000FFFFu;
  return e | (o << 16);
}

// One CTA per tile (slab s, row tile b): copy the tile's codes row by row in
// 16-byte chunks (nibbles interleaved), then gather its metadata.  Rows past
// N are written as 0.
__global__ void __launch_bounds__(256) relayout_kernel(LayoutParams p) {
  const Geom& g = p.g;
  const int s = blockIdx.x / g.NB;
  const int b = blockIdx.x % g.NB;
  const int gs = slab_groups(g, s);
  uint8_t* tile = p.out + tile_offset(g, s, b);
  const int chunks_per_row = gs * 4;
  const int words_per_row = g.K / 8;

  for (int c = threadIdx.x; c < kTileRows * chunks_per_row; c += blockDim.x) {
    const int r = c / chunks_per_row;
    const int cc = c % chunks_per_row;
    const int n = b * kTileRows + r;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (n < g.N) {
      v = __ldg(reinterpret_cast<const uint4*>(p.qweight + (size_t)n * words_per_row +
                                               s * kSlabGroups * 16) + cc);
      v = make_uint4(interleave_word(v.x), interleave_word(v.y), interleave_word(v.z),
                     interleave_word(v.w));
    }
    *reinterpret_cast<uint4*>(tile + r * gs * kCodeBytesPerGroupRow + cc * 16) = v;
  }
  uint8_t* mbase = tile + kTileRows * gs * kCodeBytesPerGroupRow;
  for (int e = threadIdx.x; e < kTileRows * gs; e += blockDim.x) {
    const int r = e / gs;
    const int gg = s * kSlabGroups + e % gs;
    const int n = b * kTileRows + r;
    const size_t mi = (size_t)n * g.NG + gg;
    if (g.sym) {
      reinterpret_cast<uint16_t*>(mbase)[e] = (n < g.N) ? p.scales[mi] : 0;
    } else {
      reinterpret_cast<uint32_t*>(mbase)[e] =
          (n < g.N) ? ((uint32_t)p.scales[mi] | ((uint32_t)p.zeros[mi] << 16)) : 0u;
    }
  }
}

// ------------------------------------------------------------------ launchers

cudaError_t launch_quantize(const void* W, const float* awq, int N, int K, int sym,
                            uint32_t* qweight, void* scales, void* zeros, int* d_status,
                            cudaStream_t stream, int num_sms) {
  QuantParams p;
  p.W = static_cast<const uint4*>(W);
  p.awq = awq;
  p.qweight = qweight;
  p.scales = static_cast<uint16_t*>(scales);
  p.zeros = static_cast<uint16_t*>(zeros);
  p.d_status = d_status;
  p.groups = (long long)N * (K / kGroup);
  p.NG = K / kGroup;
  p.sym = sym;
  if (d_status) {
    cudaError_t e = cudaMemsetAsync(d_status, 0, sizeof(int), stream);
    if (e != cudaSuccess) return e;
  }
  const long long quarters_needed = (p.groups + 1) / 2;   // two groups per quarter warp
  long long blocks = (quarters_needed + 31) / 32;
  const long long cap = (long long)num_sms * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  quantize_rtn_kernel<<<(unsigned)blocks, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_relayout(const uint32_t* qweight, const void* scales, const void* zeros,
                            int N, int K, int sym, void* packed, cudaStream_t stream) {
  LayoutParams p;
  p.qweight = qweight;
  p.scales = static_cast<const uint16_t*>(scales);
  p.zeros = static_cast<const uint16_t*>(zeros);
  p.out = static_cast<uint8_t*>(packed);
  p.g = make_geom(N, K, sym);
  const long long tiles = (long long)p.g.NS * p.g.NB;
  relayout_kernel<<<(unsigned)tiles, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace wq
