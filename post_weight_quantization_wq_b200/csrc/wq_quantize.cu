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
  uint32_t word;
  uint16_t s16, z16;
  bool bad;
};

// One half-warp (16 lanes) quantizes one group; lane `hl` holds elements
// 8*hl .. 8*hl+7 of the group, so it produces exactly one packed word.
__device__ __forceinline__ GroupResult quantize_group(const uint4 raw, const float* awq_k,
                                                      unsigned mask, int sym) {
  float w[8];
  const uint32_t r32[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    w[2 * i] = __uint_as_float(r32[i] << 16);
    w[2 * i + 1] = __uint_as_float(r32[i] & 0xFFFF0000u);
  }
  if (awq_k) {
    const float4 a0 = __ldg(reinterpret_cast<const float4*>(awq_k));
    const float4 a1 = __ldg(reinterpret_cast<const float4*>(awq_k) + 1);
    const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = __fmul_rn(w[i], a[i]);   // W' = W diag(s)
  }
  bool bad = false;
  float amax = 0.0f, mn = w[0], mx = w[0];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    bad |= !isfinite(w[i]);
    amax = fmaxf(amax, fabsf(w[i]));
    mn = fminf(mn, w[i]);
    mx = fmaxf(mx, w[i]);
  }
  bad = __any_sync(mask, bad);
#pragma unroll
  for (int o = 8; o >= 1; o >>= 1) {
    amax = fmaxf(amax, __shfl_xor_sync(mask, amax, o));
    mn = fminf(mn, __shfl_xor_sync(mask, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(mask, mx, o));
  }

  GroupResult res;
  res.word = 0;
  res.s16 = 0;
  res.z16 = 0;
  float sf = 1.0f, zf = 0.0f;
  if (!bad) {
    float range = sym ? amax : __fsub_rn(mx, mn);
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
  const float lo = sym ? -7.0f : 0.0f, hi = sym ? 7.0f : 15.0f;
  uint32_t word = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float t = __fadd_rn(rintf(__fdiv_rn(w[i], sf)), zf);
    t = fminf(fmaxf(t, lo), hi);
    const int code = static_cast<int>(t) + (sym ? 8 : 0);
    word |= static_cast<uint32_t>(code & 0xF) << (4 * i);
  }
  res.word = word;
  res.bad = false;
  return res;
}

__global__ void __launch_bounds__(256) quantize_rtn_kernel(QuantParams p) {
  const int lane = threadIdx.x & 31;
  const int hl = lane & 15;
  const unsigned mask = (lane < 16) ? 0x0000FFFFu : 0xFFFF0000u;
  const long long nhalf = (long long)gridDim.x * (blockDim.x / 16);
  long long gid = ((long long)blockIdx.x * blockDim.x + threadIdx.x) / 16;

  // Two groups per iteration so each lane keeps two 16-byte loads in flight.
  for (; gid < p.groups; gid += 2 * nhalf) {
    const long long gid2 = gid + nhalf;
    const bool has2 = gid2 < p.groups;
    const uint4 raw1 = __ldcs(p.W + gid * 16 + hl);
    uint4 raw2 = make_uint4(0, 0, 0, 0);
    if (has2) raw2 = __ldcs(p.W + gid2 * 16 + hl);

    const float* a1 = p.awq ? p.awq + (gid % p.NG) * kGroup + 8 * hl : nullptr;
    GroupResult r1 = quantize_group(raw1, a1, mask, p.sym);
    p.qweight[gid * 16 + hl] = r1.word;
    if (hl == 0) {
      p.scales[gid] = r1.s16;
      if (!p.sym) p.zeros[gid] = r1.z16;
      if (r1.bad && p.d_status) atomicAdd(p.d_status, 1);
    }
    if (has2) {
      const float* a2 = p.awq ? p.awq + (gid2 % p.NG) * kGroup + 8 * hl : nullptr;
      GroupResult r2 = quantize_group(raw2, a2, mask, p.sym);
      p.qweight[gid2 * 16 + hl] = r2.word;
      if (hl == 0) {
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
  const long long halves_needed = (p.groups + 1) / 2;
  long long blocks = (halves_needed + 15) / 16;
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
