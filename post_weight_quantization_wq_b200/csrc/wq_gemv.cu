// wq_gemv.cu -- W4A16 decode linear for M = 1..8 activation rows on the CUDA
// cores:  y[m][n] = sum_g s16[n][g] * sum_{k in g} x'[m][k] * (q[n][k] - z[n][g]).
//
// Weight-only 4-bit decode is bound by the bytes of the weights ("推理优化中
// “用精度换性能“的核心技术：量化", section 一; "3.6 量化(Quantization)",
// section 为什么重要): the weights are dequantized in registers inside the
// matmul kernel and multiplied with 16-bit activations, accumulating in fp32
// ("3.6 量化(Quantization)", section 仅权重 vs 权重 + 激活; "大模型量化全景解析",
// section dtype、storage dtype、compute dtype).
//
// Design (B200, sm_100a):
//   * persistent grid; CTA c owns the contiguous run [t0, t1) of the tile
//     sequence u = b * NS + s (row tile b of 128 output rows, K-slab s of 512
//     inputs), so it walks the slabs of one row tile after another and keeps
//     each row's running sum in registers;
//   * one producer warp streams every tile (32 KB of nibbles + its fp16
//     metadata, contiguous in memory) together with the matching slab of x
//     (and of the AWQ factor) into a ring of shared-memory stages with 1-D
//     bulk async copies (cp.async.bulk) that complete on mbarriers; eight
//     consumer warps compute;
//   * dequantization in registers: a nibble at bit 4i of a word, OR-ed into
//     the fp32 pattern of 2^(23-4i), is the float 2^(23-4i) + q (one LOP3);
//     a packed fp32x2 subtraction gives two exact codes and packed fp32x2 FMAs
//     accumulate x * q; per (row, group) the sum is corrected by z * sum(x)
//     and scaled by the fp16 scale in fp32;
//   * a half warp owns one row of a tile: lane p covers inputs 32p..32p+31
//     of the slab; the 16 lanes' partial sums of several rows are combined
//     with a transposing shuffle reduction;
//   * a row tile whose slabs are split between CTAs (only at the ends of a
//     CTA's run) is finished through the workspace: each piece writes its
//     fp32 partial, and the last piece to arrive (an atomic counter per 16
//     rows) adds the pieces in slab order and resets the counter, so y does
//     not depend on the order the GPU runs the CTAs in;
//   * every wait is bounded (globaltimer): on timeout the kernel records the
//     device error word, stops issuing copies, waits (bounded) for its copies
//     in flight and returns.
#include "wq_common.cuh"

namespace wq {

struct GemvParams {
  const uint8_t* packed;
  const uint16_t* x;       // bf16 [M][K]
  const float* inv_s;      // fp32 [K] or nullptr
  float* y;                // fp32 [M][N]
  float* partials;         // fp32 [NS][MP][Npad]
  unsigned* counters;      // one per 16 rows
  int* err;                // device error word
  Geom g;
  int M;                   // rows of x / y (<= MP)
  long long tiles;         // NS * NB
  unsigned long long wait_ns;
  unsigned long long drain_ns;
};

constexpr int kConsumerWarps = 8;
constexpr int kGemvThreads = (kConsumerWarps + 1) * 32;
constexpr int kMaxFullTile = kTileRows * kSlabGroups * (kCodeBytesPerGroupRow + 4);
constexpr int kInvBytes = kSlabK * 4;

template <int MP>
struct StageLayout {
  static constexpr int kX = kMaxFullTile;                 // bf16 [MP][512]
  static constexpr int kInv = kX + MP * kSlabK * 2;       // fp32 [512]
  static constexpr int kBytes = kInv + kInvBytes;
};

// Sum v[] over the 16 lanes of a half warp.  After the call, for V >= 16 a
// lane holds V/16 sums, v[i] being the sum of index i + (V/16)*p; for V < 16
// a lane holds one sum, of index p >> (4 - log2 V).  (p = lane & 15.)
template <int V>
__device__ __forceinline__ void half_transpose_reduce(float (&v)[V], int p) {
  int C = V;
#pragma unroll
  for (int mk = 8; mk >= 1; mk >>= 1) {
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

template <int V>
struct ReduceMap {
  static constexpr int kLog = (V >= 16) ? 4 : (V >= 8 ? 3 : (V >= 4 ? 2 : (V >= 2 ? 1 : 0)));
  static constexpr int kPerLane = (V >= 16) ? V / 16 : 1;
  __device__ static bool writer(int p) { return V >= 16 || (p & ((16 >> kLog) - 1)) == 0; }
  __device__ static int index(int i, int p) { return V >= 16 ? i + kPerLane * p : (p >> (4 - kLog)); }
};

// CTA that owns tile u when T tiles are split evenly over G CTAs
// (t0(c) = floor(c*T/G)).
__device__ __forceinline__ int owner_cta(long long u, long long T, int G) {
  return (int)(((u + 1) * G + T - 1) / T) - 1;
}

template <int MP, int JR, int STAGES, int MINB>
__global__ void __launch_bounds__(kGemvThreads, MINB) gemv_w4a16_kernel(GemvParams prm) {
  using SL = StageLayout<MP>;
  extern __shared__ __align__(128) uint8_t smem[];
  const Geom g = prm.g;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + STAGES * SL::kBytes);
  uint64_t* empty_bar = full_bar + STAGES;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty_bar + STAGES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const long long t0 = (long long)blockIdx.x * prm.tiles / G;
  const long long t1 = (long long)(blockIdx.x + 1) * prm.tiles / G;
  const int ntiles = (int)(t1 - t0);

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], kConsumerWarps);
    }
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  // Rows of x beyond M are never copied in: zero them once in every stage.
  for (int st = 0; st < STAGES; ++st)
    for (int i = threadIdx.x + prm.M * kSlabK / 8; i < MP * kSlabK / 8; i += blockDim.x)
      reinterpret_cast<uint4*>(smem + st * SL::kBytes + SL::kX)[i] = make_uint4(0, 0, 0, 0);
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < ntiles; ++i) {
        const int st = i % STAGES;
        if (i >= STAGES) {
          if (!mbar_wait_bounded(&empty_bar[st], ((i / STAGES) - 1) & 1, prm.wait_ns)) {
            atomicOr(prm.err, kDevErrTimeout);
            *abort_flag = 1;
          }
        }
        if (*abort_flag) break;
        const long long u = t0 + i;
        const int b = (int)(u / g.NS), s = (int)(u % g.NS);
        const int gs = slab_groups(g, s);
        const uint32_t tbytes = (uint32_t)tile_bytes(g, gs);
        const uint32_t xbytes = gs * kGroup * 2;
        const uint32_t ibytes = prm.inv_s ? gs * kGroup * 4 : 0;
        uint8_t* stage = smem + st * SL::kBytes;
        mbar_arrive_expect_tx(&full_bar[st], tbytes + prm.M * xbytes + ibytes);
        bulk_copy_g2s(stage, prm.packed + tile_offset(g, s, b), tbytes, &full_bar[st]);
        for (int m = 0; m < prm.M; ++m)
          bulk_copy_g2s(stage + SL::kX + m * kSlabK * 2, prm.x + (size_t)m * g.K + s * kSlabK,
                        xbytes, &full_bar[st]);
        if (ibytes)
          bulk_copy_g2s(stage + SL::kInv, prm.inv_s + s * kSlabK, ibytes, &full_bar[st]);
        issued = i + 1;
      }
      if (*abort_flag) {
        // Wait (bounded) for every copy still in flight before the CTA exits.
        for (int st = 0; st < STAGES && st < issued; ++st) {
          const int uses = (issued - 1 - st) / STAGES + 1;   // copies issued on stage st
          mbar_wait_bounded(&full_bar[st], (uses - 1) & 1, prm.drain_ns);
        }
      }
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int h = lane >> 4;          // row of the pair handled by this half warp
  const int p = lane & 15;          // 32-input chunk of the slab
  constexpr int V = JR * MP;
  constexpr int kPasses = 8 / JR;
  using RM = ReduceMap<V>;
  const uint32_t E0 = 0x4B000000u, E1 = 0x49000000u, E2 = 0x47000000u, E3 = 0x45000000u;
  const float2 negE01 = make_float2(-8388608.0f, -524288.0f);
  const float2 negE23 = make_float2(-32768.0f, -2048.0f);
  const bool awq = prm.inv_s != nullptr;

  float run[kPasses][RM::kPerLane];
#pragma unroll
  for (int a = 0; a < kPasses; ++a)
#pragma unroll
    for (int i2 = 0; i2 < RM::kPerLane; ++i2) run[a][i2] = 0.0f;
  int piece_s0 = -1;                // first slab of the current row tile in this CTA
  bool aborted = false;

  for (int i = 0; i < ntiles; ++i) {
    const long long u = t0 + i;
    const int b = (int)(u / g.NS), s = (int)(u % g.NS);
    const int gs = slab_groups(g, s);
    const int st = i % STAGES;
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
      const uint16_t* xsm = reinterpret_cast<const uint16_t*>(stage + SL::kX);
      const float* ism = reinterpret_cast<const float*>(stage + SL::kInv);
      const int pitch = gs * kCodeBytesPerGroupRow;
      const bool active = p < gs * 4;
      const int grp = p >> 2;

#pragma unroll 1
      for (int pass = 0; pass < kPasses; ++pass) {
        const int jb = pass * JR;
        uint4 c[JR];
        float sc[JR], zc[JR];
#pragma unroll
        for (int j = 0; j < JR; ++j) {
          const int r = warp * 16 + 2 * (jb + j) + h;
          c[j] = make_uint4(0, 0, 0, 0);
          sc[j] = 0.0f;
          zc[j] = 0.0f;
          if (active) {
            c[j] = *reinterpret_cast<const uint4*>(stage + r * pitch + p * 16);
            if (g.sym) {
              sc[j] = __half2float(reinterpret_cast<const __half*>(meta)[r * gs + grp]);
              zc[j] = 8.0f;
            } else {
              const __half2 sz = reinterpret_cast<const __half2*>(meta)[r * gs + grp];
              sc[j] = __low2float(sz);
              zc[j] = __high2float(sz);
            }
          }
        }
        float2 acc[JR][MP];
        float2 xs2[MP];
#pragma unroll
        for (int m = 0; m < MP; ++m) {
          xs2[m] = make_float2(0.0f, 0.0f);
#pragma unroll
          for (int j = 0; j < JR; ++j) acc[j][m] = make_float2(0.0f, 0.0f);
        }

#pragma unroll
        for (int wd = 0; wd < 4; ++wd) {
          // x' for the 8 inputs of word wd, as fp32 pairs (bf16 -> fp32 is a shift)
          float2 xv[MP][4];
          float4 ia = make_float4(1.f, 1.f, 1.f, 1.f), ib = ia;
          if (awq && active) {
            ia = *reinterpret_cast<const float4*>(ism + 32 * p + 8 * wd);
            ib = *reinterpret_cast<const float4*>(ism + 32 * p + 8 * wd + 4);
          }
#pragma unroll
          for (int m = 0; m < MP; ++m) {
            const uint4 xb = *reinterpret_cast<const uint4*>(xsm + m * kSlabK + 32 * p + 8 * wd);
            xv[m][0] = make_float2(__uint_as_float(xb.x << 16), __uint_as_float(xb.x & 0xFFFF0000u));
            xv[m][1] = make_float2(__uint_as_float(xb.y << 16), __uint_as_float(xb.y & 0xFFFF0000u));
            xv[m][2] = make_float2(__uint_as_float(xb.z << 16), __uint_as_float(xb.z & 0xFFFF0000u));
            xv[m][3] = make_float2(__uint_as_float(xb.w << 16), __uint_as_float(xb.w & 0xFFFF0000u));
            if (awq) {
              xv[m][0] = __fmul2_rn(xv[m][0], make_float2(ia.x, ia.y));
              xv[m][1] = __fmul2_rn(xv[m][1], make_float2(ia.z, ia.w));
              xv[m][2] = __fmul2_rn(xv[m][2], make_float2(ib.x, ib.y));
              xv[m][3] = __fmul2_rn(xv[m][3], make_float2(ib.z, ib.w));
            }
            xs2[m] = __fadd2_rn(xs2[m], __fadd2_rn(__fadd2_rn(xv[m][0], xv[m][1]),
                                                 __fadd2_rn(xv[m][2], xv[m][3])));
          }
#pragma unroll
          for (int j = 0; j < JR; ++j) {
            const uint32_t lo = wd == 0 ? c[j].x : wd == 1 ? c[j].y : wd == 2 ? c[j].z : c[j].w;
            const uint32_t hi = lo >> 16;
            const float2 q01 = __fadd2_rn(make_float2(__uint_as_float((lo & 0xFu) | E0),
                                                      __uint_as_float((lo & 0xF0u) | E1)),
                                          negE01);
            const float2 q23 = __fadd2_rn(make_float2(__uint_as_float((lo & 0xF00u) | E2),
                                                      __uint_as_float((lo & 0xF000u) | E3)),
                                          negE23);
            const float2 q45 = __fadd2_rn(make_float2(__uint_as_float((hi & 0xFu) | E0),
                                                      __uint_as_float((hi & 0xF0u) | E1)),
                                          negE01);
            const float2 q67 = __fadd2_rn(make_float2(__uint_as_float((hi & 0xF00u) | E2),
                                                      __uint_as_float((hi & 0xF000u) | E3)),
                                          negE23);
#pragma unroll
            for (int m = 0; m < MP; ++m) {
              float2 a = acc[j][m];
              a = __ffma2_rn(q01, xv[m][0], a);
              a = __ffma2_rn(q23, xv[m][1], a);
              a = __ffma2_rn(q45, xv[m][2], a);
              a = __ffma2_rn(q67, xv[m][3], a);
              acc[j][m] = a;
            }
          }
        }

        // partial of (row, m) over this lane's 32 inputs: s16 * (sum x*q - z * sum x)
        float v[V];
#pragma unroll
        for (int j = 0; j < JR; ++j)
#pragma unroll
          for (int m = 0; m < MP; ++m)
            v[j * MP + m] = active ? sc[j] * ((acc[j][m].x + acc[j][m].y) -
                                              zc[j] * (xs2[m].x + xs2[m].y))
                                   : 0.0f;
        half_transpose_reduce<V>(v, p);
#pragma unroll
        for (int i2 = 0; i2 < RM::kPerLane; ++i2) run[pass][i2] += v[i2];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[st]);
    }

    // ---- end of this CTA's piece of row tile b: write y or a partial
    const bool piece_end = (s == g.NS - 1) || (i == ntiles - 1);
    if (piece_end) {
      const bool whole = (piece_s0 == 0) && (s == g.NS - 1);
      if (whole) {
        if (!aborted && RM::writer(p)) {
#pragma unroll
          for (int pass = 0; pass < kPasses; ++pass)
#pragma unroll
            for (int i2 = 0; i2 < RM::kPerLane; ++i2) {
              const int idx = RM::index(i2, p);
              const int j = idx / MP, m = idx % MP;
              const int n = b * kTileRows + warp * 16 + 2 * (pass * JR + j) + h;
              if (m < prm.M && n < g.N) prm.y[(size_t)m * g.N + n] = run[pass][i2];
            }
        }
      } else {
        // Partial piece: its slot is its first slab.
        if (!aborted && RM::writer(p)) {
#pragma unroll
          for (int pass = 0; pass < kPasses; ++pass)
#pragma unroll
            for (int i2 = 0; i2 < RM::kPerLane; ++i2) {
              const int idx = RM::index(i2, p);
              const int j = idx / MP, m = idx % MP;
              const int n = b * kTileRows + warp * 16 + 2 * (pass * JR + j) + h;
              if (m < prm.M)
                prm.partials[((size_t)piece_s0 * MP + m) * g.Npad + n] = run[pass][i2];
            }
        }
        __threadfence();
        __syncwarp();
        const long long ub = (long long)b * g.NS;
        const int c_first = owner_cta(ub, prm.tiles, G);
        const int c_last = owner_cta(ub + g.NS - 1, prm.tiles, G);
        unsigned prev = 0;
        unsigned* ctr = prm.counters + (size_t)b * (kTileRows / kRowsPerCounter) + warp;
        if (lane == 0) prev = atomicAdd(ctr, 1u);
        prev = __shfl_sync(0xFFFFFFFFu, prev, 0);
        if (prev == (unsigned)(c_last - c_first)) {
          // Last piece: add all pieces in slab order, reset the counter.
          __threadfence();
          if (!aborted) {
            for (int e = lane; e < kRowsPerCounter * prm.M; e += 32) {
              const int n = b * kTileRows + warp * kRowsPerCounter + (e % kRowsPerCounter);
              const int m = e / kRowsPerCounter;
              float tot = 0.0f;
              for (int c2 = c_first; c2 <= c_last; ++c2) {
                const long long tc = (long long)c2 * prm.tiles / G;
                const int sa = (int)((tc > ub ? tc : ub) - ub);
                tot += __ldcg(prm.partials + ((size_t)sa * MP + m) * g.Npad + n);
              }
              if (n < g.N) prm.y[(size_t)m * g.N + n] = tot;
            }
          }
          if (lane == 0) *ctr = 0u;
        }
      }
#pragma unroll
      for (int a = 0; a < kPasses; ++a)
#pragma unroll
        for (int i2 = 0; i2 < RM::kPerLane; ++i2) run[a][i2] = 0.0f;
      piece_s0 = -1;
    }
  }
}

// ------------------------------------------------------------------ launcher

struct GemvConfig {
  const void* fn;
  size_t smem;
};

template <int MP, int JR, int STAGES, int MINB>
static GemvConfig gemv_config() {
  GemvConfig c;
  c.fn = reinterpret_cast<const void*>(&gemv_w4a16_kernel<MP, JR, STAGES, MINB>);
  c.smem = (size_t)STAGES * StageLayout<MP>::kBytes + 2 * STAGES * sizeof(uint64_t) + 16;
  return c;
}

static int padded_m(int M) { return M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : 8; }

static GemvConfig pick_gemv(int M) {
  switch (padded_m(M)) {
    case 1: return gemv_config<1, 8, 3, 2>();
    case 2: return gemv_config<2, 4, 3, 2>();
    case 4: return gemv_config<4, 4, 4, 1>();
    default: return gemv_config<8, 2, 4, 1>();
  }
}

size_t gemv_workspace_bytes(int M, int N, int K) {
  const Geom g = make_geom(N, K, 1);
  if (g.NS <= 1) return 0;
  return (size_t)kCounterBytes + (size_t)g.NS * padded_m(M) * g.Npad * sizeof(float);
}

cudaError_t launch_gemv(const void* x, const float* inv_s, const void* packed, int M, int N,
                        int K, int sym, float* y, void* workspace, int* err, int num_sms,
                        unsigned long long wait_ns, cudaStream_t stream) {
  GemvParams prm;
  prm.g = make_geom(N, K, sym);
  prm.packed = static_cast<const uint8_t*>(packed);
  prm.x = static_cast<const uint16_t*>(x);
  prm.inv_s = inv_s;
  prm.y = y;
  prm.counters = static_cast<unsigned*>(workspace);
  prm.partials = workspace ? reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kCounterBytes)
                           : nullptr;
  prm.err = err;
  prm.M = M;
  prm.tiles = (long long)prm.g.NS * prm.g.NB;
  prm.wait_ns = wait_ns;
  prm.drain_ns = 1000000000ull;

  const GemvConfig c = pick_gemv(M);
  int per_sm = 0;
  cudaError_t e = kernel_setup(c.fn, c.smem, kGemvThreads, &per_sm);
  if (e != cudaSuccess) return e;
  long long grid = (long long)num_sms * per_sm;
  if (grid > prm.tiles) grid = prm.tiles;
  void* args[] = {&prm};
  return cudaLaunchKernel(c.fn, dim3((unsigned)grid), dim3(kGemvThreads), args, c.smem, stream);
}

}  // namespace wq
