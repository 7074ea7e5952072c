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
//   * persistent grid, every CTA streams a contiguous run of layout tiles
//     (128 rows x 512 inputs: 32 KB of nibbles + 1-2 KB of fp16 metadata, one
//     contiguous block in memory) through a ring of shared-memory stages with
//     1-D bulk async copies (cp.async.bulk) completing on mbarriers; one
//     producer warp issues the copies, eight consumer warps compute;
//   * tiles are ordered slab-major, so a CTA keeps one K-slab of activations
//     (fp32, with the AWQ factor applied once) in shared memory for many
//     tiles;
//   * dequantization in registers: a nibble at bit 4i of a word, OR-ed into
//     the fp32 pattern of 2^(23-4i), is the float 2^(23-4i) + q (one LOP3);
//     one packed fp32x2 subtraction of the constants gives two exact codes,
//     and packed fp32x2 FMAs accumulate x * q; per (row, group) the sum is
//     corrected by z * sum(x) and scaled by s16 in fp32;
//   * a half warp owns one row: lane p covers inputs 32p..32p+31 of the slab;
//     the 16 lanes' partial sums of several rows are combined with a
//     transposing shuffle reduction;
//   * split-K across slabs: every (slab, 16-row block) writes fp32 partials to
//     the workspace; the last of the K-slabs to finish (counted with an atomic
//     per 16-row block) adds them in slab order, so the result is the same
//     whatever order the GPU runs the tiles in, and resets its counter.
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
  float* partials;         // fp32 [NS][Mp][Npad] (NS > 1)
  unsigned* counters;      // [Npad / 16]        (NS > 1)
  int* err;                // device error word
  Geom g;
  int M;                   // actual rows of x / y (<= Mp)
  long long tiles;         // NS * NB
  unsigned long long wait_ns;
  unsigned long long drain_ns;
};

constexpr int kConsumerWarps = 8;
constexpr int kGemvThreads = (kConsumerWarps + 1) * 32;
constexpr int kXPitch = kSlabK + kSlabK / 8;     // 4 pad floats per 32 inputs

__device__ __forceinline__ int xpad(int k) { return k + ((k >> 5) << 2); }

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

template <int MP, int JR, int STAGES, int MINB>
__global__ void __launch_bounds__(kGemvThreads, MINB) gemv_w4a16_kernel(GemvParams prm) {
  extern __shared__ __align__(128) uint8_t smem[];
  const Geom g = prm.g;
  const long long full_tile = g.full_tile;
  uint8_t* ring = smem;
  float* xs = reinterpret_cast<float*>(smem + STAGES * full_tile);
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(xs + MP * kXPitch);
  uint64_t* empty_bar = full_bar + STAGES;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty_bar + STAGES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long t0 = (long long)blockIdx.x * prm.tiles / gridDim.x;
  const long long t1 = (long long)(blockIdx.x + 1) * prm.tiles / gridDim.x;
  const int ntiles = (int)(t1 - t0);

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], kConsumerWarps);
    }
    *abort_flag = 0;
    fence_mbarrier_init();
  }
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
            break;
          }
        }
        if (*abort_flag) break;
        const long long t = t0 + i;
        const int s = (int)(t / g.NB), b = (int)(t % g.NB);
        const uint32_t bytes = (uint32_t)tile_bytes(g, slab_groups(g, s));
        mbar_arrive_expect_tx(&full_bar[st], bytes);
        bulk_copy_g2s(ring + st * full_tile, prm.packed + tile_offset(g, s, b), bytes,
                      &full_bar[st]);
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
  const int h = lane >> 4;          // row within the pair handled by this half warp
  const int p = lane & 15;          // 32-input chunk of the slab
  constexpr int V = JR * MP;
  using RM = ReduceMap<V>;
  const uint32_t E0 = 0x4B000000u, E1 = 0x49000000u, E2 = 0x47000000u, E3 = 0x45000000u;
  const float2 negE01 = make_float2(-8388608.0f, -524288.0f);
  const float2 negE23 = make_float2(-32768.0f, -2048.0f);

  float xsum[MP];
  int cur_s = -1;
  bool aborted = false;

  for (int i = 0; i < ntiles; ++i) {
    const long long t = t0 + i;
    const int s = (int)(t / g.NB), b = (int)(t % g.NB);
    const int gs = slab_groups(g, s);
    const int st = i % STAGES;

    if (s != cur_s) {
      // Stage this slab's activations (fp32, AWQ factor applied) once.  Every
      // consumer warp takes part, aborted or not, so the barrier always fills.
      named_barrier_sync(1, kConsumerWarps * 32);
      const int kbase = s * kSlabK;
      for (int idx = threadIdx.x; idx < MP * kSlabK; idx += kConsumerWarps * 32) {
        const int m = idx / kSlabK, k = idx % kSlabK, kk = kbase + k;
        float v = 0.0f;
        if (m < prm.M && kk < g.K) {
          v = __uint_as_float((uint32_t)prm.x[(size_t)m * g.K + kk] << 16);
          if (prm.inv_s) v = __fmul_rn(v, __ldg(prm.inv_s + kk));
        }
        xs[m * kXPitch + xpad(k)] = v;
      }
      named_barrier_sync(1, kConsumerWarps * 32);
#pragma unroll
      for (int m = 0; m < MP; ++m) {
        float a = 0.0f;
        const float4* xp = reinterpret_cast<const float4*>(xs + m * kXPitch + xpad(32 * p));
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 v = xp[q];
          a += (v.x + v.y) + (v.z + v.w);
        }
        xsum[m] = a;
      }
      cur_s = s;
    }

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
      const uint8_t* tile = ring + st * full_tile;
      const uint8_t* meta = tile + kTileRows * gs * kCodeBytesPerGroupRow;
      const int pitch = gs * kCodeBytesPerGroupRow;
      const bool active = p < gs * 4;
      const int grp = p >> 2;

#pragma unroll 1
      for (int jb = 0; jb < 8; jb += JR) {
        uint4 c[JR];
        float sc[JR], zc[JR];
#pragma unroll
        for (int j = 0; j < JR; ++j) {
          const int r = warp * 16 + 2 * (jb + j) + h;
          c[j] = make_uint4(0, 0, 0, 0);
          sc[j] = 0.0f;
          zc[j] = 0.0f;
          if (active) {
            c[j] = *reinterpret_cast<const uint4*>(tile + r * pitch + p * 16);
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
#pragma unroll
        for (int j = 0; j < JR; ++j)
#pragma unroll
          for (int m = 0; m < MP; ++m) acc[j][m] = make_float2(0.0f, 0.0f);

#pragma unroll
        for (int wd = 0; wd < 4; ++wd) {
          float2 xv[MP][4];
#pragma unroll
          for (int m = 0; m < MP; ++m) {
            const float4* xp =
                reinterpret_cast<const float4*>(xs + m * kXPitch + xpad(32 * p + 8 * wd));
            const float4 a = xp[0], bq = xp[1];
            xv[m][0] = make_float2(a.x, a.y);
            xv[m][1] = make_float2(a.z, a.w);
            xv[m][2] = make_float2(bq.x, bq.y);
            xv[m][3] = make_float2(bq.z, bq.w);
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

        // y partial of (row, m) over this lane's 32 inputs:
        //   s16 * (sum x*q - z * sum x)
        float v[V];
#pragma unroll
        for (int j = 0; j < JR; ++j)
#pragma unroll
          for (int m = 0; m < MP; ++m)
            v[j * MP + m] = active ? sc[j] * ((acc[j][m].x + acc[j][m].y) - zc[j] * xsum[m]) : 0.0f;
        half_transpose_reduce<V>(v, p);

        if (RM::writer(p)) {
#pragma unroll
          for (int i2 = 0; i2 < RM::kPerLane; ++i2) {
            const int idx = RM::index(i2, p);
            const int j = idx / MP, m = idx % MP;
            const int n = b * kTileRows + warp * 16 + 2 * (jb + j) + h;
            if (m < prm.M) {
              if (g.NS == 1) {
                if (n < g.N) prm.y[(size_t)m * g.N + n] = v[i2];
              } else {
                prm.partials[((size_t)s * MP + m) * g.Npad + n] = v[i2];
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[st]);
    }

    // ---- split-K completion: the last slab to finish a 16-row block sums it
    if (g.NS > 1) {
      __threadfence();
      __syncwarp();
      unsigned prev = 0;
      unsigned* ctr = prm.counters + (size_t)b * (kTileRows / kRowsPerCounter) + warp;
      if (lane == 0) prev = atomicAdd(ctr, 1u);
      prev = __shfl_sync(0xFFFFFFFFu, prev, 0);
      if (prev == (unsigned)(g.NS - 1)) {
        __threadfence();
        if (!aborted) {
          for (int e = lane; e < kRowsPerCounter * prm.M; e += 32) {
            const int n = b * kTileRows + warp * kRowsPerCounter + (e % kRowsPerCounter);
            const int m = e / kRowsPerCounter;
            float acc = 0.0f;
            const float* src = prm.partials + (size_t)m * g.Npad + n;
            const size_t slab_stride = (size_t)MP * g.Npad;
#pragma unroll 8
            for (int s2 = 0; s2 < g.NS; ++s2) acc += __ldcg(src + s2 * slab_stride);
            if (n < g.N) prm.y[(size_t)m * g.N + n] = acc;
          }
        }
        if (lane == 0) *ctr = 0u;
      }
    }
  }
}

// ------------------------------------------------------------------ launcher

struct GemvConfig {
  const void* fn;
  int stages;
  size_t smem;
};

template <int MP, int JR, int STAGES, int MINB>
static GemvConfig gemv_config(const Geom& g) {
  GemvConfig c;
  c.fn = reinterpret_cast<const void*>(&gemv_w4a16_kernel<MP, JR, STAGES, MINB>);
  c.stages = STAGES;
  c.smem = (size_t)STAGES * g.full_tile + (size_t)MP * kXPitch * sizeof(float) +
           2 * STAGES * sizeof(uint64_t) + 16;
  return c;
}

static GemvConfig pick_gemv(int M, const Geom& g) {
  if (M <= 1) return gemv_config<1, 8, 3, 2>(g);
  if (M <= 2) return gemv_config<2, 4, 3, 2>(g);
  if (M <= 4) return gemv_config<4, 4, 4, 1>(g);
  return gemv_config<8, 2, 4, 1>(g);
}

size_t gemv_workspace_bytes(int M, int N, int K) {
  const Geom g = make_geom(N, K, 1);
  if (g.NS <= 1) return 0;
  const int MP = M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : 8;
  return (size_t)kCounterBytes + (size_t)g.NS * MP * g.Npad * sizeof(float);
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

  const GemvConfig c = pick_gemv(M, prm.g);
  int per_sm = 0;
  cudaError_t e = kernel_setup(c.fn, c.smem, kGemvThreads, &per_sm);
  if (e != cudaSuccess) return e;
  long long grid = (long long)num_sms * per_sm;
  if (grid > prm.tiles) grid = prm.tiles;
  void* args[] = {&prm};
  return cudaLaunchKernel(c.fn, dim3((unsigned)grid), dim3(kGemvThreads), args, c.smem, stream);
}

}  // namespace wq
