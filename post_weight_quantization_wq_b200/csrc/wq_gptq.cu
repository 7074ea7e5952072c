// wq_gptq.cu -- GPTQ: per-group 4-bit quantization of W [N][K] column by
// column, each column's rounding error fed back into the columns not yet
// quantized through the inverse Hessian of calibration inputs X [T][K]
// ("3.6 量化(Quantization)", section GPTQ: minimize ||W X - W_hat X||^2 with
// H = 2 X X^T, update W[:, F] -= e_j / [H^-1]_jj * [H^-1]_{j,F};
// "推理优化中“用精度换性能“的核心技术：量化", section 四.2: columns in natural
// order, per-column error feedback; "大模型量化全景解析", section 六.2: a
// damping term for numerical stability).  The output is the RTN format
// (codes, fp16 scales and zeros per group of 128), so wq_pack_layout and the
// linears consume it unchanged.
//
// The update rows of the restricted inverses are those of the upper
// triangular U with H^-1 = U^T U, and U = R^-1 for the upper triangular R
// with H = R R^T (the Cholesky factor of H with its index order reversed).
// With the residuals d_i = w_i - w_hat_i of the columns already quantized
// (original weights minus their dequantized values), the weight column j
// holds, when it is quantized,
//     w_j + (1 / R_jj) * sum_{i<j} d_i R_ij,
// and at the start of a group B of 128 columns (where the group's scale and
// zero are fixed from its 128 current weights) the group holds
//     W_B + (sum_{i<j0} d_i R_iB) R_BB^-1.
// So the GPU needs one Cholesky factorization of H and a 128 x 128
// triangular inverse per group, no K x K inverse:
//   1. H = 2 X^T X + damp * mean(diag H) * I in fp64 (GEMM);
//   2. rotate H by 180 degrees (H' = J H J), blocked lower Cholesky
//      H' = L L^T (64 x 64 diagonal blocks in one CTA, panel and trailing
//      updates as GEMMs), rotate back: R = J L J is upper, H = R R^T;
//   3. per group of 128 columns: invert R_BB, form the group's current
//      weights (GEMM), run the 128 columns of every row in order (one warp
//      per row: code, residual, in-group feedback), then add the group's
//      residuals times R[B, later] to the feedback accumulator (GEMM).
// Everything is fp64 (the pages fix no precision); the group parameters
// follow the RTN rules on the current weights rounded to fp32.
#include "wq_common.cuh"

namespace wq {

// ------------------------------------------------------------------ fp64 GEMM
// (GemmF64 is declared in wq_common.cuh.)

constexpr int kFB = 64;       // tile rows and columns
constexpr int kFK = 16;       // k per smem stage

__global__ void __launch_bounds__(256) gemm_f64_kernel(const GemmF64 p) {
  const int ti = blockIdx.y, tj = blockIdx.x;
  if (p.lower && tj > ti) return;
  __shared__ double As[kFK][kFB];
  __shared__ double Bs[kFK][kFB];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;   // this thread: rows ty + 16 r, columns tx + 16 c
  const int i0 = ti * kFB, j0 = tj * kFB;
  const bool a_kfast = (p.a_k == 1);
  const bool b_jfast = (p.b_j == 1);
  double acc[4][4];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[r][c] = 0.0;
  double ra[4], rb[4];
  auto load = [&](int k0) {
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int e = tid + 256 * t;
      const int ai = a_kfast ? e / kFK : e % kFB;
      const int ak = a_kfast ? e % kFK : e / kFB;
      const int gi = i0 + ai, gk = k0 + ak;
      ra[t] = (gi < p.M && gk < p.K) ? p.A[(long long)gi * p.a_i + (long long)gk * p.a_k] : 0.0;
      const int bj = b_jfast ? e % kFB : e / kFK;
      const int bk = b_jfast ? e / kFB : e % kFK;
      const int gj = j0 + bj, gk2 = k0 + bk;
      rb[t] = (gj < p.N && gk2 < p.K) ? p.B[(long long)gk2 * p.b_k + (long long)gj * p.b_j] : 0.0;
    }
  };
  auto store = [&]() {
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int e = tid + 256 * t;
      const int ai = a_kfast ? e / kFK : e % kFB;
      const int ak = a_kfast ? e % kFK : e / kFB;
      As[ak][ai] = ra[t];
      const int bj = b_jfast ? e % kFB : e / kFK;
      const int bk = b_jfast ? e / kFB : e % kFK;
      Bs[bk][bj] = rb[t];
    }
  };
  load(0);
  for (int k0 = 0; k0 < p.K; k0 += kFK) {
    __syncthreads();
    store();
    __syncthreads();
    if (k0 + kFK < p.K) load(k0 + kFK);     // next stage in flight during the math
#pragma unroll
    for (int kk = 0; kk < kFK; ++kk) {
      double a[4], b[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) a[r] = As[kk][ty + 16 * r];
#pragma unroll
      for (int c = 0; c < 4; ++c) b[c] = Bs[kk][tx + 16 * c];
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][c] = fma(a[r], b[c], acc[r][c]);
    }
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int gi = i0 + ty + 16 * r;
    if (gi >= p.M) continue;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int gj = j0 + tx + 16 * c;
      if (gj >= p.N) continue;
      double* cp = p.C + (long long)gi * p.ldc + gj;
      *cp = p.beta == 0.0 ? p.alpha * acc[r][c] : fma(p.alpha, acc[r][c], p.beta * *cp);
    }
  }
}

cudaError_t gemm_f64(const GemmF64& p, cudaStream_t stream) {
  if (p.M <= 0 || p.N <= 0) return cudaSuccess;
  dim3 grid((p.N + kFB - 1) / kFB, (p.M + kFB - 1) / kFB);
  gemm_f64_kernel<<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ helpers

__global__ void bf16_to_f64_kernel(const uint16_t* __restrict__ x, double* __restrict__ y,
                                   long long n) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x)
    y[i] = (double)__uint_as_float((uint32_t)x[i] << 16);
}

// H += damp * mean(diag H) * I; one CTA, the diagonal summed in a fixed order.
__global__ void __launch_bounds__(256) damp_kernel(double* H, int K, double damp) {
  __shared__ double part[256];
  double s = 0.0;
  for (int i = threadIdx.x; i < K; i += 256) s += H[(long long)i * K + i];
  part[threadIdx.x] = s;
  __syncthreads();
  for (int w = 128; w >= 1; w >>= 1) {
    if (threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
    __syncthreads();
  }
  const double add = damp * (part[0] / K);
  for (int i = threadIdx.x; i < K; i += 256) H[(long long)i * K + i] += add;
}

// In place: A(i, j) <-> A(K-1-i, K-1-j) for a K x K row-major matrix (the
// reversal J A J).
__global__ void rotate180_kernel(double* A, long long n) {
  const long long half = n / 2;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < half;
       e += (long long)gridDim.x * blockDim.x) {
    const double t = A[e];
    A[e] = A[n - 1 - e];
    A[n - 1 - e] = t;
  }
}

// Lower Cholesky of the 64 x 64 diagonal block at (r0, r0) of A (lda), in
// place (the block's upper part is zeroed), and the inverse of the factor
// into Linv [64][64] (row-major, lower).  A pivot that is not positive sets
// bit 2 of *status and is replaced by 1 so the rest stays finite.
constexpr int kPotrfSmem = 2 * 64 * 65 * (int)sizeof(double);

__global__ void __launch_bounds__(256) potrf64_kernel(double* A, long long lda, int r0,
                                                      double* Linv, int* status) {
  extern __shared__ double potrf_smem[];
  double (*S)[65] = reinterpret_cast<double (*)[65]>(potrf_smem);
  double (*X)[65] = reinterpret_cast<double (*)[65]>(potrf_smem + 64 * 65);
  const int tid = threadIdx.x;
  for (int e = tid; e < 64 * 64; e += 256) {
    const int i = e / 64, j = e % 64;
    S[i][j] = (j <= i) ? A[(long long)(r0 + i) * lda + r0 + j] : 0.0;
  }
  __syncthreads();
  for (int k = 0; k < 64; ++k) {
    if (tid == 0) {
      double d = S[k][k];
      if (!(d > 0.0)) {
        if (status) atomicOr(status, 2);
        d = 1.0;
      }
      S[k][k] = sqrt(d);
    }
    __syncthreads();
    for (int i = k + 1 + tid; i < 64; i += 256) S[i][k] /= S[k][k];
    __syncthreads();
    const int m = 63 - k;                  // trailing size
    for (int e = tid; e < m * m; e += 256) {
      const int i = k + 1 + e / m, j = k + 1 + e % m;
      if (j <= i) S[i][j] -= S[i][k] * S[j][k];
    }
    __syncthreads();
  }
  // inverse of the lower factor, one column per thread: L X = I
  if (tid < 64) {
    const int c = tid;
    for (int i = 0; i < 64; ++i) {
      double v = (i == c) ? 1.0 : 0.0;
      for (int k = c; k < i; ++k) v -= S[i][k] * X[k][c];
      X[i][c] = (i < c) ? 0.0 : v / S[i][i];
    }
  }
  __syncthreads();
  for (int e = tid; e < 64 * 64; e += 256) {
    const int i = e / 64, j = e % 64;
    A[(long long)(r0 + i) * lda + r0 + j] = (j <= i) ? S[i][j] : 0.0;
    Linv[e] = X[i][j];
  }
}

__global__ void copy_panel_kernel(const double* __restrict__ src, double* __restrict__ dst,
                                  long long ldd, int rows) {
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < (long long)rows * 64;
       e += (long long)gridDim.x * blockDim.x)
    dst[(e / 64) * ldd + (e % 64)] = src[e];
}

// Inverse of the 128 x 128 upper triangular block R[j0.., j0..] (ldr) into
// Rinv [128][128] (row-major, upper): one column per thread, back
// substitution; the block sits in shared memory.
__global__ void __launch_bounds__(128) trinv_upper128_kernel(const double* R, long long ldr,
                                                             int j0, double* Rinv) {
  extern __shared__ double U[];           // [128][129]
  const int c = threadIdx.x;
  for (int e = c; e < 128 * 128; e += 128) {
    const int i = e / 128, j = e % 128;
    U[i * 129 + j] = (j >= i) ? R[(long long)(j0 + i) * ldr + j0 + j] : 0.0;
  }
  for (int i = 0; i < 128; ++i) Rinv[i * 128 + c] = 0.0;
  __syncthreads();
  for (int i = 127; i >= 0; --i) {
    double v = (i == c) ? 1.0 : 0.0;
    for (int k = i + 1; k <= c; ++k) v -= U[i * 129 + k] * Rinv[k * 128 + c];
    if (i <= c) Rinv[i * 128 + c] = v / U[i * 129 + i];
  }
}

// ------------------------------------------------------------------ one group

struct GptqRows {
  const uint16_t* W;       // bf16 [N][K]
  const double* acc;       // [N][K]: sum_{i<j0} d_i R_ij (feedback of earlier groups)
  const double* cur0;      // [N][128]: acc_B R_BB^-1 (block-start correction)
  const double* R;         // [K][K], upper
  double* delta;           // out [N][128]: residuals d of this group
  uint32_t* qweight;       // [N][K/8]
  uint16_t* scales;        // [N][K/128]
  uint16_t* zeros;         // [N][K/128] or null (symmetric)
  int* status;
  int N, K, j0, sym;
};

constexpr int kGptqWarps = 8;
constexpr int kGptqRowsPerWarp = 4;

// One warp per row; lane l holds the columns l, l+32, l+64, l+96 of the
// group.  R_BB (the group's 128 x 128 block of R) sits in shared memory.
__global__ void __launch_bounds__(kGptqWarps * 32) gptq_group_kernel(const GptqRows p) {
  extern __shared__ double Rs[];           // [128][128]
  __shared__ uint8_t codes[kGptqWarps][128];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int e = threadIdx.x; e < 128 * 128; e += kGptqWarps * 32) {
    const int i = e / 128, j = e % 128;
    Rs[e] = p.R[(long long)(p.j0 + i) * p.K + p.j0 + j];
  }
  __syncthreads();
  const int g = p.j0 / kGroup;
  const int NG = p.K / kGroup;
  const double qlo = p.sym ? -7.0 : 0.0, qhi = p.sym ? 7.0 : 15.0;
  for (int rr = 0; rr < kGptqRowsPerWarp; ++rr) {
    const int n = (blockIdx.x * kGptqWarps + warp) * kGptqRowsPerWarp + rr;
    if (n >= p.N) break;                   // warp-uniform
    double w[4], a[4], in[4];
    float cur32[4];
    bool bad = false;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int c = lane + 32 * t;
      const long long idx = (long long)n * p.K + p.j0 + c;
      w[t] = (double)__uint_as_float((uint32_t)p.W[idx] << 16);
      a[t] = p.acc[idx];
      in[t] = 0.0;
      cur32[t] = (float)(w[t] + p.cur0[(long long)n * 128 + c]);
      bad |= !isfinite(cur32[t]);
    }
    // group scale and zero from the block-start weights rounded to fp32
    // (the RTN rules: range floored at 1e-8, IEEE divisions, fp16 RNE)
    float mn = fminf(fminf(cur32[0], cur32[1]), fminf(cur32[2], cur32[3]));
    float mx = fmaxf(fmaxf(cur32[0], cur32[1]), fmaxf(cur32[2], cur32[3]));
    float am = fmaxf(fmaxf(fabsf(cur32[0]), fabsf(cur32[1])), fmaxf(fabsf(cur32[2]), fabsf(cur32[3])));
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, o));
      mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
      am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, o));
    }
    bad = __any_sync(0xFFFFFFFFu, bad);
    uint16_t hs = 0x7E00, hz = 0x7E00;
    double s = 1.0, z = 0.0;
    if (!bad) {
      float range = p.sym ? am : __fsub_rn(mx, mn);
      if (range < 1e-8f) range = 1e-8f;
      hs = __half_as_ushort(__float2half_rn(__fdiv_rn(range, p.sym ? 7.0f : 15.0f)));
      if (hs == 0) hs = 0x0001;
      if ((hs & 0x7C00u) == 0x7C00u) bad = true;
    }
    if (!bad) {
      const float sf = __half2float(__ushort_as_half(hs));
      s = (double)sf;
      if (!p.sym) {
        const float zf = __fadd_rn(rintf(__fdiv_rn(-mn, sf)), 0.0f);
        hz = __half_as_ushort(__float2half_rn(zf));
        if ((hz & 0x7C00u) == 0x7C00u) bad = true;
        z = (double)__half2float(__ushort_as_half(hz));
      }
    }
    if (bad) {
      hs = 0x7E00;
      hz = 0x7E00;
      if (lane == 0 && p.status) atomicOr(p.status, 1);
    }
    // the 128 columns in order
    double qv[4], dv[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
#pragma unroll 4
      for (int jj = 0; jj < 32; ++jj) {
        const int j = 32 * t + jj;
        double d = 0.0, q = 0.0;
        if (lane == jj) {
          const double cur = w[t] + (a[t] + in[t]) / Rs[j * 128 + j];
          q = bad ? (p.sym ? -8.0 : 0.0) : fmin(fmax(rint(cur / s) + z, qlo), qhi);
          d = w[t] - s * (q - z);
          qv[t] = q;
          dv[t] = d;
        }
        d = __shfl_sync(0xFFFFFFFFu, d, jj);
#pragma unroll
        for (int t2 = 0; t2 < 4; ++t2)
          if (32 * t2 + lane > j) in[t2] = fma(d, Rs[j * 128 + 32 * t2 + lane], in[t2]);
      }
    }
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int c = lane + 32 * t;
      p.delta[(long long)n * 128 + c] = bad ? 0.0 : dv[t];
      codes[warp][c] = (uint8_t)((int)qv[t] + (p.sym ? 8 : 0));
    }
    __syncwarp();
    if (lane < 16) {
      uint32_t word = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) word |= ((uint32_t)codes[warp][8 * lane + i] & 0xFu) << (4 * i);
      p.qweight[(long long)n * (p.K / 8) + p.j0 / 8 + lane] = word;
    }
    if (lane == 0) {
      p.scales[(long long)n * NG + g] = hs;
      if (!p.sym) p.zeros[(long long)n * NG + g] = hz;
    }
    __syncwarp();
  }
}

// ------------------------------------------------------------------ driver

struct GptqWs {
  double *X64, *H, *Linv, *panel, *Rinv, *cur0, *delta, *acc;
};

static size_t align256(size_t b) { return (b + 255) / 256 * 256; }

static size_t gptq_layout(int T, int N, int K, GptqWs* w, uint8_t* base) {
  size_t off = 0;
  auto take = [&](double** p, size_t count) {
    if (w) *p = reinterpret_cast<double*>(base + off);
    off += align256(count * sizeof(double));
  };
  double* dummy = nullptr;
  take(w ? &w->X64 : &dummy, (size_t)T * K);
  take(w ? &w->H : &dummy, (size_t)K * K);
  take(w ? &w->Linv : &dummy, 64 * 64);
  take(w ? &w->panel : &dummy, (size_t)K * 64);
  take(w ? &w->Rinv : &dummy, 128 * 128);
  take(w ? &w->cur0 : &dummy, (size_t)N * 128);
  take(w ? &w->delta : &dummy, (size_t)N * 128);
  take(w ? &w->acc : &dummy, (size_t)N * K);
  return off;
}

size_t gptq_workspace_bytes(int T, int N, int K) { return gptq_layout(T, N, K, nullptr, nullptr); }

cudaError_t launch_gptq(const void* W, const void* X, int T, int N, int K, int sym, double damp,
                        uint32_t* qweight, void* scales, void* zeros, void* workspace,
                        int* d_status, cudaStream_t stream) {
  GptqWs w;
  gptq_layout(T, N, K, &w, static_cast<uint8_t*>(workspace));
  cudaError_t e;
  if (d_status && (e = cudaMemsetAsync(d_status, 0, sizeof(int), stream)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(w.acc, 0, (size_t)N * K * sizeof(double), stream)) != cudaSuccess)
    return e;
  static bool attr_set[64] = {false};
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    if ((e = cudaFuncSetAttribute(gptq_group_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  128 * 128 * 8)) != cudaSuccess)
      return e;
    if ((e = cudaFuncSetAttribute(potrf64_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  kPotrfSmem)) != cudaSuccess)
      return e;
    if ((e = cudaFuncSetAttribute(trinv_upper128_kernel,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, 128 * 129 * 8)) !=
        cudaSuccess)
      return e;
    attr_set[dev] = true;
  }

  // 1. H = 2 X^T X (+ damping)
  bf16_to_f64_kernel<<<1024, 256, 0, stream>>>(static_cast<const uint16_t*>(X), w.X64,
                                               (long long)T * K);
  GemmF64 h{w.X64, 1, K, w.X64, K, 1, w.H, K, K, K, T, 2.0, 0.0, 0};
  if ((e = gemm_f64(h, stream)) != cudaSuccess) return e;
  if (damp != 0.0) damp_kernel<<<1, 256, 0, stream>>>(w.H, K, damp);
  // 2. H' = J H J, lower Cholesky in place, R = J L J
  const long long kk = (long long)K * K;
  rotate180_kernel<<<1024, 256, 0, stream>>>(w.H, kk);
  for (int r0 = 0; r0 < K; r0 += 64) {
    potrf64_kernel<<<1, 256, kPotrfSmem, stream>>>(w.H, K, r0, w.Linv, d_status);
    const int below = K - r0 - 64;
    if (below <= 0) break;
    // panel P = A[below rows, block] * Linv^T
    GemmF64 pn{w.H + (long long)(r0 + 64) * K + r0, K, 1, w.Linv, 1, 64, w.panel, 64,
               below, 64, 64, 1.0, 0.0, 0};
    if ((e = gemm_f64(pn, stream)) != cudaSuccess) return e;
    copy_panel_kernel<<<256, 256, 0, stream>>>(w.panel, w.H + (long long)(r0 + 64) * K + r0, K,
                                               below);
    // trailing lower update A22 -= P P^T
    GemmF64 tr{w.panel, 64, 1, w.panel, 1, 64, w.H + (long long)(r0 + 64) * K + (r0 + 64), K,
               below, below, 64, -1.0, 1.0, 1};
    if ((e = gemm_f64(tr, stream)) != cudaSuccess) return e;
  }
  rotate180_kernel<<<1024, 256, 0, stream>>>(w.H, kk);
  const double* R = w.H;
  // 3. groups of 128 columns in order
  const int grid_rows = (N + kGptqWarps * kGptqRowsPerWarp - 1) / (kGptqWarps * kGptqRowsPerWarp);
  for (int j0 = 0; j0 < K; j0 += kGroup) {
    trinv_upper128_kernel<<<1, 128, 128 * 129 * 8, stream>>>(R, K, j0, w.Rinv);
    GemmF64 c0{w.acc + j0, K, 1, w.Rinv, 128, 1, w.cur0, 128, N, 128, 128, 1.0, 0.0, 0};
    if ((e = gemm_f64(c0, stream)) != cudaSuccess) return e;
    GptqRows pr{static_cast<const uint16_t*>(W), w.acc, w.cur0, R, w.delta, qweight,
                static_cast<uint16_t*>(scales), static_cast<uint16_t*>(zeros), d_status,
                N, K, j0, sym};
    gptq_group_kernel<<<grid_rows, kGptqWarps * 32, 128 * 128 * 8, stream>>>(pr);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int rest = K - j0 - kGroup;
    if (rest > 0) {
      GemmF64 up{w.delta, 128, 1, R + (long long)j0 * K + j0 + kGroup, K, 1, w.acc + j0 + kGroup,
                 K, N, rest, 128, 1.0, 1.0, 0};
      if ((e = gemm_f64(up, stream)) != cudaSuccess) return e;
    }
  }
  return cudaGetLastError();
}

}  // namespace wq
