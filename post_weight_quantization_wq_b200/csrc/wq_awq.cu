// wq_awq.cu -- AWQ scale search: for alpha on the grid i / n_grid, scale the
// input channels by s = s_X^alpha (s_X the mean activation magnitude of each
// channel over the calibration rows), quantize W diag(s) with per-group RTN,
// and measure the layer's output error on the calibration inputs with the
// activations divided by s; keep the alpha with the smallest error
// ("3.6 量化(Quantization)", section AWQ: s = s_X^alpha, alpha searched in
// [0, 1] per layer on calibration data, y = sum_j quant(s_j w_j) x_j / s_j;
// "后训练量化（PTQ, Post-Training Quantization）", section AWQ).
//
// Per alpha:
//   1. s_j = m_j / exp(mean_j log m_j), m_j = s_X,j^alpha (fp64; the geometric
//      mean normalization of the scale), rounded to fp32 -- the format the
//      quantizer takes;
//   2. the RTN quantizer of wq_quantize.cu on W with the AWQ factor s (codes,
//      fp16 scales and zeros, bit-identical to wq_quantize_rtn);
//   3. D = X Delta^T with Delta[n][k] = W[n][k] - w_hat'[n][k] / s_k in fp64
//      (w_hat' = s16 (q - z16), exact), i.e. the difference between the
//      unquantized layer and the AWQ-folded quantized one on every
//      calibration row, by the fp64 GEMM kernel;
//   4. loss = sum of D^2, reduced in a fixed order (deterministic).
// Then the first alpha with the smallest loss is chosen and its s written out.
#include "wq_common.cuh"

namespace wq {

cudaError_t launch_quantize(const void* W, const float* awq, int N, int K, int sym,
                            uint32_t* qweight, void* scales, void* zeros, int* d_status,
                            cudaStream_t stream, int num_sms);

// s_X,j = max(mean_t |X[t][j]|, 1e-8) in fp64.  The sum of T bf16 magnitudes
// is exact in fp64 (8 significant bits each), so the order does not matter.
__global__ void awq_channel_mean_kernel(const uint16_t* __restrict__ X, int T, int K,
                                        double* __restrict__ sx) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= K) return;
  double acc = 0.0;
  for (int t = 0; t < T; ++t) acc += fabs((double)__uint_as_float((uint32_t)X[(size_t)t * K + j] << 16));
  const double m = acc / T;
  sx[j] = m < 1e-8 ? 1e-8 : m;
}

constexpr int kScaleThreads = 1024;

// s = s_X^alpha / geometric mean, rounded to fp32 (one CTA; the mean of the
// logarithms is summed in a fixed order).
__global__ void __launch_bounds__(kScaleThreads) awq_scale_kernel(const double* __restrict__ sx,
                                                                  int K, double alpha,
                                                                  double* __restrict__ m_tmp,
                                                                  float* __restrict__ s) {
  __shared__ double part[kScaleThreads];
  double acc = 0.0;
  for (int j = threadIdx.x; j < K; j += kScaleThreads) {
    const double m = pow(sx[j], alpha);
    m_tmp[j] = m;
    acc += log(m);
  }
  part[threadIdx.x] = acc;
  __syncthreads();
  for (int w = kScaleThreads / 2; w >= 1; w >>= 1) {
    if (threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
    __syncthreads();
  }
  const double geo = exp(part[0] / K);
  for (int j = threadIdx.x; j < K; j += kScaleThreads) s[j] = (float)(m_tmp[j] / geo);
}

// Delta[n][k] = W[n][k] - s16 (q - z16) / s_k in fp64 from the canonical codes.
__global__ void awq_delta_kernel(const uint16_t* __restrict__ W, const uint32_t* __restrict__ qw,
                                 const uint16_t* __restrict__ scales,
                                 const uint16_t* __restrict__ zeros, const float* __restrict__ s,
                                 int N, int K, int sym, double* __restrict__ delta) {
  const long long total = (long long)N * K;
  const int NG = K / kGroup;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int n = (int)(e / K), k = (int)(e % K);
    const uint32_t word = qw[(size_t)n * (K / 8) + k / 8];
    const int code = (int)((word >> (4 * (k & 7))) & 0xFu);
    const size_t gi = (size_t)n * NG + k / kGroup;
    const double sc = (double)__half2float(__ushort_as_half(scales[gi]));
    const double z = sym ? 8.0 : (double)__half2float(__ushort_as_half(zeros[gi]));
    const double what = sc * ((double)code - z);
    const double w = (double)__uint_as_float((uint32_t)W[e] << 16);
    delta[e] = w - what / (double)s[k];
  }
}

constexpr int kSumThreads = 256;
constexpr int kSumBlocks = 256;

// Partial sums of squares over a fixed split of the elements, then one CTA
// adds the partials in order: the same result on every run.
__global__ void __launch_bounds__(kSumThreads) sumsq_partial_kernel(const double* __restrict__ d,
                                                                    long long n,
                                                                    double* __restrict__ part) {
  __shared__ double sh[kSumThreads];
  double acc = 0.0;
  for (long long e = blockIdx.x * (long long)kSumThreads + threadIdx.x; e < n;
       e += (long long)kSumBlocks * kSumThreads)
    acc = fma(d[e], d[e], acc);
  sh[threadIdx.x] = acc;
  __syncthreads();
  for (int w = kSumThreads / 2; w >= 1; w >>= 1) {
    if (threadIdx.x < w) sh[threadIdx.x] += sh[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) part[blockIdx.x] = sh[0];
}

__global__ void __launch_bounds__(kSumBlocks) sum_partials_kernel(const double* __restrict__ part,
                                                                  double* __restrict__ out) {
  __shared__ double sh[kSumBlocks];
  sh[threadIdx.x] = part[threadIdx.x];
  __syncthreads();
  for (int w = kSumBlocks / 2; w >= 1; w >>= 1) {
    if (threadIdx.x < w) sh[threadIdx.x] += sh[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) *out = sh[0];
}

// The first index of the smallest loss; its scale to s_out.
__global__ void awq_pick_kernel(const double* __restrict__ losses, int n, const float* __restrict__ s_all,
                                int K, int* __restrict__ best, float* __restrict__ s_out) {
  __shared__ int bi;
  if (threadIdx.x == 0) {
    int b = 0;
    for (int i = 1; i < n; ++i)
      if (losses[i] < losses[b]) b = i;
    bi = b;
    *best = b;
  }
  __syncthreads();
  for (int j = threadIdx.x; j < K; j += blockDim.x) s_out[j] = s_all[(size_t)bi * K + j];
}

struct AwqWs {
  double *sx, *mtmp, *X64, *delta, *D, *part;
  float* s_all;
  uint32_t* qweight;
  uint16_t *scales, *zeros;
};

static size_t align256(size_t b) { return (b + 255) / 256 * 256; }

static size_t awq_layout(int T, int N, int K, int n_grid, AwqWs* w, uint8_t* base) {
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t* p = base ? base + off : nullptr;
    off += align256(bytes);
    return p;
  };
  uint8_t* p;
  p = take((size_t)K * 8);                   if (w) w->sx = reinterpret_cast<double*>(p);
  p = take((size_t)K * 8);                   if (w) w->mtmp = reinterpret_cast<double*>(p);
  p = take((size_t)T * K * 8);               if (w) w->X64 = reinterpret_cast<double*>(p);
  p = take((size_t)N * K * 8);               if (w) w->delta = reinterpret_cast<double*>(p);
  p = take((size_t)T * N * 8);               if (w) w->D = reinterpret_cast<double*>(p);
  p = take((size_t)kSumBlocks * 8);          if (w) w->part = reinterpret_cast<double*>(p);
  p = take((size_t)(n_grid + 1) * K * 4);    if (w) w->s_all = reinterpret_cast<float*>(p);
  p = take((size_t)N * K / 2);               if (w) w->qweight = reinterpret_cast<uint32_t*>(p);
  p = take((size_t)N * (K / kGroup) * 2);    if (w) w->scales = reinterpret_cast<uint16_t*>(p);
  p = take((size_t)N * (K / kGroup) * 2);    if (w) w->zeros = reinterpret_cast<uint16_t*>(p);
  return off;
}

size_t awq_workspace_bytes(int T, int N, int K, int n_grid) {
  return awq_layout(T, N, K, n_grid, nullptr, nullptr);
}

__global__ void awq_bf16_to_f64_kernel(const uint16_t* __restrict__ x, double* __restrict__ y,
                                       long long n) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x)
    y[i] = (double)__uint_as_float((uint32_t)x[i] << 16);
}

cudaError_t launch_awq_search(const void* W, const void* X, int T, int N, int K, int sym,
                              int n_grid, double* losses, float* s_out, int* best,
                              void* workspace, int num_sms, cudaStream_t stream) {
  AwqWs w;
  awq_layout(T, N, K, n_grid, &w, static_cast<uint8_t*>(workspace));
  const uint16_t* Wb = static_cast<const uint16_t*>(W);
  const uint16_t* Xb = static_cast<const uint16_t*>(X);
  cudaError_t e;
  awq_channel_mean_kernel<<<(K + 255) / 256, 256, 0, stream>>>(Xb, T, K, w.sx);
  awq_bf16_to_f64_kernel<<<1024, 256, 0, stream>>>(Xb, w.X64, (long long)T * K);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const long long nk = (long long)N * K;
  const unsigned dgrid = (unsigned)((nk + 255) / 256 < 8192 ? (nk + 255) / 256 : 8192);
  for (int i = 0; i <= n_grid; ++i) {
    const double alpha = (double)i / n_grid;
    float* s = w.s_all + (size_t)i * K;
    awq_scale_kernel<<<1, kScaleThreads, 0, stream>>>(w.sx, K, alpha, w.mtmp, s);
    if ((e = launch_quantize(W, s, N, K, sym, w.qweight, w.scales, sym ? nullptr : w.zeros,
                             nullptr, stream, num_sms)) != cudaSuccess)
      return e;
    awq_delta_kernel<<<dgrid, 256, 0, stream>>>(Wb, w.qweight, w.scales, sym ? nullptr : w.zeros,
                                                s, N, K, sym, w.delta);
    GemmF64 d{w.X64, K, 1, w.delta, 1, K, w.D, N, T, N, K, 1.0, 0.0, 0};
    if ((e = gemm_f64(d, stream)) != cudaSuccess) return e;
    sumsq_partial_kernel<<<kSumBlocks, kSumThreads, 0, stream>>>(w.D, (long long)T * N, w.part);
    sum_partials_kernel<<<1, kSumBlocks, 0, stream>>>(w.part, losses + i);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  awq_pick_kernel<<<1, 256, 0, stream>>>(losses, n_grid + 1, w.s_all, K, best, s_out);
  return cudaGetLastError();
}

}  // namespace wq
