// wq_api.cu -- the extern "C" entry points declared in include/wq.h: argument
// validation, per-device launch state and the device error word.
#include <atomic>
#include <mutex>

#include "wq_common.cuh"

namespace wq {
cudaError_t launch_quantize(const void* W, const float* awq, int N, int K, int sym,
                            uint32_t* qweight, void* scales, void* zeros, int* d_status,
                            cudaStream_t stream, int num_sms);
cudaError_t launch_relayout(const uint32_t* qweight, const void* scales, const void* zeros,
                            int N, int K, int sym, void* packed, cudaStream_t stream);
size_t gemv_workspace_bytes(int M, int N, int K);
long long gemv_grid(long long tiles, int teams, int num_sms, int ctas_per_sm);
int gemv_teams(int M, bool awq);
long long gemv_tiles(int N, int K);
cudaError_t launch_gemv(const void* x, const float* inv_s, const void* packed, int M, int N,
                        int K, int sym, float* y, void* workspace, int* err, int num_sms,
                        unsigned long long wait_ns, cudaStream_t stream);
size_t gemm_workspace_bytes(int M, int N, int K);
void gemm_force_fold(int on);
void gemv_force_cuda_cores(int on);
bool gemv_tc_supported(int M, int K);
bool gemv_forced_cuda_cores();
size_t gptq_workspace_bytes(int T, int N, int K);
size_t awq_workspace_bytes(int T, int N, int K, int n_grid);
cudaError_t launch_nvfp4_quantize(const void* A, int R, int C, uint8_t* codes, uint8_t* scales,
                                  float* tensor_scale, int* d_status, int sf_atom, int num_sms,
                                  cudaStream_t stream);
cudaError_t launch_nvfp4_sf_relayout(const uint8_t* sf, int N, int K, uint8_t* out,
                                     cudaStream_t stream);
size_t nvfp4_linear_workspace_bytes(int M, int N, int K);
cudaError_t launch_nvfp4_linear(const void* x, const uint8_t* packed, const float* w_scale, int M,
                                int N, int K, float* y, void* workspace, int* err, int num_sms,
                                unsigned long long wait_ns, cudaStream_t stream);
cudaError_t launch_awq_search(const void* W, const void* X, int T, int N, int K, int sym,
                              int n_grid, double* losses, float* s_out, int* best,
                              void* workspace, int num_sms, cudaStream_t stream);
cudaError_t launch_gptq(const void* W, const void* X, int T, int N, int K, int sym, double damp,
                        uint32_t* qweight, void* scales, void* zeros, void* workspace,
                        int* d_status, cudaStream_t stream);
cudaError_t launch_gemm(const void* x, const void* packed, int M, int N, int K, int sym,
                        float* y, void* workspace, int* err, int num_sms,
                        unsigned long long wait_ns, cudaStream_t stream);
}  // namespace wq

namespace wq {

cudaError_t kernel_setup(const void* fn, size_t smem, int threads, int* ctas_per_sm) {
  // The dynamic shared-memory limit is an attribute of the kernel, so it is
  // only ever raised (to the largest size requested on this device so far).
  struct Entry {
    int dev;
    const void* fn;
    size_t smem;
    int per_sm;
  };
  struct Limit {
    int dev;
    const void* fn;
    size_t smem;
  };
  static std::mutex mu;
  static Entry cache[256];
  static Limit limits[128];
  static int used = 0, nlimits = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i)
    if (cache[i].dev == dev && cache[i].fn == fn && cache[i].smem == smem) {
      *ctas_per_sm = cache[i].per_sm;
      return cudaSuccess;
    }
  Limit* lim = nullptr;
  for (int i = 0; i < nlimits; ++i)
    if (limits[i].dev == dev && limits[i].fn == fn) lim = &limits[i];
  if (!lim || lim->smem < smem) {
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (!lim && nlimits < 128) lim = &limits[nlimits++], lim->dev = dev, lim->fn = fn;
    if (lim) lim->smem = smem;
  }
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, threads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  if (used < 256) cache[used++] = Entry{dev, fn, smem, per_sm};
  *ctas_per_sm = per_sm;
  return cudaSuccess;
}

}  // namespace wq

// One error word per GPU that loads the library: kernels OR bits into it when
// a bounded wait gives up; wq_last_device_status reads and clears it.
__device__ int g_wq_device_error;

namespace {

constexpr int kMaxDevices = 64;
constexpr unsigned long long kDefaultWaitNs = 2000000000ull;   // 2 s

struct DeviceState {
  std::once_flag once;
  int* err = nullptr;
  int num_sms = 0;
  cudaError_t init_error = cudaSuccess;
};
DeviceState g_devices[kMaxDevices];
std::atomic<unsigned long long> g_wait_ns{kDefaultWaitNs};

// Per-device set-up, done once with that device current: the address of the
// error word and the SM count.
DeviceState* device_state(cudaError_t* e) {
  int dev = 0;
  *e = cudaGetDevice(&dev);
  if (*e != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxDevices) {
    *e = cudaErrorInvalidDevice;
    return nullptr;
  }
  DeviceState* d = &g_devices[dev];
  std::call_once(d->once, [d, dev]() {
    cudaError_t err = cudaGetSymbolAddress(reinterpret_cast<void**>(&d->err), g_wq_device_error);
    if (err == cudaSuccess)
      err = cudaDeviceGetAttribute(&d->num_sms, cudaDevAttrMultiProcessorCount, dev);
    d->init_error = err;
  });
  *e = d->init_error;
  return *e == cudaSuccess ? d : nullptr;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

wq_status check_dims(int N, int K, int group_size) {
  if (N <= 0 || K <= 0) return WQ_ERR_INVALID_ARG;
  if (group_size != WQ_GROUP_SIZE) return WQ_ERR_UNSUPPORTED_SHAPE;
  if (K % WQ_GROUP_SIZE != 0) return WQ_ERR_UNSUPPORTED_SHAPE;
  if (N > WQ_MAX_DIM || K > WQ_MAX_DIM) return WQ_ERR_UNSUPPORTED_SHAPE;
  return WQ_OK;
}

wq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? WQ_OK : WQ_ERR_CUDA; }

wq_status check_linear(const void* x, const float* inv_s, const void* packed, int M, int Mlo,
                       int Mhi, int N, int K, int group_size, int symmetric, int layout, float* y,
                       void* workspace, size_t ws_bytes, bool gemm) {
  wq_status st = check_dims(N, K, group_size);
  if (st != WQ_OK) return st;
  if (M < Mlo || M > Mhi) return WQ_ERR_UNSUPPORTED_SHAPE;
  if (symmetric != 0 && symmetric != 1) return WQ_ERR_INVALID_ARG;
  if (layout != WQ_LAYOUT_TILED) return WQ_ERR_INVALID_ARG;
  if (!x || !packed || !y) return WQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(packed) || !aligned16(y) || (inv_s && !aligned16(inv_s)))
    return WQ_ERR_MISALIGNED;
  const size_t need = gemm ? wq::gemm_workspace_bytes(M, N, K) : wq::gemv_workspace_bytes(M, N, K);
  if (need > 0) {
    if (!workspace || ws_bytes < need) return WQ_ERR_WORKSPACE_TOO_SMALL;
    if (!aligned16(workspace)) return WQ_ERR_MISALIGNED;
  }
  return WQ_OK;
}

}  // namespace

namespace wq {
cudaError_t launch_pdl(const void* fn, dim3 grid, dim3 block, void** args, size_t smem,
                       cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelExC(&cfg, fn, args);
}

// Error-word address, SM count and wait limit of the current device (set up
// on first use), for entry points defined in other files of the library.
cudaError_t device_info(int** err, int* num_sms, unsigned long long* wait_ns) {
  cudaError_t e;
  DeviceState* d = device_state(&e);
  if (!d) return e;
  *err = d->err;
  *num_sms = d->num_sms;
  *wait_ns = g_wait_ns.load();
  return cudaSuccess;
}
}  // namespace wq

extern "C" {

const char* wq_status_string(int status) {
  switch (status) {
    case WQ_OK: return "WQ_OK";
    case WQ_ERR_INVALID_ARG: return "WQ_ERR_INVALID_ARG";
    case WQ_ERR_UNSUPPORTED_SHAPE: return "WQ_ERR_UNSUPPORTED_SHAPE";
    case WQ_ERR_MISALIGNED: return "WQ_ERR_MISALIGNED";
    case WQ_ERR_WORKSPACE_TOO_SMALL: return "WQ_ERR_WORKSPACE_TOO_SMALL";
    case WQ_ERR_NONFINITE: return "WQ_ERR_NONFINITE";
    case WQ_ERR_TIMEOUT: return "WQ_ERR_TIMEOUT";
    case WQ_ERR_CUDA: return "WQ_ERR_CUDA";
    default: return "WQ_ERR_UNKNOWN";
  }
}

int wq_abi_version(void) { return WQ_ABI_VERSION; }

wq_status wq_quantize_rtn(const void* W, const float* awq_scale, int N, int K, int group_size,
                          int symmetric, uint32_t* qweight, void* scales, void* zeros,
                          int* d_status, wq_stream_t stream) {
  wq_status st = check_dims(N, K, group_size);
  if (st != WQ_OK) return st;
  if (symmetric != 0 && symmetric != 1) return WQ_ERR_INVALID_ARG;
  if (!W || !qweight || !scales) return WQ_ERR_INVALID_ARG;
  if (symmetric ? (zeros != nullptr) : (zeros == nullptr)) return WQ_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(qweight) || !aligned16(scales) ||
      (zeros && !aligned16(zeros)) || (awq_scale && !aligned16(awq_scale)))
    return WQ_ERR_MISALIGNED;
  if (d_status && (reinterpret_cast<uintptr_t>(d_status) & 3u)) return WQ_ERR_MISALIGNED;
  cudaError_t e;
  DeviceState* d = device_state(&e);
  if (!d) return WQ_ERR_CUDA;
  return from_cuda(wq::launch_quantize(W, awq_scale, N, K, symmetric, qweight, scales, zeros,
                                       d_status, reinterpret_cast<cudaStream_t>(stream),
                                       d->num_sms));
}

size_t wq_packed_bytes(int N, int K, int group_size, int symmetric, int layout) {
  if (check_dims(N, K, group_size) != WQ_OK) return 0;
  if (layout != WQ_LAYOUT_TILED || (symmetric != 0 && symmetric != 1)) return 0;
  return (size_t)wq::make_geom(N, K, symmetric).total;
}

wq_status wq_pack_layout(const uint32_t* qweight, const void* scales, const void* zeros, int N,
                         int K, int group_size, int symmetric, int layout, void* packed,
                         size_t packed_bytes, wq_stream_t stream) {
  wq_status st = check_dims(N, K, group_size);
  if (st != WQ_OK) return st;
  if (symmetric != 0 && symmetric != 1) return WQ_ERR_INVALID_ARG;
  if (layout != WQ_LAYOUT_TILED) return WQ_ERR_INVALID_ARG;
  if (!qweight || !scales || !packed) return WQ_ERR_INVALID_ARG;
  if (symmetric ? (zeros != nullptr) : (zeros == nullptr)) return WQ_ERR_INVALID_ARG;
  if (!aligned16(qweight) || !aligned16(scales) || !aligned16(packed) ||
      (zeros && !aligned16(zeros)))
    return WQ_ERR_MISALIGNED;
  if (packed_bytes < wq_packed_bytes(N, K, group_size, symmetric, layout))
    return WQ_ERR_INVALID_ARG;
  cudaError_t e;
  if (!device_state(&e)) return WQ_ERR_CUDA;
  return from_cuda(wq::launch_relayout(qweight, scales, zeros, N, K, symmetric, packed,
                                       reinterpret_cast<cudaStream_t>(stream)));
}

size_t wq_workspace_bytes(int M, int N, int K) {
  if (N <= 0 || K <= 0 || K % WQ_GROUP_SIZE || N > WQ_MAX_DIM || K > WQ_MAX_DIM) return 0;
  if (M >= 1 && M <= 8) return wq::gemv_workspace_bytes(M, N, K);
  if (M >= 9 && M <= WQ_GEMM_MAX_M) return wq::gemm_workspace_bytes(M, N, K);
  return 0;
}

size_t wq_gemm_workspace_bytes(int M, int N, int K) {
  if (N <= 0 || K <= 0 || K % WQ_GROUP_SIZE || N > WQ_MAX_DIM || K > WQ_MAX_DIM) return 0;
  if (M < 1 || M > WQ_GEMM_MAX_M) return 0;
  return wq::gemm_workspace_bytes(M, N, K);
}

wq_status wq_gemv_w4a16(const void* x, const float* inv_act_scale, const void* packed, int M,
                        int N, int K, int group_size, int symmetric, int layout, float* y,
                        void* workspace, size_t ws_bytes, wq_stream_t stream) {
  wq_status st = check_linear(x, inv_act_scale, packed, M, 1, 8, N, K, group_size, symmetric,
                              layout, y, workspace, ws_bytes, false);
  if (st != WQ_OK) return st;
  cudaError_t e;
  DeviceState* d = device_state(&e);
  if (!d) return WQ_ERR_CUDA;
  return from_cuda(wq::launch_gemv(x, inv_act_scale, packed, M, N, K, symmetric, y, workspace,
                                   d->err, d->num_sms, g_wait_ns.load(),
                                   reinterpret_cast<cudaStream_t>(stream)));
}

wq_status wq_gemm_w4a16(const void* x, const float* inv_act_scale, const void* packed, int M,
                        int N, int K, int group_size, int symmetric, int layout, float* y,
                        void* workspace, size_t ws_bytes, wq_stream_t stream) {
  wq_status st = check_linear(x, inv_act_scale, packed, M, 1, WQ_GEMM_MAX_M, N, K, group_size,
                              symmetric, layout, y, workspace, ws_bytes, true);
  if (st != WQ_OK) return st;
  if (inv_act_scale) return WQ_ERR_INVALID_ARG;
  cudaError_t e;
  DeviceState* d = device_state(&e);
  if (!d) return WQ_ERR_CUDA;
  return from_cuda(wq::launch_gemm(x, packed, M, N, K, symmetric, y, workspace, d->err,
                                   d->num_sms, g_wait_ns.load(),
                                   reinterpret_cast<cudaStream_t>(stream)));
}

size_t wq_gptq_workspace_bytes(int T, int N, int K) {
  if (check_dims(N, K, WQ_GROUP_SIZE) != WQ_OK || K > WQ_GPTQ_MAX_K || T < 1 ||
      T > WQ_GPTQ_MAX_T)
    return 0;
  return wq::gptq_workspace_bytes(T, N, K);
}

wq_status wq_gptq_quantize(const void* W, const void* X, int T, int N, int K, int group_size,
                           int symmetric, double damp, uint32_t* qweight, void* scales,
                           void* zeros, void* workspace, size_t ws_bytes, int* d_status,
                           wq_stream_t stream) {
  wq_status st = check_dims(N, K, group_size);
  if (st != WQ_OK) return st;
  if (K > WQ_GPTQ_MAX_K || T < 1 || T > WQ_GPTQ_MAX_T) return WQ_ERR_UNSUPPORTED_SHAPE;
  if (symmetric != 0 && symmetric != 1) return WQ_ERR_INVALID_ARG;
  if (!(damp >= 0.0) || damp > 1e6) return WQ_ERR_INVALID_ARG;
  if (!W || !X || !qweight || !scales) return WQ_ERR_INVALID_ARG;
  if (symmetric ? (zeros != nullptr) : (zeros == nullptr)) return WQ_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(X) || !aligned16(qweight) || !aligned16(scales) ||
      (zeros && !aligned16(zeros)))
    return WQ_ERR_MISALIGNED;
  if (d_status && (reinterpret_cast<uintptr_t>(d_status) & 3u)) return WQ_ERR_MISALIGNED;
  const size_t need = wq::gptq_workspace_bytes(T, N, K);
  if (!workspace || ws_bytes < need) return WQ_ERR_WORKSPACE_TOO_SMALL;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return WQ_ERR_MISALIGNED;
  cudaError_t e;
  if (!device_state(&e)) return WQ_ERR_CUDA;
  return from_cuda(wq::launch_gptq(W, X, T, N, K, symmetric, damp, qweight, scales, zeros,
                                   workspace, d_status, reinterpret_cast<cudaStream_t>(stream)));
}

size_t wq_awq_search_workspace_bytes(int T, int N, int K, int n_grid) {
  if (check_dims(N, K, WQ_GROUP_SIZE) != WQ_OK || T < 1 || T > WQ_AWQ_MAX_T || n_grid < 1 ||
      n_grid > WQ_AWQ_MAX_GRID)
    return 0;
  return wq::awq_workspace_bytes(T, N, K, n_grid);
}

wq_status wq_awq_search(const void* W, const void* X, int T, int N, int K, int group_size,
                        int symmetric, int n_grid, double* losses, float* scale_out, int* best,
                        void* workspace, size_t ws_bytes, wq_stream_t stream) {
  wq_status st = check_dims(N, K, group_size);
  if (st != WQ_OK) return st;
  if (T < 1 || T > WQ_AWQ_MAX_T) return WQ_ERR_UNSUPPORTED_SHAPE;
  if (n_grid < 1 || n_grid > WQ_AWQ_MAX_GRID) return WQ_ERR_INVALID_ARG;
  if (symmetric != 0 && symmetric != 1) return WQ_ERR_INVALID_ARG;
  if (!W || !X || !losses || !scale_out || !best) return WQ_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(X) || !aligned16(losses) || !aligned16(scale_out) ||
      (reinterpret_cast<uintptr_t>(best) & 3u))
    return WQ_ERR_MISALIGNED;
  const size_t need = wq::awq_workspace_bytes(T, N, K, n_grid);
  if (!workspace || ws_bytes < need) return WQ_ERR_WORKSPACE_TOO_SMALL;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return WQ_ERR_MISALIGNED;
  cudaError_t e;
  DeviceState* d = device_state(&e);
  if (!d) return WQ_ERR_CUDA;
  return from_cuda(wq::launch_awq_search(W, X, T, N, K, symmetric, n_grid, losses, scale_out,
                                         best, workspace, d->num_sms,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

wq_status wq_nvfp4_quantize(const void* A, int R, int C, uint8_t* codes, uint8_t* block_scales,
                            float* tensor_scale, int* d_status, wq_stream_t stream) {
  wq_status st = check_dims(R, C, WQ_GROUP_SIZE);
  if (st != WQ_OK) return st;
  if (!A || !codes || !block_scales || !tensor_scale) return WQ_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(codes) || !aligned16(block_scales) ||
      (reinterpret_cast<uintptr_t>(tensor_scale) & 3u) ||
      (d_status && (reinterpret_cast<uintptr_t>(d_status) & 3u)))
    return WQ_ERR_MISALIGNED;
  cudaError_t e;
  DeviceState* d = device_state(&e);
  if (!d) return WQ_ERR_CUDA;
  return from_cuda(wq::launch_nvfp4_quantize(A, R, C, codes, block_scales, tensor_scale, d_status,
                                             0, d->num_sms,
                                             reinterpret_cast<cudaStream_t>(stream)));
}

size_t wq_nvfp4_packed_bytes(int N, int K) {
  if (check_dims(N, K, WQ_GROUP_SIZE) != WQ_OK) return 0;
  return (size_t)N * K / 2 + (size_t)((N + 127) / 128) * (K / 64) * 512;
}

wq_status wq_nvfp4_pack_layout(const uint8_t* codes, const uint8_t* block_scales, int N, int K,
                               void* packed, size_t packed_bytes, wq_stream_t stream) {
  wq_status st = check_dims(N, K, WQ_GROUP_SIZE);
  if (st != WQ_OK) return st;
  if (!codes || !block_scales || !packed) return WQ_ERR_INVALID_ARG;
  if (!aligned16(codes) || !aligned16(block_scales) || !aligned16(packed))
    return WQ_ERR_MISALIGNED;
  if (packed_bytes < wq_nvfp4_packed_bytes(N, K)) return WQ_ERR_INVALID_ARG;
  cudaError_t e;
  if (!device_state(&e)) return WQ_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  e = cudaMemcpyAsync(packed, codes, (size_t)N * K / 2, cudaMemcpyDeviceToDevice, s);
  if (e != cudaSuccess) return WQ_ERR_CUDA;
  return from_cuda(wq::launch_nvfp4_sf_relayout(
      block_scales, N, K, static_cast<uint8_t*>(packed) + (size_t)N * K / 2, s));
}

size_t wq_nvfp4_linear_workspace_bytes(int M, int N, int K) {
  if (check_dims(N, K, WQ_GROUP_SIZE) != WQ_OK || M < 1 || M > WQ_NVFP4_MAX_M) return 0;
  return wq::nvfp4_linear_workspace_bytes(M, N, K);
}

wq_status wq_nvfp4_linear(const void* x, const void* packed, const float* w_tensor_scale, int M,
                          int N, int K, float* y, void* workspace, size_t ws_bytes,
                          wq_stream_t stream) {
  wq_status st = check_dims(N, K, WQ_GROUP_SIZE);
  if (st != WQ_OK) return st;
  if (M < 1 || M > WQ_NVFP4_MAX_M) return WQ_ERR_UNSUPPORTED_SHAPE;
  if (!x || !packed || !w_tensor_scale || !y) return WQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(packed) || !aligned16(y) ||
      (reinterpret_cast<uintptr_t>(w_tensor_scale) & 3u))
    return WQ_ERR_MISALIGNED;
  const size_t need = wq::nvfp4_linear_workspace_bytes(M, N, K);
  if (!workspace || ws_bytes < need) return WQ_ERR_WORKSPACE_TOO_SMALL;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return WQ_ERR_MISALIGNED;
  cudaError_t e;
  DeviceState* d = device_state(&e);
  if (!d) return WQ_ERR_CUDA;
  return from_cuda(wq::launch_nvfp4_linear(x, static_cast<const uint8_t*>(packed), w_tensor_scale,
                                           M, N, K, y, workspace, d->err, d->num_sms,
                                           g_wait_ns.load(),
                                           reinterpret_cast<cudaStream_t>(stream)));
}

wq_status wq_last_device_status(wq_stream_t stream) {
  cudaError_t e;
  DeviceState* d = device_state(&e);
  if (!d) return WQ_ERR_CUDA;
  e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return WQ_ERR_CUDA;
  int word = 0;
  e = cudaMemcpy(&word, d->err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return WQ_ERR_CUDA;
  if (word) {
    const int zero = 0;
    e = cudaMemcpy(d->err, &zero, sizeof(int), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return WQ_ERR_CUDA;
    if (word & wq::kDevErrTimeout) return WQ_ERR_TIMEOUT;
  }
  return WQ_OK;
}

// Test hook: the time a kernel's bounded wait gives before it records a
// timeout (default 2 s).  Lowering it to 0 makes waits that are not already
// satisfied give up at once, which exercises the timeout path without
// stalling the GPU.  Not part of the stable ABI.
void wq_debug_set_wait_limit_ns(unsigned long long ns) { g_wait_ns.store(ns ? ns : 1ull); }

// Test hook: 1 makes wq_gemm_w4a16 use its many-row kernel for every M (for
// comparisons at the skinny sizes); 0 restores the choice by M.  Not part of
// the stable ABI.
void wq_debug_gemm_force_fold(int on) { wq::gemm_force_fold(on ? 1 : 0); }

void wq_debug_gemv_force_cuda_cores(int on) { wq::gemv_force_cuda_cores(on ? 1 : 0); }

// Test hook: how wq_gemv_w4a16 splits its tiles for a given SM count and
// occupancy (host arithmetic only, no device call).  Not part of the stable ABI.
wq_status wq_debug_gemv_split(int M, int N, int K, int awq, int num_sms, int ctas_per_sm,
                              long long* tiles, int* teams, long long* grid) {
  if (M < 1 || M > 8 || N < 1 || K < wq::kGroup || K % wq::kGroup != 0 || num_sms < 1 ||
      ctas_per_sm < 1 || !tiles || !teams || !grid)
    return WQ_ERR_INVALID_ARG;
  *tiles = wq::gemv_tiles(N, K);
  if (!wq::gemv_forced_cuda_cores() && wq::gemv_tc_supported(M, K)) {
    // tensor-core decode kernel: one CTA per SM, one team each
    *teams = 1;
    *grid = *tiles < num_sms ? *tiles : num_sms;
    return WQ_OK;
  }
  *teams = wq::gemv_teams(M, awq != 0);
  *grid = wq::gemv_grid(*tiles, *teams, num_sms, ctas_per_sm);
  return WQ_OK;
}

}  // extern "C"
