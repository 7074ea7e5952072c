// wq_gemv_static.cu -- wq_gemv_w4a16 for callers that cannot allocate device
// memory.
//
// wq_gemv_w4a16 needs a caller-provided workspace for its split-K partial sums
// and completion counters.  Some callers have no way to provide one: code that
// runs where cudaMalloc is off limits (inside a framework's custom-op hook
// that forbids allocation, a stream-captured region whose memory pool is
// fixed, or a plugin whose host application owns every device allocation).
// This entry point runs the same GEMV kernel with its scratch in a
// fixed-size array that lives in this library's device image, so it needs no
// allocation at all.  The array is kWqStaticScratchBytes long (8 MiB; every
// GPU that loads the library keeps it until the process exits), which covers
// any shape whose wq_workspace_bytes(M, N, K) fits in it; larger requests are
// refused with WQ_ERR_WORKSPACE_TOO_SMALL.
#include <mutex>

#include "wq_common.cuh"

namespace wq {
cudaError_t device_info(int** err, int* num_sms, unsigned long long* wait_ns);
size_t gemv_workspace_bytes(int M, int N, int K);
cudaError_t launch_gemv(const void* x, const float* inv_s, const void* packed, int M, int N,
                        int K, int sym, float* y, void* workspace, int* err, int num_sms,
                        unsigned long long wait_ns, cudaStream_t stream);
}  // namespace wq

namespace {

constexpr size_t kWqStaticScratchBytes = WQ_STATIC_SCRATCH_BYTES;

// The scratch itself: counters first (they must read zero when a call starts),
// then the partial sums.  Shared by every call on the device.
static __device__ __align__(256) unsigned char g_wq_static_scratch[kWqStaticScratchBytes];

constexpr int kMaxDev = 64;
struct StaticScratch {
  std::once_flag once;
  void* ptr = nullptr;              // device address of g_wq_static_scratch
  cudaError_t err = cudaSuccess;
};
StaticScratch g_static[kMaxDev];

// Once per device, with that device current: the device address of the array.
// In host code the array's name is only a host-side stand-in, so the address
// must come from cudaGetSymbolAddress.
void* static_scratch(cudaError_t* e) {
  int dev = 0;
  *e = cudaGetDevice(&dev);
  if (*e != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxDev) {
    *e = cudaErrorInvalidDevice;
    return nullptr;
  }
  StaticScratch* s = &g_static[dev];
  std::call_once(s->once, [s]() {
    s->err = cudaGetSymbolAddress(&s->ptr, g_wq_static_scratch);
    if (s->err != cudaSuccess) s->ptr = nullptr;
  });
  *e = s->err;
  return s->ptr;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" wq_status wq_gemv_w4a16_static(const void* x, const float* inv_act_scale,
                                           const void* packed, int M, int N, int K,
                                           int group_size, int symmetric, int layout, float* y,
                                           wq_stream_t stream) {
  if (N <= 0 || K <= 0) return WQ_ERR_INVALID_ARG;
  if (group_size != WQ_GROUP_SIZE || K % WQ_GROUP_SIZE != 0) return WQ_ERR_UNSUPPORTED_SHAPE;
  if (N > WQ_MAX_DIM || K > WQ_MAX_DIM || M < 1 || M > 8) return WQ_ERR_UNSUPPORTED_SHAPE;
  if (symmetric != 0 && symmetric != 1) return WQ_ERR_INVALID_ARG;
  if (layout != WQ_LAYOUT_TILED) return WQ_ERR_INVALID_ARG;
  if (!x || !packed || !y) return WQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(packed) || !aligned16(y) ||
      (inv_act_scale && !aligned16(inv_act_scale)))
    return WQ_ERR_MISALIGNED;
  const size_t need = wq::gemv_workspace_bytes(M, N, K);
  if (need > kWqStaticScratchBytes) return WQ_ERR_WORKSPACE_TOO_SMALL;

  cudaError_t e;
  void* scratch = static_scratch(&e);
  if (!scratch) return WQ_ERR_CUDA;
  int* err = nullptr;
  int num_sms = 0;
  unsigned long long wait_ns = 0;
  e = wq::device_info(&err, &num_sms, &wait_ns);
  if (e != cudaSuccess) return WQ_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (need > 0) {
    // The completion counters this shape uses must start at zero; a call that
    // was cut short could have left some set, so clear them on the stream.
    const wq::Geom g = wq::make_geom(N, K, symmetric);
    const size_t counter_bytes = (size_t)g.NB * (wq::kTileRows / wq::kRowsPerCounter) * 4;
    e = cudaMemsetAsync(scratch, 0, counter_bytes, st);
    if (e != cudaSuccess) return WQ_ERR_CUDA;
  }
  e = wq::launch_gemv(x, inv_act_scale, packed, M, N, K, symmetric, y,
                      need > 0 ? scratch : nullptr, err, num_sms, wait_ns, st);
  return e == cudaSuccess ? WQ_OK : WQ_ERR_CUDA;
}
