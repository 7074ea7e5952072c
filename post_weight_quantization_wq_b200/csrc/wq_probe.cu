// wq_probe.cu -- a read-only streaming kernel that measures how fast this GPU
// can read HBM, as a ceiling for the weight-streaming linears (which read
// their weights once and write almost nothing).  The quantization pages have
// no counterpart: it is a measurement helper, not part of the method.
//
// Every thread reads 16-byte vectors in a grid-stride loop with a streaming
// (evict-first, no L1 allocation) load and XORs them into a register; one
// atomicXor per warp publishes the checksum so the loads cannot be dropped.
#include "wq_common.cuh"

namespace wq {
cudaError_t device_info(int** err, int* num_sms, unsigned long long* wait_ns);
}  // namespace wq

namespace {

__global__ void __launch_bounds__(512) stream_read_kernel(const uint4* __restrict__ src,
                                                           size_t n16, uint32_t* out) {
  uint32_t acc = 0;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  // four independent loads in flight per thread
  for (; i + 3 * stride < n16; i += 4 * stride) {
    const uint4 a = __ldcs(src + i), b = __ldcs(src + i + stride),
                c = __ldcs(src + i + 2 * stride), d = __ldcs(src + i + 3 * stride);
    acc ^= a.x ^ a.y ^ a.z ^ a.w ^ b.x ^ b.y ^ b.z ^ b.w ^ c.x ^ c.y ^ c.z ^ c.w ^ d.x ^ d.y ^
           d.z ^ d.w;
  }
  for (; i < n16; i += stride) {
    const uint4 a = __ldcs(src + i);
    acc ^= a.x ^ a.y ^ a.z ^ a.w;
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) acc ^= __shfl_xor_sync(0xFFFFFFFFu, acc, o);
  if ((threadIdx.x & 31) == 0) atomicXor(out, acc);
}

}  // namespace

extern "C" wq_status wq_stream_read_probe(const void* buf, size_t bytes, uint32_t* out,
                                          wq_stream_t stream) {
  if (!buf || !out || bytes == 0 || bytes % 16) return WQ_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(buf) % 16 || reinterpret_cast<uintptr_t>(out) % 4)
    return WQ_ERR_MISALIGNED;
  int* err = nullptr;
  int num_sms = 0;
  unsigned long long wait_ns = 0;
  if (wq::device_info(&err, &num_sms, &wait_ns) != cudaSuccess) return WQ_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(out, 0, sizeof(uint32_t), s) != cudaSuccess) return WQ_ERR_CUDA;
  const size_t n16 = bytes / 16;
  size_t blocks = (size_t)num_sms * 4;
  const size_t need = (n16 + 511) / 512;
  if (blocks > need) blocks = need;
  stream_read_kernel<<<(unsigned)blocks, 512, 0, s>>>(static_cast<const uint4*>(buf), n16, out);
  return cudaGetLastError() == cudaSuccess ? WQ_OK : WQ_ERR_CUDA;
}
