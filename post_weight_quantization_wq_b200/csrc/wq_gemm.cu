// wq_gemm.cu -- W4A16 skinny GEMM (M = 16..64) on the tensor cores.
#include "wq_common.cuh"

namespace wq {

size_t gemm_workspace_bytes(int M, int N, int K) {
  const Geom g = make_geom(N, K, 1);
  if (g.NS <= 1) return 0;
  return (size_t)kCounterBytes + (size_t)g.NS * 64 * g.Npad * sizeof(float);
}

cudaError_t launch_gemm(const void*, const void*, int, int, int, int, float*, void*, int*, int,
                        unsigned long long, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace wq
