// Chunkwise-parallel PRISM scan on the 5th-generation tensor cores (tcgen05).
#include "common.cuh"

namespace prism {

bool chunk_tc_supported(int d_k, int d_v, int L, int W, int chunk, int dtype) {
  (void)d_k; (void)d_v; (void)L; (void)W; (void)chunk; (void)dtype;
  return false;
}

cudaError_t launch_chunk_tc(const ScanParams& p, cudaStream_t stream) {
  (void)p; (void)stream;
  return cudaErrorNotSupported;
}

}  // namespace prism
