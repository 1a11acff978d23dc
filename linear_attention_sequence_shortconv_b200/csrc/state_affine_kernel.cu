// Composition step of per-segment state maps: out = S M + N for every (batch, head).
//
// The PRISM state update (ICML 2026 PRISM write-up, 核心迭代形式 / 架构形式)
//
//   S_t = S_{t-1} gamma_t (I - beta_t k_t k_t^T) + beta_t v_t k_t^T + sum_l alpha_l r_l u_l^T
//
// is affine in the state, and so is any run of it over a segment of tokens:
// S_end = S_start M + N, with M (d_k x d_k) the ordered product of the transitions
// and N (d_v x d_k) the segment's end state from a zero start.  Sequence sharding
// folds the maps of earlier segments into a segment's start state with this step.
// The work is tiny (d_v d_k^2 per head), so it is a plain CUDA-core kernel: one block
// per state row, the row staged in shared memory, columns over threads, a fixed
// summation order (deterministic).
#include "common.cuh"

namespace prism {
namespace {

constexpr int kAffThreads = 128;

__global__ void __launch_bounds__(kAffThreads)
    state_affine_kernel(const float* S, const float* M, const float* N, float* out, int d_v, int d_k) {
  __shared__ float srow[PRISM_MAX_HEAD_DIM];
  const int i = blockIdx.x;
  const size_t bh = blockIdx.y;
  const size_t row = (bh * d_v + i) * d_k;
  for (int c = threadIdx.x; c < d_k; c += kAffThreads) srow[c] = S[row + c];
  __syncthreads();  // the row is read before any of it is written (out may alias S)
  const float* m = M + bh * (size_t)d_k * d_k;
  for (int j = threadIdx.x; j < d_k; j += kAffThreads) {
    float acc = N ? N[row + j] : 0.f;
    for (int c = 0; c < d_k; ++c) acc += srow[c] * m[(size_t)c * d_k + j];
    out[row + j] = acc;
  }
}

}  // namespace

cudaError_t launch_state_affine(const float* S, const float* M, const float* N, float* out, int BH, int d_v, int d_k,
                                cudaStream_t stream) {
  state_affine_kernel<<<dim3(d_v, BH), kAffThreads, 0, stream>>>(S, M, N, out, d_v, d_k);
  return cudaGetLastError();
}

}  // namespace prism
