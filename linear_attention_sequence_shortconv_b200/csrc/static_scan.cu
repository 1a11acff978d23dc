// prism_scan_fwd_static: the scan for callers that cannot allocate device memory.  The
// PRISM write-ups have no counterpart of this entry point; it is a service of this library.
//
// Its scratch is a file-scope device array in this translation unit, which the CUDA
// runtime registers as a module of its own.  With lazy module loading (the default of
// CUDA 12 and of PyTorch), the array is therefore reserved only on a device where this
// entry point has run, not on every device that runs one of the library's other calls.
#include <mutex>

#include "common.cuh"

namespace prism {
int device_setup(int** status_out);
int check_sizes(int B, int T, int H, int d_k, int d_v, int L, int W, int chunk, int dtype);
}  // namespace prism

namespace {

constexpr int kMaxDevices = 64;
constexpr size_t kStaticWorkspaceBytes = (size_t)PRISM_STATIC_WORKSPACE_BYTES;

// The scratch.  In host code this name is only a host-side handle of the symbol, never
// a device address: kernels get the address looked up below.
static __device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];

std::mutex g_static_mutex;
void* g_static_ws_ptr[kMaxDevices] = {};

// Device address of g_static_workspace on the current device, looked up once per device
// (with that device current) and cached.
int static_workspace(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PRISM_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return PRISM_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_static_mutex);
  if (!g_static_ws_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_workspace) != cudaSuccess || !ptr) return PRISM_ERR_CUDA;
    g_static_ws_ptr[dev] = ptr;
  }
  *out = g_static_ws_ptr[dev];
  return PRISM_OK;
}

}  // namespace

extern "C" int prism_scan_fwd_static(const void* q, const void* k, const void* v, const float* gamma,
                                     const float* beta, const void* u, const float* alpha, const void* gain,
                                     const float* conv_w, const float* S0, const int32_t* lengths, int B, int T,
                                     int H, int d_k, int d_v, int L, int W, int chunk, int dtype, void* o,
                                     float* S_final, prism_stream_t stream, int chain, const void* conv_state) {
  if (chain != PRISM_CHAIN_LINEAR && chain != PRISM_CHAIN_GELU) return PRISM_ERR_INVALID_ARG;
  int rc = prism::check_sizes(B, T, H, d_k, d_v, L, W, chunk, dtype);
  if (rc != PRISM_OK) return rc;
  const size_t need = prism_scan_fwd_workspace_size(B, T, H, d_k, d_v, L, W, chunk, dtype);
  if (need > kStaticWorkspaceBytes) return PRISM_ERR_WORKSPACE;
  void* ws = nullptr;
  if (need > 0) {
    int* status = nullptr;
    rc = prism::device_setup(&status);  // architecture check before this module's symbol is touched
    if (rc != PRISM_OK) return rc;
    rc = static_workspace(&ws);
    if (rc != PRISM_OK) return rc;
  }
  return prism_scan_fwd_ex(q, k, v, gamma, beta, u, alpha, gain, conv_w, S0, lengths, B, T, H, d_k, d_v, L, W,
                           chunk, dtype, o, S_final, ws, need > 0 ? kStaticWorkspaceBytes : 0, stream, chain,
                           conv_state);
}
