// C ABI of the PRISM scan: argument checks, launch planning, status word.
// Declarations and documentation: include/prism.h.
#include <atomic>
#include <mutex>

#include "common.cuh"

namespace prism {
cudaError_t launch_recurrent_scan(const ScanParams& p, int dtype, cudaStream_t stream);
cudaError_t launch_prologue(const void* v, const float* alpha, const void* gain, const float* conv_w,
                            const int32_t* lengths, int B, int T, int H, int d_v, int L, int W,
                            int dtype, float* rho, cudaStream_t stream, int chain);
bool chunk_scan_supported(int d_k, int d_v, int L, int W, int chunk, int dtype);
cudaError_t launch_chunk_scan(const ScanParams& p, cudaStream_t stream);
size_t chunk_scan_workspace_bytes(int B, int T, int H, int D, int L);
int chunk_scan_launches(int B, int T, int H, int L);
int chunk_scan_split_chunks(int B, int T, int H, int L);
bool chunk_fp32_supported(int d_k, int d_v, int chunk, int dtype);
cudaError_t launch_chunk_fp32(const ScanParams& p, cudaStream_t stream);
cudaError_t launch_decode_step(const DecodeParams& p, int dtype, cudaStream_t stream);
cudaError_t launch_scan_bwd(const BwdParams& p, int dtype, cudaStream_t stream);
size_t bwd_smem_bytes(int d_k, int d_v, int L);
int bwd_row_blocks(int d_k, int d_v);
bool chunk_bwd_supported(int d_k, int d_v, int L);
size_t chunk_bwd_smem_bytes(int d);
cudaError_t launch_chunk_bwd(const ChunkBwdParams& p, int dtype, cudaStream_t stream);
cudaError_t launch_state_affine(const float* S, const float* M, const float* N, float* out, int BH, int d_v, int d_k,
                                cudaStream_t stream);
}  // namespace prism

namespace {

// One status word per device: kernels record PRISM_ERR_TIMEOUT here when a
// bounded wait gives up; prism_stream_status reads and clears it.
__device__ int g_status_word;

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
int* g_status_ptr[kMaxDevices] = {};
int g_arch_ok[kMaxDevices] = {};  // 0 unknown, 1 sm_100, -1 other
constexpr long long kDefaultSpinLimit = 1ll << 18;  // polls; each may suspend up to 20 us
std::atomic<long long> g_spin_limit{kDefaultSpinLimit};
std::atomic<void*> g_split_event{nullptr};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool ranges_overlap(const void* a, size_t a_bytes, const void* b, size_t b_bytes) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + b_bytes && y < x + a_bytes;
}
bool head_dim_ok(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }

}  // namespace

namespace prism {
// Device-side status word address and architecture check for the current device.
int device_setup(int** status_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PRISM_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return PRISM_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_arch_ok[dev] == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return PRISM_ERR_CUDA;
    g_arch_ok[dev] = (major == 10 && minor == 0) ? 1 : -1;
  }
  if (g_arch_ok[dev] != 1) return PRISM_ERR_UNSUPPORTED;
  if (!g_status_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_status_word) != cudaSuccess) return PRISM_ERR_CUDA;
    g_status_ptr[dev] = static_cast<int*>(ptr);
  }
  *status_out = g_status_ptr[dev];
  return PRISM_OK;
}

int check_sizes(int B, int T, int H, int d_k, int d_v, int L, int W, int chunk, int dtype) {
  if (B < 1 || T < 1 || H < 1 || d_k < 1 || d_v < 1 || L < 1 || W < 1 || chunk < 1)
    return PRISM_ERR_INVALID_ARG;
  if (dtype != PRISM_BF16 && dtype != PRISM_FP32) return PRISM_ERR_INVALID_ARG;
  if (!head_dim_ok(d_k) || !head_dim_ok(d_v)) return PRISM_ERR_UNSUPPORTED;
  if (L > PRISM_MAX_L || W > PRISM_MAX_W) return PRISM_ERR_UNSUPPORTED;
  if (chunk != 16 && chunk != 32 && chunk != 64) return PRISM_ERR_UNSUPPORTED;
  // element counts must fit the 64-bit index arithmetic with a wide margin
  const double elems = (double)B * T * H * (double)(L > 1 ? L - 1 : 1) * (d_k > d_v ? d_k : d_v);
  if (elems > 9.0e15) return PRISM_ERR_UNSUPPORTED;
  return PRISM_OK;
}
}  // namespace prism

namespace {
using prism::check_sizes;
using prism::device_setup;

// one thread: the device-side index check on (i, n), nothing accessed
__global__ void bounds_probe_kernel(long long i, long long n, int* status) { prism::in_bounds(i, n, status); }

}  // namespace

extern "C" {

int prism_debug_bounds(void) { return prism::kDebugBounds ? 1 : 0; }

int prism_debug_bounds_probe(long long i, long long n, prism_stream_t stream) {
  if (!prism::kDebugBounds) return PRISM_ERR_UNSUPPORTED;
  int* status = nullptr;
  const int rc = device_setup(&status);
  if (rc != PRISM_OK) return rc;
  bounds_probe_kernel<<<1, 1, 0, reinterpret_cast<cudaStream_t>(stream)>>>(i, n, status);
  return cudaGetLastError() == cudaSuccess ? PRISM_OK : PRISM_ERR_CUDA;
}

int prism_version(void) {
  return (PRISM_VERSION_MAJOR << 16) | (PRISM_VERSION_MINOR << 8) | PRISM_VERSION_PATCH;
}

const char* prism_status_string(int code) {
  switch (code) {
    case PRISM_OK: return "PRISM_OK";
    case PRISM_ERR_INVALID_ARG: return "PRISM_ERR_INVALID_ARG: a required pointer is NULL or a size is out of range";
    case PRISM_ERR_UNSUPPORTED: return "PRISM_ERR_UNSUPPORTED: valid arguments this build does not implement (head size, width, chunk, alignment or device)";
    case PRISM_ERR_WORKSPACE: return "PRISM_ERR_WORKSPACE: workspace smaller than prism_scan_fwd_workspace_size()";
    case PRISM_ERR_CUDA: return "PRISM_ERR_CUDA: a CUDA runtime call or kernel launch failed";
    case PRISM_ERR_TIMEOUT: return "PRISM_ERR_TIMEOUT: a bounded device-side wait expired";
    case PRISM_ERR_BOUNDS: return "PRISM_ERR_BOUNDS: a kernel computed an index outside its buffer (debug build)";
    default: return "PRISM: unknown status code";
  }
}

void prism_set_split_event(void* event) { g_split_event.store(event); }

void prism_set_spin_limit(long long limit) {
  g_spin_limit.store(limit > 0 ? limit : kDefaultSpinLimit);
}

size_t prism_scan_fwd_workspace_size(int B, int T, int H, int d_k, int d_v, int L, int W, int chunk,
                                     int dtype) {
  if (check_sizes(B, T, H, d_k, d_v, L, W, chunk, dtype) != PRISM_OK) return 0;
  // the tensor-core scan keeps the residual write vectors (bf16, the shape of gain) and, when
  // it cuts a long sequence over few chains into segments, three fp32 states per segment
  if (prism::chunk_scan_supported(d_k, d_v, L, W, chunk, dtype))
    return prism::chunk_scan_workspace_bytes(B, T, H, d_k, L);
  return 0;
}

int prism_scan_fwd(const void* q, const void* k, const void* v, const float* gamma, const float* beta,
                   const void* u, const float* alpha, const void* gain, const float* conv_w,
                   const float* S0, const int32_t* lengths, int B, int T, int H, int d_k, int d_v,
                   int L, int W, int chunk, int dtype, void* o, float* S_final, void* workspace,
                   size_t workspace_bytes, prism_stream_t stream) {
  return prism_scan_fwd_ex(q, k, v, gamma, beta, u, alpha, gain, conv_w, S0, lengths, B, T, H, d_k, d_v, L, W,
                           chunk, dtype, o, S_final, workspace, workspace_bytes, stream, PRISM_CHAIN_LINEAR,
                           nullptr);
}

int prism_scan_fwd_ex(const void* q, const void* k, const void* v, const float* gamma, const float* beta,
                      const void* u, const float* alpha, const void* gain, const float* conv_w,
                      const float* S0, const int32_t* lengths, int B, int T, int H, int d_k, int d_v,
                      int L, int W, int chunk, int dtype, void* o, float* S_final, void* workspace,
                      size_t workspace_bytes, prism_stream_t stream, int chain, const void* conv_state) {
  if (chain != PRISM_CHAIN_LINEAR && chain != PRISM_CHAIN_GELU) return PRISM_ERR_INVALID_ARG;
  int rc = check_sizes(B, T, H, d_k, d_v, L, W, chunk, dtype);
  if (rc != PRISM_OK) return rc;
  if (!q || !k || !v || !gamma || !beta || !conv_w || !o) return PRISM_ERR_INVALID_ARG;
  if (L > 1 && (!u || !alpha || !gain)) return PRISM_ERR_INVALID_ARG;
  if (W == 1) conv_state = nullptr;  // no history to read
  const void* ptrs[] = {q, k, v, gamma, beta, conv_w, o, S0, lengths, S_final, workspace,
                        L > 1 ? u : nullptr, L > 1 ? alpha : nullptr, L > 1 ? gain : nullptr, conv_state};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return PRISM_ERR_UNSUPPORTED;
  const size_t need = prism_scan_fwd_workspace_size(B, T, H, d_k, d_v, L, W, chunk, dtype);
  if (need > 0 && (!workspace || workspace_bytes < need)) return PRISM_ERR_WORKSPACE;
  int* status = nullptr;
  rc = device_setup(&status);
  if (rc != PRISM_OK) return rc;

  prism::ScanParams p{q, k, v, gamma, beta, L > 1 ? u : nullptr, L > 1 ? alpha : nullptr,
                      L > 1 ? gain : nullptr, conv_w, S0, lengths, o, S_final,
                      B, T, H, d_k, d_v, L, W, chunk, status, g_spin_limit.load(), chain,
                      need > 0 ? workspace : nullptr};
  p.conv_state = conv_state;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t err;
  if (prism::chunk_scan_supported(d_k, d_v, L, W, chunk, dtype)) {
    if (L > 1) p.split_event = g_split_event.exchange(nullptr);
    err = prism::launch_chunk_scan(p, s);
  } else if (prism::chunk_fp32_supported(d_k, d_v, chunk, dtype))
    err = prism::launch_chunk_fp32(p, s);
  else
    err = prism::launch_recurrent_scan(p, dtype, s);
  return err == cudaSuccess ? PRISM_OK : PRISM_ERR_CUDA;
}

int prism_scan_fwd_host(const void* host_q, const void* host_k, const void* host_v, const float* host_gamma,
                        const float* host_beta, const void* host_u, const float* host_alpha, const void* host_gain,
                        const float* host_conv_w, const float* host_S0, const int32_t* host_lengths, void* dev_q,
                        void* dev_k, void* dev_v, float* dev_gamma, float* dev_beta, void* dev_u, float* dev_alpha,
                        void* dev_gain, float* dev_conv_w, float* dev_S0, int32_t* dev_lengths, int B, int T,
                        int H, int dk, int dv, int L, int W, int chunk, int dtype, void* dev_o,
                        float* dev_S_final, void* host_o, float* host_S_final, void* workspace,
                        size_t workspace_bytes, prism_stream_t stream) {
  int rc = check_sizes(B, T, H, dk, dv, L, W, chunk, dtype);
  if (rc != PRISM_OK) return rc;
  if (!host_q || !host_k || !host_v || !host_gamma || !host_beta || !host_conv_w || !host_o) return PRISM_ERR_INVALID_ARG;
  if (L > 1 && (!host_u || !host_alpha || !host_gain)) return PRISM_ERR_INVALID_ARG;
  if ((host_S0 && !dev_S0) || (host_lengths && !dev_lengths)) return PRISM_ERR_INVALID_ARG;
  const size_t need = prism_scan_fwd_workspace_size(B, T, H, dk, dv, L, W, chunk, dtype);
  if (need > 0 && (!workspace || workspace_bytes < need)) return PRISM_ERR_WORKSPACE;
  const size_t es = dtype == PRISM_FP32 ? 4 : 2;
  const size_t toks = (size_t)B * T * H;
  const size_t m = (size_t)(L - 1);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  struct Copy { void* dst; const void* src; size_t bytes; };
  const Copy in[] = {
      {dev_q, host_q, toks * dk * es}, {dev_k, host_k, toks * dk * es}, {dev_v, host_v, toks * dv * es},
      {dev_gamma, host_gamma, toks * 4}, {dev_beta, host_beta, toks * 4},
      {dev_u, L > 1 ? host_u : nullptr, toks * m * dk * es}, {dev_alpha, L > 1 ? host_alpha : nullptr, toks * m * 4},
      {dev_gain, L > 1 ? host_gain : nullptr, toks * m * dv * es},
      {dev_conv_w, host_conv_w, (size_t)H * dv * W * 4},
      {dev_S0, host_S0, (size_t)B * H * dv * dk * 4}, {dev_lengths, host_lengths, (size_t)B * 4}};
  for (const Copy& c : in) {
    if (!c.src || c.bytes == 0) continue;
    if (!c.dst) return PRISM_ERR_INVALID_ARG;
    if (cudaMemcpyAsync(c.dst, c.src, c.bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
      return PRISM_ERR_CUDA;
  }
  rc = prism_scan_fwd(dev_q, dev_k, dev_v, dev_gamma, dev_beta, dev_u, dev_alpha, dev_gain, dev_conv_w,
                      host_S0 ? dev_S0 : nullptr, host_lengths ? dev_lengths : nullptr, B, T, H, dk, dv, L, W,
                      chunk, dtype, dev_o, host_S_final ? dev_S_final : nullptr, workspace, workspace_bytes,
                      stream);
  if (rc != PRISM_OK) return rc;
  if (cudaMemcpyAsync(host_o, dev_o, toks * dv * es, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return PRISM_ERR_CUDA;
  if (host_S_final && dev_S_final &&
      cudaMemcpyAsync(host_S_final, dev_S_final, (size_t)B * H * dv * dk * 4, cudaMemcpyDeviceToHost, s) !=
          cudaSuccess)
    return PRISM_ERR_CUDA;
  return PRISM_OK;
}

int prism_prologue_fwd(const void* v, const float* alpha, const void* gain, const float* conv_w,
                       const int32_t* lengths, int B, int T, int H, int d_v, int L, int W, int dtype,
                       float* rho_out, prism_stream_t stream) {
  return prism_prologue_fwd_ex(v, alpha, gain, conv_w, lengths, B, T, H, d_v, L, W, dtype, rho_out, stream,
                               PRISM_CHAIN_LINEAR);
}

int prism_prologue_fwd_ex(const void* v, const float* alpha, const void* gain, const float* conv_w,
                          const int32_t* lengths, int B, int T, int H, int d_v, int L, int W, int dtype,
                          float* rho_out, prism_stream_t stream, int chain) {
  if (chain != PRISM_CHAIN_LINEAR && chain != PRISM_CHAIN_GELU) return PRISM_ERR_INVALID_ARG;
  int rc = check_sizes(B, T, H, d_v, d_v, L, W, 64, dtype);
  if (rc != PRISM_OK) return rc;
  if (L < 2 || !v || !alpha || !gain || !conv_w || !rho_out) return PRISM_ERR_INVALID_ARG;
  const void* ptrs[] = {v, alpha, gain, conv_w, lengths, rho_out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return PRISM_ERR_UNSUPPORTED;
  int* status = nullptr;
  rc = device_setup(&status);
  if (rc != PRISM_OK) return rc;
  cudaError_t err = prism::launch_prologue(v, alpha, gain, conv_w, lengths, B, T, H, d_v, L, W, dtype,
                                           rho_out, reinterpret_cast<cudaStream_t>(stream), chain);
  return err == cudaSuccess ? PRISM_OK : PRISM_ERR_CUDA;
}

int prism_scan_fwd_launches(int B, int T, int H, int d_k, int d_v, int L, int W, int chunk, int dtype) {
  if (check_sizes(B, T, H, d_k, d_v, L, W, chunk, dtype) != PRISM_OK) return 0;
  if (prism::chunk_scan_supported(d_k, d_v, L, W, chunk, dtype)) return prism::chunk_scan_launches(B, T, H, L);
  return 1;
}

int prism_scan_fwd_split_chunks(int B, int T, int H, int d_k, int d_v, int L, int W, int chunk, int dtype) {
  if (check_sizes(B, T, H, d_k, d_v, L, W, chunk, dtype) != PRISM_OK) return 0;
  if (!prism::chunk_scan_supported(d_k, d_v, L, W, chunk, dtype)) return 0;
  return prism::chunk_scan_split_chunks(B, T, H, L);
}

int prism_scan_fwd_uses_tensor_cores(int d_k, int d_v, int L, int W, int chunk, int dtype) {
  if (check_sizes(1, 1, 1, d_k, d_v, L, W, chunk, dtype) != PRISM_OK) return 0;
  return prism::chunk_scan_supported(d_k, d_v, L, W, chunk, dtype) ? 1 : 0;
}

int prism_stream_status(prism_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return PRISM_ERR_CUDA;
  int* status = nullptr;
  int rc = device_setup(&status);
  if (rc != PRISM_OK) return rc;
  int value = 0, zero = 0;
  if (cudaMemcpy(&value, status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return PRISM_ERR_CUDA;
  if (value != PRISM_OK && cudaMemcpy(status, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
    return PRISM_ERR_CUDA;
  return value;
}

int prism_state_affine(const float* S, const float* M, const float* N, float* out, int BH, int d_v, int d_k,
                       prism_stream_t stream) {
  if (!S || !M || !out || BH < 1 || d_v < 1 || d_k < 1) return PRISM_ERR_INVALID_ARG;
  if (!head_dim_ok(d_k) || !head_dim_ok(d_v) || BH > 65535) return PRISM_ERR_UNSUPPORTED;
  // out may be S or N exactly (every element is read by the thread that writes it, after
  // its row has been staged); any other overlap with S, M or N would be read after write
  const size_t sn_bytes = (size_t)BH * d_v * d_k * sizeof(float), m_bytes = (size_t)BH * d_k * d_k * sizeof(float);
  if (ranges_overlap(out, sn_bytes, M, m_bytes)) return PRISM_ERR_INVALID_ARG;
  if (out != S && ranges_overlap(out, sn_bytes, S, sn_bytes)) return PRISM_ERR_INVALID_ARG;
  if (N && out != N && ranges_overlap(out, sn_bytes, N, sn_bytes)) return PRISM_ERR_INVALID_ARG;
  int* status = nullptr;
  const int rc = device_setup(&status);
  if (rc != PRISM_OK) return rc;
  const cudaError_t err =
      prism::launch_state_affine(S, M, N, out, BH, d_v, d_k, reinterpret_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? PRISM_OK : PRISM_ERR_CUDA;
}

int prism_decode_step(const void* q, const void* k, const void* v, const float* gamma, const float* beta,
                      const void* u, const float* alpha, const void* gain, const float* conv_w,
                      void* conv_state, float* S, int B, int H, int d_k, int d_v, int L, int W, int dtype,
                      int chain, void* o, prism_stream_t stream) {
  if (chain != PRISM_CHAIN_LINEAR && chain != PRISM_CHAIN_GELU) return PRISM_ERR_INVALID_ARG;
  int rc = check_sizes(B, 1, H, d_k, d_v, L, W, 16, dtype);
  if (rc != PRISM_OK) return rc;
  if (!q || !k || !v || !gamma || !beta || !conv_w || !S || !o) return PRISM_ERR_INVALID_ARG;
  if (L > 1 && (!u || !alpha || !gain)) return PRISM_ERR_INVALID_ARG;
  if (W > 1 && !conv_state) return PRISM_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, gamma, beta, u, alpha, gain, conv_w, conv_state, S, o};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return PRISM_ERR_UNSUPPORTED;
  int* status = nullptr;
  rc = device_setup(&status);
  if (rc != PRISM_OK) return rc;
  prism::DecodeParams p{q, k, v, gamma, beta, L > 1 ? u : nullptr, L > 1 ? alpha : nullptr, L > 1 ? gain : nullptr,
                        conv_w, W > 1 ? conv_state : nullptr, S, o, B, H, d_k, d_v, L, W, chain, status};
  cudaError_t err = prism::launch_decode_step(p, dtype, reinterpret_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? PRISM_OK : PRISM_ERR_CUDA;
}

namespace {

// Workspace of the chunked backward: the forward and adjoint records (fp32).
struct ChunkBwdWs {
  size_t states, psi, Hn, gk, gu, hs, part, total;
  ChunkBwdWs(int B, int T, int H, int d, int L, int W) {
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t NC = (size_t)(T + prism::kBwdChunk - 1) / prism::kBwdChunk;
    const size_t tok = (size_t)B * T * H;
    size_t o = 0;
    states = o; o += al((size_t)B * H * (NC + 1) * d * d * 4);
    Hn = o;     o += al((size_t)B * H * NC * d * d * 4);
    psi = o;    o += al(tok * d * 4);
    gk = o;     o += al(tok * d * 4);
    gu = o;     o += al(tok * (size_t)(L - 1) * d * 4);
    hs = o;     o += al((size_t)B * H * NC * d * 4);
    part = o;   o += al((size_t)B * NC * H * d * W * 4);
    total = o;
  }
};

}  // namespace

size_t prism_scan_bwd_workspace_size(int B, int T, int H, int d_k, int d_v, int L, int W, int dtype) {
  if (check_sizes(B, T, H, d_k, d_v, L, W, 16, dtype) != PRISM_OK) return 0;
  if (prism::chunk_bwd_supported(d_k, d_v, L)) return ChunkBwdWs(B, T, H, d_k, L, W).total;
  auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const size_t nv = (size_t)(L + 1) * d_k + (L + 1);
  return al((size_t)B * H * T * d_v * d_k * 4) + al((size_t)B * H * d_v * W * 4) +
         al((size_t)B * T * H * prism::bwd_row_blocks(d_k, d_v) * nv * 4);
}

int prism_scan_bwd(const void* q, const void* k, const void* v, const float* gamma, const float* beta,
                   const void* u, const float* alpha, const void* gain, const float* conv_w, const float* S0,
                   const int32_t* lengths, const void* dO, const float* dS_final, int B, int T, int H, int d_k,
                   int d_v, int L, int W, int dtype, int chain, float* dq, float* dk, float* dv, float* dgamma,
                   float* dbeta, float* du, float* dalpha, float* dgain, float* dconv_w, float* dS0,
                   void* workspace, size_t workspace_bytes, prism_stream_t stream) {
  if (chain != PRISM_CHAIN_LINEAR && chain != PRISM_CHAIN_GELU) return PRISM_ERR_INVALID_ARG;
  int rc = check_sizes(B, T, H, d_k, d_v, L, W, 16, dtype);
  if (rc != PRISM_OK) return rc;
  if (!q || !k || !v || !gamma || !beta || !conv_w || !dO) return PRISM_ERR_INVALID_ARG;
  if (!dq || !dk || !dv || !dgamma || !dbeta || !dconv_w || !dS0) return PRISM_ERR_INVALID_ARG;
  if (L > 1 && (!u || !alpha || !gain || !du || !dalpha || !dgain)) return PRISM_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, gamma, beta, conv_w, S0, lengths, dO, dS_final, dq, dk, dv, dgamma, dbeta,
                        dconv_w, dS0, workspace, L > 1 ? u : nullptr, L > 1 ? alpha : nullptr,
                        L > 1 ? gain : nullptr, L > 1 ? du : nullptr, L > 1 ? dalpha : nullptr,
                        L > 1 ? dgain : nullptr};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return PRISM_ERR_UNSUPPORTED;
  if (!prism::chunk_bwd_supported(d_k, d_v, L) && prism::bwd_smem_bytes(d_k, d_v, L) > 227u * 1024u)
    return PRISM_ERR_UNSUPPORTED;
  const size_t need = prism_scan_bwd_workspace_size(B, T, H, d_k, d_v, L, W, dtype);
  if (!workspace || workspace_bytes < need) return PRISM_ERR_WORKSPACE;
  int* status = nullptr;
  rc = device_setup(&status);
  if (rc != PRISM_OK) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t toks = (size_t)B * T * H, m = (size_t)(L - 1);
  // gradients of padded steps stay zero
  struct Z { void* p; size_t bytes; };
  const Z zs[] = {{dq, toks * d_k * 4}, {dk, toks * d_k * 4}, {dv, toks * d_v * 4}, {dgamma, toks * 4},
                  {dbeta, toks * 4}, {du, toks * m * d_k * 4}, {dalpha, toks * m * 4}, {dgain, toks * m * d_v * 4}};
  for (const Z& z : zs)
    if (z.p && z.bytes && cudaMemsetAsync(z.p, 0, z.bytes, s) != cudaSuccess) return PRISM_ERR_CUDA;
  if (prism::chunk_bwd_supported(d_k, d_v, L)) {
    // chunked backward: forward records at chunk boundaries, the adjoint pass, then
    // every chunk's gradients in parallel
    const ChunkBwdWs ws(B, T, H, d_k, L, W);
    char* wsb = static_cast<char*>(workspace);
    float* rec_states = reinterpret_cast<float*>(wsb + ws.states);
    float* rec_psi = reinterpret_cast<float*>(wsb + ws.psi);
    prism::ScanParams fp{q, k, v, gamma, beta, L > 1 ? u : nullptr, L > 1 ? alpha : nullptr,
                         L > 1 ? gain : nullptr, conv_w, S0, lengths, nullptr, nullptr, B, T, H, d_k, d_v, L, W, 16,
                         status, g_spin_limit.load(), chain, nullptr, nullptr, rec_states, rec_psi};
    cudaError_t err = prism::launch_recurrent_scan(fp, dtype, s);
    if (err != cudaSuccess) return PRISM_ERR_CUDA;
    prism::ChunkBwdParams cp{q, k, v, gamma, beta, L > 1 ? u : nullptr, L > 1 ? alpha : nullptr,
                             L > 1 ? gain : nullptr, conv_w, lengths, dO, dS_final, rec_states, rec_psi,
                             reinterpret_cast<float*>(wsb + ws.Hn), reinterpret_cast<float*>(wsb + ws.gk),
                             reinterpret_cast<float*>(wsb + ws.gu), reinterpret_cast<float*>(wsb + ws.hs),
                             reinterpret_cast<float*>(wsb + ws.part), dq, dk, dv, dgamma, dbeta,
                             L > 1 ? du : nullptr, L > 1 ? dalpha : nullptr, L > 1 ? dgain : nullptr, dconv_w, dS0,
                             B, T, H, d_k, L, W, chain, status};
    err = prism::launch_chunk_bwd(cp, dtype, s);
    return err == cudaSuccess ? PRISM_OK : PRISM_ERR_CUDA;
  }
  float* states = static_cast<float*>(workspace);
  auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
  char* wsb = static_cast<char*>(workspace);
  const size_t off_conv = al((size_t)B * H * T * d_v * d_k * 4);
  const size_t off_part = off_conv + al((size_t)B * H * d_v * W * 4);
  float* dconv_part = reinterpret_cast<float*>(wsb + off_conv);
  float* part = reinterpret_cast<float*>(wsb + off_part);
  // forward that records S_t after every valid token (no outputs)
  prism::ScanParams fp{q, k, v, gamma, beta, L > 1 ? u : nullptr, L > 1 ? alpha : nullptr, L > 1 ? gain : nullptr,
                       conv_w, S0, lengths, nullptr, nullptr, B, T, H, d_k, d_v, L, W, 16, status,
                       g_spin_limit.load(), chain, nullptr, states};
  cudaError_t err = prism::launch_recurrent_scan(fp, dtype, s);
  if (err != cudaSuccess) return PRISM_ERR_CUDA;
  prism::BwdParams bp{q, k, v, gamma, beta, L > 1 ? u : nullptr, L > 1 ? alpha : nullptr, L > 1 ? gain : nullptr,
                      conv_w, S0, lengths, dO, dS_final, states, dq, dk, dv, dgamma, dbeta,
                      L > 1 ? du : nullptr, L > 1 ? dalpha : nullptr, L > 1 ? dgain : nullptr, dconv_part, part,
                      dconv_w, dS0, B, T, H, d_k, d_v, L, W, chain, status};
  err = prism::launch_scan_bwd(bp, dtype, s);
  return err == cudaSuccess ? PRISM_OK : PRISM_ERR_CUDA;
}

}  // extern "C"
