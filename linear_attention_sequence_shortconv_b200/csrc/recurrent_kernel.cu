// Token-by-token PRISM scan on CUDA cores (fp32 arithmetic, fp32 or bf16 I/O).
//
// This is the fp32 path of prism_scan_fwd and the path for every shape the
// tensor-core chunk kernel does not cover.  It evaluates the recurrence of the
// PRISM write directly (ICML 2026 PRISM write-up, 核心迭代形式 and 架构形式;
// technical summary 2.1-2.2):
//
//   a = sum_i w_i v_{t-i};  r_0 = v_t - a;  r_l = (1 - g_l) r_{l-1}
//   S <- gamma S (I - beta k k^T) + beta v k^T + sum_l alpha_l r_l u_l^T;  o_t = S q_t
//
// The rows of S are independent recurrences: row c only needs (S k)_c, a dot
// product inside the row.  Each row is held by LPR = d_k / 4 lanes (4 fp32
// elements per lane), so the per-token reductions are warp shuffles and a
// block of 256 threads carries 256 / LPR rows of one (batch, head) pair.
#include "common.cuh"

namespace prism {

template <typename T, int LPR>
__global__ void __launch_bounds__(256) recurrent_scan_kernel(ScanParams p) {
  constexpr int RPB = 256 / LPR;  // rows per block
  const int j = threadIdx.x % LPR;  // lane within the row: owns d_k elements 4j..4j+3
  const int row = blockIdx.x * RPB + threadIdx.x / LPR;
  const int h = blockIdx.y, b = blockIdx.z;
  const int T_ = p.T, H = p.H, dk = p.d_k, dv = p.d_v, m = p.L - 1, W = p.W;
  const bool row_ok = row < dv;
  const int c = row_ok ? row : dv - 1;  // idle rows shadow the last real row (no stores)
  const int len = p.lengths ? min(max(p.lengths[b], 0), T_) : T_;

  const T* q = static_cast<const T*>(p.q);
  const T* k = static_cast<const T*>(p.k);
  const T* v = static_cast<const T*>(p.v);
  const T* u = static_cast<const T*>(p.u);
  const T* g = static_cast<const T*>(p.gain);
  T* o = static_cast<T*>(p.o);

  float w[PRISM_MAX_W];
#pragma unroll
  for (int i = 0; i < PRISM_MAX_W; ++i) w[i] = (i < W) ? p.conv_w[((size_t)h * dv + c) * W + i] : 0.f;
  float hist[PRISM_MAX_W];  // hist[i] = v_{t-1-i}[c]
#pragma unroll
  for (int i = 0; i < PRISM_MAX_W; ++i) hist[i] = 0.f;

  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
  const size_t sbase = (((size_t)b * H + h) * dv + c) * dk + 4 * j;
  if (p.S0) s = __ldg(reinterpret_cast<const float4*>(p.S0 + sbase));

  for (int t = 0; t < len; ++t) {
    const size_t tok = ((size_t)b * T_ + t) * H + h;  // token-head index
    const float4 kk = ld4<T>(k + tok * dk + 4 * j);
    const float4 qq = ld4<T>(q + tok * dk + 4 * j);
    const float vt = ld1<T>(v + tok * dv + c);
    const float gam = __ldg(p.gamma + tok);
    const float bet = __ldg(p.beta + tok);

    // (S_{t-1} k_t)_c
    float sk = s.x * kk.x + s.y * kk.y + s.z * kk.z + s.w * kk.w;
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) sk += __shfl_xor_sync(0xffffffffu, sk, off);

    // ShortConv anchor and anchor residual
    float a = w[0] * vt;
#pragma unroll
    for (int i = 1; i < PRISM_MAX_W; ++i) a += w[i] * hist[i - 1];
    float r = vt - a;
#pragma unroll
    for (int i = PRISM_MAX_W - 1; i > 0; --i) hist[i] = hist[i - 1];
    hist[0] = vt;

    // gated delta write: gamma S (I - beta k k^T) + beta v k^T
    const float coef = bet * (vt - gam * sk);
    s.x = gam * s.x + coef * kk.x;
    s.y = gam * s.y + coef * kk.y;
    s.z = gam * s.z + coef * kk.z;
    s.w = gam * s.w + coef * kk.w;

    // rank-m residual write
    for (int l = 0; l < m; ++l) {
      const size_t tl = tok * m + l;
      r *= 1.f - ld1<T>(g + tl * dv + c);
      const float rho = __ldg(p.alpha + tl) * r;
      const float4 uu = ld4<T>(u + tl * dk + 4 * j);
      s.x += rho * uu.x;
      s.y += rho * uu.y;
      s.z += rho * uu.z;
      s.w += rho * uu.w;
    }

    float oq = s.x * qq.x + s.y * qq.y + s.z * qq.z + s.w * qq.w;
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) oq += __shfl_xor_sync(0xffffffffu, oq, off);
    if (row_ok && j == 0) st1<T>(o + tok * dv + c, oq);
  }
  if (row_ok && j == 0)
    for (int t = len; t < T_; ++t) st1<T>(o + (((size_t)b * T_ + t) * H + h) * dv + c, 0.f);
  if (row_ok && p.S_final) *reinterpret_cast<float4*>(p.S_final + sbase) = s;
}

template <typename T, int LPR>
static cudaError_t launch_lpr(const ScanParams& p, cudaStream_t stream) {
  constexpr int RPB = 256 / LPR;
  dim3 grid((p.d_v + RPB - 1) / RPB, p.H, p.B);
  recurrent_scan_kernel<T, LPR><<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_t(const ScanParams& p, cudaStream_t stream) {
  switch (p.d_k) {
    case 16: return launch_lpr<T, 4>(p, stream);
    case 32: return launch_lpr<T, 8>(p, stream);
    case 64: return launch_lpr<T, 16>(p, stream);
    case 128: return launch_lpr<T, 32>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_recurrent_scan(const ScanParams& p, int dtype, cudaStream_t stream) {
  if (dtype == PRISM_FP32) return launch_t<float>(p, stream);
  return launch_t<__nv_bfloat16>(p, stream);
}

}  // namespace prism
