// PRISM prologue on its own: ShortConv anchor, anchor residual and the
// residual chain (closed-form linear or exact GELU steps), giving rho_{t,l} = alpha_{t,l} r_{t,l}.
//
// ICML 2026 PRISM write-up, 消除 Token 间串行 (a short convolution of the input
// replaces the global state as the anchor) and 消除 Step 间串行 (with the GELU
// absorbed into the preconditioner the residual chain is element-wise linear
// and has a closed form: r_l = prod_{j<=l} (1 - g_j) * r_0).
//
// Element-wise and HBM-bound: one thread per (token, head, group of 4 channels),
// consecutive threads on consecutive channel groups, so every load and the
// float4 stores of rho are coalesced.
#include "common.cuh"

namespace prism {

struct PrologueParams {
  const void* v;
  const float* alpha;
  const void* gain;
  const float* conv_w;
  const int32_t* lengths;
  float* rho;
  int B, T, H, d_v, L, W, chain;
};

template <typename T>
__global__ void __launch_bounds__(256) prologue_kernel(PrologueParams p) {
  const int groups = p.d_v / 4;
  const size_t n_threads = (size_t)p.B * p.T * p.H * groups;
  const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n_threads) return;
  const int cg = (int)(idx % groups);
  const size_t tok = idx / groups;  // ((b*T + t)*H + h)
  const int h = (int)(tok % p.H);
  const int t = (int)((tok / p.H) % p.T);
  const int b = (int)(tok / ((size_t)p.H * p.T));
  const int m = p.L - 1, dv = p.d_v, c0 = 4 * cg;
  float4* out = reinterpret_cast<float4*>(p.rho + (tok * m) * dv + c0);
  const int len = p.lengths ? p.lengths[b] : p.T;
  if (t >= len) {
    for (int l = 0; l < m; ++l) out[(size_t)l * dv / 4] = make_float4(0.f, 0.f, 0.f, 0.f);
    return;
  }
  const T* v = static_cast<const T*>(p.v);
  const T* g = static_cast<const T*>(p.gain);
  const float4 vt = ld4<T>(v + tok * dv + c0);
  float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int i = 0; i < p.W && i <= t; ++i) {
    const float4 vi = (i == 0) ? vt : ld4<T>(v + (tok - (size_t)i * p.H) * dv + c0);
    const float* w = p.conv_w + ((size_t)h * dv + c0) * p.W + i;
    a.x += __ldg(w) * vi.x;
    a.y += __ldg(w + p.W) * vi.y;
    a.z += __ldg(w + 2 * p.W) * vi.z;
    a.w += __ldg(w + 3 * p.W) * vi.w;
  }
  float4 r = make_float4(vt.x - a.x, vt.y - a.y, vt.z - a.z, vt.w - a.w);
  for (int l = 0; l < m; ++l) {
    const size_t tl = tok * m + l;
    const float4 gg = ld4<T>(g + tl * dv + c0);
    r.x = chain_step(r.x, gg.x, p.chain);
    r.y = chain_step(r.y, gg.y, p.chain);
    r.z = chain_step(r.z, gg.z, p.chain);
    r.w = chain_step(r.w, gg.w, p.chain);
    const float al = __ldg(p.alpha + tl);
    out[(size_t)l * dv / 4] = make_float4(al * r.x, al * r.y, al * r.z, al * r.w);
  }
}

cudaError_t launch_prologue(const void* v, const float* alpha, const void* gain, const float* conv_w,
                            const int32_t* lengths, int B, int T, int H, int d_v, int L, int W,
                            int dtype, float* rho, cudaStream_t stream, int chain) {
  PrologueParams p{v, alpha, gain, conv_w, lengths, rho, B, T, H, d_v, L, W, chain};
  const size_t n = (size_t)B * T * H * (d_v / 4);
  const unsigned blocks = (unsigned)((n + 255) / 256);
  if (dtype == PRISM_FP32)
    prologue_kernel<float><<<blocks, 256, 0, stream>>>(p);
  else
    prologue_kernel<__nv_bfloat16><<<blocks, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace prism
