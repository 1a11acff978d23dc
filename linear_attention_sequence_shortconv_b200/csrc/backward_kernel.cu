// Backward of the PRISM scan: gradients of L = <o, dO> + <S_final, dS_final> with
// respect to q, k, v, gamma, beta, u, alpha, gain, conv_w and S0 (fp32 gradients).
//
// Token-by-token reverse recurrence on CUDA cores, the first correct path of the
// backward.  With G_t = dL/dS_t (future contributions plus dO_t q_t^T), p = S_{t-1} k_t,
// gk = G_t k_t, for the update S_t = gamma S_{t-1} (I - beta k k^T) + beta v k^T + sum_l
// alpha_l r_l u_l^T and the readout o_t = S_t q_t:
//   dq_t = S_t^T dO_t
//   dk_t = G_t^T (beta v - gamma beta p) - gamma beta S_{t-1}^T gk
//   du_l = alpha_l G_t^T r_l,    dalpha_l = r_l . (G_t u_l),   dr_l = alpha_l G_t u_l
//   dgamma_t = <G_t, S_{t-1}> - beta gk . p,   dbeta_t = gk . (v - gamma p)
//   dv_t = beta gk + dr_0 + sum_i w_i da_{t+i}   (da = -dr_0; the ShortConv anchor)
//   G_{t-1} += gamma (G_t - beta gk k^T);  dS0 = G_{-1}
// and the residual chain taken backwards channel by channel.  The states S_t are
// recorded by the token-by-token forward kernel into the workspace.
//
// The rows of G are independent in the reverse recurrence, so each (b, h) is split into
// row blocks of kBwdThreads / LPR rows, one CTA each; LPR lanes per row c of G (EPL =
// d_k / LPR elements each), so the per-row dot products are shuffles.  The per-token sums
// over rows (dq, dk, du and the scalar gradients) are reduced inside each warp with
// shuffles, across the CTA's warps in shared memory, and across row blocks by a separate
// kernel from per-block partials in the workspace; dconv_w is summed per (b, h, row) and
// reduced over the batch the same way, so every result is deterministic.
#include "common.cuh"

namespace prism {

int bwd_row_blocks(int d_k, int d_v);

namespace {

constexpr int kBwdThreads = 256;  // per CTA: kBwdThreads / LPR rows of G

template <int LPR>
__device__ __forceinline__ float row_sum(float x) {
#pragma unroll
  for (int off = LPR / 2; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}
// sum over the rows of a warp (lanes with the same position j in their row)
template <int LPR>
__device__ __forceinline__ float warp_rows_sum(float x) {
#pragma unroll
  for (int off = LPR; off < 32; off <<= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

template <typename T, int EPL>
__device__ __forceinline__ void ld_slice(const T* src, float* dst) {
#pragma unroll
  for (int e = 0; e < EPL; e += 4) {
    const float4 f = ld4<T>(src + e);
    dst[e] = f.x;
    dst[e + 1] = f.y;
    dst[e + 2] = f.z;
    dst[e + 3] = f.w;
  }
}

// d/dx of x Phi(x): Phi(x) + x phi(x)
__device__ __forceinline__ float gelu_grad(float x) {
  return 0.5f * (1.f + erff(x * 0.7071067811865476f)) + x * 0.3989422804014327f * __expf(-0.5f * x * x);
}

// ML, MW: compile-time bounds of L and W (the per-channel chain and window arrays stay in
// registers).
template <typename T, int LPR, int EPL, int CH, int ML, int MW>
__global__ void __launch_bounds__(kBwdThreads) scan_bwd_kernel(BwdParams p) {
  extern __shared__ float red[];  // [warps][NV] per-warp partial sums of one token
  constexpr int RB = kBwdThreads / LPR;  // rows per block
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
  const int rb = blockIdx.x, nrb = gridDim.x;
  const int c_raw = rb * RB + tid / LPR, j = tid % LPR;
  const int bh = blockIdx.y, b = bh / p.H, h = bh % p.H;
  // debug build: a block outside the batch touches no memory (block-uniform)
  if (!in_bounds(bh, (long long)p.B * p.H, p.status)) return;
  const int T_ = p.T, H = p.H, dk = p.d_k, dv = p.d_v, m = p.L - 1, W = p.W;
  const int NV = (2 + m) * dk + (2 + m);
  const int len = p.lengths ? min(max(p.lengths[b], 0), T_) : T_;
  const T* q = static_cast<const T*>(p.q);
  const T* k = static_cast<const T*>(p.k);
  const T* v = static_cast<const T*>(p.v);
  const T* u = static_cast<const T*>(p.u);
  const T* g = static_cast<const T*>(p.gain);
  const T* dO = static_cast<const T*>(p.dO);
  // rows past d_v (a partly empty block) shadow the last row and contribute nothing
  const bool row_ok = c_raw < dv;
  const int c = row_ok ? c_raw : dv - 1;
  const float rv = row_ok ? 1.f : 0.f;

  float w[MW];
#pragma unroll
  for (int i = 0; i < MW; ++i) w[i] = i < W ? __ldg(p.conv_w + ((size_t)h * dv + c) * W + i) : 0.f;
  float G[EPL];
  if (p.dS_final) {
    ld_slice<float, EPL>(p.dS_final + ((size_t)bh * dv + c) * dk + EPL * j, G);
  } else {
#pragma unroll
    for (int e = 0; e < EPL; ++e) G[e] = 0.f;
  }
  float da_later[MW];  // da_later[i] = da_{t+i} for i = 1 .. W-1
  float dw[MW];        // dconv_w of channel c, this (b, h)
#pragma unroll
  for (int i = 0; i < MW; ++i) da_later[i] = dw[i] = 0.f;

  // state slices: S_t of the token being processed and S_{t-1}, each requested one token
  // ahead (S_{t-2} is in flight while token t is processed)
  auto load_state = [&](int tt, float* dst) {  // S_tt; tt = -1 is the initial state
    if (tt >= 0) {
      ld_slice<float, EPL>(p.states + (((size_t)bh * T_ + tt) * dv + c) * dk + EPL * j, dst);
    } else if (p.S0) {
      ld_slice<float, EPL>(p.S0 + ((size_t)bh * dv + c) * dk + EPL * j, dst);
    } else {
#pragma unroll
      for (int e = 0; e < EPL; ++e) dst[e] = 0.f;
    }
  };
  float st[EPL], sp_next[EPL];
  if (len > 0) {
    load_state(len - 1, st);
    load_state(len - 2, sp_next);
  }

  for (int t = len - 1; t >= 0; --t) {
    const size_t th = ((size_t)b * T_ + t) * H + h;
    float sp[EPL];  // S_{t-1}
#pragma unroll
    for (int e = 0; e < EPL; ++e) sp[e] = sp_next[e];
    if (t >= 1) load_state(t - 2, sp_next);  // for the next token
    float qv[EPL], kv[EPL];
    ld_slice<T, EPL>(q + th * dk + EPL * j, qv);
    ld_slice<T, EPL>(k + th * dk + EPL * j, kv);
    const float doc = ld1<T>(dO + th * dv + c);
    const float gam = __ldg(p.gamma + th), bet = __ldg(p.beta + th);
    const float vt = ld1<T>(v + th * dv + c);

    // G_t = G + dO_t q_t^T; row dot products
#pragma unroll
    for (int e = 0; e < EPL; ++e) G[e] += doc * qv[e];
    float pk = 0.f, gk = 0.f, gs = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      pk += sp[e] * kv[e];
      gk += G[e] * kv[e];
      gs += G[e] * sp[e];
    }
    pk = row_sum<LPR>(pk);
    gk = row_sum<LPR>(gk);
    gs = row_sum<LPR>(gs);

    // residual chain of channel c, recomputed: r[0] = v - a, r[l] = chain step
    float hv[MW];  // hv[i] = v_{t-i}[c]
    hv[0] = vt;
#pragma unroll
    for (int i = 1; i < MW; ++i) hv[i] = (i < W && t - i >= 0) ? ld1<T>(v + (th - (size_t)i * H) * dv + c) : 0.f;
    float a = 0.f;
#pragma unroll
    for (int i = 0; i < MW; ++i) a += w[i] * hv[i];
    float r[ML];
    float gl[ML];
    r[0] = vt - a;
#pragma unroll
    for (int l = 1; l < ML; ++l) {
      if (l <= m) {
        gl[l] = ld1<T>(g + (th * m + (l - 1)) * dv + c);
        r[l] = chain_step(r[l - 1], gl[l], CH);
      }
    }

    // per-warp partial sums over rows: dq, dk, du_l (vectors), dgamma, dbeta, dalpha_l
    float* rw = red + warp * NV;
    {
      const float ck = rv * (bet * vt - gam * bet * pk), cs = rv * gam * bet * gk, cq = rv * doc;
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        const float dqe = warp_rows_sum<LPR>(cq * st[e]);
        const float dke = warp_rows_sum<LPR>(ck * G[e] - cs * sp[e]);
        if (lane < LPR) {
          rw[EPL * j + e] = dqe;
          rw[dk + EPL * j + e] = dke;
        }
      }
    }
    float dr_write[ML];
#pragma unroll
    for (int l = 1; l < ML; ++l) {
      if (l <= m) {
        const T* ul = u + (th * m + (l - 1)) * dk + EPL * j;
        float uv[EPL];
        ld_slice<T, EPL>(ul, uv);
        float gu = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) gu += G[e] * uv[e];
        gu = row_sum<LPR>(gu);
        const float al = __ldg(p.alpha + th * m + (l - 1));
        dr_write[l] = al * gu;
        const float ar = rv * al * r[l];
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          const float due = warp_rows_sum<LPR>(ar * G[e]);
          if (lane < LPR) rw[(1 + l) * dk + EPL * j + e] = due;
        }
        const float dal = warp_rows_sum<LPR>(j == 0 ? rv * r[l] * gu : 0.f);
        if (lane == 0) rw[(2 + m) * dk + 2 + (l - 1)] = dal;
      }
    }
    {
      const float dg = warp_rows_sum<LPR>(j == 0 ? rv * (gs - bet * gk * pk) : 0.f);
      const float db = warp_rows_sum<LPR>(j == 0 ? rv * gk * (vt - gam * pk) : 0.f);
      if (lane == 0) {
        rw[(2 + m) * dk] = dg;
        rw[(2 + m) * dk + 1] = db;
      }
    }
    __syncthreads();
    float* pout = p.part + (th * nrb + rb) * NV;  // this block's sums over its rows
    for (int idx = tid; idx < NV; idx += blockDim.x) {
      float sum = 0.f;
      for (int ww = 0; ww < nwarps; ++ww) sum += red[ww * NV + idx];
      pout[idx] = sum;
    }

    // channel c: residual chain backwards, the anchor, dv
    float dr = 0.f;
#pragma unroll
    for (int l = ML - 1; l >= 1; --l) {
      if (l <= m) {
        dr += dr_write[l];
        float dgl, pass;
        if (CH == PRISM_CHAIN_GELU) {
          const float x = gl[l] * r[l - 1];
          const float gp = gelu_grad(x);
          dgl = -dr * r[l - 1] * gp;
          pass = 1.f - gl[l] * gp;
        } else {
          dgl = -dr * r[l - 1];
          pass = 1.f - gl[l];
        }
        if (row_ok && j == 0) p.dgain[(th * m + (l - 1)) * dv + c] = dgl;
        dr *= pass;
      }
    }
    const float da = -dr;  // dL/da_t (r_0 = v_t - a_t)
    float dvt = bet * gk + dr + w[0] * da;
#pragma unroll
    for (int i = 1; i < MW; ++i) dvt += w[i] * da_later[i];
    if (row_ok && j == 0) p.dv[th * dv + c] = dvt;
#pragma unroll
    for (int i = 0; i < MW; ++i) dw[i] += da * hv[i];
#pragma unroll
    for (int i = MW - 1; i >= 2; --i) da_later[i] = da_later[i - 1];
    da_later[1] = da;

    // G_{t-1} = gamma (G_t - beta gk k^T); S_{t-1} becomes the next token's S_t
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      G[e] = gam * (G[e] - bet * gk * kv[e]);
      st[e] = sp[e];
    }
    __syncthreads();  // red is rewritten by the next token
  }
  if (!row_ok) return;
  float* d0 = p.dS0 + ((size_t)bh * dv + c) * dk + EPL * j;
#pragma unroll
  for (int e = 0; e < EPL; e += 4) *reinterpret_cast<float4*>(d0 + e) = make_float4(G[e], G[e + 1], G[e + 2], G[e + 3]);
  if (j == 0)
    for (int i = 0; i < W; ++i) p.dconv_part[((size_t)bh * dv + c) * W + i] = dw[i];
}

// dq, dk, du, dgamma, dbeta, dalpha of every valid token: the sums of the row blocks'
// partials, in a fixed order.  One thread per (token-head, entry).
__global__ void bwd_rows_reduce_kernel(BwdParams p, int nrb) {
  const int dk = p.d_k, m = p.L - 1, NV = (2 + m) * dk + (2 + m);
  const size_t total = (size_t)p.B * p.T * p.H * NV;
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= total) return;
  const size_t th = i / NV;
  const int idx = (int)(i % NV);
  const int b = (int)(th / ((size_t)p.T * p.H)), t = (int)((th / p.H) % p.T);
  const int len = p.lengths ? min(max(p.lengths[b], 0), p.T) : p.T;
  if (t >= len) return;  // padded steps keep their zero gradients
  const float* src = p.part + th * nrb * NV + idx;
  float sum = 0.f;
  for (int r = 0; r < nrb; ++r) sum += src[(size_t)r * NV];
  if (idx < dk) {
    p.dq[th * dk + idx] = sum;
  } else if (idx < 2 * dk) {
    p.dk[th * dk + idx - dk] = sum;
  } else if (idx < (2 + m) * dk) {
    const int l = idx / dk - 2, e = idx % dk;
    p.du[(th * m + l) * dk + e] = sum;
  } else {
    const int s2 = idx - (2 + m) * dk;
    if (s2 == 0) p.dgamma[th] = sum;
    else if (s2 == 1) p.dbeta[th] = sum;
    else p.dalpha[th * m + (s2 - 2)] = sum;
  }
}

// dconv_w[h, c, i] = sum_b dconv_part[b, h, c, i], in a fixed order
__global__ void dconv_reduce_kernel(const float* part, float* dconv_w, int B, int H, int dv, int W) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  const int n = H * dv * W;
  if (idx >= n) return;
  float s = 0.f;
  for (int b = 0; b < B; ++b) s += part[(size_t)b * n + idx];
  dconv_w[idx] = s;
}

template <typename T, int LPR, int EPL, int CH, int ML, int MW>
cudaError_t launch_bwd_bounds(const BwdParams& p, cudaStream_t stream) {
  const int threads = kBwdThreads;
  const int NV = (2 + p.L - 1) * p.d_k + (2 + p.L - 1);
  const size_t smem = (size_t)(threads / 32) * NV * sizeof(float);
  const dim3 grid(bwd_row_blocks(p.d_k, p.d_v), p.B * p.H);
  cudaError_t err =
      cudaFuncSetAttribute(scan_bwd_kernel<T, LPR, EPL, CH, ML, MW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
  if (err != cudaSuccess) return err;
  scan_bwd_kernel<T, LPR, EPL, CH, ML, MW><<<grid, threads, smem, stream>>>(p);
  return cudaGetLastError();
}

template <typename T, int LPR, int EPL, int CH>
cudaError_t launch_bwd_shape(const BwdParams& p, cudaStream_t stream) {
  const bool small_l = p.L <= 4, small_w = p.W <= 4;
  if (small_l && small_w) return launch_bwd_bounds<T, LPR, EPL, CH, 4, 4>(p, stream);
  if (small_l) return launch_bwd_bounds<T, LPR, EPL, CH, 4, PRISM_MAX_W>(p, stream);
  if (small_w) return launch_bwd_bounds<T, LPR, EPL, CH, PRISM_MAX_L, 4>(p, stream);
  return launch_bwd_bounds<T, LPR, EPL, CH, PRISM_MAX_L, PRISM_MAX_W>(p, stream);
}

template <typename T, int CH>
cudaError_t launch_bwd_t(const BwdParams& p, cudaStream_t stream) {
  switch (p.d_k) {  // lanes per row as in the forward token-by-token kernel
    case 16: return launch_bwd_shape<T, 4, 4, CH>(p, stream);
    case 32: return launch_bwd_shape<T, 8, 4, CH>(p, stream);
    case 64: return launch_bwd_shape<T, 8, 8, CH>(p, stream);
    case 128: return launch_bwd_shape<T, 8, 16, CH>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

size_t bwd_smem_bytes(int d_k, int d_v, int L) {
  (void)d_v;
  (void)d_k;
  return (size_t)(kBwdThreads / 32) * ((size_t)(L + 1) * d_k + (L + 1)) * sizeof(float);
}

// row blocks per (b, h): kBwdThreads / LPR rows each (a block may be partly empty)
int bwd_row_blocks(int d_k, int d_v) {
  const int rb = kBwdThreads / (d_k == 16 ? 4 : 8);
  return (d_v + rb - 1) / rb;
}

cudaError_t launch_scan_bwd(const BwdParams& p, int dtype, cudaStream_t stream) {
  cudaError_t err;
  if (dtype == PRISM_FP32)
    err = p.chain == PRISM_CHAIN_GELU ? launch_bwd_t<float, PRISM_CHAIN_GELU>(p, stream)
                                      : launch_bwd_t<float, PRISM_CHAIN_LINEAR>(p, stream);
  else
    err = p.chain == PRISM_CHAIN_GELU ? launch_bwd_t<__nv_bfloat16, PRISM_CHAIN_GELU>(p, stream)
                                      : launch_bwd_t<__nv_bfloat16, PRISM_CHAIN_LINEAR>(p, stream);
  if (err != cudaSuccess) return err;
  {
    const int nrb = bwd_row_blocks(p.d_k, p.d_v);
    const size_t total = (size_t)p.B * p.T * p.H * ((p.L + 1) * p.d_k + (p.L + 1));
    bwd_rows_reduce_kernel<<<(unsigned)((total + 255) / 256), 256, 0, stream>>>(p, nrb);
  }
  const int n = p.H * p.d_v * p.W;
  dconv_reduce_kernel<<<(n + 255) / 256, 256, 0, stream>>>(p.dconv_part, p.dconv_w, p.B, p.H, p.d_v, p.W);
  return cudaGetLastError();
}

}  // namespace prism
