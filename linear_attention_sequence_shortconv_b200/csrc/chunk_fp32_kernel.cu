// Chunkwise PRISM scan in fp32 on CUDA cores: the fp32 build of the chunk form.
//
// The same decomposition the tensor-core scan runs, with every product in fp32
// FMAs (the chunkwise scan of the ICML 2026 PRISM write-up, 消除 Token 间串行, and
// the technical summary 2.1: the state update is affine in S with input-only
// coefficients, so a chunk is a few dense products and one triangular solve).
// With S_n the state before chunk n, c_t the in-chunk cumulative log decay
// (b_t = e^{c_t}, D[t,i] = e^{c_t - c_i}) and rho_{t,l} = alpha_{t,l} r_{t,l}:
//
//   A[t,i]    = beta_t D[t,i] k_t.k_i              (i < t)
//   T         = (I + A)^{-1}                        (unit lower triangular)
//   X         = diag(beta) V - sum_l Bku_l P_l,     Bku_l[t,i] = beta_t D[t,i] k_t.u_{i,l}  (i < t)
//   U' = T X,  W' = T diag(beta b) K,  Delta = U' - W' S_n^T
//   O         = diag(b) Q S_n^T + (M<= . D . Q K^T) Delta + sum_l (M<= . D . Q U_l^T) P_l
//   S_{n+1}   = b_C S_n + Delta^T diag(b_C / b) K + sum_l P_l^T diag(b_C / b) U_l
//
// Delta stacks delta_t = beta_t (v_t - gamma_t S_{t-1} k_t).  Tokens past a row's
// length are exact no-ops (gamma = 1, beta = alpha = 0) and their outputs are zero.
// Every decay factor is e^{c_t - c_i} with i <= t, so none exceeds 1.
//
// One CTA per (batch row, head) walks the chunks in order; the tiles of a chunk sit
// in shared memory with rows padded by one word, so that the column-parallel loops
// read them without bank conflicts.  Only block-wide barriers, no waits on flags.
#include "common.cuh"

namespace prism {
namespace {

constexpr int kF32Threads = 256;

template <int D, int C>
struct F32Layout {
  static constexpr int LD = D + 1, LC = C + 1;
  static constexpr int kTileCD = C * LD, kTileDD = D * LD, kTileCC = C * LC;
  // C x D tiles: K, Q, X (diag(beta) V, then Delta), V, U (then U'), P, R (residual), W', O
  static constexpr int K = 0, Q = K + kTileCD, X = Q + kTileCD, V = X + kTileCD, U = V + kTileCD,
                       P = U + kTileCD, R = P + kTileCD, Wp = R + kTileCD, O = Wp + kTileCD;
  // D x D: the state and the sum of the residual writes' state updates
  static constexpr int S = O + kTileCD, Sadd = S + kTileDD;
  // C x C: A then the masked products, and T
  static constexpr int M = Sadd + kTileDD, T = M + kTileCC;
  // per-token scalars and the ShortConv history (W - 1 <= 7 rows of v before the chunk)
  static constexpr int lc = T + kTileCC, bet = lc + C, eb = bet + C, ec = eb + C, hist = ec + C;
  static constexpr int floats = hist + 7 * D;
  static constexpr int bytes = floats * 4;
};

template <int D, int C>
__global__ void __launch_bounds__(kF32Threads) chunk_fp32_kernel(ScanParams p) {
  using Ly = F32Layout<D, C>;
  constexpr int LD = Ly::LD, LC = Ly::LC;
  extern __shared__ float sm[];
  float *sK = sm + Ly::K, *sQ = sm + Ly::Q, *sX = sm + Ly::X, *sV = sm + Ly::V, *sU = sm + Ly::U;
  float *sP = sm + Ly::P, *sR = sm + Ly::R, *sW = sm + Ly::Wp, *sO = sm + Ly::O;
  float *sS = sm + Ly::S, *sSa = sm + Ly::Sadd, *sM = sm + Ly::M, *sT = sm + Ly::T;
  float *slc = sm + Ly::lc, *sbet = sm + Ly::bet, *shist = sm + Ly::hist;
  float *seb = sm + Ly::eb, *sec = sm + Ly::ec;  // b_t = e^{c_t} and b_C / b_t

  const int tid = threadIdx.x;
  const int h = blockIdx.x, b = blockIdx.y;
  const int T_ = p.T, H = p.H, W = p.W, m = p.L - 1;
  const int len = p.lengths ? min(max(p.lengths[b], 0), T_) : T_;
  const float* q = static_cast<const float*>(p.q);
  const float* k = static_cast<const float*>(p.k);
  const float* v = static_cast<const float*>(p.v);
  const float* u = static_cast<const float*>(p.u);
  const float* gain = static_cast<const float*>(p.gain);
  const float* conv_state = static_cast<const float*>(p.conv_state);
  float* o = static_cast<float*>(p.o);
  const size_t bh = (size_t)b * H + h;
  int* status = p.status;
  // extents of the buffers (the debug build checks every index against them)
  const long long n_tok = (long long)p.B * T_ * H, n_x = n_tok * D, n_u = n_x * max(m, 1);

  // S_0 and the v rows before token 0 (the caller's ShortConv history, or zeros)
  for (int e = tid; e < D * D; e += kF32Threads) {
    const int c = e / D, j = e % D;
    sS[c * LD + j] = p.S0 && in_bounds((long long)(bh * D * D + e), (long long)p.B * H * D * D, status)
                         ? p.S0[bh * D * D + e]
                         : 0.f;
  }
  for (int e = tid; e < (W - 1) * D; e += kF32Threads)
    shist[e] = conv_state && in_bounds((long long)(bh * (W - 1) * D + e), (long long)p.B * H * (W - 1) * D, status)
                   ? conv_state[bh * (W - 1) * D + e]
                   : 0.f;

  const int nchunks = (len + C - 1) / C;
  for (int n = 0; n < nchunks; ++n) {
    const int t0 = n * C, nv = min(C, len - t0);
    __syncthreads();  // the previous chunk's readers of every tile are done
    // ---- tiles of the chunk (padded tokens: zero vectors, gamma = 1, beta = 0)
    for (int e = tid; e < C * D; e += kF32Threads) {
      const int t = e / D, c = e % D;
      const size_t g = (((size_t)b * T_ + t0 + t) * H + h) * D + c;
      const bool ok = t < nv && in_bounds((long long)g, n_x, status);
      sK[t * LD + c] = ok ? k[g] : 0.f;
      sQ[t * LD + c] = ok ? q[g] : 0.f;
      sV[t * LD + c] = ok ? v[g] : 0.f;
      sO[t * LD + c] = 0.f;
    }
    for (int e = tid; e < D * D; e += kF32Threads) sSa[(e / D) * LD + e % D] = 0.f;
    if (tid < C) {
      const size_t g = ((size_t)b * T_ + t0 + tid) * H + h;
      const bool ok = tid < nv && in_bounds((long long)g, n_tok, status);
      slc[tid] = ok ? logf(p.gamma[g]) : 0.f;  // prefix-summed below
      sbet[tid] = ok ? p.beta[g] : 0.f;
    }
    __syncthreads();
    if (tid == 0) {
      float acc = 0.f;
      for (int t = 0; t < C; ++t) {
        acc += slc[t];
        slc[t] = acc;
      }
      for (int t = 0; t < C; ++t) {
        seb[t] = expf(slc[t]);
        sec[t] = expf(acc - slc[t]);
      }
    }
    // ---- r_0 = v - sum_i w_i v_{t-i} (ShortConv anchor, history before the chunk)
    for (int e = tid; e < C * D; e += kF32Threads) {
      const int t = e / D, c = e % D;
      float a = 0.f;
      for (int i = 0; i < W; ++i) {
        const int tau = t - i;
        const float vi = tau >= 0 ? sV[tau * LD + c] : shist[(W - 1 + tau) * D + c];
        const long long wi = ((long long)h * D + c) * W + i;
        if (in_bounds(wi, (long long)H * D * W, status)) a = fmaf(p.conv_w[wi], vi, a);
      }
      sR[t * LD + c] = t < nv ? sV[t * LD + c] - a : 0.f;
    }
    __syncthreads();
    // ---- A (strictly lower) and X = diag(beta) V
    for (int e = tid; e < C * C; e += kF32Threads) {
      const int t = e / C, i = e % C;
      float a = 0.f;
      if (i < t) {
        for (int j = 0; j < D; ++j) a = fmaf(sK[t * LD + j], sK[i * LD + j], a);
        a *= sbet[t] * expf(slc[t] - slc[i]);
      }
      sM[t * LC + i] = a;
    }
    for (int e = tid; e < C * D; e += kF32Threads) {
      const int t = e / D, c = e % D;
      sX[t * LD + c] = sbet[t] * sV[t * LD + c];
    }
    __syncthreads();
    // ---- T = (I + A)^{-1} by forward substitution, one column per thread
    if (tid < C) {
      const int j = tid;
      for (int t = 0; t < C; ++t) {
        float x = t == j ? 1.f : 0.f;
        if (t > j) {
          for (int i = j; i < t; ++i) x = fmaf(-sM[t * LC + i], sT[i * LC + j], x);
        }
        sT[t * LC + j] = x;
      }
    }
    // ---- the residual directions: chain step, P_l, and their three products
    for (int l = 0; l < m; ++l) {
      __syncthreads();  // T done (l = 0) / the previous direction's products are done
      for (int e = tid; e < C * D; e += kF32Threads) {
        const int t = e / D, c = e % D;
        const size_t g = ((((size_t)b * T_ + t0 + t) * H + h) * m + l) * D + c;
        const bool ok = t < nv && in_bounds((long long)g, n_u, status);
        const float r = ok ? chain_step(sR[t * LD + c], gain[g], p.chain) : 0.f;
        const float al = ok ? p.alpha[(((size_t)b * T_ + t0 + t) * H + h) * m + l] : 0.f;
        sR[t * LD + c] = r;
        sP[t * LD + c] = al * r;
        sU[t * LD + c] = ok ? u[g] : 0.f;
      }
      __syncthreads();
      // Bku_l (strictly lower)
      for (int e = tid; e < C * C; e += kF32Threads) {
        const int t = e / C, i = e % C;
        float a = 0.f;
        if (i < t) {
          for (int j = 0; j < D; ++j) a = fmaf(sK[t * LD + j], sU[i * LD + j], a);
          a *= sbet[t] * expf(slc[t] - slc[i]);
        }
        sM[t * LC + i] = a;
      }
      // the state update of this direction: Sadd += P_l^T diag(b_C / b) U_l
      for (int e = tid; e < D * D; e += kF32Threads) {
        const int c = e / D, j = e % D;
        float a = sSa[c * LD + j];
        for (int i = 0; i < C; ++i) a = fmaf(sP[i * LD + c] * sec[i], sU[i * LD + j], a);
        sSa[c * LD + j] = a;
      }
      __syncthreads();
      // X -= Bku_l P_l
      for (int e = tid; e < C * D; e += kF32Threads) {
        const int t = e / D, c = e % D;
        float a = sX[t * LD + c];
        for (int i = 0; i < t; ++i) a = fmaf(-sM[t * LC + i], sP[i * LD + c], a);
        sX[t * LD + c] = a;
      }
      __syncthreads();
      // (M<= . D . Q U_l^T), then O += it times P_l
      for (int e = tid; e < C * C; e += kF32Threads) {
        const int t = e / C, i = e % C;
        float a = 0.f;
        if (i <= t) {
          for (int j = 0; j < D; ++j) a = fmaf(sQ[t * LD + j], sU[i * LD + j], a);
          a *= expf(slc[t] - slc[i]);
        }
        sM[t * LC + i] = a;
      }
      __syncthreads();
      for (int e = tid; e < C * D; e += kF32Threads) {
        const int t = e / D, c = e % D;
        float a = sO[t * LD + c];
        for (int i = 0; i <= t; ++i) a = fmaf(sM[t * LC + i], sP[i * LD + c], a);
        sO[t * LD + c] = a;
      }
    }
    __syncthreads();
    // ---- U' = T X (into U) and W' = T diag(beta b) K
    for (int e = tid; e < C * D; e += kF32Threads) {
      const int t = e / D, c = e % D;
      float a = 0.f, w = 0.f;
      for (int i = 0; i <= t; ++i) {
        const float ti = sT[t * LC + i];
        a = fmaf(ti, sX[i * LD + c], a);
        w = fmaf(ti * sbet[i] * seb[i], sK[i * LD + c], w);
      }
      sU[t * LD + c] = a;
      sW[t * LD + c] = w;
    }
    // (M<= . D . Q K^T)
    for (int e = tid; e < C * C; e += kF32Threads) {
      const int t = e / C, i = e % C;
      float a = 0.f;
      if (i <= t) {
        for (int j = 0; j < D; ++j) a = fmaf(sQ[t * LD + j], sK[i * LD + j], a);
        a *= expf(slc[t] - slc[i]);
      }
      sM[t * LC + i] = a;
    }
    __syncthreads();
    // ---- Delta = U' - W' S_n^T (into X); diag(b) Q S_n^T onto O
    for (int e = tid; e < C * D; e += kF32Threads) {
      const int t = e / D, c = e % D;
      float dl = sU[t * LD + c], qs = 0.f;
      for (int j = 0; j < D; ++j) {
        const float s = sS[c * LD + j];
        dl = fmaf(-sW[t * LD + j], s, dl);
        qs = fmaf(sQ[t * LD + j], s, qs);
      }
      sX[t * LD + c] = dl;
      sO[t * LD + c] = fmaf(seb[t], qs, sO[t * LD + c]);
    }
    __syncthreads();
    // ---- O += (M<= . D . Q K^T) Delta, written out for the valid tokens
    for (int e = tid; e < C * D; e += kF32Threads) {
      const int t = e / D, c = e % D;
      float a = sO[t * LD + c];
      for (int i = 0; i <= t; ++i) a = fmaf(sM[t * LC + i], sX[i * LD + c], a);
      const size_t oi = (((size_t)b * T_ + t0 + t) * H + h) * D + c;
      if (t < nv && in_bounds((long long)oi, n_x, status)) o[oi] = a;
    }
    // ---- S_{n+1} = b_C S_n + Delta^T diag(b_C / b) K + Sadd
    for (int e = tid; e < D * D; e += kF32Threads) {
      const int c = e / D, j = e % D;
      float a = seb[C - 1] * sS[c * LD + j] + sSa[c * LD + j];
      for (int i = 0; i < C; ++i) a = fmaf(sX[i * LD + c] * sec[i], sK[i * LD + j], a);
      sS[c * LD + j] = a;  // each element is read and written by this thread only
    }
    // ---- the last W - 1 rows of v for the next chunk's anchor (every chunk but the last is full)
    for (int e = tid; e < (W - 1) * D; e += kF32Threads) {
      const int i = e / D, c = e % D;
      shist[e] = sV[(C - (W - 1) + i) * LD + c];
    }
  }
  __syncthreads();
  for (size_t e = tid; e < (size_t)(T_ - len) * D; e += kF32Threads) {
    const int t = len + (int)(e / D), c = (int)(e % D);
    const size_t oi = (((size_t)b * T_ + t) * H + h) * D + c;
    if (in_bounds((long long)oi, n_x, status)) o[oi] = 0.f;
  }
  if (p.S_final)
    for (int e = tid; e < D * D; e += kF32Threads)
      if (in_bounds((long long)(bh * D * D + e), (long long)p.B * H * D * D, status))
        p.S_final[bh * D * D + e] = sS[(e / D) * LD + e % D];
}

template <int D, int C>
cudaError_t launch_dc(const ScanParams& p, cudaStream_t stream) {
  constexpr int smem = F32Layout<D, C>::bytes;
  cudaError_t err = cudaFuncSetAttribute(chunk_fp32_kernel<D, C>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  chunk_fp32_kernel<D, C><<<dim3(p.H, p.B), kF32Threads, smem, stream>>>(p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const ScanParams& p, cudaStream_t stream) {
  switch (p.chunk) {
    case 16: return launch_dc<D, 16>(p, stream);
    case 32: return launch_dc<D, 32>(p, stream);
    default: return launch_dc<D, 64>(p, stream);
  }
}

}  // namespace

bool chunk_fp32_supported(int d_k, int d_v, int chunk, int dtype) {
  return dtype == PRISM_FP32 && d_k == d_v && (d_k == 16 || d_k == 32 || d_k == 64) &&
         (chunk == 16 || chunk == 32 || chunk == 64);
}

cudaError_t launch_chunk_fp32(const ScanParams& p, cudaStream_t stream) {
  switch (p.d_k) {
    case 16: return launch_d<16>(p, stream);
    case 32: return launch_d<32>(p, stream);
    default: return launch_d<64>(p, stream);
  }
}

}  // namespace prism
