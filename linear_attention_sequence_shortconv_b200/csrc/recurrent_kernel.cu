// Token-by-token PRISM scan on CUDA cores (fp32 arithmetic, fp32 or bf16 I/O).
//
// This is the fp32 path of prism_scan_fwd and the path for every shape the
// tensor-core chunk kernel does not cover (long context with L = 8 among them).
// It evaluates the recurrence of the PRISM write directly (ICML 2026 PRISM
// write-up, 核心迭代形式 and 架构形式; technical summary 2.1-2.2):
//
//   a = sum_i w_i v_{t-i};  r_0 = v_t - a;  r_l = (1 - g_l) r_{l-1}
//   S <- gamma S (I - beta k k^T) + beta v k^T + sum_l alpha_l r_l u_l^T;  o_t = S q_t
//
// The rows of S are independent recurrences: row c only needs (S k)_c, a dot
// product inside the row.  Each row is held by LPR lanes (EPL = d_k / LPR fp32
// elements per lane), so the two per-token reductions are log2(LPR)-step warp
// shuffles.  Blocks of 64 threads carry 64 / LPR rows of one (batch, head), so
// even 8 (batch, head) chains of 128 rows fill 128 blocks.  The next token's
// inputs are loaded one token ahead into registers (directions and gains too
// when L - 1 <= MPF), so the loop waits on the shuffles, not on memory.
#include "common.cuh"

namespace prism {
namespace {

constexpr int kBlock = 64;
constexpr int MPF = 7;  // residual directions prefetched one token ahead

// Groups of 4 consecutive row elements kept in their I/O encoding until used: bf16 as one
// 8-byte word pair, fp32 as a float4.
template <typename T>
struct Raw4;
template <>
struct Raw4<float> {
  float4 w;
  __device__ void load(const float* p) { w = __ldg(reinterpret_cast<const float4*>(p)); }
  __device__ float4 get() const { return w; }
};
template <>
struct Raw4<__nv_bfloat16> {
  uint2 w;
  __device__ void load(const __nv_bfloat16* p) { w = __ldg(reinterpret_cast<const uint2*>(p)); }
  __device__ float4 get() const {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.y));
    return make_float4(a.x, a.y, b.x, b.y);
  }
};

template <typename T, int EPL>
struct RowVec {  // the EPL elements one lane holds of a d_k vector
  Raw4<T> r[EPL / 4];
  __device__ void load(const T* p) {
#pragma unroll
    for (int e = 0; e < EPL / 4; ++e) r[e].load(p + 4 * e);
  }
  __device__ float dot(const float* s) const {
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < EPL / 4; ++e) {
      const float4 f = r[e].get();
      acc += s[4 * e] * f.x + s[4 * e + 1] * f.y + s[4 * e + 2] * f.z + s[4 * e + 3] * f.w;
    }
    return acc;
  }
  __device__ void axpy(float a, float* s) const {  // s += a * this
#pragma unroll
    for (int e = 0; e < EPL / 4; ++e) {
      const float4 f = r[e].get();
      s[4 * e] += a * f.x; s[4 * e + 1] += a * f.y; s[4 * e + 2] += a * f.z; s[4 * e + 3] += a * f.w;
    }
  }
};

template <int LPR>
__device__ __forceinline__ float row_sum(float x) {
#pragma unroll
  for (int off = LPR / 2; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

// Inputs of one token for one row-lane.
template <typename T, int EPL, int MP>
struct Tok {
  RowVec<T, EPL> k, q, u[MP > 0 ? MP : 1];
  float v, gam, bet, g[MP > 0 ? MP : 1], al[MP > 0 ? MP : 1];
};

template <typename T, int LPR, int EPL, int MP>
__global__ void __launch_bounds__(kBlock) recurrent_scan_kernel(ScanParams p) {
  constexpr int RPB = kBlock / LPR;  // rows per block
  const int j = threadIdx.x % LPR;   // lane within the row: owns d_k elements EPL*j .. EPL*j+EPL-1
  const int row = blockIdx.x * RPB + threadIdx.x / LPR;
  const int h = blockIdx.y, b = blockIdx.z;
  const int T_ = p.T, H = p.H, dk = p.d_k, dv = p.d_v, m = p.L - 1, W = p.W;
  const bool row_ok = row < dv;
  const int c = row_ok ? row : dv - 1;  // idle rows shadow the last real row (no stores)
  const int len = p.lengths ? min(max(p.lengths[b], 0), T_) : T_;
  const bool prefetch_dirs = (m <= MP);

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

  float s[EPL];
  const size_t sbase = (((size_t)b * H + h) * dv + c) * dk + EPL * j;
#pragma unroll
  for (int e = 0; e < EPL; e += 4) {
    const float4 f = p.S0 ? __ldg(reinterpret_cast<const float4*>(p.S0 + sbase + e)) : make_float4(0.f, 0.f, 0.f, 0.f);
    s[e] = f.x; s[e + 1] = f.y; s[e + 2] = f.z; s[e + 3] = f.w;
  }

  auto fetch = [&](int t, Tok<T, EPL, MP>& x) {
    const size_t tok = ((size_t)b * T_ + t) * H + h;
    x.k.load(k + tok * dk + EPL * j);
    x.q.load(q + tok * dk + EPL * j);
    x.v = ld1<T>(v + tok * dv + c);
    x.gam = __ldg(p.gamma + tok);
    x.bet = __ldg(p.beta + tok);
    if (prefetch_dirs) {
#pragma unroll
      for (int l = 0; l < MP; ++l) {
        if (l < m) {
          const size_t tl = tok * m + l;
          x.u[l].load(u + tl * dk + EPL * j);
          x.g[l] = ld1<T>(g + tl * dv + c);
          x.al[l] = __ldg(p.alpha + tl);
        }
      }
    }
  };

  Tok<T, EPL, MP> cur, nxt;
  if (len > 0) fetch(0, cur);
  for (int t = 0; t < len; ++t) {
    if (t + 1 < len) fetch(t + 1, nxt);
    const size_t tok = ((size_t)b * T_ + t) * H + h;

    // (S_{t-1} k_t)_c
    const float sk = row_sum<LPR>(cur.k.dot(s));

    // ShortConv anchor and anchor residual
    const float vt = cur.v;
    float a = w[0] * vt;
#pragma unroll
    for (int i = 1; i < PRISM_MAX_W; ++i) a += w[i] * hist[i - 1];
    float r = vt - a;
#pragma unroll
    for (int i = PRISM_MAX_W - 1; i > 0; --i) hist[i] = hist[i - 1];
    hist[0] = vt;

    // gated delta write: gamma S (I - beta k k^T) + beta v k^T
    const float gam = cur.gam;
    const float coef = cur.bet * (vt - gam * sk);
#pragma unroll
    for (int e = 0; e < EPL; ++e) s[e] *= gam;
    cur.k.axpy(coef, s);

    // rank-m residual write
    if (prefetch_dirs) {
#pragma unroll
      for (int l = 0; l < MP; ++l) {
        if (l < m) {
          r *= 1.f - cur.g[l];
          cur.u[l].axpy(cur.al[l] * r, s);
        }
      }
    } else {
      for (int l = 0; l < m; ++l) {
        const size_t tl = tok * m + l;
        r *= 1.f - ld1<T>(g + tl * dv + c);
        RowVec<T, EPL> uu;
        uu.load(u + tl * dk + EPL * j);
        uu.axpy(__ldg(p.alpha + tl) * r, s);
      }
    }

    const float oq = row_sum<LPR>(cur.q.dot(s));
    if (row_ok && j == 0) st1<T>(o + tok * dv + c, oq);
    cur = nxt;
  }
  if (row_ok && j == 0)
    for (int t = len; t < T_; ++t) st1<T>(o + (((size_t)b * T_ + t) * H + h) * dv + c, 0.f);
  if (row_ok && p.S_final) {
#pragma unroll
    for (int e = 0; e < EPL; e += 4)
      *reinterpret_cast<float4*>(p.S_final + sbase + e) = make_float4(s[e], s[e + 1], s[e + 2], s[e + 3]);
  }
}

template <typename T, int LPR, int EPL>
cudaError_t launch_shape(const ScanParams& p, cudaStream_t stream) {
  constexpr int RPB = kBlock / LPR;
  dim3 grid((p.d_v + RPB - 1) / RPB, p.H, p.B);
  constexpr int MPMAX = sizeof(T) == 2 ? MPF : 3;  // fp32 inputs: prefetch at most 3 directions
  if (p.L - 1 <= 3)
    recurrent_scan_kernel<T, LPR, EPL, 3><<<grid, kBlock, 0, stream>>>(p);
  else
    recurrent_scan_kernel<T, LPR, EPL, MPMAX><<<grid, kBlock, 0, stream>>>(p);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_t(const ScanParams& p, cudaStream_t stream) {
  switch (p.d_k) {  // 8 lanes per row (4 for d_k = 16); EPL = d_k / LPR elements per lane
    case 16: return launch_shape<T, 4, 4>(p, stream);
    case 32: return launch_shape<T, 8, 4>(p, stream);
    case 64: return launch_shape<T, 8, 8>(p, stream);
    case 128: return launch_shape<T, 8, 16>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_recurrent_scan(const ScanParams& p, int dtype, cudaStream_t stream) {
  if (dtype == PRISM_FP32) return launch_t<float>(p, stream);
  return launch_t<__nv_bfloat16>(p, stream);
}

}  // namespace prism
