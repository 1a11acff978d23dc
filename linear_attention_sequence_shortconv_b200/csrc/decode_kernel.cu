// One recurrent step of the PRISM scan for every (batch row, head): the O(1)-state
// inference form of the recurrence (ICML 2026 PRISM write-up, 背景 and Rank-1 写入瓶颈:
// a linear-attention layer keeps a fixed-size state and updates it once per token).
//
// Per (b, h), with the ShortConv history hist = v_{t-W+1..t-1} carried in conv_state:
//   a = w[:,0] v_t + sum_{i>=1} w[:,i] v_{t-i};  r = v_t - a;  r_l = chain step(r_{l-1}, g_l)
//   S <- gamma S (I - beta k k^T) + beta v k^T + sum_l alpha_l r_l u_l^T;   o = S q
//
// HBM-bound on the state: S is read and written once (8 d_v d_k bytes per (b, h)).
// One CTA per (b, h); a state row is spread over kLanes lanes that hold interleaved
// float4 groups of it (element j = 16 i + 4 lane + e), so the four lanes of a row
// read 64 contiguous bytes per load and both row reductions are two shuffles.
#include "common.cuh"

namespace prism {

namespace {

constexpr int kLanes = 4;        // lanes per state row
constexpr int kMaxGroups = 8;    // float4 groups per lane: d_k <= 16 * kMaxGroups = 128

// coherent load (conv_state is rewritten by the same kernel, so no read-only path)
__device__ __forceinline__ float ld_plain(const float* p) { return *p; }
__device__ __forceinline__ float ld_plain(const __nv_bfloat16* p) { return __bfloat162float(*p); }

template <typename T>
__global__ void __launch_bounds__(kLanes * 128) decode_step_kernel(DecodeParams p) {
  extern __shared__ float sh[];  // k [d_k], q [d_k], u [m][d_k] as fp32
  const int bh = blockIdx.x, h = bh % p.H;
  const int dk = p.d_k, dv = p.d_v, m = p.L - 1;
  // debug build: a block or a state row outside the batch reads and writes no global memory
  // (no early return: every thread still meets the barrier below)
  const bool bh_ok = in_bounds(bh, (long long)p.B * p.H, p.status);
  float* sk = sh;
  float* sq = sh + dk;
  float* su = sh + 2 * dk;
  const T* kin = static_cast<const T*>(p.k) + (size_t)bh * dk;
  const T* qin = static_cast<const T*>(p.q) + (size_t)bh * dk;
  const T* uin = static_cast<const T*>(p.u) + (size_t)bh * m * dk;
  for (int j = threadIdx.x; j < dk; j += blockDim.x) {
    sk[j] = bh_ok ? ld1<T>(kin + j) : 0.f;
    sq[j] = bh_ok ? ld1<T>(qin + j) : 0.f;
  }
  for (int j = threadIdx.x; j < m * dk; j += blockDim.x) su[j] = bh_ok ? ld1<T>(uin + j) : 0.f;

  const int c = threadIdx.x / kLanes, lane = threadIdx.x % kLanes;
  const bool ok = bh_ok && in_bounds(c, dv, p.status);
  const int groups = dk / (4 * kLanes);
  float* Srow = p.S + ((size_t)bh * dv + c) * dk;
  float4 s[kMaxGroups];
#pragma unroll
  for (int i = 0; i < kMaxGroups; ++i)
    if (i < groups) s[i] = ok ? *reinterpret_cast<const float4*>(Srow + 16 * i + 4 * lane) : make_float4(0.f, 0.f, 0.f, 0.f);
  const float gam = ok ? __ldg(p.gamma + bh) : 1.f, bet = ok ? __ldg(p.beta + bh) : 0.f;
  const float vc = ok ? ld1<T>(static_cast<const T*>(p.v) + (size_t)bh * dv + c) : 0.f;
  // ShortConv anchor from the carried history (oldest first)
  const float* w = p.conv_w + ((size_t)h * dv + c) * p.W;
  T* hist = static_cast<T*>(p.conv_state) + (size_t)bh * (p.W - 1) * dv + c;
  float hv[PRISM_MAX_W];
  float a = ok ? __ldg(w) * vc : 0.f;
#pragma unroll
  for (int i = 1; i < PRISM_MAX_W; ++i) {
    hv[i] = 0.f;
    if (ok && i < p.W) {
      hv[i] = ld_plain(hist + (size_t)(p.W - 1 - i) * dv);  // v_{t-i}
      a += __ldg(w + i) * hv[i];
    }
  }
  __syncthreads();

  // (S k)_c
  float part = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxGroups; ++i) {
    if (i < groups) {
      const float4 kk = *reinterpret_cast<const float4*>(sk + 16 * i + 4 * lane);
      part += s[i].x * kk.x + s[i].y * kk.y + s[i].z * kk.z + s[i].w * kk.w;
    }
  }
  part += __shfl_xor_sync(0xffffffffu, part, 1);
  part += __shfl_xor_sync(0xffffffffu, part, 2);
  // S_c <- gamma (S_c - beta (S k)_c k) + beta v_c k
  const float ck = bet * (vc - gam * part);
#pragma unroll
  for (int i = 0; i < kMaxGroups; ++i) {
    if (i < groups) {
      const float4 kk = *reinterpret_cast<const float4*>(sk + 16 * i + 4 * lane);
      s[i].x = gam * s[i].x + ck * kk.x;
      s[i].y = gam * s[i].y + ck * kk.y;
      s[i].z = gam * s[i].z + ck * kk.z;
      s[i].w = gam * s[i].w + ck * kk.w;
    }
  }
  // residual chain and its rank-m write
  if (m > 0 && ok) {
    const T* g = static_cast<const T*>(p.gain) + (size_t)bh * m * dv + c;
    const float* al = p.alpha + (size_t)bh * m;
    float r = vc - a;
    for (int l = 0; l < m; ++l) {
      r = chain_step(r, ld1<T>(g + (size_t)l * dv), p.chain);
      const float rho = __ldg(al + l) * r;
      const float* ul = su + l * dk;
#pragma unroll
      for (int i = 0; i < kMaxGroups; ++i) {
        if (i < groups) {
          const float4 uu = *reinterpret_cast<const float4*>(ul + 16 * i + 4 * lane);
          s[i].x += rho * uu.x;
          s[i].y += rho * uu.y;
          s[i].z += rho * uu.z;
          s[i].w += rho * uu.w;
        }
      }
    }
  }
  // o_c = S_c q, state written back in place
  float oc = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxGroups; ++i) {
    if (i < groups) {
      const float4 qq = *reinterpret_cast<const float4*>(sq + 16 * i + 4 * lane);
      oc += s[i].x * qq.x + s[i].y * qq.y + s[i].z * qq.z + s[i].w * qq.w;
      if (ok) *reinterpret_cast<float4*>(Srow + 16 * i + 4 * lane) = s[i];
    }
  }
  oc += __shfl_xor_sync(0xffffffffu, oc, 1);
  oc += __shfl_xor_sync(0xffffffffu, oc, 2);
  if (lane == 0 && ok) {
    st1<T>(static_cast<T*>(p.o) + (size_t)bh * dv + c, oc);
    // history <- (v_{t-W+2}, ..., v_t), oldest first: slot W-2-i takes v_{t-i}; this thread
    // read channel c's old history above, so the shift reuses those values
#pragma unroll
    for (int i = 0; i < PRISM_MAX_W - 1; ++i)
      if (i < p.W - 1) st1<T>(hist + (size_t)(p.W - 2 - i) * dv, i == 0 ? vc : hv[i]);
  }
}

}  // namespace

cudaError_t launch_decode_step(const DecodeParams& p, int dtype, cudaStream_t stream) {
  const int threads = kLanes * p.d_v;
  const size_t smem = (size_t)(p.L + 1) * p.d_k * sizeof(float);
  if (dtype == PRISM_FP32)
    decode_step_kernel<float><<<p.B * p.H, threads, smem, stream>>>(p);
  else
    decode_step_kernel<__nv_bfloat16><<<p.B * p.H, threads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace prism
