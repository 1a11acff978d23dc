// Shared device helpers of the PRISM scan kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "prism.h"

namespace prism {

// Sizes and pointers of one prism_scan_fwd call (device pointers).
struct ScanParams {
  const void* q;
  const void* k;
  const void* v;
  const float* gamma;
  const float* beta;
  const void* u;
  const float* alpha;
  const void* gain;
  const float* conv_w;
  const float* S0;
  const int32_t* lengths;
  void* o;
  float* S_final;
  int B, T, H, d_k, d_v, L, W, chunk;
  int* status;            // per-device status word (PRISM_OK / PRISM_ERR_TIMEOUT)
  long long spin_limit;   // bound of every device-side wait
  int chain;              // PRISM_CHAIN_LINEAR or PRISM_CHAIN_GELU
  void* workspace;        // prism_scan_fwd_workspace_size() bytes (NULL when that is 0)
  float* states;          // token-by-token path only: S_t after every valid token,
                          // [B, H, T, d_v, d_k] fp32 (NULL: not recorded)
  // records for the chunked backward (token-by-token path; NULL: not recorded)
  float* rec_states;      // S at every 64-token chunk boundary, [B, H, NC + 1, d_v, d_k] fp32:
                          // slot 0 the initial state, slot n the state after token 64 n - 1,
                          // slot ceil(len / 64) the state after the last valid token
  float* rec_psi;         // v_t - gamma_t S_{t-1} k_t per valid token, [B, T, H, d_v] fp32
  void* split_event;      // tensor-core path: cudaEvent_t recorded after the residual-write launch (or NULL)
  const void* conv_state; // [B, H, W - 1, d_v]: v before token 0, oldest first (NULL: zeros)
};

// Tokens per chunk of the chunked backward.
constexpr int kBwdChunk = 64;

// Pointers and sizes of one prism_decode_step call (device pointers).
struct DecodeParams {
  const void* q;
  const void* k;
  const void* v;
  const float* gamma;
  const float* beta;
  const void* u;
  const float* alpha;
  const void* gain;
  const float* conv_w;
  void* conv_state;
  float* S;
  void* o;
  int B, H, d_k, d_v, L, W, chain;
  int* status;  // device status word (the debug build's bounds checks record there)
};

// Pointers and sizes of one prism_scan_bwd call (device pointers).
struct BwdParams {
  const void* q;
  const void* k;
  const void* v;
  const float* gamma;
  const float* beta;
  const void* u;
  const float* alpha;
  const void* gain;
  const float* conv_w;
  const float* S0;
  const int32_t* lengths;
  const void* dO;
  const float* dS_final;
  const float* states;  // [B, H, T, d_v, d_k]: S_t after every valid token
  float* dq;
  float* dk;
  float* dv;
  float* dgamma;
  float* dbeta;
  float* du;
  float* dalpha;
  float* dgain;
  float* dconv_part;  // [B, H, d_v, W] (workspace)
  float* part;        // [B*T*H, row blocks, NV] per-token partial sums over a block's rows (workspace)
  float* dconv_w;     // [H, d_v, W]
  float* dS0;
  int B, T, H, d_k, d_v, L, W, chain;
  int* status;        // device status word (the debug build's bounds checks record there)
};

// Pointers and sizes of the chunked backward (d_k = d_v = d; device pointers).
// NC = ceil(T / kBwdChunk).  The records are fp32 and live in the workspace.
struct ChunkBwdParams {
  const void* q;
  const void* k;
  const void* v;
  const float* gamma;
  const float* beta;
  const void* u;
  const float* alpha;
  const void* gain;
  const float* conv_w;
  const int32_t* lengths;
  const void* dO;
  const float* dS_final;
  const float* states;  // [B, H, NC + 1, d, d]: S at the chunk boundaries (forward record)
  const float* psi;     // [B, T, H, d]: v_t - gamma_t S_{t-1} k_t (forward record)
  float* Hn;            // [B, H, NC, d, d]: gradient flowing into the end of chunk n from later tokens
  float* gk;            // [B, T, H, d]: G_t k_t
  float* gu;            // [B, T, H, L - 1, d]: G_t u_{t,l}
  float* hs;            // [B, H, NC, d]: row partials of <H_n, S_{n+1}>
  float* dconv_part;    // [B, NC, H, d, W]: per-chunk dconv_w partials
  float* dq;
  float* dk;
  float* dv;
  float* dgamma;
  float* dbeta;
  float* du;
  float* dalpha;
  float* dgain;
  float* dconv_w;
  float* dS0;
  int B, T, H, d, L, W, chain;
  int* status;          // device status word (the debug build's bounds checks record there)
};

// One step of the residual chain.  Exact form (gist.science PRISM explainer, 2.2
// Input-Anchored Loop Unrolling, Residual Update): r <- r - GELU(p * r), GELU in its
// erf form.  Linearised form (ICML 2026 PRISM write-up, 消除 Step 间串行: the GELU is
// absorbed into the preconditioner): r <- (1 - g) r.
__device__ __forceinline__ float chain_step(float r, float g, int chain) {
  if (chain == PRISM_CHAIN_GELU) {
    const float x = g * r;
    return r - 0.5f * x * (1.f + erff(x * 0.7071067811865476f));
  }
  return r * (1.f - g);
}

// ---------------------------------------------------------------- element I/O
template <typename T>
__device__ __forceinline__ float ld1(const T* p);
template <>
__device__ __forceinline__ float ld1<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float ld1<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(__ldg(p));
}

// four consecutive elements starting at p (p 4-element aligned)
template <typename T>
__device__ __forceinline__ float4 ld4(const T* p);
template <>
__device__ __forceinline__ float4 ld4<float>(const float* p) {
  return __ldg(reinterpret_cast<const float4*>(p));
}
template <>
__device__ __forceinline__ float4 ld4<__nv_bfloat16>(const __nv_bfloat16* p) {
  uint2 raw = __ldg(reinterpret_cast<const uint2*>(p));
  __nv_bfloat162 lo = *reinterpret_cast<__nv_bfloat162*>(&raw.x);
  __nv_bfloat162 hi = *reinterpret_cast<__nv_bfloat162*>(&raw.y);
  float2 a = __bfloat1622float2(lo), b = __bfloat1622float2(hi);
  return make_float4(a.x, a.y, b.x, b.y);
}

template <typename T>
__device__ __forceinline__ void st1(T* p, float x);
template <>
__device__ __forceinline__ void st1<float>(float* p, float x) { *p = x; }
template <>
__device__ __forceinline__ void st1<__nv_bfloat16>(__nv_bfloat16* p, float x) {
  *p = __float2bfloat16_rn(x);
}

// In-chunk cumulative log decay of a 64-token chunk, one warp: lane owns tokens 2 lane and
// 2 lane + 1 with gates g0, g1 (1 for padded steps); returns G of those tokens and G_63.  The
// chunk scan and the residual-write launch both call this, so that their per-chunk decisions
// (such as whether e^{-G} stays finite) agree bit for bit.
__device__ __forceinline__ void chunk_log_decay(float g0, float g1, int lane, float& G0, float& G1, float& G63) {
  const float lg0 = __logf(g0), lg1 = __logf(g1);
  float x = lg0 + lg1;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  G63 = __shfl_sync(0xffffffffu, x, 31);
  G0 = x - lg1;
  G1 = x;
}

// A chunk takes the factored decay e^{G_t - G_i} = e^{G_t} e^{-G_i} (and the residual write
// vectors scaled by e^{G_63 - G_i}) when its total log decay keeps e^{-G} finite.
__device__ __forceinline__ bool chunk_decay_fast(float G63) { return G63 >= -60.f; }

__device__ __forceinline__ void record_status(int* status, int code) {
  if (status) atomicCAS(status, PRISM_OK, code);
}

// The debug build (compiled with PRISM_DEBUG_BOUNDS, libprism_debug.so) checks the global
// indices the kernels compute against the extents of their buffers, and the innermost
// coordinate of every TMA copy against the 16-byte rule.  A failed check records
// PRISM_ERR_BOUNDS in the status word and the access is skipped, so a bad index shows up
// in prism_stream_status instead of as a fault.  The release build compiles every check to
// `true`.
#ifdef PRISM_DEBUG_BOUNDS
constexpr bool kDebugBounds = true;
#else
constexpr bool kDebugBounds = false;
#endif

// 0 <= i < n (always true in the release build)
__device__ __forceinline__ bool in_bounds(long long i, long long n, int* status) {
  if (!kDebugBounds) return true;
  if (i >= 0 && i < n) return true;
  record_status(status, PRISM_ERR_BOUNDS);
  return false;
}

// a TMA box of bf16 elements starting at innermost coordinate x inside [0, extent): x a
// multiple of 8 (16 bytes) and x + box <= extent (always true in the release build)
__device__ __forceinline__ bool tma_x_ok(int x, int box, int extent, int* status) {
  if (!kDebugBounds) return true;
  if (x >= 0 && (x & 7) == 0 && x + box <= extent) return true;
  record_status(status, PRISM_ERR_BOUNDS);
  return false;
}

}  // namespace prism
