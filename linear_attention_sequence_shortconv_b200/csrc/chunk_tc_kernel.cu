// Chunkwise-parallel PRISM scan on the 5th-generation tensor cores (tcgen05).
//
// One CTA owns one (batch row, head) chain and walks its chunks of C = 64 tokens
// in order, with the state S (d_v x d_k, fp32) resident in tensor memory.  Every
// input element is read from HBM once and o is written once; the ShortConv
// prologue (anchor, residual chain, residual-write vectors rho) runs inside the
// same kernel.  Sources: ICML 2026 PRISM write-up (核心迭代形式, 消除 Token 间串行,
// 消除 Step 间串行, 架构形式) and the PRISM technical summary (2.1, 2.2), which fix
// the recurrence; its chunkwise form below is derived from that recurrence.
//
// Chunk algebra (token-local indices t, i in [0, 64); S_n = state before the chunk;
// G_t = sum_{j<=t} log gamma_j; D[t,i] = exp(G_t - G_i); c_i = exp(G_63 - G_i);
// rho_{i,l} = alpha_{i,l} r_{i,l}; P stacks rho (rows (i,l)), U stacks u):
//   A   [t,i]     = beta_t D[t,i] k_t.k_i            (i < t)
//   Bku [t,(i,l)] = beta_t D[t,i] k_t.u_{i,l}        (i < t)
//   QK  [t,i]     = D[t,i] q_t.k_i,  QU[t,(i,l)] = D[t,i] q_t.u_{i,l}   (i <= t)
//   T   = (I + A)^{-1}
//   X   = diag(beta) V - Bku P - diag(beta e^G) K S_n^T
//   Delta = T X        (the delta-rule corrections delta_t = beta_t (v_t - gamma_t S_{t-1} k_t))
//   O   = diag(e^G) Q S_n^T + QU P + (QK T) X
//   S_{n+1} = e^{G_63} S_n + Delta^T diag(c) K + P^T diag(c) U
//
// Tensor-core products (bf16 operands, fp32 accumulators in TMEM, M = 128):
//   MMA1  [K;Q] x [K;U]^T          -> R1   (token rows; N = 64 + 64m)
//   MMA3  S_n  x [K;Q]^T           -> D3   (state rows c; N = 128)
//   MMAQT [T;QK] x T               -> R1+128 (rows 64..127 = QK T)
//   MMA2  P^T x [Bku;QU]^T         -> R1   ((Bku P)^T | (QU P)^T)
//   MMA4  X^T x [T;QKT]^T          -> R1+128 (Delta^T | (QKT X)^T)
//   MMA5  (diag(c)P)^T U + (diag(c)Delta)^T K  accumulated onto e^{G_63} S_n in RS
// CUDA cores do the ShortConv prologue, the decay/mask epilogues and the 64x64
// unit-lower-triangular inverse T (blocked forward substitution in fp32).
//
// Smem operands use the 128-byte swizzle; K, Q and U arrive by TMA (zero fill past
// T), everything else is written by the CTA's threads.  Every mbarrier wait is
// bounded; on a timeout the CTA records PRISM_ERR_TIMEOUT, drains its own
// in-flight copies and MMAs, frees TMEM and exits.
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "sm100.cuh"

namespace prism {
namespace {

using namespace sm100;

constexpr int kC = 64;           // chunk length
constexpr int kThreads = 256;    // 8 warps: warp w reads TMEM lanes 32*(w%4).., column half w/4
constexpr uint32_t kAtom = 16384;  // one 128-row, 128-byte-wide swizzle atom column
constexpr long long kDrainLimit = 1ll << 26;

template <int D, int M>
struct Layout {
  static constexpr int NA = D / 64;            // atom columns along d
  static constexpr int UR = 64 * M;            // rows (i,l) of U / P per chunk
  static constexpr uint32_t U_ATOM = UR * 128;  // atom stride of U / P / P~
  static constexpr uint32_t OFF_KQ = 0;
  static constexpr uint32_t SZ_KQ = NA * kAtom;
  static constexpr uint32_t OFF_U = OFF_KQ + SZ_KQ;
  static constexpr uint32_t SZ_U = NA * U_ATOM;
  static constexpr uint32_t OFF_P = OFF_U + SZ_U;
  static constexpr uint32_t SZ_P = NA * U_ATOM;
  static constexpr uint32_t OFF_BQ = OFF_P + SZ_P;
  static constexpr uint32_t SZ_BQ = M * kAtom;  // [Bku;QU] (128 x 64m), later P~ (64m x D)
  static constexpr uint32_t OFF_TQ = OFF_BQ + SZ_BQ;
  static constexpr uint32_t OFF_SXA = OFF_TQ + kAtom;  // S bf16 | A,T fp32 | X^T, Delta~^T
  static constexpr uint32_t OFF_SMALL = OFF_SXA + 2 * kAtom;
  static constexpr uint32_t BYTES = OFF_SMALL + 1024;
  // + alignment slack; never below 116 KB so that one CTA (and one 512-column TMEM
  // allocation) is resident per SM
  static constexpr uint32_t SMEM_ALLOC = (BYTES + 1024 > 116u * 1024u) ? BYTES + 1024 : 116u * 1024u;
  static_assert(SMEM_ALLOC <= 232448, "exceeds the 227 KB opt-in shared memory of sm_100");
  static constexpr int LDA = 68;  // fp32 row stride of A / T in the SXA region
  static_assert(SZ_BQ >= SZ_P, "P~ must fit where [Bku;QU] was");
  static_assert(64 * LDA * 4 + 3 * 256 * 4 <= 2 * kAtom, "A/T + Y scratch must fit in SXA");
};

struct TcArgs {
  const __nv_bfloat16* v;
  const float* gamma;
  const float* beta;
  const float* alpha;
  const __nv_bfloat16* gain;
  const float* conv_w;
  const float* S0;
  const int32_t* lengths;
  __nv_bfloat16* o;
  float* S_final;
  int B, T, H, W;
  int* status;
  long long spin_limit;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// 8 consecutive fp32 values -> one 16-byte store of bf16 at smem byte address `addr`.
__device__ __forceinline__ void st_bf16x8(uint8_t* base, uint32_t off, const float* x) {
  uint4 u;
  u.x = pack_bf16x2(x[0], x[1]);
  u.y = pack_bf16x2(x[2], x[3]);
  u.z = pack_bf16x2(x[4], x[5]);
  u.w = pack_bf16x2(x[6], x[7]);
  *reinterpret_cast<uint4*>(base + off) = u;
}

__device__ __forceinline__ void ld_bf16x8(const __nv_bfloat16* p, float* x) {
  uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    float2 f = __bfloat1622float2(h[e]);
    x[2 * e] = f.x;
    x[2 * e + 1] = f.y;
  }
}

// Warp-uniform bounded wait (lane 0 polls, the result is broadcast).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, long long limit, int* status) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, limit, status);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

__device__ __forceinline__ uint64_t kdesc(uint32_t base, int kk, uint32_t atom_stride) {
  return sdesc_sw128(base + (uint32_t)(kk >> 2) * atom_stride + (uint32_t)(kk & 3) * 32u, 16, 1024);
}
__device__ __forceinline__ uint64_t mndesc(uint32_t base, int kk, uint32_t lbo) {
  return sdesc_sw128(base + (uint32_t)kk * 2048u, lbo, 1024);
}

template <int D, int M>
__global__ void __launch_bounds__(kThreads, 1)
    prism_chunk_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                          const __grid_constant__ CUtensorMap map_u, TcArgs p) {
  using Ly = Layout<D, M>;
  constexpr int NA = Ly::NA, UR = Ly::UR, LDA = Ly::LDA;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sKQ = sm + Ly::OFF_KQ;
  uint8_t* sU = sm + Ly::OFF_U;
  uint8_t* sP = sm + Ly::OFF_P;
  uint8_t* sBQ = sm + Ly::OFF_BQ;
  uint8_t* sTQ = sm + Ly::OFF_TQ;
  uint8_t* sSXA = sm + Ly::OFF_SXA;
  float* sG = reinterpret_cast<float*>(sm + Ly::OFF_SMALL);  // [64] cumulative log decay
  float* sBeta = sG + 64;                                     // [64]
  float* sCdec = sG + 128;                                    // [64] exp(G_63 - G_i)
  uint64_t* bar_load = reinterpret_cast<uint64_t*>(sm + Ly::OFF_SMALL + 768);
  uint64_t* bar_mma = bar_load + 1;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bar_load + 2);
  int* s_abort = reinterpret_cast<int*>(bar_load + 3);
  float* sA = reinterpret_cast<float*>(sSXA);          // [64][LDA] fp32: A, then T in place
  float* sY = sA + 64 * LDA;                           // [3][16][16] fp32 scratch of the inverse
  uint8_t* sX = sSXA;                                  // X^T      bf16 [128][64] K-major
  uint8_t* sDl = sSXA + kAtom;                         // Delta~^T bf16 [128][64] K-major

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q4 = warp & 3, hf = warp >> 2;
  const int row = 32 * q4 + lane;  // TMEM lane of this thread
  const int bh = blockIdx.x, b = bh / p.H, h = bh % p.H;
  const int T = p.T, H = p.H;
  const int len = p.lengths ? min(max(p.lengths[b], 0), T) : T;
  const int nchunks = (len + kC - 1) / kC;
  const long long lim = p.spin_limit;

  if (tid == 0) {
    mbar_init(bar_load, 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
    *s_abort = 0;
    tma_prefetch_desc(&map_q);
    tma_prefetch_desc(&map_k);
    if (M > 0) tma_prefetch_desc(&map_u);
  }
  if (warp == 0) {
    tmem_alloc(s_tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const uint32_t tl = tmem + ((uint32_t)(32 * q4) << 16);  // this warp's lane base
  constexpr uint32_t R1 = 0, D3 = 256, RS = 384;

  const uint32_t aKQ = smem_u32(sKQ), aU = smem_u32(sU), aP = smem_u32(sP), aBQ = smem_u32(sBQ);
  const uint32_t aTQ = smem_u32(sTQ), aS = smem_u32(sSXA), aX = smem_u32(sX), aDl = smem_u32(sDl);
  constexpr uint32_t kLoadBytes = 2 * NA * 8192 + NA * UR * 128;
  uint32_t ph_load = 0, ph_mma = 0;
  // (thread 0) phase of a TMA batch / MMA commit that is in flight and not yet observed, or -1
  int load_inflight = -1, mma_inflight = -1;

  auto issue_loads = [&](int t0) {
    mbar_arrive_expect_tx(bar_load, kLoadBytes);
#pragma unroll
    for (int a = 0; a < NA; ++a) {
      tma_load_4d(sKQ + a * kAtom, &map_k, bar_load, 64 * a, h, t0, b);
      tma_load_4d(sKQ + a * kAtom + 8192, &map_q, bar_load, 64 * a, h, t0, b);
      if (M > 0) tma_load_5d(sU + a * Ly::U_ATOM, &map_u, bar_load, 64 * a, 0, h, t0, b);
    }
  };

  // ---- initial state: RS <- S0 (or 0), bf16 copy -> SXA (A operand of MMA3)
  const bool lane_ok = row < D;  // state rows c in [0, D)
  if (q4 < NA * 2) {             // warps that own real state rows (all for D=128, lanes < 64 for D=64)
#pragma unroll
    for (int cc = 0; cc < D / 64; ++cc) {
      const int j0 = hf * (D / 2) + 32 * cc;
      float s[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) s[e] = 0.f;
      if (p.S0 && lane_ok) {
        const float4* src = reinterpret_cast<const float4*>(p.S0 + (((size_t)b * H + h) * D + row) * D + j0);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float4 f = __ldg(src + e);
          s[4 * e] = f.x; s[4 * e + 1] = f.y; s[4 * e + 2] = f.z; s[4 * e + 3] = f.w;
        }
      }
      tmem_st32(tl + RS + j0, s);
#pragma unroll
      for (int e = 0; e < 4; ++e) st_bf16x8(sSXA, sw128_offset(row, j0 + 8 * e, kAtom), s + 8 * e);
    }
  }
  if (tid == 0 && nchunks > 0) {
    issue_loads(0);
    load_inflight = (int)ph_load;
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();

  // ShortConv taps of the 8 channels this thread handles in the prologue
  constexpr int CPT = D / 8;           // threads per token in the prologue
  constexpr int TPP = kThreads / CPT;  // tokens per prologue pass
  const int pc8 = (tid % CPT) * 8;
  float cw[4][8];
#pragma unroll
  for (int w = 0; w < 4; ++w)
#pragma unroll
    for (int e = 0; e < 8; ++e) cw[w][e] = (w < p.W) ? __ldg(p.conv_w + ((size_t)h * D + pc8 + e) * p.W + w) : 0.f;

  bool aborted = false;
  for (int n = 0; n < nchunks && !aborted; ++n) {
    const int t0 = n * kC;
    const int nv = min(kC, len - t0);

    // ---------------- A: wait for K,Q,U; MMA1 + MMA3; prologue; decay prefix
    bool ok = warp_wait(bar_load, ph_load, lim, p.status);
    if (tid == 0) {
      if (ok) load_inflight = -1;
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4 * NA; ++kk) {
          const uint64_t a = kdesc(aKQ, kk, kAtom);
          mma_bf16(tmem + R1, a, a, idesc_bf16(128, 64, 0, 0), kk > 0);
          if (M > 0) mma_bf16(tmem + R1 + 64, a, kdesc(aU, kk, Ly::U_ATOM), idesc_bf16(128, UR, 0, 0), kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < 4 * NA; ++kk)
          mma_bf16(tmem + D3, kdesc(aS, kk, kAtom), kdesc(aKQ, kk, kAtom), idesc_bf16(128, 128, 0, 0), kk > 0);
        mma_commit(bar_mma);
        mma_inflight = (int)ph_mma;
      }
    }
    ph_load ^= 1;
    if (!ok && lane == 0) atomicExch(s_abort, 1);
    // in-chunk cumulative log decay and step sizes (padded steps: gamma = 1, beta = 0)
    if (tid < 64) {
      const bool valid = tid < nv;
      const size_t th = ((size_t)b * T + t0 + tid) * H + h;
      const float g = valid ? __logf(__ldg(p.gamma + th)) : 0.f;
      float x = g;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
      }
      sG[tid] = x;
      sBeta[tid] = valid ? __ldg(p.beta + th) : 0.f;
    }
    // prologue: rho_{i,l} = alpha_{i,l} prod_{j<=l}(1 - g_j) (v_i - sum_w cw_w v_{i-w}) -> P (bf16)
    if (M > 0) {
#pragma unroll 1
      for (int pass = 0; pass < kC / TPP; ++pass) {
        const int i = pass * TPP + tid / CPT;
        const int t = t0 + i;
        if (i < nv) {
          float vv[8], r[8];
          const size_t th = ((size_t)b * T + t) * H + h;
          ld_bf16x8(p.v + th * D + pc8, vv);
#pragma unroll
          for (int e = 0; e < 8; ++e) r[e] = vv[e] - cw[0][e] * vv[e];
#pragma unroll
          for (int w = 1; w < 4; ++w) {
            if (w < p.W && t - w >= 0) {
              float hv[8];
              ld_bf16x8(p.v + (th - (size_t)w * H) * D + pc8, hv);
#pragma unroll
              for (int e = 0; e < 8; ++e) r[e] -= cw[w][e] * hv[e];
            }
          }
#pragma unroll
          for (int l = 0; l < M; ++l) {
            float gg[8], rho[8];
            ld_bf16x8(p.gain + (th * M + l) * D + pc8, gg);
            const float al = __ldg(p.alpha + th * M + l);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              r[e] *= 1.f - gg[e];
              rho[e] = al * r[e];
            }
            st_bf16x8(sP, sw128_offset(i * M + l, pc8, Ly::U_ATOM), rho);
          }
        } else {
          float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int l = 0; l < M; ++l) st_bf16x8(sP, sw128_offset(i * M + l, pc8, Ly::U_ATOM), z);
        }
      }
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid >= 32 && tid < 64) sG[tid] += sG[31];  // combine the two warp scans
    __syncthreads();
    if (*s_abort) { aborted = true; break; }

    // ---------------- B: epilogue of MMA1 -> A (fp32), [Bku;QU], QK (bf16)
    ok = warp_wait(bar_mma, ph_mma, lim, p.status);
    ph_mma ^= 1;
    if (tid == 0 && ok) mma_inflight = -1;
    if (!ok && lane == 0) atomicExch(s_abort, 1);
    tc_fence_after();
    if (tid < 64) sCdec[tid] = __expf(sG[63] - sG[tid]);
    if (ok) {
      const bool krow = row < 64;
      const int t = krow ? row : row - 64;
      const float Gt = sG[t];
      const float bt = krow ? sBeta[t] : 1.f;
      constexpr int NCH = (64 + UR) / 32;  // 32-column pieces of R1
#pragma unroll 1
      for (int ch = hf * (NCH / 2); ch < (hf + 1) * (NCH / 2); ++ch) {
        const int j0 = 32 * ch;
        float x[32];
        tmem_ld32(tl + R1 + j0, x);
        if (j0 < 64) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int i = j0 + e;
            const bool keep = krow ? (i < t) : (i <= t);
            x[e] = keep ? bt * __expf(Gt - sG[i]) * x[e] : 0.f;
          }
          if (krow) {
            float4* dst = reinterpret_cast<float4*>(sA + t * LDA + j0);
#pragma unroll
            for (int e = 0; e < 8; ++e) dst[e] = make_float4(x[4 * e], x[4 * e + 1], x[4 * e + 2], x[4 * e + 3]);
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) st_bf16x8(sTQ, sw128_offset(row, j0 + 8 * e, kAtom), x + 8 * e);
          }
        } else {
          const int k0 = j0 - 64;  // column (i,l) = k0 + e
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int i = (k0 + e) / (M > 0 ? M : 1);
            const bool keep = krow ? (i < t) : (i <= t);
            x[e] = keep ? bt * __expf(Gt - sG[i]) * x[e] : 0.f;
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) st_bf16x8(sBQ, sw128_offset(row, k0 + 8 * e, kAtom), x + 8 * e);
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (*s_abort) { aborted = true; break; }

    // ---------------- C: T = (I + A)^{-1} in place (fp32), blocked by 16
    {
      // diagonal 16x16 blocks: thread (blk, j) solves column j by forward substitution
      float xcol[16];
      const int blk = tid >> 4, j = tid & 15;
      if (tid < 64) {
#pragma unroll
        for (int r = 0; r < 16; ++r) {
          float acc = 0.f;
#pragma unroll
          for (int s = 0; s < r; ++s) acc += sA[(16 * blk + r) * LDA + 16 * blk + s] * xcol[s];
          xcol[r] = (r < j) ? 0.f : (r == j ? 1.f : -acc);
        }
      }
      __syncthreads();
      if (tid < 64) {
#pragma unroll
        for (int r = 0; r < 16; ++r) sA[(16 * blk + r) * LDA + 16 * blk + j] = xcol[r];
      }
      __syncthreads();
      // block rows I = 1..3: Y_IJ = sum_{K=J}^{I-1} A_IK T_KJ, then T_IJ = -T_II Y_IJ
#pragma unroll 1
      for (int I = 1; I < 4; ++I) {
        for (int e = tid; e < 256 * I; e += kThreads) {
          const int J = e >> 8, r = (e >> 4) & 15, s = e & 15;
          float acc = 0.f;
          for (int kx = 16 * J; kx < 16 * I; ++kx) acc += sA[(16 * I + r) * LDA + kx] * sA[kx * LDA + 16 * J + s];
          sY[e] = acc;
        }
        __syncthreads();
        for (int e = tid; e < 256 * I; e += kThreads) {
          const int J = e >> 8, r = (e >> 4) & 15, s = e & 15;
          float acc = 0.f;
          for (int u = 0; u <= r; ++u) acc += sA[(16 * I + r) * LDA + 16 * I + u] * sY[(J << 8) + (u << 4) + s];
          sA[(16 * I + r) * LDA + 16 * J + s] = -acc;
        }
        __syncthreads();
      }
      // T (fp32, lower incl. unit diagonal; upper part holds A's zeros) -> bf16 rows 0..63 of TQ
      for (int e = tid; e < 64 * 8; e += kThreads) {
        const int t = e >> 3, c8 = (e & 7) * 8;
        const float4 lo = *reinterpret_cast<const float4*>(sA + t * LDA + c8);
        const float4 hi = *reinterpret_cast<const float4*>(sA + t * LDA + c8 + 4);
        const float v8[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
        st_bf16x8(sTQ, sw128_offset(t, c8, kAtom), v8);
      }
    }
    fence_proxy_async_smem();
    __syncthreads();

    // ---------------- D: MMA QK*T and MMA2; rescale RS by exp(G_63)
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem + R1 + 128, kdesc(aTQ, kk, kAtom), mndesc(aTQ, kk, kAtom), idesc_bf16(128, 64, 0, 1), kk > 0);
      if (M > 0) {
#pragma unroll
        for (int kk = 0; kk < UR / 16; ++kk)
          mma_bf16(tmem + R1, mndesc(aP, kk, Ly::U_ATOM), kdesc(aBQ, kk, kAtom), idesc_bf16(128, 128, 1, 0), kk > 0);
      }
      mma_commit(bar_mma);
      mma_inflight = (int)ph_mma;
    }
    const float blast = __expf(sG[63]);
    if (q4 < NA * 2) {
#pragma unroll
      for (int cc = 0; cc < D / 64; ++cc) {
        const int j0 = hf * (D / 2) + 32 * cc;
        float s[32];
        tmem_ld32(tl + RS + j0, s);
#pragma unroll
        for (int e = 0; e < 32; ++e) s[e] *= blast;
        tmem_st32(tl + RS + j0, s);
      }
    }

    // ---------------- E: QKT -> TQ rows 64..127; P~ = diag(c) P -> BQ; X^T -> SXA; O partial
    ok = warp_wait(bar_mma, ph_mma, lim, p.status);
    ph_mma ^= 1;
    if (tid == 0 && ok) mma_inflight = -1;
    if (!ok && lane == 0) atomicExch(s_abort, 1);
    tc_fence_after();
    float opart[32];
    if (ok) {
      if (q4 >= 2) {  // lanes 64..127 hold (QK T)[t, i], t = row - 64; column half hf
        float x[32];
        tmem_ld32(tl + R1 + 128 + 32 * hf, x);
#pragma unroll
        for (int e = 0; e < 4; ++e) st_bf16x8(sTQ, sw128_offset(row, 32 * hf + 8 * e, kAtom), x + 8 * e);
      }
      if (M > 0) {
        for (int e = tid; e < UR * D / 8; e += kThreads) {
          const int r = e / (D / 8), c8 = (e % (D / 8)) * 8;
          const uint32_t off = sw128_offset(r, c8, Ly::U_ATOM);
          const float sc = sCdec[r / (M > 0 ? M : 1)];
          uint4 u = *reinterpret_cast<const uint4*>(sP + off);
          __nv_bfloat162* hx = reinterpret_cast<__nv_bfloat162*>(&u);
          float f[8];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            float2 ff = __bfloat1622float2(hx[k]);
            f[2 * k] = sc * ff.x;
            f[2 * k + 1] = sc * ff.y;
          }
          st_bf16x8(sBQ, off, f);
        }
      }
      if (q4 < NA * 2) {  // state rows c = row; tokens t = 32*hf + e
        const int tb = 32 * hf;
        float y[32], d2[32];
        tmem_ld32(tl + D3 + tb, y);
        if (M > 0) tmem_ld32(tl + R1 + tb, d2);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int t = tb + e;
          const float bet = sBeta[t];
          const float vtc = (t < nv) ? __bfloat162float(p.v[(((size_t)b * T + t0 + t) * H + h) * D + row]) : 0.f;
          float xv = bet * (vtc - __expf(sG[t]) * y[e]);
          if (M > 0) xv -= d2[e];
          y[e] = xv;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) st_bf16x8(sX, sw128_offset(row, tb + 8 * e, kAtom), y + 8 * e);
        tmem_ld32(tl + D3 + 64 + tb, opart);
        if (M > 0) tmem_ld32(tl + R1 + 64 + tb, d2);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          opart[e] *= __expf(sG[tb + e]);
          if (M > 0) opart[e] += d2[e];
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (*s_abort) { aborted = true; break; }

    // ---------------- F: MMA4 (Delta^T | (QKT X)^T) and MMA5a (RS += P~^T U)
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem + R1 + 128, kdesc(aX, kk, kAtom), kdesc(aTQ, kk, kAtom), idesc_bf16(128, 128, 0, 0), kk > 0);
      if (M > 0) {
#pragma unroll
        for (int kk = 0; kk < UR / 16; ++kk)
          mma_bf16(tmem + RS, mndesc(aBQ, kk, Ly::U_ATOM), mndesc(aU, kk, Ly::U_ATOM), idesc_bf16(128, D, 1, 1), 1);
      }
      mma_commit(bar_mma);
      mma_inflight = (int)ph_mma;
    }

    // ---------------- G: Delta~^T -> SXA; o = O partial + (QKT X)
    ok = warp_wait(bar_mma, ph_mma, lim, p.status);
    ph_mma ^= 1;
    if (tid == 0 && ok) mma_inflight = -1;
    if (!ok && lane == 0) atomicExch(s_abort, 1);
    tc_fence_after();
    if (ok && q4 < NA * 2) {
      const int tb = 32 * hf;
      float x[32];
      tmem_ld32(tl + R1 + 128 + tb, x);
#pragma unroll
      for (int e = 0; e < 32; ++e) x[e] *= sCdec[tb + e];
#pragma unroll
      for (int e = 0; e < 4; ++e) st_bf16x8(sDl, sw128_offset(row, tb + 8 * e, kAtom), x + 8 * e);
      tmem_ld32(tl + R1 + 192 + tb, x);
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int t = t0 + tb + e;
        if (t < T) p.o[(((size_t)b * T + t) * H + h) * D + row] = __float2bfloat16_rn(tb + e < nv ? opart[e] + x[e] : 0.f);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (*s_abort) { aborted = true; break; }

    // ---------------- H: MMA5b (RS += Delta~^T K)
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem + RS, kdesc(aDl, kk, kAtom), mndesc(aKQ, kk, kAtom), idesc_bf16(128, D, 0, 1), 1);
      mma_commit(bar_mma);
      mma_inflight = (int)ph_mma;
    }

    // ---------------- I: next chunk's loads; S_{n+1} -> bf16 SXA (and S_final)
    ok = warp_wait(bar_mma, ph_mma, lim, p.status);
    ph_mma ^= 1;
    if (tid == 0) {
      if (ok) mma_inflight = -1;
      if (ok && n + 1 < nchunks) {
        issue_loads(t0 + kC);
        load_inflight = (int)ph_load;
      }
    }
    if (!ok && lane == 0) atomicExch(s_abort, 1);
    tc_fence_after();
    if (ok && q4 < NA * 2) {
      const bool last = n + 1 == nchunks;
#pragma unroll
      for (int cc = 0; cc < D / 64; ++cc) {
        const int j0 = hf * (D / 2) + 32 * cc;
        float s[32];
        tmem_ld32(tl + RS + j0, s);
#pragma unroll
        for (int e = 0; e < 4; ++e) st_bf16x8(sSXA, sw128_offset(row, j0 + 8 * e, kAtom), s + 8 * e);
        if (last && p.S_final) {
          float4* dst = reinterpret_cast<float4*>(p.S_final + (((size_t)b * H + h) * D + row) * D + j0);
#pragma unroll
          for (int e = 0; e < 8; ++e) dst[e] = make_float4(s[4 * e], s[4 * e + 1], s[4 * e + 2], s[4 * e + 3]);
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (*s_abort) { aborted = true; break; }
  }

  if (!aborted) {
    // rows with no valid token: S_final = S0 (still in RS); zero the outputs past the last chunk
    if (nchunks == 0 && p.S_final && q4 < NA * 2) {
#pragma unroll
      for (int cc = 0; cc < D / 64; ++cc) {
        const int j0 = hf * (D / 2) + 32 * cc;
        float s[32];
        tmem_ld32(tl + RS + j0, s);
        float4* dst = reinterpret_cast<float4*>(p.S_final + (((size_t)b * H + h) * D + row) * D + j0);
#pragma unroll
        for (int e = 0; e < 8; ++e) dst[e] = make_float4(s[4 * e], s[4 * e + 1], s[4 * e + 2], s[4 * e + 3]);
      }
    }
    const int tz = nchunks * kC;
    const __nv_bfloat16 zero = __float2bfloat16_rn(0.f);
    for (size_t e = tid; e < (size_t)max(T - tz, 0) * D; e += kThreads) {
      const int t = tz + (int)(e / D), c = (int)(e % D);
      p.o[(((size_t)b * T + t) * H + h) * D + c] = zero;
    }
  } else if (tid == 0) {
    // drain this CTA's own copies and MMAs before giving the memory back
    if (load_inflight >= 0) mbar_wait(bar_load, (uint32_t)load_inflight, kDrainLimit, p.status);
    if (mma_inflight >= 0) mbar_wait(bar_mma, (uint32_t)mma_inflight, kDrainLimit, p.status);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

bool encode(CUtensorMap* map, const void* ptr, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
            const cuuint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int M>
cudaError_t launch_dm(const ScanParams& p, cudaStream_t stream) {
  using Ly = Layout<D, M>;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(prism_chunk_tc_kernel<D, M>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    Ly::SMEM_ALLOC);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const cuuint64_t B = p.B, T = p.T, H = p.H;
  CUtensorMap mq, mk, mu;
  const cuuint64_t dims4[4] = {(cuuint64_t)D, H, T, B};
  const cuuint64_t str4[3] = {(cuuint64_t)D * 2, H * D * 2, T * H * D * 2};
  const cuuint32_t box4[4] = {64, 1, 64, 1};
  if (!encode(&mq, p.q, 4, dims4, str4, box4) || !encode(&mk, p.k, 4, dims4, str4, box4))
    return cudaErrorInvalidValue;
  if (M > 0) {
    const cuuint64_t dims5[5] = {(cuuint64_t)D, (cuuint64_t)M, H, T, B};
    const cuuint64_t str5[4] = {(cuuint64_t)D * 2, (cuuint64_t)M * D * 2, H * M * D * 2, T * H * M * D * 2};
    const cuuint32_t box5[5] = {64, (cuuint32_t)M, 1, 64, 1};
    if (!encode(&mu, p.u, 5, dims5, str5, box5)) return cudaErrorInvalidValue;
  } else {
    mu = mk;
  }
  TcArgs a{static_cast<const __nv_bfloat16*>(p.v), p.gamma, p.beta, p.alpha,
           static_cast<const __nv_bfloat16*>(p.gain), p.conv_w, p.S0, p.lengths,
           static_cast<__nv_bfloat16*>(p.o), p.S_final, p.B, p.T, p.H, p.W, p.status, p.spin_limit};
  prism_chunk_tc_kernel<D, M><<<p.B * p.H, kThreads, Ly::SMEM_ALLOC, stream>>>(mq, mk, mu, a);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const ScanParams& p, cudaStream_t stream) {
  switch (p.L - 1) {
    case 0: return launch_dm<D, 0>(p, stream);
    case 1: return launch_dm<D, 1>(p, stream);
    case 2: return launch_dm<D, 2>(p, stream);
    case 3: return launch_dm<D, 3>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

bool chunk_tc_supported(int d_k, int d_v, int L, int W, int chunk, int dtype) {
  return dtype == PRISM_BF16 && chunk == kC && d_k == d_v && (d_k == 64 || d_k == 128) && L >= 1 && L <= 4 &&
         W >= 1 && W <= 4;
}

cudaError_t launch_chunk_tc(const ScanParams& p, cudaStream_t stream) {
  if (p.d_k == 128) return launch_d<128>(p, stream);
  if (p.d_k == 64) return launch_d<64>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace prism
