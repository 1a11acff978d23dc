// Chunkwise-parallel PRISM scan on the 5th-generation tensor cores (tcgen05).
//
// One CTA owns one (batch row, head) chain and walks its chunks of C = 64 tokens
// in order, with the state S (d_v x d_k, fp32) resident in tensor memory.  Every
// input element is read from HBM once and o is written once; the ShortConv
// prologue (anchor, residual chain, residual-write vectors rho) runs inside the
// scan kernel.  Sources: ICML 2026 PRISM write-up (核心迭代形式, 消除 Token 间串行,
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
// Two launches per call.  The preparation kernel (one CTA per (b, h, chunk), all chunks
// at once) computes T = (I + A)^{-1} of every chunk: A from K K^T on the tensor cores,
// the inverse by blocked forward substitution in fp32 on CUDA cores, stored as bf16 in
// the workspace.  The scan kernel then walks the chunks of each chain in order and
// TMA-loads each chunk's T next to its K, Q and U tiles.
//
// Tensor-core products of the scan kernel (bf16 operands, fp32 accumulators in TMEM,
// M = 128):
//   MMA1  [K;Q] x [K;U]^T          -> R1   (token rows; N = 64 + 64m; only QK, Bku, QU used)
//   MMA3  S_n  x [K;Q]^T           -> D3   (state rows c; N = 128)
//   MMAQT [T;QK] x T               -> R1+128 (rows 64..127 = QK T)
//   MMA2  P^T x [Bku;QU]^T         -> R1   ((Bku P)^T | (QU P)^T)
//   MMA4  X^T x [T;QKT]^T          -> R1+128 (Delta^T | (QKT X)^T)
//   MMA5  (diag(c)P)^T U + (diag(c)Delta)^T K  accumulated onto e^{G_63} S_n in RS
// CUDA cores do the ShortConv prologue of the next chunk and the decay/mask epilogues.
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
constexpr int kThreads = 512;    // 16 warps: warp w reads TMEM lanes 32*(w%4).., column quarter w/4
constexpr uint32_t kAtom = 16384;  // one 128-row, 128-byte-wide swizzle atom column
constexpr long long kDrainLimit = 1ll << 18;  // polls of up to 20 us each

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
  // [Bku;QU] (128 x 64m); between MMA2 and the next epilogue, the next prologue's v tile
  // (NA atom columns of 72 rows, 9 KB apart) and the ShortConv taps
  static constexpr uint32_t SZ_VT = NA * 9216u + D * 16u;  // v tile + ShortConv taps (W <= 4)
  static constexpr uint32_t SZ_BQ = M == 0 ? 0u : (M * kAtom > SZ_VT ? M * kAtom : SZ_VT);
  static constexpr uint32_t OFF_TQ = OFF_BQ + SZ_BQ;
  static constexpr uint32_t OFF_SXA = OFF_TQ + kAtom;  // S bf16 | X^T, Delta~^T
  static constexpr uint32_t OFF_SMALL = OFF_SXA + 2 * kAtom;  // gate tables, barriers
  static constexpr uint32_t BYTES = OFF_SMALL + 2048;
  // + alignment slack; never below 116 KB so that one CTA (and one 512-column TMEM
  // allocation) is resident per SM
  static constexpr uint32_t SMEM_ALLOC = (BYTES + 1024 > 116u * 1024u) ? BYTES + 1024 : 116u * 1024u;
  static_assert(SMEM_ALLOC <= 232448, "exceeds the 227 KB opt-in shared memory of sm_100");
};

struct TcArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* u;
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
  int B, T, H, W, NC;
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

// element e (0..7) of 8 packed bf16
__device__ __forceinline__ float bf16_at(const uint4& u, int e) {
  const uint32_t w = e < 2 ? u.x : e < 4 ? u.y : e < 6 ? u.z : u.w;
  return __uint_as_float((e & 1) ? (w & 0xffff0000u) : (w << 16));
}

// Warp-uniform bounded wait (lane 0 polls, the result is broadcast).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, long long limit, int* status) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, limit, status);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// The scan kernel's CTA: kThreads worker threads (16 warps) and one MMA warp that issues
// every tcgen05.mma.  A tcgen05.mma sequence holds its issuing thread for about its
// execution time; in a warp of its own that no longer stalls the workers, who meet on
// barrier 1 and hand operands over through mbarriers.
constexpr int kMmaWarp = kThreads / 32;
constexpr int kCtaThreads = kThreads + 32;

__device__ __forceinline__ void worker_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kThreads) : "memory"); }
// Barrier 1 with an OR over the workers' votes: every worker gets the same answer.
__device__ __forceinline__ bool worker_sync_or(int v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred q, p;\n\t"
      "setp.ne.s32 q, %1, 0;\n\t"
      "bar.red.or.pred p, 1, %2, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(v), "n"(kThreads)
      : "memory");
  return r != 0;
}

// Bounded, warp-uniform wait of the MMA warp; also gives up once the abort flag is set.
__device__ __forceinline__ bool mma_warp_wait(uint64_t* bar, uint32_t parity, long long limit, int* status,
                                              const volatile int* abort_flag) {
  bool ok = false;
  if ((threadIdx.x & 31) == 0) {
    const uint32_t hint = limit < 1024 ? 0u : 20000u;
    for (long long i = 0; i < limit && !ok; ++i) {
      if (mbar_try_wait_suspend(bar, parity, hint)) ok = true;
      else if (*abort_flag) break;
    }
    if (!ok && !*abort_flag) record_status(status, PRISM_ERR_TIMEOUT);
  }
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

__device__ __forceinline__ uint64_t kdesc(uint32_t base, int kk, uint32_t atom_stride) {
  return sdesc_sw128(base + (uint32_t)(kk >> 2) * atom_stride + (uint32_t)(kk & 3) * 32u, 16, 1024);
}
__device__ __forceinline__ uint64_t mndesc(uint32_t base, int kk, uint32_t lbo) {
  return sdesc_sw128(base + (uint32_t)kk * 2048u, lbo, 1024);
}

// T = (I + A)^{-1} in place, for a strictly lower-triangular 64 x 64 fp32 A in sA (row
// stride LDA, zeros on and above the diagonal), by blocked forward substitution: the four
// 16 x 16 diagonal blocks column by column, then the 16 -> 32 and 32 -> 64 merges
// T_21 = -T_22 A_21 T_11.  All kPrepThreads (128) threads call it (it synchronises
// internally); on return sA holds T (unit lower triangular, zeros above).  sY: 1024 fp32.
constexpr int kPrepThreads = 128;

template <int LDA>
__device__ __forceinline__ void invert_unit_lower64(float* sA, float* sY, int tid) {
  // (1) diagonal blocks: thread (blk, j) solves column j of block blk
  {
    float xcol[16];
    const int blk = tid >> 4, j = tid & 15;
    if (tid < 64) {
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        float acc = 0.f;
#pragma unroll
        for (int s2 = 0; s2 < r; ++s2) acc += sA[(16 * blk + r) * LDA + 16 * blk + s2] * xcol[s2];
        xcol[r] = (r < j) ? 0.f : (r == j ? 1.f : -acc);
      }
    }
    __syncthreads();
    if (tid < 64) {
#pragma unroll
      for (int r = 0; r < 16; ++r) sA[(16 * blk + r) * LDA + 16 * blk + j] = xcol[r];
    }
    __syncthreads();
  }
  // (2) 16 -> 32: T_{I,I-1} = -T_II (A_{I,I-1} T_{I-1,I-1}) for I = 1, 3.  Thread: one row r
  // of one of the two blocks, four consecutive columns.
  {
    const int pr = tid >> 6, r = (tid >> 2) & 15, c0 = (tid & 3) * 4;
    const int I = 2 * pr + 1, J = 2 * pr;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const float a = sA[(16 * I + r) * LDA + 16 * J + u];
      const float4 t = *reinterpret_cast<const float4*>(sA + (16 * J + u) * LDA + 16 * J + c0);
      acc[0] += a * t.x;
      acc[1] += a * t.y;
      acc[2] += a * t.z;
      acc[3] += a * t.w;
    }
    *reinterpret_cast<float4*>(sY + pr * 256 + r * 16 + c0) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    __syncthreads();
    acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      if (u <= r) {
        const float a = sA[(16 * I + r) * LDA + 16 * I + u];
        const float4 y = *reinterpret_cast<const float4*>(sY + pr * 256 + u * 16 + c0);
        acc[0] += a * y.x;
        acc[1] += a * y.y;
        acc[2] += a * y.z;
        acc[3] += a * y.w;
      }
    }
    *reinterpret_cast<float4*>(sA + (16 * I + r) * LDA + 16 * J + c0) =
        make_float4(-acc[0], -acc[1], -acc[2], -acc[3]);
    __syncthreads();
  }
  // (3) 32 -> 64: T[32:64, 0:32] = -T2 (A21 T1).  Thread: two rows, four consecutive columns.
  {
    const int r0 = (tid >> 3) * 2, c0 = (tid & 7) * 4;
    float acc[2][4] = {};
#pragma unroll 8
    for (int u = 0; u < 32; ++u) {  // Y2 = A21 T1
      const float4 t = *reinterpret_cast<const float4*>(sA + u * LDA + c0);
#pragma unroll
      for (int i2 = 0; i2 < 2; ++i2) {
        const float a = sA[(32 + r0 + i2) * LDA + u];
        acc[i2][0] += a * t.x;
        acc[i2][1] += a * t.y;
        acc[i2][2] += a * t.z;
        acc[i2][3] += a * t.w;
      }
    }
#pragma unroll
    for (int i2 = 0; i2 < 2; ++i2)
      *reinterpret_cast<float4*>(sY + (r0 + i2) * 32 + c0) = make_float4(acc[i2][0], acc[i2][1], acc[i2][2], acc[i2][3]);
    __syncthreads();
#pragma unroll
    for (int i2 = 0; i2 < 2; ++i2) acc[i2][0] = acc[i2][1] = acc[i2][2] = acc[i2][3] = 0.f;
    const int ulim = r0 + 2;  // T2 is lower triangular: only u <= r0 + 1 contribute
#pragma unroll 8
    for (int u = 0; u < ulim; ++u) {  // T21 = -T2 Y2
      const float4 y = *reinterpret_cast<const float4*>(sY + u * 32 + c0);
#pragma unroll
      for (int i2 = 0; i2 < 2; ++i2) {
        const float a = sA[(32 + r0 + i2) * LDA + 32 + u];
        acc[i2][0] += a * y.x;
        acc[i2][1] += a * y.y;
        acc[i2][2] += a * y.z;
        acc[i2][3] += a * y.w;
      }
    }
    // rows 32..63, columns 0..31 held A21, which the first product has consumed
#pragma unroll
    for (int i2 = 0; i2 < 2; ++i2)
      *reinterpret_cast<float4*>(sA + (32 + r0 + i2) * LDA + c0) =
          make_float4(-acc[i2][0], -acc[i2][1], -acc[i2][2], -acc[i2][3]);
    __syncthreads();
  }
}

// ---------------------------------------------------------------- chunk preparation
// The part of every chunk that depends on neither the state nor the other chunks, done
// for all (b, h, chunk) at once before the scan: the in-chunk gate prefix G, the masked
// decayed Gram matrix A[t,i] = beta_t e^{G_t - G_i} k_t.k_i (i < t; K K^T on the tensor
// cores) and T = (I + A)^{-1}, stored as bf16 [B, H, NC, 64, 64] in the workspace.
// Taking the inverse off the scan's sequential chunk loop spreads it over every SM.
struct PrepArgs {
  const float* gamma;
  const float* beta;
  const int32_t* lengths;
  __nv_bfloat16* Tws;
  int T, H, NC;
  int* status;
  long long spin_limit;
};

constexpr int kPrepLDA = 68;  // fp32 row stride of A / T (bank-conflict padding)

constexpr uint32_t kPrepAtom = 8192;  // 64 rows x 128 bytes: one swizzle-atom column of K

template <int D>
struct PrepLayout {
  static constexpr int NA = D / 64;
  // K tile: NA atom columns of 64 rows, 8 KB apart.  The M = 128 MMA also reads the 64
  // rows that follow each one (the next atom column, or A below): those accumulator
  // lanes are never read.
  static constexpr uint32_t OFF_K = 0;
  static constexpr uint32_t OFF_A = NA * kPrepAtom;             // [64][kPrepLDA] fp32
  static constexpr uint32_t OFF_Y = OFF_A + 64 * kPrepLDA * 4;  // 1024 fp32 inverse scratch
  static constexpr uint32_t OFF_SMALL = OFF_Y + 4096;           // G, beta, e^{-G} [64] each; barriers
  static constexpr uint32_t BYTES = OFF_SMALL + 1024;
  static constexpr uint32_t SMEM_ALLOC = BYTES + 1024;  // + alignment slack
};

template <int D>
__global__ void __launch_bounds__(kPrepThreads) prism_chunk_prep_kernel(const __grid_constant__ CUtensorMap map_k,
                                                                       PrepArgs p) {
  using Ly = PrepLayout<D>;
  constexpr int NA = Ly::NA, LDA = kPrepLDA;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = sm + Ly::OFF_K;
  float* sA = reinterpret_cast<float*>(sm + Ly::OFF_A);
  float* sY = reinterpret_cast<float*>(sm + Ly::OFF_Y);
  float* sG = reinterpret_cast<float*>(sm + Ly::OFF_SMALL);
  float* sBeta = sG + 64;
  float* sEn = sG + 192;  // e^{-G_i} (chunks with log-decay >= -60)
  uint64_t* bar_load = reinterpret_cast<uint64_t*>(sm + Ly::OFF_SMALL + 512);
  uint64_t* bar_mma = bar_load + 1;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bar_load + 2);
  int* s_abort = reinterpret_cast<int*>(bar_load + 3);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = blockIdx.x % p.NC, bh = blockIdx.x / p.NC, b = bh / p.H, h = bh % p.H;
  const int len = p.lengths ? min(max(p.lengths[b], 0), p.T) : p.T;
  const int t0 = n * kC;
  if (t0 >= len) return;  // the scan never reaches this chunk (uniform over the CTA)
  const int nv = min(kC, len - t0);
  const long long lim = p.spin_limit;

  if (tid == 0) {  // the K tile is requested first: its latency overlaps the gate loads below
    mbar_init(bar_load, 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
    *s_abort = 0;
    mbar_arrive_expect_tx(bar_load, NA * 8192);
#pragma unroll
    for (int a = 0; a < NA; ++a) tma_load_4d(sK + a * kPrepAtom, &map_k, bar_load, 64 * a, h, t0, b);
  }
  if (warp == 0) {
    tmem_alloc(s_tmem, 64);
    tmem_relinquish();
  }
  if (warp == 2) {  // gate prefix; lane owns tokens 2 lane, 2 lane + 1; padded steps: gamma = 1, beta = 0
    float gl[2], bl[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int t = 2 * lane + e;
      const bool valid = t < nv;
      const size_t th = ((size_t)b * p.T + min(t0 + t, p.T - 1)) * p.H + h;
      gl[e] = valid ? __ldg(p.gamma + th) : 1.f;
      bl[e] = valid ? __ldg(p.beta + th) : 0.f;
    }
    const float lg0 = __logf(gl[0]), lg1 = __logf(gl[1]);
    float x = lg0 + lg1;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    sG[2 * lane] = x - lg1;
    sG[2 * lane + 1] = x;
    sBeta[2 * lane] = bl[0];
    sBeta[2 * lane + 1] = bl[1];
    if (__shfl_sync(0xffffffffu, x, 31) >= -60.f) {  // e^{-G} stays finite: factor the decays
      sEn[2 * lane] = __expf(lg1 - x);
      sEn[2 * lane + 1] = __expf(-x);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  bool mma_issued = false;
  if (tid == 0) {
    if (mbar_wait(bar_load, 0, lim, p.status)) {
      tc_fence_after();
      // K K^T with M = 128 (accumulator lanes 64..127 are not read)
      const uint32_t aK = smem_u32(sK);
#pragma unroll
      for (int kk = 0; kk < 4 * NA; ++kk)
        mma_bf16(tmem, kdesc(aK, kk, kPrepAtom), kdesc(aK, kk, kPrepAtom), idesc_bf16(128, 64, 0, 0), kk > 0);
      mma_commit(bar_mma);
      mma_issued = true;
    } else {
      *s_abort = 1;
    }
  }
  const bool load_failed = __syncthreads_or(*s_abort) != 0;  // uniform decision
  if (!load_failed && warp < 2) {  // TMEM lanes 0..63 = token rows t
    const bool ok = warp_wait(bar_mma, 0, lim, p.status);
    if (ok) {
      tc_fence_after();
      const int t = 32 * warp + lane;
      const float Gt = sG[t], bt = sBeta[t];
      const bool fast = sG[63] >= -60.f;  // as decided where sEn was written
      const float rs = fast ? bt * __expf(Gt) : 0.f;
      const uint32_t tl = tmem + ((uint32_t)(32 * warp) << 16);
#pragma unroll
      for (int pc = 0; pc < 4; ++pc) {
        float x[16];
        tmem_ld16(tl + 16 * pc, x);
        if (fast) {  // e^{G_t - G_i} = e^{G_t} e^{-G_i}
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int i = 16 * pc + e;
            x[e] = (i < t) ? rs * sEn[i] * x[e] : 0.f;
          }
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int i = 16 * pc + e;
            x[e] = (i < t) ? bt * __expf(Gt - sG[i]) * x[e] : 0.f;
          }
        }
        float4* dst = reinterpret_cast<float4*>(sA + t * LDA + 16 * pc);
#pragma unroll
        for (int e = 0; e < 4; ++e) dst[e] = make_float4(x[4 * e], x[4 * e + 1], x[4 * e + 2], x[4 * e + 3]);
      }
    } else if (lane == 0) {
      atomicExch(s_abort, 1);
    }
  }
  tc_fence_before();
  const bool failed = __syncthreads_or(*s_abort) != 0;  // uniform: the inverse synchronises internally
  if (!failed) {
    invert_unit_lower64<LDA>(sA, sY, tid);
#pragma unroll
    for (int q = 0; q < 4; ++q) {  // T -> bf16 rows of 128 bytes, 16 bytes per thread and pass
      const int e = q * kPrepThreads + tid, t = e >> 3, c8 = (e & 7) * 8;
      const float4 lo = *reinterpret_cast<const float4*>(sA + t * LDA + c8);
      const float4 hi = *reinterpret_cast<const float4*>(sA + t * LDA + c8 + 4);
      uint4 u;
      u.x = pack_bf16x2(lo.x, lo.y);
      u.y = pack_bf16x2(lo.z, lo.w);
      u.z = pack_bf16x2(hi.x, hi.y);
      u.w = pack_bf16x2(hi.z, hi.w);
      *reinterpret_cast<uint4*>(p.Tws + (((size_t)bh * p.NC + n) * 64 + t) * 64 + c8) = u;
    }
  } else if (tid == 0) {  // drain this CTA's own copy and MMA before its memory is reused
    mbar_wait(bar_load, 0, kDrainLimit, p.status);
    if (mma_issued) mbar_wait(bar_mma, 0, kDrainLimit, p.status);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 64);
}

// ---------------------------------------------------------------- the scan
// CH: residual chain step (PRISM_CHAIN_LINEAR or PRISM_CHAIN_GELU), fixed at compile
// time so the linear chain carries none of the GELU step's code or registers.
template <int D, int M, int CH>
__global__ void __launch_bounds__(kCtaThreads, 1)
    prism_chunk_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                          const __grid_constant__ CUtensorMap map_u, const __grid_constant__ CUtensorMap map_v,
                          const __grid_constant__ CUtensorMap map_g, const __grid_constant__ CUtensorMap map_o,
                          const __grid_constant__ CUtensorMap map_t, TcArgs p) {
  using Ly = Layout<D, M>;
  constexpr int NA = Ly::NA, UR = Ly::UR;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sKQ = sm + Ly::OFF_KQ;
  uint8_t* sU = sm + Ly::OFF_U;
  uint8_t* sP = sm + Ly::OFF_P;
  uint8_t* sBQ = sm + Ly::OFF_BQ;
  uint8_t* sTQ = sm + Ly::OFF_TQ;
  uint8_t* sSXA = sm + Ly::OFF_SXA;
  float* sG = reinterpret_cast<float*>(sm + Ly::OFF_SMALL);  // [2][64] in-chunk cumulative log decay
  float* sBeta = sG + 128;                                    // [2][64]
  float* sCdec = sG + 256;                                    // [64] exp(G_63 - G_t)
  float* sEp = sG + 320;                                      // [64] exp(G_t)
  float* sEn = sG + 384;                                      // [64] exp(-G_t) (fast path only)
  uint64_t* bar_load = reinterpret_cast<uint64_t*>(sm + Ly::OFF_SMALL + 1792);
  uint64_t* bar_mma = bar_load + 1;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bar_load + 2);
  int* s_abort = reinterpret_cast<int*>(bar_load + 3);
  uint64_t* bar_drain = bar_load + 4;  // one commit on the abort path: every MMA issued has completed
  uint64_t* bar_pre = bar_load + 5;    // gain and v tiles of the next prologue
  uint64_t* bar_mma1 = bar_load + 6;   // MMA1 of a chunk (issued while the previous one finishes)
  // worker -> MMA warp hand-overs, one arrival per chunk each: operands of MMA1 requested
  // (F), S_n in bf16 (A), [Bku;QU] and QK written (B), X written (E), Delta~ written (G)
  uint64_t* go_F = bar_load + 7;
  uint64_t* go_A = bar_load + 8;
  uint64_t* go_B = bar_load + 9;
  uint64_t* go_E = bar_load + 10;
  uint64_t* go_G = bar_load + 11;
  uint8_t* sX = sSXA;                          // X^T      bf16 [128][64] K-major
  uint8_t* sDl = sSXA + kAtom;                 // Delta~^T bf16 [128][64] K-major

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q4 = warp & 3, cq = warp >> 2;  // TMEM lane quarter, column quarter
  const int row = 32 * q4 + lane;           // TMEM lane of this thread
  const bool srow = q4 < 2 * NA;            // this warp owns state rows c = row < D
  const int bh = blockIdx.x, b = bh / p.H, h = bh % p.H;
  const int T = p.T, H = p.H;
  const int len = p.lengths ? min(max(p.lengths[b], 0), T) : T;
  const int nchunks = (len + kC - 1) / kC;
  const long long lim = p.spin_limit;

  if (tid == 0) {
    mbar_init(bar_load, 1);
    mbar_init(bar_mma, 1);
    mbar_init(bar_drain, 1);
    mbar_init(bar_pre, 1);
    mbar_init(bar_mma1, 1);
    mbar_init(go_F, 1);
    mbar_init(go_A, 1);
    mbar_init(go_B, 1);
    mbar_init(go_E, 1);
    mbar_init(go_G, 1);
    fence_mbar_init();
    *s_abort = 0;
    tma_prefetch_desc(&map_q);
    tma_prefetch_desc(&map_k);
    tma_prefetch_desc(&map_v);
    tma_prefetch_desc(&map_t);
    if (M > 0) {
      tma_prefetch_desc(&map_u);
      tma_prefetch_desc(&map_g);
    }
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
  constexpr int SP = D / 64;  // 16-column pieces of a state-row quarter

  const uint32_t aKQ = smem_u32(sKQ), aU = smem_u32(sU), aP = smem_u32(sP), aBQ = smem_u32(sBQ);
  const uint32_t aTQ = smem_u32(sTQ), aS = smem_u32(sSXA), aX = smem_u32(sX), aDl = smem_u32(sDl);
  uint32_t ph_load = 0, ph_mma = 0, ph_pre = 0, ph_mma1 = 0;
  int pre_inflight = -1;  // (thread 0) phase of the prologue tiles in flight, or -1
  int load_inflight = -1;  // (thread 0) parity of the last closed load phase (the MMA warp consumes it)
  bool load_open = false;  // (thread 0) next chunk's Q/U loads issued, closing arrival not yet made

  // The next chunk's tiles are loaded as soon as their buffers are free: Q once MMA1/MMA3 have
  // read it, U once MMA5a has, K (with the arrival that closes the phase) once MMA5b has.
  auto load_q = [&](int t0) {
    load_open = true;
    mbar_expect_tx(bar_load, NA * 8192);
#pragma unroll
    for (int a = 0; a < NA; ++a) tma_load_4d(sKQ + a * kAtom + 8192, &map_q, bar_load, 64 * a, h, t0, b);
  };
  auto load_u = [&](int t0) {
    if (M > 0) {
      load_open = true;
      mbar_expect_tx(bar_load, NA * UR * 128);
#pragma unroll
      for (int a = 0; a < NA; ++a)
#pragma unroll
        for (int l = 0; l < M; ++l)  // direction-major rows: row l*64 + i
          tma_load_5d(sU + a * Ly::U_ATOM + l * 8192, &map_u, bar_load, 64 * a, l, h, t0, b);
    }
  };
  auto load_k_arrive = [&](int t0) {
    load_open = false;
    load_inflight = (int)ph_load;
    ph_load ^= 1;
    mbar_arrive_expect_tx(bar_load, NA * 8192);
#pragma unroll
    for (int a = 0; a < NA; ++a) tma_load_4d(sKQ + a * kAtom, &map_k, bar_load, 64 * a, h, t0, b);
  };
  // T = (I + A)^{-1} of chunk nn (from the preparation kernel) -> rows 0..63 of TQ
  auto load_t = [&](int nn) {
    load_open = true;
    mbar_expect_tx(bar_load, 8192);
    tma_load_4d(sTQ, &map_t, bar_load, 0, 0, nn, bh);
  };
  auto issue_loads = [&](int t0) {
    load_q(t0);
    load_u(t0);
    load_t(t0 / kC);
    load_k_arrive(t0);
  };
  // Prologue tiles of chunk nn: its gain rows into P's buffer (the prologue turns them into
  // P in place) and 72 rows of v, t0-8 .. t0+63 (the ShortConv history included; zero fill
  // before the sequence start and past T), into the [Bku;QU] buffer.
  constexpr uint32_t VT_ATOM = 72 * 128;
  auto load_pre = [&](int nn) {
    const int tn = nn * kC;
    mbar_arrive_expect_tx(bar_pre, NA * (M * 8192 + VT_ATOM));
#pragma unroll
    for (int a = 0; a < NA; ++a) {
      tma_load_4d(sBQ + a * VT_ATOM, &map_v, bar_pre, 64 * a, h, tn - 8, b);
#pragma unroll
      for (int l = 0; l < M; ++l)
        tma_load_5d(sP + a * Ly::U_ATOM + l * 8192, &map_g, bar_pre, 64 * a, l, h, tn, b);
    }
    pre_inflight = (int)ph_pre;
  };
  constexpr int CPT = D / 8;           // threads per token in the prologue
  constexpr int TPP = kThreads / CPT;  // tokens per prologue pass
  const int pc8 = (tid % CPT) * 8;
  // ShortConv taps of this head, conv_w[h, :, :] (D*W <= 4*D fp32), staged in shared memory
  // for the prologue tap-major ([w][c]: a lane's 8 channels of one tap are 32 contiguous
  // bytes, so a token's 16 lanes read 512 contiguous bytes): one element per thread.
  const float* cw_head = p.conv_w + (size_t)h * D * p.W;
  const bool tap_thread = tid < D * p.W;

  // Gate prefix of chunk n into buffer buf (one warp): G_t = sum_{j<=t} log gamma_j and
  // beta_t; padded steps count as gamma = 1, beta = 0.  gate_load issues the loads (lane owns
  // tokens 2*lane, 2*lane+1), gate_scan finishes from those registers.
  auto gate_load = [&](int n, float (&gl)[4]) {
    const int t0 = n * kC;
    const int nv = min(kC, len - t0);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int t = 2 * lane + e;
      const bool valid = t < nv;
      const size_t th = ((size_t)b * T + min(t0 + t, T - 1)) * H + h;
      gl[e] = valid ? __ldg(p.gamma + th) : 1.f;
      gl[2 + e] = valid ? __ldg(p.beta + th) : 0.f;
    }
  };
  auto gate_scan = [&](const float (&gl)[4], int buf) {
    const float lg0 = __logf(gl[0]), lg1 = __logf(gl[1]);
    float x = lg0 + lg1;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    sG[buf * 64 + 2 * lane] = x - lg1;
    sG[buf * 64 + 2 * lane + 1] = x;
    sBeta[buf * 64 + 2 * lane] = gl[2];
    sBeta[buf * 64 + 2 * lane + 1] = gl[3];
  };

  // Chunk prologue: rho_{i,l} = alpha_{i,l} r_{i,l} -> P (bf16), from the chunk's gain and v
  // tiles (load_pre) and its alpha values (load_alpha); needs the chunk's gate prefix in buf.
  constexpr int NPASS = kC / TPP;
  constexpr int M1 = M > 0 ? M : 1;
  auto load_alpha = [&](int n, float (&al)[NPASS][M1]) {
    const int t0 = n * kC;
    const int nv = min(kC, len - t0);
#pragma unroll
    for (int pass = 0; pass < NPASS; ++pass) {
      const int i = pass * TPP + tid / CPT;
      const size_t th = ((size_t)b * T + min(t0 + i, T - 1)) * H + h;
#pragma unroll
      for (int l = 0; l < M1; ++l) al[pass][l] = (M > 0 && i < nv) ? __ldg(p.alpha + th * M + l) : 0.f;
    }
  };
  auto prologue = [&](int n, int buf, const float* taps, const float (&al)[NPASS][M1]) {
    const int t0 = n * kC;
    const int nv = min(kC, len - t0);
    // Fast path (chunk log-decay >= -60): write P~ = diag(c) P with c_i = e^{G_63 - G_i}; the
    // U-columns of [Bku;QU] then carry e^{G_t - G_63} instead of e^{G_t - G_i} (same product).
    const float G63 = sG[buf * 64 + 63];
    const bool pfast = G63 >= -60.f;
    if (M > 0) {
#pragma unroll
      for (int pass = 0; pass < NPASS; ++pass) {
        const int i = pass * TPP + tid / CPT;
        if (i >= nv) {  // padded step: rho = 0
          const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int l = 0; l < M; ++l) st_bf16x8(sP, sw128_offset(l * 64 + i, pc8, Ly::U_ATOM), z);
          continue;
        }
        const float ci = pfast ? __expf(G63 - sG[buf * 64 + i]) : 1.f;
        float r[8];
        {
          const uint4 v0 = *reinterpret_cast<const uint4*>(sBQ + sw128_offset(8 + i, pc8, VT_ATOM));
          float a[8];
          const float4 lo0 = *reinterpret_cast<const float4*>(taps + pc8);
          const float4 hi0 = *reinterpret_cast<const float4*>(taps + pc8 + 4);
          const float t0v[8] = {lo0.x, lo0.y, lo0.z, lo0.w, hi0.x, hi0.y, hi0.z, hi0.w};
#pragma unroll
          for (int e = 0; e < 8; ++e) a[e] = t0v[e] * bf16_at(v0, e);
#pragma unroll
          for (int w = 1; w < 4; ++w) {
            if (w < p.W) {
              const uint4 vw = *reinterpret_cast<const uint4*>(sBQ + sw128_offset(8 + i - w, pc8, VT_ATOM));
              const float4 lo = *reinterpret_cast<const float4*>(taps + w * D + pc8);
              const float4 hi = *reinterpret_cast<const float4*>(taps + w * D + pc8 + 4);
              const float tw[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
              for (int e = 0; e < 8; ++e) a[e] += tw[e] * bf16_at(vw, e);
            }
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) r[e] = bf16_at(v0, e) - a[e];
        }
#pragma unroll
        for (int l = 0; l < M; ++l) {
          const uint32_t off = sw128_offset(l * 64 + i, pc8, Ly::U_ATOM);
          const uint4 g = *reinterpret_cast<const uint4*>(sP + off);  // gain, replaced by rho below
          float rho[8];
          const float alc = al[pass][l] * ci;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            r[e] = chain_step(r[e], bf16_at(g, e), CH);
            rho[e] = alc * r[e];
          }
          st_bf16x8(sP, off, rho);
        }
      }
    }
  };

  if (warp == kMmaWarp) {
    // ---- the MMA warp: lane 0 issues, in the order the workers hand the operands over
    const volatile int* abort_flag = s_abort;
    uint32_t pF = 0, pA = 0, pB = 0, pE = 0, pG = 0, pL = 0;
    bool ok = true;
    for (int n = 0; n < nchunks && ok; ++n) {
      // MMA1: [K;Q] x [K;U]^T -> R1 once the chunk's K, Q, U, T are in
      ok = mma_warp_wait(go_F, pF, lim, p.status, abort_flag) && mma_warp_wait(bar_load, pL, lim, p.status, abort_flag);
      pF ^= 1;
      pL ^= 1;
      if (!ok) break;
      if (lane == 0) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4 * NA; ++kk) {
          const uint64_t a = kdesc(aKQ, kk, kAtom);
          mma_bf16(tmem + R1, a, a, idesc_bf16(128, 64, 0, 0), kk > 0);
          if (M > 0) mma_bf16(tmem + R1 + 64, a, kdesc(aU, kk, Ly::U_ATOM), idesc_bf16(128, UR, 0, 0), kk > 0);
        }
        mma_commit(bar_mma1);
      }
      __syncwarp();
      // MMA3: S_n x [K;Q]^T -> D3, covered by the next commit (step E reads D3 after it)
      ok = mma_warp_wait(go_A, pA, lim, p.status, abort_flag);
      pA ^= 1;
      if (!ok) break;
      if (lane == 0) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4 * NA; ++kk)
          mma_bf16(tmem + D3, kdesc(aS, kk, kAtom), kdesc(aKQ, kk, kAtom), idesc_bf16(128, 128, 0, 0), kk > 0);
      }
      __syncwarp();
      // MMA2: (Bku P)^T | (QU P)^T -> R1 and [T;QK] x T, committed for step E; then MMA5a:
      // P~^T U or P^T (diag(c) U) onto RS, which only the state pass needs (covered by the
      // commit after MMA4)
      ok = mma_warp_wait(go_B, pB, lim, p.status, abort_flag);
      pB ^= 1;
      if (!ok) break;
      if (lane == 0) {
        tc_fence_after();
        if (M > 0) {
#pragma unroll
          for (int kk = 0; kk < UR / 16; ++kk)
            mma_bf16(tmem + R1, mndesc(aP, kk, Ly::U_ATOM), kdesc(aBQ, kk, kAtom), idesc_bf16(128, 128, 1, 0),
                     kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + R1 + 128, kdesc(aTQ, kk, kAtom), mndesc(aTQ, kk, kAtom), idesc_bf16(128, 64, 0, 1),
                   kk > 0);
        mma_commit(bar_mma);
        if (M > 0) {
#pragma unroll
          for (int kk = 0; kk < UR / 16; ++kk)
            mma_bf16(tmem + RS, mndesc(aP, kk, Ly::U_ATOM), mndesc(aU, kk, Ly::U_ATOM), idesc_bf16(128, D, 1, 1),
                     1);
        }
      }
      __syncwarp();
      // MMA4: X^T x [T;QKT]^T -> Delta^T | (QKT X)^T in R1+128
      ok = mma_warp_wait(go_E, pE, lim, p.status, abort_flag);
      pE ^= 1;
      if (!ok) break;
      if (lane == 0) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + R1 + 128, kdesc(aX, kk, kAtom), kdesc(aTQ, kk, kAtom), idesc_bf16(128, 128, 0, 0),
                   kk > 0);
        mma_commit(bar_mma);
      }
      __syncwarp();
      // MMA5b: Delta~^T K onto RS
      ok = mma_warp_wait(go_G, pG, lim, p.status, abort_flag);
      pG ^= 1;
      if (!ok) break;
      if (lane == 0) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + RS, kdesc(aDl, kk, kAtom), mndesc(aKQ, kk, kAtom), idesc_bf16(128, D, 0, 1), 1);
        mma_commit(bar_mma);
      }
      __syncwarp();
    }
    if (!ok && lane == 0) atomicExch(s_abort, 1);
    if (lane == 0) {  // every MMA issued has completed before the tensor memory is freed
      mma_commit(bar_drain);
      mbar_wait(bar_drain, 0u, kDrainLimit, p.status);
    }
    __syncwarp();
  } else {
  // ---- initial state: RS <- S0 (or 0), bf16 copy -> SXA (A operand of MMA3); chunk 0 prologue
  if (srow) {
#pragma unroll
    for (int pc = 0; pc < SP; ++pc) {
      const int j0 = cq * (D / 4) + 16 * pc;
      float s[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) s[e] = 0.f;
      if (p.S0) {
        const float4* src = reinterpret_cast<const float4*>(p.S0 + (((size_t)b * H + h) * D + row) * D + j0);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float4 f = __ldg(src + e);
          s[4 * e] = f.x; s[4 * e + 1] = f.y; s[4 * e + 2] = f.z; s[4 * e + 3] = f.w;
        }
      }
      st_bf16x8(sSXA, sw128_offset(row, j0, kAtom), s);
      st_bf16x8(sSXA, sw128_offset(row, j0 + 8, kAtom), s + 8);
    }
  }
  if (tid == 0 && nchunks > 0) {
    issue_loads(0);
    mbar_arrive(go_F);  // MMA1 of chunk 0 as soon as its tiles are in
    if (M > 0) load_pre(0);
  }
  float al0[NPASS][M1];
  if (nchunks > 0) load_alpha(0, al0);
  float* taps0 = reinterpret_cast<float*>(sTQ + 8192);  // rows 64..127 of TQ: free until chunk 0's epilogue
  if (nchunks > 0 && warp == 0) {
    float gl[4];
    gate_load(0, gl);
    gate_scan(gl, 0);
  }
  // warp 2 holds the gates of the chunk after the current one in registers, requested a
  // whole chunk before its scan (step C) needs them
  float gl_next[4] = {1.f, 1.f, 0.f, 0.f};
  if (warp == 2 && nchunks > 1) gate_load(1, gl_next);
  if (M > 0 && tap_thread) taps0[(tid % p.W) * D + tid / p.W] = __ldg(cw_head + tid);
  worker_sync();
  if (srow) {  // RS <- exp(G_63 of chunk 0) S0 (undecayed S0 when there is no chunk: S_final)
    const float b0 = nchunks > 0 ? __expf(sG[63]) : 1.f;
#pragma unroll
    for (int pc = 0; pc < SP; ++pc) {
      const int j0 = cq * (D / 4) + 16 * pc;
      float s[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) s[e] = 0.f;
      if (p.S0) {
        const float4* src = reinterpret_cast<const float4*>(p.S0 + (((size_t)b * H + h) * D + row) * D + j0);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float4 f = __ldg(src + e);
          s[4 * e] = b0 * f.x; s[4 * e + 1] = b0 * f.y; s[4 * e + 2] = b0 * f.z; s[4 * e + 3] = b0 * f.w;
        }
      }
      tmem_st16(tl + RS + j0, s);
    }
  }
  if (nchunks > 0 && M > 0) {
    const bool okp = warp_wait(bar_pre, ph_pre, lim, p.status);
    if (okp) {
      if (tid == 0) pre_inflight = -1;
      prologue(0, 0, taps0, al0);
    } else if (lane == 0) {
      atomicExch(s_abort, 1);
    }
  }
  ph_pre ^= 1;
  fence_proxy_async_smem();
  tc_fence_before();
  worker_sync();

  bool aborted = false;
  for (int n = 0; n < nchunks && !aborted; ++n) {
    const int t0 = n * kC;
    const int nv = min(kC, len - t0);
    const int cur = n & 1;
    const float* G = sG + cur * 64;
    const float* Bt = sBeta + cur * 64;

    // ---------------- A: hand S_n (bf16) to the MMA warp for MMA3 (S_n x [K;Q]^T; MMA1 of this
    // chunk was issued during the previous one); per-chunk decay tables
    if (tid == 0) mbar_arrive(go_A);  // S_n (bf16) is in SXA: MMA3
    const bool fast = G[63] >= -60.f;  // exp(-G) stays finite: factor D[t,i] = e^{G_t} e^{-G_i}
    if (tid < 64) {
      sEp[tid] = __expf(G[tid]);
      sEn[tid] = fast ? __expf(-G[tid]) : 0.f;
      sCdec[tid] = __expf(G[63] - G[tid]);
    }
    if (worker_sync_or(*s_abort)) { aborted = true; break; }  // uniform: every setter votes

    // ---------------- B: epilogue of MMA1 -> [Bku;QU], QK (bf16) (exact path: U <- diag(c) U);
    // then the MMA warp issues MMA2 and QK*T (committed for step E) and MMA5a
    bool ok = warp_wait(bar_mma1, ph_mma1, lim, p.status);
    ph_mma1 ^= 1;
    if (!ok && lane == 0) atomicExch(s_abort, 1);
    float gl_after[4] = {1.f, 1.f, 0.f, 0.f};  // warp 2: gates of chunk n+2
    if (warp == 2 && n + 2 < nchunks) gate_load(n + 2, gl_after);
    tc_fence_after();
    if (ok) {
      const bool krow = row < 64;
      const int t = krow ? row : row - 64;
      const int tlim = krow ? t : t + 1;  // keep column i < tlim
      const float Gt = G[t];
      const float rs = (krow ? Bt[t] : 1.f) * sEp[t];
      const float rsu = fast ? (krow ? Bt[t] : 1.f) * __expf(Gt - G[63]) : 0.f;
      constexpr int NP = (64 + UR) / 16;  // 16-column pieces of R1
      constexpr int PQ = NP / 4;           // pieces of this thread's column quarter
      constexpr int PB = PQ >= 2 ? 2 : 1;  // pieces per TMEM wait
#pragma unroll
      for (int pb = 0; pb < PQ; pb += PB) {
      uint32_t raw[PB][16];
#pragma unroll
      for (int k = 0; k < PB; ++k)
        if (pb + k < PQ) tmem_ld16_async(tl + R1 + 16 * (cq * PQ + pb + k), raw[k]);
      tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < PB; ++k) {
        if (pb + k >= PQ) break;
        const int pc = pb + k;
        const int j0 = 16 * (cq * PQ + pc);
        if (krow && j0 < 64) continue;  // K K^T: only the preparation kernel needs it (for T)
        float x[16];
        if (j0 < 64) {  // K / Q columns: D[t,i] = e^{G_t - G_i}
          if (fast) {
            float en[16];
#pragma unroll
            for (int e = 0; e < 16; e += 4) {
              const float4 f = *reinterpret_cast<const float4*>(sEn + j0 + e);
              en[e] = f.x; en[e + 1] = f.y; en[e + 2] = f.z; en[e + 3] = f.w;
            }
#pragma unroll
            for (int e = 0; e < 16; ++e) x[e] = (j0 + e < tlim) ? rs * en[e] * __uint_as_float(raw[k][e]) : 0.f;
          } else {
            const float bk = krow ? Bt[t] : 1.f;
#pragma unroll
            for (int e = 0; e < 16; ++e)
              x[e] = (j0 + e < tlim) ? bk * __expf(Gt - G[j0 + e]) * __uint_as_float(raw[k][e]) : 0.f;
          }
        } else {  // U columns (l, i): fast path e^{G_t - G_63} (P holds P~), else e^{G_t - G_i}
          const int i0 = (j0 - 64) & 63;
          if (fast) {
#pragma unroll
            for (int e = 0; e < 16; ++e) x[e] = (i0 + e < tlim) ? rsu * __uint_as_float(raw[k][e]) : 0.f;
          } else {
            const float bk = krow ? Bt[t] : 1.f;
#pragma unroll
            for (int e = 0; e < 16; ++e)
              x[e] = (i0 + e < tlim) ? bk * __expf(Gt - G[i0 + e]) * __uint_as_float(raw[k][e]) : 0.f;
          }
        }
        if (j0 < 64) {  // QK (rows 64..127 of TQ)
          st_bf16x8(sTQ, sw128_offset(row, j0, kAtom), x);
          st_bf16x8(sTQ, sw128_offset(row, j0 + 8, kAtom), x + 8);
        } else {
          st_bf16x8(sBQ, sw128_offset(row, j0 - 64, kAtom), x);
          st_bf16x8(sBQ, sw128_offset(row, j0 - 56, kAtom), x + 8);
        }
      }
      }
    }
    if (ok && M > 0 && !fast) {
      // exact path: U <- diag(c) U in place, so that MMA5a = P^T (diag(c) U) runs next to MMA2
      // (both read the unscaled P); MMA1, the other reader of U, has completed
      for (int e = tid; e < UR * D / 8; e += kThreads) {
        const int r = e / (D / 8), c8 = (e % (D / 8)) * 8;
        const uint32_t off = sw128_offset(r, c8, Ly::U_ATOM);
        const uint4 u = *reinterpret_cast<const uint4*>(sU + off);
        const float sc = sCdec[r & 63];
        float f[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) f[k] = sc * bf16_at(u, k);
        st_bf16x8(sU, off, f);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    if (worker_sync_or(*s_abort)) { aborted = true; break; }  // uniform: every setter votes
    if (tid == 0) mbar_arrive(go_B);  // MMA2, MMA5a, QK*T

    // ---------------- C: the next chunk's gate prefix; the tap element this thread stages for
    // the next prologue and the values of v it needs for X (their latency hides behind the MMAs)
    if (warp == 2 && n + 1 < nchunks) gate_scan(gl_next, cur ^ 1);
#pragma unroll
    for (int e = 0; e < 4; ++e) gl_next[e] = gl_after[e];
    const float tap_reg = (M > 0 && tap_thread) ? __ldg(cw_head + tid) : 0.f;
    float al_next[NPASS][M1];  // alpha of the next chunk, for its prologue
    // (padded steps have beta = 0, so any in-range token may stand in for them)
    __nv_bfloat16 vraw16[16];  // converted where X is formed, so the loads are not waited on here
    {
      const int tb = 16 * cq;
      const int rr = srow ? row : 0;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int t = min(t0 + tb + e, T - 1);
        vraw16[e] = p.v[(((size_t)b * T + t) * H + h) * D + rr];
      }
    }
    // ---------------- E: QKT -> TQ rows 64..127; X^T -> SXA; O partial parked in TMEM; the next
    // chunk's Q requested; then MMA4
    ok = warp_wait(bar_mma, ph_mma, lim, p.status);
    ph_mma ^= 1;
    if (tid == 0 && ok) {
      if (n + 1 < nchunks) load_q(t0 + kC);  // MMA1 and MMA3, the readers of Q, are done
    }
    if (n + 1 < nchunks) load_alpha(n + 1, al_next);
    if (!ok && lane == 0) atomicExch(s_abort, 1);
    tc_fence_after();
    if (ok) {
      float opart[16];
      if (q4 >= 2) {  // lanes 64..127 hold (QK T)[t, i], t = row - 64
        float x[16];
        tmem_ld16(tl + R1 + 128 + 16 * cq, x);
        st_bf16x8(sTQ, sw128_offset(row, 16 * cq, kAtom), x);
        st_bf16x8(sTQ, sw128_offset(row, 16 * cq + 8, kAtom), x + 8);
      }
      if (srow) {  // state row c = row; tokens t = 16*cq + e
        const int tb = 16 * cq;
        float y[16], d2[16];
        tmem_ld16(tl + D3 + tb, y);
        if (M > 0) tmem_ld16(tl + R1 + tb, d2);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float xv = Bt[tb + e] * (__bfloat162float(vraw16[e]) - sEp[tb + e] * y[e]);
          if (M > 0) xv -= d2[e];
          y[e] = xv;
        }
        st_bf16x8(sX, sw128_offset(row, tb, kAtom), y);
        st_bf16x8(sX, sw128_offset(row, tb + 8, kAtom), y + 8);
        tmem_ld16(tl + D3 + 64 + tb, opart);
        if (M > 0) tmem_ld16(tl + R1 + 64 + tb, d2);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          opart[e] *= sEp[tb + e];
          if (M > 0) opart[e] += d2[e];
        }
        tmem_st16(tl + D3 + 64 + tb, opart);  // parked until step G (no MMA writes D3 before then)
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    if (worker_sync_or(*s_abort)) { aborted = true; break; }  // uniform: every setter votes
    if (tid == 0) mbar_arrive(go_E);  // MMA4

    // ---------------- G: the next chunk's T, U, gain and v tiles requested (MMA4 and MMA5a are
    // done); Delta~^T -> SXA; o = O partial + (QKT X) -> TMA store; then MMA5b
    ok = warp_wait(bar_mma, ph_mma, lim, p.status);
    ph_mma ^= 1;
    if (tid == 0 && ok) {
      if (n + 1 < nchunks) {  // MMA4 (last reader of TQ) and MMA5a (last of P, U) have completed
        load_t(n + 1);
        load_u(t0 + kC);
        if (M > 0) load_pre(n + 1);
      }
    }
    if (!ok && lane == 0) atomicExch(s_abort, 1);
    tc_fence_after();
    if (ok && srow) {
      const int tb = 16 * cq;
      float x[16];
      tmem_ld16(tl + R1 + 128 + tb, x);
#pragma unroll
      for (int e = 0; e < 16; ++e) x[e] *= sCdec[tb + e];
      st_bf16x8(sDl, sw128_offset(row, tb, kAtom), x);
      st_bf16x8(sDl, sw128_offset(row, tb + 8, kAtom), x + 8);
      float opart[16];
      tmem_ld16(tl + R1 + 192 + tb, x);
      tmem_ld16(tl + D3 + 64 + tb, opart);
      // o tile [64 tokens][D] bf16 in the X buffer (MMA4 has consumed X), stored by TMA below
#pragma unroll
      for (int e = 0; e < 16; ++e)
        *reinterpret_cast<__nv_bfloat16*>(sX + sw128_offset(tb + e, row, 8192)) =
            __float2bfloat16_rn(tb + e < nv ? opart[e] + x[e] : 0.f);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    if (worker_sync_or(*s_abort)) { aborted = true; break; }  // uniform: every setter votes
    if (tid == 0) {
      mbar_arrive(go_G);  // MMA5b
#pragma unroll
      for (int a = 0; a < NA; ++a) tma_store_4d(&map_o, sX + a * 8192, 64 * a, h, t0, b);
      bulk_commit_group();
    }

    // ---------------- F: next chunk's prologue while MMA5b runs.  Warp 0 first waits for MMA5b
    // and requests the next chunk's K (MMA5b has read K), so that load overlaps the prologue.
    bool ok5 = true;
    if (warp == 0) {
      ok5 = warp_wait(bar_mma, ph_mma, lim, p.status);
      if (tid == 0 && ok5 && n + 1 < nchunks) {
        load_k_arrive(t0 + kC);
        mbar_arrive(go_F);  // MMA1 of the next chunk once its tiles are in (R1 is free)
      }
      if (!ok5 && lane == 0) atomicExch(s_abort, 1);
    }
    if (n + 1 < nchunks) {
      float* taps = reinterpret_cast<float*>(sBQ + NA * VT_ATOM);  // behind the v tile
      if (M > 0 && tap_thread) taps[(tid % p.W) * D + tid / p.W] = tap_reg;
      worker_sync();
      if (M > 0) {
        const bool okp = warp_wait(bar_pre, ph_pre, lim, p.status);
        if (okp) {
          if (tid == 0) pre_inflight = -1;
          prologue(n + 1, cur ^ 1, taps, al_next);
        } else if (lane == 0) {
          atomicExch(s_abort, 1);
        }
      }
      ph_pre ^= 1;
    }
    fence_proxy_async_smem();

    // ---------------- I: S_{n+1} -> bf16 SXA (and S_final)
    ok = warp == 0 ? ok5 : warp_wait(bar_mma, ph_mma, lim, p.status);
    ph_mma ^= 1;
    if (!ok && lane == 0) atomicExch(s_abort, 1);
    if (tid == 0) bulk_wait_read_all();  // the o tile in SXA has been read by the TMA store
    worker_sync();
    tc_fence_after();
    if (ok && srow) {
      // RS <- exp(G_63 of chunk n+1) S_{n+1}, the decayed state MMA5a / MMA5b of chunk n+1
      // accumulate onto; the bf16 copy (A operand of MMA3) and S_final stay undecayed
      const bool last = n + 1 == nchunks;
      const float bnext = last ? 1.f : __expf(sG[(cur ^ 1) * 64 + 63]);
#pragma unroll
      for (int pc = 0; pc < SP; ++pc) {
        const int j0 = cq * (D / 4) + 16 * pc;
        float s[16];
        tmem_ld16(tl + RS + j0, s);
        st_bf16x8(sSXA, sw128_offset(row, j0, kAtom), s);
        st_bf16x8(sSXA, sw128_offset(row, j0 + 8, kAtom), s + 8);
        if (last) {
          if (p.S_final) {
            float4* dst = reinterpret_cast<float4*>(p.S_final + (((size_t)b * H + h) * D + row) * D + j0);
#pragma unroll
            for (int e = 0; e < 4; ++e) dst[e] = make_float4(s[4 * e], s[4 * e + 1], s[4 * e + 2], s[4 * e + 3]);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) s[e] *= bnext;
          tmem_st16_async(tl + RS + j0, s);
        }
      }
      tmem_wait_st();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    if (worker_sync_or(*s_abort)) { aborted = true; break; }  // uniform: every setter votes
  }

  if (!aborted) {
    // rows with no valid token: S_final = S0 (still in RS); zero the outputs past the last chunk
    if (nchunks == 0 && p.S_final && srow) {
#pragma unroll
      for (int pc = 0; pc < SP; ++pc) {
        const int j0 = cq * (D / 4) + 16 * pc;
        float s[16];
        tmem_ld16(tl + RS + j0, s);
        float4* dst = reinterpret_cast<float4*>(p.S_final + (((size_t)b * H + h) * D + row) * D + j0);
#pragma unroll
        for (int e = 0; e < 4; ++e) dst[e] = make_float4(s[4 * e], s[4 * e + 1], s[4 * e + 2], s[4 * e + 3]);
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
    if (load_open) {  // close the phase so the copies already issued can complete it
      mbar_arrive(bar_load);
      load_inflight = (int)ph_load;
    }
    if (load_inflight >= 0) mbar_wait(bar_load, (uint32_t)load_inflight, kDrainLimit, p.status);
    if (pre_inflight >= 0) mbar_wait(bar_pre, (uint32_t)pre_inflight, kDrainLimit, p.status);
  }
  if (tid == 0) bulk_wait_all();
  }  // workers
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

int num_chunks(int T) { return (T + kC - 1) / kC; }

// T tiles of every (b, h, chunk) into the workspace: one CTA per tile.
template <int D>
cudaError_t launch_prep(const ScanParams& p, const CUtensorMap& mk, cudaStream_t stream) {
  using Ly = PrepLayout<D>;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(prism_chunk_prep_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    Ly::SMEM_ALLOC);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const int NC = num_chunks(p.T);
  PrepArgs a{p.gamma, p.beta, p.lengths, static_cast<__nv_bfloat16*>(p.workspace), p.T, p.H, NC, p.status,
             p.spin_limit};
  prism_chunk_prep_kernel<D><<<p.B * p.H * NC, kPrepThreads, Ly::SMEM_ALLOC, stream>>>(mk, a);
  return cudaGetLastError();
}

template <int D, int M, int CH>
cudaError_t launch_dm(const ScanParams& p, cudaStream_t stream) {
  using Ly = Layout<D, M>;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(prism_chunk_tc_kernel<D, M, CH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    Ly::SMEM_ALLOC);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const cuuint64_t B = p.B, T = p.T, H = p.H;
  const int NC = num_chunks(p.T);
  CUtensorMap mq, mk, mu, mv, mg, mo;
  const cuuint64_t dims4[4] = {(cuuint64_t)D, H, T, B};
  const cuuint64_t str4[3] = {(cuuint64_t)D * 2, H * D * 2, T * H * D * 2};
  const cuuint32_t box4[4] = {64, 1, 64, 1};
  const cuuint32_t box_v[4] = {64, 1, 72, 1};  // a chunk's v rows and 8 rows of ShortConv history
  if (!encode(&mq, p.q, 4, dims4, str4, box4) || !encode(&mk, p.k, 4, dims4, str4, box4) ||
      !encode(&mv, p.v, 4, dims4, str4, box_v) || !encode(&mo, p.o, 4, dims4, str4, box4))
    return cudaErrorInvalidValue;
  if (M > 0) {
    const cuuint64_t dims5[5] = {(cuuint64_t)D, (cuuint64_t)M, H, T, B};
    const cuuint64_t str5[4] = {(cuuint64_t)D * 2, (cuuint64_t)M * D * 2, H * M * D * 2, T * H * M * D * 2};
    const cuuint32_t box5[5] = {64, 1, 1, 64, 1};
    if (!encode(&mu, p.u, 5, dims5, str5, box5) || !encode(&mg, p.gain, 5, dims5, str5, box5))
      return cudaErrorInvalidValue;
  } else {
    mu = mk;
    mg = mk;
  }
  CUtensorMap mt;  // T tiles [B*H][NC][64][64] bf16 in the workspace
  const cuuint64_t dimsT[4] = {64, 64, (cuuint64_t)NC, B * H};
  const cuuint64_t strT[3] = {128, 8192, (cuuint64_t)NC * 8192};
  const cuuint32_t boxT[4] = {64, 64, 1, 1};
  if (!encode(&mt, p.workspace, 4, dimsT, strT, boxT)) return cudaErrorInvalidValue;
  cudaError_t err = launch_prep<D>(p, mk, stream);
  if (err != cudaSuccess) return err;
  TcArgs a{static_cast<const __nv_bfloat16*>(p.q), static_cast<const __nv_bfloat16*>(p.k),
           static_cast<const __nv_bfloat16*>(p.u), static_cast<const __nv_bfloat16*>(p.v), p.gamma, p.beta, p.alpha,
           static_cast<const __nv_bfloat16*>(p.gain), p.conv_w, p.S0, p.lengths,
           static_cast<__nv_bfloat16*>(p.o), p.S_final, p.B, p.T, p.H, p.W, NC, p.status, p.spin_limit};
  prism_chunk_tc_kernel<D, M, CH><<<p.B * p.H, kCtaThreads, Ly::SMEM_ALLOC, stream>>>(mq, mk, mu, mv, mg, mo, mt, a);
  return cudaGetLastError();
}

template <int D, int CH>
cudaError_t launch_dc(const ScanParams& p, cudaStream_t stream) {
  switch (p.L - 1) {
    case 1: return launch_dm<D, 1, CH>(p, stream);
    case 2: return launch_dm<D, 2, CH>(p, stream);
    case 3: return launch_dm<D, 3, CH>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

template <int D>
cudaError_t launch_d(const ScanParams& p, cudaStream_t stream) {
  if (p.L == 1) return launch_dm<D, 0, PRISM_CHAIN_LINEAR>(p, stream);  // no residual chain at L = 1
  if (p.chain == PRISM_CHAIN_GELU) return launch_dc<D, PRISM_CHAIN_GELU>(p, stream);
  return launch_dc<D, PRISM_CHAIN_LINEAR>(p, stream);
}

}  // namespace

bool chunk_tc_supported(int d_k, int d_v, int L, int W, int chunk, int dtype) {
  return dtype == PRISM_BF16 && chunk == kC && d_k == d_v && (d_k == 64 || d_k == 128) && L >= 1 && L <= 4 &&
         W >= 1 && W <= 4;
}

size_t chunk_tc_workspace_bytes(int B, int T, int H) { return (size_t)B * H * num_chunks(T) * 8192; }

cudaError_t launch_chunk_tc(const ScanParams& p, cudaStream_t stream) {
  if (p.d_k == 128) return launch_d<128>(p, stream);
  if (p.d_k == 64) return launch_d<64>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace prism
