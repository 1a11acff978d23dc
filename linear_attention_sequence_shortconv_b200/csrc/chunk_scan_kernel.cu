// Chunkwise-parallel PRISM scan on the 5th-generation tensor cores (tcgen05): a launch of
// residual_write_kernel (the residual write vectors of every token), then the scan.
//
// One scan CTA owns one (batch row, head) chain and walks its chunks of C = 64 tokens in
// order; the fp32 state S (d_v x d_k) stays in tensor memory for the whole sequence (or
// segment: long sequences over few chains are cut into segments, and a sequence whose
// chains leave SMs idle runs in two halves; see the host side at the end).
// Sources: ICML 2026 PRISM write-up (核心迭代形式, 消除 Token 间串行, 消除 Step 间串行,
// 架构形式) and the PRISM technical summary (2.1, 2.2), which fix the recurrence; the
// chunk form below is derived from it.
//
// Chunk algebra (token-local t, i in [0, 64); S_n = state before the chunk; G_t =
// sum_{j<=t} log gamma_j; e_t = e^{G_t}; D[t,i] = e^{G_t - G_i}; c_i = e^{G_63 - G_i};
// rho_{i,l} = alpha_{i,l} r_{i,l}; P_l stacks rho_{.,l} over tokens, U_l stacks u_{.,l}):
//
//   A[t,i]     = beta_t D[t,i] k_t.k_i        (i < t)      T = (I + A)^{-1}
//   Bku_l[t,i] = beta_t D[t,i] k_t.u_{i,l}    (i < t)
//   Mqk[t,i]   = D[t,i] q_t.k_i               (i <= t)     Mqu_l[t,i] = D[t,i] q_t.u_{i,l}  (i <= t)
//   X0  = diag(beta) V - sum_l Bku_l P_l
//   U'  = T X0,                 W' = T diag(beta e) K
//   O_0 = Mqk U' + sum_l Mqu_l P_l,  Q' = diag(e) Q - Mqk W'
//   Delta = U' - W' S_n^T  (the delta-rule corrections beta_t (v_t - gamma_t S_{t-1} k_t))
//   O     = O_0 + Q' S_n^T
//   S_{n+1} = e^{G_63} S_n + Delta^T diag(c) K + sum_l P_l^T diag(c) U_l
//
// Everything but the last three lines is independent of the state, so the state-dependent
// chain of a chunk is two MMAs (Q'/W' against S_n, Delta~ against K) and two short
// tensor-memory epilogues; the rest (the masked Gram products, the inverse, W', Q', U', O_0
// and the residual state write) is worked off by other warps.  The residual chain itself
// (rho, and P~ below) depends on neither the state nor the keys: residual_write_kernel
// computes it for every chunk of every chain at once, before the scan, and the scan loads
// P~ by TMA.
//
// Tensor-core products (bf16 operands, fp32 accumulators in TMEM, M = 128, one issuing
// thread each; "x^T" operands come from TMEM or MN-major shared memory):
//   key     [K;Q] x K^T                     -> RKQ (token rows: A | Mqk)
//   MqkT    [T;Mqk] x T                     -> RKQ (rows 64..127: Mqk T)
//   a_l     [K;Q] x U_l^T                   -> RU[s] (token rows: Bku_l | Mqu_l)
//   b_l     P~_l^T x [Bku_l;Mqu_l]^T        -> ACC  (state rows: (Bku P)^T | (Mqu P)^T)
//   e_l     P~_l^T x U~_l                   -> RS   (the residual write of the chunk)
//   d       [T;MqkT] x (diag(beta e) K)     -> RW   ([W'; Mqk W'])
//   c       X0^T x [T;MqkT]^T               -> ACC  ([U'^T | O_0^T])
//   one     S_n (TMEM) x [-W';Q']^T         -> ACC  ([Delta^T | O^T])
//   two     Delta~^T (TMEM) x K             -> RS   (S_{n+1})
// "Fast" chunks (G_63 >= -60) factor the decay as e^{G_t - G_63} c_i: the residual-write
// launch writes P~ = diag(c) P and U~ = U; other chunks use e^{G_t - G_i} per element,
// P~ = P and U~ = diag(c) U (scaled in place).
//
// Warp roles (448 threads): warps 0-7 the epilogue group EG (Bku/Mqu epilogues, X0,
// [-W'; Q'], the state epilogues, o), warps 8-11 the key group KG (gate prefix, A and Mqk, the
// inverse, Mqk T, K^, W'/Q'; issues its own MMAs), warp 12 the MMA warp (every other MMA),
// warp 13 the TMA warp.  Hand-overs go through mbarriers; every wait is bounded and gives
// up once another agent has set the abort flag, so a missed arrival records
// PRISM_ERR_TIMEOUT instead of hanging the GPU.
#include <cuda.h>

#include <algorithm>
#include <cmath>
#include <functional>
#include <mutex>

#include "common.cuh"
#include "sm100.cuh"

namespace prism {
namespace {

using namespace sm100;

constexpr int kC = 64;            // chunk length
constexpr int kEG = 256;          // epilogue group threads (warps 0-7)
constexpr int kKG = 128;          // key group threads (warps 8-11)
constexpr int kMW = 12;           // MMA warp
constexpr int kTW = 13;           // TMA warp
constexpr int kThreads = 448;
constexpr uint32_t kAtom128 = 16384;  // one 128-row, 128-byte-wide swizzle atom column
constexpr uint32_t kAtom64 = 8192;    // the same with 64 rows
constexpr long long kDrainLimit = 1ll << 18;
constexpr int kWsLd = 68;  // fp32 row stride of the inverse's scratch (bank padding)
constexpr int kRankRows = 1024;  // rows the scan ranks by length (longest first) when chains exceed SMs
constexpr int kPlanSMs = 148;    // SMs of a B200: the segment plan and the chain order assume them

// TMEM columns
// RU: [K;Q] U_l^T, two slots (directions alternate); RW ([W'; Mqk W']) reuses them once the
// direction loop is done.
constexpr uint32_t kRS = 0, kACC = 128, kSB = 256, kRKQ = 320, kRU = 384, kRW = 384;

// NU: shared-memory slots for U_l (direction j uses slot j % NU); P~_l always has two.
// With NU = 3 (many residual directions) the chunk's v tile has no buffer of its own: it
// is loaded into the [-W'; Q'] buffer once the key group's inverse scratch there is free,
// and read before [-W'; Q'] is written.
template <int D, int NU>
struct Lay {
  static_assert(NU == 2 || NU == 3, "U slots");
  static constexpr int NA = D / 64;
  static constexpr bool kVinWQ = NU == 3;
  static constexpr uint32_t KQ = 0;                          // [K;Q] per atom column
  static constexpr uint32_t KB = KQ + NA * kAtom128;         // K for the state update
  static constexpr uint32_t UB = KB + NA * kAtom64;          // U_l, NU slots
  static constexpr uint32_t PB = UB + NU * NA * kAtom64;     // P~_l, two slots
  static constexpr uint32_t BQ = PB + 2 * NA * kAtom64;      // [Bku_l;Mqu_l], two slots; slot 0 also X0^T
  static constexpr uint32_t VB = BQ + 2 * kAtom128;          // v (64 rows), unless it goes to WQ
  static constexpr uint32_t ZB = VB + (kVinWQ ? 0 : NA * kAtom64);  // [T; Mqk | MqkT]
  static constexpr uint32_t WQ = ZB + kAtom128;              // [-W'; Q']
  static constexpr uint32_t WS_BYTES = 64 * kWsLd * 4 + 4096;
  // the inverse's scratch lives in WQ when it fits (WQ is free while the inverse runs)
  static constexpr uint32_t WS = (NA * kAtom128 >= WS_BYTES) ? WQ : WQ + NA * kAtom128;
  static constexpr uint32_t SMALL = (WS == WQ) ? WQ + NA * kAtom128 : WS + ((WS_BYTES + 1023) / 1024) * 1024;
  static constexpr uint32_t BYTES = SMALL + 4096;
  static constexpr uint32_t ALLOC = BYTES + 1024;
  static_assert(ALLOC <= 232448, "exceeds the 227 KB opt-in shared memory of sm_100");
};

// One launch of the scan kernel.  A sequence may be cut into P segments of Ts tokens
// (Ts a multiple of 64), one CTA each; CTA (b, h, p) scans tokens [p Ts, min((p+1) Ts, len)),
// the last segment up to len (the two halves in time have a shorter first segment).
// Its start state is S0 (p = 0), else the identity (s_in_identity), else S_in[b, h, p],
// else zero; its end state goes to S_out[b, h, p] when S_out is set, else to S_final from
// the last segment.  writes_off treats v and the residual writes as zero (the transitions
// alone); write_o = 0 skips the outputs.
struct ScanArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const float* gamma;
  const float* beta;
  const float* alpha;
  const float* conv_w;
  const float* S0;
  const int32_t* lengths;
  __nv_bfloat16* o;
  float* S_final;
  const float* S_in;   // [B, H, P, D, D] or NULL
  float* S_out;        // [B, H, P, D, D] or NULL
  int B, T, H, W, m;   // m: residual directions of this launch (0 when writes are off)
  int P, Ts;
  int s_in_identity, write_o, writes_off;
  int seg_only;        // >= 0: this launch runs only that segment of every chain (one CTA per chain)
  int* status;
  long long spin_limit;
};

// Per-chunk gate tables (two slots: chunk n uses slot n & 1).
struct Gates {
  float G[64], beta[64], e[64], en[64], c[64], rr[64];
  int fast, nv, pad0, pad1;
};

// Barriers (one 8-byte word each, in shared memory).
enum Bar {
  kKqFull, kKqFree, kKbFull, kVFull, kVFree, kWsFree, kUFull0, kUFull1, kUFull2, kPFull0, kPFull1, kUFree0,
  kUFree1, kUFree2, kPFree0, kPFree1, kRuFull0, kRuFull1,
  kEpiDone0, kEpiDone1, kE1Done, kKqkFree, kBkupDone, kX0Ready, kZReady, kWqReady, kAccFull, kDlReady, kRsFull,
  kGates0, kGates1, kGFree0, kGFree1, kKgMma, kDrain, kKgDrain, kRwFull, kNumBars
};

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ void st_bf16x8(uint8_t* base, uint32_t off, const float* x) {
  uint4 u;
  u.x = pack_bf16x2(x[0], x[1]);
  u.y = pack_bf16x2(x[2], x[3]);
  u.z = pack_bf16x2(x[4], x[5]);
  u.w = pack_bf16x2(x[6], x[7]);
  *reinterpret_cast<uint4*>(base + off) = u;
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
  f[0] = bf16_lo(u.x); f[1] = bf16_hi(u.x); f[2] = bf16_lo(u.y); f[3] = bf16_hi(u.y);
  f[4] = bf16_lo(u.z); f[5] = bf16_hi(u.z); f[6] = bf16_lo(u.w); f[7] = bf16_hi(u.w);
}

// ---------------------------------------------------------------- TMEM helpers
__device__ __forceinline__ void tmem_ld32_raw(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32_raw(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]),
      "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]),
      "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st16_raw(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T: the A operand from tensor memory (lane = row of A,
// bf16 pairs packed per 32-bit column).
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ uint64_t kdesc(uint32_t base, int kk, uint32_t atom_stride) {
  return sdesc_sw128(base + (uint32_t)(kk >> 2) * atom_stride + (uint32_t)(kk & 3) * 32u, 16, 1024);
}
__device__ __forceinline__ uint64_t mndesc(uint32_t base, int kk, uint32_t lbo) {
  return sdesc_sw128(base + (uint32_t)kk * 2048u, lbo, 1024);
}
// The same descriptors for K step kk from the step-0 descriptor: only the 14-bit start
// address field (address / 16, bits 0-13) changes, and every address stays inside shared
// memory, so the field never carries into the others.  Saves the issuing thread the full
// descriptor arithmetic per MMA.
__device__ __forceinline__ uint64_t kdesc_step(uint64_t d0, int kk, uint32_t atom_stride) {
  return d0 + (((uint32_t)(kk >> 2) * atom_stride + (uint32_t)(kk & 3) * 32u) >> 4);
}
__device__ __forceinline__ uint64_t mndesc_step(uint64_t d0, int kk) { return d0 + (uint64_t)kk * 128u; }

// ---------------------------------------------------------------- barriers and waits
__device__ __forceinline__ void kg_sync() { asm volatile("bar.sync 2, 128;" ::: "memory"); }
__device__ __forceinline__ bool kg_sync_or(int v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred q, p;\n\tsetp.ne.s32 q, %1, 0;\n\tbar.red.or.pred p, 2, 128, q;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(v)
      : "memory");
  return r != 0;
}

// Bounded wait for the phase of parity `par`: false once the abort flag is set, or after
// `limit` polls (then PRISM_ERR_TIMEOUT is recorded and the abort flag set).
__device__ __forceinline__ bool bwait(uint64_t* bar, uint32_t par, long long limit, int* status,
                                      volatile int* abort_flag) {
  const uint32_t hint = limit < 1024 ? 0u : 20000u;
  for (long long i = 0; i < limit; ++i) {
    if (mbar_try_wait_suspend(bar, par, hint)) return true;
    if (*abort_flag) return false;
  }
  record_status(status, PRISM_ERR_TIMEOUT);
  *abort_flag = 1;
  return false;
}
// The same for a whole warp: lane 0 waits, the answer is broadcast.
__device__ __forceinline__ bool wwait(uint64_t* bar, uint32_t par, long long limit, int* status,
                                      volatile int* abort_flag) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = bwait(bar, par, limit, status, abort_flag) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// T = (I + A)^{-1} in place for a strictly lower-triangular 64 x 64 fp32 A (row stride
// kWsLd, zeros on and above the diagonal) by blocked forward substitution: the four
// 16 x 16 diagonal blocks column by column, then the 16 -> 32 and 32 -> 64 merges
// T_21 = -T_22 A_21 T_11.  Called by the key group's 128 threads (tid 0..127); sY holds
// 1024 fp32 of scratch.
__device__ __forceinline__ void invert_unit_lower64(float* sA, float* sY, int tid) {
  constexpr int LDA = kWsLd;
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
    kg_sync();
    if (tid < 64) {
#pragma unroll
      for (int r = 0; r < 16; ++r) sA[(16 * blk + r) * LDA + 16 * blk + j] = xcol[r];
    }
    kg_sync();
  }
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
    kg_sync();
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
    kg_sync();
  }
  {
    const int r0 = (tid >> 3) * 2, c0 = (tid & 7) * 4;
    float acc[2][4] = {};
#pragma unroll 8
    for (int u = 0; u < 32; ++u) {
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
    kg_sync();
#pragma unroll
    for (int i2 = 0; i2 < 2; ++i2) acc[i2][0] = acc[i2][1] = acc[i2][2] = acc[i2][3] = 0.f;
    const int ulim = r0 + 2;
#pragma unroll 8
    for (int u = 0; u < ulim; ++u) {
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
#pragma unroll
    for (int i2 = 0; i2 < 2; ++i2)
      *reinterpret_cast<float4*>(sA + (32 + r0 + i2) * LDA + c0) =
          make_float4(-acc[i2][0], -acc[i2][1], -acc[i2][2], -acc[i2][3]);
    kg_sync();
  }
}

// ---------------------------------------------------------------- the kernel
template <int D, int NU>
__global__ void __launch_bounds__(kThreads, 1)
    prism_scan_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                      const __grid_constant__ CUtensorMap map_u, const __grid_constant__ CUtensorMap map_v,
                      const __grid_constant__ CUtensorMap map_g, ScanArgs p) {
  using Ly = Lay<D, NU>;
  constexpr int NA = Ly::NA;
  constexpr bool VW = Ly::kVinWQ;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sKQ = sm + Ly::KQ;
  uint8_t* sKB = sm + Ly::KB;
  uint8_t* sBQ0 = sm + Ly::BQ;
  uint8_t* sVB = VW ? sm + Ly::WQ : sm + Ly::VB;  // the chunk's v tile
  uint8_t* sZB = sm + Ly::ZB;
  uint8_t* sWQ = sm + Ly::WQ;
  float* sWS = reinterpret_cast<float*>(sm + Ly::WS);
  Gates* sGates = reinterpret_cast<Gates*>(sm + Ly::SMALL);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Ly::SMALL + 2 * sizeof(Gates));
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + kNumBars);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  static_assert(2 * sizeof(Gates) + 8 * kNumBars + 12 <= 4096, "small region");

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // The chain of this CTA.  With ragged lengths and one CTA per chain, the CTA of rank r
  // takes a head of the (r / H)-th longest row (ties: the lower row first): CTAs start in
  // rank order, so when there are more chains than SMs the long rows start first and the
  // short ones fill in behind them.
  int chain = p.seg_only >= 0 ? (int)blockIdx.x : (int)blockIdx.x / p.P;
  if (p.lengths && (p.P == 1 || p.seg_only >= 0) && p.B <= kRankRows && p.B * p.H > kPlanSMs) {
    int* s_pick = reinterpret_cast<int*>(s_tmem + 2);
    int* s_len = reinterpret_cast<int*>(sBQ0);  // scratch: the [Bku;Mqu] tiles are not in use yet
    for (int r = tid; r < p.B; r += kThreads) s_len[r] = min(max(p.lengths[r], 0), p.T);
    __syncthreads();
    const int want = chain / p.H;
    for (int cand = tid; cand < p.B; cand += kThreads) {
      const int lc = s_len[cand];
      int rank = 0;
      for (int o = 0; o < p.B; ++o) {
        const int lo = s_len[o];
        rank += (lo > lc || (lo == lc && o < cand)) ? 1 : 0;
      }
      if (rank == want) *s_pick = cand;
    }
    __syncthreads();
    chain = *s_pick * p.H + chain % p.H;
  }
  const int bh = chain;
  const int seg = p.seg_only >= 0 ? p.seg_only : (int)blockIdx.x % p.P, b = bh / p.H, h = bh % p.H;
  const int T = p.T, H = p.H, m = p.m;
  // debug build: a chain or segment outside the plan does no work
  const bool cta_ok = in_bounds(bh, (long long)p.B * H, p.status) && in_bounds(seg, p.P, p.status);
  const int len = !cta_ok ? 0 : p.lengths ? min(max(p.lengths[b], 0), T) : T;
  const int tok0 = seg * p.Ts;                         // first token of this CTA's segment
  const int seg_end = seg == p.P - 1 ? T : min(tok0 + p.Ts, T);  // end of the segment (the last: T)
  const int vend = min(len, seg_end);                  // end of its valid tokens
  const int nchunks = vend > tok0 ? (vend - tok0 + kC - 1) / kC : 0;
  const long long lim = p.spin_limit;
  int* status = p.status;
  const size_t DD = (size_t)D * D;
  const float* S_start = !cta_ok ? nullptr
                         : seg == 0 ? (p.S0 ? p.S0 + (size_t)bh * DD : nullptr)
                                    : (p.S_in ? p.S_in + ((size_t)bh * p.P + seg) * DD : nullptr);
  const bool start_identity = seg > 0 && p.s_in_identity;
  float* S_end = !cta_ok ? nullptr
                 : p.S_out ? p.S_out + ((size_t)bh * p.P + seg) * DD
                           : (seg == p.P - 1 && p.S_final ? p.S_final + (size_t)bh * DD : nullptr);

  if (tid == 0) {
    // one arrival each, except the epilogue group's hand-overs: one per warp (8, or the 4
    // warps of the Delta half), so that its warps never wait for one another
    for (int i = 0; i < kNumBars; ++i) {
      const bool eg8 = i == kE1Done || i == kEpiDone0 || i == kEpiDone1 || i == kX0Ready || i == kVFree ||
                       i == kWqReady || i == kKqFree || i == kGFree0 || i == kGFree1;
      mbar_init(&bars[i], i == kDlReady ? 4 : eg8 ? 8 : 1);
    }
    fence_mbar_init();
    *s_abort = 0;
  }
  if (warp == 0) {
    tmem_alloc(s_tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  // this CTA holds its SM: a kernel launched after this one with programmatic dependent
  // launch (the residual write of a second half) may start once every CTA has got here
  if (tid == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const uint32_t aKQ = smem_u32(sKQ), aKB = smem_u32(sKB), aZB = smem_u32(sZB), aWQ = smem_u32(sWQ);
  const uint32_t aUB0 = smem_u32(sm + Ly::UB), aPB0 = smem_u32(sm + Ly::PB), aBQ0 = smem_u32(sBQ0);

  if (warp == kTW) {
    // ================================================================ TMA warp
    // Lane 0 issues every load in one fixed order that follows the order in which their
    // buffers are released, waiting (bounded) for each release.  Per chunk n: P~ of the
    // directions from the third on (two slots) and U from the (NU + 1)-th on (NU slots);
    // with v in the [-W'; Q'] buffer, the chunk's v (once the key group's inverse scratch
    // there is free); then the next chunk's first NU U, first two P~, (v), [K;Q] and K.
    // Every wait is on a release that needs only loads issued before it, so the order
    // cannot deadlock.
    if (lane == 0) {
      int n_kq = 0, n_v = 0, n_kb = 0, nu[3] = {0, 0, 0}, np[2] = {0, 0};  // loads issued per stream
      // debug build: the coordinates of a tile of direction l at token t0 (the innermost,
      // 64 a, is a multiple of 8 inside [0, D) by construction); on a failure the CTA aborts
      auto tile_ok = [&](int l, int t0) -> bool {
        const bool ok = in_bounds(l, max(m, 1), status) && in_bounds(t0, T, status) && in_bounds(h, H, status) &&
                        in_bounds(b, p.B, status) && tma_x_ok(64 * (NA - 1), 64, D, status);
        if (!ok) *s_abort = 1;
        return ok;
      };
      auto prefetch = [&](int n) {  // every tile of chunk n into L2
        const int t0 = tok0 + n * kC;
        for (int a = 0; a < NA; ++a) {
          tma_prefetch_l2_4d(&map_k, 64 * a, h, t0, b);
          tma_prefetch_l2_4d(&map_q, 64 * a, h, t0, b);
          if (!p.writes_off) tma_prefetch_l2_4d(&map_v, 64 * a, h, t0, b);
          for (int l = 0; l < m; ++l) {
            tma_prefetch_l2_5d(&map_u, 64 * a, l, h, t0, b);
            tma_prefetch_l2_5d(&map_g, 64 * a, l, h, t0, b);
          }
        }
      };
      // U_l of direction j into slot j % NU; with NU = 2 P~_l comes with it on the same
      // barrier (both slots are freed by the same MMAs), else it has its own (ld_p)
      auto ld_u = [&](int j) -> bool {
        const int s = j % NU;
        if (j >= NU && !bwait(&bars[kUFree0 + s], ((j / NU) - 1) & 1, lim, status, s_abort)) return false;
        const int t0 = tok0 + (j / m) * kC, l = j % m;
        if (!tile_ok(l, t0)) return false;
        mbar_arrive_expect_tx(&bars[kUFull0 + s], (NU == 2 ? 2 : 1) * NA * kAtom64);
        for (int a = 0; a < NA; ++a) {
          tma_load_5d(sm + Ly::UB + (s * NA + a) * kAtom64, &map_u, &bars[kUFull0 + s], 64 * a, l, h, t0, b);
          if (NU == 2)
            tma_load_5d(sm + Ly::PB + (s * NA + a) * kAtom64, &map_g, &bars[kUFull0 + s], 64 * a, l, h, t0, b);
        }
        ++nu[s];
        return true;
      };
      auto ld_p = [&](int j) -> bool {  // P~_l of direction j into slot j % 2 (NU = 3)
        if (NU == 2) return true;
        const int s = j & 1;
        if (j >= 2 && !bwait(&bars[kPFree0 + s], ((j >> 1) - 1) & 1, lim, status, s_abort)) return false;
        const int t0 = tok0 + (j / m) * kC, l = j % m;
        if (!tile_ok(l, t0)) return false;
        mbar_arrive_expect_tx(&bars[kPFull0 + s], NA * kAtom64);
        for (int a = 0; a < NA; ++a)
          tma_load_5d(sm + Ly::PB + (s * NA + a) * kAtom64, &map_g, &bars[kPFull0 + s], 64 * a, l, h, t0, b);
        ++np[s];
        return true;
      };
      auto ld_kq = [&](int n) -> bool {
        if (n >= 1 && !bwait(&bars[kKqFree], (n - 1) & 1, lim, status, s_abort)) return false;
        const int t0 = tok0 + n * kC;
        if (!tile_ok(0, t0)) return false;
        mbar_arrive_expect_tx(&bars[kKqFull], 2 * NA * kAtom64);
        for (int a = 0; a < NA; ++a) {
          tma_load_4d(sKQ + a * kAtom128, &map_k, &bars[kKqFull], 64 * a, h, t0, b);
          tma_load_4d(sKQ + a * kAtom128 + kAtom64, &map_q, &bars[kKqFull], 64 * a, h, t0, b);
        }
        if (n + 2 < nchunks) prefetch(n + 2);
        ++n_kq;
        return true;
      };
      // v of chunk n: into its own buffer once the epilogue group has read chunk n - 1's,
      // or (VW) into the [-W'; Q'] buffer once the key group's inverse scratch there is free
      auto ld_v = [&](int n) -> bool {
        if (p.writes_off) return true;
        if (VW ? !bwait(&bars[kWsFree], n & 1, lim, status, s_abort)
               : (n >= 1 && !bwait(&bars[kVFree], (n - 1) & 1, lim, status, s_abort)))
          return false;
        if (!tile_ok(0, tok0 + n * kC)) return false;
        mbar_arrive_expect_tx(&bars[kVFull], NA * kAtom64);
        for (int a = 0; a < NA; ++a)
          tma_load_4d(sVB + a * kAtom64, &map_v, &bars[kVFull], 64 * a, h, tok0 + n * kC, b);
        ++n_v;
        return true;
      };
      auto ld_kb = [&](int n) -> bool {
        if (n >= 1 && !bwait(&bars[kRsFull], (n - 1) & 1, lim, status, s_abort)) return false;
        if (!tile_ok(0, tok0 + n * kC)) return false;
        mbar_arrive_expect_tx(&bars[kKbFull], NA * kAtom64);
        for (int a = 0; a < NA; ++a)
          tma_load_4d(sKB + a * kAtom64, &map_k, &bars[kKbFull], 64 * a, h, tok0 + n * kC, b);
        ++n_kb;
        return true;
      };
      bool ok = true;
      if (nchunks > 0) {
        tma_prefetch_desc(&map_q);
        tma_prefetch_desc(&map_k);
        tma_prefetch_desc(&map_v);
        if (m > 0) {
          tma_prefetch_desc(&map_u);
          tma_prefetch_desc(&map_g);
        }
        if (nchunks > 1) prefetch(1);
        ok = ld_kq(0) && (VW || ld_v(0)) && ld_kb(0);
        for (int l = 0; l < min(m, NU) && ok; ++l) ok = ld_u(l);
        for (int l = 0; l < min(m, 2) && ok; ++l) ok = ld_p(l);
      }
      for (int n = 0; n < nchunks && ok; ++n) {
        for (int l = 2; l < m && ok; ++l) {
          if (l >= NU) ok = ld_u(n * m + l);
          ok = ok && ld_p(n * m + l);
        }
        if (VW) ok = ok && ld_v(n);
        if (n + 1 < nchunks && ok) {
          for (int l = 0; l < min(m, NU) && ok; ++l) ok = ld_u((n + 1) * m + l);
          for (int l = 0; l < min(m, 2) && ok; ++l) ok = ld_p((n + 1) * m + l);
          ok = ok && (VW || ld_v(n + 1)) && ld_kq(n + 1) && ld_kb(n + 1);
        }
      }
      // drain on an abort: the last phase of every barrier a load was issued on has completed
      if (*s_abort) {
        if (n_kq > 0) mbar_wait(&bars[kKqFull], (n_kq - 1) & 1, kDrainLimit, status);
        if (n_v > 0) mbar_wait(&bars[kVFull], (n_v - 1) & 1, kDrainLimit, status);
        if (n_kb > 0) mbar_wait(&bars[kKbFull], (n_kb - 1) & 1, kDrainLimit, status);
#pragma unroll
        for (int s2 = 0; s2 < 3; ++s2)
          if (nu[s2] > 0) mbar_wait(&bars[kUFull0 + s2], (nu[s2] - 1) & 1, kDrainLimit, status);
#pragma unroll
        for (int s2 = 0; s2 < 2; ++s2)
          if (np[s2] > 0) mbar_wait(&bars[kPFull0 + s2], (np[s2] - 1) & 1, kDrainLimit, status);
      }
    }
    __syncwarp();
  } else if (warp == kMW) {
    // ================================================================ MMA warp (lane 0 issues)
    if (lane == 0) {
      bool ok = true;
      int j = 0;
      // MMA-b and MMA-e of direction jj (direction l of chunk n)
      auto do_be = [&](int n, int jj, int l) -> bool {
        const int s = jj & 1, su = jj % NU;
        if (!bwait(&bars[kEpiDone0 + s], (jj >> 1) & 1, lim, status, s_abort)) return false;
        if (NU == 3 && !bwait(&bars[kPFull0 + s], (jj >> 1) & 1, lim, status, s_abort)) return false;
        if (l == 0 && !bwait(&bars[kE1Done], n & 1, lim, status, s_abort)) return false;
        tc_fence_after();
        const uint32_t aP = aPB0 + s * NA * kAtom64, aU = aUB0 + su * NA * kAtom64, aB = aBQ0 + s * kAtom128;
        const uint64_t dP = mndesc(aP, 0, kAtom64), dB = kdesc(aB, 0, kAtom128), dU = mndesc(aU, 0, kAtom64);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + kACC, mndesc_step(dP, kk), kdesc_step(dB, kk, kAtom128), idesc_bf16(128, 128, 1, 0),
                   (l > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + kRS, mndesc_step(dP, kk), mndesc_step(dU, kk), idesc_bf16(128, D, 1, 1), 1);
        if (NU == 3) mma_commit(&bars[kPFree0 + s]);
        mma_commit(&bars[kUFree0 + su]);
        if (l == m - 1) mma_commit(&bars[kBkupDone]);
        return true;
      };
      for (int n = 0; n < nchunks && ok; ++n) {
        if (m > 0) {
          // MMA-a of every direction, each followed by MMA-b/e of the direction before it
          ok = bwait(&bars[kKqFull], n & 1, lim, status, s_abort);
          for (int l = 0; l < m && ok; ++l) {
            const int jj = j + l, s = jj & 1, su = jj % NU;
            ok = bwait(&bars[kUFull0 + su], (jj / NU) & 1, lim, status, s_abort);
            if (!ok) break;
            tc_fence_after();
            const uint64_t dKQ = kdesc(aKQ, 0, kAtom128), dU = kdesc(aUB0 + su * NA * kAtom64, 0, kAtom64);
#pragma unroll
            for (int kk = 0; kk < 4 * NA; ++kk)
              mma_bf16(tmem + kRU + 64 * s, kdesc_step(dKQ, kk, kAtom128), kdesc_step(dU, kk, kAtom64),
                       idesc_bf16(128, 64, 0, 0), kk > 0);
            mma_commit(&bars[kRuFull0 + s]);
            if (l == m - 1) mma_commit(&bars[kKqkFree]);
            if (l >= 1) ok = do_be(n, jj - 1, l - 1);
          }
          if (ok) ok = do_be(n, j + m - 1, m - 1);
          j += m;
        } else {
          ok = bwait(&bars[kE1Done], n & 1, lim, status, s_abort);
        }
        // MMA-c: [U'^T | O_0^T] onto ACC (nothing to add when the writes are off)
        if (ok && !p.writes_off) {
          ok = bwait(&bars[kX0Ready], n & 1, lim, status, s_abort) && bwait(&bars[kZReady], n & 1, lim, status, s_abort);
          if (ok) {
            tc_fence_after();
            const uint64_t dX = kdesc(aBQ0, 0, kAtom128), dZ = kdesc(aZB, 0, kAtom128);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16(tmem + kACC, kdesc_step(dX, kk, kAtom128), kdesc_step(dZ, kk, kAtom128),
                       idesc_bf16(128, 128, 0, 0), (m > 0 || kk > 0) ? 1u : 0u);
          }
        }
        // MMA1: S_n x [-W';Q']^T onto ACC
        if (ok) ok = bwait(&bars[kWqReady], n & 1, lim, status, s_abort);
        if (ok) {
          tc_fence_after();
          const uint64_t dW = kdesc(aWQ, 0, kAtom128);
#pragma unroll
          for (int kk = 0; kk < 4 * NA; ++kk)
            mma_ts(tmem + kACC, tmem + kSB + 8 * kk, kdesc_step(dW, kk, kAtom128), idesc_bf16(128, 128, 0, 0),
                   (!p.writes_off || kk > 0) ? 1u : 0u);
          mma_commit(&bars[kAccFull]);
        }
        // MMA2: Delta~^T x K onto RS
        if (ok) ok = bwait(&bars[kDlReady], n & 1, lim, status, s_abort) && bwait(&bars[kKbFull], n & 1, lim, status, s_abort);
        if (ok) {
          tc_fence_after();
          const uint64_t dK = mndesc(aKB, 0, kAtom64);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ts(tmem + kRS, tmem + kSB + 8 * kk, mndesc_step(dK, kk), idesc_bf16(128, D, 0, 1), 1);
          mma_commit(&bars[kRsFull]);
        }
      }
      // every MMA this thread issued has completed before TMEM is freed
      mma_commit(&bars[kDrain]);
      mbar_wait(&bars[kDrain], 0, kDrainLimit, status);
    }
    __syncwarp();
  } else if (warp >= 8) {
    // ================================================================ key group
    const int kt = tid - kEG;  // 0..127
    const int q4 = warp & 3;
    const int row = 32 * q4 + lane;  // TMEM lane
    const uint32_t tl = tmem + ((uint32_t)(32 * q4) << 16);
    uint32_t ph_kg = 0;
    bool ok = true;
    auto kg_mma_wait = [&]() -> bool {
      const bool r = wwait(&bars[kKgMma], ph_kg, lim, status, s_abort);
      ph_kg ^= 1;
      return r;
    };
    // gate prefix and decay tables of chunk n into slot n & 1 (warp 8; the key
    // group meets on its barrier afterwards)
    auto gates = [&](int n) {
      if (warp != 8) return;
      Gates& gq = sGates[n & 1];
      const int t0 = tok0 + n * kC;
      const int nv = min(kC, vend - t0);
      float gl[2], bl[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int t = 2 * lane + e;
        const bool valid = t < nv;
        const size_t th = ((size_t)b * T + min(t0 + t, T - 1)) * H + h;
        const bool ld = valid && in_bounds((long long)th, (long long)p.B * T * H, status);
        gl[e] = ld ? __ldg(p.gamma + th) : 1.f;
        bl[e] = ld ? __ldg(p.beta + th) : 0.f;
      }
      float Gv[2], G63;
      chunk_log_decay(gl[0], gl[1], lane, Gv[0], Gv[1], G63);
      const bool fast = chunk_decay_fast(G63);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int t = 2 * lane + e;
        gq.G[t] = Gv[e];
        gq.beta[t] = bl[e];
        gq.e[t] = __expf(Gv[e]);
        gq.en[t] = fast ? __expf(-Gv[e]) : 0.f;
        gq.c[t] = __expf(G63 - Gv[e]);
        gq.rr[t] = fast ? __expf(Gv[e] - G63) : 0.f;
      }
      if (lane == 0) {
        gq.fast = fast ? 1 : 0;
        gq.nv = nv;
      }
    };
    if (nchunks > 0) {
      gates(0);
      kg_sync();
      if (kt == 0) mbar_arrive(&bars[kGates0]);
    }
    for (int n = 0; n < nchunks; ++n) {
      const int g = n & 1;
      Gates& gt = sGates[g];
      bool fail = false;
      const bool fast = gt.fast != 0;
      // ---- key product [K;Q] K^T
      fail = !wwait(&bars[kKqFull], n & 1, lim, status, s_abort);
      // the inverse's scratch and ZB are free once MMA-c and MMA1 of the previous chunk are
      // done; the key product waits for them too, so it does not hold up MMA1 on the tensor pipe
      if (!fail && n >= 1) fail = !wwait(&bars[kAccFull], (n - 1) & 1, lim, status, s_abort);
      if (kg_sync_or(fail)) break;
      if (kt == 0) {
        tc_fence_after();
        const uint64_t dKQ = kdesc(aKQ, 0, kAtom128);
#pragma unroll
        for (int kk = 0; kk < 4 * NA; ++kk) {
          const uint64_t a = kdesc_step(dKQ, kk, kAtom128);
          mma_bf16(tmem + kRKQ, a, a, idesc_bf16(128, 64, 0, 0), kk > 0);
        }
        mma_commit(&bars[kKgMma]);
      }
      fail = !kg_mma_wait();
      if (kg_sync_or(fail)) break;
      tc_fence_after();
      {  // A (token rows 0..63, fp32 into the inverse's scratch) and Mqk (rows 64..127, bf16 into ZB)
        const bool krow = row < 64;
        const int t = krow ? row : row - 64;
        const float bt = krow ? gt.beta[t] : 1.f;
        const float et = gt.e[t], Gt = gt.G[t];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t raw[32];
          tmem_ld32_raw(tl + kRKQ + 32 * half, raw);
          tmem_wait_ld();
          float x[32];
          const int tlim = krow ? t : t + 1;  // keep columns i < tlim
          const int br = q4 & 1;              // this warp's 32-row block against the column half
          if (fast && br < half) {            // above the diagonal: nothing kept
#pragma unroll
            for (int e = 0; e < 32; ++e) x[e] = 0.f;
          } else if (fast) {  // D[t,i] = e^{G_t} e^{-G_i}
            const float rt = bt * et;
            const int lim_e = br > half ? 32 : tlim - 32 * half;
#pragma unroll
            for (int e4 = 0; e4 < 32; e4 += 4) {
              const float4 en = *reinterpret_cast<const float4*>(gt.en + 32 * half + e4);
              const float f[4] = {en.x, en.y, en.z, en.w};
#pragma unroll
              for (int k2 = 0; k2 < 4; ++k2) {
                const int e = e4 + k2;
                x[e] = e < lim_e ? rt * f[k2] * __uint_as_float(raw[e]) : 0.f;
              }
            }
          } else {  // strongly decaying chunk: e^{G_t - G_i} per element
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int i = 32 * half + e;
              x[e] = (i < tlim) ? bt * __expf(Gt - gt.G[i]) * __uint_as_float(raw[e]) : 0.f;
            }
          }
          if (krow) {
            float4* dst = reinterpret_cast<float4*>(sWS + t * kWsLd + 32 * half);
#pragma unroll
            for (int e = 0; e < 8; ++e) dst[e] = make_float4(x[4 * e], x[4 * e + 1], x[4 * e + 2], x[4 * e + 3]);
          } else {
#pragma unroll
            for (int c8 = 0; c8 < 32; c8 += 8) st_bf16x8(sZB, sw128_offset(row, 32 * half + c8, kAtom128), x + c8);
          }
        }
      }
      kg_sync();
      invert_unit_lower64(sWS, sWS + 64 * kWsLd, kt);
      // T -> rows 0..63 of ZB (bf16)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int e = q * kKG + kt, t = e >> 3, c8 = (e & 7) * 8;
        float f[8];
        const float4 lo = *reinterpret_cast<const float4*>(sWS + t * kWsLd + c8);
        const float4 hi = *reinterpret_cast<const float4*>(sWS + t * kWsLd + c8 + 4);
        f[0] = lo.x; f[1] = lo.y; f[2] = lo.z; f[3] = lo.w; f[4] = hi.x; f[5] = hi.y; f[6] = hi.z; f[7] = hi.w;
        st_bf16x8(sZB, sw128_offset(t, c8, kAtom128), f);
      }
      fence_proxy_async_smem();
      kg_sync();
      if (VW && kt == 0) mbar_arrive(&bars[kWsFree]);  // the inverse's scratch is free: this chunk's v may land
      // ---- Mqk T
      if (kt == 0) {
        tc_fence_after();
        const uint64_t dZk = kdesc(aZB, 0, kAtom128), dZm = mndesc(aZB, 0, kAtom128);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + kRKQ, kdesc_step(dZk, kk, kAtom128), mndesc_step(dZm, kk), idesc_bf16(128, 64, 0, 1),
                   kk > 0);
        mma_commit(&bars[kKgMma]);
      }
      fail = !kg_mma_wait();
      if (kg_sync_or(fail)) break;
      tc_fence_after();
      if (row >= 64) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t raw[32];
          tmem_ld32_raw(tl + kRKQ + 32 * half, raw);
          tmem_wait_ld();
          float x[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) x[e] = __uint_as_float(raw[e]);
#pragma unroll
          for (int c8 = 0; c8 < 32; c8 += 8) st_bf16x8(sZB, sw128_offset(row, 32 * half + c8, kAtom128), x + c8);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      kg_sync();
      if (kt == 0) mbar_arrive(&bars[kZReady]);
      // ---- K^ = diag(beta e) K in place (rows 0..63 of KQ) once the direction loop is done with K
      if (m > 0) fail = !wwait(&bars[kKqkFree], n & 1, lim, status, s_abort);
      if (kg_sync_or(fail)) break;
      for (int e = kt; e < 64 * (D / 8); e += kKG) {
        const int t = e / (D / 8), c8 = (e % (D / 8)) * 8;
        const uint32_t off = sw128_offset(t, c8, kAtom128);
        const float sc = gt.beta[t] * gt.e[t];
        float f[8];
        unpack8(*reinterpret_cast<const uint4*>(sKQ + off), f);
#pragma unroll
        for (int k2 = 0; k2 < 8; ++k2) f[k2] *= sc;
        st_bf16x8(sKQ, off, f);
      }
      fence_proxy_async_smem();
      // RW shares columns with RU: free once the direction loop's MMAs are done
      if (m > 0) fail = !wwait(&bars[kBkupDone], n & 1, lim, status, s_abort);
      if (kg_sync_or(fail)) break;
      // ---- [W'; Mqk W'] = [T; MqkT] K^ into RW; the epilogue group turns it into [-W'; Q']
      if (kt == 0) {
        tc_fence_after();
        const uint64_t dZk = kdesc(aZB, 0, kAtom128), dKm = mndesc(aKQ, 0, kAtom128);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + kRW, kdesc_step(dZk, kk, kAtom128), mndesc_step(dKm, kk), idesc_bf16(128, D, 0, 1),
                   kk > 0);
        mma_commit(&bars[kRwFull]);
      }
      // ---- gates of the next chunk, into the slot chunk n - 1 used (free once the epilogue
      // group has started chunk n)
      if (n + 1 < nchunks) {
        if (n >= 1) fail = !wwait(&bars[kGFree0 + (g ^ 1)], ((n - 1) >> 1) & 1, lim, status, s_abort);
        if (kg_sync_or(fail)) break;
        gates(n + 1);
        kg_sync();
        if (kt == 0) mbar_arrive(&bars[kGates0 + (g ^ 1)]);
      }
      ok = true;
    }
    (void)ok;
    if (kt == 0) {  // the group's own MMAs have completed before TMEM is freed
      mma_commit(&bars[kKgDrain]);
      mbar_wait(&bars[kKgDrain], 0, kDrainLimit, status);
    }
  } else {
    // ================================================================ epilogue group
    const int q4 = warp & 3, ch = warp >> 2;
    const int row = 32 * q4 + lane;  // TMEM lane: state row c, or token row
    const uint32_t tl = tmem + ((uint32_t)(32 * q4) << 16);
    const bool srow = row < D;
    bool aborted = false;
    int j = 0;
    // chunk 0's v tile (later chunks' arrive while the state MMAs of the chunk before run;
    // with v in the [-W'; Q'] buffer, each chunk's is waited for in X0)
    if (!VW && nchunks > 0 && !p.writes_off) {
      if (!wwait(&bars[kVFull], 0, lim, status, s_abort)) aborted = true;
    }
    for (int n = 0; n < nchunks && !aborted; ++n) {
      const int g = n & 1;
      Gates& gt = sGates[g];
      const int t0 = tok0 + n * kC;
      bool fail = !wwait(&bars[kGates0 + g], (n >> 1) & 1, lim, status, s_abort);
      // ---- E1: S_n -> bf16 into SB (A operand of MMA1), RS <- e^{G_63} S_n
      if (!fail && n >= 1) fail = !wwait(&bars[kRsFull], (n - 1) & 1, lim, status, s_abort);
      if (fail) { aborted = true; break; }
      if (n >= 1 && lane == 0) mbar_arrive(&bars[kGFree0 + (g ^ 1)]);  // this warp is done with chunk n-1's gates
      tc_fence_after();
      if (srow) {  // this thread: state row c = row, columns [ch*D/2, ch*D/2 + D/2), 32 at a time
        const float e63 = gt.e[63];
#pragma unroll
        for (int pc = 0; pc < D / 64; ++pc) {
          const int c0 = ch * (D / 2) + 32 * pc;
          uint32_t raw[32];
          if (n == 0) {  // the segment's start state: S0, the identity, a folded state or zero
            const float4* src = reinterpret_cast<const float4*>(S_start + (size_t)row * D + c0);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float4 f = S_start ? __ldg(src + e) : make_float4(0.f, 0.f, 0.f, 0.f);
              raw[4 * e] = __float_as_uint(f.x);
              raw[4 * e + 1] = __float_as_uint(f.y);
              raw[4 * e + 2] = __float_as_uint(f.z);
              raw[4 * e + 3] = __float_as_uint(f.w);
            }
            if (start_identity) {
#pragma unroll
              for (int e = 0; e < 32; ++e) raw[e] = __float_as_uint(c0 + e == row ? 1.f : 0.f);
            }
          } else {
            tmem_ld32_raw(tl + kRS + c0, raw);
            tmem_wait_ld();
          }
          uint32_t pk[16];
          const float2 e2 = make_float2(e63, e63);
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const float2 sv = make_float2(__uint_as_float(raw[2 * c]), __uint_as_float(raw[2 * c + 1]));
            pk[c] = pack_bf16x2(sv.x, sv.y);
            const float2 sc = __fmul2_rn(e2, sv);
            raw[2 * c] = __float_as_uint(sc.x);
            raw[2 * c + 1] = __float_as_uint(sc.y);
          }
          tmem_st16_raw(tl + kSB + c0 / 2, pk);
          tmem_st32_raw(tl + kRS + c0, raw);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kE1Done]);
      const bool fast = gt.fast != 0;
      const int nv = gt.nv;
      // ---- direction loop: the epilogue ([Bku_l; Mqu_l]) of every direction
      for (int l = 0; l < m; ++l, ++j) {
        const int s = j & 1, su = j % NU;
        uint8_t* sU = sm + Ly::UB + su * NA * kAtom64;
        uint8_t* sB = sBQ0 + s * kAtom128;
        fail = !wwait(&bars[kUFull0 + su], (j / NU) & 1, lim, status, s_abort);
        if (fail) { aborted = true; break; }
        fail = !wwait(&bars[kRuFull0 + s], (j >> 1) & 1, lim, status, s_abort);
        if (fail) { aborted = true; break; }
        tc_fence_after();
        // epilogue: RU[s] (token rows) -> [Bku_l; Mqu_l] bf16 in BQ[s]
        {
          const bool krow = row < 64;
          const int t = krow ? row : row - 64;
          const float bt = krow ? gt.beta[t] : 1.f;
          uint32_t raw[32];
          tmem_ld32_raw(tl + kRU + 64 * s + 32 * ch, raw);
          tmem_wait_ld();
          float x[32];
          // the masks are causal: against this warp's 32-token block of rows, the 32-column
          // piece [32 ch, 32 ch + 32) is entirely kept, entirely zero or the diagonal block
          const int br = q4 & 1;
          if (fast && br != ch) {
            const float f = br > ch ? bt * gt.rr[t] : 0.f;
            const float2 f2 = make_float2(f, f);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const float2 y = __fmul2_rn(f2, make_float2(__uint_as_float(raw[e]), __uint_as_float(raw[e + 1])));
              x[e] = y.x;
              x[e + 1] = y.y;
            }
          } else if (fast) {
            const float f = bt * gt.rr[t];
            const int lim_e = krow ? lane : lane + 1;  // keep columns e < lim_e of the piece
#pragma unroll
            for (int e = 0; e < 32; ++e) x[e] = e < lim_e ? f * __uint_as_float(raw[e]) : 0.f;
          } else {  // strongly decaying chunk
            const float Gt = gt.G[t];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int i = 32 * ch + e;
              x[e] = (krow ? i < t : i <= t) ? bt * __expf(Gt - gt.G[i]) * __uint_as_float(raw[e]) : 0.f;
            }
          }
#pragma unroll
          for (int c8 = 0; c8 < 32; c8 += 8) st_bf16x8(sB, sw128_offset(row, 32 * ch + c8, kAtom128), x + c8);
        }
        if (!fast) {  // U~ = diag(c) U in place (MMA-a, its other reader, has completed)
          for (int e = tid; e < 64 * (D / 8); e += kEG) {
            const int i = e / (D / 8), c8 = (e % (D / 8)) * 8;
            const uint32_t off = sw128_offset(i, c8 & 63, kAtom64) + (c8 >> 6) * kAtom64;
            float f[8];
            unpack8(*reinterpret_cast<const uint4*>(sU + off), f);
            const float ci = gt.c[i];
#pragma unroll
            for (int k2 = 0; k2 < 8; ++k2) f[k2] *= ci;
            st_bf16x8(sU, off, f);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[kEpiDone0 + s]);
      }
      if (aborted) break;
      // ---- X0^T = beta V - (Bku P)^T -> BQ slot 0 (K-major rows c); ACC's Delta half zeroed
      if (!p.writes_off) {
      float x[32];  // beta_t v_t[c], read while the last direction's MMAs finish
      if (VW) {
        fail = !wwait(&bars[kVFull], n & 1, lim, status, s_abort);
        if (fail) { aborted = true; break; }
      }
      if (srow) {
        const uint8_t* vcol = sVB + (row >> 6) * kAtom64;
#pragma unroll
        for (int e4 = 0; e4 < 32; e4 += 4) {
          const float4 b4 = *reinterpret_cast<const float4*>(gt.beta + 32 * ch + e4);
          const float bb[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
          for (int k2 = 0; k2 < 4; ++k2) {
            const int t = 32 * ch + e4 + k2;
            const float vv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(vcol + sw128_offset(t, row & 63, kAtom64)));
            x[e4 + k2] = bb[k2] * vv;
          }
        }
      }
      if (m > 0) fail = !wwait(&bars[kBkupDone], n & 1, lim, status, s_abort);
      if (fail) { aborted = true; break; }
      tc_fence_after();
      if (srow) {
        if (m > 0) {
          uint32_t raw[32];
          tmem_ld32_raw(tl + kACC + 32 * ch, raw);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float2 y = __fadd2_rn(make_float2(x[e], x[e + 1]),
                                        make_float2(-__uint_as_float(raw[e]), -__uint_as_float(raw[e + 1])));
            x[e] = y.x;
            x[e + 1] = y.y;
          }
        }
#pragma unroll
        for (int c8 = 0; c8 < 32; c8 += 8) st_bf16x8(sBQ0, sw128_offset(row, 32 * ch + c8, kAtom128), x + c8);
        if (m > 0) {
          uint32_t z[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) z[e] = 0u;
          tmem_st32_raw(tl + kACC + 32 * ch, z);
          tmem_wait_st();
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars[kX0Ready]);
        if (!VW) mbar_arrive(&bars[kVFree]);
      }
      }
      // ---- [-W'; Q'] -> WQ (Q' = e Q - Mqk W'): token rows, this warp's half of the columns
      fail = !wwait(&bars[kRwFull], n & 1, lim, status, s_abort);
      if (fail) { aborted = true; break; }
      // with v in this buffer: every warp of the group has read it (X0Ready completes only
      // when all eight have arrived; a bounded wait, like every other one)
      if (VW && !p.writes_off) {
        fail = !wwait(&bars[kX0Ready], n & 1, lim, status, s_abort);
        if (fail) { aborted = true; break; }
      }
      tc_fence_after();
      {
        const bool wrow = row < 64;
        const int t = wrow ? row : row - 64;
        const float et = gt.e[t];
#pragma unroll
        for (int pc = 0; pc < D / 64; ++pc) {
          const int c0 = ch * (D / 2) + 32 * pc;
          uint32_t raw[32];
          tmem_ld32_raw(tl + kRW + c0, raw);
          tmem_wait_ld();
#pragma unroll
          for (int c8 = 0; c8 < 32; c8 += 8) {
            const int d0 = c0 + c8;
            float f[8];
            if (wrow) {
#pragma unroll
              for (int k2 = 0; k2 < 8; ++k2) f[k2] = -__uint_as_float(raw[c8 + k2]);
            } else {
              float qv[8];
              unpack8(*reinterpret_cast<const uint4*>(sKQ + sw128_offset(64 + t, d0, kAtom128)), qv);
#pragma unroll
              for (int k2 = 0; k2 < 8; ++k2) f[k2] = et * qv[k2] - __uint_as_float(raw[c8 + k2]);
            }
            st_bf16x8(sWQ, sw128_offset(row, d0, kAtom128), f);
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars[kWqReady]);
        mbar_arrive(&bars[kKqFree]);
      }
      // the next chunk's v tile, loaded while MMA-c and MMA1 run
      if (!VW && n + 1 < nchunks && !p.writes_off) {
        fail = !wwait(&bars[kVFull], (n + 1) & 1, lim, status, s_abort);
        if (fail) { aborted = true; break; }
      }
      // ---- E2: Delta~^T -> SB (bf16, TMEM); O^T -> o
      fail = !wwait(&bars[kAccFull], n & 1, lim, status, s_abort);
      if (fail) { aborted = true; break; }
      tc_fence_after();
      if (ch == 0) {  // Delta~^T[c, t] = c_t Delta^T[c, t] -> bf16 into SB (A operand of MMA2)
        if (srow) {
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t raw[32];
            tmem_ld32_raw(tl + kACC + 32 * half, raw);
            tmem_wait_ld();
            uint32_t pk[16];
#pragma unroll
            for (int e4 = 0; e4 < 8; ++e4) {
              const float4 c4 = *reinterpret_cast<const float4*>(gt.c + 32 * half + 4 * e4);
              const float2 d0 = __fmul2_rn(make_float2(c4.x, c4.y),
                                           make_float2(__uint_as_float(raw[4 * e4]), __uint_as_float(raw[4 * e4 + 1])));
              const float2 d1 = __fmul2_rn(make_float2(c4.z, c4.w),
                                           make_float2(__uint_as_float(raw[4 * e4 + 2]), __uint_as_float(raw[4 * e4 + 3])));
              pk[2 * e4] = pack_bf16x2(d0.x, d0.y);
              pk[2 * e4 + 1] = pack_bf16x2(d1.x, d1.y);
            }
            tmem_st16_raw(tl + kSB + 16 * half, pk);
          }
          tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[kDlReady]);
      } else if (srow && p.write_o) {  // o[t0 + t, c] = O^T[c, t]; zero past the sequence's length
        __nv_bfloat16* op = p.o + (((size_t)b * T + t0) * H + h) * D + row;
        const int tmax = min(kC, seg_end - t0);
        // debug build: the first and the last token row this thread writes (the rows between
        // lie between them)
        const long long o0 = (((long long)b * T + t0) * H + h) * D + row, on = (long long)p.B * T * H * D;
        const bool o_ok = in_bounds(o0, on, status) && in_bounds(o0 + (long long)(tmax - 1) * H * D, on, status);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t raw[32];
          tmem_ld32_raw(tl + kACC + 64 + 32 * half, raw);
          tmem_wait_ld();
          if (!o_ok) {
          } else if (nv == kC) {  // a full chunk: every token valid and inside the tensor
#pragma unroll
            for (int e = 0; e < 32; ++e)
              op[(size_t)(32 * half + e) * H * D] = __float2bfloat16_rn(__uint_as_float(raw[e]));
          } else {  // the last chunk of a sequence
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int t = 32 * half + e;
              if (t < tmax) op[(size_t)t * H * D] = __float2bfloat16_rn(t < nv ? __uint_as_float(raw[e]) : 0.f);
            }
          }
        }
      }
    }
    // ---- the final state, and o past the last chunk
    if (!aborted && nchunks > 0) {
      const bool okf = wwait(&bars[kRsFull], (nchunks - 1) & 1, lim, status, s_abort);
      if (okf) {
        tc_fence_after();
        if (srow && S_end) {
#pragma unroll
          for (int pc = 0; pc < D / 64; ++pc) {
            const int c0 = ch * (D / 2) + 32 * pc;
            uint32_t raw[32];
            tmem_ld32_raw(tl + kRS + c0, raw);
            tmem_wait_ld();
            float4* dst = reinterpret_cast<float4*>(S_end + (size_t)row * D + c0);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              dst[e] = make_float4(__uint_as_float(raw[4 * e]), __uint_as_float(raw[4 * e + 1]),
                                   __uint_as_float(raw[4 * e + 2]), __uint_as_float(raw[4 * e + 3]));
          }
        }
      } else {
        aborted = true;
      }
    }
    if (!aborted) {
      if (nchunks == 0 && S_end) {  // no valid token: the end state is the start state
        for (int e = tid; e < D * D; e += kEG)
          S_end[e] = start_identity ? (e / D == e % D ? 1.f : 0.f) : (S_start ? S_start[e] : 0.f);
      }
      if (p.write_o && cta_ok) {  // o = 0 for the segment's tokens past its last chunk
        const int tz = tok0 + nchunks * kC;
        const __nv_bfloat16 zero = __float2bfloat16_rn(0.f);
        for (size_t e = tid; e < (size_t)max(seg_end - tz, 0) * D; e += kEG) {
          const int t = tz + (int)(e / D), c = (int)(e % D);
          const size_t oi = (((size_t)b * T + t) * H + h) * D + c;
          if (in_bounds((long long)oi, (long long)p.B * T * H * D, status)) p.o[oi] = zero;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------- residual write vectors
// rho_{t,l} = alpha_{t,l} r_{t,l} of every token, written as P~ (bf16, the layout of gain:
// [B, T, H, L - 1, D]) for the scan to load by TMA.  r_{t,0} = v_t - ShortConv anchor,
// r_{t,l} = chain step of r_{t,l-1} with gain g_{t,l}.  In a chunk whose decay is factored
// (chunk_decay_fast), P~ = e^{G_63 - G_t} rho; else P~ = rho.  Nothing here depends on the
// state, so every chunk of every chain runs at once, in CTAs of kPrepThreads threads over
// prep_tokens(D) tokens of one chunk.  A thread owns 8 channels of 2 consecutive tokens: it
// loads each v row of their ShortConv window once and the gain rows of up to kPrepLevels
// levels at the same time, so that enough 16-byte loads are in flight to keep HBM busy.
// Two tokens rather than four: 80 registers, six CTAs per SM, twice as many shorter CTAs,
// whose load, compute and store phases overlap better (the 130M-LM step 1.7% faster).
// Chunks wholly past a row's length are skipped (the scan never reads them); padded tokens
// of a chunk get zeros.  A launch covers chunks [nc0, nc0 + ncn) of every chain.
constexpr int kPrepThreads = 128;
constexpr int kPrepTPT = 2;     // consecutive tokens per thread
constexpr int kPrepLevels = 3;  // residual levels whose gain rows are loaded together
__host__ __device__ constexpr int prep_tokens(int D) { return kPrepThreads * kPrepTPT / (D / 8); }

__device__ __forceinline__ uint4 ldg16(const __nv_bfloat16* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }

template <int D, int CH, int WM>  // WM >= W: taps of a head in shared memory
__global__ void __launch_bounds__(kPrepThreads, WM <= 4 ? 6 : 3)
    residual_write_kernel(const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ gain,
                          const float* __restrict__ alpha, const float* __restrict__ gamma,
                          const float* __restrict__ conv_w, const int32_t* __restrict__ lengths,
                          const __nv_bfloat16* __restrict__ conv_state, __nv_bfloat16* __restrict__ ptil, int B,
                          int T, int H, int W, int m, int nc0, int ncn, int* status) {
  constexpr int CPT = D / 8;              // threads per token row
  constexpr int TPT = kPrepTPT;
  constexpr int PB = kC / prep_tokens(D);  // CTAs per chunk
  constexpr int NV = TPT + WM - 1;        // v rows of the threads' ShortConv window
  constexpr int LB = kPrepLevels;
  static_assert(PB >= 1 && kC % prep_tokens(D) == 0, "CTA tiling of a chunk");
  __shared__ float s_c[kC];  // e^{G_63 - G_t} (1 when the chunk's decay is not factored)
  __shared__ __align__(16) float s_taps[WM][D];  // ShortConv taps of the head, tap-major
  const int part = blockIdx.x % PB, cidx = blockIdx.x / PB;
  const int n = nc0 + cidx % ncn, bh = cidx / ncn, b = bh / H, h = bh % H;
  if (!in_bounds(bh, (long long)B * H, status)) return;  // debug build: a chain outside the batch
  const int len = lengths ? min(max(lengths[b], 0), T) : T;
  const int t0 = n * kC;
  if (t0 >= len) return;
  const int tid = threadIdx.x, lane = tid & 31;
  const int c8 = (tid % CPT) * 8, i0 = part * prep_tokens(D) + (tid / CPT) * TPT;
  const size_t row0 = ((size_t)b * T + t0 + i0) * H + h;  // (token, head) row of the first token
  // every load first: the v window, then the gain rows and alphas of the first LB levels
  uint4 vr[NV];
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int t = t0 + i0 - (WM - 1) + j;
    const size_t vi = (((size_t)b * T + t) * H + h) * D + c8;
    const size_t ci = (((size_t)b * H + h) * (W - 1) + (W - 1 + t)) * D + c8;
    if (t >= 0)
      vr[j] = t < T && in_bounds((long long)vi + 7, (long long)B * T * H * D, status) ? ldg16(v + vi)
                                                                                       : make_uint4(0, 0, 0, 0);
    else  // before token 0: the sequence's ShortConv history (rows W - 1 + t), else zero
      vr[j] = (conv_state && t >= 1 - W && in_bounds((long long)ci + 7, (long long)B * H * (W - 1) * D, status))
                  ? ldg16(conv_state + ci)
                  : make_uint4(0, 0, 0, 0);
  }
  uint4 gr[LB][TPT];
  float al[LB][TPT];
  auto load_levels = [&](int l0) {
#pragma unroll
    for (int j = 0; j < LB; ++j)
#pragma unroll
      for (int a = 0; a < TPT; ++a) {
        const size_t th = row0 + (size_t)a * H;
        const bool ok = l0 + j < m && t0 + i0 + a < len &&
                        in_bounds((long long)((th * m + l0 + j) * D + c8) + 7, (long long)B * T * H * m * D, status);
        gr[j][a] = ok ? ldg16(gain + (th * m + l0 + j) * D + c8) : make_uint4(0, 0, 0, 0);
        al[j][a] = ok ? __ldg(alpha + th * m + l0 + j) : 0.f;
      }
  };
  load_levels(0);
  for (int e = tid; e < WM * D; e += kPrepThreads) {
    const int w = e / D, c = e % D;
    s_taps[w][c] = w < W && in_bounds(((long long)h * D + c) * W + w, (long long)H * D * W, status)
                       ? __ldg(conv_w + ((size_t)h * D + c) * W + w)
                       : 0.f;
  }
  if (tid < 32) {
    const int nv = min(kC, len - t0);
    float gl[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int t = 2 * lane + e;
      const size_t gi = ((size_t)b * T + t0 + t) * H + h;
      gl[e] = t < nv && in_bounds((long long)gi, (long long)B * T * H, status) ? __ldg(gamma + gi) : 1.f;
    }
    float G0, G1, G63;
    chunk_log_decay(gl[0], gl[1], lane, G0, G1, G63);
    const bool fast = chunk_decay_fast(G63);
    s_c[2 * lane] = fast ? __expf(G63 - G0) : 1.f;
    s_c[2 * lane + 1] = fast ? __expf(G63 - G1) : 1.f;
  }
  __syncthreads();  // s_taps, s_c
  float r[TPT][8];
  {
    auto tap8 = [&](int w, float* t8) {
      const float4 x = *reinterpret_cast<const float4*>(&s_taps[w][c8]);
      const float4 y = *reinterpret_cast<const float4*>(&s_taps[w][c8 + 4]);
      t8[0] = x.x; t8[1] = x.y; t8[2] = x.z; t8[3] = x.w; t8[4] = y.x; t8[5] = y.y; t8[6] = y.z; t8[7] = y.w;
    };
#pragma unroll
    for (int a = 0; a < TPT; ++a) {
      float vt[8], tw[8];
      unpack8(vr[a + WM - 1], vt);
      tap8(0, tw);
#pragma unroll
      for (int e = 0; e < 8; ++e) r[a][e] = vt[e] - tw[e] * vt[e];
#pragma unroll
      for (int w = 1; w < WM; ++w) {
        if (w < W) {
          float vw[8];
          unpack8(vr[a + WM - 1 - w], vw);
          tap8(w, tw);
#pragma unroll
          for (int e = 0; e < 8; ++e) r[a][e] -= tw[e] * vw[e];
        }
      }
    }
  }
  float cs[TPT];
#pragma unroll
  for (int a = 0; a < TPT; ++a) cs[a] = s_c[i0 + a];
  for (int l0 = 0; l0 < m; l0 += LB) {
    if (l0 > 0) load_levels(l0);
#pragma unroll
    for (int j = 0; j < LB; ++j) {
      if (l0 + j < m) {
#pragma unroll
        for (int a = 0; a < TPT; ++a) {
          const int t = t0 + i0 + a;
          if (t < T) {
            float gv[8], rho[8];
            unpack8(gr[j][a], gv);
            const float sc = cs[a] * al[j][a];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              r[a][e] = chain_step(r[a][e], gv[e], CH);
              rho[e] = sc * r[a][e];
            }
            uint4 u = make_uint4(0, 0, 0, 0);
            if (t < len) {
              u.x = pack_bf16x2(rho[0], rho[1]);
              u.y = pack_bf16x2(rho[2], rho[3]);
              u.z = pack_bf16x2(rho[4], rho[5]);
              u.w = pack_bf16x2(rho[6], rho[7]);
            }
            const size_t pi = ((row0 + (size_t)a * H) * m + l0 + j) * D + c8;
            if (in_bounds((long long)pi + 7, (long long)B * T * H * m * D, status))
              *reinterpret_cast<uint4*>(ptil + pi) = u;
          }
        }
      }
    }
  }
}

// ---------------------------------------------------------------- segment fold
// The start states of the segments of a cut sequence.  A segment maps its start state S
// to S M_p + N_p (M_p: the scan of the segment from the identity with the writes off;
// N_p: from a zero start, or from S0 for the first segment, whose N is therefore already
// its exact end state).  Sst[1] = N_0, Sst[p] = Sst[p-1] M_{p-1} + N_{p-1}.  Rows of the
// state are independent, so one block carries one row through all segments.
template <int D>
__global__ void __launch_bounds__(D) segment_fold_kernel(const float* N, const float* M, float* Sst, int P) {
  __shared__ float srow[D];
  const int c = blockIdx.x, j = threadIdx.x;
  const size_t bh = blockIdx.y, DD = (size_t)D * D;
  float x = N[(bh * P) * DD + (size_t)c * D + j];
  Sst[(bh * P + 1) * DD + (size_t)c * D + j] = x;
  for (int q = 2; q < P; ++q) {
    srow[j] = x;
    __syncthreads();
    const float* m = M + (bh * P + q - 1) * DD;
    float acc = N[(bh * P + q - 1) * DD + (size_t)c * D + j];
#pragma unroll 8
    for (int i = 0; i < D; ++i) acc += srow[i] * m[(size_t)i * D + j];
    __syncthreads();
    x = acc;
    Sst[(bh * P + q) * DD + (size_t)c * D + j] = x;
  }
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

// Segments of a long sequence over few chains: planned for the 148 SMs of a B200 on every
// device, so that the plan (and with it the rounding of the results and the workspace size)
// is a function of the sizes alone.  A plan cuts only sequences of at least 32 chunks whose
// chains fill under half of those SMs, into segments of at least 16 chunks.
struct SegPlan {
  int P, Ts;
};
SegPlan plan_segments(int B, int T, int H) {
  const int nc = (T + kC - 1) / kC, chains = B * H;
  if (2 * chains > kPlanSMs || nc < 32) return {1, nc * kC};
  const int P = std::min(kPlanSMs / chains, nc / 16);
  if (P < 2) return {1, nc * kC};
  const int cps = (nc + P - 1) / P;  // chunks per segment
  return {(nc + cps - 1) / cps, cps * kC};
}

// Two halves in time.  When the chains of a sequence leave SMs idle during the scan (and
// the sequence is not cut into segments), the scan runs in two launches: chunks
// [0, nA), then chunks [nA, NC) from the first launch's end states.  The residual write
// of the second half runs beside the first scan launch, on the SMs that launch leaves
// idle, so only the first half's residual write precedes the scan.  The first launch is
// cut where that write should end about when the first scan does.  On the idle SMs the
// write of one chunk of every chain takes about x = 0.28 chains / idle SMs chunk times of
// the scan, so nA = NC x / (1 + x), at least a quarter of the chunks.  The constant is
// measured on the 130M-LM layer (96 chains): its step time is lowest at nA = 11 of 32
// chunks (x = 0.52), 2% below nA = 16, and within 1% from 10 to 13.
constexpr int kSplitIdleSMs = 24;  // SMs the chains must leave idle
constexpr double kSplitWriteCost = 0.28;
struct TimeSplit {
  bool on;
  int nA;  // chunks of the first half
};
TimeSplit time_split(int B, int T, int H, int L) {
  const int nc = (T + kC - 1) / kC;
  const bool on = L > 1 && plan_segments(B, T, H).P == 1 && B * H + kSplitIdleSMs <= kPlanSMs && nc >= 8;
  const int chains = B * H, idle = std::max(kPlanSMs - chains, 1);
  const double x = kSplitWriteCost * chains / idle;
  const int nA = (int)std::ceil(nc * x / (1.0 + x));
  return {on, std::max((nc + 3) / 4, std::min(nc - 1, nA))};
}

// The side stream of a device for the two halves: the first scan launch, then the second
// half's residual write as a programmatic dependent launch, which starts once every CTA of
// the scan holds its SM (so it takes only the SMs the scan leaves idle) and does not wait
// for the scan to finish.  Fork and join through events on the caller's stream; the join
// event, recorded after both, completes once both have.  Created on first use; a mutex
// keeps the record / wait sequences of concurrent callers from interleaving.
struct SideStreams {
  cudaStream_t hi = nullptr;
  cudaEvent_t forked = nullptr, joined = nullptr;
};
constexpr int kMaxSideDevices = 64;
std::mutex g_side_mutex;
SideStreams g_side[kMaxSideDevices];

cudaError_t side_streams(SideStreams** out) {  // with g_side_mutex held
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxSideDevices) return cudaErrorInvalidDevice;
  SideStreams& x = g_side[dev];
  if (!x.hi) {
    int least = 0, greatest = 0;
    if ((e = cudaDeviceGetStreamPriorityRange(&least, &greatest)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&x.forked, cudaEventDisableTiming)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&x.joined, cudaEventDisableTiming)) != cudaSuccess) return e;
    if ((e = cudaStreamCreateWithPriority(&x.hi, cudaStreamNonBlocking, greatest)) != cudaSuccess) return e;
  }
  *out = &x;
  return cudaSuccess;
}

// The workspace: P~ (bf16, the shape of gain), 256-byte aligned, then the segments' states
// or the two halves' hand-over states.
size_t ptil_bytes(int B, int T, int H, int D, int L) {
  const size_t b = (size_t)B * T * H * (L - 1) * D * 2;
  return (b + 255) & ~size_t(255);
}

template <int D, int NU>
cudaError_t set_smem_attr() {
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(prism_scan_kernel<D, NU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    Lay<D, NU>::ALLOC);
  });
  return attr_err;
}

// The scan launches of one call (the residual write vectors are in the workspace): one
// launch, two halves, or the segments' three launches and fold.  NU: U slots (3 when a
// chunk has four or more residual directions, so that their loads run ahead).
template <int D, int NU>
cudaError_t launch_scans(const ScanParams& p, cudaStream_t stream, const CUtensorMap& mq, const CUtensorMap& mk,
                         const CUtensorMap& mu, const CUtensorMap& mv, const CUtensorMap& mg, int m,
                         const TimeSplit& split,
                         const std::function<cudaError_t(int, int, cudaStream_t, bool)>& residual) {
  using Ly = Lay<D, NU>;
  const cudaError_t attr_err = set_smem_attr<D, NU>();
  if (attr_err != cudaSuccess) return attr_err;
  const int NC = (p.T + kC - 1) / kC;
  const SegPlan plan = plan_segments(p.B, p.T, p.H);
  ScanArgs a{static_cast<const __nv_bfloat16*>(p.q), static_cast<const __nv_bfloat16*>(p.k),
             static_cast<const __nv_bfloat16*>(p.v), p.gamma, p.beta, p.alpha, p.conv_w, p.S0, p.lengths,
             static_cast<__nv_bfloat16*>(p.o), p.S_final, nullptr, nullptr, p.B, p.T, p.H, p.W, m,
             plan.P, plan.Ts, 0, 1, 0, -1, p.status, p.spin_limit};
  const int grid = p.B * p.H * plan.P;
  if (split.on) {
    // the two halves as segments 0 and 1 of a 2-segment plan, one launch each; the first
    // writes its end states to hand[b, h, 1], where the second reads its start states
    float* hand = reinterpret_cast<float*>(static_cast<char*>(p.workspace) + ptil_bytes(p.B, p.T, p.H, D, p.L));
    ScanArgs aA = a;
    aA.P = 2;
    aA.Ts = split.nA * kC;
    aA.seg_only = 0;
    aA.S_out = hand + (size_t)D * D;
    ScanArgs aB = aA;
    aB.seg_only = 1;
    aB.S_out = nullptr;
    aB.S_in = hand;
    {
      std::lock_guard<std::mutex> lock(g_side_mutex);
      SideStreams* ss = nullptr;
      cudaError_t e = side_streams(&ss);
      if (e == cudaSuccess) e = cudaEventRecord(ss->forked, stream);
      if (e == cudaSuccess) e = cudaStreamWaitEvent(ss->hi, ss->forked, 0);
      if (e != cudaSuccess) return e;
      prism_scan_kernel<D, NU><<<p.B * p.H, kThreads, Ly::ALLOC, ss->hi>>>(mq, mk, mu, mv, mg, aA);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
      if ((e = residual(split.nA, NC - split.nA, ss->hi, true)) != cudaSuccess) return e;
      if ((e = cudaEventRecord(ss->joined, ss->hi)) != cudaSuccess) return e;
      if ((e = cudaStreamWaitEvent(stream, ss->joined, 0)) != cudaSuccess) return e;
    }
    prism_scan_kernel<D, NU><<<p.B * p.H, kThreads, Ly::ALLOC, stream>>>(mq, mk, mu, mv, mg, aB);
    return cudaGetLastError();
  }
  if (plan.P == 1) {
    prism_scan_kernel<D, NU><<<grid, kThreads, Ly::ALLOC, stream>>>(mq, mk, mu, mv, mg, a);
    return cudaGetLastError();
  }
  // a long sequence over few chains: P segments side by side, three scans and a fold
  const size_t seg_states = (size_t)p.B * p.H * plan.P * D * D;
  float* wsN = reinterpret_cast<float*>(static_cast<char*>(p.workspace) + ptil_bytes(p.B, p.T, p.H, D, p.L));
  float* wsM = wsN + seg_states;
  float* wsS = wsM + seg_states;
  ScanArgs aN = a;  // each segment from a zero start (the first from S0): N_p
  aN.S_out = wsN;
  aN.write_o = 0;
  aN.S_final = nullptr;
  prism_scan_kernel<D, NU><<<grid, kThreads, Ly::ALLOC, stream>>>(mq, mk, mu, mv, mg, aN);
  ScanArgs aM = aN;  // the transitions alone from the identity: M_p
  aM.S_out = wsM;
  aM.s_in_identity = 1;
  aM.writes_off = 1;
  aM.m = 0;
  prism_scan_kernel<D, NU><<<grid, kThreads, Ly::ALLOC, stream>>>(mq, mk, mu, mv, mg, aM);
  segment_fold_kernel<D><<<dim3(D, p.B * p.H), D, 0, stream>>>(wsN, wsM, wsS, plan.P);
  ScanArgs aF = a;  // every segment again from its exact start state: o and S_final
  aF.S_in = wsS;
  prism_scan_kernel<D, NU><<<grid, kThreads, Ly::ALLOC, stream>>>(mq, mk, mu, mv, mg, aF);
  return cudaGetLastError();
}

template <int D, int CH>
cudaError_t launch_dc(const ScanParams& p, cudaStream_t stream) {
  const cuuint64_t B = p.B, T = p.T, H = p.H;
  const int m = p.L - 1;
  CUtensorMap mq, mk, mu, mv, mg;
  const cuuint64_t dims4[4] = {(cuuint64_t)D, H, T, B};
  const cuuint64_t str4[3] = {(cuuint64_t)D * 2, H * D * 2, T * H * D * 2};
  const cuuint32_t box4[4] = {64, 1, 64, 1};
  const cuuint32_t box_v[4] = {64, 1, 64, 1};
  if (!encode(&mq, p.q, 4, dims4, str4, box4) || !encode(&mk, p.k, 4, dims4, str4, box4) ||
      !encode(&mv, p.v, 4, dims4, str4, box_v))
    return cudaErrorInvalidValue;
  __nv_bfloat16* ptil = static_cast<__nv_bfloat16*>(p.workspace);  // P~, the layout of gain
  const int NC = (p.T + kC - 1) / kC;
  const TimeSplit split = time_split(p.B, p.T, p.H, p.L);
  const __nv_bfloat16* vv = static_cast<const __nv_bfloat16*>(p.v);
  const __nv_bfloat16* gg = static_cast<const __nv_bfloat16*>(p.gain);
  const __nv_bfloat16* cs = static_cast<const __nv_bfloat16*>(p.conv_state);
  // the residual write of chunks [nc0, nc0 + ncn); `dependent`: as a programmatic dependent
  // launch of the kernel before it on the stream
  auto residual = [&](int nc0, int ncn, cudaStream_t st, bool dependent) -> cudaError_t {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.B * p.H * ncn * (kC / prep_tokens(D)));
    cfg.blockDim = dim3(kPrepThreads);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = dependent ? 1 : 0;
    if (p.W <= 4)
      return cudaLaunchKernelEx(&cfg, residual_write_kernel<D, CH, 4>, vv, gg, p.alpha, p.gamma, p.conv_w,
                                p.lengths, cs, ptil, p.B, p.T, p.H, p.W, m, nc0, ncn, p.status);
    return cudaLaunchKernelEx(&cfg, residual_write_kernel<D, CH, PRISM_MAX_W>, vv, gg, p.alpha, p.gamma, p.conv_w,
                              p.lengths, cs, ptil, p.B, p.T, p.H, p.W, m, nc0, ncn, p.status);
  };
  if (m > 0) {
    const cuuint64_t dims5[5] = {(cuuint64_t)D, (cuuint64_t)m, H, T, B};
    const cuuint64_t str5[4] = {(cuuint64_t)D * 2, (cuuint64_t)m * D * 2, H * m * D * 2, T * H * m * D * 2};
    const cuuint32_t box5[5] = {64, 1, 1, 64, 1};
    if (!encode(&mu, p.u, 5, dims5, str5, box5) || !encode(&mg, ptil, 5, dims5, str5, box5))
      return cudaErrorInvalidValue;
    const cudaError_t e = residual(0, split.on ? split.nA : NC, stream, false);
    if (e != cudaSuccess) return e;
    if (p.split_event) {
      const cudaError_t e = cudaEventRecord(static_cast<cudaEvent_t>(p.split_event), stream);
      if (e != cudaSuccess) return e;
    }
  } else {
    mu = mk;
    mg = mk;
  }
  if (m >= 4) return launch_scans<D, 3>(p, stream, mq, mk, mu, mv, mg, m, split, residual);
  return launch_scans<D, 2>(p, stream, mq, mk, mu, mv, mg, m, split, residual);
}

template <int D>
cudaError_t launch_d(const ScanParams& p, cudaStream_t stream) {
  if (p.L > 1 && p.chain == PRISM_CHAIN_GELU) return launch_dc<D, PRISM_CHAIN_GELU>(p, stream);
  return launch_dc<D, PRISM_CHAIN_LINEAR>(p, stream);
}

}  // namespace

bool chunk_scan_supported(int d_k, int d_v, int L, int W, int chunk, int dtype) {
  return dtype == PRISM_BF16 && chunk == kC && d_k == d_v && (d_k == 64 || d_k == 128) && L >= 1 &&
         L <= PRISM_MAX_L && W >= 1 && W <= PRISM_MAX_W;
}

size_t chunk_scan_workspace_bytes(int B, int T, int H, int D, int L) {
  const SegPlan plan = plan_segments(B, T, H);
  const size_t states = plan.P > 1 ? 3 * (size_t)B * H * plan.P * D * D
                                   : (time_split(B, T, H, L).on ? 2 * (size_t)B * H * D * D : 0);
  return ptil_bytes(B, T, H, D, L) + states * sizeof(float);
}

int chunk_scan_split_chunks(int B, int T, int H, int L) {
  const TimeSplit s = time_split(B, T, H, L);
  return s.on ? s.nA : 0;
}

int chunk_scan_launches(int B, int T, int H, int L) {
  if (time_split(B, T, H, L).on) return 4;  // two residual-write launches, two scan launches
  return (L > 1 ? 1 : 0) + (plan_segments(B, T, H).P == 1 ? 1 : 4);
}

cudaError_t launch_chunk_scan(const ScanParams& p, cudaStream_t stream) {
  if (p.d_k == 128) return launch_d<128>(p, stream);
  if (p.d_k == 64) return launch_d<64>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace prism
