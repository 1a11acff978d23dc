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
// shuffles.  Blocks of 64 threads carry 64 / LPR rows of one (batch, head), so a
// handful of (batch, head) chains still spreads over many SMs.
//
// The loop over tokens is sequential, so its inputs must be on-chip when it gets
// to them: tiles of TT tokens (k, q, u of the head; v and gains of the block's
// rows; gamma, beta, alpha) stream into double-buffered shared memory with
// cp.async while the previous tile is being scanned.
#include <algorithm>

#include "common.cuh"

namespace prism {
namespace {

constexpr int kBlock = 64;
constexpr int kTileBytes = 48 * 1024;  // per buffer, at most

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

// 4 consecutive elements from shared memory as fp32
template <typename T>
__device__ __forceinline__ float4 ld4_smem(const T* p);
template <>
__device__ __forceinline__ float4 ld4_smem<float>(const float* p) { return *reinterpret_cast<const float4*>(p); }
template <>
__device__ __forceinline__ float4 ld4_smem<__nv_bfloat16>(const __nv_bfloat16* p) {
  const uint2 w = *reinterpret_cast<const uint2*>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.y));
  return make_float4(a.x, a.y, b.x, b.y);
}

template <int LPR>
__device__ __forceinline__ float row_sum(float x) {
#pragma unroll
  for (int off = LPR / 2; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

// Shared-memory layout of one tile of TT tokens (byte offsets, each 16-byte aligned).
struct TileLayout {
  int TT, dk, m, rpb, es;
  int off_k, off_q, off_u, off_v, off_g, off_gam, off_bet, off_al, bytes;
  __host__ __device__ TileLayout(int TT_, int dk_, int m_, int rpb_, int es_)
      : TT(TT_), dk(dk_), m(m_), rpb(rpb_), es(es_) {
    auto al16 = [](int x) { return (x + 15) & ~15; };
    off_k = 0;
    off_q = al16(off_k + TT * dk * es);
    off_u = al16(off_q + TT * dk * es);
    off_v = al16(off_u + TT * m * dk * es);
    off_g = al16(off_v + TT * rpb * es);
    off_gam = al16(off_g + TT * m * rpb * es);
    off_bet = al16(off_gam + TT * 4);
    off_al = al16(off_bet + TT * 4);
    bytes = al16(off_al + TT * m * 4);
  }
};

template <typename T>
int tile_tokens(int dk, int m, int rpb, int budget) {
  for (int TT = 32; TT > 1; TT >>= 1)
    if (TileLayout(TT, dk, m, rpb, sizeof(T)).bytes <= budget) return TT;
  return 1;
}

// CH: residual chain step (PRISM_CHAIN_LINEAR or PRISM_CHAIN_GELU), fixed at compile time.
template <typename T, int LPR, int EPL, int CH>
__global__ void __launch_bounds__(kBlock) recurrent_scan_kernel(ScanParams p, int TT) {
  constexpr int RPB = kBlock / LPR;  // rows per block
  extern __shared__ __align__(16) uint8_t smem[];
  const int tid = threadIdx.x;
  const int j = tid % LPR;  // lane within the row: owns d_k elements 4 j + 4 LPR g + (0..3), g < EPL / 4
  const int lrow = tid / LPR;
  const int row0 = blockIdx.x * RPB;
  const int row = row0 + lrow;
  const int h = blockIdx.y, b = blockIdx.z;
  const int T_ = p.T, H = p.H, dk = p.d_k, dv = p.d_v, m = p.L - 1, W = p.W;
  const bool row_ok = row < dv;
  const int c = row_ok ? row : dv - 1;  // idle rows shadow the last real row (no stores)
  // debug build: a block outside the batch or the heads reads and writes nothing
  const bool blk_ok = in_bounds(b, p.B, p.status) && in_bounds(h, H, p.status);
  const int len = !blk_ok ? 0 : p.lengths ? min(max(p.lengths[b], 0), T_) : T_;
  const long long n_o = (long long)p.B * T_ * H * dv;
  const TileLayout L(TT, dk, m, RPB, (int)sizeof(T));
  const int nrows = min(RPB, dv - row0);  // rows of this block that exist

  const T* q = static_cast<const T*>(p.q);
  const T* k = static_cast<const T*>(p.k);
  const T* v = static_cast<const T*>(p.v);
  const T* u = static_cast<const T*>(p.u);
  const T* g = static_cast<const T*>(p.gain);
  T* o = static_cast<T*>(p.o);

  // cooperative async load of tile `ti` (tokens ti*TT ..) into buffer `buf`
  auto load_tile = [&](int ti, int buf) {
    uint8_t* base = smem + buf * L.bytes;
    const int t0 = ti * TT, nt = min(TT, len - t0);
    // debug build: the tile's last (token, head) row lies inside the tensors
    if (nt > 0 && !in_bounds(((long long)b * T_ + t0 + nt - 1) * H + h, (long long)p.B * T_ * H, p.status)) return;
    const int vec = 16 / (int)sizeof(T);  // elements per 16-byte chunk
    const int kchunks = dk / vec;
    // k, q: [nt][dk]
    for (int e = tid; e < nt * kchunks; e += kBlock) {
      const int i = e / kchunks, cc = e % kchunks;
      const size_t tok = ((size_t)b * T_ + t0 + i) * H + h;
      cp_async16(base + L.off_k + (i * dk + cc * vec) * sizeof(T), k + tok * dk + cc * vec);
      cp_async16(base + L.off_q + (i * dk + cc * vec) * sizeof(T), q + tok * dk + cc * vec);
    }
    // u: [nt][m][dk] (contiguous per token)
    for (int e = tid; e < nt * m * kchunks; e += kBlock) {
      const int i = e / (m * kchunks), r = e % (m * kchunks);
      const size_t tok = ((size_t)b * T_ + t0 + i) * H + h;
      cp_async16(base + L.off_u + ((size_t)i * m * dk + r * vec) * sizeof(T), u + tok * m * dk + r * vec);
    }
    // v, gains of this block's rows: [nt][rpb], [nt][m][rpb] (a block's rows are contiguous:
    // 16-byte copies when the whole block exists, element copies at a ragged d_v edge)
    const int rbytes = RPB * (int)sizeof(T);
    if (nrows == RPB && rbytes % 16 == 0) {
      const int rch = rbytes / 16;
      for (int e = tid; e < nt * (1 + m) * rch; e += kBlock) {
        const int i = e / ((1 + m) * rch), r = e % ((1 + m) * rch), l = r / rch, cc = r % rch;
        const size_t tok = ((size_t)b * T_ + t0 + i) * H + h;
        const T* src = (l == 0 ? v + tok * dv : g + (tok * m + (l - 1)) * dv) + row0 + cc * (16 / (int)sizeof(T));
        uint8_t* dst = base + (l == 0 ? L.off_v + i * rbytes : L.off_g + (i * m + (l - 1)) * rbytes) + cc * 16;
        cp_async16(dst, src);
      }
    } else {
      for (int e = tid; e < nt * (1 + m) * nrows; e += kBlock) {
        const int i = e / ((1 + m) * nrows), r = e % ((1 + m) * nrows), l = r / nrows, cr = r % nrows;
        const size_t tok = ((size_t)b * T_ + t0 + i) * H + h;
        const T* src = l == 0 ? v + tok * dv + row0 + cr : g + (tok * m + (l - 1)) * dv + row0 + cr;
        T* dst = reinterpret_cast<T*>(base + (l == 0 ? L.off_v : L.off_g)) +
                 (l == 0 ? i * RPB + cr : (i * m + (l - 1)) * RPB + cr);
        if (sizeof(T) == 4)
          cp_async4(dst, src);
        else
          *dst = *src;  // 2-byte elements at a ragged edge: plain copy (cp.async needs >= 4 bytes)
      }
    }
    // gates: gamma, beta [nt], alpha [nt][m]
    for (int e = tid; e < nt * (2 + m); e += kBlock) {
      const int i = e / (2 + m), r = e % (2 + m);
      const size_t tok = ((size_t)b * T_ + t0 + i) * H + h;
      const float* src = r == 0 ? p.gamma + tok : (r == 1 ? p.beta + tok : p.alpha + tok * m + (r - 2));
      float* dst = reinterpret_cast<float*>(base + (r == 0 ? L.off_gam : (r == 1 ? L.off_bet : L.off_al))) +
                   (r < 2 ? i : i * m + (r - 2));
      cp_async4(dst, src);
    }
  };

  float w[PRISM_MAX_W];
#pragma unroll
  for (int i = 0; i < PRISM_MAX_W; ++i) w[i] = (i < W) ? p.conv_w[((size_t)h * dv + c) * W + i] : 0.f;
  float hist[PRISM_MAX_W];  // hist[i] = v_{t-1-i}[c]; before token 0 the sequence's history (or zero)
  const T* cs = static_cast<const T*>(p.conv_state);
#pragma unroll
  for (int i = 0; i < PRISM_MAX_W; ++i)
    hist[i] = (cs && blk_ok && i < W - 1) ? ld1<T>(cs + (((size_t)b * H + h) * (W - 1) + (W - 2 - i)) * dv + c) : 0.f;

  float s[EPL];
  const size_t sbase = (((size_t)b * H + h) * dv + c) * dk + 4 * j;
#pragma unroll
  for (int e = 0; e < EPL; e += 4) {
    const float4 f = p.S0 && blk_ok ? __ldg(reinterpret_cast<const float4*>(p.S0 + sbase + e * LPR))
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
    s[e] = f.x; s[e + 1] = f.y; s[e + 2] = f.z; s[e + 3] = f.w;
  }

  const int NCr = (T_ + kBwdChunk - 1) / kBwdChunk;  // chunk-boundary record slots: NCr + 1
  float* rec_row = p.rec_states ? p.rec_states + (((size_t)b * H + h) * (NCr + 1) * dv + c) * dk + 4 * j : nullptr;
  if (rec_row && row_ok) {
#pragma unroll
    for (int e = 0; e < EPL; e += 4)
      *reinterpret_cast<float4*>(rec_row + e * LPR) = make_float4(s[e], s[e + 1], s[e + 2], s[e + 3]);
  }

  const int ntiles = (len + TT - 1) / TT;
  if (ntiles > 0) load_tile(0, 0);
  cp_async_commit();
  for (int ti = 0; ti < ntiles; ++ti) {
    const int buf = ti & 1;
    if (ti + 1 < ntiles) load_tile(ti + 1, buf ^ 1);
    cp_async_commit();
    cp_async_wait_1();  // tile ti has landed (the next may still be in flight)
    __syncthreads();
    const uint8_t* base = smem + buf * L.bytes;
    const T* sk_ = reinterpret_cast<const T*>(base + L.off_k);
    const T* sq_ = reinterpret_cast<const T*>(base + L.off_q);
    const T* su_ = reinterpret_cast<const T*>(base + L.off_u);
    const T* sv_ = reinterpret_cast<const T*>(base + L.off_v);
    const T* sg_ = reinterpret_cast<const T*>(base + L.off_g);
    const float* sgam = reinterpret_cast<const float*>(base + L.off_gam);
    const float* sbet = reinterpret_cast<const float*>(base + L.off_bet);
    const float* sal = reinterpret_cast<const float*>(base + L.off_al);
    const int t0 = ti * TT, nt = min(TT, len - t0);
    const int cr = row_ok ? lrow : 0;
    for (int i = 0; i < nt; ++i) {
      const T* kk = sk_ + i * dk + 4 * j;
      float sk = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; e += 4) {
        const float4 f = ld4_smem<T>(kk + e * LPR);
        sk += s[e] * f.x + s[e + 1] * f.y + s[e + 2] * f.z + s[e + 3] * f.w;
      }
      sk = row_sum<LPR>(sk);

      // ShortConv anchor and anchor residual
      const float vt = to_f<T>(sv_[i * RPB + cr]);
      float a = w[0] * vt;
#pragma unroll
      for (int z = 1; z < PRISM_MAX_W; ++z) a += w[z] * hist[z - 1];
      float r = vt - a;
#pragma unroll
      for (int z = PRISM_MAX_W - 1; z > 0; --z) hist[z] = hist[z - 1];
      hist[0] = vt;

      // gated delta write: gamma S (I - beta k k^T) + beta v k^T
      const float gam = sgam[i];
      const float psi = vt - gam * sk;
      const float coef = sbet[i] * psi;
      if (p.rec_psi && row_ok && j == 0) p.rec_psi[(((size_t)b * T_ + t0 + i) * H + h) * dv + c] = psi;
#pragma unroll
      for (int e = 0; e < EPL; e += 4) {
        const float4 f = ld4_smem<T>(kk + e * LPR);
        s[e] = gam * s[e] + coef * f.x;
        s[e + 1] = gam * s[e + 1] + coef * f.y;
        s[e + 2] = gam * s[e + 2] + coef * f.z;
        s[e + 3] = gam * s[e + 3] + coef * f.w;
      }
      // rank-m residual write
      for (int l = 0; l < m; ++l) {
        r = chain_step(r, to_f<T>(sg_[(i * m + l) * RPB + cr]), CH);
        const float rho = sal[i * m + l] * r;
        const T* uu = su_ + ((size_t)i * m + l) * dk + 4 * j;
#pragma unroll
        for (int e = 0; e < EPL; e += 4) {
          const float4 f = ld4_smem<T>(uu + e * LPR);
          s[e] += rho * f.x;
          s[e + 1] += rho * f.y;
          s[e + 2] += rho * f.z;
          s[e + 3] += rho * f.w;
        }
      }
      const int tn = t0 + i + 1;  // tokens done
      if (rec_row && row_ok && (tn % kBwdChunk == 0 || tn == len)) {  // a chunk boundary
        float* dst = rec_row + (size_t)((tn + kBwdChunk - 1) / kBwdChunk) * dv * dk;
#pragma unroll
        for (int e = 0; e < EPL; e += 4)
          *reinterpret_cast<float4*>(dst + e * LPR) = make_float4(s[e], s[e + 1], s[e + 2], s[e + 3]);
      }
      if (p.states && row_ok) {  // S_t of this row, for the backward pass
        float* dst = p.states + ((((size_t)b * H + h) * T_ + t0 + i) * dv + c) * dk + 4 * j;
#pragma unroll
        for (int e = 0; e < EPL; e += 4)
          *reinterpret_cast<float4*>(dst + e * LPR) = make_float4(s[e], s[e + 1], s[e + 2], s[e + 3]);
      }
      if (o) {  // no readout in the recording launches of the backward
        const T* qq = sq_ + i * dk + 4 * j;
        float oq = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; e += 4) {
          const float4 f = ld4_smem<T>(qq + e * LPR);
          oq += s[e] * f.x + s[e + 1] * f.y + s[e + 2] * f.z + s[e + 3] * f.w;
        }
        oq = row_sum<LPR>(oq);
        const size_t oi = (((size_t)b * T_ + t0 + i) * H + h) * dv + c;
        if (row_ok && j == 0 && in_bounds((long long)oi, n_o, p.status)) st1<T>(o + oi, oq);
      }
    }
    __syncthreads();  // the buffer is refilled next iteration
  }
  cp_async_wait_0();
  if (o && row_ok && j == 0 && blk_ok)
    for (int t = len; t < T_; ++t) {
      const size_t oi = (((size_t)b * T_ + t) * H + h) * dv + c;
      if (in_bounds((long long)oi, n_o, p.status)) st1<T>(o + oi, 0.f);
    }
  if (row_ok && p.S_final && blk_ok) {
#pragma unroll
    for (int e = 0; e < EPL; e += 4)
      *reinterpret_cast<float4*>(p.S_final + sbase + e * LPR) = make_float4(s[e], s[e + 1], s[e + 2], s[e + 3]);
  }
}

int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      n = 148;
  }
  return n;
}

template <typename T, int LPR, int EPL, int CH>
cudaError_t launch_chain(const ScanParams& p, cudaStream_t stream) {
  constexpr int RPB = kBlock / LPR;
  // Every block walks the whole sequence, so all of them must be resident at once (a
  // second wave would double the time): the double-buffered tile shrinks with the
  // blocks each SM has to hold (about 200 KB of shared memory per SM in all).
  dim3 grid((p.d_v + RPB - 1) / RPB, p.H, p.B);
  const long long nblocks = (long long)grid.x * grid.y * grid.z;
  const long long per_sm = (nblocks + sm_count() - 1) / sm_count();
  const int budget = (int)std::min<long long>(kTileBytes, (200 * 1024) / (2 * std::max<long long>(per_sm, 1)));
  const int TT = tile_tokens<T>(p.d_k, p.L - 1, RPB, budget);
  const int smem = 2 * TileLayout(TT, p.d_k, p.L - 1, RPB, sizeof(T)).bytes;
  cudaError_t err = cudaFuncSetAttribute(recurrent_scan_kernel<T, LPR, EPL, CH>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  recurrent_scan_kernel<T, LPR, EPL, CH><<<grid, kBlock, smem, stream>>>(p, TT);
  return cudaGetLastError();
}

template <typename T, int LPR, int EPL>
cudaError_t launch_shape(const ScanParams& p, cudaStream_t stream) {
  if (p.chain == PRISM_CHAIN_GELU) return launch_chain<T, LPR, EPL, PRISM_CHAIN_GELU>(p, stream);
  return launch_chain<T, LPR, EPL, PRISM_CHAIN_LINEAR>(p, stream);
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
