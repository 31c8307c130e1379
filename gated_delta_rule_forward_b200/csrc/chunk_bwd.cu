// Chunk-parallel kernels of the chunked backward for the five variants.
// "Gated DeltaNet-2" (technical core) asks for a gate-aware backward that
// keeps the chunkwise structure; this one
// reverses the forward's chunk algebra ("Kaczmarz Linear Attention", KLA
// update rule and implementation):
//     forward, per chunk:  E = U' - W S0,  O = Qg S0 + P E,  S_C = Gamma_C S0 + Kt^T E
//     backward, dS the gradient of the chunk's end state:
//         dE  = Kt dS + P^T dO
//         dS0 = Gamma_C dS + Qg^T dO - W^T dE
// The recurrence in dS is the forward carry's own form with the operands
// exchanged (Kt where -W was, -W where Kt was, R = P^T dO where U' was and
// F = Qg^T dO as an extra state term), so it runs on the forward's carry
// kernel over "reverse records" that bwd_rev_prep_kernel builds here from the
// forward's records, with the chunks in reverse order.  Every other gradient
// is local to a chunk given its start state S0 and dS; bwd_local_kernel
// computes them per chunk, dE included (the records carry beta in P and Kt,
// so the carry's own residual is Diag(beta) dE, which cannot be divided
// back where beta vanishes).  With scalar decay, g the chunk-local cumulative
// log decay, D_tr = e^(g_t - g_r) for r <= t, e = e^g and f = e^(g_C - g)
// (channel decay and GDN-2's gates: see bwd_local_kernel):
//     dE = Diag(f) K dS + P^T dO,  P = scale tril(D o Q K^T)
//     G = K K^T,  A = tril(Diag(beta) (D o G), -1),  T = (I + A)^-1
//     E = T Diag(beta) V - T Diag(beta e) K S0,  dW = -dE S0^T,  dP = tril(dO E^T)
//     dT = dE V^T Diag(beta) + dW K^T Diag(beta e),  dA = tril(-T^T dT T^T, -1)
//     N1 = Diag(beta) (dA o D),  N2 = scale (dP o D)
//     dk = Diag(f) E dS^T + Diag(beta e) T^T dW + N1 K + N1^T K + N2^T Q
//     dq = scale Diag(e) dO S0^T + N2 K,   dv = Diag(beta) T^T dE
//     dbeta = rowsum(V o T^T dE) + e o rowsum(K o T^T dW) + rowsum(dA o D o G)
//     dg_t = sum_i [dq o Q + (Diag(beta e) T^T dW + N1 K - Diag(f) E dS^T - N1^T K - N2^T Q) o K]_ti
//            (+ sum(Diag(f) E dS^T o K) + e^(g_C) sum(dS o S0) at the chunk's last token)
//     dlog_g_t = sum of dg_s over the chunk's tokens s >= t
// and for KLA, beta = eta / (||k||^2 + eps): d eta = dbeta / (||k||^2 + eps),
// dk -= 2 dbeta beta / (||k||^2 + eps) k.  Decay enters only through D, e and
// f, all at most 1, so no factor overflows however strong the decay.
//
// The reverse carry's fp16 operands need the gradients near unit scale: dO and
// the final-state gradient are scaled by a power of two s (max |.| to [0.5, 1)),
// and the local kernel and the initial-state gradient divide it out again.
// The forward carry keeps every chunk's start state in fp16 for scalar decay
// (the operand its MMAs took) and in fp32 for channel decay; the reverse carry
// keeps its states in fp32.
#include <algorithm>
#include <type_traits>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "chunk_bwd.cuh"
#include "chunk_common.cuh"
#include "chunk_record.cuh"
#include "chunk_split.cuh"

// Device-side error word of this file (bit 1: a reverse-record operand beyond
// the fp16 range).
__device__ int g_gdr_bwd_error = 0;

namespace gdr {
namespace tc {
namespace {

constexpr int NT = 256;
constexpr float F16_SAFE_BWD = 60000.f;
constexpr float LOG2E_BWD = 1.4426950408889634f;

// ---------------------------------------------------------------- warp-tile products
// The products run on the tensor cores through the warp-level tf32 MMA
// (m16n8k8, fp32 accumulation): a CTA's eight warps tile an M x N product
// (M, N in {64, 128}) into 16-row tiles, each of W warps covering 16 rows and
// N * RT / (8 W) columns, RT = M / 16 row tiles.  Operands come from shared or global
// memory through views that may transpose them, so every product of the
// chunk algebra is written as it reads.
//
// A matrix operand: element (r, c) is p[r * ld + c], or p[c * ld + r] for TR.
// GLOBAL operands are read through the read-only cache; an EXACT fp32 operand
// holds tf32 values already (the solve's T), so it needs no second tf32 part.
template <typename E, bool TR, bool GLOBAL = false, bool EXACT = false>
struct Mat {
  using elem = E;
  static constexpr bool kTr = TR;
  static constexpr bool kGlobal = GLOBAL;
  static constexpr bool kExact = EXACT || std::is_same<E, __nv_bfloat16>::value || std::is_same<E, __half>::value;
  const E *p;
  int ld;
};

template <typename E, bool G>
__device__ __forceinline__ float ld1(const E *p);
template <>
__device__ __forceinline__ float ld1<float, false>(const float *p) { return *p; }
template <>
__device__ __forceinline__ float ld1<float, true>(const float *p) { return __ldg(p); }
template <>
__device__ __forceinline__ float ld1<__nv_bfloat16, false>(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
template <>
__device__ __forceinline__ float ld1<__half, false>(const __half *p) { return __half2float(*p); }

template <typename V>
__device__ __forceinline__ float at(const V &m, int r, int c) {
  return ld1<typename V::elem, V::kGlobal>(m.p + (V::kTr ? c * m.ld + r : r * m.ld + c));
}
// Channel decay (KDA): a bf16 tile of K or Q scaled element by element by
// 2^(sg (gamma[t][i] - ref[i])), gamma the chunk-local cumulative log2 decay per
// token t and channel i (an fp32 tile of row stride LDG in shared memory) and
// ref a per-channel vector.  Element (r, c) is the (token, channel) one, or the
// (channel, token) one for TR; a GLOBAL tile has token rows ld apart and reads
// zero past the chunk's n tokens.
constexpr int LDG = DK + 4;
template <bool TR, bool GLOBAL = false>
struct Fac {
  using elem = float;
  static constexpr bool kTr = TR;
  static constexpr bool kGlobal = GLOBAL;
  static constexpr bool kExact = false;
  const __nv_bfloat16 *x;
  int ld, n;
  const float *g, *ref;
  float sg;
};
template <bool TR, bool GLOBAL>
__device__ __forceinline__ float at(const Fac<TR, GLOBAL> &m, int r, int c) {
  const int t = TR ? c : r, i = TR ? r : c;
  float x;
  if constexpr (GLOBAL) {
    x = t < m.n ? __bfloat162float(__ldg(m.x + t * m.ld + i)) : 0.f;
  } else {
    x = __bfloat162float(m.x[t * m.ld + i]);
  }
  return x * ex2(m.sg * (m.g[t * LDG + i] - m.ref[i]));
}
// A bf16 tile in global memory with token rows ld apart, zero past the chunk's n tokens.
template <bool TR>
struct GB {
  using elem = __nv_bfloat16;
  static constexpr bool kTr = TR;
  static constexpr bool kGlobal = true;
  static constexpr bool kExact = true;
  const __nv_bfloat16 *x;
  int ld, n;
};
template <bool TR>
__device__ __forceinline__ float at(const GB<TR> &m, int r, int c) {
  const int t = TR ? c : r, j = TR ? r : c;
  return t < m.n ? __bfloat162float(__ldg(m.x + t * m.ld + j)) : 0.f;
}

// GDN-2: a factored key tile times a gate per (token, channel) read from global
// memory, K o gate o 2^(sg (gamma - ref)), gate = the erase gate b (GM 1) or
// w - b (GM 2); zero past the chunk's n tokens.
template <bool TR, int GM>
struct FacG {
  using elem = float;
  static constexpr bool kTr = TR;
  static constexpr bool kGlobal = false;
  static constexpr bool kExact = false;
  const __nv_bfloat16 *x;
  int ld, n;
  const float *g, *ref;
  float sg;
  const float *eb, *ww;
  int gld;
};
template <bool TR, int GM>
__device__ __forceinline__ float at(const FacG<TR, GM> &m, int r, int c) {
  const int t = TR ? c : r, i = TR ? r : c;
  if (t >= m.n) return 0.f;
  float gt = __ldg(m.eb + t * m.gld + i);
  if (GM == 2) gt = __ldg(m.ww + t * m.gld + i) - gt;
  return __bfloat162float(m.x[t * m.ld + i]) * gt * ex2(m.sg * (m.g[t * LDG + i] - m.ref[i]));
}

// ... or such a gated key tile staged in shared memory as fp32 (rows of LDG).
template <bool TR>
struct FacF {
  using elem = float;
  static constexpr bool kTr = TR;
  static constexpr bool kGlobal = false;
  static constexpr bool kExact = false;
  const float *x, *g, *ref;
  float sg;
};
template <bool TR>
__device__ __forceinline__ float at(const FacF<TR> &m, int r, int c) {
  const int t = TR ? c : r, i = TR ? r : c;
  return m.x[t * LDG + i] * ex2(m.sg * (m.g[t * LDG + i] - m.ref[i]));
}

// The warp tile of rows m0 .. m0 + 15 and columns n0 .. n0 + 8 NT - 1 of an M x N
// product shared by W warps.
template <int M, int N, int W = 8>
struct Tiling {
  static constexpr int RT = M / 16;          // row tiles
  static constexpr int CH = W / RT;          // column parts
  static constexpr int NT = N / 8 / CH;      // 8-column MMA tiles per warp
  static_assert(CH >= 1 && NT >= 1, "tiling");
  static __device__ __forceinline__ int m0(int w) { return 16 * (w % RT); }
  static __device__ __forceinline__ int n0(int w) { return (w / RT) * (N / CH); }
};

// acc (+/-)= A(m0.., k) ks[k] B(k, n0..) over k < K (a multiple of 8); ks, a
// per-k factor in shared memory, may be null.  acc[j] is the m16n8 fragment of
// columns n0 + 8 j .. n0 + 8 j + 7: {D[g][2t], D[g][2t+1], D[g+8][2t], D[g+8][2t+1]}
// with g = lane / 4, t = lane % 4.  PRECISE: each fp32 operand is split into
// two tf32 parts, x = hi + lo, and the product taken as a_hi b_hi + a_lo b_hi +
// a_hi b_lo (three-pass tf32: about fp32 accuracy; a bf16 operand is exact in
// tf32 and has no lo part, so its products take two passes).  Otherwise one
// tf32 pass (for results that are stored in fp16 anyway).
template <typename V>
__device__ __forceinline__ void split(const V &m, int r, int c, float scale, uint32_t &hi, uint32_t &lo) {
  const float x = at(m, r, c) * scale;
  hi = V::kExact && scale == 1.f ? __float_as_uint(x) : to_tf32(x);
  lo = to_tf32(x - __uint_as_float(hi));
}
template <int NT, bool NEG, typename MA, typename MB, bool PRECISE = true>
__device__ __forceinline__ void wmm(float (&acc)[NT][4], const MA a, const MB b, int K, int m0, int n0, int lane,
                                    const float *ks = nullptr) {
  constexpr bool a_exact = !PRECISE || MA::kExact;
  const bool b_exact = !PRECISE || (MB::kExact && ks == nullptr);
  const int g = lane >> 2, t = lane & 3;
#pragma unroll 2
  for (int k0 = 0; k0 < K; k0 += 8) {
    uint32_t ah[4], al[4];
    split(a, m0 + g, k0 + t, 1.f, ah[0], al[0]);
    split(a, m0 + g + 8, k0 + t, 1.f, ah[1], al[1]);
    split(a, m0 + g, k0 + t + 4, 1.f, ah[2], al[2]);
    split(a, m0 + g + 8, k0 + t + 4, 1.f, ah[3], al[3]);
    if (NEG) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        ah[e] ^= 0x80000000u;
        al[e] ^= 0x80000000u;
      }
    }
    const float s0 = ks != nullptr ? ks[k0 + t] : 1.f, s1 = ks != nullptr ? ks[k0 + t + 4] : 1.f;
    // all B fragments first, then the passes as three sweeps over the tiles, so
    // that consecutive MMAs accumulate into different fragments
    uint32_t bh[NT][2], bl[NT][2];
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      split(b, k0 + t, n0 + 8 * j + g, s0, bh[j][0], bl[j][0]);
      split(b, k0 + t + 4, n0 + 8 * j + g, s1, bh[j][1], bl[j][1]);
    }
    if (!b_exact) {
#pragma unroll
      for (int j = 0; j < NT; ++j) mma_tf32_16x8x8(acc[j], ah, bl[j][0], bl[j][1]);
    }
    if (!a_exact) {
#pragma unroll
      for (int j = 0; j < NT; ++j) mma_tf32_16x8x8(acc[j], al, bh[j][0], bh[j][1]);
    }
#pragma unroll
    for (int j = 0; j < NT; ++j) mma_tf32_16x8x8(acc[j], ah, bh[j][0], bh[j][1]);
  }
}

// One tf32 pass, for the products whose rounding the gradients absorb (see
// bwd_local_kernel).
template <int NT, bool NEG, typename MA, typename MB>
__device__ __forceinline__ void wmm1(float (&acc)[NT][4], const MA a, const MB b, int K, int m0, int n0, int lane,
                                     const float *ks = nullptr) {
  wmm<NT, NEG, MA, MB, false>(acc, a, b, K, m0, n0, lane, ks);
}

// f(row, col, value) for each accumulator element of a warp tile; each_je
// also passes the fragment indices (j, e), compile-time constants after
// unrolling, for per-column register arrays.
template <int NT, typename F>
__device__ __forceinline__ void each(float (&acc)[NT][4], int m0, int n0, int lane, F f) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int j = 0; j < NT; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) f(m0 + g + 8 * (e >> 1), n0 + 8 * j + 2 * t + (e & 1), acc[j][e]);
}
template <int NT, typename F>
__device__ __forceinline__ void each_je(float (&acc)[NT][4], int m0, int n0, int lane, F f) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int j = 0; j < NT; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) f(j, e, m0 + g + 8 * (e >> 1), n0 + 8 * j + 2 * t + (e & 1), acc[j][e]);
}

template <int NT>
__device__ __forceinline__ void zero(float (&acc)[NT][4]) {
#pragma unroll
  for (int j = 0; j < NT; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;
}

// Sums over the lanes of a quad (the four lanes that share a row of a fragment)
// and over the eight quads (the lanes that share a column).
__device__ __forceinline__ float quad_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  return x + __shfl_xor_sync(0xffffffffu, x, 2);
}
__device__ __forceinline__ float column_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 4);
  x += __shfl_xor_sync(0xffffffffu, x, 8);
  return x + __shfl_xor_sync(0xffffffffu, x, 16);
}

// The power of two s with s * max|gradient| in [0.5, 1) (1 when the maximum is
// zero or not finite).
__device__ __forceinline__ float grad_scale(const uint32_t *absmax) {
  const float m = __uint_as_float(*absmax);
  if (!(m > 0.f) || !(m < 3.0e38f)) return 1.f;
  int ex;
  frexpf(m, &ex);
  ex = max(-120, min(120, ex));
  return ldexpf(1.f, -ex);
}

// ---------------------------------------------------------------- gradient scale
__global__ void bwd_absmax_kernel(const __nv_bfloat16 *d_o, size_t n_o, const float *d_final, size_t n_f,
                                  uint32_t *out) {
  float m = 0.f;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  const uint4 *o8 = reinterpret_cast<const uint4 *>(d_o);   // n_o is a multiple of 8 (d_v is)
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_o / 8; i += stride) {
    float x[8];
    unpack8(__ldg(o8 + i), x);
#pragma unroll
    for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(x[e]));
  }
  if (d_final != nullptr)
    for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_f; i += stride)
      m = fmaxf(m, fabsf(__ldg(d_final + i)));
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  // one atomic per block (not per warp): thousands of atomics on one word serialise
  __shared__ float wmax[32];
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = threadIdx.x < (blockDim.x >> 5) ? wmax[threadIdx.x] : 0.f;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (threadIdx.x == 0) atomicMax(out, __float_as_uint(m));   // non-negative floats order as integers
  }
}

__global__ void bwd_scale_state_kernel(const float *d_final, size_t n, const uint32_t *absmax, float *x0) {
  const float s = grad_scale(absmax);
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride)
    x0[i] = d_final != nullptr ? s * __ldg(d_final + i) : 0.f;
}

__global__ void bwd_unscale_kernel(const float *xf, size_t n, const uint32_t *absmax, float *d_s0) {
  const float inv = 1.f / grad_scale(absmax);
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride)
    d_s0[i] = __ldg(xf + i) * inv;
}

// ---------------------------------------------------------------- reverse records
struct RevPrepParams {
  int T, H, NC;
  uint32_t rb_f, rb_r;   // bytes of a forward record / a reverse record
  bool chan;             // Gamma_C stored as d_k values in the forward record
  const __nv_bfloat16 *d_o;
  const uint8_t *fwd;
  uint8_t *rev;
  const uint32_t *absmax;
};

// One CTA per forward record (b, h, c); it writes reverse record (b, h, NC-1-c)
// in the channel-decay + GDN-2 record format the carry's third mode reads:
//     -W slot of REC_WQ <- Kt,  REC_K <- -W,
//     U' slot <- R^T = (s dO)^T P,  Gamma_C as d_k values,
//     the state term <- F^T = (s dO)^T Qg.
// The Qg slots, P and the output term stay unwritten: the reverse carry runs
// without outputs and reads none of them.
//
// Every operand is exact in 16 bits (s dO in bf16, s a power of two; P and Qg
// are the record's fp16), so the tiles stay 16-bit in shared memory (44 KB at
// d_v = 128, three CTAs per SM) and one tf32 pass is exact per product; F^T is
// taken in two 64-column halves, and both products go from the fragments
// straight to the record.
template <int DV>
__global__ void __launch_bounds__(NT, 3) bwd_rev_prep_kernel(const RevPrepParams p) {
  constexpr int NS = DV / 64;
  constexpr int LDO = DV + 8, LDP = C + 8, LDQ = DK + 8;   // 16-bit rows, 16 bytes of padding
  extern __shared__ float4 smem_rev[];
  __nv_bfloat16 *sO = reinterpret_cast<__nv_bfloat16 *>(smem_rev);   // [C][LDO] s dO, rows t
  __half *sP = reinterpret_cast<__half *>(sO + C * LDO);               // [C][LDP] P, rows t
  __half *sQ = sP + C * LDP;                                           // [C][LDQ] Qg, rows t
  const int tid = threadIdx.x;
  const int r = blockIdx.x;
  const int bh = r / p.NC, c = r - bh * p.NC;
  const int b = bh / p.H, h = bh - b * p.H;
  const uint8_t *src = p.fwd + static_cast<size_t>(r) * p.rb_f;
  uint8_t *dst = p.rev + (static_cast<size_t>(bh) * p.NC + (p.NC - 1 - c)) * p.rb_r;
  const float s = grad_scale(p.absmax);

#pragma unroll
  for (int i = tid; i < C * DV / 8; i += NT) {
    const int t = i / (DV / 8), v8 = (i % (DV / 8)) * 8;
    const int tg = c * C + t;
    float x[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (tg < p.T)
      unpack8(__ldg(reinterpret_cast<const uint4 *>(p.d_o + ((static_cast<size_t>(b) * p.T + tg) * p.H + h) * DV + v8)),
              x);
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] *= s;
    st_chunk_bf16(reinterpret_cast<uint8_t *>(sO + t * LDO + v8), x);
  }
#pragma unroll
  for (int i = tid; i < C * C / 8; i += NT) {   // P: the record's swizzled rows, 16 bytes at a time
    const int t = i >> 3, j = i & 7;
    *reinterpret_cast<uint4 *>(sP + t * LDP + 8 * j) = *reinterpret_cast<const uint4 *>(src + REC_P + sw128(t, j));
  }
#pragma unroll
  for (int i = tid; i < C * DK / 8; i += NT) {   // Qg: two 64-channel atoms
    const int t = i >> 4, a = (i >> 3) & 1, j = i & 7;
    *reinterpret_cast<uint4 *>(sQ + t * LDQ + 64 * a + 8 * j) =
        *reinterpret_cast<const uint4 *>(src + REC_WQ + a * 16384 + 8192 + sw128(t, j));
  }
  // tile copies (16-byte units)
  for (int i = tid; i < 1024; i += NT) {
    const int a = i >> 9, j = i & 511;
    *reinterpret_cast<uint4 *>(dst + REC_WQ + a * 16384 + 16 * j) =
        *reinterpret_cast<const uint4 *>(src + REC_K + a * 8192 + 16 * j);
    *reinterpret_cast<uint4 *>(dst + REC_K + a * 8192 + 16 * j) =
        *reinterpret_cast<const uint4 *>(src + REC_WQ + a * 16384 + 16 * j);
  }
  if (tid < DK) {
    const float *g = reinterpret_cast<const float *>(src + rec_sc(NS));
    reinterpret_cast<float *>(dst + rec_sc(NS))[tid] = p.chan ? g[tid] : g[0];
  }
  __syncthreads();

  const int warp = tid >> 5, lane = tid & 31;
  float vmax = 0.f;
  using TL = Tiling<DV, 64>;
  const int m0 = TL::m0(warp), n0 = TL::n0(warp);
  using OT = Mat<__nv_bfloat16, true>;
  using HM = Mat<__half, false>;
  {   // R^T [v][t]: the U' slot's rows v, 128-byte swizzled
    float acc[TL::NT][4];
    zero(acc);
    wmm<TL::NT, false, OT, HM, false>(acc, OT{sO, LDO}, HM{sP, LDP}, C, m0, n0, lane);
    const int g = lane >> 2, tq = lane & 3;
#pragma unroll
    for (int j = 0; j < TL::NT; ++j)
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {   // two adjacent tokens per 4-byte store
        const int v = m0 + g + 8 * h2, t = n0 + 8 * j + 2 * tq;
        const float x0 = acc[j][2 * h2], x1 = acc[j][2 * h2 + 1];
        vmax = fmaxf(vmax, fmaxf(fabsf(x0), fabsf(x1)));
        *reinterpret_cast<uint32_t *>(dst + REC_U + sw128(v, t >> 3) + (t & 7) * 2) = pack_f16x2(x0, x1);
      }
  }
  uint8_t *fdst = dst + rec_bytes_chan(NS) + 8192 * NS;   // F^T [v][i]: unswizzled rows of d_k values
#pragma unroll 1
  for (int hh = 0; hh < 2; ++hh) {
    float acc[TL::NT][4];
    zero(acc);
    wmm<TL::NT, false, OT, HM, false>(acc, OT{sO, LDO}, HM{sQ + 64 * hh, LDQ}, C, m0, n0, lane);
    const int g = lane >> 2, tq = lane & 3;
#pragma unroll
    for (int j = 0; j < TL::NT; ++j)
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int v = m0 + g + 8 * h2, i = 64 * hh + n0 + 8 * j + 2 * tq;
        const float x0 = acc[j][2 * h2], x1 = acc[j][2 * h2 + 1];
        vmax = fmaxf(vmax, fmaxf(fabsf(x0), fabsf(x1)));
        *reinterpret_cast<uint32_t *>(fdst + (v * DK + i) * 2) = pack_f16x2(x0, x1);
      }
  }
  if (vmax > F16_SAFE_BWD) atomicOr(&g_gdr_bwd_error, 2);
}

// ---------------------------------------------------------------- chunk-local gradients
struct LocalParams {
  int T, H, NC;
  bool decay, kla;
  float eps, scale;
  const __nv_bfloat16 *q, *k, *v, *d_o;
  const float *beta, *log_g;   // log_g [B,T,H], or [B,T,H,d_k] with channel decay
  const void *s0s;          // chunk start states: fp16 as the forward carry's MMAs take them
                            // (scalar decay), fp32 (channel decay)
  const float *dss;         // (scaled) end-state gradients in reverse chunk order
  const uint32_t *absmax;
  __nv_bfloat16 *dq, *dk, *dv;
  float *dbeta, *dlog_g;    // dlog_g laid out as log_g
  // GDN-2: the gates, their gradients, and per-chunk scratch in the forward and
  // reverse records' slots (dead once the reverse carry has run)
  const float *erase_b, *write_w;
  float *d_erase, *d_write;
  uint8_t *scr_f, *scr_r;
  uint32_t rb_f, rb_r;
};

// CHAN: channel decay, with the decay tile after the scalars; at d_v = 128 Q and
// V are then read from global memory (through the read-only cache) to make room.
template <int DV, bool CHAN>
struct LocalSmem {
  static constexpr bool kQVGlobal = CHAN && DV == 128;
  static constexpr int LDB = DK + 8;    // bf16 rows of K, Q
  static constexpr int LDBV = DV + 8;   // bf16 rows of V, dO
  static constexpr int LDF = DV + 4;    // fp32 rows of dE, E
  static constexpr int LDW = DK + 4;    // fp32 rows of W
  static constexpr int LDC = C + 4;     // fp32 rows of C-wide tiles (dW^T, X, dP)
  static constexpr int LDS = DV + 8;    // fp16 rows of S0 (over dE, A, P)
  static constexpr int LDSE = DV + 4;   // fp16 rows of S0's second staging (over E)
  static constexpr int LDH = 66;        // fp32 rows of a 64-column half of dS (over W) or of S0 (over E)
  static constexpr size_t K = 0;
  static constexpr size_t Q = K + C * LDB * 2;
  static constexpr size_t V = Q + (kQVGlobal ? 0 : C * LDB * 2);
  static constexpr size_t O = V + (kQVGlobal ? 0 : C * LDBV * 2);
  static constexpr size_t E = O + C * LDBV * 2;
  static constexpr size_t W = E + static_cast<size_t>(std::max(C * LDF, C * LDC)) * 4;
  static constexpr size_t TT = W + static_cast<size_t>(std::max(C * LDW, DK * LDC)) * 4;
  static constexpr size_t DE = TT + C * LD * 4;   // DE, A and P are contiguous: S0's staging before dE and P exist
  static constexpr size_t A = DE + C * LDF * 4;
  static constexpr size_t P = A + C * LD * 4;
  static constexpr size_t SC = P + C * LDC * 4;
  static constexpr size_t GAM = SC + (9 * C + 4 + (CHAN ? 5 * DK : 0)) * 4;   // [C][LDG] gamma
  static constexpr size_t BYTES = GAM + (CHAN ? C * LDG * 4 : 0);
  static_assert(BYTES <= 232448 && GAM % 16 == 0, "shared memory");
  static_assert(A + C * LD * 4 + C * LDC * 4 - DE >= static_cast<size_t>(DK) * LDF * 4, "S0 staging over dE, A, P");
  static_assert(std::max(C * LDW, DK * LDC) >= DK * LDH, "a half of dS over W");
  static_assert(std::max(C * LDF, C * LDC) * 4 >= DK * LDSE * 2, "S0 (fp16) over E");
  static constexpr bool kS0HalvesOverE = std::max(C * LDF, C * LDC) >= DK * LDH;   // fp32 S0: d_v = 128
};

// One CTA of NTL threads per chunk (b, h, c): sixteen warps share each
// product, so that the chunk's chain of small dependent products runs with
// twice the warps in flight of an eight-warp CTA (one CTA fits an SM).
//
// With channel decay (CHAN, KDA: "Gated DeltaNet-2", what is new) the decay
// enters the products element by element.  With gamma the chunk-local
// cumulative log decay per token and channel, factored around token m = 31 as
// the forward's preparation factors it (whose range check bounds every factor
// by 2^120), a = e^(gamma - gamma_m), b = e^(gamma_m - gamma), e = e^gamma and
// f = e^(gamma_C - gamma), all (token x channel):
//     G~ = (K o a)(K o b)^T,  A = tril(Diag(beta) G~, -1),  P = scale tril((Q o a)(K o b)^T)
//     W = T Diag(beta) (K o e),  dE = (K o f) dS + P^T dO,  dT = (dE V^T + dW (K o e)^T) Diag(beta)
//     N1 = Diag(beta) dA,  N2 = scale dP
//     X1 = f o (E dS^T),  Y1 = e o (Diag(beta) T^T dW) + a o (N1 (K o b)),
//     Y2 = b o (N1^T (K o a) + N2^T (Q o a))
//     dk = X1 + Y1 + Y2,  dq = scale e o (dO S0^T) + a o (N2 (K o b))
//     dbeta = rowsum(V o T^T dE) + rowsum((K o e) o T^T dW) + rowsum(dA o G~)
//     dg = dq o Q + (Y1 - X1 - Y2) o K, plus sum_t (X1 o K)_t + e^(gamma_C) o rowsum(dS o S0)
//     at the chunk's last token; dlog_g = per-channel suffix sums of dg over the chunk.
//
// Precision: fp32 operands are split into two tf32 parts (wmm) except in the
// products that take one pass (wmm1): dT, X = dT T^T and dA (not for GDN-2,
// whose d erase is a small difference of gradients built from them); KDA's
// factored Gram and P products; and, with scalar decay, the dk and dq products
// with N1 and N2.  Measured against the fp64 oracle (the 350M layer and small ragged
// and strong-decay cases of every variant), this moved no gradient past 5e-3
// of its RMS (d log g 6.0e-3 -> 5.8e-3, dk 2.3e-3 -> 4.8e-3); one pass for
// E, dW or the dE, U', W products moved d log g to 1.5-2.9e-2, and KDA's dk
// products at one pass 2.6e-2.
//
// GDN-2 (G2, with CHAN) has erase and write gates in place of beta: with
// a = b o k, d = (w - b) o k and the factors above (a_ for the middle-token
// factor a), the chunk's forward is A = tril((K o a_)(a o b)^T, -1), A^d likewise
// with d, T = (I + A)^-1, Zt = I - A^d, E = T Zt V - W S0 with W = T (K o e),
// P^a, P^d = scale tril((Q o a_)(a or d o b)^T), and
//     dE = (a o f) dS + P^a^T dO,  tU = T^T dE,  dv = Zt^T tU + P^d^T dO + (d o f) dS
//     dT = dE V^T Zt^T + dW (K o e)^T,  dA = tril(-T^T dT T^T, -1),  dA^d = -tril(tU V^T, -1)
//     dk = a_ o (dA (a o b) + dA^d (d o b)) + e o T^T dW + b o da + (w - b) o dd
//     da = b o (dA^T (K o a_) + N2a^T (Q o a_)) + f o (E dS^T)
//     dd = b o (dA^d^T (K o a_) + N2d^T (Q o a_)) + f o (V dS^T)
//     dq = scale e o (dO S0^T) + a_ o (N2a (a o b) + N2d (d o b))
//     d erase = k o (da - dd),  d write = k o dd,  N2a = scale tril(dO E^T), N2d = scale tril(dO V^T)
//     dg = dq o Q + (a_ o dKa + e o T^T dW) o K - da o a - dd o d, plus the f parts of
//     da o a + dd o d summed over the chunk and e^(gamma_C) o rowsum(dS o S0) at its last token.
// I - A^d, P^d, dA^d, da, dd and the (d o f) dS term go through global scratch: this
// chunk's slots of the forward and reverse records, which nothing reads any more.
//
// At d_v = 128 (KDA and GDN-2) the factored and gated key / query tiles are
// staged whole in shared memory as fp32 wherever a region of that size is
// free between its own uses (E, W, dE), so that a fragment element is one
// load rather than a factor evaluation; elsewhere the views evaluate them.
constexpr int NTL = 512;
template <int DV, bool CHAN, bool G2 = false>
__global__ void __launch_bounds__(NTL, 1) bwd_local_kernel(const LocalParams p) {
  static_assert(CHAN || !G2, "GDN-2 has channel decay");
  using L = LocalSmem<DV, CHAN>;
  constexpr bool QVG = L::kQVGlobal;
  constexpr int LDB = L::LDB, LDBV = L::LDBV, LDF = L::LDF, LDW = L::LDW, LDC = L::LDC;
  static_assert(NTL == 4 * DK, "the channel scans run four 16-token parts per channel");
  extern __shared__ float4 smem_loc[];
  uint8_t *sm = reinterpret_cast<uint8_t *>(smem_loc);
  __nv_bfloat16 *sK = reinterpret_cast<__nv_bfloat16 *>(sm + L::K);
  __nv_bfloat16 *sQ = reinterpret_cast<__nv_bfloat16 *>(sm + L::Q);
  __nv_bfloat16 *sV = reinterpret_cast<__nv_bfloat16 *>(sm + L::V);
  __nv_bfloat16 *sO = reinterpret_cast<__nv_bfloat16 *>(sm + L::O);
  float *sdE = reinterpret_cast<float *>(sm + L::DE);
  float *sE = reinterpret_cast<float *>(sm + L::E);    // E, later X = dT T^T (and staged tiles between)
  float *sW = reinterpret_cast<float *>(sm + L::W);    // W, later dW^T (and staged tiles between)
  float *sA = reinterpret_cast<float *>(sm + L::A);    // A^T for the solve, later dT, dA, N1
  float *sT = reinterpret_cast<float *>(sm + L::TT);   // T
  float *sP = reinterpret_cast<float *>(sm + L::P);    // dP, later N2
  float *sbeta = reinterpret_cast<float *>(sm + L::SC);
  float *sbe = sbeta + C;     // beta e
  float *see = sbe + C;       // e
  float *sff = see + C;       // f
  float *sscan = sff + C;     // per-warp scan of the log2 decay
  float *sG = sscan + C;      // cumulative log2 decay
  float *sdb = sG + C;        // dbeta
  float *sdg = sdb + C;       // dg
  float *snk = sdg + C;       // ||k||^2
  float *sred = snk + C;      // [0] sum X1 o K, [1] sum dS o S0
  // channel decay: gamma_m, gamma_C, zeros, and per channel sum_t X1 o K and sum_v dS o S0
  float *sgm = sred + 4, *sgC = sgm + DK, *szero = sgC + DK, *sx1k = szero + DK, *sss = sx1k + DK;
  float *sgam = reinterpret_cast<float *>(sm + L::GAM);   // [C][LDG] cumulative log2 decay

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x / p.NC, c = blockIdx.x - bh * p.NC;
  const int b = bh / p.H, h = bh - b * p.H;
  const int t0 = c * C, n = min(C, p.T - t0);
  const float s = grad_scale(p.absmax), inv_s = 1.f / s;
  const size_t rc = static_cast<size_t>(bh) * p.NC + (p.NC - 1 - c);   // reverse-order index of this chunk
  // S0 in fp16 with scalar decay; in fp32 with channel decay, whose d log g its fp16
  // rounding would move to ~2e-2 of RMS on long sequences
  using S0E = std::conditional_t<CHAN, float, __half>;
  const S0E *S0 = static_cast<const S0E *>(p.s0s) + static_cast<size_t>(blockIdx.x) * DK * DV;
  const float *dS = p.dss + rc * DK * DV;
  auto row = [&](int t) { return (static_cast<size_t>(b) * p.T + t0 + t) * p.H + h; };
  // GDN-2 scratch: [I - A^d | P^d | dA^d] (C x C each) and [da | dd] (C x d_k), (d o f) dS (C x d_v)
  float *scZ = G2 ? reinterpret_cast<float *>(p.scr_f + static_cast<size_t>(blockIdx.x) * p.rb_f) : nullptr;
  float *scPd = G2 ? scZ + C * C : nullptr, *scAd = G2 ? scPd + C * C : nullptr;
  float *scDa = G2 ? reinterpret_cast<float *>(p.scr_r + rc * p.rb_r) : nullptr;
  float *scDd = G2 ? scDa + C * DK : nullptr, *scDv = G2 ? scDd + C * DK : nullptr;

  // ---- inputs: bf16 tiles (zero past T)
#pragma unroll
  for (int i = tid; i < C * DK / 8; i += NTL) {
    const int t = i / (DK / 8), j = i % (DK / 8);
    uint4 uq = make_uint4(0u, 0u, 0u, 0u), uk = uq;
    if (t < n) {
      if constexpr (!QVG) uq = __ldg(reinterpret_cast<const uint4 *>(p.q + row(t) * DK) + j);
      uk = __ldg(reinterpret_cast<const uint4 *>(p.k + row(t) * DK) + j);
    }
    if constexpr (!QVG) *reinterpret_cast<uint4 *>(sQ + t * LDB + 8 * j) = uq;
    *reinterpret_cast<uint4 *>(sK + t * LDB + 8 * j) = uk;
  }
#pragma unroll
  for (int i = tid; i < C * DV / 8; i += NTL) {
    const int t = i / (DV / 8), j = i % (DV / 8);
    uint4 uv = make_uint4(0u, 0u, 0u, 0u), uo = uv;
    if (t < n) {
      if constexpr (!QVG) uv = __ldg(reinterpret_cast<const uint4 *>(p.v + row(t) * DV) + j);
      uo = __ldg(reinterpret_cast<const uint4 *>(p.d_o + row(t) * DV) + j);
    }
    if constexpr (!QVG) *reinterpret_cast<uint4 *>(sV + t * LDBV + 8 * j) = uv;
    *reinterpret_cast<uint4 *>(sO + t * LDBV + 8 * j) = uo;
  }
  if constexpr (CHAN) {   // log g per channel (zero past T: no decay)
#pragma unroll
    for (int i = tid; i < C * DK / 4; i += NTL) {
      const int t = i / (DK / 4), j = i % (DK / 4);
      float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
      if (t < n) x = __ldg(reinterpret_cast<const float4 *>(p.log_g + row(t) * DK) + j);
      *reinterpret_cast<float4 *>(sgam + t * LDG + 4 * j) = x;
    }
  }
  if (tid < C) {
    sdb[tid] = 0.f;
    sdg[tid] = 0.f;
  }
  if (tid < 4) sred[tid] = 0.f;
  __syncthreads();

  // ---- token scalars (threads 0-63): beta (KLA: eta / (||k||^2 + eps)), the
  // cumulative log2 decay, e and f
  if (tid < C) {
    const int t = tid;
    float bt = 0.f, lg = 0.f, nk = 0.f;
    for (int i = 0; i < DK; ++i) {
      const float x = __bfloat162float(sK[t * LDB + i]);
      nk = fmaf(x, x, nk);
    }
    if (t < n) {
      if constexpr (!G2) bt = __ldg(p.beta + row(t));
      if (!CHAN && p.decay) lg = __ldg(p.log_g + row(t));
    }
    if (p.kla) bt = bt / (nk + p.eps);
    snk[t] = nk;
    sbeta[t] = bt;
    float x = lg * LOG2E_BWD;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    sscan[t] = x;
  }
  __syncthreads();
  if (tid < C) {
    const int t = tid;
    sG[t] = sscan[t] + (t >= 32 ? sscan[31] : 0.f);
  }
  __syncthreads();
  if (tid < C) {
    const int t = tid;
    const float e = ex2(sG[t]);
    see[t] = e;
    sff[t] = ex2(sG[n - 1] - sG[t]);
    sbe[t] = sbeta[t] * e;
  }
  __syncthreads();
  if constexpr (CHAN) {   // gamma: per-channel prefix sums in log2 units, four 16-token parts
    const int i = tid % DK, part = tid / DK;
    float *stot = sdE;   // part totals (dE holds nothing yet)
    float run = 0.f;
    for (int t = 16 * part; t < 16 * part + 16; ++t) {
      run = fmaf(sgam[t * LDG + i], LOG2E_BWD, run);
      sgam[t * LDG + i] = run;
    }
    stot[part * DK + i] = run;
    __syncthreads();
    float off = 0.f;
    for (int q = 0; q < part; ++q) off += stot[q * DK + i];
    for (int t = 16 * part; t < 16 * part + 16; ++t) sgam[t * LDG + i] += off;
    __syncthreads();
    if (tid < DK) {
      sgm[tid] = sgam[31 * LDG + tid];
      sgC[tid] = sgam[(n - 1) * LDG + tid];
      szero[tid] = 0.f;
      sx1k[tid] = 0.f;
    }
    __syncthreads();
  }

  constexpr int LW = NTL / 32;
  using CC = Tiling<C, C, LW>;     // C x C products
  using CV = Tiling<C, DV, LW>;    // C x d_v
  using CK = Tiling<C, DK, LW>;    // C x d_k
  using KC = Tiling<DK, C, LW>;    // d_k x C (the transposed gradient tiles)
  const int mc = CC::m0(warp), nc = CC::n0(warp);
  const int mv = CV::m0(warp), nv = CV::n0(warp);
  const int mk = CK::m0(warp), nk = CK::n0(warp);
  const int mt = KC::m0(warp), nt = KC::n0(warp);
  using BK = Mat<__nv_bfloat16, false>;   // a bf16 tile as stored
  using BKT = Mat<__nv_bfloat16, true>;   // ... transposed
  using F = Mat<float, false>;
  using FT = Mat<float, true>;
  using HS = Mat<__half, false>;          // an fp16 tile (S0)
  using FG = Mat<float, false, true>;     // a global fp32 matrix (S0)
  using TX = Mat<float, false, false, true>;   // T (tf32 values from the solve)
  using TXT = Mat<float, true, false, true>;   // ... transposed
  // channel decay: K o 2^(sg (gamma - ref)) and Q o a, V as stored or read from global memory
  auto kfac = [&](const float *ref, float sg) { return Fac<false>{sK, LDB, C, sgam, ref, sg}; };
  auto kfacT = [&](const float *ref, float sg) { return Fac<true>{sK, LDB, C, sgam, ref, sg}; };
  auto qa = [&]() {
    if constexpr (QVG) return Fac<false, true>{p.q + row(0) * DK, p.H * DK, n, sgam, sgm, 1.f};
    else return Fac<false>{sQ, LDB, C, sgam, sgm, 1.f};
  };
  auto qaT = [&]() {
    if constexpr (QVG) return Fac<true, true>{p.q + row(0) * DK, p.H * DK, n, sgam, sgm, 1.f};
    else return Fac<true>{sQ, LDB, C, sgam, sgm, 1.f};
  };
  auto vm = [&]() {
    if constexpr (QVG) return GB<false>{p.v + row(0) * DV, p.H * DV, n};
    else return BK{sV, LDBV};
  };
  auto vmT = [&]() {
    if constexpr (QVG) return GB<true>{p.v + row(0) * DV, p.H * DV, n};
    else return BKT{sV, LDBV};
  };
  auto qat = [&](int t, int i) {
    if constexpr (QVG) return t < n ? __bfloat162float(__ldg(p.q + row(t) * DK + i)) : 0.f;
    else return __bfloat162float(sQ[t * LDB + i]);
  };
  auto vat = [&](int t, int v) {
    if constexpr (QVG) return t < n ? __bfloat162float(__ldg(p.v + row(t) * DV + v)) : 0.f;
    else return __bfloat162float(sV[t * LDBV + v]);
  };
  auto vmTh = [&](int h0) {   // columns h0 .. of V, transposed
    if constexpr (QVG) return GB<true>{p.v + row(0) * DV + h0, p.H * DV, n};
    else return BKT{sV + h0, LDBV};
  };
  // GDN-2: the gated key tiles (a o 2^.., d o 2^..) and the gates themselves
  const float *ebp = G2 ? p.erase_b + row(0) * DK : nullptr, *wwp = G2 ? p.write_w + row(0) * DK : nullptr;
  const int gld = p.H * DK;
  auto afacT = [&](const float *ref, float sg) { return FacG<true, 1>{sK, LDB, n, sgam, ref, sg, ebp, wwp, gld}; };
  auto dfacT = [&](const float *ref, float sg) { return FacG<true, 2>{sK, LDB, n, sgam, ref, sg, ebp, wwp, gld}; };
  auto afac = [&](const float *ref, float sg) { return FacG<false, 1>{sK, LDB, n, sgam, ref, sg, ebp, wwp, gld}; };
  auto dfac = [&](const float *ref, float sg) { return FacG<false, 2>{sK, LDB, n, sgam, ref, sg, ebp, wwp, gld}; };
  auto gate = [&](const float *gp, int t, int i) { return t < n ? __ldg(gp + t * gld + i) : 0.f; };
  // At d_v = 128 the gated key tiles a = b o k and d = (w - b) o k are staged in
  // shared memory (fp32, rows of LDG) where a region of that size is free: for
  // the two Gram products, for P^a and P^d, and for the dk and dq products.
  constexpr bool GST = G2 && DV == 128;
  auto stage_gated = [&](float *ta, float *td) {
#pragma unroll
    for (int u = tid; u < C * DK / 4; u += NTL) {
      const int t = u / (DK / 4), i4 = 4 * (u % (DK / 4));
      float4 e4 = make_float4(0.f, 0.f, 0.f, 0.f), w4 = e4;
      if (t < n) {
        e4 = __ldg(reinterpret_cast<const float4 *>(ebp + t * gld + i4));
        w4 = __ldg(reinterpret_cast<const float4 *>(wwp + t * gld + i4));
      }
      const float k0 = __bfloat162float(sK[t * LDB + i4]), k1 = __bfloat162float(sK[t * LDB + i4 + 1]),
                  k2 = __bfloat162float(sK[t * LDB + i4 + 2]), k3 = __bfloat162float(sK[t * LDB + i4 + 3]);
      if (ta != nullptr)
        *reinterpret_cast<float4 *>(ta + t * LDG + i4) = make_float4(e4.x * k0, e4.y * k1, e4.z * k2, e4.w * k3);
      if (td != nullptr)
        *reinterpret_cast<float4 *>(td + t * LDG + i4) =
            make_float4((w4.x - e4.x) * k0, (w4.y - e4.y) * k1, (w4.z - e4.z) * k2, (w4.w - e4.w) * k3);
    }
  };
  // the staged tiles' views (regions: E and W at the start and at the end, W and dE for P^a and P^d)
  auto fsT = [&](const float *tile, const float *ref, float sg) { return FacF<true>{tile, sgam, ref, sg}; };
  // KDA at d_v = 128: the factored tiles x o 2^(sg (gamma - ref)) (x = K, or Q) staged whole as fp32
  // (rows of LDG) where a region of that size is free, the same values the factored views compute
  constexpr bool KST = CHAN && !G2 && DV == 128;
  auto stage_fac = [&](float *dst, bool from_q, const float *ref, float sg) {
#pragma unroll
    for (int u = tid; u < C * DK / 4; u += NTL) {
      const int t = u / (DK / 4), i4 = 4 * (u % (DK / 4));
      float x[4];
      if (from_q) {
        if constexpr (QVG) {
          uint2 raw = make_uint2(0u, 0u);
          if (t < n) raw = __ldg(reinterpret_cast<const uint2 *>(p.q + row(t) * DK + i4));
          const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
          const float2 a0 = __bfloat1622float2(h2[0]), a1 = __bfloat1622float2(h2[1]);
          x[0] = a0.x; x[1] = a0.y; x[2] = a1.x; x[3] = a1.y;
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) x[e] = __bfloat162float(sQ[t * LDB + i4 + e]);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) x[e] = __bfloat162float(sK[t * LDB + i4 + e]);
      }
      const float4 g4 = *reinterpret_cast<const float4 *>(sgam + t * LDG + i4);
      const float4 r4 = *reinterpret_cast<const float4 *>(ref + i4);
      *reinterpret_cast<float4 *>(dst + t * LDG + i4) =
          make_float4(x[0] * ex2(sg * (g4.x - r4.x)), x[1] * ex2(sg * (g4.y - r4.y)), x[2] * ex2(sg * (g4.z - r4.z)),
                      x[3] * ex2(sg * (g4.w - r4.w)));
    }
  };

  // ---- A = tril(Diag(beta) (D o K K^T), -1), stored transposed and tf32-rounded for the solve
  {
    float g[CC::NT][4];
    zero(g);
    if constexpr (GST) {   // a over E, d over W, K o a_ over dE (nothing yet)
      stage_gated(sE, sW);
      stage_fac(sdE, false, sgm, 1.f);
      __syncthreads();
      wmm<CC::NT, false>(g, F{sdE, LDG}, fsT(sE, sgm, -1.f), DK, mc, nc, lane);
    } else if constexpr (G2) {
      wmm<CC::NT, false>(g, kfac(sgm, 1.f), afacT(sgm, -1.f), DK, mc, nc, lane);
    } else if constexpr (KST) {   // K o a_ over E, K o b over W
      stage_fac(sE, false, sgm, 1.f);
      stage_fac(sW, false, sgm, -1.f);
      __syncthreads();
      wmm1<CC::NT, false>(g, F{sE, LDG}, FT{sW, LDG}, DK, mc, nc, lane);
    } else if constexpr (CHAN) {
      wmm1<CC::NT, false>(g, kfac(sgm, 1.f), kfacT(sgm, -1.f), DK, mc, nc, lane);
    } else {
      wmm<CC::NT, false>(g, BK{sK, LDB}, BKT{sK, LDB}, DK, mc, nc, lane);
    }
    each(g, mc, nc, lane, [&](int t, int r, float &x) {
      const float d = CHAN ? 1.f : ex2(sG[t] - sG[r]);
      sA[r * LD + t] = tf32r(r < t ? (G2 ? 1.f : sbeta[t]) * d * x : 0.f);
    });
  }
  __syncthreads();
  solve_unit_lower_64(sA, sT, tid, warp, lane);   // ends with a barrier
  for (int i = tid; i < C * C; i += NTL) {
    const int m = i / C, j = i % C;
    if (j > m) sT[m * LD + j] = 0.f;
  }
  __syncthreads();

  if constexpr (G2) {   // Zt = I - tril((K o a_)(d o b)^T, -1) to scratch, then R = T Zt (over P)
    {
      float g[CC::NT][4];
      zero(g);
      if constexpr (GST) {
        wmm<CC::NT, false>(g, F{sdE, LDG}, fsT(sW, sgm, -1.f), DK, mc, nc, lane);
      } else {
        wmm<CC::NT, false>(g, kfac(sgm, 1.f), dfacT(sgm, -1.f), DK, mc, nc, lane);
      }
      each(g, mc, nc, lane,
           [&](int t, int r, float &x) { scZ[t * C + r] = r == t ? 1.f : (r < t ? -x : 0.f); });
    }
    __syncthreads();
    float acc[CC::NT][4];
    zero(acc);
    wmm<CC::NT, false>(acc, TX{sT, LD}, F{scZ, C}, C, mc, nc, lane);
    each(acc, mc, nc, lane, [&](int t, int r, float &x) { sP[t * LDC + r] = x; });
    __syncthreads();
  }
  // ---- U' = T Diag(beta) V (GDN-2: T Zt V) and W = T Diag(beta e) K; E = U' - W S0
  float ue[CV::NT][4];
  zero(ue);
  if constexpr (G2) {
    wmm<CV::NT, false>(ue, F{sP, LDC}, vm(), C, mv, nv, lane);
  } else {
    wmm<CV::NT, false>(ue, TX{sT, LD}, vm(), C, mv, nv, lane, sbeta);
  }
  {
    float w[CK::NT][4];
    zero(w);
    if constexpr (G2) {
      wmm<CK::NT, false>(w, TX{sT, LD}, kfac(szero, 1.f), C, mk, nk, lane);
    } else if constexpr (KST) {   // K o e over E (E not yet computed)
      stage_fac(sE, false, szero, 1.f);
      __syncthreads();
      wmm<CK::NT, false>(w, TX{sT, LD}, F{sE, LDG}, C, mk, nk, lane, sbeta);
    } else if constexpr (CHAN) {
      wmm<CK::NT, false>(w, TX{sT, LD}, kfac(szero, 1.f), C, mk, nk, lane, sbeta);
    } else {
      wmm<CK::NT, false>(w, TX{sT, LD}, BK{sK, LDB}, C, mk, nk, lane, sbe);
    }
    each(w, mk, nk, lane, [&](int t, int i, float &x) { sW[t * LDW + i] = x; });
  }
  // S0 through shared memory (over dE, A and P, none of which holds data yet):
  // E = U' - W S0 and dq's first part, scale Diag(e) dO S0^T
  float dqT[KC::NT][4];
  if constexpr (G2) __syncthreads();   // R (over P) is read before S0 lands over it
  if constexpr (CHAN) {
    float *sS = reinterpret_cast<float *>(sm + L::DE);
#pragma unroll
    for (int i = tid; i < DK * DV / 4; i += NTL) {
      const int r = i / (DV / 4), c4 = i % (DV / 4);
      *reinterpret_cast<float4 *>(sS + r * LDF + 4 * c4) = __ldg(reinterpret_cast<const float4 *>(S0) + i);
    }
    __syncthreads();
    wmm<CV::NT, true>(ue, F{sW, LDW}, F{sS, LDF}, DK, mv, nv, lane);
    each(ue, mv, nv, lane, [&](int t, int v, float &x) { sE[t * LDF + v] = x; });
    zero(dqT);
    wmm<KC::NT, false>(dqT, F{sS, LDF}, BKT{sO, LDBV}, DV, mt, nt, lane);
  } else {
    __half *sS = reinterpret_cast<__half *>(sm + L::DE);
#pragma unroll
    for (int i = tid; i < DK * DV / 8; i += NTL) {
      const int r = i / (DV / 8), c8 = i % (DV / 8);
      *reinterpret_cast<uint4 *>(sS + r * L::LDS + 8 * c8) = __ldg(reinterpret_cast<const uint4 *>(S0) + i);
    }
    __syncthreads();
    wmm<CV::NT, true>(ue, F{sW, LDW}, HS{sS, L::LDS}, DK, mv, nv, lane);
    each(ue, mv, nv, lane, [&](int t, int v, float &x) { sE[t * LDF + v] = x; });
    zero(dqT);
    wmm<KC::NT, false>(dqT, HS{sS, L::LDS}, BKT{sO, LDBV}, DV, mt, nt, lane);
  }
  each(dqT, mt, nt, lane, [&](int i, int t, float &x) { x *= p.scale * (CHAN ? ex2(sgam[t * LDG + i]) : see[t]); });
  __syncthreads();   // S0's staging is read: P may overwrite it
  if constexpr (GST) {   // a over W (dead since E), d over dE (nothing yet) for P^a and P^d
    stage_gated(sW, sdE);
    __syncthreads();
  }
  // ---- dE = Diag(f) K dS + P^T dO, P = scale tril(D o Q K^T) (into dP's tile first).  The
  // reverse carry's own dE is Diag(beta) dE (its records carry beta in P and Kt), so it is
  // recomputed here rather than divided by beta.
  {
    float gq[CC::NT][4];
    zero(gq);
    if constexpr (GST) {
      wmm<CC::NT, false>(gq, qa(), fsT(sW, sgm, -1.f), DK, mc, nc, lane);
    } else if constexpr (G2) {
      wmm<CC::NT, false>(gq, qa(), afacT(sgm, -1.f), DK, mc, nc, lane);
    } else if constexpr (KST) {   // Q o a_ over W (dead since E), K o b over dE (nothing yet)
      stage_fac(sW, true, sgm, 1.f);
      stage_fac(sdE, false, sgm, -1.f);
      __syncthreads();
      wmm1<CC::NT, false>(gq, F{sW, LDG}, FT{sdE, LDG}, DK, mc, nc, lane);
    } else if constexpr (CHAN) {
      wmm1<CC::NT, false>(gq, qa(), kfacT(sgm, -1.f), DK, mc, nc, lane);
    } else {
      wmm<CC::NT, false>(gq, BK{sQ, LDB}, BKT{sK, LDB}, DK, mc, nc, lane);
    }
    each(gq, mc, nc, lane, [&](int t, int r, float &x) {
      sP[t * LDC + r] = r <= t ? p.scale * (CHAN ? 1.f : ex2(sG[t] - sG[r])) * x : 0.f;
    });
  }
  if constexpr (G2) {   // P^d to scratch
    float gq[CC::NT][4];
    zero(gq);
    if constexpr (GST) {
      wmm<CC::NT, false>(gq, qa(), fsT(sdE, sgm, -1.f), DK, mc, nc, lane);
    } else {
      wmm<CC::NT, false>(gq, qa(), dfacT(sgm, -1.f), DK, mc, nc, lane);
    }
    each(gq, mc, nc, lane, [&](int t, int r, float &x) { scPd[t * C + r] = r <= t ? p.scale * x : 0.f; });
  }
  __syncthreads();
  // ---- with dS through shared memory in 64-column halves (over W, which E has
  // finished reading): dE's columns of the half, and dk^T's first part
  // (Diag(f) E dS^T)^T / s accumulated over the halves
  float dkT[KC::NT][4];
  float dgp[KC::NT][2];   // scalar decay: this thread's column sums toward dg_t (columns n0 + 8 j + 2 t + e)
  float dgT[KC::NT][4];   // channel decay: dg^T, the tile of dkT
  float x1k = 0.f;
  zero(dkT);
  zero(dgT);
#pragma unroll
  for (int j = 0; j < KC::NT; ++j) dgp[j][0] = dgp[j][1] = 0.f;
  auto add_dg = [&](int j, int e, float y) {
    if constexpr (CHAN) {
      dgT[j][e] += y;
    } else {
      dgp[j][e & 1] += y;
    }
  };
  {
    using CH = Tiling<C, 64, LW>;
    const int mh = CH::m0(warp), nh = CH::n0(warp);
    float *sH = reinterpret_cast<float *>(sm + L::W);
    for (int h = 0; h < DV / 64; ++h) {
#pragma unroll
      for (int i = tid; i < DK * 32; i += NTL) {   // float2 pairs of the half
        const int r = i >> 5, c2 = i & 31;
        *reinterpret_cast<float2 *>(sH + r * L::LDH + 2 * c2) =
            __ldg(reinterpret_cast<const float2 *>(dS + r * DV + 64 * h) + c2);
      }
      __syncthreads();
      float acc[CH::NT][4];
      zero(acc);
      if constexpr (G2) {
        wmm<CH::NT, false>(acc, afac(sgC, -1.f), F{sH, L::LDH}, DK, mh, nh, lane);
        each(acc, mh, nh, lane, [&](int, int, float &x) { x *= inv_s; });
      } else if constexpr (CHAN) {
        wmm<CH::NT, false>(acc, kfac(sgC, -1.f), F{sH, L::LDH}, DK, mh, nh, lane);
        each(acc, mh, nh, lane, [&](int, int, float &x) { x *= inv_s; });
      } else {
        wmm<CH::NT, false>(acc, BK{sK, LDB}, F{sH, L::LDH}, DK, mh, nh, lane);
        each(acc, mh, nh, lane, [&](int t, int, float &x) { x *= sff[t] * inv_s; });
      }
      wmm<CH::NT, false>(acc, FT{sP, LDC}, BK{sO + 64 * h, LDBV}, C, mh, nh, lane);
      each(acc, mh, nh, lane, [&](int t, int v, float &x) { sdE[t * LDF + 64 * h + v] = x; });
      wmm<KC::NT, false>(dkT, F{sH, L::LDH}, FT{sE + 64 * h, LDF}, 64, mt, nt, lane);
      if constexpr (G2) {   // V dS^T (in dgT, still zero) and (d o f) dS / s to scratch
        wmm<KC::NT, false>(dgT, F{sH, L::LDH}, vmTh(64 * h), 64, mt, nt, lane);
        zero(acc);
        wmm<CH::NT, false>(acc, dfac(sgC, -1.f), F{sH, L::LDH}, DK, mh, nh, lane);
        each(acc, mh, nh, lane, [&](int t, int v, float &x) { scDv[t * DV + 64 * h + v] = x * inv_s; });
      }
      __syncthreads();   // the half is read before the next one (or dW^T) lands over it
    }
  }
  if constexpr (G2) {   // f o E dS^T and f o V dS^T start da and dd; their sum with a, d for the last token
    float x1r[2] = {0.f, 0.f};
    each_je(dkT, mt, nt, lane, [&](int j, int e, int i, int t, float &x) {
      const float f = ex2(sgC[i] - sgam[t * LDG + i]) * inv_s;
      const float da = x * f, dd = dgT[j][e] * f;
      scDa[t * DK + i] = da;
      scDd[t * DK + i] = dd;
      const float kv = __bfloat162float(sK[t * LDB + i]), eb = gate(ebp, t, i), ww = gate(wwp, t, i);
      x1r[e >> 1] += (da * eb + dd * (ww - eb)) * kv;
      x = 0.f;
      dgT[j][e] = 0.f;
    });
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const float s2 = quad_sum(x1r[h2]);
      if ((lane & 3) == 0) atomicAdd(&sx1k[mt + (lane >> 2) + 8 * h2], s2);
    }
  } else {
    float x1r[2] = {0.f, 0.f};   // channel decay: rows mt + g, mt + g + 8 of sum_t X1 o K
    each_je(dkT, mt, nt, lane, [&](int j, int e, int i, int t, float &x) {
      x *= (CHAN ? ex2(sgC[i] - sgam[t * LDG + i]) : sff[t]) * inv_s;
      const float y = x * __bfloat162float(sK[t * LDB + i]);
      if constexpr (CHAN) {
        x1r[e >> 1] += y;
      } else {
        x1k += y;
      }
      add_dg(j, e, -y);
    });
    if constexpr (CHAN) {
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const float s2 = quad_sum(x1r[h2]);
        if ((lane & 3) == 0) atomicAdd(&sx1k[mt + (lane >> 2) + 8 * h2], s2);
      }
    }
  }
  // ---- dP = tril(dO E^T)
  {
    float acc[CC::NT][4];
    zero(acc);
    wmm<CC::NT, false>(acc, BK{sO, LDBV}, FT{sE, LDF}, DV, mc, nc, lane);
    each(acc, mc, nc, lane, [&](int t, int r, float &x) { sP[t * LDC + r] = r <= t ? x : 0.f; });
  }
  // ---- dW^T = -S0 dE^T  (d_k x C, over W), S0 through shared memory again, over
  // E once dP has read it (fp32 S0: in halves at d_v = 128, else from global memory)
  {
    float acc[KC::NT][4];
    zero(acc);
    if constexpr (!CHAN) {
      __syncthreads();   // dP has read E
      __half *sH = reinterpret_cast<__half *>(sm + L::E);
#pragma unroll
      for (int i = tid; i < DK * DV / 8; i += NTL) {
        const int r = i / (DV / 8), c8 = i % (DV / 8);
        const uint4 u = __ldg(reinterpret_cast<const uint4 *>(S0) + i);   // rows of LDSE halves: 8-byte aligned
        *reinterpret_cast<uint2 *>(sH + r * L::LDSE + 8 * c8) = make_uint2(u.x, u.y);
        *reinterpret_cast<uint2 *>(sH + r * L::LDSE + 8 * c8 + 4) = make_uint2(u.z, u.w);
      }
      __syncthreads();
      wmm<KC::NT, true>(acc, HS{sH, L::LDSE}, FT{sdE, LDF}, DV, mt, nt, lane);
    } else if constexpr (L::kS0HalvesOverE) {
      __syncthreads();   // dP has read E
      float *sH = reinterpret_cast<float *>(sm + L::E);
      for (int h = 0; h < DV / 64; ++h) {
#pragma unroll
        for (int i = tid; i < DK * 32; i += NTL) {
          const int r = i >> 5, c2 = i & 31;
          *reinterpret_cast<float2 *>(sH + r * L::LDH + 2 * c2) =
              __ldg(reinterpret_cast<const float2 *>(S0 + r * DV + 64 * h) + c2);
        }
        __syncthreads();
        wmm<KC::NT, true>(acc, F{sH, L::LDH}, FT{sdE + 64 * h, LDF}, 64, mt, nt, lane);
        __syncthreads();
      }
    } else {
      wmm<KC::NT, true>(acc, FG{reinterpret_cast<const float *>(S0), DV}, FT{sdE, LDF}, DV, mt, nt, lane);
    }
    each(acc, mt, nt, lane, [&](int i, int t, float &x) { sW[i * LDC + t] = x; });
  }
  __syncthreads();

  // ---- dv = Diag(beta) T^T dE;  dbeta += rowsum(V o T^T dE)
  // (GDN-2: tU = T^T dE over E, dv = Zt^T tU + P^d^T dO + (d o f) dS, dA^d = -tril(tU V^T, -1))
  if constexpr (G2) {
    {
      float acc[CV::NT][4];
      zero(acc);
      wmm<CV::NT, false>(acc, TXT{sT, LD}, F{sdE, LDF}, C, mv, nv, lane);
      each(acc, mv, nv, lane, [&](int t, int v, float &x) { sE[t * LDF + v] = x; });
    }
    __syncthreads();
    {
      float acc[CV::NT][4];
      zero(acc);
      wmm<CV::NT, false>(acc, FT{scZ, C}, F{sE, LDF}, C, mv, nv, lane);
      wmm<CV::NT, false>(acc, FT{scPd, C}, BK{sO, LDBV}, C, mv, nv, lane);
      each(acc, mv, nv, lane, [&](int t, int v, float &x) { x += scDv[t * DV + v]; });
      const int g = lane >> 2, tq = lane & 3;
#pragma unroll
      for (int j = 0; j < CV::NT; ++j)
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int t = mv + g + 8 * h2, v = nv + 8 * j + 2 * tq;
          if (t < n)
            *reinterpret_cast<uint32_t *>(p.dv + row(t) * DV + v) =
                pack_bf16x2(acc[j][2 * h2], acc[j][2 * h2 + 1]);
        }
    }
    {
      float acc[CC::NT][4];
      zero(acc);
      wmm<CC::NT, true>(acc, F{sE, LDF}, vmT(), DV, mc, nc, lane);
      each(acc, mc, nc, lane, [&](int t, int r, float &x) { scAd[t * C + r] = r < t ? x : 0.f; });
    }
  } else {
    float acc[CV::NT][4];
    zero(acc);
    wmm<CV::NT, false>(acc, TXT{sT, LD}, F{sdE, LDF}, C, mv, nv, lane);
    float part[2] = {0.f, 0.f};   // rows g and g + 8 of the tile
    each_je(acc, mv, nv, lane, [&](int, int e, int t, int v, float &x) {
      part[e >> 1] = fmaf(vat(t, v), x, part[e >> 1]);
      x *= sbeta[t];
    });
    const int g = lane >> 2, tq = lane & 3;
#pragma unroll
    for (int j = 0; j < CV::NT; ++j)
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {   // two adjacent values per store
        const int t = mv + g + 8 * h2, v = nv + 8 * j + 2 * tq;
        if (t < n)
          *reinterpret_cast<uint32_t *>(p.dv + row(t) * DV + v) = pack_bf16x2(acc[j][2 * h2], acc[j][2 * h2 + 1]);
      }
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const float s2 = quad_sum(part[h2]);
      if (tq == 0) atomicAdd(&sdb[mv + g + 8 * h2], s2);
    }
  }
  // ---- (T^T dW)^T = dW^T T:  dk += Diag(beta e) T^T dW;  dbeta += e o rowsum(K o T^T dW)
  {
    float acc[KC::NT][4];
    zero(acc);
    wmm<KC::NT, false>(acc, F{sW, LDC}, TX{sT, LD}, C, mt, nt, lane);
    float dbp[KC::NT][2];
#pragma unroll
    for (int j = 0; j < KC::NT; ++j) dbp[j][0] = dbp[j][1] = 0.f;
#pragma unroll
    for (int j = 0; j < KC::NT; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = mt + (lane >> 2) + 8 * (e >> 1), t = nt + 8 * j + 2 * (lane & 3) + (e & 1);
        const float kv = __bfloat162float(sK[t * LDB + i]);
        const float et = CHAN ? ex2(sgam[t * LDG + i]) : see[t];
        const float y = (G2 ? et : CHAN ? sbeta[t] * et : sbe[t]) * acc[j][e];
        dkT[j][e] += y;
        add_dg(j, e, y * kv);
        dbp[j][e & 1] = fmaf(et * kv, acc[j][e], dbp[j][e & 1]);
      }
    if constexpr (!G2) {
#pragma unroll
      for (int j = 0; j < KC::NT; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float s2 = column_sum(dbp[j][e]);
          if (lane < 4) atomicAdd(&sdb[nt + 8 * j + 2 * lane + e], s2);
        }
    }
  }
  // ---- dT = dE V^T Diag(beta) + dW K^T Diag(beta e)  (over A^T, dead since the solve;
  // GDN-2: dE V^T Zt^T + dW (K o e)^T)
  if constexpr (G2) {
    float a2[CC::NT][4];
    {   // (full precision: d erase is the small difference of two gradients built from these)
      float a1[CC::NT][4];
      zero(a1);
      wmm<CC::NT, false>(a1, F{sdE, LDF}, vmT(), DV, mc, nc, lane);
      each(a1, mc, nc, lane, [&](int t, int r, float &x) { sA[t * LD + r] = x; });
    }
    zero(a2);
    if constexpr (GST) {   // K o e over E, once every warp has read tU there
      __syncthreads();
      stage_fac(sE, false, szero, 1.f);
      __syncthreads();
      wmm<CC::NT, false>(a2, FT{sW, LDC}, FT{sE, LDG}, DK, mc, nc, lane);
    } else {
      wmm<CC::NT, false>(a2, FT{sW, LDC}, kfacT(szero, 1.f), DK, mc, nc, lane);
      __syncthreads();
    }
    wmm<CC::NT, false>(a2, F{sA, LD}, FT{scZ, C}, C, mc, nc, lane);
    __syncthreads();
    each(a2, mc, nc, lane, [&](int t, int r, float &x) { sA[t * LD + r] = x; });
  } else {
    float a1[CC::NT][4], a2[CC::NT][4];
    zero(a1);
    zero(a2);
    wmm1<CC::NT, false>(a1, F{sdE, LDF}, vmT(), DV, mc, nc, lane);
    if constexpr (KST) {   // K o e over E (dead since dW)
      stage_fac(sE, false, szero, 1.f);
      __syncthreads();
      wmm1<CC::NT, false>(a2, FT{sW, LDC}, FT{sE, LDG}, DK, mc, nc, lane);
    } else if constexpr (CHAN) {
      wmm1<CC::NT, false>(a2, FT{sW, LDC}, kfacT(szero, 1.f), DK, mc, nc, lane);
    } else {
      wmm1<CC::NT, false>(a2, FT{sW, LDC}, BKT{sK, LDB}, DK, mc, nc, lane);
    }
#pragma unroll
    for (int j = 0; j < CC::NT; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int t = mc + (lane >> 2) + 8 * (e >> 1), r = nc + 8 * j + 2 * (lane & 3) + (e & 1);
        sA[t * LD + r] = CHAN ? sbeta[r] * (a1[j][e] + a2[j][e]) : sbeta[r] * a1[j][e] + sbe[r] * a2[j][e];
      }
  }
  __syncthreads();
  // ---- X = dT T^T (over E), then dA = tril(-T^T X, -1) (over dT)
  {
    float acc[CC::NT][4];
    zero(acc);
    if constexpr (G2) {
      wmm<CC::NT, false>(acc, F{sA, LD}, TXT{sT, LD}, C, mc, nc, lane);
    } else {
      wmm1<CC::NT, false>(acc, F{sA, LD}, TXT{sT, LD}, C, mc, nc, lane);
    }
    each(acc, mc, nc, lane, [&](int t, int r, float &x) { sE[t * LDC + r] = x; });
  }
  __syncthreads();
  {
    float acc[CC::NT][4];
    zero(acc);
    if constexpr (G2) {
      wmm<CC::NT, true>(acc, TXT{sT, LD}, F{sE, LDC}, C, mc, nc, lane);
    } else {
      wmm1<CC::NT, true>(acc, TXT{sT, LD}, F{sE, LDC}, C, mc, nc, lane);
    }
    each(acc, mc, nc, lane, [&](int t, int r, float &x) { sA[t * LD + r] = r < t ? x : 0.f; });
  }
  __syncthreads();
  // ---- G = K K^T again: dbeta += rowsum(dA o D o G); N1 = Diag(beta) (dA o D), N2 = scale (dP o D)
  // (GDN-2: N1 = dA; N2a = scale dP in place, N2d = scale tril(dO V^T) over T, dead since dA)
  if constexpr (G2) {
    for (int i = tid; i < C * C; i += NTL) {
      const int t = i / C, r = i % C;
      sP[t * LDC + r] *= p.scale;
    }
    float acc[CC::NT][4];
    zero(acc);
    wmm<CC::NT, false>(acc, BK{sO, LDBV}, vmT(), DV, mc, nc, lane);
    each(acc, mc, nc, lane, [&](int t, int r, float &x) { sT[t * LD + r] = r <= t ? p.scale * x : 0.f; });
  } else {
    if constexpr (KST) {   // K o a_ over E (X is dead), K o b over W (dW^T is dead), Q o a_ over dE
      stage_fac(sE, false, sgm, 1.f);
      stage_fac(sW, false, sgm, -1.f);
      stage_fac(sdE, true, sgm, 1.f);
      __syncthreads();
    }
    float g[CC::NT][4];
    zero(g);
    if constexpr (KST) {
      wmm1<CC::NT, false>(g, F{sE, LDG}, FT{sW, LDG}, DK, mc, nc, lane);
    } else if constexpr (CHAN) {
      wmm1<CC::NT, false>(g, kfac(sgm, 1.f), kfacT(sgm, -1.f), DK, mc, nc, lane);
    } else {
      wmm<CC::NT, false>(g, BK{sK, LDB}, BKT{sK, LDB}, DK, mc, nc, lane);
    }
    float part[2] = {0.f, 0.f};
    each_je(g, mc, nc, lane, [&](int, int e, int t, int r, float &x) {
      const float d = r <= t ? (CHAN ? 1.f : ex2(sG[t] - sG[r])) : 0.f;
      const float da = sA[t * LD + r];
      // dA is strictly lower; above the diagonal the factored Gram may overflow (0 inf = NaN)
      if (r < t) part[e >> 1] = fmaf(da * d, x, part[e >> 1]);
      sA[t * LD + r] = sbeta[t] * da * d;
      sP[t * LDC + r] = p.scale * sP[t * LDC + r] * d;
    });
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const float s2 = quad_sum(part[h2]);
      if ((lane & 3) == 0) atomicAdd(&sdb[mc + (lane >> 2) + 8 * h2], s2);
    }
  }
  __syncthreads();
  // ---- dk += N1 K + N1^T K + N2^T Q   (as K^T N1^T, K^T N1, Q^T N2)
  if constexpr (G2) {
    if constexpr (GST) {   // a over E (X is dead), d over W (dW^T is dead), K o a_ over dE (dead)
      stage_gated(sE, sW);
      stage_fac(sdE, false, sgm, 1.f);
      __syncthreads();
    }
    {   // dKa = dA (a o b) + dA^d (d o b): dk += a_ o dKa, dg += dKa o Ka
      float acc[KC::NT][4];
      zero(acc);
      if constexpr (GST) {
        wmm<KC::NT, false>(acc, fsT(sE, sgm, -1.f), FT{sA, LD}, C, mt, nt, lane);
        wmm<KC::NT, false>(acc, fsT(sW, sgm, -1.f), FT{scAd, C}, C, mt, nt, lane);
      } else {
        wmm<KC::NT, false>(acc, afacT(sgm, -1.f), FT{sA, LD}, C, mt, nt, lane);
        wmm<KC::NT, false>(acc, dfacT(sgm, -1.f), FT{scAd, C}, C, mt, nt, lane);
      }
      each_je(acc, mt, nt, lane, [&](int j, int e, int i, int t, float &x) {
        x *= ex2(sgam[t * LDG + i] - sgm[i]);
        add_dg(j, e, x * __bfloat162float(sK[t * LDB + i]));
        dkT[j][e] += x;
      });
    }
    {   // da += b o (dA^T Ka + N2a^T Qa),  dd += b o (dA^d^T Ka + N2d^T Qa)
      float acc[KC::NT][4];
      zero(acc);
      if constexpr (GST) {
        wmm<KC::NT, false>(acc, FT{sdE, LDG}, F{sA, LD}, C, mt, nt, lane);
      } else {
        wmm<KC::NT, false>(acc, kfacT(sgm, 1.f), F{sA, LD}, C, mt, nt, lane);
      }
      wmm<KC::NT, false>(acc, qaT(), F{sP, LDC}, C, mt, nt, lane);
      each(acc, mt, nt, lane,
           [&](int i, int t, float &x) { scDa[t * DK + i] += x * ex2(sgm[i] - sgam[t * LDG + i]); });
      zero(acc);
      if constexpr (GST) {
        wmm<KC::NT, false>(acc, FT{sdE, LDG}, F{scAd, C}, C, mt, nt, lane);
      } else {
        wmm<KC::NT, false>(acc, kfacT(sgm, 1.f), F{scAd, C}, C, mt, nt, lane);
      }
      wmm<KC::NT, false>(acc, qaT(), F{sT, LD}, C, mt, nt, lane);
      each(acc, mt, nt, lane,
           [&](int i, int t, float &x) { scDd[t * DK + i] += x * ex2(sgm[i] - sgam[t * LDG + i]); });
    }
    {   // dq += a_ o (N2a (a o b) + N2d (d o b))
      float acc[KC::NT][4];
      zero(acc);
      if constexpr (GST) {
        wmm<KC::NT, false>(acc, fsT(sE, sgm, -1.f), FT{sP, LDC}, C, mt, nt, lane);
        wmm<KC::NT, false>(acc, fsT(sW, sgm, -1.f), FT{sT, LD}, C, mt, nt, lane);
      } else {
        wmm<KC::NT, false>(acc, afacT(sgm, -1.f), FT{sP, LDC}, C, mt, nt, lane);
        wmm<KC::NT, false>(acc, dfacT(sgm, -1.f), FT{sT, LD}, C, mt, nt, lane);
      }
      each_je(acc, mt, nt, lane,
              [&](int j, int e, int i, int t, float &x) { dqT[j][e] += x * ex2(sgam[t * LDG + i] - sgm[i]); });
    }
    // the gates' gradients; dk += b o da + (w - b) o dd;  dg -= da o a + dd o d
    each_je(dkT, mt, nt, lane, [&](int j, int e, int i, int t, float &x) {
      const float da = scDa[t * DK + i], dd = scDd[t * DK + i];
      const float kv = __bfloat162float(sK[t * LDB + i]), eb = gate(ebp, t, i), ww = gate(wwp, t, i);
      x += eb * da + (ww - eb) * dd;
      add_dg(j, e, -(da * eb + dd * (ww - eb)) * kv);
      if (t < n) {
        p.d_erase[row(t) * DK + i] = kv * (da - dd);
        p.d_write[row(t) * DK + i] = kv * dd;
      }
    });
  } else {
    float acc[KC::NT][4];
    zero(acc);
    if constexpr (KST) {
      wmm<KC::NT, false>(acc, FT{sW, LDG}, FT{sA, LD}, C, mt, nt, lane);
    } else if constexpr (CHAN) {
      wmm<KC::NT, false>(acc, kfacT(sgm, -1.f), FT{sA, LD}, C, mt, nt, lane);
    } else {
      wmm1<KC::NT, false>(acc, BKT{sK, LDB}, FT{sA, LD}, C, mt, nt, lane);
    }
    each_je(acc, mt, nt, lane, [&](int j, int e, int i, int t, float &x) {
      if constexpr (CHAN) x *= ex2(sgam[t * LDG + i] - sgm[i]);
      add_dg(j, e, x * __bfloat162float(sK[t * LDB + i]));
      dkT[j][e] += x;
    });
    zero(acc);
    if constexpr (KST) {
      wmm<KC::NT, false>(acc, FT{sE, LDG}, F{sA, LD}, C, mt, nt, lane);
      wmm<KC::NT, false>(acc, FT{sdE, LDG}, F{sP, LDC}, C, mt, nt, lane);
    } else if constexpr (CHAN) {
      wmm<KC::NT, false>(acc, kfacT(sgm, 1.f), F{sA, LD}, C, mt, nt, lane);
      wmm<KC::NT, false>(acc, qaT(), F{sP, LDC}, C, mt, nt, lane);
    } else {
      wmm1<KC::NT, false>(acc, BKT{sK, LDB}, F{sA, LD}, C, mt, nt, lane);
      wmm1<KC::NT, false>(acc, BKT{sQ, LDB}, F{sP, LDC}, C, mt, nt, lane);
    }
    each_je(acc, mt, nt, lane, [&](int j, int e, int i, int t, float &x) {
      if constexpr (CHAN) x *= ex2(sgm[i] - sgam[t * LDG + i]);
      add_dg(j, e, -x * __bfloat162float(sK[t * LDB + i]));
      dkT[j][e] += x;
    });
  }
  // ---- dq += N2 K (GDN-2: above)
  if constexpr (G2) {
  } else if constexpr (CHAN) {
    float acc[KC::NT][4];
    zero(acc);
    if constexpr (KST) {
      wmm<KC::NT, false>(acc, FT{sW, LDG}, FT{sP, LDC}, C, mt, nt, lane);
    } else {
      wmm<KC::NT, false>(acc, kfacT(sgm, -1.f), FT{sP, LDC}, C, mt, nt, lane);
    }
    each_je(acc, mt, nt, lane,
            [&](int j, int e, int i, int t, float &x) { dqT[j][e] += x * ex2(sgam[t * LDG + i] - sgm[i]); });
  } else {
    wmm1<KC::NT, false>(dqT, BKT{sK, LDB}, FT{sP, LDC}, C, mt, nt, lane);
  }
  each_je(dqT, mt, nt, lane, [&](int j, int e, int i, int t, float &x) { add_dg(j, e, x * qat(t, i)); });

  // ---- reductions: dg_t over the rows; sum(X1 o K); sum(dS o S0)
  {
    const float4 *a = reinterpret_cast<const float4 *>(dS);
    if constexpr (CHAN) {   // per state row (fp32 S0): DV / 4 lanes a row, every thread the same number of rows
      const float4 *bb = reinterpret_cast<const float4 *>(S0);
      constexpr int GL = DV / 4;
      static_assert((DK * DV / 4) % NTL == 0 && 32 % GL == 0, "row groups");
#pragma unroll 4
      for (int i = tid; i < DK * DV / 4; i += NTL) {
        const float4 x = __ldg(a + i), y = __ldg(bb + i);
        float ss = fmaf(x.x, y.x, fmaf(x.y, y.y, fmaf(x.z, y.z, x.w * y.w)));
#pragma unroll
        for (int o = GL / 2; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (lane % GL == 0) sss[i / GL] = ss;
      }
    } else {   // fp16 S0: eight products at a time
      const uint4 *bb = reinterpret_cast<const uint4 *>(S0);
      float ss = 0.f;
#pragma unroll
      for (int i = tid; i < DK * DV / 8; i += NTL) {
        const float4 x0 = __ldg(a + 2 * i), x1 = __ldg(a + 2 * i + 1);
        const uint4 w = __ldg(bb + i);
        const __half2 *y = reinterpret_cast<const __half2 *>(&w);
        const float2 y0 = __half22float2(y[0]), y1 = __half22float2(y[1]), y2 = __half22float2(y[2]),
                     y3 = __half22float2(y[3]);
        ss = fmaf(x0.x, y0.x, fmaf(x0.y, y0.y, fmaf(x0.z, y1.x, fmaf(x0.w, y1.y, ss))));
        ss = fmaf(x1.x, y2.x, fmaf(x1.y, y2.y, fmaf(x1.z, y3.x, fmaf(x1.w, y3.y, ss))));
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) {
        ss += __shfl_xor_sync(0xffffffffu, ss, o);
        x1k += __shfl_xor_sync(0xffffffffu, x1k, o);
      }
      if (lane == 0) {
        atomicAdd(&sred[0], x1k);
        atomicAdd(&sred[1], ss);
      }
#pragma unroll
      for (int j = 0; j < KC::NT; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float s2 = column_sum(dgp[j][e]);
          if (lane < 4) atomicAdd(&sdg[nt + 8 * j + 2 * lane + e], s2);
        }
    }
  }
  __syncthreads();

  // ---- KLA: beta = eta / (||k||^2 + eps) adds -2 dbeta beta / (||k||^2 + eps) k to dk;
  // then dk and dq through bf16 tiles (over W and E, both dead) for row-contiguous stores
  __nv_bfloat16 *stk = reinterpret_cast<__nv_bfloat16 *>(sE);
  __nv_bfloat16 *stq = reinterpret_cast<__nv_bfloat16 *>(sW);
  each(dkT, mt, nt, lane, [&](int i, int t, float &x) {
    if (p.kla) x = fmaf(-2.f * sdb[t] * sbeta[t] / (snk[t] + p.eps), __bfloat162float(sK[t * LDB + i]), x);
    stk[t * LDB + i] = __float2bfloat16_rn(x);
  });
  each(dqT, mt, nt, lane, [&](int i, int t, float &x) { stq[t * LDB + i] = __float2bfloat16_rn(x); });
  if constexpr (CHAN) {   // dg over the decay tile, which nothing reads any more
    each(dgT, mt, nt, lane, [&](int i, int t, float &x) { sgam[t * LDG + i] = x; });
  }
  __syncthreads();
  for (int i = tid; i < C * DK / 8; i += NTL) {
    const int t = i / (DK / 8), j = i % (DK / 8);
    if (t < n) {
      reinterpret_cast<uint4 *>(p.dk + row(t) * DK)[j] = *reinterpret_cast<const uint4 *>(stk + t * LDB + 8 * j);
      reinterpret_cast<uint4 *>(p.dq + row(t) * DK)[j] = *reinterpret_cast<const uint4 *>(stq + t * LDB + 8 * j);
    }
  }
  // ---- dbeta (d eta for KLA) and dlog_g = suffix sums of dg over the chunk's tokens
  if (tid < C) {
    const int t = tid;
    if (!G2 && t < n) p.dbeta[row(t)] = p.kla ? sdb[t] / (snk[t] + p.eps) : sdb[t];
    if (!CHAN && p.decay && p.dlog_g != nullptr) {
      float x = 0.f;
      if (t < n) x = sdg[t] + (t == n - 1 ? sred[0] + ex2(sG[n - 1]) * sred[1] * inv_s : 0.f);
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_down_sync(0xffffffffu, x, o);
        if (lane + o < 32) x += y;
      }
      sscan[t] = x;   // suffix sums within each warp
    }
  }
  __syncthreads();
  if (!CHAN && tid < C && p.decay && p.dlog_g != nullptr) {
    const int t = tid;
    const float x = sscan[t] + (t < 32 ? sscan[32] : 0.f);
    if (t < n) p.dlog_g[row(t)] = x;
  }
  if constexpr (CHAN) {   // per-channel suffix sums of dg, four 16-token parts per channel
    if (p.dlog_g != nullptr) {
      const int i = tid % DK, part = tid / DK;
      float *stot = sdE;   // part totals (dE is dead)
      float run = 0.f;
      for (int t = 16 * part + 15; t >= 16 * part; --t) {
        float x = t < n ? sgam[t * LDG + i] : 0.f;
        if (t == n - 1) x += sx1k[i] + ex2(sgC[i]) * sss[i] * inv_s;
        run += x;
        sgam[t * LDG + i] = run;
      }
      stot[part * DK + i] = run;
      __syncthreads();
      float off = 0.f;
      for (int q = part + 1; q < NTL / DK; ++q) off += stot[q * DK + i];
      for (int t = 16 * part; t < 16 * part + 16 && t < n; ++t) p.dlog_g[row(t) * DK + i] = sgam[t * LDG + i] + off;
    }
  }
}

int grid_for(size_t n) { return static_cast<int>(std::min<size_t>((n + 255) / 256, 4096)); }

}  // namespace
}  // namespace tc

BwdLayout bwd_layout(int variant, int B, int T, int H, int dv) {
  using namespace tc;
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t NC = (static_cast<size_t>(T) + C - 1) / C, bh = static_cast<size_t>(B) * H, ns = dv / 64;
  const size_t rb_f = variant == kGDN2 ? rec_bytes_gdn2(static_cast<int>(ns))
                      : variant == kKDA ? rec_bytes_chan(static_cast<int>(ns))
                                        : rec_bytes(static_cast<int>(ns));
  BwdLayout L;
  L.fwd_rec = 0;
  L.rev_rec = up(bh * NC * rb_f);
  L.s0s = L.rev_rec + up(bh * NC * rec_bytes_gdn2(static_cast<int>(ns)));
  const bool chan = variant == kKDA || variant == kGDN2;
  L.dss = L.s0s + up(bh * NC * DK * dv * (chan ? 4 : 2));   // S0: fp32 with channel decay
  L.x0 = L.dss + up(bh * NC * DK * dv * 4);
  L.xf = L.x0 + up(bh * DK * dv * 4);
  L.maps = L.xf + up(bh * DK * dv * 4);
  L.maps_bytes = gdr_split_segment_bytes(B, T, H, dv);
  L.absmax = L.maps + up(L.maps_bytes);
  L.total = L.absmax + 256;
  return L;
}

}  // namespace gdr

bool gdr_bwd_supported(int variant, int dtype_bf16, int dk, int dv) {
  using namespace gdr;
  const bool v = variant == kDeltaNet || variant == kGatedDeltaNet || variant == kKLA || variant == kKDA ||
                 variant == kGDN2;
  return v && dtype_bf16 && dk == 128 && (dv == 64 || dv == 128);
}

size_t gdr_bwd_workspace_bytes(int variant, int B, int T, int H, int dv) {
  return gdr::bwd_layout(variant, B, T, H, dv).total;
}

cudaError_t gdr_bwd_launch_scale(const gdr::BwdProblem &p, uint32_t *absmax, float *x0, cudaStream_t s) {
  using namespace gdr::tc;
  const gdr::FwdProblem &f = p.f;
  cudaError_t e = cudaMemsetAsync(absmax, 0, sizeof(uint32_t), s);
  if (e != cudaSuccess) return e;
  const size_t n_o = static_cast<size_t>(f.B) * f.T * f.H * f.dv, n_s = static_cast<size_t>(f.B) * f.H * f.dk * f.dv;
  // a grid-stride sweep of 16-byte loads (d_o) and floats (d_final), one atomic per block
  const int grid = static_cast<int>(std::min<size_t>((std::max(n_o / 8, n_s) + 255) / 256, 1024));
  bwd_absmax_kernel<<<std::max(grid, 1), 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(p.d_o), n_o, p.d_final,
                                                      n_s, absmax);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  bwd_scale_state_kernel<<<grid_for(n_s), 256, 0, s>>>(p.d_final, n_s, absmax, x0);
  return cudaGetLastError();
}

cudaError_t gdr_bwd_launch_rev_prep(const gdr::BwdProblem &p, const uint8_t *fwd_rec, uint8_t *rev_rec,
                                    const uint32_t *absmax, cudaStream_t s) {
  using namespace gdr::tc;
  const gdr::FwdProblem &f = p.f;
  RevPrepParams rp;
  rp.T = f.T; rp.H = f.H; rp.NC = (f.T + C - 1) / C;
  const int ns = f.dv / 64;
  rp.chan = f.variant == gdr::kKDA || f.variant == gdr::kGDN2;
  rp.rb_f = f.variant == gdr::kGDN2 ? rec_bytes_gdn2(ns) : rp.chan ? rec_bytes_chan(ns) : rec_bytes(ns);
  rp.rb_r = rec_bytes_gdn2(ns);
  rp.d_o = static_cast<const __nv_bfloat16 *>(p.d_o);
  rp.fwd = fwd_rec; rp.rev = rev_rec; rp.absmax = absmax;
  const int grid = f.B * f.H * rp.NC;
  auto run = [&](auto kern, int dv) {
    const size_t smem = (static_cast<size_t>(C) * (dv + 8) + C * (C + 8) + C * (DK + 8)) * 2;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    kern<<<grid, NT, smem, s>>>(rp);
    return cudaGetLastError();
  };
  return f.dv == 128 ? run(bwd_rev_prep_kernel<128>, 128) : run(bwd_rev_prep_kernel<64>, 64);
}

cudaError_t gdr_bwd_launch_local(const gdr::BwdProblem &p, const void *s0s, const float *dss,
                                 const uint32_t *absmax, uint8_t *fwd_rec, uint8_t *rev_rec, cudaStream_t s) {
  using namespace gdr::tc;
  const gdr::FwdProblem &f = p.f;
  LocalParams lp;
  lp.T = f.T; lp.H = f.H; lp.NC = (f.T + C - 1) / C;
  lp.decay = f.variant != gdr::kDeltaNet;
  lp.kla = f.variant == gdr::kKLA;
  lp.eps = f.eps; lp.scale = f.scale;
  lp.q = static_cast<const __nv_bfloat16 *>(f.q);
  lp.k = static_cast<const __nv_bfloat16 *>(f.k);
  lp.v = static_cast<const __nv_bfloat16 *>(f.v);
  lp.d_o = static_cast<const __nv_bfloat16 *>(p.d_o);
  lp.beta = f.beta; lp.log_g = f.log_g;
  lp.s0s = s0s; lp.dss = dss; lp.absmax = absmax;
  lp.dq = static_cast<__nv_bfloat16 *>(p.dq);
  lp.dk = static_cast<__nv_bfloat16 *>(p.dk);
  lp.dv = static_cast<__nv_bfloat16 *>(p.dv);
  lp.dbeta = p.dbeta; lp.dlog_g = p.dlog_g;
  lp.erase_b = f.erase_b; lp.write_w = f.write_w;
  lp.d_erase = p.d_erase; lp.d_write = p.d_write;
  lp.scr_f = fwd_rec; lp.scr_r = rev_rec;
  lp.rb_f = rec_bytes_gdn2(f.dv / 64); lp.rb_r = rec_bytes_gdn2(f.dv / 64);
  const int grid = f.B * f.H * lp.NC;
  auto run = [&](auto kern, size_t smem) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    kern<<<grid, NTL, smem, s>>>(lp);
    return cudaGetLastError();
  };
  if (f.variant == gdr::kGDN2)
    return f.dv == 128 ? run(bwd_local_kernel<128, true, true>, LocalSmem<128, true>::BYTES)
                       : run(bwd_local_kernel<64, true, true>, LocalSmem<64, true>::BYTES);
  if (f.variant == gdr::kKDA)
    return f.dv == 128 ? run(bwd_local_kernel<128, true>, LocalSmem<128, true>::BYTES)
                       : run(bwd_local_kernel<64, true>, LocalSmem<64, true>::BYTES);
  return f.dv == 128 ? run(bwd_local_kernel<128, false>, LocalSmem<128, false>::BYTES)
                     : run(bwd_local_kernel<64, false>, LocalSmem<64, false>::BYTES);
}

cudaError_t gdr_bwd_launch_unscale(const gdr::BwdProblem &p, const float *xf, const uint32_t *absmax,
                                   cudaStream_t s) {
  using namespace gdr::tc;
  if (p.d_s0 == nullptr) return cudaSuccess;
  const size_t n = static_cast<size_t>(p.f.B) * p.f.H * p.f.dk * p.f.dv;
  bwd_unscale_kernel<<<grid_for(n), 256, 0, s>>>(xf, n, absmax, p.d_s0);
  return cudaGetLastError();
}

int gdr_bwd_read_device_error(cudaStream_t s) {
  if (cudaStreamSynchronize(s) != cudaSuccess) return -1;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_gdr_bwd_error, sizeof(int)) != cudaSuccess) return -1;
  if (v != 0) {
    const int z = 0;
    if (cudaMemcpyToSymbol(g_gdr_bwd_error, &z, sizeof(int)) != cudaSuccess) return -1;
  }
  return v;
}
