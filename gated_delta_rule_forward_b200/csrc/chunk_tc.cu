// Chunked gated delta-rule forward on sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Chunk form of the recurrence.  Within a chunk of C = 64 tokens with start
// state S0, cumulative log decay gamma_t = sum_{r<=t} log g_r (inclusive),
// Gamma_t = exp(gamma_t), and a_t = c_t = beta_t k_t, unrolling
//     S_t = S~_t + beta_t k_t u_t^T,   u_t = v_t - S~_t^T k_t   ("Kaczmarz Linear
//     Attention", KLA update rule; the residual form of the delta rule)
// gives, with u_t stacked into U (C x dv):
//     u_t = v_t - Gamma_t S0^T k_t - sum_{r<t} beta_r (Gamma_t/Gamma_r)(k_t.k_r) u_r
//  => (I + A) U = V - Diag(Gamma) K S0,   A_tr = beta_r (Gamma_t/Gamma_r) k_t.k_r  (r < t)
//  => U = T V - (T Diag(Gamma)) K S0 = U' - W S0,  T = (I + A)^{-1}
//     O = Diag(Gamma) Q S0 + P U,           P_tr = beta_r (Gamma_t/Gamma_r) q_t.k_r (r <= t)
//     S_C = Gamma_C S0 + K^T Diag(beta_r Gamma_C / Gamma_r) U
// This is the chunkwise WY / UT form that "Gated DeltaNet-2" (technical core)
// and "Kaczmarz Linear Attention" (implementation) describe: the decay enters
// only through the asymmetric factors Gamma_t/Gamma_r of the erase terms, and
// KLA differs from Gated DeltaNet only in the diagonal Diag(beta).  Here KLA's
// ||k_t||^2 is the diagonal of K K^T, which the kernel computes anyway.
//
// One CTA owns one (batch, head, 64-column slice of v) and sweeps the chunks
// in order; the fp32 state slice (128 x 64) stays in registers (thread i holds
// row i) for the whole sequence.  Per chunk:
//   MMA1  [K;Q] K^T            (M128 N64 K128)  -> G = K K^T, H = Q K^T
//   SIMT  A, P (decay, beta, scale), KLA beta, T = (I + A)^{-1}
//   MMA2  W = T Diag(Gamma) K  (M64 N128 K64),   U' = T V (M64 N64 K64)
//   MMA3  E = U' - W S0        (M64 N64 K128, negated A, accumulating on U')
//         Y = Q S0             (M64 N64 K128)
//   MMA4  dS = K^T Diag(w) E   (M128 N64 K64),   Z = P E (M64 N64 K64)
//   SIMT  S = Gamma_C S + dS;  o_t = scale Gamma_t y_t + z_t
// Operands are bf16 in shared memory (128-byte swizzled tiles; q, k, v arrive
// by TMA, the rest is written by the threads), accumulators fp32 in TMEM.
// The operands that carry the state and the residuals -- S0, E, Diag(w) E and
// P -- are split into two bf16 terms x = hi + lo (hi = bf16(x), lo =
// bf16(x - hi)), and each product takes the hi*hi, hi*lo and lo*hi terms, so
// those products keep ~16 bits of precision; a single bf16 rounding there
// (2^-9 relative) would leave errors of a few percent of the output RMS on
// heavy-tailed outputs.  T, W and the raw q, k, v tiles stay single bf16.
// No cluster, no multicast.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdio>
#include <mutex>

#include "chunk_tc.cuh"
#include "tc_util.cuh"

// Device-side error word: set (never cleared by a kernel) when a bounded wait
// gives up; read and cleared by gdr_device_status().
__device__ int g_gdr_device_error = 0;

namespace gdr {
namespace tc {
namespace {

constexpr int C = 64;         // chunk length
constexpr int DK = 128;       // key dim handled by this kernel
constexpr int BV = 64;        // value columns per CTA
constexpr int NTHREADS = 128;
constexpr float LOG2E = 1.4426950408889634f;

// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t OFF_KQ = 0;          // 2 stages x [Kb0 | Qb0 | Kb1 | Qb1], 8 KB each
constexpr uint32_t KQ_STAGE = 32768;
constexpr uint32_t OFF_V = 65536;       // 2 stages x 8 KB
constexpr uint32_t V_STAGE = 8192;
constexpr uint32_t OFF_W = 81920;       // W: [b0 | b1]
constexpr uint32_t OFF_TP = 98304;      // T Diag(Gamma)
constexpr uint32_t OFF_TT = 106496;     // T
constexpr uint32_t OFF_P = 114688;      // P hi
constexpr uint32_t OFF_PL = 122880;     // P lo
constexpr uint32_t OFF_E = 131072;      // E hi   [r][v]
constexpr uint32_t OFF_EL = 139264;     // E lo
constexpr uint32_t OFF_EW = 147456;     // Diag(w) E hi
constexpr uint32_t OFF_EWL = 155648;    // Diag(w) E lo
constexpr uint32_t OFF_S = 163840;      // S0 hi [i][v], 128 rows
constexpr uint32_t OFF_SL = 180224;     // S0 lo
constexpr uint32_t OFF_A = 196608;      // A^T fp32, 64 x 68
constexpr uint32_t A_LD = 68;
constexpr uint32_t OFF_SC = OFF_A + 64 * A_LD * 4;   // scalars: 5 x 64 floats
constexpr uint32_t OFF_BAR = OFF_SC + 5 * 64 * 4;    // 3 mbarriers + TMEM slot
constexpr uint32_t SMEM_USED = OFF_BAR + 64;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;    // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// TMEM columns (fp32 accumulators)
constexpr uint32_t COL_G = 0;     // M128 x 64: G (lanes 0-63), H (lanes 64-127)
constexpr uint32_t COL_W = 64;    // M64 x 128
constexpr uint32_t COL_E = 192;   // M64 x 64: U', then E
constexpr uint32_t COL_Y = 256;   // M64 x 64: Q S0
constexpr uint32_t COL_S = 320;   // M128 x 64: dS
constexpr uint32_t COL_Z = 384;   // M64 x 64: P E
constexpr uint32_t TMEM_COLS = 512;

constexpr uint32_t ID_M128_N64_KK = idesc_bf16(128, 64, false, false);
constexpr uint32_t ID_M64_N128_KMN = idesc_bf16(64, 128, false, true);
constexpr uint32_t ID_M64_N64_KMN = idesc_bf16(64, 64, false, true);
constexpr uint32_t ID_M64_N64_KMN_NEG = idesc_bf16(64, 64, false, true, true);
constexpr uint32_t ID_M128_N64_MNMN = idesc_bf16(128, 64, true, true);

struct Params {
  int T, H, dv;
  const float *beta, *log_g, *s0;
  float *s_final;
  __nv_bfloat16 *o;
  float eps, scale;
};

// Store a row of 64 floats as two bf16 rows: hi = bf16(x), lo = bf16(x - hi).
__device__ __forceinline__ void st_row64_split(uint8_t *hi_tile, uint8_t *lo_tile, uint32_t r, const float *x) {
  float lo[64];
#pragma unroll
  for (int j = 0; j < 64; ++j) lo[j] = x[j] - __bfloat162float(__float2bfloat16_rn(x[j]));
  st_row64(hi_tile, r, x);
  st_row64(lo_tile, r, lo);
}

template <int VAR>
__global__ void __launch_bounds__(NTHREADS, 1)
    chunk_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int v0 = blockIdx.x * BV, h = blockIdx.y, b = blockIdx.z;
  const int NC = (p.T + C - 1) / C;

  uint64_t *bar_full = reinterpret_cast<uint64_t *>(sm + OFF_BAR);  // [2]
  uint64_t *bar_mma = bar_full + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_full + 3);
  float *sc_beta = reinterpret_cast<float *>(sm + OFF_SC);   // beta_t (KLA: Kaczmarz step)
  float *sc_g2 = sc_beta + 64;                               // gamma_t * log2(e)
  float *sc_wf = sc_g2 + 64;                                 // beta_r Gamma_C / Gamma_r
  float *sc_G = sc_wf + 64;                                  // Gamma_t
  float *sc_tmp = sc_G + 64;
  float *At = reinterpret_cast<float *>(sm + OFF_A);        // At[r][t] = A[t][r]

  if (warp == 0) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar_full[0], 1);
    mbar_init(&bar_full[1], 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }

  // state row i = tid, columns v0 .. v0+63, fp32 in registers
  float S[64];
  {
    const float *src = p.s0 ? p.s0 + ((static_cast<size_t>(b) * p.H + h) * DK + tid) * p.dv + v0 : nullptr;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      float4 f = src ? __ldg(reinterpret_cast<const float4 *>(src) + j) : make_float4(0.f, 0.f, 0.f, 0.f);
      S[4 * j] = f.x; S[4 * j + 1] = f.y; S[4 * j + 2] = f.z; S[4 * j + 3] = f.w;
    }
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;

  auto issue_chunk = [&](int c, int s) {
    uint8_t *kq = sm + OFF_KQ + s * KQ_STAGE;
    mbar_expect_tx(&bar_full[s], 5 * 8192);
    tma_load_4d(kq + 0, &tm_k, &bar_full[s], 0, h, c * C, b);
    tma_load_4d(kq + 8192, &tm_q, &bar_full[s], 0, h, c * C, b);
    tma_load_4d(kq + 16384, &tm_k, &bar_full[s], 64, h, c * C, b);
    tma_load_4d(kq + 24576, &tm_q, &bar_full[s], 64, h, c * C, b);
    tma_load_4d(sm + OFF_V + s * V_STAGE, &tm_v, &bar_full[s], v0, h, c * C, b);
  };
  if (tid == 0) {
    issue_chunk(0, 0);
    if (NC > 1) issue_chunk(1, 1);
  }
  st_row64_split(sm + OFF_S, sm + OFF_SL, tid, S);
  fence_async_smem();
  __syncthreads();

  uint32_t mma_phase = 0;
  int bad = 0;
  const uint32_t s_tile = smem_u32(sm + OFF_S), sl_tile = smem_u32(sm + OFF_SL);

  for (int c = 0; c < NC; ++c) {
    const int s = c & 1;
    const int t0 = c * C;
    const uint32_t kq = smem_u32(sm + OFF_KQ + s * KQ_STAGE);
    const uint32_t vt = smem_u32(sm + OFF_V + s * V_STAGE);

    // ---- (a) gates: beta_t, cumulative log2 decay
    if (tid < 64) {
      const int t = t0 + tid;
      float lg = 0.f, bt = 0.f;
      if (t < p.T) {
        const size_t th = (static_cast<size_t>(b) * p.T + t) * p.H + h;
        if constexpr (scalar_decay(VAR)) lg = __ldg(p.log_g + th);
        bt = __ldg(p.beta + th);
      }
      float x = lg * LOG2E;  // inclusive scan within the warp
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      sc_tmp[tid] = x;
      sc_beta[tid] = bt;
    }
    __syncthreads();
    if (tid < 64) sc_g2[tid] = sc_tmp[tid] + (tid >= 32 ? sc_tmp[31] : 0.f);

    // ---- (b) chunk inputs landed?
    if (!mbar_wait(&bar_full[s], (c >> 1) & 1)) bad = 1;
    if (__syncthreads_or(bad)) break;

    // ---- (c) MMA1: [K;Q] K^T
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t a = kq + (kk >> 2) * 16384 + (kk & 3) * 32;
        mma_bf16(tmem + COL_G, sdesc(a, 16, 1024), sdesc(a, 16, 1024), ID_M128_N64_KK, kk > 0);
      }
      mma_commit(bar_mma);
    }
    if (!mbar_wait(bar_mma, mma_phase)) bad = 1;
    mma_phase ^= 1;
    tc_fence_after();

    // ---- (d) A (warps 0-1, rows t = tid), P (warps 2-3, rows t = tid - 64)
    {
      float g[64];
      tmem_ld64(tmem + lane_base + COL_G, g);
      const int row = tid & 63;
      if constexpr (VAR == kKLA) {
        if (warp < 2) {
          float kk = 0.f;
#pragma unroll
          for (int r = 0; r < 64; ++r) kk = (r == row) ? g[r] : kk;
          const float eta = sc_beta[row];
          sc_beta[row] = (eta == 0.f) ? 0.f : eta / (kk + p.eps);   // Kaczmarz step
        }
      }
      __syncthreads();
      if (tid < 64) {
        sc_wf[tid] = sc_beta[tid] * ex2(sc_g2[63] - sc_g2[tid]);
        sc_G[tid] = ex2(sc_g2[tid]);
      }
      const float g2t = sc_g2[row];
      if (warp < 2) {
#pragma unroll
        for (int r = 0; r < 64; ++r) {
          const float a = (r < row) ? g[r] * sc_beta[r] * ex2(g2t - sc_g2[r]) : 0.f;
          At[r * A_LD + row] = a;
        }
      } else {
#pragma unroll
        for (int r = 0; r < 64; ++r) g[r] = (r <= row) ? p.scale * g[r] * sc_beta[r] * ex2(g2t - sc_g2[r]) : 0.f;
        st_row64_split(sm + OFF_P, sm + OFF_PL, row, g);
      }
    }
    tc_fence_before();
    __syncthreads();

    // ---- (e) T = (I + A)^{-1} (warps 0-1, column n = tid)
    if (warp < 2) {
      const int n = tid;
      float x[64];
#pragma unroll
      for (int m = 0; m < 64; ++m) x[m] = (m == n) ? 1.f : 0.f;
      // right-looking substitution: x[m] -= A[m][l] x[l] for m > l
#pragma unroll
      for (int l = 0; l < 63; ++l) {
        const float xl = x[l];
        const float *col = At + l * A_LD;   // A[.][l]
#pragma unroll
        for (int m4 = (l + 1) & ~3; m4 < 64; m4 += 4) {
          const float4 a4 = *reinterpret_cast<const float4 *>(col + m4);
          if (m4 + 0 > l) x[m4 + 0] = fmaf(-a4.x, xl, x[m4 + 0]);
          if (m4 + 1 > l) x[m4 + 1] = fmaf(-a4.y, xl, x[m4 + 1]);
          if (m4 + 2 > l) x[m4 + 2] = fmaf(-a4.z, xl, x[m4 + 2]);
          if (m4 + 3 > l) x[m4 + 3] = fmaf(-a4.w, xl, x[m4 + 3]);
        }
      }
      const float Gn = sc_G[n];
      __nv_bfloat16 *tt = reinterpret_cast<__nv_bfloat16 *>(sm + OFF_TT);
      __nv_bfloat16 *tp = reinterpret_cast<__nv_bfloat16 *>(sm + OFF_TP);
#pragma unroll
      for (int m = 0; m < 64; ++m) {
        const uint32_t off = (sw128(m, n >> 3) >> 1) + (n & 7);
        tt[off] = __float2bfloat16_rn(x[m]);
        tp[off] = __float2bfloat16_rn(x[m] * Gn);
      }
    }
    fence_async_smem();
    __syncthreads();

    // ---- (f) MMA2: W = T Diag(Gamma) K, U' = T V
    if (tid == 0) {
      tc_fence_after();
      const uint32_t tp = smem_u32(sm + OFF_TP), tt = smem_u32(sm + OFF_TT);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem + COL_W, sdesc(tp + kk * 32, 16, 1024), sdesc(kq + kk * 2048, 16384, 1024),
                 ID_M64_N128_KMN, kk > 0);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem + COL_E, sdesc(tt + kk * 32, 16, 1024), sdesc(vt + kk * 2048, 8192, 1024),
                 ID_M64_N64_KMN, kk > 0);
      mma_commit(bar_mma);
    }
    if (!mbar_wait(bar_mma, mma_phase)) bad = 1;
    mma_phase ^= 1;
    tc_fence_after();

    // ---- (g) W (M64 layout: warp w, lanes 0-15 hold rows 16w + lane) -> bf16 tile
    {
      float w[64];
      tmem_ld64(tmem + lane_base + COL_W, w);
      if (lane < 16) st_row64(sm + OFF_W, warp * 16 + lane, w);
      tmem_ld64(tmem + lane_base + COL_W + 64, w);
      if (lane < 16) st_row64(sm + OFF_W + 8192, warp * 16 + lane, w);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- (h) MMA3: E = U' - W (S0hi + S0lo) ; Y = Q (S0hi + S0lo)
    if (tid == 0) {
      tc_fence_after();
      const uint32_t wt = smem_u32(sm + OFF_W), qt = kq + 8192;
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        const uint32_t st = part ? sl_tile : s_tile;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16(tmem + COL_E, sdesc(wt + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024),
                   sdesc(st + kk * 2048, 8192, 1024), ID_M64_N64_KMN_NEG, 1);
      }
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        const uint32_t st = part ? sl_tile : s_tile;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16(tmem + COL_Y, sdesc(qt + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                   sdesc(st + kk * 2048, 8192, 1024), ID_M64_N64_KMN, part + kk > 0);
      }
      mma_commit(bar_mma);
    }
    if (!mbar_wait(bar_mma, mma_phase)) bad = 1;
    mma_phase ^= 1;
    tc_fence_after();

    // ---- (i) E -> bf16 tiles E and Diag(w) E  (rows r = 16w + lane)
    {
      float e[64];
      tmem_ld64(tmem + lane_base + COL_E, e);
      if (lane < 16) {
        const int r = warp * 16 + lane;
        st_row64_split(sm + OFF_E, sm + OFF_EL, r, e);
        const float wr = sc_wf[r];
#pragma unroll
        for (int j = 0; j < 64; ++j) e[j] *= wr;
        st_row64_split(sm + OFF_EW, sm + OFF_EWL, r, e);
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- (j) MMA4: dS = K^T Diag(w) (Ehi + Elo) ; Z = Phi Ehi + Phi Elo + Plo Ehi
    if (tid == 0) {
      tc_fence_after();
      const uint32_t ew = smem_u32(sm + OFF_EW), ewl = smem_u32(sm + OFF_EWL);
      const uint32_t et = smem_u32(sm + OFF_E), etl = smem_u32(sm + OFF_EL);
      const uint32_t pt = smem_u32(sm + OFF_P), ptl = smem_u32(sm + OFF_PL);
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        const uint32_t bt = part ? ewl : ew;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + COL_S, sdesc(kq + kk * 2048, 16384, 1024), sdesc(bt + kk * 2048, 8192, 1024),
                   ID_M128_N64_MNMN, part + kk > 0);
      }
#pragma unroll
      for (int part = 0; part < 3; ++part) {
        const uint32_t at = part == 2 ? ptl : pt;
        const uint32_t bt = part == 1 ? etl : et;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + COL_Z, sdesc(at + kk * 32, 16, 1024), sdesc(bt + kk * 2048, 8192, 1024),
                   ID_M64_N64_KMN, part + kk > 0);
      }
      mma_commit(bar_mma);
    }
    if (!mbar_wait(bar_mma, mma_phase)) bad = 1;
    mma_phase ^= 1;
    tc_fence_after();

    // ---- (k) state update (row i = tid) and output rows (16w + lane)
    {
      float d[64];
      tmem_ld64(tmem + lane_base + COL_S, d);
      const float gc = ex2(sc_g2[63]);
#pragma unroll
      for (int j = 0; j < 64; ++j) S[j] = fmaf(gc, S[j], d[j]);
      st_row64_split(sm + OFF_S, sm + OFF_SL, tid, S);
      float y[64];
      tmem_ld64(tmem + lane_base + COL_Y, y);
      tmem_ld64(tmem + lane_base + COL_Z, d);
      const int tr = (warp * 16 + lane) & 63;
      const float fy = p.scale * sc_G[tr];
#pragma unroll
      for (int j = 0; j < 64; ++j) d[j] = fmaf(fy, y[j], d[j]);
      const int t = t0 + warp * 16 + lane;
      if (lane < 16 && t < p.T) {
        uint4 *dst = reinterpret_cast<uint4 *>(p.o + ((static_cast<size_t>(b) * p.T + t) * p.H + h) * p.dv + v0);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          uint4 u;
          u.x = pack_bf16x2(d[8 * j + 0], d[8 * j + 1]);
          u.y = pack_bf16x2(d[8 * j + 2], d[8 * j + 3]);
          u.z = pack_bf16x2(d[8 * j + 4], d[8 * j + 5]);
          u.w = pack_bf16x2(d[8 * j + 6], d[8 * j + 7]);
          dst[j] = u;
        }
      }
    }
    fence_async_smem();
    tc_fence_before();
    if (__syncthreads_or(bad)) break;

    // ---- (l) refill this stage with chunk c + 2
    if (tid == 0 && c + 2 < NC) issue_chunk(c + 2, s);
  }

  if (bad) {
    if (tid == 0) atomicExch(&g_gdr_device_error, 1);
  } else if (p.s_final) {
    float4 *dst = reinterpret_cast<float4 *>(p.s_final + ((static_cast<size_t>(b) * p.H + h) * DK + tid) * p.dv + v0);
#pragma unroll
    for (int j = 0; j < 16; ++j) dst[j] = make_float4(S[4 * j], S[4 * j + 1], S[4 * j + 2], S[4 * j + 3]);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// [B, T, H, D] bf16 tensor, box of 64 (D) x 1 (H) x 64 (T) x 1 (B), 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *base, int B, int T, int H, int D) {
  auto enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)T * H * D * 2};
  const cuuint32_t box[4] = {64, 1, 64, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int VAR>
cudaError_t launch_variant(const FwdProblem &p, cudaStream_t stream, std::string *err) {
  // per call: the attribute is per device, and callers may switch devices
  cudaError_t e = cudaFuncSetAttribute(chunk_fwd_kernel<VAR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)SMEM_BYTES);
  if (e != cudaSuccess) {
    *err = "cudaFuncSetAttribute: ";
    return e;
  }
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, p.q, p.B, p.T, p.H, p.dk) || !make_map(&mk, p.k, p.B, p.T, p.H, p.dk) ||
      !make_map(&mv, p.v, p.B, p.T, p.H, p.dv)) {
    *err = "cuTensorMapEncodeTiled failed: ";
    return cudaErrorInvalidValue;
  }
  Params kp;
  kp.T = p.T; kp.H = p.H; kp.dv = p.dv;
  kp.beta = p.beta; kp.log_g = p.log_g; kp.s0 = p.s0; kp.s_final = p.s_final;
  kp.o = static_cast<__nv_bfloat16 *>(p.o);
  kp.eps = p.eps; kp.scale = p.scale;
  const dim3 grid(p.dv / BV, p.H, p.B), block(NTHREADS);
  chunk_fwd_kernel<VAR><<<grid, block, SMEM_BYTES, stream>>>(mq, mk, mv, kp);
  e = cudaGetLastError();
  if (e != cudaSuccess) *err = "launch: ";
  return e;
}

}  // namespace
}  // namespace tc
}  // namespace gdr

bool gdr_chunk_tc_supported(int variant, int dk, int dv) {
  using namespace gdr;
  const bool v = variant == kDeltaNet || variant == kGatedDeltaNet || variant == kKLA;
  return v && dk == 128 && (dv == 64 || dv == 128);
}

int gdr_chunk_tc_launches(int, int, int, int, int) { return 1; }

cudaError_t gdr_launch_chunk_tc(const gdr::FwdProblem &p, cudaStream_t stream, std::string *err) {
  using namespace gdr;
  switch (p.variant) {
    case kDeltaNet: return tc::launch_variant<kDeltaNet>(p, stream, err);
    case kGatedDeltaNet: return tc::launch_variant<kGatedDeltaNet>(p, stream, err);
    case kKLA: return tc::launch_variant<kKLA>(p, stream, err);
    default: *err = "variant not covered: "; return cudaErrorInvalidValue;
  }
}

int gdr_read_device_error(cudaStream_t stream) {
  int h = 0, zero = 0;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return -1;
  if (cudaMemcpyFromSymbol(&h, g_gdr_device_error, sizeof(int)) != cudaSuccess) return -1;
  if (h) cudaMemcpyToSymbol(g_gdr_device_error, &zero, sizeof(int));
  return h;
}
