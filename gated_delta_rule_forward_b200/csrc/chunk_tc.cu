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
//     O = Diag(scale Gamma) Q S0 + P U,     P_tr = scale beta_r (Gamma_t/Gamma_r) q_t.k_r (r <= t)
//     S_C = Gamma_C S0 + K^T Diag(beta_r Gamma_C / Gamma_r) U
// This is the chunkwise WY / UT form that "Gated DeltaNet-2" (technical core)
// and "Kaczmarz Linear Attention" (implementation) describe: the decay enters
// only through the asymmetric factors Gamma_t/Gamma_r of the erase terms, and
// KLA differs from Gated DeltaNet only in the diagonal Diag(beta).  KLA's
// ||k_t||^2 is the diagonal of K K^T, which the kernel computes anyway.
//
// One CTA of 8 warps owns one (batch, head, 64-column slice of v) and sweeps
// the chunks in order.  The fp32 state slice (128 x 64) lives in registers:
// warp w holds rows 32 (w % 4) + lane, columns 32 (w / 4) .. +31.  Per chunk:
//   MMA1  [K;Q] K^T (bf16)              M128 N64  K128 -> G = K K^T | H = Q K^T
//   SIMT  A, P (decay, beta, scale; KLA beta from diag G); fp16 copies of K
//         and Diag(scale Gamma) Q; T = (I + A)^{-1} by a 16x16-blocked solve
//   MMA2  W = T Diag(Gamma) K (bf16)     M64  N128 K64
//         [0; T] V (bf16)                M128 N64  K64  -> lanes 64-127: U'
//   MMA3  + [Diag(scale Gamma) Q; -W] S0 (fp16)  M128 N64 K128
//         -> lanes 0-63: Diag(scale Gamma) Q S0, lanes 64-127: E = U' - W S0
//   MMA4  dS = K^T Diag(w) E (fp16)      M128 N64  K64
//         + [P; *] E (fp16)              M128 N64  K64  -> lanes 0-63: O
//   SIMT  S = Gamma_C S + dS; o rows
// q, k, v arrive by 4-d TMA (128-byte swizzle, two stages, no multicast); all
// other operands are written by the threads into swizzled tiles.  The
// operands that carry the state and the residuals (S0, E, Diag(w) E, P, W and
// the q/k copies they meet) are fp16: its 11-bit significand keeps those
// products near 2^-12 relative error, where bf16 (8 bits) left a few percent
// of the output RMS on heavy-tailed outputs.  fp16's range limits |S|, |E| to
// 6.5e4; a kernel that sees larger values raises the range flag that
// gdr_device_status() reports.  T, its Gamma-scaled copy and raw q, k, v stay
// bf16.
#include "chunk_tc.cuh"
#include "chunk_common.cuh"
#include "tma_host.cuh"
#include "tc_util.cuh"

// Device-side error word, read and cleared by gdr_device_status():
// bit 0 = a bounded wait gave up, bit 1 = an fp16 operand left its range.
__device__ int g_gdr_device_error = 0;

namespace gdr {
namespace tc {
namespace {

constexpr int C = 64;         // chunk length
constexpr int DK = 128;       // key dim handled by this kernel
constexpr int BV = 64;        // value columns per CTA
constexpr int NTHREADS = 256;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float F16_SAFE = 60000.f;

// shared memory map (bytes from a 1024-aligned base); 8 KB tiles are 64 rows x 128 B
constexpr uint32_t OFF_KQ = 0;          // 2 stages x [Kb0 | Qb0 | Kb1 | Qb1] bf16 (TMA)
constexpr uint32_t KQ_STAGE = 32768;
constexpr uint32_t OFF_V = 65536;       // 2 stages x V bf16 (TMA)
constexpr uint32_t V_STAGE = 8192;
constexpr uint32_t OFF_QW = 81920;      // fp16 [Qg b0 | -W b0 | Qg b1 | -W b1]
constexpr uint32_t OFF_K16 = 114688;    // fp16 [K b0 | K b1]
constexpr uint32_t OFF_ZT = 131072;     // bf16 [zero | T]
constexpr uint32_t OFF_TP = 147456;     // bf16 T Diag(Gamma)
constexpr uint32_t OFF_P = 155648;      // fp16 P (rows 0-63 of an M128 operand; E16 follows)
constexpr uint32_t OFF_E = 163840;      // fp16 E  [r][v]
constexpr uint32_t OFF_EW = 172032;     // fp16 Diag(w) E
constexpr uint32_t OFF_TF = OFF_QW;     // fp32 T during the solve, 64 x 72 (aliases Qg / -W)
constexpr uint32_t OFF_S = 180224;      // fp16 S0 [i][v], 128 rows
constexpr uint32_t OFF_A = 196608;      // fp32 A^T [r][t], 64 x 72
constexpr uint32_t OFF_SC = OFF_A + 64 * LD * 4;   // scalars: 5 x 64 floats
constexpr uint32_t OFF_BAR = OFF_SC + 5 * 64 * 4;    // 3 mbarriers + TMEM slot
constexpr uint32_t SMEM_USED = OFF_BAR + 64;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;    // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// TMEM columns (fp32 accumulators)
constexpr uint32_t COL_G = 0;     // M128 x 64: G (lanes 0-63), H (lanes 64-127)
constexpr uint32_t COL_W = 64;    // M64 x 128
constexpr uint32_t COL_YE = 192;  // M128 x 64: lanes 0-63 Q S0 (+ P E), lanes 64-127 U' then E
constexpr uint32_t COL_S = 256;   // M128 x 64: dS
constexpr uint32_t TMEM_COLS = 512;

constexpr uint32_t ID_G = idesc_bf16(128, 64, false, false);        // [K;Q] K^T
constexpr uint32_t ID_W = idesc_bf16(64, 128, false, true);         // T' K
constexpr uint32_t ID_U = idesc_bf16(128, 64, false, true);         // [0;T] V
constexpr uint32_t ID_YE = idesc_f16(128, 64, false, true);         // [Qg;-W] S0
constexpr uint32_t ID_DS = idesc_f16(128, 64, true, true);          // K^T Ew
constexpr uint32_t ID_PE = idesc_f16(128, 64, false, true);         // [P;*] E

struct Params {
  int T, H, dv;
  const float *beta, *log_g, *s0;
  float *s_final;
  __nv_bfloat16 *o;
  float eps, scale;
};


template <int VAR>
__global__ void __launch_bounds__(NTHREADS, 1)
    chunk_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quad = warp & 3, half = warp >> 2;            // TMEM lane quadrant, column half
  const int row = quad * 32 + lane;                       // this thread's TMEM lane (M128 layout)
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
  float *At = reinterpret_cast<float *>(sm + OFF_A);        // At[r * LD + t] = A[t][r]
  float *Tf = reinterpret_cast<float *>(sm + OFF_TF);

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
  // zero tile (rows 0-63 of the [0; T] operand)
  for (int i = tid; i < 512; i += NTHREADS)
    reinterpret_cast<uint4 *>(sm + OFF_ZT)[i] = make_uint4(0u, 0u, 0u, 0u);

  // state: row `row`, columns v0 + 32 half .. +31
  float S[32];
  {
    const float *src =
        p.s0 ? p.s0 + ((static_cast<size_t>(b) * p.H + h) * DK + row) * p.dv + v0 + 32 * half : nullptr;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float4 f = src ? __ldg(reinterpret_cast<const float4 *>(src) + j) : make_float4(0.f, 0.f, 0.f, 0.f);
      S[4 * j] = f.x; S[4 * j + 1] = f.y; S[4 * j + 2] = f.z; S[4 * j + 3] = f.w;
    }
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;

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
  // fp16 S0 tile, this thread's 32 columns = four 16-byte chunks of row `row`
#pragma unroll
  for (int j = 0; j < 4; ++j) st_chunk_f16(sm + OFF_S + sw128(row, 4 * half + j), S + 8 * j);

  // gates of chunk 0 (prefetched one chunk ahead from here on)
  float pf_lg = 0.f, pf_bt = 0.f;
  auto load_gates = [&](int c) {
    pf_lg = 0.f;
    pf_bt = 0.f;
    const int t = c * C + tid;
    if (tid < 64 && t < p.T) {
      const size_t th = (static_cast<size_t>(b) * p.T + t) * p.H + h;
      if constexpr (scalar_decay(VAR)) pf_lg = __ldg(p.log_g + th);
      pf_bt = __ldg(p.beta + th);
    }
  };
  load_gates(0);
  fence_async_smem();
  __syncthreads();

  uint32_t mma_phase = 0;
  int bad = 0;
  float smax = 0.f;                                    // largest |fp16 operand| seen (range check)
  const uint32_t s_tile = smem_u32(sm + OFF_S);

  for (int c = 0; c < NC; ++c) {
    const int s = c & 1;
    const int t0 = c * C;
    const uint32_t kq = smem_u32(sm + OFF_KQ + s * KQ_STAGE);
    const uint32_t vt = smem_u32(sm + OFF_V + s * V_STAGE);
    uint8_t *kq_ptr = sm + OFF_KQ + s * KQ_STAGE;

    // ---- (a) gates: beta_t, cumulative log2 decay; prefetch the next chunk's
    if (tid < 64) {
      float x = pf_lg * LOG2E;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      sc_tmp[tid] = x;
      sc_beta[tid] = pf_bt;
    }
    if (c + 1 < NC) load_gates(c + 1);
    __syncthreads();
    if (tid < 64) {
      const float g2 = sc_tmp[tid] + (tid >= 32 ? sc_tmp[31] : 0.f);
      sc_g2[tid] = g2;
      sc_G[tid] = ex2(g2);
    }

    // ---- (b) chunk inputs landed?
    if (!mbar_wait(&bar_full[s], (c >> 1) & 1)) bad = 1;
    if (__syncthreads_or(bad)) break;

    // ---- (c) MMA1: [K;Q] K^T; meanwhile the fp16 copy of K
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t a = kq + (kk >> 2) * 16384 + (kk & 3) * 32;
        mma_ss(tmem + COL_G, sdesc(a, 16, 1024), sdesc(a, 16, 1024), ID_G, kk > 0);
      }
      mma_commit(bar_mma);
    }
    {
      // fp16 copy of K: 2 atoms x 64 rows x 8 chunks = 1024 chunks; 4 per thread
#pragma unroll
      for (int it = 0; it < 4; ++it) {
        const int idx = it * NTHREADS + tid;
        const int kb = idx >> 9, r = (idx >> 3) & 63, j = idx & 7;
        const uint32_t off = sw128(r, j);
        float x[8];
        unpack8(*reinterpret_cast<const uint4 *>(kq_ptr + kb * 16384 + off), x);
        st_chunk_f16(sm + OFF_K16 + kb * 8192 + off, x);
      }
    }
    if (!mbar_wait(bar_mma, mma_phase)) bad = 1;
    mma_phase ^= 1;
    tc_fence_after();

    // ---- (d) A (lanes 0-63) and P (lanes 64-127); this thread: 32 columns
    {
      float g[32];
      tmem_ld32(tmem + lane_base + COL_G + 32 * half, g);
      const int t = row & 63;
      const int r0 = 32 * half;
      if constexpr (VAR == kKLA) {
        if (quad < 2 && (t >> 5) == half) {
          float kk = 0.f;
#pragma unroll
          for (int r = 0; r < 32; ++r) kk = (r0 + r == t) ? g[r] : kk;
          const float eta = sc_beta[t];
          sc_beta[t] = (eta == 0.f) ? 0.f : eta / (kk + p.eps);   // Kaczmarz step
        }
      }
      __syncthreads();
      // decay factors 2^(g2_t - g2_r) = rowf_t * colf_r with the reference at the
      // first column of each 32-column half (rowf <= 1 where used, colf >= 1);
      // exact per element when the chunk's decay span could overflow the split
      const bool fast = sc_g2[0] - sc_g2[63] < 120.f;
      if (tid < 64) {
        sc_wf[tid] = sc_beta[tid] * ex2(sc_g2[63] - sc_g2[tid]);
        sc_tmp[tid] = sc_beta[tid] * ex2(sc_g2[tid & 32] - sc_g2[tid]);
      }
      __syncthreads();
      const float g2t = sc_g2[t];
      const float rowf = (t >= r0) ? ex2(g2t - sc_g2[r0]) : 0.f;
      float fac[32];
      if (fast) {
#pragma unroll
        for (int r4 = 0; r4 < 32; r4 += 4) {
          const float4 cb = *reinterpret_cast<const float4 *>(sc_tmp + r0 + r4);
          fac[r4 + 0] = cb.x * rowf; fac[r4 + 1] = cb.y * rowf;
          fac[r4 + 2] = cb.z * rowf; fac[r4 + 3] = cb.w * rowf;
        }
      } else {
#pragma unroll
        for (int r = 0; r < 32; ++r) fac[r] = sc_beta[r0 + r] * ex2(g2t - sc_g2[r0 + r]);
      }
      if (quad < 2) {
#pragma unroll
        for (int r = 0; r < 32; ++r) At[(r0 + r) * LD + t] = (r0 + r < t) ? tf32r(g[r] * fac[r]) : 0.f;
      } else {
#pragma unroll
        for (int r = 0; r < 32; ++r) g[r] = (r0 + r <= t) ? p.scale * g[r] * fac[r] : 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) st_chunk_f16(sm + OFF_P + sw128(t, 4 * half + j), g + 8 * j);
      }
    }
    tc_fence_before();
    __syncthreads();

    // ---- (e) T = (I + A)^{-1}
    solve_unit_lower_64(At, Tf, tid, warp, lane);
    // T and T Diag(Gamma) as bf16 tiles (rows m, 16 columns per thread); upper part zero
    {
      const int m = tid >> 2, n0 = (tid & 3) * 16;
      float tv[16], tg[16];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const float4 f = *reinterpret_cast<const float4 *>(Tf + m * LD + n0 + 4 * q4);
        tv[4 * q4 + 0] = f.x; tv[4 * q4 + 1] = f.y; tv[4 * q4 + 2] = f.z; tv[4 * q4 + 3] = f.w;
      }
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int n = n0 + e;
        tv[e] = (n <= m) ? tv[e] : 0.f;
        tg[e] = tv[e] * sc_G[n];
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        st_chunk_bf16(sm + OFF_ZT + 8192 + sw128(m, 2 * (tid & 3) + j), tv + 8 * j);
        st_chunk_bf16(sm + OFF_TP + sw128(m, 2 * (tid & 3) + j), tg + 8 * j);
      }
    }
    fence_async_smem();
    __syncthreads();

    // ---- (f) MMA2: W = T Diag(Gamma) K ; lanes 64-127 of YE = T V (lanes 0-63 = 0)
    if (tid == 0) {
      tc_fence_after();
      const uint32_t tp = smem_u32(sm + OFF_TP), zt = smem_u32(sm + OFF_ZT);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ss(tmem + COL_W, sdesc(tp + kk * 32, 16, 1024), sdesc(kq + kk * 2048, 16384, 1024), ID_W, kk > 0);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ss(tmem + COL_YE, sdesc(zt + kk * 32, 16, 1024), sdesc(vt + kk * 2048, 8192, 1024), ID_U, kk > 0);
      mma_commit(bar_mma);
    }
    if (!mbar_wait(bar_mma, mma_phase)) bad = 1;
    mma_phase ^= 1;
    tc_fence_after();

    // ---- (g) -W (M64 layout: rows 16 quad + lane for lane < 16) -> fp16, columns 64 half ..;
    // and the fp16 copy of Diag(scale Gamma) Q (the T scratch that shared this tile is dead)
    {
#pragma unroll
      for (int it = 0; it < 4; ++it) {
        const int idx = it * NTHREADS + tid;
        const int kb = idx >> 9, r = (idx >> 3) & 63, j = idx & 7;
        const uint32_t off = sw128(r, j);
        float x[8];
        unpack8(*reinterpret_cast<const uint4 *>(kq_ptr + kb * 16384 + 8192 + off), x);
        const float f = p.scale * sc_G[r];
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] *= f;
        st_chunk_f16(sm + OFF_QW + kb * 16384 + off, x);
      }
    }
    {
      float w[32];
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        tmem_ld32(tmem + lane_base + COL_W + 64 * half + 32 * part, w);
        if (lane < 16) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            smax = fmaxf(smax, fabsf(w[e]));
            w[e] = -w[e];
          }
#pragma unroll
          for (int j = 0; j < 4; ++j)
            st_chunk_f16(sm + OFF_QW + half * 16384 + 8192 + sw128(quad * 16 + lane, 4 * part + j), w + 8 * j);
        }
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- (h) MMA3: YE += [Diag(scale Gamma) Q; -W] S0
    if (tid == 0) {
      tc_fence_after();
      const uint32_t qw = smem_u32(sm + OFF_QW);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ss(tmem + COL_YE, sdesc(qw + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                 sdesc(s_tile + kk * 2048, 8192, 1024), ID_YE, 1);
      mma_commit(bar_mma);
    }
    if (!mbar_wait(bar_mma, mma_phase)) bad = 1;
    mma_phase ^= 1;
    tc_fence_after();

    // ---- (i) E (lanes 64-127) -> fp16 tiles E and Diag(w) E
    if (quad >= 2) {
      float e[32];
      tmem_ld32(tmem + lane_base + COL_YE + 32 * half, e);
      const int r = row - 64;
#pragma unroll
      for (int j = 0; j < 32; ++j) smax = fmaxf(smax, fabsf(e[j]));
#pragma unroll
      for (int j = 0; j < 4; ++j) st_chunk_f16(sm + OFF_E + sw128(r, 4 * half + j), e + 8 * j);
      const float wr = sc_wf[r];
#pragma unroll
      for (int j = 0; j < 32; ++j) e[j] *= wr;
#pragma unroll
      for (int j = 0; j < 4; ++j) st_chunk_f16(sm + OFF_EW + sw128(r, 4 * half + j), e + 8 * j);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- (j) MMA4: dS = K^T Diag(w) E ; YE += [P; *] E
    if (tid == 0) {
      tc_fence_after();
      const uint32_t k16 = smem_u32(sm + OFF_K16), ew = smem_u32(sm + OFF_EW);
      const uint32_t et = smem_u32(sm + OFF_E), pt = smem_u32(sm + OFF_P);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ss(tmem + COL_S, sdesc(k16 + kk * 2048, 8192, 1024), sdesc(ew + kk * 2048, 8192, 1024), ID_DS,
                 kk > 0);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ss(tmem + COL_YE, sdesc(pt + kk * 32, 16, 1024), sdesc(et + kk * 2048, 8192, 1024), ID_PE, 1);
      mma_commit(bar_mma);
    }
    if (!mbar_wait(bar_mma, mma_phase)) bad = 1;
    mma_phase ^= 1;
    tc_fence_after();

    // ---- (k) state update (all lanes) and output rows (lanes 0-63)
    {
      float d[32];
      tmem_ld32(tmem + lane_base + COL_S + 32 * half, d);
      const float gc = ex2(sc_g2[63]);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        S[j] = fmaf(gc, S[j], d[j]);
        smax = fmaxf(smax, fabsf(S[j]));
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) st_chunk_f16(sm + OFF_S + sw128(row, 4 * half + j), S + 8 * j);
      if (quad < 2) {
        tmem_ld32(tmem + lane_base + COL_YE + 32 * half, d);
        const int t = t0 + row;
        if (t < p.T) {
          uint8_t *dst = reinterpret_cast<uint8_t *>(
              p.o + ((static_cast<size_t>(b) * p.T + t) * p.H + h) * p.dv + v0 + 32 * half);
#pragma unroll
          for (int j = 0; j < 4; ++j) st_chunk_bf16(dst + 16 * j, d + 8 * j);
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
    if (tid == 0) atomicOr(&g_gdr_device_error, 1);
  } else {
    if (smax > F16_SAFE) atomicOr(&g_gdr_device_error, 2);
    if (p.s_final) {
      float4 *dst = reinterpret_cast<float4 *>(
          p.s_final + ((static_cast<size_t>(b) * p.H + h) * DK + row) * p.dv + v0 + 32 * half);
#pragma unroll
      for (int j = 0; j < 8; ++j) dst[j] = make_float4(S[4 * j], S[4 * j + 1], S[4 * j + 2], S[4 * j + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
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
  const bool v = variant == kDeltaNet || variant == kGatedDeltaNet || variant == kKLA || variant == kKDA;
  return v && dk == 128 && (dv == 64 || dv == 128);
}

int gdr_chunk_tc_launches(int, int, int, int, int) { return 1; }

cudaError_t gdr_launch_chunk_tc(const gdr::FwdProblem &p, cudaStream_t stream, std::string *err) {
  using namespace gdr;
  switch (p.variant) {
    case kDeltaNet: return tc::launch_variant<kDeltaNet>(p, stream, err);
    case kGatedDeltaNet: return tc::launch_variant<kGatedDeltaNet>(p, stream, err);
    case kKLA: return tc::launch_variant<kKLA>(p, stream, err);
    case kKDA: return gdr_launch_chunk_chan(p, stream, err);
    default: *err = "variant not covered: "; return cudaErrorInvalidValue;
  }
}

int gdr_read_device_error(cudaStream_t stream) {
  int h = 0, zero = 0;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return -1;
  if (cudaMemcpyFromSymbol(&h, g_gdr_device_error, sizeof(int)) != cudaSuccess) return -1;
  if (h) cudaMemcpyToSymbol(g_gdr_device_error, &zero, sizeof(int));
  const int hc = gdr_read_chan_error();
  const int hs = gdr_read_split_error();
  if (hc < 0 || hs < 0) return -1;
  return h | hc | hs;
}
