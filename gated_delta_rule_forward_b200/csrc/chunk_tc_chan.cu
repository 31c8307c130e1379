// Chunked forward for channel-wise decay (KDA) on sm_100a tensor cores.
//
// KDA ("Gated DeltaNet-2", what is new / technical core: the decay of Kimi
// Delta Attention is a vector g_t in R^{dk} acting on the rows of the state)
// with a_t = c_t = beta_t k_t.  Within a chunk, gamma_t[i] = sum_{r<=t} log g_r[i]
// per channel, and the chunk form of the scalar-decay kernel holds with the
// decay moved inside the products ("decay absorbed into asymmetric erase
// factors", technical core):
//     A_tr = beta_r sum_i k_t[i] k_r[i] e^{gamma_t[i] - gamma_r[i]}     (r < t)
//     P_tr = beta_r sum_i scale q_t[i] k_r[i] e^{gamma_t[i] - gamma_r[i]} (r <= t)
//     T = (I + A)^{-1};  W = T (K o e^{gamma});  U' = T V;  E = U' - W S0
//     O = (scale Q o e^{gamma}) S0 + P E
//     S_C = Diag(e^{gamma_C}) S0 + Kt^T E,  Kt[r][i] = beta_r k_r[i] e^{gamma_C[i] - gamma_r[i]}
// The e^{gamma_t - gamma_r} factor is split around the chunk's middle token m:
// [K o e^{gamma - gamma_m}; scale Q o e^{gamma - gamma_m}] (K o e^{gamma_m - gamma})^T.
// Its factors span up to e^{|gamma_0 - gamma_63|}, beyond fp16's range, and one
// bf16 rounding there alone leaves ~2.5% of the output RMS, so these two
// operands are tf32: fp32 range with an 11-bit significand like fp16's.
// MMA1 runs in two 64-channel halves so the fp32 operands fit in shared
// memory.  The channel log-decay tile (64 x 128 fp32) arrives by TMA
// one chunk ahead and is scanned in place.  Everything after T follows the
// scalar-decay kernel (fp16 carry operands, stacked [Qg; -W] S0, P E
// accumulated onto the output rows); see chunk_tc.cu for the shared
// derivation and precision argument.
#include "chunk_common.cuh"
#include "chunk_tc.cuh"
#include "tc_util.cuh"
#include "tma_host.cuh"

// Device-side error word of this file (see gdr_device_status()):
// bit 0 = a bounded wait gave up, bit 1 = an operand left its range.
__device__ int g_gdr_chan_error = 0;

namespace gdr {
namespace tc {
namespace {

constexpr int C = 64;
constexpr int DK = 128;
constexpr int BV = 64;
constexpr int NTHREADS = 256;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float F16_SAFE = 60000.f;
constexpr float SPAN_SAFE = 120.f;     // |gamma_t - gamma_m| (log2 units) the fp32 factors can carry

// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t OFF_KQ = 0;          // 2 stages x [Kb0 | Qb0 | Kb1 | Qb1] bf16 (TMA)
constexpr uint32_t KQ_STAGE = 32768;
constexpr uint32_t OFF_V = 65536;       // 2 stages x V bf16 (TMA)
constexpr uint32_t V_STAGE = 8192;
constexpr uint32_t OFF_LG = 81920;      // fp32 [64][128]: log g (TMA), then e^{gamma - gamma_m}
constexpr uint32_t OFF_S = 114688;      // fp16 S0 [i][v], 128 rows
constexpr uint32_t OFF_KT = 131072;     // fp16 Kt [Kb0 | Kb1]
constexpr uint32_t OFF_ZT = 147456;     // bf16 [zero | T]
constexpr uint32_t OFF_R = 163840;      // phase-shared region (60 KB), see below
constexpr uint32_t OFF_P = OFF_R;                    // fp16 P (d .. j); rows 64-127 of [P; *] follow
constexpr uint32_t OFF_XF = OFF_R + 8192;            // (c) tf32 [K o G; Q o G], 128 rows x 2 atoms of 32 ch
constexpr uint32_t OFF_YF = OFF_R + 40960;           // (c) tf32 K o G^-1, 64 rows x 2 atoms of 32 ch
constexpr uint32_t OFF_A = OFF_R + 8192;             // (d, e) fp32 A^T, 64 x LD
constexpr uint32_t OFF_TF = OFF_R + 26624;           // (e) fp32 T, 64 x LD
constexpr uint32_t OFF_KG = OFF_R + 45056;           // (e, f) bf16 K o e^{gamma} [Kb0 | Kb1]
constexpr uint32_t OFF_QW = OFF_R + 8192;            // (g, h) fp16 [Qg b0 | -W b0 | Qg b1 | -W b1]
constexpr uint32_t OFF_E = OFF_R + 40960;            // (i, j) fp16 E
constexpr uint32_t OFF_SC = OFF_R + 61440;           // scalars
constexpr uint32_t OFF_BAR = OFF_SC + 384 * 4;       // mbarriers + TMEM slot
constexpr uint32_t SMEM_USED = OFF_BAR + 64;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(OFF_KG % 1024 == 0 && OFF_E % 1024 == 0 && OFF_XF % 1024 == 0 && OFF_YF % 1024 == 0,
              "tile alignment");

constexpr uint32_t COL_G = 0;     // M128 x 64
constexpr uint32_t COL_W = 64;    // M64 x 128
constexpr uint32_t COL_YE = 192;  // M128 x 64
constexpr uint32_t COL_S = 256;   // M128 x 64
constexpr uint32_t TMEM_COLS = 512;

constexpr uint32_t ID_G = idesc_tf32(128, 64, false, false);
constexpr uint32_t ID_W = idesc_bf16(64, 128, false, true);
constexpr uint32_t ID_U = idesc_bf16(128, 64, false, true);
constexpr uint32_t ID_YE = idesc_f16(128, 64, false, true);
constexpr uint32_t ID_DS = idesc_f16(128, 64, true, true);
constexpr uint32_t ID_PE = idesc_f16(128, 64, false, true);

struct Params {
  int T, H, dv;
  const float *beta, *s0;
  float *s_final;
  __nv_bfloat16 *o;
  float scale;
};


template <int VAR>
__global__ void __launch_bounds__(NTHREADS, 1)
    chunk_chan_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                      const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quad = warp & 3, half = warp >> 2;
  const int row = quad * 32 + lane;
  const int v0 = blockIdx.x * BV, h = blockIdx.y, b = blockIdx.z;
  const int NC = (p.T + C - 1) / C;

  uint64_t *bar_full = reinterpret_cast<uint64_t *>(sm + OFF_BAR);  // [2]
  uint64_t *bar_mma = bar_full + 2;
  uint64_t *bar_lg = bar_full + 3;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_full + 4);
  float *sc_beta = reinterpret_cast<float *>(sm + OFF_SC);   // [64]
  float *sc_gm = sc_beta + 64;                               // [128] gamma_m * log2 e per channel
  float *sc_tmp = sc_gm + 128;                               // [128]
  float *sc_gc = sc_tmp + 128;                               // [64]   (unused slack)
  float *Gr = reinterpret_cast<float *>(sm + OFF_LG);        // [64][128]
  float *At = reinterpret_cast<float *>(sm + OFF_A);
  float *Tf = reinterpret_cast<float *>(sm + OFF_TF);
  (void)sc_gc;

  if (warp == 0) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar_full[0], 1);
    mbar_init(&bar_full[1], 1);
    mbar_init(bar_mma, 1);
    mbar_init(bar_lg, 1);
    fence_mbar_init();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_g);
  }
  for (int i = tid; i < 512; i += NTHREADS)
    reinterpret_cast<uint4 *>(sm + OFF_ZT)[i] = make_uint4(0u, 0u, 0u, 0u);

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
  auto issue_gates = [&](int c) {
    mbar_expect_tx(bar_lg, 64 * DK * 4);
    tma_load_4d(sm + OFF_LG, &tm_g, bar_lg, 0, h, c * C, b);
  };
  if (tid == 0) {
    issue_gates(0);
    issue_chunk(0, 0);
    if (NC > 1) issue_chunk(1, 1);
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) st_chunk_f16(sm + OFF_S + sw128(row, 4 * half + j), S + 8 * j);

  float pf_bt = 0.f;
  auto load_beta = [&](int c) {
    pf_bt = 0.f;
    const int t = c * C + tid;
    if (tid < 64 && t < p.T) pf_bt = __ldg(p.beta + (static_cast<size_t>(b) * p.T + t) * p.H + h);
  };
  load_beta(0);
  fence_async_smem();
  __syncthreads();

  uint32_t mma_phase = 0;
  int bad = 0, range = 0;
  float smax = 0.f;
  const uint32_t s_tile = smem_u32(sm + OFF_S);

  for (int c = 0; c < NC; ++c) {
    const int s = c & 1;
    const int t0 = c * C;
    const uint32_t kq = smem_u32(sm + OFF_KQ + s * KQ_STAGE);
    const uint32_t vt = smem_u32(sm + OFF_V + s * V_STAGE);
    uint8_t *kq_ptr = sm + OFF_KQ + s * KQ_STAGE;

    // ---- (a) gates: beta; per-channel cumulative log2 decay, in place, then
    // G_r = e^{gamma - gamma_m} with m = token 31
    if (tid < 64) sc_beta[tid] = pf_bt;
    if (c + 1 < NC) load_beta(c + 1);
    if (!mbar_wait(bar_lg, c & 1)) bad = 1;
    if (__syncthreads_or(bad)) break;
    {
      const int ch = tid & 127, hh = tid >> 7;
      float run = 0.f;
#pragma unroll 8
      for (int t = 32 * hh; t < 32 * hh + 32; ++t) {
        run += Gr[t * DK + ch] * LOG2E;
        Gr[t * DK + ch] = run;
      }
      if (hh == 0) sc_tmp[ch] = run;     // gamma at token 31 = the reference gamma_m
      __syncthreads();
      const float gm = sc_tmp[ch];
      if (hh == 0) sc_gm[ch] = gm;
#pragma unroll 8
      for (int t = 32 * hh; t < 32 * hh + 32; ++t) {
        float d = Gr[t * DK + ch] + (hh ? gm : 0.f) - gm;
        if (d > SPAN_SAFE || d < -SPAN_SAFE) {
          range = 1;
          d = fminf(fmaxf(d, -SPAN_SAFE), SPAN_SAFE);
        }
        Gr[t * DK + ch] = ex2(d);
      }
    }

    // ---- (b) chunk inputs landed?
    if (!mbar_wait(&bar_full[s], (c >> 1) & 1)) bad = 1;
    if (__syncthreads_or(bad)) break;

    // ---- (c) MMA1 in two 64-channel halves: [K o G; Q o G] (K o G^-1)^T in tf32;
    // also Kt = beta_r K o G_63 / G_r (fp16)
#pragma unroll 1
    for (int hp = 0; hp < 2; ++hp) {
#pragma unroll
      for (int it = 0; it < 4; ++it) {
        const int u = it * NTHREADS + tid;      // 1024 units: (t, 4-channel group j4)
        const int t = u >> 4, j4 = u & 15;
        const int ch0 = 64 * hp + 4 * j4;
        const uint32_t bf = sw128(t, j4 >> 1) + 8 * (j4 & 1);   // 4 bf16 values of the input tiles
        float kx[4], qx[4];
        unpack4(*reinterpret_cast<const uint2 *>(kq_ptr + hp * 16384 + bf), kx);
        unpack4(*reinterpret_cast<const uint2 *>(kq_ptr + hp * 16384 + 8192 + bf), qx);
        const float4 g4 = *reinterpret_cast<const float4 *>(Gr + t * DK + ch0);
        const float4 h4 = *reinterpret_cast<const float4 *>(Gr + 63 * DK + ch0);
        const float g[4] = {g4.x, g4.y, g4.z, g4.w}, g63[4] = {h4.x, h4.y, h4.z, h4.w};
        const float bt = sc_beta[t];
        float kg[4], qg[4], ig[4], kt[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float inv = __frcp_rn(g[e]);
          kg[e] = tf32r(kx[e] * g[e]);
          qg[e] = tf32r(p.scale * qx[e] * g[e]);
          ig[e] = tf32r(kx[e] * inv);
          kt[e] = bt * kx[e] * (g63[e] * inv);
        }
        // fp32 tiles: 32-channel atoms of 128-byte rows; 16-byte chunk j4 mod 8 of the row
        const uint32_t xa = (j4 >> 3) * 16384, ya = (j4 >> 3) * 8192;
        *reinterpret_cast<float4 *>(sm + OFF_XF + xa + sw128(t, j4 & 7)) = make_float4(kg[0], kg[1], kg[2], kg[3]);
        *reinterpret_cast<float4 *>(sm + OFF_XF + xa + sw128(64 + t, j4 & 7)) =
            make_float4(qg[0], qg[1], qg[2], qg[3]);
        *reinterpret_cast<float4 *>(sm + OFF_YF + ya + sw128(t, j4 & 7)) = make_float4(ig[0], ig[1], ig[2], ig[3]);
        *reinterpret_cast<uint2 *>(sm + OFF_KT + hp * 8192 + bf) =
            make_uint2(pack_f16x2(kt[0], kt[1]), pack_f16x2(kt[2], kt[3]));
      }
      fence_async_smem();
      __syncthreads();
      if (tid == 0) {
        tc_fence_after();
        const uint32_t xf = smem_u32(sm + OFF_XF), yf = smem_u32(sm + OFF_YF);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_tf32(tmem + COL_G, sdesc(xf + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                   sdesc(yf + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024), ID_G, hp + kk > 0);
        mma_commit(bar_mma);
      }
      if (!mbar_wait(bar_mma, mma_phase)) bad = 1;
      mma_phase ^= 1;
      tc_fence_after();
    }

    // ---- (d) A (lanes 0-63) and P (lanes 64-127); decay already inside the products
    {
      float g[32];
      tmem_ld32(tmem + lane_base + COL_G + 32 * half, g);
      const int t = row & 63;
      const int r0 = 32 * half;
      if (quad < 2) {
#pragma unroll
        for (int r = 0; r < 32; ++r) At[(r0 + r) * LD + t] = (r0 + r < t) ? tf32r(g[r] * sc_beta[r0 + r]) : 0.f;
      } else {
#pragma unroll
        for (int r = 0; r < 32; ++r) g[r] = (r0 + r <= t) ? g[r] * sc_beta[r0 + r] : 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) st_chunk_f16(sm + OFF_P + sw128(t, 4 * half + j), g + 8 * j);
      }
    }
    tc_fence_before();
    __syncthreads();

    // ---- (e) T = (I + A)^{-1}; T as bf16; K o e^{gamma} as bf16 (B operand of W)
    solve_unit_lower_64(At, Tf, tid, warp, lane);
    {
      const int m = tid >> 2, n0 = (tid & 3) * 16;
      float tv[16];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const float4 f = *reinterpret_cast<const float4 *>(Tf + m * LD + n0 + 4 * q4);
        tv[4 * q4 + 0] = f.x; tv[4 * q4 + 1] = f.y; tv[4 * q4 + 2] = f.z; tv[4 * q4 + 3] = f.w;
      }
#pragma unroll
      for (int e = 0; e < 16; ++e) tv[e] = (n0 + e <= m) ? tv[e] : 0.f;
#pragma unroll
      for (int j = 0; j < 2; ++j) st_chunk_bf16(sm + OFF_ZT + 8192 + sw128(m, 2 * (tid & 3) + j), tv + 8 * j);
    }
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int u = it * NTHREADS + tid;        // 1024 units: (atom, t, chunk j)
      const int kb = u >> 9, t = (u >> 3) & 63, j = u & 7;
      const int ch0 = 64 * kb + 8 * j;
      float kx[8];
      unpack8(*reinterpret_cast<const uint4 *>(kq_ptr + kb * 16384 + sw128(t, j)), kx);
#pragma unroll
      for (int e = 0; e < 8; ++e) kx[e] *= Gr[t * DK + ch0 + e] * ex2(sc_gm[ch0 + e]);
      st_chunk_bf16(sm + OFF_KG + kb * 8192 + sw128(t, j), kx);
    }
    fence_async_smem();
    __syncthreads();

    // ---- (f) MMA2: W = T (K o e^{gamma}) ; lanes 64-127 of YE = T V (lanes 0-63 = 0)
    if (tid == 0) {
      tc_fence_after();
      const uint32_t zt = smem_u32(sm + OFF_ZT), kg = smem_u32(sm + OFF_KG);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ss(tmem + COL_W, sdesc(zt + 8192 + kk * 32, 16, 1024), sdesc(kg + kk * 2048, 8192, 1024), ID_W,
                 kk > 0);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ss(tmem + COL_YE, sdesc(zt + kk * 32, 16, 1024), sdesc(vt + kk * 2048, 8192, 1024), ID_U, kk > 0);
      mma_commit(bar_mma);
    }
    if (!mbar_wait(bar_mma, mma_phase)) bad = 1;
    mma_phase ^= 1;
    tc_fence_after();

    // ---- (g) -W -> fp16; fp16 copy of scale Q o e^{gamma}; this thread's state-row
    // decay e^{gamma_C}; then the decay tile is free for the next chunk's gates
    const float gc_row = Gr[63 * DK + row] * ex2(sc_gm[row]);
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int u = it * NTHREADS + tid;
      const int kb = u >> 9, t = (u >> 3) & 63, j = u & 7;
      const int ch0 = 64 * kb + 8 * j;
      float x[8];
      unpack8(*reinterpret_cast<const uint4 *>(kq_ptr + kb * 16384 + 8192 + sw128(t, j)), x);
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] *= p.scale * Gr[t * DK + ch0 + e] * ex2(sc_gm[ch0 + e]);
      st_chunk_f16(sm + OFF_QW + kb * 16384 + sw128(t, j), x);
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
    if (tid == 0 && c + 1 < NC) issue_gates(c + 1);

    // ---- (h) MMA3: YE += [Qg; -W] S0
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

    // ---- (i) E (lanes 64-127) -> fp16
    if (quad >= 2) {
      float e[32];
      tmem_ld32(tmem + lane_base + COL_YE + 32 * half, e);
      const int r = row - 64;
#pragma unroll
      for (int j = 0; j < 32; ++j) smax = fmaxf(smax, fabsf(e[j]));
#pragma unroll
      for (int j = 0; j < 4; ++j) st_chunk_f16(sm + OFF_E + sw128(r, 4 * half + j), e + 8 * j);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- (j) MMA4: dS = Kt^T E ; YE += [P; *] E
    if (tid == 0) {
      tc_fence_after();
      const uint32_t kt = smem_u32(sm + OFF_KT), et = smem_u32(sm + OFF_E), pt = smem_u32(sm + OFF_P);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ss(tmem + COL_S, sdesc(kt + kk * 2048, 8192, 1024), sdesc(et + kk * 2048, 8192, 1024), ID_DS,
                 kk > 0);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ss(tmem + COL_YE, sdesc(pt + kk * 32, 16, 1024), sdesc(et + kk * 2048, 8192, 1024), ID_PE, 1);
      mma_commit(bar_mma);
    }
    if (!mbar_wait(bar_mma, mma_phase)) bad = 1;
    mma_phase ^= 1;
    tc_fence_after();

    // ---- (k) state update (row decay e^{gamma_C[row]}) and output rows (lanes 0-63)
    {
      float d[32];
      tmem_ld32(tmem + lane_base + COL_S + 32 * half, d);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        S[j] = fmaf(gc_row, S[j], d[j]);
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
    if (tid == 0) atomicOr(&g_gdr_chan_error, 1);
  } else {
    if (smax > F16_SAFE || range) atomicOr(&g_gdr_chan_error, 2);
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
cudaError_t launch_chan(const FwdProblem &p, cudaStream_t stream, std::string *err) {
  cudaError_t e = cudaFuncSetAttribute(chunk_chan_kernel<VAR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)SMEM_BYTES);
  if (e != cudaSuccess) {
    *err = "cudaFuncSetAttribute: ";
    return e;
  }
  CUtensorMap mq, mk, mv, mg;
  if (!make_map(&mq, p.q, p.B, p.T, p.H, p.dk) || !make_map(&mk, p.k, p.B, p.T, p.H, p.dk) ||
      !make_map(&mv, p.v, p.B, p.T, p.H, p.dv) || !make_map_f32_rows(&mg, p.log_g, p.B, p.T, p.H, p.dk)) {
    *err = "cuTensorMapEncodeTiled failed: ";
    return cudaErrorInvalidValue;
  }
  Params kp;
  kp.T = p.T; kp.H = p.H; kp.dv = p.dv;
  kp.beta = p.beta; kp.s0 = p.s0; kp.s_final = p.s_final;
  kp.o = static_cast<__nv_bfloat16 *>(p.o);
  kp.scale = p.scale;
  const dim3 grid(p.dv / BV, p.H, p.B), block(NTHREADS);
  chunk_chan_kernel<VAR><<<grid, block, SMEM_BYTES, stream>>>(mq, mk, mv, mg, kp);
  e = cudaGetLastError();
  if (e != cudaSuccess) *err = "launch: ";
  return e;
}

}  // namespace
}  // namespace tc
}  // namespace gdr

cudaError_t gdr_launch_chunk_chan(const gdr::FwdProblem &p, cudaStream_t stream, std::string *err) {
  using namespace gdr;
  if (p.variant == kKDA) return tc::launch_chan<kKDA>(p, stream, err);
  *err = "variant not covered: ";
  return cudaErrorInvalidValue;
}

int gdr_read_chan_error() {
  int h = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&h, g_gdr_chan_error, sizeof(int)) != cudaSuccess) return -1;
  if (h) cudaMemcpyToSymbol(g_gdr_chan_error, &zero, sizeof(int));
  return h;
}
