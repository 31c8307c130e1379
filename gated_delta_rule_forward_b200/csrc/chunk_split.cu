// Two-kernel chunked forward for the scalar-decay variants (DeltaNet, Gated
// DeltaNet, KLA): a chunk-parallel preparation kernel and a sequential carry
// kernel, with the per-chunk products passed through a workspace.
//
// The chunk algebra is the one of chunk_tc.cu ("Kaczmarz Linear Attention",
// KLA update rule and implementation; "Gated DeltaNet-2", technical core):
//     T = (I + A)^{-1},  W = T Diag(Gamma) K,  U' = T V,  E = U' - W S0
//     O = Diag(scale Gamma) Q S0 + P E,   S_C = Gamma_C S0 + K^T Diag(w) E.
// Everything that does not depend on S0 -- A, P, the solve, W, U' -- is the
// bulk of the work and is independent across chunks.  The preparation kernel
// computes it with one CTA per (batch, head, chunk) over the whole machine (two
// CTAs per SM) instead of inside the sequential sweep, and it is shared by all
// value slices of a head.  The carry kernel then does only what depends on the
// state: [Diag(scale Gamma) Q; -W] S0, E, K^T Diag(w) E and P E, and the state
// update, one CTA per (batch, head, 64-column value slice).
//
// Workspace record per (b, h, chunk), all tile images in the 128-byte-swizzled
// layout the tensor cores read, so the carry kernel bulk-copies them into
// shared memory unchanged:
//     REC_W   fp16 -W, K-major atoms [d_k 0-63 | 64-127]         16 KB
//     REC_U   fp16 U' per 64-column value slice                  8 KB x NS
//     REC_P   fp16 P (rows t, columns r)                          8 KB
//     REC_SC  fp32 scale Gamma_t [64], w_r [64], Gamma_C          1 KB
#include <mutex>

#include "chunk_common.cuh"
#include "chunk_tc.cuh"
#include "tc_util.cuh"
#include "tma_host.cuh"

// Device-side error word of this file (see gdr_device_status()).
__device__ int g_gdr_split_error = 0;

// Fixed scratch for gdr_forward_chunked_noalloc(): the two-kernel path's
// workspace for callers that cannot allocate device memory.  It is part of
// this library's device image, so every GPU that loads the library holds it
// until the process exits.  All calls share it; the preparation kernel fully
// rewrites the records a call uses before the carry kernel reads them, so
// nothing needs clearing between calls, and calls that overlap on the GPU race.
constexpr size_t kFixedScratchBytes = size_t(32) << 20;
static __device__ __align__(256) uint8_t g_split_fixed_scratch[kFixedScratchBytes];

namespace gdr {
namespace tc {
namespace {

constexpr int C = 64;
constexpr int DK = 128;
constexpr int NTHREADS = 256;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float F16_SAFE = 60000.f;

__host__ __device__ constexpr uint32_t rec_u(int) { return 16384; }
__host__ __device__ constexpr uint32_t rec_p(int ns) { return 16384 + 8192 * ns; }
__host__ __device__ constexpr uint32_t rec_sc(int ns) { return rec_p(ns) + 8192; }
__host__ __device__ constexpr uint32_t rec_bytes(int ns) { return rec_sc(ns) + 1024; }

// ------------------------------------------------------------------ preparation kernel
namespace prep {
constexpr uint32_t OFF_KQ = 0;          // bf16 [Kb0 | Qb0 | Kb1 | Qb1] (TMA)
constexpr uint32_t OFF_V = 32768;       // bf16 V, one 8 KB box per value slice (TMA)
constexpr uint32_t OFF_A = 49152;       // fp32 A^T, 64 x LD
constexpr uint32_t OFF_TF = OFF_A + 64 * LD * 4;
constexpr uint32_t OFF_T = 86016;       // bf16 T
constexpr uint32_t OFF_TP = 94208;      // bf16 T Diag(Gamma)
constexpr uint32_t OFF_SC = 102400;     // scalars: 5 x 64 floats
constexpr uint32_t OFF_BAR = OFF_SC + 5 * 64 * 4;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 64 + 1024;
static_assert(OFF_TF + 64 * LD * 4 <= OFF_T, "layout");
constexpr uint32_t COL_G = 0;     // M128 x 64 (dead before W)
constexpr uint32_t COL_W = 0;     // M64 x 128
constexpr uint32_t COL_U = 128;   // M64 x dv
constexpr uint32_t TMEM_COLS = 256;
}  // namespace prep

struct PrepParams {
  int T, H, dv, NC;
  const float *beta, *log_g;
  uint8_t *ws;
  float eps, scale;
};

template <int VAR>
__global__ void __launch_bounds__(NTHREADS, 2)
    chunk_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const PrepParams p) {
  using namespace prep;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quad = warp & 3, half = warp >> 2;
  const int row = quad * 32 + lane;
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int NS = p.dv / 64;
  const int t0 = c * C;

  uint64_t *bar_in = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
  uint64_t *bar_mma = bar_in + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_in + 2);
  float *sc_beta = reinterpret_cast<float *>(sm + OFF_SC);
  float *sc_g2 = sc_beta + 64;
  float *sc_wf = sc_g2 + 64;
  float *sc_G = sc_wf + 64;
  float *sc_tmp = sc_G + 64;
  float *At = reinterpret_cast<float *>(sm + OFF_A);
  float *Tf = reinterpret_cast<float *>(sm + OFF_TF);
  uint8_t *rec = p.ws + ((static_cast<size_t>(b) * p.H + h) * p.NC + c) * rec_bytes(NS);

  if (warp == 0) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar_in, 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
    mbar_expect_tx(bar_in, 4 * 8192 + NS * 8192);
    tma_load_4d(sm + OFF_KQ + 0, &tm_k, bar_in, 0, h, t0, b);
    tma_load_4d(sm + OFF_KQ + 8192, &tm_q, bar_in, 0, h, t0, b);
    tma_load_4d(sm + OFF_KQ + 16384, &tm_k, bar_in, 64, h, t0, b);
    tma_load_4d(sm + OFF_KQ + 24576, &tm_q, bar_in, 64, h, t0, b);
    for (int sl = 0; sl < NS; ++sl) tma_load_4d(sm + OFF_V + sl * 8192, &tm_v, bar_in, 64 * sl, h, t0, b);
  }
  // gates: beta_t, cumulative log2 decay, Gamma_t
  if (tid < 64) {
    const int t = t0 + tid;
    float lg = 0.f, bt = 0.f;
    if (t < p.T) {
      const size_t th = (static_cast<size_t>(b) * p.T + t) * p.H + h;
      if constexpr (scalar_decay(VAR)) lg = __ldg(p.log_g + th);
      bt = __ldg(p.beta + th);
    }
    float x = lg * LOG2E;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    sc_tmp[tid] = x;
    sc_beta[tid] = bt;
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
  if (tid < 64) {
    const float g2 = sc_tmp[tid] + (tid >= 32 ? sc_tmp[31] : 0.f);
    sc_g2[tid] = g2;
    sc_G[tid] = ex2(g2);
  }
  int bad = 0;
  if (!mbar_wait(bar_in, 0)) bad = 1;
  bad = __syncthreads_or(bad);
  const uint32_t kq = smem_u32(sm + OFF_KQ);
  uint32_t mma_phase = 0;

  // MMA1: [K;Q] K^T
  if (!bad && tid == 0) {
    tc_fence_after();
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint32_t a = kq + (kk >> 2) * 16384 + (kk & 3) * 32;
      mma_bf16(tmem + COL_G, sdesc(a, 16, 1024), sdesc(a, 16, 1024), idesc_bf16(128, 64, false, false), kk > 0);
    }
    mma_commit(bar_mma);
  }
  if (!bad && !mbar_wait(bar_mma, mma_phase)) bad = 1;
  bad = __syncthreads_or(bad);
  mma_phase ^= 1;
  tc_fence_after();

  // A (lanes 0-63) -> A^T scratch; P (lanes 64-127) -> fp16 record tile
  if (!bad) {
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
      for (int j = 0; j < 4; ++j) st_chunk_f16(rec + rec_p(NS) + sw128(t, 4 * half + j), g + 8 * j);
    }
  }
  tc_fence_before();
  __syncthreads();

  // T = (I + A)^{-1}; T and T Diag(Gamma) as bf16 tiles
  solve_unit_lower_64(At, Tf, tid, warp, lane);
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
      tv[e] = (n0 + e <= m) ? tv[e] : 0.f;
      tg[e] = tv[e] * sc_G[n0 + e];
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      st_chunk_bf16(sm + OFF_T + sw128(m, 2 * (tid & 3) + j), tv + 8 * j);
      st_chunk_bf16(sm + OFF_TP + sw128(m, 2 * (tid & 3) + j), tg + 8 * j);
    }
  }
  // per-row scalars of the record: scale Gamma_t, w_r, Gamma_C
  if (tid < 64) {
    float *rs = reinterpret_cast<float *>(rec + rec_sc(NS));
    rs[tid] = p.scale * sc_G[tid];
    rs[64 + tid] = sc_wf[tid];
    if (tid == 0) rs[128] = sc_G[63];
  }
  fence_async_smem();
  __syncthreads();

  // MMA2: W = T Diag(Gamma) K (M64 N128); U' = T V (M64 N dv)
  if (!bad && tid == 0) {
    tc_fence_after();
    const uint32_t tp = smem_u32(sm + OFF_TP), tt = smem_u32(sm + OFF_T), vt = smem_u32(sm + OFF_V);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_bf16(tmem + COL_W, sdesc(tp + kk * 32, 16, 1024), sdesc(kq + kk * 2048, 16384, 1024),
               idesc_bf16(64, 128, false, true), kk > 0);
    const uint32_t id_u = NS == 2 ? idesc_bf16(64, 128, false, true) : idesc_bf16(64, 64, false, true);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_bf16(tmem + COL_U, sdesc(tt + kk * 32, 16, 1024), sdesc(vt + kk * 2048, 8192, 1024), id_u, kk > 0);
    mma_commit(bar_mma);
  }
  if (!bad && !mbar_wait(bar_mma, mma_phase)) bad = 1;
  bad = __syncthreads_or(bad);
  mma_phase ^= 1;
  tc_fence_after();

  // -W and U' (M64 layout: rows 16 quad + lane, lane < 16) -> fp16 record tiles.
  // Column half `half` of W is d_k atom `half`; of U' it is value slice `half`.
  float wmax = 0.f;
  if (!bad) {
    float w[32];
#pragma unroll
    for (int part = 0; part < 2; ++part) {
      tmem_ld32(tmem + lane_base + COL_W + 64 * half + 32 * part, w);
      if (lane < 16) {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          wmax = fmaxf(wmax, fabsf(w[e]));
          w[e] = -w[e];
        }
#pragma unroll
        for (int j = 0; j < 4; ++j)
          st_chunk_f16(rec + half * 8192 + sw128(quad * 16 + lane, 4 * part + j), w + 8 * j);
      }
    }
    if (half < NS) {
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        tmem_ld32(tmem + lane_base + COL_U + 64 * half + 32 * part, w);
        if (lane < 16) {
#pragma unroll
          for (int e = 0; e < 32; ++e) wmax = fmaxf(wmax, fabsf(w[e]));
#pragma unroll
          for (int j = 0; j < 4; ++j)
            st_chunk_f16(rec + rec_u(NS) + half * 8192 + sw128(quad * 16 + lane, 4 * part + j), w + 8 * j);
        }
      }
    }
  }
  if (bad && tid == 0) atomicOr(&g_gdr_split_error, 1);
  if (wmax > F16_SAFE) atomicOr(&g_gdr_split_error, 2);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ------------------------------------------------------------------ carry kernel
// Software-pipelined over chunks: the critical path is MMA3(c) -> E -> dS(c)
// -> S -> MMA3(c+1); the fp16 copies for chunk c+1 are made while MMA4(c)
// runs, and the output rows of chunk c are written while MMA3(c+1) runs.
// TMEM output tiles and the Diag(w) K copy are double-buffered for that.
namespace carry {
constexpr uint32_t STAGE = 82944;       // 81 KB per chunk stage
constexpr uint32_t S_KQ = 0;            // bf16 raw [Kb0 | Qb0 | Kb1 | Qb1] (TMA)
constexpr uint32_t S_QW = 32768;        // fp16 [Qg b0 | -W b0 | Qg b1 | -W b1] (Qg by threads, -W bulk)
constexpr uint32_t S_P = 65536;         // fp16 P (bulk); the U' tile follows as rows 64-127 of [P; *]
constexpr uint32_t S_U = 73728;         // fp16 U' of this slice (bulk)
constexpr uint32_t S_SC = 81920;        // fp32 scale Gamma_t [64], w_r [64], Gamma_C (bulk)
constexpr uint32_t OFF_KT = 2 * STAGE;  // 2 x fp16 Diag(w) K [Kb0 | Kb1]
constexpr uint32_t OFF_E = OFF_KT + 2 * 16384;
constexpr uint32_t OFF_S = OFF_E + 8192;
constexpr uint32_t OFF_BAR = OFF_S + 16384;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 64 + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(STAGE % 1024 == 0 && OFF_KT % 1024 == 0 && OFF_S % 1024 == 0, "alignment");
constexpr uint32_t COL_YE = 0;    // 2 x (M128 x 64): lanes 0-63 Qg S0 + P E, lanes 64-127 -W S0
constexpr uint32_t COL_S = 128;   // M128 x 64: dS
constexpr uint32_t TMEM_COLS = 256;
}  // namespace carry

struct CarryParams {
  int T, H, dv, NC;
  const uint8_t *ws;
  const float *s0;
  float *s_final;
  __nv_bfloat16 *o;
};

__global__ void __launch_bounds__(NTHREADS, 1)
    chunk_carry_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const CarryParams p) {
  using namespace carry;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quad = warp & 3, half = warp >> 2;
  const int row = quad * 32 + lane;
  const int sl = blockIdx.x, v0 = 64 * sl, h = blockIdx.y, b = blockIdx.z;
  const int NS = p.dv / 64, NC = p.NC;

  uint64_t *bar_full = reinterpret_cast<uint64_t *>(sm + OFF_BAR);   // [2] chunk inputs
  uint64_t *bar_e = bar_full + 2;                                    // MMA3 done
  uint64_t *bar_s = bar_full + 3;                                    // dS done
  uint64_t *bar_o = bar_full + 4;                                    // P E done
  uint64_t *bar_drain = bar_full + 5;                                // error path only
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_full + 6);

  if (warp == 0) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar_full[0], 1);
    mbar_init(&bar_full[1], 1);
    mbar_init(bar_e, 1);
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    mbar_init(bar_drain, 1);
    fence_mbar_init();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
  }
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
  const size_t rb = rec_bytes(NS);
  const uint8_t *recs = p.ws + (static_cast<size_t>(b) * p.H + h) * NC * rb;
  const uint32_t s_tile = smem_u32(sm + OFF_S), e_tile = smem_u32(sm + OFF_E);

  // load phases issued into / seen landing in stage 0 (low 16 bits) and 1 (high 16 bits)
  uint32_t n_issued = 0, n_landed = 0;
  auto issue_chunk = [&](int c, int s) {
    n_issued += 1u << (16 * s);
    uint8_t *st = sm + s * STAGE;
    const uint8_t *rec = recs + c * rb;
    uint64_t *bar = &bar_full[s];
    mbar_expect_tx(bar, 4 * 8192 + 2 * 8192 + 8192 + 8192 + 1024);
    tma_load_4d(st + S_KQ + 0, &tm_k, bar, 0, h, c * C, b);
    tma_load_4d(st + S_KQ + 8192, &tm_q, bar, 0, h, c * C, b);
    tma_load_4d(st + S_KQ + 16384, &tm_k, bar, 64, h, c * C, b);
    tma_load_4d(st + S_KQ + 24576, &tm_q, bar, 64, h, c * C, b);
    bulk_load(st + S_QW + 8192, rec + 0, 8192, bar);
    bulk_load(st + S_QW + 24576, rec + 8192, 8192, bar);
    bulk_load(st + S_P, rec + rec_p(NS), 8192, bar);
    bulk_load(st + S_U, rec + rec_u(NS) + sl * 8192, 8192, bar);
    bulk_load(st + S_SC, rec + rec_sc(NS), 1024, bar);
  };
  // fp16 Diag(scale Gamma) Q into the stage and fp16 Diag(w) K into buffer kbuf
  // (1024 + 1024 sixteen-byte chunks, 8 per thread)
  auto convert = [&](int s, int kbuf) {
    uint8_t *st = sm + s * STAGE;
    const float *rs = reinterpret_cast<const float *>(st + S_SC);
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      const int u = it * NTHREADS + tid;
      const int isq = u >> 10, kb = (u >> 9) & 1, r = (u >> 3) & 63, j = u & 7;
      const uint32_t off = sw128(r, j);
      float x[8];
      unpack8(*reinterpret_cast<const uint4 *>(st + S_KQ + kb * 16384 + isq * 8192 + off), x);
      const float f = rs[isq ? r : 64 + r];
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] *= f;
      st_chunk_f16(isq ? st + S_QW + kb * 16384 + off : sm + OFF_KT + kbuf * 16384 + kb * 8192 + off, x);
    }
  };
  // YE[yb] = [Qg; -W] S0 of stage s
  auto issue_mma3 = [&](int s, int yb) {
    tc_fence_after();
    const uint32_t qw = smem_u32(sm + s * STAGE + S_QW);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
      mma_bf16(tmem + COL_YE + 64 * yb, sdesc(qw + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
               sdesc(s_tile + kk * 2048, 8192, 1024), idesc_f16(128, 64, false, true), kk > 0);
    mma_commit(bar_e);
  };

  int bad = 0;
  float smax = 0.f;
  if (tid == 0) {
    issue_chunk(0, 0);
    if (NC > 1) issue_chunk(1, 1);
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) st_chunk_f16(sm + OFF_S + sw128(row, 4 * half + j), S + 8 * j);
  if (mbar_wait(&bar_full[0], 0)) n_landed += 1;
  else bad = 1;
  bad = __syncthreads_or(bad);
  if (!bad) convert(0, 0);
  fence_async_smem();
  bad = __syncthreads_or(bad);
  if (!bad && tid == 0) issue_mma3(0, 0);

  for (int c = 0; c < NC && !bad; ++c) {
    const int s = c & 1, yb = c & 1;
    uint8_t *st = sm + s * STAGE;
    const float *rs = reinterpret_cast<const float *>(st + S_SC);
    const uint32_t ye = tmem + COL_YE + 64 * yb;

    // (1) E = U' - W S0 (lanes 64-127) -> fp16
    if (!mbar_wait(bar_e, c & 1)) bad = 1;
    tc_fence_after();
    if (quad >= 2) {
      float e[32], u[8];
      tmem_ld32(lane_base + ye + 32 * half, e);
      const int r = row - 64;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 raw = *reinterpret_cast<const uint4 *>(st + S_U + sw128(r, 4 * half + j));
        const __half2 *hp = reinterpret_cast<const __half2 *>(&raw);
#pragma unroll
        for (int q2 = 0; q2 < 4; ++q2) {
          const float2 f = __half22float2(hp[q2]);
          u[2 * q2] = f.x;
          u[2 * q2 + 1] = f.y;
        }
#pragma unroll
        for (int e8 = 0; e8 < 8; ++e8) {
          e[8 * j + e8] += u[e8];
          smax = fmaxf(smax, fabsf(e[8 * j + e8]));
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) st_chunk_f16(sm + OFF_E + sw128(r, 4 * half + j), e + 8 * j);
    }
    fence_async_smem();
    tc_fence_before();
    if ((bad = __syncthreads_or(bad))) break;

    // (2) dS = (Diag(w) K)^T E ; YE[yb] += [P; *] E
    if (tid == 0) {
      tc_fence_after();
      const uint32_t kt = smem_u32(sm + OFF_KT + yb * 16384), pt = smem_u32(st + S_P);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem + COL_S, sdesc(kt + kk * 2048, 8192, 1024), sdesc(e_tile + kk * 2048, 8192, 1024),
                 idesc_f16(128, 64, true, true), kk > 0);
      mma_commit(bar_s);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(ye, sdesc(pt + kk * 32, 16, 1024), sdesc(e_tile + kk * 2048, 8192, 1024),
                 idesc_f16(128, 64, false, true), 1);
      mma_commit(bar_o);
    }

    // (3) while MMA4 runs: the next chunk's fp16 copies
    if (c + 1 < NC) {
      if (!mbar_wait(&bar_full[s ^ 1], ((c + 1) >> 1) & 1)) {
        bad = 1;
      } else {
        n_landed += 1u << (16 * (s ^ 1));
        convert(s ^ 1, yb ^ 1);
      }
    }

    // (4) state update: S = Gamma_C S + dS -> fp16 tile; then MMA3 of the next chunk
    if (!mbar_wait(bar_s, c & 1)) bad = 1;
    tc_fence_after();
    {
      float d[32];
      tmem_ld32(tmem + lane_base + COL_S + 32 * half, d);
      const float gc = rs[128];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        S[j] = fmaf(gc, S[j], d[j]);
        smax = fmaxf(smax, fabsf(S[j]));
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) st_chunk_f16(sm + OFF_S + sw128(row, 4 * half + j), S + 8 * j);
    }
    fence_async_smem();
    tc_fence_before();
    if ((bad = __syncthreads_or(bad))) break;
    if (tid == 0 && c + 1 < NC) issue_mma3(s ^ 1, yb ^ 1);

    // (5) while MMA3 of the next chunk runs: output rows of this chunk (lanes 0-63)
    if (!mbar_wait(bar_o, c & 1)) bad = 1;
    tc_fence_after();
    if (quad < 2) {
      float d[32];
      tmem_ld32(lane_base + ye + 32 * half, d);
      const int t = c * C + row;
      if (t < p.T) {
        uint8_t *dst = reinterpret_cast<uint8_t *>(
            p.o + ((static_cast<size_t>(b) * p.T + t) * p.H + h) * p.dv + v0 + 32 * half);
#pragma unroll
        for (int j = 0; j < 4; ++j) st_chunk_bf16(dst + 16 * j, d + 8 * j);
      }
    }
    tc_fence_before();
    if ((bad = __syncthreads_or(bad))) break;
    if (tid == 0 && c + 2 < NC) issue_chunk(c + 2, s);
  }

  if (bad) {
    // a wait gave up: report it, then let this CTA's MMAs and copies in
    // flight finish (each wait again bounded) before TMEM is released
    if (tid == 0) {
      atomicOr(&g_gdr_split_error, 1);
      mma_commit(bar_drain);
      mbar_wait(bar_drain, 0);
      for (int st = 0; st < 2; ++st) {
        const uint32_t got = (n_landed >> (16 * st)) & 0xffff, sent = (n_issued >> (16 * st)) & 0xffff;
        if (got < sent) mbar_wait(&bar_full[st], got & 1);
      }
    }
  } else {
    if (smax > F16_SAFE) atomicOr(&g_gdr_split_error, 2);
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
cudaError_t launch_split(const FwdProblem &p, void *ws, cudaStream_t stream, std::string *err) {
  cudaError_t e = cudaFuncSetAttribute(chunk_prep_kernel<VAR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)prep::SMEM_BYTES);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(chunk_carry_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)carry::SMEM_BYTES);
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
  const int NC = (p.T + C - 1) / C;
  PrepParams pp;
  pp.T = p.T; pp.H = p.H; pp.dv = p.dv; pp.NC = NC;
  pp.beta = p.beta; pp.log_g = p.log_g; pp.ws = static_cast<uint8_t *>(ws);
  pp.eps = p.eps; pp.scale = p.scale;
  chunk_prep_kernel<VAR><<<dim3(NC, p.H, p.B), NTHREADS, prep::SMEM_BYTES, stream>>>(mq, mk, mv, pp);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    *err = "prep launch: ";
    return e;
  }
  CarryParams cp;
  cp.T = p.T; cp.H = p.H; cp.dv = p.dv; cp.NC = NC;
  cp.ws = static_cast<const uint8_t *>(ws); cp.s0 = p.s0; cp.s_final = p.s_final;
  cp.o = static_cast<__nv_bfloat16 *>(p.o);
  chunk_carry_kernel<<<dim3(p.dv / 64, p.H, p.B), NTHREADS, carry::SMEM_BYTES, stream>>>(mq, mk, cp);
  e = cudaGetLastError();
  if (e != cudaSuccess) *err = "carry launch: ";
  return e;
}

}  // namespace
}  // namespace tc
}  // namespace gdr

bool gdr_split_supported(int variant, int dk, int dv) {
  using namespace gdr;
  const bool v = variant == kDeltaNet || variant == kGatedDeltaNet || variant == kKLA;
  return v && dk == 128 && (dv == 64 || dv == 128);
}

size_t gdr_split_workspace_bytes(int B, int T, int H, int dv) {
  const size_t NC = (static_cast<size_t>(T) + 63) / 64;
  return static_cast<size_t>(B) * H * NC * gdr::tc::rec_bytes(dv / 64);
}

cudaError_t gdr_launch_split(const gdr::FwdProblem &p, void *ws, cudaStream_t stream, std::string *err) {
  using namespace gdr;
  switch (p.variant) {
    case kDeltaNet: return tc::launch_split<kDeltaNet>(p, ws, stream, err);
    case kGatedDeltaNet: return tc::launch_split<kGatedDeltaNet>(p, ws, stream, err);
    case kKLA: return tc::launch_split<kKLA>(p, ws, stream, err);
    default: *err = "variant not covered: "; return cudaErrorInvalidValue;
  }
}

int gdr_read_split_error() {
  int h = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&h, g_gdr_split_error, sizeof(int)) != cudaSuccess) return -1;
  if (h) cudaMemcpyToSymbol(g_gdr_split_error, &zero, sizeof(int));
  return h;
}

size_t gdr_split_fixed_scratch_bytes() { return kFixedScratchBytes; }

// Device address of the fixed scratch on the current device.  Host code only
// holds a stand-in for the array, so the address is looked up with
// cudaGetSymbolAddress, once per device, while that device is current.
cudaError_t gdr_split_fixed_scratch(void **ptr) {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static void *addr[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_split_fixed_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *ptr = addr[dev];
  return cudaSuccess;
}
