// Two-kernel chunked forward for all five variants (DeltaNet, Gated DeltaNet,
// KLA, KDA, Gated DeltaNet-2): chunk-parallel preparation kernels and a
// sequential carry kernel, with the per-chunk products passed through a
// workspace.
//
// The chunk algebra ("Kaczmarz Linear Attention",
// KLA update rule and implementation; "Gated DeltaNet-2", technical core):
//     T = (I + A)^{-1},  W = T Diag(Gamma) K,  U' = T V,  E = U' - W S0
//     O = Diag(scale Gamma) Q S0 + P E,   S_C = Gamma_C S0 + K^T Diag(w) E.
// Everything that does not depend on S0 -- A, P, the solve, W, U' and the
// scaled copies Qg = Diag(scale Gamma) Q and Kt = Diag(w) K -- is the bulk of
// the work and is independent across chunks.  A preparation kernel computes
// it per (batch, head, chunk) over the whole machine instead of inside the
// sequential sweep; there is one for the scalar decays (DeltaNet, GDN, KLA),
// one for the per-channel decay of KDA (Gamma_C a vector, the Gram product
// in tf32 around the middle token) and one for GDN-2, whose separate erase
// and write gates add two state-free terms (P^d V into the output and
// D~^T V into the state) that its record carries precomputed.
//
// The carry kernel does only what depends on the state, one CTA per
// (batch, head), in transposed form so that the state is the tensor-memory
// operand of every product:
//     Y_W = S0^T (-W)^T,  Y_Q = S0^T Qg^T,  E^T = U'^T + Y_W,
//     dS^T = E^T Kt,  O^T = Y_Q + E^T P^T,  S_C^T = Gamma_C S0^T + dS^T.
// Lane v of tensor memory is value column v; S^T and E^T are written there in
// fp16 by the threads that own them and read by the MMAs from there, so the
// sweep moves no operand through shared memory except the record itself.
// Its template MODE picks the decay of the state update: a scalar Gamma_C,
// a per-channel Gamma_C, or the per-channel one plus the GDN-2 terms.
//
// The carry's B*H CTAs leave the rest of the device idle.  With few long
// sequences the carry is segmented: each sequence is cut into G segments, the
// affine maps of the segments (S -> M_g S + D_g, computed by one state-only
// launch of the carry kernel) are chained by a small kernel into each
// segment's start state, and a last launch runs all segments at once from
// their start states.  Otherwise, where the idle SMs pay for it, the sweep is
// pipelined: the chunks are cut in two, and the second part's preparation
// runs on the SMs beside the first part's carry.  Consecutive grids are
// chained by programmatic dependent launch (griddepcontrol).
//
// Workspace record per (b, h, chunk).  The tiles the MMAs read are images of
// the 128-byte-swizzled shared-memory layout, so the carry kernel bulk-copies
// the whole record into shared memory unchanged:
//     REC_WQ  fp16 [-W; Qg] per d_k atom: [-W 0-63 | Qg 0-63 | -W 64-127 | Qg 64-127],
//             rows t, K-major (the N = 128 operand of one product)   32 KB
//     REC_K   fp16 Kt, rows t, atoms [d_k 0-63 | 64-127] (read as the MN-major operand)  16 KB
//     REC_P   fp16 P, rows t, columns r                            8 KB
//     REC_U   fp16 U'^T, rows v, columns t (swizzled 16-byte chunks) 8 KB per 64 values
//     REC_SC  fp32 Gamma_C: one value padded to 16 bytes, or d_k values
//     GDN-2 only: the P^d V and D~^T V terms, 24 KB per 64 values
#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "chunk_bwd.cuh"
#include "chunk_common.cuh"
#include "chunk_record.cuh"
#include "chunk_split.cuh"
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

constexpr int NTHREADS = 256;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float F16_SAFE = 60000.f;


// ------------------------------------------------------------------ preparation kernel
// Three CTAs share an SM (72 KB of shared memory, 128 tensor-memory columns
// and at most 80 registers a thread each), so buffers are reused by phase:
//   Q slots: Q, then (once the Qg conversion has read it) this record's V;
//   A^T scratch: A for the solve, then the bf16 tiles T and T Diag(Gamma rk);
//   T scratch: fp32 T from the solve, then the staging image of -W, which a
//   bulk copy writes to the record.
namespace prep {
constexpr int CTAS_PER_SM = 3;
constexpr uint32_t OFF_KQ = 0;          // bf16 [Kb0 | Qb0 | Kb1 | Qb1] (TMA); V lands in the Q slots
constexpr uint32_t OFF_V = OFF_KQ + 8192;   // V slice sl at OFF_V + 16384 sl (the Q slots)
constexpr uint32_t OFF_A = 32768;       // fp32 A^T, 64 x LD
constexpr uint32_t OFF_T = OFF_A;       // after the solve: bf16 T
constexpr uint32_t OFF_TP = OFF_A + 8192;   // after the solve: bf16 T Diag(Gamma rk)
constexpr uint32_t OFF_TF = OFF_A + 64 * LD * 4;   // fp32 T, 64 x LD
constexpr uint32_t OFF_WS = OFF_TF;     // after the T tiles: fp16 -W image [atom 0 | atom 1], 16 KB
constexpr uint32_t OFF_SC = OFF_TF + 64 * LD * 4;   // scalars: 8 x 64 floats
constexpr uint32_t OFF_BAR = OFF_SC + 8 * 64 * 4;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 64 + 1024;
static_assert(OFF_TP + 8192 <= OFF_TF && 16384 <= 64 * LD * 4, "phase reuse");
static_assert(OFF_A % 1024 == 0 && OFF_TP % 1024 == 0 && OFF_WS % 1024 == 0, "tile alignment");
static_assert(CTAS_PER_SM * (SMEM_BYTES + 1024) <= 233472, "three CTAs per SM");
constexpr uint32_t COL_G = 0;     // M128 x 64: [K; Q] K^T (dead before W)
constexpr uint32_t COL_W = 0;     // M128 x 64: W^T (lane = d_k channel, columns t)
constexpr uint32_t COL_U = 64;    // M128 x 64: U'^T (lane = value column, columns t)
constexpr uint32_t TMEM_COLS = 128;
}  // namespace prep

struct PrepParams {
  int B, T, H, dv, NC;
  bool raw;      // raw-input mode: unit q (and k), gates from their logits
  int c0, ncr;   // the launch prepares chunks [c0, c0 + ncr) of every (b, h)
  const float *beta, *log_g;
  const float *erase_b, *write_w;   // GDN-2 only
  uint8_t *ws;
  float eps, scale;
};

// Launch-local record r (chunk fastest) -> batch, head, chunk.
struct RecIdx {
  int b, h, c;
};
__device__ __forceinline__ RecIdx rec_idx(const PrepParams &p, int r) {
  const int bh = r / p.ncr;
  return {bh / p.H, bh % p.H, p.c0 + (r - bh * p.ncr)};
}
__device__ __forceinline__ size_t rec_index(const PrepParams &p, const RecIdx &x) {
  return (static_cast<size_t>(x.b) * p.H + x.h) * p.NC + x.c;
}

template <int VAR, bool RAW>
__global__ void __launch_bounds__(NTHREADS, prep::CTAS_PER_SM)
    chunk_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const PrepParams p) {
  using namespace prep;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quad = warp & 3, half = warp >> 2;
  const int row = quad * 32 + lane;
  const int NS = p.dv / 64;
  const int total = p.ncr * p.H * p.B;   // records of this launch, chunk index fastest

  uint64_t *bar_q = reinterpret_cast<uint64_t *>(sm + OFF_BAR);   // Q landed
  uint64_t *bar_k = bar_q + 1;          // K landed
  uint64_t *bar_v = bar_q + 2;          // V landed
  uint64_t *bar_mma = bar_q + 3;        // MMA1, then MMA2 (W^T and U'^T)
  uint64_t *bar_drain = bar_q + 4;      // error path only
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_q + 5);
  float *sc_beta = reinterpret_cast<float *>(sm + OFF_SC);
  float *sc_g2 = sc_beta + 64;
  float *sc_wf = sc_g2 + 64;
  float *sc_G = sc_wf + 64;
  float *sc_tmp = sc_G + 64;
  float *sc_rk = sc_tmp + 64;   // raw-input mode: 1 / ||k_t|| (keys normalised here), else 1
  float *sc_qn = sc_rk + 64;    // raw-input mode: 1 / ||q_t||
  float *sc_scan = sc_qn + 64;  // per-warp prefix sums of the log decay
  float *At = reinterpret_cast<float *>(sm + OFF_A);
  float *Tf = reinterpret_cast<float *>(sm + OFF_TF);

  // TMA loads of record r's Q, K and V (thread 0), each on its own barrier:
  // the next record's Q and K once MMA2 has read this record's K and V (V sits
  // in the Q slots), this record's V once its Qg conversion has read Q.
  uint32_t issued = 0, landed = 0;   // thread 0: loads issued / seen landing (q | k << 8 | v << 16)
  auto issue_q = [&](int r) {
    const RecIdx x = rec_idx(p, r);
    mbar_expect_tx(bar_q, 2 * 8192);
    tma_load_4d(sm + OFF_KQ + 8192, &tm_q, bar_q, 0, x.h, x.c * C, x.b);
    tma_load_4d(sm + OFF_KQ + 24576, &tm_q, bar_q, 64, x.h, x.c * C, x.b);
    issued += 1u;
  };
  auto issue_k = [&](int r) {
    const RecIdx x = rec_idx(p, r);
    mbar_expect_tx(bar_k, 2 * 8192);
    tma_load_4d(sm + OFF_KQ + 0, &tm_k, bar_k, 0, x.h, x.c * C, x.b);
    tma_load_4d(sm + OFF_KQ + 16384, &tm_k, bar_k, 64, x.h, x.c * C, x.b);
    issued += 1u << 8;
  };
  auto issue_v = [&](int r) {
    const RecIdx x = rec_idx(p, r);
    mbar_expect_tx(bar_v, NS * 8192);
    for (int sl = 0; sl < NS; ++sl) tma_load_4d(sm + OFF_V + sl * 16384, &tm_v, bar_v, 64 * sl, x.h, x.c * C, x.b);
    issued += 1u << 16;
  };
  // log decay and beta of token `tid` of record r (threads 0-63)
  auto load_gates = [&](int r, float &lg, float &bt) {
    const RecIdx x = rec_idx(p, r);
    const int c = x.c, h = x.h, b = x.b;
    const int t = c * C + tid;
    lg = 0.f;
    bt = 0.f;
    if (t < p.T) {
      const size_t th = (static_cast<size_t>(b) * p.T + t) * p.H + h;
      if constexpr (scalar_decay(VAR)) lg = __ldg(p.log_g + th);
      bt = __ldg(p.beta + th);
      if constexpr (RAW) {
        if constexpr (scalar_decay(VAR)) lg = raw_log_decay(lg);
        bt = raw_gate(bt);
      }
    }
  };

  if (warp == 0) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar_q, 1);
    mbar_init(bar_k, 1);
    mbar_init(bar_v, 1);
    mbar_init(bar_mma, 1);
    mbar_init(bar_drain, 1);
    fence_mbar_init();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    if (static_cast<int>(blockIdx.x) < total) {
      issue_q(blockIdx.x);
      issue_k(blockIdx.x);
    }
  }
  if (tid < 64) sc_rk[tid] = 1.f;   // rewritten per record only where keys are normalised here
  float lg_next = 0.f, bt_next = 0.f;
  if (tid < 64 && static_cast<int>(blockIdx.x) < total) load_gates(blockIdx.x, lg_next, bt_next);
  // every CTA of this persistent grid is resident from the start, so the carry
  // kernel may launch now: its CTAs take SMs as preparation CTAs finish and
  // wait for this grid to complete before they read a record
  griddep_launch_dependents();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
  const uint32_t kq = smem_u32(sm + OFF_KQ);
  uint32_t mma_phase = 0;
  int bad = 0;
  float wmax = 0.f;

  // Persistent over records: each of the next record's loads is issued as soon
  // as this record no longer reads its buffer.
  for (int r = blockIdx.x; r < total; r += gridDim.x) {
    const uint32_t ph = ((r - blockIdx.x) / gridDim.x) & 1;   // phase of the input and U' barriers
    const bool more = r + static_cast<int>(gridDim.x) < total;
    uint8_t *rec = p.ws + rec_index(p, rec_idx(p, r)) * rec_bytes(NS);
    // gates (warps 0 and 1, meeting at a 64-thread barrier): beta_t, cumulative
    // log2 decay, Gamma_t; and, where beta is the column coefficient (no
    // Kaczmarz step, no keys normalised here), the column factors of A, P, Kt
    constexpr bool diag_pass = VAR == kKLA || RAW;   // the coefficient needs ||k_t||^2 from MMA1
    if (tid < 64) {
      float x = lg_next * LOG2E;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      sc_scan[tid] = x;
      sc_beta[tid] = bt_next;
      if (more) load_gates(r + gridDim.x, lg_next, bt_next);
      named_bar_sync(2, 64);
      const float g2 = sc_scan[tid] + (tid >= 32 ? sc_scan[31] : 0.f);
      sc_g2[tid] = g2;
      sc_G[tid] = ex2(g2);
      if constexpr (!diag_pass) {
        named_bar_sync(2, 64);
        sc_wf[tid] = sc_beta[tid] * ex2(sc_g2[63] - g2);
        sc_tmp[tid] = sc_beta[tid] * ex2(sc_g2[tid & 32] - g2);
      }
    }
    if (!mbar_wait(bar_q, ph) || !mbar_wait(bar_k, ph)) bad = 1;
    else if (tid == 0) landed += 1u | (1u << 8);
    bad = __syncthreads_or(bad);
    if (bad) break;
    if constexpr (RAW) tile_row_inv_norms(sm + OFF_KQ + 8192, 16384, sc_qn, tid);   // read after MMA1's barrier

    // MMA1: [K;Q] K^T
    if (!bad && tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t a = kq + (kk >> 2) * 16384 + (kk & 3) * 32;
        mma_ss(tmem + COL_G, sdesc(a, 16, 1024), sdesc(a, 16, 1024), idesc_bf16(128, 64, false, false), kk > 0);
      }
      mma_commit(bar_mma);
    }
    if (!bad && tid == 0 && !mbar_wait(bar_mma, mma_phase)) bad = 1;   // one waiter; the rest sleep in the barrier
    bad = __syncthreads_or(bad);
    mma_phase ^= 1;
    tc_fence_after();

    // A (lanes 0-63) -> A^T scratch; P (lanes 64-127) -> fp16 record tile.  The
    // column coefficient c_r is beta_r, or for KLA the Kaczmarz step
    // eta_r / (||k_r||^2 + eps), ||k_r||^2 being the diagonal of K K^T.  In the
    // raw-input mode the recurrence sees the unit keys khat = k / ||k|| (not
    // for KLA): the Gram entries of the raw keys are scaled by 1/||k_t|| (row
    // factor rk_t) and 1/||k_r|| (in c_r = beta_r / ||k_r||), and W and Kt take
    // the same factors, so no separate normalisation pass is needed.
    if (!bad) {
      float g[32];
      tmem_ld32(tmem + lane_base + COL_G + 32 * half, g);
      const int t = row & 63;
      const int r0 = 32 * half;
      if constexpr (diag_pass) {
        if (quad < 2 && (t >> 5) == half) {
          float kk = 0.f;
#pragma unroll
          for (int r = 0; r < 32; ++r) kk = (r0 + r == t) ? g[r] : kk;
          const float bt = sc_beta[t];
          if constexpr (VAR == kKLA) {
            sc_beta[t] = (bt == 0.f) ? 0.f : bt / (kk + p.eps);   // Kaczmarz step
          } else {
            const float rk = kk > 0.f ? rsqrtf(kk) : 0.f;
            sc_beta[t] = bt * rk;
            sc_rk[t] = rk;
          }
        }
        __syncthreads();
        if (tid < 64) {
          sc_wf[tid] = sc_beta[tid] * ex2(sc_g2[63] - sc_g2[tid]);
          sc_tmp[tid] = sc_beta[tid] * ex2(sc_g2[tid & 32] - sc_g2[tid]);
        }
        __syncthreads();
      }
      const bool fast = sc_g2[0] - sc_g2[63] < 120.f;
      const float g2t = sc_g2[t];
      // column factor of entry (t, r0 + r): c_r Gamma_t / Gamma_r, factored
      // through the block's first column where the decay range allows it
      const float rowf = (t >= r0) ? ex2(g2t - sc_g2[r0]) : 0.f;
      auto emit = [&](auto fac) {
        if (quad < 2) {
          const float rkt = sc_rk[t];
#pragma unroll
          for (int r = 0; r < 32; ++r) At[(r0 + r) * LD + t] = (r0 + r < t) ? tf32r(rkt * g[r] * fac(r)) : 0.f;
        } else {
          const float qs = RAW ? p.scale * sc_qn[t] : p.scale;
#pragma unroll
          for (int r = 0; r < 32; ++r) g[r] = (r0 + r <= t) ? qs * g[r] * fac(r) : 0.f;
#pragma unroll
          for (int j = 0; j < 4; ++j) st_chunk_f16(rec + REC_P + sw128(t, 4 * half + j), g + 8 * j);
        }
      };
      if (fast) emit([&](int r) { return sc_tmp[r0 + r] * rowf; });
      else emit([&](int r) { return sc_beta[r0 + r] * ex2(g2t - sc_g2[r0 + r]); });
    }
    tc_fence_before();   // the tensor-memory reads above, ordered by the barrier after the conversion

    // Gamma_C, and the fp16 copies Qg = Diag(scale Gamma) Q and Kt = Diag(w) K
    // (2048 sixteen-byte chunks in the swizzled image of the bf16 tiles)
    if (tid == 0) *reinterpret_cast<float4 *>(rec + rec_sc(NS)) = make_float4(sc_G[63], 0.f, 0.f, 0.f);
    float qkmax = 0.f;
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      const int u = it * NTHREADS + tid;
      const int isq = u >> 10, kb = (u >> 9) & 1, r = (u >> 3) & 63, j = u & 7;
      const uint32_t off = sw128(r, j);
      float x[8];
      unpack8(*reinterpret_cast<const uint4 *>(sm + OFF_KQ + kb * 16384 + isq * 8192 + off), x);
      const float f = isq ? p.scale * sc_G[r] * (RAW ? sc_qn[r] : 1.f) : sc_wf[r];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        x[e] *= f;
        qkmax = fmaxf(qkmax, fabsf(x[e]));
      }
      st_chunk_f16(rec + (isq ? REC_WQ + kb * 16384 + 8192 : REC_K + kb * 8192) + off, x);
    }
    // Q is consumed: this record's V lands in its slots during the solve.  The
    // previous record's -W bulk copy must have read the T scratch before the
    // solve writes it.
    if (tid == 0) bulk_wait_read();
    __syncthreads();
    if (tid == 0) issue_v(r);
    if (NS == 1) {   // d_v = 64: the transposed U' product reads a 128-row V operand
      for (int i = tid; i < 512; i += NTHREADS)
        reinterpret_cast<uint4 *>(sm + OFF_V + 16384)[i] = make_uint4(0u, 0u, 0u, 0u);
    }

    // T = (I + A)^{-1}; T (for U' = T V) and T Diag(Gamma rk) (for W = T Diag(Gamma) K,
    // the keys normalised in the raw-input mode) as bf16 tiles
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
        tg[e] = tv[e] * sc_G[n0 + e] * sc_rk[n0 + e];
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        st_chunk_bf16(sm + OFF_T + sw128(m, 2 * (tid & 3) + j), tv + 8 * j);
        st_chunk_bf16(sm + OFF_TP + sw128(m, 2 * (tid & 3) + j), tg + 8 * j);
      }
    }
    fence_async_smem();
    __syncthreads();

    // MMA2: W^T = K^T (T Diag(Gamma rk))^T (M128 over d_k, N64) and U'^T = V^T T^T
    // (M128 over d_v, N64), both with the d_k / d_v operand MN-major
    if (tid == 0) {
      if (!mbar_wait(bar_v, ph)) {
        bad = 1;
      } else {
        landed += 1u << 16;
        tc_fence_after();
        const uint32_t tp = smem_u32(sm + OFF_TP), tt = smem_u32(sm + OFF_T), vt = smem_u32(sm + OFF_V);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss(tmem + COL_W, sdesc(kq + kk * 2048, 16384, 1024), sdesc(tp + kk * 32, 16, 1024),
                 idesc_bf16(128, 64, true, false), kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss(tmem + COL_U, sdesc(vt + kk * 2048, 16384, 1024), sdesc(tt + kk * 32, 16, 1024),
                 idesc_bf16(128, 64, true, false), kk > 0);
        mma_commit(bar_mma);
      }
    }
    if (!bad && tid == 0 && !mbar_wait(bar_mma, mma_phase)) bad = 1;   // one waiter; the rest sleep in the barrier
    bad = __syncthreads_or(bad);
    mma_phase ^= 1;
    if (bad) break;
    tc_fence_after();
    // K and V (in the Q slots) are consumed: the next record's Q and K land during the epilogues
    if (tid == 0 && more) {
      issue_q(r + gridDim.x);
      issue_k(r + gridDim.x);
    }

    // -W^T (lane = d_k channel i, tokens 32 half ..) -> the staging image of the
    // record's -W tile (rows t, 64-channel atoms, 128-byte swizzle); U'^T (lane v =
    // value column, columns t) -> fp16 record tile
    wmax = fmaxf(wmax, qkmax);
    {
      float w[32];
      tmem_ld32(tmem + lane_base + COL_W + 32 * half, w);
      uint8_t *ws = sm + OFF_WS + (row >> 6) * 8192 + (row & 7) * 2;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        wmax = fmaxf(wmax, fabsf(w[e]));
        *reinterpret_cast<__half *>(ws + sw128(32 * half + e, (row & 63) >> 3)) = __float2half_rn(-w[e]);
      }
      tmem_ld32(tmem + lane_base + COL_U + 32 * half, w);
      if (row < p.dv) {
#pragma unroll
        for (int e = 0; e < 32; ++e) wmax = fmaxf(wmax, fabsf(w[e]));
#pragma unroll
        for (int j = 0; j < 4; ++j) st_chunk_f16(rec + REC_U + sw128(row, 4 * half + j), w + 8 * j);
      }
    }
    // tensor-memory reads done before the next record's MMA1; the -W image to the record
    fence_async_smem();
    tc_fence_before();
    bad = __syncthreads_or(bad);
    if (bad) break;
    if (tid == 0) {
      bulk_store(rec + REC_WQ, sm + OFF_WS, 8192);
      bulk_store(rec + REC_WQ + 16384, sm + OFF_WS + 8192, 8192);
      bulk_commit();
    }
  }

  if (bad && tid == 0) {
    // a wait gave up: report it, then let the MMAs and loads in flight
    // finish (each wait again bounded) before tensor memory is released
    atomicOr(&g_gdr_split_error, 1);
    mma_commit(bar_drain);
    mbar_wait(bar_drain, 0);
    uint64_t *bars[3] = {bar_q, bar_k, bar_v};
    for (int i = 0; i < 3; ++i) {
      const uint32_t n_issued = (issued >> (8 * i)) & 0xffu, n_landed = (landed >> (8 * i)) & 0xffu;
      if (n_issued != n_landed) mbar_wait(bars[i], n_landed & 1u);
    }
  }
  if (tid == 0) bulk_wait_all();   // the last record's -W copy
  if (wmax > F16_SAFE) atomicOr(&g_gdr_split_error, 2);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
  // Launched as a programmatic dependent of a carry grid (the pipelined
  // sweep), this grid completes only after that carry, so whatever is ordered
  // after it is ordered after both.  Without such a launch this returns at once.
  griddep_wait();
}

// ------------------------------------------------------------------ preparation kernel, channel decay
// KDA ("Gated DeltaNet-2", what is new / technical core: a decay vector g_t in
// R^{dk} on the state rows).  The chunk-local products take the decay inside,
// factored around the chunk's middle token m with G_t[i] = e^{gamma_t[i] - gamma_m[i]}:
//     A_tr = beta_r [K o G; .](K o G^-1)^T,  P_tr = beta_r [.; scale Q o G](K o G^-1)^T,
//     W = T (K o e^gamma),  Qg = scale Q o e^gamma,  Kt_r = beta_r k_r o e^{gamma_C - gamma_r},
// and the state decays row by row with e^{gamma_C}.  The factors G span beyond
// fp16's range and one bf16 rounding of them leaves ~2.5% of the output RMS,
// so MMA1 takes tf32 operands (fp32 range, an 11-bit significand), in two
// 64-channel halves.  The record is the scalar-decay record with Gamma_C a
// vector of d_k values.
namespace prepc {
constexpr float SPAN_SAFE = 120.f;      // |gamma_t - gamma_m| (log2 units) the fp32 factors carry
constexpr uint32_t OFF_KQ = 0;          // bf16 [Kb0 | Qb0 | Kb1 | Qb1] (TMA)
constexpr uint32_t OFF_V = 32768;       // bf16 V, one 8 KB box per value slice (TMA)
constexpr uint32_t OFF_LG = 49152;      // fp32 [64][128]: log g (TMA), then G
constexpr uint32_t OFF_R = 81920;       // phase-shared region
constexpr uint32_t OFF_XF = OFF_R;              // (c) tf32 [K o G; Q o G], 128 rows x 2 atoms of 32 channels
constexpr uint32_t OFF_YF = OFF_R + 32768;      // (c) tf32 K o G^-1, 64 rows x 2 atoms
constexpr uint32_t OFF_KG = OFF_R + 49152;      // (c..f) bf16 K o e^gamma [Kb0 | Kb1]
constexpr uint32_t OFF_A = OFF_R;               // (d, e) fp32 A^T, 64 x LD
constexpr uint32_t OFF_TF = OFF_R + 18432;      // (e) fp32 T, 64 x LD
constexpr uint32_t OFF_T = OFF_R + 36864;       // (e, f) bf16 T
constexpr uint32_t OFF_SC = OFF_R + 65536;      // beta [64], e^{gamma_m} [128], scratch [128], 1/||k|| [64], 1/||q|| [64]
constexpr uint32_t OFF_BAR = OFF_SC + 448 * 4;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 64 + 1024;
static_assert(OFF_TF + 64 * LD * 4 <= OFF_T && OFF_T + 8192 <= OFF_KG, "phase region layout");
static_assert(OFF_XF % 1024 == 0 && OFF_YF % 1024 == 0 && OFF_KG % 1024 == 0 && OFF_T % 1024 == 0, "alignment");
constexpr uint32_t COL_G = 0;     // M128 x 64
constexpr uint32_t COL_W = 64;    // M64 x 128
constexpr uint32_t COL_U = 192;   // M128 x 64: U'^T
constexpr uint32_t TMEM_COLS = 256;
}  // namespace prepc

template <bool RAW>
__global__ void __launch_bounds__(NTHREADS, 1)
    chunk_prep_chan_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                           const PrepParams p) {
  using namespace prepc;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quad = warp & 3, half = warp >> 2;
  const int row = quad * 32 + lane;
  const int NS = p.dv / 64;
  const int total = p.ncr * p.H * p.B;   // records of this launch, chunk index fastest

  uint64_t *bar_kq = reinterpret_cast<uint64_t *>(sm + OFF_BAR);   // K, Q landed
  uint64_t *bar_lg = bar_kq + 1;                                      // log g landed
  uint64_t *bar_mma = bar_kq + 2;
  uint64_t *bar_v = bar_kq + 3;                                       // V landed
  uint64_t *bar_drain = bar_kq + 4;                                   // error path only
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_kq + 5);
  float *sc_beta = reinterpret_cast<float *>(sm + OFF_SC);   // [64]
  float *sc_em = sc_beta + 64;                               // [128] e^{gamma_m} per channel
  float *sc_tmp = sc_em + 128;                               // [128]
  float *sc_kn = sc_tmp + 128;                               // [64] raw-input mode: 1 / ||k_t||
  float *sc_qn = sc_kn + 64;                                 // [64] raw-input mode: 1 / ||q_t||
  float *Gr = reinterpret_cast<float *>(sm + OFF_LG);        // [64][128]
  float *At = reinterpret_cast<float *>(sm + OFF_A);
  float *Tf = reinterpret_cast<float *>(sm + OFF_TF);
  uint8_t *kq_ptr = sm + OFF_KQ;

  // loads of record r (thread 0): log g and K, Q first, V once MMA2 no longer reads it
  uint32_t issued = 0, landed = 0;   // thread 0: loads issued / seen landing (lg | kq << 8 | v << 16)
  auto issue_kq_lg = [&](int r) {
    const RecIdx x = rec_idx(p, r);
    const int c = x.c, h = x.h, b = x.b;
    mbar_expect_tx(bar_lg, 64 * DK * 4);
    tma_load_4d(sm + OFF_LG, &tm_g, bar_lg, 0, h, c * C, b);
    mbar_expect_tx(bar_kq, 4 * 8192);
    tma_load_4d(sm + OFF_KQ + 0, &tm_k, bar_kq, 0, h, c * C, b);
    tma_load_4d(sm + OFF_KQ + 8192, &tm_q, bar_kq, 0, h, c * C, b);
    tma_load_4d(sm + OFF_KQ + 16384, &tm_k, bar_kq, 64, h, c * C, b);
    tma_load_4d(sm + OFF_KQ + 24576, &tm_q, bar_kq, 64, h, c * C, b);
    issued += 1u | (1u << 8);
  };
  auto issue_v = [&](int r) {
    const RecIdx x = rec_idx(p, r);
    const int c = x.c, h = x.h, b = x.b;
    mbar_expect_tx(bar_v, NS * 8192);
    for (int sl = 0; sl < NS; ++sl) tma_load_4d(sm + OFF_V + sl * 8192, &tm_v, bar_v, 64 * sl, h, c * C, b);
    issued += 1u << 16;
  };
  auto load_beta = [&](int r) -> float {   // threads 0-63
    const RecIdx x = rec_idx(p, r);
    const int c = x.c, h = x.h, b = x.b;
    const int t = c * C + tid;
    if (t >= p.T) return 0.f;
    const float bt = __ldg(p.beta + (static_cast<size_t>(b) * p.T + t) * p.H + h);
    return RAW ? raw_gate(bt) : bt;
  };

  if (warp == 0) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar_kq, 1);
    mbar_init(bar_lg, 1);
    mbar_init(bar_mma, 1);
    mbar_init(bar_v, 1);
    mbar_init(bar_drain, 1);
    fence_mbar_init();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_g);
    if (static_cast<int>(blockIdx.x) < total) {
      issue_kq_lg(blockIdx.x);
      issue_v(blockIdx.x);
    }
  }
  if (NS == 1) {   // d_v = 64: the transposed U' product reads a 128-row V operand
    for (int i = tid; i < 512; i += NTHREADS)
      reinterpret_cast<uint4 *>(sm + OFF_V + 8192)[i] = make_uint4(0u, 0u, 0u, 0u);
  }
  float bt_next = (tid < 64 && static_cast<int>(blockIdx.x) < total) ? load_beta(blockIdx.x) : 0.f;
  griddep_launch_dependents();   // persistent grid: the carry may launch now (see chunk_prep_kernel)
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
  int bad = 0, range = 0;
  uint32_t mma_phase = 0;
  float wmax_all = 0.f;

  // Persistent over records (one CTA per SM): the next record's log g, K and Q
  // are loaded once MMA1 has consumed this record's, its V once MMA2 has.
  for (int r = blockIdx.x; r < total; r += gridDim.x) {
    const uint32_t ph = ((r - blockIdx.x) / gridDim.x) & 1;   // phase of the input barriers
    uint8_t *rec = p.ws + rec_index(p, rec_idx(p, r)) * rec_bytes_chan(NS);
    if (tid < 64) {
      sc_beta[tid] = bt_next;
      if (r + static_cast<int>(gridDim.x) < total) bt_next = load_beta(r + gridDim.x);
    }
    __syncthreads();

    // (a) per-channel cumulative log2 decay in place, then G = 2^(gamma - gamma_m), m = token 31
    if (!mbar_wait(bar_lg, ph)) bad = 1;
    else if (tid == 0) landed += 1u;
    bad = __syncthreads_or(bad);
    if (!bad) {
      const int ch = tid & 127, hh = tid >> 7;
      const int valid = p.T - rec_idx(p, r).c * C;   // tokens of this chunk inside the sequence
      float run = 0.f;
#pragma unroll 8
      for (int t = 32 * hh; t < 32 * hh + 32; ++t) {
        // raw-input mode: -softplus of the logit; past the sequence's end the
        // padding decays nothing (a zero logit would decay by one half)
        const float lg = Gr[t * DK + ch];
        run += (RAW ? (t < valid ? raw_log_decay(lg) : 0.f) : lg) * LOG2E;
        Gr[t * DK + ch] = run;
      }
      if (hh == 0) sc_tmp[ch] = run;   // gamma at token 31
      __syncthreads();
      const float gm = sc_tmp[ch];
      if (hh == 0) sc_em[ch] = ex2(gm);
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
    __syncthreads();
    // Gamma_C per channel into the record
    if (!bad && tid < DK) reinterpret_cast<float *>(rec + rec_sc(NS))[tid] = Gr[63 * DK + tid] * sc_em[tid];

    // (b) K and Q landed?
    if (!mbar_wait(bar_kq, ph)) bad = 1;
    else if (tid == 0) landed += 1u << 8;
    bad = __syncthreads_or(bad);
    if (RAW && !bad) {   // unit q and k
      tile_row_inv_norms(kq_ptr, 16384, sc_kn, tid);
      tile_row_inv_norms(kq_ptr + 8192, 16384, sc_qn, tid);
      __syncthreads();
    }
    float qkmax = 0.f;

    // (c) MMA1 in two 64-channel halves; the record's Kt and Qg, and K o e^gamma for MMA2
#pragma unroll 1
    for (int hp = 0; hp < 2 && !bad; ++hp) {
#pragma unroll
      for (int it = 0; it < 4; ++it) {
        const int u = it * NTHREADS + tid;      // 1024 units: (t, 4-channel group j4)
        const int t = u >> 4, j4 = u & 15;
        const int ch0 = 64 * hp + 4 * j4;
        const uint32_t bf = sw128(t, j4 >> 1) + 8 * (j4 & 1);   // 4 values of a 16-bit tile row
        float kx[4], qx[4];
        unpack4(*reinterpret_cast<const uint2 *>(kq_ptr + hp * 16384 + bf), kx);
        unpack4(*reinterpret_cast<const uint2 *>(kq_ptr + hp * 16384 + 8192 + bf), qx);
        if constexpr (RAW) {
          const float kn = sc_kn[t], qn = sc_qn[t];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            kx[e] *= kn;
            qx[e] *= qn;
          }
        }
        const float4 g4 = *reinterpret_cast<const float4 *>(Gr + t * DK + ch0);
        const float4 h4 = *reinterpret_cast<const float4 *>(Gr + 63 * DK + ch0);
        const float4 m4 = *reinterpret_cast<const float4 *>(sc_em + ch0);
        const float g[4] = {g4.x, g4.y, g4.z, g4.w}, g63[4] = {h4.x, h4.y, h4.z, h4.w};
        const float em[4] = {m4.x, m4.y, m4.z, m4.w};
        const float bt = sc_beta[t];
        float kg[4], qg[4], ig[4], kt[4], qo[4], ke[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float inv = rcp_approx(g[e]);
          kg[e] = tf32r(kx[e] * g[e]);
          qg[e] = tf32r(p.scale * qx[e] * g[e]);
          ig[e] = tf32r(kx[e] * inv);
          kt[e] = bt * kx[e] * (g63[e] * inv);
          qo[e] = p.scale * qx[e] * g[e] * em[e];
          ke[e] = kx[e] * g[e] * em[e];
          qkmax = fmaxf(qkmax, fmaxf(fabsf(kt[e]), fabsf(qo[e])));
        }
        const uint32_t xa = (j4 >> 3) * 16384, ya = (j4 >> 3) * 8192;
        *reinterpret_cast<float4 *>(sm + OFF_XF + xa + sw128(t, j4 & 7)) = make_float4(kg[0], kg[1], kg[2], kg[3]);
        *reinterpret_cast<float4 *>(sm + OFF_XF + xa + sw128(64 + t, j4 & 7)) = make_float4(qg[0], qg[1], qg[2], qg[3]);
        *reinterpret_cast<float4 *>(sm + OFF_YF + ya + sw128(t, j4 & 7)) = make_float4(ig[0], ig[1], ig[2], ig[3]);
        *reinterpret_cast<uint2 *>(rec + REC_K + hp * 8192 + bf) =
            make_uint2(pack_f16x2(kt[0], kt[1]), pack_f16x2(kt[2], kt[3]));
        *reinterpret_cast<uint2 *>(rec + REC_WQ + hp * 16384 + 8192 + bf) =
            make_uint2(pack_f16x2(qo[0], qo[1]), pack_f16x2(qo[2], qo[3]));
        *reinterpret_cast<uint2 *>(sm + OFF_KG + hp * 8192 + bf) =
            make_uint2(pack_bf16x2(ke[0], ke[1]), pack_bf16x2(ke[2], ke[3]));
      }
      fence_async_smem();
      __syncthreads();
      if (tid == 0) {
        tc_fence_after();
        const uint32_t xf = smem_u32(sm + OFF_XF), yf = smem_u32(sm + OFF_YF);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_tf32(tmem + COL_G, sdesc(xf + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                   sdesc(yf + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024), idesc_tf32(128, 64, false, false),
                   hp + kk > 0);
        mma_commit(bar_mma);
      }
      if (tid == 0 && !mbar_wait(bar_mma, mma_phase)) bad = 1;   // one waiter; the rest sleep in the barrier
      bad = __syncthreads_or(bad);
      mma_phase ^= 1;
      tc_fence_after();
    }

    // log g, K and Q are consumed: the next record's are loaded from here on
    if (!bad && tid == 0 && r + static_cast<int>(gridDim.x) < total) issue_kq_lg(r + gridDim.x);

    // (d) A (lanes 0-63) -> A^T scratch; P (lanes 64-127) -> fp16 record tile
    if (!bad) {
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
        for (int j = 0; j < 4; ++j) st_chunk_f16(rec + REC_P + sw128(t, 4 * half + j), g + 8 * j);
      }
    }
    tc_fence_before();
    __syncthreads();

    // (e) T = (I + A)^{-1} as a bf16 tile
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
      for (int j = 0; j < 2; ++j) st_chunk_bf16(sm + OFF_T + sw128(m, 2 * (tid & 3) + j), tv + 8 * j);
    }
    fence_async_smem();
    __syncthreads();

    // (f) MMA2: W = T (K o e^gamma) (M64 N128); U'^T = V^T T^T (M128 over d_v, N64)
    if (!bad && tid == 0 && !mbar_wait(bar_v, ph)) bad = 1;
    else if (!bad && tid == 0) landed += 1u << 16;
    if (!bad && tid == 0) {
      tc_fence_after();
      const uint32_t tt = smem_u32(sm + OFF_T), kg = smem_u32(sm + OFF_KG), vt = smem_u32(sm + OFF_V);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ss(tmem + COL_W, sdesc(tt + kk * 32, 16, 1024), sdesc(kg + kk * 2048, 8192, 1024),
                 idesc_bf16(64, 128, false, true), kk > 0);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ss(tmem + COL_U, sdesc(vt + kk * 2048, 8192, 1024), sdesc(tt + kk * 32, 16, 1024),
                 idesc_bf16(128, 64, true, false), kk > 0);
      mma_commit(bar_mma);
    }
    if (!bad && tid == 0 && !mbar_wait(bar_mma, mma_phase)) bad = 1;   // one waiter; the rest sleep in the barrier
    bad = __syncthreads_or(bad);
    mma_phase ^= 1;
    tc_fence_after();
    // V is consumed: the next record's is loaded during the epilogue
    if (!bad && tid == 0 && r + static_cast<int>(gridDim.x) < total) issue_v(r + gridDim.x);

    // (g) -W (M64 layout) and U'^T -> fp16 record tiles
    float wmax = qkmax;
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
            st_chunk_f16(rec + REC_WQ + half * 16384 + sw128(quad * 16 + lane, 4 * part + j), w + 8 * j);
        }
      }
      tmem_ld32(tmem + lane_base + COL_U + 32 * half, w);
      if (row < p.dv) {
#pragma unroll
        for (int e = 0; e < 32; ++e) wmax = fmaxf(wmax, fabsf(w[e]));
#pragma unroll
        for (int j = 0; j < 4; ++j) st_chunk_f16(rec + REC_U + sw128(row, 4 * half + j), w + 8 * j);
      }
    }
    wmax_all = fmaxf(wmax_all, wmax);
    // tensor-memory reads done before the next record's MMA1
    tc_fence_before();
    __syncthreads();
    if (bad) break;
  }

  if (bad && tid == 0) {
    // a wait gave up: report it, then let the MMAs and loads in flight finish
    // (each wait again bounded) before tensor memory is released
    atomicOr(&g_gdr_split_error, 1);
    mma_commit(bar_drain);
    mbar_wait(bar_drain, 0);
    uint64_t *bars[3] = {bar_lg, bar_kq, bar_v};
    for (int i = 0; i < 3; ++i) {
      const uint32_t n_issued = (issued >> (8 * i)) & 0xffu, n_landed = (landed >> (8 * i)) & 0xffu;
      if (n_issued != n_landed) mbar_wait(bars[i], n_landed & 1u);
    }
  }
  if (range || wmax_all > F16_SAFE) atomicOr(&g_gdr_split_error, 2);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
  // Launched as a programmatic dependent of a carry grid (the pipelined
  // sweep), this grid completes only after that carry, so whatever is ordered
  // after it is ordered after both.  Without such a launch this returns at once.
  griddep_wait();
}

// ------------------------------------------------------------------ preparation kernel, GDN-2
// GDN-2 ("Gated DeltaNet-2", technical core, read as in the header of gdr.h):
// channel decay, erase vector a_t = b_t o k_t, write vector c_t = w_t o k_t.
// With d_t = c_t - a_t the chunk form keeps the residual of the scalar
// kernels (an exact rearrangement of the per-token recurrence):
//     A = Gram(K, a), A^d = Gram(K, d) (strictly lower), P^a, P^d = Gram(scale Q, .) (lower),
//     T = (I + A)^{-1},  R = T (I - A^d),  W = T (K o e^gamma),  U' = R V,  E = U' - W S0
//     O = (scale Q o e^gamma) S0 + P^a E + P^d V
//     S_C = e^{gamma_C} o S0 + At^T E + Dt^T V,   At, Dt rows a_r, d_r o e^{gamma_C - gamma_r}
// where Gram(X, Y)_tr = sum_i x_t[i] y_r[i] e^{gamma_t[i] - gamma_r[i]}, factored
// around the middle token as for KDA and computed as one tf32 product
// [K o G; scale Q o G] [a o G^-1; d o G^-1]^T.  The record is the channel-decay
// record (At in the Kt slot, P^a in the P slot) followed by the two terms
// that do not involve the state, (P^d V)^T and (Dt^T V)^T, which the carry
// adds to the output and to the state.
namespace prepg {
constexpr float SPAN_SAFE = 120.f;
constexpr uint32_t OFF_KQ = 0;          // bf16 [Kb0 | Qb0 | Kb1 | Qb1] (TMA)
constexpr uint32_t OFF_V = 32768;       // V boxes: bf16 (TMA), fp16 from (e) on
constexpr uint32_t OFF_LG = 49152;      // fp32 [64][128]: log g (TMA), then G
constexpr uint32_t OFF_R = 81920;       // phase-shared region
constexpr uint32_t OFF_XF = OFF_R;              // (c) tf32 [K o G; Q o G], 2 atoms x 128 rows
constexpr uint32_t OFF_YF = OFF_R + 32768;      // (c) tf32 [a o G^-1; d o G^-1], 2 atoms x 128 rows
constexpr uint32_t OFF_A = OFF_R;               // (d, e) fp32 A^T
constexpr uint32_t OFF_TF = OFF_R + 18432;      // (e) fp32 T
constexpr uint32_t OFF_T = OFF_R + 36864;       // fp16 T, rows t
constexpr uint32_t OFF_IAD = OFF_R + 45056;     // fp16 I - A^d, rows r (MN-major operand)
constexpr uint32_t OFF_PD = OFF_R + 53248;      // fp16 P^d, rows t
constexpr uint32_t OFF_RT = OFF_R + 61440;      // fp16 R, rows t
constexpr uint32_t OFF_KG = OFF_R + 69632;      // (c..f) fp16 K o e^gamma [Kb0 | Kb1]
constexpr uint32_t OFF_DT = OFF_R + 86016;      // (c..f) fp16 Dt [b0 | b1], rows r (MN-major operand)
constexpr uint32_t OFF_SC = OFF_R + 102400;     // e^{gamma_m} [128], scratch [128], 1/||k|| [64], 1/||q|| [64]
constexpr uint32_t OFF_BAR = OFF_SC + 384 * 4;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 64 + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(OFF_TF + 64 * LD * 4 <= OFF_T && OFF_YF + 32768 <= OFF_KG, "phase region layout");
static_assert((OFF_T | OFF_IAD | OFF_PD | OFF_RT | OFF_KG | OFF_DT | OFF_XF | OFF_YF) % 1024 == 0, "alignment");
constexpr uint32_t COL_G = 0;     // (c, d) M128 x 128: [A | A^d ; P^a | P^d]
constexpr uint32_t COL_SD = 0;    // (f, g) M128 x 128: (Dt^T V)^T
constexpr uint32_t COL_R = 128;   // M64 x 64
constexpr uint32_t COL_W = 192;   // M64 x 128
constexpr uint32_t COL_U = 320;   // M128 x 64: U'^T
constexpr uint32_t COL_OD = 384;  // M128 x 64: (P^d V)^T
constexpr uint32_t TMEM_COLS = 512;
}  // namespace prepg

template <bool RAW>
__global__ void __launch_bounds__(NTHREADS, 1)
    chunk_prep_gdn2_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                           const PrepParams p) {
  using namespace prepg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quad = warp & 3, half = warp >> 2;
  const int row = quad * 32 + lane;
  const int NS = p.dv / 64;
  const int total = p.ncr * p.H * p.B;   // records of this launch, chunk index fastest

  uint64_t *bar_kq = reinterpret_cast<uint64_t *>(sm + OFF_BAR);   // K, Q landed
  uint64_t *bar_lg = bar_kq + 1;                                      // log g landed
  uint64_t *bar_mma = bar_kq + 2;
  uint64_t *bar_v = bar_kq + 3;                                       // V landed
  uint64_t *bar_drain = bar_kq + 4;                                   // error path only
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_kq + 5);
  float *sc_em = reinterpret_cast<float *>(sm + OFF_SC);     // [128] e^{gamma_m} per channel
  float *sc_tmp = sc_em + 128;                               // [128]
  float *sc_kn = sc_tmp + 128;                               // [64] raw-input mode: 1 / ||k_t||
  float *sc_qn = sc_kn + 64;                                 // [64] raw-input mode: 1 / ||q_t||
  float *Gr = reinterpret_cast<float *>(sm + OFF_LG);        // [64][128]
  float *At = reinterpret_cast<float *>(sm + OFF_A);
  float *Tf = reinterpret_cast<float *>(sm + OFF_TF);
  uint8_t *kq_ptr = sm + OFF_KQ;

  // loads of record r (thread 0): log g and K, Q first, V once the last product no longer reads it
  uint32_t issued = 0, landed = 0;   // thread 0: loads issued / seen landing (lg | kq << 8 | v << 16)
  auto issue_kq_lg = [&](int r) {
    const RecIdx x = rec_idx(p, r);
    mbar_expect_tx(bar_lg, 64 * DK * 4);
    tma_load_4d(sm + OFF_LG, &tm_g, bar_lg, 0, x.h, x.c * C, x.b);
    mbar_expect_tx(bar_kq, 4 * 8192);
    tma_load_4d(sm + OFF_KQ + 0, &tm_k, bar_kq, 0, x.h, x.c * C, x.b);
    tma_load_4d(sm + OFF_KQ + 8192, &tm_q, bar_kq, 0, x.h, x.c * C, x.b);
    tma_load_4d(sm + OFF_KQ + 16384, &tm_k, bar_kq, 64, x.h, x.c * C, x.b);
    tma_load_4d(sm + OFF_KQ + 24576, &tm_q, bar_kq, 64, x.h, x.c * C, x.b);
    issued += 1u | (1u << 8);
  };
  auto issue_v = [&](int r) {
    const RecIdx x = rec_idx(p, r);
    mbar_expect_tx(bar_v, NS * 8192);
    for (int sl = 0; sl < NS; ++sl) tma_load_4d(sm + OFF_V + sl * 8192, &tm_v, bar_v, 64 * sl, x.h, x.c * C, x.b);
    issued += 1u << 16;
  };
  // erase / write gates of the (t, 4-channel) units this thread builds in pass hp
  // of record r, loaded one pass ahead so that no pass waits for global memory
  float4 ebs[2][4], wrs[2][4];
  auto load_gates = [&](int r, int hp) {
    const RecIdx x = rec_idx(p, r);
    const int t0 = x.c * C;
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int t = (it * NTHREADS + tid) >> 4, ch0 = 64 * hp + 4 * (tid & 15);
      ebs[hp][it] = wrs[hp][it] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (t0 + t < p.T) {
        const size_t gi = ((static_cast<size_t>(x.b) * p.T + t0 + t) * p.H + x.h) * DK + ch0;
        ebs[hp][it] = __ldg(reinterpret_cast<const float4 *>(p.erase_b + gi));
        wrs[hp][it] = __ldg(reinterpret_cast<const float4 *>(p.write_w + gi));
        if constexpr (RAW) {
          float4 &e4 = ebs[hp][it], &w4 = wrs[hp][it];
          e4 = make_float4(raw_gate(e4.x), raw_gate(e4.y), raw_gate(e4.z), raw_gate(e4.w));
          w4 = make_float4(raw_gate(w4.x), raw_gate(w4.y), raw_gate(w4.z), raw_gate(w4.w));
        }
      }
    }
  };

  if (warp == 0) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar_kq, 1);
    mbar_init(bar_lg, 1);
    mbar_init(bar_mma, 1);
    mbar_init(bar_v, 1);
    mbar_init(bar_drain, 1);
    fence_mbar_init();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_g);
    if (static_cast<int>(blockIdx.x) < total) {
      issue_kq_lg(blockIdx.x);
      issue_v(blockIdx.x);
    }
  }
  if (NS == 1) {   // d_v = 64: the transposed products read a 128-row V operand
    for (int i = tid; i < 512; i += NTHREADS)
      reinterpret_cast<uint4 *>(sm + OFF_V + 8192)[i] = make_uint4(0u, 0u, 0u, 0u);
  }
  griddep_launch_dependents();   // persistent grid: the carry may launch now (see chunk_prep_kernel)
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
  int bad = 0, range = 0;
  uint32_t mma_phase = 0;
  float wmax_all = 0.f;

  // Persistent over records (one CTA per SM): the next record's log g, K and Q
  // are loaded once MMA1 has consumed this record's, its V once the last
  // product has.
  for (int r = blockIdx.x; r < total; r += gridDim.x) {
    const uint32_t ph = ((r - blockIdx.x) / gridDim.x) & 1;   // phase of the input barriers
    uint8_t *rec = p.ws + rec_index(p, rec_idx(p, r)) * rec_bytes_gdn2(NS);
    uint8_t *rec_od = rec + rec_bytes_chan(NS);          // (P^d V)^T, rows v x 64 t fp16
    uint8_t *rec_sd = rec_od + 8192 * NS;                // (Dt^T V)^T, rows v x 128 i fp16
    load_gates(r, 0);

    // (a) per-channel cumulative log2 decay in place, then G = 2^(gamma - gamma_m), m = token 31
    if (!mbar_wait(bar_lg, ph)) bad = 1;
    else if (tid == 0) landed += 1u;
    bad = __syncthreads_or(bad);
    if (!bad) {
      const int ch = tid & 127, hh = tid >> 7;
      const int valid = p.T - rec_idx(p, r).c * C;   // tokens of this chunk inside the sequence
      float run = 0.f;
#pragma unroll 8
      for (int t = 32 * hh; t < 32 * hh + 32; ++t) {
        // raw-input mode: -softplus of the logit; past the sequence's end the
        // padding decays nothing (a zero logit would decay by one half)
        const float lg = Gr[t * DK + ch];
        run += (RAW ? (t < valid ? raw_log_decay(lg) : 0.f) : lg) * LOG2E;
        Gr[t * DK + ch] = run;
      }
      if (hh == 0) sc_tmp[ch] = run;
      __syncthreads();
      const float gm = sc_tmp[ch];
      if (hh == 0) sc_em[ch] = ex2(gm);
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
    __syncthreads();
    if (!bad && tid < DK) reinterpret_cast<float *>(rec + rec_sc(NS))[tid] = Gr[63 * DK + tid] * sc_em[tid];

    // (b) K and Q landed?
    if (!mbar_wait(bar_kq, ph)) bad = 1;
    else if (tid == 0) landed += 1u << 8;
    bad = __syncthreads_or(bad);
    if (RAW && !bad) {   // unit q and k
      tile_row_inv_norms(kq_ptr, 16384, sc_kn, tid);
      tile_row_inv_norms(kq_ptr + 8192, 16384, sc_qn, tid);
      __syncthreads();
    }
    float qkmax = 0.f;

    // (c) MMA1 in two 64-channel halves; the record's At and Qg; K o e^gamma and Dt for MMA2
#pragma unroll
    for (int hp = 0; hp < 2; ++hp) {
      if (bad) break;
      if (hp == 0) load_gates(r, 1);
#pragma unroll
      for (int it = 0; it < 4; ++it) {
        const int u = it * NTHREADS + tid;      // 1024 units: (t, 4-channel group j4)
        const int t = u >> 4, j4 = u & 15;
        const int ch0 = 64 * hp + 4 * j4;
        const uint32_t bf = sw128(t, j4 >> 1) + 8 * (j4 & 1);
        float kx[4], qx[4];
        unpack4(*reinterpret_cast<const uint2 *>(kq_ptr + hp * 16384 + bf), kx);
        unpack4(*reinterpret_cast<const uint2 *>(kq_ptr + hp * 16384 + 8192 + bf), qx);
        if constexpr (RAW) {
          const float kn = sc_kn[t], qn = sc_qn[t];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            kx[e] *= kn;
            qx[e] *= qn;
          }
        }
        const float4 eb = ebs[hp][it], wr = wrs[hp][it];
        const float4 g4 = *reinterpret_cast<const float4 *>(Gr + t * DK + ch0);
        const float4 h4 = *reinterpret_cast<const float4 *>(Gr + 63 * DK + ch0);
        const float4 m4 = *reinterpret_cast<const float4 *>(sc_em + ch0);
        const float g[4] = {g4.x, g4.y, g4.z, g4.w}, g63[4] = {h4.x, h4.y, h4.z, h4.w};
        const float em[4] = {m4.x, m4.y, m4.z, m4.w};
        const float ebv[4] = {eb.x, eb.y, eb.z, eb.w}, wrv[4] = {wr.x, wr.y, wr.z, wr.w};
        float kg[4], qg[4], af[4], df[4], at[4], dt[4], qo[4], ke[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float inv = rcp_approx(g[e]);
          const float a = ebv[e] * kx[e], d = (wrv[e] - ebv[e]) * kx[e];
          kg[e] = tf32r(kx[e] * g[e]);
          qg[e] = tf32r(p.scale * qx[e] * g[e]);
          af[e] = tf32r(a * inv);
          df[e] = tf32r(d * inv);
          at[e] = a * (g63[e] * inv);
          dt[e] = d * (g63[e] * inv);
          qo[e] = p.scale * qx[e] * g[e] * em[e];
          ke[e] = kx[e] * g[e] * em[e];
          qkmax = fmaxf(qkmax, fmaxf(fabsf(at[e]), fabsf(qo[e])));
        }
        const uint32_t xa = (j4 >> 3) * 16384;
        const uint32_t sw = sw128(t, j4 & 7), sw64 = sw128(64 + t, j4 & 7);
        *reinterpret_cast<float4 *>(sm + OFF_XF + xa + sw) = make_float4(kg[0], kg[1], kg[2], kg[3]);
        *reinterpret_cast<float4 *>(sm + OFF_XF + xa + sw64) = make_float4(qg[0], qg[1], qg[2], qg[3]);
        *reinterpret_cast<float4 *>(sm + OFF_YF + xa + sw) = make_float4(af[0], af[1], af[2], af[3]);
        *reinterpret_cast<float4 *>(sm + OFF_YF + xa + sw64) = make_float4(df[0], df[1], df[2], df[3]);
        *reinterpret_cast<uint2 *>(rec + REC_K + hp * 8192 + bf) =
            make_uint2(pack_f16x2(at[0], at[1]), pack_f16x2(at[2], at[3]));
        *reinterpret_cast<uint2 *>(rec + REC_WQ + hp * 16384 + 8192 + bf) =
            make_uint2(pack_f16x2(qo[0], qo[1]), pack_f16x2(qo[2], qo[3]));
        *reinterpret_cast<uint2 *>(sm + OFF_KG + hp * 8192 + bf) =
            make_uint2(pack_f16x2(ke[0], ke[1]), pack_f16x2(ke[2], ke[3]));
        *reinterpret_cast<uint2 *>(sm + OFF_DT + hp * 8192 + bf) =
            make_uint2(pack_f16x2(dt[0], dt[1]), pack_f16x2(dt[2], dt[3]));
      }
      fence_async_smem();
      __syncthreads();
      if (tid == 0) {
        tc_fence_after();
        const uint32_t xf = smem_u32(sm + OFF_XF), yf = smem_u32(sm + OFF_YF);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_tf32(tmem + COL_G, sdesc(xf + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                   sdesc(yf + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024), idesc_tf32(128, 128, false, false),
                   hp + kk > 0);
        mma_commit(bar_mma);
      }
      if (tid == 0 && !mbar_wait(bar_mma, mma_phase)) bad = 1;   // one waiter; the rest sleep in the barrier
      bad = __syncthreads_or(bad);
      mma_phase ^= 1;
      tc_fence_after();
    }

    // log g, K and Q are consumed: the next record's are loaded from here on
    if (!bad && tid == 0 && r + static_cast<int>(gridDim.x) < total) issue_kq_lg(r + gridDim.x);

    // (d) rows t of K (lanes 0-63): A -> A^T scratch, I - A^d -> fp16 rows; rows t of Q
    // (lanes 64-127): P^a -> fp16 record tile, P^d -> fp16 tile.  Column half `half`
    // selects the a or the d block.
    if (!bad) {
      float g[64];
      tmem_ld64(tmem + lane_base + COL_G + 64 * half, g);
      const int t = row & 63;
      if (quad < 2) {
        if (half == 0) {
#pragma unroll
          for (int r2 = 0; r2 < 64; ++r2) At[r2 * LD + t] = (r2 < t) ? tf32r(g[r2]) : 0.f;
        } else {
#pragma unroll
          for (int r2 = 0; r2 < 64; ++r2) g[r2] = (r2 < t) ? -g[r2] : (r2 == t ? 1.f : 0.f);
#pragma unroll
          for (int j = 0; j < 8; ++j) st_chunk_f16(sm + OFF_IAD + sw128(t, j), g + 8 * j);
        }
      } else {
#pragma unroll
        for (int r2 = 0; r2 < 64; ++r2) g[r2] = (r2 <= t) ? g[r2] : 0.f;
        if (half == 0) {
#pragma unroll
          for (int j = 0; j < 8; ++j) st_chunk_f16(rec + REC_P + sw128(t, j), g + 8 * j);
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) st_chunk_f16(sm + OFF_PD + sw128(t, j), g + 8 * j);
        }
      }
    }
    tc_fence_before();
    __syncthreads();

    // (e) T = (I + A)^{-1} as fp16 rows; then R = T (I - A^d).  The V tile turns
    // fp16 in place (exact from bf16) so that every product of this kernel after
    // MMA1 has fp16 operands: the GDN-2 terms pass more roundings into the state
    // than the other variants' and bf16 there leaves ~2% of the state RMS.
    solve_unit_lower_64(At, Tf, tid, warp, lane);
    float tmax = 0.f;
    {
      const int m = tid >> 2, n0 = (tid & 3) * 16;
      float tv[16];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const float4 f = *reinterpret_cast<const float4 *>(Tf + m * LD + n0 + 4 * q4);
        tv[4 * q4 + 0] = f.x; tv[4 * q4 + 1] = f.y; tv[4 * q4 + 2] = f.z; tv[4 * q4 + 3] = f.w;
      }
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        tv[e] = (n0 + e <= m) ? tv[e] : 0.f;
        tmax = fmaxf(tmax, fabsf(tv[e]));
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) st_chunk_f16(sm + OFF_T + sw128(m, 2 * (tid & 3) + j), tv + 8 * j);
    }
    fence_async_smem();
    __syncthreads();
    if (!bad && tid == 0) {
      tc_fence_after();
      const uint32_t tt = smem_u32(sm + OFF_T), iad = smem_u32(sm + OFF_IAD);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ss(tmem + COL_R, sdesc(tt + kk * 32, 16, 1024), sdesc(iad + kk * 2048, 8192, 1024),
               idesc_f16(64, 64, false, true), kk > 0);
      mma_commit(bar_mma);
    }
    // V landed? then to fp16 in place (the R product does not read it)
    if (!bad && !mbar_wait(bar_v, ph)) bad = 1;
    else if (!bad && tid == 0) landed += 1u << 16;
    bad = __syncthreads_or(bad);
    if (!bad) {
      for (int i = tid; i < NS * 512; i += NTHREADS) {
        uint4 *chunk = reinterpret_cast<uint4 *>(sm + OFF_V) + i;
        float x[8];
        unpack8(*chunk, x);
        st_chunk_f16(reinterpret_cast<uint8_t *>(chunk), x);
      }
    }
    if (!bad && tid == 0 && !mbar_wait(bar_mma, mma_phase)) bad = 1;   // one waiter; the rest sleep in the barrier
    bad = __syncthreads_or(bad);
    mma_phase ^= 1;
    tc_fence_after();
    if (!bad) {   // R (M64 layout: rows 16 quad + lane, lane < 16) -> fp16 rows t
      float w[32];
      tmem_ld32(tmem + lane_base + COL_R + 32 * half, w);
      if (lane < 16) {
#pragma unroll
        for (int e = 0; e < 32; ++e) tmax = fmaxf(tmax, fabsf(w[e]));
#pragma unroll
        for (int j = 0; j < 4; ++j) st_chunk_f16(sm + OFF_RT + sw128(quad * 16 + lane, 4 * half + j), w + 8 * j);
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // (f) W = T (K o e^gamma); U'^T = V^T R^T; (P^d V)^T = V^T P^d^T; (Dt^T V)^T = V^T Dt
    if (!bad && tid == 0) {
      tc_fence_after();
      const uint32_t tt = smem_u32(sm + OFF_T), kg = smem_u32(sm + OFF_KG), vt = smem_u32(sm + OFF_V);
      const uint32_t rt = smem_u32(sm + OFF_RT), pd = smem_u32(sm + OFF_PD), dtt = smem_u32(sm + OFF_DT);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t va = sdesc(vt + kk * 2048, 8192, 1024);
        mma_ss(tmem + COL_W, sdesc(tt + kk * 32, 16, 1024), sdesc(kg + kk * 2048, 8192, 1024),
               idesc_f16(64, 128, false, true), kk > 0);
        mma_ss(tmem + COL_U, va, sdesc(rt + kk * 32, 16, 1024), idesc_f16(128, 64, true, false), kk > 0);
        mma_ss(tmem + COL_OD, va, sdesc(pd + kk * 32, 16, 1024), idesc_f16(128, 64, true, false), kk > 0);
        mma_ss(tmem + COL_SD, va, sdesc(dtt + kk * 2048, 8192, 1024), idesc_f16(128, 128, true, true), kk > 0);
      }
      mma_commit(bar_mma);
    }
    if (!bad && tid == 0 && !mbar_wait(bar_mma, mma_phase)) bad = 1;   // one waiter; the rest sleep in the barrier
    bad = __syncthreads_or(bad);
    mma_phase ^= 1;
    tc_fence_after();
    // V is consumed: the next record's is loaded during the epilogue
    if (!bad && tid == 0 && r + static_cast<int>(gridDim.x) < total) issue_v(r + gridDim.x);

    // (g) -W (M64 layout), U'^T, (P^d V)^T and (Dt^T V)^T -> fp16 record tiles
    float wmax = fmaxf(qkmax, tmax);
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
            st_chunk_f16(rec + REC_WQ + half * 16384 + sw128(quad * 16 + lane, 4 * part + j), w + 8 * j);
        }
      }
      tmem_ld32(tmem + lane_base + COL_U + 32 * half, w);
      if (row < p.dv) {
#pragma unroll
        for (int e = 0; e < 32; ++e) wmax = fmaxf(wmax, fabsf(w[e]));
#pragma unroll
        for (int j = 0; j < 4; ++j) st_chunk_f16(rec + REC_U + sw128(row, 4 * half + j), w + 8 * j);
      }
      tmem_ld32(tmem + lane_base + COL_OD + 32 * half, w);
      if (row < p.dv) {
#pragma unroll
        for (int e = 0; e < 32; ++e) wmax = fmaxf(wmax, fabsf(w[e]));
#pragma unroll
        for (int j = 0; j < 4; ++j) st_chunk_f16(rec_od + row * 128 + half * 64 + 16 * j, w + 8 * j);
      }
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        tmem_ld32(tmem + lane_base + COL_SD + 64 * half + 32 * part, w);
        if (row < p.dv) {
#pragma unroll
          for (int e = 0; e < 32; ++e) wmax = fmaxf(wmax, fabsf(w[e]));
#pragma unroll
          for (int j = 0; j < 4; ++j)
            st_chunk_f16(rec_sd + row * 256 + half * 128 + part * 64 + 16 * j, w + 8 * j);
        }
      }
    }
    wmax_all = fmaxf(wmax_all, wmax);
    // tensor-memory reads done before the next record's MMA1
    tc_fence_before();
    __syncthreads();
    if (bad) break;
  }

  if (bad && tid == 0) {
    // a wait gave up: report it, then let the MMAs and loads in flight finish
    // (each wait again bounded) before tensor memory is released
    atomicOr(&g_gdr_split_error, 1);
    mma_commit(bar_drain);
    mbar_wait(bar_drain, 0);
    uint64_t *bars[3] = {bar_lg, bar_kq, bar_v};
    for (int i = 0; i < 3; ++i) {
      const uint32_t n_issued = (issued >> (8 * i)) & 0xffu, n_landed = (landed >> (8 * i)) & 0xffu;
      if (n_issued != n_landed) mbar_wait(bars[i], n_landed & 1u);
    }
  }
  if (range || wmax_all > F16_SAFE) atomicOr(&g_gdr_split_error, 2);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
  // programmatic dependent of a carry grid (the pipelined sweep): complete
  // only after it (see chunk_prep_chan_kernel)
  griddep_wait();
}

// ------------------------------------------------------------------ carry kernel
// One CTA per (b, h) sweeps the chunks in order, warp-specialised: warp 16
// issues the record copies and the MMAs; compute warp w (0-15) owns value
// column v = 32 (w mod 4) + lane of S^T (its tensor-memory lane) and the
// quarter w / 4 of its d_k range (fp32 registers), of E^T's tokens and of the
// output tokens.  The two sides hand over through mbarriers only:
//     issuer:  Y(c) = S^T [-W; Qg]^T -> bar_e      compute: E^T(c) -> bar_ea
//              dS^T(c), Y_Q += E^T P^T -> bar_s/o           S^T(c) -> bar_sa, bar_sa1
//              record c+2 (after bar_done of c-1)           output rows (c) -> bar_done
// Y is double-buffered so Y(c+1) runs while the output rows of c are written;
// records arrive by bulk copy two chunks ahead of their use.
namespace carry {
constexpr int NSTAGE = 3;
constexpr int NCOMPUTE = 16;
constexpr int NTHREADS_CARRY = (NCOMPUTE + 1) * 32;
constexpr uint32_t STAGE = 74752;        // record image (<= 74240 bytes), 1 KB aligned
constexpr uint32_t OFF_BAR = NSTAGE * STAGE;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(STAGE % 1024 == 0 && STAGE >= rec_bytes(2) && STAGE >= rec_bytes_chan(2), "stage layout");
constexpr uint32_t COL_Y = 0;      // 2 x 128: [(-W S0)^T | (Qg S0)^T + (P E)^T], [v][t]
constexpr uint32_t COL_DS = 256;   // 128: dS^T, [v][i]
constexpr uint32_t COL_SA = 384;   // 64: fp16 S^T, d_k packed two per column (MMA operand)
constexpr uint32_t COL_EA = 448;   // 32: fp16 E^T, tokens packed two per column (MMA operand)
constexpr uint32_t TMEM_COLS = 512;
constexpr long long WAIT_LIMIT = 1ll << 31;   // cycles, about a second
}  // namespace carry

// Segments: a launch holds up to two passes over segments of seg_len chunks,
// counted from chunk c_base.
// CTA (h, b, z) with z < z_split belongs to pass A and sweeps segment z of its
// (b, h): initial state s0 + z s0_seg_stride (zeros if s0 is null, or for
// z > 0 under CARRY_S0_FIRST; the identity under CARRY_IDENTITY), final state
// to s_final + z s_final_seg_stride (only the last segment under
// CARRY_LAST_FINAL).  CTA z >= z_split belongs to pass B: segment
// seg_first_b + (z - z_split) with flags_b, no initial state but the identity
// or zeros, final state to s_final_b + (z - z_split) s_final_b_seg_stride.
enum CarryFlags : int {
  CARRY_IDENTITY = 1,     // start from S = I (d_v = 128): the segment's transition map
  CARRY_NO_VALUES = 2,    // U' and GDN-2's state-free terms taken as zero
  CARRY_NO_OUTPUT = 4,    // write no output rows
  CARRY_LAST_FINAL = 8,   // only the last segment writes s_final
  CARRY_S0_FIRST = 16,    // only segment 0 starts from s0, the others from zero
  CARRY_FAULT_MISSING_COPY = 32,   // host fault injection (see the issuer's prologue)
  CARRY_WRITE_STATES = 64,   // write every chunk's start state to `states` ([B,H,NC,d_k,d_v], fp32)
  CARRY_STATES_F16 = 128,    // ... in fp16 instead: the state as this kernel's MMAs take it
  CARRY_SNAPSHOTS = 256,     // write the state at every interior chunk c_first + c that is a multiple of snap_len
};

struct CarryParams {
  int T, H, dv, NC;
  int seg_len, flags;
  uint32_t rec_bytes;    // bytes per record
  uint32_t copy_bytes;   // leading bytes of a record that go through shared memory
  const uint8_t *ws;
  const float *s0;
  float *s_final;
  size_t s0_seg_stride, s_final_seg_stride;   // elements between segments' states
  size_t s0_bh_stride, s_final_bh_stride;     // elements between (b, h) states (d_k d_v when packed)
  int c_base;                                 // chunk of segment 0's start
  int z_split;                                // CTAs z >= z_split run pass B
  int seg_first_b, flags_b;
  float *s_final_b;
  size_t s_final_b_seg_stride;
  __nv_bfloat16 *o;
  void *states;    // CARRY_WRITE_STATES output, indexed by (b, h, chunk)
  // CARRY_SNAPSHOTS: the state at chunk x = n snap_len goes to snap (pass A) or
  // snap_b (pass B) + (n - 1) snap_stride, packed [B, H, d_k, d_v] within a slot
  int snap_len;
  float *snap, *snap_b;
  size_t snap_stride;
};

// max |x_i| over 16 values as a tree (four levels instead of a chain of 16).
__device__ __forceinline__ float max_abs16(const float *x) {
  float m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = fmaxf(fabsf(x[2 * i]), fabsf(x[2 * i + 1]));
#pragma unroll
  for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
    for (int i = 0; i < w; ++i) m[i] = fmaxf(m[i], m[i + w]);
  return m[0];
}

// Bounded wait: gives up after carry::WAIT_LIMIT cycles (raising `abort`) or
// once another warp has raised `abort`.
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t phase, volatile int *abort) {
  if (mbar_try_wait(bar, phase)) return true;
  const long long start = clock64();
  while (!mbar_try_wait(bar, phase)) {
    if (*abort) return false;
    if (clock64() - start > carry::WAIT_LIMIT) {
      *abort = 1;
      return false;
    }
  }
  return true;
}

// MODE 0: scalar Gamma_C.  MODE 1: Gamma_C a vector of d_k values (channel
// decay).  MODE 2: as 1, plus the record's (P^d V)^T and (Dt^T V)^T terms added
// to the output and to the state (GDN-2); each compute thread loads its share
// of them from the record one chunk ahead.
// 17 warps: one SM sub-partition holds five of them, so 96 registers per thread.
template <int MODE>
__global__ void __launch_bounds__(carry::NTHREADS_CARRY, 1) chunk_carry_kernel(const CarryParams p) {
  constexpr bool CHAN = MODE >= 1;
  using namespace carry;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x, b = blockIdx.y;
  const bool pass_b = static_cast<int>(blockIdx.z) >= p.z_split;
  const int zi = pass_b ? blockIdx.z - p.z_split : blockIdx.z;      // index within the pass
  const int flags = pass_b ? p.flags_b : p.flags;
  const int c_first = p.c_base + (pass_b ? p.seg_first_b + zi : zi) * p.seg_len;   // this CTA's first chunk
  const int NS = p.dv / 64, NC = min(p.seg_len, p.NC - c_first);   // chunks of this CTA
  const bool values = !(flags & CARRY_NO_VALUES);
  // A carry without outputs copies only -W, Kt, U' (unless NO_VALUES) and the decay of
  // each record, and takes neither Qg's half of the Y product nor E^T P^T.
  const bool lite = (flags & CARRY_NO_OUTPUT) != 0;

  uint64_t *bar_full = reinterpret_cast<uint64_t *>(sm + OFF_BAR);   // [NSTAGE] records landed
  uint64_t *bar_e = bar_full + NSTAGE;    // Y(c) done
  uint64_t *bar_s = bar_e + 1;            // dS^T(c) done
  uint64_t *bar_o = bar_e + 2;            // E^T P^T (c) done
  uint64_t *bar_ea = bar_e + 3;           // E^T(c) in tensor memory (16 warps)
  uint64_t *bar_sa = bar_e + 4;           // S^T (scalar decay), or its first half-rows, in tensor memory (16 warps)
  uint64_t *bar_done = bar_e + 5;         // chunk c's Y read and stage released (16 warps)
  uint64_t *bar_drain = bar_e + 6;        // error path only
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_e + 7);
  volatile int *abort = reinterpret_cast<volatile int *>(bar_e + 8);
  uint64_t *bar_sa1 = bar_e + 9;          // S^T's second half-rows in tensor memory (16 warps)

  if (warp == 0) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < NSTAGE; ++i) mbar_init(&bar_full[i], 1);
    mbar_init(bar_e, 1);
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    mbar_init(bar_ea, NCOMPUTE);
    mbar_init(bar_sa, NCOMPUTE);
    mbar_init(bar_sa1, NCOMPUTE);
    mbar_init(bar_done, NCOMPUTE);
    mbar_init(bar_drain, 1);
    *abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t rb = p.rec_bytes;
  // every CTA of this grid holds its SM: a preparation grid launched as this
  // grid's programmatic dependent (the pipelined sweep) may take the others
  griddep_launch_dependents();

  // issuer's view of the record copies: stage has a copy in flight / phase parity to wait for
  uint32_t pend = 0, par = 0;
  float smax = 0.f;
  float S[32];
  const int quad = warp & 3, part = (warp >> 2) & 3;
  const int v = quad * 32 + lane;
  const bool has_v = quad * 32 < p.dv;   // warp-uniform (d_v is 64 or 128)
  const uint32_t lrow = tmem + (static_cast<uint32_t>(quad * 32) << 16);

  if (warp == NCOMPUTE) {
    // ---------------------------------------------------------------- issuer
    if (lane == 0) {
      const uint8_t *recs = p.ws + ((static_cast<size_t>(b) * p.H + h) * p.NC + c_first) * rb;
      auto issue_chunk = [&](int c) {
        const int s = c % NSTAGE;
        const uint8_t *src = recs + static_cast<size_t>(c) * rb;
        uint8_t *dst = sm + s * STAGE;
        if (lite) {   // -W's two atoms, Kt, then U' (unless NO_VALUES) and the decay
          const uint32_t tail = values ? REC_U : rec_sc(NS);
          mbar_expect_tx(&bar_full[s], 32768 + (p.copy_bytes - tail));
          bulk_load(dst + REC_WQ, src + REC_WQ, 8192, &bar_full[s]);
          bulk_load(dst + REC_WQ + 16384, src + REC_WQ + 16384, 8192, &bar_full[s]);
          bulk_load(dst + REC_K, src + REC_K, 16384, &bar_full[s]);
          bulk_load(dst + tail, src + tail, p.copy_bytes - tail, &bar_full[s]);
        } else {
          mbar_expect_tx(&bar_full[s], p.copy_bytes);
          bulk_load(dst, src, p.copy_bytes, &bar_full[s]);
        }
        // MODE 2: the rest of the record, which the compute threads read themselves
        // (without outputs, its state term only)
        if constexpr (MODE == 2) {
          const uint32_t skip = lite ? 8192u * NS : 0u;
          prefetch_l2(src + p.copy_bytes + skip, rb - p.copy_bytes - skip);
        }
        pend |= 1u << s;
      };
      auto wait_full = [&](int c) -> bool {
        const int s = c % NSTAGE;
        if (!wait_or_abort(&bar_full[s], (c / NSTAGE) & 1, abort)) return false;
        pend &= ~(1u << s);
        par ^= 1u << s;
        return true;
      };
      // Y(c) = S^T [-W; Qg]^T over d_k in 16-row steps.  With channel decay (a
      // longer S update) the even steps (each compute warp's first 16 rows) go as
      // soon as those are stored and the odd ones after the rest; with a scalar
      // decay the state is handed off whole (the second hand-off costs more than
      // it saves there).
      const uint32_t id_y = lite ? idesc_f16(128, 64, false, false) : idesc_f16(128, 128, false, false);
      auto issue_y = [&](int c) -> bool {
        const uint32_t st = smem_u32(sm + (c % NSTAGE) * STAGE);
        if constexpr (MODE == 0) {
          if (!wait_or_abort(bar_sa, c & 1, abort)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tmem + COL_Y + 128 * (c & 1), tmem + COL_SA + 8 * kk,
                   sdesc(st + REC_WQ + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024), id_y, kk > 0);
          mma_commit(bar_e);
          return true;
        }
#pragma unroll
        for (int odd = 0; odd < 2; ++odd) {
          if (!wait_or_abort(odd ? bar_sa1 : bar_sa, c & 1, abort)) return false;
          tc_fence_after();
#pragma unroll
          for (int k2 = 0; k2 < 4; ++k2) {
            const int kk = 2 * k2 + odd;
            mma_ts(tmem + COL_Y + 128 * (c & 1), tmem + COL_SA + 8 * kk,
                   sdesc(st + REC_WQ + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024), id_y, kk > 0);
          }
        }
        mma_commit(bar_e);
        return true;
      };
      griddep_wait();   // the records are the preparation kernel's output
      // CARRY_FAULT_MISSING_COPY (host fault injection): CTA (0, 0, 0) never copies
      // record 1 nor expects its bytes, so the waits for it give up after their limit
      const bool inject = (flags & CARRY_FAULT_MISSING_COPY) && (blockIdx.x | blockIdx.y | blockIdx.z) == 0;
      for (int c = 0; c < NSTAGE && c < NC; ++c)
        if (!(inject && c == 1)) issue_chunk(c);
      bool ok = wait_full(0) && issue_y(0);
      // Waits follow the order in which the compute warps arrive (done(c-1)
      // before E(c) before S(c)), so no barrier can complete a phase the
      // issuer has not waited for yet.
      for (int c = 0; ok && c < NC; ++c) {
        // chunk c-1 fully consumed: its stage takes record c+2 (without outputs, whose
        // record takes four copies, they are issued after the dS product, off its path)
        if (c >= 1) {
          if (!(ok = wait_or_abort(bar_done, (c - 1) & 1, abort))) break;
          if (!lite && c + 2 < NC) issue_chunk(c + 2);
        }
        // dS^T = E^T Kt ; Y_Q += E^T P^T
        if (!(ok = wait_or_abort(bar_ea, c & 1, abort))) break;
        tc_fence_after();
        const uint32_t st = smem_u32(sm + (c % NSTAGE) * STAGE);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ts(tmem + COL_DS, tmem + COL_EA + 8 * kk, sdesc(st + REC_K + kk * 2048, 8192, 1024),
                 idesc_f16(128, 128, false, true), kk > 0);
        mma_commit(bar_s);
        if (lite && c >= 1 && c + 2 < NC) issue_chunk(c + 2);
        if (!lite) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ts(tmem + COL_Y + 128 * (c & 1) + 64, tmem + COL_EA + 8 * kk, sdesc(st + REC_P + kk * 32, 16, 1024),
                   idesc_f16(128, 64, false, false), 1);
          mma_commit(bar_o);
        }
        if (c + 1 < NC) {
          if (!(ok = wait_full(c + 1) && issue_y(c + 1))) break;
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- compute warps
    griddep_wait();   // the initial state and the records may be the previous grid's output
    {
      const size_t base = (static_cast<size_t>(b) * p.H + h) * p.s0_bh_stride + static_cast<size_t>(32 * part) * p.dv + v;
      const bool from_s0 = !pass_b && p.s0 != nullptr && has_v && (zi == 0 || !(flags & CARRY_S0_FIRST));
#pragma unroll
      for (int k = 0; k < 32; ++k)
        S[k] = (flags & CARRY_IDENTITY) ? (32 * part + k == v ? 1.f : 0.f)
               : from_s0 ? __ldg(p.s0 + zi * p.s0_seg_stride + base + static_cast<size_t>(k) * p.dv) : 0.f;
    }
    // S^T rows 32 part + 16 hv .. + 15 as fp16 pairs into columns 16 part + 8 hv ..
    // (the Y product's K-step 2 part + hv), then that half's hand-off
    auto store_half = [&](int hv) {
      uint32_t r[8];
#pragma unroll
      for (int m = 0; m < 8; ++m) r[m] = pack_f16x2(S[16 * hv + 2 * m], S[16 * hv + 2 * m + 1]);
      tmem_st8(lrow + COL_SA + 16 * part + 8 * hv, r);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(hv ? bar_sa1 : bar_sa);
    };
    // scalar decay: S^T's 32 rows in one store and one hand-off
    auto store_whole = [&]() {
      uint32_t r[16];
#pragma unroll
      for (int m = 0; m < 16; ++m) r[m] = pack_f16x2(S[2 * m], S[2 * m + 1]);
      tmem_st16(lrow + COL_SA + 16 * part, r);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_sa);
    };
    if constexpr (MODE == 0) {
      store_whole();
    } else {
      store_half(0);
      store_half(1);
    }
    // MODE 2: this thread's (Dt^T V)^T (rows 32 part ..) and (P^d V)^T (tokens 16 part ..),
    // each loaded from L2 (the issuer prefetches records there) just before the wait that
    // precedes its use; short live ranges keep them out of local memory, where a pending
    // load would stall its spill store
    uint4 od_raw[2], sd_raw[4];
    auto local_terms = [&](int c) {
      return p.ws + ((static_cast<size_t>(b) * p.H + h) * p.NC + c_first + c) * rb + p.copy_bytes;
    };
    auto load_sd = [&](int c) {
      const uint4 *sd = reinterpret_cast<const uint4 *>(local_terms(c) + 8192 * NS + v * 256 + part * 64);
#pragma unroll
      for (int j = 0; j < 4; ++j) sd_raw[j] = (has_v && values) ? __ldg(sd + j) : make_uint4(0u, 0u, 0u, 0u);
    };
    auto load_od = [&](int c) {
      const uint4 *od = reinterpret_cast<const uint4 *>(local_terms(c) + v * 128 + part * 32);
#pragma unroll
      for (int j = 0; j < 2; ++j) od_raw[j] = (has_v && values) ? __ldg(od + j) : make_uint4(0u, 0u, 0u, 0u);
    };
    const size_t chunk0 = (static_cast<size_t>(b) * p.H + h) * p.NC + c_first;   // this CTA's first chunk, all (b, h)
    for (int c = 0; c < NC; ++c) {
      uint8_t *st = sm + (c % NSTAGE) * STAGE;
      const uint32_t y = lrow + COL_Y + 128 * (c & 1);
      if ((flags & CARRY_WRITE_STATES) && has_v) {   // S at the chunk's start: rows 32 part .., column v
        const size_t at = ((chunk0 + c) * DK + 32 * part) * p.dv + v;
        if (flags & CARRY_STATES_F16) {
          __half *dst = static_cast<__half *>(p.states) + at;
#pragma unroll
          for (int k = 0; k < 32; ++k) dst[static_cast<size_t>(k) * p.dv] = __float2half_rn(S[k]);
        } else {
          float *dst = static_cast<float *>(p.states) + at;
#pragma unroll
          for (int k = 0; k < 32; ++k) dst[static_cast<size_t>(k) * p.dv] = S[k];
        }
      }
      if ((flags & CARRY_SNAPSHOTS) && has_v && c > 0 && (c_first + c) % p.snap_len == 0) {
        float *dst = (pass_b ? p.snap_b : p.snap) + static_cast<size_t>((c_first + c) / p.snap_len - 1) * p.snap_stride +
                     ((static_cast<size_t>(b) * p.H + h) * DK + 32 * part) * p.dv + v;
#pragma unroll
        for (int k = 0; k < 32; ++k) dst[static_cast<size_t>(k) * p.dv] = S[k];
      }

      // E^T = U'^T + Y_W, tokens 16 part .. 16 part + 15; U'^T is read from the
      // stage before Y(c) is waited for
      bool ok = wait_or_abort(&bar_full[c % NSTAGE], (c / NSTAGE) & 1, abort);
      if (!__all_sync(0xffffffffu, ok)) break;
      uint4 u_raw[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
      if (has_v && values) {
#pragma unroll
        for (int j = 0; j < 2; ++j) u_raw[j] = *reinterpret_cast<const uint4 *>(st + REC_U + sw128(v, 2 * part + j));
      }
      ok = wait_or_abort(bar_e, c & 1, abort);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      {
        float e[16];
        tmem_ld16(y + 16 * part, e);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const __half2 *hp = reinterpret_cast<const __half2 *>(&u_raw[j]);
#pragma unroll
          for (int q2 = 0; q2 < 4; ++q2) {
            const float2 f = __half22float2(hp[q2]);
            e[8 * j + 2 * q2] += f.x;
            e[8 * j + 2 * q2 + 1] += f.y;
          }
        }
        uint32_t r[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) r[m] = pack_f16x2(e[2 * m], e[2 * m + 1]);
        tmem_st8(lrow + COL_EA + 8 * part, r);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_ea);
        smax = fmaxf(smax, max_abs16(e));   // the range check, after the hand-off
      }
      if constexpr (MODE == 2) load_sd(c);

      // S^T = Gamma_C S^T + dS^T, d_k rows 32 part .. 32 part + 31 (Gamma_C per row
      // for channel decay)
      ok = wait_or_abort(bar_s, c & 1, abort);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      {
        const float *gcv = reinterpret_cast<const float *>(st + rec_sc(NS)) + (CHAN ? 32 * part : 0);
        if constexpr (MODE == 0) {   // both halves of dS^T in one wait, one hand-off
          float d0[16], d1[16];
          tmem_ld16(lrow + COL_DS + 32 * part, d0);
          tmem_ld16(lrow + COL_DS + 32 * part + 16, d1);
          tmem_wait_ld();
          const float gc = gcv[0];
#pragma unroll
          for (int m = 0; m < 16; ++m) {
            S[m] = fmaf(gc, S[m], d0[m]);
            S[16 + m] = fmaf(gc, S[16 + m], d1[m]);
          }
          store_whole();
        } else if constexpr (MODE == 1) {   // channel decay: half by half (registers)
#pragma unroll
          for (int hv = 0; hv < 2; ++hv) {
            float d[16];
            tmem_ld16(lrow + COL_DS + 32 * part + 16 * hv, d);
            tmem_wait_ld();
#pragma unroll
            for (int m = 0; m < 16; ++m) S[16 * hv + m] = fmaf(gcv[16 * hv + m], S[16 * hv + m], d[m]);
            store_half(hv);
          }
        } else {   // GDN-2: two halves of 16 rows keep its extra terms in registers
#pragma unroll
          for (int hv = 0; hv < 2; ++hv) {
            float d[16];
            tmem_ld16(lrow + COL_DS + 32 * part + 16 * hv, d);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const __half2 *hp = reinterpret_cast<const __half2 *>(&sd_raw[2 * hv + j]);
#pragma unroll
              for (int q2 = 0; q2 < 4; ++q2) {
                const float2 f = __half22float2(hp[q2]);
                d[8 * j + 2 * q2] += f.x;
                d[8 * j + 2 * q2 + 1] += f.y;
              }
            }
#pragma unroll
            for (int m = 0; m < 16; ++m) S[16 * hv + m] = fmaf(gcv[16 * hv + m], S[16 * hv + m], d[m]);
          }
          store_half(0);
          store_half(1);
        }
        smax = fmaxf(smax, fmaxf(max_abs16(S), max_abs16(S + 16)));   // after the hand-off
        if constexpr (MODE == 2) {
          if (!lite) load_od(c);
        }
      }

      // output rows: tokens 16 part .. 16 part + 15 of value columns 32 quad .., transposed
      // through this warp's 1 KB of the stage's (now unused) U'^T tile into 16-byte stores.
      // Without outputs the stage is released once the S update is done: every MMA that
      // reads it completed before bar_s.
      if (!lite) {
        ok = wait_or_abort(bar_o, c & 1, abort);
        if (!__all_sync(0xffffffffu, ok)) break;
        tc_fence_after();
      }
      if (!lite) {
        float yo[16];
        tmem_ld16(y + 64 + 16 * part, yo);
        tmem_wait_ld();
        if constexpr (MODE == 2) {
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const __half2 *hp = reinterpret_cast<const __half2 *>(&od_raw[j]);
#pragma unroll
            for (int q2 = 0; q2 < 4; ++q2) {
              const float2 f = __half22float2(hp[q2]);
              yo[8 * j + 2 * q2] += f.x;
              yo[8 * j + 2 * q2 + 1] += f.y;
            }
          }
        }
        if (has_v) {
          uint8_t *tile = st + REC_U + (quad * 4 + part) * 1024;
#pragma unroll
          for (int m = 0; m < 16; ++m)
            *reinterpret_cast<__nv_bfloat16 *>(tile + m * 64 + lane * 2) = __float2bfloat16_rn(yo[m]);
          __syncwarp();
#pragma unroll
          for (int it = 0; it < 2; ++it) {
            const int q = it * 32 + lane, tr = q >> 2, piece = q & 3;
            const int t = (c_first + c) * C + 16 * part + tr;
            const uint4 val = *reinterpret_cast<const uint4 *>(tile + tr * 64 + piece * 16);
            if (t < p.T)
              *reinterpret_cast<uint4 *>(p.o + ((static_cast<size_t>(b) * p.T + t) * p.H + h) * p.dv + 32 * quad +
                                         8 * piece) = val;
          }
        }
      }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_done);
    }
  }

  __syncthreads();
  const bool failed = *abort != 0;
  if (failed) {
    // a wait gave up: report it, then let the MMAs and copies in flight
    // finish (each wait again bounded) before tensor memory is released
    if (warp == NCOMPUTE && lane == 0) {
      atomicOr(&g_gdr_split_error, 1);
      mma_commit(bar_drain);
      mbar_wait(bar_drain, 0);
      for (int s = 0; s < NSTAGE; ++s)
        if (pend >> s & 1u) mbar_wait(&bar_full[s], par >> s & 1u);
    }
  } else if (warp < NCOMPUTE) {
    if (smax > F16_SAFE) atomicOr(&g_gdr_split_error, 2);
    const bool write_final = !(flags & CARRY_LAST_FINAL) || zi + 1 == p.z_split;
    float *sf = pass_b ? p.s_final_b : p.s_final;
    if (sf != nullptr && has_v && write_final) {
      float *dst = sf + zi * (pass_b ? p.s_final_b_seg_stride : p.s_final_seg_stride) +
                   (static_cast<size_t>(b) * p.H + h) * (pass_b ? static_cast<size_t>(DK) * p.dv : p.s_final_bh_stride) +
                   static_cast<size_t>(32 * part) * p.dv + v;
#pragma unroll
      for (int k = 0; k < 32; ++k) dst[static_cast<size_t>(k) * p.dv] = S[k];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// Chunk range of a preparation launch and the SMs its persistent grid is sized for.
struct PrepRange {
  int c0 = 0, ncr = 0;   // chunks [c0, c0 + ncr); ncr = 0: all
  int sms = 0;           // 0: the whole device
  bool after_carry = false;   // launched as the programmatic dependent of the carry before it
};

template <typename... KArgs, typename... Args>
cudaError_t launch_maybe_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                             bool pdl, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  return e == cudaSuccess ? cudaGetLastError() : e;
}

template <int VAR>
cudaError_t launch_prep(const FwdProblem &p, int NC, uint8_t *ws, const PrepRange &rg, cudaStream_t stream,
                        std::string *err) {
  auto kern = p.raw ? chunk_prep_kernel<VAR, true> : chunk_prep_kernel<VAR, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)prep::SMEM_BYTES);
  // all of the unified L1 as shared memory, so that three preparation CTAs fit on an SM
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
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
  PrepParams pp;
  pp.B = p.B; pp.T = p.T; pp.H = p.H; pp.dv = p.dv; pp.NC = NC; pp.raw = p.raw;
  pp.c0 = rg.c0; pp.ncr = rg.ncr > 0 ? rg.ncr : NC;
  pp.beta = p.beta; pp.log_g = p.log_g; pp.ws = ws;
  pp.eps = p.eps; pp.scale = p.scale;
  // persistent grid: as many CTAs as fit on the device (or on rg.sms SMs) at once, none idle
  int dev = 0, sms = 0, per_sm = 0;
  e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess)
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, NTHREADS, prep::SMEM_BYTES);
  if (e != cudaSuccess) {
    *err = "occupancy query: ";
    return e;
  }
  // The occupancy query may report fewer CTAs per SM than are resident once
  // the carveout applies (72 KB of shared memory and 80 x 256 registers each),
  // so the grid is sized for at least prep::CTAS_PER_SM.  A CTA that does not
  // fit only starts later; no CTA waits on another.
  if (rg.sms > 0) sms = std::min(sms, rg.sms);
  const long long records = static_cast<long long>(pp.ncr) * p.H * p.B;
  const int grid = static_cast<int>(
      std::min<long long>(records, static_cast<long long>(std::max(per_sm, prep::CTAS_PER_SM)) * sms));
  e = launch_maybe_pdl(kern, dim3(grid), dim3(NTHREADS), prep::SMEM_BYTES, stream, rg.after_carry,
                       mq, mk, mv, pp);
  if (e != cudaSuccess) *err = "prep launch: ";
  return e;
}

cudaError_t launch_prep_gdn2(const FwdProblem &p, int NC, uint8_t *ws, const PrepRange &rg, cudaStream_t stream,
                             std::string *err) {
  auto kern = p.raw ? chunk_prep_gdn2_kernel<true> : chunk_prep_gdn2_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)prepg::SMEM_BYTES);
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
  PrepParams pp;
  pp.B = p.B; pp.T = p.T; pp.H = p.H; pp.dv = p.dv; pp.NC = NC; pp.raw = p.raw;
  pp.c0 = rg.c0; pp.ncr = rg.ncr > 0 ? rg.ncr : NC;
  pp.beta = nullptr; pp.log_g = p.log_g; pp.erase_b = p.erase_b; pp.write_w = p.write_w; pp.ws = ws;
  pp.eps = p.eps; pp.scale = p.scale;
  int dev = 0, sms = 0;
  e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) {
    *err = "device query: ";
    return e;
  }
  if (rg.sms > 0) sms = std::min(sms, rg.sms);
  const long long records = static_cast<long long>(pp.ncr) * p.H * p.B;
  const int grid = static_cast<int>(std::min<long long>(records, sms));   // one CTA per SM, persistent
  e = launch_maybe_pdl(kern, dim3(grid), dim3(NTHREADS), prepg::SMEM_BYTES, stream,
                       rg.after_carry, mq, mk, mv, mg, pp);
  if (e != cudaSuccess) *err = "prep launch: ";
  return e;
}

cudaError_t launch_prep_chan(const FwdProblem &p, int NC, uint8_t *ws, const PrepRange &rg, cudaStream_t stream,
                             std::string *err) {
  auto kern = p.raw ? chunk_prep_chan_kernel<true> : chunk_prep_chan_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)prepc::SMEM_BYTES);
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
  PrepParams pp;
  pp.B = p.B; pp.T = p.T; pp.H = p.H; pp.dv = p.dv; pp.NC = NC; pp.raw = p.raw;
  pp.c0 = rg.c0; pp.ncr = rg.ncr > 0 ? rg.ncr : NC;
  pp.beta = p.beta; pp.log_g = p.log_g; pp.ws = ws;
  pp.eps = p.eps; pp.scale = p.scale;
  int dev = 0, sms = 0;
  e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) {
    *err = "device query: ";
    return e;
  }
  if (rg.sms > 0) sms = std::min(sms, rg.sms);
  const long long records = static_cast<long long>(pp.ncr) * p.H * p.B;
  const int grid = static_cast<int>(std::min<long long>(records, sms));   // one CTA per SM, persistent
  e = launch_maybe_pdl(kern, dim3(grid), dim3(NTHREADS), prepc::SMEM_BYTES, stream,
                       rg.after_carry, mq, mk, mv, mg, pp);
  if (e != cudaSuccess) *err = "prep launch: ";
  return e;
}

// Start states of phase 2's parts (see SegPlan), for one (b, h) and 16 value
// columns per CTA, in fp32.  The segment starts form the chain
//     S_start[0] = s0 (zeros if null),  S_start[1] = D_0,
//     S_start[g + 1] = M_g S_start[g] + D_g  (g = 1 .. G - 2),
// where D_0 is segment 0's end state from s0 itself and, for g >= 1, M_g is the
// transition map of segment g (the carry from the identity with the values
// taken as zero, d_k x d_k, stored at index g - 1) and D_g its end state from
// zero (d_k x d_v).  A part that starts j chunks into segment g (0 < j < L)
// starts from the same affine map after j chunks, which phase 1 leaves as
// snapshots of both carries: S = M_g(j) S_start[g] + D_g(j), or D_0(j) itself
// in segment 0.  `items` lists the steps in order: a chain step (0x8000 | part
// << 8 | g) forms S_start[g + 1] and, where a part starts there, writes it as
// that part's state; a part step (its index) forms a part inside a segment.
// Part 0 is S_start[0].
struct ChainItems {
  static constexpr int kMax = 16 + 64;
  int n = 0;
  uint16_t it[kMax];
};
namespace chain {
constexpr int NT = 512;                         // threads: 32 row groups x 16 k-slices
constexpr int SC_FLOATS = DK * 16 + (DK / 8) * 4;   // S_start[g] for 16 columns, padded (see sc_at)
constexpr size_t SMEM_BYTES = 2 * 8 * NT * 16;  // two steps' maps, 8 float4 per thread
// Row k of the 16-column start state: the 16 k-slices of a warp read rows 8
// apart, so each group of 8 rows is shifted by 4 banks.
__device__ __forceinline__ int sc_at(int k) { return k * 16 + (k >> 3) * 4; }
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_one() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
}  // namespace chain
// Each thread forms a 4 x 16 block of the product (rows 4 rg .. 4 rg + 3, the
// CTA's 16 columns) over its 8-wide k-slice; the 16 k-slices of a row group
// (half a warp) then sum by shuffles, each lane keeping 4 of the 64 values.
// The maps of the next step are copied into shared memory (each thread its
// own 8 float4) while the current one is formed.
__global__ void __launch_bounds__(chain::NT, 1) segment_chain_kernel(const float *s0, const float *M, const float *D,
                                                                    const float *snapM, const float *snapD,
                                                                    float *S_part, const ChainItems items, int L,
                                                                    int Lp, int H, int dv) {
  using namespace chain;
  __shared__ __align__(16) float Sc[SC_FLOATS];
  extern __shared__ float4 stage[];   // [2][8][NT]
  const int sl = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const size_t BH = static_cast<size_t>(gridDim.z) * H, bh = static_cast<size_t>(b) * H + h;
  const size_t slot = BH * DK * dv, mslot = BH * DK * DK;
  const int rg = tid >> 4, ks = tid & 15;
  const int r0 = 4 * rg, kb = 8 * ks;
  // after the reduction: row 4 rg + ks / 4, columns 4 (ks % 4) .. + 3 of the CTA's 16
  const int orow = r0 + (ks >> 2), ocol = 4 * (ks & 3);
  const size_t at = (bh * DK + orow) * dv + 16 * sl + ocol;
  for (int e = tid; e < DK * 16; e += NT) {
    const int k = e >> 4, j = e & 15;
    const size_t a = (bh * DK + k) * dv + 16 * sl + j;
    const float x = s0 != nullptr ? s0[a] : 0.f;
    Sc[sc_at(k) + j] = x;
    S_part[a] = x;
  }
  // the map of step n, or null where the step copies
  auto map_of = [&](int n) -> const float * {
    const int it = items.it[n];
    const int g = (it & 0x8000) ? (it & 0xff) : it * Lp / L;
    if (g == 0) return nullptr;
    return (it & 0x8000) ? M + (g - 1) * mslot : snapM + (it - 1) * mslot;
  };
  // this thread's part of a map: float4 j = 2 rho + half is M[r0 + rho][kb + 4 half .. + 3]
  auto fetch = [&](int n, int buf) {
    const float *m = n < items.n ? map_of(n) : nullptr;
    if (m != nullptr) {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        cp_async16(&stage[(buf * 8 + j) * NT + tid], m + (bh * DK + r0 + (j >> 1)) * DK + kb + 4 * (j & 1));
    }
    cp_async_commit();
  };
  fetch(0, 0);
  __syncthreads();
  for (int n = 0; n < items.n; ++n) {
    const int it = items.it[n];
    const bool chain_step = (it & 0x8000) != 0;
    const bool has_map = map_of(n) != nullptr;   // uniform over the CTA
    fetch(n + 1, (n + 1) & 1);
    const float *Dp = chain_step ? D + (it & 0xff) * slot : snapD + (it - 1) * slot;
    const float4 dd = __ldg(reinterpret_cast<const float4 *>(Dp + at));
    float acc[64];
#pragma unroll
    for (int e = 0; e < 64; ++e) acc[e] = 0.f;
    cp_async_wait_one();   // this step's map (the thread's own copies)
    if (has_map) {
      const float4 *st = stage + (n & 1) * 8 * NT + tid;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float4 mr[4];
#pragma unroll
        for (int rho = 0; rho < 4; ++rho) mr[rho] = st[(2 * rho + half) * NT];
#pragma unroll
        for (int kq = 0; kq < 4; ++kq) {
          const float4 *sr = reinterpret_cast<const float4 *>(&Sc[sc_at(kb + 4 * half + kq)]);
          float sv[16];
#pragma unroll
          for (int j4 = 0; j4 < 4; ++j4) {
            const float4 x = sr[j4];
            sv[4 * j4] = x.x; sv[4 * j4 + 1] = x.y; sv[4 * j4 + 2] = x.z; sv[4 * j4 + 3] = x.w;
          }
#pragma unroll
          for (int rho = 0; rho < 4; ++rho) {
            const float m = kq == 0 ? mr[rho].x : kq == 1 ? mr[rho].y : kq == 2 ? mr[rho].z : mr[rho].w;
#pragma unroll
            for (int c = 0; c < 16; ++c) acc[16 * rho + c] = fmaf(m, sv[c], acc[16 * rho + c]);
          }
        }
      }
    }
    // sum over the 16 k-slices: each round keeps the half of the values that
    // its lane bit selects; lane ks ends with values 4 ks .. 4 ks + 3
#pragma unroll
    for (int w = 32, mask = 8; w >= 4; w >>= 1, mask >>= 1) {
      const bool up = (ks & mask) != 0;
#pragma unroll
      for (int e = 0; e < w; ++e) {
        const float send = up ? acc[e] : acc[w + e];
        acc[e] = (up ? acc[w + e] : acc[e]) + __shfl_xor_sync(0xffffffffu, send, mask);
      }
    }
    const float4 out = make_float4(acc[0] + dd.x, acc[1] + dd.y, acc[2] + dd.z, acc[3] + dd.w);
    if (chain_step) {
      __syncthreads();   // every thread is done reading S_start[g]
      *reinterpret_cast<float4 *>(&Sc[sc_at(orow) + ocol]) = out;
      const int part = (it >> 8) & 0x7f;
      if (part > 0) *reinterpret_cast<float4 *>(S_part + part * slot + at) = out;
      __syncthreads();
    } else {
      *reinterpret_cast<float4 *>(S_part + it * slot + at) = out;
    }
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
}

struct CarryLaunch {
  int c_base = 0;
  int segments = 1, seg_len = 0, flags = 0;
  const float *s0 = nullptr;
  float *s_final = nullptr;
  size_t s0_stride = 0, s_final_stride = 0;
  size_t s0_bh_stride = 0, s_final_bh_stride = 0;   // 0: d_k d_v (packed [B, H, d_k, d_v])
  // optional pass B in the same launch
  int segments_b = 0, seg_first_b = 0, flags_b = 0;
  float *s_final_b = nullptr;
  size_t s_final_b_stride = 0;
  void *states = nullptr;    // CARRY_WRITE_STATES output
  int snap_len = 0;          // CARRY_SNAPSHOTS
  float *snap = nullptr, *snap_b = nullptr;
  size_t snap_stride = 0;
};

// `pdl`: launched with programmatic stream serialization, so that its CTAs may
// start (allocate, set up) while the grid before it on the stream finishes;
// every thread waits for that grid's completion before it reads the initial
// state or a record.
template <int MODE>
cudaError_t launch_carry(const FwdProblem &p, int NC, const uint8_t *ws, const CarryLaunch &l, bool pdl,
                         cudaStream_t stream, std::string *err) {
  cudaError_t e = cudaFuncSetAttribute(chunk_carry_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)carry::SMEM_BYTES);
  if (e != cudaSuccess) {
    *err = "cudaFuncSetAttribute: ";
    return e;
  }
  CarryParams cp;
  cp.T = p.T; cp.H = p.H; cp.dv = p.dv; cp.NC = NC;
  cp.seg_len = l.seg_len; cp.flags = l.flags;
  const int ns = p.dv / 64;
  cp.rec_bytes = MODE == 2 ? rec_bytes_gdn2(ns) : MODE == 1 ? rec_bytes_chan(ns) : rec_bytes(ns);
  cp.copy_bytes = MODE == 0 ? rec_bytes(ns) : rec_bytes_chan(ns);
  cp.ws = ws; cp.s0 = l.s0; cp.s_final = l.s_final;
  cp.s0_seg_stride = l.s0_stride; cp.s_final_seg_stride = l.s_final_stride;
  cp.c_base = l.c_base;
  cp.s0_bh_stride = l.s0_bh_stride ? l.s0_bh_stride : static_cast<size_t>(DK) * p.dv;
  cp.s_final_bh_stride = l.s_final_bh_stride ? l.s_final_bh_stride : static_cast<size_t>(DK) * p.dv;
  cp.z_split = l.segments;
  cp.seg_first_b = l.seg_first_b; cp.flags_b = l.flags_b;
  cp.s_final_b = l.s_final_b; cp.s_final_b_seg_stride = l.s_final_b_stride;
  cp.o = static_cast<__nv_bfloat16 *>(p.o);
  cp.states = l.states;
  cp.snap_len = l.snap_len; cp.snap = l.snap; cp.snap_b = l.snap_b; cp.snap_stride = l.snap_stride;
  // GDR_FAULT=wait (host-side fault injection for the failure-path tests): CTA
  // (0, 0, 0) never copies chunk 1's record, so its waits give up after their
  // limit (about a second).
  const char *fault = std::getenv("GDR_FAULT");
  if (fault != nullptr && std::strcmp(fault, "wait") == 0) {
    cp.flags |= CARRY_FAULT_MISSING_COPY;
    cp.flags_b |= CARRY_FAULT_MISSING_COPY;
  }
  e = launch_maybe_pdl(chunk_carry_kernel<MODE>, dim3(p.H, p.B, l.segments + l.segments_b),
                       dim3(carry::NTHREADS_CARRY), carry::SMEM_BYTES, stream, pdl, cp);
  if (e != cudaSuccess) *err = "carry launch: ";
  return e;
}

// Carry over segments when too few (b, h) sequences fill the machine: each of G
// segments of a sequence gets its own CTA.  Phase 1, one launch, computes the
// affine map S_end = M_g S_start + D_g of every segment but the last: D_g is
// the end state from zero, except that segment 0 starts from s0 itself, so
// D_0 is already S_start[1] and segment 0 needs no M; M_g (g >= 1) is the
// carry from the identity with the values taken as zero.  That is 2G - 3
// state-only CTAs per (b, h), all resident at once.  A chain kernel turns the
// maps into start states; phase 2 runs the sequence from them with outputs.
//
// Phase 2 needs one CTA per part where phase 1 needs about two per segment, so
// it may cut the sequence finer: P parts of Lp chunks.  A part that starts
// inside segment g (g < G - 1) starts from the segment's map and offset after
// the chunks before it, which phase 1's two carries leave there as snapshots;
// no part may start inside the last segment, which phase 1 does not run.  The
// plan minimises the sequential time in units of about 0.4 us, measured on the
// 64k-token sweep: a phase-1 chunk (no outputs) 4, a phase-2 chunk 5, a
// product of the chain 10.  The sequential depth drops from NC chunks to about
// L + Lp.
struct SegPlan {
  int G = 1, L = 0;    // phase 1: segments of L chunks
  int P = 1, Lp = 0;   // phase 2: parts of Lp chunks (P = G, Lp = L unless cut finer)
  bool finer() const { return G > 1 && Lp != L; }
};
constexpr int kMaxParts = 64;
// SMs of the current device, 0 if there is none.
int device_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return sms;
}
// Products the chain kernel forms for a plan: one per segment start after the
// second, one per part starting strictly inside a segment other than the first.
int seg_products(int G, int L, int P, int Lp) {
  int n = G - 2;
  for (int p = 1; p < P; ++p)
    if (p * Lp >= L && (p * Lp) % L != 0) ++n;
  return n;
}
SegPlan seg_plan_for(int B, int H, int dv, int NC, int sms) {
  SegPlan sp;
  sp.L = NC;
  const long long bh = static_cast<long long>(B) * H;
  if (dv != 128 || NC < 64 || bh <= 0 || sms <= 0) return sp;
  // phase 1 runs (2G - 3) bh CTAs, at most one per SM
  const int G = static_cast<int>(std::min<long long>(16, (sms / bh + 3) / 2));
  if (G < 3) return sp;
  sp.L = (NC + G - 1) / G;
  sp.G = (NC + sp.L - 1) / sp.L;
  sp.P = sp.G;
  sp.Lp = sp.L;
  auto cost = [](int G1, int L1, int P, int Lp) { return 4LL * L1 + 5LL * Lp + 10LL * seg_products(G1, L1, P, Lp); };
  long long best = cost(sp.G, sp.L, sp.P, sp.Lp);
  const int pmax = static_cast<int>(std::min<long long>(std::min<long long>(sms / bh, NC), kMaxParts));
  const SegPlan base = sp;
  for (int P0 = base.G + 1; P0 <= pmax; ++P0) {
    const int Lp = (NC + P0 - 1) / P0, P = (NC + Lp - 1) / Lp;
    if (P <= base.G) continue;
    // the shortest phase-1 segments that leave no part start inside the last one
    for (int L1 = base.L; L1 <= base.L + Lp; ++L1) {
      const int G1 = (NC + L1 - 1) / L1;
      if (G1 < 3) break;
      if (static_cast<long long>(G1 - 1) * L1 < static_cast<long long>(P - 1) * Lp) continue;
      const long long c = cost(G1, L1, P, Lp);
      if (c < best) {
        best = c;
        sp.G = G1; sp.L = L1; sp.P = P; sp.Lp = Lp;
      }
      break;
    }
  }
  return sp;
}
SegPlan seg_plan(int B, int H, int dv, int NC) {
  if (dv != 128 || NC < 64) return seg_plan_for(B, H, dv, NC, 0);
  return seg_plan_for(B, H, dv, NC, device_sms());
}
// The chain kernel's steps for a plan (see segment_chain_kernel); false if a
// part would start inside the last segment.
bool chain_items(const SegPlan &sp, ChainItems *ci) {
  ci->n = 0;
  int p = 1;
  for (int g = 0; g + 1 < sp.G; ++g) {
    for (; p < sp.P && p * sp.Lp < (g + 1) * sp.L; ++p) ci->it[ci->n++] = static_cast<uint16_t>(p);
    int at_start = 0;
    if (p < sp.P && p * sp.Lp == (g + 1) * sp.L) at_start = p++;
    ci->it[ci->n++] = static_cast<uint16_t>(0x8000 | (at_start << 8) | g);
  }
  return p == sp.P;
}
// Floats of the maps, offsets, part start states and snapshots.
size_t seg_extra_floats(int B, int H, int dv, const SegPlan &sp) {
  if (sp.G == 1) return 0;
  const size_t bh = static_cast<size_t>(B) * H;
  size_t n = (sp.G - 2) * bh * DK * DK + (sp.G - 1) * bh * DK * dv + sp.P * bh * DK * dv;
  if (sp.finer()) n += (sp.P - 1) * bh * (DK * dv + DK * DK);
  return n;
}

// Pipelined sweep.  The carry runs B*H CTAs, one per SM, and leaves the other
// SMs idle; when enough are left, the sequences are cut at chunk c_split and
// four grids run back to back on the caller's stream, each launched as the
// programmatic dependent of the one before it:
//     prep [0, c_split) on the whole device;
//     carry [0, c_split), its CTAs taking SMs as the first preparation drains;
//     prep [c_split, NC), launched once every carry CTA holds its SM and sized
//         for the SMs the carry leaves; its last step waits for the carry grid;
//     carry [c_split, NC) from the first carry's end states.
// A grid waits only for the completion of the grid before it (griddepcontrol),
// never on another's progress.  c_split minimises a cost model fitted to B200
// measurements: a persistent preparation grid takes about P0 + P1 * (records
// per CTA) us, a carry about C0 + C1 * (chunks) us; the plan is taken only where
// the model expects at least 3% over the serial sweep.
struct PipePlan {
  int c_split = 0;   // 0: serial
  int prep_sms = 0;  // SMs the second preparation grid is sized for
};
PipePlan pipe_plan_for(int variant, int B, int H, int NC, int sms) {
  PipePlan pp;
  const long long bh = static_cast<long long>(B) * H;
  if (NC < 4 || bh <= 0 || sms - bh < 16) return pp;
  // per variant family: scalar decay (three preparation CTAs per SM), KDA, GDN-2 (one each)
  const int fam = variant == kGDN2 ? 2 : variant == kKDA ? 1 : 0;
  const double slots = fam ? 1.0 : 3.0;                       // preparation CTAs per SM
  const double P0 = fam ? 13.0 : 9.0;                         // us
  const double P1 = fam == 2 ? 15.0 : fam ? 10.8 : 11.5;      // us per record per CTA
  const double C0 = fam == 2 ? 2.5 : fam ? 2.1 : 2.4;         // us
  const double C1 = fam == 2 ? 3.1 : fam ? 1.85 : 2.1;        // us per chunk
  auto prep = [&](double records, double ctas) { return P0 + P1 * records / ctas; };
  const double serial = prep(double(NC) * bh, slots * sms) + C0 + C1 * NC;
  double best = serial;
  for (int cs = 1; cs < NC; ++cs) {
    const double t = prep(double(cs) * bh, slots * sms) +
                     std::max(C0 + C1 * cs, prep(double(NC - cs) * bh, slots * (sms - bh))) + C0 + C1 * (NC - cs) + 2.0;
    if (t < best) {
      best = t;
      pp.c_split = cs;
    }
  }
  if (best > 0.97 * serial) pp.c_split = 0;
  pp.prep_sms = static_cast<int>(sms - bh);
  return pp;
}
PipePlan pipe_plan(int variant, int B, int H, int NC) {
  if (NC < 4) return PipePlan();
  return pipe_plan_for(variant, B, H, NC, device_sms());
}

template <int VAR>
cudaError_t launch_prep_any(const FwdProblem &p, int NC, uint8_t *w, const PrepRange &rg, cudaStream_t stream,
                            std::string *err) {
  if constexpr (VAR == kKDA) return launch_prep_chan(p, NC, w, rg, stream, err);
  else if constexpr (VAR == kGDN2) return launch_prep_gdn2(p, NC, w, rg, stream, err);
  else return launch_prep<VAR>(p, NC, w, rg, stream, err);
}

template <int VAR>
cudaError_t launch_pipelined(const FwdProblem &p, int NC, uint8_t *w, const PipePlan &pp, cudaStream_t stream,
                             std::string *err) {
  constexpr int MODE = VAR == kGDN2 ? 2 : VAR == kKDA ? 1 : 0;
  const int cs = pp.c_split, ns = p.dv / 64;
  const size_t rb = MODE == 2 ? rec_bytes_gdn2(ns) : MODE == 1 ? rec_bytes_chan(ns) : rec_bytes(ns);
  // The first carry's end states go to each sequence's chunk-0 record, which
  // that carry CTA has consumed by then and the second preparation never writes.
  float *mid = reinterpret_cast<float *>(w);
  const size_t mid_bh = static_cast<size_t>(NC) * rb / sizeof(float);
  PrepRange r1;
  r1.ncr = cs;
  cudaError_t e = launch_prep_any<VAR>(p, NC, w, r1, stream, err);
  if (e != cudaSuccess) return e;
  CarryLaunch l1;
  l1.seg_len = cs;
  l1.s0 = p.s0;
  l1.s_final = mid;
  l1.s_final_bh_stride = mid_bh;
  if ((e = launch_carry<MODE>(p, NC, w, l1, true, stream, err)) != cudaSuccess) return e;
  PrepRange r2;
  r2.c0 = cs;
  r2.ncr = NC - cs;
  r2.sms = pp.prep_sms;
  r2.after_carry = true;
  if ((e = launch_prep_any<VAR>(p, NC, w, r2, stream, err)) != cudaSuccess) return e;
  CarryLaunch l2;
  l2.c_base = cs;
  l2.seg_len = NC - cs;
  l2.s0 = mid;
  l2.s0_bh_stride = mid_bh;
  l2.s_final = p.s_final;
  return launch_carry<MODE>(p, NC, w, l2, true, stream, err);
}

// The carry over segments (few long sequences, sp.G > 1) on the records at
// `records`, with the segment maps, offsets and start states at `maps`
// (seg_extra_floats floats): phase 1, the chain of start states, then phase 2,
// every segment from its start state with flags2 added (the forward: none, so
// with outputs; the backward's carries: no outputs, chunk states kept).
template <int MODE>
cudaError_t launch_segmented(const FwdProblem &p, int NC, const SegPlan &sp, const uint8_t *records, uint8_t *maps,
                             const float *s0, float *s_final, int flags2, void *states, cudaStream_t stream,
                             std::string *err) {
  const size_t bh = static_cast<size_t>(p.B) * p.H;
  ChainItems items;
  if (!chain_items(sp, &items)) {
    *err = "segment plan: ";
    return cudaErrorInvalidValue;
  }
  float *Mb = reinterpret_cast<float *>(maps);
  float *Db = Mb + (sp.G - 2) * bh * DK * DK;
  float *Ss = Db + (sp.G - 1) * bh * DK * p.dv;
  float *snapD = Ss + sp.P * bh * DK * p.dv;               // used when the parts are finer
  float *snapM = snapD + (sp.P - 1) * bh * DK * p.dv;
  CarryLaunch m;   // phase 1, pass A: end states of segments 0 .. G-2 (segment 0 from s0, the rest from zero)
  m.segments = sp.G - 1; m.seg_len = sp.L;
  m.flags = CARRY_NO_OUTPUT | CARRY_S0_FIRST;
  m.s0 = s0;
  m.s_final = Db; m.s_final_stride = bh * DK * p.dv;
  // pass B: transition maps of segments 1 .. G-2
  m.segments_b = sp.G - 2; m.seg_first_b = 1;
  m.flags_b = CARRY_IDENTITY | CARRY_NO_VALUES | CARRY_NO_OUTPUT;
  m.s_final_b = Mb; m.s_final_b_stride = bh * DK * DK;
  if (sp.finer()) {   // both passes leave their state where a part starts inside the segment
    m.flags |= CARRY_SNAPSHOTS;
    m.flags_b |= CARRY_SNAPSHOTS;
    m.snap_len = sp.Lp;
    m.snap = snapD; m.snap_b = snapM;
    m.snap_stride = bh * DK * p.dv;
  }
  cudaError_t e = launch_carry<MODE>(p, NC, records, m, true, stream, err);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(segment_chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(chain::SMEM_BYTES));
  if (e != cudaSuccess) {
    *err = "cudaFuncSetAttribute: ";
    return e;
  }
  segment_chain_kernel<<<dim3(p.dv / 16, p.H, p.B), chain::NT, chain::SMEM_BYTES, stream>>>(
      s0, Mb, Db, snapM, snapD, Ss, items, sp.L, sp.Lp, p.H, p.dv);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    *err = "segment chain launch: ";
    return e;
  }
  CarryLaunch f;   // phase 2: every part from its start
  f.segments = sp.P; f.seg_len = sp.Lp;
  f.flags = CARRY_LAST_FINAL | flags2;
  f.s0 = Ss; f.s0_stride = bh * DK * p.dv;
  f.s_final = s_final;
  f.states = states;
  return launch_carry<MODE>(p, NC, records, f, true, stream, err);
}

// `ws_bytes` is the workspace the call may use: a segmented plan whose maps do
// not fit beside the records falls back to the unsegmented sweep.
template <int VAR>
cudaError_t launch_split(const FwdProblem &p, void *ws, size_t ws_bytes, cudaStream_t stream, std::string *err) {
  constexpr int MODE = VAR == kGDN2 ? 2 : VAR == kKDA ? 1 : 0;
  const int NC = (p.T + C - 1) / C;
  uint8_t *w = static_cast<uint8_t *>(ws);
  SegPlan sp = seg_plan(p.B, p.H, p.dv, NC);
  if (sp.G > 1 && gdr_split_workspace_bytes(VAR, p.B, p.T, p.H, p.dv) > ws_bytes) sp = SegPlan{1, NC};
  if (sp.G == 1) {
    const PipePlan pp = pipe_plan(VAR, p.B, p.H, NC);
    if (pp.c_split > 0) return launch_pipelined<VAR>(p, NC, w, pp, stream, err);
  }
  cudaError_t e = launch_prep_any<VAR>(p, NC, w, PrepRange(), stream, err);
  if (e != cudaSuccess) return e;
  if (sp.G == 1) {
    CarryLaunch l;
    l.seg_len = NC;
    l.s0 = p.s0;
    l.s_final = p.s_final;
    return launch_carry<MODE>(p, NC, w, l, true, stream, err);
  }
  const size_t bh = static_cast<size_t>(p.B) * p.H, ns = p.dv / 64;
  const size_t rec = MODE == 2 ? rec_bytes_gdn2(ns) : MODE == 1 ? rec_bytes_chan(ns) : rec_bytes(ns);
  const size_t rec_total = (bh * NC * rec + 255) / 256 * 256;
  return launch_segmented<MODE>(p, NC, sp, w, w + rec_total, p.s0, p.s_final, 0, nullptr, stream, err);
}

// The backward's steps on the stream (each the programmatic dependent of the
// one before where the kernel supports it): the forward's records; a carry
// that keeps every chunk's start state (no outputs); the gradient scale and
// the reverse records; the reverse carry (third carry mode, over the reverse
// records) keeping every chunk's end-state gradient; the chunk-local
// gradients; the initial state's gradient.  Both carries run segmented where
// the forward's would (few long sequences).
template <int VAR>
cudaError_t launch_backward(const BwdProblem &bp, uint8_t *w, cudaStream_t stream, std::string *err) {
  constexpr int MODE = VAR == kKDA ? 1 : VAR == kGDN2 ? 2 : 0;
  const FwdProblem &p = bp.f;
  const int NC = (p.T + C - 1) / C;
  const BwdLayout L = bwd_layout(VAR, p.B, p.T, p.H, p.dv);
  // chunk start states in fp16 (the forward carry's own operand) for scalar decay, in fp32 for
  // channel decay; the reverse carry's states, whose fp16 rounding the gate gradients do not
  // absorb, in fp32
  void *s0s = w + L.s0s;
  float *dss = reinterpret_cast<float *>(w + L.dss);
  const int s0_f16 = MODE == 0 ? CARRY_STATES_F16 : 0;
  float *x0 = reinterpret_cast<float *>(w + L.x0), *xf = reinterpret_cast<float *>(w + L.xf);
  uint32_t *absmax = reinterpret_cast<uint32_t *>(w + L.absmax);
  const SegPlan sp = L.maps_bytes > 0 ? seg_plan(p.B, p.H, p.dv, NC) : SegPlan{1, NC};
  cudaError_t e = launch_prep_any<VAR>(p, NC, w + L.fwd_rec, PrepRange(), stream, err);
  if (e != cudaSuccess) return e;
  if (sp.G > 1) {
    e = launch_segmented<MODE>(p, NC, sp, w + L.fwd_rec, w + L.maps, p.s0, nullptr,
                               CARRY_NO_OUTPUT | CARRY_WRITE_STATES | s0_f16, s0s, stream, err);
  } else {
    CarryLaunch lf;
    lf.seg_len = NC;
    lf.flags = CARRY_NO_OUTPUT | CARRY_WRITE_STATES | s0_f16;
    lf.s0 = p.s0;
    lf.states = s0s;
    e = launch_carry<MODE>(p, NC, w + L.fwd_rec, lf, true, stream, err);
  }
  if (e != cudaSuccess) return e;
  if ((e = gdr_bwd_launch_scale(bp, absmax, x0, stream)) != cudaSuccess) {
    *err = "gradient scale: ";
    return e;
  }
  if ((e = gdr_bwd_launch_rev_prep(bp, w + L.fwd_rec, w + L.rev_rec, absmax, stream)) != cudaSuccess) {
    *err = "reverse records: ";
    return e;
  }
  if (sp.G > 1) {
    e = launch_segmented<2>(p, NC, sp, w + L.rev_rec, w + L.maps, x0, xf, CARRY_NO_OUTPUT | CARRY_WRITE_STATES,
                            dss, stream, err);
  } else {
    CarryLaunch lr;
    lr.seg_len = NC;
    lr.flags = CARRY_NO_OUTPUT | CARRY_WRITE_STATES;
    lr.s0 = x0;
    lr.s_final = xf;
    lr.states = dss;
    e = launch_carry<2>(p, NC, w + L.rev_rec, lr, true, stream, err);
  }
  if (e != cudaSuccess) return e;
  if ((e = gdr_bwd_launch_local(bp, s0s, dss, absmax, w + L.fwd_rec, w + L.rev_rec, stream)) != cudaSuccess) {
    *err = "local gradients: ";
    return e;
  }
  if ((e = gdr_bwd_launch_unscale(bp, xf, absmax, stream)) != cudaSuccess) *err = "initial-state gradient: ";
  return e;
}

}  // namespace
}  // namespace tc
}  // namespace gdr

cudaError_t gdr_launch_backward(const gdr::BwdProblem &p, void *ws, size_t ws_bytes, cudaStream_t stream,
                                std::string *err) {
  using namespace gdr;
  if (ws_bytes < bwd_layout(p.f.variant, p.f.B, p.f.T, p.f.H, p.f.dv).total) {
    *err = "workspace smaller than gdr_backward_workspace_size(): ";
    return cudaErrorInvalidValue;
  }
  uint8_t *w = static_cast<uint8_t *>(ws);
  switch (p.f.variant) {
    case kDeltaNet: return tc::launch_backward<kDeltaNet>(p, w, stream, err);
    case kGatedDeltaNet: return tc::launch_backward<kGatedDeltaNet>(p, w, stream, err);
    case kKLA: return tc::launch_backward<kKLA>(p, w, stream, err);
    case kKDA: return tc::launch_backward<kKDA>(p, w, stream, err);
    case kGDN2: return tc::launch_backward<kGDN2>(p, w, stream, err);
    default: *err = "variant not covered by the backward: "; return cudaErrorInvalidValue;
  }
}

bool gdr_split_supported(int variant, int dk, int dv) {
  using namespace gdr;
  const bool v = variant == kDeltaNet || variant == kGatedDeltaNet || variant == kKLA || variant == kKDA ||
                 variant == kGDN2;
  return v && dk == 128 && (dv == 64 || dv == 128);
}

size_t gdr_split_record_bytes(int variant, int dv) {
  return variant == gdr::kGDN2  ? gdr::tc::rec_bytes_gdn2(dv / 64)
         : variant == gdr::kKDA ? gdr::tc::rec_bytes_chan(dv / 64)
                                : gdr::tc::rec_bytes(dv / 64);
}

size_t gdr_split_segment_bytes(int B, int T, int H, int dv) {
  const int NC = (T + 63) / 64;
  const gdr::tc::SegPlan sp = gdr::tc::seg_plan(B, H, dv, NC);
  return sp.G == 1 ? 0 : 4 * gdr::tc::seg_extra_floats(B, H, dv, sp);
}

size_t gdr_split_workspace_bytes(int variant, int B, int T, int H, int dv) {
  const size_t NC = (static_cast<size_t>(T) + 63) / 64;
  const size_t records = static_cast<size_t>(B) * H * NC * gdr_split_record_bytes(variant, dv);
  const gdr::tc::SegPlan sp = gdr::tc::seg_plan(B, H, dv, static_cast<int>(NC));
  if (sp.G == 1) return records;
  return (records + 255) / 256 * 256 + 4 * gdr::tc::seg_extra_floats(B, H, dv, sp);
}

void gdr_split_plan(int variant, int B, int T, int H, int dv, int sms, int *segments, int *segment_chunks,
                    int *split_chunk, int *parts, int *part_chunks) {
  const int NC = (T + 63) / 64;
  const gdr::tc::SegPlan sp = gdr::tc::seg_plan_for(B, H, dv, NC, sms);
  *segments = sp.G;
  *segment_chunks = sp.L;
  *split_chunk = sp.G == 1 ? gdr::tc::pipe_plan_for(variant, B, H, NC, sms).c_split : 0;
  if (parts != nullptr) *parts = sp.G == 1 ? 1 : sp.P;
  if (part_chunks != nullptr) *part_chunks = sp.G == 1 ? sp.L : sp.Lp;
}

int gdr_split_launches(int variant, int B, int T, int H, int dv) {
  const int NC = (T + 63) / 64;
  if (gdr::tc::seg_plan(B, H, dv, NC).G > 1) return 4;
  return gdr::tc::pipe_plan(variant, B, H, NC).c_split > 0 ? 4 : 2;
}

cudaError_t gdr_launch_split(const gdr::FwdProblem &p, void *ws, size_t ws_bytes, cudaStream_t stream,
                             std::string *err) {
  using namespace gdr;
  switch (p.variant) {
    case kDeltaNet: return tc::launch_split<kDeltaNet>(p, ws, ws_bytes, stream, err);
    case kGatedDeltaNet: return tc::launch_split<kGatedDeltaNet>(p, ws, ws_bytes, stream, err);
    case kKLA: return tc::launch_split<kKLA>(p, ws, ws_bytes, stream, err);
    case kKDA: return tc::launch_split<kKDA>(p, ws, ws_bytes, stream, err);
    case kGDN2: return tc::launch_split<kGDN2>(p, ws, ws_bytes, stream, err);
    default: *err = "variant not covered: "; return cudaErrorInvalidValue;
  }
}

int gdr_read_device_error(cudaStream_t stream) {
  int h = 0, zero = 0;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return -1;
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
