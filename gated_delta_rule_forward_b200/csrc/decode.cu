// Single-token recurrent decode of the gated delta rule (bandwidth-bound).
//
// Per (sequence, head) the fp32 state S [dk][dv] is read once and written
// once; everything else (q, k, v, gates, o) is ~1% of the bytes.  One CTA of
// 256 threads owns one (sequence, head):
//   - thread (rg, cq): cq = tid % (dv/4) picks four adjacent value columns,
//     rg = tid / (dv/4) picks the rows rg, rg + RG, rg + 2 RG, ... so that
//     every warp reads and writes whole 512-byte state rows with float4
//     accesses (fully coalesced), and all of a thread's loads are issued
//     before any is used (dk*dv/256 floats in flight per thread);
//   - x = S~^T k and y = S~^T q are reduced in the same pass: per-thread
//     partial sums, then one shared-memory reduction across row groups;
//   - the update S = S~ - a x^T + c v^T is written straight from registers
//     (in place) and o = scale * (y - (a.q) x + (c.q) v).
// Recurrence as in "Kaczmarz Linear Attention" (KLA update rule) and the
// erase/write reading of "Gated DeltaNet-2" (technical core).  In the raw-input
// mode q and k are scaled to unit norm and the gates taken from their logits
// on the load path (a few hundred bytes beside the 128 KB state stream).
#include "common.cuh"

namespace gdr {
namespace {

constexpr int kDecodeThreads = 256;

template <int DK, int DV, typename IO, int VAR>
__global__ void __launch_bounds__(kDecodeThreads, 2) decode_kernel(const DecodeProblem p) {
  constexpr int TPR = DV / 4;                   // threads per state row
  constexpr int RG = kDecodeThreads / TPR;      // row groups
  constexpr int RPT = DK / RG;                  // rows per thread
  static_assert(RPT >= 1 && DK % RG == 0, "shape");
  __shared__ float kf[DK], qf[DK], gf[DK], af[DK], cf[DK];
  __shared__ float vf[DV];
  __shared__ __align__(16) float red_x[RG][DV];
  __shared__ __align__(16) float red_y[RG][DV];

  const int tid = threadIdx.x;
  const int cq = tid % TPR, rg = tid / TPR;
  const long nh = blockIdx.x;
  float4 *__restrict__ st = reinterpret_cast<float4 *>(p.state + (size_t)nh * DK * DV);

  // 1. issue every state load of this thread first
  float4 s[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) s[r] = st[(size_t)(rg + RG * r) * (DV / 4) + cq];

  // 2. small vectors into shared memory (fp32)
  const IO *q = static_cast<const IO *>(p.q) + nh * DK;
  const IO *k = static_cast<const IO *>(p.k) + nh * DK;
  const IO *v = static_cast<const IO *>(p.v) + nh * DV;
  const bool raw = p.raw;
  __shared__ float inv_qk[2];
  if (raw && tid < 64) {   // raw-input mode: warp 0 sums q^2, warp 1 k^2
    const IO *x = tid < 32 ? q : k;
    float ss = 0.f;
    for (int i = tid & 31; i < DK; i += 32) {
      const float e = ld_io<IO>(x + i);
      ss = fmaf(e, e, ss);
    }
    ss = warp_sum(ss);
    if ((tid & 31) == 0) inv_qk[tid >> 5] = (tid >= 32 && VAR == kKLA) ? 1.f : raw_inv_norm(ss);
  }
  if (raw) __syncthreads();
  if (tid < DK) {
    const float kk = ld_io<IO>(k + tid) * (raw ? inv_qk[1] : 1.f);
    kf[tid] = kk;
    qf[tid] = ld_io<IO>(q + tid) * (raw ? inv_qk[0] : 1.f);
    if constexpr (scalar_decay(VAR) || channel_decay(VAR)) {
      const float lg = __ldg(p.log_g + (scalar_decay(VAR) ? nh : nh * DK + tid));
      gf[tid] = expf(raw ? raw_log_decay(lg) : lg);
    } else {
      gf[tid] = 1.f;
    }
    if constexpr (VAR == kGDN2) {
      const float eb = __ldg(p.erase_b + nh * DK + tid), ww = __ldg(p.write_w + nh * DK + tid);
      af[tid] = (raw ? raw_gate(eb) : eb) * kk;
      cf[tid] = (raw ? raw_gate(ww) : ww) * kk;
    }
  }
  if (tid < DV) vf[tid] = ld_io<IO>(v + tid);
  __syncthreads();

  // 3. per-warp scalar dot products over dk: (k.q, k.k) or ((b.k).q, (w.k).q)
  const int lane = tid & 31;
  float s1 = 0.f, s2 = 0.f;
#pragma unroll
  for (int i = lane; i < DK; i += 32) {
    if constexpr (VAR == kGDN2) {
      s1 = fmaf(af[i], qf[i], s1);
      s2 = fmaf(cf[i], qf[i], s2);
    } else {
      s1 = fmaf(kf[i], qf[i], s1);
      s2 = fmaf(kf[i], kf[i], s2);
    }
  }
  s1 = warp_sum(s1);
  s2 = warp_sum(s2);
  float step = 0.f;
  if constexpr (VAR != kGDN2) {
    step = __ldg(p.beta + nh);                        // beta, or eta for KLA
    if (raw) step = raw_gate(step);
    if constexpr (VAR == kKLA) step = step / (s2 + p.eps);
  }

  // 4. decay and partial readouts over this thread's rows
  float px[4] = {0.f, 0.f, 0.f, 0.f}, py[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const int i = rg + RG * r;
    const float g = gf[i], ki = kf[i], qi = qf[i];
    s[r].x *= g; s[r].y *= g; s[r].z *= g; s[r].w *= g;
    px[0] = fmaf(s[r].x, ki, px[0]); px[1] = fmaf(s[r].y, ki, px[1]);
    px[2] = fmaf(s[r].z, ki, px[2]); px[3] = fmaf(s[r].w, ki, px[3]);
    py[0] = fmaf(s[r].x, qi, py[0]); py[1] = fmaf(s[r].y, qi, py[1]);
    py[2] = fmaf(s[r].z, qi, py[2]); py[3] = fmaf(s[r].w, qi, py[3]);
  }
  reinterpret_cast<float4 *>(red_x[rg])[cq] = make_float4(px[0], px[1], px[2], px[3]);
  reinterpret_cast<float4 *>(red_y[rg])[cq] = make_float4(py[0], py[1], py[2], py[3]);
  __syncthreads();
  float x[4] = {0.f, 0.f, 0.f, 0.f}, y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int g = 0; g < RG; ++g) {
    const float4 a = reinterpret_cast<const float4 *>(red_x[g])[cq];
    const float4 bq = reinterpret_cast<const float4 *>(red_y[g])[cq];
    x[0] += a.x; x[1] += a.y; x[2] += a.z; x[3] += a.w;
    y[0] += bq.x; y[1] += bq.y; y[2] += bq.z; y[3] += bq.w;
  }
  const float4 v4 = reinterpret_cast<const float4 *>(vf)[cq];
  const float vv[4] = {v4.x, v4.y, v4.z, v4.w};

  // 5. write the updated state from registers
  if constexpr (VAR == kGDN2) {
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
      const int i = rg + RG * r;
      const float a = af[i], c = cf[i];
      s[r].x = fmaf(-a, x[0], fmaf(c, vv[0], s[r].x));
      s[r].y = fmaf(-a, x[1], fmaf(c, vv[1], s[r].y));
      s[r].z = fmaf(-a, x[2], fmaf(c, vv[2], s[r].z));
      s[r].w = fmaf(-a, x[3], fmaf(c, vv[3], s[r].w));
      st[(size_t)i * (DV / 4) + cq] = s[r];
    }
  } else {
    const float e[4] = {vv[0] - x[0], vv[1] - x[1], vv[2] - x[2], vv[3] - x[3]};
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
      const int i = rg + RG * r;
      const float a = step * kf[i];
      s[r].x = fmaf(a, e[0], s[r].x);
      s[r].y = fmaf(a, e[1], s[r].y);
      s[r].z = fmaf(a, e[2], s[r].z);
      s[r].w = fmaf(a, e[3], s[r].w);
      st[(size_t)i * (DV / 4) + cq] = s[r];
    }
  }

  // 6. output
  if (rg == 0) {
    IO *o = static_cast<IO *>(p.o) + nh * DV + 4 * cq;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float out;
      if constexpr (VAR == kGDN2) out = y[c] - s1 * x[c] + s2 * vv[c];
      else out = fmaf(step * s1, vv[c] - x[c], y[c]);
      st_io<IO>(o + c, p.scale * out);
    }
  }
}

template <int DK, int DV, typename IO>
cudaError_t launch_shape(const DecodeProblem &p, cudaStream_t s) {
  const dim3 grid((unsigned)((long)p.N * p.H)), block(kDecodeThreads);
  switch (p.variant) {
    case kDeltaNet: decode_kernel<DK, DV, IO, kDeltaNet><<<grid, block, 0, s>>>(p); break;
    case kGatedDeltaNet: decode_kernel<DK, DV, IO, kGatedDeltaNet><<<grid, block, 0, s>>>(p); break;
    case kKDA: decode_kernel<DK, DV, IO, kKDA><<<grid, block, 0, s>>>(p); break;
    case kGDN2: decode_kernel<DK, DV, IO, kGDN2><<<grid, block, 0, s>>>(p); break;
    case kKLA: decode_kernel<DK, DV, IO, kKLA><<<grid, block, 0, s>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

template <typename IO>
cudaError_t launch_io(const DecodeProblem &p, cudaStream_t s) {
  if (p.dk == 128 && p.dv == 128) return launch_shape<128, 128, IO>(p, s);
  if (p.dk == 128 && p.dv == 64) return launch_shape<128, 64, IO>(p, s);
  if (p.dk == 64 && p.dv == 128) return launch_shape<64, 128, IO>(p, s);
  if (p.dk == 64 && p.dv == 64) return launch_shape<64, 64, IO>(p, s);
  return cudaErrorInvalidValue;
}

}  // namespace
}  // namespace gdr

cudaError_t gdr_launch_decode(const gdr::DecodeProblem &p, cudaStream_t s) {
  return p.bf16_io ? gdr::launch_io<__nv_bfloat16>(p, s) : gdr::launch_io<float>(p, s);
}
