// Device helpers shared by the libgdr kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdr {

// Variant ids, the same numbering as gdr_variant_t in include/gdr.h.
enum Variant : int { kDeltaNet = 0, kGatedDeltaNet = 1, kKDA = 2, kGDN2 = 3, kKLA = 4 };

__host__ __device__ constexpr bool scalar_decay(int v) { return v == kGatedDeltaNet || v == kKLA; }
__host__ __device__ constexpr bool channel_decay(int v) { return v == kKDA || v == kGDN2; }

// Problem description handed from the ABI layer to the launchers.  `raw`:
// q, k, beta and the gates arrive as raw projections and logits, and the
// kernels apply the input transforms on their load paths (see raw_* below).
struct FwdProblem {
  int variant, B, T, H, dk, dv;
  bool bf16_io, raw;
  const void *q, *k, *v;
  const float *beta, *log_g, *erase_b, *write_w;
  const float *s0;
  float *s_final;
  void *o;
  float eps, scale;
};

struct DecodeProblem {
  int variant, N, H, dk, dv;
  bool bf16_io, raw;
  const void *q, *k, *v;
  const float *beta, *log_g, *erase_b, *write_w;
  float *state;
  void *o;
  float eps, scale;
};

// ---- I/O element access -----------------------------------------------------
template <typename IO> __device__ __forceinline__ float ld_io(const IO *p);
template <> __device__ __forceinline__ float ld_io<float>(const float *p) { return __ldg(p); }
template <> __device__ __forceinline__ float ld_io<__nv_bfloat16>(const __nv_bfloat16 *p) {
  return __bfloat162float(__ldg(p));
}

template <typename IO> __device__ __forceinline__ void st_io(IO *p, float x);
template <> __device__ __forceinline__ void st_io<float>(float *p, float x) { *p = x; }
template <> __device__ __forceinline__ void st_io<__nv_bfloat16>(__nv_bfloat16 *p, float x) {
  *p = __float2bfloat16_rn(x);
}

// Load 8 consecutive I/O elements (16-byte aligned for bf16, 32-byte for fp32).
template <typename IO> __device__ __forceinline__ void ld8(const IO *p, float (&x)[8]);
template <> __device__ __forceinline__ void ld8<float>(const float *p, float (&x)[8]) {
  float4 a = __ldg(reinterpret_cast<const float4 *>(p));
  float4 b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
template <> __device__ __forceinline__ void ld8<__nv_bfloat16>(const __nv_bfloat16 *p, float (&x)[8]) {
  uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}

// Store 8 consecutive I/O elements.
template <typename IO> __device__ __forceinline__ void st8(IO *p, const float (&x)[8]);
template <> __device__ __forceinline__ void st8<float>(float *p, const float (&x)[8]) {
  reinterpret_cast<float4 *>(p)[0] = make_float4(x[0], x[1], x[2], x[3]);
  reinterpret_cast<float4 *>(p)[1] = make_float4(x[4], x[5], x[6], x[7]);
}
template <> __device__ __forceinline__ void st8<__nv_bfloat16>(__nv_bfloat16 *p, const float (&x)[8]) {
  uint4 u;
  __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
  *reinterpret_cast<uint4 *>(p) = u;
}

// Input transforms of the raw-input mode (the parameterisation the workloads
// use): a decay logit x gives log g = -softplus(x) (so g = sigmoid(-x) in
// (0, 1)); beta / eta and the GDN-2 erase and write gates are sigmoid of their
// logits; q and k are scaled to unit L2 norm (KLA's keys are not: its step
// eta / (||k||^2 + eps) carries their norm), with the norm floored at 1e-6.
__device__ __forceinline__ float raw_log_decay(float x) { return -(fmaxf(x, 0.f) + log1pf(expf(-fabsf(x)))); }
__device__ __forceinline__ float raw_gate(float x) { return 1.f / (1.f + expf(-x)); }
__device__ __forceinline__ float raw_inv_norm(float sumsq) { return 1.f / fmaxf(sqrtf(sumsq), 1e-6f); }

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

}  // namespace gdr

// Launchers implemented in the .cu files; each returns cudaGetLastError().
cudaError_t gdr_launch_token_forward(const gdr::FwdProblem &p, cudaStream_t stream);
cudaError_t gdr_launch_decode(const gdr::DecodeProblem &p, cudaStream_t stream);
