// Shared pieces of the chunked tensor-core kernels.
#pragma once

#include "common.cuh"
#include "tc_util.cuh"

namespace gdr {
namespace tc {

constexpr int LD = 72;   // row stride (floats) of A^T and T scratch: conflict-free MMA fragments

// Round to tf32 and keep as float: the solve stores its operands pre-rounded.
__device__ __forceinline__ float tf32r(float x) { return __uint_as_float(to_tf32(x)); }

// Raw-input mode: 1 / ||row|| (floored as raw_inv_norm does) of the 64 rows of
// a bf16 tile stored as two 64-element atoms of 128-byte swizzled rows (atom 1
// at atom0 + atom_stride), into out[0..63].  256 threads, four per row; every
// thread of the block must call it.
__device__ __forceinline__ void tile_row_inv_norms(const uint8_t *atom0, uint32_t atom_stride, float *out, int tid) {
  const int row = tid >> 2, qtr = tid & 3;
  const uint8_t *a = atom0 + (qtr >> 1) * atom_stride;
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    float x[8];
    unpack8(*reinterpret_cast<const uint4 *>(a + sw128(row, 4 * (qtr & 1) + j)), x);
#pragma unroll
    for (int e = 0; e < 8; ++e) ss = fmaf(x[e], x[e], ss);
  }
  ss += __shfl_xor_sync(0xffffffffu, ss, 1);
  ss += __shfl_xor_sync(0xffffffffu, ss, 2);
  if (qtr == 0) out[row] = raw_inv_norm(ss);
}

// T = (I + A)^{-1} for a strictly lower-triangular 64 x 64 A (C = 64), 16x16-blocked.
// At[r * LD + t] holds A[t][r] pre-rounded to tf32 (written by the caller); the
// result lands in Tf[m * LD + n] (rows m, columns n; the strictly upper part is
// scratch).  Diagonal blocks D_i by forward substitution (fp32, one thread per
// column); then, level by level (i - j = 1, 2, 3), X = sum_{l=j}^{i-1} A_il T_lj
// and T_ij = -D_i X with warp-level tf32 MMAs, one warp per 16x8 half block
// (X is parked in the unused upper block (j, i)).  Needs >= 6 warps; every
// thread of the block must call it (it contains block-wide barriers).
__device__ __forceinline__ void solve_unit_lower_64(const float *At, float *Tf, int tid, int warp, int lane) {
  if (tid < 64) {
    const int bk = tid >> 4, j = tid & 15, o = 16 * bk;
    float x[16];
#pragma unroll
    for (int m = 0; m < 16; ++m) x[m] = (m == j) ? 1.f : 0.f;
#pragma unroll
    for (int l = 0; l < 15; ++l) {
      const float xl = x[l];
      const float *col = At + (o + l) * LD + o;   // A[o + m][o + l], m = 0..15
#pragma unroll
      for (int m4 = 0; m4 < 16; m4 += 4) {
        if (m4 + 3 <= l) continue;
        const float4 a4 = *reinterpret_cast<const float4 *>(col + m4);
        if (m4 + 0 > l) x[m4 + 0] = fmaf(-a4.x, xl, x[m4 + 0]);
        if (m4 + 1 > l) x[m4 + 1] = fmaf(-a4.y, xl, x[m4 + 1]);
        if (m4 + 2 > l) x[m4 + 2] = fmaf(-a4.z, xl, x[m4 + 2]);
        if (m4 + 3 > l) x[m4 + 3] = fmaf(-a4.w, xl, x[m4 + 3]);
      }
    }
#pragma unroll
    for (int m = 0; m < 16; ++m) Tf[(o + m) * LD + o + j] = tf32r(x[m]);
  }
  __syncthreads();
  {
    const int fg = lane >> 2, ft = lane & 3;   // fragment row group / thread in group
#pragma unroll
    for (int lev = 1; lev <= 3; ++lev) {
      if (warp < 2 * (4 - lev)) {
        const int i = lev + (warp >> 1), jb = i - lev, nh = warp & 1;
        // X[:, half nh] = A[16i.., 16jb .. 16i) * T[16jb .. 16i, 16jb + 8nh ..]   (K = 16 lev)
        float xa[4] = {0.f, 0.f, 0.f, 0.f};
        const int nb = 16 * jb + 8 * nh + fg;
#pragma unroll
        for (int ks = 0; ks < 2 * lev; ++ks) {
          const int k0 = 16 * jb + 8 * ks;
          uint32_t a[4];
          a[0] = __float_as_uint(At[(k0 + ft) * LD + 16 * i + fg]);
          a[1] = __float_as_uint(At[(k0 + ft) * LD + 16 * i + fg + 8]);
          a[2] = __float_as_uint(At[(k0 + ft + 4) * LD + 16 * i + fg]);
          a[3] = __float_as_uint(At[(k0 + ft + 4) * LD + 16 * i + fg + 8]);
          mma_tf32_16x8x8(xa, a, __float_as_uint(Tf[(k0 + ft) * LD + nb]),
                          __float_as_uint(Tf[(k0 + ft + 4) * LD + nb]));
        }
        {
          const int n = 16 * i + 8 * nh + 2 * ft;     // scratch: upper block (jb, i)
          Tf[(16 * jb + fg) * LD + n] = tf32r(xa[0]);
          Tf[(16 * jb + fg) * LD + n + 1] = tf32r(xa[1]);
          Tf[(16 * jb + fg + 8) * LD + n] = tf32r(xa[2]);
          Tf[(16 * jb + fg + 8) * LD + n + 1] = tf32r(xa[3]);
        }
        __syncwarp();
        // T_ij[:, half nh] = -D_i X[:, half nh]   (K = 16)
        float ta[4] = {0.f, 0.f, 0.f, 0.f};
        const int nx = 16 * i + 8 * nh + fg;
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
          const int k0 = 8 * ks;
          uint32_t a[4];
          a[0] = __float_as_uint(-Tf[(16 * i + fg) * LD + 16 * i + k0 + ft]);
          a[1] = __float_as_uint(-Tf[(16 * i + fg + 8) * LD + 16 * i + k0 + ft]);
          a[2] = __float_as_uint(-Tf[(16 * i + fg) * LD + 16 * i + k0 + ft + 4]);
          a[3] = __float_as_uint(-Tf[(16 * i + fg + 8) * LD + 16 * i + k0 + ft + 4]);
          mma_tf32_16x8x8(ta, a, __float_as_uint(Tf[(16 * jb + k0 + ft) * LD + nx]),
                          __float_as_uint(Tf[(16 * jb + k0 + ft + 4) * LD + nx]));
        }
        {
          const int n = 16 * jb + 8 * nh + 2 * ft;
          Tf[(16 * i + fg) * LD + n] = tf32r(ta[0]);
          Tf[(16 * i + fg) * LD + n + 1] = tf32r(ta[1]);
          Tf[(16 * i + fg + 8) * LD + n] = tf32r(ta[2]);
          Tf[(16 * i + fg + 8) * LD + n + 1] = tf32r(ta[3]);
        }
      }
      __syncthreads();
    }
  }
}

}  // namespace tc
}  // namespace gdr
