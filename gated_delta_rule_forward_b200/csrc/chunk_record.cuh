// Layout of the per-(batch, head, chunk) record that the chunked kernels pass
// through the workspace: fp16 tiles stored as images of the 128-byte-swizzled
// shared-memory layout (rows of 64 elements, 16-byte chunks XOR-ed with the
// row index mod 8), so that a record is bulk-copied into shared memory
// unchanged and read there by the tensor-core MMAs.
//     REC_WQ  [-W 0-63 | Qg 0-63 | -W 64-127 | Qg 64-127], rows t        32 KB
//     REC_K   Kt, rows t, d_k atoms [0-63 | 64-127]                        16 KB
//     REC_P   P, rows t, columns r                                          8 KB
//     REC_U   U'^T, rows v, columns t                           8 KB per 64 values
//     rec_sc  fp32 Gamma_C: one value padded to 16 bytes, or d_k values
//     GDN-2 only, unswizzled: (P^d V)^T [v][t] (8 KB per 64 values), then
//             (Dt^T V)^T [v][i] (16 KB per 64 values)
#pragma once

#include <cstdint>

namespace gdr {
namespace tc {

constexpr int C = 64;     // tokens per chunk
constexpr int DK = 128;   // key width of the chunked kernels

constexpr uint32_t REC_WQ = 0;
constexpr uint32_t REC_K = 32768;
constexpr uint32_t REC_P = 49152;
constexpr uint32_t REC_U = 57344;
__host__ __device__ constexpr uint32_t rec_sc(int ns) { return REC_U + 8192 * ns; }
__host__ __device__ constexpr uint32_t rec_bytes(int ns) { return rec_sc(ns) + 16; }
// channel decay: Gamma_C is a vector of d_k = 128 floats
__host__ __device__ constexpr uint32_t rec_bytes_chan(int ns) { return rec_sc(ns) + 4 * 128; }
// GDN-2: the channel-decay record, then (P^d V)^T (8 KB per 64 values) and (Dt^T V)^T (16 KB per 64 values)
__host__ __device__ constexpr uint32_t rec_bytes_gdn2(int ns) { return rec_bytes_chan(ns) + 24576 * ns; }

}  // namespace tc
}  // namespace gdr
