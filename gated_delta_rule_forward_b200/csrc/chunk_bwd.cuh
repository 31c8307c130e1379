// Chunked backward of the five variants: its chunk-parallel kernels
// (chunk_bwd.cu) and the orchestration over the forward's preparation and
// carry kernels (chunk_split.cu).
#pragma once
#include <cstdint>
#include <string>
#include <cuda_fp16.h>

#include "common.cuh"

namespace gdr {

struct BwdProblem {
  FwdProblem f;            // the forward's inputs and shape (f.o and f.s_final unused)
  const void *d_o;         // [B,T,H,dv] I/O dtype: gradient of the outputs
  const float *d_final;    // [B,H,dk,dv] gradient of the final state, or null (zero)
  void *dq, *dk, *dv;      // [B,T,H,dk], [B,T,H,dk], [B,T,H,dv] I/O dtype
  float *dbeta;            // [B,T,H]: d beta, or d eta for KLA; null for GDN-2
  float *dlog_g;           // [B,T,H] (GDN, KLA) or [B,T,H,dk] (KDA, GDN-2); null for DeltaNet
  float *d_s0;             // [B,H,dk,dv] gradient of the initial state, or null
  float *d_erase, *d_write;   // [B,T,H,dk] GDN-2's erase and write gate gradients
};

// Byte offsets of the backward's workspace regions (each 256-byte aligned).
struct BwdLayout {
  size_t fwd_rec;   // the forward's per-chunk records
  size_t rev_rec;   // the reverse carry's records, chunks in reverse order
  size_t s0s;       // start state of every chunk   [B,H,NC,dk,dv] fp16 (KDA: fp32)
  size_t dss;       // end-state gradient (scaled), reverse chunk order [B,H,NC,dk,dv] fp32
  size_t x0, xf;    // reverse carry's start (scaled d_final) and end (scaled d_s0) [B,H,dk,dv]
  size_t maps, maps_bytes;   // the segmented carries' maps and start states (0 bytes: unsegmented)
  size_t absmax;    // the gradients' magnitude (one fp32 word)
  size_t total;
};
BwdLayout bwd_layout(int variant, int B, int T, int H, int dv);

}  // namespace gdr

// The backward covers all five variants with bf16 I/O, dk = 128 and dv in
// {64, 128}.
bool gdr_bwd_supported(int variant, int dtype_bf16, int dk, int dv);
size_t gdr_bwd_workspace_bytes(int variant, int B, int T, int H, int dv);

// The steps after the forward records and chunk states exist.  `absmax`,
// `x0`, `xf`, the record and state pointers are regions of the workspace.
cudaError_t gdr_bwd_launch_scale(const gdr::BwdProblem &p, uint32_t *absmax, float *x0, cudaStream_t s);
cudaError_t gdr_bwd_launch_rev_prep(const gdr::BwdProblem &p, const uint8_t *fwd_rec, uint8_t *rev_rec,
                                    const uint32_t *absmax, cudaStream_t s);
// GDN-2 uses each chunk's slots of the forward and reverse records (dead by
// then) as scratch.
cudaError_t gdr_bwd_launch_local(const gdr::BwdProblem &p, const void *s0s, const float *dss,
                                  const uint32_t *absmax, uint8_t *fwd_rec, uint8_t *rev_rec, cudaStream_t s);
cudaError_t gdr_bwd_launch_unscale(const gdr::BwdProblem &p, const float *xf, const uint32_t *absmax,
                                   cudaStream_t s);
// Read and clear this file's device error word (bit 1: an fp16 operand of the
// reverse records left its range).  Synchronises `s`; -1 on a CUDA error.
int gdr_bwd_read_device_error(cudaStream_t s);

// The whole backward (chunk_split.cu): the forward's preparation and a carry
// that keeps every chunk's start state, the reverse records, the reverse carry,
// the chunk-local gradients.
cudaError_t gdr_launch_backward(const gdr::BwdProblem &p, void *ws, size_t ws_bytes, cudaStream_t s,
                                std::string *err);
