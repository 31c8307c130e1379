// Chunked tensor-core forward (tcgen05 + TMEM + TMA, chunk C = 64, bf16 I/O).
#pragma once
#include <string>

#include "common.cuh"

// True when the chunked kernel covers (variant, dk, dv) with bf16 I/O.
bool gdr_chunk_tc_supported(int variant, int dk, int dv);
// Kernel launches one forward call makes on this path.
int gdr_chunk_tc_launches(int B, int T, int H, int dk, int dv);
// Enqueue the forward; on failure *err names the failing step.
cudaError_t gdr_launch_chunk_tc(const gdr::FwdProblem &p, cudaStream_t stream, std::string *err);
// Synchronise `stream`, then read and clear the device error word (1 when a
// bounded wait inside a kernel gave up, 0 otherwise, -1 on a CUDA error).
int gdr_read_device_error(cudaStream_t stream);
// Channel-wise decay kernel (chunk_tc_chan.cu) and its error word.
cudaError_t gdr_launch_chunk_chan(const gdr::FwdProblem &p, cudaStream_t stream, std::string *err);
int gdr_read_chan_error();
// Two-kernel path (chunk_split.cu): chunk-parallel preparation + sequential carry.
bool gdr_split_supported(int variant, int dk, int dv);
size_t gdr_split_workspace_bytes(int variant, int B, int T, int H, int dv);
size_t gdr_split_record_bytes(int variant, int dv);   // bytes of one (b, h, chunk) record
int gdr_split_launches(int variant, int B, int T, int H, int dv);   // kernel launches of one two-kernel-path call
// The two-kernel path's schedule on a device with `sms` SMs (no device query).
void gdr_split_plan(int variant, int B, int T, int H, int dv, int sms, int *segments, int *segment_chunks,
                    int *split_chunk);
// ws_bytes: the workspace at ws; a segmented plan that needs more runs unsegmented.
cudaError_t gdr_launch_split(const gdr::FwdProblem &p, void *ws, size_t ws_bytes, cudaStream_t stream,
                             std::string *err);
int gdr_read_split_error();
// Fixed scratch of the no-allocation entry point (chunk_split.cu).
size_t gdr_split_fixed_scratch_bytes();
cudaError_t gdr_split_fixed_scratch(void **ptr);
