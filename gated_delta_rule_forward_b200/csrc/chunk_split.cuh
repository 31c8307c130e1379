// Chunked tensor-core forward (tcgen05 + TMEM + TMA, chunk C = 64, bf16 I/O):
// chunk-parallel preparation kernels and the sequential carry (chunk_split.cu).
#pragma once
#include <string>

#include "common.cuh"

// Synchronise `stream`, then read and clear the device error word (bit 0: a
// bounded wait inside a kernel gave up; bit 1: an operand left its range; -1
// on a CUDA error).
int gdr_read_device_error(cudaStream_t stream);
bool gdr_split_supported(int variant, int dk, int dv);
size_t gdr_split_workspace_bytes(int variant, int B, int T, int H, int dv);
size_t gdr_split_record_bytes(int variant, int dv);   // bytes of one (b, h, chunk) record
// Bytes of the segmented carry's maps, offsets and start states on the current device (0 when not segmented).
size_t gdr_split_segment_bytes(int B, int T, int H, int dv);
int gdr_split_launches(int variant, int B, int T, int H, int dv);   // kernel launches of one two-kernel-path call
// The two-kernel path's schedule on a device with `sms` SMs (no device query);
// parts / part_chunks (either may be null): the segmented carry's second phase.
void gdr_split_plan(int variant, int B, int T, int H, int dv, int sms, int *segments, int *segment_chunks,
                    int *split_chunk, int *parts = nullptr, int *part_chunks = nullptr);
// ws_bytes: the workspace at ws; a segmented plan that needs more runs unsegmented.
cudaError_t gdr_launch_split(const gdr::FwdProblem &p, void *ws, size_t ws_bytes, cudaStream_t stream,
                             std::string *err);
// Fixed scratch of the no-allocation entry point (chunk_split.cu).
size_t gdr_split_fixed_scratch_bytes();
cudaError_t gdr_split_fixed_scratch(void **ptr);
