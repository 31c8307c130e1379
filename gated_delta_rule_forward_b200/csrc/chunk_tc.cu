#include "chunk_tc.cuh"

bool gdr_chunk_tc_supported(int, int, int) { return false; }
int gdr_chunk_tc_launches(int, int, int, int, int) { return 0; }
cudaError_t gdr_launch_chunk_tc(const gdr::FwdProblem &, cudaStream_t, std::string *err) {
  *err = "not built";
  return cudaErrorNotSupported;
}
