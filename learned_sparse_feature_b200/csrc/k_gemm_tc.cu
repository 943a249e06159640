// tcgen05 (5th-generation tensor core) kernels: placeholder until the sm_100a
// GEMM and attention kernels land.
#include "sg_internal.cuh"

namespace sg {
bool tc_available() { return false; }
cudaError_t launch_gemm_tc(const GemmArgs&, int, int, cudaStream_t) { return cudaErrorNotSupported; }
cudaError_t launch_attention_tc(const AttnArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace sg
