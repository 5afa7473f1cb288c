// Tensor-core (tcgen05) kernels.  Placeholder until the sm_100a kernels land:
// every problem runs on the CUDA-core kernels.
#include "jfa_common.cuh"

namespace jfa {
bool tc_supported(const jfa_problem&, int, int) { return false; }
size_t tc_workspace_extra(const jfa_problem&, int) { return 0; }
cudaError_t tc_forward(const jfa_problem&, const AttnArgs&, void*, cudaStream_t) { return cudaErrorNotSupported; }
cudaError_t tc_backward(const jfa_problem&, const AttnArgs&, const AttnArgs&, void*, cudaStream_t) { return cudaErrorNotSupported; }
int tc_fwd_tile() { return 128; }
int tc_bwd_tile() { return 128; }
}  // namespace jfa
