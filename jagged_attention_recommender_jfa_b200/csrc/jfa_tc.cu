// Dispatch to the tensor-core (tcgen05) kernels: which problems they take and
// how they are launched.
#include "jfa_common.cuh"

namespace jfa {

cudaError_t tc_forward_launch(const jfa_problem& p, const AttnArgs& a, cudaStream_t st);

// Forward: bf16 storage, head_dim 128, any activation and bias kind.
bool tc_supported(const jfa_problem& p, int act, int backward) {
    (void)act;
    if (backward) return false;
    return p.dtype == JFA_BF16 && p.head_dim == 128;
}

size_t tc_workspace_extra(const jfa_problem&, int) { return 0; }

cudaError_t tc_forward(const jfa_problem& p, const AttnArgs& a, void*, cudaStream_t st) {
    return tc_forward_launch(p, a, st);
}

cudaError_t tc_backward(const jfa_problem&, const AttnArgs&, const AttnArgs&, void*, cudaStream_t) {
    return cudaErrorNotSupported;
}

int tc_fwd_tile() { return 128; }
int tc_bwd_tile() { return 128; }

}  // namespace jfa
