// Dispatch to the tensor-core (tcgen05) kernels: which problems they take and
// how they are launched.
#include "jfa_common.cuh"

namespace jfa {

cudaError_t tc_forward_launch(const jfa_problem& p, const AttnArgs& a, cudaStream_t st);
cudaError_t tc_backward_launch(const jfa_problem& p, const AttnArgs& a, const AttnArgs& kv,
                               cudaStream_t st);

// bf16 storage, head_dim 128, any activation and bias kind.
bool tc_supported(const jfa_problem& p, int act, int backward) {
    (void)act;
    (void)backward;
    return p.dtype == JFA_BF16 && p.head_dim == 128;
}

// The backward keeps an fp32 dQ accumulator [total_q][heads][128].
size_t tc_workspace_extra(const jfa_problem& p, int backward) {
    if (!backward) return 0;
    return sizeof(float) * (size_t)p.total_q * p.heads * p.head_dim;
}

cudaError_t tc_forward(const jfa_problem& p, const AttnArgs& a, void*, cudaStream_t st) {
    return tc_forward_launch(p, a, st);
}

cudaError_t tc_backward(const jfa_problem& p, const AttnArgs& a, const AttnArgs& kv,
                        void* ws_extra, cudaStream_t st) {
    AttnArgs aq = a, akv = kv;
    aq.dq_acc = reinterpret_cast<float*>(ws_extra);
    akv.dq_acc = aq.dq_acc;
    return tc_backward_launch(p, aq, akv, st);
}

int tc_fwd_tile() { return 128; }
int tc_bwd_tile() { return 128; }

}  // namespace jfa
