// Persistent tcgen05 block-sparse attention kernel (placeholder until the
// tensor-core kernel lands: the launcher reports "not supported").
#include "bsa_internal.cuh"

namespace bsa {

cudaError_t launch_attn_tc(const bsa_plan& p, const void* qp, const void* kp, const void* vp,
                           const int32_t* row_ptr, const int32_t* col_idx, const int32_t* work,
                           int32_t* counter, void* o, cudaStream_t s) {
    (void)p; (void)qp; (void)kp; (void)vp; (void)row_ptr; (void)col_idx; (void)work;
    (void)counter; (void)o; (void)s;
    return cudaErrorNotSupported;
}

}  // namespace bsa
