// la_tc.cu -- tensor-core path dispatch.
#include "la_tc.cuh"

namespace la {
namespace tc {

bool supports(const Shape &, la_dtype) { return false; }
size_t workspace_size(la_op, const Shape &, la_dtype) { return 0; }
la_status state_fwd(bool, const void *, const void *, const void *, void *, float *, const Shape &, la_dtype, float,
                    void *, cudaStream_t) {
    return LA_ERR_UNSUPPORTED;
}
la_status state_bwd(bool, const void *, const void *, const void *, const void *, const float *, void *, void *,
                    void *, const Shape &, la_dtype, float, void *, cudaStream_t) {
    return LA_ERR_UNSUPPORTED;
}
la_status decay_fwd(const void *, const void *, const void *, void *, const DecayArgs &, const Shape &, la_dtype,
                    void *, cudaStream_t) {
    return LA_ERR_UNSUPPORTED;
}
la_status decay_bwd(const void *, const void *, const void *, const void *, const DecayArgs &, void *, void *, void *,
                    const Shape &, la_dtype, void *, cudaStream_t) {
    return LA_ERR_UNSUPPORTED;
}

}  // namespace tc
}  // namespace la
