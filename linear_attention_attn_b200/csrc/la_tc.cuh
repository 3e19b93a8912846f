// la_tc.cuh -- the tensor-core (tcgen05 / TMA) path for fp16 and bf16 (not part of the ABI).
#pragma once

#include "la_internal.cuh"

namespace la {
namespace tc {

// True when the tensor-core kernels cover this op, shape and dtype.
bool supports(la_op op, const Shape &s, la_dtype dt);
size_t workspace_size(la_op op, const Shape &s, la_dtype dt);
size_t state_workspace_size(la_op op, const Shape &s);
// Fault word of the tensor-core kernels (nonzero when a wait ran out); cleared on read.
unsigned int read_and_clear_fault();
la_status state_fwd(bool bidir, const void *q, const void *k, const void *v, void *o, float *state,
                    const Shape &s, la_dtype dt, float eps, void *ws, cudaStream_t st);
la_status state_bwd(bool bidir, const void *q, const void *k, const void *v, const void *g,
                    const float *state, void *dq, void *dk, void *dv, const Shape &s, la_dtype dt,
                    float eps, void *ws, cudaStream_t st);
la_status decay_fwd(const void *q, const void *k, const void *v, void *o, const DecayArgs &dec,
                    const Shape &s, la_dtype dt, void *ws, cudaStream_t st);
la_status decay_bwd(const void *q, const void *k, const void *v, const void *g, const DecayArgs &dec,
                    void *dq, void *dk, void *dv, const Shape &s, la_dtype dt, void *ws, cudaStream_t st);

}  // namespace tc
}  // namespace la
