// la_tc.cuh -- the tensor-core (tcgen05 / TMA) path for fp16 and bf16 (not part of the ABI).
#pragma once

#include <cuda.h>

#include "la_internal.cuh"

namespace la {
namespace tc {

// True when the tensor-core kernels cover this op, shape and dtype.
bool supports(la_op op, const Shape &s, la_dtype dt);
size_t workspace_size(la_op op, const Shape &s, la_dtype dt);
size_t state_workspace_size(la_op op, const Shape &s);
// Fault word of the tensor-core kernels (nonzero when a wait ran out); cleared on read.
unsigned int read_and_clear_fault();
unsigned int read_and_clear_state_fault();
unsigned int read_and_clear_retention_fault();
unsigned int read_and_clear_debug_fault();

// [BH, T, D] 16-bit tensor map: boxes of box_rows x 64 columns, 128-byte swizzle.
la_status make_tensor_map(CUtensorMap *m, const void *ptr, const Shape &s, bool bf16, int box_rows);
la_status retention_map(CUtensorMap *m, const void *ptr, const Shape &s, bool bf16);
// Chunked causal decay forward on tensor cores (bf16 or fp16 storage, D = 64 or 128).
la_status retention_fwd(const void *q, const void *k, const void *v, void *o, const float *sin, float *sout,
                        const DecayArgs &dec, const Shape &s, bool bf16, cudaStream_t st);
// sin: state S entering the segment (or null); rin: R = sum_{t >= end} gamma^(t-end) q_t^T dO_t
// entering from the right (or null); rout: R at the segment's first row (or null).  [BH, D, D].
la_status retention_bwd(const void *q, const void *k, const void *v, const void *g, const float *sin,
                        const float *rin, float *rout, const DecayArgs &dec, void *dq, void *dk, void *dv,
                        const Shape &s, bool bf16, cudaStream_t st);
la_status state_fwd(bool bidir, const void *q, const void *k, const void *v, void *o, float *state,
                    const Shape &s, la_dtype dt, float eps, void *ws, cudaStream_t st);
la_status state_bwd(bool bidir, const void *q, const void *k, const void *v, const void *g,
                    const float *state, void *dq, void *dk, void *dv, const Shape &s, la_dtype dt,
                    float eps, void *ws, cudaStream_t st);
la_status decay_fwd(const void *q, const void *k, const void *v, void *o, const float *sin, float *sout,
                    const DecayArgs &dec, const Shape &s, la_dtype dt, void *ws, cudaStream_t st);
// One stage of the state form (Stage in la_internal.cuh).
la_status state_stage(Stage stage, la_feature f, const void *x, const void *y, const float *sin, float *sout,
                      void *out1, void *out2, const Shape &s, la_dtype dt, float eps, void *ws, cudaStream_t st);
la_status decay_bwd(const void *q, const void *k, const void *v, const void *g, const float *sin,
                    const float *rin, float *rout, const DecayArgs &dec, void *dq, void *dk, void *dv,
                    const Shape &s, la_dtype dt, void *ws, cudaStream_t st);

}  // namespace tc
}  // namespace la
