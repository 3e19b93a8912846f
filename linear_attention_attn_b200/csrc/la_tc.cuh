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
la_status retention_map_f32(CUtensorMap *m, void *ptr, const Shape &s);
// Chunked causal decay forward on tensor cores (bf16 or fp16 storage, D = 64 or 128).
la_status retention_fwd(const void *q, const void *k, const void *v, void *o, const float *sin, float *sout,
                        const DecayArgs &dec, const Shape &s, bool bf16, cudaStream_t st);
// sin: state S entering the segment (or null); rin: R = sum_{t >= end} gamma^(t-end) q_t^T dO_t
// entering from the right (or null); rout: R at the segment's first row (or null).  [BH, D, D].
// dq32, dk32 (or null; D = 64 only): dq and dk written in fp32 there instead of dq, dk.
la_status retention_bwd(const void *q, const void *k, const void *v, const void *g, const float *sin,
                        const float *rin, float *rout, const DecayArgs &dec, void *dq, void *dk, void *dv,
                        const Shape &s, bool bf16, cudaStream_t st, float *dq32 = nullptr, float *dk32 = nullptr);
// Causal linear attention with the norm term on features q, k formed by the caller (D = 64):
// o_t = q_t S_t / n_t with n_t = q_t . z_t + eps.  With dout not null, o receives
// du = dout / n instead and dn (fp32 [BH, T]) -(dout . o) / n.
la_status retention_norm_fwd(const void *q, const void *k, const void *v, void *o, const void *dout, float *dn,
                             const DecayArgs &dec, float eps, const Shape &s, bool bf16, cudaStream_t st);
// Causal linear attention with the norm term (D = 64, fp16; has_decay = 0: gamma = 1; phi:
// f = elu + 1, else the identity); workspace causal_norm_workspace(op, s, phi) bytes.
bool causal_norm_supported(const Shape &s, la_dtype dt);
size_t causal_norm_workspace(la_op op, const Shape &s, bool phi);
la_status causal_norm_fwd(const void *q, const void *k, const void *v, void *o, const DecayArgs &dec, int has_decay,
                          bool phi, const Shape &s, la_dtype dt, float eps, void *ws, cudaStream_t st);
la_status causal_norm_bwd(const void *q, const void *k, const void *v, const void *dout, void *dq, void *dk,
                          void *dv, const DecayArgs &dec, int has_decay, bool phi, const Shape &s, la_dtype dt,
                          float eps, void *ws, cudaStream_t st);
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
