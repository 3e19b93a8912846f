// la_tc.cu -- which ops and shapes the tensor-core path covers, and its workspace.
#include "la_tc.cuh"

namespace la {
namespace tc {

bool supports(la_op op, const Shape &s, la_dtype dt) {
    if (dt != LA_F16 && dt != LA_BF16) return false;
    switch (op) {
    case LA_OP_BIDIR_FWD:
    case LA_OP_BIDIR_BWD:
    case LA_OP_SIMPLE_FWD:
    case LA_OP_SIMPLE_BWD:
    case LA_OP_STATE_REDUCE:
    case LA_OP_STATE_APPLY:
    case LA_OP_STATE_BWD_Q:
    case LA_OP_STATE_BWD_KV: return s.D == 64;
    case LA_OP_CHUNK_DECAY_FWD:
    case LA_OP_CHUNK_DECAY_BWD: return s.D == 64 || s.D == 128;
    case LA_OP_CAUSAL_NORM_FWD:
    case LA_OP_CAUSAL_NORM_BWD: return causal_norm_supported(s, dt);
    default: return false;
    }
}

unsigned int read_and_clear_fault() {
    const unsigned int a = read_and_clear_state_fault(), b = read_and_clear_retention_fault(),
                       c = read_and_clear_debug_fault();
    if (a == 0xFFFFFFFFu || b == 0xFFFFFFFFu || c == 0xFFFFFFFFu) return 0xFFFFFFFFu;
    return a | b | c;
}

size_t workspace_size(la_op op, const Shape &s, la_dtype) {
    switch (op) {
    case LA_OP_BIDIR_FWD:
    case LA_OP_BIDIR_BWD:
    case LA_OP_SIMPLE_FWD:
    case LA_OP_SIMPLE_BWD:
    case LA_OP_STATE_REDUCE:
    case LA_OP_STATE_BWD_Q: return state_workspace_size(op, s);
    case LA_OP_CAUSAL_NORM_FWD:
    case LA_OP_CAUSAL_NORM_BWD: return causal_norm_workspace(op, s, true);   // the larger, with elu + 1
    default: return 0;
    }
}

la_status decay_fwd(const void *q, const void *k, const void *v, void *o, const float *sin, float *sout,
                    const DecayArgs &dec, const Shape &s, la_dtype dt, void *, cudaStream_t st) {
    return retention_fwd(q, k, v, o, sin, sout, dec, s, dt == LA_BF16, st);
}
la_status decay_bwd(const void *q, const void *k, const void *v, const void *g, const float *sin, const float *rin,
                    float *rout, const DecayArgs &dec, void *dq, void *dk, void *dv, const Shape &s, la_dtype dt,
                    void *, cudaStream_t st) {
    return retention_bwd(q, k, v, g, sin, rin, rout, dec, dq, dk, dv, s, dt == LA_BF16, st);
}

}  // namespace tc
}  // namespace la
