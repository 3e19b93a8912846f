// la_api.cu -- the C entry points: argument validation, workspace layout,
// path selection, launch accounting and the optional per-kernel timing.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <string>
#include <vector>

#include "la_internal.cuh"
#include "la_tc.cuh"

namespace la {

// ---------------------------------------------------------------- errors --

static thread_local std::string g_last_error;

void set_error(const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
}

la_status cuda_fail(cudaError_t e, const char *what) {
    set_error("%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
    return LA_ERR_CUDA;
}

la_status launch_fail(cudaError_t e, const char *what, const void *kernel, dim3 block, size_t smem) {
    cudaFuncAttributes fa;
    memset(&fa, 0, sizeof fa);
    cudaGetLastError();
    if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) cudaGetLastError();
    set_error("%s: %s (%s); block %u threads, %zu B dynamic shared memory; kernel: %d registers, "
              "%zu B local, %zu B static shared, at most %d threads",
              what, cudaGetErrorString(e), cudaGetErrorName(e), block.x * block.y * block.z, smem, fa.numRegs,
              (size_t)fa.localSizeBytes, (size_t)fa.sharedSizeBytes, fa.maxThreadsPerBlock);
    return LA_ERR_CUDA;
}

static la_status fail(la_status s, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

// ------------------------------------------------- launches and profiling --

static std::atomic<long long> g_launches{0};
static std::atomic<int> g_prof_on{0};

struct ProfEntry {
    const char *name;
    cudaEvent_t start, stop;
};
static std::mutex g_prof_mu;
static std::vector<ProfEntry> g_prof;            // recorded, not yet collected
static std::vector<cudaEvent_t> g_event_pool;     // reusable events
static thread_local const char *t_pending_name = nullptr;
static thread_local cudaEvent_t t_pending_start = nullptr;

static cudaEvent_t take_event() {
    {
        std::lock_guard<std::mutex> lk(g_prof_mu);
        if (!g_event_pool.empty()) {
            cudaEvent_t e = g_event_pool.back();
            g_event_pool.pop_back();
            return e;
        }
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

// Launches still to pass before the injected failure (-1: none armed).
static std::atomic<long long> g_fail_after{-1};

bool injected_launch_failure(const char *name) {
    long long n = g_fail_after.load(std::memory_order_relaxed);
    while (n >= 0) {
        if (g_fail_after.compare_exchange_weak(n, n - 1, std::memory_order_relaxed)) {
            if (n > 0) return false;
            set_error("%s: injected launch failure (la_debug_fail_launch)", name);
            return true;
        }
    }
    return false;
}

void prof_before(const char *name, cudaStream_t s) {
    t_pending_name = nullptr;
    if (!g_prof_on.load(std::memory_order_relaxed)) return;
    cudaEvent_t e = take_event();
    if (!e) return;
    cudaEventRecord(e, s);
    t_pending_name = name;
    t_pending_start = e;
}

void prof_after(cudaStream_t s) {
    if (!t_pending_name) return;
    cudaEvent_t e = take_event();
    if (!e) return;
    cudaEventRecord(e, s);
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof.push_back({t_pending_name, t_pending_start, e});
    t_pending_name = nullptr;
}

// ----------------------------------------------------- shapes / workspace --

int state_splits(const Shape &s, int rows_per_unit) {
    // Aim at about two CTAs per SM of a 148-SM part, never fewer rows per split
    // than one unit, never more than 64 splits.
    const long long target = 296;
    long long want = (target + s.BH() - 1) / s.BH();
    long long max_units = (s.T + rows_per_unit - 1) / rows_per_unit;
    if (want > max_units) want = max_units;
    if (want > 64) want = 64;
    if (want < 1) want = 1;
    return (int)want;
}

size_t state_bytes(const Shape &s, long long copies) {
    size_t b = (size_t)s.BH() * (size_t)copies * (size_t)s.D * (size_t)(s.D + 1) * sizeof(float);
    return (b + 255) & ~(size_t)255;
}

static thread_local bool t_allow_null = false;   // set while validating a T == 0 call

static bool path_tc(la_op op, const Shape &s, la_dtype dt) { return tc::supports(op, s, dt); }

static la_status validate(const Shape &s, la_dtype dt) {
    t_allow_null = (s.T == 0);
    if (s.B < 1 || s.H < 1 || s.T < 0) return fail(LA_ERR_INVALID_ARG, "B, H must be >= 1 and T >= 0");
    if (dt != LA_F32 && dt != LA_F16 && dt != LA_BF16) return fail(LA_ERR_UNSUPPORTED, "unknown dtype %d", (int)dt);
    if (s.D != 64 && s.D != 128) return fail(LA_ERR_UNSUPPORTED, "D must be 64 or 128 (got %d)", s.D);
    if ((double)s.B * s.H * s.T * s.D >= 2147483648.0)
        return fail(LA_ERR_UNSUPPORTED, "tensor too large (B*H*T*D must be < 2^31)");
    if (s.BH() > 65535) return fail(LA_ERR_UNSUPPORTED, "B*H must be <= 65535");
    return LA_OK;
}

static la_status check_ptr(const void *p, const char *name) {
    if (!p && t_allow_null) return LA_OK;
    if (!p) return fail(LA_ERR_INVALID_ARG, "%s is NULL", name);
    if (((uintptr_t)p) & 15) return fail(LA_ERR_ALIGNMENT, "%s is not 16-byte aligned", name);
    return LA_OK;
}

static size_t ws_size(la_op op, const Shape &s, la_dtype dt) {
    if (path_tc(op, s, dt)) return tc::workspace_size(op, s, dt);
    return simt::workspace_size(op, s);
}

static la_status check_ws(la_op op, const Shape &s, la_dtype dt, void *ws, size_t ws_bytes) {
    const size_t need = ws_size(op, s, dt);
    if (need == 0) return LA_OK;
    if (!ws) return fail(LA_ERR_WORKSPACE, "workspace is NULL but %zu bytes are needed", need);
    if (((uintptr_t)ws) & 255) return fail(LA_ERR_ALIGNMENT, "workspace is not 256-byte aligned");
    if (ws_bytes < need) return fail(LA_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", ws_bytes, need);
    return LA_OK;
}

#define LA_TRY(x)                     \
    do {                              \
        la_status _rc = (x);          \
        if (_rc != LA_OK) return _rc; \
    } while (0)

// Common front half of the bidir / simple entry points.
static la_status state_fwd_entry(bool bidir, const void *q, const void *k, const void *v, void *o, float *state,
                                 int B, int H, int T, int D, la_dtype dt, float eps, void *ws, size_t ws_bytes,
                                 void *stream) {
    const Shape s{B, H, T, D};
    const la_op op = bidir ? LA_OP_BIDIR_FWD : LA_OP_SIMPLE_FWD;
    LA_TRY(validate(s, dt));
    if (!(eps >= 0.f)) return fail(LA_ERR_INVALID_ARG, "eps must be >= 0");
    LA_TRY(check_ptr(q, "q"));
    LA_TRY(check_ptr(k, "k"));
    LA_TRY(check_ptr(v, "v"));
    LA_TRY(check_ptr(o, "o"));
    if (state && (((uintptr_t)state) & 15)) return fail(LA_ERR_ALIGNMENT, "state is not 16-byte aligned");
    LA_TRY(check_ws(op, s, dt, ws, ws_bytes));
    cudaStream_t st = (cudaStream_t)stream;
    if (T == 0) {
        if (state) {
            cudaError_t e = cudaMemsetAsync(state, 0, (size_t)s.BH() * D * (D + 1) * sizeof(float), st);
            if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(state)");
        }
        return LA_OK;
    }
    if (path_tc(op, s, dt)) return tc::state_fwd(bidir, q, k, v, o, state, s, dt, eps, ws, st);
    return simt::state_fwd(bidir, q, k, v, o, state, s, dt, eps, ws, st);
}

static la_status state_bwd_entry(bool bidir, const void *q, const void *k, const void *v, const void *g,
                                 const float *state, void *dq, void *dk, void *dv, int B, int H, int T, int D,
                                 la_dtype dt, float eps, void *ws, size_t ws_bytes, void *stream) {
    const Shape s{B, H, T, D};
    const la_op op = bidir ? LA_OP_BIDIR_BWD : LA_OP_SIMPLE_BWD;
    LA_TRY(validate(s, dt));
    if (!(eps >= 0.f)) return fail(LA_ERR_INVALID_ARG, "eps must be >= 0");
    LA_TRY(check_ptr(q, "q"));
    LA_TRY(check_ptr(k, "k"));
    LA_TRY(check_ptr(v, "v"));
    LA_TRY(check_ptr(g, "dout"));
    LA_TRY(check_ptr(dq, "dq"));
    LA_TRY(check_ptr(dk, "dk"));
    LA_TRY(check_ptr(dv, "dv"));
    if (state && (((uintptr_t)state) & 15)) return fail(LA_ERR_ALIGNMENT, "state is not 16-byte aligned");
    LA_TRY(check_ws(op, s, dt, ws, ws_bytes));
    if (T == 0) return LA_OK;
    cudaStream_t st = (cudaStream_t)stream;
    if (path_tc(op, s, dt)) return tc::state_bwd(bidir, q, k, v, g, state, dq, dk, dv, s, dt, eps, ws, st);
    return simt::state_bwd(bidir, q, k, v, g, state, dq, dk, dv, s, dt, eps, ws, st);
}

static la_status decay_args(const float *decay, int H, DecayArgs *out) {
    if (!decay) return fail(LA_ERR_INVALID_ARG, "decay is NULL");
    if (H > LA_MAX_DECAY_HEADS) return fail(LA_ERR_UNSUPPORTED, "H=%d exceeds %d for the decay op", H, LA_MAX_DECAY_HEADS);
    memset(out, 0, sizeof *out);
    for (int h = 0; h < H; ++h) {
        const float g = decay[h];
        if (!(g > 0.f && g <= 1.f)) return fail(LA_ERR_INVALID_ARG, "decay[%d]=%g is not in (0, 1]", h, (double)g);
        out->gamma[h] = g;
    }
    return LA_OK;
}

// Front half of the sequence-parallel stage entry points.
static la_status check_state(const void *p, const char *name) {
    if (!p) return fail(LA_ERR_INVALID_ARG, "%s is NULL", name);
    if (((uintptr_t)p) & 15) return fail(LA_ERR_ALIGNMENT, "%s is not 16-byte aligned", name);
    return LA_OK;
}

static la_status stage_entry(Stage stage, la_op op, la_feature f, const void *x, const void *y, const float *sin,
                             float *sout, void *out1, void *out2, int B, int H, int T, int D, la_dtype dt, float eps,
                             void *ws, size_t ws_bytes, void *stream) {
    const Shape s{B, H, T, D};
    LA_TRY(validate(s, dt));
    if (f != LA_FEATURE_IDENTITY && f != LA_FEATURE_ELU1 && f != LA_FEATURE_NORM)
        return fail(LA_ERR_UNSUPPORTED, "unknown feature map %d", (int)f);
    if (!(eps >= 0.f) || !isfinite(eps)) return fail(LA_ERR_INVALID_ARG, "eps must be finite and >= 0");
    const char *xn = stage == Stage::Reduce || stage == Stage::BwdKV ? "k" : "q";
    LA_TRY(check_ptr(x, xn));
    if (stage != Stage::Apply) LA_TRY(check_ptr(y, stage == Stage::BwdQ ? "dout" : "v"));
    if (sin) LA_TRY(check_state(sin, "state"));
    if (stage != Stage::Reduce && !sin) return fail(LA_ERR_INVALID_ARG, "state is NULL");
    if (stage == Stage::Reduce || stage == Stage::BwdQ) LA_TRY(check_state(sout, stage == Stage::Reduce ? "state" : "dstate"));
    if (stage != Stage::Reduce) LA_TRY(check_ptr(out1, stage == Stage::Apply ? "o" : (stage == Stage::BwdQ ? "dq" : "dk")));
    if (stage == Stage::BwdKV) LA_TRY(check_ptr(out2, "dv"));
    LA_TRY(check_ws(op, s, dt, ws, ws_bytes));
    cudaStream_t st = (cudaStream_t)stream;
    if (T == 0) {
        if (sout) {
            cudaError_t e = cudaMemsetAsync(sout, 0, state_bytes(s, 1), st);
            if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
        }
        return LA_OK;
    }
    if (path_tc(op, s, dt)) return tc::state_stage(stage, f, x, y, sin, sout, out1, out2, s, dt, eps, ws, st);
    return simt::state_stage(stage, f, x, y, sin, sout, out1, out2, s, dt, eps, ws, st);
}

}  // namespace la

using namespace la;

extern "C" {

size_t la_workspace_size(la_op op, int B, int H, int T, int D, la_dtype dtype) {
    const Shape s{B, H, T, D};
    if (s.B < 1 || s.H < 1 || s.T < 0 || (s.D != 64 && s.D != 128)) return 0;
    if (dtype != LA_F32 && dtype != LA_F16 && dtype != LA_BF16) return 0;
    if ((int)op < 0 || (int)op > (int)LA_OP_GATED_BWD) return 0;
    return ws_size(op, s, dtype);
}

la_status la_bidir_fwd(const void *q, const void *k, const void *v, void *o, float *state, int B, int H, int T,
                       int D, la_dtype dtype, float eps, void *workspace, size_t workspace_bytes, void *stream) {
    return state_fwd_entry(true, q, k, v, o, state, B, H, T, D, dtype, eps, workspace, workspace_bytes, stream);
}

la_status la_simple_fwd(const void *q, const void *k, const void *v, void *o, float *state, int B, int H, int T,
                        int D, la_dtype dtype, void *workspace, size_t workspace_bytes, void *stream) {
    return state_fwd_entry(false, q, k, v, o, state, B, H, T, D, dtype, 0.f, workspace, workspace_bytes, stream);
}

la_status la_bidir_bwd(const void *q, const void *k, const void *v, const void *dout, const float *state, void *dq,
                       void *dk, void *dv, int B, int H, int T, int D, la_dtype dtype, float eps, void *workspace,
                       size_t workspace_bytes, void *stream) {
    return state_bwd_entry(true, q, k, v, dout, state, dq, dk, dv, B, H, T, D, dtype, eps, workspace,
                           workspace_bytes, stream);
}

la_status la_simple_bwd(const void *q, const void *k, const void *v, const void *dout, const float *state, void *dq,
                        void *dk, void *dv, int B, int H, int T, int D, la_dtype dtype, void *workspace,
                        size_t workspace_bytes, void *stream) {
    return state_bwd_entry(false, q, k, v, dout, state, dq, dk, dv, B, H, T, D, dtype, 0.f, workspace,
                           workspace_bytes, stream);
}

static la_status decay_fwd_entry(const void *q, const void *k, const void *v, void *o, const float *sin, float *sout,
                                 const float *decay, int B, int H, int T, int D, la_dtype dtype, void *workspace,
                                 size_t workspace_bytes, void *stream, bool state_entry) {
    const Shape s{B, H, T, D};
    LA_TRY(validate(s, dtype));
    // o == NULL on the state entry point: the state only (q is then not read either)
    const bool sonly = state_entry && !o;
    if (sonly && !sout) return fail(LA_ERR_INVALID_ARG, "o and state_out are both NULL: nothing to compute");
    if (!sonly) LA_TRY(check_ptr(q, "q"));
    LA_TRY(check_ptr(k, "k"));
    LA_TRY(check_ptr(v, "v"));
    if (!sonly) LA_TRY(check_ptr(o, "o"));
    if (sin) LA_TRY(check_state(sin, "state_in"));
    if (sout) LA_TRY(check_state(sout, "state_out"));
    DecayArgs dec;
    LA_TRY(decay_args(decay, H, &dec));
    LA_TRY(check_ws(LA_OP_CHUNK_DECAY_FWD, s, dtype, workspace, workspace_bytes));
    cudaStream_t st = (cudaStream_t)stream;
    if (T == 0) {   // the state passes through unchanged
        if (!sout) return LA_OK;
        const size_t bytes = (size_t)s.BH() * D * D * sizeof(float);
        cudaError_t e = sin ? (sin == sout ? cudaSuccess : cudaMemcpyAsync(sout, sin, bytes, cudaMemcpyDeviceToDevice, st))
                            : cudaMemsetAsync(sout, 0, bytes, st);
        return e == cudaSuccess ? LA_OK : cuda_fail(e, "state copy");
    }
    if (path_tc(LA_OP_CHUNK_DECAY_FWD, s, dtype))
        return tc::decay_fwd(q, k, v, o, sin, sout, dec, s, dtype, workspace, st);
    return simt::decay_fwd(q, k, v, o, sin, sout, dec, s, dtype, st);
}

la_status la_chunk_decay_fwd(const void *q, const void *k, const void *v, void *o, const float *decay, int B, int H,
                             int T, int D, la_dtype dtype, void *workspace, size_t workspace_bytes, void *stream) {
    return decay_fwd_entry(q, k, v, o, nullptr, nullptr, decay, B, H, T, D, dtype, workspace, workspace_bytes, stream,
                           false);
}

la_status la_chunk_decay_fwd_state(const void *q, const void *k, const void *v, void *o, const float *state_in,
                                   float *state_out, const float *decay, int B, int H, int T, int D, la_dtype dtype,
                                   void *workspace, size_t workspace_bytes, void *stream) {
    return decay_fwd_entry(q, k, v, o, state_in, state_out, decay, B, H, T, D, dtype, workspace, workspace_bytes,
                           stream, true);
}

static la_status decay_bwd_entry(const void *q, const void *k, const void *v, const void *dout, const float *sin,
                                 const float *rin, float *rout, const float *decay, void *dq, void *dk, void *dv,
                                 int B, int H, int T, int D, la_dtype dtype, void *workspace, size_t workspace_bytes,
                                 void *stream, bool dq_optional) {
    const Shape s{B, H, T, D};
    LA_TRY(validate(s, dtype));
    // dq, dk and dv all NULL on the state entry point: R at the first row only (k, v not read)
    const bool sonly = dq_optional && !dq && !dk && !dv;
    if (sonly && !rout) return fail(LA_ERR_INVALID_ARG, "dq, dk, dv and dstate_out are all NULL: nothing to compute");
    LA_TRY(check_ptr(q, "q"));
    if (!sonly) LA_TRY(check_ptr(k, "k"));
    if (!sonly) LA_TRY(check_ptr(v, "v"));
    LA_TRY(check_ptr(dout, "dout"));
    if (dq || !dq_optional) LA_TRY(check_ptr(dq, "dq"));
    if (!sonly) LA_TRY(check_ptr(dk, "dk"));
    if (!sonly) LA_TRY(check_ptr(dv, "dv"));
    if (sin) LA_TRY(check_state(sin, "state_in"));
    if (rin) LA_TRY(check_state(rin, "dstate_in"));
    if (rout) {
        LA_TRY(check_state(rout, "dstate_out"));
        // dstate_out is written while other CTAs still read state_in and dstate_in
        const size_t bytes = (size_t)s.BH() * D * D * sizeof(float);
        auto overlaps = [&](const float *a) {
            return a && (const char *)a < (const char *)rout + bytes && (const char *)rout < (const char *)a + bytes;
        };
        if (overlaps(sin) || overlaps(rin))
            return fail(LA_ERR_INVALID_ARG, "dstate_out overlaps state_in or dstate_in");
    }
    DecayArgs dec;
    LA_TRY(decay_args(decay, H, &dec));
    LA_TRY(check_ws(LA_OP_CHUNK_DECAY_BWD, s, dtype, workspace, workspace_bytes));
    cudaStream_t st = (cudaStream_t)stream;
    if (T == 0) {   // R passes through unchanged
        if (!rout) return LA_OK;
        const size_t bytes = (size_t)s.BH() * D * D * sizeof(float);
        cudaError_t e = rin ? cudaMemcpyAsync(rout, rin, bytes, cudaMemcpyDeviceToDevice, st)
                            : cudaMemsetAsync(rout, 0, bytes, st);
        return e == cudaSuccess ? LA_OK : cuda_fail(e, "dstate copy");
    }
    if (path_tc(LA_OP_CHUNK_DECAY_BWD, s, dtype))
        return tc::decay_bwd(q, k, v, dout, sin, rin, rout, dec, dq, dk, dv, s, dtype, workspace, st);
    return simt::decay_bwd(q, k, v, dout, sin, rin, rout, dec, dq, dk, dv, s, dtype, st);
}

la_status la_chunk_decay_bwd(const void *q, const void *k, const void *v, const void *dout, const float *decay,
                             void *dq, void *dk, void *dv, int B, int H, int T, int D, la_dtype dtype,
                             void *workspace, size_t workspace_bytes, void *stream) {
    return decay_bwd_entry(q, k, v, dout, nullptr, nullptr, nullptr, decay, dq, dk, dv, B, H, T, D, dtype, workspace,
                           workspace_bytes, stream, false);
}

la_status la_chunk_decay_bwd_state(const void *q, const void *k, const void *v, const void *dout,
                                   const float *state_in, const float *dstate_in, float *dstate_out,
                                   const float *decay, void *dq, void *dk, void *dv, int B, int H, int T, int D,
                                   la_dtype dtype, void *workspace, size_t workspace_bytes, void *stream) {
    return decay_bwd_entry(q, k, v, dout, state_in, dstate_in, dstate_out, decay, dq, dk, dv, B, H, T, D, dtype,
                           workspace, workspace_bytes, stream, true);
}

// Common front half of the causal-norm entry points.
static la_status causal_entry(const Shape &s, la_dtype dt, const float *decay, la_feature f, float eps,
                              DecayArgs *dec, int *has_decay) {
    LA_TRY(validate(s, dt));
    // the norm term is always on here: LA_FEATURE_NORM is the identity feature map as well
    if (f != LA_FEATURE_IDENTITY && f != LA_FEATURE_ELU1 && f != LA_FEATURE_NORM)
        return fail(LA_ERR_UNSUPPORTED, "unknown feature map %d", (int)f);
    if (!(eps >= 0.f) || !isfinite(eps)) return fail(LA_ERR_INVALID_ARG, "eps must be finite and >= 0");
    *has_decay = decay != nullptr;
    if (decay) LA_TRY(decay_args(decay, s.H, dec));
    return LA_OK;
}

la_status la_causal_norm_fwd(const void *q, const void *k, const void *v, void *o, const float *decay,
                             la_feature feature, float eps, int B, int H, int T, int D, la_dtype dtype,
                             void *workspace, size_t workspace_bytes, void *stream) {
    const Shape s{B, H, T, D};
    DecayArgs dec;
    int has_decay = 0;
    LA_TRY(causal_entry(s, dtype, decay, feature, eps, &dec, &has_decay));
    LA_TRY(check_ptr(q, "q"));
    LA_TRY(check_ptr(k, "k"));
    LA_TRY(check_ptr(v, "v"));
    LA_TRY(check_ptr(o, "o"));
    LA_TRY(check_ws(LA_OP_CAUSAL_NORM_FWD, s, dtype, workspace, workspace_bytes));
    if (T == 0) return LA_OK;
    if (path_tc(LA_OP_CAUSAL_NORM_FWD, s, dtype))
        return tc::causal_norm_fwd(q, k, v, o, dec, has_decay, feature == LA_FEATURE_ELU1, s, dtype, eps, workspace,
                                   (cudaStream_t)stream);
    return simt::causal_norm_fwd(q, k, v, o, dec, has_decay, feature == LA_FEATURE_ELU1, s, dtype, eps, workspace,
                                 (cudaStream_t)stream);
}

la_status la_causal_norm_bwd(const void *q, const void *k, const void *v, const void *dout, const float *decay,
                             la_feature feature, float eps, void *dq, void *dk, void *dv, int B, int H, int T, int D,
                             la_dtype dtype, void *workspace, size_t workspace_bytes, void *stream) {
    const Shape s{B, H, T, D};
    DecayArgs dec;
    int has_decay = 0;
    LA_TRY(causal_entry(s, dtype, decay, feature, eps, &dec, &has_decay));
    LA_TRY(check_ptr(q, "q"));
    LA_TRY(check_ptr(k, "k"));
    LA_TRY(check_ptr(v, "v"));
    LA_TRY(check_ptr(dout, "dout"));
    LA_TRY(check_ptr(dq, "dq"));
    LA_TRY(check_ptr(dk, "dk"));
    LA_TRY(check_ptr(dv, "dv"));
    LA_TRY(check_ws(LA_OP_CAUSAL_NORM_BWD, s, dtype, workspace, workspace_bytes));
    if (T == 0) return LA_OK;
    if (path_tc(LA_OP_CAUSAL_NORM_BWD, s, dtype))
        return tc::causal_norm_bwd(q, k, v, dout, dq, dk, dv, dec, has_decay, feature == LA_FEATURE_ELU1, s, dtype,
                                   eps, workspace, (cudaStream_t)stream);
    return simt::causal_norm_bwd(q, k, v, dout, dq, dk, dv, dec, has_decay, feature == LA_FEATURE_ELU1, s, dtype, eps,
                                 workspace, (cudaStream_t)stream);
}

static la_status fmap_entry(bool bwd, la_fmap kind, float p, const void *x, const void *dy, void *out, int B,
                            int H, int T, int D, la_dtype dt, void *stream) {
    t_allow_null = (T == 0);
    if (B < 1 || H < 1 || T < 0) return fail(LA_ERR_INVALID_ARG, "B, H must be >= 1 and T >= 0");
    if (dt != LA_F32 && dt != LA_F16 && dt != LA_BF16) return fail(LA_ERR_UNSUPPORTED, "unknown dtype %d", (int)dt);
    if (D != 32 && D != 64 && D != 128) return fail(LA_ERR_UNSUPPORTED, "D must be 32, 64 or 128 (got %d)", D);
    if (kind != LA_FMAP_FOCUSED && kind != LA_FMAP_POLARITY && kind != LA_FMAP_POLARITY_SWAP)
        return fail(LA_ERR_UNSUPPORTED, "unknown feature map kind %d", (int)kind);
    if (!(p >= 1.f) || !isfinite(p)) return fail(LA_ERR_INVALID_ARG, "p must be finite and >= 1");
    const long long rows = (long long)B * H * T;
    if ((double)rows * D * 2 >= 2147483648.0) return fail(LA_ERR_UNSUPPORTED, "tensor too large");
    LA_TRY(check_ptr(x, "x"));
    if (bwd) LA_TRY(check_ptr(dy, "dy"));
    LA_TRY(check_ptr(out, bwd ? "dx" : "y"));
    if (rows == 0) return LA_OK;
    return feature_map(bwd, (int)kind, p, x, dy, out, rows, D, dt, (cudaStream_t)stream);
}

la_status la_feature_map_fwd(la_fmap kind, float p, const void *x, void *y, int B, int H, int T, int D, la_dtype dtype,
                             void *stream) {
    return fmap_entry(false, kind, p, x, nullptr, y, B, H, T, D, dtype, stream);
}

la_status la_feature_map_bwd(la_fmap kind, float p, const void *x, const void *dy, void *dx, int B, int H, int T,
                             int D, la_dtype dtype, void *stream) {
    return fmap_entry(true, kind, p, x, dy, dx, B, H, T, D, dtype, stream);
}

la_status la_gated_fwd(const void *q, const void *k, const void *v, const void *g, void *o, int B, int H, int T,
                       int D, la_dtype dtype, void *workspace, size_t workspace_bytes, void *stream) {
    const Shape s{B, H, T, D};
    LA_TRY(validate(s, dtype));
    LA_TRY(check_ptr(q, "q"));
    LA_TRY(check_ptr(k, "k"));
    LA_TRY(check_ptr(v, "v"));
    LA_TRY(check_ptr(g, "g"));
    LA_TRY(check_ptr(o, "o"));
    LA_TRY(check_ws(LA_OP_GATED_FWD, s, dtype, workspace, workspace_bytes));
    if (T == 0) return LA_OK;
    return simt::gated_fwd(q, k, v, g, o, s, dtype, workspace, (cudaStream_t)stream);
}

la_status la_gated_bwd(const void *q, const void *k, const void *v, const void *g, const void *dout, void *dq,
                       void *dk, void *dv, void *dg, int B, int H, int T, int D, la_dtype dtype, void *workspace,
                       size_t workspace_bytes, void *stream) {
    const Shape s{B, H, T, D};
    LA_TRY(validate(s, dtype));
    LA_TRY(check_ptr(q, "q"));
    LA_TRY(check_ptr(k, "k"));
    LA_TRY(check_ptr(v, "v"));
    LA_TRY(check_ptr(g, "g"));
    LA_TRY(check_ptr(dout, "dout"));
    LA_TRY(check_ptr(dq, "dq"));
    LA_TRY(check_ptr(dk, "dk"));
    LA_TRY(check_ptr(dv, "dv"));
    LA_TRY(check_ptr(dg, "dg"));
    LA_TRY(check_ws(LA_OP_GATED_BWD, s, dtype, workspace, workspace_bytes));
    if (T == 0) return LA_OK;
    return simt::gated_bwd(q, k, v, g, dout, dq, dk, dv, dg, s, dtype, workspace, (cudaStream_t)stream);
}

la_status la_chunk_decay_scan(const float *states, const long long *gaps, int n, const float *decay, float *out,
                              int B, int H, int D, void *stream) {
    LA_TRY(validate(Shape{B, H, 1, D}, LA_F32));
    if (n < 1 || n > LA_MAX_SCAN_SEGMENTS)
        return fail(LA_ERR_UNSUPPORTED, "n=%d segments, must be in [1, %d]", n, LA_MAX_SCAN_SEGMENTS);
    if (!gaps) return fail(LA_ERR_INVALID_ARG, "gaps is NULL");
    LA_TRY(check_state(states, "states"));
    LA_TRY(check_state(out, "out"));
    DecayArgs dec;
    LA_TRY(decay_args(decay, H, &dec));
    return decay_scan(states, gaps, n, dec, out, B, H, D, (cudaStream_t)stream);
}

la_status la_state_reduce(const void *k, const void *v, float *state, int B, int H, int T, int D, la_dtype dtype,
                          la_feature feature, void *workspace, size_t workspace_bytes, void *stream) {
    return stage_entry(Stage::Reduce, LA_OP_STATE_REDUCE, feature, k, v, nullptr, state, nullptr, nullptr, B, H, T, D,
                       dtype, 0.f, workspace, workspace_bytes, stream);
}

la_status la_state_apply(const void *q, const float *state, void *o, int B, int H, int T, int D, la_dtype dtype,
                         la_feature feature, float eps, void *stream) {
    return stage_entry(Stage::Apply, LA_OP_STATE_APPLY, feature, q, nullptr, state, nullptr, o, nullptr, B, H, T, D,
                       dtype, eps, nullptr, 0, stream);
}

la_status la_state_bwd_q(const void *q, const void *dout, const float *state, void *dq, float *dstate, int B, int H,
                         int T, int D, la_dtype dtype, la_feature feature, float eps, void *workspace,
                         size_t workspace_bytes, void *stream) {
    return stage_entry(Stage::BwdQ, LA_OP_STATE_BWD_Q, feature, q, dout, state, dstate, dq, nullptr, B, H, T, D, dtype,
                       eps, workspace, workspace_bytes, stream);
}

la_status la_state_bwd_kv(const void *k, const void *v, const float *dstate, void *dk, void *dv, int B, int H, int T,
                          int D, la_dtype dtype, la_feature feature, void *stream) {
    return stage_entry(Stage::BwdKV, LA_OP_STATE_BWD_KV, feature, k, v, dstate, nullptr, dk, dv, B, H, T, D, dtype,
                       0.f, nullptr, 0, stream);
}

la_status la_chunk_decay_step(const void *q, const void *k, const void *v, void *o, float *state,
                              const float *decay, int B, int H, int D, la_dtype dtype, void *stream) {
    const Shape s{B, H, 1, D};
    LA_TRY(validate(s, dtype));
    LA_TRY(check_ptr(q, "q"));
    LA_TRY(check_ptr(k, "k"));
    LA_TRY(check_ptr(v, "v"));
    LA_TRY(check_ptr(o, "o"));
    LA_TRY(check_ptr(state, "state"));
    DecayArgs dec;
    LA_TRY(decay_args(decay, H, &dec));
    return decay_step(q, k, v, o, state, dec, B, H, D, dtype, (cudaStream_t)stream);
}

const char *la_status_string(la_status status) {
    switch (status) {
    case LA_OK: return "LA_OK";
    case LA_ERR_INVALID_ARG: return "LA_ERR_INVALID_ARG";
    case LA_ERR_UNSUPPORTED: return "LA_ERR_UNSUPPORTED";
    case LA_ERR_ALIGNMENT: return "LA_ERR_ALIGNMENT";
    case LA_ERR_WORKSPACE: return "LA_ERR_WORKSPACE";
    case LA_ERR_CUDA: return "LA_ERR_CUDA";
    case LA_ERR_TIMEOUT: return "LA_ERR_TIMEOUT";
    }
    return "LA_ERR_UNKNOWN";
}

const char *la_last_error(void) { return g_last_error.c_str(); }

la_status la_device_check(void) {
    const unsigned int f = tc::read_and_clear_fault();
    if (f == 0xFFFFFFFFu) return fail(LA_ERR_CUDA, "could not read the device fault word");
    if (f) return fail(LA_ERR_TIMEOUT, "a tensor-core kernel wait ran out (fault bits 0x%08x)", f);
    return LA_OK;
}

long long la_launch_count(void) { return g_launches.load(); }

la_status la_debug_fail_launch(int after) {
    if (after < -1) return fail(LA_ERR_INVALID_ARG, "after must be >= -1 (got %d)", after);
    g_fail_after.store(after);
    return LA_OK;
}

int la_prof_enable(int enabled) { return g_prof_on.exchange(enabled ? 1 : 0); }

int la_prof_collect(la_prof_record *records, int max_records) {
    std::vector<ProfEntry> entries;
    {
        std::lock_guard<std::mutex> lk(g_prof_mu);
        entries.swap(g_prof);
    }
    struct Agg {
        const char *name;
        long long n;
        double ms;
    };
    std::vector<Agg> agg;
    int rc = 0;
    for (const ProfEntry &e : entries) {
        float ms = 0.f;
        if (cudaEventSynchronize(e.stop) != cudaSuccess || cudaEventElapsedTime(&ms, e.start, e.stop) != cudaSuccess) {
            rc = -1;
        }
        size_t i = 0;
        for (; i < agg.size(); ++i)
            if (strcmp(agg[i].name, e.name) == 0) break;
        if (i == agg.size()) agg.push_back({e.name, 0, 0.0});
        agg[i].n += 1;
        agg[i].ms += ms;
    }
    {
        std::lock_guard<std::mutex> lk(g_prof_mu);
        for (const ProfEntry &e : entries) {
            g_event_pool.push_back(e.start);
            g_event_pool.push_back(e.stop);
        }
    }
    if (rc) return -1;
    for (size_t i = 0; i < agg.size() && (int)i < max_records; ++i) {
        records[i].name = agg[i].name;
        records[i].launches = agg[i].n;
        records[i].total_ms = agg[i].ms;
    }
    return (int)agg.size();
}

}  // extern "C"
