// la_internal.cuh -- shared declarations of the library's CUDA sources (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/la.h"

namespace la {

// ---------------------------------------------------------------- errors --
void set_error(const char *fmt, ...);
la_status cuda_fail(cudaError_t e, const char *what);
// A failed launch: the error text also gives the kernel's registers, local memory
// and thread limit next to the block and shared memory asked for.
la_status launch_fail(cudaError_t e, const char *what, const void *kernel, dim3 block, size_t smem);

// ------------------------------------------------------------- launching --
// Every kernel goes through launch(): it counts launches and, when profiling
// is on, brackets the launch with two events on its stream.
void prof_before(const char *name, cudaStream_t s);
void prof_after(cudaStream_t s);
void count_launch();
// Test hook (la_debug_fail_launch): true when this launch is to fail without running;
// the error text is then set.  Checked before any CUDA call of the launch.
bool injected_launch_failure(const char *name);

template <typename Kernel, typename... Args>
la_status launch(const char *name, Kernel kernel, dim3 grid, dim3 block, size_t smem,
                 cudaStream_t stream, Args... args) {
    if (grid.x == 0 || grid.y == 0 || grid.z == 0) return LA_OK;
    if (injected_launch_failure(name)) return LA_ERR_CUDA;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return cuda_fail(e, name);
    }
    prof_before(name, stream);
    kernel<<<grid, block, smem, stream>>>(args...);
    cudaError_t e = cudaGetLastError();
    prof_after(stream);
    count_launch();
    if (e != cudaSuccess) return cuda_fail(e, name);
    return LA_OK;
}

// Launch with programmatic stream serialization: the kernel may start while the
// previous kernel in the stream is finishing.  Only for kernels that execute
// griddepcontrol.wait before touching global memory (the tensor-core kernels).
// (With per-kernel profiling on, the events between kernels keep plain order.)

template <typename Kernel, typename... Args>
la_status launch_pdl(const char *name, Kernel kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                     Args... args) {
    if (grid.x == 0 || grid.y == 0 || grid.z == 0) return LA_OK;
    if (injected_launch_failure(name)) return LA_ERR_CUDA;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return cuda_fail(e, name);
    }
    prof_before(name, stream);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
    if (e == cudaSuccess) e = cudaGetLastError();
    prof_after(stream);
    count_launch();
    if (e != cudaSuccess) return launch_fail(e, name, reinterpret_cast<const void *>(kernel), block, smem);
    return LA_OK;
}

// ---------------------------------------------------------- element I/O --
template <typename T> struct io;
template <> struct io<float> {
    static __device__ __forceinline__ float ld(const float *p) { return __ldg(p); }
    static __device__ __forceinline__ void st(float *p, float x) { *p = x; }
};
template <> struct io<__half> {
    static __device__ __forceinline__ float ld(const __half *p) { return __half2float(__ldg(p)); }
    static __device__ __forceinline__ void st(__half *p, float x) { *p = __float2half_rn(x); }
};
template <> struct io<__nv_bfloat16> {
    static __device__ __forceinline__ float ld(const __nv_bfloat16 *p) { return __bfloat162float(__ldg(p)); }
    static __device__ __forceinline__ void st(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }
};

// Feature map of bidirectional linear attention: elu(x) + 1, i.e. x + 1 for
// x > 0 and exp(x) for x <= 0, and its derivative (1, resp. exp(x)).
__device__ __forceinline__ float feature(float x) { return x > 0.f ? x + 1.f : expf(x); }
__device__ __forceinline__ float feature_grad(float x) { return x > 0.f ? 1.f : expf(x); }

// Per-head decays of the chunked causal op travel by value.
struct DecayArgs {
    float gamma[LA_MAX_DECAY_HEADS];
};

// Stages of the state form, run separately for a sequence split along T:
//   Reduce  k, v            -> [S | z] of the tokens passed
//   Apply   q, [S | z]      -> o
//   BwdQ    q, dO, [S | z]  -> dq and the tokens' [dS | dz]
//   BwdKV   k, v, [dS | dz] -> dk, dv
enum class Stage { Reduce, Apply, BwdQ, BwdKV };

// ------------------------------------------------------ shape / workspace --
struct Shape {
    int B, H, T, D;
    long long BH() const { return (long long)B * H; }
};

// Split count of the T-reductions: a function of (B, H, T) only, so results
// are deterministic for a shape whatever GPU runs them.
int state_splits(const Shape &s, int rows_per_unit);

// Bytes of one [BH, D, D+1] fp32 state block, rounded up to 256.
size_t state_bytes(const Shape &s, long long copies);

// Combine of per-segment states of the decay op: out = sum_i gamma^gaps[i] states[i]
// over the i with gaps[i] >= 0 (n <= LA_MAX_SCAN_SEGMENTS, gaps on the host).
la_status decay_scan(const float *states, const long long *gaps, int n, const DecayArgs &dec, float *out, int B,
                     int H, int D, cudaStream_t st);

// Row-wise feature map (kind 0 focusing, 1 polarity split, 2 swapped split) of `rows`
// rows of D in {32, 64, 128}, or its backward (dx = J^T dy) when bwd.
la_status feature_map(bool bwd, int kind, float p, const void *x, const void *dy, void *out, long long rows, int D,
                      la_dtype dt, cudaStream_t st);

// One recurrent (decode) step of the decay op: S <- gamma S + k^T v, o = q S,
// with q, k, v, o [B,H,D] and the fp32 state [B,H,D,D] updated in place.
la_status decay_step(const void *q, const void *k, const void *v, void *o, float *state, const DecayArgs &dec, int B,
                     int H, int D, la_dtype dt, cudaStream_t st);

// ------------------------------------------------------------ SIMT path --
// Plain CUDA-core kernels (fp32 FMA).  They implement every op for every
// dtype; the fp16/bf16 ops at D in {64,128} normally run on the tensor-core
// path instead.
namespace simt {
size_t workspace_size(la_op op, const Shape &s);
la_status state_fwd(bool bidir, const void *q, const void *k, const void *v, void *o, float *state,
                    const Shape &s, la_dtype dt, float eps, void *ws, cudaStream_t st);
la_status state_bwd(bool bidir, const void *q, const void *k, const void *v, const void *g,
                    const float *state, void *dq, void *dk, void *dv, const Shape &s, la_dtype dt,
                    float eps, void *ws, cudaStream_t st);
la_status decay_fwd(const void *q, const void *k, const void *v, void *o, const float *sin, float *sout,
                    const DecayArgs &dec, const Shape &s, la_dtype dt, cudaStream_t st);
la_status decay_bwd(const void *q, const void *k, const void *v, const void *g, const float *sin,
                    const float *rin, float *rout, const DecayArgs &dec, void *dq, void *dk, void *dv,
                    const Shape &s, la_dtype dt, cudaStream_t st);
la_status state_stage(Stage stage, la_feature f, const void *x, const void *y, const float *sin, float *sout,
                      void *out1, void *out2, const Shape &s, la_dtype dt, float eps, void *ws, cudaStream_t st);
// Causal linear attention with the norm term (has_decay = 0: gamma = 1; phi: elu + 1,
// else the identity).  The workspaces hold the chunk states (sequences of more than one
// chunk) and, for the backward, (n_t, dn_t) of every row before them.
la_status causal_norm_fwd(const void *q, const void *k, const void *v, void *o, const DecayArgs &dec, int has_decay,
                          bool phi, const Shape &s, la_dtype dt, float eps, void *ws, cudaStream_t st);
la_status causal_norm_bwd(const void *q, const void *k, const void *v, const void *g, void *dq, void *dk, void *dv,
                          const DecayArgs &dec, int has_decay, bool phi, const Shape &s, la_dtype dt, float eps,
                          void *ws, cudaStream_t st);
// Gated linear attention (log gates g, the decay exp(g) per token and key dimension).
la_status gated_fwd(const void *q, const void *k, const void *v, const void *g, void *o, const Shape &s, la_dtype dt,
                    void *ws, cudaStream_t st);
la_status gated_bwd(const void *q, const void *k, const void *v, const void *g, const void *dout, void *dq, void *dk,
                    void *dv, void *dg, const Shape &s, la_dtype dt, void *ws, cudaStream_t st);
}  // namespace simt

}  // namespace la
