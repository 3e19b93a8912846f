// la_static_scratch.cu -- la_bidir_fwd_static: the bidirectional forward for callers that
// cannot allocate device memory.
//
// Some callers have no way to allocate device memory of their own: code running
// inside a host framework that owns the CUDA allocator and hands out only the
// tensors it manages, plugins loaded into an inference server, or embedded
// runtimes that are forbidden from calling cudaMalloc after start-up.  They
// cannot provide the scratch buffer that la_bidir_fwd needs for its split
// reductions.  This entry point takes that scratch from a fixed-size array
// compiled into the library instead, so the caller passes only inputs and
// outputs.
//
// The array lives in every GPU's memory once the library's module is loaded on
// that GPU, and stays until the process exits.  All calls share it: calls that
// overlap on the GPU (different streams, or different host threads, without
// ordering between them) race on it and may return wrong results.  Its contents
// are whatever the previous call left; the kernels never read scratch they have
// not written in the same call, so nothing has to be cleared between calls.
//
// The array's device address belongs to the CUDA context that loaded the module:
// after cudaDeviceReset, or when a driver-API user releases and re-creates the
// primary context, the module is loaded again and the array may move.  So the
// address is cached per device together with the unique id of the context it was
// looked up in, and looked up again whenever the current context is another one.
#include <mutex>
#include <stdio.h>

#include <cuda.h>

#include "la_internal.cuh"

namespace la {
namespace {

// Largest scratch the entry point can use (bytes).  Shapes whose workspace need
// (la_workspace_size(LA_OP_BIDIR_FWD, ...)) exceeds it are rejected.
constexpr size_t kStaticScratchBytes = (size_t)LA_STATIC_SCRATCH_BYTES;

// The scratch itself.  In host code this name is only the host-side shadow of the
// symbol; its device address is taken with cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
struct ScratchEntry {
    unsigned long long ctx_id;   // id of the context the address was looked up in
    void *addr;                  // null: not looked up yet
};
static ScratchEntry g_scratch[kMaxDevices];
static std::mutex g_scratch_mu;

// Driver calls that name the current context, resolved at run time (the library
// does not link against libcuda).
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

static bool driver_fn(const char *name, void **fn) {
    cudaDriverEntryPointQueryResult q;
    return cudaGetDriverEntryPoint(name, fn, cudaEnableDefault, &q) == cudaSuccess &&
           q == cudaDriverEntryPointSuccess && *fn;
}

// Id of the context current on this thread; false when there is none yet.
static bool current_ctx_id(unsigned long long *id) {
    static CtxGetCurrentFn get_cur = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *a = nullptr, *b = nullptr;
        if (driver_fn("cuCtxGetCurrent", &a) && driver_fn("cuCtxGetId", &b)) {
            get_cur = reinterpret_cast<CtxGetCurrentFn>(a);
            get_id = reinterpret_cast<CtxGetIdFn>(b);
        }
    });
    if (!get_cur || !get_id) return false;
    CUcontext ctx = nullptr;
    if (get_cur(&ctx) != CUDA_SUCCESS || !ctx) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the scratch in the current device's current context.  The
// lookup (first call on a device, or in a new context) must not happen while
// `stream` is being captured into a graph: it may load the library's module.
static la_status scratch_address(cudaStream_t stream, void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) {
        set_error("device ordinal %d is beyond the %d devices the static scratch supports", dev, kMaxDevices);
        return LA_ERR_UNSUPPORTED;
    }
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    unsigned long long id = 0;
    const bool have_id = current_ctx_id(&id);
    ScratchEntry &ent = g_scratch[dev];
    if (ent.addr && have_id && ent.ctx_id == id) {
        *out = ent.addr;
        return LA_OK;
    }
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    e = cudaStreamIsCapturing(stream, &cap);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamIsCapturing");
    if (cap != cudaStreamCaptureStatusNone) {
        set_error("la_bidir_fwd_static: the first call on a device (or in a new CUDA context) looks up the "
                  "static scratch and must not run during stream capture; call it once before capturing");
        return LA_ERR_INVALID_ARG;
    }
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
    // the lookup made the runtime's context current if none was
    if (!current_ctx_id(&id)) {
        set_error("la_bidir_fwd_static: no current CUDA context after the scratch lookup");
        return LA_ERR_CUDA;
    }
    ent.ctx_id = id;
    ent.addr = p;
    *out = p;
    return LA_OK;
}

}  // namespace
}  // namespace la

extern "C" size_t la_static_scratch_bytes(void) { return la::kStaticScratchBytes; }

extern "C" la_status la_bidir_fwd_static(const void *q, const void *k, const void *v, void *o, float *state, int B,
                                         int H, int T, int D, la_dtype dtype, float eps, void *stream) {
    const size_t need = la_workspace_size(LA_OP_BIDIR_FWD, B, H, T, D, dtype);
    if (need > la::kStaticScratchBytes) {
        la::set_error("la_bidir_fwd_static: this shape needs %zu bytes of scratch but the static scratch holds "
                      "%zu; use la_bidir_fwd with a caller-provided workspace",
                      need, la::kStaticScratchBytes);
        return LA_ERR_WORKSPACE;
    }
    // Nothing to look up when no scratch is used: an invalid shape or dtype (which
    // la_bidir_fwd reports) needs none.
    if (need == 0) return la_bidir_fwd(q, k, v, o, state, B, H, T, D, dtype, eps, nullptr, 0, stream);
    void *scratch = nullptr;
    la_status rc = la::scratch_address((cudaStream_t)stream, &scratch);
    if (rc != LA_OK) return rc;
    return la_bidir_fwd(q, k, v, o, state, B, H, T, D, dtype, eps, scratch, la::kStaticScratchBytes, stream);
}
