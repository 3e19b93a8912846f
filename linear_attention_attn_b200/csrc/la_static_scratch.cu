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
#include <mutex>
#include <stdio.h>

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
static void *g_scratch_addr[kMaxDevices];
static std::mutex g_scratch_mu;

// Device address of the scratch on the current device, looked up once per device.
static la_status scratch_address(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) {
        set_error("device ordinal %d is beyond the %d devices the static scratch supports", dev, kMaxDevices);
        return LA_ERR_UNSUPPORTED;
    }
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return LA_OK;
}

}  // namespace
}  // namespace la

extern "C" la_status la_bidir_fwd_static(const void *q, const void *k, const void *v, void *o, float *state, int B,
                                         int H, int T, int D, la_dtype dtype, float eps, void *stream) {
    const size_t need = la_workspace_size(LA_OP_BIDIR_FWD, B, H, T, D, dtype);
    if (need > la::kStaticScratchBytes) {
        la::set_error("la_bidir_fwd_static: this shape needs %zu bytes of scratch but the static scratch holds "
                      "%zu; use la_bidir_fwd with a caller-provided workspace",
                      need, la::kStaticScratchBytes);
        return LA_ERR_WORKSPACE;
    }
    void *scratch = nullptr;
    la_status rc = la::scratch_address(&scratch);
    if (rc != LA_OK) return rc;
    return la_bidir_fwd(q, k, v, o, state, B, H, T, D, dtype, eps, scratch, la::kStaticScratchBytes, stream);
}
