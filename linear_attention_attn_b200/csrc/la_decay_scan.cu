// la_decay_scan.cu -- the combine step of the decay op (retention) over the
// segments of one sequence split along T (one segment per rank):
//   out[b,h] = sum over i < n with gap_i >= 0 of gamma_h^gap_i * states[i,b,h]
// in the order i = 0, 1, ... (deterministic).  For the forward, states are the
// segments' end states from a zero state and gap_i the number of tokens
// between segment i and the target segment (the state entering it is the
// exclusive scan of the decayed end states); for the backward, states are the
// segments' reverse-sweep R at their first token and gap_i counts the tokens
// between the target segment and segment i.  Linear attention's recurrent
// form S_t = gamma S_{t-1} + k_t^T v_t ("flash-linear-attention" README,
// FusedRecurrent) makes the state after a span of tokens gamma^len S + (the
// span's own state), which is what the sum unrolls.
//
// HBM bound: n + 1 arrays of B H D^2 fp32 values, read and written once with
// float4 loads by 256-thread CTAs, grid (D^2 / 1024, B H).
#include "la_internal.cuh"

#include <math.h>

namespace la {
namespace {

constexpr int kScanThreads = 256;

struct ScanArgs {
    long long gap[LA_MAX_SCAN_SEGMENTS];
};

__global__ void __launch_bounds__(kScanThreads)
decay_scan_kernel(const float4 *__restrict__ states, float4 *out, ScanArgs a, DecayArgs dec, int n, int H,
                  int per_head4, long long BH) {
    __shared__ float w[LA_MAX_SCAN_SEGMENTS];
    const long long bh = blockIdx.y;
    const double gamma = dec.gamma[bh % H];
    for (int i = threadIdx.x; i < n; i += blockDim.x)
        w[i] = a.gap[i] < 0 ? 0.f : (float)pow(gamma, (double)a.gap[i]);
    __syncthreads();
    const int e = blockIdx.x * kScanThreads + threadIdx.x;
    if (e >= per_head4) return;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i = 0; i < n; ++i) {
        if (a.gap[i] < 0) continue;
        const float4 x = states[((long long)i * BH + bh) * per_head4 + e];
        acc.x = fmaf(w[i], x.x, acc.x);
        acc.y = fmaf(w[i], x.y, acc.y);
        acc.z = fmaf(w[i], x.z, acc.z);
        acc.w = fmaf(w[i], x.w, acc.w);
    }
    out[bh * per_head4 + e] = acc;
}

}  // namespace

la_status decay_scan(const float *states, const long long *gaps, int n, const DecayArgs &dec, float *out, int B,
                     int H, int D, cudaStream_t st) {
    ScanArgs a;
    for (int i = 0; i < n; ++i) a.gap[i] = gaps[i];
    const long long BH = (long long)B * H;
    const int per_head4 = D * D / 4;
    const dim3 grid((unsigned)((per_head4 + kScanThreads - 1) / kScanThreads), (unsigned)BH);
    return launch("decay_scan", decay_scan_kernel, grid, dim3(kScanThreads), 0, st,
                  reinterpret_cast<const float4 *>(states), reinterpret_cast<float4 *>(out), a, dec, n, H,
                  per_head4, BH);
}

}  // namespace la
