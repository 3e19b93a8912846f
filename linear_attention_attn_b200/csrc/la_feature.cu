// la_feature.cu -- row-wise feature maps applied before the bidirectional op with
// the norm term on caller-formed features (LA_FEATURE_NORM), and their backward:
//   focusing function (focused linear attention): y = relu(x), f = (|y| / |y^p|) y^p
//   polarity split:  f = [relu(x)^p, relu(-x)^p]  (or the halves swapped)
// "Flash Bi-directional Linear Attention" README, the list of models the library
// serves (Focused-LA, PolaFormer); the maps themselves are those models' feature
// maps, written from their definitions.  |.| is the 2-norm over the row's D
// entries, y^p elementwise; a row with no positive entry maps to 0.
//
// One warp per row, lane l holding entries E l .. E l + E - 1 (E = D / 32), the row
// norms reduced with xor shuffles in a fixed order; fp32 arithmetic.  Bound by HBM:
// a row of D inputs in, D or 2 D outputs out (backward: x and dy in, dx out).
#include "la_internal.cuh"

#include <math.h>

namespace la {
namespace {

constexpr int kRowsPerBlock = 8;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
    return v;
}

// r^p for r >= 0 (0 at r = 0 for every p > 0)
__device__ __forceinline__ float pow_pos(float r, float p) { return r > 0.f ? powf(r, p) : 0.f; }

template <typename T, int D, int KIND>
__global__ void __launch_bounds__(32 * kRowsPerBlock)
fmap_fwd(const T *__restrict__ x, T *__restrict__ y, long long rows, float p) {
    constexpr int E = D / 32;
    const long long row = (long long)blockIdx.x * kRowsPerBlock + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;                     // whole warps leave together
    float xv[E];
#pragma unroll
    for (int e = 0; e < E; ++e) xv[e] = io<T>::ld(x + row * D + lane * E + e);
    if (KIND == 0) {
        float a2 = 0.f, b2 = 0.f, u[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const float r = fmaxf(xv[e], 0.f);
            u[e] = pow_pos(r, p);
            a2 = fmaf(r, r, a2);
            b2 = fmaf(u[e], u[e], b2);
        }
        a2 = warp_sum(a2);
        b2 = warp_sum(b2);
        const float sc = b2 > 0.f ? sqrtf(a2 / b2) : 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) io<T>::st(y + row * D + lane * E + e, sc * u[e]);
    } else {
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const float pos = pow_pos(fmaxf(xv[e], 0.f), p), neg = pow_pos(fmaxf(-xv[e], 0.f), p);
            io<T>::st(y + row * 2 * D + lane * E + e, KIND == 1 ? pos : neg);
            io<T>::st(y + row * 2 * D + D + lane * E + e, KIND == 1 ? neg : pos);
        }
    }
}

// dx = J^T dy.  Focusing function, a = |y|, b = |y^p|, s = dy . y^p:
//   dx_j = [x_j > 0] ((a / b) p y_j^(p-1) dy_j + s y_j / (a b) - s a p y_j^(2p-1) / b^3).
// Polarity split: relu(x)^p has slope p x^(p-1) on x > 0, relu(-x)^p slope -p (-x)^(p-1) on x < 0.
template <typename T, int D, int KIND>
__global__ void __launch_bounds__(32 * kRowsPerBlock)
fmap_bwd(const T *__restrict__ x, const T *__restrict__ dy, T *__restrict__ dx, long long rows, float p) {
    constexpr int E = D / 32;
    const long long row = (long long)blockIdx.x * kRowsPerBlock + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    float xv[E];
#pragma unroll
    for (int e = 0; e < E; ++e) xv[e] = io<T>::ld(x + row * D + lane * E + e);
    if (KIND == 0) {
        float a2 = 0.f, b2 = 0.f, s = 0.f, g[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const float r = fmaxf(xv[e], 0.f), u = pow_pos(r, p);
            g[e] = io<T>::ld(dy + row * D + lane * E + e);
            a2 = fmaf(r, r, a2);
            b2 = fmaf(u, u, b2);
            s = fmaf(g[e], u, s);
        }
        a2 = warp_sum(a2);
        b2 = warp_sum(b2);
        s = warp_sum(s);
        const float a = sqrtf(a2), b = sqrtf(b2);
#pragma unroll
        for (int e = 0; e < E; ++e) {
            float d = 0.f;
            if (xv[e] > 0.f && b > 0.f) {
                const float r = xv[e], rp1 = pow_pos(r, p - 1.f), rp = rp1 * r;
                d = (a / b) * p * rp1 * g[e] + s * r / (a * b) - s * a * p * rp * rp1 / (b2 * b);
            }
            io<T>::st(dx + row * D + lane * E + e, d);
        }
    } else {
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const float xe = xv[e];
            const float gp = io<T>::ld(dy + row * 2 * D + (KIND == 1 ? 0 : D) + lane * E + e);
            const float gn = io<T>::ld(dy + row * 2 * D + (KIND == 1 ? D : 0) + lane * E + e);
            float d = 0.f;
            if (xe > 0.f) d = gp * p * pow_pos(xe, p - 1.f);
            if (xe < 0.f) d = -gn * p * pow_pos(-xe, p - 1.f);
            io<T>::st(dx + row * D + lane * E + e, d);
        }
    }
}

template <typename T, int D>
la_status fmap_t(bool bwd, int kind, float p, const void *x, const void *dy, void *out, long long rows,
                 cudaStream_t st) {
    const dim3 grid((unsigned)((rows + kRowsPerBlock - 1) / kRowsPerBlock)), block(32 * kRowsPerBlock);
    const T *xs = (const T *)x;
    if (!bwd) {
        T *y = (T *)out;
        if (kind == 0) return launch("feature_map_fwd", fmap_fwd<T, D, 0>, grid, block, 0, st, xs, y, rows, p);
        if (kind == 1) return launch("feature_map_fwd", fmap_fwd<T, D, 1>, grid, block, 0, st, xs, y, rows, p);
        return launch("feature_map_fwd", fmap_fwd<T, D, 2>, grid, block, 0, st, xs, y, rows, p);
    }
    const T *g = (const T *)dy;
    T *dx = (T *)out;
    if (kind == 0) return launch("feature_map_bwd", fmap_bwd<T, D, 0>, grid, block, 0, st, xs, g, dx, rows, p);
    if (kind == 1) return launch("feature_map_bwd", fmap_bwd<T, D, 1>, grid, block, 0, st, xs, g, dx, rows, p);
    return launch("feature_map_bwd", fmap_bwd<T, D, 2>, grid, block, 0, st, xs, g, dx, rows, p);
}

template <typename T>
la_status fmap_d(bool bwd, int kind, float p, const void *x, const void *dy, void *out, long long rows, int D,
                 cudaStream_t st) {
    if (D == 32) return fmap_t<T, 32>(bwd, kind, p, x, dy, out, rows, st);
    if (D == 64) return fmap_t<T, 64>(bwd, kind, p, x, dy, out, rows, st);
    return fmap_t<T, 128>(bwd, kind, p, x, dy, out, rows, st);
}

}  // namespace

la_status feature_map(bool bwd, int kind, float p, const void *x, const void *dy, void *out, long long rows, int D,
                      la_dtype dt, cudaStream_t st) {
    switch (dt) {
    case LA_F32: return fmap_d<float>(bwd, kind, p, x, dy, out, rows, D, st);
    case LA_F16: return fmap_d<__half>(bwd, kind, p, x, dy, out, rows, D, st);
    default: return fmap_d<__nv_bfloat16>(bwd, kind, p, x, dy, out, rows, D, st);
    }
}

}  // namespace la
