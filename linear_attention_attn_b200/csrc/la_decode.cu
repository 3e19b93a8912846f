// la_decode.cu -- one recurrent step of causal linear attention with per-head
// decay (retention) for decoding: S <- gamma S + k^T v, o = q S.
//
// "flash-linear-attention" README, "Different forms of linear attention"
// (FusedRecurrent: the recurrent form, one token at a time).  The step reads and
// writes the fp32 D x D state once, so it is bound by HBM: 2 D^2 * 4 bytes of
// state traffic per (b, h) against 4 D elements of q, k, v, o.
//
// One CTA per (b, h), 8 warps.  Warp w takes state rows i = w, w + 8, ...; lane
// l takes columns D/32 * l .. D/32 * l + D/32 - 1, so every row is read and
// written as one coalesced 512-byte (D = 128) or 256-byte (D = 64) segment.  The
// 8 warps' partial outputs are summed in warp order (deterministic).
#include "la_internal.cuh"

namespace la {
namespace {

constexpr int kStepWarps = 8;

template <int N> struct vecf;
template <> struct vecf<4> {
    static __device__ __forceinline__ void ld(const float *p, float (&x)[4]) {
        const float4 v = *reinterpret_cast<const float4 *>(p);
        x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
    }
    static __device__ __forceinline__ void st(float *p, const float (&x)[4]) {
        *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]);
    }
};
template <> struct vecf<2> {
    static __device__ __forceinline__ void ld(const float *p, float (&x)[2]) {
        const float2 v = *reinterpret_cast<const float2 *>(p);
        x[0] = v.x; x[1] = v.y;
    }
    static __device__ __forceinline__ void st(float *p, const float (&x)[2]) {
        *reinterpret_cast<float2 *>(p) = make_float2(x[0], x[1]);
    }
};

template <typename T, int D>
__global__ void __launch_bounds__(kStepWarps * 32)
decay_step_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v, T *__restrict__ o,
                  float *__restrict__ state, DecayArgs dec, int H) {
    constexpr int CPL = D / 32;
    __shared__ float sq[D], sk[D];
    __shared__ float part[kStepWarps][D];
    const int bh = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float gamma = dec.gamma[bh % H];
    const size_t vo = (size_t)bh * D;
    for (int i = threadIdx.x; i < D; i += blockDim.x) {
        sq[i] = io<T>::ld(q + vo + i);
        sk[i] = io<T>::ld(k + vo + i);
    }
    float vj[CPL], acc[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        vj[c] = io<T>::ld(v + vo + lane * CPL + c);
        acc[c] = 0.f;
    }
    __syncthreads();
    float *sh = state + (size_t)bh * D * D + lane * CPL;
#pragma unroll 4
    for (int i = warp; i < D; i += kStepWarps) {
        float x[CPL];
        vecf<CPL>::ld(sh + (size_t)i * D, x);
        const float ki = sk[i], qi = sq[i];
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            x[c] = fmaf(gamma, x[c], ki * vj[c]);
            acc[c] = fmaf(qi, x[c], acc[c]);
        }
        vecf<CPL>::st(sh + (size_t)i * D, x);
    }
#pragma unroll
    for (int c = 0; c < CPL; ++c) part[warp][lane * CPL + c] = acc[c];
    __syncthreads();
    for (int j = threadIdx.x; j < D; j += blockDim.x) {
        float r = 0.f;
#pragma unroll
        for (int w = 0; w < kStepWarps; ++w) r += part[w][j];
        io<T>::st(o + vo + j, r);
    }
}

template <typename T>
la_status step_t(const void *q, const void *k, const void *v, void *o, float *state, const DecayArgs &dec, int B,
                 int H, int D, cudaStream_t st) {
    const dim3 grid((unsigned)((long long)B * H)), block(kStepWarps * 32);
    if (D == 64)
        return launch("decay_step", decay_step_kernel<T, 64>, grid, block, 0, st, (const T *)q, (const T *)k,
                      (const T *)v, (T *)o, state, dec, H);
    return launch("decay_step", decay_step_kernel<T, 128>, grid, block, 0, st, (const T *)q, (const T *)k,
                  (const T *)v, (T *)o, state, dec, H);
}

}  // namespace

la_status decay_step(const void *q, const void *k, const void *v, void *o, float *state, const DecayArgs &dec, int B,
                     int H, int D, la_dtype dt, cudaStream_t st) {
    switch (dt) {
    case LA_F32: return step_t<float>(q, k, v, o, state, dec, B, H, D, st);
    case LA_F16: return step_t<__half>(q, k, v, o, state, dec, B, H, D, st);
    default: return step_t<__nv_bfloat16>(q, k, v, o, state, dec, B, H, D, st);
    }
}

}  // namespace la
