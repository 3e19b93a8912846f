// la_simt.cu -- CUDA-core (fp32 FMA) kernels for every op and dtype.
//
// This is the straightforward path: every contraction is a loop of fp32
// FMAs over shared-memory tiles.  It carries fp32 inputs (where the tensor
// cores would round operands) and is the reference GPU implementation that
// the tensor-core kernels are checked against besides the CPU oracle.
//
// Bidirectional / simple_la ("Flash Bi-directional Linear Attention" README,
// intro and "Update": linear_attn with and without the norm term):
//   state_partial  per (b,h, T-split): S_part = sum phi(k)^T v, z_part = sum phi(k)
//   combine        fixed-order sum of the splits          -> state [BH, D, D+1]
//   output         o_t = phi(q_t) S / (phi(q_t).z + eps)
//   bwd_q          dq and the per-split partials of dS, dz
//   bwd_k          dk = (v dS^T + dz) phi'(k),  dv = phi(k) dS
// Retention ("flash-linear-attention" README, "Benchmarks" and "Different
// forms of linear attention", FusedRecurrent): one CTA per (b,h) walks T
// with the D x D state held in registers, one state column (or row) per
// thread.
// Causal linear attention with the norm term and gated linear attention (the
// same recurrent form, with the norm term of the bidirectional op, resp. gates
// per token and key dimension): the sequence in chunks of 256 tokens, each
// chunk's own state from a zero state (causal_chunk_state / gated_chunk_state),
// a scan over the chunks (chunk_scan), and one CTA per (b,h, chunk) walking its
// chunk with the state held once in register blocks of four columns.
#include "la_internal.cuh"

#include <string.h>

namespace la {
namespace simt {

constexpr int kTile = 32;      // rows per shared-memory tile
constexpr int kRetTile = 16;   // rows per tile in the recurrent (retention) kernels
constexpr int kThreads = 256;
constexpr int kCausalChunk = 256;   // tokens per chunk of the causal-norm and gated kernels (whole tiles)
static_assert(kCausalChunk % kRetTile == 0, "chunks hold whole recurrent tiles");

inline int causal_chunks(int T_len) { return T_len <= kCausalChunk ? 1 : (T_len + kCausalChunk - 1) / kCausalChunk; }
inline size_t round256(size_t n) { return (n + 255) / 256 * 256; }
// (n_t, dn_t) of every row of the causal-norm backward
inline size_t nd_bytes(const Shape &s) { return round256((size_t)s.BH() * s.T * sizeof(float2)); }
// the [B H][chunk][D][D + 1] fp32 chunk states; none for a single chunk
inline size_t causal_state_bytes(const Shape &s) {
    const int nc = causal_chunks(s.T);
    return nc > 1 ? round256((size_t)s.BH() * nc * s.D * (s.D + 1) * sizeof(float)) : 0;
}
// gated: dq in fp32; the [B H][chunk][D][D] states and the [B H][chunk][D] factors (or totals)
inline size_t dq32_bytes(const Shape &s) { return round256((size_t)s.BH() * s.T * s.D * sizeof(float)); }
inline size_t gated_e_bytes(const Shape &s) {
    return round256((size_t)s.BH() * causal_chunks(s.T) * s.D * s.D * sizeof(float));
}
inline size_t gated_a_bytes(const Shape &s) {
    return round256((size_t)s.BH() * causal_chunks(s.T) * s.D * sizeof(float));
}
inline size_t gated_state_bytes(const Shape &s) {
    return causal_chunks(s.T) > 1 ? gated_e_bytes(s) + gated_a_bytes(s) : 0;
}

// ------------------------------------------------------------ reductions --

// Partial S (and z for bidir) over rows [split*rps, min(T, (split+1)*rps)) of
// head blockIdx.y.  Thread (ti, tj) owns the R x R block S[ti*R.., tj*R..].
template <typename T, int D, bool BIDIR, bool PHI = BIDIR>
__global__ void __launch_bounds__(kThreads)
state_partial(const T *__restrict__ k, const T *__restrict__ v, float *__restrict__ part,
              int T_len, int nsplit, int rps) {
    constexpr int R = D / 16;
    __shared__ float ks[kTile][D];
    __shared__ float vs[kTile][D];
    const int split = blockIdx.x, bh = blockIdx.y;
    const long long base = (long long)bh * T_len * D;
    const int t0 = split * rps;
    const int t1 = min(T_len, t0 + rps);
    const int ti = threadIdx.x / 16, tj = threadIdx.x % 16;
    float acc[R][R];
    float zacc[R];
#pragma unroll
    for (int x = 0; x < R; ++x) {
        zacc[x] = 0.f;
#pragma unroll
        for (int y = 0; y < R; ++y) acc[x][y] = 0.f;
    }
    for (int ts = t0; ts < t1; ts += kTile) {
        for (int e = threadIdx.x; e < kTile * D; e += kThreads) {
            const int r = e / D, c = e % D, t = ts + r;
            float kk = 0.f, vv = 0.f;
            if (t < t1) {
                kk = io<T>::ld(k + base + (long long)t * D + c);
                if (PHI) kk = feature(kk);
                vv = io<T>::ld(v + base + (long long)t * D + c);
            }
            ks[r][c] = kk;
            vs[r][c] = vv;
        }
        __syncthreads();
#pragma unroll 4
        for (int r = 0; r < kTile; ++r) {
            float a[R], b[R];
#pragma unroll
            for (int x = 0; x < R; ++x) {
                a[x] = ks[r][ti * R + x];
                b[x] = vs[r][tj * R + x];
            }
#pragma unroll
            for (int x = 0; x < R; ++x) {
                if (BIDIR) zacc[x] += a[x];
#pragma unroll
                for (int y = 0; y < R; ++y) acc[x][y] = fmaf(a[x], b[y], acc[x][y]);
            }
        }
        __syncthreads();
    }
    float *out = part + ((long long)bh * nsplit + split) * D * (D + 1);
#pragma unroll
    for (int x = 0; x < R; ++x) {
#pragma unroll
        for (int y = 0; y < R; ++y) out[(ti * R + x) * (D + 1) + tj * R + y] = acc[x][y];
        if (tj == 0) out[(ti * R + x) * (D + 1) + D] = BIDIR ? zacc[x] : 0.f;
    }
}

// out[bh][e] = sum_{s=0..nsplit-1} part[bh][s][e], always in that order.
__global__ void __launch_bounds__(kThreads)
combine(const float *__restrict__ part, float *__restrict__ out, int nsplit, int n) {
    const long long bh = blockIdx.x;
    for (int e = threadIdx.x; e < n; e += kThreads) {
        float s = 0.f;
        for (int sp = 0; sp < nsplit; ++sp) s += part[(bh * nsplit + sp) * n + e];
        out[bh * n + e] = s;
    }
}

// --------------------------------------------------------------- outputs --

// o_t = f(q_t) S / (f(q_t).z + eps)  (bidir)  or  q_t S  (simple).
// 32 rows per CTA, 8 threads per row, thread cg owns columns cg + 8c.
template <typename T, int D, bool BIDIR, bool PHI = BIDIR>
__global__ void __launch_bounds__(kThreads)
output(const T *__restrict__ q, const float *__restrict__ state, T *__restrict__ o, int T_len, float eps) {
    constexpr int TPR = kThreads / kTile;
    constexpr int CPT = D / TPR;
    constexpr int LD = D + 1;
    extern __shared__ float sm[];
    float *S = sm;              // D x D
    float *z = S + D * D;       // D
    float *qs = z + D;          // kTile x LD
    const int bh = blockIdx.y;
    const int row0 = blockIdx.x * kTile;
    const long long base = (long long)bh * T_len * D;
    const float *st = state + (long long)bh * D * (D + 1);
    for (int e = threadIdx.x; e < D * D; e += kThreads) S[e] = st[(e / D) * (D + 1) + e % D];
    for (int e = threadIdx.x; e < D; e += kThreads) z[e] = st[e * (D + 1) + D];
    for (int e = threadIdx.x; e < kTile * D; e += kThreads) {
        const int r = e / D, c = e % D, t = row0 + r;
        float x = t < T_len ? io<T>::ld(q + base + (long long)t * D + c) : 0.f;
        qs[r * LD + c] = (PHI && t < T_len) ? feature(x) : x;
    }
    __syncthreads();
    const int r = threadIdx.x / TPR, cg = threadIdx.x % TPR, t = row0 + r;
    float acc[CPT];
#pragma unroll
    for (int c = 0; c < CPT; ++c) acc[c] = 0.f;
    float n = eps;
    for (int i = 0; i < D; ++i) {
        const float qi = qs[r * LD + i];
        if (BIDIR) n = fmaf(qi, z[i], n);
#pragma unroll
        for (int c = 0; c < CPT; ++c) acc[c] = fmaf(qi, S[i * D + cg + TPR * c], acc[c]);
    }
    if (t < T_len) {
#pragma unroll
        for (int c = 0; c < CPT; ++c)
            io<T>::st(o + base + (long long)t * D + cg + TPR * c, BIDIR ? acc[c] / n : acc[c]);
    }
}

// ------------------------------------------------------------- backward ---

// Query side of the backward pass over rows [split*rps, ...) of one head:
// writes dq and the split's partial (dS | dz) into part.
template <typename T, int D, bool BIDIR, bool PHI = BIDIR>
__global__ void __launch_bounds__(kThreads)
bwd_q(const T *__restrict__ q, const T *__restrict__ g, const float *__restrict__ state,
      T *__restrict__ dq, float *__restrict__ part, int T_len, int nsplit, int rps, float eps) {
    constexpr int TPR = kThreads / kTile;
    constexpr int CPT = D / TPR;
    constexpr int LD = D + 1;
    constexpr int R = D / 16;
    extern __shared__ float sm[];
    float *S = sm;                 // D x LD
    float *z = S + D * LD;         // D
    float *qraw = z + D;           // kTile x LD
    float *qf = qraw + kTile * LD; // kTile x LD   (feature of q, 0 on padded rows)
    float *gs = qf + kTile * LD;   // kTile x LD   (g, then g / n)
    float *wr = gs + kTile * LD;   // kTile        (-(g.o)/n)
    const int split = blockIdx.x, bh = blockIdx.y;
    const long long base = (long long)bh * T_len * D;
    const int t0 = split * rps;
    const int t1 = min(T_len, t0 + rps);
    const float *st = state + (long long)bh * D * (D + 1);
    for (int e = threadIdx.x; e < D * D; e += kThreads) S[(e / D) * LD + e % D] = st[(e / D) * (D + 1) + e % D];
    for (int e = threadIdx.x; e < D; e += kThreads) z[e] = BIDIR ? st[e * (D + 1) + D] : 0.f;
    const int ti = threadIdx.x / 16, tj = threadIdx.x % 16;
    float acc[R][R];
    float zacc[R];
#pragma unroll
    for (int x = 0; x < R; ++x) {
        zacc[x] = 0.f;
#pragma unroll
        for (int y = 0; y < R; ++y) acc[x][y] = 0.f;
    }
    const int r = threadIdx.x / TPR, cg = threadIdx.x % TPR;
    for (int ts = t0; ts < t1; ts += kTile) {
        __syncthreads();
        for (int e = threadIdx.x; e < kTile * D; e += kThreads) {
            const int rr = e / D, c = e % D, t = ts + rr;
            float x = 0.f, gg = 0.f;
            if (t < t1) {
                x = io<T>::ld(q + base + (long long)t * D + c);
                gg = io<T>::ld(g + base + (long long)t * D + c);
            }
            qraw[rr * LD + c] = x;
            qf[rr * LD + c] = (PHI && t < t1) ? feature(x) : x;
            gs[rr * LD + c] = gg;
        }
        __syncthreads();
        // Phase A: per-row outputs.
        const int t = ts + r;
        float n = eps;
        float gdot = 0.f;
        if (BIDIR) {
            float u[CPT];
#pragma unroll
            for (int c = 0; c < CPT; ++c) u[c] = 0.f;
            for (int i = 0; i < D; ++i) {
                const float qi = qf[r * LD + i];
                n = fmaf(qi, z[i], n);
#pragma unroll
                for (int c = 0; c < CPT; ++c) u[c] = fmaf(qi, S[i * LD + cg + TPR * c], u[c]);
            }
            if (t >= t1) n = 1.f;  // padded row: keep 0/0 out of the tile (its g is 0)
#pragma unroll
            for (int c = 0; c < CPT; ++c) gdot = fmaf(gs[r * LD + cg + TPR * c], u[c] / n, gdot);
#pragma unroll
            for (int m = 1; m < TPR; m <<= 1) gdot += __shfl_xor_sync(0xffffffffu, gdot, m);
        }
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
            const int i = cg + TPR * c;
            float a = 0.f;
            for (int j = 0; j < D; ++j) a = fmaf(gs[r * LD + j], S[i * LD + j], a);
            if (BIDIR) a = (a - gdot * z[i]) / n * (PHI ? feature_grad(qraw[r * LD + i]) : 1.f);
            if (t < t1) io<T>::st(dq + base + (long long)t * D + i, a);
        }
        __syncthreads();
        if (BIDIR) {
#pragma unroll
            for (int c = 0; c < CPT; ++c) gs[r * LD + cg + TPR * c] /= n;
            if (cg == 0) wr[r] = t < t1 ? -gdot / n : 0.f;
        }
        __syncthreads();
        // Phase B: dS += f(q)^T (g/n), dz += f(q)^T w.
#pragma unroll 4
        for (int rr = 0; rr < kTile; ++rr) {
            float a[R], b[R];
#pragma unroll
            for (int x = 0; x < R; ++x) {
                a[x] = qf[rr * LD + ti * R + x];
                b[x] = gs[rr * LD + tj * R + x];
            }
            const float w = BIDIR ? wr[rr] : 0.f;
#pragma unroll
            for (int x = 0; x < R; ++x) {
                if (BIDIR) zacc[x] = fmaf(a[x], w, zacc[x]);
#pragma unroll
                for (int y = 0; y < R; ++y) acc[x][y] = fmaf(a[x], b[y], acc[x][y]);
            }
        }
    }
    float *out = part + ((long long)bh * nsplit + split) * D * (D + 1);
#pragma unroll
    for (int x = 0; x < R; ++x) {
#pragma unroll
        for (int y = 0; y < R; ++y) out[(ti * R + x) * (D + 1) + tj * R + y] = acc[x][y];
        if (tj == 0) out[(ti * R + x) * (D + 1) + D] = zacc[x];
    }
}

// Key/value side: dk = (v dS^T + dz) f'(k),  dv = f(k) dS.
template <typename T, int D, bool BIDIR, bool PHI = BIDIR>
__global__ void __launch_bounds__(kThreads)
bwd_k(const T *__restrict__ k, const T *__restrict__ v, const float *__restrict__ dstate,
      T *__restrict__ dk, T *__restrict__ dv, int T_len) {
    constexpr int TPR = kThreads / kTile;
    constexpr int CPT = D / TPR;
    constexpr int LD = D + 1;
    extern __shared__ float sm[];
    float *dS = sm;                // D x LD
    float *dz = dS + D * LD;       // D
    float *kraw = dz + D;          // kTile x LD
    float *kf = kraw + kTile * LD; // kTile x LD
    float *vs = kf + kTile * LD;   // kTile x LD
    const int bh = blockIdx.y;
    const int row0 = blockIdx.x * kTile;
    const long long base = (long long)bh * T_len * D;
    const float *st = dstate + (long long)bh * D * (D + 1);
    for (int e = threadIdx.x; e < D * D; e += kThreads) dS[(e / D) * LD + e % D] = st[(e / D) * (D + 1) + e % D];
    for (int e = threadIdx.x; e < D; e += kThreads) dz[e] = BIDIR ? st[e * (D + 1) + D] : 0.f;
    for (int e = threadIdx.x; e < kTile * D; e += kThreads) {
        const int r = e / D, c = e % D, t = row0 + r;
        float x = 0.f, y = 0.f;
        if (t < T_len) {
            x = io<T>::ld(k + base + (long long)t * D + c);
            y = io<T>::ld(v + base + (long long)t * D + c);
        }
        kraw[r * LD + c] = x;
        kf[r * LD + c] = PHI ? feature(x) : x;
        vs[r * LD + c] = y;
    }
    __syncthreads();
    const int r = threadIdx.x / TPR, cg = threadIdx.x % TPR, t = row0 + r;
    if (t >= T_len) return;
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
        const int i = cg + TPR * c;
        float a = dz[i];
        for (int j = 0; j < D; ++j) a = fmaf(dS[i * LD + j], vs[r * LD + j], a);
        if (PHI) a *= feature_grad(kraw[r * LD + i]);
        io<T>::st(dk + base + (long long)t * D + i, a);
    }
    float acc[CPT];
#pragma unroll
    for (int c = 0; c < CPT; ++c) acc[c] = 0.f;
    for (int i = 0; i < D; ++i) {
        const float ki = kf[r * LD + i];
#pragma unroll
        for (int c = 0; c < CPT; ++c) acc[c] = fmaf(ki, dS[i * LD + cg + TPR * c], acc[c]);
    }
#pragma unroll
    for (int c = 0; c < CPT; ++c) io<T>::st(dv + base + (long long)t * D + cg + TPR * c, acc[c]);
}

// ------------------------------------------------------------ retention ---

// Loads rows [ts, ts+kRetTile) of up to four [T, D] tensors of one head into
// fp32 shared tiles (zero past T).
template <typename T, int D, int N, int NT>
__device__ __forceinline__ void load_rows(const T *const (&src)[N], float (*dst)[kRetTile][D], long long base,
                                          int ts, int T_len) {
    // NT threads; every load of the tile is issued before the first shared-memory store
    constexpr int PER = (kRetTile * D + NT - 1) / NT;
    float x[N][PER];
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        const int e = threadIdx.x + u * NT, t = ts + e / D;
#pragma unroll
        for (int m = 0; m < N; ++m)
            x[m][u] = e < kRetTile * D && t < T_len ? io<T>::ld(src[m] + base + (long long)t * D + e % D) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        const int e = threadIdx.x + u * NT;
        if (e < kRetTile * D) {
#pragma unroll
            for (int m = 0; m < N; ++m) dst[m][e / D][e % D] = x[m][u];
        }
    }
}

// 16 bytes of T as floats
template <typename T> struct vec16;
template <> struct vec16<float> {
    static constexpr int n = 4;
    static __device__ __forceinline__ void unpack(const uint4 &u, float *f) {
        f[0] = __uint_as_float(u.x), f[1] = __uint_as_float(u.y);
        f[2] = __uint_as_float(u.z), f[3] = __uint_as_float(u.w);
    }
};
template <> struct vec16<__half> {
    static constexpr int n = 8;
    static __device__ __forceinline__ void unpack(const uint4 &u, float *f) {
        const unsigned w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __half2 h;
            memcpy(&h, &w[i], 4);
            const float2 x = __half22float2(h);
            f[2 * i] = x.x, f[2 * i + 1] = x.y;
        }
    }
};
template <> struct vec16<__nv_bfloat16> {
    static constexpr int n = 8;
    static __device__ __forceinline__ void unpack(const uint4 &u, float *f) {
        const unsigned w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 h;
            memcpy(&h, &w[i], 4);
            const float2 x = __bfloat1622float2(h);
            f[2 * i] = x.x, f[2 * i + 1] = x.y;
        }
    }
};

// A tile of N row blocks by 16-byte loads into registers (rows are contiguous and 16-byte aligned:
// D e is a multiple of 16 and the tensors start 16-byte aligned; rows at or past T_len read as 0),
// then into shared memory as floats; NT threads, every load issued before the first store.
template <typename T, int D, int NT>
struct TileVec {
    static constexpr int VE = vec16<T>::n, NV = kRetTile * D / VE, PER = (NV + NT - 1) / NT;
};
template <typename T, int D, int N, int NT>
__device__ __forceinline__ void fetch_rows(const T *const (&src)[N], uint4 (&x)[N][TileVec<T, D, NT>::PER],
                                           long long base, int ts, int T_len) {
    using V = TileVec<T, D, NT>;
#pragma unroll
    for (int u = 0; u < V::PER; ++u) {
        const int vi = threadIdx.x + u * NT, t = ts + vi * V::VE / D;
#pragma unroll
        for (int m = 0; m < N; ++m) {
            const T *at = src[m] + base + (long long)ts * D + (long long)vi * V::VE;
            x[m][u] = vi < V::NV && t < T_len ? __ldg(reinterpret_cast<const uint4 *>(at)) : make_uint4(0u, 0u, 0u, 0u);
        }
    }
}
template <typename T, int D, int N, int NT>
__device__ __forceinline__ void stash_rows(const uint4 (&x)[N][TileVec<T, D, NT>::PER], float (*dst)[kRetTile][D]) {
    using V = TileVec<T, D, NT>;
#pragma unroll
    for (int u = 0; u < V::PER; ++u) {
        const int vi = threadIdx.x + u * NT;
        if (vi < V::NV) {
#pragma unroll
            for (int m = 0; m < N; ++m) {
                float f[V::VE];
                vec16<T>::unpack(x[m][u], f);
                float *d = &dst[m][0][0] + vi * V::VE;
#pragma unroll
                for (int w = 0; w < V::VE; w += 4)
                    *reinterpret_cast<float4 *>(d + w) = make_float4(f[w], f[w + 1], f[w + 2], f[w + 3]);
            }
        }
    }
}

// Forward recurrence, thread j holds column j of S:
//   S_t = gamma S_{t-1} + k_t^T v_t,   o_t[j] = sum_i q_t[i] S_t[i][j].
// OUT = false: the state only (q is not read, o not written; q must still point at a
// readable tensor of the same shape, e.g. k).
template <typename T, int D, bool OUT>
__global__ void __launch_bounds__(D)
ret_fwd(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v, T *__restrict__ o,
        DecayArgs dec, int T_len, int H, const float *__restrict__ sin, float *__restrict__ sout) {
    __shared__ float tiles[3][kRetTile][D];
    const int bh = blockIdx.x;
    const float gamma = dec.gamma[bh % H];
    const long long base = (long long)bh * T_len * D;
    const int j = threadIdx.x;
    float S[D];   // column j of the state (S[i] = S[i][j]); the entering state, or zero
#pragma unroll
    for (int i = 0; i < D; ++i) S[i] = sin ? sin[((long long)bh * D + i) * D + j] : 0.f;
    const T *const src[3] = {q, k, v};
    for (int ts = 0; ts < T_len; ts += kRetTile) {
        __syncthreads();
        load_rows<T, D, 3, D>(src, tiles, base, ts, T_len);
        __syncthreads();
        const int nr = min(kRetTile, T_len - ts);
        for (int r = 0; r < nr; ++r) {
            const float vj = tiles[2][r][j];
            float acc = 0.f;
#pragma unroll
            for (int i = 0; i < D; ++i) {
                S[i] = fmaf(gamma, S[i], tiles[1][r][i] * vj);
                if (OUT) acc = fmaf(tiles[0][r][i], S[i], acc);
            }
            if (OUT) io<T>::st(o + base + (long long)(ts + r) * D + j, acc);
        }
    }
    if (sout) {
#pragma unroll
        for (int i = 0; i < D; ++i) sout[((long long)bh * D + i) * D + j] = S[i];
    }
}

// Backward, forward sweep, thread i holds row i of S: dq_t[i] = sum_j S_t[i][j] g_t[j],
// S starting from the state entering the segment (sin) or zero.
template <typename T, int D>
__global__ void __launch_bounds__(D)
ret_bwd_dq(const T *__restrict__ k, const T *__restrict__ v, const T *__restrict__ g, T *__restrict__ dq,
           DecayArgs dec, int T_len, int H, const float *__restrict__ sin) {
    __shared__ float tiles[3][kRetTile][D];
    const int bh = blockIdx.x;
    const float gamma = dec.gamma[bh % H];
    const long long base = (long long)bh * T_len * D;
    const int i = threadIdx.x;
    float S[D];
#pragma unroll
    for (int j = 0; j < D; ++j) S[j] = sin ? sin[((long long)bh * D + i) * D + j] : 0.f;
    const T *const src[3] = {k, v, g};
    for (int ts = 0; ts < T_len; ts += kRetTile) {
        __syncthreads();
        load_rows<T, D, 3, D>(src, tiles, base, ts, T_len);
        __syncthreads();
        const int nr = min(kRetTile, T_len - ts);
        for (int r = 0; r < nr; ++r) {
            const float ki = tiles[0][r][i];
            float acc = 0.f;
#pragma unroll
            for (int j = 0; j < D; ++j) {
                S[j] = fmaf(gamma, S[j], ki * tiles[1][r][j]);
                acc = fmaf(S[j], tiles[2][r][j], acc);
            }
            io<T>::st(dq + base + (long long)(ts + r) * D + i, acc);
        }
    }
}

// Backward, reverse sweep over R_s = gamma R_{s+1} + q_s^T g_s.  Threads
// 0..D-1 hold row i of R (dk_s[i] = sum_j R[i][j] v_s[j]); threads D..2D-1
// hold column j of R (dv_s[j] = sum_i k_s[i] R[i][j]).  R starts from rin (R one
// past the segment's last row) or zero; rout receives R at the segment's first row.
// OUT = false: R only (rout), no dk, dv: k and v are not read (they must still point at
// readable tensors of the same shape, e.g. q and g).
template <typename T, int D, bool OUT>
__global__ void __launch_bounds__(2 * D)
ret_bwd_dkdv(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
             const T *__restrict__ g, T *__restrict__ dk, T *__restrict__ dv, DecayArgs dec, int T_len, int H,
             const float *__restrict__ rin, float *__restrict__ rout) {
    __shared__ float tiles[4][kRetTile][D];
    const int bh = blockIdx.x;
    const float gamma = dec.gamma[bh % H];
    const long long base = (long long)bh * T_len * D;
    const bool row_side = threadIdx.x < D;
    const int idx = row_side ? threadIdx.x : threadIdx.x - D;
    float Rr[D];
    const float *rb = rin ? rin + (long long)bh * D * D : nullptr;
#pragma unroll
    for (int m = 0; m < D; ++m) Rr[m] = rin ? (row_side ? rb[idx * D + m] : rb[m * D + idx]) : 0.f;
    const T *const src[4] = {q, k, v, g};
    const int ntiles = (T_len + kRetTile - 1) / kRetTile;
    for (int tile = ntiles - 1; tile >= 0; --tile) {
        const int ts = tile * kRetTile;
        __syncthreads();
        load_rows<T, D, 4, 2 * D>(src, tiles, base, ts, T_len);
        __syncthreads();
        const int nr = min(kRetTile, T_len - ts);
        for (int r = nr - 1; r >= 0; --r) {
            float acc = 0.f;
            if (row_side) {
                const float qi = tiles[0][r][idx];
#pragma unroll
                for (int j = 0; j < D; ++j) {
                    Rr[j] = fmaf(gamma, Rr[j], qi * tiles[3][r][j]);
                    if (OUT) acc = fmaf(Rr[j], tiles[2][r][j], acc);
                }
                if (OUT) io<T>::st(dk + base + (long long)(ts + r) * D + idx, acc);
            } else if (OUT) {
                const float gj = tiles[3][r][idx];
#pragma unroll
                for (int i = 0; i < D; ++i) {
                    Rr[i] = fmaf(gamma, Rr[i], tiles[0][r][i] * gj);
                    acc = fmaf(tiles[1][r][i], Rr[i], acc);
                }
                io<T>::st(dv + base + (long long)(ts + r) * D + idx, acc);
            }
        }
    }
    if (rout && row_side) {
#pragma unroll
        for (int j = 0; j < D; ++j) rout[((long long)bh * D + idx) * D + j] = Rr[j];
    }
}

// ----------------------------------------------- causal with the norm term ---
// Causal linear attention with the norm term and a per-head decay (gamma = 1 for
// plain causal linear attention), the recurrent form:
//   S_t = gamma S_{t-1} + f(k_t)^T v_t,  z_t = gamma z_{t-1} + f(k_t)
//   o_t = f(q_t) S_t / (f(q_t) . z_t + eps),  f = elu + 1 (PHI) or the identity.
// z is the state's column for a value that is always 1.

// f applied in place to the first `n` tiles of a tile stack (rows past the sequence
// are never read).
template <int D, bool PHI>
__device__ __forceinline__ void feature_tiles(float (*tiles)[kRetTile][D], int n) {
    if (PHI) {
        for (int e = threadIdx.x; e < n * kRetTile * D; e += blockDim.x) {
            float *x = &tiles[e / (kRetTile * D)][(e / D) % kRetTile][e % D];
            *x = feature(*x);
        }
    }
}
// f'(x) from f(x): elu + 1 is x + 1 > 1 for x > 0 (slope 1) and exp(x) <= 1 otherwise.
template <bool PHI>
__device__ __forceinline__ float feature_grad_of(float fx) { return PHI ? (fx > 1.f ? 1.f : fx) : 1.f; }

// The state is held in register blocks: the threads of a column group (P adjacent lanes) hold
// four columns of it, thread p the rows part_entry(p, 0 ..), and partial sums meet through xor
// shuffles among those lanes (fixed order).
// forward: column groups of four, each over D / 8 threads of 8 rows
template <int D> constexpr int causal_fwd_parts() { return D / 8; }
template <int D> constexpr int causal_fwd_threads() { return D / 4 * causal_fwd_parts<D>(); }
// dq sweep: column groups of four, each over 8 threads of D / 8 rows
template <int D> constexpr int causal_bwd_q_threads() { return D / 4 * 8; }
template <int D> constexpr int causal_bwd_kv_threads() { return D / 4 * 8; }   // as the dq sweep

template <int P>
__device__ __forceinline__ float line_sum(float s) {
#pragma unroll
    for (int m = 1; m < P; m <<= 1) s += __shfl_xor_sync(0xffffffffu, s, m);
    return s;
}

// A line's D entries are dealt to its P parts in float4 groups, round robin: part p holds
// group m = entries 4 p + 4 P m .. 4 p + 4 P m + 3, its i-th entry part_entry(p, i).  The P
// parts of a line (adjacent lanes) then read one contiguous 16 P-byte span of a shared-memory
// row per group, a single conflict-free 128-bit load each.
template <int P>
__device__ __forceinline__ int part_entry(int p, int i) { return 4 * p + 4 * P * (i >> 2) + (i & 3); }
template <int P>
__device__ __forceinline__ float4 part_group(const float *row, int p, int m) {
    return *reinterpret_cast<const float4 *>(row + 4 * p + 4 * P * m);
}
__device__ __forceinline__ float f4(const float4 &x, int e) { return e == 0 ? x.x : e == 1 ? x.y : e == 2 ? x.z : x.w; }
// The P parts (adjacent lanes, P a power of two >= 4) of a group of four lines each hold partial
// sums col[0..3] of the four lines; returns the whole sum of line (p & 3) in part p.  Fixed order:
// halves above the first four lanes first, then two exchange rounds (3 shuffles for P = 4).
template <int P>
__device__ __forceinline__ float group_reduce_scatter(const float (&col)[4], int p) {
    float c0 = col[0], c1 = col[1], c2 = col[2], c3 = col[3];
#pragma unroll
    for (int m = P / 2; m >= 4; m >>= 1) {
        c0 += __shfl_xor_sync(0xffffffffu, c0, m);
        c1 += __shfl_xor_sync(0xffffffffu, c1, m);
        c2 += __shfl_xor_sync(0xffffffffu, c2, m);
        c3 += __shfl_xor_sync(0xffffffffu, c3, m);
    }
    const bool hi = p & 2, odd = p & 1;
    float k0 = hi ? c2 : c0, k1 = hi ? c3 : c1;           // lines kept: 2 hi + 0, 2 hi + 1
    k0 += __shfl_xor_sync(0xffffffffu, hi ? c0 : c2, 2);
    k1 += __shfl_xor_sync(0xffffffffu, hi ? c1 : c3, 2);
    float kk = odd ? k1 : k0;                             // line 2 hi + odd
    kk += __shfl_xor_sync(0xffffffffu, odd ? k0 : k1, 1);
    return kk;
}

// s <- gamma s + x y, or s + x y without a decay (one FMA)
template <bool DECAY>
__device__ __forceinline__ float decay_fma(float gamma, float s, float x, float y) {
    return DECAY ? fmaf(gamma, s, x * y) : fmaf(x, y, s);
}

// ---- chunks along T.  One CTA per head runs the recurrence over too few threads to fill the
// GPU (B H CTAs), so the sequence is cut into chunks of kCausalChunk tokens, one CTA per (head,
// chunk), each starting from the state that the tokens before its chunk leave (the backward's
// reverse sweep: after its chunk).  Those states come from two short passes: every chunk's own
// state from a zero state (a sum of weighted outer products, no recurrence), then a scan over
// the chunks of one head:  S_in[c] = gamma^L S_in[c-1] + E[c-1]  (reverse: from the last chunk).
// States are [B H][chunk][D][D + 1] fp32, the last column z (forward) or r (reverse).
template <int D, int W = D + 1>
__device__ __forceinline__ const float *chunk_state(const float *st, int bh, int c) {
    return st ? st + ((long long)bh * gridDim.y + c) * D * W : nullptr;
}

// token rows per shared-memory tile of causal_chunk_state (two buffers of a and b rows: 32 KB)
template <int D> constexpr int chunk_state_rows() { return 2048 / D; }

// One tile of causal_chunk_state's inputs into registers: thread x holds entries x + 256 u of
// the tile's rows (rows at or past s1 are not read); rc: the c value of row x (x < the tile's rows).
template <typename T, int D, bool REV, int EPT>
__device__ __forceinline__ void chunk_fetch(const T *__restrict__ a, const T *__restrict__ b,
                                            const float2 *__restrict__ ndh, int ts, int s1, float (&ra)[EPT],
                                            float (&rb)[EPT], float (&rn)[EPT], float &rc) {
#pragma unroll
    for (int u = 0; u < EPT; ++u) {
        const int e = threadIdx.x + 256 * u, t = ts + e / D;
        if (t < s1) {
            ra[u] = io<T>::ld(a + (long long)t * D + e % D);
            rb[u] = io<T>::ld(b + (long long)t * D + e % D);
            if (REV) rn[u] = ndh[t].x;
        }
    }
    if (threadIdx.x < chunk_state_rows<D>()) {
        const int t = ts + threadIdx.x;
        rc = t < s1 ? (REV ? ndh[t].y : 1.f) : 0.f;
    }
}

// E[c] = sum over the chunk's tokens t of w_t a_t^T [b_t | c_t]:
//   forward (REV false): a = f(k), b = v, c = 1, w_t = gamma^(s1 - 1 - t)  (the state after the
//     chunk's last token s1 - 1, from a zero state before its first);
//   reverse (REV true):  a = f(q), b = dout / n, c = dn, w_t = gamma^(t - s0)  (R, r at the chunk's
//     first token s0, from a zero state after its last).
// 256 threads as 16 x 16; thread (ti, tj) accumulates rows 4 ti + 64 m + 0..3 by columns
// 4 tj + 64 n + 0..3 (float4 reads of the staged rows), and rows' c column for tj = 0.  Tiles
// are double buffered: the next tile's loads are in flight while the current one is summed.
template <typename T, int D, bool PHI, bool REV>
__global__ void __launch_bounds__(256)
causal_chunk_state(const T *__restrict__ a_src, const T *__restrict__ b_src, const float2 *__restrict__ nd,
                   float *__restrict__ E, DecayArgs dec, int has_decay, int T_len, int H, int L) {
    constexpr int G = D / 64;                  // float4 groups per thread and side
    constexpr int R = chunk_state_rows<D>(), EPT = R * D / 256;
    __shared__ __align__(16) float As[2][R][D];
    __shared__ __align__(16) float Bs[2][R][D];
    __shared__ float Cs[2][R];
    const int c = blockIdx.x, bh = blockIdx.y, nc = gridDim.x;
    if (REV ? c == 0 : c == nc - 1) return;    // no other chunk starts from this one's state
    const int s0 = c * L, s1 = min(T_len, s0 + L);
    const float gamma = has_decay ? dec.gamma[bh % H] : 1.f;
    const long long base = (long long)bh * T_len * D;
    const T *const a_h = a_src + base, *const b_h = b_src + base;
    const float2 *const ndh = REV ? nd + (long long)bh * T_len : nullptr;
    const int tj = threadIdx.x & 15, ti = threadIdx.x >> 4;
    float acc[4 * G][4 * G], accc[4 * G];
#pragma unroll
    for (int m = 0; m < 4 * G; ++m) {
        accc[m] = 0.f;
#pragma unroll
        for (int n = 0; n < 4 * G; ++n) acc[m][n] = 0.f;
    }
    float ra[EPT], rb[EPT], rn[EPT], rc = 0.f;
#pragma unroll
    for (int u = 0; u < EPT; ++u) ra[u] = rb[u] = rn[u] = 0.f;
    chunk_fetch<T, D, REV, EPT>(a_h, b_h, ndh, s0, s1, ra, rb, rn, rc);
    int buf = 0;
    for (int ts = s0; ts < s1; ts += R, buf ^= 1) {
        const int nr = min(R, s1 - ts);
        // the registers of this tile into buffer `buf` (last read two tiles ago, before the
        // barrier of the previous tile)
#pragma unroll
        for (int u = 0; u < EPT; ++u) {
            const int e = threadIdx.x + 256 * u, r = e / D, t = ts + r;
            float av = 0.f, bv = 0.f;
            if (r < nr) {
                const float w = has_decay ? powf(gamma, (float)(REV ? t - s0 : s1 - 1 - t)) : 1.f;
                av = (PHI ? feature(ra[u]) : ra[u]) * w;
                bv = REV ? rb[u] * (1.f / rn[u]) : rb[u];
            }
            As[buf][r][e % D] = av;
            Bs[buf][r][e % D] = bv;
        }
        if (threadIdx.x < R) Cs[buf][threadIdx.x] = rc;
        __syncthreads();
        if (ts + R < s1) chunk_fetch<T, D, REV, EPT>(a_h, b_h, ndh, ts + R, s1, ra, rb, rn, rc);
        for (int r = 0; r < nr; ++r) {
            float a[4 * G], b[4 * G];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float4 x = *reinterpret_cast<const float4 *>(&As[buf][r][64 * g + 4 * ti]);
                const float4 y = *reinterpret_cast<const float4 *>(&Bs[buf][r][64 * g + 4 * tj]);
                a[4 * g] = x.x, a[4 * g + 1] = x.y, a[4 * g + 2] = x.z, a[4 * g + 3] = x.w;
                b[4 * g] = y.x, b[4 * g + 1] = y.y, b[4 * g + 2] = y.z, b[4 * g + 3] = y.w;
            }
            const float cr = Cs[buf][r];
#pragma unroll
            for (int m = 0; m < 4 * G; ++m) {
#pragma unroll
                for (int n = 0; n < 4 * G; ++n) acc[m][n] = fmaf(a[m], b[n], acc[m][n]);
                accc[m] = fmaf(a[m], cr, accc[m]);
            }
        }
    }
    float *out = E + ((long long)bh * nc + c) * D * (D + 1);
#pragma unroll
    for (int m = 0; m < 4 * G; ++m) {
        const int i = 64 * (m / 4) + 4 * ti + m % 4;
#pragma unroll
        for (int n = 0; n < 4 * G; ++n) out[i * (D + 1) + 64 * (n / 4) + 4 * tj + n % 4] = acc[m][n];
        if (tj == 0) out[i * (D + 1) + D] = accc[m];
    }
}

// In place over the nc chunk states of each head: the state entering chunk c (forward) or the
// reverse state entering it from the chunks after it (rev), in chunk order:
//   run <- f_c run + own_c,  f_c = A[c][i] for a state row i (gated), else gamma^L.
// Every chunk but the last (rev: the first) has L tokens; the state of the last chunk visited
// is never read.  States hold per_head values, rows of row_len.
__global__ void __launch_bounds__(256)
chunk_scan(float *__restrict__ E, const float *__restrict__ A, DecayArgs dec, int has_decay, int H, int nc,
           int per_head, int row_len, int L, int rev) {
    const int bh = blockIdx.y, e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= per_head) return;
    const int rows = per_head / row_len, i = e / row_len;
    const float fl = has_decay ? (float)pow((double)dec.gamma[bh % H], (double)L) : 1.f;
    float *p = E + (long long)bh * nc * per_head + e;
    float run = 0.f;
    constexpr int kBatch = 8;                  // chunks whose loads are in flight together
    for (int n0 = 0; n0 < nc; n0 += kBatch) {
        float own[kBatch], f[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int n = n0 + u, c = rev ? nc - 1 - n : n;
            own[u] = n < nc - 1 ? p[(long long)c * per_head] : 0.f;
            f[u] = !A || n >= nc ? fl : A[((long long)bh * nc + c) * rows + i];
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int n = n0 + u, c = rev ? nc - 1 - n : n;
            if (n < nc) {
                p[(long long)c * per_head] = run;
                run = fmaf(f[u], run, own[u]);
            }
        }
    }
}

// Forward: the columns of S in groups of four; thread p of group g holds S[i][4 g + c] (c < 4)
// for its eight rows i = part_entry(p, .), so each k and q entry it reads serves four columns;
// group 0 also holds z (the column of a value that is always 1) for its rows.
template <typename T, int D, bool PHI, bool DECAY>
__global__ void __launch_bounds__(causal_fwd_threads<D>())
causal_fwd(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v, T *__restrict__ o,
           const float *__restrict__ st_in, DecayArgs dec, int has_decay, int T_len, int H, int L, float eps) {
    constexpr int P = causal_fwd_parts<D>(), DP = 8, C = 4;
    __shared__ __align__(16) float tiles[3][kRetTile][D];
    __shared__ float acc[kRetTile][D + 1];
    const int bh = blockIdx.x, s0 = blockIdx.y * L, s1 = min(T_len, s0 + L);
    const float gamma = has_decay ? dec.gamma[bh % H] : 1.f;
    const long long base = (long long)bh * T_len * D;
    const int grp = threadIdx.x / P, pp = threadIdx.x % P, j0 = C * grp;
    const bool zgrp = grp == 0, warp0 = threadIdx.x < 32;
    const float *const S0 = chunk_state<D>(st_in, bh, blockIdx.y);
    float S[C][DP], Sz[DP];
#pragma unroll
    for (int i = 0; i < DP; ++i) {
        const int x = part_entry<P>(pp, i);
#pragma unroll
        for (int c = 0; c < C; ++c) S[c][i] = S0 ? S0[x * (D + 1) + j0 + c] : 0.f;
        Sz[i] = S0 && zgrp ? S0[x * (D + 1) + D] : 0.f;
    }
    const T *const src[3] = {q, k, v};
    constexpr int NT = causal_fwd_threads<D>();
    for (int ts = s0; ts < s1; ts += kRetTile) {
        __syncthreads();
        {
            uint4 x[3][TileVec<T, D, NT>::PER];
            fetch_rows<T, D, 3, NT>(src, x, base, ts, T_len);
            stash_rows<T, D, 3, NT>(x, tiles);
        }
        __syncthreads();
        feature_tiles<D, PHI>(tiles, 2);
        __syncthreads();
        const int nr = min(kRetTile, s1 - ts);
#pragma unroll 2
        for (int r = 0; r < nr; ++r) {
            const float4 vv = *reinterpret_cast<const float4 *>(&tiles[2][r][j0]);
            float a[C][4], az[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                az[e] = 0.f;
#pragma unroll
                for (int c = 0; c < C; ++c) a[c][e] = 0.f;
            }
#pragma unroll
            for (int m = 0; m < DP / 4; ++m) {
                const float4 kk = part_group<P>(tiles[1][r], pp, m), qq = part_group<P>(tiles[0][r], pp, m);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float ke = f4(kk, e), qe = f4(qq, e);
#pragma unroll
                    for (int c = 0; c < C; ++c) {
                        S[c][4 * m + e] = decay_fma<DECAY>(gamma, S[c][4 * m + e], ke, f4(vv, c));
                        a[c][e] = fmaf(qe, S[c][4 * m + e], a[c][e]);
                    }
                    if (zgrp) {
                        Sz[4 * m + e] = DECAY ? fmaf(gamma, Sz[4 * m + e], ke) : Sz[4 * m + e] + ke;
                        az[e] = fmaf(qe, Sz[4 * m + e], az[e]);
                    }
                }
            }
            float col[C];
#pragma unroll
            for (int c = 0; c < C; ++c) col[c] = (a[c][0] + a[c][1]) + (a[c][2] + a[c][3]);
            const float mine = group_reduce_scatter<P>(col, pp);
            if (pp < C) acc[r][j0 + pp] = mine;
            if (warp0) {                          // group 0 (lanes 0 .. P - 1 of warp 0): n_t - eps
                const float zs = line_sum<P>((az[0] + az[1]) + (az[2] + az[3]));
                if (threadIdx.x == 0) acc[r][D] = zs;
            }
        }
        __syncthreads();
        for (int e = threadIdx.x; e < nr * D; e += blockDim.x) {
            const int r = e / D, c = e % D;
            io<T>::st(o + base + (long long)(ts + r) * D + c, acc[r][c] / (acc[r][D] + eps));
        }
    }
}

// Row sums over the four column groups of a warp (lane bits 3 and 4), scattered: each lane
// enters partial sums v[0 .. N) of N rows and leaves with the whole sums of N / 4 of them,
// rows (lane & 16 ? N / 2 : 0) + (lane & 8 ? N / 4 : 0) + x for x < N / 4.  Fixed order.
template <int N>
__device__ __forceinline__ void rows_reduce_scatter(const float (&v)[N], float (&out)[N / 4], int lane) {
    const bool b4 = lane & 16, b3 = lane & 8;
    float h[N / 2];
#pragma unroll
    for (int x = 0; x < N / 2; ++x)
        h[x] = (b4 ? v[N / 2 + x] : v[x]) + __shfl_xor_sync(0xffffffffu, b4 ? v[x] : v[N / 2 + x], 16);
#pragma unroll
    for (int x = 0; x < N / 4; ++x)
        out[x] = (b3 ? h[N / 4 + x] : h[x]) + __shfl_xor_sync(0xffffffffu, b3 ? h[x] : h[N / 4 + x], 8);
}

// Backward, forward sweep: dq, and per row (n_t, dn_t) for the reverse sweep, with
// u_t = f(q_t) S_t, n_t = f(q_t) . z_t + eps, dn_t = -(dout_t . u_t) / n_t^2:
//   df(q)_t[i] = (sum_j S_t[i][j] dout_t[j]) / n_t + z_t[i] dn_t,  dq = df(q) f'(q).
// S is held once, in blocks: thread p of column group g holds S[i][4 g + c] (c < 4) for the D / 8
// rows i = part_entry(p, .), and forms from them both the column sums u_t (over the 8 threads of
// the group) and the row sums of dq (over the column groups: the four of a warp by shuffles, the
// warps through shared memory); group 0 also holds z.  Each k, q entry read serves four columns
// and each v, dO entry D / 8 rows.
template <typename T, int D, bool PHI, bool DECAY>
__global__ void __launch_bounds__(causal_bwd_q_threads<D>())
causal_bwd_q(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v, const T *__restrict__ g,
             T *__restrict__ dq, float2 *__restrict__ nd, const float *__restrict__ st_in, DecayArgs dec, int has_decay,
             int T_len, int H, int L, float eps) {
    constexpr int P = 8, DP = D / P, C = 4, NT = causal_bwd_q_threads<D>(), W = NT / 32;
    extern __shared__ __align__(16) float dsm[];   // causal_bwd_q_smem<D>() bytes
    float(*tiles)[kRetTile][D] = reinterpret_cast<float(*)[kRetTile][D]>(dsm);   // f(q), f(k), v, dout
    float(*U)[D + 1] = reinterpret_cast<float(*)[D + 1]>(dsm + 4 * kRetTile * D);  // dout_t[j] u_t[j], n_t - eps
    float(*Z)[D] = reinterpret_cast<float(*)[D]>(dsm + 4 * kRetTile * D + kRetTile * (D + 1));   // z_t
    float(*A)[kRetTile][D] = reinterpret_cast<float(*)[kRetTile][D]>(dsm + 5 * kRetTile * D + kRetTile * (D + 1));
    float2 *info = reinterpret_cast<float2 *>(dsm + (5 + W) * kRetTile * D + kRetTile * (D + 1));   // (1 / n_t, dn_t)
    const int bh = blockIdx.x, s0 = blockIdx.y * L, s1 = min(T_len, s0 + L);
    const float gamma = has_decay ? dec.gamma[bh % H] : 1.f;
    const long long base = (long long)bh * T_len * D;
    const int grp = threadIdx.x / P, pp = threadIdx.x % P, j0 = C * grp;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool zgrp = grp == 0;
    const int rbase = (lane & 16 ? DP / 2 : 0) + (lane & 8 ? DP / 4 : 0);   // rows this lane's dq sums cover
    const float *const S0 = chunk_state<D>(st_in, bh, blockIdx.y);
    float S[C][DP], Sz[DP];
#pragma unroll
    for (int i = 0; i < DP; ++i) {
        const int x = part_entry<P>(pp, i);
#pragma unroll
        for (int c = 0; c < C; ++c) S[c][i] = S0 ? S0[x * (D + 1) + j0 + c] : 0.f;
        Sz[i] = S0 && zgrp ? S0[x * (D + 1) + D] : 0.f;
    }
    const T *const src[4] = {q, k, v, g};
    for (int ts = s0; ts < s1; ts += kRetTile) {
        __syncthreads();
        {
            uint4 x[4][TileVec<T, D, NT>::PER];
            fetch_rows<T, D, 4, NT>(src, x, base, ts, T_len);
            stash_rows<T, D, 4, NT>(x, tiles);
        }
        __syncthreads();
        feature_tiles<D, PHI>(tiles, 2);
        __syncthreads();
        const int nr = min(kRetTile, s1 - ts);
#pragma unroll 2
        for (int r = 0; r < nr; ++r) {
            const float4 vv = *reinterpret_cast<const float4 *>(&tiles[2][r][j0]);
            const float4 gv = *reinterpret_cast<const float4 *>(&tiles[3][r][j0]);
            float au[C][4], ad[DP], az[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                az[e] = 0.f;
#pragma unroll
                for (int c = 0; c < C; ++c) au[c][e] = 0.f;
            }
#pragma unroll
            for (int i = 0; i < DP; ++i) ad[i] = 0.f;
#pragma unroll
            for (int m = 0; m < DP / 4; ++m) {
                const float4 kk = part_group<P>(tiles[1][r], pp, m), qq = part_group<P>(tiles[0][r], pp, m);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int i = 4 * m + e;
                    const float ke = f4(kk, e), qe = f4(qq, e);
#pragma unroll
                    for (int c = 0; c < C; ++c) {
                        S[c][i] = decay_fma<DECAY>(gamma, S[c][i], ke, f4(vv, c));
                        au[c][e] = fmaf(qe, S[c][i], au[c][e]);
                        ad[i] = fmaf(S[c][i], f4(gv, c), ad[i]);
                    }
                    if (zgrp) {
                        Sz[i] = DECAY ? fmaf(gamma, Sz[i], ke) : Sz[i] + ke;
                        az[e] = fmaf(qe, Sz[i], az[e]);
                    }
                }
            }
            float col[C];
#pragma unroll
            for (int c = 0; c < C; ++c) col[c] = (au[c][0] + au[c][1]) + (au[c][2] + au[c][3]);
            const float u = group_reduce_scatter<P>(col, pp);
            if (pp < C) U[r][j0 + pp] = u * f4(gv, pp);
            if (warp == 0) {                      // group 0 (lanes 0 .. 7 of warp 0): n_t - eps
                const float zs = line_sum<P>((az[0] + az[1]) + (az[2] + az[3]));
                if (lane == 0) U[r][D] = zs;
            }
            if (zgrp) {
#pragma unroll
                for (int i = 0; i < DP; ++i) Z[r][part_entry<P>(pp, i)] = Sz[i];
            }
            float rs[DP / 4];
            rows_reduce_scatter<DP>(ad, rs, lane);
#pragma unroll
            for (int x = 0; x < DP / 4; ++x) A[warp][r][part_entry<P>(pp, rbase + x)] = rs[x];
        }
        __syncthreads();
        for (int r = warp; r < nr; r += W) {      // dout_t . u_t, a warp per row, fixed order
            float p = 0.f;
            for (int jj = lane; jj < D; jj += 32) p += U[r][jj];
#pragma unroll
            for (int m = 16; m > 0; m >>= 1) p += __shfl_xor_sync(0xffffffffu, p, m);
            if (lane == 0) {
                const float n = U[r][D] + eps, inv = 1.f / n;
                const float dn = -p * inv * inv;
                info[r] = make_float2(inv, dn);
                nd[(long long)bh * T_len + ts + r] = make_float2(n, dn);
            }
        }
        __syncthreads();
        for (int e = threadIdx.x; e < nr * D; e += NT) {
            const int r = e / D, c = e % D;
            const float2 in = info[r];
            float a = 0.f;
#pragma unroll
            for (int w = 0; w < W; ++w) a += A[w][r][c];
            const float d = fmaf(a, in.x, Z[r][c] * in.y);
            io<T>::st(dq + base + (long long)(ts + r) * D + c, d * feature_grad_of<PHI>(tiles[0][r][c]));
        }
    }
}

template <int D>
constexpr size_t causal_bwd_q_smem() {
    constexpr int W = causal_bwd_q_threads<D>() / 32;
    return (size_t)((5 + W) * kRetTile * D + kRetTile * (D + 1)) * sizeof(float) + kRetTile * sizeof(float2);
}
static_assert(((5 + 4) * kRetTile * 64 + kRetTile * 65) % 2 == 0 &&
                  ((5 + 8) * kRetTile * 128 + kRetTile * 129) % 2 == 0,
              "the float2 block of causal_bwd_q starts 8-byte aligned");

// Backward, reverse sweep over R_s = gamma R_{s+1} + f(q_s)^T du_s and r_s = gamma r_{s+1} +
// f(q_s) dn_s with du_s = dout_s / n_s:
//   dk_s[i] = (sum_j R[i][j] v_s[j] + r[i]) f'(k_s[i]),  dv_s[j] = sum_i f(k_s)[i] R[i][j].
// R is held in blocks as S in the dq sweep: thread p of column group g holds R[i][4 g + c] for the
// D / 8 rows i = part_entry(p, .); the column sums (dv) meet over the group's 8 threads, the row
// sums (dk) over the column groups (shuffles within a warp, shared memory across warps); group 0
// also holds r.
template <typename T, int D, bool PHI, bool DECAY>
__global__ void __launch_bounds__(causal_bwd_kv_threads<D>())
causal_bwd_kv(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v, const T *__restrict__ g,
              const float2 *__restrict__ nd, T *__restrict__ dk, T *__restrict__ dv, const float *__restrict__ st_in,
              DecayArgs dec, int has_decay, int T_len, int H, int L) {
    constexpr int P = 8, DP = D / P, C = 4, NT = causal_bwd_kv_threads<D>(), W = NT / 32;
    extern __shared__ __align__(16) float dsm[];   // causal_bwd_kv_smem<D>() bytes
    float(*tiles)[kRetTile][D] = reinterpret_cast<float(*)[kRetTile][D]>(dsm);   // f(q), f(k), v, dout (then du)
    float(*A)[kRetTile][D] = tiles + 4;                                          // per warp: row sums of dk
    float(*DV)[D] = reinterpret_cast<float(*)[D]>(dsm + (4 + W) * kRetTile * D);  // dv
    float(*Rr)[D] = DV + kRetTile;                                               // r_s
    float2 *info = reinterpret_cast<float2 *>(dsm + (6 + W) * kRetTile * D);    // (1 / n_s, dn_s)
    const int bh = blockIdx.x, s0 = blockIdx.y * L, s1 = min(T_len, s0 + L);
    const float gamma = has_decay ? dec.gamma[bh % H] : 1.f;
    const long long base = (long long)bh * T_len * D;
    const int grp = threadIdx.x / P, pp = threadIdx.x % P, j0 = C * grp;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool zgrp = grp == 0;
    const int rbase = (lane & 16 ? DP / 2 : 0) + (lane & 8 ? DP / 4 : 0);
    // the entering [R | r] (the tokens after this chunk)
    const float *const R0 = chunk_state<D>(st_in, bh, blockIdx.y);
    float R[C][DP], ri[DP];
#pragma unroll
    for (int i = 0; i < DP; ++i) {
        const int x = part_entry<P>(pp, i);
#pragma unroll
        for (int c = 0; c < C; ++c) R[c][i] = R0 ? R0[x * (D + 1) + j0 + c] : 0.f;
        ri[i] = R0 && zgrp ? R0[x * (D + 1) + D] : 0.f;
    }
    const T *const src[4] = {q, k, v, g};
    for (int ts = s0 + (s1 - s0 - 1) / kRetTile * kRetTile; ts >= s0; ts -= kRetTile) {
        __syncthreads();
        {
            uint4 x[4][TileVec<T, D, NT>::PER];
            fetch_rows<T, D, 4, NT>(src, x, base, ts, T_len);
            stash_rows<T, D, 4, NT>(x, tiles);
        }
        const int nr = min(kRetTile, s1 - ts);
        if (threadIdx.x < nr) {
            const float2 x = nd[(long long)bh * T_len + ts + threadIdx.x];
            info[threadIdx.x] = make_float2(1.f / x.x, x.y);
        }
        __syncthreads();
        feature_tiles<D, PHI>(tiles, 2);
        for (int e = threadIdx.x; e < nr * D; e += NT) tiles[3][e / D][e % D] *= info[e / D].x;   // du
        __syncthreads();
#pragma unroll 2
        for (int r = nr - 1; r >= 0; --r) {
            const float4 du = *reinterpret_cast<const float4 *>(&tiles[3][r][j0]);
            const float4 vv = *reinterpret_cast<const float4 *>(&tiles[2][r][j0]);
            const float dn = info[r].y;
            float av[C][4], ak[DP];
#pragma unroll
            for (int e = 0; e < 4; ++e)
#pragma unroll
                for (int c = 0; c < C; ++c) av[c][e] = 0.f;
#pragma unroll
            for (int i = 0; i < DP; ++i) ak[i] = 0.f;
#pragma unroll
            for (int m = 0; m < DP / 4; ++m) {
                const float4 qq = part_group<P>(tiles[0][r], pp, m), kk = part_group<P>(tiles[1][r], pp, m);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int i = 4 * m + e;
                    const float qe = f4(qq, e), ke = f4(kk, e);
#pragma unroll
                    for (int c = 0; c < C; ++c) {
                        R[c][i] = decay_fma<DECAY>(gamma, R[c][i], qe, f4(du, c));
                        ak[i] = fmaf(R[c][i], f4(vv, c), ak[i]);
                        av[c][e] = fmaf(ke, R[c][i], av[c][e]);
                    }
                    if (zgrp) ri[i] = DECAY ? fmaf(gamma, ri[i], qe * dn) : fmaf(qe, dn, ri[i]);
                }
            }
            float col[C];
#pragma unroll
            for (int c = 0; c < C; ++c) col[c] = (av[c][0] + av[c][1]) + (av[c][2] + av[c][3]);
            const float dvj = group_reduce_scatter<P>(col, pp);
            if (pp < C) DV[r][j0 + pp] = dvj;
            if (zgrp) {
#pragma unroll
                for (int i = 0; i < DP; ++i) Rr[r][part_entry<P>(pp, i)] = ri[i];
            }
            float rs[DP / 4];
            rows_reduce_scatter<DP>(ak, rs, lane);
#pragma unroll
            for (int x = 0; x < DP / 4; ++x) A[warp][r][part_entry<P>(pp, rbase + x)] = rs[x];
        }
        __syncthreads();
        for (int e = threadIdx.x; e < nr * D; e += NT) {   // the tile's rows, coalesced
            const int r = e / D, c = e % D;
            const long long at = base + (long long)(ts + r) * D + c;
            float a = Rr[r][c];
#pragma unroll
            for (int w = 0; w < W; ++w) a += A[w][r][c];
            io<T>::st(dk + at, a * feature_grad_of<PHI>(tiles[1][r][c]));
            io<T>::st(dv + at, DV[r][c]);
        }
    }
}

template <int D>
constexpr size_t causal_bwd_kv_smem() {
    constexpr int W = causal_bwd_kv_threads<D>() / 32;
    return (size_t)((6 + W) * kRetTile * D) * sizeof(float) + kRetTile * sizeof(float2);
}

// ------------------------------------------------------ gated linear attention ---
// Per-token, per-key-dimension decay, the recurrent form:
//   S_t = diag(a_t) S_{t-1} + k_t^T v_t,  o_t = q_t S_t,  a_t = exp(g_t), g the log gates.
// The state is held in register blocks as in the causal-norm kernels.

// exp of a gate tile in place (rows past the sequence are never read)
template <int D>
__device__ __forceinline__ void exp_tile(float (*tile)[D]) {
    for (int e = threadIdx.x; e < kRetTile * D; e += blockDim.x) tile[e / D][e % D] = expf(tile[e / D][e % D]);
}
// the state in blocks of four columns by D / 8 rows per thread, as the causal-norm sweeps
template <int D> constexpr int gated_threads() { return D / 4 * 8; }

// ---- chunks along T, as for the causal-norm kernels.  A chunk's own state from a zero state
// weights each token by the product of the gates between it and the chunk's end (forward) or
// start (reverse), exp of a running sum of log gates per key dimension i:
//   forward (REV false): E[c][i][j] = sum_t exp(sum_{u=t+1}^{s1-1} g_u[i]) k_t[i] v_t[j],
//     A[c][i] = exp(sum_{u=s0}^{s1-1} g_u[i])   (S after the chunk = diag(A) S before + E);
//   reverse (REV true):  E[c][i][j] = sum_t exp(sum_{u=s0+1}^{t} g_u[i]) q_t[i] dout_t[j],
//     A[c][i] = exp(sum_{u=s0+1}^{s1} g_u[i])   (R at s0 = E + diag(A) R at s1; no g past T).
// E is [B H][chunk][D][D], A [B H][chunk][D]; the 256 threads form the weights (256 / D per key
// dimension) and accumulate rows 4 ti + 64 m + 0..3 by columns 4 tj + 64 n + 0..3 as
// causal_chunk_state.
template <typename T, int D, bool REV>
__global__ void __launch_bounds__(256)
gated_chunk_state(const T *__restrict__ a_src, const T *__restrict__ b_src, const T *__restrict__ g,
                  float *__restrict__ E, float *__restrict__ A, int T_len, int L) {
    constexpr int G = D / 64, R = chunk_state_rows<D>(), TPC = 256 / D, RPT = R / TPC;
    __shared__ __align__(16) float As[R][D];
    __shared__ __align__(16) float Bs[R][D];
    __shared__ float Gs[R][D];
    __shared__ float Part[TPC][D];
    const int c = blockIdx.x, bh = blockIdx.y, nc = gridDim.x;
    if (REV ? c == 0 : c == nc - 1) return;    // no other chunk starts from this one's state
    const int s0 = c * L, s1 = min(T_len, s0 + L), ntiles = (s1 - s0 + R - 1) / R;
    const long long base = (long long)bh * T_len * D;
    const int tj = threadIdx.x & 15, ti = threadIdx.x >> 4;
    float acc[4 * G][4 * G];
#pragma unroll
    for (int m = 0; m < 4 * G; ++m)
#pragma unroll
        for (int n = 0; n < 4 * G; ++n) acc[m][n] = 0.f;
    float run = 0.f;                           // the running sum of log gates of dimension threadIdx.x % D
    // the tiles in the order they are summed (forward: from the chunk's end), each fetched into
    // registers while the one before it is weighted and summed
    constexpr int EPT = R * D / 256;
    float ra[EPT], rb[EPT], rg[EPT];
    const T *const a_h = a_src + base, *const b_h = b_src + base, *const g_h = g + base;
#define LA_GATED_FETCH(N_)                                                              \
    do {                                                                                \
        const int ts_ = s0 + (REV ? (N_) : ntiles - 1 - (N_)) * R, nr_ = min(R, s1 - ts_); \
        _Pragma("unroll") for (int u = 0; u < EPT; ++u) {                               \
            const int e = threadIdx.x + 256 * u, r = e / D;                             \
            const long long at = (long long)(ts_ + r) * D + e % D;                      \
            ra[u] = r < nr_ ? io<T>::ld(a_h + at) : 0.f;                                \
            rb[u] = r < nr_ ? io<T>::ld(b_h + at) : 0.f;                                \
            rg[u] = r < nr_ ? io<T>::ld(g_h + at) : 0.f;                                \
        }                                                                               \
    } while (0)
    LA_GATED_FETCH(0);
    for (int n = 0; n < ntiles; ++n) {
        const int ts = s0 + (REV ? n : ntiles - 1 - n) * R, nr = min(R, s1 - ts);
        __syncthreads();                       // the previous tile is summed
#pragma unroll
        for (int u = 0; u < EPT; ++u) {
            const int e = threadIdx.x + 256 * u;
            As[e / D][e % D] = ra[u];
            Bs[e / D][e % D] = rb[u];
            Gs[e / D][e % D] = REV && ts + e / D == s0 ? 0.f : rg[u];   // the reverse sums start after s0
        }
        __syncthreads();
        if (n + 1 < ntiles) LA_GATED_FETCH(n + 1);
        // the weights: running sums of the log gates of key dimension i over the tile, its rows
        // split over TPC threads of RPT rows each (thread part qd; parts meet in shared memory)
        const int i = threadIdx.x % D, qd = threadIdx.x / D;
        float loc = 0.f;
#pragma unroll
        for (int j = 0; j < RPT; ++j) loc += Gs[qd * RPT + j][i];
        Part[qd][i] = loc;
        __syncthreads();
        float before = 0.f, after = 0.f;        // the parts of the rows before and after this part's
#pragma unroll
        for (int q2 = 0; q2 < TPC; ++q2) {
            if (q2 < qd) before += Part[q2][i];
            if (q2 > qd) after += Part[q2][i];
        }
        if (REV) {                              // exp of the sum up to and including the row
            float sum = run + before;
#pragma unroll
            for (int j = 0; j < RPT; ++j) {
                sum += Gs[qd * RPT + j][i];
                As[qd * RPT + j][i] *= expf(sum);
            }
        } else {                                // exp of the sum of the rows after it
            float sum = run + after;
#pragma unroll
            for (int j = RPT - 1; j >= 0; --j) {
                As[qd * RPT + j][i] *= expf(sum);
                sum += Gs[qd * RPT + j][i];
            }
        }
#pragma unroll
        for (int q2 = 0; q2 < TPC; ++q2) run += Part[q2][i];
        __syncthreads();
        for (int r = 0; r < nr; ++r) {
            float a[4 * G], b[4 * G];
#pragma unroll
            for (int gq = 0; gq < G; ++gq) {
                const float4 x = *reinterpret_cast<const float4 *>(&As[r][64 * gq + 4 * ti]);
                const float4 y = *reinterpret_cast<const float4 *>(&Bs[r][64 * gq + 4 * tj]);
                a[4 * gq] = x.x, a[4 * gq + 1] = x.y, a[4 * gq + 2] = x.z, a[4 * gq + 3] = x.w;
                b[4 * gq] = y.x, b[4 * gq + 1] = y.y, b[4 * gq + 2] = y.z, b[4 * gq + 3] = y.w;
            }
#pragma unroll
            for (int m = 0; m < 4 * G; ++m)
#pragma unroll
                for (int n2 = 0; n2 < 4 * G; ++n2) acc[m][n2] = fmaf(a[m], b[n2], acc[m][n2]);
        }
    }
#undef LA_GATED_FETCH
    float *out = E + ((long long)bh * nc + c) * D * D;
#pragma unroll
    for (int m = 0; m < 4 * G; ++m) {
        const int i = 64 * (m / 4) + 4 * ti + m % 4;
#pragma unroll
        for (int n = 0; n < 4 * G; ++n) out[i * D + 64 * (n / 4) + 4 * tj + n % 4] = acc[m][n];
    }
    if (threadIdx.x < D) {
        const float next = REV && s1 < T_len ? io<T>::ld(g + base + (long long)s1 * D + threadIdx.x) : 0.f;
        A[((long long)bh * nc + c) * D + threadIdx.x] = expf(run + next);
    }
}

// dg of a sequence cut into chunks: each chunk's part (fp32, summed over its own rows from the
// end) plus the totals of the chunks after it.
template <typename T, int D>
__global__ void __launch_bounds__(256)
gated_dg_carry(const float *__restrict__ part, const float *__restrict__ totals, T *__restrict__ dg, int T_len,
               int L) {
    __shared__ float carry[D];
    const int c = blockIdx.x, bh = blockIdx.y, nc = gridDim.x;
    if (threadIdx.x < D) {
        float sum = 0.f;
        for (int c2 = nc - 1; c2 > c; --c2) sum += totals[((long long)bh * nc + c2) * D + threadIdx.x];
        carry[threadIdx.x] = sum;
    }
    __syncthreads();
    const int s0 = c * L, s1 = min(T_len, s0 + L);
    const long long base = (long long)bh * T_len * D;
    for (long long e = (long long)s0 * D + threadIdx.x; e < (long long)s1 * D; e += blockDim.x)
        io<T>::st(dg + base + e, part[base + e] + carry[e % D]);
}

// Forward: thread p of column group g holds S[i][4 g + c] (c < 4) for the D / 8 rows
// i = part_entry(p, .); o_t[j] is a column sum over the group's 8 threads.
template <typename T, int D>
__global__ void __launch_bounds__(gated_threads<D>())
gated_fwd(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v, const T *__restrict__ g,
          T *__restrict__ o, const float *__restrict__ st_in, int T_len, int L) {
    constexpr int P = 8, DP = D / P, C = 4, NT = gated_threads<D>();
    __shared__ __align__(16) float tiles[4][kRetTile][D];      // q, k, v, a = exp(g)
    __shared__ float acc[kRetTile][D];
    const int s0 = blockIdx.y * L, s1 = min(T_len, s0 + L);
    const long long base = (long long)blockIdx.x * T_len * D;
    const int grp = threadIdx.x / P, pp = threadIdx.x % P, j0 = C * grp;
    const float *const S0 = chunk_state<D, D>(st_in, blockIdx.x, blockIdx.y);
    float S[C][DP];
#pragma unroll
    for (int i = 0; i < DP; ++i)
#pragma unroll
        for (int c = 0; c < C; ++c) S[c][i] = S0 ? S0[part_entry<P>(pp, i) * D + j0 + c] : 0.f;
    const T *const src[4] = {q, k, v, g};
    for (int ts = s0; ts < s1; ts += kRetTile) {
        __syncthreads();
        {
            uint4 x[4][TileVec<T, D, NT>::PER];
            fetch_rows<T, D, 4, NT>(src, x, base, ts, T_len);
            stash_rows<T, D, 4, NT>(x, tiles);
        }
        __syncthreads();
        exp_tile<D>(tiles[3]);
        __syncthreads();
        const int nr = min(kRetTile, s1 - ts);
#pragma unroll 2
        for (int r = 0; r < nr; ++r) {
            const float4 vv = *reinterpret_cast<const float4 *>(&tiles[2][r][j0]);
            float a[C][4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
#pragma unroll
                for (int c = 0; c < C; ++c) a[c][e] = 0.f;
#pragma unroll
            for (int m = 0; m < DP / 4; ++m) {
                const float4 aa = part_group<P>(tiles[3][r], pp, m), kk = part_group<P>(tiles[1][r], pp, m),
                             qq = part_group<P>(tiles[0][r], pp, m);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int i = 4 * m + e;
#pragma unroll
                    for (int c = 0; c < C; ++c) {
                        S[c][i] = fmaf(f4(aa, e), S[c][i], f4(kk, e) * f4(vv, c));
                        a[c][e] = fmaf(f4(qq, e), S[c][i], a[c][e]);
                    }
                }
            }
            float col[C];
#pragma unroll
            for (int c = 0; c < C; ++c) col[c] = (a[c][0] + a[c][1]) + (a[c][2] + a[c][3]);
            const float oj = group_reduce_scatter<P>(col, pp);
            if (pp < C) acc[r][j0 + pp] = oj;
        }
        __syncthreads();
        for (int e = threadIdx.x; e < nr * D; e += NT)
            io<T>::st(o + base + (long long)(ts + e / D) * D + e % D, acc[e / D][e % D]);
    }
}

// Backward, forward sweep: dq_t[i] = sum_j S_t[i][j] dout_t[j], row sums over the column groups
// (the four of a warp by shuffles, the warps through shared memory).
template <typename T, int D>
__global__ void __launch_bounds__(gated_threads<D>())
gated_bwd_q(const T *__restrict__ k, const T *__restrict__ v, const T *__restrict__ g, const T *__restrict__ dout,
            T *__restrict__ dq, float *__restrict__ dq32, const float *__restrict__ st_in, int T_len, int L) {
    constexpr int P = 8, DP = D / P, C = 4, NT = gated_threads<D>(), W = NT / 32;
    extern __shared__ __align__(16) float dsm[];   // gated_bwd_q_smem<D>() bytes
    float(*tiles)[kRetTile][D] = reinterpret_cast<float(*)[kRetTile][D]>(dsm);   // k, v, a = exp(g), dout
    float(*A)[kRetTile][D] = tiles + 4;                                          // per warp: row sums of dq
    const int s0 = blockIdx.y * L, s1 = min(T_len, s0 + L);
    const long long base = (long long)blockIdx.x * T_len * D;
    const int grp = threadIdx.x / P, pp = threadIdx.x % P, j0 = C * grp;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rbase = (lane & 16 ? DP / 2 : 0) + (lane & 8 ? DP / 4 : 0);
    const float *const S0 = chunk_state<D, D>(st_in, blockIdx.x, blockIdx.y);
    float S[C][DP];
#pragma unroll
    for (int i = 0; i < DP; ++i)
#pragma unroll
        for (int c = 0; c < C; ++c) S[c][i] = S0 ? S0[part_entry<P>(pp, i) * D + j0 + c] : 0.f;
    const T *const src[4] = {k, v, g, dout};
    for (int ts = s0; ts < s1; ts += kRetTile) {
        __syncthreads();
        {
            uint4 x[4][TileVec<T, D, NT>::PER];
            fetch_rows<T, D, 4, NT>(src, x, base, ts, T_len);
            stash_rows<T, D, 4, NT>(x, tiles);
        }
        __syncthreads();
        exp_tile<D>(tiles[2]);
        __syncthreads();
        const int nr = min(kRetTile, s1 - ts);
#pragma unroll 2
        for (int r = 0; r < nr; ++r) {
            const float4 vv = *reinterpret_cast<const float4 *>(&tiles[1][r][j0]);
            const float4 gv = *reinterpret_cast<const float4 *>(&tiles[3][r][j0]);
            float ad[DP];
#pragma unroll
            for (int i = 0; i < DP; ++i) ad[i] = 0.f;
#pragma unroll
            for (int m = 0; m < DP / 4; ++m) {
                const float4 aa = part_group<P>(tiles[2][r], pp, m), kk = part_group<P>(tiles[0][r], pp, m);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int i = 4 * m + e;
#pragma unroll
                    for (int c = 0; c < C; ++c) {
                        S[c][i] = fmaf(f4(aa, e), S[c][i], f4(kk, e) * f4(vv, c));
                        ad[i] = fmaf(S[c][i], f4(gv, c), ad[i]);
                    }
                }
            }
            float rs[DP / 4];
            rows_reduce_scatter<DP>(ad, rs, lane);
#pragma unroll
            for (int x = 0; x < DP / 4; ++x) A[warp][r][part_entry<P>(pp, rbase + x)] = rs[x];
        }
        __syncthreads();
        for (int e = threadIdx.x; e < nr * D; e += NT) {
            const int r = e / D, c = e % D;
            float d = 0.f;
#pragma unroll
            for (int w = 0; w < W; ++w) d += A[w][r][c];
            const long long at = base + (long long)(ts + r) * D + c;
            io<T>::st(dq + at, d);
            dq32[at] = d;                            // unrounded, for the log gates' gradient
        }
    }
}

template <int D>
constexpr size_t gated_bwd_q_smem() { return (size_t)(4 + gated_threads<D>() / 32) * kRetTile * D * sizeof(float); }

// Backward, reverse sweep over R_t = q_t^T dout_t + diag(a_{t+1}) R_{t+1} (R after the sequence
// is 0): dk_t[i] = sum_j R[i][j] v_t[j] (row sums over the column groups), dv_t[j] = sum_i k_t[i]
// R[i][j] (column sums over a group's 8 threads), R held in blocks as S in the forward.  a_{t+1}
// of a tile's last row is the first row of the tile after it (kept in `anext`).  The log gates'
// gradient comes out of the same reverse walk: with G_t = sum_{s<=t} g_s,
// o_t = sum_{s<=t} (q_t e^{G_t}) . (k_s e^{-G_s}) v_s, so dL/dG_t = q_t dq_t - k_t dk_t and
// dg_t = sum_{s>=t} (q_s dq_s - k_s dk_s), summed by thread i of each key dimension in fp32 from
// the unrounded dq (dq32) and dk.
template <typename T, int D>
__global__ void __launch_bounds__(gated_threads<D>())
gated_bwd_kv(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v, const T *__restrict__ g,
             const T *__restrict__ dout, float *__restrict__ dq32, T *__restrict__ dk, T *__restrict__ dv,
             T *__restrict__ dg, const float *__restrict__ st_in, float *__restrict__ totals, int T_len, int L) {
    constexpr int P = 8, DP = D / P, C = 4, NT = gated_threads<D>(), W = NT / 32;
    extern __shared__ __align__(16) float dsm[];   // gated_bwd_kv_smem<D>() bytes
    float(*tiles)[kRetTile][D] = reinterpret_cast<float(*)[kRetTile][D]>(dsm);   // q, k, v, dout, a = exp(g)
    float(*A)[kRetTile][D] = tiles + 5;                                          // per warp: row sums of dk
    float(*DV)[D] = reinterpret_cast<float(*)[D]>(dsm + (5 + W) * kRetTile * D);  // dv
    float *anext = dsm + (6 + W) * kRetTile * D;     // a of the row after the tile (0 past the sequence)
    const int s0 = blockIdx.y * L, s1 = min(T_len, s0 + L);
    const long long base = (long long)blockIdx.x * T_len * D;
    const int grp = threadIdx.x / P, pp = threadIdx.x % P, j0 = C * grp;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rbase = (lane & 16 ? DP / 2 : 0) + (lane & 8 ? DP / 4 : 0);
    // the entering R (the tokens after this chunk)
    const float *const R0 = chunk_state<D, D>(st_in, blockIdx.x, blockIdx.y);
    float R[C][DP];
#pragma unroll
    for (int i = 0; i < DP; ++i)
#pragma unroll
        for (int c = 0; c < C; ++c) R[c][i] = R0 ? R0[part_entry<P>(pp, i) * D + j0 + c] : 0.f;
    float accg = 0.f;                            // thread i < D: sum over the chunk's rows after t of dL/dG[i]
    for (int e = threadIdx.x; e < D; e += NT)    // the first gate after the chunk
        anext[e] = s1 < T_len ? expf(io<T>::ld(g + base + (long long)s1 * D + e)) : 0.f;
    const T *const src[5] = {q, k, v, dout, g};
    for (int ts = s0 + (s1 - s0 - 1) / kRetTile * kRetTile; ts >= s0; ts -= kRetTile) {
        __syncthreads();
        {
            uint4 x[5][TileVec<T, D, NT>::PER];
            fetch_rows<T, D, 5, NT>(src, x, base, ts, T_len);
            stash_rows<T, D, 5, NT>(x, tiles);
        }
        __syncthreads();
        exp_tile<D>(tiles[4]);
        __syncthreads();
        const int nr = min(kRetTile, s1 - ts);
        float dqv[kRetTile];                     // thread i < D: this tile's dq32[., i], loaded during the sweep
        if (threadIdx.x < D) {
#pragma unroll
            for (int r = 0; r < kRetTile; ++r)
                dqv[r] = r < nr ? dq32[base + (long long)(ts + r) * D + threadIdx.x] : 0.f;
        }
#pragma unroll 2
        for (int r = nr - 1; r >= 0; --r) {
            const float *an = r + 1 < nr ? tiles[4][r + 1] : anext;    // a_{t+1}
            const float4 gv = *reinterpret_cast<const float4 *>(&tiles[3][r][j0]);
            const float4 vv = *reinterpret_cast<const float4 *>(&tiles[2][r][j0]);
            float ak[DP], av[C][4];
#pragma unroll
            for (int i = 0; i < DP; ++i) ak[i] = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e)
#pragma unroll
                for (int c = 0; c < C; ++c) av[c][e] = 0.f;
#pragma unroll
            for (int m = 0; m < DP / 4; ++m) {
                const float4 aa = part_group<P>(an, pp, m), qq = part_group<P>(tiles[0][r], pp, m),
                             kk = part_group<P>(tiles[1][r], pp, m);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int i = 4 * m + e;
#pragma unroll
                    for (int c = 0; c < C; ++c) {
                        R[c][i] = fmaf(f4(aa, e), R[c][i], f4(qq, e) * f4(gv, c));
                        ak[i] = fmaf(R[c][i], f4(vv, c), ak[i]);
                        av[c][e] = fmaf(f4(kk, e), R[c][i], av[c][e]);
                    }
                }
            }
            float col[C];
#pragma unroll
            for (int c = 0; c < C; ++c) col[c] = (av[c][0] + av[c][1]) + (av[c][2] + av[c][3]);
            const float dvj = group_reduce_scatter<P>(col, pp);
            if (pp < C) DV[r][j0 + pp] = dvj;
            float rs[DP / 4];
            rows_reduce_scatter<DP>(ak, rs, lane);
#pragma unroll
            for (int x = 0; x < DP / 4; ++x) A[warp][r][part_entry<P>(pp, rbase + x)] = rs[x];
        }
        __syncthreads();
        for (int e = threadIdx.x; e < nr * D; e += NT) {
            const int r = e / D, c = e % D;
            float a = 0.f;
#pragma unroll
            for (int w = 0; w < W; ++w) a += A[w][r][c];
            const long long at = base + (long long)(ts + r) * D + c;
            io<T>::st(dk + at, a);
            io<T>::st(dv + at, DV[r][c]);
        }
        if (threadIdx.x < D) {
            const int i = threadIdx.x;
#pragma unroll
            for (int r = kRetTile - 1; r >= 0; --r) {
                if (r >= nr) continue;
                const long long at = base + (long long)(ts + r) * D + i;
                float dki = 0.f;
#pragma unroll
                for (int w = 0; w < W; ++w) dki += A[w][r][i];
                accg = fmaf(tiles[0][r][i], dqv[r], accg);
                accg = fmaf(-tiles[1][r][i], dki, accg);
                // one chunk: dg itself; several: the chunk's part in fp32, in place of dq32
                // (this thread's own element, read above), completed by gated_dg_carry
                if (totals) dq32[at] = accg;
                else io<T>::st(dg + at, accg);
            }
        }
        for (int e = threadIdx.x; e < D; e += NT) anext[e] = tiles[4][0][e];
    }
    if (totals && threadIdx.x < D) totals[((long long)blockIdx.x * gridDim.y + blockIdx.y) * D + threadIdx.x] = accg;
}

template <int D>
constexpr size_t gated_bwd_kv_smem() {
    return (size_t)((6 + gated_threads<D>() / 32) * kRetTile * D + D) * sizeof(float);
}

// -------------------------------------------------------------- drivers ---

namespace {

int simt_splits(const Shape &s) { return state_splits(s, kTile); }

template <typename T, int D>
la_status state_fwd_t(bool bidir, const T *q, const T *k, const T *v, T *o, float *state, const Shape &s,
                      float eps, void *ws, cudaStream_t st) {
    const int nsplit = simt_splits(s);
    const int rps = (s.T + nsplit - 1) / nsplit;
    float *part = (float *)ws;
    float *stt = state ? state : (float *)((char *)ws + state_bytes(s, nsplit));
    const dim3 g1(nsplit, (unsigned)s.BH());
    la_status rc = bidir ? launch("simt_state_partial", state_partial<T, D, true>, g1, dim3(kThreads), 0, st, k, v,
                                  part, s.T, nsplit, rps)
                         : launch("simt_state_partial", state_partial<T, D, false>, g1, dim3(kThreads), 0, st, k, v,
                                  part, s.T, nsplit, rps);
    if (rc) return rc;
    rc = launch("simt_combine", combine, dim3((unsigned)s.BH()), dim3(kThreads), 0, st, (const float *)part, stt,
                nsplit, D * (D + 1));
    if (rc) return rc;
    const size_t smem = (size_t)(D * D + D + kTile * (D + 1)) * sizeof(float);
    const dim3 g2((s.T + kTile - 1) / kTile, (unsigned)s.BH());
    return bidir ? launch("simt_output", output<T, D, true>, g2, dim3(kThreads), smem, st, q, (const float *)stt, o,
                          s.T, eps)
                 : launch("simt_output", output<T, D, false>, g2, dim3(kThreads), smem, st, q, (const float *)stt, o,
                          s.T, eps);
}

template <typename T, int D>
la_status state_bwd_t(bool bidir, const T *q, const T *k, const T *v, const T *g, const float *state, T *dq,
                      T *dk, T *dv, const Shape &s, float eps, void *ws, cudaStream_t st) {
    const int nsplit = simt_splits(s);
    const int rps = (s.T + nsplit - 1) / nsplit;
    char *w = (char *)ws;
    float *part = (float *)w;
    float *stt = (float *)(w + state_bytes(s, nsplit));
    float *dstate = (float *)(w + state_bytes(s, nsplit) + state_bytes(s, 1));
    la_status rc;
    const dim3 g1(nsplit, (unsigned)s.BH());
    if (!state) {
        rc = bidir ? launch("simt_state_partial", state_partial<T, D, true>, g1, dim3(kThreads), 0, st, k, v, part,
                            s.T, nsplit, rps)
                   : launch("simt_state_partial", state_partial<T, D, false>, g1, dim3(kThreads), 0, st, k, v, part,
                            s.T, nsplit, rps);
        if (rc) return rc;
        rc = launch("simt_combine", combine, dim3((unsigned)s.BH()), dim3(kThreads), 0, st, (const float *)part, stt,
                    nsplit, D * (D + 1));
        if (rc) return rc;
        state = stt;
    }
    const size_t smemq = (size_t)(D * (D + 1) + D + 3 * kTile * (D + 1) + kTile) * sizeof(float);
    rc = bidir ? launch("simt_bwd_q", bwd_q<T, D, true>, g1, dim3(kThreads), smemq, st, q, g, state, dq, part, s.T,
                        nsplit, rps, eps)
               : launch("simt_bwd_q", bwd_q<T, D, false>, g1, dim3(kThreads), smemq, st, q, g, state, dq, part, s.T,
                        nsplit, rps, eps);
    if (rc) return rc;
    rc = launch("simt_combine", combine, dim3((unsigned)s.BH()), dim3(kThreads), 0, st, (const float *)part, dstate,
                nsplit, D * (D + 1));
    if (rc) return rc;
    const size_t smemk = (size_t)(D * (D + 1) + D + 3 * kTile * (D + 1)) * sizeof(float);
    const dim3 g2((s.T + kTile - 1) / kTile, (unsigned)s.BH());
    return bidir ? launch("simt_bwd_k", bwd_k<T, D, true>, g2, dim3(kThreads), smemk, st, k, v,
                          (const float *)dstate, dk, dv, s.T)
                 : launch("simt_bwd_k", bwd_k<T, D, false>, g2, dim3(kThreads), smemk, st, k, v,
                          (const float *)dstate, dk, dv, s.T);
}

// One stage of the state form (see Stage): the same kernels as state_fwd_t /
// state_bwd_t, with the state passed in or handed out instead of kept inside.
template <typename T, int D, bool BIDIR, bool PHI>
la_status stage_tt(Stage stage, const T *x, const T *y, const float *sin, float *sout, T *out1, T *out2,
                   const Shape &s, float eps, void *ws, cudaStream_t st) {
    const int nsplit = simt_splits(s);
    const int rps = (s.T + nsplit - 1) / nsplit;
    float *part = (float *)ws;
    const dim3 g1(nsplit, (unsigned)s.BH());
    const dim3 g2((s.T + kTile - 1) / kTile, (unsigned)s.BH());
    la_status rc;
    switch (stage) {
    case Stage::Reduce:
        rc = launch("simt_state_partial", state_partial<T, D, BIDIR, PHI>, g1, dim3(kThreads), 0, st, x, y, part,
                    s.T, nsplit, rps);
        if (rc) return rc;
        return launch("simt_combine", combine, dim3((unsigned)s.BH()), dim3(kThreads), 0, st, (const float *)part, sout,
                      nsplit, D * (D + 1));
    case Stage::Apply: {
        const size_t smem = (size_t)(D * D + D + kTile * (D + 1)) * sizeof(float);
        return launch("simt_output", output<T, D, BIDIR, PHI>, g2, dim3(kThreads), smem, st, x, sin, out1, s.T, eps);
    }
    case Stage::BwdQ: {
        const size_t smemq = (size_t)(D * (D + 1) + D + 3 * kTile * (D + 1) + kTile) * sizeof(float);
        rc = launch("simt_bwd_q", bwd_q<T, D, BIDIR, PHI>, g1, dim3(kThreads), smemq, st, x, y, sin, out1, part, s.T,
                    nsplit, rps, eps);
        if (rc) return rc;
        return launch("simt_combine", combine, dim3((unsigned)s.BH()), dim3(kThreads), 0, st, (const float *)part, sout,
                      nsplit, D * (D + 1));
    }
    default: {
        const size_t smemk = (size_t)(D * (D + 1) + D + 3 * kTile * (D + 1)) * sizeof(float);
        return launch("simt_bwd_k", bwd_k<T, D, BIDIR, PHI>, g2, dim3(kThreads), smemk, st, x, y, sin, out1, out2, s.T);
    }
    }
}

template <typename T, int D>
la_status stage_t(Stage stage, la_feature f, const T *x, const T *y, const float *sin, float *sout, T *out1, T *out2,
                  const Shape &s, float eps, void *ws, cudaStream_t st) {
    if (f == LA_FEATURE_ELU1) return stage_tt<T, D, true, true>(stage, x, y, sin, sout, out1, out2, s, eps, ws, st);
    if (f == LA_FEATURE_NORM) return stage_tt<T, D, true, false>(stage, x, y, sin, sout, out1, out2, s, eps, ws, st);
    return stage_tt<T, D, false, false>(stage, x, y, sin, sout, out1, out2, s, eps, ws, st);
}

template <typename T>
la_status stage_d(Stage stage, la_feature f, const void *x, const void *y, const float *sin, float *sout, void *out1,
                  void *out2, const Shape &s, float eps, void *ws, cudaStream_t st) {
    if (s.D == 64)
        return stage_t<T, 64>(stage, f, (const T *)x, (const T *)y, sin, sout, (T *)out1, (T *)out2, s, eps, ws, st);
    return stage_t<T, 128>(stage, f, (const T *)x, (const T *)y, sin, sout, (T *)out1, (T *)out2, s, eps, ws, st);
}

template <typename T>
la_status state_fwd_d(bool bidir, const void *q, const void *k, const void *v, void *o, float *state, const Shape &s,
                      float eps, void *ws, cudaStream_t st) {
    if (s.D == 64)
        return state_fwd_t<T, 64>(bidir, (const T *)q, (const T *)k, (const T *)v, (T *)o, state, s, eps, ws, st);
    return state_fwd_t<T, 128>(bidir, (const T *)q, (const T *)k, (const T *)v, (T *)o, state, s, eps, ws, st);
}

template <typename T>
la_status state_bwd_d(bool bidir, const void *q, const void *k, const void *v, const void *g, const float *state,
                      void *dq, void *dk, void *dv, const Shape &s, float eps, void *ws, cudaStream_t st) {
    if (s.D == 64)
        return state_bwd_t<T, 64>(bidir, (const T *)q, (const T *)k, (const T *)v, (const T *)g, state, (T *)dq,
                                  (T *)dk, (T *)dv, s, eps, ws, st);
    return state_bwd_t<T, 128>(bidir, (const T *)q, (const T *)k, (const T *)v, (const T *)g, state, (T *)dq,
                               (T *)dk, (T *)dv, s, eps, ws, st);
}

template <typename T, int D>
la_status decay_fwd_t(const T *q, const T *k, const T *v, T *o, const float *sin, float *sout, const DecayArgs &dec,
                      const Shape &s, cudaStream_t st) {
    if (!o)   // the state only
        return launch("simt_ret_state", ret_fwd<T, D, false>, dim3((unsigned)s.BH()), dim3(D), 0, st, k, k, v, o, dec,
                      s.T, s.H, sin, sout);
    return launch("simt_ret_fwd", ret_fwd<T, D, true>, dim3((unsigned)s.BH()), dim3(D), 0, st, q, k, v, o, dec, s.T,
                  s.H, sin, sout);
}

template <typename T, int D>
la_status decay_bwd_t(const T *q, const T *k, const T *v, const T *g, const float *sin, const float *rin, float *rout,
                      const DecayArgs &dec, T *dq, T *dk, T *dv, const Shape &s, cudaStream_t st) {
    if (!dq && !dk && !dv)   // R at the first row only
        return launch("simt_ret_bwd_state", ret_bwd_dkdv<T, D, false>, dim3((unsigned)s.BH()), dim3(2 * D), 0, st, q,
                      q, g, g, dk, dv, dec, s.T, s.H, rin, rout);
    if (dq) {   // dq == null: dk, dv only
        la_status rc = launch("simt_ret_bwd_dq", ret_bwd_dq<T, D>, dim3((unsigned)s.BH()), dim3(D), 0, st, k, v, g,
                              dq, dec, s.T, s.H, sin);
        if (rc) return rc;
    }
    return launch("simt_ret_bwd_dkdv", ret_bwd_dkdv<T, D, true>, dim3((unsigned)s.BH()), dim3(2 * D), 0, st, q, k, v,
                  g, dk, dv, dec, s.T, s.H, rin, rout);
}

}  // namespace

size_t workspace_size(la_op op, const Shape &s) {
    switch (op) {
    case LA_OP_BIDIR_FWD:
    case LA_OP_SIMPLE_FWD:
        return state_bytes(s, simt_splits(s)) + state_bytes(s, 1);
    case LA_OP_BIDIR_BWD:
    case LA_OP_SIMPLE_BWD:
        return state_bytes(s, simt_splits(s)) + 2 * state_bytes(s, 1);
    case LA_OP_STATE_REDUCE:
    case LA_OP_STATE_BWD_Q:
        return state_bytes(s, simt_splits(s));
    case LA_OP_CAUSAL_NORM_FWD:   // the chunk states
        return causal_state_bytes(s);
    case LA_OP_CAUSAL_NORM_BWD:   // (n_t, dn_t) of every row, then the chunk states
        return nd_bytes(s) + causal_state_bytes(s);
    case LA_OP_GATED_FWD:         // the chunk states and factors
        return gated_state_bytes(s);
    case LA_OP_GATED_BWD:         // dq in fp32 for the log gates' gradient, the chunk states, factors, totals
        return dq32_bytes(s) + gated_state_bytes(s) + (causal_chunks(s.T) > 1 ? gated_a_bytes(s) : 0);
    default:
        return 0;
    }
}

la_status state_stage(Stage stage, la_feature f, const void *x, const void *y, const float *sin, float *sout,
                      void *out1, void *out2, const Shape &s, la_dtype dt, float eps, void *ws, cudaStream_t st) {
    switch (dt) {
    case LA_F32: return stage_d<float>(stage, f, x, y, sin, sout, out1, out2, s, eps, ws, st);
    case LA_F16: return stage_d<__half>(stage, f, x, y, sin, sout, out1, out2, s, eps, ws, st);
    default: return stage_d<__nv_bfloat16>(stage, f, x, y, sin, sout, out1, out2, s, eps, ws, st);
    }
}

la_status state_fwd(bool bidir, const void *q, const void *k, const void *v, void *o, float *state, const Shape &s,
                    la_dtype dt, float eps, void *ws, cudaStream_t st) {
    switch (dt) {
    case LA_F32: return state_fwd_d<float>(bidir, q, k, v, o, state, s, eps, ws, st);
    case LA_F16: return state_fwd_d<__half>(bidir, q, k, v, o, state, s, eps, ws, st);
    default: return state_fwd_d<__nv_bfloat16>(bidir, q, k, v, o, state, s, eps, ws, st);
    }
}

la_status state_bwd(bool bidir, const void *q, const void *k, const void *v, const void *g, const float *state,
                    void *dq, void *dk, void *dv, const Shape &s, la_dtype dt, float eps, void *ws, cudaStream_t st) {
    switch (dt) {
    case LA_F32: return state_bwd_d<float>(bidir, q, k, v, g, state, dq, dk, dv, s, eps, ws, st);
    case LA_F16: return state_bwd_d<__half>(bidir, q, k, v, g, state, dq, dk, dv, s, eps, ws, st);
    default: return state_bwd_d<__nv_bfloat16>(bidir, q, k, v, g, state, dq, dk, dv, s, eps, ws, st);
    }
}

la_status decay_fwd(const void *q, const void *k, const void *v, void *o, const float *sin, float *sout,
                    const DecayArgs &dec, const Shape &s, la_dtype dt, cudaStream_t st) {
#define LA_RET_FWD(TY)                                                                                                 \
    return s.D == 64 ? decay_fwd_t<TY, 64>((const TY *)q, (const TY *)k, (const TY *)v, (TY *)o, sin, sout, dec, s, st) \
                     : decay_fwd_t<TY, 128>((const TY *)q, (const TY *)k, (const TY *)v, (TY *)o, sin, sout, dec, s, st)
    switch (dt) {
    case LA_F32: LA_RET_FWD(float);
    case LA_F16: LA_RET_FWD(__half);
    default: LA_RET_FWD(__nv_bfloat16);
    }
#undef LA_RET_FWD
}

la_status decay_bwd(const void *q, const void *k, const void *v, const void *g, const float *sin, const float *rin,
                    float *rout, const DecayArgs &dec, void *dq, void *dk, void *dv, const Shape &s, la_dtype dt,
                    cudaStream_t st) {
#define LA_RET_BWD(TY)                                                                                              \
    return s.D == 64 ? decay_bwd_t<TY, 64>((const TY *)q, (const TY *)k, (const TY *)v, (const TY *)g, sin, rin,      \
                                           rout, dec, (TY *)dq, (TY *)dk, (TY *)dv, s, st)                           \
                     : decay_bwd_t<TY, 128>((const TY *)q, (const TY *)k, (const TY *)v, (const TY *)g, sin, rin,     \
                                            rout, dec, (TY *)dq, (TY *)dk, (TY *)dv, s, st)
    switch (dt) {
    case LA_F32: LA_RET_BWD(float);
    case LA_F16: LA_RET_BWD(__half);
    default: LA_RET_BWD(__nv_bfloat16);
    }
#undef LA_RET_BWD
}

namespace {

// The chunk states (forward, then reverse for the backward) of every head, scanned in place.
template <typename T, int D, bool PHI, bool REV>
la_status causal_states(const void *a, const void *b, const float2 *nd, float *E, const DecayArgs &dec, int has_decay,
                        const Shape &s, cudaStream_t st) {
    const int nc = causal_chunks(s.T), per_head = D * (D + 1);
    la_status rc = launch(REV ? "simt_causal_norm_state_rev" : "simt_causal_norm_state",
                          causal_chunk_state<T, D, PHI, REV>, dim3((unsigned)nc, (unsigned)s.BH()), dim3(256), 0, st,
                          (const T *)a, (const T *)b, nd, E, dec, has_decay, s.T, s.H, kCausalChunk);
    if (rc) return rc;
    return launch("simt_chunk_scan", chunk_scan, dim3((unsigned)((per_head + 255) / 256), (unsigned)s.BH()), dim3(256),
                  0, st, E, (const float *)nullptr, dec, has_decay, s.H, nc, per_head, D + 1, kCausalChunk, (int)REV);
}

template <typename T, int D, bool PHI>
la_status causal_fwd_t(const void *q, const void *k, const void *v, void *o, const DecayArgs &dec, int has_decay,
                       const Shape &s, float eps, void *ws, cudaStream_t st) {
    const int nc = causal_chunks(s.T);
    float *E = nc > 1 ? (float *)ws : nullptr;
    if (E) {
        const la_status rc = causal_states<T, D, PHI, false>(k, v, nullptr, E, dec, has_decay, s, st);
        if (rc) return rc;
    }
    const auto kern = has_decay ? causal_fwd<T, D, PHI, true> : causal_fwd<T, D, PHI, false>;
    return launch("simt_causal_norm_fwd", kern, dim3((unsigned)s.BH(), (unsigned)nc), dim3(causal_fwd_threads<D>()), 0,
                  st, (const T *)q, (const T *)k, (const T *)v, (T *)o, (const float *)E, dec, has_decay, s.T, s.H,
                  kCausalChunk, eps);
}

template <typename T, int D, bool PHI>
la_status causal_bwd_t(const void *q, const void *k, const void *v, const void *g, void *dq, void *dk, void *dv,
                       const DecayArgs &dec, int has_decay, const Shape &s, float eps, void *ws, cudaStream_t st) {
    const int nc = causal_chunks(s.T);
    float2 *nd = (float2 *)ws;
    float *E = nc > 1 ? (float *)((char *)ws + nd_bytes(s)) : nullptr;
    const dim3 grid((unsigned)s.BH(), (unsigned)nc);
    la_status rc;
    if (E && (rc = causal_states<T, D, PHI, false>(k, v, nullptr, E, dec, has_decay, s, st))) return rc;
    const auto kq = has_decay ? causal_bwd_q<T, D, PHI, true> : causal_bwd_q<T, D, PHI, false>;
    const auto kkv = has_decay ? causal_bwd_kv<T, D, PHI, true> : causal_bwd_kv<T, D, PHI, false>;
    rc = launch("simt_causal_norm_bwd_q", kq, grid, dim3(causal_bwd_q_threads<D>()), causal_bwd_q_smem<D>(), st,
                (const T *)q, (const T *)k, (const T *)v, (const T *)g, (T *)dq, nd, (const float *)E, dec, has_decay,
                s.T, s.H, kCausalChunk, eps);
    if (rc) return rc;
    // the reverse states need every row's (n, dn) from the dq pass; they reuse the forward's buffer
    if (E && (rc = causal_states<T, D, PHI, true>(q, g, nd, E, dec, has_decay, s, st))) return rc;
    return launch("simt_causal_norm_bwd_kv", kkv, grid, dim3(causal_bwd_kv_threads<D>()), causal_bwd_kv_smem<D>(), st,
                  (const T *)q, (const T *)k, (const T *)v, (const T *)g, (const float2 *)nd, (T *)dk, (T *)dv,
                  (const float *)E, dec, has_decay, s.T, s.H, kCausalChunk);
}

// dtype x D x feature map dispatch of F<T, D, PHI>(args...)
#define LA_CAUSAL_DISPATCH(F, ...)                                                                  \
    do {                                                                                           \
        if (dt == LA_F32) {                                                                        \
            if (s.D == 64) return phi ? F<float, 64, true>(__VA_ARGS__) : F<float, 64, false>(__VA_ARGS__); \
            return phi ? F<float, 128, true>(__VA_ARGS__) : F<float, 128, false>(__VA_ARGS__);     \
        }                                                                                          \
        if (dt == LA_F16) {                                                                        \
            if (s.D == 64) return phi ? F<__half, 64, true>(__VA_ARGS__) : F<__half, 64, false>(__VA_ARGS__); \
            return phi ? F<__half, 128, true>(__VA_ARGS__) : F<__half, 128, false>(__VA_ARGS__);   \
        }                                                                                          \
        if (s.D == 64)                                                                             \
            return phi ? F<__nv_bfloat16, 64, true>(__VA_ARGS__) : F<__nv_bfloat16, 64, false>(__VA_ARGS__); \
        return phi ? F<__nv_bfloat16, 128, true>(__VA_ARGS__) : F<__nv_bfloat16, 128, false>(__VA_ARGS__); \
    } while (0)

}  // namespace

la_status causal_norm_fwd(const void *q, const void *k, const void *v, void *o, const DecayArgs &dec, int has_decay,
                          bool phi, const Shape &s, la_dtype dt, float eps, void *ws, cudaStream_t st) {
    LA_CAUSAL_DISPATCH(causal_fwd_t, q, k, v, o, dec, has_decay, s, eps, ws, st);
}

la_status causal_norm_bwd(const void *q, const void *k, const void *v, const void *g, void *dq, void *dk, void *dv,
                          const DecayArgs &dec, int has_decay, bool phi, const Shape &s, la_dtype dt, float eps,
                          void *ws, cudaStream_t st) {
    LA_CAUSAL_DISPATCH(causal_bwd_t, q, k, v, g, dq, dk, dv, dec, has_decay, s, eps, ws, st);
}
#undef LA_CAUSAL_DISPATCH

namespace {

// The gated chunk states and factors of every head, scanned in place.
template <typename T, int D, bool REV>
la_status gated_states(const void *a, const void *b, const void *g, float *E, float *A, const Shape &s,
                       cudaStream_t st) {
    const int nc = causal_chunks(s.T);
    la_status rc = launch(REV ? "simt_gated_state_rev" : "simt_gated_state", gated_chunk_state<T, D, REV>,
                          dim3((unsigned)nc, (unsigned)s.BH()), dim3(256), 0, st, (const T *)a, (const T *)b,
                          (const T *)g, E, A, s.T, kCausalChunk);
    if (rc) return rc;
    return launch("simt_chunk_scan", chunk_scan, dim3((unsigned)((D * D + 255) / 256), (unsigned)s.BH()), dim3(256), 0,
                  st, E, (const float *)A, DecayArgs{}, 0, s.H, nc, D * D, D, kCausalChunk, (int)REV);
}

template <typename T, int D>
la_status gated_fwd_t(const void *q, const void *k, const void *v, const void *g, void *o, const Shape &s, void *ws,
                      cudaStream_t st) {
    const int nc = causal_chunks(s.T);
    float *E = nc > 1 ? (float *)ws : nullptr;
    float *A = E ? (float *)((char *)ws + gated_e_bytes(s)) : nullptr;
    if (E) {
        const la_status rc = gated_states<T, D, false>(k, v, g, E, A, s, st);
        if (rc) return rc;
    }
    return launch("simt_gated_fwd", gated_fwd<T, D>, dim3((unsigned)s.BH(), (unsigned)nc), dim3(gated_threads<D>()),
                  0, st, (const T *)q, (const T *)k, (const T *)v, (const T *)g, (T *)o, (const float *)E, s.T,
                  kCausalChunk);
}

template <typename T, int D>
la_status gated_bwd_t(const void *q, const void *k, const void *v, const void *g, const void *dout, void *dq,
                      void *dk, void *dv, void *dg, const Shape &s, void *ws, cudaStream_t st) {
    const int nc = causal_chunks(s.T);
    const dim3 grid((unsigned)s.BH(), (unsigned)nc);
    float *dq32 = (float *)ws;
    char *rest = (char *)ws + dq32_bytes(s);
    float *E = nc > 1 ? (float *)rest : nullptr;
    float *A = E ? (float *)(rest + gated_e_bytes(s)) : nullptr;
    float *totals = E ? (float *)(rest + gated_e_bytes(s) + gated_a_bytes(s)) : nullptr;
    la_status rc;
    if (E && (rc = gated_states<T, D, false>(k, v, g, E, A, s, st))) return rc;
    rc = launch("simt_gated_bwd_q", gated_bwd_q<T, D>, grid, dim3(gated_threads<D>()), gated_bwd_q_smem<D>(), st,
                (const T *)k, (const T *)v, (const T *)g, (const T *)dout, (T *)dq, dq32, (const float *)E, s.T,
                kCausalChunk);
    if (rc) return rc;
    if (E && (rc = gated_states<T, D, true>(q, dout, g, E, A, s, st))) return rc;
    rc = launch("simt_gated_bwd_kv", gated_bwd_kv<T, D>, grid, dim3(gated_threads<D>()), gated_bwd_kv_smem<D>(), st,
                (const T *)q, (const T *)k, (const T *)v, (const T *)g, (const T *)dout, dq32, (T *)dk, (T *)dv,
                (T *)dg, (const float *)E, totals, s.T, kCausalChunk);
    if (rc || !E) return rc;
    return launch("simt_gated_dg_carry", gated_dg_carry<T, D>, dim3((unsigned)nc, (unsigned)s.BH()), dim3(256), 0, st,
                  (const float *)dq32, (const float *)totals, (T *)dg, s.T, kCausalChunk);
}

#define LA_GATED_DISPATCH(F, ...)                                                     \
    do {                                                                              \
        if (dt == LA_F32) return s.D == 64 ? F<float, 64>(__VA_ARGS__) : F<float, 128>(__VA_ARGS__); \
        if (dt == LA_F16) return s.D == 64 ? F<__half, 64>(__VA_ARGS__) : F<__half, 128>(__VA_ARGS__); \
        return s.D == 64 ? F<__nv_bfloat16, 64>(__VA_ARGS__) : F<__nv_bfloat16, 128>(__VA_ARGS__); \
    } while (0)

}  // namespace

la_status gated_fwd(const void *q, const void *k, const void *v, const void *g, void *o, const Shape &s, la_dtype dt,
                    void *ws, cudaStream_t st) {
    LA_GATED_DISPATCH(gated_fwd_t, q, k, v, g, o, s, ws, st);
}

la_status gated_bwd(const void *q, const void *k, const void *v, const void *g, const void *dout, void *dq, void *dk,
                    void *dv, void *dg, const Shape &s, la_dtype dt, void *ws, cudaStream_t st) {
    LA_GATED_DISPATCH(gated_bwd_t, q, k, v, g, dout, dq, dk, dv, dg, s, ws, st);
}
#undef LA_GATED_DISPATCH

}  // namespace simt
}  // namespace la
