// la_tc_causal.cu -- causal linear attention with the norm term at D = 64, fp16, on the
// tensor cores, built on the retention kernel (la_tc_retention.cu).
//
// "flash-linear-attention" README, "Different forms of linear attention": the chunkwise form
// of causal linear attention; the norm term and the feature map f as in the bidirectional
// op.  With S_t = gamma S_{t-1} + f(k_t)^T v_t, z_t = gamma z_{t-1} + f(k_t),
// n_t = f(q_t) . z_t + eps and o_t = f(q_t) S_t / n_t:
//   f(q), f(k) are formed once into the workspace (one elementwise pass);
//   forward   the retention kernel with the norm term: a column of ones next to v carries z
//             through the same products, and the epilogue divides by n_t;
//   backward  du_t = dout_t / n_t and dn_t = -(dout_t . o_t) / n_t from a forward pass that
//             also reads dout (prep); then the retention backward on (f(q), f(k), v, du) gives
//               dq~_t = sum_{s<=t} gamma^(t-s) (du_t . v_s) f(k_s)     (= S_t du_t)
//               dk~_s = sum_{t>=s} gamma^(t-s) (v_s . du_t) f(q_t)     (= R_s v_s)
//               dv_s  = sum_{t>=s} gamma^(t-s) (f(k_s) . f(q_t)) du_t  (= f(k_s) R_s);
//             dq~ and dk~ kept in fp32 (the dn terms below cancel much of them: at T = 1
//             exactly, up to eps); the terms of dn, z_t dn_t and
//             r_s = sum_{t>=s} gamma^(t-s) f(q_t) dn_t, and the derivative of f come last, on
//             CUDA cores:
//               dq_t = (dq~_t + z_t dn_t) f'(q_t),  dk_s = (dk~_s + r_s) f'(k_s),
//             with f'(x) = min(f(x), 1) for f = elu + 1.
// These are the gradients of sum(o * dout) the recurrent form gives (la.h states them).
// bf16 stays on the CUDA-core kernels: du rounded to bf16 (8 significant bits) loses too much
// to the cancellation between dq~ and z dn (gradients 7e-3 off at T = 700, beyond 5e-3).
#include "la_tc.cuh"
#include "la_tc_common.cuh"

#include <algorithm>

#ifndef LA_TRY
#define LA_TRY(x)                     \
    do {                              \
        la_status _rc = (x);          \
        if (_rc != LA_OK) return _rc; \
    } while (0)
#endif

namespace la {
namespace tc {

namespace {

constexpr int kL = 64;   // rows per chunk of the sums of dn's terms; 8 groups of 8 rows

template <bool BF>
__device__ __forceinline__ void unpack8(const uint4 u, float (&x)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2 f = h2<BF>::to_f2(w[j]);
        x[2 * j] = f.x;
        x[2 * j + 1] = f.y;
    }
}
template <bool BF>
__device__ __forceinline__ uint4 pack8(const float (&x)[8]) {
    return make_uint4(h2<BF>::from_f2(x[0], x[1]), h2<BF>::from_f2(x[2], x[3]), h2<BF>::from_f2(x[4], x[5]),
                      h2<BF>::from_f2(x[6], x[7]));
}
// gamma^m from log2 gamma (m >= 0; gamma = 1 gives 1)
__device__ __forceinline__ float gpow(float l2g, int m) { return m == 0 ? 1.f : exp2f((float)m * l2g); }

// f(q), f(k) with f = elu + 1, 8 elements (16 bytes) per step, grid-stride.
template <bool BF>
__global__ void __launch_bounds__(256)
phi_pair_kernel(const uint4 *__restrict__ q, const uint4 *__restrict__ k, uint4 *__restrict__ qf,
                uint4 *__restrict__ kf, long long n8) {
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (long long)gridDim.x * blockDim.x) {
        float a[8], b[8];
        unpack8<BF>(q[i], a);
        unpack8<BF>(k[i], b);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            a[j] = phi_f(a[j]);
            b[j] = phi_f(b[j]);
        }
        qf[i] = pack8<BF>(a);
        kf[i] = pack8<BF>(b);
    }
}

// Threads of the two kernels below: one CTA of 64 per (b, h, chunk of kL rows from row t0);
// thread (g, j) = (tid / 8, tid % 8) takes rows 8 g .. 8 g + 7 of the chunk (a group) and
// dimensions 8 j .. 8 j + 7, as 16-byte vectors.  fq, fk are f(q), f(k) (q, k themselves for
// the identity map).  Within a group, from its rows alone:
//   zl = sum_{s in group} gamma^(last - s) f(k_s),  rl = sum_{t in group} gamma^(t - first) f(q_t) dn_t.
template <bool BF>
__device__ __forceinline__ void group_sums(const uint16_t *fq, const uint16_t *fk, const float *dn, long long row0,
                                           int a, int b, int d0, float g, float (&zl)[8], float (&rl)[8]) {
#pragma unroll
    for (int j = 0; j < 8; ++j) zl[j] = rl[j] = 0.f;
    for (int i = a; i <= b; ++i) {
        float x[8];
        unpack8<BF>(*reinterpret_cast<const uint4 *>(fk + (row0 + i) * 64 + d0), x);
#pragma unroll
        for (int j = 0; j < 8; ++j) zl[j] = fmaf(g, zl[j], x[j]);
    }
    for (int i = b; i >= a; --i) {
        float x[8];
        unpack8<BF>(*reinterpret_cast<const uint4 *>(fq + (row0 + i) * 64 + d0), x);
        const float w = dn[row0 + i];
#pragma unroll
        for (int j = 0; j < 8; ++j) rl[j] = fmaf(g, rl[j], x[j] * w);
    }
}

// Each chunk's own parts, parts [BH, nch, 2, 64] fp32:
//   Z_c = sum_{s in c} gamma^(t_last - s) f(k_s)   (z at the chunk's last row, from the chunk)
//   P_c = sum_{t in c} gamma^(t - t0) f(q_t) dn_t  (r at the chunk's first row, from the chunk)
template <bool BF>
__global__ void __launch_bounds__(64)
dn_parts_kernel(const uint16_t *__restrict__ fq, const uint16_t *__restrict__ fk, const float *__restrict__ dn,
                float *__restrict__ parts, DecayArgs dec, int T, int H, int nch) {
    __shared__ float sz[8][64], sr[8][64];
    const int bh = blockIdx.x / nch, c = blockIdx.x % nch, tid = threadIdx.x;
    const int grp = tid >> 3, d0 = 8 * (tid & 7);
    const float g = dec.gamma[bh % H], l2g = log2f(g);
    const int t0 = c * kL, rows = min(kL, T - t0);
    const long long row0 = (long long)bh * T + t0;
    const int a = 8 * grp, b = min(a + 7, rows - 1);
    float zl[8], rl[8];
    group_sums<BF>(fq, fk, dn, row0, a, b, d0, g, zl, rl);
    const float wz = b >= a ? gpow(l2g, rows - 1 - b) : 0.f, wr = b >= a ? gpow(l2g, a) : 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        sz[grp][d0 + j] = wz * zl[j];
        sr[grp][d0 + j] = wr * rl[j];
    }
    __syncthreads();
    float z = 0.f, r = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        z += sz[e][tid];
        r += sr[e][tid];
    }
    float *p = parts + ((long long)bh * nch + c) * 128;
    p[tid] = z;
    p[64 + tid] = r;
}

// z entering the chunk and r leaving it from the other chunks' parts (Horner over whole
// chunks: only the last may be shorter, and it is never passed over), carried to each group,
// then the group's rows in order (z) and in reverse (r):
//   dq_t = (dq~_t + z_t dn_t) f'(q_t),  dk_s = (dk~_s + r_s) f'(k_s)
// from dq~, dk~ in fp32; f'(x) = min(f(x), 1) for elu + 1 (phi), 1 for the identity.
template <bool BF>
__global__ void __launch_bounds__(64)
dn_apply_kernel(const uint16_t *__restrict__ fq, const uint16_t *__restrict__ fk, const float *__restrict__ dn,
                const float *__restrict__ parts, const float *__restrict__ dq32, const float *__restrict__ dk32,
                uint16_t *__restrict__ dq, uint16_t *__restrict__ dk, DecayArgs dec, int phi, int T, int H, int nch) {
    __shared__ float sz[8][64], sr[8][64], zc[64], rc[64];
    const int bh = blockIdx.x / nch, c = blockIdx.x % nch, tid = threadIdx.x;
    const int grp = tid >> 3, d0 = 8 * (tid & 7);
    const float g = dec.gamma[bh % H], l2g = log2f(g), gL = gpow(l2g, kL);
    const int t0 = c * kL, rows = min(kL, T - t0);
    const long long row0 = (long long)bh * T + t0;
    {
        const float *pb = parts + (long long)bh * nch * 128;
        float z = 0.f, r = 0.f;
        for (int cc = 0; cc < c; ++cc) z = fmaf(gL, z, pb[cc * 128 + tid]);
        for (int cc = nch - 1; cc > c; --cc) r = fmaf(gL, r, pb[cc * 128 + 64 + tid]);
        zc[tid] = z;
        rc[tid] = r;
    }
    const int a = 8 * grp, b = min(a + 7, rows - 1);
    float zl[8], rl[8];
    group_sums<BF>(fq, fk, dn, row0, a, b, d0, g, zl, rl);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        sz[grp][d0 + j] = zl[j];
        sr[grp][d0 + j] = rl[j];
    }
    __syncthreads();
    if (b < a) return;
    // z at row a - 1 and r at row b + 1 (groups before this one are whole; none after a short one)
    float z[8], r[8];
    const int ngrp = (rows + 7) / 8;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        float zz = gpow(l2g, a) * zc[d0 + j];
        for (int e = 0; e < grp; ++e) zz += gpow(l2g, 8 * (grp - 1 - e)) * sz[e][d0 + j];
        float rr = gpow(l2g, rows - 1 - b) * rc[d0 + j];
        for (int e = grp + 1; e < ngrp; ++e) rr += gpow(l2g, 8 * (e - grp - 1)) * sr[e][d0 + j];
        z[j] = zz;
        r[j] = rr;
    }
    for (int i = a; i <= b; ++i) {
        const long long e = (row0 + i) * 64 + d0;
        float fkv[8], fqv[8], acc[8];
        unpack8<BF>(*reinterpret_cast<const uint4 *>(fk + e), fkv);
        unpack8<BF>(*reinterpret_cast<const uint4 *>(fq + e), fqv);
        const float4 lo = *reinterpret_cast<const float4 *>(dq32 + e), hi = *reinterpret_cast<const float4 *>(dq32 + e + 4);
        const float x[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
        const float w = dn[row0 + i];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            z[j] = fmaf(g, z[j], fkv[j]);
            acc[j] = fmaf(z[j], w, x[j]) * (phi ? fminf(fqv[j], 1.f) : 1.f);
        }
        *reinterpret_cast<uint4 *>(dq + e) = pack8<BF>(acc);
    }
    for (int i = b; i >= a; --i) {
        const long long e = (row0 + i) * 64 + d0;
        float fkv[8], fqv[8], acc[8];
        unpack8<BF>(*reinterpret_cast<const uint4 *>(fk + e), fkv);
        unpack8<BF>(*reinterpret_cast<const uint4 *>(fq + e), fqv);
        const float4 lo = *reinterpret_cast<const float4 *>(dk32 + e), hi = *reinterpret_cast<const float4 *>(dk32 + e + 4);
        const float x[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
        const float w = dn[row0 + i];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            r[j] = fmaf(g, r[j], fqv[j] * w);
            acc[j] = (x[j] + r[j]) * (phi ? fminf(fkv[j], 1.f) : 1.f);
        }
        *reinterpret_cast<uint4 *>(dk + e) = pack8<BF>(acc);
    }
}

struct CausalWs {
    uint16_t *fq, *fk, *du;
    float *dn, *parts, *dq32, *dk32;
};

static size_t align256(size_t b) { return (b + 255) & ~(size_t)255; }

// Workspace: f(q), f(k) (elu + 1 only) for both passes; the backward adds du (16-bit), dn,
// the chunk parts and dq~, dk~ (fp32).
static size_t ws_bytes(la_op op, const Shape &s, bool phi, CausalWs *w, void *base) {
    const size_t t16 = align256((size_t)s.BH() * s.T * s.D * 2), t32 = align256((size_t)s.BH() * s.T * s.D * 4);
    const size_t rowf = align256((size_t)s.BH() * s.T * sizeof(float));
    const size_t nch = (size_t)((s.T + kL - 1) / kL), partb = align256((size_t)s.BH() * nch * 128 * sizeof(float));
    char *p = static_cast<char *>(base);
    size_t off = 0;
    auto take = [&](size_t b) -> char * { char *r = p ? p + off : nullptr; off += b; return r; };
    CausalWs x{};
    if (phi) {
        x.fq = reinterpret_cast<uint16_t *>(take(t16));
        x.fk = reinterpret_cast<uint16_t *>(take(t16));
    }
    if (op == LA_OP_CAUSAL_NORM_BWD) {
        x.du = reinterpret_cast<uint16_t *>(take(t16));
        x.dn = reinterpret_cast<float *>(take(rowf));
        x.parts = reinterpret_cast<float *>(take(partb));
        x.dq32 = reinterpret_cast<float *>(take(t32));
        x.dk32 = reinterpret_cast<float *>(take(t32));
    }
    if (w) *w = x;
    return off;
}

static DecayArgs decay_or_one(const DecayArgs &dec, int has_decay, int H) {
    DecayArgs d = dec;
    if (!has_decay)
        for (int h = 0; h < H; ++h) d.gamma[h] = 1.f;
    return d;
}

static la_status phi_pair(const void *q, const void *k, const CausalWs &w, const Shape &s, cudaStream_t st) {
    const long long n8 = (long long)s.BH() * s.T * s.D / 8;
    const unsigned grid = (unsigned)std::min<long long>((n8 + 255) / 256, 148LL * 8);
    return launch("tc_causal_norm_phi", phi_pair_kernel<false>, dim3(grid), dim3(256), 0, st,
                  static_cast<const uint4 *>(q), static_cast<const uint4 *>(k), reinterpret_cast<uint4 *>(w.fq),
                  reinterpret_cast<uint4 *>(w.fk), n8);
}

}  // namespace

bool causal_norm_supported(const Shape &s, la_dtype dt) { return s.D == 64 && dt == LA_F16; }

size_t causal_norm_workspace(la_op op, const Shape &s, bool phi) { return ws_bytes(op, s, phi, nullptr, nullptr); }

la_status causal_norm_fwd(const void *q, const void *k, const void *v, void *o, const DecayArgs &dec, int has_decay,
                          bool phi, const Shape &s, la_dtype, float eps, void *ws, cudaStream_t st) {
    const DecayArgs d = decay_or_one(dec, has_decay, s.H);
    CausalWs w;
    ws_bytes(LA_OP_CAUSAL_NORM_FWD, s, phi, &w, ws);
    if (phi) LA_TRY(phi_pair(q, k, w, s, st));
    return retention_norm_fwd(phi ? w.fq : q, phi ? w.fk : k, v, o, nullptr, nullptr, d, eps, s, false, st);
}

la_status causal_norm_bwd(const void *q, const void *k, const void *v, const void *dout, void *dq, void *dk,
                          void *dv, const DecayArgs &dec, int has_decay, bool phi, const Shape &s, la_dtype,
                          float eps, void *ws, cudaStream_t st) {
    const DecayArgs d = decay_or_one(dec, has_decay, s.H);
    CausalWs w;
    ws_bytes(LA_OP_CAUSAL_NORM_BWD, s, phi, &w, ws);
    if (phi) LA_TRY(phi_pair(q, k, w, s, st));
    const void *fq = phi ? (const void *)w.fq : q, *fk = phi ? (const void *)w.fk : k;
    // du and dn
    LA_TRY(retention_norm_fwd(fq, fk, v, w.du, dout, w.dn, d, eps, s, false, st));
    // dq~ (fp32), dv, dk~ (fp32)
    LA_TRY(retention_bwd(fq, fk, v, w.du, nullptr, nullptr, nullptr, d, dq, dk, dv, s, false, st, w.dq32, w.dk32));
    const int nch = (s.T + kL - 1) / kL;
    const dim3 grid((unsigned)(s.BH() * nch));
    const auto *fq16 = static_cast<const uint16_t *>(fq), *fk16 = static_cast<const uint16_t *>(fk);
    LA_TRY(launch("tc_causal_norm_dn_parts", dn_parts_kernel<false>, grid, dim3(64), 0, st, fq16, fk16,
                  (const float *)w.dn, w.parts, d, s.T, s.H, nch));
    return launch("tc_causal_norm_dn_apply", dn_apply_kernel<false>, grid, dim3(64), 0, st, fq16, fk16,
                  (const float *)w.dn, (const float *)w.parts, (const float *)w.dq32, (const float *)w.dk32,
                  static_cast<uint16_t *>(dq), static_cast<uint16_t *>(dk), d, (int)phi, s.T, s.H, nch);
}

}  // namespace tc
}  // namespace la
