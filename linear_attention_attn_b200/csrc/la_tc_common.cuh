// la_tc_common.cuh -- pieces shared by the tensor-core kernels: the persistent tile
// partition, the 16-bit element helpers, the feature-map transform of a swizzled
// tile, state gathering and operand building.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <string.h>

#include "la_internal.cuh"
#include "la_tc_ptx.cuh"

namespace la {
namespace tc {

constexpr int kGrid = 148;          // persistent CTAs; fixed so partial-slot layout depends on the shape only
constexpr int kRows = 128;          // rows of q/k/v per tile (the UMMA M of the row-wise products)
// Warp roles: 0 TMA producer, 1 UMMA issuer + TMEM owner, 2..9 feature-map
// ("transform") warps, 10..13 epilogue warps (warp w reads TMEM lanes 32*(w%4)..).
constexpr int kXw0 = 2, kXWarps = 8, kXThreads = kXWarps * 32;
constexpr int kEw0 = 10, kEWarps = 4;
constexpr int kThreads = 448;
constexpr int kWorkers = kEWarps * 32;   // epilogue threads (named barriers 1 and 2)
constexpr int kTileBytes = kRows * 128;   // 128 rows x 64 16-bit elements, 128-byte swizzled
constexpr int kStateElems = 64 * 65;      // one fp32 [64][65] state block: S | z

// ------------------------------------------------------------- partition --
// Tiles of all heads, head-major (x = h * nt + j), split into G contiguous
// ranges with G = min(kGrid, N): CTA c takes [start(c), start(c+1)), never
// empty.  The CTAs touching head h are first_cta(h) .. last_cta(h); CTA c writes
// its partial of head h into slot c - first_cta(h), so a head's slots are
// 0 .. last_cta(h) - first_cta(h), all written.
struct Partition {
    long long N;
    int nt;
    int G;
    __host__ __device__ long long start(int c) const { return (long long)c * N / G; }
    __host__ __device__ int cta_of(long long x) const { return (int)(((x + 1) * G - 1) / N); }
    __host__ __device__ int first_cta(int h) const { return cta_of((long long)h * nt); }
    __host__ __device__ int last_cta(int h) const { return cta_of((long long)h * nt + nt - 1); }
};

__host__ __device__ inline int grid_for(long long N) { return N < kGrid ? (int)N : kGrid; }

// Upper bound of last_cta(h) - first_cta(h) + 1 over heads (G <= kGrid CTAs over BH heads).
__host__ __device__ inline int max_slots(int BH) { return (kGrid + BH - 1) / BH + 1; }

// ------------------------------------------------------------ 16-bit I/O --
// Packed pairs travel as uint32_t.  Reinterpreting a local through a pointer of
// another type breaks C++'s aliasing rules (the optimiser may then assume the
// two never alias); memcpy is the defined bit copy and compiles to a register
// move.
template <typename To, typename From>
__device__ __forceinline__ To bit_cast32(const From &x) {
    static_assert(sizeof(To) == 4 && sizeof(From) == 4, "32-bit values only");
    To t;
    memcpy(&t, &x, 4);
    return t;
}

template <bool BF16> struct h2;
template <> struct h2<false> {
    static __device__ __forceinline__ float2 to_f2(uint32_t u) { return __half22float2(bit_cast32<__half2>(u)); }
    static __device__ __forceinline__ uint32_t from_f2(float a, float b) {
        return bit_cast32<uint32_t>(__floats2half2_rn(a, b));
    }
    static __device__ __forceinline__ uint16_t one() { return 0x3C00u; }
};
template <> struct h2<true> {
    // bf16 is the upper half of an fp32: widening is a shift
    static __device__ __forceinline__ float2 to_f2(uint32_t u) {
        return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
    }
    static __device__ __forceinline__ uint32_t from_f2(float a, float b) {
        return bit_cast32<uint32_t>(__floats2bfloat162_rn(a, b));
    }
    static __device__ __forceinline__ uint16_t one() { return 0x3F80u; }
};

__device__ __forceinline__ float phi_f(float x) { return x > 0.f ? x + 1.f : __expf(x); }

// elu+1 on two packed fp16 values without leaving fp16:
//   phi(x) = max(x, 0) + 2^(min(x, 0) * log2(e))
// (x > 0 gives x + 2^0 = x + 1, x <= 0 gives e^x).  ex2.approx.f16x2 handles
// both halves in one special-function operation.
__device__ __forceinline__ uint32_t phi_h2(uint32_t x) {
    const __half2 hx = bit_cast32<__half2>(x);
    const __half2 zero = __float2half2_rn(0.f);
    const __half2 l2e = __float2half2_rn(1.4426950408889634f);
    const __half2 a = __hmul2(__hmin2(hx, zero), l2e);
    const uint32_t ai = bit_cast32<uint32_t>(a);
    uint32_t ei;
    asm("ex2.approx.f16x2 %0, %1;" : "=r"(ei) : "r"(ai));
    return bit_cast32<uint32_t>(__hadd2(__hmax2(hx, zero), bit_cast32<__half2>(ei)));
}

// The tile transforms below apply elu+1 when PHI is set and leave the values as
// they are otherwise (features computed by the caller): then only the zeroing of
// rows past the sequence end remains, and every lo part is zero (a 16-bit value
// is its own 16-bit rounding).

// Feature map elu+1 applied in place to row `row` of a 128-byte-swizzled tile
// (the row's 8 chunks are visited in an order that spreads banks); rows that
// lie past the sequence end are zeroed when `zero` is set.
template <bool BF16, bool PHI = true>
__device__ __forceinline__ void phi_row_inplace(uint8_t *tile, int row, bool zero) {
    if (!PHI && !zero) return;
    uint8_t *p = tile + row * 128;
#pragma unroll
    for (int it = 0; it < 8; ++it) {
        uint4 *c = reinterpret_cast<uint4 *>(p + ((it ^ (row & 7)) << 4));
        uint4 u = *c;
        if (zero) {
            u = make_uint4(0u, 0u, 0u, 0u);
        } else {
            uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float2 f = h2<BF16>::to_f2(w[k]);
                w[k] = h2<BF16>::from_f2(phi_f(f.x), phi_f(f.y));
            }
            u = make_uint4(w[0], w[1], w[2], w[3]);
        }
        *c = u;
    }
}

// Feature map of one whole row of a 128-byte-swizzled tile in place, all eight
// 16-byte chunks loaded before any is transformed (one shared-memory round trip
// per row).  SPLIT keeps lo = round(phi(x) - hi) at the same position of lo_tile.
template <bool BF16, bool SPLIT, bool PHI = true>
__device__ __forceinline__ void phi_row_batched(uint8_t *tile, uint8_t *lo_tile, int row) {
    if (!PHI) {
        if (SPLIT) {
#pragma unroll
            for (int c = 0; c < 8; ++c)
                *reinterpret_cast<uint4 *>(lo_tile + row * 128 + ((c ^ (row & 7)) << 4)) = make_uint4(0u, 0u, 0u, 0u);
        }
        return;
    }
    uint8_t *p = tile + row * 128;
    uint4 u[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) u[c] = *reinterpret_cast<const uint4 *>(p + ((c ^ (row & 7)) << 4));
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint32_t w[4] = {u[c].x, u[c].y, u[c].z, u[c].w}, l[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            if (!BF16 && !SPLIT) {
                w[k] = phi_h2(w[k]);
            } else {
                const float2 f = h2<BF16>::to_f2(w[k]);
                const float a = phi_f(f.x), b = phi_f(f.y);
                w[k] = h2<BF16>::from_f2(a, b);
                if (SPLIT) {
                    const float2 hv = h2<BF16>::to_f2(w[k]);
                    l[k] = h2<BF16>::from_f2(a - hv.x, b - hv.y);
                }
            }
        }
        const int off = (c ^ (row & 7)) << 4;
        *reinterpret_cast<uint4 *>(p + off) = make_uint4(w[0], w[1], w[2], w[3]);
        if (SPLIT) *reinterpret_cast<uint4 *>(lo_tile + row * 128 + off) = make_uint4(l[0], l[1], l[2], l[3]);
    }
}

// Feature map with a two-term result: hi = round(phi(x)) replaces x in place,
// lo = round(phi(x) - hi) goes to the same position of `lo_tile`.
template <bool BF16, bool PHI = true>
__device__ __forceinline__ void phi_row_split(uint8_t *tile, uint8_t *lo_tile, int row) {
    uint8_t *p = tile + row * 128;
    uint8_t *q = lo_tile + row * 128;
    if (!PHI) {
#pragma unroll
        for (int it = 0; it < 8; ++it) *reinterpret_cast<uint4 *>(q + ((it ^ (row & 7)) << 4)) = make_uint4(0u, 0u, 0u, 0u);
        return;
    }
#pragma unroll
    for (int it = 0; it < 8; ++it) {
        const int off = (it ^ (row & 7)) << 4;
        uint4 u = *reinterpret_cast<uint4 *>(p + off);
        uint32_t w[4] = {u.x, u.y, u.z, u.w}, l[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            float2 f = h2<BF16>::to_f2(w[k]);
            const float a = phi_f(f.x), b = phi_f(f.y);
            w[k] = h2<BF16>::from_f2(a, b);
            const float2 hv = h2<BF16>::to_f2(w[k]);
            l[k] = h2<BF16>::from_f2(a - hv.x, b - hv.y);
        }
        *reinterpret_cast<uint4 *>(p + off) = make_uint4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<uint4 *>(q + off) = make_uint4(l[0], l[1], l[2], l[3]);
    }
}

// The transform warps split a tile into 256 half rows: thread xi handles row
// xi % 128, logical chunks 4 * (xi / 128) .. + 3 (chunk order spreads banks).
template <bool BF16, bool PHI = true>
__device__ __forceinline__ void phi_half_row(uint8_t *tile, int xi, bool zero) {
    if (!PHI && !zero) return;
    const int row = xi & 127, c0 = (xi >> 7) * 4;
    uint8_t *p = tile + row * 128;
#pragma unroll
    for (int it = 0; it < 4; ++it) {
        uint4 *c = reinterpret_cast<uint4 *>(p + (((c0 + it) ^ (row & 7)) << 4));
        uint4 u = *c;
        if (zero) {
            u = make_uint4(0u, 0u, 0u, 0u);
        } else if (!BF16) {
            u = make_uint4(phi_h2(u.x), phi_h2(u.y), phi_h2(u.z), phi_h2(u.w));
        } else {
            uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 f = h2<BF16>::to_f2(w[k]);
                w[k] = h2<BF16>::from_f2(phi_f(f.x), phi_f(f.y));
            }
            u = make_uint4(w[0], w[1], w[2], w[3]);
        }
        *c = u;
    }
}

// As phi_half_row, keeping lo = round(phi(x) - hi) in lo_tile (zeroing both when `zero`).
template <bool BF16, bool PHI = true>
__device__ __forceinline__ void phi_half_row_split(uint8_t *tile, uint8_t *lo_tile, int xi, bool zero) {
    const int row = xi & 127, c0 = (xi >> 7) * 4;
#pragma unroll
    for (int it = 0; it < 4; ++it) {
        const int off = row * 128 + (((c0 + it) ^ (row & 7)) << 4);
        uint4 u = *reinterpret_cast<uint4 *>(tile + off);
        uint32_t w[4] = {u.x, u.y, u.z, u.w}, l[4] = {0u, 0u, 0u, 0u};
        if (zero) {
            w[0] = w[1] = w[2] = w[3] = 0u;
        } else if (PHI) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 f = h2<BF16>::to_f2(w[k]);
                const float a = phi_f(f.x), b = phi_f(f.y);
                w[k] = h2<BF16>::from_f2(a, b);
                const float2 hv = h2<BF16>::to_f2(w[k]);
                l[k] = h2<BF16>::from_f2(a - hv.x, b - hv.y);
            }
        }
        *reinterpret_cast<uint4 *>(tile + off) = make_uint4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<uint4 *>(lo_tile + off) = make_uint4(l[0], l[1], l[2], l[3]);
    }
}

// 16 elements (logical columns 16*c16 .. +15) of row `row` of a swizzled tile.
template <bool BF16>
__device__ __forceinline__ void load_chunk16(const uint8_t *tile, int row, int c16, float (&out)[16]) {
    const uint8_t *p = tile + row * 128;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint4 u = *reinterpret_cast<const uint4 *>(p + (((2 * c16 + h) ^ (row & 7)) << 4));
        const float2 a = h2<BF16>::to_f2(u.x), b = h2<BF16>::to_f2(u.y), d = h2<BF16>::to_f2(u.z),
                     e = h2<BF16>::to_f2(u.w);
        out[h * 8 + 0] = a.x; out[h * 8 + 1] = a.y; out[h * 8 + 2] = b.x; out[h * 8 + 3] = b.y;
        out[h * 8 + 4] = d.x; out[h * 8 + 5] = d.y; out[h * 8 + 6] = e.x; out[h * 8 + 7] = e.y;
    }
}

template <bool BF16>
__device__ __forceinline__ void store_chunk16(uint8_t *tile, int row, int c16, const float (&v)[16]) {
    uint8_t *p = tile + row * 128;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint4 u;
        u.x = h2<BF16>::from_f2(v[h * 8 + 0], v[h * 8 + 1]);
        u.y = h2<BF16>::from_f2(v[h * 8 + 2], v[h * 8 + 3]);
        u.z = h2<BF16>::from_f2(v[h * 8 + 4], v[h * 8 + 5]);
        u.w = h2<BF16>::from_f2(v[h * 8 + 6], v[h * 8 + 7]);
        *reinterpret_cast<uint4 *>(p + (((2 * c16 + h) ^ (row & 7)) << 4)) = u;
    }
}

// Reads the 64 elements of row `row` of a swizzled 16-bit tile into fp32.
template <bool BF16>
__device__ __forceinline__ void load_row(const uint8_t *tile, int row, float (&out)[64]) {
    const uint8_t *p = tile + row * 128;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint4 u = *reinterpret_cast<const uint4 *>(p + ((c ^ (row & 7)) << 4));
        float2 a = h2<BF16>::to_f2(u.x), b = h2<BF16>::to_f2(u.y), d = h2<BF16>::to_f2(u.z),
               e = h2<BF16>::to_f2(u.w);
        out[c * 8 + 0] = a.x; out[c * 8 + 1] = a.y; out[c * 8 + 2] = b.x; out[c * 8 + 3] = b.y;
        out[c * 8 + 4] = d.x; out[c * 8 + 5] = d.y; out[c * 8 + 6] = e.x; out[c * 8 + 7] = e.y;
    }
}

// Writes 64 fp32 values as row `row` of a swizzled 16-bit tile (round to nearest even).
template <bool BF16>
__device__ __forceinline__ void store_row(uint8_t *tile, int row, const float (&v)[64]) {
    uint8_t *p = tile + row * 128;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint4 u;
        u.x = h2<BF16>::from_f2(v[c * 8 + 0], v[c * 8 + 1]);
        u.y = h2<BF16>::from_f2(v[c * 8 + 2], v[c * 8 + 3]);
        u.z = h2<BF16>::from_f2(v[c * 8 + 4], v[c * 8 + 5]);
        u.w = h2<BF16>::from_f2(v[c * 8 + 6], v[c * 8 + 7]);
        *reinterpret_cast<uint4 *>(p + ((c ^ (row & 7)) << 4)) = u;
    }
}

// 64 fp32 accumulator columns [col, col+64) of this warp's TMEM lanes.
__device__ __forceinline__ void tmem_row64(uint32_t taddr, float (&v)[64]) {
    float a[16], b[16], c[16], d[16];
    tmem_ld16(taddr + 0, a);
    tmem_ld16(taddr + 16, b);
    tmem_ld16(taddr + 32, c);
    tmem_ld16(taddr + 48, d);
    tmem_ld_wait(a, b);
    reg_keep(c);
    reg_keep(d);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        v[i] = a[i];
        v[16 + i] = b[i];
        v[32 + i] = c[i];
        v[48 + i] = d[i];
    }
}

// ------------------------------------------------------------- state I/O --
// stage[e] = sum over s in [0, nslots) of src[s * kStateElems + e], in slot order
// (a fixed order: the result does not depend on which CTA finished first).
// Blocks are 16-byte aligned, so the copy runs on float4s with all of a slot's
// loads in flight at once.  Returns this thread's max |stage[e]| over its elements.
__device__ __forceinline__ float gather_state(const float *__restrict__ src, int nslots, float *stage, int tid) {
    constexpr int N4 = kStateElems / 4;                  // 1040 float4 per block
    constexpr int PER = (N4 + kWorkers - 1) / kWorkers;  // 9 per thread
    const float4 *s4 = reinterpret_cast<const float4 *>(src);
    float4 acc[PER];
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        const int e = tid + u * kWorkers;
        acc[u] = e < N4 ? __ldg(s4 + e) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int sl = 1; sl < nslots; ++sl) {
        float4 nx[PER];
#pragma unroll
        for (int u = 0; u < PER; ++u) {
            const int e = tid + u * kWorkers;
            nx[u] = e < N4 ? __ldg(s4 + (long long)sl * N4 + e) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < PER; ++u) {
            acc[u].x += nx[u].x;
            acc[u].y += nx[u].y;
            acc[u].z += nx[u].z;
            acc[u].w += nx[u].w;
        }
    }
    float m = 0.f;
    float4 *st4 = reinterpret_cast<float4 *>(stage);
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        const int e = tid + u * kWorkers;
        if (e < N4) {
            st4[e] = acc[u];
            m = fmaxf(m, fmaxf(fmaxf(fabsf(acc[u].x), fabsf(acc[u].y)), fmaxf(fabsf(acc[u].z), fabsf(acc[u].w))));
        }
    }
    return m;
}

// Max over the 128 worker threads (named barrier 2); `red` is 4 floats of smem.
__device__ __forceinline__ float workers_max(float m, float *red, int tid) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((tid & 31) == 0) red[tid >> 5] = m;
    named_bar(2, kWorkers);
    m = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    named_bar(2, kWorkers);
    return m;
}

// Power-of-two scale that puts max |x| = m in [2^13, 2^14) for fp16 operands
// (range and subnormal safety); bf16 shares fp32's range and needs none.
template <bool BF16>
__device__ __forceinline__ float operand_scale(float m) {
    if (BF16 || !(m > 0.f) || !isfinite(m)) return 1.f;
    int e;
    frexpf(m, &e);                        // m = f * 2^e, f in [0.5, 1)
    e = 14 - e;
    e = e < -100 ? -100 : (e > 100 ? 100 : e);
    return ldexpf(1.f, e);
}

// This worker thread's max |stage[e]| over the float4s gather_state would have given it.
__device__ __forceinline__ float stage_absmax(const float *stage, int tid) {
    const float4 *st4 = reinterpret_cast<const float4 *>(stage);
    float m = 0.f;
    for (int e = tid; e < kStateElems / 4; e += kWorkers) {
        const float4 a = st4[e];
        m = fmaxf(m, fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(a.z), fabsf(a.w))));
    }
    return m;
}

// Two-term 16-bit split (bf16 or fp16) of 16 fp32 values, packed in pairs: hi = round(x),
// lo = round(x - hi) (x - hi is exact in fp32).
template <bool BF16 = true>
__device__ __forceinline__ void split_hi_lo16_packed(const float (&x)[16], uint32_t (&hw)[8], uint32_t (&lw)[8]) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        hw[k] = h2<BF16>::from_f2(x[2 * k], x[2 * k + 1]);
        const float2 hv = h2<BF16>::to_f2(hw[k]);
        lw[k] = h2<BF16>::from_f2(x[2 * k] - hv.x, x[2 * k + 1] - hv.y);
    }
}

// store_chunk16 with the 16 values already packed in pairs.
__device__ __forceinline__ void store_chunk16_packed(uint8_t *tile, int row, int c16, const uint32_t (&w)[8]) {
    uint8_t *p = tile + row * 128;
#pragma unroll
    for (int h = 0; h < 2; ++h)
        *reinterpret_cast<uint4 *>(p + (((2 * c16 + h) ^ (row & 7)) << 4)) =
            make_uint4(w[4 * h], w[4 * h + 1], w[4 * h + 2], w[4 * h + 3]);
}

// (head, tile-in-head) of the tile indices x0, x0 + 1, ... of a Partition, advanced
// without a 64-bit division per tile (an emulated division costs hundreds of cycles).
struct TileCursor {
    long long x;
    int h, j, nt;
    __device__ __forceinline__ TileCursor(long long x0, int nt_)
        : x(x0), h((int)(x0 / nt_)), j((int)(x0 % nt_)), nt(nt_) {}
    __device__ __forceinline__ void next() {
        ++x;
        if (++j == nt) { j = 0; ++h; }
    }
    __device__ __forceinline__ bool last_of_head() const { return j + 1 == nt; }
};

// Rows [0, nrows) of a K-major 128-byte-swizzled 16-bit operand (64 K values per
// row) from the fp32 state block [64][65] in shared memory, scaled by sc:
//   COLUMNS:  row n, element i = stage[i][n]  (column n of S; n == 64 is z when
//             with_z, and rows without a source are zero)
//   !COLUMNS: row n, element i = stage[n][i]  (row n of S)
// hi = round(x), lo = round(x - hi) (lo only with NOPS == 2).  The 128 worker
// threads take (row, 8-element chunk) pairs, consecutive rows in consecutive
// threads, so neither the reads (row stride 65 words) nor the swizzled 16-byte
// writes conflict.  The loop stays rolled: this runs once per head, and an
// unrolled copy costs more in cold instruction fetch than it saves.
template <bool BF16, int NOPS, bool COLUMNS>
__device__ __forceinline__ void build_state_operand(const float *stage, float sc, int nrows, bool with_z, uint8_t *op0,
                                                    uint8_t *op1, int tid) {
#pragma unroll 1
    for (int task = tid; task < nrows * 8; task += kWorkers) {
        const int n = task % nrows, c = task / nrows;
        float x[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int i = 8 * c + k;
            if (COLUMNS)
                x[k] = (n < 64 || (n == 64 && with_z)) ? stage[i * 65 + n] * sc : 0.f;
            else
                x[k] = stage[n * 65 + i] * sc;
        }
        const int off = n * 128 + ((c ^ (n & 7)) << 4);
        uint4 u;
        u.x = h2<BF16>::from_f2(x[0], x[1]);
        u.y = h2<BF16>::from_f2(x[2], x[3]);
        u.z = h2<BF16>::from_f2(x[4], x[5]);
        u.w = h2<BF16>::from_f2(x[6], x[7]);
        *reinterpret_cast<uint4 *>(op0 + off) = u;
        if (NOPS == 2) {
            const uint32_t hw[4] = {u.x, u.y, u.z, u.w};
            uint32_t lw[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 hv = h2<BF16>::to_f2(hw[k]);
                lw[k] = h2<BF16>::from_f2(x[2 * k] - hv.x, x[2 * k + 1] - hv.y);
            }
            *reinterpret_cast<uint4 *>(op1 + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
    }
}

// sum_i |stage[i][64]| (the z column), the same value in every lane of the warp.
__device__ __forceinline__ float warp_abs_z_sum(const float *stage, int lane) {
    float v = fabsf(stage[lane * 65 + 64]) + fabsf(stage[(lane + 32) * 65 + 64]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

}  // namespace tc
}  // namespace la
