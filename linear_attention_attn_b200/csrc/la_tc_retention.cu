// la_tc_retention.cu -- tensor-core kernel of causal linear attention with a per-head
// scalar decay (retention), forward, bf16 storage, D = 128, fp32 accumulation.
//
// "flash-linear-attention" README, "Benchmarks" (RetNet) and "Different forms of
// linear attention" (FusedChunk: chunkwise, the inter-chunk state kept on chip,
// one program per (b, h)).  With chunk c covering rows cC .. cC+C-1 (C = 64),
// local indices i, j in [0, C), M_ij = gamma^(i-j) [i >= j], and the state
// entering chunk c, S_c = sum_{s < cC} gamma^(cC-1-s) k_s^T v_s (S_0 = 0):
//   O_c     = ((Q_c K_c^T) o M) V_c + diag(gamma^(i+1)) Q_c S_c
//   S_{c+1} = gamma^C S_c + K_c^T diag(gamma^(C-1-j)) V_c
// which is o_t = sum_{s<=t} gamma^(t-s) (q_t . k_s) v_s regrouped by chunk.
//
// One CTA per (b, h) walks the chunks in order.  Warp 0 streams q/k/v chunks
// with TMA (two 64-column boxes per 64-row chunk, 128-byte swizzle); warp 1
// issues the UMMAs of chunk c in the order dS, O_intra, P of chunk c + 1,
// O_inter, so that dS (which does not depend on the state), O_intra and the
// next P run while the state is being carried; warps 2..5 form the masked
// P~ = P o M (hi + lo bf16; the M = 64 accumulator rows spread over all 32
// lanes of a warp); warps 6..9 combine the two output accumulators and store
// o; warps 10..17 hold the fp32 state S <- gamma^C S + dS in registers, write
// it to shared memory as the bf16 hi + lo B operand of Q S, and form
// K^ = diag(gamma^(C-1-j)) K of the next chunk (hi + lo) while Q S runs.  The
// chain from one chunk to the next is O_inter (reads S_c) -> state operand
// write -> O_inter of the next chunk.
//   P       M=64  N=64  K=128  A = Q (K-major)        B = K (K-major)
//   O_intra M=64  N=128 K=64   A = P~ hi, lo (K-major) B = V (MN-major)
//   O_inter M=64  N=128 K=128  A = Q (K-major)        B = S hi, lo (MN-major)
//   dS      M=128 N=128 K=64   A = K^ hi, lo (MN-major) B = V (MN-major)
//
// The backward reuses the same kernel: with R_s = sum_{t>=s} gamma^(t-s) q_t^T dO_t,
//   dq_t = sum_{s<=t} gamma^(t-s) (dO_t . v_s) k_s   = retention(dO, V, K)
//   dv_s = sum_{t>=s} gamma^(t-s) (k_s . q_t) dO_t   = retention run backwards in time on (K, Q, dO)
//   dk_s = sum_{t>=s} gamma^(t-s) (v_s . dO_t) q_t   = retention run backwards in time on (V, dO, Q)
// Backwards in time ("rev") the chunks are visited last to first, the mask is
// gamma^(j-i) [j >= i], the inter-chunk row scale gamma^(C-i), and the state
// update weights gamma^j k_j; the three passes run as one grid of 3 B H CTAs.
#include "la_tc.cuh"
#include "la_tc_common.cuh"

#include <mutex>
#include <string.h>

namespace la {
namespace tc {

__device__ unsigned int g_ret_fault = 0;

namespace {

#define LA_RWAIT(bar, par, code) mbar_wait((bar), (par), s_abort, &g_ret_fault, (code))

constexpr int kC = 64;                    // chunk rows
constexpr int kBox = kC * 128;            // one [64 rows x 64 cols] bf16 box, 8 KB
constexpr int kTile128 = 2 * kBox;        // a [64 x 128] chunk tile: two boxes

__device__ __forceinline__ uint8_t *align1024r(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Four 8-element chunks (4 part .. 4 part + 3 of the row's 16, across the two boxes)
// of row `row` of a [64 x 128] tile, scaled by f, as the bf16 hi tile and (if lo_too)
// the lo tile, lo = round(x f - hi), kTile128 bytes further.
static __device__ __noinline__ void scale_split_row(const uint8_t *src, uint8_t *dst, int row, int part, float f,
                                                    bool lo_too) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int ch = part * 4 + i;
        const int off = (ch >> 3) * kBox + row * 128 + (((ch & 7) ^ (row & 7)) << 4);
        const uint4 u = *reinterpret_cast<const uint4 *>(src + off);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 x = h2<true>::to_f2(w[k]);
            const float a = x.x * f, b = x.y * f;
            hi[k] = h2<true>::from_f2(a, b);
            const float2 hv = h2<true>::to_f2(hi[k]);
            lo[k] = h2<true>::from_f2(a - hv.x, b - hv.y);
        }
        *reinterpret_cast<uint4 *>(dst + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        if (lo_too) *reinterpret_cast<uint4 *>(dst + kTile128 + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
}

// Stores 16 columns (16*c16 .. +15, c16 in 0..7) of row `row` of a 128-column tile
// kept as boxes of 64 columns, `box_bytes` apart.
__device__ __forceinline__ void st16_wide(uint8_t *t, int box_bytes, int row, int c16, const float (&v)[16]) {
    store_chunk16<true>(t + (c16 >> 2) * box_bytes, row, c16 & 3, v);
}

// Warp roles: 0 TMA, 1 UMMA, 2..5 decay mask, 6..9 output, 10..17 state and K^
// (two warps per TMEM lane quadrant, 64 state columns each).
constexpr int kRXWarps = 4, kROw0 = 6, kROWarps = 4, kRSw0 = 10, kRSWarps = 8;   // mask warps 2..5
constexpr int kRThreads = (kRSw0 + kRSWarps) * 32;

struct RetLayout {
    static constexpr int NST = 2;
    static constexpr int qoff = 0;                              // [NST] q chunk (2 boxes)
    static constexpr int koff = qoff + NST * kTile128;
    static constexpr int voff = koff + NST * kTile128;
    static constexpr int khoff = voff + NST * kTile128;         // k^ hi, lo
    static constexpr int ptoff = khoff + 2 * kTile128;          // P~ hi, lo: [64 x 64] each
    static constexpr int soff = ptoff + 2 * kBox;               // S hi, lo: [128 x 128] each (2 x 16 KB)
    static constexpr int ooff = soff + 2 * 2 * 16384;           // output staging chunk
    static constexpr int gpoff = ooff + kTile128;               // gamma^k, k = 0..128
    static constexpr int baroff = gpoff + 132 * 4;
    static constexpr int nbars = 2 * NST + 10;
    static constexpr int misc = baroff + nbars * 8;
    static constexpr int bytes = misc + 32 + 1024;
    static_assert(bytes <= 227 * 1024, "shared memory of one CTA");
};

// Up to three retention passes in one launch: pass p reads (q, k, v) through
// maps q[p], k[p], v[p], writes o[p], forwards (rev = 0) or backwards in time.
struct RetJobs {
    CUtensorMap q[3], k[3], v[3], o[3];
    int rev[3];
    // Per pass: the state entering the pass's first chunk in its own direction of time
    // [BH, D, D] fp32 (row = key-side index), or null for zero; sin_t[p] != 0 reads it
    // transposed.  sout[p]: the state after the pass's last chunk, or null.
    const float *sin[3];
    float *sout[3];
    int sin_t[3];
    // Per pass, which operands carry a bf16 lo part besides the hi part (fp32 = hi + lo):
    // kLoK (K^ of dS), kLoP (P~ of O_intra), kLoS (S of O_inter).  The launches set all
    // three: each lo left out adds about 6e-4 to the relative L2 error of the output.
    int lo[3];
};
constexpr int kLoK = 1, kLoP = 2, kLoS = 4;

// Grid: one CTA per (pass, b, h), pass = blockIdx.x / BH.  decay[h] = gamma_h.
__global__ void __launch_bounds__(kRThreads, 1)
retention_kernel(const __grid_constant__ RetJobs jobs, DecayArgs dec, int T, int H, int BH) {
    using L = RetLayout;
    constexpr int NST = L::NST;
    constexpr uint32_t ID_P = idesc_f16(64, 64, true, false, false);
    constexpr uint32_t ID_OI = idesc_f16(64, 128, true, false, true);
    constexpr uint32_t ID_DS = idesc_f16(128, 128, true, true, true);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024r(smem_raw);
    uint8_t *sQ = smem + L::qoff;
    uint8_t *sK = smem + L::koff;
    uint8_t *sV = smem + L::voff;
    uint8_t *sKh = smem + L::khoff;      // hi at +0, lo at +kTile128
    uint8_t *sPt = smem + L::ptoff;      // hi at +0, lo at +kBox
    uint8_t *sS = smem + L::soff;        // hi at +0 (2 atoms of 16 KB), lo at +32 KB
    uint8_t *sO = smem + L::ooff;
    float *gpow = reinterpret_cast<float *>(smem + L::gpoff);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::baroff);
    uint64_t *empty = full + NST;
    uint64_t *pfull = empty + NST;       // P = Q K^T in TMEM
    uint64_t *ptready = pfull + 1;       // P read, P~ written (feature-map warps)
    uint64_t *khready = ptready + 1;     // K^ written
    uint64_t *dsfull = khready + 1;      // dS = K^^T V in TMEM
    uint64_t *dsread = dsfull + 1;       // dS read (state warps)
    uint64_t *sready = dsread + 1;       // state operand holds S_c (phase c)
    uint64_t *sfree = sready + 1;        // Q S of the chunk done reading the state operand
    uint64_t *ofull = sfree + 1;         // O_intra and O_inter in TMEM
    uint64_t *oread = ofull + 1;         // ... read (output warps)
    uint64_t *drain = oread + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::misc);
    int *s_abort = reinterpret_cast<int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int pass = blockIdx.x / BH;
    const int bh = blockIdx.x % BH;
    const bool rev = jobs.rev[pass] != 0;
    const int lo_mask = jobs.lo[pass];
    const int nlk = (lo_mask & kLoK) ? 2 : 1, nlp = (lo_mask & kLoP) ? 2 : 1, nls = (lo_mask & kLoS) ? 2 : 1;
    const CUtensorMap *tmQ = &jobs.q[pass], *tmK = &jobs.k[pass], *tmV = &jobs.v[pass], *tmO = &jobs.o[pass];
    const float gamma = dec.gamma[bh % H];
    const int nchunks = (T + kC - 1) / kC;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(pfull, 1);
        mbar_init(ptready, kRXWarps);
        mbar_init(khready, kRSWarps);
        mbar_init(dsfull, 1);
        mbar_init(dsread, kRSWarps);
        mbar_init(sready, kRSWarps);
        mbar_init(sfree, 1);
        mbar_init(ofull, 1);
        mbar_init(oread, kROWarps);
        mbar_init(drain, 1);
        *s_abort = 0;
        fence_mbar_init();
    }
    if (threadIdx.x < 129) {
        // gamma^k in fp32 as exp2(k log2 gamma): k = 0..C for the masks and row scales
        const float l2g = log2f(gamma);
        gpow[threadIdx.x] = threadIdx.x == 0 ? 1.f : exp2f((float)threadIdx.x * l2g);
    }
    if (warp >= kRSw0) {
        // S_0 = 0: the state operand (hi and lo, 4 x 16 KB), 16 bytes per thread per step
        for (int i = threadIdx.x - kRSw0 * 32; i < 4 * 16384 / 16; i += kRSWarps * 32)
            reinterpret_cast<uint4 *>(sS)[i] = make_uint4(0u, 0u, 0u, 0u);
        fence_async_smem();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch(tmQ);
        tma_prefetch(tmK);
        tma_prefetch(tmV);
        tma_prefetch(tmO);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // Everything above touched only shared memory and TMEM: with a programmatic
    // launch it overlapped the previous kernel.  Global memory waits for it here;
    // dependents are released only once this kernel is past its own wait.
    grid_dependency_wait();
    if (threadIdx.x == 0) grid_launch_dependents();
    constexpr uint32_t cP = 0, cOI = 64, cOX = 192, cDS = 320;

    if (warp == 0) {
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            int issued = 0;
            for (int it = 0; it < nchunks; ++it) {
                const int c = rev ? nchunks - 1 - it : it;
                if (!LA_RWAIT(&empty[s], ph ^ 1, 0x1u)) break;
                mbar_arrive_expect_tx(&full[s], 3 * kTile128);
                for (int b = 0; b < 2; ++b) {
                    tma_load_3d(sQ + s * kTile128 + b * kBox, tmQ, &full[s], 64 * b, c * kC, bh);
                    tma_load_3d(sK + s * kTile128 + b * kBox, tmK, &full[s], 64 * b, c * kC, bh);
                    tma_load_3d(sV + s * kTile128 + b * kBox, tmV, &full[s], 64 * b, c * kC, bh);
                }
                ++issued;
                if (++s == NST) { s = 0; ph ^= 1; }
            }
            if (*s_abort) {
                for (int i = issued - 1; i >= 0 && i >= issued - NST; --i)
                    mbar_wait_slow(smem_u32(&full[i % NST]), (uint32_t)((i / NST) & 1), nullptr, &g_ret_fault, 0x200u);
            }
        }
    } else if (warp == 1) {
        // UMMA issue, per chunk c: dS (independent of the state), O_intra, P of
        // chunk c + 1 (so that its decay mask overlaps the rest of chunk c), then
        // Q S once the state warps have written S_c.
        if (lane == 0) {
            auto issue_p = [&](int sp) {
                const uint64_t dq = sdesc_sw128(smem_u32(sQ + sp * kTile128), 16, 1024);
                const uint64_t dk = sdesc_sw128(smem_u32(sK + sp * kTile128), 16, 1024);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * kBox + (kk & 3) * 32;
                    umma_f16_ss(tmem + cP, desc_at(dq, off), desc_at(dk, off), ID_P, kk ? 1u : 0u);
                }
                umma_commit(pfull);
            };
            int s = 0;
            uint32_t ph = 0;
            bool ok = nchunks > 0 && LA_RWAIT(&full[0], 0, 0x4u);
            if (ok) {
                tc_fence_after();
                issue_p(0);
            }
            for (int it = 0; it < nchunks && ok; ++it) {
                const uint32_t pc = (uint32_t)(it & 1), pp = pc ^ 1u;
                const int sn = s + 1 == NST ? 0 : s + 1;
                const uint32_t phn = s + 1 == NST ? ph ^ 1u : ph;
                const uint64_t dq = sdesc_sw128(smem_u32(sQ + s * kTile128), 16, 1024);
                const uint64_t dv = sdesc_sw128(smem_u32(sV + s * kTile128), kBox, 1024);
                // dS = K^^T V
                if (!LA_RWAIT(khready, pc, 0x80u)) break;
                if (it > 0 && !LA_RWAIT(dsread, pp, 0x40u)) break;
                tc_fence_after();
                const uint64_t dkh = sdesc_sw128(smem_u32(sKh), kBox, 1024);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
                    for (int op = 0; op < nlk; ++op)
                        umma_f16_ss(tmem + cDS, desc_at(dkh, op * kTile128 + kk * 2048), desc_at(dv, kk * 2048), ID_DS,
                                    (kk | op) ? 1u : 0u);
                }
                umma_commit(dsfull);
                // O_intra = P~ V (the mask has read P: its accumulator is free)
                if (!LA_RWAIT(ptready, pc, 0x10u)) break;
                if (it > 0 && !LA_RWAIT(oread, pp, 0x20u)) break;
                tc_fence_after();
                const uint64_t dpt = sdesc_sw128(smem_u32(sPt), 16, 1024);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
                    for (int op = 0; op < nlp; ++op)
                        umma_f16_ss(tmem + cOI, desc_at(dpt, op * kBox + kk * 32), desc_at(dv, kk * 2048), ID_OI,
                                    (kk | op) ? 1u : 0u);
                }
                // P of the next chunk
                if (it + 1 < nchunks) {
                    if (!LA_RWAIT(&full[sn], phn, 0x4u)) break;
                    tc_fence_after();
                    issue_p(sn);
                }
                // O_inter = Q S_c
                if (!LA_RWAIT(sready, pc, 0x1000u)) break;
                tc_fence_after();
                const uint64_t ds = sdesc_sw128(smem_u32(sS), 16384, 1024);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * kBox + (kk & 3) * 32;
#pragma unroll
                    for (int op = 0; op < nls; ++op)
                        umma_f16_ss(tmem + cOX, desc_at(dq, off), desc_at(ds, op * 32768 + kk * 2048), ID_OI,
                                    (kk | op) ? 1u : 0u);
                }
                umma_commit(ofull);
                umma_commit(sfree);
                umma_commit(&empty[s]);
                s = sn;
                ph = phn;
            }
            umma_commit(drain);
            mbar_wait_slow(smem_u32(drain), 0, nullptr, &g_ret_fault, 0x400u);
        }
    } else if (warp < kROw0) {
        // Decay-mask warps: P~ = P o M as hi + lo (warp w reads TMEM lane quadrant w % 4,
        // where chunk rows 16 (w % 4) + l sit in lanes l = 0..15).
        const int sub = warp & 3;
        const uint32_t lanes = (uint32_t)(32 * sub) << 16;
        const int ri = 16 * sub + (lane & 15), hcol = lane >> 4;   // row; column half (M = 64 rows in lanes 0..15)
        for (int it = 0; it < nchunks; ++it) {
            const uint32_t pc = (uint32_t)(it & 1);
            // P~ of the previous chunk: its O_intra completed before this chunk's P, which pfull tracks
            const bool got = __all_sync(0xffffffffu, LA_RWAIT(pfull, pc, 0x400u));
            if (!got) break;
            __syncwarp();   // converged for the .sync.aligned TMEM loads
            tc_fence_after();
            // lanes 0..15 take columns 0..31 of their row, lanes 16..31 columns 32..63
#pragma unroll
            for (int h16 = 0; h16 < 2; ++h16) {
                const int c16 = 2 * hcol + h16;
                float x[16];
                tmem_ld16_halves<32>(tmem + cP + lanes + 16 * h16, x);
                tmem_ld_wait(x);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int j = 16 * c16 + e;
                    const int dlt = rev ? j - ri : ri - j;     // causal: i >= j; backwards: j >= i
                    x[e] = dlt >= 0 ? x[e] * gpow[dlt] : 0.f;
                }
                uint32_t hw[8], lw[8];
                split_hi_lo16_packed(x, hw, lw);
                store_chunk16_packed(sPt, ri, c16, hw);
                if (nlp == 2) store_chunk16_packed(sPt + kBox, ri, c16, lw);
            }
            tc_fence_before();
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(ptready);
        }
    } else if (warp < kRSw0) {
        // Output warps: o = O_intra + diag(gamma^(i+1)) O_inter (backwards: gamma^(C-i)),
        // staged and stored with TMA.  Named barrier 1 (these 128 threads) is
        // reached by all of them whatever the waits return.
        const int ot = threadIdx.x - kROw0 * 32;
        const int sub = warp & 3;
        const uint32_t lanes = (uint32_t)(32 * sub) << 16;
        const int ri = 16 * sub + (lane & 15), hcol = lane >> 4;   // row; column half (M = 64 rows in lanes 0..15)
        bool live = true;
        for (int it = 0; it < nchunks; ++it) {
            const int c = rev ? nchunks - 1 - it : it;
            const uint32_t pc = (uint32_t)(it & 1);
            if (ot == 0) tma_store_wait_read<0>();
            named_bar(1, kROWarps * 32);
            bool got = live && LA_RWAIT(ofull, pc, 0x800u);
            got = __all_sync(0xffffffffu, got);
            live = live && got;
            if (got) {
                __syncwarp();   // converged for the .sync.aligned TMEM loads
                tc_fence_after();
                // backwards the entering state sits one past the chunk's last valid row
                const int rows = min(kC, T - c * kC);
                const float g1 = rev ? (ri < rows ? gpow[rows - ri] : 0.f) : gpow[ri + 1];
                // lanes 0..15 take columns 0..63 of their row, lanes 16..31 columns 64..127
#pragma unroll
                for (int h16 = 0; h16 < 4; ++h16) {
                    float a[16], b[16];
                    tmem_ld16_halves<64>(tmem + cOI + lanes + 16 * h16, a);
                    tmem_ld16_halves<64>(tmem + cOX + lanes + 16 * h16, b);
                    tmem_ld_wait(a, b);
#pragma unroll
                    for (int i = 0; i < 16; ++i) a[i] = fmaf(g1, b[i], a[i]);
                    st16_wide(sO, kBox, ri, 4 * hcol + h16, a);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(oread);
            }
            fence_async_smem();
            named_bar(1, kROWarps * 32);
            if (ot == 0 && live) {
                tma_store_3d(tmO, sO, 0, c * kC, bh);
                tma_store_3d(tmO, sO + kBox, 64, c * kC, bh);
                tma_store_commit();
            }
        }
        if (ot == 0) tma_store_wait_all<0>();
    } else {
        // State warps: S_{c+1} = gamma^C S_c + dS_c in fp32 registers; thread (d, half)
        // holds columns 64 half .. 64 half + 63 of state row d (its TMEM lane) and
        // writes them as the bf16 hi + lo operand of Q S.
        const int sub = warp & 3, half = (warp - kRSw0) >> 2;
        const uint32_t lanes = (uint32_t)(32 * sub) << 16;
        const int d = 32 * sub + lane;
        const float gC = gpow[kC];
        // decay over the partial chunk at the end of the sequence: the last chunk
        // forwards, the first one backwards
        const float gLast = gpow[min(kC, T - (nchunks - 1) * kC)];
        float st[64];
        const float *sin = jobs.sin[pass];
        float *sout = jobs.sout[pass];
        const long long srow = ((long long)bh * 128 + d) * 128 + 64 * half;   // this thread's 64 state entries
        if (sin) {   // S_0 given: registers and the hi + lo operand of the first Q S
            if (jobs.sin_t[pass]) {   // st[c] = sin[64 half + c][d]: lanes read consecutive d
                const float *col = sin + (long long)bh * 128 * 128 + (long long)(64 * half) * 128 + d;
#pragma unroll
                for (int c = 0; c < 64; ++c) st[c] = col[(long long)c * 128];
            } else {
#pragma unroll
                for (int c4 = 0; c4 < 16; ++c4) {
                    const float4 x = *reinterpret_cast<const float4 *>(sin + srow + 4 * c4);
                    st[4 * c4] = x.x;
                    st[4 * c4 + 1] = x.y;
                    st[4 * c4 + 2] = x.z;
                    st[4 * c4 + 3] = x.w;
                }
            }
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                uint32_t hw[8], lw[8];
                split_hi_lo16_packed(*reinterpret_cast<const float(*)[16]>(&st[16 * c4]), hw, lw);
                store_chunk16_packed(sS + half * 16384, d, c4, hw);
                if (nls == 2) store_chunk16_packed(sS + 32768 + half * 16384, d, c4, lw);
            }
            fence_async_smem();
        } else {
#pragma unroll
            for (int i = 0; i < 64; ++i) st[i] = 0.f;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(sready);                // S_0
        // K^ = diag(gamma^(C-1-j)) K of chunk iteration itk as hi + lo, written while Q S of
        // the previous chunk runs: thread kt takes row kt % 64 and the 8-element chunks
        // 4 (kt / 64) .. + 3 of the row's 16.  Forwards in time the weights count back from
        // the chunk's last valid row, so that the state after a partial last chunk is the
        // state after token T - 1.
        const int kt = threadIdx.x - kRSw0 * 32;
        const int krow = kt & 63, kpart = kt >> 6;
        auto build_khat = [&](int itk) -> bool {
            const int sk = itk % NST;
            if (!__all_sync(0xffffffffu, LA_RWAIT(&full[sk], (uint32_t)((itk / NST) & 1), 0x100u))) return false;
            const int rows = min(kC, T - (rev ? nchunks - 1 - itk : itk) * kC);
            const float f = rev ? gpow[krow] : (krow < rows ? gpow[rows - 1 - krow] : 0.f);
            scale_split_row(sK + sk * kTile128, sKh, krow, kpart, f, nlk == 2);
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(khready);
            return true;
        };
        const bool k0 = nchunks > 0 && build_khat(0);
        for (int it = 0; it < nchunks && k0; ++it) {
            const uint32_t pc = (uint32_t)(it & 1);
            bool got = __all_sync(0xffffffffu, LA_RWAIT(dsfull, pc, 0x1000u));
            if (!got) break;
            __syncwarp();   // converged for the .sync.aligned TMEM loads
            tc_fence_after();
            const uint32_t base = tmem + cDS + lanes + 64u * half;
            const float g = (it == (rev ? 0 : nchunks - 1)) ? gLast : gC;
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                float a[16];
                tmem_ld16(base + 16 * c4, a);
                tmem_ld_wait(a);
#pragma unroll
                for (int i = 0; i < 16; ++i) st[16 * c4 + i] = fmaf(g, st[16 * c4 + i], a[i]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(dsread);
            // dS_c is complete, so it has read K^_c: the buffer takes K^ of the next chunk
            if (it + 1 < nchunks && !build_khat(it + 1)) break;
            got = __all_sync(0xffffffffu, LA_RWAIT(sfree, pc, 0x2000u));   // Q S_c has read the operand
            if (!got) break;
            // the 64 columns are columns 0..63 of box `half` (each box holds 64 state columns)
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                uint32_t hw[8], lw[8];
                split_hi_lo16_packed(*reinterpret_cast<const float(*)[16]>(&st[16 * c4]), hw, lw);
                store_chunk16_packed(sS + half * 16384, d, c4, hw);
                if (nls == 2) store_chunk16_packed(sS + 32768 + half * 16384, d, c4, lw);
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(sready);
        }
        if (sout && !*s_abort) {   // S after the last chunk
#pragma unroll
            for (int c4 = 0; c4 < 16; ++c4)
                *reinterpret_cast<float4 *>(sout + srow + 4 * c4) =
                    make_float4(st[4 * c4], st[4 * c4 + 1], st[4 * c4 + 2], st[4 * c4 + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

#ifndef LA_TRY
#define LA_TRY(x)                     \
    do {                              \
        la_status _rc = (x);          \
        if (_rc != LA_OK) return _rc; \
    } while (0)
#endif

}  // namespace

la_status retention_fwd(const void *q, const void *k, const void *v, void *o, const float *sin, float *sout,
                        const DecayArgs &dec, const Shape &s, cudaStream_t st) {
    RetJobs jobs;
    memset(&jobs, 0, sizeof jobs);
    jobs.sin[0] = sin;
    jobs.sout[0] = sout;
    jobs.lo[0] = kLoK | kLoP | kLoS;
    LA_TRY(retention_map(&jobs.q[0], q, s));
    LA_TRY(retention_map(&jobs.k[0], k, s));
    LA_TRY(retention_map(&jobs.v[0], v, s));
    LA_TRY(retention_map(&jobs.o[0], o, s));
    return launch_pdl("tc_retention_fwd", retention_kernel, dim3((unsigned)s.BH()), dim3(kRThreads),
                  (size_t)RetLayout::bytes, st, jobs, dec, s.T, s.H, (int)s.BH());
}

la_status retention_bwd(const void *q, const void *k, const void *v, const void *g, const float *sin,
                        const float *rin, float *rout, const DecayArgs &dec, void *dq, void *dk, void *dv,
                        const Shape &s, cudaStream_t st) {
    RetJobs jobs;
    memset(&jobs, 0, sizeof jobs);
    // dq = retention(dO, V, K); dv = reverse retention(K, Q, dO); dk = reverse retention(V, dO, Q).
    // Their states are S^T (S = sum k^T v), R and R^T (R = sum gamma^(t-s) q_t^T dO_t).
    // dq == null leaves out the first pass.
    struct Pass {
        const void *q, *k, *v;
        void *o;
        int rev;
        const float *sin;
        int sin_t;
        float *sout;
    };
    const Pass all[3] = {{g, v, k, dq, 0, sin, 1, nullptr},
                         {k, q, g, dv, 1, rin, 0, rout},
                         {v, g, q, dk, 1, rin, 1, nullptr}};
    int np = 0;
    for (int p = dq ? 0 : 1; p < 3; ++p, ++np) {
        LA_TRY(retention_map(&jobs.q[np], all[p].q, s));
        LA_TRY(retention_map(&jobs.k[np], all[p].k, s));
        LA_TRY(retention_map(&jobs.v[np], all[p].v, s));
        LA_TRY(retention_map(&jobs.o[np], all[p].o, s));
        jobs.rev[np] = all[p].rev;
        jobs.sin[np] = all[p].sin;
        jobs.sin_t[np] = all[p].sin_t;
        jobs.sout[np] = all[p].sout;
        jobs.lo[np] = kLoK | kLoP | kLoS;
    }
    return launch_pdl("tc_retention_bwd", retention_kernel, dim3((unsigned)(np * s.BH())), dim3(kRThreads),
                  (size_t)RetLayout::bytes, st, jobs, dec, s.T, s.H, (int)s.BH());
}

unsigned int read_and_clear_retention_fault() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_ret_fault, sizeof v) != cudaSuccess) return 0xFFFFFFFFu;
    if (v) cudaMemcpyToSymbol(g_ret_fault, &zero, sizeof zero);
    return v;
}

}  // namespace tc
}  // namespace la

