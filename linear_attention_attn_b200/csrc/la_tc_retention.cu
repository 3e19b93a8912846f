// la_tc_retention.cu -- tensor-core kernel of causal linear attention with a per-head
// scalar decay (retention), forward and backward, bf16 or fp16 storage, D = 64 or 128,
// fp32 accumulation.
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
// with TMA (two 64-column boxes per 64-row chunk, 128-byte swizzle) into three
// stages, so the loads of the next two chunks are in flight while one is
// computed; warp 1 issues the UMMAs; warps 2..5 form the masked P~ = P o M (hi +
// lo bf16; the M = 64 accumulator rows spread over all 32 lanes of a warp); warps
// 6..9 combine the two output parts and store o; warps 10..17 hold the fp32 state
// in registers and form K^ = diag(gamma^(C-1-j)) K of the next chunk (hi + lo).
// The outputs are computed transposed, O^T = V^T P~^T + S^T Q^T (M = 128, the
// value dimension), so that the state, kept by the state warps as S^T, is the
// A operand of O_inter^T straight from tensor memory (bf16 hi + lo, written with
// tcgen05.st): it needs no shared memory, which goes to the third stage.  The
// chain from one chunk to the next is O_inter^T (reads S_c) -> state operand
// write -> O_inter^T of the next chunk.
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

// NCH 8-element chunks (NCH part .. NCH part + NCH - 1 of the row's 16, across the two
// boxes) of row `row` of a [64 x 128] tile, scaled by f, as the bf16 hi tile and (if
// lo_too) the lo tile, lo = round(x f - hi), kTile128 bytes further.
template <int NCH, bool BF>
static __device__ __noinline__ void scale_split_row(const uint8_t *src, uint8_t *dst, int row, int part, float f,
                                                    bool lo_too) {
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
        const int ch = part * NCH + i;
        const int off = (ch >> 3) * kBox + row * 128 + (((ch & 7) ^ (row & 7)) << 4);
        const uint4 u = *reinterpret_cast<const uint4 *>(src + off);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 x = h2<BF>::to_f2(w[k]);
            const float a = x.x * f, b = x.y * f;
            hi[k] = h2<BF>::from_f2(a, b);
            const float2 hv = h2<BF>::to_f2(hi[k]);
            lo[k] = h2<BF>::from_f2(a - hv.x, b - hv.y);
        }
        *reinterpret_cast<uint4 *>(dst + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        if (lo_too) *reinterpret_cast<uint4 *>(dst + kTile128 + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
}

// Warp roles: 0 TMA, 1 UMMA, 2..5 decay mask, 6..9 output, 10..17 state and K^
// (two warps per TMEM lane quadrant, 64 state columns each).
constexpr int kRXWarps = 4, kROw0 = 6, kROWarps = 4, kRSw0 = 10, kRSWarps = 8;   // mask warps 2..5
constexpr int kRThreads = (kRSw0 + kRSWarps) * 32;

// Shared memory: three stages of q/k/v chunks (so that the loads of the next two
// chunks are in flight while one is computed), K^ and P~ (hi + lo each), the output
// staging chunk, the decay powers and the barriers.  The state lives in tensor memory.
struct RetLayout {
    static constexpr int NST = 3;
    static constexpr int qoff = 0;                              // [NST] q chunk (2 boxes)
    static constexpr int koff = qoff + NST * kTile128;
    static constexpr int voff = koff + NST * kTile128;
    static constexpr int khoff = voff + NST * kTile128;         // K^ hi, lo
    static constexpr int ptoff = khoff + 2 * kTile128;          // P~ hi, lo: [64 x 64] each
    static constexpr int ooff = ptoff + 2 * kBox;               // output staging chunk
    static constexpr int gpoff = ooff + kTile128;               // gamma^k, k = -64..128
    static constexpr int denoff = gpoff + 196 * 4;              // [2][64] 1 / denominators (norm term)
    static constexpr int dotoff = denoff + 2 * 64 * 4;          // [2][64] dout . o partial sums (prep)
    static constexpr int baroff = dotoff + 2 * 64 * 4;
    static constexpr int nbars = 2 * NST + 22;
    static constexpr int misc = baroff + nbars * 8;
    static constexpr int bytes = misc + 32 + 1024;
    static_assert(bytes <= 227 * 1024, "shared memory of one CTA");
};

// Tensor memory (512 columns): P of two consecutive chunks (M = 64, 64 columns each),
// the transposed output (M = 128: lane d, column = row of the chunk), dS^T, and the
// state S^T as the A operand of O_inter^T, bf16 hi then lo (lane d, 64 columns each
// holding 128 16-bit K values).  The output takes columns 128..255 in one of two ways
// (see retention_kernel): two accumulators of consecutive chunks (cO, cO + 64), or
// O_intra^T and O_inter^T of one chunk (cOI, cOX).
constexpr uint32_t cP = 0, cO = 128, cOI = 128, cOX = 192, cDS = 256, cSA = 384;

// Reference row of the folded output (see retention_kernel).
constexpr int kM = 32;

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
    // sonly[p] != 0: the pass computes its state only (sout), no output: only k and v
    // are loaded, and per chunk only K^ and dS^T are formed.
    int sonly[3];
    // D = 64 only: o32[p] != 0 writes the pass's output in fp32 (map o[p] of fp32 [BH, T, 64],
    // boxes of 32 columns), for a caller that adds to it before rounding.
    int o32[3];
    // Kernels with the norm term (NORM): eps of the denominators.  prep != 0 turns the
    // forward into the first step of the backward: with dout (map g) loaded chunk by chunk,
    // the output written is du = dout / n (n = f(q) . z + eps) instead of o, and dn receives
    // -(dout . o) / n of every row, [BH, T] fp32.
    CUtensorMap g;
    float eps;
    int prep;
    float *dn;
};

// Grid: one CTA per (pass, b, h), pass = blockIdx.x / BH.  decay[h] = gamma_h.
//
// FOLD: the two output parts share one accumulator, so that consecutive chunks can
// use two of them and the epilogue of one chunk overlaps the products of the next.
// With g_i the row scale of the inter-chunk part (gamma^(i+1); backwards
// gamma^(rows-i)) and a reference row m = 32,
//   o_i = f_i (sum_j w'_ij P_ij v_j + q_i (gamma^m S)),  f_i = g_i / gamma^m,
//   w'_ij = w_ij gamma^m / g_i = gamma^(m-1-j) (j <= i)   [backwards gamma^(j+m-rows), j >= i],
// so the state operand is written as gamma^m S and the epilogue multiplies row i by
// f_i.  Every factor lies within gamma^(+-64) of 1, which stays far inside the fp32 and
// bf16 ranges for gamma >= 1/8 (fp16: gamma >= 0.9, see fold_ok); smaller decays use
// FOLD = false, where O_intra^T and O_inter^T keep accumulators of their own and the
// epilogue forms O_intra + g_i O_inter.
//
// Per chunk c the UMMAs are issued in the order P(c + 1), dS^T(c), O_intra^T(c),
// O_inter^T(c): P of the next chunk goes to the other P buffer as soon as its data has
// arrived, so the decay mask of chunk c + 1 overlaps the rest of chunk c, and every
// product whose operands are ready is queued ahead of O_inter^T, the one that waits
// for the state.  Every operand of the 16-bit products is exact or split hi + lo
// (K^, P~, S), so the products carry fp32 accuracy into the fp32 accumulators.
//   P           M=64  N=64  K=128  A = Q (K-major)            B = K (K-major)
//   dS^T        M=128 N=128 K=64   A = V^T (MN-major)         B = K^ hi, lo (MN-major)
//   O_intra^T   M=128 N=64  K=64   A = V^T (MN-major)         B = P~ hi, lo (K-major)
//   O_inter^T   M=128 N=64  K=128  A = S^T hi, lo (tensor mem) B = Q (K-major)
//
// NORM (D = 64, forward in time): causal linear attention with the norm term,
// o_t = f(q_t) S_t / (f(q_t) . z_t + eps) with z_t the decayed sum of f(k_s).  The unused
// first box of every v stage holds a column of ones (value index -1, TMEM lane 0), so the
// same products carry z through the state (lane 0 of S^T) and give each row's denominator
// in lane 0 of the output accumulator; the epilogue divides by it.
template <bool FOLD, int NBOX, bool BF, bool NORM>
__global__ void __launch_bounds__(kRThreads, 1)
retention_kernel(const __grid_constant__ RetJobs jobs, DecayArgs dec, int T, int H, int BH) {
    static_assert(!NORM || NBOX == 1, "the norm term needs the free first box of v (D = 64)");
    using L = RetLayout;
    constexpr int NST = L::NST;
    constexpr uint32_t ID_P = idesc_f16(64, 64, BF, false, false);
    constexpr uint32_t ID_OIT = idesc_f16(128, 64, BF, true, false);
    constexpr uint32_t ID_OXT = idesc_f16(128, 64, BF, false, false);
    constexpr uint32_t ID_DST = idesc_f16(128, 64 * NBOX, BF, true, true);   // N = the key dimensions
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024r(smem_raw);
    uint8_t *sQ = smem + L::qoff;
    uint8_t *sK = smem + L::koff;
    uint8_t *sV = smem + L::voff;
    uint8_t *sKh = smem + L::khoff;      // hi at +0, lo at +kTile128
    uint8_t *sPt = smem + L::ptoff;      // hi at +0, lo at +kBox
    uint8_t *sO = smem + L::ooff;
    float *gexp = reinterpret_cast<float *>(smem + L::gpoff);   // gexp[k + 64] = gamma^k
#define GP(k) gexp[(k) + 64]
    float *sDen = reinterpret_cast<float *>(smem + L::denoff);   // NORM: 1 / (f(q) . z + eps) per row
    float *sDot = reinterpret_cast<float *>(smem + L::dotoff);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::baroff);
    uint64_t *empty = full + NST;
    uint64_t *pfull = empty + NST;       // [2] P of a chunk in TMEM buffer (chunk & 1)
    uint64_t *ptready = pfull + 2;       // P read, P~ written (mask warps)
    uint64_t *ptfree = ptready + 1;      // O_intra^T done reading P~
    uint64_t *khready = ptfree + 1;      // K^ written
    uint64_t *dsfull = khready + 1;      // dS^T = V^T K^ in TMEM
    uint64_t *dsread = dsfull + 1;       // dS^T read (state warps)
    uint64_t *sready = dsread + 1;       // state operand holds S_c (phase c)
    uint64_t *sfree = sready + 1;        // O_inter^T of the chunk done reading the state operand
    uint64_t *ofull = sfree + 1;         // [2] the output of a chunk in TMEM (FOLD: per buffer)
    uint64_t *oread = ofull + 2;         // [2] ... read (output warps)
    uint64_t *drain = oread + 2;
    uint64_t *gfull = drain + 1;         // [2] prep: the dout chunk in its buffer (iteration & 1)
    uint64_t *denready = gfull + 2;      // [2] NORM: sDen[iteration & 1] written
    uint64_t *denfree = denready + 2;    // [2] NORM: ... read
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::misc);
    int *s_abort = reinterpret_cast<int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int pass = blockIdx.x / BH;
    const int bh = blockIdx.x % BH;
    const bool rev = jobs.rev[pass] != 0;
    const bool sonly = jobs.sonly[pass] != 0;
    const CUtensorMap *tmQ = &jobs.q[pass], *tmK = &jobs.k[pass], *tmV = &jobs.v[pass], *tmO = &jobs.o[pass];
    const float gamma = dec.gamma[bh % H];
    const int nchunks = (T + kC - 1) / kC;
    // NBOX = 1 (D = 64): one 64-column box of each tile is loaded and stored, the other is
    // zero, so every product keeps its D = 128 shape (with K = 64 where the key dimensions
    // are summed) and the extra dimensions contribute nothing.  q and k take the first box;
    // v, and so the output, the second: the value dimensions (the TMEM lanes of dS^T, of the
    // state operand and of the output) are then lanes 64..127, whose warps run on other
    // schedulers than the TMA and UMMA-issuing warps.
    constexpr int nbox = NBOX, D = 64 * NBOX;
    constexpr int vbox = 2 - NBOX;             // box of v's (and o's) columns 0..63

    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(&pfull[0], 1);
        mbar_init(&pfull[1], 1);
        mbar_init(ptready, kRXWarps);
        mbar_init(ptfree, 1);
        mbar_init(khready, kRSWarps);
        mbar_init(dsfull, 1);
        mbar_init(dsread, kRSWarps);
        mbar_init(sready, kRSWarps);
        mbar_init(sfree, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ofull[b], 1);
            mbar_init(&oread[b], kROWarps);
        }
        mbar_init(drain, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&gfull[b], 1);
            mbar_init(&denready[b], 1);
            mbar_init(&denfree[b], 2);
        }
        *s_abort = 0;
        fence_mbar_init();
    }
    if (threadIdx.x < 193) {
        // gamma^k in fp32 as exp2(k log2 gamma), k = -64..128: the masks, row scales and
        // the folded output's factors
        const float l2g = log2f(gamma);
        const int k = (int)threadIdx.x - 64;
        gexp[threadIdx.x] = k == 0 ? 1.f : exp2f((float)k * l2g);
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch(tmQ);
        tma_prefetch(tmK);
        tma_prefetch(tmV);
        tma_prefetch(tmO);
        if (NORM && jobs.prep) tma_prefetch(&jobs.g);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    if (NBOX == 1) {
        // the unused boxes: the second of q, k of every stage and of K^ hi, lo, the first of v
        // (3 NST + 2 boxes of 8 KB)
        constexpr int nz = 3 * NST + 2;
        for (int i = threadIdx.x; i < nz * (kBox / 16); i += kRThreads) {
            const int b = i / (kBox / 16), e = i % (kBox / 16);
            uint8_t *base = b < 2 * NST ? smem + L::qoff + b * kTile128 + kBox
                          : b < 3 * NST ? smem + L::qoff + b * kTile128
                                        : sKh + (b - 3 * NST) * kTile128 + kBox;
            // NORM: column 0 of v's first box is one (the 16-byte chunk of row e / 8 that
            // the swizzle puts column 0 in)
            const bool one = NORM && b >= 2 * NST && b < 3 * NST && (e & 7) == ((e >> 3) & 7);
            *reinterpret_cast<uint4 *>(base + e * 16) = make_uint4(one ? h2<BF>::one() : 0u, 0u, 0u, 0u);
        }
        fence_async_smem();
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

    if (warp == 0) {
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            int issued = 0;
            for (int it = 0; it < nchunks; ++it) {
                const int c = rev ? nchunks - 1 - it : it;
                if (!LA_RWAIT(&empty[s], ph ^ 1, 0x1u)) break;
                mbar_arrive_expect_tx(&full[s], (sonly ? 2 : 3) * nbox * kBox);
                for (int b = 0; b < nbox; ++b) {
                    if (!sonly) tma_load_3d(sQ + s * kTile128 + b * kBox, tmQ, &full[s], 64 * b, c * kC, bh);
                    tma_load_3d(sK + s * kTile128 + b * kBox, tmK, &full[s], 64 * b, c * kC, bh);
                    tma_load_3d(sV + s * kTile128 + (b + vbox) * kBox, tmV, &full[s], 64 * b, c * kC, bh);
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
        // The whole warp runs the issue loop in step (waits included); one elected lane
        // issues each UMMA and commit, so the descriptors stay warp-uniform.
#define LA_WWAIT(bar, par, code) __all_sync(0xffffffffu, LA_RWAIT((bar), (par), (code)))
        auto issue_p = [&](int c) {   // P = Q K^T of chunk iteration c into buffer c & 1
            const int sp = c % NST;
            const uint64_t dq = sdesc_sw128(smem_u32(sQ + sp * kTile128), 16, 1024);
            const uint64_t dk = sdesc_sw128(smem_u32(sK + sp * kTile128), 16, 1024);
#pragma unroll
            for (int kk = 0; kk < 4 * NBOX; ++kk) {   // K = the key dimensions
                const uint32_t off = (kk >> 2) * kBox + (kk & 3) * 32;
                umma_f16_ss_warp(tmem + cP + 64u * (uint32_t)(c & 1), desc_at(dq, off), desc_at(dk, off), ID_P,
                                 kk ? 1u : 0u);
            }
            umma_commit_warp(&pfull[c & 1]);
        };
        if (sonly) {
            // state only: dS^T of every chunk, released as soon as it has read the stage
            const uint64_t dkh = sdesc_sw128(smem_u32(sKh), kBox, 1024);
            for (int it = 0; it < nchunks; ++it) {
                const uint32_t pc = (uint32_t)(it & 1), pp = pc ^ 1u;
                const int s = it % NST;
                if (!LA_WWAIT(khready, pc, 0x80u)) break;
                if (it > 0 && !LA_WWAIT(dsread, pp, 0x40u)) break;
                tc_fence_after();
                const uint64_t dv = sdesc_sw128(smem_u32(sV + s * kTile128), kBox, 1024);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
                    for (int op = 0; op < 2; ++op)
                        umma_f16_ss_warp(tmem + cDS, desc_at(dv, kk * 2048), desc_at(dkh, op * kTile128 + kk * 2048),
                                         ID_DST, (kk | op) ? 1u : 0u);
                }
                umma_commit_warp(dsfull);
                umma_commit_warp(&empty[s]);
            }
        }
        bool ok = !sonly && nchunks > 0 && LA_WWAIT(&full[0], 0, 0x4u);
        if (ok) {
            tc_fence_after();
            issue_p(0);
        }
        const uint64_t dkh = sdesc_sw128(smem_u32(sKh), kBox, 1024);
        const uint64_t dpt = sdesc_sw128(smem_u32(sPt), 16, 1024);
        for (int it = 0; it < nchunks && ok; ++it) {
            const uint32_t pc = (uint32_t)(it & 1), pp = pc ^ 1u;
            const int s = it % NST;
            // P of the next chunk: its buffer was last read by the mask of chunk it - 1,
            // which finished before O_intra^T(it - 1) was issued
            if (it + 1 < nchunks) {
                if (!LA_WWAIT(&full[(it + 1) % NST], (uint32_t)(((it + 1) / NST) & 1), 0x4u)) break;
                tc_fence_after();
                issue_p(it + 1);
            }
            const uint64_t dv = sdesc_sw128(smem_u32(sV + s * kTile128), kBox, 1024);
            // dS^T = V^T K^
            if (!LA_WWAIT(khready, pc, 0x80u)) break;
            if (it > 0 && !LA_WWAIT(dsread, pp, 0x40u)) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
                for (int op = 0; op < 2; ++op)
                    umma_f16_ss_warp(tmem + cDS, desc_at(dv, kk * 2048), desc_at(dkh, op * kTile128 + kk * 2048),
                                     ID_DST, (kk | op) ? 1u : 0u);
            }
            umma_commit_warp(dsfull);
            // O_intra^T = V^T P~^T, once the output warps have read what its accumulator
            // held (FOLD: the chunk before the previous one; else the previous chunk)
            const int ob = FOLD ? (it & 1) : 0;
            const uint32_t cIn = FOLD ? cO + 64u * (uint32_t)ob : cOI;
            const uint32_t cEx = FOLD ? cIn : cOX;
            if (!LA_WWAIT(ptready, pc, 0x10u)) break;
            if (FOLD ? it >= 2 && !LA_WWAIT(&oread[ob], (uint32_t)(((it >> 1) & 1) ^ 1), 0x20u)
                     : it > 0 && !LA_WWAIT(&oread[0], pp, 0x20u))
                break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
                for (int op = 0; op < 2; ++op)
                    umma_f16_ss_warp(tmem + cIn, desc_at(dv, kk * 2048), desc_at(dpt, op * kBox + kk * 32), ID_OIT,
                                     (kk | op) ? 1u : 0u);
            }
            umma_commit_warp(ptfree);
            // O_inter^T = S^T Q^T once the state warps have written S_c
            if (!LA_WWAIT(sready, pc, 0x1000u)) break;
            tc_fence_after();
            const uint64_t dq = sdesc_sw128(smem_u32(sQ + s * kTile128), 16, 1024);
#pragma unroll
            for (int kk = 0; kk < 4 * NBOX; ++kk) {   // K = the key dimensions
                const uint32_t off = (kk >> 2) * kBox + (kk & 3) * 32;
#pragma unroll
                for (int op = 0; op < 2; ++op)
                    umma_f16_ts_warp(tmem + cEx, tmem + cSA + 64u * op + 8u * kk, desc_at(dq, off), ID_OXT,
                                     (FOLD || (kk | op)) ? 1u : 0u);
            }
            umma_commit_warp(&ofull[ob]);
            umma_commit_warp(sfree);
            umma_commit_warp(&empty[s]);
        }
        umma_commit_warp(drain);
        mbar_wait_slow(smem_u32(drain), 0, nullptr, &g_ret_fault, 0x400u);
        __syncwarp();
#undef LA_WWAIT
    } else if (warp < kROw0) {
        // Decay-mask warps: P~ = P o M as hi + lo (warp w reads TMEM lane quadrant w % 4,
        // where chunk rows 16 (w % 4) + l sit in lanes l = 0..15).
        const int sub = warp & 3;
        const uint32_t lanes = (uint32_t)(32 * sub) << 16;
        const int ri = 16 * sub + (lane & 15), hcol = lane >> 4;   // row; column half (M = 64 rows in lanes 0..15)
        for (int it = 0; it < (sonly ? 0 : nchunks); ++it) {
            const uint32_t pc = (uint32_t)(it & 1);
            const int rows = min(kC, T - (rev ? nchunks - 1 - it : it) * kC);
            if (!__all_sync(0xffffffffu, LA_RWAIT(&pfull[it & 1], (uint32_t)((it >> 1) & 1), 0x400u))) break;
            // P~ of the previous chunk has been read by its O_intra^T
            if (it > 0 && !__all_sync(0xffffffffu, LA_RWAIT(ptfree, pc ^ 1u, 0x8u))) break;
            __syncwarp();   // converged for the .sync.aligned TMEM loads
            tc_fence_after();
            // lanes 0..15 take columns 0..31 of their row, lanes 16..31 columns 32..63
#pragma unroll
            for (int h16 = 0; h16 < 2; ++h16) {
                const int c16 = 2 * hcol + h16;
                float x[16];
                tmem_ld16_halves_sync<32>(tmem + cP + 64u * (uint32_t)(it & 1) + lanes + 16 * h16, x);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int j = 16 * c16 + e;
                    const int dlt = rev ? j - ri : ri - j;     // causal: i >= j; backwards: j >= i
                    const float wgt = FOLD ? (rev ? GP(j + kM - rows) : GP(kM - 1 - j)) : GP(dlt);
                    x[e] = dlt >= 0 ? x[e] * wgt : 0.f;
                }
                uint32_t hw[8], lw[8];
                split_hi_lo16_packed<BF>(x, hw, lw);
                store_chunk16_packed(sPt, ri, c16, hw);
                store_chunk16_packed(sPt + kBox, ri, c16, lw);
            }
            tc_fence_before();
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(ptready);
        }
    } else if (warp < kRSw0) {
        // Output warps: o = O_intra + diag(gamma^(i+1)) O_inter (backwards: gamma^(rows-i);
        // folded: f_i times the one accumulator), from the transposed parts (TMEM lane d,
        // column = row i of the chunk).  Each warp takes its 32 lanes as two groups of 16
        // in rounds of 16 columns: a 16x256b TMEM load gives the MMA-fragment layout of a
        // [16 d x 16 i] block, and stmatrix .trans writes its four 8x8 parts transposed, as
        // 16-byte rows of the staging chunk (row i, 8 consecutive d).  Named barrier 1
        // (the warps that write the staging chunk: all four, or with D = 64 the two of lanes
        // 64..127) is reached by all of them whatever the waits return.  With D = 64 the other
        // two warps hold no output: they run ahead, releasing each accumulator as soon as it is
        // full, and (NORM) the first of them forms the chunk's reciprocal denominators from
        // lane 0 (the column of ones) into sDen[it & 1] a chunk ahead of their use.
        const int ot = threadIdx.x - kROw0 * 32;
        const int sub = warp & 3;
        const int q4 = lane & 3;                            // fragment: columns 2 q4 (+1) of lanes lane / 4 (+8)
        const int mk = lane >> 3, mj = lane & 7;            // stmatrix: matrix mk, stored row mj
        // prep (forward only): the dout chunk of iteration it in the unused second box of K^
        // hi (it even) or lo (it odd), loaded one iteration ahead
        const bool prep = NORM && jobs.prep;
        const bool out32 = NBOX == 1 && jobs.o32[pass];
        auto gbuf = [&](int it) -> uint8_t * { return sKh + (it & 1) * kTile128 + kBox; };
        if (prep && ot == 0 && nchunks > 0) {
            mbar_arrive_expect_tx(&gfull[0], kBox);
            tma_load_3d(gbuf(0), &jobs.g, &gfull[0], 0, 0, bh);
        }
        auto scale_in = [&](int rows, int i) -> float {   // FOLD: f_i; else g_i of the inter-chunk part
            if (FOLD) return rev ? (i < rows ? GP(rows - i - kM) : 0.f) : GP(i + 1 - kM);
            return rev ? (i < rows ? GP(rows - i) : 0.f) : GP(i + 1);
        };
        constexpr int kStageThreads = (NBOX == 1 ? 2 : kROWarps) * 32;   // named barrier 1
        bool live = true;
        if (NBOX == 1 && sub < 2) {
            for (int it = 0; it < (sonly ? 0 : nchunks); ++it) {
                const int c = rev ? nchunks - 1 - it : it;
                const int rows = min(kC, T - c * kC);
                const int ob = FOLD ? (it & 1) : 0;
                if (!__all_sync(0xffffffffu, LA_RWAIT(&ofull[ob], FOLD ? (uint32_t)((it >> 1) & 1) : (uint32_t)(it & 1),
                                                      0x800u)))
                    break;
                __syncwarp();   // converged for the .sync.aligned TMEM loads
                tc_fence_after();
                if (NORM && sub == 0) {
                    // sDen[it & 1] was last read for iteration it - 2
                    if (it >= 2 && !__all_sync(0xffffffffu, LA_RWAIT(&denfree[it & 1], (uint32_t)(((it >> 1) & 1) ^ 1),
                                                                      0x20000u)))
                        break;
                    float *den = sDen + 64 * (it & 1);
                    // threads 0..3 hold lane 0, columns 16 h + 2 t, +1, +8, +9 (16x256b layout)
#pragma unroll 1
                    for (int h = 0; h < 4; ++h) {
                        uint32_t r[8];
                        float x0, x1, x8, x9;
                        const int c0 = 16 * h + 2 * q4;
                        if (FOLD) {
                            tmem_ld16x256b_x2_sync(tmem + cO + 64u * (uint32_t)ob + 16 * h, r);
                            x0 = scale_in(rows, c0) * __uint_as_float(r[0]);
                            x1 = scale_in(rows, c0 + 1) * __uint_as_float(r[1]);
                            x8 = scale_in(rows, c0 + 8) * __uint_as_float(r[4]);
                            x9 = scale_in(rows, c0 + 9) * __uint_as_float(r[5]);
                        } else {
                            uint32_t xi[8];
                            tmem_ld16x256b_x2_sync(tmem + cOI + 16 * h, xi);
                            tmem_ld16x256b_x2_sync(tmem + cOX + 16 * h, r);
                            x0 = fmaf(scale_in(rows, c0), __uint_as_float(r[0]), __uint_as_float(xi[0]));
                            x1 = fmaf(scale_in(rows, c0 + 1), __uint_as_float(r[1]), __uint_as_float(xi[1]));
                            x8 = fmaf(scale_in(rows, c0 + 8), __uint_as_float(r[4]), __uint_as_float(xi[4]));
                            x9 = fmaf(scale_in(rows, c0 + 9), __uint_as_float(r[5]), __uint_as_float(xi[5]));
                        }
                        // the reciprocals, once per row (approximate reciprocal: a few fp32 ulp)
                        if (lane < 4) {
                            *reinterpret_cast<float2 *>(den + c0) =
                                make_float2(__fdividef(1.f, x0 + jobs.eps), __fdividef(1.f, x1 + jobs.eps));
                            *reinterpret_cast<float2 *>(den + c0 + 8) =
                                make_float2(__fdividef(1.f, x8 + jobs.eps), __fdividef(1.f, x9 + jobs.eps));
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&denready[it & 1]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&oread[ob]);
            }
        } else {
        for (int it = 0; it < (sonly ? 0 : nchunks); ++it) {
            const int c = rev ? nchunks - 1 - it : it;
            const uint32_t pc = (uint32_t)(it & 1);
            if (ot == 0) tma_store_wait_read<0>();
            named_bar(1, kStageThreads);
            // the buffer of iteration it + 1 was last read in iteration it - 1, now complete
            if (prep && ot == 0 && it + 1 < nchunks) {
                mbar_arrive_expect_tx(&gfull[(it + 1) & 1], kBox);
                tma_load_3d(gbuf(it + 1), &jobs.g, &gfull[(it + 1) & 1], 0, (it + 1) * kC, bh);
            }
            const int ob = FOLD ? (it & 1) : 0;
            bool got = live && LA_RWAIT(&ofull[ob], FOLD ? (uint32_t)((it >> 1) & 1) : pc, 0x800u);
            got = __all_sync(0xffffffffu, got);
            live = live && got;
            // backwards the entering state sits one past the chunk's last valid row
            const int rows = min(kC, T - c * kC);
            auto scale = [&](int i) -> float { return scale_in(rows, i); };
            if (got) {
                __syncwarp();   // converged for the .sync.aligned TMEM loads
                tc_fence_after();
            }
            const float *den = sDen + 64 * (it & 1);
            if (NORM && got) {
                got = __all_sync(0xffffffffu, LA_RWAIT(&denready[it & 1], (uint32_t)((it >> 1) & 1), 0x40000u));
                live = live && got;
            }
            if (got) {
                const uint8_t *gb = gbuf(it);
                if (prep) {
                    got = __all_sync(0xffffffffu, LA_RWAIT(&gfull[it & 1], (uint32_t)((it >> 1) & 1), 0x8000u));
                    live = live && got;
                }
#pragma unroll 1
                for (int h = 0; h < 4; ++h) {
                    const int i0 = 16 * h + 2 * q4;
                    float pA = 0.f, pB = 0.f, pC = 0.f, pD = 0.f;   // prep: dout . o of rows i0, +1, +8, +9
                    float f0 = scale(i0), f1 = scale(i0 + 1), f8 = scale(i0 + 8), f9 = scale(i0 + 9);
                    // NORM: each row times the reciprocal of its denominator
                    const float u0 = NORM ? den[i0] : 1.f, u1 = NORM ? den[i0 + 1] : 1.f;
                    const float u8 = NORM ? den[i0 + 8] : 1.f, u9 = NORM ? den[i0 + 9] : 1.f;
                    if (FOLD) {
                        f0 *= u0;
                        f1 *= u1;
                        f8 *= u8;
                        f9 *= u9;
                    }
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        const int dbase = 32 * sub + 16 * half;
                        const uint32_t tl = (uint32_t)dbase << 16;
                        uint32_t r[8];
                        float y[8];
                        if (FOLD) {
                            tmem_ld16x256b_x2_sync(tmem + cO + 64u * (uint32_t)ob + tl + 16 * h, r);
                            y[0] = f0 * __uint_as_float(r[0]);
                            y[1] = f1 * __uint_as_float(r[1]);
                            y[2] = f0 * __uint_as_float(r[2]);
                            y[3] = f1 * __uint_as_float(r[3]);
                            y[4] = f8 * __uint_as_float(r[4]);
                            y[5] = f9 * __uint_as_float(r[5]);
                            y[6] = f8 * __uint_as_float(r[6]);
                            y[7] = f9 * __uint_as_float(r[7]);
                        } else {
                            uint32_t x[8];
                            tmem_ld16x256b_x2_sync(tmem + cOI + tl + 16 * h, r);
                            tmem_ld16x256b_x2_sync(tmem + cOX + tl + 16 * h, x);
                            const float fs[8] = {f0, f1, f0, f1, f8, f9, f8, f9};
                            const float us[8] = {u0, u1, u0, u1, u8, u9, u8, u9};
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                y[e] = us[e] * fmaf(fs[e], __uint_as_float(x[e]), __uint_as_float(r[e]));
                        }
                        if (h == 3 && half == 1) {
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&oread[ob]);
                        }
                        if (prep && got) {
                            // y holds o: the sums dout . o, and du = dout / n in its place.  The
                            // dout tile is laid out as the staging chunk (row i, value index d =
                            // lane - 64), so ldmatrix .trans gives it in y's fragment layout.
                            const int grow = 16 * h + mj + (mk >= 2 ? 8 : 0);
                            const int gd = dbase - 64 + ((mk & 1) ? 8 : 0);
                            uint32_t w0, w1, w2, w3;
                            ldmatrix_x4_trans(smem_u32(gb + grow * 128 + (((gd >> 3) ^ (grow & 7)) << 4)), w0, w1, w2, w3);
                            const float2 e0 = h2<BF>::to_f2(w0), e1 = h2<BF>::to_f2(w1), e2 = h2<BF>::to_f2(w2),
                                         e3 = h2<BF>::to_f2(w3);
                            const float g0 = e0.x, g1 = e0.y, g2 = e1.x, g3 = e1.y, g4 = e2.x, g5 = e2.y, g6 = e3.x,
                                        g7 = e3.y;
                            pA += y[0] * g0 + y[2] * g2;
                            pB += y[1] * g1 + y[3] * g3;
                            pC += y[4] * g4 + y[6] * g6;
                            pD += y[5] * g5 + y[7] * g7;
                            y[0] = g0 * u0;
                            y[1] = g1 * u1;
                            y[2] = g2 * u0;
                            y[3] = g3 * u1;
                            y[4] = g4 * u8;
                            y[5] = g5 * u9;
                            y[6] = g6 * u8;
                            y[7] = g7 * u9;
                        }
                        if (NBOX == 1 && out32) {
                            // fp32 staging: two boxes of [64 rows x 32 columns], 128-byte swizzle
                            const int d0 = dbase - 64 + (lane >> 2);
                            auto put = [&](int i, int d, float x) {
                                *reinterpret_cast<float *>(sO + (d >> 5) * kBox + i * 128 +
                                                           ((((d & 31) >> 2) ^ (i & 7)) << 4) + (d & 3) * 4) = x;
                            };
                            put(i0, d0, y[0]);
                            put(i0 + 1, d0, y[1]);
                            put(i0, d0 + 8, y[2]);
                            put(i0 + 1, d0 + 8, y[3]);
                            put(i0 + 8, d0, y[4]);
                            put(i0 + 9, d0, y[5]);
                            put(i0 + 8, d0 + 8, y[6]);
                            put(i0 + 9, d0 + 8, y[7]);
                            continue;
                        }
                        // matrices: (d 0..7, i 0..7), (d 8..15, i 0..7), (d 0..7, i 8..15), (d 8..15, i 8..15)
                        const int row = 16 * h + mj + (mk >= 2 ? 8 : 0);
                        const int dch = dbase + ((mk & 1) ? 8 : 0);
                        const uint32_t sa = smem_u32(sO + (dch >> 6) * kBox + row * 128 +
                                                     ((((dch & 63) >> 3) ^ (row & 7)) << 4));
                        stmatrix_x4_trans(sa, h2<BF>::from_f2(y[0], y[1]), h2<BF>::from_f2(y[2], y[3]),
                                          h2<BF>::from_f2(y[4], y[5]), h2<BF>::from_f2(y[6], y[7]));
                    }
                    if (prep) {
                        // over the 8 lane groups of the warp, then one part per warp in sDot
#pragma unroll
                        for (int m = 4; m < 32; m <<= 1) {
                            pA += __shfl_xor_sync(0xffffffffu, pA, m);
                            pB += __shfl_xor_sync(0xffffffffu, pB, m);
                            pC += __shfl_xor_sync(0xffffffffu, pC, m);
                            pD += __shfl_xor_sync(0xffffffffu, pD, m);
                        }
                        if (lane < 4) {
                            float *dst = sDot + (sub - 2) * 64;
                            dst[i0] = pA;
                            dst[i0 + 1] = pB;
                            dst[i0 + 8] = pC;
                            dst[i0 + 9] = pD;
                        }
                    }
                }
            }
            if (prep && sub >= 2) {
                // dn = -(dout . o) / n of the chunk's rows, from the two warps' parts
                named_bar(3, 64);
                if (sub == 2 && got) {
#pragma unroll
                    for (int r2 = 0; r2 < 2; ++r2) {
                        const int i = lane + 32 * r2;
                        if (i < rows)
                            jobs.dn[(long long)bh * T + (long long)c * kC + i] = -(sDot[i] + sDot[64 + i]) * den[i];
                    }
                }
            }
            if (NORM) {   // den read for this chunk
                __syncwarp();
                if (lane == 0) mbar_arrive(&denfree[it & 1]);
            }
            fence_async_smem();
            named_bar(1, kStageThreads);
            if (ot == 0 && live) {
                if (NBOX == 1 && out32) {
                    tma_store_3d(tmO, sO, 0, c * kC, bh);
                    tma_store_3d(tmO, sO + kBox, 32, c * kC, bh);
                } else {
                    tma_store_3d(tmO, sO + vbox * kBox, 0, c * kC, bh);
                    if (NBOX == 2) tma_store_3d(tmO, sO + kBox, 64, c * kC, bh);
                }
                tma_store_commit();
            }
        }
        if (ot == 0) tma_store_wait_all<0>();
        if (prep && ot == 0) {
            // every dout load has landed before the shared memory goes (an early exit may
            // leave the last ones unread): the last phase of each buffer
            for (int b = 0; b < 2; ++b) {
                const int nb = (nchunks + 1 - b) / 2;
                if (nb > 0) mbar_wait_slow(smem_u32(&gfull[b]), (uint32_t)((nb - 1) & 1), nullptr, &g_ret_fault, 0x10000u);
            }
        }
        }
    } else {
        // State warps: S^T_{c+1} = gamma^C S^T_c + dS^T_c in fp32 registers; thread (d, half)
        // holds row d of S^T (column d of S), entries SC half .. SC half + SC - 1 (its TMEM
        // lane of dS^T), and writes them as the bf16 hi + lo A operand of O_inter^T.  D = 128:
        // SC = 64.  D = 64: the value dimensions sit in lanes 64..127 (d = 64 + value index),
        // whose rows split their 64 entries (SC = 32); the warps of lanes 0..63, which would
        // hold zeros, only keep the barriers' counts.
        constexpr int SC = 64 / (3 - NBOX);
        const int sub = warp & 3, half = (warp - kRSw0) >> 2;
        const uint32_t lanes = (uint32_t)(32 * sub) << 16;
        const int d = 32 * sub + lane;
        // (NORM: lane 0, the column of ones, carries z; its warps hold the rest of lanes 0..31 as zeros)
        const bool sact = NBOX == 2 || sub >= 2 || (NORM && sub == 0);
        const int dv = d - 64 * vbox;          // the value dimension of lane d
        const int col0 = SC * half;
        const float gC = GP(kC);
        const float gm = FOLD ? GP(kM) : 1.f;   // the state operand holds gamma^m S (FOLD)
        // decay over the partial chunk at the end of the sequence: the last chunk
        // forwards, the first one backwards
        const float gLast = GP(min(kC, T - (nchunks - 1) * kC));
        float st[SC];
        const float *sin = jobs.sin[pass];
        float *sout = jobs.sout[pass];
        const long long sbase = (long long)bh * D * D;
        if (sin && sact && dv >= 0) {
            if (jobs.sin_t[pass]) {   // sin holds S^T: row d, entries col0 ..
#pragma unroll
                for (int c4 = 0; c4 < SC / 4; ++c4) {
                    const float4 x = *reinterpret_cast<const float4 *>(sin + sbase + (long long)dv * D + col0 + 4 * c4);
                    st[4 * c4] = x.x;
                    st[4 * c4 + 1] = x.y;
                    st[4 * c4 + 2] = x.z;
                    st[4 * c4 + 3] = x.w;
                }
            } else {                  // sin holds S: column d (lanes read consecutive d)
#pragma unroll
                for (int c = 0; c < SC; ++c) st[c] = sin[sbase + (long long)(col0 + c) * D + dv];
            }
        } else {
#pragma unroll
            for (int i = 0; i < SC; ++i) st[i] = 0.f;
        }
        // The state operand: this thread's SC entries as SC / 2 packed columns of its lane,
        // hi at cSA + col0 / 2, lo 64 columns further, in rounds of 8 columns.
        auto write_state = [&]() {
            if (sact) {
#pragma unroll
            for (int r = 0; r < SC / 16; ++r) {
                uint32_t hw[8], lw[8];
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const float a = gm * st[16 * r + 2 * m], b = gm * st[16 * r + 2 * m + 1];
                    hw[m] = h2<BF>::from_f2(a, b);
                    const float2 hv = h2<BF>::to_f2(hw[m]);
                    lw[m] = h2<BF>::from_f2(a - hv.x, b - hv.y);
                }
                tmem_st8(tmem + cSA + lanes + col0 / 2 + 8 * r, hw);
                tmem_st8(tmem + cSA + 64 + lanes + col0 / 2 + 8 * r, lw);
            }
            tmem_st_wait();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(sready);
        };
        if (!sonly) write_state();                         // S_0
        // K^ = diag(gamma^(C-1-j)) K of chunk iteration itk as hi + lo: thread kt takes row
        // kt % 64 and the 8-element chunks 2 NBOX (kt / 64) .. + 2 NBOX - 1 of the row's 16
        // (with D = 64 the first box only).  Forwards in time the weights count back from the
        // chunk's last valid row, so that the state after a partial last chunk is the state
        // after token T - 1.
        const int kt = threadIdx.x - kRSw0 * 32;
        const int krow = kt & 63, kpart = kt >> 6;
        auto build_khat = [&](int itk) -> bool {
            const int sk = itk % NST;
            if (!__all_sync(0xffffffffu, LA_RWAIT(&full[sk], (uint32_t)((itk / NST) & 1), 0x100u))) return false;
            const int rows = min(kC, T - (rev ? nchunks - 1 - itk : itk) * kC);
            const float f = rev ? GP(krow) : (krow < rows ? GP(rows - 1 - krow) : 0.f);
            scale_split_row<2 * NBOX, BF>(sK + sk * kTile128, sKh, krow, kpart, f, true);
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(khready);
            return true;
        };
        const bool k0 = nchunks > 0 && build_khat(0);
        for (int it = 0; it < nchunks && k0; ++it) {
            const uint32_t pc = (uint32_t)(it & 1);
            if (!__all_sync(0xffffffffu, LA_RWAIT(dsfull, pc, 0x1000u))) break;
            __syncwarp();   // converged for the .sync.aligned TMEM loads
            tc_fence_after();
            const uint32_t base = tmem + cDS + lanes + (uint32_t)col0;
            const float g = (it == (rev ? 0 : nchunks - 1)) ? gLast : gC;
            if (sact) {
#pragma unroll
            for (int c4 = 0; c4 < SC / 16; ++c4) {
                float a[16];
                tmem_ld16_sync(base + 16 * c4, a);
#pragma unroll
                for (int i = 0; i < 16; ++i) st[16 * c4 + i] = fmaf(g, st[16 * c4 + i], a[i]);
            }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(dsread);
            if (it + 1 == nchunks) break;                  // st holds the state after the sequence
            // dS^T_c is complete, so it has read K^_c: the buffer takes K^ of the next chunk
            if (!build_khat(it + 1)) break;
            if (sonly) continue;                           // nothing reads the state operand
            if (!__all_sync(0xffffffffu, LA_RWAIT(sfree, pc, 0x2000u))) break;   // O_inter^T(c) read S_c
            __syncwarp();
            tc_fence_after();
            write_state();
        }
        if (sout && sact && dv >= 0 && !*s_abort) {   // S after the last chunk: column d of S, lanes write consecutive d
#pragma unroll
            for (int c = 0; c < SC; ++c) sout[sbase + (long long)(col0 + c) * D + dv] = st[c];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
#undef GP
}

// The folded output stores the masked products scaled by gamma^(m-1-j) (up to gamma^-32) and the
// state operand as gamma^m S (gamma^32) in the 16-bit type: bf16 has the fp32 exponent range,
// which gamma >= 1/8 keeps them far inside; fp16 (largest value 65504, smallest normal 6.1e-5)
// takes the fold only for gamma >= 0.9 (factors within 29 and 1/29 of 1).
static bool fold_ok(const DecayArgs &dec, int H, bool bf16) {
    const float lo = bf16 ? 0.125f : 0.9f;
    for (int h = 0; h < H; ++h)
        if (!(dec.gamma[h] >= lo)) return false;
    return true;
}

#ifndef LA_TRY
#define LA_TRY(x)                     \
    do {                              \
        la_status _rc = (x);          \
        if (_rc != LA_OK) return _rc; \
    } while (0)
#endif

// One launch of `passes` x BH CTAs: the folded kernel when every decay allows it (launch
// name `folded`), else the one with two output accumulators (`unfolded`); D = 64 or 128.
template <int NBOX, bool BF>
static la_status launch_retention_t(const char *folded, const char *unfolded, int passes, const RetJobs &jobs,
                                    const DecayArgs &dec, const Shape &s, cudaStream_t st) {
    const dim3 grid((unsigned)(passes * s.BH())), block(kRThreads);
    const size_t smem = (size_t)RetLayout::bytes;
    return fold_ok(dec, s.H, BF)
               ? launch_pdl(folded, retention_kernel<true, NBOX, BF, false>, grid, block, smem, st, jobs, dec, s.T, s.H,
                            (int)s.BH())
               : launch_pdl(unfolded, retention_kernel<false, NBOX, BF, false>, grid, block, smem, st, jobs, dec, s.T,
                            s.H, (int)s.BH());
}

static la_status launch_retention(const char *folded, const char *unfolded, int passes, const RetJobs &jobs,
                                  const DecayArgs &dec, const Shape &s, bool bf16, cudaStream_t st) {
    if (s.D == 64)
        return bf16 ? launch_retention_t<1, true>(folded, unfolded, passes, jobs, dec, s, st)
                    : launch_retention_t<1, false>(folded, unfolded, passes, jobs, dec, s, st);
    return bf16 ? launch_retention_t<2, true>(folded, unfolded, passes, jobs, dec, s, st)
                : launch_retention_t<2, false>(folded, unfolded, passes, jobs, dec, s, st);
}

}  // namespace

la_status retention_fwd(const void *q, const void *k, const void *v, void *o, const float *sin, float *sout,
                        const DecayArgs &dec, const Shape &s, bool bf16, cudaStream_t st) {
    RetJobs jobs;
    memset(&jobs, 0, sizeof jobs);
    jobs.sin[0] = sin;
    jobs.sout[0] = sout;
    jobs.sonly[0] = o == nullptr;   // the state only: q and o are not touched (their maps stand in as k's)
    LA_TRY(retention_map(&jobs.q[0], o ? q : k, s, bf16));
    LA_TRY(retention_map(&jobs.k[0], k, s, bf16));
    LA_TRY(retention_map(&jobs.v[0], v, s, bf16));
    LA_TRY(retention_map(&jobs.o[0], o ? o : k, s, bf16));
    return o ? launch_retention("tc_retention_fwd", "tc_retention_fwd_unfolded", 1, jobs, dec, s, bf16, st)
             : launch_retention("tc_retention_state", "tc_retention_state_unfolded", 1, jobs, dec, s, bf16, st);
}

la_status retention_norm_fwd(const void *q, const void *k, const void *v, void *o, const void *dout, float *dn,
                             const DecayArgs &dec, float eps, const Shape &s, bool bf16, cudaStream_t st) {
    if (s.D != 64) return LA_ERR_UNSUPPORTED;
    RetJobs jobs;
    memset(&jobs, 0, sizeof jobs);
    LA_TRY(retention_map(&jobs.q[0], q, s, bf16));
    LA_TRY(retention_map(&jobs.k[0], k, s, bf16));
    LA_TRY(retention_map(&jobs.v[0], v, s, bf16));
    LA_TRY(retention_map(&jobs.o[0], o, s, bf16));
    jobs.eps = eps;
    if (dout) {
        LA_TRY(retention_map(&jobs.g, dout, s, bf16));
        jobs.prep = 1;
        jobs.dn = dn;
    }
    const char *name = dout ? (fold_ok(dec, s.H, bf16) ? "tc_causal_norm_prep" : "tc_causal_norm_prep_unfolded")
                            : (fold_ok(dec, s.H, bf16) ? "tc_causal_norm_fwd" : "tc_causal_norm_fwd_unfolded");
    const dim3 grid((unsigned)s.BH()), block(kRThreads);
    const size_t smem = (size_t)RetLayout::bytes;
    if (fold_ok(dec, s.H, bf16))
        return bf16 ? launch_pdl(name, retention_kernel<true, 1, true, true>, grid, block, smem, st, jobs, dec, s.T,
                                 s.H, (int)s.BH())
                    : launch_pdl(name, retention_kernel<true, 1, false, true>, grid, block, smem, st, jobs, dec, s.T,
                                 s.H, (int)s.BH());
    return bf16 ? launch_pdl(name, retention_kernel<false, 1, true, true>, grid, block, smem, st, jobs, dec, s.T, s.H,
                             (int)s.BH())
                : launch_pdl(name, retention_kernel<false, 1, false, true>, grid, block, smem, st, jobs, dec, s.T, s.H,
                             (int)s.BH());
}

la_status retention_bwd(const void *q, const void *k, const void *v, const void *g, const float *sin,
                        const float *rin, float *rout, const DecayArgs &dec, void *dq, void *dk, void *dv,
                        const Shape &s, bool bf16, cudaStream_t st, float *dq32, float *dk32) {
    RetJobs jobs;
    memset(&jobs, 0, sizeof jobs);
    // dq = retention(dO, V, K); dv = reverse retention(K, Q, dO); dk = reverse retention(V, dO, Q).
    // Their states are S^T (S = sum k^T v), R and R^T (R = sum gamma^(t-s) q_t^T dO_t).
    // dq == null leaves out the first pass; dq, dk and dv all null leave only the second, as a
    // state-only pass (R at the first row, rout).
    const bool sonly = !dq && !dk && !dv;
    if (sonly) {
        jobs.rev[0] = 1;
        jobs.sin[0] = rin;
        jobs.sout[0] = rout;
        jobs.sonly[0] = 1;
        LA_TRY(retention_map(&jobs.q[0], q, s, bf16));
        LA_TRY(retention_map(&jobs.k[0], q, s, bf16));
        LA_TRY(retention_map(&jobs.v[0], g, s, bf16));
        LA_TRY(retention_map(&jobs.o[0], q, s, bf16));
        return launch_retention("tc_retention_state", "tc_retention_state_unfolded", 1, jobs, dec, s, bf16, st);
    }
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
        LA_TRY(retention_map(&jobs.q[np], all[p].q, s, bf16));
        LA_TRY(retention_map(&jobs.k[np], all[p].k, s, bf16));
        LA_TRY(retention_map(&jobs.v[np], all[p].v, s, bf16));
        float *o32 = p == 0 ? dq32 : p == 2 ? dk32 : nullptr;
        if (o32) {
            LA_TRY(retention_map_f32(&jobs.o[np], o32, s));
            jobs.o32[np] = 1;
        } else {
            LA_TRY(retention_map(&jobs.o[np], all[p].o, s, bf16));
        }
        jobs.rev[np] = all[p].rev;
        jobs.sin[np] = all[p].sin;
        jobs.sin_t[np] = all[p].sin_t;
        jobs.sout[np] = all[p].sout;
    }
    return launch_retention("tc_retention_bwd", "tc_retention_bwd_unfolded", np, jobs, dec, s, bf16, st);
}

unsigned int read_and_clear_retention_fault() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_ret_fault, sizeof v) != cudaSuccess) return 0xFFFFFFFFu;
    if (v) cudaMemcpyToSymbol(g_ret_fault, &zero, sizeof zero);
    return v;
}

}  // namespace tc
}  // namespace la

