// la_tc_state.cu -- tensor-core kernels of bidirectional linear attention and simple_la
// (fp16 / bf16 storage, D = 64, fp32 accumulation in TMEM).
//
// "Flash Bi-directional Linear Attention" README (intro; "Update": simple_la is
// linear_attn without the norm term).  Forward, with f = elu+1 (bidir) or the
// identity (simple):
//   state_reduce:  S = sum_t f(k_t)^T v_t, z = sum_t f(k_t)     (per CTA partial, fp32)
//   output:        o_t = f(q_t) S / (f(q_t).z + eps)  (bidir)  |  q_t S  (simple)
// Backward (hand-derived; see include/la.h):
//   bwd_q:   n_t, o_t recomputed; dq_t = (g_t S^T - (g_t.o_t) z)/n_t * f'(q_t);
//            partial dS = sum_t f(q_t)^T g_t/n_t, dz = -sum_t f(q_t)(g_t.o_t)/n_t
//   bwd_kv:  dk_s = (v_s dS^T + dz) * f'(k_s),  dv_s = f(k_s) dS
//
// Every kernel is persistent: kGrid CTAs split the head-major list of 128-row
// tiles into contiguous ranges (Partition).  Warp 0 streams q/k/v/dO tiles with
// TMA into a ring of 128-byte-swizzled stages; warp 1 owns TMEM and issues the
// tcgen05 UMMAs (fp32 accumulators in TMEM); warps 2..9 apply the feature map in
// place (half a row each); warps 10..13 run the epilogues (TMEM -> registers ->
// swizzled staging -> TMA store) and build the per-head state operand.  A reduction's per-CTA partial goes to slot
// (cta - first_cta(head)) of the workspace; its consumer sums the slots in slot
// order, so results are deterministic.
//
// The D x D state operand of the row-wise products is stored K-major with the
// state's column index as the row: row n holds S[0..63][n], row 64 holds z.
// Read K-major it is [S | z]^T (for f(q)[S | z]); read MN-major (its first 64
// rows) it is S (for g S^T).  fp16 operands carry a power-of-two scale chosen
// per head (range); bf16 operands are split hi + lo (precision).
#include "la_tc.cuh"
#include "la_tc_common.cuh"

#include <cudaTypedefs.h>
#include <mutex>

namespace la {
namespace tc {

// Fault word of the tensor-core kernels (a wait ran out): read by la_device_check().
__device__ unsigned int g_tc_fault = 0;

namespace {

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

#ifndef LA_TRY
#define LA_TRY(x)                     \
    do {                              \
        la_status _rc = (x);          \
        if (_rc != LA_OK) return _rc; \
    } while (0)
#endif

// Waits used by every role; codes identify the barrier in the fault word.
#define LA_WAIT(bar, par, code) mbar_wait((bar), (par), s_abort, &g_tc_fault, (code))
// The UMMA-issuing warps run their loops with all 32 lanes in step (every lane waits, one
// elected lane issues each UMMA and commit), so the descriptors stay warp-uniform: issued
// by one lane alone, each UMMA first moved its operands to uniform registers, and on a
// scheduler shared with busy warps that cost ~140 cycles an instruction.
#define LA_WWAIT(bar, par, code) __all_sync(0xffffffffu, LA_WAIT((bar), (par), (code)))

// ============================================================ state_reduce ==
// Partial (S | z) of every (CTA, head) segment.  UMMA M = 64 (the state row i),
// N = 64 (+16 with the ones block that yields z), K = 128 tile rows:
//   A = f(K)^T read MN-major from the k tile, B = [V | 1] read MN-major.
// bf16 bidir also multiplies in lo = round(f(k) - hi) (its own tile), so S and z
// carry f(k) to fp32 accuracy.
template <bool BIDIR, bool BF16>
struct ReduceLayout {
    static constexpr bool KLO = BIDIR && BF16;
    static constexpr int NST = KLO ? 4 : 6;
    static constexpr int koff = 0;
    static constexpr int voff = koff + NST * kTileBytes;
    static constexpr int kloff = voff + NST * kTileBytes;
    static constexpr int onesoff = kloff + (KLO ? NST * kTileBytes : 0);
    static constexpr int baroff = onesoff + kTileBytes;
    static constexpr int nbars = 3 * NST + 5;
    static constexpr int misc = baroff + nbars * 8;
    static constexpr int bytes = misc + 32 + 1024;
    static_assert(bytes <= 227 * 1024, "shared memory of one CTA");
};

template <bool BIDIR, bool BF16, bool PHI>
__global__ void __launch_bounds__(kThreads, 1)
state_reduce_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    float *__restrict__ part, int T, int BH, int nt, int maxslots) {
    using L = ReduceLayout<BIDIR, BF16>;
    constexpr int NST = L::NST;
    constexpr bool KLO = L::KLO;
    constexpr int N = BIDIR ? 80 : 64;
    constexpr uint32_t IDESC = idesc_f16(64, N, BF16, true, true);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *sK = smem + L::koff;
    uint8_t *sV = smem + L::voff;
    uint8_t *sKlo = smem + L::kloff;
    uint8_t *sOnes = smem + L::onesoff;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::baroff);
    uint64_t *xf = full + NST;
    uint64_t *empty = xf + NST;
    uint64_t *accfull = empty + NST;   // [2]
    uint64_t *accfree = accfull + 2;   // [2]
    uint64_t *drain = accfree + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::misc);
    int *s_abort = reinterpret_cast<int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Partition P{(long long)BH * nt, nt, grid_for((long long)BH * nt)};
    const int cta = blockIdx.x;
    const long long x0 = P.start(cta), x1 = P.start(cta + 1);
    if (x0 >= x1) return;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&xf[s], kXWarps);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&accfull[a], 1);
            mbar_init(&accfree[a], kEWarps);
        }
        mbar_init(drain, 1);
        *s_abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch(&tmK);
        tma_prefetch(&tmV);
    }
    if (BIDIR && warp >= kEw0) {
        // ones block: column 0 (state column 64) = 1 for every tile row, zeros elsewhere
        const int r = threadIdx.x - kEw0 * 32;
        uint8_t *p = sOnes + r * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4 *>(p + c * 16) = make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint16_t *>(sOnes + sw128_offset(r, 0)) = h2<BF16>::one();
        fence_async_smem();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 256);
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

    if (warp == 0) {
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            long long issued = 0;
            for (TileCursor t(x0, nt); t.x < x1; t.next()) {
                const int h = t.h, j = t.j;
                if (!LA_WAIT(&empty[s], ph ^ 1, 0x1u)) break;
                mbar_arrive_expect_tx(&full[s], 2 * kTileBytes);
                tma_load_3d(sK + s * kTileBytes, &tmK, &full[s], 0, j * kRows, h);
                tma_load_3d(sV + s * kTileBytes, &tmV, &full[s], 0, j * kRows, h);
                ++issued;
                if (++s == NST) { s = 0; ph ^= 1; }
            }
            if (*s_abort) {   // let the loads in flight land before the CTA's smem goes away
                for (long long i = issued - 1; i >= 0 && i >= issued - NST; --i)
                    mbar_wait_slow(smem_u32(&full[i % NST]), (uint32_t)((i / NST) & 1), nullptr, &g_tc_fault, 0x200u);
            }
        }
    } else if (warp == 1) {
        int s = 0, a = 0;
        uint32_t ph = 0, aph = 0;
        bool seg_start = true;
        for (TileCursor t(x0, nt); t.x < x1; t.next()) {
            const long long x = t.x;
            const bool seg_end = (x + 1 == x1) || t.last_of_head();
            if (seg_start) {
                if (!LA_WWAIT(&accfree[a], aph ^ 1, 0x2u)) break;
            }
            if (!LA_WWAIT(BIDIR ? &xf[s] : &full[s], ph, 0x4u)) break;
            tc_fence_after();
            const uint32_t d = tmem + (uint32_t)a * 128u;
            const uint32_t aV = smem_u32(sV + s * kTileBytes);
            const uint32_t lbo = BIDIR ? (smem_u32(sOnes) - aV) : (uint32_t)kTileBytes;
            const uint64_t dk = sdesc_sw128(smem_u32(sK + s * kTileBytes), kTileBytes, 1024);
            const uint64_t dkl = sdesc_sw128(smem_u32(sKlo + s * kTileBytes), kTileBytes, 1024);
            const uint64_t dv = sdesc_sw128(aV, lbo, 1024);
#pragma unroll
            for (int kk = 0; kk < kRows / 16; ++kk) {
                umma_f16_ss_warp(d, desc_at(dk, kk * 2048), desc_at(dv, kk * 2048), IDESC,
                                 (seg_start && kk == 0) ? 0u : 1u);
                if (KLO) umma_f16_ss_warp(d, desc_at(dkl, kk * 2048), desc_at(dv, kk * 2048), IDESC, 1u);
            }
            umma_commit_warp(&empty[s]);
            if (seg_end) {
                umma_commit_warp(&accfull[a]);
                a ^= 1;
                if (a == 0) aph ^= 1;
            }
            seg_start = seg_end;
            if (++s == NST) { s = 0; ph ^= 1; }
        }
        umma_commit_warp(drain);
        mbar_wait_slow(smem_u32(drain), 0, nullptr, &g_tc_fault, 0x400u);
        __syncwarp();
    } else if (warp < kEw0) {
        if (BIDIR) {
            const int xi = threadIdx.x - kXw0 * 32;
            int s = 0;
            uint32_t ph = 0;
            for (TileCursor t(x0, nt); t.x < x1; t.next()) {
                const int j = t.j;
                const bool got = __all_sync(0xffffffffu, LA_WAIT(&full[s], ph, 0x8u));
                if (!got) break;
                const bool pad = j * kRows + (xi & 127) >= T;   // rows past the end: f(0) = 1 must not count
                if (KLO)
                    phi_half_row_split<BF16, PHI>(sK + s * kTileBytes, sKlo + s * kTileBytes, xi, pad);
                else
                    phi_half_row<BF16, PHI>(sK + s * kTileBytes, xi, pad);
                fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&xf[s]);
                if (++s == NST) { s = 0; ph ^= 1; }
            }
        }
    } else {
        const int sub = warp & 3;
        int a = 0;
        uint32_t aph = 0;
        for (TileCursor t(x0, nt); t.x < x1; t.next()) {
                const long long x = t.x;
            const int h = t.h;
            const bool seg_end = (x + 1 == x1) || t.last_of_head();
            if (!seg_end) continue;
            const bool got = __all_sync(0xffffffffu, LA_WAIT(&accfull[a], aph, 0x10u));
            if (!got) break;
            tc_fence_after();
            // M = 64 accumulator: state row i = 16*sub + l sits in TMEM lane 32*sub + l (l < 16)
            const uint32_t base = tmem + (uint32_t)a * 128u + ((uint32_t)(32 * sub) << 16);
            float v[64];
            tmem_row64(base, v);
            float zz = 0.f;
            if (BIDIR) {
                float t16[16];
                tmem_ld16(base + 64, t16);
                tmem_ld_wait(t16);
                zz = t16[0];
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&accfree[a]);
            if (lane < 16) {
                const int i = 16 * sub + lane;
                const int slot = cta - P.first_cta(h);
                float4 *dst = reinterpret_cast<float4 *>(part + ((long long)h * maxslots + slot) * kStateElems);
                // row i of the [64][65] block: 65 floats starting at i*65 (not 16-byte aligned): scalar stores
                float *d1 = reinterpret_cast<float *>(dst) + i * 65;
#pragma unroll
                for (int c = 0; c < 64; ++c) d1[c] = v[c];
                d1[64] = zz;
            }
            a ^= 1;
            if (a == 0) aph ^= 1;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ================================================================= output ==
// o = f(q) [S | z] / n per tile: UMMA M = 128 rows, N = 80 (64 + z + pad) or 64,
// K = 64, A = f(Q) tile K-major, B = state operand K-major (hi [+ lo]).  The
// epilogue warps build the operand of the CTA's next head into the second of
// two operand buffers while the current head's tiles stream.
struct OutputLayout {
    static constexpr int NST = 6, OST = 2, OPB = 80 * 128;
    static constexpr int qoff = 0;
    static constexpr int ooff = qoff + NST * kTileBytes;
    static constexpr int opoff = ooff + OST * kTileBytes;      // [buffer][hi, lo]
    static constexpr int stageoff = opoff + 4 * OPB;
    static constexpr int redoff = stageoff + kStateElems * 4;
    static constexpr int baroff = redoff + 32;
    static constexpr int nbars = 3 * NST + 2 + 2 + 2 + 1;
    static constexpr int misc = baroff + nbars * 8;
    static constexpr int bytes = misc + 32 + 1024;
    static_assert(bytes <= 227 * 1024, "shared memory of one CTA");
};

template <bool BIDIR, bool BF16, bool PHI>
__global__ void __launch_bounds__(kThreads, 1)
output_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
              const float *__restrict__ src, int src_per_head, int src_single, float *__restrict__ state_out, int T,
              int BH, int nt, float eps, int early_loads) {
    using L = OutputLayout;
    constexpr int NST = L::NST, OST = L::OST, OPB = L::OPB;
    constexpr int NOPS = BF16 ? 2 : 1;
    constexpr int N = BIDIR ? 80 : 64;
    constexpr uint32_t IDESC = idesc_f16(128, N, BF16, false, false);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *sQ = smem + L::qoff;
    uint8_t *sO = smem + L::ooff;
    uint8_t *sOp = smem + L::opoff;
    float *stage = reinterpret_cast<float *>(smem + L::stageoff);
    float *red = reinterpret_cast<float *>(smem + L::redoff);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::baroff);
    uint64_t *xf = full + NST;
    uint64_t *empty = xf + NST;
    uint64_t *accfull = empty + NST;
    uint64_t *accempty = accfull + 2;
    uint64_t *opready = accempty + 2;   // [2]
    uint64_t *drain = opready + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::misc);
    int *s_abort = reinterpret_cast<int *>(tmem_slot + 1);
    float *s_scale = reinterpret_cast<float *>(tmem_slot + 2);   // [2]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Partition P{(long long)BH * nt, nt, grid_for((long long)BH * nt)};
    const int cta = blockIdx.x;
    const long long x0 = P.start(cta), x1 = P.start(cta + 1);
    if (x0 >= x1) return;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&xf[s], kXWarps);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&accfull[a], 1);
            mbar_init(&accempty[a], kEWarps);
            mbar_init(&opready[a], 1);
        }
        mbar_init(drain, 1);
        *s_abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch(&tmQ);
        tma_prefetch(&tmO);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // Everything above touched only shared memory and TMEM: with a programmatic
    // launch it overlapped the previous kernel.  With `early_loads` (the previous
    // kernel is the first kernel of the same call, which writes none of this
    // kernel's inputs) the TMA producer starts streaming inputs right away; every
    // other access to global memory waits for the previous kernel here.
    if (!(early_loads && warp == 0)) grid_dependency_wait();
    if (threadIdx.x == 64) grid_launch_dependents();

    if (warp == 0) {
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            long long issued = 0;
            for (TileCursor t(x0, nt); t.x < x1; t.next()) {
                const int h = t.h, j = t.j;
                if (!LA_WAIT(&empty[s], ph ^ 1, 0x1u)) break;
                mbar_arrive_expect_tx(&full[s], kTileBytes);
                tma_load_3d(sQ + s * kTileBytes, &tmQ, &full[s], 0, j * kRows, h);
                ++issued;
                if (++s == NST) { s = 0; ph ^= 1; }
            }
            if (*s_abort) {
                for (long long i = issued - 1; i >= 0 && i >= issued - NST; --i)
                    mbar_wait_slow(smem_u32(&full[i % NST]), (uint32_t)((i / NST) & 1), nullptr, &g_tc_fault, 0x200u);
            }
        }
    } else if (warp == 1) {
        int s = 0, a = 0, hidx = -1;
        uint32_t ph = 0, aph = 0;
        long long prev_h = -1;
        for (TileCursor t(x0, nt); t.x < x1; t.next()) {
            const long long h = t.h;
            if (h != prev_h) {
                ++hidx;
                prev_h = h;
                if (!LA_WWAIT(&opready[hidx & 1], (uint32_t)((hidx >> 1) & 1), 0x20u)) break;
            }
            if (!LA_WWAIT(BIDIR ? &xf[s] : &full[s], ph, 0x4u)) break;
            if (!LA_WWAIT(&accempty[a], aph ^ 1, 0x2u)) break;
            tc_fence_after();
            const uint32_t d = tmem + (uint32_t)a * 128u;
            const uint64_t dq = sdesc_sw128(smem_u32(sQ + s * kTileBytes), 16, 1024);
            const uint64_t dop = sdesc_sw128(smem_u32(sOp + (hidx & 1) * 2 * OPB), 16, 1024);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
                for (int op = 0; op < NOPS; ++op)
                    umma_f16_ss_warp(d, desc_at(dq, kk * 32), desc_at(dop, op * OPB + kk * 32), IDESC,
                                     (kk | op) ? 1u : 0u);
            }
            umma_commit_warp(&empty[s]);
            umma_commit_warp(&accfull[a]);
            a ^= 1;
            if (a == 0) aph ^= 1;
            if (++s == NST) { s = 0; ph ^= 1; }
        }
        umma_commit_warp(drain);
        mbar_wait_slow(smem_u32(drain), 0, nullptr, &g_tc_fault, 0x400u);
        __syncwarp();
    } else if (warp < kEw0) {
        if (BIDIR) {
            const int xi = threadIdx.x - kXw0 * 32;
            int s = 0;
            uint32_t ph = 0;
            for (TileCursor t(x0, nt); t.x < x1; t.next()) {
                const bool got = __all_sync(0xffffffffu, LA_WAIT(&full[s], ph, 0x8u));
                if (!got) break;
                phi_half_row<BF16, PHI>(sQ + s * kTileBytes, xi, false);   // rows past T are never stored
                fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&xf[s]);
                if (++s == NST) { s = 0; ph ^= 1; }
            }
        }
    } else {
        // Epilogue warps.  Every named barrier is reached by all 128 of them whatever
        // the mbarrier waits return (a failed wait only skips work).
        const int tid = threadIdx.x - kEw0 * 32;
        const int sub = warp & 3;
        const int row = sub * 32 + lane;
        int a = 0, ob = 0, hidx = -1;
        uint32_t aph = 0;
        long long cur_h = -1;
        bool live = true;
        auto build = [&](long long h, int buf) {
            const float *srch = src + h * (long long)src_per_head;
            const int ns = src_single ? 1 : (P.last_cta((int)h) - P.first_cta((int)h) + 1);
            float m = gather_state(srch, ns, stage, tid);
            named_bar(1, kWorkers);
            if (state_out && h * nt >= x0) {   // this CTA holds the head's first tile: it writes the state
                float4 *dst = reinterpret_cast<float4 *>(state_out + h * (long long)kStateElems);
                const float4 *st4 = reinterpret_cast<const float4 *>(stage);
                for (int e = tid; e < kStateElems / 4; e += kWorkers) dst[e] = st4[e];
            }
            if (!BF16) m = workers_max(m, red, tid);
            const float sc = operand_scale<BF16>(m);
            uint8_t *op0 = sOp + buf * 2 * OPB;
            build_state_operand<BF16, NOPS, true>(stage, sc, 80, BIDIR, op0, op0 + OPB, tid);
            if (tid == 0) s_scale[buf] = sc;
            fence_async_smem();
            named_bar(1, kWorkers);
            if (tid == 0) mbar_arrive(&opready[buf]);
        };
        for (TileCursor t(x0, nt); t.x < x1; t.next()) {
                const long long x = t.x;
            const long long h = t.h;
            const int j = t.j;
            if (h != cur_h) {
                ++hidx;
                cur_h = h;
                if (hidx == 0) build(h, 0);
            }
            // ---- epilogue of tile x
            if (tid == 0) tma_store_wait_read<OST - 1>();
            named_bar(1, kWorkers);
            bool got = live && LA_WAIT(&accfull[a], aph, 0x10u);
            got = __all_sync(0xffffffffu, got);
            live = live && got;
            if (got) {
                tc_fence_after();
                const uint32_t base = tmem + (uint32_t)a * 128u + ((uint32_t)(32 * sub) << 16);
                const float sc = s_scale[hidx & 1];
                float inv = 1.f / sc;
                if (BIDIR) {
                    float t16[16];
                    tmem_ld16(base + 64, t16);
                    tmem_ld_wait(t16);
                    inv = 1.f / (t16[0] + eps * sc);
                }
                float v[64];
                tmem_row64(base, v);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&accempty[a]);
#pragma unroll
                for (int c = 0; c < 64; ++c) v[c] *= inv;
                store_row<BF16>(sO + ob * kTileBytes, row, v);
            }
            fence_async_smem();
            named_bar(1, kWorkers);
            if (tid == 0 && live) {
                tma_store_3d(&tmO, sO + ob * kTileBytes, 0, j * kRows, (int)h);
                tma_store_commit();
            }
            if (++ob == OST) ob = 0;
            a ^= 1;
            if (a == 0) aph ^= 1;
            // ---- the next head's operand, into the other buffer (its last user, the
            //      head before this one, has finished all its UMMAs)
            const bool first_of_head = (x == x0) || (j == 0);
            if (first_of_head && (h + 1) * nt < x1) build(h + 1, (hidx + 1) & 1);
        }
        if (tid == 0) tma_store_wait_all<0>();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ================================================================== bwd_q ==
// Per tile: MMA1 [u | q.z] = f(Q) [S | z] (M=128, N=80), MMA2 g S^T (M=128, N=64,
// B = the state operand read MN-major); the epilogue warps form n, o, g.o and dq
// and write g/n (in place over the dO tile) and w = -(g.o)/n; MMA3 accumulates
// [dS | dz] += f(Q)^T [g/n | w] (M=64, N=80, both MN-major).  The 16 columns of
// w's MN atom live in one zero-filled tile shared by the stages: stage s owns
// columns 16 s .. 16 s + 15 (w in the first, zeros after), and MMA3's
// descriptor points its second atom there (a start 32 s bytes into a 128-byte
// row, as a K step does for K-major operands).  bf16 bidir also keeps
// lo = round(f(q) - hi): MMA1 adds f(Q)_lo S_hi and f'(q) = min(hi + lo, 1).
// Warp roles of bwd_q: 0 TMA, 1 UMMA (MMA1, MMA2), 2..5 feature map, 6..9 dq,
// 10..13 epilogue, 14 UMMA (MMA3).
constexpr int kQXWarps = 4, kQDw0 = kXw0 + kQXWarps, kQDWarps = 4, kQU2 = kEw0 + kEWarps;
constexpr int kQThreads = (kQU2 + 1) * 32;
static_assert(kQDw0 + kQDWarps == kEw0, "bwd_q warp roles");

template <bool BIDIR, bool BF16>
struct BwdQLayout {
    static constexpr bool QLO = BIDIR && BF16;
    static constexpr int NST = BIDIR ? (QLO ? 2 : 4) : 4, OST = 2, OPB = 80 * 128;
    static constexpr int qoff = 0;
    static constexpr int goff = qoff + NST * kTileBytes;
    static constexpr int woff = goff + NST * kTileBytes;
    static constexpr int qloff = woff + (BIDIR ? kTileBytes : 0);   // one w tile shared by the stages
    static constexpr int dqoff = qloff + (QLO ? NST * kTileBytes : 0);
    static constexpr int opoff = dqoff + OST * kTileBytes;
    static constexpr int stageoff = opoff + 2 * OPB;
    static constexpr int zsoff = stageoff + kStateElems * 4;        // [3][64] z of three heads
    static constexpr int iscoff = zsoff + 3 * 64 * 4;                // [3] 1 / operand scale
    static constexpr int rioff = iscoff + 16;                        // [2][128] (g.o, 1/n) per row
    static constexpr int redoff = rioff + 2 * 128 * 8;
    static constexpr int baroff = redoff + 32;
    static constexpr int nbars = 4 * NST + 10;
    static constexpr int misc = baroff + nbars * 8;
    static constexpr int bytes = misc + 32 + 1024;
    static_assert(bytes <= 227 * 1024, "shared memory of one CTA");
    static_assert(kStateElems * 4 <= 2 * OPB, "the operand block stages a [dS | dz] partial");
};

template <bool BIDIR, bool BF16, bool PHI>
__global__ void __launch_bounds__(kQThreads, 1)
bwd_q_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmG,
             const __grid_constant__ CUtensorMap tmDQ, const float *__restrict__ src, int src_per_head,
             int src_single, float *__restrict__ dpart, int T, int BH, int nt, int maxslots, float eps,
             int early_loads) {
    using L = BwdQLayout<BIDIR, BF16>;
    constexpr int NST = L::NST, OPB = L::OPB;
    constexpr bool QLO = L::QLO;
    constexpr int NOPS = BF16 ? 2 : 1;
    constexpr int N3 = BIDIR ? 80 : 64;
    constexpr uint32_t IDESC1 = idesc_f16(128, 80, BF16, false, false);
    constexpr uint32_t IDESC2 = idesc_f16(128, 64, BF16, false, true);
    constexpr uint32_t IDESC3 = idesc_f16(64, N3, BF16, true, true);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *sQ = smem + L::qoff;
    uint8_t *sG = smem + L::goff;
    uint8_t *sW = smem + L::woff;
    uint8_t *sQlo = smem + L::qloff;
    uint8_t *sDQ = smem + L::dqoff;
    uint8_t *sOp = smem + L::opoff;
    float *stage = reinterpret_cast<float *>(smem + L::stageoff);
    float *zs = reinterpret_cast<float *>(smem + L::zsoff);
    float *red = reinterpret_cast<float *>(smem + L::redoff);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::baroff);
    uint64_t *xf = full + NST;
    uint64_t *gnready = xf + NST;
    uint64_t *empty = gnready + NST;
    uint64_t *acc12full = empty + NST;   // [2]
    uint64_t *acc12empty = acc12full + 2;
    uint64_t *accSfull = acc12empty + 2;
    uint64_t *accSfree = accSfull + 1;
    uint64_t *opready = accSfree + 1;
    uint64_t *drain = opready + 1;
    uint64_t *drain2 = drain + 1;
    uint64_t *stfull = drain2 + 1;       // a head's state copied into the staging block ahead of its build
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::misc);
    int *s_abort = reinterpret_cast<int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Partition P{(long long)BH * nt, nt, grid_for((long long)BH * nt)};
    const int cta = blockIdx.x;
    const long long x0 = P.start(cta), x1 = P.start(cta + 1);
    if (x0 >= x1) return;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&xf[s], kQXWarps);
            mbar_init(&gnready[s], kEWarps);
            mbar_init(&empty[s], BIDIR ? 1 + kQDWarps : 1);   // MMA3, and the dq pass that reads f(q)
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc12full[b], 1);
            mbar_init(&acc12empty[b], BIDIR ? kEWarps + kQDWarps : kQDWarps);
        }
        mbar_init(accSfull, 1);
        mbar_init(accSfree, kEWarps);
        mbar_init(opready, 1);
        mbar_init(drain, 1);
        mbar_init(drain2, 1);
        mbar_init(stfull, 1);
        *s_abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch(&tmQ);
        tma_prefetch(&tmG);
        tma_prefetch(&tmDQ);
    }
    if (BIDIR && warp >= kEw0 && warp < kQU2) {   // the w tile: zero except column 16 s of stage s, written per tile
        const int r = threadIdx.x - kEw0 * 32;
        uint8_t *p = sW + r * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4 *>(p + c * 16) = make_uint4(0u, 0u, 0u, 0u);
        fence_async_smem();
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
    // launch it overlapped the previous kernel.  With `early_loads` (the previous
    // kernel is the first kernel of the same call, which writes none of this
    // kernel's inputs) the TMA producer starts streaming inputs right away; every
    // other access to global memory waits for the previous kernel here.
    if (!(early_loads && warp == 0)) grid_dependency_wait();
    if (threadIdx.x == 64) grid_launch_dependents();
    constexpr uint32_t kAccS = 176;    // columns 176..255: the M=64 [dS | dz] accumulator

    if (warp == 0) {
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            long long issued = 0;
            if (src_single) {   // the first head's state, ahead of the tile stream
                mbar_arrive_expect_tx(stfull, kStateElems * 4);
                bulk_load(stage, src + (x0 / nt) * (long long)src_per_head, kStateElems * 4, stfull);
            }
            for (TileCursor t(x0, nt); t.x < x1; t.next()) {
                const int h = t.h, j = t.j;
                if (!LA_WAIT(&empty[s], ph ^ 1, 0x1u)) break;
                mbar_arrive_expect_tx(&full[s], 2 * kTileBytes);
                tma_load_3d(sQ + s * kTileBytes, &tmQ, &full[s], 0, j * kRows, h);
                tma_load_3d(sG + s * kTileBytes, &tmG, &full[s], 0, j * kRows, h);
                ++issued;
                if (++s == NST) { s = 0; ph ^= 1; }
            }
            if (*s_abort) {
                for (long long i = issued - 1; i >= 0 && i >= issued - NST; --i)
                    mbar_wait_slow(smem_u32(&full[i % NST]), (uint32_t)((i / NST) & 1), nullptr, &g_tc_fault, 0x200u);
                if (src_single) mbar_wait_slow(smem_u32(stfull), 0, nullptr, &g_tc_fault, 0x200u);
            }
        }
    } else if (warp == 1) {
        int s = 0, b = 0;
        uint32_t ph = 0, bph = 0, oph = 0;
        long long prev_h = -1;
        bool dead = false;
        for (TileCursor t(x0, nt); t.x < x1 && !dead; t.next()) {
            const long long h = t.h;
            if (h != prev_h) {
                if (!LA_WWAIT(opready, oph, 0x20u)) break;
                oph ^= 1;
                prev_h = h;
            }
            if (!LA_WWAIT(BIDIR ? &xf[s] : &full[s], ph, 0x4u)) break;
            if (!LA_WWAIT(&acc12empty[b], bph ^ 1, 0x2u)) break;
            tc_fence_after();
            const uint32_t d1 = tmem + (uint32_t)b * 256u, d2 = d1 + 96u;
            const uint64_t dq = sdesc_sw128(smem_u32(sQ + s * kTileBytes), 16, 1024);
            const uint64_t dg = sdesc_sw128(smem_u32(sG + s * kTileBytes), 16, 1024);
            const uint64_t dql = sdesc_sw128(smem_u32(sQlo + s * kTileBytes), 16, 1024);
            const uint64_t dok = sdesc_sw128(smem_u32(sOp), 16, 1024);     // state operand read K-major
            const uint64_t dom = sdesc_sw128(smem_u32(sOp), OPB, 1024);    // ... and MN-major
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
                for (int op = 0; op < NOPS; ++op) {
                    if (BIDIR)
                        umma_f16_ss_warp(d1, desc_at(dq, kk * 32), desc_at(dok, op * OPB + kk * 32), IDESC1,
                                         (kk | op) ? 1u : 0u);
                    umma_f16_ss_warp(d2, desc_at(dg, kk * 32), desc_at(dom, op * OPB + kk * 2048), IDESC2,
                                     (kk | op) ? 1u : 0u);
                }
                if (QLO) umma_f16_ss_warp(d1, desc_at(dql, kk * 32), desc_at(dok, kk * 32), IDESC1, 1u);
            }
            umma_commit_warp(&acc12full[b]);
            b ^= 1;
            if (b == 0) bph ^= 1;
            if (++s == NST) { s = 0; ph ^= 1; }
        }
        umma_commit_warp(drain);
        mbar_wait_slow(smem_u32(drain), 0, nullptr, &g_tc_fault, 0x400u);
        __syncwarp();
    } else if (warp == kQU2) {
        // Second UMMA issuer: MMA3 of every tile, in tile order, once the epilogue
        // warps have written its g/n and w.  A thread's issue rate, not the tensor
        // pipe, bounds these small-N UMMAs while the other warps of its scheduler
        // are busy, so the two UMMA groups of a tile come from two schedulers.
        int s = 0;
        uint32_t ph = 0;
        long long seg = 0;                     // segments started (accS free parity)
        for (TileCursor t(x0, nt); t.x < x1; t.next()) {
            const bool seg_start = (t.x == x0) || t.j == 0;
            const bool seg_end = (t.x + 1 == x1) || t.last_of_head();
            if (seg_start) {
                if (!LA_WWAIT(accSfree, (uint32_t)((seg & 1) ^ 1), 0x40u)) break;
                ++seg;
            }
            if (!LA_WWAIT(&gnready[s], ph, 0x80u)) break;
            tc_fence_after();
            const uint32_t aG = smem_u32(sG + s * kTileBytes);
            // the second MN atom of [g/n | w] starts at column 16 s of the shared w tile
            const uint32_t lbo = BIDIR ? smem_u32(sW) + 32u * (uint32_t)s - aG : (uint32_t)kTileBytes;
            const uint64_t dq = sdesc_sw128(smem_u32(sQ + s * kTileBytes), kTileBytes, 1024);
            const uint64_t dg = sdesc_sw128(aG, lbo, 1024);
#pragma unroll
            for (int kk = 0; kk < kRows / 16; ++kk)
                umma_f16_ss_warp(tmem + kAccS, desc_at(dq, kk * 2048), desc_at(dg, kk * 2048), IDESC3,
                                 (seg_start && kk == 0) ? 0u : 1u);
            umma_commit_warp(&empty[s]);
            if (seg_end) umma_commit_warp(accSfull);
            if (++s == NST) { s = 0; ph ^= 1; }
        }
        umma_commit_warp(drain2);
        mbar_wait_slow(smem_u32(drain2), 0, nullptr, &g_tc_fault, 0x400u);
        __syncwarp();
    } else if (warp < kQDw0) {
        // Feature-map warps (bidir): f(q) in place, one row per thread.
        if (BIDIR) {
            const int r = threadIdx.x - kXw0 * 32;
            int s = 0;
            uint32_t ph = 0;
            for (TileCursor t(x0, nt); t.x < x1; t.next()) {
                const bool got = __all_sync(0xffffffffu, LA_WAIT(&full[s], ph, 0x8u));
                if (!got) break;
                phi_row_batched<BF16, QLO, PHI>(sQ + s * kTileBytes, sQlo + s * kTileBytes, r);
                fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&xf[s]);
                if (++s == NST) { s = 0; ph ^= 1; }
            }
        }
    } else if (warp < kEw0) {
        // dq warps: dq = ((g S^T - (g.o) z) / n) f'(q) from TMEM (g S^T) and the
        // epilogue warps' per-row (g.o, 1/n); warp w reads TMEM lane quadrant w % 4.
        // Named barrier 3 (these 128 threads) is reached by all whatever the waits return.
        const int sub = warp & 3;
        const int row = sub * 32 + lane;
        const bool storer = threadIdx.x == kQDw0 * 32;
        const float2 *rinfo = reinterpret_cast<const float2 *>(smem + L::rioff);
        const float *isc3 = reinterpret_cast<const float *>(smem + L::iscoff);
        bool live = true;
        int s = 0, b = 0, hidx = -1;
        uint32_t ph = 0, bph = 0;
        long long prev_h = -1;
        for (TileCursor t(x0, nt); t.x < x1; t.next()) {
            if (t.h != prev_h) {
                ++hidx;
                prev_h = t.h;
            }
            const int zb = hidx % 3;
            if (storer) tma_store_wait_read<L::OST - 1>();   // staging buffer x % OST is free
            named_bar(3, kQDWarps * 32);
            uint8_t *sDQx = sDQ + (int)(t.x & (L::OST - 1)) * kTileBytes;
            bool got = live && LA_WAIT(&gnready[s], ph, 0x80u);
            got = got && LA_WAIT(&acc12full[b], bph, 0x10u);
            got = __all_sync(0xffffffffu, got);
            live = live && got;
            if (got) {
                tc_fence_after();
                float gdot = 0.f, inv = 1.f;
                if (BIDIR) {
                    const float2 ri = rinfo[b * 128 + row];
                    gdot = ri.x;
                    inv = ri.y;
                }
                const float *zsb = zs + zb * 64;
                const float isc = isc3[zb];
                const uint32_t d2 = tmem + (uint32_t)b * 256u + 96u + ((uint32_t)(32 * sub) << 16);
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    float a0[16], a1[16];
                    tmem_ld16(d2 + 32 * hf, a0);
                    tmem_ld16(d2 + 32 * hf + 16, a1);
                    tmem_ld_wait(a0, a1);
                    if (hf == 1) {   // every TMEM read of this accumulator pair is complete
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&acc12empty[b]);
                    }
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        const int c16 = 2 * hf + cc;
                        float dq[16];
                        if (BIDIR) {
                            float qf[16];
                            load_chunk16<BF16>(sQ + s * kTileBytes, row, c16, qf);
                            if (QLO) {
                                float ql[16];
                                load_chunk16<BF16>(sQlo + s * kTileBytes, row, c16, ql);
#pragma unroll
                                for (int i = 0; i < 16; ++i) qf[i] += ql[i];
                            }
                            const float4 *z4 = reinterpret_cast<const float4 *>(zsb + 16 * c16);
#pragma unroll
                            for (int i4 = 0; i4 < 4; ++i4) {
                                const float4 zz = z4[i4];
                                const float zv[4] = {zz.x, zz.y, zz.z, zz.w};
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const int i = 4 * i4 + e;
                                    const float acc = cc ? a1[i] : a0[i];
                                    dq[i] = (acc - gdot * zv[e]) * inv * (PHI ? fminf(qf[i], 1.f) : 1.f);
                                }
                            }
                        } else {
#pragma unroll
                            for (int i = 0; i < 16; ++i) dq[i] = (cc ? a1[i] : a0[i]) * isc;
                        }
                        store_chunk16<BF16>(sDQx, row, c16, dq);
                    }
                }
                if (BIDIR) {   // f(q) of this stage is no longer read
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&empty[s]);
                }
            }
            fence_async_smem();
            named_bar(3, kQDWarps * 32);
            if (storer && live) {
                tma_store_3d(&tmDQ, sDQx, 0, t.j * kRows, t.h);
                tma_store_commit();
            }
            if (++s == NST) { s = 0; ph ^= 1; }
            b ^= 1;
            if (b == 0) bph ^= 1;
        }
        if (storer) tma_store_wait_all<0>();
    } else if (warp < kQU2) {
        // Epilogue warps (every named barrier is reached by all 128 whatever the waits return).
        const int tid = threadIdx.x - kEw0 * 32;
        const int sub = warp & 3;
        const int row = sub * 32 + lane;
        int s = 0, b = 0;
        uint32_t ph = 0, bph = 0, sfull_ph = 0;
        long long cur_h = -1;
        bool live = true;
        float cur_sc = 1.f, cur_scn = 1.f;

        float *isc3 = reinterpret_cast<float *>(smem + L::iscoff);
        int hidx = -1;
        int copies = src_single ? 1 : 0;   // bulk copies of a head's state into the staging block so far
        int landed = 0;                    // ... seen complete
        auto build = [&](long long h, int zb) {
            const float *srch = src + h * (long long)src_per_head;
            const int ns = src_single ? 1 : (P.last_cta((int)h) - P.first_cta((int)h) + 1);
            float m;
            if (src_single) {   // copied ahead: the first head by the TMA thread, the next ones below
                if (LA_WAIT(stfull, (uint32_t)(hidx & 1), 0x800u))
                    ++landed;
                else
                    live = false;
                m = stage_absmax(stage, tid);
            } else {
                m = gather_state(srch, ns, stage, tid);
            }
            named_bar(1, kWorkers);
            if (!BF16) m = workers_max(m, red, tid);
            const float sc = operand_scale<BF16>(m);
            const float zsum = BIDIR ? warp_abs_z_sum(stage, tid & 31) : 0.f;
            float scn = 1.f;
            if (BIDIR && zsum > 0.f && isfinite(zsum)) {
                int e;
                frexpf(zsum, &e);
                e = e < -100 ? -100 : (e > 100 ? 100 : e);
                scn = ldexpf(1.f, e - 1);
            }
            build_state_operand<BF16, NOPS, true>(stage, sc, 80, BIDIR, sOp, sOp + OPB, tid);
            if (tid < 64) zs[zb * 64 + tid] = stage[tid * 65 + 64] * sc;
            if (tid == 0) isc3[zb] = 1.f / sc;
            fence_async_smem();
            named_bar(1, kWorkers);
            cur_sc = sc;
            cur_scn = scn;
            if (tid == 0) mbar_arrive(opready);
            // the staging block is read: the next head of this CTA's range comes in behind
            // the current head's tiles instead of at the switch
            if (src_single && tid == 0 && live && (h + 1) * nt < x1) {
                mbar_arrive_expect_tx(stfull, kStateElems * 4);
                bulk_load(stage, src + (h + 1) * (long long)src_per_head, kStateElems * 4, stfull);
                ++copies;
            }
        };

        // [dS | dz] partial of the segment of head hs that just ended.  It is staged in the
        // state operand block: its last readers, MMA1 and MMA2 of the segment's last tile,
        // completed before acc12full, which these warps waited for in that tile's epilogue,
        // and the next head's operand is built only after the copy (the staging block holds
        // that head's state, copied in ahead).
        float *accst = reinterpret_cast<float *>(sOp);
        auto read_accS = [&](int hs, float scn) {
            bool got = live && LA_WAIT(accSfull, sfull_ph, 0x100u);
            got = __all_sync(0xffffffffu, got);
            live = live && got;
            sfull_ph ^= 1;
            if (got) {
                tc_fence_after();
                const uint32_t base = tmem + kAccS + ((uint32_t)(32 * sub) << 16);
                float v[64];
                tmem_row64(base, v);
                float zz = 0.f;
                if (BIDIR) {
                    float t16[16];
                    tmem_ld16(base + 64, t16);
                    tmem_ld_wait(t16);
                    zz = t16[0];
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(accSfree);
                if (lane < 16) {   // row i of [dS | dz] into the operand block (stride 65: no bank conflicts)
                    const int i = 16 * sub + lane;
                    const float is = 1.f / scn;
#pragma unroll
                    for (int c = 0; c < 64; ++c) accst[i * 65 + c] = v[c] * is;
                    accst[i * 65 + 64] = zz * is;
                }
            }
            named_bar(1, kWorkers);
            if (live) {            // the slot as one contiguous, coalesced 16.6 KB copy
                float4 *dst = reinterpret_cast<float4 *>(dpart + ((long long)hs * maxslots + (cta - P.first_cta(hs))) *
                                                                     kStateElems);
                const float4 *src4 = reinterpret_cast<const float4 *>(accst);
                for (int e = tid; e < kStateElems / 4; e += kWorkers) dst[e] = src4[e];
            }
            named_bar(1, kWorkers);   // the operand block is free for the next head's operand
        };

        float2 *rinfo = reinterpret_cast<float2 *>(smem + L::rioff);
        for (TileCursor t(x0, nt); t.x < x1; t.next()) {
            const long long x = t.x;
            const long long h = t.h;
            if (h != cur_h) {
                ++hidx;
                build(h, hidx % 3);
                cur_h = h;
            }
            // ---- first half of the epilogue of tile x (stage s, accumulator pair b):
            //      n, g.o, g/n and w; the feature-map warps form dq from g S^T
            bool got = live && LA_WAIT(&acc12full[b], bph, 0x10u);
            got = __all_sync(0xffffffffu, got);
            live = live && got;
            if (got && BIDIR) {
                tc_fence_after();
                const uint32_t d1 = tmem + (uint32_t)b * 256u + ((uint32_t)(32 * sub) << 16);
                float u[64], t16[16];   // u = f(q) S, t16[0] = f(q).z (one wait for all five loads)
                tmem_ld16(d1 + 64, t16);
                tmem_row64(d1, u);
                reg_keep(t16);   // loaded before the wait inside tmem_row64
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc12empty[b]);
                const float inv = 1.f / (t16[0] + eps * cur_sc);
                const float gsc = inv * cur_sc * cur_scn;
                uint8_t *tg = sG + s * kTileBytes;
                float gdot = 0.f;
#pragma unroll
                for (int c16 = 0; c16 < 4; ++c16) {
                    float g[16];
                    load_chunk16<BF16>(tg, row, c16, g);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        gdot = fmaf(g[i], u[16 * c16 + i], gdot);
                        g[i] *= gsc;
                    }
                    store_chunk16<BF16>(tg, row, c16, g);   // g/n (scaled) over dO: MMA2 is done with it
                }
                gdot *= inv;
                rinfo[b * 128 + row] = make_float2(gdot, inv);
                const float w = -gdot * gsc;
                // columns 16 s .. 16 s + 7 of the w tile: (w, 0, ..., 0)
                const uint32_t wbits = BF16 ? (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(w))
                                            : (uint32_t)__half_as_ushort(__float2half_rn(w));
                *reinterpret_cast<uint4 *>(sW + sw128_offset(row, 16 * s)) = make_uint4(wbits, 0u, 0u, 0u);
                fence_async_smem();
            }
            __syncwarp();
            if (lane == 0 && got) mbar_arrive(&gnready[s]);
            const bool seg_end = (x + 1 == x1) || t.last_of_head();
            if (seg_end) read_accS((int)h, cur_scn);
            if (++s == NST) { s = 0; ph ^= 1; }
            b ^= 1;
            if (b == 0) bph ^= 1;
        }
        // a copy issued after the last wait that gave up lands before the CTA exits (only the
        // last one can be unseen: no copy is issued once a wait has failed)
        if (tid == 0 && copies > landed)
            mbar_wait_slow(smem_u32(stfull), (uint32_t)((copies - 1) & 1), nullptr, &g_tc_fault, 0x800u);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ================================================================= bwd_kv ==
// Per tile: MMA_a  v dS^T (A = V tile, B = dS operand K-major),
//           MMA_b  f(K) dS (A = f(K) tile, B = dS operand read MN-major);
// dk = (v dS^T + dz) f'(k), dv = f(k) dS.  The dS operand rows are dS's rows.
struct BwdKvLayout {
    static constexpr int NST = 4, OST = 1, OPB = 64 * 128;
    static constexpr int koff = 0;
    static constexpr int voff = koff + NST * kTileBytes;
    static constexpr int dkoff = voff + NST * kTileBytes;
    static constexpr int dvoff = dkoff + OST * kTileBytes;
    static constexpr int opoff = dvoff + OST * kTileBytes;
    static constexpr int stageoff = opoff + 2 * OPB;
    static constexpr int dzoff = stageoff + kStateElems * 4;
    static constexpr int redoff = dzoff + 64 * 4;
    static constexpr int baroff = redoff + 32;
    static constexpr int nbars = 3 * NST + 4 + 2;
    static constexpr int misc = baroff + nbars * 8;
    static constexpr int bytes = misc + 32 + 1024;
    static_assert(bytes <= 227 * 1024, "shared memory of one CTA");
};

template <bool BIDIR, bool BF16, bool PHI>
__global__ void __launch_bounds__(kThreads, 1)
bwd_kv_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
              const __grid_constant__ CUtensorMap tmDK, const __grid_constant__ CUtensorMap tmDV,
              const float *__restrict__ src, int src_per_head, int src_single, int T, int BH, int nt,
              int early_loads) {
    using L = BwdKvLayout;
    constexpr int NST = L::NST, OPB = L::OPB;
    constexpr int NOPS = BF16 ? 2 : 1;
    constexpr uint32_t IDESC_A = idesc_f16(128, 64, BF16, false, false);
    constexpr uint32_t IDESC_B = idesc_f16(128, 64, BF16, false, true);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *sK = smem + L::koff;
    uint8_t *sV = smem + L::voff;
    uint8_t *sDK = smem + L::dkoff;
    uint8_t *sDV = smem + L::dvoff;
    uint8_t *sOp = smem + L::opoff;
    float *stage = reinterpret_cast<float *>(smem + L::stageoff);
    float *dz = reinterpret_cast<float *>(smem + L::dzoff);
    float *red = reinterpret_cast<float *>(smem + L::redoff);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::baroff);
    uint64_t *xf = full + NST;
    uint64_t *empty = xf + NST;
    uint64_t *accfull = empty + NST;
    uint64_t *accempty = accfull + 2;
    uint64_t *opready = accempty + 2;
    uint64_t *drain = opready + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::misc);
    int *s_abort = reinterpret_cast<int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Partition P{(long long)BH * nt, nt, grid_for((long long)BH * nt)};
    const int cta = blockIdx.x;
    const long long x0 = P.start(cta), x1 = P.start(cta + 1);
    if (x0 >= x1) return;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&xf[s], kXWarps);
            mbar_init(&empty[s], BIDIR ? 1 + kEWarps : 1);   // UMMA commit (+ the epilogue warps read f(k))
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&accfull[b], 1);
            mbar_init(&accempty[b], kEWarps);
        }
        mbar_init(opready, 1);
        mbar_init(drain, 1);
        *s_abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch(&tmK);
        tma_prefetch(&tmV);
        tma_prefetch(&tmDK);
        tma_prefetch(&tmDV);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // Everything above touched only shared memory and TMEM: with a programmatic
    // launch it overlapped the previous kernel.  With `early_loads` (the previous
    // kernel is the first kernel of the same call, which writes none of this
    // kernel's inputs) the TMA producer starts streaming inputs right away; every
    // other access to global memory waits for the previous kernel here.
    if (!(early_loads && warp == 0)) grid_dependency_wait();
    if (threadIdx.x == 64) grid_launch_dependents();

    if (warp == 0) {
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            long long issued = 0;
            for (TileCursor t(x0, nt); t.x < x1; t.next()) {
                const int h = t.h, j = t.j;
                if (!LA_WAIT(&empty[s], ph ^ 1, 0x1u)) break;
                mbar_arrive_expect_tx(&full[s], 2 * kTileBytes);
                tma_load_3d(sK + s * kTileBytes, &tmK, &full[s], 0, j * kRows, h);
                tma_load_3d(sV + s * kTileBytes, &tmV, &full[s], 0, j * kRows, h);
                ++issued;
                if (++s == NST) { s = 0; ph ^= 1; }
            }
            if (*s_abort) {
                for (long long i = issued - 1; i >= 0 && i >= issued - NST; --i)
                    mbar_wait_slow(smem_u32(&full[i % NST]), (uint32_t)((i / NST) & 1), nullptr, &g_tc_fault, 0x200u);
            }
        }
    } else if (warp == 1) {
        int s = 0, b = 0;
        uint32_t ph = 0, bph = 0, oph = 0;
        long long prev_h = -1;
        for (TileCursor t(x0, nt); t.x < x1; t.next()) {
            const long long h = t.h;
            if (h != prev_h) {
                if (!LA_WWAIT(opready, oph, 0x20u)) break;
                oph ^= 1;
                prev_h = h;
            }
            if (!LA_WWAIT(BIDIR ? &xf[s] : &full[s], ph, 0x4u)) break;
            if (!LA_WWAIT(&accempty[b], bph ^ 1, 0x2u)) break;
            tc_fence_after();
            const uint32_t da = tmem + (uint32_t)b * 128u, db = da + 64u;
            const uint64_t dk = sdesc_sw128(smem_u32(sK + s * kTileBytes), 16, 1024);
            const uint64_t dv = sdesc_sw128(smem_u32(sV + s * kTileBytes), 16, 1024);
            const uint64_t dok = sdesc_sw128(smem_u32(sOp), 16, 1024);
            const uint64_t dom = sdesc_sw128(smem_u32(sOp), OPB, 1024);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
                for (int op = 0; op < NOPS; ++op) {
                    umma_f16_ss_warp(da, desc_at(dv, kk * 32), desc_at(dok, op * OPB + kk * 32), IDESC_A,
                                     (kk | op) ? 1u : 0u);
                    umma_f16_ss_warp(db, desc_at(dk, kk * 32), desc_at(dom, op * OPB + kk * 2048), IDESC_B,
                                     (kk | op) ? 1u : 0u);
                }
            }
            umma_commit_warp(&empty[s]);
            umma_commit_warp(&accfull[b]);
            b ^= 1;
            if (b == 0) bph ^= 1;
            if (++s == NST) { s = 0; ph ^= 1; }
        }
        umma_commit_warp(drain);
        mbar_wait_slow(smem_u32(drain), 0, nullptr, &g_tc_fault, 0x400u);
        __syncwarp();
    } else if (warp < kEw0) {
        if (BIDIR) {
            const int xi = threadIdx.x - kXw0 * 32;
            int s = 0;
            uint32_t ph = 0;
            for (TileCursor t(x0, nt); t.x < x1; t.next()) {
                const bool got = __all_sync(0xffffffffu, LA_WAIT(&full[s], ph, 0x8u));
                if (!got) break;
                phi_half_row<BF16, PHI>(sK + s * kTileBytes, xi, false);
                fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&xf[s]);
                if (++s == NST) { s = 0; ph ^= 1; }
            }
        }
    } else {
        const int tid = threadIdx.x - kEw0 * 32;
        const int sub = warp & 3;
        const int row = sub * 32 + lane;
        int s = 0, b = 0;
        uint32_t bph = 0;
        long long cur_h = -1;
        bool live = true;
        float cur_isd = 1.f;
        for (TileCursor t(x0, nt); t.x < x1; t.next()) {
            const long long h = t.h;
            const int j = t.j;
            if (h != cur_h) {
                // the previous head's UMMAs are complete (its last epilogue waited on them)
                const float *srch = src + h * (long long)src_per_head;
                const int ns = src_single ? 1 : (P.last_cta((int)h) - P.first_cta((int)h) + 1);
                float m = gather_state(srch, ns, stage, tid);
                named_bar(1, kWorkers);
                if (!BF16) m = workers_max(m, red, tid);
                const float sd = operand_scale<BF16>(m);
                build_state_operand<BF16, NOPS, false>(stage, sd, 64, false, sOp, sOp + OPB, tid);
                if (tid < 64) dz[tid] = BIDIR ? stage[tid * 65 + 64] : 0.f;
                fence_async_smem();
                named_bar(1, kWorkers);
                cur_isd = 1.f / sd;
                if (tid == 0) mbar_arrive(opready);
                cur_h = h;
            }
            // ---- epilogue of tile x
            if (tid == 0) tma_store_wait_read<0>();
            named_bar(1, kWorkers);
            bool got = live && LA_WAIT(&accfull[b], bph, 0x10u);
            got = __all_sync(0xffffffffu, got);
            live = live && got;
            if (got) {
                tc_fence_after();
                const uint32_t da = tmem + (uint32_t)b * 128u + ((uint32_t)(32 * sub) << 16), db = da + 64u;
#pragma unroll
                for (int c16 = 0; c16 < 4; ++c16) {
                    float aa[16], bb[16], out[16];
                    tmem_ld16(da + 16 * c16, aa);
                    tmem_ld16(db + 16 * c16, bb);
                    if (BIDIR) {
                        float kf[16];
                        load_chunk16<BF16>(sK + s * kTileBytes, row, c16, kf);
                        tmem_ld_wait(aa, bb);
#pragma unroll
                        for (int i = 0; i < 16; ++i) out[i] = fmaf(aa[i], cur_isd, dz[16 * c16 + i]) * (PHI ? fminf(kf[i], 1.f) : 1.f);
                    } else {
                        tmem_ld_wait(aa, bb);
#pragma unroll
                        for (int i = 0; i < 16; ++i) out[i] = aa[i] * cur_isd;
                    }
                    store_chunk16<BF16>(sDK, row, c16, out);
#pragma unroll
                    for (int i = 0; i < 16; ++i) out[i] = bb[i] * cur_isd;
                    store_chunk16<BF16>(sDV, row, c16, out);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&accempty[b]);
                    if (BIDIR) mbar_arrive(&empty[s]);   // f(k) read: the stage may be reloaded
                }
            }
            fence_async_smem();
            named_bar(1, kWorkers);
            if (tid == 0 && live) {
                tma_store_3d(&tmDK, sDK, 0, j * kRows, (int)h);
                tma_store_3d(&tmDV, sDV, 0, j * kRows, (int)h);
                tma_store_commit();
            }
            if (++s == NST) s = 0;
            b ^= 1;
            if (b == 0) bph ^= 1;
        }
        if (tid == 0) tma_store_wait_all<0>();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ================================================================ combine ==
// state[h] = sum over the head's partial slots 0 .. ns(h) - 1 in slot order (the
// order every consumer's gather uses, so the sum is the same bits).
__global__ void __launch_bounds__(256)
combine_partials_kernel(const float *__restrict__ part, float *__restrict__ out, int BH, int nt, int maxslots) {
    const Partition P{(long long)BH * nt, nt, grid_for((long long)BH * nt)};
    const int h = blockIdx.x;
    const int ns = P.last_cta(h) - P.first_cta(h) + 1;
    const float4 *src = reinterpret_cast<const float4 *>(part + (long long)h * maxslots * kStateElems);
    float4 *dst = reinterpret_cast<float4 *>(out + (long long)h * kStateElems);
    for (int e = threadIdx.x; e < kStateElems / 4; e += blockDim.x) {
        float4 a = src[e];
        for (int sl = 1; sl < ns; ++sl) {
            const float4 b = src[(long long)sl * (kStateElems / 4) + e];
            a.x += b.x;
            a.y += b.y;
            a.z += b.z;
            a.w += b.w;
        }
        dst[e] = a;
    }
}

// =================================================================== host ==

using EncodeFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                              const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeFn encode_fn() {
    static EncodeFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeFn>(p);
    });
    return fn;
}

}  // namespace

// [BH, T, D] 16-bit tensor, boxes of `box_rows` rows x 64 columns, 128-byte swizzle, zero fill.
la_status make_tensor_map(CUtensorMap *m, const void *ptr, const Shape &s, bool bf16, int box_rows) {
    EncodeFn enc = encode_fn();
    if (!enc) {
        set_error("cuTensorMapEncodeTiled is unavailable from the driver");
        return LA_ERR_CUDA;
    }
    const cuuint64_t dims[3] = {(cuuint64_t)s.D, (cuuint64_t)s.T, (cuuint64_t)s.BH()};
    const cuuint64_t strides[2] = {(cuuint64_t)s.D * 2, (cuuint64_t)s.T * s.D * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    CUresult r = enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                     const_cast<void *>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        set_error("cuTensorMapEncodeTiled failed (%d)", (int)r);
        return LA_ERR_CUDA;
    }
    return LA_OK;
}

la_status retention_map(CUtensorMap *m, const void *ptr, const Shape &s, bool bf16) {
    return make_tensor_map(m, ptr, s, bf16, 64);
}

// [BH, T, 64] fp32 tensor, boxes of 64 rows x 32 columns (128 bytes), 128-byte swizzle.
la_status retention_map_f32(CUtensorMap *m, void *ptr, const Shape &s) {
    EncodeFn enc = encode_fn();
    if (!enc) {
        set_error("cuTensorMapEncodeTiled is unavailable from the driver");
        return LA_ERR_CUDA;
    }
    const cuuint64_t dims[3] = {(cuuint64_t)s.D, (cuuint64_t)s.T, (cuuint64_t)s.BH()};
    const cuuint64_t strides[2] = {(cuuint64_t)s.D * 4, (cuuint64_t)s.T * s.D * 4};
    const cuuint32_t box[3] = {32, 64, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, ptr, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        set_error("cuTensorMapEncodeTiled failed (%d)", (int)r);
        return LA_ERR_CUDA;
    }
    return LA_OK;
}

namespace {

static la_status tensor_map(CUtensorMap *m, const void *ptr, const Shape &s, bool bf16) {
    return make_tensor_map(m, ptr, s, bf16, kRows);
}

static size_t partial_bytes(const Shape &s) {
    size_t b = (size_t)s.BH() * (size_t)max_slots((int)s.BH()) * kStateElems * sizeof(float);
    return (b + 255) & ~(size_t)255;
}

// Launch names (string literals: the profiler keeps the pointers): "<base>" for elu+1 with
// the norm term, "<base>_norm" for the norm term on features the caller computed,
// "<base>_simple" for neither.
#define LA_KNAME(base) (!BIDIR ? base "_simple" : (PHI ? base : base "_norm"))

template <bool BIDIR, bool BF16, bool PHI>
static la_status launch_reduce(const CUtensorMap &mk, const CUtensorMap &mv, float *part, const Shape &s, int nt,
                               cudaStream_t st) {
    return launch_pdl(LA_KNAME("tc_state_reduce"), state_reduce_kernel<BIDIR, BF16, PHI>,
                  dim3(grid_for((long long)s.BH() * nt)), dim3(kThreads), (size_t)ReduceLayout<BIDIR, BF16>::bytes, st, mk, mv, part, s.T, (int)s.BH(), nt,
                  max_slots((int)s.BH()));
}

template <bool BIDIR, bool BF16, bool PHI>
static la_status fwd_t(const void *q, const void *k, const void *v, void *o, float *state, const Shape &s,
                       float eps, void *ws, cudaStream_t st) {
    CUtensorMap mq, mk, mv, mo;
    LA_TRY(tensor_map(&mq, q, s, BF16));
    LA_TRY(tensor_map(&mk, k, s, BF16));
    LA_TRY(tensor_map(&mv, v, s, BF16));
    LA_TRY(tensor_map(&mo, o, s, BF16));
    const int nt = (s.T + kRows - 1) / kRows;
    const int ms = max_slots((int)s.BH());
    float *part = (float *)ws;
    LA_TRY((launch_reduce<BIDIR, BF16, PHI>(mk, mv, part, s, nt, st)));
    return launch_pdl(LA_KNAME("tc_output"), output_kernel<BIDIR, BF16, PHI>, dim3(grid_for((long long)s.BH() * nt)), dim3(kThreads),
                  (size_t)OutputLayout::bytes, st, mq, mo, (const float *)part, ms * kStateElems, 0, state, s.T, (int)s.BH(), nt,
                  eps, 1);
}

template <bool BIDIR, bool BF16, bool PHI>
static la_status bwd_t(const void *q, const void *k, const void *v, const void *g, const float *state, void *dq,
                       void *dk, void *dv, const Shape &s, float eps, void *ws, cudaStream_t st) {
    CUtensorMap mq, mk, mv, mg, mdq, mdk, mdv;
    LA_TRY(tensor_map(&mq, q, s, BF16));
    LA_TRY(tensor_map(&mk, k, s, BF16));
    LA_TRY(tensor_map(&mv, v, s, BF16));
    LA_TRY(tensor_map(&mg, g, s, BF16));
    LA_TRY(tensor_map(&mdq, dq, s, BF16));
    LA_TRY(tensor_map(&mdk, dk, s, BF16));
    LA_TRY(tensor_map(&mdv, dv, s, BF16));
    const int nt = (s.T + kRows - 1) / kRows;
    const int ms = max_slots((int)s.BH());
    float *dpart = (float *)ws;
    float *spart = (float *)((char *)ws + partial_bytes(s));
    const float *src = state;
    int per_head = kStateElems, single = 1;
    if (!state) {
        LA_TRY((launch_reduce<BIDIR, BF16, PHI>(mk, mv, spart, s, nt, st)));
        src = spart;
        per_head = ms * kStateElems;
        single = 0;
    }
    LA_TRY(launch_pdl(LA_KNAME("tc_bwd_q"), bwd_q_kernel<BIDIR, BF16, PHI>, dim3(grid_for((long long)s.BH() * nt)), dim3(kQThreads),
                  (size_t)BwdQLayout<BIDIR, BF16>::bytes, st, mq, mg, mdq, src, per_head, single, dpart, s.T, (int)s.BH(),
                  nt, ms, eps, state ? 0 : 1));
    return launch_pdl(LA_KNAME("tc_bwd_kv"), bwd_kv_kernel<BIDIR, BF16, PHI>, dim3(grid_for((long long)s.BH() * nt)), dim3(kThreads),
                  (size_t)BwdKvLayout::bytes, st, mk, mv, mdk, mdv, (const float *)dpart, ms * kStateElems, 0, s.T,
                  (int)s.BH(), nt, 1);
}

// The state form in separate stages, for a sequence split along T (see the
// sequence-parallel entry points): the caller sums the stages' states across
// the shards between them.
template <bool BIDIR, bool BF16, bool PHI>
static la_status stage_t(Stage stage, const void *x, const void *y, const float *sin, float *sout, void *out1,
                         void *out2, const Shape &s, float eps, void *ws, cudaStream_t st) {
    const int nt = (s.T + kRows - 1) / kRows;
    const int ms = max_slots((int)s.BH());
    float *part = (float *)ws;
    switch (stage) {
    case Stage::Reduce: {   // x = k, y = v -> sout = [S | z]
        CUtensorMap mk, mv;
        LA_TRY(tensor_map(&mk, x, s, BF16));
        LA_TRY(tensor_map(&mv, y, s, BF16));
        LA_TRY((launch_reduce<BIDIR, BF16, PHI>(mk, mv, part, s, nt, st)));
        return launch("tc_combine", combine_partials_kernel, dim3((unsigned)s.BH()), dim3(256), 0, st,
                      (const float *)part, sout, (int)s.BH(), nt, ms);
    }
    case Stage::Apply: {    // x = q, sin = [S | z] -> out1 = o
        CUtensorMap mq, mo;
        LA_TRY(tensor_map(&mq, x, s, BF16));
        LA_TRY(tensor_map(&mo, out1, s, BF16));
        return launch_pdl(LA_KNAME("tc_output"), output_kernel<BIDIR, BF16, PHI>,
                          dim3(grid_for((long long)s.BH() * nt)), dim3(kThreads), (size_t)OutputLayout::bytes, st, mq,
                          mo, sin, kStateElems, 1, (float *)nullptr, s.T, (int)s.BH(), nt, eps, 0);
    }
    case Stage::BwdQ: {     // x = q, y = dO, sin = [S | z] -> out1 = dq, sout = [dS | dz]
        CUtensorMap mq, mg, mdq;
        LA_TRY(tensor_map(&mq, x, s, BF16));
        LA_TRY(tensor_map(&mg, y, s, BF16));
        LA_TRY(tensor_map(&mdq, out1, s, BF16));
        LA_TRY(launch_pdl(LA_KNAME("tc_bwd_q"), bwd_q_kernel<BIDIR, BF16, PHI>,
                          dim3(grid_for((long long)s.BH() * nt)), dim3(kQThreads), (size_t)BwdQLayout<BIDIR, BF16>::bytes,
                          st, mq, mg, mdq, sin, kStateElems, 1, part, s.T, (int)s.BH(), nt, ms, eps, 0));
        return launch("tc_combine", combine_partials_kernel, dim3((unsigned)s.BH()), dim3(256), 0, st,
                      (const float *)part, sout, (int)s.BH(), nt, ms);
    }
    default: {              // x = k, y = v, sin = [dS | dz] -> out1 = dk, out2 = dv
        CUtensorMap mk, mv, mdk, mdv;
        LA_TRY(tensor_map(&mk, x, s, BF16));
        LA_TRY(tensor_map(&mv, y, s, BF16));
        LA_TRY(tensor_map(&mdk, out1, s, BF16));
        LA_TRY(tensor_map(&mdv, out2, s, BF16));
        return launch_pdl(LA_KNAME("tc_bwd_kv"), bwd_kv_kernel<BIDIR, BF16, PHI>,
                          dim3(grid_for((long long)s.BH() * nt)), dim3(kThreads), (size_t)BwdKvLayout::bytes, st, mk,
                          mv, mdk, mdv, sin, kStateElems, 1, s.T, (int)s.BH(), nt, 0);
    }
    }
}

}  // namespace

size_t state_workspace_size(la_op op, const Shape &s) {
    switch (op) {
    case LA_OP_BIDIR_FWD:
    case LA_OP_SIMPLE_FWD: return partial_bytes(s);
    case LA_OP_BIDIR_BWD:
    case LA_OP_SIMPLE_BWD: return 2 * partial_bytes(s);
    case LA_OP_STATE_REDUCE:
    case LA_OP_STATE_BWD_Q: return partial_bytes(s);
    default: return 0;
    }
}

la_status state_stage(Stage stage, la_feature f, const void *x, const void *y, const float *sin, float *sout,
                      void *out1, void *out2, const Shape &s, la_dtype dt, float eps, void *ws, cudaStream_t st) {
    const bool bf = dt == LA_BF16;
    if (f == LA_FEATURE_ELU1)
        return bf ? stage_t<true, true, true>(stage, x, y, sin, sout, out1, out2, s, eps, ws, st)
                  : stage_t<true, false, true>(stage, x, y, sin, sout, out1, out2, s, eps, ws, st);
    if (f == LA_FEATURE_NORM)
        return bf ? stage_t<true, true, false>(stage, x, y, sin, sout, out1, out2, s, eps, ws, st)
                  : stage_t<true, false, false>(stage, x, y, sin, sout, out1, out2, s, eps, ws, st);
    return bf ? stage_t<false, true, false>(stage, x, y, sin, sout, out1, out2, s, eps, ws, st)
              : stage_t<false, false, false>(stage, x, y, sin, sout, out1, out2, s, eps, ws, st);
}

la_status state_fwd(bool bidir, const void *q, const void *k, const void *v, void *o, float *state, const Shape &s,
                    la_dtype dt, float eps, void *ws, cudaStream_t st) {
    const bool bf = dt == LA_BF16;
    if (bidir) return bf ? fwd_t<true, true, true>(q, k, v, o, state, s, eps, ws, st)
                         : fwd_t<true, false, true>(q, k, v, o, state, s, eps, ws, st);
    return bf ? fwd_t<false, true, false>(q, k, v, o, state, s, eps, ws, st)
              : fwd_t<false, false, false>(q, k, v, o, state, s, eps, ws, st);
}

la_status state_bwd(bool bidir, const void *q, const void *k, const void *v, const void *g, const float *state,
                    void *dq, void *dk, void *dv, const Shape &s, la_dtype dt, float eps, void *ws, cudaStream_t st) {
    const bool bf = dt == LA_BF16;
    if (bidir) return bf ? bwd_t<true, true, true>(q, k, v, g, state, dq, dk, dv, s, eps, ws, st)
                         : bwd_t<true, false, true>(q, k, v, g, state, dq, dk, dv, s, eps, ws, st);
    return bf ? bwd_t<false, true, false>(q, k, v, g, state, dq, dk, dv, s, eps, ws, st)
              : bwd_t<false, false, false>(q, k, v, g, state, dq, dk, dv, s, eps, ws, st);
}

unsigned int read_and_clear_state_fault() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_tc_fault, sizeof v) != cudaSuccess) return 0xFFFFFFFFu;
    if (v) cudaMemcpyToSymbol(g_tc_fault, &zero, sizeof zero);
    return v;
}

}  // namespace tc
}  // namespace la
