// draft_tc.cu -- tensor-core (tcgen05 / TMEM / TMA) Markov-bias tile kernel
// for bf16 rounds, fused with the drafting softmax epilogue (and, in a second
// mode, with the residual mass of verification).
//
// Method (paperlayer.ai summary of DSpark, §3.1; menfem.com KB entry,
// "Methodology": rank-256 factorisation; llm-wiki.hwlabs.dev study 116,
// draft-generation figure): Delta_i = E_i W with E_i[b] = U[x_{i-1}[b]], added
// to the backbone logits L[i] before the temperature softmax.
//
// Persistent, warp-specialised CTA (one per SM), 608 threads, 512 TMEM columns.
// A CTA owns 128 rows and walks 256-column tiles; one 128 x 256 x 16 MMA per
// K step (a chain of MMAs into one accumulator costs about the same per
// instruction for N = 128 and N = 256 on this part, so the wide tile doubles
// tensor throughput).
//   warp 0      TMA producer of the B operand: the transition-factor tile
//               Wt[n0:n0+256, :] one 64-deep k-block at a time through a ring
//               (128-byte swizzle, evict-last: W is reused by every position
//               and M-block and stays in L2).
//   warp 1      TMEM owner and MMA issuer: 128 x 256 x 16 bf16 MMAs, A and B
//               from shared memory, into one of two 256-column fp32
//               accumulators.
//   warp 2      TMA producer of the logits L[:, i, :] in 128 x 64 segments
//               (128-byte swizzle, evict-first; drafting only).
//   warps 3-18  epilogue: warp e owns TMEM lane quarter (warp % 4) and the
//               64-column segment (e / 4) of every tile: Delta from TMEM plus
//               the logits give the 64-column partials (max, lowest argmax,
//               sum of exp((y - max) / T)).
// Drafting runs every position of the round in one cooperative launch: after
// a position's tiles the CTAs meet at a grid barrier, the epilogue warps
// finalize two rows per CTA (256 threads per row: the token draw, its
// probability, and the token's U row staged for the next position), meet
// again, and one thread loads the staged rows as the next position's A
// operand with TMA.  The producers run straight across position boundaries.
// At the first position (and for the residual rows) the epilogue warps gather
// the A rows U[previous token] into shared memory themselves.
// Delta never leaves the SM.  Every mbarrier and grid-barrier wait is bounded
// by a clock budget; on expiry the CTA raises a timeout bit in the status
// word, drains its own copies and MMAs, frees TMEM and returns.
#include <algorithm>

#include "common.cuh"
#include "finalize.cuh"
#include "kernels.cuh"
#include "tc.cuh"

namespace dspark {

namespace {

constexpr int kM = 128;             // rows (requests) per CTA
constexpr int kBN = 256;            // MMA N: columns per tile
constexpr int kSeg = 64;            // columns per logit segment = per partial
constexpr int kSegs = kBN / kSeg;   // 4
constexpr int kKB = 64;             // bf16 elements per 128-byte k-block
constexpr int kABlockBytes = kM * 128;     // one k-block of A (16 KB)
constexpr int kStageBytes = kBN * 128;     // one k-block of B (32 KB)
constexpr int kSegBytes = kM * kSeg * 2;   // one logit segment (16 KB)
constexpr int kEpiWarp0 = 3;
constexpr int kEpiWarps = 16;
constexpr int kThreads = (kEpiWarp0 + kEpiWarps) * 32;   // 608
constexpr int kTmemCols = 2 * kBN;                        // two accumulators
constexpr long long kWaitBudget = 4000000000LL;          // ~2 s of SM clock

struct TcLayout {
    int nkb, sB, sL;
    uint32_t a_off, b_off, l_off, bar_off, total;
};

// Every epilogue warp group owns one logit slot (segment sg of each tile goes
// to slot sg), so a group only ever waits on phases of its own slot (drafting
// only; the residual pass reads its rows from global memory); the B ring takes
// what shared memory is left (3 stages for r <= 256, 1 for r = 512).  With the
// RNN head's rows (residual pass only) A holds a high and a low bf16 part.
__host__ __device__ inline TcLayout tc_layout(int r, int mode, int rnn) {
    TcLayout t;
    t.nkb = (r + kKB - 1) / kKB;
    t.sL = mode == 0 ? kSegs : 0;
    const int na = t.nkb * (rnn ? 2 : 1);
    const int fixed = na * kABlockBytes + t.sL * kSegBytes + 256 + 1024;
    int sB = (227 * 1024 - fixed) / kStageBytes;
    t.sB = sB > 3 ? 3 : (sB < 1 ? 1 : sB);   // B ring depth
    t.a_off = 0;
    t.b_off = t.a_off + na * kABlockBytes;
    t.l_off = t.b_off + t.sB * kStageBytes;
    t.bar_off = t.l_off + t.sL * kSegBytes;
    t.total = t.bar_off + 256 + 1024;   // barriers, base alignment
    return t;
}

// Epilogue modes: drafting partials, or residual mass for verification.
enum { kEpiDraft = 0, kEpiResidual = 1 };

struct TcEpi {
    const float *temp;
    int B, G, V, nParts;
    long long budget;         // clock budget of the bounded waits (drains keep their own)
    WsHeader *hdr;
    FinArgs fin;              // drafting: the per-row finalize of every position
    uint32_t *grid_count;     // drafting: grid-barrier counter (zeroed before the launch)
    const __nv_bfloat16 *U;   // [V, r]: A-operand rows are U[previous token]
    const int32_t *x0;        // [B] last committed tokens
    const int32_t *x;         // [B, G] draft tokens (drafting: earlier positions of this call)
    const float *H;           // residual, RNN head: the states [B, G, r] (A rows split high/low); else null
    const __nv_bfloat16 *L;   // drafting and residual: backbone logits [B, G, V]
    // drafting: 64-column partials per request row
    float2 *part;
    // residual: rows are the queued rejections; per 64 columns the sum of
    // max(0, p_t - p_d) with p_d rebuilt from L + Delta and the drafting stats
    const uint32_t *nrows;
    const int32_t *res_b, *res_k;
    const float *res_mt, *res_zt, *rowmax, *rowsum;
    const __nv_bfloat16 *Tlog;
    float *rp;
};

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1) markov_tile_tc(const __grid_constant__ CUtensorMap mapW,
                                                              const __grid_constant__ CUtensorMap mapL,
                                                              const __grid_constant__ CUtensorMap mapE, int r,
                                                              int nTilesN, const TcEpi ep)
{
    extern __shared__ unsigned char smem_raw[];
    const int rnn = (MODE == kEpiResidual && ep.H != nullptr) ? 1 : 0;
    const TcLayout lay = tc_layout(r, MODE, rnn);
    const uint32_t raw_u32 = tc::smem_u32(smem_raw);
    unsigned char *base = smem_raw + (((raw_u32 + 1023) & ~1023u) - raw_u32);
    unsigned char *sA = base + lay.a_off;
    unsigned char *sB = base + lay.b_off;
    unsigned char *sL = base + lay.l_off;
    const int SB = lay.sB, SL = lay.sL, nkb = lay.nkb;
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + lay.bar_off);
    uint64_t *a_full = bars;                 // A is in shared memory (one phase per position)
    uint64_t *b_full = a_full + 1;           // SB
    uint64_t *b_empty = b_full + SB;         // SB
    uint64_t *l_full = b_empty + SB;         // SL
    uint64_t *l_empty = l_full + SL;         // SL (4 warps, one per lane quarter)
    uint64_t *acc_full = l_empty + SL;       // 2
    uint64_t *acc_empty = acc_full + 2;      // 2 (16 warps)
    uint64_t *drain = acc_empty + 2;         // 1
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    __shared__ int epi_flag;                 // epilogue-wide verdict of the last grid barrier
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int B = ep.B, V = ep.V, nParts = ep.nParts;
    const int npos = (MODE == kEpiDraft) ? ep.G : 1;
    WsHeader *hdr = ep.hdr;
    // Residual rows are counted on the device: the CTAs split over the
    // M-blocks that hold queued rows only, so a round with at most 128
    // rejections runs every CTA on one M-block.
    const int nrows = (MODE == kEpiResidual) ? (int)*reinterpret_cast<const volatile uint32_t *>(ep.nrows) : B;
    if (nrows <= 0) return;
    const int nMB = (nrows + kM - 1) / kM;
    const int mb = blockIdx.x % nMB;
    const int m0 = mb * kM;
    const int first_tile = blockIdx.x / nMB;
    const int tile_step = ((int)gridDim.x - mb + nMB - 1) / nMB;
    // (Drafting grids never exceed the tile count: every CTA meets the grid barriers.)
    if (MODE == kEpiResidual && first_tile >= nTilesN) return;

    if (threadIdx.x == 0) {
        tc::mbar_init(a_full, 1);
        for (int q = 0; q < SB; ++q) { tc::mbar_init(&b_full[q], 1); tc::mbar_init(&b_empty[q], 1); }
        for (int q = 0; q < SL; ++q) { tc::mbar_init(&l_full[q], 1); tc::mbar_init(&l_empty[q], 4); }
        for (int q = 0; q < 2; ++q) { tc::mbar_init(&acc_full[q], 1); tc::mbar_init(&acc_empty[q], kEpiWarps); }
        tc::mbar_init(drain, 1);
        *abort_flag = 0;
        tc::fence_barrier_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, kTmemCols);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------ B producer
        if (lane == 0) {
            tc::prefetch_tmap(&mapW);
            const uint64_t keep = tc::policy_evict_last();
            int g = 0;
            bool ok = true;
            // The factor does not depend on the drawn tokens: the ring runs on
            // into the next position while the rows are finalized.
            for (int pos = 0; pos < npos && ok; ++pos) {
            for (int t = first_tile; t < nTilesN && ok; t += tile_step) {
                const int n0 = t * kBN;
                for (int kb = 0; kb < nkb; ++kb, ++g) {
                    const int s = g % SB;
                    if (!tc::mbar_wait_bounded(&b_empty[s], ((g / SB) & 1) ^ 1, abort_flag, ep.budget)) {
                        ok = false;
                        break;
                    }
                    tc::mbar_arrive_expect_tx(&b_full[s], kStageBytes);
                    tc::tma_load_2d(sB + s * kStageBytes, &mapW, &b_full[s], kb * kKB, n0, keep);
                }
            }
            }
            if (!ok) {
                // Give up: wait (bounded, ignoring the abort flag) for every copy
                // this thread issued so that none lands after the CTA exits.
                int dummy = 0;
                volatile int *no_abort = &dummy;
                for (int q = 0; q < SB && g - 1 - q >= 0; ++q) {
                    const int gg = g - 1 - q;
                    tc::mbar_wait_bounded(&b_full[gg % SB], (gg / SB) & 1, no_abort, kWaitBudget / 4);
                }
                flag_status(hdr, DSPARK_DEV_TIMEOUT);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = tc::idesc_bf16_f32(kM, kBN);
            const uint32_t a_addr = tc::smem_u32(sA), b_addr = tc::smem_u32(sB);
            bool ok = true;
            int g = 0, j = 0;
            for (int pos = 0; pos < npos && ok; ++pos) {
            ok = tc::mbar_wait_bounded(a_full, pos & 1, abort_flag, ep.budget);
            tc::tc_fence_after();
            for (int t = first_tile; t < nTilesN && ok; t += tile_step, ++j) {
                const int ab = j & 1;
                if (!tc::mbar_wait_bounded(&acc_empty[ab], ((j >> 1) & 1) ^ 1, abort_flag, ep.budget)) {
                    ok = false;
                    break;
                }
                tc::tc_fence_after();
                const uint32_t d = tmem_base + ab * kBN;
                for (int kb = 0; kb < nkb; ++kb, ++g) {
                    const int s = g % SB;
                    if (!tc::mbar_wait_bounded(&b_full[s], (g / SB) & 1, abort_flag, ep.budget)) {
                        ok = false;
                        break;
                    }
                    tc::tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < kKB / 16; ++kk) {
                        const uint64_t ad = tc::sw128_desc(a_addr + kb * kABlockBytes + kk * 32);
                        const uint64_t bd = tc::sw128_desc(b_addr + s * kStageBytes + kk * 32);
                        tc::mma_bf16(d, ad, bd, idesc, (kb | kk) != 0);
                        if (rnn) {
                            const uint64_t al = tc::sw128_desc(a_addr + (nkb + kb) * kABlockBytes + kk * 32);
                            tc::mma_bf16(d, al, bd, idesc, 1u);
                        }
                    }
                    tc::mma_commit(&b_empty[s]);
                }
                if (!ok) break;
                tc::mma_commit(&acc_full[ab]);
            }
            }
            // Drain: every MMA issued above has completed once this arrives.
            tc::mma_commit(drain);
            int dummy = 0;
            tc::mbar_wait_bounded(drain, 0, &dummy, kWaitBudget / 4);
            if (!ok) flag_status(hdr, DSPARK_DEV_TIMEOUT);
        }
    } else if (warp == 2) {
        // ------------------------------------------------------ logit producer
        if (MODE == kEpiDraft && lane == 0) {
            tc::prefetch_tmap(&mapL);
            const uint64_t stream = tc::policy_evict_first();
            int g = 0;
            bool ok = true;
            for (int pos = 0; pos < npos && ok; ++pos) {   // (the logits neither)
            for (int t = first_tile; t < nTilesN && ok; t += tile_step) {
                for (int sg = 0; sg < kSegs; ++sg, ++g) {
                    const int q = g % SL;
                    if (!tc::mbar_wait_bounded(&l_empty[q], ((g / SL) & 1) ^ 1, abort_flag, ep.budget)) {
                        ok = false;
                        break;
                    }
                    tc::mbar_arrive_expect_tx(&l_full[q], kSegBytes);
                    tc::tma_load_3d(sL + q * kSegBytes, &mapL, &l_full[q], t * kBN + sg * kSeg, pos, m0, stream);
                }
            }
            }
            if (!ok) {
                int dummy = 0;
                volatile int *no_abort = &dummy;
                for (int q = 0; q < SL && g - 1 - q >= 0; ++q) {
                    const int gg = g - 1 - q;
                    tc::mbar_wait_bounded(&l_full[gg % SL], (gg / SL) & 1, no_abort, kWaitBudget / 4);
                }
                flag_status(hdr, DSPARK_DEV_TIMEOUT);
            }
        }
    } else {
        const int ew = warp - kEpiWarp0;       // 0..15
        const int quarter = warp & 3;          // TMEM lane quarter this warp may access
        const int sg = ew >> 2;                // 64-column segment of every tile (0..3)
        const int row = quarter * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        const bool leader = ew == 0 && lane == 0;
        // Named barrier 1: the 16 epilogue warps only.
        auto epi_sync = [&]() { asm volatile("bar.sync 1, %0;" ::"r"(kEpiWarps * 32) : "memory"); };
        // A operand into shared memory: row `row` is U[prev] -- x0 at the
        // first position, or for a queued rejection the token before it.
        // This warp writes k-blocks kb = sg, sg + 4, ... of its 32 rows in the
        // 128-byte-swizzled K-major layout (zeros past r); then one thread
        // completes the A phase for the MMA warp.
        auto gather_A = [&](int prev) {
            const __nv_bfloat16 *urow = ep.U + (size_t)prev * r;
            for (int kb = sg; kb < nkb; kb += kSegs) {
                uint4 v[8];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const int k = kb * kKB + c * 8;
                    v[c] = (k < r) ? ld_nc16(urow + k) : make_uint4(0, 0, 0, 0);
                }
                unsigned char *dst = sA + kb * kABlockBytes + row * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4 *>(dst + ((c ^ (row & 7)) << 4)) = v[c];
            }
            tc::fence_proxy_async_smem();   // generic writes -> tensor-core reads
            epi_sync();
            if (leader) tc::mbar_arrive(a_full);
        };
        // RNN head's rows: the fp32 state h (row `row` of A) split into bf16
        // high parts (k-blocks 0..nkb-1) and low parts (nkb..2nkb-1).
        auto gather_A_state = [&](const float *hrow) {
            for (int kb = sg; kb < nkb; kb += kSegs) {
                unsigned char *dhi = sA + kb * kABlockBytes + row * 128;
                unsigned char *dlo = sA + (nkb + kb) * kABlockBytes + row * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const int k = kb * kKB + c * 8;
                    float h8[8];
                    if (hrow != nullptr && k < r) {
                        const float4 p0 = *reinterpret_cast<const float4 *>(hrow + k);
                        const float4 p1 = *reinterpret_cast<const float4 *>(hrow + k + 4);
                        h8[0] = p0.x; h8[1] = p0.y; h8[2] = p0.z; h8[3] = p0.w;
                        h8[4] = p1.x; h8[5] = p1.y; h8[6] = p1.z; h8[7] = p1.w;
                    } else {
#pragma unroll
                        for (int e = 0; e < 8; ++e) h8[e] = 0.f;
                    }
                    uint32_t hi4[4], lo4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const __nv_bfloat16 a0 = __float2bfloat16_rn(h8[2 * e]), a1 = __float2bfloat16_rn(h8[2 * e + 1]);
                        const __nv_bfloat16 b0 = __float2bfloat16_rn(h8[2 * e] - __bfloat162float(a0));
                        const __nv_bfloat16 b1 = __float2bfloat16_rn(h8[2 * e + 1] - __bfloat162float(a1));
                        hi4[e] = (uint32_t)__bfloat16_as_ushort(a0) | ((uint32_t)__bfloat16_as_ushort(a1) << 16);
                        lo4[e] = (uint32_t)__bfloat16_as_ushort(b0) | ((uint32_t)__bfloat16_as_ushort(b1) << 16);
                    }
                    *reinterpret_cast<uint4 *>(dhi + ((c ^ (row & 7)) << 4)) = make_uint4(hi4[0], hi4[1], hi4[2], hi4[3]);
                    *reinterpret_cast<uint4 *>(dlo + ((c ^ (row & 7)) << 4)) = make_uint4(lo4[0], lo4[1], lo4[2], lo4[3]);
                }
            }
            tc::fence_proxy_async_smem();
            epi_sync();
            if (leader) tc::mbar_arrive(a_full);
        };
        if (MODE == kEpiDraft) {
            // ------------------------------------------ drafting epilogue
            // One online pass per 32-column chunk: y = L + Delta, chunk max,
            // then the running sum of exp((y - max) / T), rescaled when the
            // max grows.  The lowest argmax is tracked only in warps holding a
            // greedy row.
            const int b = m0 + row;
            const bool rowok = b < B;
            float invT = 0.f;
            if (rowok) {
                const float Tb = ep.temp[b];
                invT = Tb > 0.f ? 1.f / Tb : 0.f;
            }
            const float cexp = invT * kLog2e;      // exp((y - m) / T) = 2^((y - m) * cexp)
            const bool warp_greedy = __any_sync(0xffffffffu, rowok && invT == 0.f);
            const bool warp_soft = __any_sync(0xffffffffu, rowok && invT > 0.f);
            // All CTAs' epilogue warps meet; false (uniform across the
            // epilogue) when any role of this CTA aborted or the wait ran out.
            auto grid_sync = [&](uint32_t target) -> bool {
                epi_sync();
                if (leader) {
                    bool ok = *abort_flag == 0;
                    if (ok) {
                        __threadfence();
                        atomicAdd(ep.grid_count, 1u);
                        const long long t0 = clock64();
                        while (tc::ld_acquire_gpu(ep.grid_count) < target) {
                            if (*abort_flag || clock64() - t0 > ep.budget) { ok = false; break; }
                            __nanosleep(32);
                        }
                    }
                    if (!ok) {
                        *abort_flag = 1;
                        flag_status(hdr, DSPARK_DEV_TIMEOUT);
                    }
                    epi_flag = ok ? 0 : 1;
                }
                epi_sync();
                return epi_flag == 0;
            };
            // Finalize: epilogue warps 0-7 and 8-15 are two 256-thread groups
            // (named barriers 2 and 3), each with scratch in the A region,
            // which no MMA reads between a position's last tile and the next
            // position's A load.
            const int grp = ew >> 3;
            const Grp fg{(ew & 7) * 32 + lane, 256, ew & 7, 8, 2 + grp};
            FinScratch *fsc = reinterpret_cast<FinScratch *>(sA + grp * 4096);
            float *furow = reinterpret_cast<float *>(sA + 8192 + grp * 2048);

            const uint32_t nblk = gridDim.x;
            int j = 0;
            for (int pos = 0; pos < ep.G; ++pos) {
                if (pos == 0) {
                    int prev = 0;
                    if (rowok) {
                        prev = ep.x0[b];
                        if (prev < 0 || prev >= V) {
                            flag_status(hdr, DSPARK_DEV_TOKEN_RANGE);
                            prev = prev < 0 ? 0 : V - 1;
                        }
                    }
                    gather_A(prev);
                }
                for (int t = first_tile; t < nTilesN; t += tile_step, ++j) {
                    const int ab = j & 1;
                    const int gl = j * kSegs + sg, q = gl % SL;
                    // Every lane waits; the vote keeps the warp converged for the
                    // warp-collective TMEM loads below even if the budget runs out.
                    bool ok = tc::mbar_wait_bounded(&l_full[q], (gl / SL) & 1, abort_flag, ep.budget);
                    ok = ok && tc::mbar_wait_bounded(&acc_full[ab], (j >> 1) & 1, abort_flag, ep.budget);
                    if (!__all_sync(0xffffffffu, ok)) break;
                    tc::tc_fence_after();
                    // This thread's 64 logits: one 128-byte row of the swizzled segment.
                    const unsigned char *lsrc = sL + q * kSegBytes + row * 128;
                    uint4 cur[8];
    #pragma unroll
                    for (int u = 0; u < 8; ++u)
                        cur[u] = *reinterpret_cast<const uint4 *>(lsrc + ((u ^ (row & 7)) << 4));
                    // The segment is in registers: hand the slot back to the
                    // producer now, so the next tile's copy overlaps this one's math.
                    tc::fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(&l_empty[q]);
                    const uint32_t taddr = tmem_base + lane_addr + ab * kBN + sg * kSeg;
                    const int cbase = t * kBN + sg * kSeg;
                    const bool whole = cbase + kSeg <= V;   // no column of this segment lies past V
                    float m = -INFINITY, s = 0.f;
                    int am = 0x7fffffff;
    #pragma unroll
                    for (int c = 0; c < kSeg / 32; ++c) {
                        float y[32];
                        tc::tmem_ld32(taddr + c * 32, y);
                        // y = L + Delta, two columns per instruction.
    #pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const uint4 qv = cur[c * 4 + u];
                            const uint32_t wq[4] = {qv.x, qv.y, qv.z, qv.w};
    #pragma unroll
                            for (int h = 0; h < 4; ++h) {
                                const float2 yy = add2(make_float2(y[u * 8 + 2 * h], y[u * 8 + 2 * h + 1]),
                                                       make_float2(bf16lo(wq[h]), bf16hi(wq[h])));
                                y[u * 8 + 2 * h] = yy.x;
                                y[u * 8 + 2 * h + 1] = yy.y;
                            }
                        }
                        if (!whole) {
    #pragma unroll
                            for (int e = 0; e < 32; ++e)
                                if (cbase + c * 32 + e >= V) y[e] = -INFINITY;
                        }
                        // Chunk max: a tree of three-input maxima.
                        float t11[11];
    #pragma unroll
                        for (int e = 0; e < 10; ++e) t11[e] = max3(y[3 * e], y[3 * e + 1], y[3 * e + 2]);
                        t11[10] = fmaxf(y[30], y[31]);
                        const float cm = max3(max3(t11[0], t11[1], t11[2]), max3(t11[3], t11[4], t11[5]),
                                              max3(max3(t11[6], t11[7], t11[8]), t11[9], t11[10]));
                        if (warp_greedy && cm > m) {
                            int ix = 0x7fffffff;
    #pragma unroll
                            for (int e = 31; e >= 0; --e)
                                if (y[e] == cm) ix = e;
                            am = cbase + c * 32 + ix;
                        }
                        const float mn = fmaxf(m, cm);
                        if (warp_soft) {
                            // exp((y - mn) / T) = 2^(y * cexp - mn * cexp): one fused
                            // multiply-add per two columns, then the two ex2.
                            const float2 c2 = make_float2(cexp, cexp);
                            const float nmc = -mn * cexp;
                            const float2 n2 = make_float2(nmc, nmc);
                            float2 s2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                                            make_float2(0.f, 0.f)};   // four independent pairs of sums
    #pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                const float2 arg = fma2(make_float2(y[2 * e], y[2 * e + 1]), c2, n2);
                                s2[e & 3] = add2(s2[e & 3], make_float2(fast_exp2(arg.x), fast_exp2(arg.y)));
                            }
                            const float2 p01 = add2(s2[0], s2[1]), p23 = add2(s2[2], s2[3]);
                            const float2 pall = add2(p01, p23);
                            const float acc = pall.x + pall.y;
                            s = (m == -INFINITY ? 0.f : s * fast_exp2((m - mn) * cexp)) + acc;
                        }
                        m = mn;
                    }
                    tc::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(&acc_empty[ab]);
                    const int p = t * kSegs + sg;
                    if (rowok && p < nParts) {
                        const size_t o = (size_t)b * nParts + p;
                        // One 8-byte record: the finalize reads Z's terms for a sampled row,
                        // the argmax for a greedy one.
                        ep.part[o] = make_float2(m, invT > 0.f ? s : __int_as_float(am));
                    }
                }
                // Every CTA's partials of this position are written.
                if (!grid_sync(nblk * (2u * pos + 1u))) break;
                for (int bb = (int)blockIdx.x * 2 + grp; bb < B; bb += 2 * (int)nblk)
                    finalize_row<__nv_bfloat16>(fg, fsc, furow, ep.fin, bb, pos);
                tc::fence_proxy_async_all();   // E rows and the scratch, before async-proxy use
                // Every row's token (and staged U row) of this position is written.
                if (!grid_sync(nblk * (2u * pos + 2u))) break;
                if (pos + 1 < ep.G && leader) {
                    tc::fence_proxy_async_all();
                    tc::mbar_arrive_expect_tx(a_full, (uint32_t)nkb * kABlockBytes);
                    const uint64_t once = tc::policy_evict_first();
                    for (int kb = 0; kb < nkb; ++kb)
                        tc::tma_load_2d(sA + kb * kABlockBytes, &mapE, a_full, kb * kKB, m0, once);
                }
            }
        } else {
            if (rnn) {
                const int sidx = m0 + row;
                const float *hrow = nullptr;
                if (sidx < nrows) hrow = ep.H + ((size_t)ep.res_b[sidx] * ep.G + ep.res_k[sidx]) * r;
                gather_A_state(hrow);
            } else {
                int prev = 0;
                const int sidx = m0 + row;
                if (sidx < nrows) {
                    const int bq = ep.res_b[sidx], k = ep.res_k[sidx];
                    prev = (k == 0) ? ep.x0[bq] : ep.x[(size_t)bq * ep.G + k - 1];
                    prev = min(max(prev, 0), V - 1);
                }
                gather_A(prev);
            }
            // ------------------------------------------ residual epilogue
            const int sidx = m0 + row;
            const bool rowok = sidx < nrows;
            float invT = 0.f, Md = 0.f, rZd = 0.f, Mt = 0.f, rZt = 0.f;
            const __nv_bfloat16 *Lrow = ep.L, *Trow = ep.Tlog;
            if (rowok) {
                const int b = ep.res_b[sidx], k = ep.res_k[sidx];
                invT = 1.f / fmaxf(ep.temp[b], 1e-30f);
                const size_t ro = (size_t)b * ep.G + k;
                Md = ep.rowmax[ro];
                rZd = 1.f / ep.rowsum[ro];
                Mt = ep.res_mt[sidx];
                rZt = 1.f / ep.res_zt[sidx];
                Lrow = ep.L + ro * V;
                Trow = ep.Tlog + ((size_t)b * (ep.G + 1) + k) * V;
            }
            int j = 0;
            for (int t = first_tile; t < nTilesN; t += tile_step, ++j) {
                const int ab = j & 1;
                const int cbase = t * kBN + sg * kSeg;
                const bool ok = tc::mbar_wait_bounded(&acc_full[ab], (j >> 1) & 1, abort_flag, ep.budget);
                if (!__all_sync(0xffffffffu, ok)) break;
                tc::tc_fence_after();
                const uint32_t taddr = tmem_base + lane_addr + ab * kBN + sg * kSeg;
                float qs = 0.f;
#pragma unroll
                for (int c = 0; c < kSeg / 32; ++c) {
                    uint4 lq[4], tq[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int c8 = cbase + c * 32 + u * 8;
                        const bool in = rowok && c8 < V;
                        lq[u] = in ? ld_nc16(Lrow + c8) : make_uint4(0, 0, 0, 0);
                        tq[u] = in ? ld_nc16(Trow + c8) : make_uint4(0, 0, 0, 0);
                    }
                    float d[32];
                    tc::tmem_ld32(taddr + c * 32, d);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const uint4 a = lq[u], bq = tq[u];
                        const float l8[8] = {bf16lo(a.x), bf16hi(a.x), bf16lo(a.y), bf16hi(a.y),
                                             bf16lo(a.z), bf16hi(a.z), bf16lo(a.w), bf16hi(a.w)};
                        const float t8[8] = {bf16lo(bq.x), bf16hi(bq.x), bf16lo(bq.y), bf16hi(bq.y),
                                             bf16lo(bq.z), bf16hi(bq.z), bf16lo(bq.w), bf16hi(bq.w)};
                        const bool in = rowok && (cbase + c * 32 + u * 8) < V;
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float pt = exp_e((t8[e] - Mt) * invT) * rZt;
                            const float pd = exp_e(((l8[e] - Md) + d[u * 8 + e]) * invT) * rZd;
                            if (in) qs += fmaxf(pt - pd, 0.f);
                        }
                    }
                }
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&acc_empty[ab]);
                const int p = t * kSegs + sg;
                if (rowok && p < nParts) ep.rp[(size_t)sidx * nParts + p] = qs;
            }
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem_base, kTmemCols);
    }
}

// ------------------------------------------------------------------ host
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (fn == nullptr) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// Tensor map of the transition factor Wt [V, r] (bf16): 64 x 128 boxes,
// 128-byte swizzle, rows past V and columns past r read as zero.
bool map_factor(CUtensorMap *m, const void *Wt, int V, int r) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[2] = {(cuuint64_t)r, (cuuint64_t)V};
    cuuint64_t strides[1] = {(cuuint64_t)r * 2};
    cuuint32_t box[2] = {kKB, kBN};   // 64 x 256: one k-block of a 256-column tile
    cuuint32_t es[2] = {1, 1};
    CUresult res = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(Wt), dims, strides, box, es,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return res == CUDA_SUCCESS;
}

// Tensor map of the logits L [B, G, V] (bf16) as a 3-D tensor (V, G, B):
// 64-column x 1 x 128-row boxes, 128-byte swizzle, out-of-range reads as zero.
bool map_logits(CUtensorMap *m, const void *L, int B, int G, int V) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[3] = {(cuuint64_t)V, (cuuint64_t)G, (cuuint64_t)B};
    cuuint64_t strides[2] = {(cuuint64_t)V * 2, (cuuint64_t)G * V * 2};
    cuuint32_t box[3] = {kSeg, 1, kM};
    cuuint32_t es[3] = {1, 1, 1};
    CUresult res = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(L), dims, strides, box, es,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return res == CUDA_SUCCESS;
}

// Tensor map of the staged A rows E [B, r] (bf16): 64 x 128 boxes (one
// k-block of one 128-row block), 128-byte swizzle, rows past B read as zero.
bool map_stage(CUtensorMap *m, const void *E, int B, int r) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[2] = {(cuuint64_t)r, (cuuint64_t)B};
    cuuint64_t strides[1] = {(cuuint64_t)r * 2};
    cuuint32_t box[2] = {kKB, kM};
    cuuint32_t es[2] = {1, 1};
    CUresult res = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(E), dims, strides, box, es,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return res == CUDA_SUCCESS;
}

template <int MODE>
cudaError_t launch_markov_tc(const void *Wt, int r, const TcEpi &ep, const void *E, cudaStream_t st) {
    CUtensorMap mW, mL, mE;
    if (!map_factor(&mW, Wt, ep.V, r)) return cudaErrorInvalidValue;
    if (!map_logits(&mL, ep.L, ep.B, ep.G, ep.V)) return cudaErrorInvalidValue;
    if (MODE == kEpiDraft && ep.G > 1) {
        if (!map_stage(&mE, E, ep.B, r)) return cudaErrorInvalidValue;
    } else {
        mE = mW;   // unused
    }
    const TcLayout lay = tc_layout(r, MODE, (MODE == kEpiResidual && ep.H != nullptr) ? 1 : 0);
    cudaError_t e = cudaFuncSetAttribute(markov_tile_tc<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)lay.total);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int nTilesN = (ep.V + kBN - 1) / kBN;
    const int nMB = (ep.B + kM - 1) / kM;
    int grid = std::min(sms, nMB * nTilesN);
    grid = std::max(grid, nMB);
    if (MODE == kEpiResidual) {
        markov_tile_tc<MODE><<<grid, kThreads, lay.total, st>>>(mW, mL, mE, r, nTilesN, ep);
        return cudaGetLastError();
    }
    // Drafting: every CTA must be resident for the grid barriers, which a
    // cooperative launch guarantees (or refuses).
    int per_sm = 0;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, markov_tile_tc<MODE>, kThreads, lay.total)) !=
        cudaSuccess)
        return e;
    if (per_sm < 1 || grid > per_sm * sms) return cudaErrorCooperativeLaunchTooLarge;
    if ((e = cudaMemsetAsync(ep.grid_count, 0, sizeof(uint32_t), st)) != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = lay.total;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, markov_tile_tc<MODE>, mW, mL, mE, r, nTilesN, ep);
}

}  // namespace

cudaError_t launch_draft_tc(const DraftArgs &a, const DraftWs &w, const FinArgs &f, cudaStream_t st) {
    TcEpi ep{};
    ep.temp = a.temp; ep.B = a.B; ep.G = a.G; ep.V = a.V; ep.nParts = w.nTiles; ep.hdr = w.hdr;
    ep.budget = wait_budget(kWaitBudget);
    ep.U = static_cast<const __nv_bfloat16 *>(a.U); ep.x0 = a.x0; ep.x = a.x_out;
    ep.L = static_cast<const __nv_bfloat16 *>(a.L);
    ep.part = w.part;
    ep.fin = f;
    ep.grid_count = &w.hdr->pad[2];
    return launch_markov_tc<kEpiDraft>(a.Wt, a.r, ep, w.E, st);
}

cudaError_t launch_residual_tile_tc(const ResidualTcArgs &a, cudaStream_t st) {
    TcEpi ep{};
    ep.temp = a.temp; ep.B = a.B; ep.G = a.G; ep.V = a.V; ep.nParts = a.nParts; ep.hdr = a.hdr;
    ep.budget = wait_budget(kWaitBudget);
    ep.U = a.U; ep.x0 = a.x0; ep.x = a.x; ep.L = a.L;
    ep.nrows = a.nrows; ep.res_b = a.res_b; ep.res_k = a.res_k; ep.res_mt = a.res_mt; ep.res_zt = a.res_zt;
    ep.H = a.H;
    ep.rowmax = a.rowmax; ep.rowsum = a.rowsum; ep.Tlog = a.Tlog; ep.rp = a.rp;
    return launch_markov_tc<kEpiResidual>(a.Wt, a.r, ep, nullptr, st);
}

}  // namespace dspark
