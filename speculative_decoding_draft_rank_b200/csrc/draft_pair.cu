// draft_pair.cu -- tensor-core drafting on CTA pairs for batches of more than
// 128 requests: the Markov-bias product Delta_i = E_i W (E_i[b] = U[x_{i-1}[b]])
// of a 256-row block is one M = 256 MMA per K step shared by the two CTAs of a
// cluster (tcgen05 cta_group::2), fused with the drafting softmax epilogue.
//
// Method (paperlayer.ai summary of DSpark, §3.1 Semi-autoregressive
// generation; menfem.com KB entry, "Methodology": rank-256 factorisation;
// llm-wiki.hwlabs.dev study 116, draft-generation figure): each position's
// logits L[i] + Delta_i go through a temperature softmax and an inverse-CDF
// draw; the drawn token selects the next position's U row.
//
// Why pairs: a 128-row CTA streams every 256-column tile of the transition
// factor (128 KB) through its shared memory for every position, twice per
// 256 requests, while it also streams the logits from HBM; with M = 256 the
// pair reads each tile once (each CTA loads its own 128 columns of it and the
// MMA reads both halves), halving the factor's L2 traffic per position.
//
// Roles per CTA (608 threads), the same in both CTAs of a pair except the MMA:
//   warp 0      TMA producer of this CTA's half of the B tile: Wt rows
//               [n0 + 128 * rank, +128) one 64-deep k-block at a time through
//               a ring; completion is counted on the even CTA's barrier.
//   warp 1      TMEM owner (512 columns, allocated for the pair); in the even
//               CTA the MMA issuer: 256 x 256 x 16 bf16 MMAs into one of two
//               256-column accumulators, each CTA receiving its 128 rows.
//   warp 2      TMA producer of this CTA's logit rows L[m0 : m0 + 128, i, :]
//               in 128 x 64 segments.
//   warps 3-18  epilogue on this CTA's accumulator rows: the 64-column
//               partials (max, lowest argmax, sum of exp((y - max) / T)) of
//               y = L + Delta; Delta never leaves the SM.
// Positions are separated by a grid barrier, the per-row finalize (inverse
// CDF, token, U row staged for the next position) and a second grid barrier,
// as in the single-CTA kernel of draft_tc.cu.  The two producers do not wait
// for that window: the logits and the factor do not depend on the drawn
// tokens, so they fill the free ring slots with the next position's first
// tiles while the rows are finalized.  Every mbarrier and grid-barrier
// wait is bounded; a CTA that gives up raises DSPARK_DEV_TIMEOUT, lets its
// copies in flight land, and both CTAs of the pair meet at a cluster barrier
// before the pair's tensor memory is freed.
#include <algorithm>

#include "common.cuh"
#include "finalize.cuh"
#include "kernels.cuh"
#include "tc.cuh"

namespace dspark {

namespace {

constexpr int kPM = 128;                      // rows per CTA (256 per pair)
constexpr int kPBN = 256;                     // MMA N: columns per tile
constexpr int kPHalf = kPBN / 2;              // columns of the B tile each CTA stages
constexpr int kPSeg = 64;                     // columns per logit segment = per partial
constexpr int kPSegs = kPBN / kPSeg;          // 4
constexpr int kPKB = 64;                      // bf16 elements per 128-byte k-block
constexpr int kPABytes = kPM * 128;           // one k-block of A (16 KB)
constexpr int kPBStage = kPHalf * 128;        // one k-block of this CTA's half of B (16 KB)
constexpr int kPSegBytes = kPM * kPSeg * 2;   // one logit segment (16 KB)
constexpr int kPEpi0 = 3;
constexpr int kPEpiWarps = 16;
constexpr int kPThreads = (kPEpi0 + kPEpiWarps) * 32;   // 608
constexpr int kPTmemCols = 2 * kPBN;                     // two accumulators
constexpr long long kPWaitBudget = 4000000000LL;        // ~2 s of SM clock
constexpr long long kPDrainCycles = 2000000LL;          // ~1 ms: copies in flight land long before

// Heads: the Markov head's A rows are U[previous token] (bf16, one MMA per
// K step); the RNN head's are its fp32 state split into bf16 high and low
// parts (two MMAs per K step into the same accumulator).
enum { kHeadMarkov = 0, kHeadRnn = 1 };

struct PairLayout {
    int nkb, sB, sL;
    uint32_t a_off, b_off, l_off, bar_off, total;
};

// The B ring takes what is left under ~200 KB (2 to 6 stages; deeper rings
// under the full 227 KB measured slower).  Each of the four logit consumer
// groups (one per 64-column segment) owns one slot: with fewer slots than
// groups a slot would pass between groups whose parity waits can alias.
__host__ __device__ inline PairLayout pair_layout(int r, int head) {
    PairLayout t;
    t.nkb = (r + kPKB - 1) / kPKB;
    t.sL = kPSegs;
    const int na = t.nkb * (head == kHeadRnn ? 2 : 1);
    const int fixed = na * kPABytes + t.sL * kPSegBytes + 256 + 1024;
    int sB = (200 * 1024 - fixed) / kPBStage;
    t.sB = sB > 6 ? 6 : (sB < 2 ? 2 : sB);
    t.a_off = 0;
    t.b_off = t.a_off + na * kPABytes;
    t.l_off = t.b_off + t.sB * kPBStage;
    t.bar_off = t.l_off + t.sL * kPSegBytes;
    t.total = t.bar_off + 256 + 1024;
    return t;
}

struct PairEpi {
    const float *temp;
    int B, G, V, nParts, nPB;   // nPB: 256-row blocks
    long long budget;
    WsHeader *hdr;
    FinArgs fin;
    uint32_t *grid_count;
    const __nv_bfloat16 *U;
    const int32_t *x0;
    float2 *part;
};

template <int HEAD>
__global__ void __launch_bounds__(kPThreads, 1)
    markov_pair_tc(const __grid_constant__ CUtensorMap mapW, const __grid_constant__ CUtensorMap mapL,
                   const __grid_constant__ CUtensorMap mapE, int r, int nTilesN, const PairEpi ep)
{
    extern __shared__ unsigned char smem_raw[];
    const PairLayout lay = pair_layout(r, HEAD);
    const uint32_t raw_u32 = tc::smem_u32(smem_raw);
    unsigned char *base = smem_raw + (((raw_u32 + 1023) & ~1023u) - raw_u32);
    unsigned char *sA = base + lay.a_off;
    unsigned char *sB = base + lay.b_off;
    unsigned char *sL = base + lay.l_off;
    const int SB = lay.sB, SL = lay.sL, nkb = lay.nkb;
    const int na = HEAD == kHeadRnn ? 2 * nkb : nkb;   // A k-blocks (RNN: high parts, then low parts)
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + lay.bar_off);
    uint64_t *a_full = bars;                 // even CTA: both CTAs' A rows are in (one phase per position)
    uint64_t *b_full = a_full + 1;           // SB, even CTA: both halves of a B stage landed
    uint64_t *b_empty = b_full + SB;         // SB, each CTA: the pair's MMAs are done with the stage
    uint64_t *l_full = b_empty + SB;         // SL, local
    uint64_t *l_empty = l_full + SL;         // SL, local (4 warps, one per lane quarter)
    uint64_t *acc_full = l_empty + SL;       // 2, each CTA: an accumulator is complete
    uint64_t *acc_empty = acc_full + 2;      // 2, even CTA: both CTAs' 32 epilogue warps drained it
    uint64_t *drain = acc_empty + 2;         // 1, even CTA
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    __shared__ int epi_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = tc::cluster_ctarank();
    const bool even = rank == 0;
    const int B = ep.B, V = ep.V, nParts = ep.nParts, nPB = ep.nPB;
    WsHeader *hdr = ep.hdr;
    // Tile schedule of the pair (identical in both CTAs).
    const int cl = blockIdx.x >> 1, nCl = gridDim.x >> 1;
    const int pb = cl % nPB;
    const int m0 = (2 * pb + (int)rank) * kPM;
    const int first_tile = cl / nPB;
    const int tile_step = (nCl - pb + nPB - 1) / nPB;

    if (threadIdx.x == 0) {
        tc::mbar_init(a_full, 2);
        for (int q = 0; q < SB; ++q) { tc::mbar_init(&b_full[q], 1); tc::mbar_init(&b_empty[q], 1); }
        for (int q = 0; q < SL; ++q) { tc::mbar_init(&l_full[q], 1); tc::mbar_init(&l_empty[q], 4); }
        for (int q = 0; q < 2; ++q) { tc::mbar_init(&acc_full[q], 1); tc::mbar_init(&acc_empty[q], 2 * kPEpiWarps); }
        tc::mbar_init(drain, 1);
        *abort_flag = 0;
        tc::fence_barrier_init();
    }
    if (warp == 1) {
        tc::tmem_alloc_pair(tmem_slot, kPTmemCols);
        tc::tmem_relinquish_pair();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::cluster_sync();   // both CTAs' barriers and tensor memory exist before any cross-CTA use
    tc::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // The even CTA's barriers, as shared::cluster addresses.
    const uint32_t a_full0 = tc::mapa_shared(tc::smem_u32(a_full), 0);
    const uint32_t acc_empty0 = tc::mapa_shared(tc::smem_u32(acc_empty), 0);

    if (warp == 0) {
        // ------------------------------------------------------ B producer
        if (lane == 0) {
            tc::prefetch_tmap(&mapW);
            const uint64_t keep = tc::policy_evict_last();
            int g = 0;
            bool ok = true;
            for (int pos = 0; pos < ep.G && ok; ++pos) {
                for (int t = first_tile; t < nTilesN && ok; t += tile_step) {
                    const int n0 = t * kPBN + (int)rank * kPHalf;
                    for (int kb = 0; kb < nkb; ++kb, ++g) {
                        const int s = g % SB;
                        if (!tc::mbar_wait_bounded(&b_empty[s], ((g / SB) & 1) ^ 1, abort_flag, ep.budget)) {
                            ok = false;
                            break;
                        }
                        if (even) tc::mbar_arrive_expect_tx(&b_full[s], 2u * kPBStage);
                        tc::tma_load_2d_pair(sB + s * kPBStage, &mapW, tc::mapa_shared(tc::smem_u32(&b_full[s]), 0),
                                             kb * kPKB, n0, keep);
                    }
                }
            }
            if (!ok) flag_status(hdr, DSPARK_DEV_TIMEOUT);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer (even CTA)
        if (even && lane == 0) {
            const uint32_t idesc = tc::idesc_bf16_f32(2 * kPM, kPBN);
            const uint32_t a_addr = tc::smem_u32(sA), b_addr = tc::smem_u32(sB);
            bool ok = true;
            int g = 0, j = 0;
            for (int pos = 0; pos < ep.G && ok; ++pos) {
                ok = tc::mbar_wait_bounded(a_full, pos & 1, abort_flag, ep.budget);
                tc::tc_fence_after();
                for (int t = first_tile; t < nTilesN && ok; t += tile_step, ++j) {
                    const int ab = j & 1;
                    if (!tc::mbar_wait_bounded(&acc_empty[ab], ((j >> 1) & 1) ^ 1, abort_flag, ep.budget)) {
                        ok = false;
                        break;
                    }
                    tc::tc_fence_after();
                    const uint32_t d = tmem_base + ab * kPBN;
                    for (int kb = 0; kb < nkb; ++kb, ++g) {
                        const int s = g % SB;
                        if (!tc::mbar_wait_bounded(&b_full[s], (g / SB) & 1, abort_flag, ep.budget)) {
                            ok = false;
                            break;
                        }
                        tc::tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < kPKB / 16; ++kk) {
                            const uint64_t ad = tc::sw128_desc(a_addr + kb * kPABytes + kk * 32);
                            const uint64_t bd = tc::sw128_desc(b_addr + s * kPBStage + kk * 32);
                            tc::mma_bf16_pair(d, ad, bd, idesc, (kb | kk) != 0);
                            if (HEAD == kHeadRnn) {
                                const uint64_t al = tc::sw128_desc(a_addr + (nkb + kb) * kPABytes + kk * 32);
                                tc::mma_bf16_pair(d, al, bd, idesc, 1u);
                            }
                        }
                        const uint32_t be = tc::smem_u32(&b_empty[s]);
                        tc::mma_commit_pair(tc::mapa_shared(be, 0));
                        tc::mma_commit_pair(tc::mapa_shared(be, 1));
                    }
                    if (!ok) break;
                    const uint32_t af = tc::smem_u32(&acc_full[ab]);
                    tc::mma_commit_pair(tc::mapa_shared(af, 0));
                    tc::mma_commit_pair(tc::mapa_shared(af, 1));
                }
            }
            // Drain: every MMA issued above has completed once this arrives.
            tc::mma_commit_pair(tc::mapa_shared(tc::smem_u32(drain), 0));
            int dummy = 0;
            tc::mbar_wait_bounded(drain, 0, &dummy, kPWaitBudget / 4);
            if (!ok) flag_status(hdr, DSPARK_DEV_TIMEOUT);
        }
    } else if (warp == 2) {
        // ------------------------------------------------------ logit producer
        if (lane == 0) {
            tc::prefetch_tmap(&mapL);
            const uint64_t stream = tc::policy_evict_first();
            int g = 0;
            bool ok = true;
            for (int pos = 0; pos < ep.G && ok; ++pos) {
                for (int t = first_tile; t < nTilesN && ok; t += tile_step) {
                    for (int sg = 0; sg < kPSegs; ++sg, ++g) {
                        const int q = g % SL;
                        if (!tc::mbar_wait_bounded(&l_empty[q], ((g / SL) & 1) ^ 1, abort_flag, ep.budget)) {
                            ok = false;
                            break;
                        }
                        tc::mbar_arrive_expect_tx(&l_full[q], kPSegBytes);
                        tc::tma_load_3d(sL + q * kPSegBytes, &mapL, &l_full[q], t * kPBN + sg * kPSeg, pos, m0,
                                        stream);
                    }
                }
            }
            if (!ok) {
                int dummy = 0;
                volatile int *no_abort = &dummy;
                for (int q = 0; q < SL && g - 1 - q >= 0; ++q) {
                    const int gg = g - 1 - q;
                    tc::mbar_wait_bounded(&l_full[gg % SL], (gg / SL) & 1, no_abort, kPWaitBudget / 4);
                }
                flag_status(hdr, DSPARK_DEV_TIMEOUT);
            }
        }
    } else {
        // ------------------------------------------------------ epilogue
        const int ew = warp - kPEpi0;          // 0..15
        const int quarter = warp & 3;          // TMEM lane quarter this warp may access
        const int sg = ew >> 2;                // 64-column segment of every tile (0..3)
        const int row = quarter * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        const bool leader = ew == 0 && lane == 0;
        auto epi_sync = [&]() { asm volatile("bar.sync 1, %0;" ::"r"(kPEpiWarps * 32) : "memory"); };
        // This CTA's A rows are in: the even CTA's MMA counts one arrival per CTA.
        auto a_arrive = [&]() {
            if (even) tc::mbar_arrive(a_full);
            else tc::mbar_arrive_remote_release(a_full0);
        };
        const int b = m0 + row;
        const bool rowok = b < B;
        float invT = 0.f;
        if (rowok) {
            const float Tb = ep.temp[b];
            invT = Tb > 0.f ? 1.f / Tb : 0.f;
        }
        const float cexp = invT * kLog2e;
        const bool warp_greedy = __any_sync(0xffffffffu, rowok && invT == 0.f);
        const bool warp_soft = __any_sync(0xffffffffu, rowok && invT > 0.f);
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
        const int grp = ew >> 3;
        const Grp fg{(ew & 7) * 32 + lane, 256, ew & 7, 8, 2 + grp};
        FinScratch *fsc = reinterpret_cast<FinScratch *>(sA + grp * 4096);
        float *furow = reinterpret_cast<float *>(sA + 8192 + grp * 2048);

        // Position 0: the A rows gathered into the 128-byte-swizzled K-major
        // layout by the epilogue warps (k-blocks sg, sg + 4, ...): U[x_0]
        // (Markov head), or the first state h_1 = tanh(U[x_0]) split into
        // high and low bf16 parts (RNN head; the pairs on the first tiles also
        // write h_1 to the state output).
        {
            int prev = 0;
            if (rowok) {
                prev = ep.x0[b];
                if (prev < 0 || prev >= V) {
                    flag_status(hdr, DSPARK_DEV_TOKEN_RANGE);
                    prev = prev < 0 ? 0 : V - 1;
                }
            }
            const __nv_bfloat16 *urow = ep.U + (size_t)prev * r;
            for (int kb = sg; kb < nkb; kb += kPSegs) {
                uint4 v[8];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const int k = kb * kPKB + c * 8;
                    v[c] = (k < r) ? ld_nc16(urow + k) : make_uint4(0, 0, 0, 0);
                }
                unsigned char *dst = sA + kb * kPABytes + row * 128;
                if (HEAD == kHeadRnn) {
                    unsigned char *dlo = sA + (nkb + kb) * kPABytes + row * 128;
                    float *hrow = ep.fin.H + ((size_t)b * ep.G) * r + kb * kPKB;
                    const bool write_h = rowok && first_tile == 0;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint32_t w4[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
                        uint32_t hi4[4], lo4[4];
                        float h8[8];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float h0 = tanhf(bf16lo(w4[e])), h1 = tanhf(bf16hi(w4[e]));
                            const __nv_bfloat16 a0 = __float2bfloat16_rn(h0), a1 = __float2bfloat16_rn(h1);
                            const __nv_bfloat16 b0 = __float2bfloat16_rn(h0 - __bfloat162float(a0));
                            const __nv_bfloat16 b1 = __float2bfloat16_rn(h1 - __bfloat162float(a1));
                            hi4[e] = (uint32_t)__bfloat16_as_ushort(a0) | ((uint32_t)__bfloat16_as_ushort(a1) << 16);
                            lo4[e] = (uint32_t)__bfloat16_as_ushort(b0) | ((uint32_t)__bfloat16_as_ushort(b1) << 16);
                            h8[2 * e] = h0;
                            h8[2 * e + 1] = h1;
                        }
                        *reinterpret_cast<uint4 *>(dst + ((c ^ (row & 7)) << 4)) = make_uint4(hi4[0], hi4[1], hi4[2], hi4[3]);
                        *reinterpret_cast<uint4 *>(dlo + ((c ^ (row & 7)) << 4)) = make_uint4(lo4[0], lo4[1], lo4[2], lo4[3]);
                        if (write_h && kb * kPKB + c * 8 < r) {
                            *reinterpret_cast<float4 *>(hrow + c * 8) = make_float4(h8[0], h8[1], h8[2], h8[3]);
                            *reinterpret_cast<float4 *>(hrow + c * 8 + 4) = make_float4(h8[4], h8[5], h8[6], h8[7]);
                        }
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4 *>(dst + ((c ^ (row & 7)) << 4)) = v[c];
                }
            }
            tc::fence_proxy_async_smem();
            epi_sync();
            if (leader) a_arrive();
        }

        const uint32_t nblk = gridDim.x;
        int j = 0;
        for (int pos = 0; pos < ep.G; ++pos) {
            for (int t = first_tile; t < nTilesN; t += tile_step, ++j) {
                const int ab = j & 1;
                const int gl = j * kPSegs + sg, q = gl % SL;
                bool ok = tc::mbar_wait_bounded(&l_full[q], (gl / SL) & 1, abort_flag, ep.budget);
                ok = ok && tc::mbar_wait_bounded(&acc_full[ab], (j >> 1) & 1, abort_flag, ep.budget);
                if (!__all_sync(0xffffffffu, ok)) break;
                tc::tc_fence_after();
                const unsigned char *lsrc = sL + q * kPSegBytes + row * 128;
                uint4 cur[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) cur[u] = *reinterpret_cast<const uint4 *>(lsrc + ((u ^ (row & 7)) << 4));
                tc::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&l_empty[q]);
                const uint32_t taddr = tmem_base + lane_addr + ab * kPBN + sg * kPSeg;
                const int cbase = t * kPBN + sg * kPSeg;
                const bool whole = cbase + kPSeg <= V;
                // Both 32-column halves of the segment's accumulator in one round trip.
                uint32_t yr[2][32];
                tc::tmem_ld32_nowait(taddr, yr[0]);
                tc::tmem_ld32_nowait(taddr + 32, yr[1]);
                tc::tmem_ld_wait();
                // The accumulator is in registers: hand it back to the MMA.
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive_remote(acc_empty0 + ab * 8);
                float m = -INFINITY, s = 0.f;
                int am = 0x7fffffff;
#pragma unroll
                for (int c = 0; c < kPSeg / 32; ++c) {
                    float y[32];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const uint4 qv = cur[c * 4 + u];
                        const uint32_t wq[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
                        for (int h = 0; h < 4; ++h) {
                            const float2 yy = add2(make_float2(__uint_as_float(yr[c][u * 8 + 2 * h]),
                                                               __uint_as_float(yr[c][u * 8 + 2 * h + 1])),
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
                        const float2 c2 = make_float2(cexp, cexp);
                        const float nmc = -mn * cexp;
                        const float2 n2 = make_float2(nmc, nmc);
                        float2 s2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                                        make_float2(0.f, 0.f)};
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
                const int p = t * kPSegs + sg;
                if (rowok && p < nParts) {
                    const size_t o = (size_t)b * nParts + p;
                    // One 8-byte record: the finalize reads Z's terms for a sampled row,
                    // the argmax for a greedy one.
                    ep.part[o] = make_float2(m, invT > 0.f ? s : __int_as_float(am));
                }
            }
            if (!grid_sync(nblk * (2u * pos + 1u))) break;
            for (int bb = (int)blockIdx.x * 2 + grp; bb < B; bb += 2 * (int)nblk)
                finalize_row<__nv_bfloat16>(fg, fsc, furow, ep.fin, bb, pos);
            tc::fence_proxy_async_all();
            if (!grid_sync(nblk * (2u * pos + 2u))) break;
            if (pos + 1 < ep.G && leader) {
                // The next position's A rows: this CTA's staged U[x_pos] rows,
                // counted on the even CTA's barrier (it expects both halves).
                tc::fence_proxy_async_all();
                const uint64_t once = tc::policy_evict_first();
                if (even) tc::mbar_arrive_expect_tx(a_full, 2u * (uint32_t)na * kPABytes);
                for (int kb = 0; kb < nkb; ++kb) {
                    tc::tma_load_2d_pair(sA + kb * kPABytes, &mapE, a_full0, kb * kPKB, m0, once);
                    if (HEAD == kHeadRnn)   // the low parts sit B rows below the high parts
                        tc::tma_load_2d_pair(sA + (nkb + kb) * kPABytes, &mapE, a_full0, kb * kPKB, B + m0, once);
                }
                if (!even) tc::mbar_arrive_remote_release(a_full0);
            }
        }
    }

    // A CTA that gave up lets its copies in flight land (some complete on the
    // other CTA's barriers, so they are not waited for one by one).
    if (threadIdx.x == 0 && *abort_flag) {
        const long long t0 = clock64();
        while (clock64() - t0 < kPDrainCycles) __nanosleep(1000);
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::cluster_sync();   // the pair's MMAs, commits and remote arrivals are all done
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc_pair(tmem_base, kPTmemCols);
    }
}

// ------------------------------------------------------------------ host
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn pair_encode_fn() {
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

// 2-D bf16 map of a [rows, r] row-major matrix in 64 x `box_rows` boxes,
// 128-byte swizzle, out-of-range reads as zero.
bool pair_map_2d(CUtensorMap *m, const void *base, int rows, int r, int box_rows) {
    EncodeTiledFn fn = pair_encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[2] = {(cuuint64_t)r, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)r * 2};
    cuuint32_t box[2] = {kPKB, (cuuint32_t)box_rows};
    cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool pair_map_logits(CUtensorMap *m, const void *L, int B, int G, int V) {
    EncodeTiledFn fn = pair_encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[3] = {(cuuint64_t)V, (cuuint64_t)G, (cuuint64_t)B};
    cuuint64_t strides[2] = {(cuuint64_t)V * 2, (cuuint64_t)G * V * 2};
    cuuint32_t box[3] = {kPSeg, 1, kPM};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(L), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int HEAD>
cudaError_t launch_pair(const DraftArgs &a, const DraftWs &w, const FinArgs &f, cudaStream_t st) {
    PairEpi ep{};
    ep.temp = a.temp; ep.B = a.B; ep.G = a.G; ep.V = a.V; ep.nParts = w.nTiles; ep.hdr = w.hdr;
    ep.budget = wait_budget(kPWaitBudget);
    ep.fin = f;
    ep.grid_count = &w.hdr->pad[2];
    ep.U = static_cast<const __nv_bfloat16 *>(a.U);
    ep.x0 = a.x0;
    ep.part = w.part;
    const int nMB = (a.B + kPM - 1) / kPM;
    ep.nPB = (nMB + 1) / 2;
    CUtensorMap mW, mL, mE;
    if (!pair_map_2d(&mW, a.Wt, a.V, a.r, kPHalf)) return cudaErrorInvalidValue;
    if (!pair_map_logits(&mL, a.L, a.B, a.G, a.V)) return cudaErrorInvalidValue;
    if (a.G > 1) {
        // The staged rows: B (Markov head) or 2B (RNN head: high, then low parts).
        if (!pair_map_2d(&mE, w.E, HEAD == kHeadRnn ? 2 * a.B : a.B, a.r, kPM)) return cudaErrorInvalidValue;
    } else {
        mE = mW;   // unused
    }
    const PairLayout lay = pair_layout(a.r, HEAD);
    cudaError_t e = cudaFuncSetAttribute(markov_pair_tc<HEAD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)lay.total);
    if (e != cudaSuccess) return e;
    const int nTilesN = (a.V + kPBN - 1) / kPBN;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kPThreads);
    cfg.dynamicSmemBytes = lay.total;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // Every CTA must be resident for the grid barriers: at most as many
    // pairs as fit on the GPU at once (a GPC with an odd SM count leaves one
    // SM without a partner).
    int maxc = 0;
    cfg.gridDim = dim3(2);
    if ((e = cudaOccupancyMaxActiveClusters(&maxc, markov_pair_tc<HEAD>, &cfg)) != cudaSuccess) return e;
    if (maxc < ep.nPB) return cudaErrorCooperativeLaunchTooLarge;
    const int pairs = std::max(ep.nPB, std::min(maxc, ep.nPB * nTilesN));
    cfg.gridDim = dim3(2 * pairs);
    if ((e = cudaMemsetAsync(ep.grid_count, 0, sizeof(uint32_t), st)) != cudaSuccess) return e;
    // A plain cluster launch: the grid fits the GPU at once by the check
    // above, and every CTA waits on the grid barriers with a bounded spin.
    return cudaLaunchKernelEx(&cfg, markov_pair_tc<HEAD>, mW, mL, mE, a.r, nTilesN, ep);
}

}  // namespace

cudaError_t launch_draft_pair(const DraftArgs &a, const DraftWs &w, const FinArgs &f, cudaStream_t st) {
    return f.H != nullptr ? launch_pair<kHeadRnn>(a, w, f, st) : launch_pair<kHeadMarkov>(a, w, f, st);
}

}  // namespace dspark
