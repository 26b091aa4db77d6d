// draft_tc.cu -- tensor-core (tcgen05 / TMEM / TMA) Markov-bias tile kernel
// for bf16 rounds, fused with the drafting softmax epilogue (and, in a second
// mode, with the residual mass of verification).
//
// Method (paperlayer.ai summary of DSpark, §3.1; menfem.com KB entry,
// "Methodology": rank-256 factorisation; llm-wiki.hwlabs.dev study 116,
// draft-generation figure): Delta_i = E_i W with E_i[b] = U[x_{i-1}[b]], added
// to the backbone logits L[i] before the temperature softmax.
//
// Persistent, warp-specialised CTA (one per SM), 320 threads, 512 TMEM columns:
//   warp 0      TMA producer of the B operand: per 128-column tile the
//               transition-factor tile Wt[n0:n0+128, :] through a ring of
//               k-block stages (128-byte swizzle, evict-last: W is reused by
//               every position and m-block).
//   warp 1      TMEM owner and MMA issuer: 128 x 128 x 16 bf16 MMAs with the A
//               operand read from TMEM (the CTA's 128 gathered U rows, written
//               there once) into one of two fp32 accumulators.
//   warps 2-9   epilogue: first they copy the A rows into TMEM (lane = row),
//               then each thread owns one row and one 64-column half of every
//               tile: Delta from TMEM, its row's logits straight from global
//               memory (loaded one tile ahead), and the 64-column partials.
// Shared memory only carries the B ring, so the MMA's operand fetch does not
// compete with the logit stream.  Delta never leaves the SM.  Every mbarrier
// wait is bounded by a clock budget; on expiry the CTA raises a timeout bit in
// the status word, drains its own copies and MMAs, frees TMEM and returns.
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"
#include "tc.cuh"

namespace dspark {

namespace {

constexpr int kM = 128;            // rows (requests) per CTA
constexpr int kBN = 128;           // MMA N: columns per tile
constexpr int kPartN = 64;         // partial granularity: columns per epilogue warp
constexpr int kKB = 64;            // bf16 elements per 128-byte k-block
constexpr int kStageBytes = kBN * 128;        // one k-block of the B tile
constexpr int kStages = 8;                    // B ring depth (two tiles at r = 256)
constexpr int kThreads = 320;
constexpr int kEpiWarp0 = 2;       // first epilogue warp
constexpr int kTmemCols = 512;     // A (r/2 columns, <= 256) + two 128-column accumulators
constexpr int kAccCol0 = 256;
constexpr long long kWaitBudget = 4000000000LL;  // ~2 s of SM clock

constexpr uint32_t kSmemBytes = kStages * kStageBytes + 256 + 1024;  // ring + barriers + base alignment

// Epilogue modes: drafting partials, or residual mass for verification.
enum { kEpiDraft = 0, kEpiResidual = 1 };

struct TcEpi {
    const float *temp;
    int B, G, V, pos, nParts;
    WsHeader *hdr;
    const __nv_bfloat16 *E;   // [round_up(B,128), r] A-operand rows
    const __nv_bfloat16 *L;   // drafting and residual: backbone logits [B, G, V]
    // drafting: 64-column partials per request row
    float *part_m, *part_s;
    int32_t *part_a;
    // residual: rows are the queued rejections; per 64 columns the sum of
    // max(0, p_t - p_d) with p_d rebuilt from L + Delta and the drafting stats
    const uint32_t *nrows;
    const int32_t *res_b, *res_k;
    const float *res_mt, *res_zt, *rowmax, *rowsum;
    const __nv_bfloat16 *Tlog;
    float *rp;
};

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1) markov_tile_tc(const __grid_constant__ CUtensorMap mapW, int r,
                                                              int nTilesN, const TcEpi ep)
{
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw_u32 = tc::smem_u32(smem_raw);
    unsigned char *base = smem_raw + (((raw_u32 + 1023) & ~1023u) - raw_u32);
    unsigned char *sB = base;
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + kStages * kStageBytes);
    uint64_t *a_full = bars;                       // 8 epilogue-warp arrivals: A is in TMEM
    uint64_t *b_full = bars + 1;                   // kStages
    uint64_t *b_empty = b_full + kStages;          // kStages
    uint64_t *acc_full = b_empty + kStages;        // 2
    uint64_t *acc_empty = acc_full + 2;            // 2
    uint64_t *drain = acc_empty + 2;               // 1
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int B = ep.B, V = ep.V, nParts = ep.nParts;
    WsHeader *hdr = ep.hdr;
    const int nMB = (B + kM - 1) / kM;
    const int mb = blockIdx.x % nMB;
    const int m0 = mb * kM;
    const int first_tile = blockIdx.x / nMB;
    const int tile_step = ((int)gridDim.x - mb + nMB - 1) / nMB;
    const int nkb = (r + kKB - 1) / kKB;
    // Residual rows are counted on the device: m-blocks past the count leave now.
    const int nrows = (MODE == kEpiResidual) ? (int)*reinterpret_cast<const volatile uint32_t *>(ep.nrows) : B;
    if (m0 >= nrows) return;

    if (threadIdx.x == 0) {
        tc::mbar_init(a_full, 8);
        for (int s = 0; s < kStages; ++s) { tc::mbar_init(&b_full[s], 1); tc::mbar_init(&b_empty[s], 1); }
        for (int q = 0; q < 2; ++q) { tc::mbar_init(&acc_full[q], 1); tc::mbar_init(&acc_empty[q], 8); }
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
            for (int t = first_tile; t < nTilesN && ok; t += tile_step) {
                const int n0 = t * kBN;
                for (int kb = 0; kb < nkb; ++kb, ++g) {
                    const int s = g % kStages;
                    if (!tc::mbar_wait_bounded(&b_empty[s], ((g / kStages) & 1) ^ 1, abort_flag, kWaitBudget)) {
                        ok = false;
                        break;
                    }
                    tc::mbar_arrive_expect_tx(&b_full[s], kStageBytes);
                    tc::tma_load_2d(sB + s * kStageBytes, &mapW, &b_full[s], kb * kKB, n0, keep);
                }
            }
            if (!ok) {
                // Give up: wait (bounded, ignoring the abort flag) for every copy
                // this thread issued so that none lands after the CTA exits.
                int dummy = 0;
                volatile int *no_abort = &dummy;
                for (int q = 0; q < kStages && g - 1 - q >= 0; ++q) {
                    const int gg = g - 1 - q;
                    tc::mbar_wait_bounded(&b_full[gg % kStages], (gg / kStages) & 1, no_abort, kWaitBudget / 4);
                }
                flag_status(hdr, DSPARK_DEV_TIMEOUT);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = tc::idesc_bf16_f32(kM, kBN);
            const uint32_t b_addr = tc::smem_u32(sB);
            bool ok = tc::mbar_wait_bounded(a_full, 0, abort_flag, kWaitBudget);
            tc::tc_fence_after();
            int g = 0, j = 0;
            for (int t = first_tile; t < nTilesN && ok; t += tile_step, ++j) {
                const int ab = j & 1;
                if (!tc::mbar_wait_bounded(&acc_empty[ab], ((j >> 1) & 1) ^ 1, abort_flag, kWaitBudget)) {
                    ok = false;
                    break;
                }
                tc::tc_fence_after();
                const uint32_t d = tmem_base + kAccCol0 + ab * kBN;
                for (int kb = 0; kb < nkb; ++kb, ++g) {
                    const int s = g % kStages;
                    if (!tc::mbar_wait_bounded(&b_full[s], (g / kStages) & 1, abort_flag, kWaitBudget)) {
                        ok = false;
                        break;
                    }
                    tc::tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < kKB / 16; ++kk) {
                        const uint32_t a = tmem_base + kb * (kKB / 2) + kk * 8;   // 16 bf16 = 8 columns
                        const uint64_t bd = tc::sw128_desc(b_addr + s * kStageBytes + kk * 32);
                        tc::mma_bf16_ts(d, a, bd, idesc, (kb | kk) != 0);
                    }
                    tc::mma_commit(&b_empty[s]);
                }
                if (!ok) break;
                tc::mma_commit(&acc_full[ab]);
            }
            // Drain: every MMA issued above has completed once this arrives.
            tc::mma_commit(drain);
            int dummy = 0;
            tc::mbar_wait_bounded(drain, 0, &dummy, kWaitBudget / 4);
            if (!ok) flag_status(hdr, DSPARK_DEV_TIMEOUT);
        }
    } else {
        const int ew = warp - kEpiWarp0;
        const int quarter = warp & 3;          // TMEM lane quarter this warp may access
        const int half = ew >> 2;              // which 64-column half of every tile
        const int row = quarter * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        // ---------------------------------------------- A operand into TMEM
        // Row m0 + row of E; this warp writes the k-blocks kb = half, half+2, ...
        // (zeros past r), 32 columns per k-block.
        {
            const __nv_bfloat16 *erow = ep.E + (size_t)(m0 + row) * r;
            for (int kb = half; kb < nkb; kb += 2) {
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    uint32_t v[16];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int k = kb * kKB + h2 * 32 + q * 8;
                        uint4 x = make_uint4(0, 0, 0, 0);
                        if (k < r) x = ld_nc16(erow + k);
                        v[q * 4 + 0] = x.x; v[q * 4 + 1] = x.y; v[q * 4 + 2] = x.z; v[q * 4 + 3] = x.w;
                    }
                    tc::tmem_st16(tmem_base + lane_addr + kb * (kKB / 2) + h2 * 16, v);
                }
            }
            tc::tmem_st_wait();
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(a_full);
        }
        if (MODE == kEpiDraft) {
            // ------------------------------------------ drafting epilogue
            // One online pass per 32-column chunk: y = L + Delta, chunk max,
            // then the running sum of exp((y - max) / T), rescaled when the
            // max grows.  The lowest argmax is tracked only in warps holding a
            // greedy row.  The row's logits for the next tile are loaded
            // before waiting on this tile's accumulator.
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
            const __nv_bfloat16 *lrow = ep.L + ((size_t)(rowok ? b : 0) * ep.G + ep.pos) * V;
            uint4 lq[8];
            auto load_l = [&](int t) {
                const int cb = t * kBN + half * kPartN;
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int c8 = cb + u * 8;
                    lq[u] = (rowok && c8 < V) ? ld_nc16(lrow + c8) : make_uint4(0, 0, 0, 0);
                }
            };
            if (first_tile < nTilesN) load_l(first_tile);
            int j = 0;
            for (int t = first_tile; t < nTilesN; t += tile_step, ++j) {
                const int ab = j & 1;
                const uint32_t ph = (j >> 1) & 1;
                uint4 cur[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) cur[u] = lq[u];
                if (t + tile_step < nTilesN) load_l(t + tile_step);
                // Every lane waits; the vote keeps the warp converged for the
                // warp-collective TMEM loads below even if the budget runs out.
                const bool ok = tc::mbar_wait_bounded(&acc_full[ab], ph, abort_flag, kWaitBudget);
                if (!__all_sync(0xffffffffu, ok)) break;
                tc::tc_fence_after();
                const uint32_t taddr = tmem_base + lane_addr + kAccCol0 + ab * kBN + half * kPartN;
                const int cbase = t * kBN + half * kPartN;
                const bool whole = cbase + kPartN <= V;   // no column of this half lies past V
                float m = -INFINITY, s = 0.f;
                int am = 0x7fffffff;
#pragma unroll
                for (int c = 0; c < kPartN / 32; ++c) {
                    float y[32];
                    tc::tmem_ld32(taddr + c * 32, y);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const uint4 q = cur[c * 4 + u];
                        y[u * 8 + 0] += bf16lo(q.x); y[u * 8 + 1] += bf16hi(q.x);
                        y[u * 8 + 2] += bf16lo(q.y); y[u * 8 + 3] += bf16hi(q.y);
                        y[u * 8 + 4] += bf16lo(q.z); y[u * 8 + 5] += bf16hi(q.z);
                        y[u * 8 + 6] += bf16lo(q.w); y[u * 8 + 7] += bf16hi(q.w);
                    }
                    if (!whole) {
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (cbase + c * 32 + e >= V) y[e] = -INFINITY;
                    }
                    float cm = y[0];
#pragma unroll
                    for (int e = 1; e < 32; ++e) cm = fmaxf(cm, y[e]);
                    if (warp_greedy && cm > m) {
                        int ix = 0x7fffffff;
#pragma unroll
                        for (int e = 31; e >= 0; --e)
                            if (y[e] == cm) ix = e;
                        am = cbase + c * 32 + ix;
                    }
                    const float mn = fmaxf(m, cm);
                    if (warp_soft) {
                        float acc = 0.f;
#pragma unroll
                        for (int e = 0; e < 32; ++e) acc += fast_exp2((y[e] - mn) * cexp);
                        s = (m == -INFINITY ? 0.f : s * fast_exp2((m - mn) * cexp)) + acc;
                    }
                    m = mn;
                }
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&acc_empty[ab]);
                const int p = t * (kBN / kPartN) + half;
                if (rowok && p < nParts) {
                    const size_t o = (size_t)b * nParts + p;
                    ep.part_m[o] = m;
                    ep.part_s[o] = s;
                    ep.part_a[o] = am;
                }
            }
        } else {
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
                const uint32_t ph = (j >> 1) & 1;
                const int cbase = t * kBN + half * kPartN;
                // Issue this row's logit loads before waiting on the accumulator.
                uint4 lq[8], tq[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int c8 = cbase + u * 8;
                    if (rowok && c8 < V) {
                        lq[u] = ld_nc16(Lrow + c8);
                        tq[u] = ld_nc16(Trow + c8);
                    } else {
                        lq[u] = make_uint4(0, 0, 0, 0);
                        tq[u] = make_uint4(0, 0, 0, 0);
                    }
                }
                const bool ok = tc::mbar_wait_bounded(&acc_full[ab], ph, abort_flag, kWaitBudget);
                if (!__all_sync(0xffffffffu, ok)) break;
                tc::tc_fence_after();
                const uint32_t taddr = tmem_base + lane_addr + kAccCol0 + ab * kBN + half * kPartN;
                float qs = 0.f;
#pragma unroll
                for (int c = 0; c < kPartN / 32; ++c) {
                    float d[32];
                    tc::tmem_ld32(taddr + c * 32, d);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const uint4 a = lq[c * 4 + u], bq = tq[c * 4 + u];
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
                const int p = t * (kBN / kPartN) + half;
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
    cuuint32_t box[2] = {kKB, kBN};
    cuuint32_t es[2] = {1, 1};
    CUresult res = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(Wt), dims, strides, box, es,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return res == CUDA_SUCCESS;
}

template <int MODE>
cudaError_t launch_markov_tc(const void *Wt, int r, const TcEpi &ep, cudaStream_t st) {
    CUtensorMap mW;
    if (!map_factor(&mW, Wt, ep.V, r)) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(markov_tile_tc<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int nTilesN = (ep.V + kBN - 1) / kBN;
    const int nMB = (ep.B + kM - 1) / kM;
    int grid = std::min(sms, nMB * nTilesN);
    grid = std::max(grid, nMB);
    markov_tile_tc<MODE><<<grid, kThreads, kSmemBytes, st>>>(mW, r, nTilesN, ep);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_draft_tile_tc(const DraftArgs &a, const DraftWs &w, int pos, cudaStream_t st) {
    TcEpi ep{};
    ep.temp = a.temp; ep.B = a.B; ep.G = a.G; ep.V = a.V; ep.pos = pos; ep.nParts = w.nTiles; ep.hdr = w.hdr;
    ep.E = w.E; ep.L = static_cast<const __nv_bfloat16 *>(a.L);
    ep.part_m = w.part_m; ep.part_s = w.part_s; ep.part_a = w.part_a;
    return launch_markov_tc<kEpiDraft>(a.Wt, a.r, ep, st);
}

cudaError_t launch_residual_tile_tc(const ResidualTcArgs &a, cudaStream_t st) {
    TcEpi ep{};
    ep.temp = a.temp; ep.B = a.B; ep.G = a.G; ep.V = a.V; ep.pos = 0; ep.nParts = a.nParts; ep.hdr = a.hdr;
    ep.E = a.E; ep.L = a.L;
    ep.nrows = a.nrows; ep.res_b = a.res_b; ep.res_k = a.res_k; ep.res_mt = a.res_mt; ep.res_zt = a.res_zt;
    ep.rowmax = a.rowmax; ep.rowsum = a.rowsum; ep.Tlog = a.Tlog; ep.rp = a.rp;
    return launch_markov_tc<kEpiResidual>(a.Wt, a.r, ep, st);
}

}  // namespace dspark
