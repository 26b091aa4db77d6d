// draft_tc.cu -- tensor-core (tcgen05 / TMEM / TMA) Markov-bias tile kernel
// for bf16 rounds, fused with the drafting softmax epilogue.
//
// Method (paperlayer.ai summary of DSpark, §3.1; menfem.com KB entry,
// "Methodology": rank-256 factorisation; llm-wiki.hwlabs.dev study 116,
// draft-generation figure): Delta_i = E_i W with E_i[b] = U[x_{i-1}[b]], added
// to the backbone logits L[i] before the temperature softmax.
//
// Persistent, warp-specialised CTA (one per SM), 352 threads:
//   warp 0      TMA producer of the operands: the CTA's 128 gathered U rows
//               (A operand, kept resident), then per 128-column tile the
//               transition-factor tile Wt[n0:n0+128, :] (B operand) through
//               a ring of k-block stages (evict-last: W is reused by every
//               position and m-block).
//   warp 1      TMEM owner and MMA issuer: 128 x 128 x 16 bf16 MMAs into one
//               of two fp32 accumulators (256 TMEM columns), committed to the
//               stage-empty and accumulator-full barriers.
//   warp 2      TMA producer of the 128 x 128 slices of L[:, i, :]
//               (double-buffered, evict-first), independent of the B ring.
//   warps 3-10  epilogue: each thread owns one row (TMEM lane) and one half
//               (64 columns) of the tile; reads Delta from TMEM and L from the
//               swizzled shared tile, and writes the 64-column partials of
//               y = L + Delta: max, lowest argmax and sum of exp((y - max)/T).
// Delta never leaves the SM.  Every mbarrier wait is bounded by a clock
// budget; on expiry the CTA raises a timeout bit in the status word, drains
// its own copies and MMAs, frees TMEM and returns.
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
constexpr int kABlockBytes = kM * 128;        // one k-block of the A tile
constexpr int kLBufBytes = kM * kBN * 2;      // one L tile
constexpr int kThreads = 352;      // B producer, MMA, L producer, 8 epilogue warps
constexpr int kEpiWarp0 = 3;       // first epilogue warp
constexpr int kTmemCols = 2 * kBN;
constexpr long long kWaitBudget = 4000000000LL;  // ~2 s of SM clock

struct TcSmem {
    int nkb, stages;
    uint32_t a_off, b_off, l_off, bar_off, total;
};

__host__ __device__ inline TcSmem tc_layout(int r) {
    TcSmem s;
    s.nkb = (r + kKB - 1) / kKB;
    s.stages = s.nkb <= 4 ? 6 : 2;
    s.a_off = 0;
    s.b_off = s.a_off + s.nkb * kABlockBytes;
    s.l_off = s.b_off + s.stages * kStageBytes;
    s.bar_off = s.l_off + 2 * kLBufBytes;
    s.total = s.bar_off + 256 + 1024;  // barriers + 1024 for aligning the base
    return s;
}

// Epilogue modes: drafting partials, or residual mass for verification.
enum { kEpiDraft = 0, kEpiResidual = 1 };

struct TcEpi {
    const float *temp;
    int B, G, V, pos, nParts;
    WsHeader *hdr;
    // drafting: 64-column partials per request row
    float *part_m, *part_s;
    int32_t *part_a;
    // residual: rows are the queued rejections; per 64 columns the sum of
    // max(0, p_t - p_d) with p_d rebuilt from L + Delta and the drafting stats
    const uint32_t *nrows;
    const int32_t *res_b, *res_k;
    const float *res_mt, *res_zt, *rowmax, *rowsum;
    const __nv_bfloat16 *L, *Tlog;
    float *rp;
};

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1) markov_tile_tc(
    const __grid_constant__ CUtensorMap mapE, const __grid_constant__ CUtensorMap mapW,
    const __grid_constant__ CUtensorMap mapL, int r, int nTilesN, const TcEpi ep)
{
    extern __shared__ unsigned char smem_raw[];
    const TcSmem lay = tc_layout(r);
    const uint32_t raw_u32 = tc::smem_u32(smem_raw);
    unsigned char *base = smem_raw + (((raw_u32 + 1023) & ~1023u) - raw_u32);
    unsigned char *sA = base + lay.a_off;
    unsigned char *sB = base + lay.b_off;
    unsigned char *sL = base + lay.l_off;
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + lay.bar_off);
    uint64_t *a_full = bars;                       // 1
    uint64_t *b_full = bars + 1;                   // stages
    uint64_t *b_empty = b_full + lay.stages;       // stages
    uint64_t *l_full = b_empty + lay.stages;       // 2
    uint64_t *l_empty = l_full + 2;                // 2
    uint64_t *acc_full = l_empty + 2;              // 2
    uint64_t *acc_empty = acc_full + 2;            // 2
    uint64_t *drain = acc_empty + 2;               // 1
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int B = ep.B, V = ep.V, pos = ep.pos, nParts = ep.nParts;
    WsHeader *hdr = ep.hdr;
    const int nMB = (B + kM - 1) / kM;
    const int mb = blockIdx.x % nMB;
    const int m0 = mb * kM;
    const int first_tile = blockIdx.x / nMB;
    const int tile_step = ((int)gridDim.x - mb + nMB - 1) / nMB;
    const int S = lay.stages;
    const int nkb = lay.nkb;
    // Residual rows are counted on the device: m-blocks past the count leave now.
    const int nrows = (MODE == kEpiResidual) ? (int)*reinterpret_cast<const volatile uint32_t *>(ep.nrows) : B;
    if (m0 >= nrows) return;

    if (threadIdx.x == 0) {
        tc::mbar_init(a_full, 1);
        for (int s = 0; s < S; ++s) { tc::mbar_init(&b_full[s], 1); tc::mbar_init(&b_empty[s], 1); }
        for (int q = 0; q < 2; ++q) {
            tc::mbar_init(&l_full[q], 1);
            tc::mbar_init(&l_empty[q], 8);
            tc::mbar_init(&acc_full[q], 1);
            tc::mbar_init(&acc_empty[q], 8);
        }
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
        // ------------------------------------------------------ operand producer
        if (lane == 0) {
            tc::prefetch_tmap(&mapE);
            tc::prefetch_tmap(&mapW);
            const uint64_t keep = tc::policy_evict_last();
            tc::mbar_arrive_expect_tx(a_full, nkb * kABlockBytes);
            for (int kb = 0; kb < nkb; ++kb)
                tc::tma_load_2d(sA + kb * kABlockBytes, &mapE, a_full, kb * kKB, m0, keep);
            int g = 0;
            bool ok = true;
            for (int t = first_tile; t < nTilesN && ok; t += tile_step) {
                const int n0 = t * kBN;
                for (int kb = 0; kb < nkb; ++kb, ++g) {
                    const int s = g % S;
                    if (!tc::mbar_wait_bounded(&b_empty[s], ((g / S) & 1) ^ 1, abort_flag, kWaitBudget)) {
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
                for (int q = 0; q < S && g - 1 - q >= 0; ++q) {
                    const int gg = g - 1 - q;
                    tc::mbar_wait_bounded(&b_full[gg % S], (gg / S) & 1, no_abort, kWaitBudget / 4);
                }
                tc::mbar_wait_bounded(a_full, 0, no_abort, kWaitBudget / 4);
                flag_status(hdr, DSPARK_DEV_TIMEOUT);
            }
        }
    } else if (warp == 2) {
        // ------------------------------------------------------ logit producer
        if (MODE == kEpiDraft && lane == 0) {
            tc::prefetch_tmap(&mapL);
            const uint64_t stream = tc::policy_evict_first();
            int j = 0;
            bool ok = true;
            for (int t = first_tile; t < nTilesN; t += tile_step, ++j) {
                const int n0 = t * kBN;
                const int lb = j & 1;
                if (!tc::mbar_wait_bounded(&l_empty[lb], ((j >> 1) & 1) ^ 1, abort_flag, kWaitBudget)) {
                    ok = false;
                    break;
                }
                tc::mbar_arrive_expect_tx(&l_full[lb], kLBufBytes);
                tc::tma_load_3d(sL + lb * kLBufBytes, &mapL, &l_full[lb], n0, pos, m0, stream);
                tc::tma_load_3d(sL + lb * kLBufBytes + kLBufBytes / 2, &mapL, &l_full[lb], n0 + kPartN, pos, m0,
                                stream);
            }
            if (!ok) {
                int dummy = 0;
                volatile int *no_abort = &dummy;
                for (int q = 0; q < 2 && j - 1 - q >= 0; ++q) {
                    const int jj = j - 1 - q;
                    tc::mbar_wait_bounded(&l_full[jj & 1], (jj >> 1) & 1, no_abort, kWaitBudget / 4);
                }
                flag_status(hdr, DSPARK_DEV_TIMEOUT);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = tc::idesc_bf16_f32(kM, kBN);
            const uint32_t a_addr = tc::smem_u32(sA), b_addr = tc::smem_u32(sB);
            bool ok = tc::mbar_wait_bounded(a_full, 0, abort_flag, kWaitBudget);
            int g = 0, j = 0;
            for (int t = first_tile; t < nTilesN && ok; t += tile_step, ++j) {
                const int ab = j & 1;
                if (!tc::mbar_wait_bounded(&acc_empty[ab], ((j >> 1) & 1) ^ 1, abort_flag, kWaitBudget)) {
                    ok = false;
                    break;
                }
                tc::tc_fence_after();
                const uint32_t d = tmem_base + ab * kBN;
                for (int kb = 0; kb < nkb; ++kb, ++g) {
                    const int s = g % S;
                    if (!tc::mbar_wait_bounded(&b_full[s], (g / S) & 1, abort_flag, kWaitBudget)) {
                        ok = false;
                        break;
                    }
                    tc::tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < kKB / 16; ++kk) {
                        const uint64_t ad = tc::sw128_desc(a_addr + kb * kABlockBytes + kk * 32);
                        const uint64_t bd = tc::sw128_desc(b_addr + s * kStageBytes + kk * 32);
                        tc::mma_bf16(d, ad, bd, idesc, (kb | kk) != 0);
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
    } else if (MODE == kEpiDraft) {
        // ------------------------------------------------------ drafting epilogue
        // One online pass per 32-column chunk: y = L + Delta, chunk max, then
        // the running sum of exp((y - max) / T) rescaled when the max grows.
        // The lowest argmax is tracked only in warps that hold a greedy row.
        const int ew = warp - kEpiWarp0;
        const int quarter = warp & 3;          // TMEM lane quarter this warp may access
        const int half = ew >> 2;              // which 64-column half of the tile
        const int row = quarter * 32 + lane;
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
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        int j = 0;
        for (int t = first_tile; t < nTilesN; t += tile_step, ++j) {
            const int ab = j & 1, lb = j & 1;
            const uint32_t ph = (j >> 1) & 1;
            // Every lane waits; the vote keeps the warp converged for the
            // warp-collective TMEM loads below even if the budget runs out.
            bool ok = tc::mbar_wait_bounded(&acc_full[ab], ph, abort_flag, kWaitBudget);
            ok = ok && tc::mbar_wait_bounded(&l_full[lb], ph, abort_flag, kWaitBudget);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc::tc_fence_after();
            const uint32_t taddr = tmem_base + lane_addr + ab * kBN + half * kPartN;
            const unsigned char *lrow = sL + lb * kLBufBytes + half * (kLBufBytes / 2) + row * 128;
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
                    const int chunk = (c * 4 + u) ^ (row & 7);
                    const uint4 q = *reinterpret_cast<const uint4 *>(lrow + chunk * 16);
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
            tc::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                tc::mbar_arrive(&acc_empty[ab]);
                tc::mbar_arrive(&l_empty[lb]);
            }
            const int p = t * (kBN / kPartN) + half;
            if (rowok && p < nParts) {
                const size_t o = (size_t)b * nParts + p;
                ep.part_m[o] = m;
                ep.part_s[o] = s;
                ep.part_a[o] = am;
            }
        }
    } else {
        // ------------------------------------------------------ residual epilogue
        const int ew = warp - kEpiWarp0;
        const int quarter = warp & 3;
        const int half = ew >> 2;
        const int row = quarter * 32 + lane;
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
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
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
                    lq[u] = ld_stream16(Lrow + c8);
                    tq[u] = ld_stream16(Trow + c8);
                } else {
                    lq[u] = make_uint4(0, 0, 0, 0);
                    tq[u] = make_uint4(0, 0, 0, 0);
                }
            }
            bool ok = tc::mbar_wait_bounded(&acc_full[ab], ph, abort_flag, kWaitBudget);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc::tc_fence_after();
            const uint32_t taddr = tmem_base + lane_addr + ab * kBN + half * kPartN;
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

bool make_map(CUtensorMap *m, const void *ptr, int rank, const cuuint64_t *dims, const cuuint64_t *strides,
              const cuuint32_t *box) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint32_t es[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(ptr), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int MODE>
cudaError_t launch_markov_tc(const CUtensorMap &mE, const CUtensorMap &mW, const CUtensorMap &mL, int r,
                             const TcEpi &ep, cudaStream_t st) {
    const TcSmem lay = tc_layout(r);
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
    markov_tile_tc<MODE><<<grid, kThreads, lay.total, st>>>(mE, mW, mL, r, nTilesN, ep);
    return cudaGetLastError();
}

bool map_rows(CUtensorMap *m, const void *base, int rows, int r) {
    cuuint64_t dims[2] = {(cuuint64_t)r, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)r * 2};
    cuuint32_t box[2] = {kKB, kM};
    return make_map(m, base, 2, dims, strides, box);
}
bool map_factor(CUtensorMap *m, const void *Wt, int V, int r) {
    cuuint64_t dims[2] = {(cuuint64_t)r, (cuuint64_t)V};
    cuuint64_t strides[1] = {(cuuint64_t)r * 2};
    cuuint32_t box[2] = {kKB, kBN};
    return make_map(m, Wt, 2, dims, strides, box);
}

}  // namespace

cudaError_t launch_draft_tile_tc(const DraftArgs &a, const DraftWs &w, int pos, cudaStream_t st) {
    CUtensorMap mE, mW, mL;
    if (!map_rows(&mE, w.E, round_up(a.B, kM), a.r) || !map_factor(&mW, a.Wt, a.V, a.r))
        return cudaErrorInvalidValue;
    {
        cuuint64_t dims[3] = {(cuuint64_t)a.V, (cuuint64_t)a.G, (cuuint64_t)a.B};
        cuuint64_t strides[2] = {(cuuint64_t)a.V * 2, (cuuint64_t)a.G * a.V * 2};
        cuuint32_t box[3] = {kPartN, 1, kM};
        if (!make_map(&mL, a.L, 3, dims, strides, box)) return cudaErrorInvalidValue;
    }
    TcEpi ep{};
    ep.temp = a.temp; ep.B = a.B; ep.G = a.G; ep.V = a.V; ep.pos = pos; ep.nParts = w.nTiles; ep.hdr = w.hdr;
    ep.part_m = w.part_m; ep.part_s = w.part_s; ep.part_a = w.part_a;
    return launch_markov_tc<kEpiDraft>(mE, mW, mL, a.r, ep, st);
}

cudaError_t launch_residual_tile_tc(const ResidualTcArgs &a, cudaStream_t st) {
    CUtensorMap mE, mW;
    if (!map_rows(&mE, a.E, round_up(a.B, kM), a.r) || !map_factor(&mW, a.Wt, a.V, a.r))
        return cudaErrorInvalidValue;
    TcEpi ep{};
    ep.temp = a.temp; ep.B = a.B; ep.G = a.G; ep.V = a.V; ep.pos = 0; ep.nParts = a.nParts; ep.hdr = a.hdr;
    ep.nrows = a.nrows; ep.res_b = a.res_b; ep.res_k = a.res_k; ep.res_mt = a.res_mt; ep.res_zt = a.res_zt;
    ep.rowmax = a.rowmax; ep.rowsum = a.rowsum; ep.L = a.L; ep.Tlog = a.Tlog; ep.rp = a.rp;
    return launch_markov_tc<kEpiResidual>(mE, mW, mE, a.r, ep, st);
}

}  // namespace dspark
