// verify.cu -- stage 4, exact rejection-sampling verification.
//
// Method (menfem.com KB entry on DSpark, "Methodology": x_k is accepted with
// probability min(1, p_t(x_k) / p_d(x_k)) and the first rejection discards
// every later token; paperlayer.ai summary, §2: the longest consistent prefix
// is kept; Appendix A: with nothing admitted the target draws a fresh
// token).  A rejection at k* is replaced by a draw from the normalised
// residual max(0, p_t - p_d) at k*; a fully accepted prefix earns a bonus
// draw from p_t at row ell + 1.
//
// Launch sequence (fixed, graph-capturable; work counts live on the device):
//   plan        1 CTA: row list of the admitted target rows, rows (b, k) for
//               k = 0..ell_b (0-based), and their offsets per request.
//   rows        persistent grid over (row, 4096-column chunk) work items
//               (bf16: chunks staged in shared memory by bulk copies, two
//               stages per warp): one streaming pass over each target row,
//               giving per chunk the max, lowest argmax and sum of
//               exp((t - max) / T).
//   decide      1 CTA per request: row max / Z from the chunk partials,
//               p_t(x_k), the accept tests, the first-rejection count A, the
//               bonus draw (prefix over chunk sums, then one chunk rescanned)
//               or the greedy token; rejected rows are queued for the residual.
//   residual    Delta recomputed for the queued rows (CUDA-core GEMM tile,
//               as in drafting) fused with q = max(0, p_t - p_d) tile sums.
//   res_final   1 CTA per queued row: prefix over tile sums, one tile
//               recomputed and scanned to the replacement token.
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"
#include "tc.cuh"

namespace dspark {

constexpr int kChunk = 4096;          // columns per row work item
constexpr int kRowThreads = 256;      // threads of the row and decide kernels
constexpr int kRowQ = kChunk / (kRowThreads * 8);   // 8-column groups per thread in a chunk (fp32 rows pass)
constexpr int kColsPerThread = kChunk / kRowThreads;   // columns per thread when a block rescans a chunk
constexpr int kResRows = 32;          // queued rows per residual tile CTA
constexpr int kResCols = 256;         // columns per residual tile (fp32, CUDA cores)

__host__ __device__ inline int res_cols(int dtype) { return dtype == DSPARK_BF16 ? kTcTileN : kResCols; }

struct VerifyWs {
    WsHeader *hdr;             // pad[0] = row count, pad[1] = residual count
    int32_t *rows;             // [B*(G+1)] packed b * 32 + k
    int32_t *row_off;          // [B+1]
    float *cm, *cs;            // [B*(G+1)*nChunks] chunk max / sum
    int32_t *ca;               // [B*(G+1)*nChunks] chunk argmax
    int32_t *res_b;            // [B] queued request
    int32_t *res_k;            // [B] rejected position (0-based)
    float *res_mt, *res_zt;    // [B] target row max / Z of the rejected row
    float *rp;                 // [B*nResTiles] residual tile sums
    int nChunks, nResTiles, resCols;
};

static VerifyWs carve_verify_ws(void *ws, int B, int G, int V, int r, int dtype) {
    VerifyWs w;
    w.nChunks = (V + kChunk - 1) / kChunk;
    w.resCols = res_cols(dtype);
    w.nResTiles = (V + w.resCols - 1) / w.resCols;
    const size_t R = (size_t)B * (G + 1);
    char *p = static_cast<char *>(ws);
    w.hdr = reinterpret_cast<WsHeader *>(p); p += sizeof(WsHeader);
    w.rows = reinterpret_cast<int32_t *>(p); p += align256(sizeof(int32_t) * R);
    w.row_off = reinterpret_cast<int32_t *>(p); p += align256(sizeof(int32_t) * (B + 1));
    w.cm = reinterpret_cast<float *>(p); p += align256(sizeof(float) * R * w.nChunks);
    w.cs = reinterpret_cast<float *>(p); p += align256(sizeof(float) * R * w.nChunks);
    w.ca = reinterpret_cast<int32_t *>(p); p += align256(sizeof(int32_t) * R * w.nChunks);
    w.res_b = reinterpret_cast<int32_t *>(p); p += align256(sizeof(int32_t) * B);
    w.res_k = reinterpret_cast<int32_t *>(p); p += align256(sizeof(int32_t) * B);
    w.res_mt = reinterpret_cast<float *>(p); p += align256(sizeof(float) * B);
    w.res_zt = reinterpret_cast<float *>(p); p += align256(sizeof(float) * B);
    w.rp = reinterpret_cast<float *>(p); p += align256(sizeof(float) * (size_t)B * w.nResTiles);
    return w;
}

size_t verify_ws_bytes(int B, int G, int V, int r, int dtype) {
    const int nChunks = (V + kChunk - 1) / kChunk, rc = res_cols(dtype), nResTiles = (V + rc - 1) / rc;
    const size_t R = (size_t)B * (G + 1);
    size_t bytes = sizeof(WsHeader) + align256(4 * R) + align256(4 * (B + 1)) + 3 * align256(4 * R * nChunks) +
                   4 * align256(4 * (size_t)B) + align256(4 * (size_t)B * nResTiles);
    return bytes;
}

// Eight consecutive elements starting at index i of a row (bounds-checked;
// one or two 16-byte loads when aligned and complete).
__device__ __forceinline__ void load8(const __nv_bfloat16 *row, int i, int n, float (&v)[8]) {
    const __nv_bfloat16 *p = row + i;
    if (i + 8 <= n && (reinterpret_cast<uintptr_t>(p) & 15) == 0) {
        uint4 q = ld_stream16(p);
        v[0] = bf16lo(q.x); v[1] = bf16hi(q.x); v[2] = bf16lo(q.y); v[3] = bf16hi(q.y);
        v[4] = bf16lo(q.z); v[5] = bf16hi(q.z); v[6] = bf16lo(q.w); v[7] = bf16hi(q.w);
    } else {
#pragma unroll
        for (int q = 0; q < 8; ++q) v[q] = (i + q < n) ? __bfloat162float(p[q]) : -INFINITY;
    }
}
__device__ __forceinline__ void load8(const float *row, int i, int n, float (&v)[8]) {
    const float *p = row + i;
    if (i + 8 <= n && (reinterpret_cast<uintptr_t>(p) & 15) == 0) {
        uint4 a = ld_stream16(p), b = ld_stream16(p + 4);
        v[0] = __uint_as_float(a.x); v[1] = __uint_as_float(a.y); v[2] = __uint_as_float(a.z);
        v[3] = __uint_as_float(a.w); v[4] = __uint_as_float(b.x); v[5] = __uint_as_float(b.y);
        v[6] = __uint_as_float(b.z); v[7] = __uint_as_float(b.w);
    } else {
#pragma unroll
        for (int q = 0; q < 8; ++q) v[q] = (i + q < n) ? p[q] : -INFINITY;
    }
}

// ----------------------------------------------------------------- plan
__global__ void verify_plan(const int32_t *__restrict__ ell, int B, int G, VerifyWs w) {
    __shared__ int tot[33];
    __shared__ int carry;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    if (tid == 0) { carry = 0; w.hdr->pad[1] = 0; w.hdr->pad[kPadRowItems] = 0; }
    __syncthreads();
    for (int b0 = 0; b0 < B; b0 += blockDim.x) {
        const int b = b0 + tid;
        int n = 0;
        if (b < B) {
            int l = ell[b];
            if (l < 0 || l > G) { flag_status(w.hdr, DSPARK_DEV_ELL_RANGE); l = l < 0 ? 0 : G; }
            n = l + 1;
        }
        int inc = warp_incl_scan_i(n);
        if (lane == 31) tot[wid] = inc;
        __syncthreads();
        if (wid == 0) {
            int t = lane < (int)(blockDim.x >> 5) ? tot[lane] : 0;
            t = warp_incl_scan_i(t);
            tot[lane] = t;
        }
        __syncthreads();
        const int off = carry + inc - n + (wid > 0 ? tot[wid - 1] : 0);
        if (b < B) {
            w.row_off[b] = off;
            for (int k = 0; k < n; ++k) w.rows[off + k] = b * 32 + k;
        }
        __syncthreads();
        if (tid == 0) carry += tot[(blockDim.x >> 5) - 1];
        __syncthreads();
    }
    if (tid == 0) { w.row_off[B] = carry; w.hdr->pad[0] = carry; }
}

// ----------------------------------------------------------------- rows
// One work item = one 4096-column chunk of one admitted target row.  Each
// thread owns 16 columns (2 groups of 8 contiguous columns), loads them with
// 16-byte streaming loads one item ahead of the one it reduces, and keeps an
// online (max, sum of exp((t - max) / T)); the greedy argmax is only tracked
// for T = 0 rows.  One block merge per item writes the chunk partial.
template <typename T>
__device__ __forceinline__ void rows_load(const T *__restrict__ Tlog, const VerifyWs &w, int G, int V, int item,
                                          float (&v)[kRowQ][8]) {
    const int j = item / w.nChunks, c = item - j * w.nChunks;
    const int rk = w.rows[j], b = rk >> 5, k = rk & 31;
    const T *row = Tlog + ((size_t)b * (G + 1) + k) * V;
    const int c0 = c * kChunk, c1 = min(V, c0 + kChunk);
#pragma unroll
    for (int q = 0; q < kRowQ; ++q) {
        const int i = c0 + (q * kRowThreads + threadIdx.x) * 8;
        if (i < c1) {
            load8(row, i, c1, v[q]);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) v[q][e] = -INFINITY;
        }
    }
}

template <typename T>
__global__ void __launch_bounds__(kRowThreads) verify_rows(const T *__restrict__ Tlog,
                                                           const float *__restrict__ temp, int G,
                                                           int V, VerifyWs w) {
    __shared__ float rm[8], rs[8];
    __shared__ int ra[8];
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int nrows = *reinterpret_cast<volatile uint32_t *>(&w.hdr->pad[0]);
    const int nwork = nrows * w.nChunks;
    int item = blockIdx.x;
    if (item >= nwork) return;
    float cur[kRowQ][8], nxt[kRowQ][8];
    rows_load(Tlog, w, G, V, item, cur);
    for (; item < nwork; item += gridDim.x) {
        const int next = item + gridDim.x;
        if (next < nwork) rows_load(Tlog, w, G, V, next, nxt);
        const int j = item / w.nChunks, c = item - j * w.nChunks;
        const int b = w.rows[j] >> 5;
        float Tb = temp[b];
        Tb = Tb >= 0.f ? Tb : 0.f;
        const float cexp = Tb > 0.f ? kLog2e / Tb : 0.f;
        float m = -INFINITY;
#pragma unroll
        for (int q = 0; q < kRowQ; ++q)
#pragma unroll
            for (int e = 0; e < 8; ++e) m = fmaxf(m, cur[q][e]);
        int am = 0x7fffffff;
        float s = 0.f;
        if (Tb == 0.f) {   // whole item is one row: the branch is block-uniform
#pragma unroll
            for (int q = kRowQ - 1; q >= 0; --q)
#pragma unroll
                for (int e = 7; e >= 0; --e)
                    if (cur[q][e] == m) am = c * kChunk + (q * kRowThreads + tid) * 8 + e;
        } else if (m > -INFINITY) {
#pragma unroll
            for (int q = 0; q < kRowQ; ++q)
#pragma unroll
                for (int e = 0; e < 8; ++e) s += fast_exp2((cur[q][e] - m) * cexp);
        }
        // Warp merge of (m, s, argmax), then across the 8 warps.
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float om = __shfl_xor_sync(0xffffffffu, m, o);
            const float os = __shfl_xor_sync(0xffffffffu, s, o);
            const int oa = __shfl_xor_sync(0xffffffffu, am, o);
            const float nm = fmaxf(m, om);
            if (cexp > 0.f)
                s = (m > -INFINITY ? s * fast_exp2((m - nm) * cexp) : 0.f) +
                    (om > -INFINITY ? os * fast_exp2((om - nm) * cexp) : 0.f);
            if (om > m || (om == m && oa < am)) am = oa;
            m = nm;
        }
        if (lane == 0) { rm[wid] = m; rs[wid] = s; ra[wid] = am; }
        __syncthreads();
        if (tid == 0) {
            float M = rm[0];
            int A = ra[0];
            for (int q = 1; q < 8; ++q)
                if (rm[q] > M || (rm[q] == M && ra[q] < A)) { M = rm[q]; A = ra[q]; }
            float S = 0.f;
            if (cexp > 0.f)
                for (int q = 0; q < 8; ++q)
                    if (rm[q] > -INFINITY) S += rs[q] * fast_exp2((rm[q] - M) * cexp);
            const size_t o = (size_t)j * w.nChunks + c;
            w.cm[o] = M;
            w.cs[o] = S;
            w.ca[o] = A;
        }
        __syncthreads();
        if (next < nwork) {
#pragma unroll
            for (int q = 0; q < kRowQ; ++q)
#pragma unroll
                for (int e = 0; e < 8; ++e) cur[q][e] = nxt[q][e];
        }
    }
}

// bf16 rows: persistent CTAs (one per SM) over the (row, 4096-column chunk)
// work items.  Each warp streams its items itself: its first two are fixed,
// the rest it claims one at a time from a counter in the workspace header.
// It owns two shared-memory stages and keeps a bulk copy in flight into one
// while it reduces the other (evict-first: every target row is read once, so
// the transition factor that drafting left in L2 stays there for the residual
// pass).  As soon as a chunk's values are in registers the warp issues the
// next claimed item's copy into the stage it just read, reduces its 4096
// columns to (max, sum of exp((t - max) / T), lowest argmax) and writes the
// chunk partial -- no block barrier, no producer to wait for.  The row of an
// item comes from the compacted row list; temperatures are staged in shared
// memory.  Lane l reads the 16-byte pieces l, l + 32, ... of the chunk
// (bank-conflict free).
constexpr int kVrWarps = 12;
constexpr int kVrThreads = kVrWarps * 32;
constexpr int kVrStageBytes = kChunk * 2;            // 8 KB
constexpr int kVrPieces = kVrStageBytes / 16 / 32;   // 16-byte pieces per lane (16)
constexpr long long kVrWaitBudget = 4000000000LL;   // ~2 s of SM clock

__host__ inline size_t vr_smem_bytes(int B) {
    return (size_t)kVrWarps * 2 * kVrStageBytes + (size_t)kVrWarps * 2 * sizeof(uint64_t) + sizeof(float) * (size_t)B;
}

__global__ void __launch_bounds__(kVrThreads, 1) verify_rows_bulk(const __nv_bfloat16 *__restrict__ Tlog,
                                                                 const float *__restrict__ temp, int B, int G, int V,
                                                                 VerifyWs w, long long budget) {
    extern __shared__ __align__(128) unsigned char vr_smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(vr_smem + kVrWarps * 2 * kVrStageBytes);   // [warp][2]
    float *temp_s = reinterpret_cast<float *>(full + kVrWarps * 2);                            // [B]
    __shared__ int abort_s;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nrows = *reinterpret_cast<volatile uint32_t *>(&w.hdr->pad[0]);
    const int nwork = nrows * w.nChunks;
    if ((int)blockIdx.x >= nwork) return;
    if (threadIdx.x == 0) {
        for (int q = 0; q < kVrWarps * 2; ++q) tc::mbar_init(&full[q], 1);
        abort_s = 0;
        tc::fence_barrier_init();
    }
    for (int b = threadIdx.x; b < B; b += blockDim.x) temp_s[b] = temp[b];
    __syncthreads();
    volatile int *abort_flag = &abort_s;
    unsigned char *stage0 = vr_smem + warp * 2 * kVrStageBytes;
    uint64_t *myfull = full + warp * 2;
    // Items: a warp's first two are fixed (g and g + NW, g its index over the
    // grid's NW warps); after that each warp claims one item at a time from
    // the counter that verify_plan zeroed (claimed items are numbered from
    // 2 NW), so the warps finish together instead of some taking one item
    // more.  Lane 0 fires a claim and the claimed item's row-id load one
    // iteration before the item is issued, so both latencies pass while the
    // warp computes.  A warp's claims increase, so the first out-of-range item
    // it meets ends its work with nothing claimed left over.
    const int NW = (int)gridDim.x * kVrWarps;
    uint32_t *claim_ctr = &w.hdr->pad[kPadRowItems];
    int itA = warp * (int)gridDim.x + (int)blockIdx.x, itB = itA + NW;   // the items in stages 0 and 1
    int rkA = 0, rkB = 0, nxt_it = nwork, nxt_rk = 0, pend = nwork;
    if (lane == 0) {
        pend = 2 * NW + (int)atomicAdd(claim_ctr, 1u);
        if (itA < nwork) rkA = w.rows[itA / w.nChunks];
        if (itB < nwork) rkB = w.rows[itB / w.nChunks];
    }
    rkA = __shfl_sync(0xffffffffu, rkA, 0);
    rkB = __shfl_sync(0xffffffffu, rkB, 0);
    const uint64_t pol = tc::policy_evict_first();
    auto issue = [&](int item, int rk, int s) {   // lane 0
        const int c = item % w.nChunks;
        const int c0 = c * kChunk, ncols = min(kChunk, V - c0);
        const __nv_bfloat16 *src = Tlog + ((size_t)(rk >> 5) * (G + 1) + (rk & 31)) * V + c0;
        tc::mbar_arrive_expect_tx(&myfull[s], (uint32_t)ncols * 2);
        tc::bulk_load(stage0 + s * kVrStageBytes, src, (uint32_t)ncols * 2, &myfull[s], pol);
    };
    if (lane == 0) {
        if (itA < nwork) issue(itA, rkA, 0);
        if (itB < nwork) issue(itB, rkB, 1);
        nxt_it = pend;   // waits for the first claim while the copies fly
        if (nxt_it < nwork) {
            nxt_rk = w.rows[nxt_it / w.nChunks];
            pend = 2 * NW + (int)atomicAdd(claim_ctr, 1u);
        }
    }
    for (int k = 0;; ++k) {
        const int s = k & 1;
        const int item = s ? itB : itA;
        if (item >= nwork) break;
        const bool ok = tc::mbar_wait_bounded(&myfull[s], (k >> 1) & 1, abort_flag, budget);
        if (!__all_sync(0xffffffffu, ok)) {
            // Give up: wait (bounded, ignoring the abort flag) for this warp's
            // copies in flight (this stage's, and the other's if it holds an
            // item) so that none lands after the CTA exits.
            if (lane == 0) {
                int dummy = 0;
                tc::mbar_wait_bounded(&myfull[s], (k >> 1) & 1, &dummy, kVrWaitBudget / 4);
                if ((s ? itA : itB) < nwork)
                    tc::mbar_wait_bounded(&myfull[s ^ 1], ((k + 1) >> 1) & 1, &dummy, kVrWaitBudget / 4);
                *abort_flag = 1;
                flag_status(w.hdr, DSPARK_DEV_TIMEOUT);
            }
            break;
        }
        uint4 v[kVrPieces];
        const unsigned char *src = stage0 + s * kVrStageBytes + lane * 16;
#pragma unroll
        for (int i = 0; i < kVrPieces; ++i) v[i] = *reinterpret_cast<const uint4 *>(src + i * 512);
        const int rk = s ? rkB : rkA;
        // The stage is free once every lane's reads are done: the next copy may
        // land in it (generic reads, then async-proxy writes).
        tc::fence_proxy_async_smem();
        __syncwarp();
        // Refill this stage with the claimed item; claim the next one.
        const int nit = __shfl_sync(0xffffffffu, nxt_it, 0);
        const int nrk = __shfl_sync(0xffffffffu, nxt_rk, 0);
        if (lane == 0 && nit < nwork) {
            issue(nit, nrk, s);
            nxt_it = pend;
            if (nxt_it < nwork) {
                nxt_rk = w.rows[nxt_it / w.nChunks];
                pend = 2 * NW + (int)atomicAdd(claim_ctr, 1u);
            }
        }
        if (s) { itB = nit; rkB = nrk; } else { itA = nit; rkA = nrk; }
        const int jrow = item / w.nChunks, ch = item - jrow * w.nChunks;
        const int ncols = min(kChunk, V - ch * kChunk);
        float T = temp_s[rk >> 5];
        T = T >= 0.f ? T : 0.f;
        const float cexp = T > 0.f ? kLog2e / T : 0.f;
        if (ncols < kChunk) {   // the row's last chunk: columns past V are -inf (bf16 0xff80)
#pragma unroll
            for (int i = 0; i < kVrPieces; ++i) {
                uint32_t wq[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const int col = i * 256 + lane * 8 + 2 * h;
                    if (col >= ncols) wq[h] = (wq[h] & 0xffff0000u) | 0xff80u;
                    if (col + 1 >= ncols) wq[h] = (wq[h] & 0x0000ffffu) | 0xff800000u;
                }
                v[i] = make_uint4(wq[0], wq[1], wq[2], wq[3]);
            }
        }
        // Maximum: running three-input maxima over the value pairs.
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int i = 0; i < kVrPieces; ++i) {
            m4[0] = max3(m4[0], bf16lo(v[i].x), bf16hi(v[i].x));
            m4[1] = max3(m4[1], bf16lo(v[i].y), bf16hi(v[i].y));
            m4[2] = max3(m4[2], bf16lo(v[i].z), bf16hi(v[i].z));
            m4[3] = max3(m4[3], bf16lo(v[i].w), bf16hi(v[i].w));
        }
        float m = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        float sum = 0.f;
        int am = 0x7fffffff;
        if (cexp == 0.f) {   // greedy row (warp-uniform): the lowest index of the largest value
#pragma unroll
            for (int i = kVrPieces - 1; i >= 0; --i) {
                const uint32_t wq[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
                for (int h = 3; h >= 0; --h) {
                    if (bf16hi(wq[h]) == m) am = ch * kChunk + i * 256 + lane * 8 + 2 * h + 1;
                    if (bf16lo(wq[h]) == m) am = ch * kChunk + i * 256 + lane * 8 + 2 * h;
                }
            }
        } else if (m > -INFINITY) {
            // exp((t - m) / T) = 2^(t * cexp - m * cexp): one paired fused
            // multiply-add per two columns, then the two ex2.
            const float2 c2 = make_float2(cexp, cexp);
            const float nmc = -m * cexp;
            const float2 n2 = make_float2(nmc, nmc);
            float2 s2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                            make_float2(0.f, 0.f)};
#pragma unroll
            for (int i = 0; i < kVrPieces; ++i) {
                const uint32_t wq[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const float2 arg = fma2(make_float2(bf16lo(wq[h]), bf16hi(wq[h])), c2, n2);
                    // One column pair in four goes through the FMA-pipe polynomial
                    // instead of the special-function unit, which is the busier pipe.
                    s2[h] = add2(s2[h], h == 3 ? exp2_poly2(arg) : make_float2(fast_exp2(arg.x), fast_exp2(arg.y)));
                }
            }
            const float2 p01 = add2(s2[0], s2[1]), p23 = add2(s2[2], s2[3]);
            const float2 pall = add2(p01, p23);
            sum = pall.x + pall.y;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float om = __shfl_xor_sync(0xffffffffu, m, o);
            const float os = __shfl_xor_sync(0xffffffffu, sum, o);
            const int oa = __shfl_xor_sync(0xffffffffu, am, o);
            const float nm = fmaxf(m, om);
            if (cexp > 0.f)
                sum = (m > -INFINITY ? sum * fast_exp2((m - nm) * cexp) : 0.f) +
                      (om > -INFINITY ? os * fast_exp2((om - nm) * cexp) : 0.f);
            if (om > m || (om == m && oa < am)) am = oa;
            m = nm;
        }
        if (lane == 0) {
            const size_t o = (size_t)jrow * w.nChunks + ch;
            w.cm[o] = m;
            w.cs[o] = sum;
            w.ca[o] = am;
        }
    }
}

// Row statistics from the chunk partials of compacted row j (one warp).
__device__ __forceinline__ void row_stats(const VerifyWs &w, int j, float invT, float &M, float &Z,
                                          int &A) {
    const int lane = threadIdx.x & 31;
    const float *cm = w.cm + (size_t)j * w.nChunks;
    const float *cs = w.cs + (size_t)j * w.nChunks;
    const int32_t *ca = w.ca + (size_t)j * w.nChunks;
    float m = -INFINITY;
    int a = 0x7fffffff;
    for (int c = lane; c < w.nChunks; c += 32)
        if (cm[c] > m || (cm[c] == m && ca[c] < a)) { m = cm[c]; a = ca[c]; }
    warp_argmax(m, a);
    float z = 0.f;
    if (invT > 0.f)
        for (int c = lane; c < w.nChunks; c += 32) z += cs[c] * exp_e((cm[c] - m) * invT);
    z = warp_sum(z);
    M = m; Z = z; A = a;
}

// Inverse-CDF draw from target row j (compacted index; request b, position
// k) with row stats (M, Z): prefix over the chunk sums, then the chosen chunk
// rescanned in index order, each thread owning 32 consecutive columns loaded
// at once.  Whole block (kRowThreads threads); returns the token.
template <typename T>
__device__ int sample_target_row(const T *__restrict__ Tlog, const VerifyWs &w, int j, int b, int k,
                                 int G, int V, float M, float Z, float invT, float u) {
    __shared__ float s_c[32], s_e[32];
    __shared__ int s_i0[32], s_i1[32], s_i2[32], s_i3[32];
    __shared__ float excl_s;
    __shared__ int col_s;
    const int tid = threadIdx.x;
    const float *cm = w.cm + (size_t)j * w.nChunks;
    const float *cs = w.cs + (size_t)j * w.nChunks;
    const float target = u * Z;
    // Prefix over chunk sums (nChunks <= 256 for V <= 2^20; kRowThreads >= that).
    const float wc = tid < w.nChunks ? cs[tid] * exp_e((cm[tid] - M) * invT) : 0.f;
    float tot;
    const float inc = block_scan1(wc, s_c, &tot);
    int ch = block_min1((tid < w.nChunks && inc > target) ? tid : 0x7fffffff, s_i0);
    const bool past_mass = ch == 0x7fffffff;   // rounding left u Z at the top: a tie by definition
    if (past_mass) {
        ch = block_max1_i((tid < w.nChunks && wc > 0.f) ? tid : -1, s_i1);
        if (ch < 0) ch = w.nChunks - 1;
    }
    if (tid == ch) excl_s = inc - wc;
    __syncthreads();
    const float rem = target - excl_s;
    const T *row = Tlog + ((size_t)b * (G + 1) + k) * V;
    const int c0 = ch * kChunk, c1 = min(V, c0 + kChunk);
    const int i0 = c0 + tid * kColsPerThread;   // this thread's consecutive columns
    float e[kColsPerThread];
    float run = 0.f;
#pragma unroll
    for (int q = 0; q < kColsPerThread / 8; ++q) {
        float v[8];
        const int i = i0 + q * 8;
        if (i < c1) load8(row, i, c1, v);
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            e[q * 8 + t] = (i + t < c1) ? exp_e((v[t] - M) * invT) : 0.f;
            run += e[q * 8 + t];
        }
    }
    float rt;
    const float incl = block_scan1(run, s_e, &rt);
    int owner = block_min1((incl > rem && run > 0.f) ? tid : 0x7fffffff, s_i2);
    const bool short_slice = owner == 0x7fffffff;
    if (short_slice) owner = max(0, block_max1_i(run > 0.f ? tid : -1, s_i3));
    if (tid == owner) {
        float p = incl - run;
        int f = -1, lastpos = -1;
        float margin = 0.f;
#pragma unroll
        for (int t = 0; t < kColsPerThread; ++t) {
            if (f < 0 && e[t] > 0.f) {
                lastpos = i0 + t;
                p += e[t];
                if (p > rem) {
                    f = i0 + t;
                    margin = fminf(rem - (p - e[t]), p - rem) / Z;   // u Z to the nearer edge, over Z
                }
            }
        }
        if (f < 0) f = lastpos >= 0 ? lastpos : c1 - 1;
        if (past_mass || short_slice || !(margin >= kNearTie)) count_near_tie(w.hdr, kPadVerifyTies);
        col_s = f;
    }
    __syncthreads();
    return col_s;
}

// ----------------------------------------------------------------- decide
template <typename T>
__global__ void __launch_bounds__(kRowThreads) verify_decide(
    const T *__restrict__ Tlog, const T *__restrict__ U, const int32_t *__restrict__ x0, int r,
    const int32_t *__restrict__ x, const float *__restrict__ pd_x,
    const float *__restrict__ temp, const float *__restrict__ u_accept,
    const float *__restrict__ u_final, const int32_t *__restrict__ ell, int B, int G, int V,
    VerifyWs w, int32_t *__restrict__ acc_out, int32_t *__restrict__ tokens_out,
    int32_t *__restrict__ nout_out, float *__restrict__ pt_x_out) {
    __shared__ float rM[17], rZ[17];
    __shared__ int rA[17];
    __shared__ int acc_s[16], tie_s[16];
    __shared__ int A_s;
    const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const float Tb = sane_temp(temp[b], w.hdr);
    const float invT = Tb > 0.f ? 1.f / Tb : 0.f;
    int lb = ell[b];
    lb = lb < 0 ? 0 : (lb > G ? G : lb);
    // Thread k < G fetches what the accept test of position k needs before
    // the row statistics are in.
    const size_t o = (size_t)b * G + tid;
    int xk = 0;
    float tk = 0.f, uk = 0.f, pdk = 1.f;
    if (tid < lb) {
        xk = clamp_token(x[o], V, w.hdr);
        if (Tb > 0.f) {
            tk = to_f32(Tlog[((size_t)b * (G + 1) + tid) * V + xk]);
            uk = u_accept[o];
            pdk = pd_x[o];
        }
    }
    const int j0 = w.row_off[b];
    for (int k = wid; k <= lb; k += kRowThreads / 32) {
        float M, Z;
        int A;
        row_stats(w, j0 + k, invT, M, Z, A);
        if (lane == 0) { rM[k] = M; rZ[k] = Z; rA[k] = A; }
    }
    __syncthreads();
    if (tid < G) {
        float pt = -1.f;
        int acc = 0, tie = 0;
        if (tid < lb) {
            if (Tb == 0.f) {
                acc = rA[tid] == xk;
                pt = acc ? 1.f : 0.f;
            } else {
                pt = exp_e((tk - rM[tid]) * invT) / rZ[tid];
                const float ratio = pt / pdk;
                acc = uk < ratio;
                tie = !(fabsf(uk - ratio) >= kNearTie);
            }
        }
        acc_s[tid] = acc;
        tie_s[tid] = tie;
        if (pt_x_out != nullptr) pt_x_out[o] = pt;
    }
    __syncthreads();
    if (tid == 0) {
        int A = 0;
        while (A < lb && acc_s[A]) ++A;   // the first rejection discards the rest
        // Near-ties among the tests that decided A (later ones are discarded).
        for (int k = 0; k < lb && k <= A; ++k)
            if (tie_s[k]) count_near_tie(w.hdr, kPadVerifyTies);
        A_s = A;
        acc_out[b] = A;
        nout_out[b] = A + 1;
        if (Tb > 0.f && A < lb) {  // queue the rejected row for the residual draw
            const int slot = atomicAdd(&w.hdr->pad[1], 1u);
            w.res_b[slot] = b;
            w.res_k[slot] = A;
            w.res_mt[slot] = rM[A];
            w.res_zt[slot] = rZ[A];
        }
    }
    __syncthreads();
    const int A = A_s;
    // Token A: the greedy target token, the bonus draw from p_t at row lb
    // (a fresh token when nothing was admitted), or -1 until the residual
    // draw replaces it.
    int fin = -1;
    if (Tb == 0.f)
        fin = (rA[A] >= 0 && rA[A] < V) ? rA[A] : 0;
    else if (A == lb)   // block-uniform
        fin = sample_target_row(Tlog, w, j0 + lb, b, lb, G, V, rM[lb], rZ[lb], invT, u_final[b]);
    if (tid <= G) tokens_out[(size_t)b * (G + 1) + tid] = tid < A ? x[(size_t)b * G + tid] : (tid == A ? fin : -1);
}

// ----------------------------------------------------------------- residual
// q = max(0, p_t - p_d) tile sums for the queued rows; p_d rebuilt from
// L + U[x_{k-1}] W (CUDA-core tile GEMM) and the drafting stats.
template <typename T>
__global__ void __launch_bounds__(256) residual_tile_simt(
    const T *__restrict__ Tlog, const T *__restrict__ L, const T *__restrict__ U,
    const T *__restrict__ Wt, const int32_t *__restrict__ x0, const int32_t *__restrict__ x,
    const float *__restrict__ rowmax, const float *__restrict__ rowsum,
    const float *__restrict__ temp, int G, int V, int r, VerifyWs w) {
    __shared__ float Es[kResRows][33];
    __shared__ int prev_s[kResRows], b_s[kResRows], k_s[kResRows];
    __shared__ float red[8][kResRows];
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int nres = *reinterpret_cast<volatile uint32_t *>(&w.hdr->pad[1]);
    const int row0 = blockIdx.y * kResRows;
    if (row0 >= nres) return;
    const int tile = blockIdx.x;
    const int col = tile * kResCols + tid;
    const bool colok = col < V;
    if (tid < kResRows) {
        int s = row0 + tid, b = 0, k = 0, p = 0;
        if (s < nres) {
            b = w.res_b[s];
            k = w.res_k[s];
            p = (k == 0) ? x0[b] : x[(size_t)b * G + k - 1];
            p = min(max(p, 0), V - 1);
        }
        b_s[tid] = b; k_s[tid] = k; prev_s[tid] = p;
    }
    float acc[kResRows];
#pragma unroll
    for (int j = 0; j < kResRows; ++j) acc[j] = 0.f;
    for (int k0 = 0; k0 < r; k0 += 32) {
        __syncthreads();
        for (int e = tid; e < kResRows * 32; e += blockDim.x) {
            int rr = e >> 5, kk = e & 31;
            float v = 0.f;
            if (row0 + rr < nres && k0 + kk < r) v = ld_elem(U, (size_t)prev_s[rr] * r + k0 + kk);
            Es[rr][kk] = v;
        }
        __syncthreads();
        float wv[32];
#pragma unroll
        for (int kk = 0; kk < 32; ++kk)
            wv[kk] = (colok && k0 + kk < r) ? ld_elem(Wt, (size_t)col * r + k0 + kk) : 0.f;
#pragma unroll
        for (int j = 0; j < kResRows; ++j) {
            float a = acc[j];
#pragma unroll
            for (int kk = 0; kk < 32; ++kk) a = fmaf(Es[j][kk], wv[kk], a);
            acc[j] = a;
        }
    }
#pragma unroll
    for (int j = 0; j < kResRows; ++j) {
        const int s = row0 + j;
        float q = 0.f;
        if (s < nres && colok) {
            const int b = b_s[j], k = k_s[j];
            const float Tb = fmaxf(temp[b], 0.f);
            const float invT = 1.f / Tb;
            const size_t ro = (size_t)b * G + k;
            const float l = ld_elem(L, ro * V + col);
            const float pd = exp_e(((l - rowmax[ro]) + acc[j]) * invT) / rowsum[ro];
            const float t = ld_elem(Tlog, ((size_t)b * (G + 1) + k) * V + col);
            const float pt = exp_e((t - w.res_mt[s]) * invT) / w.res_zt[s];
            q = fmaxf(pt - pd, 0.f);
        }
        q = warp_sum(q);
        if (lane == 0) red[wid][j] = q;
    }
    __syncthreads();
    if (tid < kResRows && row0 + tid < nres) {
        float s = 0.f;
        for (int q = 0; q < 8; ++q) s += red[q][tid];
        w.rp[(size_t)(row0 + tid) * w.nResTiles + tile] = s;
    }
}

// Replacement token of a queued rejection: thread t owns the contiguous tile
// sums [t K, t K + K) (loaded before any barrier), one block scan gives Q and
// the thread whose range holds u Q, which walks its sums to the crossing
// tile; the block recomputes that tile's q values and scans them.
constexpr int kResChunk = 8;   // tile sums per thread held in registers

template <typename T>
__global__ void __launch_bounds__(kRowThreads) residual_final(
    const T *__restrict__ Tlog, const T *__restrict__ L, const T *__restrict__ U,
    const T *__restrict__ Wt, const int32_t *__restrict__ x0, const int32_t *__restrict__ x,
    const float *__restrict__ H, const float *__restrict__ rowmax, const float *__restrict__ rowsum,
    const float *__restrict__ temp, const float *__restrict__ u_final, int G, int V, int r,
    VerifyWs w, int32_t *__restrict__ tokens_out) {
    extern __shared__ float res_smem[];
    float *urow = res_smem;   // [r]
    __shared__ float s_loc[32], s_col[32];
    __shared__ int s_own[32], s_own2[32], s_y[32], s_y2[32];
    __shared__ int ts_s;
    __shared__ float rem_s;
    const int s = blockIdx.x, tid = threadIdx.x, nthr = blockDim.x;
    const int nres = *reinterpret_cast<volatile uint32_t *>(&w.hdr->pad[1]);
    if (s >= nres) return;
    const int nT = w.nResTiles;
    const float *tp = w.rp + (size_t)s * nT;
    const int K = (nT + nthr - 1) / nthr;
    const int t0 = min(nT, tid * K), t1 = min(nT, t0 + K);
    float cq[kResChunk];
#pragma unroll
    for (int q = 0; q < kResChunk; ++q) cq[q] = t0 + q < t1 ? tp[t0 + q] : 0.f;
    const int b = w.res_b[s], k = w.res_k[s];
    const size_t ro = (size_t)b * G + k;
    const float Tb = fmaxf(temp[b], 0.f), invT = 1.f / Tb;
    const float Md = rowmax[ro], Zd = rowsum[ro], Mt = w.res_mt[s], Zt = w.res_zt[s];
    const float u = u_final[b];
    // The rejected position's A row in fp32: U[previous token] (Markov head)
    // or the state that biased it (RNN head).
    float uv0, uv1;
    if (H != nullptr) {   // as the residual tile pass's split product saw it
        uv0 = tid < r ? split_bf16_sum(H[ro * r + tid]) : 0.f;
        uv1 = tid + nthr < r ? split_bf16_sum(H[ro * r + tid + nthr]) : 0.f;
    } else {
        const int prev = min(max((k == 0) ? x0[b] : x[ro - 1], 0), V - 1);
        uv0 = tid < r ? ld_elem(U, (size_t)prev * r + tid) : 0.f;
        uv1 = tid + nthr < r ? ld_elem(U, (size_t)prev * r + tid + nthr) : 0.f;
    }
    float loc = 0.f;
#pragma unroll
    for (int q = 0; q < kResChunk; ++q) loc += cq[q];
    for (int t = t0 + kResChunk; t < t1; ++t) loc += tp[t];   // very large vocabularies only
    if (tid < r) urow[tid] = uv0;
    if (tid + nthr < r) urow[tid + nthr] = uv1;
    float Q;
    const float incl = block_scan1(loc, s_loc, &Q);   // also publishes urow
    int y;
    if (!(Q > 0.f)) {  // empty residual (block-uniform): draw from p_t of the rejected row
        y = sample_target_row(Tlog, w, w.row_off[b] + k, b, k, G, V, Mt, Zt, invT, u);
    } else {
        const float target = u * Q;
        int owner = block_min1((incl > target && loc > 0.f) ? tid : 0x7fffffff, s_own);
        const bool past_mass = owner == 0x7fffffff;   // rounding left u Q at the top: a tie by definition
        if (past_mass) owner = max(0, block_max1_i(loc > 0.f ? tid : -1, s_own2));
        if (tid == owner) {
            float run = incl - loc, run_last = run;
            int ts = -1, last = t1 - 1;
#pragma unroll
            for (int q = 0; q < kResChunk; ++q) {
                if (ts < 0 && t0 + q < t1) {
                    if (run + cq[q] > target) {
                        ts = t0 + q;
                    } else {
                        if (cq[q] > 0.f) { last = t0 + q; run_last = run; }
                        run += cq[q];
                    }
                }
            }
            for (int t = t0 + kResChunk; t < t1 && ts < 0; ++t) {
                const float wt = tp[t];
                if (run + wt > target) {
                    ts = t;
                } else {
                    if (wt > 0.f) { last = t; run_last = run; }
                    run += wt;
                }
            }
            if (ts < 0) { ts = last; run = run_last; }
            ts_s = max(ts, 0);
            rem_s = target - run;
        }
        __syncthreads();
        const int ts = ts_s;
        const float rem = rem_s;
        // tpc consecutive threads share one column's dot product.
        const int TN = w.resCols;
        const int c0 = ts * TN;
        const int tpc = nthr / TN;
        const int col = c0 + tid / tpc, part = tid % tpc;
        const bool mine = part == 0 && col < V;
        const float lval = mine ? ld_elem(L, ro * V + col) : 0.f;
        const float tval = mine ? ld_elem(Tlog, ((size_t)b * (G + 1) + k) * V + col) : 0.f;
        float dl = 0.f;
        if (col < V) dl = dot_part(urow, Wt + (size_t)col * r, r, part, tpc);
        for (int o = tpc >> 1; o > 0; o >>= 1) dl += __shfl_xor_sync(0xffffffffu, dl, o);
        float qv = 0.f;
        if (mine) {
            const float pd = exp_e(((lval - Md) + dl) * invT) / Zd;
            const float pt = exp_e((tval - Mt) * invT) / Zt;
            qv = fmaxf(pt - pd, 0.f);
        }
        float tot;
        const float inc = block_scan1(qv, s_col, &tot);
        int ys = block_min1((mine && qv > 0.f && inc > rem) ? col : 0x7fffffff, s_y);
        const bool fell_short = ys == 0x7fffffff;
        if (fell_short) {
            ys = block_max1_i((mine && qv > 0.f) ? col : -1, s_y2);
            if (ys < 0) ys = min(c0 + TN, V) - 1;
        }
        if (mine && col == ys) {
            // The residual draw's margin: u Q to the nearer edge of the token's interval, over Q.
            const float margin = (past_mass || fell_short) ? 0.f : fminf(rem - (inc - qv), inc - rem) / Q;
            if (margin < kNearTie) count_near_tie(w.hdr, kPadVerifyTies);
        }
        y = ys;
    }
    if (tid == 0) tokens_out[(size_t)b * (G + 1) + k] = y;
}

// ----------------------------------------------------------------- host
// ----------------------------------------------------------------- diagnostics
__global__ void exp2_fma_kernel(const float *__restrict__ x, float *__restrict__ y, int n) {
    const int i = (blockIdx.x * blockDim.x + threadIdx.x) * 2;
    if (i + 1 < n) {
        const float2 v = exp2_poly2(make_float2(x[i], x[i + 1]));
        y[i] = v.x;
        y[i + 1] = v.y;
    } else if (i < n) {
        y[i] = exp2_poly2(make_float2(x[i], 0.f)).x;
    }
}

cudaError_t launch_exp2_fma(const float *x, float *y, int n, cudaStream_t st) {
    const int pairs = (n + 1) / 2;
    exp2_fma_kernel<<<(pairs + 255) / 256, 256, 0, st>>>(x, y, n);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_verify_t(const VerifyArgs &a, const VerifyWs &w, cudaStream_t st) {
    const T *Tl = static_cast<const T *>(a.Tlog);
    verify_plan<<<1, std::min(1024, (a.B + 31) / 32 * 32), 0, st>>>(a.ell, a.B, a.G, w);   // one thread per request
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int maxwork = a.B * (a.G + 1) * w.nChunks;
    if (a.dtype == DSPARK_BF16) {
        const int grid = max(1, min(maxwork, sms));
        const size_t smem = vr_smem_bytes(a.B);
        if ((e = cudaFuncSetAttribute(verify_rows_bulk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
            cudaSuccess)
            return e;
        verify_rows_bulk<<<grid, kVrThreads, smem, st>>>(static_cast<const __nv_bfloat16 *>(a.Tlog), a.temp, a.B,
                                                         a.G, a.V, w, wait_budget(kVrWaitBudget));
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    } else {
        const int grid = max(1, min(maxwork, sms * 8));
        verify_rows<T><<<grid, kRowThreads, 0, st>>>(Tl, a.temp, a.G, a.V, w);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    verify_decide<T><<<a.B, kRowThreads, 0, st>>>(Tl, static_cast<const T *>(a.U), a.x0, a.r, a.x, a.pd_x, a.temp,
                                                  a.u_accept, a.u_final, a.ell, a.B, a.G, a.V, w, a.acc_out,
                                                  a.tokens_out, a.nout_out, a.pt_x_out);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (a.dtype == DSPARK_BF16) {
        ResidualTcArgs ra{a.Wt, static_cast<const __nv_bfloat16 *>(a.U), static_cast<const __nv_bfloat16 *>(a.L),
                          static_cast<const __nv_bfloat16 *>(a.Tlog), a.x0, a.x, a.H, a.temp, a.rowmax, a.rowsum, w.res_mt,
                          w.res_zt, w.res_b, w.res_k, &w.hdr->pad[1], a.B, a.G, a.V, a.r, w.nResTiles, w.rp, w.hdr};
        if ((e = launch_residual_tile_tc(ra, st)) != cudaSuccess) return e;
    } else {
        dim3 rg(w.nResTiles, (a.B + kResRows - 1) / kResRows);
        residual_tile_simt<T><<<rg, 256, 0, st>>>(Tl, static_cast<const T *>(a.L), static_cast<const T *>(a.U),
                                                  static_cast<const T *>(a.Wt), a.x0, a.x, a.rowmax,
                                                  a.rowsum, a.temp, a.G, a.V, a.r, w);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    const size_t smem = sizeof(float) * (size_t)a.r;
    auto fin = residual_final<T>;
    if (smem > 48 * 1024) {
        if ((e = cudaFuncSetAttribute(fin, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
            cudaSuccess)
            return e;
    }
    fin<<<a.B, kRowThreads, smem, st>>>(Tl, static_cast<const T *>(a.L), static_cast<const T *>(a.U),
                                       static_cast<const T *>(a.Wt), a.x0, a.x, a.H, a.rowmax, a.rowsum, a.temp,
                                       a.u_final, a.G, a.V, a.r, w, a.tokens_out);
    return cudaGetLastError();
}

cudaError_t launch_verify(const VerifyArgs &a, void *ws, cudaStream_t st) {
    VerifyWs w = carve_verify_ws(ws, a.B, a.G, a.V, a.r, a.dtype);
    if (a.dtype == DSPARK_BF16) return launch_verify_t<__nv_bfloat16>(a, w, st);
    return launch_verify_t<float>(a, w, st);
}

}  // namespace dspark
