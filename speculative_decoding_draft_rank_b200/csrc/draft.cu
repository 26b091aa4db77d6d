// draft.cu -- stage 1, semi-autoregressive drafting with the Markov head.
//
// Method (paperlayer.ai summary of DSpark, §3.1 Semi-autoregressive
// generation; llm-wiki.hwlabs.dev study 116, draft-generation figure): for
// positions i = 1..G in turn, the backbone logits L[i] get the bias
// Delta_i = U[x_{i-1}] W, then a temperature softmax and an inverse-CDF draw.
//
// Per position two launches:
//   tile kernel   Delta tile (GEMM over the rank r) fused with the softmax
//                 epilogue: per (row, column tile) the max of y = L + Delta,
//                 the sum of exp((y - max) / T) and the argmax.  Delta never
//                 reaches HBM.  (bf16 rounds use the tcgen05 kernel of
//                 draft_tc.cu; this file holds the CUDA-core kernel used for
//                 fp32 rounds.)
//   finalize      one CTA per row: combines the tile partials into (max, Z),
//                 finds the tile where u Z falls by a prefix scan over the
//                 tile sums, recomputes that one tile's values and scans it to
//                 the sampled token; writes x_i, p_d(x_i), max and Z.
#include "common.cuh"
#include "kernels.cuh"

namespace dspark {

// ---------------------------------------------------------------------------
// CUDA-core tile kernel: 32 rows x 256 columns per CTA of 256 threads.  Each
// thread owns one column and accumulates Delta for the 32 rows over the rank.
constexpr int kSimtRows = 32;
constexpr int kSimtCols = 256;

template <typename T>
__global__ void __launch_bounds__(256) draft_tile_simt(
    const T *__restrict__ L, const T *__restrict__ U, const T *__restrict__ Wt,
    const int32_t *__restrict__ x0, const int32_t *__restrict__ xprev_base,
    const float *__restrict__ temp, int B, int G, int V, int r, int pos, int nTiles,
    float *__restrict__ part_m, float *__restrict__ part_s, int32_t *__restrict__ part_a,
    WsHeader *hdr)
{
    __shared__ float Es[kSimtRows][33];
    __shared__ int prev_s[kSimtRows];
    __shared__ float red_v[8][kSimtRows];
    __shared__ int red_i[8][kSimtRows];
    __shared__ float row_m[kSimtRows];
    __shared__ float row_invT[kSimtRows];

    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int tile = blockIdx.x;
    const int row0 = blockIdx.y * kSimtRows;
    const int col = tile * kSimtCols + tid;
    const bool colok = col < V;

    if (tid < kSimtRows) {
        int b = row0 + tid, p = 0;
        float invT = 0.f;
        if (b < B) {
            p = (pos == 0) ? clamp_token(x0[b], V, hdr) : xprev_base[(size_t)b * G + pos - 1];
            float Tb = sane_temp(temp[b], hdr);
            invT = Tb > 0.f ? 1.f / Tb : 0.f;
        }
        prev_s[tid] = p;
        row_invT[tid] = invT;
    }

    float acc[kSimtRows];
#pragma unroll
    for (int j = 0; j < kSimtRows; ++j) acc[j] = 0.f;

    for (int k0 = 0; k0 < r; k0 += 32) {
        __syncthreads();
        for (int e = tid; e < kSimtRows * 32; e += blockDim.x) {
            int rr = e >> 5, kk = e & 31;
            float v = 0.f;
            if (row0 + rr < B && k0 + kk < r) v = ld_elem(U, (size_t)prev_s[rr] * r + k0 + kk);
            Es[rr][kk] = v;
        }
        __syncthreads();
        float wv[32];
#pragma unroll
        for (int kk = 0; kk < 32; ++kk)
            wv[kk] = (colok && k0 + kk < r) ? ld_elem(Wt, (size_t)col * r + k0 + kk) : 0.f;
#pragma unroll
        for (int j = 0; j < kSimtRows; ++j) {
            float a = acc[j];
#pragma unroll
            for (int kk = 0; kk < 32; ++kk) a = fmaf(Es[j][kk], wv[kk], a);
            acc[j] = a;
        }
    }

    // Epilogue, phase 1: per-row max of y = L + Delta and its lowest argmax.
    float lv[kSimtRows];
#pragma unroll
    for (int j = 0; j < kSimtRows; ++j) {
        int b = row0 + j;
        float l = 0.f, y = -INFINITY;
        if (b < B && colok) {
            l = ld_elem(L, ((size_t)b * G + pos) * V + col);
            y = l + acc[j];
        }
        lv[j] = l;
        float v = y;
        int ix = colok ? col : 0x7fffffff;
        warp_argmax(v, ix);
        if (lane == 0) { red_v[wid][j] = v; red_i[wid][j] = ix; }
    }
    __syncthreads();
    if (tid < kSimtRows) {
        float v = red_v[0][tid];
        int ix = red_i[0][tid];
        for (int w = 1; w < 8; ++w) {
            float ov = red_v[w][tid];
            int oi = red_i[w][tid];
            if (ov > v || (ov == v && oi < ix)) { v = ov; ix = oi; }
        }
        row_m[tid] = v;
        int b = row0 + tid;
        if (b < B) {
            part_m[(size_t)b * nTiles + tile] = v;
            part_a[(size_t)b * nTiles + tile] = ix;
        }
    }
    __syncthreads();
    // Phase 2: sum of exp(((L - m) + Delta) / T) over the tile.
#pragma unroll
    for (int j = 0; j < kSimtRows; ++j) {
        float e = 0.f;
        if (row0 + j < B && colok && row_invT[j] > 0.f)
            e = exp_e(((lv[j] - row_m[j]) + acc[j]) * row_invT[j]);
        e = warp_sum(e);
        if (lane == 0) red_v[wid][j] = e;
    }
    __syncthreads();
    if (tid < kSimtRows && row0 + tid < B) {
        float s = 0.f;
        for (int w = 0; w < 8; ++w) s += red_v[w][tid];
        part_s[(size_t)(row0 + tid) * nTiles + tile] = s;
    }
}

// ---------------------------------------------------------------------------
// Finalize: one CTA of kFinThreads threads per request row.  Thread t owns the
// contiguous partials [t K, t K + K) and loads them (with the previous token
// and its U row) before any barrier, so the stage costs a few dependent
// memory round trips: one block max, one block scan of the threads' scaled
// partial sums, then the thread whose range holds u Z walks its partials to
// the crossing one, whose columns the block recomputes and scans.
constexpr int kFinThreads = 256;
constexpr int kFinChunk = 8;   // partials per thread held in registers

template <typename T>
__global__ void __launch_bounds__(kFinThreads) draft_finalize(
    const T *__restrict__ L, const T *__restrict__ U, const T *__restrict__ Wt,
    const int32_t *__restrict__ x0, const float *__restrict__ temp,
    const float *__restrict__ u_draft, int B, int G, int V, int r, int pos, int nTiles, int TN,
    const float *__restrict__ part_m, const float *__restrict__ part_s,
    const int32_t *__restrict__ part_a, int32_t *__restrict__ x_out, float *__restrict__ pd_out,
    float *__restrict__ rowmax_out, float *__restrict__ rowsum_out, __nv_bfloat16 *__restrict__ E,
    WsHeader *hdr)
{
    extern __shared__ float fin_smem[];
    float *urow = fin_smem;                 // [r] U[x_{i-1}] row
    __shared__ float s_max[32], s_loc[32], s_col[32];
    __shared__ int s_own[32], s_own2[32], s_x[32], s_x2[32];
    __shared__ int ts_s, xg_s;
    __shared__ float rem_s;

    const int b = blockIdx.x, tid = threadIdx.x, nthr = blockDim.x;
    const size_t ro = (size_t)b * G + pos;
    // bf16 rounds: the sampled token's U row is staged in E[b] for the next
    // position's tensor-core pass (16-byte pieces; r is a multiple of 16).
    auto stage_next = [&](int x) {
        if (E != nullptr && pos + 1 < G)
            for (int q = tid; q < r / 8; q += nthr)
                reinterpret_cast<uint4 *>(E + (size_t)b * r)[q] = ld_nc16(U + (size_t)x * r + q * 8);
    };
    const float *pm = part_m + (size_t)b * nTiles;
    const float *ps = part_s + (size_t)b * nTiles;
    const int K = (nTiles + nthr - 1) / nthr;
    const int t0 = min(nTiles, tid * K), t1 = min(nTiles, t0 + K);

    // Every load that depends on nothing else goes out first.
    float cm[kFinChunk], cs[kFinChunk];
#pragma unroll
    for (int q = 0; q < kFinChunk; ++q) {
        const bool in = t0 + q < t1;
        cm[q] = in ? pm[t0 + q] : -INFINITY;
        cs[q] = in ? ps[t0 + q] : 0.f;
    }
    const float Tb = sane_temp(temp[b], hdr);
    const float u = u_draft[ro];
    const int prev = (pos == 0) ? clamp_token(x0[b], V, hdr) : x_out[(size_t)b * G + pos - 1];
    // The previous token's U row (r <= 512 = 2 x kFinThreads), kept in
    // registers until after the first barrier.
    const float uv0 = tid < r ? ld_elem(U, (size_t)prev * r + tid) : 0.f;
    const float uv1 = tid + nthr < r ? ld_elem(U, (size_t)prev * r + tid + nthr) : 0.f;

    float m = -INFINITY;
#pragma unroll
    for (int q = 0; q < kFinChunk; ++q) m = fmaxf(m, cm[q]);
    for (int t = t0 + kFinChunk; t < t1; ++t) m = fmaxf(m, pm[t]);   // very large vocabularies only
    const float M = block_max1(m, s_max);

    if (Tb == 0.f) {   // greedy row (block-uniform): lowest argmax over the partials
        int first = 0x7fffffff;
        for (int t = t1 - 1; t >= t0 + kFinChunk; --t)
            if (pm[t] == M) first = t;
#pragma unroll
        for (int q = kFinChunk - 1; q >= 0; --q)
            if (t0 + q < t1 && cm[q] == M) first = t0 + q;
        first = block_min1(first, s_own);
        if (tid == 0) {
            if (first >= nTiles) first = 0;  // no partial matched (non-finite inputs)
            int x = part_a[(size_t)b * nTiles + first];
            if (x < 0 || x >= V) x = 0;
            x_out[ro] = x;
            pd_out[ro] = 1.f;
            rowmax_out[ro] = M;
            rowsum_out[ro] = 1.f;
            xg_s = x;
        }
        if (E != nullptr && pos + 1 < G) {
            __syncthreads();
            stage_next(xg_s);
        }
        return;
    }

    const float cexp = kLog2e / Tb;
    float loc = 0.f;
#pragma unroll
    for (int q = 0; q < kFinChunk; ++q) loc += cs[q] * fast_exp2((cm[q] - M) * cexp);
    for (int t = t0 + kFinChunk; t < t1; ++t) loc += ps[t] * fast_exp2((pm[t] - M) * cexp);
    if (tid < r) urow[tid] = uv0;
    if (tid + nthr < r) urow[tid + nthr] = uv1;
    float Z;
    const float incl = block_scan1(loc, s_loc, &Z);   // also publishes urow
    const float target = u * Z;
    // The first thread whose inclusive prefix passes u Z owns the crossing
    // (the last thread with mass if rounding left u Z at the top).
    int owner = block_min1((incl > target && loc > 0.f) ? tid : 0x7fffffff, s_own);
    if (owner == 0x7fffffff) owner = max(0, block_max1_i(loc > 0.f ? tid : -1, s_own2));
    if (tid == owner) {
        float run = incl - loc, run_last = run;
        int ts = -1, last = t1 - 1;
#pragma unroll
        for (int q = 0; q < kFinChunk; ++q) {
            if (ts < 0 && t0 + q < t1) {
                const float wt = cs[q] * fast_exp2((cm[q] - M) * cexp);
                if (run + wt > target) {
                    ts = t0 + q;
                } else {
                    if (wt > 0.f) { last = t0 + q; run_last = run; }
                    run += wt;
                }
            }
        }
        for (int t = t0 + kFinChunk; t < t1 && ts < 0; ++t) {
            const float wt = ps[t] * fast_exp2((pm[t] - M) * cexp);
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
    // Recompute the chosen partial's columns: tpc consecutive threads share one column.
    const int c0 = ts * TN;
    const int tpc = nthr / TN;
    const int col = c0 + tid / tpc, part = tid % tpc;
    const bool mine = part == 0 && col < V;
    const float lval = mine ? ld_elem(L, ro * V + col) : 0.f;   // issued with the factor loads
    float dl = 0.f;
    if (col < V) dl = dot_part(urow, Wt + (size_t)col * r, r, part, tpc);
    for (int o = tpc >> 1; o > 0; o >>= 1) dl += __shfl_xor_sync(0xffffffffu, dl, o);
    const float e = mine ? fast_exp2(((lval - M) + dl) * cexp) : 0.f;
    float ttot;
    const float inc = block_scan1(e, s_col, &ttot);
    int xs = block_min1((mine && inc > rem) ? col : 0x7fffffff, s_x);
    if (xs == 0x7fffffff) {  // the recomputed mass fell short: last positive column
        xs = block_max1_i((mine && e > 0.f) ? col : -1, s_x2);
        if (xs < 0) xs = min(c0 + TN, V) - 1;
    }
    if (mine && col == xs) {
        x_out[ro] = xs;
        pd_out[ro] = e / Z;
        rowmax_out[ro] = M;
        rowsum_out[ro] = Z;
    }
    stage_next(xs);
}

// ---------------------------------------------------------------------------
// Host side.
size_t draft_tiles(int V, int dtype) { return (size_t)((V + draft_tile_cols(dtype) - 1) / draft_tile_cols(dtype)); }

int draft_tile_cols(int dtype) { return dtype == DSPARK_BF16 ? kTcTileN : kSimtCols; }

size_t draft_ws_bytes(int B, int G, int V, int r, int dtype) {
    size_t nt = draft_tiles(V, dtype);
    size_t bytes = sizeof(WsHeader);
    bytes += align256(sizeof(float) * (size_t)B * nt);    // part_m
    bytes += align256(sizeof(float) * (size_t)B * nt);    // part_s
    bytes += align256(sizeof(int32_t) * (size_t)B * nt);  // part_a
    if (dtype == DSPARK_BF16) bytes += align256((size_t)B * r * 2);   // E
    return bytes;
}

DraftWs carve_draft_ws(void *ws, int B, int V, int r, int dtype) {
    DraftWs w;
    size_t nt = draft_tiles(V, dtype);
    char *p = static_cast<char *>(ws);
    w.hdr = reinterpret_cast<WsHeader *>(p);
    p += sizeof(WsHeader);
    w.part_m = reinterpret_cast<float *>(p); p += align256(sizeof(float) * (size_t)B * nt);
    w.part_s = reinterpret_cast<float *>(p); p += align256(sizeof(float) * (size_t)B * nt);
    w.part_a = reinterpret_cast<int32_t *>(p); p += align256(sizeof(int32_t) * (size_t)B * nt);
    w.E = nullptr;
    if (dtype == DSPARK_BF16) { w.E = reinterpret_cast<__nv_bfloat16 *>(p); p += align256((size_t)B * r * 2); }
    w.nTiles = (int)nt;
    return w;
}

template <typename T>
static cudaError_t launch_finalize(const DraftArgs &a, const DraftWs &w, int pos, cudaStream_t st) {
    size_t smem = sizeof(float) * (size_t)a.r;
    auto kern = draft_finalize<T>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    kern<<<a.B, kFinThreads, smem, st>>>(static_cast<const T *>(a.L), static_cast<const T *>(a.U),
                                         static_cast<const T *>(a.Wt), a.x0, a.temp, a.u_draft, a.B, a.G, a.V,
                                         a.r, pos, w.nTiles, draft_tile_cols(a.dtype), w.part_m, w.part_s,
                                         w.part_a, a.x_out, a.pd_out, a.rowmax_out, a.rowsum_out,
                                         reinterpret_cast<__nv_bfloat16 *>(w.E), w.hdr);
    return cudaGetLastError();
}

cudaError_t launch_draft(const DraftArgs &a, void *ws, cudaStream_t st) {
    DraftWs w = carve_draft_ws(ws, a.B, a.V, a.r, a.dtype);
    cudaError_t e;
    for (int pos = 0; pos < a.G; ++pos) {
        if (a.dtype == DSPARK_F32) {
            dim3 grid(w.nTiles, (a.B + kSimtRows - 1) / kSimtRows);
            draft_tile_simt<float><<<grid, 256, 0, st>>>(
                static_cast<const float *>(a.L), static_cast<const float *>(a.U),
                static_cast<const float *>(a.Wt), a.x0, a.x_out, a.temp, a.B, a.G, a.V, a.r, pos,
                w.nTiles, w.part_m, w.part_s, w.part_a, w.hdr);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
            if ((e = launch_finalize<float>(a, w, pos, st)) != cudaSuccess) return e;
        } else {
            // bf16: tensor-core tile kernel (its A rows are U[previous token]).
            if ((e = launch_draft_tile_tc(a, w, pos, st)) != cudaSuccess) return e;
            if ((e = launch_finalize<__nv_bfloat16>(a, w, pos, st)) != cudaSuccess) return e;
        }
    }
    return cudaSuccess;
}

}  // namespace dspark
