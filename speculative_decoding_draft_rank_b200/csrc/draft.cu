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
#include "finalize.cuh"
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
    float2 *__restrict__ part, WsHeader *hdr)
{
    __shared__ float Es[kSimtRows][33];
    __shared__ int prev_s[kSimtRows];
    __shared__ float red_v[8][kSimtRows];
    __shared__ int red_i[8][kSimtRows];
    __shared__ float row_m[kSimtRows];
    __shared__ int row_a[kSimtRows];
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
        row_a[tid] = ix;
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
        part[(size_t)(row0 + tid) * nTiles + tile] =
            make_float2(row_m[tid], row_invT[tid] > 0.f ? s : __int_as_float(row_a[tid]));
    }
}

// out[c][q] = in[q][c] for an n x n bf16 matrix (32 x 32 tiles through shared
// memory, 32 x 8 threads).
__global__ void transpose_bf16(const __nv_bfloat16 *__restrict__ in, __nv_bfloat16 *__restrict__ out, int n) {
    __shared__ __nv_bfloat16 tile[32][33];
    const int x0 = blockIdx.x * 32, y0 = blockIdx.y * 32;
    for (int j = threadIdx.y; j < 32; j += 8) {
        const int y = y0 + j, x = x0 + threadIdx.x;
        if (y < n && x < n) tile[j][threadIdx.x] = in[(size_t)y * n + x];
    }
    __syncthreads();
    for (int j = threadIdx.y; j < 32; j += 8) {
        const int y = x0 + j, x = y0 + threadIdx.x;   // out row = in column
        if (y < n && x < n) out[(size_t)y * n + x] = tile[threadIdx.x][j];
    }
}

// ---------------------------------------------------------------------------
// Finalize (fp32 rounds): one CTA of kFinThreads threads per request row, the
// row work in finalize.cuh.
constexpr int kFinThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kFinThreads) draft_finalize(const FinArgs a, int pos) {
    __shared__ FinScratch sc;
    __shared__ float urow[512];
    const Grp g{(int)threadIdx.x, (int)blockDim.x, (int)(threadIdx.x >> 5), (int)(blockDim.x >> 5), 0};
    finalize_row<T>(g, &sc, urow, a, blockIdx.x, pos);
}

// ---------------------------------------------------------------------------
// Host side.
size_t draft_tiles(int V, int dtype) { return (size_t)((V + draft_tile_cols(dtype) - 1) / draft_tile_cols(dtype)); }

int draft_tile_cols(int dtype) { return dtype == DSPARK_BF16 ? kTcTileN : kSimtCols; }

size_t draft_ws_bytes(int B, int G, int V, int r, int dtype) {
    size_t nt = draft_tiles(V, dtype);
    size_t bytes = sizeof(WsHeader);
    bytes += align256(sizeof(float2) * (size_t)B * nt);   // part
    if (dtype == DSPARK_BF16) bytes += align256((size_t)2 * B * r * 2);   // E (the RNN head stages two parts)
    if (dtype == DSPARK_BF16) bytes += align256((size_t)r * r * 2);       // the RNN head's transposed A
    return bytes;
}

DraftWs carve_draft_ws(void *ws, int B, int V, int r, int dtype) {
    DraftWs w;
    size_t nt = draft_tiles(V, dtype);
    char *p = static_cast<char *>(ws);
    w.hdr = reinterpret_cast<WsHeader *>(p);
    p += sizeof(WsHeader);
    w.part = reinterpret_cast<float2 *>(p); p += align256(sizeof(float2) * (size_t)B * nt);
    w.E = nullptr;
    w.AT = nullptr;
    if (dtype == DSPARK_BF16) { w.E = reinterpret_cast<__nv_bfloat16 *>(p); p += align256((size_t)2 * B * r * 2); }
    if (dtype == DSPARK_BF16) { w.AT = reinterpret_cast<__nv_bfloat16 *>(p); p += align256((size_t)r * r * 2); }
    w.nTiles = (int)nt;
    return w;
}

FinArgs fin_args(const DraftArgs &a, const DraftWs &w) {
    FinArgs f{};
    f.L = a.L; f.U = a.U; f.Wt = a.Wt; f.x0 = a.x0; f.temp = a.temp; f.u_draft = a.u_draft;
    f.B = a.B; f.G = a.G; f.V = a.V; f.r = a.r; f.nTiles = w.nTiles; f.TN = draft_tile_cols(a.dtype);
    f.part = w.part;
    f.x_out = a.x_out; f.pd_out = a.pd_out; f.rowmax_out = a.rowmax_out; f.rowsum_out = a.rowsum_out;
    f.E = w.E; f.hdr = w.hdr;
    f.Arec = static_cast<const __nv_bfloat16 *>(a.Arec);
    f.ArecT = w.AT;
    f.H = a.H_out;
    return f;
}

cudaError_t launch_draft(const DraftArgs &a, void *ws, cudaStream_t st) {
    DraftWs w = carve_draft_ws(ws, a.B, a.V, a.r, a.dtype);
    const FinArgs f = fin_args(a, w);
    // bf16: more than 128 requests (and every RNN-head round) on CTA pairs;
    // the RNN head's recurrent matrix is transposed into the workspace first.
    if (a.dtype == DSPARK_BF16) {
        if (a.H_out != nullptr) {
            dim3 grid((a.r + 31) / 32, (a.r + 31) / 32);
            transpose_bf16<<<grid, dim3(32, 8), 0, st>>>(static_cast<const __nv_bfloat16 *>(a.Arec), w.AT, a.r);
            cudaError_t e = cudaGetLastError();
            if (e != cudaSuccess) return e;
        }
        return (a.B > 128 || a.H_out != nullptr) ? launch_draft_pair(a, w, f, st) : launch_draft_tc(a, w, f, st);
    }
    cudaError_t e;
    for (int pos = 0; pos < a.G; ++pos) {
        dim3 grid(w.nTiles, (a.B + kSimtRows - 1) / kSimtRows);
        draft_tile_simt<float><<<grid, 256, 0, st>>>(
            static_cast<const float *>(a.L), static_cast<const float *>(a.U), static_cast<const float *>(a.Wt),
            a.x0, a.x_out, a.temp, a.B, a.G, a.V, a.r, pos, w.nTiles, w.part, w.hdr);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        draft_finalize<float><<<a.B, kFinThreads, 0, st>>>(f, pos);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace dspark
