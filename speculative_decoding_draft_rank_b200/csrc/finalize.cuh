// finalize.cuh -- the per-row end of one drafting position, shared by the
// standalone finalize kernel (fp32 rounds) and the persistent tensor-core
// drafting kernel (bf16 rounds).
//
// Method (paperlayer.ai summary of DSpark, §3.1 Semi-autoregressive
// generation: each position's token is drawn from the temperature softmax of
// L[i] + Delta_i; the draw here is the inverse CDF at the round's uniform u):
// the tile partials (max, sum of exp((y - max) / T), lowest argmax) of a row
// are combined into the row's max M and normaliser Z; the partial where the
// running mass passes u Z is found by a prefix over the partials, its columns
// are recomputed (Delta from U[x_{i-1}] and W) and scanned to the token.
#pragma once

#include "common.cuh"

namespace dspark {

// A group of whole warps working on one row: its thread index, size, warp
// index and warp count, and the named barrier it synchronises on (0 with the
// whole CTA as the group means __syncthreads).
struct Grp {
    int tid, n, wid, nw, bar;
    __device__ __forceinline__ void sync() const {
        if (bar == 0) __syncthreads();
        else asm volatile("bar.sync %0, %1;" ::"r"(bar), "r"(n) : "memory");
    }
};

// One-barrier group reductions (every warp publishes into its own entry of
// `slots`; each call site owns its slots, so no trailing barrier is needed).
__device__ __forceinline__ float grp_max1(const Grp &g, float v, float *slots) {
    v = warp_max(v);
    if ((threadIdx.x & 31) == 0) slots[g.wid] = v;
    g.sync();
    float r = slots[0];
    for (int w = 1; w < g.nw; ++w) r = fmaxf(r, slots[w]);
    return r;
}
__device__ __forceinline__ int grp_min1(const Grp &g, int v, int *slots) {
    v = warp_min_i(v);
    if ((threadIdx.x & 31) == 0) slots[g.wid] = v;
    g.sync();
    int r = slots[0];
    for (int w = 1; w < g.nw; ++w) r = min(r, slots[w]);
    return r;
}
__device__ __forceinline__ int grp_max1_i(const Grp &g, int v, int *slots) { return -grp_min1(g, -v, slots); }
__device__ __forceinline__ float grp_scan1(const Grp &g, float v, float *slots, float *total) {
    const float s = warp_incl_scan(v);
    if ((threadIdx.x & 31) == 31) slots[g.wid] = s;
    g.sync();
    float before = 0.f, tot = 0.f;
    for (int w = 0; w < g.nw; ++w) {
        if (w == g.wid) before = tot;
        tot += slots[w];
    }
    *total = tot;
    return before + s;
}

// Shared-memory scratch of one group (at most 8 warps).
struct FinScratch {
    float s_max[8], s_loc[8], s_col[8];
    int s_own[8], s_own2[8], s_x[8], s_x2[8];
    int ts, xg;
    float rem;
};


constexpr int kFinChunk = 8;   // partials per thread held in registers

struct FinArgs {
    const void *L, *U, *Wt;
    const int32_t *x0;
    const float *temp, *u_draft;
    int B, G, V, r, nTiles, TN;   // TN: columns per partial
    const float2 *part;            // [B, nTiles] (max, sum of exps or argmax bits)
    int32_t *x_out;
    float *pd_out, *rowmax_out, *rowsum_out;
    __nv_bfloat16 *E;              // bf16 rounds: the next position's A rows staged for TMA, else null
    // RNN head (null for the Markov head): the recurrent matrix Arec [r, r]
    // and the states H [B, G, r] fp32 (row b*G + i holds the state that
    // biases position i); E then holds the next state split into bf16 high
    // parts (rows 0..B-1) and low parts (rows B..2B-1).
    const __nv_bfloat16 *Arec;
    const __nv_bfloat16 *ArecT;    // its transpose [r, r] (row c = column c), staged per launch
    float *H;
    WsHeader *hdr;
};

// Row b at position pos.  Thread t of the group owns the contiguous partials
// [t K, t K + K) and loads them (with the previous token and its U row) before
// any barrier: one group max, one group scan of the threads' scaled partial
// sums, then the thread whose range holds u Z walks its partials to the
// crossing one, whose TN columns the group recomputes and scans.  urow holds
// r floats.  Ends with a group barrier, so the scratch may be reused.
template <typename T>
__device__ void finalize_row(const Grp &g, FinScratch *sc, float *urow, const FinArgs &a, int b, int pos) {
    const T *L = static_cast<const T *>(a.L);
    const T *U = static_cast<const T *>(a.U);
    const T *Wt = static_cast<const T *>(a.Wt);
    const int B = a.B, G = a.G, V = a.V, r = a.r, nTiles = a.nTiles, TN = a.TN;
    const int tid = g.tid, nthr = g.n;
    const size_t ro = (size_t)b * G + pos;
    // bf16 rounds: the next position's A row is staged in E for its
    // tensor-core pass.  Markov head: the sampled token's U row (16-byte
    // pieces; r is a multiple of 16).  RNN head: the next state
    // h' = tanh(h A + U[x]) from this position's state h (in urow), written
    // to H and split into bf16 high and low parts (h' = hi + lo to about 2^-17
    // relative, so two MMAs reproduce the fp32 state's product).
    auto stage_next = [&](int x) {
        if (a.E == nullptr || pos + 1 >= G) return;
        if (a.H == nullptr) {
            for (int q = tid; q < r / 8; q += nthr)
                reinterpret_cast<uint4 *>(a.E + (size_t)b * r)[q] = ld_nc16(U + (size_t)x * r + q * 8);
            return;
        }
        for (int c = tid; c < r; c += nthr) {
            // (h A)[c] as the dot product of h with column c of A, a row of
            // the transposed copy: 16-byte loads, eight in flight, summed in
            // index order.
            float acc = dot_part(urow, a.ArecT + (size_t)c * r, r, 0, 1);
            acc += ld_elem(U, (size_t)x * r + c);
            const float hn = tanhf(acc);
            a.H[(ro + 1) * r + c] = hn;
            const __nv_bfloat16 hi = __float2bfloat16_rn(hn);
            a.E[(size_t)b * r + c] = hi;
            a.E[((size_t)B + b) * r + c] = __float2bfloat16_rn(hn - __bfloat162float(hi));
        }
    };
    const float2 *pp = a.part + (size_t)b * nTiles;
    const int K = (nTiles + nthr - 1) / nthr;
    const int t0 = min(nTiles, tid * K), t1 = min(nTiles, t0 + K);

    // Every load that depends on nothing else goes out first (the partials
    // as 16-byte pieces when the thread's eight are whole and aligned).  The
    // partials are rewritten at every position by other CTAs of the same
    // launch, so they are read past L1 (ld.global.cg), never through the
    // read-only path.
    float cm[kFinChunk], cs[kFinChunk];   // cs: sums of exps (sampled rows) or argmax bits (greedy rows)
    if (t0 + kFinChunk <= t1 && (reinterpret_cast<uintptr_t>(pp + t0) & 15) == 0) {
#pragma unroll
        for (int q = 0; q < kFinChunk / 2; ++q) {
            const float4 v = __ldcg(reinterpret_cast<const float4 *>(pp + t0 + 2 * q));
            cm[2 * q] = v.x; cs[2 * q] = v.y; cm[2 * q + 1] = v.z; cs[2 * q + 1] = v.w;
        }
    } else {
#pragma unroll
        for (int q = 0; q < kFinChunk; ++q) {
            const bool in = t0 + q < t1;
            const float2 v = in ? __ldcg(pp + t0 + q) : make_float2(-INFINITY, 0.f);
            cm[q] = v.x;
            cs[q] = v.y;
        }
    }
    const float Tb = sane_temp(a.temp[b], a.hdr);
    const float u = a.u_draft[ro];
    // This position's A row in fp32 (r <= 512 = 2 x 256 threads): the
    // previous token's U row (Markov head) or the state h (RNN head).  It is
    // published to urow by the first group barrier below.
    float uv0, uv1;
    if (a.H != nullptr) {
        // The state as the tensor-core product saw it: its high and low bf16
        // parts summed, so the recomputed slice agrees with the tile partials.
        const float *hrow = a.H + ro * r;
        uv0 = tid < r ? split_bf16_sum(hrow[tid]) : 0.f;
        uv1 = tid + nthr < r ? split_bf16_sum(hrow[tid + nthr]) : 0.f;
    } else {
        const int prev = (pos == 0) ? clamp_token(a.x0[b], V, a.hdr) : a.x_out[(size_t)b * G + pos - 1];
        uv0 = tid < r ? ld_elem(U, (size_t)prev * r + tid) : 0.f;
        uv1 = tid + nthr < r ? ld_elem(U, (size_t)prev * r + tid + nthr) : 0.f;
    }
    if (tid < r) urow[tid] = uv0;
    if (tid + nthr < r) urow[tid + nthr] = uv1;

    float m = -INFINITY;
#pragma unroll
    for (int q = 0; q < kFinChunk; ++q) m = fmaxf(m, cm[q]);
    for (int t = t0 + kFinChunk; t < t1; ++t) m = fmaxf(m, __ldcg(pp + t).x);   // very large vocabularies only
    const float M = grp_max1(g, m, sc->s_max);

    if (Tb == 0.f) {   // greedy row (group-uniform): lowest argmax over the partials
        int first = 0x7fffffff;
        for (int t = t1 - 1; t >= t0 + kFinChunk; --t)
            if (__ldcg(pp + t).x == M) first = t;
#pragma unroll
        for (int q = kFinChunk - 1; q >= 0; --q)
            if (t0 + q < t1 && cm[q] == M) first = t0 + q;
        first = grp_min1(g, first, sc->s_own);
        if (tid == 0) {
            if (first >= nTiles) first = 0;  // no partial matched (non-finite inputs)
            int x = __float_as_int(__ldcg(pp + first).y);
            if (x < 0 || x >= V) x = 0;
            a.x_out[ro] = x;
            a.pd_out[ro] = 1.f;
            a.rowmax_out[ro] = M;
            a.rowsum_out[ro] = 1.f;
            sc->xg = x;
        }
        g.sync();
        stage_next(sc->xg);
        g.sync();
        return;
    }

    const float cexp = kLog2e / Tb;
    float loc = 0.f;
#pragma unroll
    for (int q = 0; q < kFinChunk; ++q) loc += cs[q] * fast_exp2((cm[q] - M) * cexp);
    for (int t = t0 + kFinChunk; t < t1; ++t) {
        const float2 v = __ldcg(pp + t);
        loc += v.y * fast_exp2((v.x - M) * cexp);
    }
    float Z;
    const float incl = grp_scan1(g, loc, sc->s_loc, &Z);
    const float target = u * Z;
    // The first thread whose inclusive prefix passes u Z owns the crossing
    // (the last thread with mass if rounding left u Z at the top).
    int owner = grp_min1(g, (incl > target && loc > 0.f) ? tid : 0x7fffffff, sc->s_own);
    const bool past_mass = owner == 0x7fffffff;   // rounding left u Z at the top: a tie by definition
    if (past_mass) owner = max(0, grp_max1_i(g, loc > 0.f ? tid : -1, sc->s_own2));
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
            const float2 v = __ldcg(pp + t);
            const float wt = v.y * fast_exp2((v.x - M) * cexp);
            if (run + wt > target) {
                ts = t;
            } else {
                if (wt > 0.f) { last = t; run_last = run; }
                run += wt;
            }
        }
        if (ts < 0) { ts = last; run = run_last; }
        sc->ts = max(ts, 0);
        sc->rem = target - run;
    }
    g.sync();
    const int ts = sc->ts;
    const float rem = sc->rem;
    // Recompute the chosen partial's columns: tpc consecutive threads share one column.
    const int c0 = ts * TN;
    const int tpc = nthr / TN;
    const int col = c0 + tid / tpc, part = tid % tpc;
    const bool mine = part == 0 && col < V;
    const float lval = mine ? ld_elem(L, ro * V + col) : 0.f;   // issued with the factor loads
    // The token is one of these columns: its U row (read to stage the next
    // position) is brought into L2 while the columns are recomputed.
    if (a.E != nullptr && pos + 1 < G) {
        const int nl = (r * (int)sizeof(T) + 127) / 128;   // 128-byte lines per U row
        for (int q = tid; q < TN * nl; q += nthr) {
            const int cc = c0 + q / nl;
            if (cc < V)
                asm volatile("prefetch.global.L2 [%0];" ::"l"(U + (size_t)cc * r + (q % nl) * (128 / sizeof(T))));
        }
    }
    float dl = 0.f;
    if (col < V) dl = dot_part(urow, Wt + (size_t)col * r, r, part, tpc);
    for (int o = tpc >> 1; o > 0; o >>= 1) dl += __shfl_xor_sync(0xffffffffu, dl, o);
    const float e = mine ? fast_exp2(((lval - M) + dl) * cexp) : 0.f;
    float ttot;
    const float inc = grp_scan1(g, e, sc->s_col, &ttot);
    int xs = grp_min1(g, (mine && inc > rem) ? col : 0x7fffffff, sc->s_x);
    const bool fell_short = xs == 0x7fffffff;
    if (fell_short) {  // the recomputed mass fell short: last positive column
        xs = grp_max1_i(g, (mine && e > 0.f) ? col : -1, sc->s_x2);
        if (xs < 0) xs = min(c0 + TN, V) - 1;
    }
    if (mine && col == xs) {
        a.x_out[ro] = xs;
        a.pd_out[ro] = e / Z;
        a.rowmax_out[ro] = M;
        a.rowsum_out[ro] = Z;
        // The draw's margin: u Z to the nearer edge of the token's interval
        // [inc - e, inc) (mass units, relative to the crossing slice), over Z.
        const float margin = (past_mass || fell_short) ? 0.f : fminf(rem - (inc - e), inc - rem) / Z;
        if (margin < kNearTie) count_near_tie(a.hdr, kPadDraftTies);
    }
    stage_next(xs);
    g.sync();
}

}  // namespace dspark
