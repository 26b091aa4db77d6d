// schedule.cu -- stage 3, Algorithm 1 (hardware-aware prefix scheduler).
//
// Method (menfem.com KB entry on DSpark, "Key Contributions": greedy global
// sort of candidate tokens by cumulative survival, incremental batch
// admission with early stopping that keeps admissions causal; paperlayer.ai
// summary, Appendix A: stop as soon as the objective drops, so admitting
// token k never looks at information from after x_k is drawn).
//
// One CTA of 1024 threads does the whole stage:
//   1. keys ~bits(S) (ascending = S descending, valid since S >= 0) and
//      position-major candidate ids i*B + b are sorted by a stable LSD radix
//      sort in shared memory (8 passes of 4 bits; each thread owns a
//      contiguous chunk, per-thread digit counts are scanned digit-major so
//      equal keys keep their id order);
//   2. fp64 block scan of the sorted survivals gives V_n = B + sum_{j<n} S_(j);
//   3. every candidate n evaluates the stop test
//      (V_n + S_(n)) t(n) < V_n t(n+1) in parallel; the first true index
//      (or the budget) is the admitted count;
//   4. admitted candidates are counted per request in shared memory -> ell.
#include "common.cuh"
#include "kernels.cuh"

namespace dspark {

constexpr int kSchedThreads = 1024;
constexpr int kSchedMaxN = 16384;
constexpr int kSchedMaxP = 64;
constexpr int kRadixBits = 4;
constexpr int kRadixBins = 1 << kRadixBits;

// Piecewise-linear profile through (kn[j], kt[j]) continued with the last slope.
__device__ __forceinline__ double profile_at(const int *kn, const double *kt, int P, double n) {
    if (P == 1) return kt[0];
    int lo = 0, hi = P - 2;  // segment index: the last j <= P-2 with kn[j] <= n
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if ((double)kn[mid] <= n) lo = mid; else hi = mid - 1;
    }
    const double slope = (kt[lo + 1] - kt[lo]) / (double)(kn[lo + 1] - kn[lo]);
    return kt[lo] + (n - (double)kn[lo]) * slope;
}

__global__ void __launch_bounds__(kSchedThreads) schedule_kernel(
    const float *__restrict__ S, int B, int G, const int32_t *__restrict__ knots_n,
    const double *__restrict__ knots_t, int P, int budget, int mode, int32_t *__restrict__ ell_out,
    int32_t *__restrict__ n_adm_out, double *__restrict__ theta_out, int32_t *__restrict__ order_out)
{
    extern __shared__ __align__(16) unsigned char sched_smem[];
    const int N = B * G;
    uint32_t *keys = reinterpret_cast<uint32_t *>(sched_smem);                  // [N]
    uint16_t *ids = reinterpret_cast<uint16_t *>(keys + kSchedMaxN);            // [N]
    uint16_t *cnt = ids + kSchedMaxN;                                          // [bins][threads]
    int *ell_s = reinterpret_cast<int *>(cnt);                                 // reused after sorting
    __shared__ int kn_s[kSchedMaxP];
    __shared__ double kt_s[kSchedMaxP];
    __shared__ int red_i[33];
    __shared__ double red_d[33];
    __shared__ int tot_s[33];

    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    for (int j = tid; j < P; j += blockDim.x) { kn_s[j] = knots_n[j]; kt_s[j] = knots_t[j]; }

    if (mode == DSPARK_SCHED_ALL) {
        double acc = 0.0;
        for (int j = tid; j < N; j += blockDim.x) acc += (double)S[j];
        acc = warp_sum_d(acc);
        if (lane == 0) red_d[wid] = acc;
        __syncthreads();
        if (tid == 0) {
            double t = 0.0;
            for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red_d[w];
            *n_adm_out = N;
            *theta_out = ((double)B + t) / profile_at(kn_s, kt_s, P, (double)N);
        }
        for (int b = tid; b < B; b += blockDim.x) ell_out[b] = G;
        if (order_out != nullptr)
            for (int j = tid; j < N; j += blockDim.x) order_out[j] = j;
        return;
    }

    // Keys and ids in position-major order (id = i*B + b).
    for (int id = tid; id < N; id += blockDim.x) {
        const int i = id / B, b = id - i * B;
        float s = S[(size_t)b * G + i];
        if (!(s >= 0.f)) s = 0.f;  // NaN or negative survival ranks last
        keys[id] = ~__float_as_uint(s);
        ids[id] = (uint16_t)id;
    }
    __syncthreads();

    const int cpt = (N + blockDim.x - 1) / blockDim.x;  // chunk per thread (<= 16)
    const int c0 = min(N, tid * cpt), c1 = min(N, c0 + cpt);
    constexpr int kMaxChunk = kSchedMaxN / kSchedThreads;
    for (int shift = 0; shift < 32; shift += kRadixBits) {
        uint32_t kr[kMaxChunk];
        uint32_t ir[kMaxChunk];
#pragma unroll
        for (int d = 0; d < kRadixBins; ++d) cnt[d * blockDim.x + tid] = 0;
#pragma unroll
        for (int j = 0; j < kMaxChunk; ++j) {
            if (c0 + j < c1) {
                kr[j] = keys[c0 + j];
                ir[j] = ids[c0 + j];
                cnt[((kr[j] >> shift) & (kRadixBins - 1)) * blockDim.x + tid]++;
            }
        }
        __syncthreads();
        // Exclusive scan of cnt in (digit, thread) order: thread t scans the
        // kRadixBins consecutive entries starting at kRadixBins * t.
        uint16_t *mine = cnt + tid * kRadixBins;
        int s = 0;
#pragma unroll
        for (int j = 0; j < kRadixBins; ++j) s += mine[j];
        const int ws = warp_incl_scan_i(s);
        if (lane == 31) tot_s[wid] = ws;
        __syncthreads();
        if (wid == 0) {
            int t = lane < (int)(blockDim.x >> 5) ? tot_s[lane] : 0;
            t = warp_incl_scan_i(t);
            tot_s[lane] = t;
        }
        __syncthreads();
        int run = ws - s + (wid > 0 ? tot_s[wid - 1] : 0);
#pragma unroll
        for (int j = 0; j < kRadixBins; ++j) {  // offsets reach N <= 16384: fits 16 bits
            const int c = mine[j];
            mine[j] = (uint16_t)run;
            run += c;
        }
        __syncthreads();
        // Stable scatter: each thread walks its chunk in order, bumping its
        // own column of offsets.
#pragma unroll
        for (int j = 0; j < kMaxChunk; ++j) {
            if (c0 + j < c1) {
                uint16_t &o = cnt[((kr[j] >> shift) & (kRadixBins - 1)) * blockDim.x + tid];
                const int p = o;
                o = (uint16_t)(p + 1);
                keys[p] = kr[j];
                ids[p] = (uint16_t)ir[j];
            }
        }
        __syncthreads();
    }

    // fp64 prefix of the sorted survivals: V_n = B + sum_{j<n} S_(j).
    double run = 0.0;
    for (int n = c0; n < c1; ++n) run += (double)__uint_as_float(~keys[n]);
    const double wsum = warp_incl_scan_d(run);
    if (lane == 31) red_d[wid] = wsum;
    __syncthreads();
    if (wid == 0) {
        double t = lane < (int)(blockDim.x >> 5) ? red_d[lane] : 0.0;
        t = warp_incl_scan_d(t);
        red_d[lane] = t;
    }
    __syncthreads();
    const double Vbase = (double)B + (wsum - run) + (wid > 0 ? red_d[wid - 1] : 0.0);
    const int limit = (budget >= 0 && budget < N) ? budget : N;
    int first_stop = 0x7fffffff;
    {
        double Vn = Vbase;
        for (int n = c0; n < c1 && n < limit; ++n) {
            const double sn = (double)__uint_as_float(~keys[n]);
            const double t0 = profile_at(kn_s, kt_s, P, (double)n);
            const double t1 = profile_at(kn_s, kt_s, P, (double)(n + 1));
            if ((Vn + sn) * t0 < Vn * t1) { first_stop = n; break; }
            Vn += sn;
        }
    }
    int nadm = block_min_i(first_stop, red_i);
    if (nadm > limit) nadm = limit;

    // Objective at the admitted count: V_nadm from the chunk that holds
    // index nadm (or the last chunk when nadm == N).
    __shared__ double Vadm_s;
    if (tid == 0) Vadm_s = (double)B;
    __syncthreads();
    if (c0 < c1 && ((nadm >= c0 && nadm < c1) || (nadm == N && c1 == N))) {
        double Vn = Vbase;
        for (int n = c0; n < nadm && n < c1; ++n) Vn += (double)__uint_as_float(~keys[n]);
        Vadm_s = Vn;
    }
    for (int b = tid; b < B; b += blockDim.x) ell_s[b] = 0;
    __syncthreads();
    for (int n = tid; n < nadm; n += blockDim.x) atomicAdd(&ell_s[ids[n] % B], 1);
    if (order_out != nullptr)
        for (int n = tid; n < N; n += blockDim.x) order_out[n] = ids[n];
    __syncthreads();
    for (int b = tid; b < B; b += blockDim.x) ell_out[b] = ell_s[b];
    if (tid == 0) {
        *n_adm_out = nadm;
        *theta_out = Vadm_s / profile_at(kn_s, kt_s, P, (double)nadm);
    }
}

size_t schedule_ws_bytes(int, int) { return sizeof(WsHeader); }

cudaError_t launch_schedule(const float *S, int B, int G, const int32_t *knots_n,
                            const double *knots_t, int P, int budget, int mode, void *,
                            int32_t *ell_out, int32_t *n_adm_out, double *theta_out,
                            int32_t *order_out, cudaStream_t st) {
    const size_t smem = sizeof(uint32_t) * kSchedMaxN + sizeof(uint16_t) * kSchedMaxN +
                        sizeof(uint16_t) * kRadixBins * kSchedThreads;
    static_assert(sizeof(uint16_t) * kRadixBins * kSchedThreads >= sizeof(int) * 4096,
                  "the count table doubles as the per-request counters");
    cudaError_t e = cudaFuncSetAttribute(schedule_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    schedule_kernel<<<1, kSchedThreads, smem, st>>>(S, B, G, knots_n, knots_t, P, budget, mode, ell_out,
                                                    n_adm_out, theta_out, order_out);
    return cudaGetLastError();
}

}  // namespace dspark
