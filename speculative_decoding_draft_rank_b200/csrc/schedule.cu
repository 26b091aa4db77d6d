// schedule.cu -- stage 3, Algorithm 1 (hardware-aware prefix scheduler).
//
// Method (menfem.com KB entry on DSpark, "Key Contributions": greedy global
// sort of candidate tokens by cumulative survival, incremental batch
// admission with early stopping that keeps admissions causal; paperlayer.ai
// summary, Appendix A: stop as soon as the objective drops, so admitting
// token k never looks at information from after x_k is drawn).
//
// The stage runs as one launch of CTAs of 1024 threads:
//   1. rank by counting, spread over the CTAs: every CTA holds the survivals
//      (position-major, candidate id i*B + b) in shared memory and each warp
//      takes one candidate c at a time: its rank in the order "S descending,
//      ties by the lower id" is #{j : S_j > S_c} + #{j : S_j = S_c, j < c},
//      counted by the 32 lanes over all candidates (ranks are unique, so the
//      candidates land in a permutation); the candidate's 64-bit key
//      (~bits(S) above the id) is written at its rank in the workspace;
//   2. the last CTA to finish (an arrival counter in the workspace header,
//      zeroed by a memset before the launch) reads the sorted keys and
//      admits: fp64 block scan of the sorted survivals gives
//      V_n = B + sum_{j<n} S_(j); every candidate n evaluates the stop test
//      (V_n + S_(n)) t(n) < V_n t(n+1) in parallel; the first true index (or
//      the budget) is the admitted count;
//   3. admitted candidates are counted per request in shared memory -> ell.
// Batches of at most 4096 candidates run as a single cluster of 16 CTAs (8
// where the GPU refuses 16) that ranks through sorted position columns
// (schedule_cluster_kernel below) and gathers the sorted keys in the first
// CTA's shared memory: cluster barriers replace the workspace round trip, the
// arrival counter and its reset.
// Variants (menfem.com KB entry, "Key Contributions"; paperlayer.ai summary,
// Appendix A): the offline global search admits the count that maximises
// Theta(n) = V_n / t(n) over every n up to the budget (lowest n on ties) --
// no early stop, so not lossless when confidence depends on drawn tokens --
// and static-threshold pruning admits the sorted candidates with
// S >= threshold, up to the budget.  The production scheduler's dynamic
// top-K (paperlayer.ai summary, §5.2 Production Scheduler: the capacity limit
// comes from historical predictions, the current candidates are ranked by
// their latest cumulative confidence) admits the first K of the sorted
// candidates, K read from device memory -- written there by an earlier
// schedule call on an earlier round -- so one captured graph serves every
// capacity.
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"
#include "schedule_variants.cuh"
#include "tc.cuh"

namespace dspark {

constexpr int kSchedThreads = 1024;
constexpr int kSchedMaxN = 16384;
constexpr int kSchedMaxP = 64;
constexpr int kSchedClusterMaxN = 4096;   // batches ranked by one cluster of CTAs

// Piecewise-linear profile through (kn[j], kt[j]) continued with the last slope.
__device__ __forceinline__ double profile_at(const int *kn, const double *kt, int P, double n) {
    if (P == 1) return kt[0];
    int lo = 0, hi = P - 2;  // segment index: the last j <= P-2 with kn[j] <= n
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if ((double)kn[mid] <= n) lo = mid; else hi = mid - 1;
    }
    return kt[lo] + (n - (double)kn[lo]) * kt[kSchedMaxP + lo];   // the segment's slope, stored by load_profile
}

// Knots and per-segment slopes into shared memory: kt[j] = t(kn[j]) and
// kt[kSchedMaxP + j] = (t(kn[j+1]) - t(kn[j])) / (kn[j+1] - kn[j]), so that
// the admission scan evaluates the profile without a division.
__device__ __forceinline__ void load_profile(const int32_t *__restrict__ knots_n, const double *__restrict__ knots_t,
                                             int P, int *kn, double *kt) {
    for (int j = threadIdx.x; j < P; j += blockDim.x) {
        kn[j] = knots_n[j];
        kt[j] = knots_t[j];
        if (j + 1 < P) kt[kSchedMaxP + j] = (knots_t[j + 1] - knots_t[j]) / (double)(knots_n[j + 1] - knots_n[j]);
    }
}

// Admission over the sorted keys [N] in shared memory (one CTA): the fp64
// prefix of the sorted survivals, the mode's count, the per-request lengths,
// the order and the objective at the admitted count.  ell_s: [B] ints of
// shared memory.
__device__ void admit_sorted(const unsigned long long *keys, int *ell_s, int B, int G, const int *kn_s,
                             const double *kt_s, int P, int budget, int mode, float threshold,
                             const int32_t *__restrict__ capacity, WsHeader *hdr, int32_t *__restrict__ ell_out,
                             int32_t *__restrict__ n_adm_out, double *__restrict__ theta_out,
                             int32_t *__restrict__ order_out) {
    __shared__ int red_i[33];
    __shared__ double red_d[33];
    const int N = B * G;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    // fp64 prefix of the sorted survivals: V_n = B + sum_{j<n} S_(j).  Thread t
    // owns the contiguous ranks [c0, c1).
    const int cpt = (N + blockDim.x - 1) / blockDim.x;
    const int c0 = min(N, tid * cpt), c1 = min(N, c0 + cpt);
    auto surv = [&](int n) { return (double)__uint_as_float(~(unsigned)(keys[n] >> 32)); };
    double run = 0.0;
    for (int n = c0; n < c1; ++n) run += surv(n);
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
    int nadm;
    if (mode == DSPARK_SCHED_GLOBAL_ARGMAX) {
        // Theta at every count: n = 0 (thread 0) and n + 1 for the thread's
        // ranks n; the block argmax keeps the lowest count among equal values.
        double best = -INFINITY;
        int bestn = 0x7fffffff;
        if (tid == 0) { best = (double)B / profile_at(kn_s, kt_s, P, 0.0); bestn = 0; }
        double Vn = Vbase;
        for (int n = c0; n < c1 && n < limit; ++n) {
            Vn += surv(n);
            const double th = Vn / profile_at(kn_s, kt_s, P, (double)(n + 1));
            if (th > best) { best = th; bestn = n + 1; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const double ob = __shfl_xor_sync(0xffffffffu, best, o);
            const int on = __shfl_xor_sync(0xffffffffu, bestn, o);
            if (ob > best || (ob == best && on < bestn)) { best = ob; bestn = on; }
        }
        __shared__ double arg_v[32];
        __shared__ int arg_n[32];
        if (lane == 0) { arg_v[wid] = best; arg_n[wid] = bestn; }
        __syncthreads();
        best = arg_v[0];
        bestn = arg_n[0];
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w)
            if (arg_v[w] > best || (arg_v[w] == best && arg_n[w] < bestn)) { best = arg_v[w]; bestn = arg_n[w]; }
        nadm = bestn;
    } else if (mode == DSPARK_SCHED_TOPK) {
        // The first K of the stable order; a negative capacity admits none
        // and is recorded.
        int kcap = *capacity;
        if (kcap < 0) {
            if (tid == 0) flag_status(hdr, DSPARK_DEV_ELL_RANGE);
            kcap = 0;
        }
        nadm = kcap < limit ? kcap : limit;
    } else if (mode == DSPARK_SCHED_THRESHOLD) {
        // The sorted survivals fall below the threshold at one index.
        int first_below = 0x7fffffff;
        for (int n = c0; n < c1; ++n)
            if (surv(n) < (double)threshold) { first_below = n; break; }
        nadm = block_min_i(first_below, red_i);
        if (nadm > limit) nadm = limit;
    } else {
        int first_stop = 0x7fffffff;
        double Vn = Vbase;
        for (int n = c0; n < c1 && n < limit; ++n) {
            const double sn = surv(n);
            const double t0 = profile_at(kn_s, kt_s, P, (double)n);
            const double t1 = profile_at(kn_s, kt_s, P, (double)(n + 1));
            if ((Vn + sn) * t0 < Vn * t1) { first_stop = n; break; }
            Vn += sn;
        }
        nadm = block_min_i(first_stop, red_i);
        if (nadm > limit) nadm = limit;
    }

    // Objective at the admitted count: V_nadm from the chunk that holds
    // index nadm (or the last chunk when nadm == N).
    __shared__ double Vadm_s;
    if (tid == 0) Vadm_s = (double)B;
    __syncthreads();
    if (c0 < c1 && ((nadm >= c0 && nadm < c1) || (nadm == N && c1 == N))) {
        double Vn = Vbase;
        for (int n = c0; n < nadm && n < c1; ++n) Vn += surv(n);
        Vadm_s = Vn;
    }
    for (int b = tid; b < B; b += blockDim.x) ell_s[b] = 0;
    __syncthreads();
    for (int n = tid; n < nadm; n += blockDim.x) atomicAdd(&ell_s[(int)(unsigned)keys[n] % B], 1);
    if (order_out != nullptr)
        for (int n = tid; n < N; n += blockDim.x) order_out[n] = (int)(unsigned)keys[n];
    __syncthreads();
    for (int b = tid; b < B; b += blockDim.x) ell_out[b] = ell_s[b];
    if (tid == 0) {
        *n_adm_out = nadm;
        if (theta_out != nullptr) *theta_out = Vadm_s / profile_at(kn_s, kt_s, P, (double)nadm);
    }
}

__global__ void __launch_bounds__(kSchedThreads) schedule_kernel(
    const float *__restrict__ S, int B, int G, const int32_t *__restrict__ knots_n,
    const double *__restrict__ knots_t, int P, int budget, int mode, float threshold,
    const int32_t *__restrict__ capacity, WsHeader *hdr, unsigned long long *__restrict__ sorted,
    int32_t *__restrict__ ell_out, int32_t *__restrict__ n_adm_out, double *__restrict__ theta_out,
    int32_t *__restrict__ order_out)
{
    extern __shared__ __align__(16) unsigned char sched_smem[];
    const int N = B * G;
    // Shared memory: the survivals (phase 1), then the sorted keys [N] and the
    // per-request counts [B] (the admitting CTA).
    int *ell_s = reinterpret_cast<int *>(sched_smem + sizeof(unsigned long long) * (size_t)N);
    __shared__ int last_s;
    __shared__ int kn_s[kSchedMaxP];
    __shared__ double kt_s[2 * kSchedMaxP];
    __shared__ double red_d[33];

    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5, nwarps = blockDim.x >> 5;
    load_profile(knots_n, knots_t, P, kn_s, kt_s);

    if (mode == DSPARK_SCHED_ALL) {   // one CTA: no order to find
        if (blockIdx.x != 0) return;
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

    // Phase 1: ranks by counting.  sv holds the survivals position-major
    // (NaN or negative survivals rank last, as 0).
    float *sv = reinterpret_cast<float *>(sched_smem);
    for (int id = tid; id < N; id += blockDim.x) {
        const int i = id / B, b = id - i * B;
        float s = S[(size_t)b * G + i];
        if (!(s >= 0.f)) s = 0.f;
        sv[id] = s;
    }
    __syncthreads();
    for (int c = (int)blockIdx.x * nwarps + wid; c < N; c += (int)gridDim.x * nwarps) {
        const float s = sv[c];
        int cnt = 0;
        for (int j = lane; j < N; j += 32) {
            const float t = sv[j];
            cnt += (t > s) | ((t == s) & (j < c));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
        if (lane == 0) sorted[cnt] = ((unsigned long long)(~__float_as_uint(s)) << 32) | (unsigned)c;
    }
    // The last CTA to finish its candidates admits.
    __threadfence();
    __syncthreads();
    if (tid == 0) last_s = atomicAdd(&hdr->pad[kPadSchedArrive], 1u) == gridDim.x - 1;
    __syncthreads();
    if (!last_s) return;
    __threadfence();
    unsigned long long *keys = reinterpret_cast<unsigned long long *>(sched_smem);   // [N]
    for (int n = tid; n < N; n += blockDim.x) keys[n] = __ldcg(sorted + n);
    __syncthreads();

    admit_sorted(keys, ell_s, B, G, kn_s, kt_s, P, budget, mode, threshold, capacity, hdr, ell_out, n_adm_out,
                 theta_out, order_out);
}

// Batches of at most kSchedClusterMaxN candidates: the grid is one cluster,
// and the rank is found in two steps instead of by comparing all pairs.  The
// order is that of the unique 64-bit keys (~bits(S) above the candidate id),
// so a candidate's rank is the number of smaller keys, summed over the G
// position columns of B candidates each:
//   1. column ranks -- each CTA takes a share of the candidates and counts,
//      within the candidate's own column, the smaller keys (B comparisons,
//      one warp per candidate); the key is stored at that place of the
//      sorted column in every CTA of the cluster (distributed shared memory);
//   2. after a cluster barrier, global ranks -- for its candidates each CTA
//      adds the G lower bounds of the key in the sorted columns (one lane per
//      column, a binary search each) and stores the key at that rank in the
//      first CTA; after a second barrier the first CTA admits.
// That is N (B + G log B) comparisons where counting over all pairs takes N^2,
// with no workspace round trip and no arrival counter.
__global__ void __launch_bounds__(kSchedThreads) schedule_cluster_kernel(
    const float *__restrict__ S, int B, int G, const int32_t *__restrict__ knots_n,
    const double *__restrict__ knots_t, int P, int budget, int mode, float threshold,
    const int32_t *__restrict__ capacity, WsHeader *hdr, int32_t *__restrict__ ell_out,
    int32_t *__restrict__ n_adm_out, double *__restrict__ theta_out, int32_t *__restrict__ order_out)
{
    extern __shared__ __align__(16) unsigned char sched_smem[];
    const int N = B * G;
    // Shared memory: every candidate's key [N] (position-major), the sorted
    // columns [G][B], then (used in the first CTA) the sorted keys [N] and the
    // per-request counts [B].
    unsigned long long *kall = reinterpret_cast<unsigned long long *>(sched_smem);
    unsigned long long *col = kall + N;
    unsigned long long *keys = col + N;
    int *ell_s = reinterpret_cast<int *>(keys + N);
    __shared__ int kn_s[kSchedMaxP];
    __shared__ double kt_s[2 * kSchedMaxP];
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5, nwarps = blockDim.x >> 5;
    tc::cluster_arrive_relaxed();   // this CTA runs; waited for before the first remote store
    load_profile(knots_n, knots_t, P, kn_s, kt_s);
    for (int id = tid; id < N; id += blockDim.x) {
        const int i = id / B, b = id - i * B;
        float s = S[(size_t)b * G + i];
        if (!(s >= 0.f)) s = 0.f;   // NaN or negative survivals rank last, as 0
        kall[id] = ((unsigned long long)(~__float_as_uint(s)) << 32) | (unsigned)id;
    }
    __syncthreads();
    tc::cluster_wait();             // every CTA of the cluster has started
    const int rank = (int)tc::cluster_ctarank(), ncta = (int)gridDim.x;
    const int step = ncta * nwarps;
    // 1. Column ranks, broadcast into every CTA's sorted columns.
    const uint32_t col_u32 = tc::smem_u32(col);
    for (int c = rank * nwarps + wid; c < N; c += step) {
        const unsigned long long k = kall[c];
        const int i = c / B;
        const unsigned long long *cc = kall + (size_t)i * B;
        int cnt = 0;
        for (int j = lane; j < B; j += 32) cnt += cc[j] < k;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
        if (lane < ncta) tc::st_cluster_u64(tc::mapa_shared(col_u32 + 8u * (uint32_t)(i * B + cnt), lane), k);
    }
    tc::cluster_sync();   // every CTA holds all G sorted columns
    // 2. Global ranks: lane i < G counts the keys below k in sorted column i.
    const uint32_t keys0 = tc::mapa_shared(tc::smem_u32(keys), 0);
    for (int c = rank * nwarps + wid; c < N; c += step) {
        const unsigned long long k = kall[c];
        int below = 0;
        if (lane < G) {
            const unsigned long long *cc = col + (size_t)lane * B;
            int lo = 0, hi = B;   // first index with cc[idx] >= k
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (cc[mid] < k) lo = mid + 1; else hi = mid;
            }
            below = lo;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) below += __shfl_xor_sync(0xffffffffu, below, o);
        if (lane == 0) tc::st_cluster_u64(keys0 + 8u * (uint32_t)below, k);
    }
    tc::cluster_sync();   // every key is in the first CTA, in order
    if (rank != 0) return;
    admit_sorted(keys, ell_s, B, G, kn_s, kt_s, P, budget, mode, threshold, capacity, hdr, ell_out, n_adm_out,
                 theta_out, order_out);
}

// Workspace: the header (status word, arrival counter) and the sorted keys.
size_t schedule_ws_bytes(int B, int G) { return sizeof(WsHeader) + align256(sizeof(unsigned long long) * (size_t)B * G); }

// Dynamic shared memory of one call: the sorted keys (which reuse the
// survivals' space) and the per-request counts.
static size_t sched_smem_bytes(int B, int G) {
    return sizeof(unsigned long long) * (size_t)B * G + sizeof(int) * (size_t)B;
}

static cudaError_t launch_sched(const float *S, int B, int G, const int32_t *knots_n, const double *knots_t, int P,
                                int budget, int mode, float threshold, const int32_t *capacity, void *ws,
                                int32_t *ell_out, int32_t *n_adm_out, double *theta_out, int32_t *order_out,
                                cudaStream_t st) {
    const size_t smem = sched_smem_bytes(B, G);
    cudaError_t e = cudaFuncSetAttribute(schedule_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(sizeof(unsigned long long) * kSchedMaxN + sizeof(int) * 4096));
    if (e != cudaSuccess) return e;
    WsHeader *hdr = static_cast<WsHeader *>(ws);
    unsigned long long *sorted = reinterpret_cast<unsigned long long *>(static_cast<char *>(ws) + sizeof(WsHeader));
    if (mode != DSPARK_SCHED_ALL && B * G <= kSchedClusterMaxN) {
        static int cluster = -1;   // CTAs of the ranking cluster (16 where the GPU allows, else 8)
        // keys, sorted columns and sorted keys [3 N] u64, the counts [B] int
        const size_t csmem = 3 * sizeof(unsigned long long) * (size_t)B * G + sizeof(int) * (size_t)B;
        if ((e = cudaFuncSetAttribute(schedule_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)(3 * sizeof(unsigned long long) * kSchedClusterMaxN +
                                            sizeof(int) * kSchedClusterMaxN))) != cudaSuccess)
            return e;
        cudaLaunchConfig_t cfg = {};
        cfg.blockDim = dim3(kSchedThreads);
        cfg.dynamicSmemBytes = csmem;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cluster < 0) {
            cluster = 8;
            if (cudaFuncSetAttribute(schedule_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
                cudaSuccess) {
                int n = 0;
                attr[0].val.clusterDim.x = 16;
                cfg.gridDim = dim3(16);
                if (cudaOccupancyMaxActiveClusters(&n, schedule_cluster_kernel, &cfg) == cudaSuccess && n >= 1)
                    cluster = 16;
            }
            cudaGetLastError();   // a refused query leaves no error behind
        }
        attr[0].val.clusterDim.x = cluster;
        cfg.gridDim = dim3(cluster);
        if ((e = cudaLaunchKernelEx(&cfg, schedule_cluster_kernel, S, B, G, knots_n, knots_t, P, budget, mode,
                                    threshold, capacity, hdr, ell_out, n_adm_out, theta_out, order_out)) !=
            cudaSuccess)
            return e;
        return cudaGetLastError();
    }
    int grid = 1;
    if (mode != DSPARK_SCHED_ALL) {
        int dev = 0, sms = 148;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const int warps = kSchedThreads / 32;
        grid = std::max(1, std::min(sms, (B * G + warps - 1) / warps));   // about one candidate per warp
        if ((e = cudaMemsetAsync(&hdr->pad[kPadSchedArrive], 0, sizeof(uint32_t), st)) != cudaSuccess) return e;
    }
    schedule_kernel<<<grid, kSchedThreads, smem, st>>>(S, B, G, knots_n, knots_t, P, budget, mode, threshold,
                                                       capacity, hdr, sorted, ell_out, n_adm_out, theta_out,
                                                       order_out);
    return cudaGetLastError();
}

cudaError_t launch_schedule(const float *S, int B, int G, const int32_t *knots_n,
                            const double *knots_t, int P, int budget, int mode, float threshold, void *ws,
                            int32_t *ell_out, int32_t *n_adm_out, double *theta_out,
                            int32_t *order_out, cudaStream_t st) {
    return launch_sched(S, B, G, knots_n, knots_t, P, budget, mode, threshold, nullptr, ws, ell_out, n_adm_out,
                        theta_out, order_out, st);
}

cudaError_t launch_schedule_topk(const float *S, int B, int G, const int32_t *capacity, int budget, void *ws,
                                 int32_t *ell_out, int32_t *n_adm_out, int32_t *order_out, cudaStream_t st) {
    return launch_sched(S, B, G, nullptr, nullptr, 0, budget, DSPARK_SCHED_TOPK, 0.f, capacity, ws, ell_out,
                        n_adm_out, nullptr, order_out, st);
}

}  // namespace dspark
