// calibration.cu -- sequential temperature scaling (STS) of the confidence
// head and the ROC-AUC of the prefix survivals.
//
// Method (paperlayer.ai summary of DSpark, §3.2 Confidence-scheduled
// verification: STS calibrates the cumulative prefix-survival probabilities
// left to right, minimising the expected calibration error of the running
// products of the per-position scores; menfem.com KB entry, "Key
// Contributions" and "Results": raw ROC-AUC 0.81-0.90, ECE 3-8 %, about 1 %
// after STS).  Readings where the pages are silent: the temperature divides
// the head's logit (c_i = sigmoid(z_i / tau_i)); the label of position i is
// "the first i draft tokens were accepted" (A >= i); ECE uses M equal-width
// bins (bin = min(M - 1, floor(s * M))), ECE = sum_bins |sum (y - s)| / N; the
// minimum is taken over a caller-given grid, first entry of the least ECE.
//
// Fit: one launch per position i over (K + 1) x P CTAs: candidate k (k = K is
// the raw chain, tau = 1) times chunk p of the N samples, P chosen so that the
// grid covers the SMs about twice.  A CTA evaluates s = S_{i-1} * sigmoid(z_i /
// tau_k) for its chunk, keeps s (every candidate's survivals, double-buffered
// across positions: the next position reads the chosen row), and bins
// (y - s) into per-thread bin columns in shared memory, summed per bin in a
// fixed order.  The last of a candidate's chunk CTAs to arrive (arrival
// counters, no waiting) sums its chunks in chunk order and forms its ECE; the
// last candidate to finish picks the first grid entry with the least.  Arithmetic in fp64: the bin of a score is a
// floating-point decision, taken here in the same precision as the
// definition is written in.
//
// ROC-AUC: one thread per positive sample, scanning every sample of the
// position through shared-memory tiles in which positives are masked out
// (NaN compares false), counting 2 per lower negative and 1 per tie; exact
// 64-bit integer totals.
#include <cmath>

#include "calibration.cuh"
#include "common.cuh"

namespace dspark {

namespace {

constexpr int kStsThreads = 256;
constexpr int kAucThreads = 256;
constexpr int kAucTile = 2048;

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

// The candidate survival of one sample: the running product times the
// calibrated score.  One function for the candidate CTAs and the chain update
// so that the chosen candidate's scores and the advanced chain agree bit for bit.
__device__ __forceinline__ double cand_survival(double prev, float z, double t) {
    return prev * (1.0 / (1.0 + exp(-((double)z / t))));
}

__device__ __forceinline__ int ece_bin(double s, int M) {
    if (!(s >= 0.0)) return 0;                    // NaN: flagged by the caller's data check
    const double f = floor(s * (double)M);
    return f >= (double)(M - 1) ? M - 1 : (int)f;
}

__device__ __forceinline__ bool valid_temp(double t) { return t > 0.0 && t < INFINITY; }

__global__ void __launch_bounds__(kStsThreads) sts_position(const float *__restrict__ z,
                                                            const int32_t *__restrict__ acc,
                                                            const float *__restrict__ grid, int N, int G, int K,
                                                            int M, int P, int chunk, int i, StsWs w,
                                                            float *tau_out, double *ece_raw_out,
                                                            double *ece_fit_out, double *ece_all_out,
                                                            float *S_out) {
    extern __shared__ double part[];   // [M][kStsThreads]: per-thread bin sums of (y - s)
    __shared__ double s_val[kStsThreads / 32];
    __shared__ int s_idx[kStsThreads / 32];
    __shared__ int s_last_chunk, s_last_cand;
    const int tid = threadIdx.x, lane = tid & 31, wd = tid >> 5;
    const int k = blockIdx.x / P, p = blockIdx.x - k * P;
    const bool raw = k == K;
    const double t = raw ? 1.0 : (double)grid[k];
    const size_t NN = (size_t)N;
    // Survivals of position i - 1: the raw chain continues the raw chain, every
    // candidate continues the row chosen at i - 1.
    const double *prev = w.cand + (size_t)((i + 1) & 1) * (K + 1) * NN +
                         (size_t)(raw ? K : (i > 0 ? (int)w.hdr->pad[1] : 0)) * NN;
    double *cur = w.cand + (size_t)(i & 1) * (K + 1) * NN + (size_t)k * NN;
    for (int m = 0; m < M; ++m) part[m * kStsThreads + tid] = 0.0;
    const int n0 = p * chunk, n1 = min(N, n0 + chunk);
    bool bad_acc = false, bad_z = false;
    for (int n = n0 + tid; n < n1; n += kStsThreads) {
        const float zf = z[(size_t)n * G + i];
        const int a = acc[n];
        const double sp = i == 0 ? 1.0 : prev[n];
        const double s = cand_survival(sp, zf, t);
        part[ece_bin(s, M) * kStsThreads + tid] += (a >= i + 1 ? 1.0 : 0.0) - s;
        cur[n] = s;
        if (raw) {
            bad_acc |= a < 0 || a > G;
            bad_z |= !(fabsf(zf) < INFINITY);
        }
        // The fitted survivals of position i - 1, once (by candidate 0's CTAs).
        if (k == 0 && i > 0 && S_out != nullptr) S_out[(size_t)n * G + i - 1] = (float)sp;
    }
    if (bad_acc) flag_status(w.hdr, DSPARK_DEV_ELL_RANGE);
    if (bad_z) flag_status(w.hdr, DSPARK_DEV_BAD_VALUE);
    __syncthreads();
    // Per-bin totals of this chunk: warp wd sums bins wd, wd + 8, ... over the
    // thread columns in lane order, then a fixed shuffle tree.
    double *mine = w.part + (size_t)blockIdx.x * M;
    for (int m = wd; m < M; m += kStsThreads / 32) {
        double v = 0.0;
        for (int j = lane; j < kStsThreads; j += 32) v += part[m * kStsThreads + j];
        v = warp_sum_d(v);
        if (lane == 0) {
            mine[m] = v;
            __threadfence();
        }
    }
    __syncthreads();
    // The last of candidate k's P chunk CTAs forms its ECE: lane m sums bin m
    // over the chunks in chunk order, |.| per bin, then a fixed shuffle tree.
    if (tid == 0) {
        __threadfence();
        s_last_chunk = atomicAdd(w.cnt + k, 1u) == (unsigned)(P - 1);
        s_last_cand = 0;
    }
    __syncthreads();
    if (!s_last_chunk) return;
    __threadfence();
    if (wd == 0) {
        double v = 0.0;
        if (lane < M) {
            const double *col = w.part + (size_t)k * P * M + lane;
            int q = 0;
            for (; q + 4 <= P; q += 4) {   // four independent loads in flight, added in order
                const double a0 = __ldcg(col + (size_t)q * M), a1 = __ldcg(col + (size_t)(q + 1) * M);
                const double a2 = __ldcg(col + (size_t)(q + 2) * M), a3 = __ldcg(col + (size_t)(q + 3) * M);
                v += a0; v += a1; v += a2; v += a3;
            }
            for (; q < P; ++q) v += __ldcg(col + (size_t)q * M);
        }
        double e = warp_sum_d(fabs(v)) / (double)N;
        if (lane == 0) {
            if (raw) {
                if (ece_raw_out != nullptr) ece_raw_out[i] = e;
            } else {
                if (!valid_temp(t)) {              // no temperature: never preferred
                    e = INFINITY;
                    flag_status(w.hdr, DSPARK_DEV_BAD_VALUE);
                }
                w.ece[k] = e;
                if (ece_all_out != nullptr) ece_all_out[(size_t)i * K + k] = e;
            }
            w.cnt[k] = 0u;                         // the next launch counts afresh
            __threadfence();
            s_last_cand = atomicAdd(&w.hdr->pad[0], 1u) == (unsigned)K;   // K + 1 candidates in all
        }
    }
    __syncthreads();
    if (!s_last_cand) return;
    __threadfence();
    // The last candidate to finish picks the first grid entry with the least
    // ECE (+inf entries lose to any finite one; all +inf: the first).
    double best = INFINITY;
    int bk = 0x7fffffff;
    for (int kk = tid; kk < K; kk += kStsThreads) {
        const double e = __ldcg(w.ece + kk);
        if (e < best || (e == best && kk < bk)) { best = e; bk = kk; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const double ob = __shfl_xor_sync(0xffffffffu, best, o);
        const int ok = __shfl_xor_sync(0xffffffffu, bk, o);
        if (ob < best || (ob == best && ok < bk)) { best = ob; bk = ok; }
    }
    if (lane == 0) { s_val[wd] = best; s_idx[wd] = bk; }
    __syncthreads();
    if (tid == 0) {
        for (int q = 1; q < kStsThreads / 32; ++q)
            if (s_val[q] < s_val[0] || (s_val[q] == s_val[0] && s_idx[q] < s_idx[0])) {
                s_val[0] = s_val[q];
                s_idx[0] = s_idx[q];
            }
        const int kstar = s_idx[0] < K ? s_idx[0] : 0;   // every entry NaN: flagged data
        tau_out[i] = grid[kstar];
        if (ece_fit_out != nullptr) ece_fit_out[i] = __ldcg(w.ece + kstar);
        w.hdr->pad[1] = (uint32_t)kstar;                  // the row the next position continues
        w.hdr->pad[0] = 0u;                               // the next launch counts afresh
    }
}

// The fitted survivals of the last position (the earlier ones are written by
// the next position's launch).
__global__ void sts_last_survivals(int N, int G, int K, StsWs w, float *S_out) {
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    if (n >= N) return;
    const double *row = w.cand + (size_t)((G - 1) & 1) * (K + 1) * N + (size_t)w.hdr->pad[1] * N;
    S_out[(size_t)n * G + G - 1] = (float)row[n];
}

// ROC-AUC counts of position i = blockIdx.y: thread p (a positive sample)
// adds 2 for every negative with a lower score and 1 for every tie.
__global__ void __launch_bounds__(kAucThreads) survival_auc_counts(const float *__restrict__ S,
                                                                   const int32_t *__restrict__ acc, int N, int G,
                                                                   unsigned long long *twice_out,
                                                                   unsigned long long *npos_out) {
    __shared__ __align__(16) float tile[kAucTile];
    __shared__ unsigned long long s_red[kAucThreads / 32];
    __shared__ unsigned s_np[kAucThreads / 32];
    const int i = blockIdx.y, tid = threadIdx.x;
    const int p = blockIdx.x * kAucThreads + tid;
    const bool pos = p < N && acc[p] >= i + 1;
    const float sp = pos ? S[(size_t)p * G + i] : 0.f;
    unsigned long long cnt = 0;
    for (int base = 0; base < N; base += kAucTile) {
        __syncthreads();
        for (int j = tid; j < kAucTile; j += kAucThreads) {
            const int q = base + j;
            // Positives and the tail are NaN: every comparison with them is false.
            tile[j] = (q < N && acc[q] < i + 1) ? S[(size_t)q * G + i] : __int_as_float(0x7fc00000);
        }
        __syncthreads();
        if (pos) {
            unsigned c = 0;   // at most 2 * kAucTile per tile
            const float4 *t4 = reinterpret_cast<const float4 *>(tile);
#pragma unroll 4
            for (int j = 0; j < kAucTile / 4; ++j) {
                const float4 q = t4[j];
                c += (sp > q.x ? 2u : 0u) + (sp == q.x ? 1u : 0u);
                c += (sp > q.y ? 2u : 0u) + (sp == q.y ? 1u : 0u);
                c += (sp > q.z ? 2u : 0u) + (sp == q.z ? 1u : 0u);
                c += (sp > q.w ? 2u : 0u) + (sp == q.w ? 1u : 0u);
            }
            cnt += c;
        }
    }
    // Block totals: counts and positives, exact in 64-bit integers.
    unsigned long long v = cnt;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const unsigned np = __popc(__ballot_sync(0xffffffffu, pos));
    if ((tid & 31) == 0) {
        s_red[tid >> 5] = v;
        s_np[tid >> 5] = np;
    }
    __syncthreads();
    if (tid == 0) {
        unsigned long long tot = 0, ntot = 0;
        for (int q = 0; q < kAucThreads / 32; ++q) { tot += s_red[q]; ntot += s_np[q]; }
        atomicAdd(twice_out + i, tot);
        atomicAdd(npos_out + i, ntot);
    }
}

// pairs[i] = positives * negatives, in place over the positive counts.
__global__ void survival_auc_pairs(int N, int G, unsigned long long *pairs) {
    const int i = threadIdx.x;
    if (i < G) pairs[i] = pairs[i] * ((unsigned long long)N - pairs[i]);
}

}  // namespace

// Chunks per candidate: enough CTAs to cover the SMs about twice, at least
// one block of threads' worth of samples per chunk.
int sts_chunks(int N, int K) {
    const int want = (2 * 148 + K) / (K + 1);
    const int most = (N + kStsThreads - 1) / kStsThreads;
    return max(1, min(want, most));
}

size_t sts_ws_bytes(int N, int K, int M) {
    const int P = sts_chunks(N, K);
    return 256 + up256(sizeof(double) * 2 * (size_t)(K + 1) * N) + up256(sizeof(double) * (size_t)(K + 1) * P * M) +
           up256(sizeof(double) * (size_t)K) + up256(sizeof(uint32_t) * (size_t)(K + 1));
}

StsWs sts_ws_carve(void *ws, int N, int K, int M) {
    const int P = sts_chunks(N, K);
    char *p = static_cast<char *>(ws);
    StsWs w;
    w.hdr = reinterpret_cast<WsHeader *>(p);
    p += 256;
    w.cand = reinterpret_cast<double *>(p);
    p += up256(sizeof(double) * 2 * (size_t)(K + 1) * N);
    w.part = reinterpret_cast<double *>(p);
    p += up256(sizeof(double) * (size_t)(K + 1) * P * M);
    w.ece = reinterpret_cast<double *>(p);
    p += up256(sizeof(double) * (size_t)K);
    w.cnt = reinterpret_cast<uint32_t *>(p);
    return w;
}

cudaError_t launch_sts_fit(const StsArgs &a, void *ws, cudaStream_t st) {
    StsWs w = sts_ws_carve(ws, a.N, a.K, a.M);
    const int P = sts_chunks(a.N, a.K);
    const int chunk = (a.N + P - 1) / P;
    cudaError_t e = cudaMemsetAsync(&w.hdr->pad[0], 0, sizeof(uint32_t), st);
    if (e != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(w.cnt, 0, sizeof(uint32_t) * (size_t)(a.K + 1), st)) != cudaSuccess) return e;
    const size_t smem = sizeof(double) * (size_t)a.M * kStsThreads;
    if (smem > 48 * 1024 &&
        (e = cudaFuncSetAttribute(sts_position, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
            cudaSuccess)
        return e;
    for (int i = 0; i < a.G; ++i) {
        sts_position<<<(a.K + 1) * P, kStsThreads, smem, st>>>(a.z, a.acc, a.grid, a.N, a.G, a.K, a.M, P, chunk, i,
                                                                w, a.tau_out, a.ece_raw_out, a.ece_fit_out,
                                                                a.ece_all_out, a.S_out);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (a.S_out != nullptr) {
        sts_last_survivals<<<(a.N + 255) / 256, 256, 0, st>>>(a.N, a.G, a.K, w, a.S_out);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_survival_auc(const float *S, const int32_t *acc, int N, int G, unsigned long long *twice_out,
                                unsigned long long *pairs_out, cudaStream_t st) {
    cudaError_t e = cudaMemsetAsync(twice_out, 0, sizeof(unsigned long long) * (size_t)G, st);
    if (e != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(pairs_out, 0, sizeof(unsigned long long) * (size_t)G, st)) != cudaSuccess) return e;
    dim3 grid((N + kAucThreads - 1) / kAucThreads, G);
    survival_auc_counts<<<grid, kAucThreads, 0, st>>>(S, acc, N, G, twice_out, pairs_out);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    survival_auc_pairs<<<1, 32, 0, st>>>(N, G, pairs_out);
    return cudaGetLastError();
}

}  // namespace dspark
