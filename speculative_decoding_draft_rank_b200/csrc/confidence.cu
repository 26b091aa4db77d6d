// confidence.cu -- stage 2, linear confidence head and prefix survival.
//
// Method (menfem.com KB entry on DSpark, "Key Contributions": a lightweight
// linear confidence head emits a per-position survival probability;
// paperlayer.ai summary, §3.2: cumulative products give the prefix survival,
// calibrated left to right by sequential temperature scaling):
//   c[b,i] = sigmoid((w . h[b,i,:] + bias) / tau[i]),  S[b,i] = prod_{j<=i} c[b,j].
//
// One CTA per request, one warp per position (G warps, at most 40 registers
// a thread): small enough to share an SM with the drafting kernel, which it
// runs beside on a side stream of the round (it does not depend on the
// drafted tokens).  Each lane keeps four 16-byte loads of h in flight; the
// warp's partial dot products are folded in a fixed order, then the first
// thread forms the running product.  HBM-bound: B*G*d*esize bytes.
#include "common.cuh"
#include "kernels.cuh"

namespace dspark {

// Partial dot product of h and w over the 8-element groups q = first,
// first + stride, ... (bf16: one 16-byte load each), four loads in flight.
__device__ __forceinline__ float dot_part8(const __nv_bfloat16 *__restrict__ h,
                                           const __nv_bfloat16 *__restrict__ w, int d, int first, int stride) {
    float acc = 0.f;
    const bool vec = ((reinterpret_cast<uintptr_t>(h) | reinterpret_cast<uintptr_t>(w)) & 15) == 0 && (d & 7) == 0;
    if (vec) {
        const uint4 *hv = reinterpret_cast<const uint4 *>(h);
        const uint4 *wv = reinterpret_cast<const uint4 *>(w);
        const int nv = d / 8;
        for (int q0 = first; q0 < nv; q0 += 4 * stride) {
            uint4 a[4], c[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int q = q0 + u * stride;
                a[u] = q < nv ? ld_stream16(hv + q) : make_uint4(0, 0, 0, 0);
                c[u] = q < nv ? __ldg(wv + q) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                acc = fmaf(bf16lo(a[u].x), bf16lo(c[u].x), acc); acc = fmaf(bf16hi(a[u].x), bf16hi(c[u].x), acc);
                acc = fmaf(bf16lo(a[u].y), bf16lo(c[u].y), acc); acc = fmaf(bf16hi(a[u].y), bf16hi(c[u].y), acc);
                acc = fmaf(bf16lo(a[u].z), bf16lo(c[u].z), acc); acc = fmaf(bf16hi(a[u].z), bf16hi(c[u].z), acc);
                acc = fmaf(bf16lo(a[u].w), bf16lo(c[u].w), acc); acc = fmaf(bf16hi(a[u].w), bf16hi(c[u].w), acc);
            }
        }
    } else {
        for (int j = first; j < d; j += stride) acc = fmaf(to_f32(h[j]), to_f32(w[j]), acc);
    }
    return acc;
}
// fp32: 4-element groups, one 16-byte load each.
__device__ __forceinline__ float dot_part8(const float *__restrict__ h, const float *__restrict__ w, int d,
                                           int first, int stride) {
    float acc = 0.f;
    const bool vec = ((reinterpret_cast<uintptr_t>(h) | reinterpret_cast<uintptr_t>(w)) & 15) == 0 && (d & 3) == 0;
    if (vec) {
        const float4 *hv = reinterpret_cast<const float4 *>(h);
        const float4 *wv = reinterpret_cast<const float4 *>(w);
        const int nv = d / 4;
        for (int q0 = first; q0 < nv; q0 += 4 * stride) {
            float4 a[4], c[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int q = q0 + u * stride;
                a[u] = q < nv ? __ldg(hv + q) : make_float4(0.f, 0.f, 0.f, 0.f);
                c[u] = q < nv ? __ldg(wv + q) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                acc = fmaf(a[u].x, c[u].x, acc); acc = fmaf(a[u].y, c[u].y, acc);
                acc = fmaf(a[u].z, c[u].z, acc); acc = fmaf(a[u].w, c[u].w, acc);
            }
        }
    } else {
        for (int j = first; j < d; j += stride) acc = fmaf(h[j], w[j], acc);
    }
    return acc;
}

template <typename T>
__global__ void __launch_bounds__(512, 3) confidence_kernel(const T *__restrict__ h, const T *__restrict__ w,
                                                          float bias, const float *__restrict__ tau, int B, int G,
                                                          int d, int P, float *__restrict__ c_out,
                                                          float *__restrict__ S_out) {
    __shared__ float part[32];
    __shared__ float cs[16];
    const int b = blockIdx.x, wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i = wid / P, p = wid - i * P;   // position, and this warp's share of its row
    if (i < G) {
        const size_t o = (size_t)b * G + i;
        float a = dot_part8(h + o * d, w, d, p * 32 + lane, 32 * P);
        a = warp_sum(a);
        if (lane == 0) part[wid] = a;
    }
    __syncthreads();
    if (threadIdx.x < G) {
        const int ii = threadIdx.x;
        float a = 0.f;
        for (int q = 0; q < P; ++q) a += part[ii * P + q];
        a += bias;
        if (tau != nullptr) a = a / tau[ii];
        const float c = 1.f / (1.f + expf(-a));
        cs[ii] = c;
        c_out[(size_t)b * G + ii] = c;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        float S = 1.f;
        for (int ii = 0; ii < G; ++ii) {
            S *= cs[ii];
            S_out[(size_t)b * G + ii] = S;
        }
    }
}

cudaError_t launch_confidence(const void *h, const void *w, float bias, const float *tau, int B,
                              int G, int d, int dtype, float *c_out, float *S_out, cudaStream_t st) {
    const int P = 1;                     // one warp per position
    const int threads = 32 * G * P;
    if (dtype == DSPARK_BF16)
        confidence_kernel<__nv_bfloat16><<<B, threads, 0, st>>>(
            static_cast<const __nv_bfloat16 *>(h), static_cast<const __nv_bfloat16 *>(w), bias, tau,
            B, G, d, P, c_out, S_out);
    else
        confidence_kernel<float><<<B, threads, 0, st>>>(static_cast<const float *>(h),
                                                        static_cast<const float *>(w), bias, tau, B, G,
                                                        d, P, c_out, S_out);
    return cudaGetLastError();
}

}  // namespace dspark
