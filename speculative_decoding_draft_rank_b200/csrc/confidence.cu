// confidence.cu -- stage 2, linear confidence head and prefix survival.
//
// Method (menfem.com KB entry on DSpark, "Key Contributions": a lightweight
// linear confidence head emits a per-position survival probability;
// paperlayer.ai summary, §3.2: cumulative products give the prefix survival,
// calibrated left to right by sequential temperature scaling):
//   c[b,i] = sigmoid((w . h[b,i,:] + bias) / tau[i]),  S[b,i] = prod_{j<=i} c[b,j].
//
// One CTA per request, one warp per position: the warp streams its hidden
// row with 16-byte loads, reduces the dot product by shuffles, and the first
// thread forms the running product.  HBM-bound: B*G*d*esize bytes.
#include "common.cuh"
#include "kernels.cuh"

namespace dspark {

template <typename T>
__device__ __forceinline__ float dot_row(const T *__restrict__ h, const T *__restrict__ w, int d);

template <>
__device__ __forceinline__ float dot_row<__nv_bfloat16>(const __nv_bfloat16 *__restrict__ h,
                                                        const __nv_bfloat16 *__restrict__ w, int d) {
    const int lane = threadIdx.x & 31;
    float acc = 0.f;
    const bool vec = ((reinterpret_cast<uintptr_t>(h) | reinterpret_cast<uintptr_t>(w)) & 15) == 0;
    int done = 0;
    if (vec) {
        const int nv = d / 8;
        const uint4 *hv = reinterpret_cast<const uint4 *>(h);
        const uint4 *wv = reinterpret_cast<const uint4 *>(w);
        for (int j = lane; j < nv; j += 32) {
            uint4 a = ld_stream16(hv + j);
            uint4 b = __ldg(wv + j);
            acc = fmaf(bf16lo(a.x), bf16lo(b.x), acc); acc = fmaf(bf16hi(a.x), bf16hi(b.x), acc);
            acc = fmaf(bf16lo(a.y), bf16lo(b.y), acc); acc = fmaf(bf16hi(a.y), bf16hi(b.y), acc);
            acc = fmaf(bf16lo(a.z), bf16lo(b.z), acc); acc = fmaf(bf16hi(a.z), bf16hi(b.z), acc);
            acc = fmaf(bf16lo(a.w), bf16lo(b.w), acc); acc = fmaf(bf16hi(a.w), bf16hi(b.w), acc);
        }
        done = nv * 8;
    }
    for (int j = done + lane; j < d; j += 32) acc = fmaf(to_f32(h[j]), to_f32(w[j]), acc);
    return warp_sum(acc);
}

template <>
__device__ __forceinline__ float dot_row<float>(const float *__restrict__ h, const float *__restrict__ w,
                                                int d) {
    const int lane = threadIdx.x & 31;
    float acc = 0.f;
    const bool vec = ((reinterpret_cast<uintptr_t>(h) | reinterpret_cast<uintptr_t>(w)) & 15) == 0;
    int done = 0;
    if (vec) {
        const int nv = d / 4;
        const float4 *hv = reinterpret_cast<const float4 *>(h);
        const float4 *wv = reinterpret_cast<const float4 *>(w);
        for (int j = lane; j < nv; j += 32) {
            float4 a = __ldg(hv + j), b = __ldg(wv + j);
            acc = fmaf(a.x, b.x, acc); acc = fmaf(a.y, b.y, acc);
            acc = fmaf(a.z, b.z, acc); acc = fmaf(a.w, b.w, acc);
        }
        done = nv * 4;
    }
    for (int j = done + lane; j < d; j += 32) acc = fmaf(h[j], w[j], acc);
    return warp_sum(acc);
}

template <typename T>
__global__ void confidence_kernel(const T *__restrict__ h, const T *__restrict__ w, float bias,
                                  const float *__restrict__ tau, int B, int G, int d,
                                  float *__restrict__ c_out, float *__restrict__ S_out) {
    __shared__ float cs[16];
    const int b = blockIdx.x, wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (wid < G) {
        const size_t o = (size_t)b * G + wid;
        float a = dot_row<T>(h + o * d, w, d) + bias;
        if (tau != nullptr) a = a / tau[wid];
        if (lane == 0) {
            float c = 1.f / (1.f + expf(-a));
            cs[wid] = c;
            c_out[o] = c;
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        float S = 1.f;
        for (int i = 0; i < G; ++i) {
            S *= cs[i];
            S_out[(size_t)b * G + i] = S;
        }
    }
}

cudaError_t launch_confidence(const void *h, const void *w, float bias, const float *tau, int B,
                              int G, int d, int dtype, float *c_out, float *S_out, cudaStream_t st) {
    const int threads = 32 * G;
    if (dtype == DSPARK_BF16)
        confidence_kernel<__nv_bfloat16><<<B, threads, 0, st>>>(
            static_cast<const __nv_bfloat16 *>(h), static_cast<const __nv_bfloat16 *>(w), bias, tau,
            B, G, d, c_out, S_out);
    else
        confidence_kernel<float><<<B, threads, 0, st>>>(static_cast<const float *>(h),
                                                        static_cast<const float *>(w), bias, tau, B, G,
                                                        d, c_out, S_out);
    return cudaGetLastError();
}

}  // namespace dspark
