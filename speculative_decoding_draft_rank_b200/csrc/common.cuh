// common.cuh -- shared device helpers of the DSpark round kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/dspark.h"

namespace dspark {

constexpr int kWarp = 32;
constexpr float kLog2e = 1.4426950408889634f;

// Workspace header: the first 256 bytes of every workspace hold the device
// status word (bit set by kernels that clamp bad data) and spare counters.
struct WsHeader {
    uint32_t status;
    uint32_t pad[63];
};
static_assert(sizeof(WsHeader) == 256, "header is 256 bytes");

__device__ __forceinline__ void flag_status(WsHeader *h, uint32_t bit) {
    atomicOr(&h->status, bit);
}

// Near-tie counters in the workspace header: sampled decisions whose uniform
// fell within kNearTie (CDF units) of an edge of the chosen interval, or of
// the accept threshold p_t / p_d.  Drafting counts into pad[8], verification
// into pad[9]; dspark_clear_device_status zeroes both.
constexpr int kPadDraftTies = 8;
constexpr int kPadVerifyTies = 9;
constexpr int kPadSchedArrive = 4;   // the scheduler's arrival counter
constexpr int kPadRowItems = 5;     // the verification row pass's item counter
constexpr float kNearTie = 1e-5f;
__device__ __forceinline__ void count_near_tie(WsHeader *h, int slot) { atomicAdd(&h->pad[slot], 1u); }

// Element loads: fp32 or bf16 widened exactly to fp32.
__device__ __forceinline__ float ld_elem(const float *p, size_t i) { return __ldg(p + i); }
__device__ __forceinline__ float ld_elem(const __nv_bfloat16 *p, size_t i) {
    return __bfloat162float(p[i]);
}
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

// Streaming (read-once) 16-byte load that does not allocate in L1.
__device__ __forceinline__ uint4 ld_stream16(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// Read-only 16-byte load through L1 (neighbouring pieces of a line hit L1).
__device__ __forceinline__ uint4 ld_nc16(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// v rounded to bf16, plus the remainder rounded to bf16: the value a product
// of the two bf16 parts of v (a high and a low part) multiplies by.
__device__ __forceinline__ float split_bf16_sum(float v) {
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    const float h = __bfloat162float(hi);
    return h + __bfloat162float(__float2bfloat16_rn(v - h));
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// exp(x) through the hardware base-2 exponential.
__device__ __forceinline__ float exp_e(float x) { return fast_exp2(x * kLog2e); }

// Two-lane fp32 arithmetic (sm_100: one instruction for both lanes,
// round-to-nearest per lane, as the scalar forms).
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
    float2 r;
    asm("{\n\t.reg .b64 pa, pb, pd;\n\tmov.b64 pa, {%2, %3};\n\tmov.b64 pb, {%4, %5};\n\t"
        "add.rn.f32x2 pd, pa, pb;\n\tmov.b64 {%0, %1}, pd;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return r;
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    float2 r;
    asm("{\n\t.reg .b64 pa, pb, pc, pd;\n\tmov.b64 pa, {%2, %3};\n\tmov.b64 pb, {%4, %5};\n\t"
        "mov.b64 pc, {%6, %7};\n\tfma.rn.f32x2 pd, pa, pb, pc;\n\tmov.b64 {%0, %1}, pd;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return r;
}
// 2^x for two arguments x <= 0 on the FMA pipe, to share the exponential work
// of a softmax with the MUFU unit: x = n + f with n = rint(x) (by the 1.5 * 2^23
// rounding constant, no conversion instruction) and f in [-1/2, 1/2]; 2^f from
// the degree-5 polynomial interpolating it at the six Chebyshev nodes of
// [-1/2, 1/2] (coefficients computed offline; max relative error 2.4e-7 in
// fp32 Horner form, about that of ex2.approx); 2^n added to the exponent
// bits.  Arguments below -125 are raised to -125 (a value of ~1e-38 in place
// of a smaller one).
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
    const float2 lo = make_float2(-125.f, -125.f);
    x = make_float2(fmaxf(x.x, lo.x), fmaxf(x.y, lo.y));
    const float2 big = make_float2(12582912.f, 12582912.f);
    const float2 t = add2(x, big);                       // n in the low mantissa bits
    const float2 f = add2(x, add2(big, make_float2(-t.x, -t.y)));   // x - n
    float2 p = make_float2(0.0013390863314270973f, 0.0013390863314270973f);
    p = fma2(p, f, make_float2(0.009676031768321991f, 0.009676031768321991f));
    p = fma2(p, f, make_float2(0.055503569543361664f, 0.055503569543361664f));
    p = fma2(p, f, make_float2(0.2402210682630539f, 0.2402210682630539f));
    p = fma2(p, f, make_float2(0.6931471824645996f, 0.6931471824645996f));
    p = fma2(p, f, make_float2(1.0000001192092896f, 1.0000001192092896f));
    const int nx = __float_as_int(t.x) - 0x4B400000, ny = __float_as_int(t.y) - 0x4B400000;
    return make_float2(__int_as_float(__float_as_int(p.x) + (nx << 23)),
                       __int_as_float(__float_as_int(p.y) + (ny << 23)));
}

// max(a, b, c) in one instruction.
__device__ __forceinline__ float max3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Dot product of a shared-memory fp32 vector u[0..r) with a global row w
// (fp32 or bf16) read in 16-byte pieces; piece q goes to the threads with
// q % tpc == part.  Eight pieces are loaded before any is used (one memory
// round trip for r <= 64 * tpc bf16); the products are accumulated in piece
// order.  The caller reduces the partial sums across the tpc threads.
__device__ __forceinline__ float dot_part(const float *u, const __nv_bfloat16 *w, int r, int part, int tpc) {
    float acc = 0.f;
    const uint4 *wv = reinterpret_cast<const uint4 *>(w);
    if ((reinterpret_cast<uintptr_t>(w) & 15) == 0 && (r & 7) == 0) {
        const int n = r / 8;
        for (int q0 = part; q0 < n; q0 += 8 * tpc) {
            uint4 v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int q = q0 + i * tpc;
                v[i] = q < n ? __ldg(wv + q) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int q = q0 + i * tpc;
                if (q < n) {
                    const float *uu = u + q * 8;
                    acc = fmaf(uu[0], bf16lo(v[i].x), acc); acc = fmaf(uu[1], bf16hi(v[i].x), acc);
                    acc = fmaf(uu[2], bf16lo(v[i].y), acc); acc = fmaf(uu[3], bf16hi(v[i].y), acc);
                    acc = fmaf(uu[4], bf16lo(v[i].z), acc); acc = fmaf(uu[5], bf16hi(v[i].z), acc);
                    acc = fmaf(uu[6], bf16lo(v[i].w), acc); acc = fmaf(uu[7], bf16hi(v[i].w), acc);
                }
            }
        }
    } else {
        for (int k = part; k < r; k += tpc) acc = fmaf(u[k], __bfloat162float(w[k]), acc);
    }
    return acc;
}
__device__ __forceinline__ float dot_part(const float *u, const float *w, int r, int part, int tpc) {
    float acc = 0.f;
    if ((reinterpret_cast<uintptr_t>(w) & 15) == 0 && (r & 3) == 0) {
        const float4 *wv = reinterpret_cast<const float4 *>(w);
        const int n = r / 4;
        for (int q0 = part; q0 < n; q0 += 8 * tpc) {
            float4 v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int q = q0 + i * tpc;
                v[i] = q < n ? __ldg(wv + q) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int q = q0 + i * tpc;
                if (q < n) {
                    const float *uu = u + q * 4;
                    acc = fmaf(uu[0], v[i].x, acc); acc = fmaf(uu[1], v[i].y, acc);
                    acc = fmaf(uu[2], v[i].z, acc); acc = fmaf(uu[3], v[i].w, acc);
                }
            }
        }
    } else {
        for (int k = part; k < r; k += tpc) acc = fmaf(u[k], w[k], acc);
    }
    return acc;
}

// ---------------------------------------------------------------------------
// Warp reductions and scans.
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ int warp_min_i(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
// (value, index) max with the lower index winning ties.
__device__ __forceinline__ void warp_argmax(float &v, int &i) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        float ov = __shfl_xor_sync(0xffffffffu, v, o);
        int oi = __shfl_xor_sync(0xffffffffu, i, o);
        if (ov > v || (ov == v && oi < i)) { v = ov; i = oi; }
    }
}
// Inclusive prefix sum across the warp (lane order).
__device__ __forceinline__ float warp_incl_scan(float v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        float n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    return v;
}
__device__ __forceinline__ double warp_incl_scan_d(double v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        double n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    return v;
}
__device__ __forceinline__ int warp_incl_scan_i(int v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    return v;
}

// Block-wide inclusive scan of one float per thread (blockDim a multiple of
// 32, at most 1024).  `smem` holds >= 33 floats.  Returns the inclusive
// prefix; *total receives the block sum.
__device__ __forceinline__ float block_incl_scan(float v, float *smem, float *total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    float s = warp_incl_scan(v);
    if (lane == 31) smem[wid] = s;
    __syncthreads();
    if (wid == 0) {
        float t = lane < nw ? smem[lane] : 0.f;
        t = warp_incl_scan(t);
        if (lane < nw) smem[lane] = t;
        if (lane == nw - 1) smem[32] = t;
    }
    __syncthreads();
    float r = s + (wid > 0 ? smem[wid - 1] : 0.f);
    *total = smem[32];
    __syncthreads();
    return r;
}

__device__ __forceinline__ float block_max(float v, float *smem) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    v = warp_max(v);
    if (lane == 0) smem[wid] = v;
    __syncthreads();
    if (wid == 0) {
        float t = lane < nw ? smem[lane] : -INFINITY;
        t = warp_max(t);
        if (lane == 0) smem[32] = t;
    }
    __syncthreads();
    float r = smem[32];
    __syncthreads();
    return r;
}

__device__ __forceinline__ int block_min_i(int v, int *smem) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    v = warp_min_i(v);
    if (lane == 0) smem[wid] = v;
    __syncthreads();
    if (wid == 0) {
        int t = lane < nw ? smem[lane] : 0x7fffffff;
        t = warp_min_i(t);
        if (lane == 0) smem[32] = t;
    }
    __syncthreads();
    int r = smem[32];
    __syncthreads();
    return r;
}

// ---------------------------------------------------------------------------
// One-barrier block reductions.  Every warp publishes its partial into its own
// entry of `slots` (blockDim/32 entries); after a single barrier each thread
// folds all entries in warp order, so every thread gets the same value.  A
// call site must own its `slots` array (no other call writes it while a slow
// warp may still read), which is what removes the trailing barrier.
__device__ __forceinline__ float block_max1(float v, float *slots) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    v = warp_max(v);
    if (lane == 0) slots[wid] = v;
    __syncthreads();
    float r = slots[0];
    for (int w = 1; w < nw; ++w) r = fmaxf(r, slots[w]);
    return r;
}
__device__ __forceinline__ int block_min1(int v, int *slots) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    v = warp_min_i(v);
    if (lane == 0) slots[wid] = v;
    __syncthreads();
    int r = slots[0];
    for (int w = 1; w < nw; ++w) r = min(r, slots[w]);
    return r;
}
__device__ __forceinline__ int block_max1_i(int v, int *slots) { return -block_min1(-v, slots); }
// Inclusive block scan in thread order; *total = block sum (same fold order
// in every thread).
__device__ __forceinline__ float block_scan1(float v, float *slots, float *total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const float s = warp_incl_scan(v);
    if (lane == 31) slots[wid] = s;
    __syncthreads();
    float before = 0.f, tot = 0.f;
    for (int w = 0; w < nw; ++w) {
        if (w == wid) before = tot;
        tot += slots[w];
    }
    *total = tot;
    return before + s;
}

// Clamp a token id to [0, V), flagging the status word when it was outside.
__device__ __forceinline__ int clamp_token(int t, int V, WsHeader *h) {
    if (t < 0 || t >= V) {
        flag_status(h, DSPARK_DEV_TOKEN_RANGE);
        t = t < 0 ? 0 : V - 1;
    }
    return t;
}
// Temperatures: negative or NaN -> 0 (greedy), flagged.
__device__ __forceinline__ float sane_temp(float T, WsHeader *h) {
    if (!(T >= 0.f)) {
        flag_status(h, DSPARK_DEV_BAD_TEMP);
        T = 0.f;
    }
    return T;
}

}  // namespace dspark
