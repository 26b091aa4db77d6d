// gather.cu -- the admitted target rows from page-locked host memory.
//
// The target forward covers only the admitted tokens (paperlayer.ai summary,
// §2 Background: one target pass checks the drafted tokens; menfem.com KB,
// "Key Contributions": the scheduler prunes low-confidence tokens from
// verification), so a round fed from the host needs rows 0..ell_b of
// request b of the target logits [B, G+1, V] and nothing else.  One launch
// pulls exactly those rows over PCIe from host memory mapped into the
// device's address space, reading ell on the device: no host round trip
// between scheduling and verification, and no per-copy overhead of one DMA
// transfer per request.
#include <cstdint>

#include "kernels.cuh"

namespace dspark {

namespace {

constexpr int kGatherThreads = 256;
constexpr int kGatherUnroll = 8;   // loads in flight per thread (host reads have PCIe latency)

// blockIdx.y = request, blockIdx.x = slice of kGatherThreads * kGatherUnroll
// units of the request's rows 0..ell_b (contiguous in the [B, G+1, V]
// layout); slices past the admitted rows return at once.  src is read with
// plain global loads (host memory, not the read-only path).
template <typename Unit>
__global__ void __launch_bounds__(kGatherThreads) gather_admitted_rows(const Unit *src, Unit *__restrict__ dst,
                                                                        const int32_t *__restrict__ ell, int G,
                                                                        size_t units_per_row) {
    const int b = blockIdx.y;
    int e = ell[b];
    e = e < 0 ? 0 : (e > G ? G : e);
    const size_t n = (size_t)(e + 1) * units_per_row;
    const size_t c0 = (size_t)blockIdx.x * (kGatherThreads * kGatherUnroll);
    if (c0 >= n) return;
    const size_t base = (size_t)b * (size_t)(G + 1) * units_per_row + c0;
    Unit v[kGatherUnroll];
#pragma unroll
    for (int u = 0; u < kGatherUnroll; ++u) {
        const size_t i = (size_t)u * kGatherThreads + threadIdx.x;
        if (c0 + i < n) v[u] = src[base + i];
    }
#pragma unroll
    for (int u = 0; u < kGatherUnroll; ++u) {
        const size_t i = (size_t)u * kGatherThreads + threadIdx.x;
        if (c0 + i < n) dst[base + i] = v[u];
    }
}

template <typename Unit>
cudaError_t launch_units(const void *src, void *dst, const int32_t *ell, int B, int G, size_t row_bytes,
                         cudaStream_t st) {
    const size_t upr = row_bytes / sizeof(Unit);
    const size_t per_cta = (size_t)kGatherThreads * kGatherUnroll;
    const size_t gx = ((size_t)(G + 1) * upr + per_cta - 1) / per_cta;
    if (gx > 0x7fffffffu) return cudaErrorInvalidValue;
    gather_admitted_rows<Unit><<<dim3((unsigned)gx, (unsigned)B), kGatherThreads, 0, st>>>(
        static_cast<const Unit *>(src), static_cast<Unit *>(dst), ell, G, upr);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gather_admitted(const void *src, void *dst, const int32_t *ell, int B, int G, int V,
                                   int elem_bytes, cudaStream_t st) {
    const size_t row_bytes = (size_t)V * (size_t)elem_bytes;
    const uintptr_t al = reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst);
    // The widest unit that divides a row and both base addresses.
    if (row_bytes % 16 == 0 && al % 16 == 0) return launch_units<uint4>(src, dst, ell, B, G, row_bytes, st);
    if (row_bytes % 4 == 0 && al % 4 == 0) return launch_units<uint32_t>(src, dst, ell, B, G, row_bytes, st);
    if (row_bytes % 2 == 0 && al % 2 == 0) return launch_units<uint16_t>(src, dst, ell, B, G, row_bytes, st);
    return launch_units<uint8_t>(src, dst, ell, B, G, row_bytes, st);
}

}  // namespace dspark
