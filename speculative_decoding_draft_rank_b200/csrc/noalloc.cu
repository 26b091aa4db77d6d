// noalloc.cu -- drafting entry point that allocates nothing.
//
// Some callers cannot allocate device memory at the point where they draft:
// an inference engine's plugin that is handed only its inputs and outputs at
// enqueue time (the engine planned all memory up front and offers no
// allocator), or a latency-critical serving loop that must never call
// cudaMalloc, which can synchronise the device and stall every stream.  For
// them dspark_draft_markov_noalloc runs the same kernels as
// dspark_draft_markov but keeps its scratch (the workspace header, the
// per-tile partials and the gathered A-operand rows) in a file-scope device
// array of fixed size that every GPU loading this library holds until exit.
#include <mutex>

#include "abi_util.cuh"
#include "common.cuh"
#include "kernels.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB per device

// The scratch itself.  In host code this name is only a stand-in for the
// device symbol; kernels receive the device address obtained below.
static __device__ __align__(256) unsigned char g_draft_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch on the current device, looked up once per
// device (with that device current) and cached.
dspark_status scratch_address(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DSPARK_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_draft_scratch) != cudaSuccess || p == nullptr) return DSPARK_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return DSPARK_OK;
}

}  // namespace

extern "C" {

size_t dspark_draft_noalloc_max_scratch(void) { return kNoAllocScratchBytes; }

dspark_status dspark_draft_markov_noalloc(const void *L, const void *U, const void *Wt, const int32_t *x0,
                                          const float *temp, const float *u_draft, int B, int G, int V,
                                          int r, int dtype, int32_t *x_out, float *pd_x_out,
                                          float *rowmax_out, float *rowsum_out, void *stream) {
    if (dspark_status s = dspark::injected("dspark_draft_markov_noalloc")) return s;
    if (dspark_status s = dspark::check_common(B, G, V, r, dtype)) return s;
    if (!L || !U || !Wt || !x0 || !temp || !u_draft || !x_out || !pd_x_out || !rowmax_out || !rowsum_out)
        return DSPARK_ERR_INVALID_ARG;
    if (dtype == DSPARK_BF16 && !(dspark::aligned16(L) && dspark::aligned16(U) && dspark::aligned16(Wt)))
        return DSPARK_ERR_INVALID_ARG;
    if (dspark::draft_ws_bytes(B, G, V, r, dtype) > kNoAllocScratchBytes) return DSPARK_ERR_WORKSPACE;
    void *ws = nullptr;
    if (dspark_status s = scratch_address(&ws)) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // The scratch keeps the previous call's contents; only the header (the
    // device status word) must start at zero.  Everything else is written
    // before it is read.
    if (cudaMemsetAsync(ws, 0, sizeof(dspark::WsHeader), st) != cudaSuccess) return DSPARK_ERR_CUDA;
    dspark::DraftArgs a{L, U, Wt, x0, temp, u_draft, B, G, V, r, dtype, x_out, pd_x_out, rowmax_out, rowsum_out};
    return dspark::launch_draft(a, ws, st) == cudaSuccess ? DSPARK_OK : DSPARK_ERR_CUDA;
}

dspark_status dspark_draft_noalloc_device_status(void *stream, uint32_t *status_out) {
    if (status_out == nullptr) return DSPARK_ERR_INVALID_ARG;
    void *ws = nullptr;
    if (dspark_status s = scratch_address(&ws)) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t v = 0;
    // Stream order: the word of the last call enqueued on `stream` (calls on
    // other streams must have been ordered before it by the caller).
    if (cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess) return DSPARK_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return DSPARK_ERR_CUDA;
    *status_out = v;
    return DSPARK_OK;
}

}  // extern "C"
