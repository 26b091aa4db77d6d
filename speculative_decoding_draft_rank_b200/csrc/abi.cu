// abi.cu -- the extern "C" entry points of libdspark: host-side argument
// checks, workspace checks, then the stage launchers.  Nothing here
// allocates memory or synchronises, except dspark_get_device_status.
#include <cstring>

#include "abi_util.cuh"
#include "calibration.cuh"
#include "common.cuh"
#include "kernels.cuh"
#include "schedule_variants.cuh"

using namespace dspark;

namespace {

dspark_status cuda_status(cudaError_t e) { return e == cudaSuccess ? DSPARK_OK : DSPARK_ERR_CUDA; }

bool sts_sizes_ok(int N, int G, int K, int M) {
    return N >= 1 && N <= (1 << 24) && G >= 1 && G <= 16 && K >= 1 && K <= 4096 && M >= 1 && M <= kStsMaxBins;
}

}  // namespace

extern "C" {

const char *dspark_version(void) { return "dspark-b200 0.1 (sm_100a)"; }

size_t dspark_draft_workspace_size(int B, int G, int V, int r, int dtype) {
    if (check_common(B, G, V, r, dtype) != DSPARK_OK) return 0;
    return draft_ws_bytes(B, G, V, r, dtype);
}

dspark_status dspark_draft_markov(const void *L, const void *U, const void *Wt, const int32_t *x0,
                                  const float *temp, const float *u_draft, int B, int G, int V, int r,
                                  int dtype, void *ws, size_t ws_bytes, int32_t *x_out,
                                  float *pd_x_out, float *rowmax_out, float *rowsum_out,
                                  void *stream) {
    if (dspark_status s = injected("dspark_draft_markov")) return s;
    if (dspark_status s = check_common(B, G, V, r, dtype)) return s;
    if (!L || !U || !Wt || !x0 || !temp || !u_draft || !x_out || !pd_x_out || !rowmax_out || !rowsum_out)
        return DSPARK_ERR_INVALID_ARG;
    if (dtype == DSPARK_BF16 && !(aligned16(L) && aligned16(U) && aligned16(Wt))) return DSPARK_ERR_INVALID_ARG;
    if (dspark_status s = check_ws(ws, ws_bytes, draft_ws_bytes(B, G, V, r, dtype))) return s;
    DraftArgs a{L, U, Wt, x0, temp, u_draft, B, G, V, r, dtype, x_out, pd_x_out, rowmax_out, rowsum_out};
    return cuda_status(launch_draft(a, ws, static_cast<cudaStream_t>(stream)));
}

dspark_status dspark_confidence(const void *h, const void *w, float bias, const float *tau, int B,
                                int G, int d, int dtype, float *c_out, float *S_out, void *stream) {
    if (dspark_status s = injected("dspark_confidence")) return s;
    if (!dtype_ok(dtype)) return DSPARK_ERR_UNSUPPORTED_DTYPE;
    if (B < 1 || B > 4096 || G < 1 || G > 16 || d < 1 || d > 65536) return DSPARK_ERR_INVALID_ARG;
    if (!h || !w || !c_out || !S_out) return DSPARK_ERR_INVALID_ARG;
    return cuda_status(launch_confidence(h, w, bias, tau, B, G, d, dtype, c_out, S_out,
                                         static_cast<cudaStream_t>(stream)));
}

size_t dspark_schedule_workspace_size(int B, int G) {
    if (B < 1 || B > 4096 || G < 1 || G > 16 || B * G > 16384) return 0;
    return schedule_ws_bytes(B, G);
}

dspark_status dspark_schedule(const float *S, int B, int G, const int32_t *knots_n,
                              const double *knots_t, int P, int budget, int mode, void *ws,
                              size_t ws_bytes, int32_t *ell_out, int32_t *n_adm_out, double *theta_out,
                              int32_t *order_out, void *stream) {
    if (dspark_status s = injected("dspark_schedule")) return s;
    if (B < 1 || B > 4096 || G < 1 || G > 16 || B * G > 16384 || P < 1 || P > 64)
        return DSPARK_ERR_INVALID_ARG;
    if (mode != DSPARK_SCHED_ALL && mode != DSPARK_SCHED_GREEDY_EARLY_STOP && mode != DSPARK_SCHED_GLOBAL_ARGMAX)
        return DSPARK_ERR_INVALID_ARG;
    if (!S || !knots_n || !knots_t || !ell_out || !n_adm_out || !theta_out) return DSPARK_ERR_INVALID_ARG;
    if (dspark_status s = check_ws(ws, ws_bytes, schedule_ws_bytes(B, G))) return s;
    return cuda_status(launch_schedule(S, B, G, knots_n, knots_t, P, budget, mode, 0.f, ws, ell_out, n_adm_out,
                                       theta_out, order_out, static_cast<cudaStream_t>(stream)));
}

dspark_status dspark_schedule_threshold(const float *S, int B, int G, float threshold, int budget, void *ws,
                                        size_t ws_bytes, int32_t *ell_out, int32_t *n_adm_out,
                                        int32_t *order_out, void *stream) {
    if (dspark_status s = injected("dspark_schedule_threshold")) return s;
    if (B < 1 || B > 4096 || G < 1 || G > 16 || B * G > 16384 || !(threshold == threshold))
        return DSPARK_ERR_INVALID_ARG;
    if (!S || !ell_out || !n_adm_out) return DSPARK_ERR_INVALID_ARG;
    if (dspark_status s = check_ws(ws, ws_bytes, schedule_ws_bytes(B, G))) return s;
    return cuda_status(launch_schedule(S, B, G, nullptr, nullptr, 0, budget, DSPARK_SCHED_THRESHOLD, threshold, ws,
                                       ell_out, n_adm_out, nullptr, order_out, static_cast<cudaStream_t>(stream)));
}

size_t dspark_sts_workspace_size(int N, int G, int K, int n_bins) {
    if (!sts_sizes_ok(N, G, K, n_bins)) return 0;
    return sts_ws_bytes(N, K, n_bins);
}

dspark_status dspark_sts_fit(const float *z, const int32_t *acc, const float *tau_grid, int N, int G, int K,
                             int n_bins, void *ws, size_t ws_bytes, float *tau_out, double *ece_raw_out,
                             double *ece_fit_out, double *ece_all_out, float *S_out, void *stream) {
    if (dspark_status s = injected("dspark_sts_fit")) return s;
    if (!sts_sizes_ok(N, G, K, n_bins) || !z || !acc || !tau_grid || !tau_out) return DSPARK_ERR_INVALID_ARG;
    if (dspark_status s = check_ws(ws, ws_bytes, sts_ws_bytes(N, K, n_bins))) return s;
    StsArgs a{z, acc, tau_grid, N, G, K, n_bins, tau_out, ece_raw_out, ece_fit_out, ece_all_out, S_out};
    return cuda_status(launch_sts_fit(a, ws, static_cast<cudaStream_t>(stream)));
}

dspark_status dspark_survival_auc(const float *S, const int32_t *acc, int N, int G, uint64_t *twice_out,
                                  uint64_t *pairs_out, void *stream) {
    if (dspark_status s = injected("dspark_survival_auc")) return s;
    if (N < 1 || N > (1 << 24) || G < 1 || G > 16 || !S || !acc || !twice_out || !pairs_out)
        return DSPARK_ERR_INVALID_ARG;
    return cuda_status(launch_survival_auc(S, acc, N, G, reinterpret_cast<unsigned long long *>(twice_out),
                                           reinterpret_cast<unsigned long long *>(pairs_out),
                                           static_cast<cudaStream_t>(stream)));
}

dspark_status dspark_schedule_topk(const float *S, int B, int G, const int32_t *capacity, int budget, void *ws,
                                   size_t ws_bytes, int32_t *ell_out, int32_t *n_adm_out, int32_t *order_out,
                                   void *stream) {
    if (dspark_status s = injected("dspark_schedule_topk")) return s;
    if (B < 1 || B > 4096 || G < 1 || G > 16 || B * G > 16384) return DSPARK_ERR_INVALID_ARG;
    if (!S || !capacity || !ell_out || !n_adm_out) return DSPARK_ERR_INVALID_ARG;
    if (dspark_status s = check_ws(ws, ws_bytes, schedule_ws_bytes(B, G))) return s;
    return cuda_status(launch_schedule_topk(S, B, G, capacity, budget, ws, ell_out, n_adm_out, order_out,
                                            static_cast<cudaStream_t>(stream)));
}

size_t dspark_verify_workspace_size(int B, int G, int V, int r, int dtype) {
    if (check_common(B, G, V, r, dtype) != DSPARK_OK) return 0;
    return verify_ws_bytes(B, G, V, r, dtype);
}

dspark_status dspark_verify(const void *Tlog, const void *L, const void *U, const void *Wt,
                            const int32_t *x0, const int32_t *x, const float *pd_x,
                            const float *rowmax, const float *rowsum, const float *temp,
                            const float *u_accept, const float *u_final, const int32_t *ell, int B,
                            int G, int V, int r, int dtype, void *ws, size_t ws_bytes,
                            int32_t *acc_out, int32_t *tokens_out, int32_t *nout_out,
                            float *pt_x_out, void *stream) {
    if (dspark_status s = injected("dspark_verify")) return s;
    if (dspark_status s = check_common(B, G, V, r, dtype)) return s;
    if (!Tlog || !L || !U || !Wt || !x0 || !x || !pd_x || !rowmax || !rowsum || !temp || !u_accept ||
        !u_final || !ell || !acc_out || !tokens_out || !nout_out)
        return DSPARK_ERR_INVALID_ARG;
    if (dtype == DSPARK_BF16 && !(aligned16(Tlog) && aligned16(L) && aligned16(U) && aligned16(Wt)))
        return DSPARK_ERR_INVALID_ARG;
    if (dspark_status s = check_ws(ws, ws_bytes, verify_ws_bytes(B, G, V, r, dtype))) return s;
    VerifyArgs a{Tlog, L, U, Wt, x0, x, nullptr, pd_x, rowmax, rowsum, temp, u_accept, u_final, ell,
                 B, G, V, r, dtype, acc_out, tokens_out, nout_out, pt_x_out};
    return cuda_status(launch_verify(a, ws, static_cast<cudaStream_t>(stream)));
}

dspark_status dspark_gather_admitted_targets(const void *Tlog_host, void *Tlog_dev, const int32_t *ell, int B,
                                             int G, int V, int dtype, void *stream) {
    if (dspark_status s = injected("dspark_gather_admitted_targets")) return s;
    if (!dtype_ok(dtype)) return DSPARK_ERR_UNSUPPORTED_DTYPE;
    if (!Tlog_host || !Tlog_dev || !ell || B < 1 || B > 4096 || G < 1 || G > 16 || V < 1 || V > (1 << 24))
        return DSPARK_ERR_INVALID_ARG;
    // The source must be page-locked host memory that the device can address,
    // the destination device memory: anything else is refused before launch.
    cudaPointerAttributes hs{}, dd{};
    if (cudaPointerGetAttributes(&hs, Tlog_host) != cudaSuccess ||
        cudaPointerGetAttributes(&dd, Tlog_dev) != cudaSuccess) {
        (void)cudaGetLastError();
        return DSPARK_ERR_INVALID_ARG;
    }
    if (hs.type != cudaMemoryTypeHost || hs.devicePointer == nullptr) return DSPARK_ERR_INVALID_ARG;
    if (dd.type != cudaMemoryTypeDevice && dd.type != cudaMemoryTypeManaged) return DSPARK_ERR_INVALID_ARG;
    return cuda_status(launch_gather_admitted(hs.devicePointer, Tlog_dev, ell, B, G, V,
                                              dtype == DSPARK_BF16 ? 2 : 4, static_cast<cudaStream_t>(stream)));
}

dspark_status dspark_draft_rnn(const void *L, const void *U, const void *Arec, const void *Wt, const int32_t *x0,
                               const float *temp, const float *u_draft, int B, int G, int V, int r, int dtype,
                               void *ws, size_t ws_bytes, int32_t *x_out, float *pd_x_out, float *rowmax_out,
                               float *rowsum_out, float *H_out, void *stream) {
    if (dspark_status s = injected("dspark_draft_rnn")) return s;
    if (dspark_status s = check_common(B, G, V, r, dtype)) return s;
    if (dtype != DSPARK_BF16) return DSPARK_ERR_UNSUPPORTED_DTYPE;
    if (r > 256) return DSPARK_ERR_INVALID_ARG;
    if (!L || !U || !Arec || !Wt || !x0 || !temp || !u_draft || !x_out || !pd_x_out || !rowmax_out ||
        !rowsum_out || !H_out)
        return DSPARK_ERR_INVALID_ARG;
    if (!(aligned16(L) && aligned16(U) && aligned16(Wt) && aligned16(H_out))) return DSPARK_ERR_INVALID_ARG;
    if (dspark_status s = check_ws(ws, ws_bytes, draft_ws_bytes(B, G, V, r, dtype))) return s;
    DraftArgs a{L, U, Wt, x0, temp, u_draft, B, G, V, r, dtype, x_out, pd_x_out, rowmax_out, rowsum_out};
    a.Arec = Arec;
    a.H_out = H_out;
    return cuda_status(launch_draft(a, ws, static_cast<cudaStream_t>(stream)));
}

dspark_status dspark_verify_rnn(const void *Tlog, const void *L, const float *H, const void *Wt, const int32_t *x,
                                const float *pd_x, const float *rowmax, const float *rowsum, const float *temp,
                                const float *u_accept, const float *u_final, const int32_t *ell, int B, int G, int V,
                                int r, int dtype, void *ws, size_t ws_bytes, int32_t *acc_out, int32_t *tokens_out,
                                int32_t *nout_out, float *pt_x_out, void *stream) {
    if (dspark_status s = injected("dspark_verify_rnn")) return s;
    if (dspark_status s = check_common(B, G, V, r, dtype)) return s;
    if (dtype != DSPARK_BF16) return DSPARK_ERR_UNSUPPORTED_DTYPE;
    if (r > 256) return DSPARK_ERR_INVALID_ARG;
    if (!Tlog || !L || !H || !Wt || !x || !pd_x || !rowmax || !rowsum || !temp || !u_accept || !u_final || !ell ||
        !acc_out || !tokens_out || !nout_out)
        return DSPARK_ERR_INVALID_ARG;
    if (!(aligned16(Tlog) && aligned16(L) && aligned16(H) && aligned16(Wt))) return DSPARK_ERR_INVALID_ARG;
    if (dspark_status s = check_ws(ws, ws_bytes, verify_ws_bytes(B, G, V, r, dtype))) return s;
    VerifyArgs a{Tlog, L, nullptr, Wt, nullptr, x, H, pd_x, rowmax, rowsum, temp, u_accept, u_final, ell,
                 B, G, V, r, dtype, acc_out, tokens_out, nout_out, pt_x_out};
    return cuda_status(launch_verify(a, ws, static_cast<cudaStream_t>(stream)));
}

dspark_status dspark_get_device_status(const void *ws, void *stream, uint32_t *status_out) {
    if (!ws || !status_out) return DSPARK_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return DSPARK_ERR_CUDA;
    uint32_t v = 0;
    if (cudaMemcpy(&v, ws, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return DSPARK_ERR_CUDA;
    *status_out = v;
    return DSPARK_OK;
}

dspark_status dspark_clear_device_status(void *ws, void *stream) {
    if (!ws) return DSPARK_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    WsHeader *h = static_cast<WsHeader *>(ws);
    if (cudaMemsetAsync(&h->status, 0, sizeof(uint32_t), st) != cudaSuccess) return DSPARK_ERR_CUDA;
    return cuda_status(cudaMemsetAsync(&h->pad[kPadDraftTies], 0, 2 * sizeof(uint32_t), st));
}

dspark_status dspark_exp2_fma(const float *x, float *y, int n, void *stream) {
    if (n < 0 || (n > 0 && (!x || !y))) return DSPARK_ERR_INVALID_ARG;
    if (n == 0) return DSPARK_OK;
    return cuda_status(launch_exp2_fma(x, y, n, static_cast<cudaStream_t>(stream)));
}

dspark_status dspark_get_near_ties(const void *ws, void *stream, uint32_t *draft_out, uint32_t *verify_out) {
    if (!ws || !draft_out || !verify_out) return DSPARK_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return DSPARK_ERR_CUDA;
    uint32_t v[2] = {0, 0};
    const WsHeader *h = static_cast<const WsHeader *>(ws);
    if (cudaMemcpy(v, &h->pad[kPadDraftTies], sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess)
        return DSPARK_ERR_CUDA;
    *draft_out = v[0];
    *verify_out = v[1];
    return DSPARK_OK;
}

}  // extern "C"
