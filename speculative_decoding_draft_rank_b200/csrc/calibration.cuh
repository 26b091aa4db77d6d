// calibration.cuh -- launchers of the confidence-calibration kernels
// (sequential temperature scaling fit, survival ROC-AUC) and their workspace.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace dspark {

constexpr int kStsMaxBins = 32;

// Fit workspace: the status header (pad[0] = the per-launch arrival counter,
// pad[1] = the candidate chosen at the previous position); every candidate's
// survivals [2][K + 1][N] fp64 (double-buffered by position parity; row K is
// the raw chain); per-CTA bin sums [(K + 1) * P][M] fp64; the candidates'
// ECE [K] fp64; per-candidate arrival counters [K + 1].
struct StsWs {
    WsHeader *hdr;
    double *cand;
    double *part;
    double *ece;
    uint32_t *cnt;
};

struct StsArgs {
    const float *z;        // [N, G] head logits
    const int32_t *acc;    // [N] accepted counts
    const float *grid;     // [K] candidate temperatures
    int N, G, K, M;
    float *tau_out;        // [G]
    double *ece_raw_out;   // [G] or null
    double *ece_fit_out;   // [G] or null
    double *ece_all_out;   // [G, K] or null
    float *S_out;          // [N, G] or null
};

int sts_chunks(int N, int K);
size_t sts_ws_bytes(int N, int K, int M);
StsWs sts_ws_carve(void *ws, int N, int K, int M);
cudaError_t launch_sts_fit(const StsArgs &a, void *ws, cudaStream_t st);
cudaError_t launch_survival_auc(const float *S, const int32_t *acc, int N, int G, unsigned long long *twice_out,
                                unsigned long long *pairs_out, cudaStream_t st);

}  // namespace dspark
