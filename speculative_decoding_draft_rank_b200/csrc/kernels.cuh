// kernels.cuh -- launch interfaces shared by the stage files of the library.
#pragma once

#include <cstdlib>

#include "common.cuh"

namespace dspark {

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Clock budget of the bounded device waits of a launch: `dflt`, or the cycle
// count in the environment variable DSPARK_WAIT_BUDGET_CYCLES when it is set
// to a positive number (a failure-path test hook: a budget of a few hundred
// cycles makes the first real wait run out).  Read when the launch is
// enqueued, so a captured graph keeps the value of its capture.
inline long long wait_budget(long long dflt) {
    const char *e = getenv("DSPARK_WAIT_BUDGET_CYCLES");
    if (e == nullptr || *e == 0) return dflt;
    const long long v = atoll(e);
    return v > 0 ? v : dflt;
}
inline int round_up(int x, int m) { return (x + m - 1) / m * m; }

// Columns per partial (max, sum, argmax) of the bf16 tensor-core drafting kernel.
constexpr int kTcTileN = 64;

// ----------------------------------------------------------------- drafting
struct DraftArgs {
    const void *L, *U, *Wt;
    const int32_t *x0;
    const float *temp, *u_draft;
    int B, G, V, r, dtype;
    int32_t *x_out;
    float *pd_out, *rowmax_out, *rowsum_out;
    const void *Arec = nullptr;   // RNN head: recurrent matrix [r, r] (bf16); null for the Markov head
    float *H_out = nullptr;       // RNN head: states [B, G, r] fp32
};

struct DraftWs {
    WsHeader *hdr;
    // Per (row, 64-column segment) partial of the drafting softmax: x = the
    // segment's max, y = its sum of exp((y - max) / T) for a sampled row, or
    // the bits of its lowest argmax (int) for a greedy row.
    float2 *part;
    __nv_bfloat16 *E;
    __nv_bfloat16 *AT;   // bf16 only: the RNN head's recurrent matrix transposed [r, r] (row c = column c of A)   // bf16 only: [B, r] rows U[x_i] staged for the next position's MMA
    int nTiles;
};

int draft_tile_cols(int dtype);
size_t draft_tiles(int V, int dtype);
size_t draft_ws_bytes(int B, int G, int V, int r, int dtype);
DraftWs carve_draft_ws(void *ws, int B, int V, int r, int dtype);
cudaError_t launch_draft(const DraftArgs &a, void *ws, cudaStream_t st);
struct FinArgs;
// bf16 rounds: every position in one cooperative launch of the tensor-core kernel.
cudaError_t launch_draft_tc(const DraftArgs &a, const DraftWs &w, const FinArgs &f, cudaStream_t st);
// bf16 rounds of more than 128 requests: the same on CTA pairs (M = 256 MMAs).
cudaError_t launch_draft_pair(const DraftArgs &a, const DraftWs &w, const FinArgs &f, cudaStream_t st);

// --------------------------------------------------------------- confidence
cudaError_t launch_confidence(const void *h, const void *w, float bias, const float *tau, int B,
                              int G, int d, int dtype, float *c_out, float *S_out, cudaStream_t st);

// ---------------------------------------------------------------- scheduler
size_t schedule_ws_bytes(int B, int G);
cudaError_t launch_schedule(const float *S, int B, int G, const int32_t *knots_n,
                            const double *knots_t, int P, int budget, int mode, float threshold, void *ws,
                            int32_t *ell_out, int32_t *n_adm_out, double *theta_out,
                            int32_t *order_out, cudaStream_t st);

// ------------------------------------------------------------- verification
struct VerifyArgs {
    const void *Tlog, *L, *U, *Wt;
    const int32_t *x0, *x;
    const float *H;   // RNN head: the drafting states [B, G, r]; null for the Markov head (U, x0 used)
    const float *pd_x, *rowmax, *rowsum, *temp, *u_accept, *u_final;
    const int32_t *ell;
    int B, G, V, r, dtype;
    int32_t *acc_out, *tokens_out, *nout_out;
    float *pt_x_out;
};
size_t verify_ws_bytes(int B, int G, int V, int r, int dtype);

// Residual pass of bf16 verification on the tensor cores: rows are the
// queued rejections (count on the device), A operand their gathered U rows.
struct ResidualTcArgs {
    const void *Wt;
    const __nv_bfloat16 *U, *L, *Tlog;
    const int32_t *x0, *x;
    const float *H;   // RNN head: states [B, G, r] (the A rows), else null
    const float *temp, *rowmax, *rowsum, *res_mt, *res_zt;
    const int32_t *res_b, *res_k;
    const uint32_t *nrows;
    int B, G, V, r, nParts;
    float *rp;
    WsHeader *hdr;
};
cudaError_t launch_residual_tile_tc(const ResidualTcArgs &a, cudaStream_t st);
cudaError_t launch_verify(const VerifyArgs &a, void *ws, cudaStream_t st);
// y = 2^x by the FMA-pipe polynomial of common.cuh (diagnostics).
cudaError_t launch_exp2_fma(const float *x, float *y, int n, cudaStream_t st);
// Rows 0..ell[b] of each request of a [B, G+1, V] array from host memory
// mapped into the device's address space (src: its device address).
cudaError_t launch_gather_admitted(const void *src, void *dst, const int32_t *ell, int B, int G, int V,
                                   int elem_bytes, cudaStream_t st);

}  // namespace dspark
