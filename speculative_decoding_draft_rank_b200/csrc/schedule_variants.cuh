// schedule_variants.cuh -- launcher of the production scheduler's dynamic
// top-K admission (the capacity read from device memory).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace dspark {

cudaError_t launch_schedule_topk(const float *S, int B, int G, const int32_t *capacity, int budget, void *ws,
                                 int32_t *ell_out, int32_t *n_adm_out, int32_t *order_out, cudaStream_t st);

}  // namespace dspark
