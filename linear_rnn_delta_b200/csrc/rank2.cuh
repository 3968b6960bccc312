// Rank-2 steps on the rank-1 kernels: data movement into and out of the
// sub-token layout.
#pragma once
#include "common.cuh"

namespace kda {

// q2[2t] = 0, q2[2t+1] = q[t]; alpha2[2t] = alpha[t], alpha2[2t+1] = 1 (per
// token row of H*d_k elements); cu2[n] = 2 cu[n] for n < n_cu (cu may be null).
cudaError_t launch_rank2_expand(bool bf16, const void *q, const void *alpha, void *q2, void *alpha2,
                                long long tokens, int row_elems, const int32_t *cu, int32_t *cu2, int n_cu,
                                cudaStream_t st);
// o[t] = o2[2t + parity] (per token row of row_elems elements).
cudaError_t launch_rank2_gather(bool bf16, const void *o2, void *o, long long tokens, int row_elems, int parity,
                                cudaStream_t st);
// x2[2t] = 0, x2[2t+1] = x[t] (per token row of row_elems elements).
cudaError_t launch_rank2_spread(bool bf16, const void *x, void *x2, long long tokens, int row_elems, cudaStream_t st);

}  // namespace kda
