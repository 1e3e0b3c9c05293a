// Dispatch of the round's contractions and attention to their kernels.
#pragma once

#include "internal.h"

namespace dspark {

// Number of split-K partials run_gemm writes for an [M, K] x [N, K]^T product.
int gemm_splits(const dspark_model* m, int M, int N, int K);
// out[z][m][n] (z < splits) = partial sums of X[m, :] . W[n, :]; fp32.
cudaError_t run_gemm(const dspark_model* m, const void* X, int64_t ldx, const MatRef& W, int M, int N, int K,
                     int splits, float* out, cudaStream_t s);
// U[m][v] = softcap(x[m] . lm_head[v]) in fp32 (no cap when final_logit_softcapping == 0).
cudaError_t run_lm_head(const dspark_model* m, const void* x, int M, float* U, cudaStream_t s);
// Context K/V of `nrows` rows of X into `dst` (the GEMM over all layers' k_proj plus the norm/RoPE epilogue).
bool project_needs_raw(const dspark_model* m);
cudaError_t run_kv_projection(const dspark_model* m, const void* X, int nrows, const RowsPlan& rp, const KvDest& dst,
                              float* raw, int splits, cudaStream_t s);
cudaError_t run_attention(const dspark_model* m, const AttnArgs& a, cudaStream_t s);

int gemm_prepare_model(dspark_model* m);
void gemm_release_model(dspark_model* m);

}  // namespace dspark
