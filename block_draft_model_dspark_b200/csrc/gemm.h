// Dispatch of the round's contractions and attention to their kernels.
#pragma once

#include "internal.h"

namespace dspark {

// Tensor-core (tcgen05) path: bf16 dense weights. CUDA-core path: the fp32
// model (its 1e-4 bar excludes TF32) and 4-bit weights.
bool use_tensor_cores(const dspark_model* m);
// fp32 elements of partial output run_gemm / run_kv_projection need for an [M, K] x [N, K]^T product.
size_t gemm_part_elems(const dspark_model* m, int M, int N, int K, bool act_pair);
// out = X @ W^T for an activation X (fp32, or its bf16 pair on tensor cores); *view reads the result.
cudaError_t run_gemm(const dspark_model* m, const ActBuf& X, const MatRef& W, int M, int N, int K, float* part,
                     PartView* view, cudaStream_t s);
// U[m][v] = softcap(x[m] . lm_head[v]) in fp32 (no cap when final_logit_softcapping == 0).
cudaError_t run_lm_head(const dspark_model* m, const ActBuf& x, int M, float* U, float* part, cudaStream_t s);
// Context K/V of `nrows` rows of the caller's hidden X (model dtype) into `dst`.
cudaError_t run_kv_projection(const dspark_model* m, const void* X, int nrows, const RowsPlan& rp, const KvDest& dst,
                              float* raw, cudaStream_t s);
cudaError_t run_attention(const dspark_model* m, const AttnArgs& a, cudaStream_t s);
// Context keys per split of the attention for A rows of at most max_ctx_len keys.
int attention_key_chunk(const dspark_model* m, int A, int max_ctx_len);

int gemm_prepare_model(dspark_model* m);
void gemm_release_model(dspark_model* m);

}  // namespace dspark
