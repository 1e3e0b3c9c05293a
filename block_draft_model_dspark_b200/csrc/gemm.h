// Dispatch of the round's contractions and attention to their kernels.
#pragma once

#include "internal.h"

namespace dspark {

// Tensor-core (tcgen05) path: bf16 dense weights. CUDA-core path: the fp32
// model (its 1e-4 bar excludes TF32) and 4-bit weights.
bool use_tensor_cores(const dspark_model* m);
// Scratch of the tensor-core GEMM's stream-K partial tiles, read back by the
// consumer through its PartView.
struct GemmScratch {
    float* part = nullptr;
};
// fp32 elements of the result buffer run_gemm / run_kv_projection write for an
// [M, K] x [N, K]^T product, and bytes of GemmScratch it needs.
size_t gemm_out_elems(const dspark_model* m, int M, int N, int K);
size_t gemm_scratch_bytes(const dspark_model* m, int M, int N, int K, bool act_pair);
GemmScratch gemm_scratch_at(void* base, size_t bytes);
// out = X @ W^T for an activation X (fp32, or its bf16 pair on tensor cores); *view reads the result.
cudaError_t run_gemm(const dspark_model* m, const ActBuf& X, const MatRef& W, int M, int N, int K, float* out,
                     const GemmScratch& sc, PartView* view, int timer_kind, cudaStream_t s);
// U[m][v] = softcap(x[m] . lm_head[v]) in fp32 (no cap when final_logit_softcapping == 0).
cudaError_t run_lm_head(const dspark_model* m, const ActBuf& x, int M, float* U, cudaStream_t s);
// Context K/V of `nrows` rows of the caller's hidden X (model dtype) into `dst`.
cudaError_t run_kv_projection(const dspark_model* m, const void* X, int nrows, const RowsPlan& rp, const KvDest& dst,
                              float* raw, const GemmScratch& sc, cudaStream_t s);
cudaError_t run_attention(const dspark_model* m, const AttnArgs& a, cudaStream_t s);
// Context keys per split of the attention for A rows of at most max_ctx_len keys.
int attention_key_chunk(const dspark_model* m, int A, int max_ctx_len);

int gemm_prepare_model(dspark_model* m);
void gemm_release_model(dspark_model* m);

}  // namespace dspark
