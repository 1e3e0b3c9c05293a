// Dispatch of the round's contractions and attention to their kernels.
#pragma once

#include "internal.h"

namespace dspark {

// Tensor-core (tcgen05) path: bf16 models, dense or 4-bit weights. CUDA-core
// path: the fp32 model (its 1e-4 bar excludes TF32).
bool use_tensor_cores(const dspark_model* m);
// Activation rows up to which a dense bf16 model's round GEMMs read the fp16
// pair (hi, lo): there both parts share one MMA of N = 2 BN, so the pair costs
// nothing while the weight stream bounds the GEMM. Above it the GEMMs are bound
// by the MMAs and read hi alone (as do the 4-bit GEMMs).
constexpr int kPairMaxRows = 128;
// Whether a round of M activation rows keeps its GEMM inputs as the fp16 pair (else hi alone).
bool act_pair(const dspark_model* m, int M);
// The activation parts (1 or 2) and the weight format (tc::kW*) of a GEMM.
struct GemmFormat { int np, wfmt; };
GemmFormat round_gemm_format(const dspark_model* m, int M);   // the round's layer GEMMs and lm-head
GemmFormat project_gemm_format(const dspark_model* m);        // the context K/V projection
GemmFormat feature_gemm_format(const dspark_model* m);        // the context feature projection (dense fc)
// Scratch of the tensor-core GEMM's stream-K partial tiles, read back by the
// consumer through its PartView.
struct GemmScratch {
    float* part = nullptr;
};
// fp32 elements of the result buffer run_gemm / run_kv_projection write for an
// [M, K] x [N, K]^T product, and bytes of GemmScratch it needs.
size_t gemm_out_elems(const dspark_model* m, int M, int N, int K);
size_t gemm_scratch_bytes(const dspark_model* m, int M, int N, int K, const GemmFormat& f);
// fp32 elements of the CUDA-core GEMM's split-K result for the same product (any model).
size_t simt_gemm_out_elems(const dspark_model* m, int M, int N, int K);
GemmScratch gemm_scratch_at(void* base, size_t bytes);
// out = X @ W^T for an activation X (fp32, or its bf16 pair on tensor cores); *view reads the result.
cudaError_t run_gemm(const dspark_model* m, const ActBuf& X, const MatRef& W, int M, int N, int K, float* out,
                     const GemmScratch& sc, PartView* view, int timer_kind, cudaStream_t s);
// U[m][v] = softcap(x[m] . lm_head[v]) in fp32 (no cap when final_logit_softcapping == 0), and
// the per-(128-entry vocabulary tile, position) statistics of U into `ts`.
cudaError_t run_lm_head(const dspark_model* m, const ActBuf& x, int M, float* U, const TileStats& ts, cudaStream_t s);
// Context K/V of `nrows` rows of the caller's hidden X (model dtype) into `dst`; x16 holds
// nrows * H fp16 values for the 4-bit GEMM's input (unused otherwise).
// raw = X @ fc^T for `nrows` rows of the caller's tap hiddens X (model dtype, [nrows, fc.k]) and fc
// [H, fc.k] (dense in the model dtype, or 4-bit affine: the CUDA-core GEMM); *view reads the result
// (deepspec.ts #projectContext, before its norm).
cudaError_t run_context_features(const dspark_model* m, const void* X, int nrows, const MatRef& fc, float* raw,
                                 const GemmScratch& sc, PartView* view, cudaStream_t s);
cudaError_t run_kv_projection(const dspark_model* m, const void* X, int nrows, const RowsPlan& rp, const KvDest& dst,
                              float* raw, const GemmScratch& sc, void* x16, cudaStream_t s);
cudaError_t run_attention(const dspark_model* m, const AttnArgs& a, cudaStream_t s);
// CUDA-core attention: context keys per split for A rows of at most max_ctx_len keys.
int attention_key_chunk(const dspark_model* m, int A, int max_ctx_len);
namespace tc {
bool attention_tc_supported(const dspark_model* m);
// V-only caches (K rebuilt from V in the tensor-core attention).
bool vonly_attention_supported(const dspark_model* m);
// Tensor-core attention: CTAs of a call for A rows, ints of its work plan and floats of its
// per-CTA partial state (one slot of 128 rows x (head_dim + 2) per CTA).
int attention_tc_grid(const dspark_model* m, int A);
size_t attention_tc_item_ints(const dspark_model* m, int A);
size_t attention_tc_partial_floats(const dspark_model* m, int grid);
}  // namespace tc


}  // namespace dspark
