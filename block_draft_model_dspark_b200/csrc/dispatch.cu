// Chooses the kernel for each contraction: CUDA-core paths for the fp32
// model (whose 1e-4 bar excludes TF32), tensor-core paths for bf16.
#include <algorithm>

#include "gemm.h"

namespace dspark {

cudaError_t launch_attention_simt(const dspark_model* m, const AttnArgs& a, cudaStream_t s);

namespace {
int simt_kps(int K, int S) {
    int kps = (K + S - 1) / S;
    return (kps + 31) / 32 * 32;
}
}  // namespace

int gemm_splits(const dspark_model* m, int M, int N, int K) {
    const int tiles = ((N + 63) / 64) * ((M + 63) / 64);
    int S = std::max(1, std::min((2 * m->num_sms + tiles - 1) / tiles, std::max(1, K / 128)));
    for (;;) {   // the split count the launch will really produce
        const int kps = simt_kps(K, S);
        const int z = (K + kps - 1) / kps;
        if (z == S) return S;
        S = z;
    }
}

double weight_bytes(const dspark_model* m, int64_t N, int64_t K) {
    if (m->d.quant) return (double)N * K * 0.5 + (double)N * (K / m->d.group) * 4.0;
    return (double)N * K * (m->d.dtype == DSPARK_DTYPE_F32 ? 4.0 : 2.0);
}

cudaError_t run_gemm(const dspark_model* m, const void* X, int64_t ldx, const MatRef& W, int M, int N, int K,
                     int splits, float* out, cudaStream_t s) {
    KernelTimer t(DSPARK_TIMER_GEMM, s, weight_bytes(m, N, K) + 4.0 * M * K + 4.0 * M * N, 2.0 * M * N * K);
    return launch_simt_gemm(X, ldx, DSPARK_DTYPE_F32, m->d.dtype, W, m->d.group, M, N, K, splits, out, N,
                            (int64_t)M * N, false, 0.f, s);
}

cudaError_t run_lm_head(const dspark_model* m, const void* x, int M, float* U, cudaStream_t s) {
    const Dims& d = m->d;
    KernelTimer t(DSPARK_TIMER_LM_HEAD, s, weight_bytes(m, d.V, d.H) + 4.0 * M * d.H + 4.0 * M * d.V,
                  2.0 * M * (double)d.V * d.H);
    return launch_simt_gemm(x, d.H, DSPARK_DTYPE_F32, d.dtype, m->lm_head, d.group, M, d.V, d.H, 1, U, d.V, 0, true,
                            d.cap, s);
}

bool project_needs_raw(const dspark_model* m) { (void)m; return true; }

cudaError_t run_kv_projection(const dspark_model* m, const void* X, int nrows, const RowsPlan& rp, const KvDest& dst,
                              float* raw, int splits, cudaStream_t s) {
    const Dims& d = m->d;
    const int N = d.Lyr * d.nKv * d.hd;
    const double es = d.dtype == DSPARK_DTYPE_F32 ? 4.0 : 2.0;
    KernelTimer t(DSPARK_TIMER_KV_PROJECT, s, weight_bytes(m, N, d.H) + es * nrows * d.H + 2.0 * es * nrows * N,
                  2.0 * nrows * (double)N * d.H);
    cudaError_t e = launch_simt_gemm(X, d.H, d.dtype, d.dtype, m->wk_all, d.group, nrows, N, d.H, splits, raw, N,
                                     (int64_t)nrows * N, false, 0.f, s);
    if (e != cudaSuccess) return e;
    return launch_kv_epilogue(m, raw, splits, (int64_t)nrows * N, rp, dst, s);
}

cudaError_t run_attention(const dspark_model* m, const AttnArgs& a, cudaStream_t s) {
    KernelTimer t(DSPARK_TIMER_ATTENTION, s, a.kv_bytes, a.flops);
    return launch_attention_simt(m, a, s);
}

int gemm_prepare_model(dspark_model* m) { (void)m; return DSPARK_OK; }
void gemm_release_model(dspark_model* m) { (void)m; }

}  // namespace dspark
