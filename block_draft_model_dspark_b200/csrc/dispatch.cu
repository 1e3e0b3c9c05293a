// Chooses the kernel for each contraction: tcgen05 tensor cores for bf16
// models (dense bf16 weights, or 4-bit weights dequantized to 16 bits in shared
// memory); CUDA cores for the fp32 model, whose 1e-4 bar excludes TF32.
#include <algorithm>

#include "gemm.h"

namespace dspark {

cudaError_t launch_attention_simt(const dspark_model* m, const AttnArgs& a, cudaStream_t s);
namespace tc {
bool attention_tc_supported(const dspark_model* m);
int attention_tc_key_tile();
cudaError_t launch_attention_tc(const dspark_model* m, const AttnArgs& a, cudaStream_t s);
}  // namespace tc

namespace {

int simt_kps(int K, int S) {
    int kps = (K + S - 1) / S;
    return (kps + 31) / 32 * 32;
}

// Split count of the CUDA-core GEMM: ~2 CTAs per SM, then the count the launch really produces.
int simt_splits(const dspark_model* m, int M, int N, int K) {
    const int tiles = ((N + 63) / 64) * ((M + 63) / 64);
    int S = std::max(1, std::min((2 * m->num_sms + tiles - 1) / tiles, std::max(1, K / 128)));
    for (;;) {
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

}  // namespace

bool use_tensor_cores(const dspark_model* m) { return m->d.dtype == DSPARK_DTYPE_BF16; }

bool act_pair(const dspark_model* m, int M) { return use_tensor_cores(m) && !m->d.quant && M <= kPairMaxRows; }

GemmFormat round_gemm_format(const dspark_model* m, int M) {
    if (m->d.quant) return {1, tc::kWQ4AsF16};
    return {act_pair(m, M) ? 2 : 1, tc::kWF16};
}

GemmFormat project_gemm_format(const dspark_model* m) { return {1, m->d.quant ? tc::kWQ4AsF16 : tc::kWBf16}; }

GemmFormat feature_gemm_format(const dspark_model*) { return {1, tc::kWBf16}; }

int attention_key_chunk(const dspark_model* m, int A, int max_ctx_len) {
    // context chunks so that A * nKv (tensor cores) or A * nH (CUDA cores) CTAs per split cover the GPU ~2x
    const Dims& d = m->d;
    const bool tcore = tc::attention_tc_supported(m);
    const int per_split = A * (tcore ? d.nKv : d.nH);
    // tensor cores: one CTA per SM (a CTA holds ~225 KB of shared memory), so one wave
    // of A * nKv * splits CTAs; CUDA cores: ~2 waves
    const int want = tcore ? std::max(1, m->num_sms / per_split)
                           : std::max(1, (2 * m->num_sms + per_split - 1) / per_split);
    const int align = tcore ? tc::attention_tc_key_tile() : 16;
    // tensor cores: >= 2 key tiles per split (each split also pays a Q tile load and
    // writes a 128-row partial O that the merge reads back). At one 4096-key row,
    // attention + merge per layer measured 30.0 us with 4 tiles per split, 27.7 with
    // 2 and 28.3 with 1 (more, smaller partials shift the time into the merge).
    const int min_chunk = tcore ? 2 * tc::attention_tc_key_tile() : 64;
    int chunk = min_chunk;
    if (max_ctx_len > 0) chunk = std::max(min_chunk, (max_ctx_len + want - 1) / want);
    return (chunk + align - 1) / align * align;
}

size_t gemm_out_elems(const dspark_model* m, int M, int N, int K) {
    if (M <= 0) return 0;
    if (use_tensor_cores(m)) return (size_t)M * N;
    return (size_t)simt_splits(m, M, N, K) * M * N;
}

size_t simt_gemm_out_elems(const dspark_model* m, int M, int N, int K) {
    return M <= 0 ? 0 : (size_t)simt_splits(m, M, N, K) * M * N;
}

size_t gemm_scratch_bytes(const dspark_model* m, int M, int N, int K, const GemmFormat& f) {
    if (M <= 0 || !use_tensor_cores(m)) return 0;
    const tc::GemmPlan p = tc::plan_gemm(m->num_sms, M, N, K, f.np, false, false, f.wfmt);
    return tc::gemm_partial_elems(p) * 4;
}

GemmScratch gemm_scratch_at(void* base, size_t bytes) {
    GemmScratch sc;
    if (base && bytes) sc.part = static_cast<float*>(base);
    return sc;
}

namespace {

// The view of a tensor-core GEMM's result: the partial tiles of a stream-K
// plan, else the plain [M, N] result.
void tc_view(const tc::GemmPlan& p, float* out, const GemmScratch& sc, PartView* v) {
    *v = PartView{};
    if (p.streamk) {
        v->mode = 1; v->p = sc.part;
        v->BN = p.BN; v->n_mt = p.n_mt; v->kb = p.kb; v->P = p.P; v->T = p.T; v->G = p.G; v->pair = p.pair;
        v->wide = (int64_t)p.T * p.G >= ((int64_t)1 << 32) || p.T > (1 << 30);
        v->set_divisor((uint32_t)p.T);
    } else {
        v->p = out; v->S = 1; v->stride = (int64_t)p.M * p.N; v->ld = p.N;
    }
}

}  // namespace

cudaError_t run_gemm(const dspark_model* m, const ActBuf& X, const MatRef& W, int M, int N, int K, float* out,
                     const GemmScratch& sc, PartView* view, int timer_kind, cudaStream_t s) {
    KernelTimer t(timer_kind, s, weight_bytes(m, N, K) + 4.0 * M * K + 4.0 * M * N, 2.0 * M * N * K);
    if (use_tensor_cores(m)) {
        const GemmFormat f = round_gemm_format(m, M);
        const tc::GemmPlan p = tc::plan_gemm(m->num_sms, M, N, K, f.np, false, false, f.wfmt);
        tc_view(p, out, sc, view);
        const void* w = m->d.quant ? W.packed : W.w16;
        return tc::launch_gemm_tc(p, w, W.n, X.hi, X.lo, out, N, 0.f, sc.part, m->ws.status, s);
    }
    const int S = simt_splits(m, M, N, K);
    *view = PartView{};
    view->p = out; view->S = S; view->stride = (int64_t)M * N; view->ld = N;
    return launch_simt_gemm(X.f32, K, DSPARK_DTYPE_F32, m->d.dtype, W, m->d.group, M, N, K, S, out, N,
                            (int64_t)M * N, false, 0.f, s);
}

cudaError_t run_lm_head(const dspark_model* m, const ActBuf& x, int M, float* U, const TileStats& ts, cudaStream_t s) {
    const Dims& d = m->d;
    const float* w2norm = d.r > 0 ? m->ws.w2norm : nullptr;
    if (use_tensor_cores(m)) {
        // the logit statistics come out of the epilogue
        KernelTimer t(DSPARK_TIMER_LM_HEAD, s, weight_bytes(m, d.V, d.H) + 4.0 * M * d.H + 4.0 * M * d.V,
                      2.0 * M * (double)d.V * d.H);
        const GemmFormat f = round_gemm_format(m, M);
        const tc::GemmPlan p = tc::plan_gemm(m->num_sms, M, d.V, d.H, f.np, true, true, f.wfmt);
        const void* w = d.quant ? m->lm_head.packed : m->lm_head.w16;
        return tc::launch_gemm_tc(p, w, d.V, x.hi, x.lo, U, d.V, d.cap, nullptr, m->ws.status, s, &ts, w2norm,
                                  m->ws.w1max_bits);
    }
    cudaError_t e;
    {
        KernelTimer t(DSPARK_TIMER_LM_HEAD, s, weight_bytes(m, d.V, d.H) + 4.0 * M * d.H + 4.0 * M * d.V,
                      2.0 * M * (double)d.V * d.H);
        e = launch_simt_gemm(x.f32, d.H, DSPARK_DTYPE_F32, d.dtype, m->lm_head, d.group, M, d.V, d.H, 1, U, d.V, 0,
                             true, d.cap, s);
    }
    if (e != cudaSuccess) return e;
    // a scan of U gives the same statistics
    KernelTimer t(DSPARK_TIMER_ROWS, s, 4.0 * M * d.V, 0.0);
    return launch_tile_stats(m, U, M, ts, s);
}

cudaError_t run_context_features(const dspark_model* m, const void* X, int nrows, const MatRef& fc, float* raw,
                                 const GemmScratch& sc, PartView* view, cudaStream_t s) {
    const Dims& d = m->d;
    const int N = d.H, K = (int)fc.k;
    const double es = d.dtype == DSPARK_DTYPE_F32 ? 4.0 : 2.0;
    KernelTimer t(DSPARK_TIMER_KV_PROJECT, s, es * ((double)N * K + (double)nrows * K + (double)nrows * N),
                  2.0 * nrows * (double)N * K);
    if (use_tensor_cores(m) && !fc.quant) {
        // the caller's rows and fc in bf16, straight from TMA (products exact in fp32); a 4-bit
        // fc takes the CUDA-core GEMM below (dequantized on load)
        const tc::GemmPlan p = tc::plan_gemm(m->num_sms, nrows, N, K, 1, false, false, tc::kWBf16);
        tc_view(p, raw, sc, view);
        return tc::launch_gemm_tc(p, fc.w, N, X, nullptr, raw, N, 0.f, sc.part, m->ws.status, s);
    }
    const int S = simt_splits(m, nrows, N, K);
    *view = PartView{};
    view->p = raw; view->S = S; view->stride = (int64_t)nrows * N; view->ld = N;
    return launch_simt_gemm(X, K, d.dtype, d.dtype, fc, d.group, nrows, N, K, S, raw, N, (int64_t)nrows * N, false,
                            0.f, s);
}

cudaError_t run_kv_projection(const dspark_model* m, const void* X, int nrows, const RowsPlan& rp, const KvDest& dst,
                              float* raw, const GemmScratch& sc, void* x16, cudaStream_t s) {
    const Dims& d = m->d;
    const int N = d.Lyr * d.nKv * d.hd;
    const double es = d.dtype == DSPARK_DTYPE_F32 ? 4.0 : 2.0;
    KernelTimer t(DSPARK_TIMER_KV_PROJECT, s, weight_bytes(m, N, d.H) + es * nrows * d.H + (dst.k ? 2.0 : 1.0) * es * nrows * N,
                  2.0 * nrows * (double)N * d.H);
    PartView view{};
    view.p = raw;
    cudaError_t e;
    if (use_tensor_cores(m)) {
        const GemmFormat f = project_gemm_format(m);
        const tc::GemmPlan p = tc::plan_gemm(m->num_sms, nrows, N, d.H, f.np, false, false, f.wfmt);
        tc_view(p, raw, sc, &view);
        if (d.quant) {
            // 4-bit k_proj is dequantized to fp16 (bf16 would round every weight to 8 bits and
            // move the cached K/V by about one bf16 unit): the caller's bf16 rows become fp16
            e = tc::f16_copy(X, (int64_t)nrows * d.H, x16, m->ws.status, s, DSPARK_DEV_RANGE);
            if (e != cudaSuccess) return e;
            X = x16;
        }
        e = tc::launch_gemm_tc(p, d.quant ? m->wk_all.packed : m->wk_all.w, N, X, nullptr, raw, N, 0.f, sc.part,
                               m->ws.status, s);
    } else {
        const int S = simt_splits(m, nrows, N, d.H);
        view.S = S; view.stride = (int64_t)nrows * N; view.ld = N;
        e = launch_simt_gemm(X, d.H, d.dtype, d.dtype, m->wk_all, d.group, nrows, N, d.H, S, raw, N,
                             (int64_t)nrows * N, false, 0.f, s);
    }
    if (e != cudaSuccess) return e;
    return launch_kv_epilogue(m, view, rp, dst, s);
}

cudaError_t run_attention(const dspark_model* m, const AttnArgs& a, cudaStream_t s) {
    KernelTimer t(DSPARK_TIMER_ATTENTION, s, a.kv_bytes, a.flops);
    if (tc::attention_tc_supported(m)) return tc::launch_attention_tc(m, a, s);
    return launch_attention_simt(m, a, s);
}


}  // namespace dspark
