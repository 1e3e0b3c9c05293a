// The C ABI of libdspark: argument validation, workspace planning and the
// launch sequence of each call. Every device-side step runs in this
// library's kernels; nothing here computes on the host except the RoPE
// inverse-frequency table and the launch plans.
#include <math.h>
#include <string.h>

#include <algorithm>
#include <string>

#include "internal.h"
#include "gemm.h"

namespace dspark {

static thread_local std::string g_error;
void set_error(const std::string& msg) { g_error = msg; }

cudaError_t launch_attention_simt(const dspark_model* m, const AttnArgs& a, cudaStream_t s);

namespace {

size_t esize(int dtype) { return dtype == DSPARK_DTYPE_F32 ? 4 : 2; }

// ------------------------------------------------------------------ config
int validate_config(const dspark_config* c, std::string* why) {
    auto fail = [&](int code, const std::string& m) { *why = m; return code; };
    if (!c) return fail(DSPARK_ERR_INVALID_ARGUMENT, "config is NULL");
    // readConfig's refusals (deepspec.ts): each would load and compute wrong math.
    if (c->attention_k_eq_v != 1)
        return fail(DSPARK_ERR_UNSUPPORTED, "attention_k_eq_v=false needs a v_proj path; this drafter wires V from k_proj");
    if (c->markov_rank > 0 && c->markov_head_vanilla != 1)
        return fail(DSPARK_ERR_UNSUPPORTED, "only the vanilla Markov head is implemented");
    if (c->hidden_activation_gelu_tanh != 1)
        return fail(DSPARK_ERR_UNSUPPORTED, "only the gelu_pytorch_tanh MLP is implemented");
    if (c->dtype != DSPARK_DTYPE_F32 && c->dtype != DSPARK_DTYPE_BF16) return fail(DSPARK_ERR_UNSUPPORTED, "dtype must be fp32 or bf16");
    if (c->quant_bits != 0 && !(c->quant_bits == 4 && c->quant_group_size == 64 && c->dtype == DSPARK_DTYPE_BF16))
        return fail(DSPARK_ERR_UNSUPPORTED, "quantized weights: only 4-bit affine, group 64, with bf16 activations");
    const int H = c->hidden_size, hd = c->global_head_dim, nH = c->num_attention_heads, nKv = c->num_global_key_value_heads;
    if (H <= 0 || H % 64 || H > 16384) return fail(DSPARK_ERR_UNSUPPORTED, "hidden_size must be a positive multiple of 64, <= 16384");
    if (c->num_hidden_layers < 1 || c->num_hidden_layers > kMaxLayers) return fail(DSPARK_ERR_UNSUPPORTED, "num_hidden_layers must be in [1, 64]");
    if (hd <= 0 || hd % 64 || hd > 256) return fail(DSPARK_ERR_UNSUPPORTED, "global_head_dim must be 64, 128, 192 or 256");
    if (nH <= 0 || nKv <= 0 || nH % nKv) return fail(DSPARK_ERR_UNSUPPORTED, "num_attention_heads must be a positive multiple of num_global_key_value_heads");
    if (c->intermediate_size <= 0 || c->intermediate_size % 64) return fail(DSPARK_ERR_UNSUPPORTED, "intermediate_size must be a positive multiple of 64");
    if (c->vocab_size < 2 || c->vocab_size > (1 << 30)) return fail(DSPARK_ERR_UNSUPPORTED, "vocab_size out of range");
    if (c->mask_token_id < 0 || c->mask_token_id >= c->vocab_size) return fail(DSPARK_ERR_INVALID_ARGUMENT, "mask_token_id outside [0, vocab_size)");
    if (c->block_size < 1 || c->block_size > 32 || c->block_size * hd > 4096)
        return fail(DSPARK_ERR_UNSUPPORTED, "block_size must be in [1, 32] with block_size * head_dim <= 4096");
    if (c->markov_rank != 0 && !(c->markov_rank >= 8 && c->markov_rank <= 256 && (c->markov_rank & (c->markov_rank - 1)) == 0))
        return fail(DSPARK_ERR_UNSUPPORTED, "markov_rank must be 0 or a power of two in [8, 256]");
    if (c->quant_bits == 4 && c->markov_rank % 64) return fail(DSPARK_ERR_UNSUPPORTED, "quantized markov_w2 needs markov_rank % 64 == 0");
    if (c->enable_confidence_head && c->confidence_head_with_markov && c->markov_rank <= 0)
        return fail(DSPARK_ERR_INVALID_ARGUMENT, "confidence_head_with_markov requires markov_rank > 0");
    if (c->quant_bits == 4 && c->enable_confidence_head && (H + (c->confidence_head_with_markov ? c->markov_rank : 0)) % 64)
        return fail(DSPARK_ERR_UNSUPPORTED, "quantized confidence head needs its input width % 64 == 0");
    if (!(c->rms_norm_eps > 0.f) || !(c->rope_theta > 0.f) || c->partial_rotary_factor < 0.f || c->partial_rotary_factor > 1.f)
        return fail(DSPARK_ERR_INVALID_ARGUMENT, "rms_norm_eps, rope_theta or partial_rotary_factor out of range");
    if (c->final_logit_softcapping < 0.f) return fail(DSPARK_ERR_INVALID_ARGUMENT, "final_logit_softcapping must be >= 0 (0 = none)");
    return DSPARK_OK;
}

Dims make_dims(const dspark_config* c) {
    Dims d{};
    d.H = c->hidden_size; d.Lyr = c->num_hidden_layers; d.nH = c->num_attention_heads;
    d.nKv = c->num_global_key_value_heads; d.hd = c->global_head_dim; d.grp = d.nH / d.nKv;
    d.I = c->intermediate_size; d.V = c->vocab_size; d.gamma = c->block_size; d.mask_id = c->mask_token_id;
    d.r = c->markov_rank; d.dtype = c->dtype; d.quant = c->quant_bits == 4; d.group = d.quant ? c->quant_group_size : 64;
    d.eps = c->rms_norm_eps; d.cap = c->final_logit_softcapping; d.conf_thr = c->confidence_threshold;
    d.conf_head = c->enable_confidence_head != 0; d.conf_markov = c->confidence_head_with_markov != 0;
    d.conf_in = d.H + (d.conf_markov ? d.r : 0);
    return d;
}

// Bytes of a stacked matrix [n, k] in the model's weight format.
struct MatBytes { size_t w, s; };
MatBytes mat_bytes(const Dims& d, int64_t n, int64_t k) {
    if (d.quant) return {align_up((size_t)n * (size_t)(k / 8) * 4, 256), align_up((size_t)n * (size_t)(k / d.group) * 2, 256)};
    return {align_up((size_t)n * (size_t)k * esize(d.dtype), 256), 0};
}

struct ModelLayout {
    size_t status, inv_freq, wqk, wqk_s, wqk_b, wgu, wgu_s, wgu_b, wk, wk_s, wk_b, w2norm, w1max, total;
    MatBytes qk, gu, kall;
};
ModelLayout model_layout(const Dims& d) {
    ModelLayout L{};
    size_t o = 0;
    auto take = [&](size_t bytes) { size_t at = o; o += align_up(bytes, 256); return at; };
    L.status = take(256);
    L.inv_freq = take(sizeof(double) * (size_t)(d.hd / 2));
    L.qk = mat_bytes(d, (int64_t)(d.nH + d.nKv) * d.hd, d.H);
    L.gu = mat_bytes(d, 2 * (int64_t)d.I, d.H);
    L.kall = mat_bytes(d, (int64_t)d.Lyr * d.nKv * d.hd, d.H);
    L.wqk = take(L.qk.w * d.Lyr);
    L.wqk_s = take(L.qk.s * d.Lyr);
    L.wqk_b = take(L.qk.s * d.Lyr);
    L.wgu = take(L.gu.w * d.Lyr);
    L.wgu_s = take(L.gu.s * d.Lyr);
    L.wgu_b = take(L.gu.s * d.Lyr);
    L.wk = take(L.kall.w);
    L.wk_s = take(L.kall.s);
    L.wk_b = take(L.kall.s);
    // markov norm bounds of the pruned walk
    const bool prune = walk_prune_model_supported(d);
    L.w2norm = take(prune ? sizeof(float) * (size_t)d.V : 0);
    L.w1max = take(prune ? sizeof(uint32_t) : 0);
    L.total = o;
    return L;
}

MatRef make_ref(const dspark_matrix& m, int64_t n, int64_t k, bool quant) {
    MatRef r;
    r.w = m.w; r.scales = static_cast<const bf16*>(m.scales); r.biases = static_cast<const bf16*>(m.biases);
    r.n = n; r.k = k; r.quant = quant;
    return r;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_matrix(const dspark_matrix& m, bool quant, const char* name, std::string* why) {
    if (!m.w || !aligned16(m.w)) { *why = std::string(name) + ": NULL or not 16-byte aligned"; return DSPARK_ERR_INVALID_ARGUMENT; }
    if (quant && (!m.scales || !m.biases)) { *why = std::string(name) + ": quantized matrix needs scales and biases"; return DSPARK_ERR_INVALID_ARGUMENT; }
    return DSPARK_OK;
}

// Copies rows [0, n) of a matrix into a stacked destination at row `row0`.
cudaError_t copy_rows(const Dims& d, const MatRef& src, void* dw, bf16* ds, bf16* db, int64_t row0, cudaStream_t s) {
    if (!d.quant) {
        const size_t rb = (size_t)src.k * esize(d.dtype);
        return cudaMemcpyAsync(static_cast<char*>(dw) + row0 * rb, src.w, rb * src.n, cudaMemcpyDeviceToDevice, s);
    }
    const size_t wb = (size_t)(src.k / 8) * 4, sb = (size_t)(src.k / d.group) * 2;
    cudaError_t e = cudaMemcpyAsync(static_cast<char*>(dw) + row0 * wb, src.w, wb * src.n, cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return e;
    e = cudaMemcpyAsync(reinterpret_cast<char*>(ds) + row0 * sb, src.scales, sb * src.n, cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return e;
    return cudaMemcpyAsync(reinterpret_cast<char*>(db) + row0 * sb, src.biases, sb * src.n, cudaMemcpyDeviceToDevice, s);
}

MatRef stacked_ref(const Dims& d, void* w, bf16* s, bf16* b, int64_t n, int64_t k) {
    MatRef r; r.w = w; r.scales = s; r.biases = b; r.n = n; r.k = k; r.quant = d.quant;
    return r;
}

// ------------------------------------------------------------------ workspace plans
struct Carve {
    size_t off = 0;
    size_t take(size_t bytes) { size_t at = off; off += align_up(bytes, 256); return at; }
};

struct DraftPlan {
    int M, attn_splits, attn_chunk, walk_blocks;
    bool pairs;   // GEMM inputs also kept as bf16 (hi, lo) pairs for the tensor-core GEMMs
    size_t h, x, part, q, kb, vb, attn_out, act, U, part_o, part_ml, prev, ticket, walk_val, walk_idx, walk_keys;
    size_t x_hi, x_lo, ao_hi, ao_lo, act_hi, act_lo, conf, gscr, gscr_bytes, total;
    bool prune;          // pruned walk ahead of the tensor-core walk
    size_t prune_words, prune_list;   // [T | cnt][M] + fail, and the candidate lists
};

DraftPlan plan_draft(const dspark_model* m, int A, int maxL) {
    const Dims& d = m->d;
    DraftPlan p{};
    p.M = A * d.gamma;
    const int Nqk = (d.nH + d.nKv) * d.hd;
    p.pairs = use_tensor_cores(m);
    const size_t part_elems = std::max({gemm_out_elems(m, p.M, Nqk, d.H), gemm_out_elems(m, p.M, d.H, d.nH * d.hd),
                                        gemm_out_elems(m, p.M, 2 * d.I, d.H), gemm_out_elems(m, p.M, d.H, d.I)});
    p.gscr_bytes = std::max({gemm_scratch_bytes(m, p.M, Nqk, d.H, p.pairs),
                             gemm_scratch_bytes(m, p.M, d.H, d.nH * d.hd, p.pairs),
                             gemm_scratch_bytes(m, p.M, 2 * d.I, d.H, p.pairs),
                             gemm_scratch_bytes(m, p.M, d.H, d.I, p.pairs)});
    const int chunk = attention_key_chunk(m, A, maxL);
    p.attn_chunk = chunk;
    p.attn_splits = maxL > 0 ? (maxL + chunk - 1) / chunk : 0;
    p.walk_blocks = walk_persistent_supported(m, A) ? walk_persistent_blocks(m)
                                                    : walk_vocab_blocks(m->num_sms, d.V, d.r, d.dtype, d.quant);
    Carve c;
    const size_t es = esize(d.dtype);
    p.h = c.take((size_t)p.M * d.H * 4);
    p.x = c.take((size_t)p.M * d.H * 4);
    p.part = c.take(part_elems * 4);
    p.q = c.take((size_t)p.M * d.nH * d.hd * 4);
    p.kb = c.take((size_t)p.M * d.nKv * d.hd * es);
    p.vb = c.take((size_t)p.M * d.nKv * d.hd * es);
    p.attn_out = c.take((size_t)p.M * d.nH * d.hd * 4);
    p.act = c.take((size_t)p.M * d.I * 4);
    p.U = c.take((size_t)p.M * d.V * 4);
    const size_t S1 = (size_t)p.attn_splits + 1;
    p.part_o = c.take((size_t)A * d.nH * S1 * d.gamma * d.hd * 4);
    p.part_ml = c.take((size_t)A * d.nH * S1 * d.gamma * 2 * 4);
    p.prev = c.take((size_t)A * 4);
    p.ticket = c.take(256);
    p.walk_keys = c.take((size_t)d.gamma * A * 8);              // tensor-core walk: per (step, row) maximum
    p.prune = m->ws.w2norm != nullptr && tc::walk_tc_supported(m, A);
    p.prune_words = c.take(p.prune ? (size_t)p.M * 8 + 4 : 0);
    p.prune_list = c.take(p.prune ? (size_t)p.M * kPruneCap * 4 : 0);
    p.walk_val = c.take((size_t)2 * p.walk_blocks * A * 4);     // two step-parity buffers (persistent walk)
    p.walk_idx = c.take((size_t)2 * p.walk_blocks * A * 4);
    const size_t pb = p.pairs ? 2 : 0;
    // each bf16 pair as one [2][M][K] block (lo right after hi): the GEMM loads both with one TMA
    p.x_hi = c.take(2 * (size_t)p.M * d.H * pb);
    p.x_lo = p.x_hi + (size_t)p.M * d.H * pb;
    p.ao_hi = c.take(2 * (size_t)p.M * d.nH * d.hd * pb);
    p.ao_lo = p.ao_hi + (size_t)p.M * d.nH * d.hd * pb;
    p.act_hi = c.take(2 * (size_t)p.M * d.I * pb);
    p.act_lo = p.act_hi + (size_t)p.M * d.I * pb;
    p.conf = c.take((size_t)p.M * 4);
    p.gscr = c.take(p.gscr_bytes);
    p.total = c.off;
    return p;
}

constexpr int64_t kProjectChunkRows = 16384;
constexpr int kMaxAppendBatch = 4096;    // cache batch rows an append handles

struct ProjectPlan {
    int64_t chunk_rows;
    size_t nvalid, row0, raw, gscr, gscr_bytes, total;
};
ProjectPlan plan_project(const dspark_model* m, int64_t rows) {
    const Dims& d = m->d;
    ProjectPlan p{};
    rows = std::max<int64_t>(rows, 1);
    p.chunk_rows = std::min<int64_t>(rows, kProjectChunkRows);
    const int N = d.Lyr * d.nKv * d.hd;
    size_t raw = gemm_out_elems(m, (int)p.chunk_rows, N, d.H);
    p.gscr_bytes = gemm_scratch_bytes(m, (int)p.chunk_rows, N, d.H, false);
    if (rows % p.chunk_rows) {
        raw = std::max(raw, gemm_out_elems(m, (int)(rows % p.chunk_rows), N, d.H));
        p.gscr_bytes = std::max(p.gscr_bytes, gemm_scratch_bytes(m, (int)(rows % p.chunk_rows), N, d.H, false));
    }
    Carve c;
    p.nvalid = c.take(kMaxAppendBatch * 4);
    p.row0 = c.take(kMaxAppendBatch * 4);
    p.raw = c.take(raw * 4);
    p.gscr = c.take(p.gscr_bytes);
    p.total = c.off;
    return p;
}

template <typename P> P* at(void* base, size_t off) { return reinterpret_cast<P*>(static_cast<char*>(base) + off); }

int project_rows(const dspark_model* m, const void* hidden, int B, int Lrows, const int32_t* n_valid,
                 const int32_t* dst_row0, const int32_t* pos0, int static_pos, const KvDest& dst, void* ws,
                 const ProjectPlan& pp, cudaStream_t s) {
    const Dims& d = m->d;
    const int64_t rows = (int64_t)B * Lrows;
    const size_t es = esize(d.dtype);
    const GemmScratch sc = gemm_scratch_at(at<void>(ws, pp.gscr), pp.gscr_bytes);
    for (int64_t r0 = 0; r0 < rows; r0 += pp.chunk_rows) {
        const int nr = (int)std::min<int64_t>(pp.chunk_rows, rows - r0);
        RowsPlan rp{};
        rp.B = B; rp.Lrows = Lrows; rp.row0 = (int)r0; rp.nrows = nr; rp.n_valid = n_valid;
        rp.dst_row0 = dst_row0; rp.pos0 = pos0; rp.static_pos = static_pos;
        const void* X = static_cast<const char*>(hidden) + (size_t)r0 * d.H * es;
        cudaError_t e = run_kv_projection(m, X, nr, rp, dst, at<float>(ws, pp.raw), sc, s);
        if (e != cudaSuccess) DSPARK_FAIL(DSPARK_ERR_CUDA, std::string("context K/V projection launch: ") + cudaGetErrorString(e));
    }
    return DSPARK_OK;
}

}  // namespace
}  // namespace dspark

using namespace dspark;

extern "C" {

const char* dspark_last_error(void) { return g_error.c_str(); }

size_t dspark_model_workspace_bytes(const dspark_config* cfg) {
    std::string why;
    if (validate_config(cfg, &why) != DSPARK_OK) return 0;
    return model_layout(make_dims(cfg)).total;
}

int dspark_model_create(const dspark_config* cfg, const dspark_weights* w, void* model_ws, size_t model_ws_bytes,
                        void* stream, dspark_model** out) {
    std::string why;
    int rc = validate_config(cfg, &why);
    if (rc != DSPARK_OK) DSPARK_FAIL(rc, why);
    if (!w || !out || !model_ws) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "weights, model_ws and out_model must be non-NULL");
    if (reinterpret_cast<uintptr_t>(model_ws) & 255u) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "model_ws must be 256-byte aligned");
    const Dims d = make_dims(cfg);
    const ModelLayout L = model_layout(d);
    if (model_ws_bytes < L.total)
        DSPARK_FAIL(DSPARK_ERR_WORKSPACE, "model_ws smaller than dspark_model_workspace_bytes(): " + std::to_string(L.total));
    if (!w->layers) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "weights.layers is NULL");
    const bool q = d.quant;
    if ((rc = check_matrix(w->embed_tokens, q, "embed_tokens", &why)) || (rc = check_matrix(w->lm_head, q, "lm_head", &why)))
        DSPARK_FAIL(rc, why);
    if (d.r > 0 && ((rc = check_matrix(w->markov_w2, q, "markov_w2", &why)) || !w->markov_w1))
        DSPARK_FAIL(rc ? rc : DSPARK_ERR_INVALID_ARGUMENT, rc ? why : "markov_w1 is NULL");
    if (d.conf_head && ((rc = check_matrix(w->confidence_proj, q, "confidence_proj", &why)) || !w->confidence_bias))
        DSPARK_FAIL(rc ? rc : DSPARK_ERR_INVALID_ARGUMENT, rc ? why : "confidence_bias is NULL");
    if (!w->norm) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "norm is NULL");
    for (int l = 0; l < d.Lyr; ++l) {
        const dspark_layer_weights& lw = w->layers[l];
        const dspark_matrix* mats[6] = {&lw.q_proj, &lw.k_proj, &lw.o_proj, &lw.gate_proj, &lw.up_proj, &lw.down_proj};
        for (auto* mm : mats)
            if ((rc = check_matrix(*mm, q, "layer matrix", &why))) DSPARK_FAIL(rc, why + " (layer " + std::to_string(l) + ")");
        if (!lw.q_norm || !lw.k_norm || !lw.input_layernorm || !lw.post_attention_layernorm || !lw.pre_feedforward_layernorm ||
            !lw.post_feedforward_layernorm || !lw.layer_scalar)
            DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "a norm gain or layer_scalar is NULL (layer " + std::to_string(l) + ")");
    }

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    dspark_model* m = new dspark_model();
    m->cfg = *cfg;
    m->d = d;
    cudaGetDevice(&m->device);
    cudaDeviceGetAttribute(&m->num_sms, cudaDevAttrMultiProcessorCount, m->device);
    char* base = static_cast<char*>(model_ws);
    m->ws.status = reinterpret_cast<int32_t*>(base + L.status);
    m->ws.inv_freq = reinterpret_cast<double*>(base + L.inv_freq);
    m->ws.wqk = base + L.wqk; m->ws.wgu = base + L.wgu; m->ws.wk_all = base + L.wk;
    m->ws.wqk_s = reinterpret_cast<bf16*>(base + L.wqk_s); m->ws.wqk_b = reinterpret_cast<bf16*>(base + L.wqk_b);
    m->ws.wgu_s = reinterpret_cast<bf16*>(base + L.wgu_s); m->ws.wgu_b = reinterpret_cast<bf16*>(base + L.wgu_b);
    m->ws.wk_all_s = reinterpret_cast<bf16*>(base + L.wk_s); m->ws.wk_all_b = reinterpret_cast<bf16*>(base + L.wk_b);

    // RoPE inverse frequencies theta^(-2k/hd) for k < floor(hd*partial)/2, 0 (identity) beyond.
    std::vector<double> inv(d.hd / 2, 0.0);
    const int rotated = (int)floor((double)d.hd * (double)cfg->partial_rotary_factor);
    for (int k = 0; k < d.hd / 2 && k < rotated / 2.0; ++k) inv[k] = pow((double)cfg->rope_theta, -2.0 * k / d.hd);

    const int64_t Nqk = (int64_t)(d.nH + d.nKv) * d.hd;
    m->layers.resize(d.Lyr);
    cudaError_t e = cudaMemsetAsync(m->ws.status, 0, 256, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(m->ws.inv_freq, inv.data(), inv.size() * sizeof(double), cudaMemcpyHostToDevice, s);
    for (int l = 0; l < d.Lyr && e == cudaSuccess; ++l) {
        const dspark_layer_weights& lw = w->layers[l];
        LayerRef& R = m->layers[l];
        const size_t wq = L.qk.w * l, sq = L.qk.s * l, wg = L.gu.w * l, sg = L.gu.s * l;
        void* qkw = base + L.wqk + wq; bf16* qks = at<bf16>(base, L.wqk_s + sq); bf16* qkb = at<bf16>(base, L.wqk_b + sq);
        void* guw = base + L.wgu + wg; bf16* gus = at<bf16>(base, L.wgu_s + sg); bf16* gub = at<bf16>(base, L.wgu_b + sg);
        const MatRef mq = make_ref(lw.q_proj, (int64_t)d.nH * d.hd, d.H, q);
        const MatRef mk = make_ref(lw.k_proj, (int64_t)d.nKv * d.hd, d.H, q);
        const MatRef mg = make_ref(lw.gate_proj, d.I, d.H, q);
        const MatRef mu = make_ref(lw.up_proj, d.I, d.H, q);
        e = copy_rows(d, mq, qkw, qks, qkb, 0, s);
        if (e == cudaSuccess) e = copy_rows(d, mk, qkw, qks, qkb, (int64_t)d.nH * d.hd, s);
        if (e == cudaSuccess) e = copy_rows(d, mg, guw, gus, gub, 0, s);
        if (e == cudaSuccess) e = copy_rows(d, mu, guw, gus, gub, d.I, s);
        if (e == cudaSuccess)
            e = copy_rows(d, mk, base + L.wk, at<bf16>(base, L.wk_s), at<bf16>(base, L.wk_b), (int64_t)l * d.nKv * d.hd, s);
        R.qk = stacked_ref(d, qkw, qks, qkb, Nqk, d.H);
        R.gu = stacked_ref(d, guw, gus, gub, 2 * (int64_t)d.I, d.H);
        R.o = make_ref(lw.o_proj, d.H, (int64_t)d.nH * d.hd, q);
        R.down = make_ref(lw.down_proj, d.H, d.I, q);
        R.q_norm = lw.q_norm; R.k_norm = lw.k_norm; R.in_norm = lw.input_layernorm;
        R.post_attn_norm = lw.post_attention_layernorm; R.pre_ff_norm = lw.pre_feedforward_layernorm;
        R.post_ff_norm = lw.post_feedforward_layernorm; R.layer_scalar = lw.layer_scalar;
    }
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);   // the host RoPE table must be consumed
    if (e != cudaSuccess) {
        delete m;
        DSPARK_FAIL(DSPARK_ERR_CUDA, std::string("model set-up copies: ") + cudaGetErrorString(e));
    }
    m->wk_all = stacked_ref(d, base + L.wk, at<bf16>(base, L.wk_s), at<bf16>(base, L.wk_b), (int64_t)d.Lyr * d.nKv * d.hd, d.H);
    m->embed = make_ref(w->embed_tokens, d.V, d.H, q);
    m->lm_head = make_ref(w->lm_head, d.V, d.H, q);
    if (d.r > 0) m->w2 = make_ref(w->markov_w2, d.V, d.r, q);
    if (d.conf_head) m->conf_proj = make_ref(w->confidence_proj, 1, d.conf_in, q);
    m->w1 = w->markov_w1;
    m->final_norm = w->norm;
    m->conf_bias = w->confidence_bias;
    // norm bounds of the pruned walk: once per model, from the weights as given
    if (walk_prune_model_supported(d) && aligned16(m->w1) && aligned16(m->w2.w)) {
        m->ws.w2norm = reinterpret_cast<float*>(base + L.w2norm);
        m->ws.w1max_bits = reinterpret_cast<uint32_t*>(base + L.w1max);
        e = launch_markov_norms(m, s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) {
            delete m;
            DSPARK_FAIL(DSPARK_ERR_CUDA, std::string("markov norm bounds: ") + cudaGetErrorString(e));
        }
    }
    rc = gemm_prepare_model(m);
    if (rc != DSPARK_OK) { delete m; return rc; }
    *out = m;
    return DSPARK_OK;
}

int dspark_model_destroy(dspark_model* m) {
    if (!m) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "model is NULL");
    gemm_release_model(m);
    delete m;
    return DSPARK_OK;
}

size_t dspark_project_workspace_bytes(const dspark_model* m, int64_t rows) {
    if (!m || rows < 0) return 0;
    return plan_project(m, rows).total;
}

int dspark_project_context_kv(const dspark_model* m, const void* hidden, int32_t B, int32_t L, int32_t static_pos,
                              const int32_t* pos0, void* k_out, void* v_out, void* ws, size_t ws_bytes, void* stream) {
    if (!m) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "model is NULL");
    if (B < 0 || L < 0) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "B and L must be >= 0");
    if ((int64_t)B * L == 0) return DSPARK_OK;
    if ((int64_t)B * L > (int64_t)1 << 30) DSPARK_FAIL(DSPARK_ERR_UNSUPPORTED, "B * L above 2^30 rows");
    if (!hidden || !k_out || !v_out || !ws) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "hidden, k_out, v_out and ws must be non-NULL");
    if (!aligned16(hidden) || !aligned16(k_out) || !aligned16(v_out)) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "buffers must be 16-byte aligned");
    if (!pos0 && static_pos < 0) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "static_pos must be >= 0");
    const ProjectPlan pp = plan_project(m, (int64_t)B * L);
    if (ws_bytes < pp.total) DSPARK_FAIL(DSPARK_ERR_WORKSPACE, "ws smaller than dspark_project_workspace_bytes(): " + std::to_string(pp.total));
    const Dims& d = m->d;
    KvDest dst{};
    dst.k = k_out; dst.v = v_out; dst.capacity = L;
    dst.batch_stride = (int64_t)L * d.nKv * d.hd;
    dst.layer_stride = (int64_t)B * dst.batch_stride;
    return project_rows(m, hidden, B, L, nullptr, nullptr, pos0, static_pos, dst, ws, pp, static_cast<cudaStream_t>(stream));
}

int dspark_append_context_kv(const dspark_model* m, const void* hidden, int32_t Lnew_max, const int32_t* n_new,
                             const int32_t* pos0, dspark_kv_cache* cache, void* ws, size_t ws_bytes, void* stream) {
    if (!m || !cache) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "model and cache must be non-NULL");
    const int B = cache->batch;
    if (B <= 0 || B > kMaxAppendBatch) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "cache.batch must be in [1, 4096]");
    if (Lnew_max < 0 || Lnew_max > cache->capacity) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "Lnew_max must be in [0, cache.capacity]");
    if ((int64_t)B * Lnew_max > (int64_t)1 << 30) DSPARK_FAIL(DSPARK_ERR_UNSUPPORTED, "batch * Lnew_max above 2^30 rows");
    if (!n_new || !pos0 || !cache->len || !cache->k || !cache->v)
        DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "n_new, pos0 and the cache's k, v, len must be non-NULL");
    if (!aligned16(cache->k) || !aligned16(cache->v)) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "cache k / v must be 16-byte aligned");
    if (Lnew_max == 0) return DSPARK_OK;
    if (!hidden || !ws || !aligned16(hidden)) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "hidden and ws must be non-NULL, 16-byte aligned");
    const ProjectPlan pp = plan_project(m, (int64_t)B * Lnew_max);
    if (ws_bytes < pp.total) DSPARK_FAIL(DSPARK_ERR_WORKSPACE, "ws smaller than dspark_project_workspace_bytes(): " + std::to_string(pp.total));
    const Dims& d = m->d;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t* nvalid = at<int32_t>(ws, pp.nvalid);
    int32_t* row0 = at<int32_t>(ws, pp.row0);
    // the counts live on the device: validate them there (a refused append writes nothing)
    cudaError_t e = launch_append_check(n_new, cache->len, B, Lnew_max, cache->capacity, nvalid, row0, m->ws.status, s);
    if (e != cudaSuccess) DSPARK_FAIL(DSPARK_ERR_CUDA, std::string("append check: ") + cudaGetErrorString(e));
    KvDest dst{};
    dst.k = cache->k; dst.v = cache->v; dst.capacity = cache->capacity;
    dst.batch_stride = (int64_t)cache->capacity * d.nKv * d.hd;
    dst.layer_stride = (int64_t)B * dst.batch_stride;
    int rc = project_rows(m, hidden, B, Lnew_max, nvalid, row0, pos0, 0, dst, ws, pp, s);
    if (rc != DSPARK_OK) return rc;
    e = launch_commit_len(cache->len, nvalid, B, s);
    if (e != cudaSuccess) DSPARK_FAIL(DSPARK_ERR_CUDA, std::string("append commit: ") + cudaGetErrorString(e));
    return DSPARK_OK;
}

size_t dspark_draft_workspace_bytes(const dspark_model* m, int32_t A, int32_t max_ctx_len) {
    if (!m || A <= 0 || max_ctx_len < 0) return 0;
    return plan_draft(m, A, max_ctx_len).total;
}

static int check_cache(const dspark_model* m, const dspark_kv_cache* c, int A, int maxL, std::string* why) {
    if (!c || !c->k || !c->v || !c->len) { *why = "cache and its k, v, len must be non-NULL"; return DSPARK_ERR_INVALID_ARGUMENT; }
    if (A <= 0 || A > c->batch) { *why = "A must be in [1, cache.batch]"; return DSPARK_ERR_INVALID_ARGUMENT; }
    if (maxL < 0 || maxL > c->capacity) { *why = "max_ctx_len must be in [0, cache.capacity]"; return DSPARK_ERR_INVALID_ARGUMENT; }
    if (!aligned16(c->k) || !aligned16(c->v)) { *why = "cache k / v must be 16-byte aligned"; return DSPARK_ERR_INVALID_ARGUMENT; }
    (void)m;
    return DSPARK_OK;
}

static AttnArgs attn_args(const dspark_model* m, const DraftPlan& p, void* ws, const dspark_kv_cache* c, int layer, int A,
                          const void* q, const void* kb, const void* vb, void* out, int io_dtype) {
    const Dims& d = m->d;
    const size_t es = esize(d.dtype);
    const size_t layer_bytes = (size_t)c->batch * c->capacity * d.nKv * d.hd * es;
    AttnArgs a{};
    a.q = q; a.kb = kb; a.vb = vb; a.out = out;
    a.q_dtype = io_dtype; a.out_dtype = io_dtype;
    a.kc = static_cast<const char*>(c->k) + layer_bytes * layer;
    a.vc = static_cast<const char*>(c->v) + layer_bytes * layer;
    a.len = c->len; a.capacity = c->capacity; a.batch = c->batch;
    a.part_o = at<float>(ws, p.part_o); a.part_ml = at<float>(ws, p.part_ml);
    a.A = A; a.n_splits = p.attn_splits; a.chunk = p.attn_chunk;
    a.status = m->ws.status;
    // algorithmic work: every valid context row's K and V once, the block K/V, q and out
    double keys = (double)A * d.gamma;
    if (c->len_host)
        for (int b = 0; b < A; ++b) keys += c->len_host[b];
    else
        keys += (double)A * c->capacity;
    const double qo = 2.0 * A * d.gamma * d.nH * d.hd * (io_dtype == DSPARK_DTYPE_F32 ? 4.0 : (double)es);
    a.kv_bytes = keys * d.nKv * d.hd * 2.0 * es + qo;
    a.flops = 4.0 * (double)d.nH * d.gamma * d.hd * keys;
    return a;
}

int dspark_attend(const dspark_model* m, int32_t layer, const dspark_kv_cache* cache, const void* q, const void* k_blk,
                  const void* v_blk, void* out, int32_t A, int32_t max_ctx_len, void* ws, size_t ws_bytes, void* stream) {
    if (!m) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "model is NULL");
    std::string why;
    int rc = check_cache(m, cache, A, max_ctx_len, &why);
    if (rc) DSPARK_FAIL(rc, why);
    if (layer < 0 || layer >= m->d.Lyr) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "layer out of range");
    if (!q || !k_blk || !v_blk || !out || !ws) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "q, k_blk, v_blk, out and ws must be non-NULL");
    const DraftPlan p = plan_draft(m, A, max_ctx_len);
    if (ws_bytes < p.total) DSPARK_FAIL(DSPARK_ERR_WORKSPACE, "ws smaller than dspark_draft_workspace_bytes(): " + std::to_string(p.total));
    const AttnArgs a = attn_args(m, p, ws, cache, layer, A, q, k_blk, v_blk, out, m->d.dtype);
    cudaError_t e = run_attention(m, a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) DSPARK_FAIL(DSPARK_ERR_CUDA, std::string("attention launch: ") + cudaGetErrorString(e));
    return DSPARK_OK;
}

int dspark_draft_rows(const dspark_model* m, const dspark_kv_cache* cache, const int32_t* anchors,
                      const int32_t* block_pos, int32_t A, int32_t max_ctx_len, int32_t* tokens, float* conf,
                      int32_t* lengths, float* base_logits, void* ws, size_t ws_bytes, void* stream) {
    if (!m) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "model is NULL");
    std::string why;
    int rc = check_cache(m, cache, A, max_ctx_len, &why);
    if (rc) DSPARK_FAIL(rc, why);
    if (!anchors || !block_pos || !tokens || !lengths || !ws)
        DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "anchors, block_pos, tokens, lengths and ws must be non-NULL");
    if (conf && !m->d.conf_head) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "conf requested but the confidence head is disabled");
    const DraftPlan p = plan_draft(m, A, max_ctx_len);
    if (ws_bytes < p.total) DSPARK_FAIL(DSPARK_ERR_WORKSPACE, "ws smaller than dspark_draft_workspace_bytes(): " + std::to_string(p.total));
    const Dims& d = m->d;
    const size_t dump_layer = (size_t)A * d.gamma * d.nH * d.hd * sizeof(float);
    if (m->attn_dump && m->attn_dump_bytes < dump_layer * d.Lyr)
        DSPARK_FAIL(DSPARK_ERR_WORKSPACE, "attention dump smaller than num_hidden_layers * A * gamma * nH * hd floats");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int M = p.M;
    float* h = at<float>(ws, p.h);
    float* part = at<float>(ws, p.part);
    float* q = at<float>(ws, p.q); void* kb = at<void>(ws, p.kb); void* vb = at<void>(ws, p.vb);
    float* U = base_logits ? base_logits : at<float>(ws, p.U);
    ActBuf x, ao, act;
    x.f32 = at<float>(ws, p.x); ao.f32 = at<float>(ws, p.attn_out); act.f32 = at<float>(ws, p.act);
    if (p.pairs) {
        x.hi = at<bf16>(ws, p.x_hi); x.lo = at<bf16>(ws, p.x_lo);
        ao.hi = at<bf16>(ws, p.ao_hi); ao.lo = at<bf16>(ws, p.ao_lo);
        act.hi = at<bf16>(ws, p.act_hi); act.lo = at<bf16>(ws, p.act_lo);
    }
    const int Nqk = (d.nH + d.nKv) * d.hd;
    PartView pv;
    const GemmScratch sc = gemm_scratch_at(at<void>(ws, p.gscr), p.gscr_bytes);
    // the persistent walk's grid-barrier counter
    cudaError_t e = cudaMemsetAsync(at<uint32_t>(ws, p.ticket), 0, sizeof(uint32_t), s);
    if (e == cudaSuccess) e = cudaMemsetAsync(at<void>(ws, p.walk_keys), 0, (size_t)d.gamma * A * 8, s);
    if (e == cudaSuccess && p.prune) e = cudaMemsetAsync(at<void>(ws, p.prune_words), 0, (size_t)M * 8 + 4, s);
    if (e == cudaSuccess) e = launch_embed(m, anchors, A, h, x, m->ws.status, s);
    for (int l = 0; l < d.Lyr && e == cudaSuccess; ++l) {
        const LayerRef& L = m->layers[l];
        e = run_gemm(m, x, L.qk, M, Nqk, d.H, part, sc, &pv, DSPARK_TIMER_GEMM_QK, s);
        if (e == cudaSuccess) e = launch_qk_epilogue(m, l, pv, A, block_pos, q, kb, vb, s);
        if (e == cudaSuccess) {
            AttnArgs a = attn_args(m, p, ws, cache, l, A, q, kb, vb, ao.f32, DSPARK_DTYPE_F32);
            a.out_hi = ao.hi; a.out_lo = ao.lo;
            e = run_attention(m, a, s);
        }
        if (e == cudaSuccess && m->attn_dump)
            e = cudaMemcpyAsync(reinterpret_cast<char*>(m->attn_dump) + dump_layer * l, ao.f32, dump_layer,
                                cudaMemcpyDeviceToDevice, s);
        if (e == cudaSuccess) e = run_gemm(m, ao, L.o, M, d.H, d.nH * d.hd, part, sc, &pv, DSPARK_TIMER_GEMM_O, s);
        if (e == cudaSuccess) e = launch_o_epilogue(m, l, pv, M, h, x, s);
        if (e == cudaSuccess) e = run_gemm(m, x, L.gu, M, 2 * d.I, d.H, part, sc, &pv, DSPARK_TIMER_GEMM_GU, s);
        if (e == cudaSuccess) e = launch_gu_epilogue(m, pv, M, act, s);
        if (e == cudaSuccess) e = run_gemm(m, act, L.down, M, d.H, d.I, part, sc, &pv, DSPARK_TIMER_GEMM_DOWN, s);
        if (e == cudaSuccess) e = launch_down_epilogue(m, l, pv, M, h, x, s);
    }
    if (e == cudaSuccess) e = run_lm_head(m, x, M, U, s);
    if (e == cudaSuccess) {
        WalkArgs wa{};
        wa.U = U; wa.tokens = tokens; wa.prev = at<int32_t>(ws, p.prev);
        wa.part_val = at<float>(ws, p.walk_val); wa.part_idx = at<int32_t>(ws, p.walk_idx);
        wa.ticket = at<uint32_t>(ws, p.ticket); wa.A = A; wa.nblk = p.walk_blocks; wa.status = m->ws.status;
        const double w2b = d.r > 0 ? (d.quant ? (double)d.V * d.r * 0.5 + (double)d.V * (d.r / d.group) * 4.0
                                              : (double)d.V * d.r * esize(d.dtype)) : 0.0;
        if (tc::walk_tc_supported(m, A)) {
            const int* skip = nullptr;
            if (p.prune) {
                PruneScratch ps;
                ps.T = at<uint32_t>(ws, p.prune_words);
                ps.cnt = at<int>(ws, p.prune_words + (size_t)M * 4);
                ps.fail = at<int>(ws, p.prune_words + (size_t)M * 8);
                ps.list = at<int>(ws, p.prune_list);
                // algorithmic bytes: the two scans of U
                KernelTimer t(DSPARK_TIMER_WALK, s, 2.0 * 4.0 * A * d.gamma * (double)d.V, 0.0);
                e = launch_walk_prune(m, U, anchors, tokens, A, ps, s);
                skip = ps.fail;
            }
            // with the pruned walk ahead, the full walk runs only when a candidate list
            // overflowed: its work is then not counted (it usually returns at once)
            const bool full_counted = skip == nullptr;
            KernelTimer t(DSPARK_TIMER_WALK, s, full_counted ? d.gamma * (w2b + 4.0 * A * d.V) : 0.0,
                          full_counted ? 2.0 * d.gamma * A * (double)d.V * d.r : 0.0);
            if (e == cudaSuccess)
                e = tc::launch_walk_tc(m, U, anchors, tokens, at<unsigned long long>(ws, p.walk_keys), wa.ticket, skip, A, s);
        } else if (walk_persistent_supported(m, A)) {
            KernelTimer t(DSPARK_TIMER_WALK, s, d.gamma * (w2b + 4.0 * A * d.V), 2.0 * d.gamma * A * (double)d.V * d.r);
            e = launch_walk_persistent(m, U, anchors, tokens, wa.part_val, wa.part_idx, wa.ticket, A, s);
        } else {
            e = launch_walk_init(anchors, wa.prev, wa.ticket, A, d.V, m->ws.status, s);
            for (int k = 0; k < d.gamma && e == cudaSuccess; ++k) {
                wa.step = k;
                KernelTimer t(DSPARK_TIMER_WALK, s, w2b + 4.0 * A * d.V, 2.0 * A * (double)d.V * d.r);
                e = launch_walk_step(m, wa, s);
            }
        }
    }
    if (e == cudaSuccess) e = launch_confidence(m, x.f32, anchors, tokens, A, conf ? conf : at<float>(ws, p.conf), lengths, s);
    if (e != cudaSuccess) DSPARK_FAIL(DSPARK_ERR_CUDA, std::string("draft round launch: ") + cudaGetErrorString(e));
    return DSPARK_OK;
}

int dspark_debug_attention_dump(dspark_model* m, float* dst, size_t bytes) {
    if (!m) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "model is NULL");
    if (dst && (reinterpret_cast<uintptr_t>(dst) & 15u)) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "dst must be 16-byte aligned");
    m->attn_dump = dst;
    m->attn_dump_bytes = dst ? bytes : 0;
    return DSPARK_OK;
}

int dspark_read_device_status(const dspark_model* m, void* stream, int32_t* status) {
    if (!m || !status) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "model and status must be non-NULL");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t v = 0;
    DSPARK_CUDA_CHECK(cudaMemcpyAsync(&v, m->ws.status, sizeof(int32_t), cudaMemcpyDeviceToHost, s));
    DSPARK_CUDA_CHECK(cudaStreamSynchronize(s));
    DSPARK_CUDA_CHECK(cudaMemsetAsync(m->ws.status, 0, sizeof(int32_t), s));
    *status = v;
    return DSPARK_OK;
}

}  // extern "C"
