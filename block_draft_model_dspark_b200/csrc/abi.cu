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
    d.r = c->markov_rank; d.dtype = c->dtype; d.quant = c->quant_bits == 4;
    d.kv_dtype = c->dtype == DSPARK_DTYPE_BF16 ? DSPARK_DTYPE_F16 : DSPARK_DTYPE_F32; d.group = d.quant ? c->quant_group_size : 64;
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
    // 4-bit models: the packed copies the tensor-core GEMM reads (per layer where stacked per layer)
    size_t pk_qk, pk_o, pk_gu, pk_down, pk_lm, pk_k;
    size_t pk_qk_b, pk_o_b, pk_gu_b, pk_down_b;       // bytes of one layer's copy
    // dense bf16 models: fp16 copies of o_proj, down_proj (per layer) and the lm-head (the
    // [q; k] and [gate; up] stacks are fp16 too; the all-layer k_proj stays bf16)
    size_t h_o, h_down, h_lm, h_o_b, h_down_b;
};
ModelLayout model_layout(const Dims& d) {
    ModelLayout L{};
    size_t o = 0;
    auto take = [&](size_t bytes) { size_t at = o; o += align_up(bytes, 256); return at; };
    L.status = take(256);
    L.inv_freq = take(sizeof(double) * (size_t)(d.hd / 2));
    // dense: stacked [q_proj; k_proj], [gate; up] and all layers' k_proj; 4-bit: packed copies instead
    if (!d.quant) {
        L.qk = mat_bytes(d, (int64_t)(d.nH + d.nKv) * d.hd, d.H);
        L.gu = mat_bytes(d, 2 * (int64_t)d.I, d.H);
        L.kall = mat_bytes(d, (int64_t)d.Lyr * d.nKv * d.hd, d.H);
    } else {
        L.pk_qk_b = tc::q4_packed_bytes((int64_t)(d.nH + d.nKv) * d.hd, d.H);
        L.pk_o_b = tc::q4_packed_bytes(d.H, (int64_t)d.nH * d.hd);
        L.pk_gu_b = tc::q4_packed_bytes(2 * (int64_t)d.I, d.H);
        L.pk_down_b = tc::q4_packed_bytes(d.H, d.I);
        L.pk_qk = take(L.pk_qk_b * d.Lyr);
        L.pk_o = take(L.pk_o_b * d.Lyr);
        L.pk_gu = take(L.pk_gu_b * d.Lyr);
        L.pk_down = take(L.pk_down_b * d.Lyr);
        L.pk_lm = take(tc::q4_packed_bytes(d.V, d.H));
        L.pk_k = take(tc::q4_packed_bytes((int64_t)d.Lyr * d.nKv * d.hd, d.H));
    }
    L.wqk = take(L.qk.w * d.Lyr);
    L.wqk_s = take(L.qk.s * d.Lyr);
    L.wqk_b = take(L.qk.s * d.Lyr);
    L.wgu = take(L.gu.w * d.Lyr);
    L.wgu_s = take(L.gu.s * d.Lyr);
    L.wgu_b = take(L.gu.s * d.Lyr);
    L.wk = take(L.kall.w);
    L.wk_s = take(L.kall.s);
    L.wk_b = take(L.kall.s);
    if (!d.quant && d.dtype == DSPARK_DTYPE_BF16) {
        L.h_o_b = align_up((size_t)d.H * d.nH * d.hd * 2, 256);
        L.h_down_b = align_up((size_t)d.H * d.I * 2, 256);
        L.h_o = take(L.h_o_b * d.Lyr);
        L.h_down = take(L.h_down_b * d.Lyr);
        L.h_lm = take((size_t)d.V * d.H * 2);
    }
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
    int attn_tc_grid;    // tensor-core attention: CTAs (0: the CUDA-core split plan)
    size_t attn_items;   // its per-item (first slot, slots) for the merge (ints)
    bool tc;      // tensor-core GEMMs: the inputs are also kept in fp16 (hi)
    bool pairs;   // ... and as the fp16 pair (hi, lo)
    size_t h, x, part, q, kb, vb, attn_out, act, U, part_o, part_ml, prev, ticket, walk_val, walk_idx, walk_keys;
    size_t x_hi, x_lo, ao_hi, ao_lo, act_hi, act_lo, conf, gscr, gscr_bytes, total;
    int n_vt;            // 128-entry vocabulary tiles of the logit statistics
    size_t st_mx, st_arg, st_se, st_lo, st_hi;     // tile statistics [n_vt][M] each
    size_t prune_cnt, prune_fail, prune_list;      // candidate counts [M], fail word, lists [M][kPruneCap]
};

DraftPlan plan_draft(const dspark_model* m, int A, int maxL) {
    const Dims& d = m->d;
    DraftPlan p{};
    p.M = A * d.gamma;
    const int Nqk = (d.nH + d.nKv) * d.hd;
    p.tc = use_tensor_cores(m);
    p.pairs = act_pair(m, p.M);
    const GemmFormat gf = round_gemm_format(m, p.M);
    const size_t part_elems = std::max({gemm_out_elems(m, p.M, Nqk, d.H), gemm_out_elems(m, p.M, d.H, d.nH * d.hd),
                                        gemm_out_elems(m, p.M, 2 * d.I, d.H), gemm_out_elems(m, p.M, d.H, d.I)});
    p.gscr_bytes = std::max({gemm_scratch_bytes(m, p.M, Nqk, d.H, gf),
                             gemm_scratch_bytes(m, p.M, d.H, d.nH * d.hd, gf),
                             gemm_scratch_bytes(m, p.M, 2 * d.I, d.H, gf),
                             gemm_scratch_bytes(m, p.M, d.H, d.I, gf)});
    const int chunk = attention_key_chunk(m, A, maxL);
    p.attn_chunk = chunk;
    p.attn_splits = maxL > 0 ? (maxL + chunk - 1) / chunk : 0;
    p.walk_blocks = walk_persistent_supported(m, A) ? walk_persistent_blocks(m)
                                                    : walk_vocab_blocks(m->num_sms, d.V, d.r, d.dtype, d.quant);
    Carve c;
    const size_t es = esize(d.kv_dtype);
    p.h = c.take((size_t)p.M * d.H * 4);
    p.x = c.take((size_t)p.M * d.H * 4);
    p.part = c.take(part_elems * 4);
    p.q = c.take((size_t)p.M * d.nH * d.hd * es);    // the attention's queries, in the KV dtype
    p.kb = c.take((size_t)p.M * d.nKv * d.hd * es);
    p.vb = c.take((size_t)p.M * d.nKv * d.hd * es);
    p.attn_out = c.take((size_t)p.M * d.nH * d.hd * 4);
    p.act = c.take((size_t)p.M * d.I * 4);
    p.U = c.take((size_t)p.M * d.V * 4);
    if (tc::attention_tc_supported(m)) {
        // one partial slot per CTA of the plan: independent of the context lengths
        p.attn_tc_grid = tc::attention_tc_grid(m, A);
        const size_t slot_f = tc::attention_tc_partial_floats(m, p.attn_tc_grid);
        p.part_o = c.take(slot_f / (d.hd + 2) * d.hd * 4);
        p.part_ml = c.take(slot_f / (d.hd + 2) * 2 * 4);
        p.attn_items = c.take(tc::attention_tc_item_ints(m, A) * 4);
    } else {
        const size_t S1 = (size_t)p.attn_splits + 1;
        p.part_o = c.take((size_t)A * d.nH * S1 * d.gamma * d.hd * 4);
        p.part_ml = c.take((size_t)A * d.nH * S1 * d.gamma * 2 * 4);
        p.attn_items = c.take(0);
    }
    p.prev = c.take((size_t)A * 4);
    p.ticket = c.take(256);
    p.walk_keys = c.take((size_t)d.gamma * A * 8);              // tensor-core walk: per (step, row) maximum
    p.n_vt = (d.V + 127) / 128;
    const size_t st = (size_t)p.n_vt * p.M * 4;
    const bool bounds = d.r > 0;
    p.st_mx = c.take(st);
    p.st_arg = c.take(st);
    p.st_se = c.take(st);
    p.st_lo = c.take(bounds ? st : 0);
    p.st_hi = c.take(bounds ? st : 0);
    p.prune_cnt = c.take((size_t)p.M * 4);
    p.prune_fail = c.take(4);
    p.prune_list = c.take(bounds ? (size_t)p.M * kPruneCap * 4 : 0);
    p.walk_val = c.take((size_t)2 * p.walk_blocks * A * 4);     // two step-parity buffers (persistent walk)
    p.walk_idx = c.take((size_t)2 * p.walk_blocks * A * 4);
    // each fp16 form as one [parts][M][K] block (lo right after hi): the GEMM loads both with one TMA
    const size_t fb = p.tc ? 2 : 0, parts = p.pairs ? 2 : 1;
    p.x_hi = c.take(parts * (size_t)p.M * d.H * fb);
    p.x_lo = p.x_hi + (size_t)p.M * d.H * fb;
    p.ao_hi = c.take(parts * (size_t)p.M * d.nH * d.hd * fb);
    p.ao_lo = p.ao_hi + (size_t)p.M * d.nH * d.hd * fb;
    p.act_hi = c.take(parts * (size_t)p.M * d.I * fb);
    p.act_lo = p.act_hi + (size_t)p.M * d.I * fb;
    p.conf = c.take((size_t)p.M * 4);
    p.gscr = c.take(p.gscr_bytes);
    p.total = c.off;
    return p;
}

constexpr int64_t kProjectChunkRows = 16384;
constexpr int kMaxAppendBatch = 4096;    // cache batch rows an append handles

struct ProjectPlan {
    int64_t chunk_rows;
    size_t nvalid, row0, raw, gscr, gscr_bytes, x16, total;
};
ProjectPlan plan_project(const dspark_model* m, int64_t rows) {
    const Dims& d = m->d;
    ProjectPlan p{};
    rows = std::max<int64_t>(rows, 1);
    p.chunk_rows = std::min<int64_t>(rows, kProjectChunkRows);
    const int N = d.Lyr * d.nKv * d.hd;
    size_t raw = gemm_out_elems(m, (int)p.chunk_rows, N, d.H);
    const GemmFormat pf = project_gemm_format(m);
    p.gscr_bytes = gemm_scratch_bytes(m, (int)p.chunk_rows, N, d.H, pf);
    if (rows % p.chunk_rows) {
        raw = std::max(raw, gemm_out_elems(m, (int)(rows % p.chunk_rows), N, d.H));
        p.gscr_bytes = std::max(p.gscr_bytes, gemm_scratch_bytes(m, (int)(rows % p.chunk_rows), N, d.H, pf));
    }
    Carve c;
    p.nvalid = c.take(kMaxAppendBatch * 4);
    p.row0 = c.take(kMaxAppendBatch * 4);
    p.raw = c.take(raw * 4);
    p.gscr = c.take(p.gscr_bytes);
    p.x16 = c.take(d.quant ? (size_t)p.chunk_rows * d.H * 2 : 0);   // 4-bit models: a chunk's rows in fp16
    p.total = c.off;
    return p;
}

template <typename P> P* at(void* base, size_t off) { return reinterpret_cast<P*>(static_cast<char*>(base) + off); }

// Workspace of the context feature projection: one chunk's GEMM result and its GEMM scratch.
struct FeaturePlan {
    int64_t chunk_rows;
    size_t raw, gscr, gscr_bytes, total;
};
FeaturePlan plan_features(const dspark_model* m, int taps, int64_t rows) {
    const Dims& d = m->d;
    const int K = taps * d.H;
    FeaturePlan p{};
    rows = std::max<int64_t>(rows, 1);
    p.chunk_rows = std::min<int64_t>(rows, kProjectChunkRows);
    const GemmFormat f = feature_gemm_format(m);
    // the larger of the model's GEMM result and the CUDA-core one (a 4-bit fc)
    auto out_elems = [&](int M) { return std::max(gemm_out_elems(m, M, d.H, K), simt_gemm_out_elems(m, M, d.H, K)); };
    size_t raw = out_elems((int)p.chunk_rows);
    p.gscr_bytes = gemm_scratch_bytes(m, (int)p.chunk_rows, d.H, K, f);
    if (rows % p.chunk_rows) {
        raw = std::max(raw, out_elems((int)(rows % p.chunk_rows)));
        p.gscr_bytes = std::max(p.gscr_bytes, gemm_scratch_bytes(m, (int)(rows % p.chunk_rows), d.H, K, f));
    }
    Carve c;
    p.raw = c.take(raw * 4);
    p.gscr = c.take(p.gscr_bytes);
    p.total = c.off;
    return p;
}

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
        cudaError_t e = run_kv_projection(m, X, nr, rp, dst, at<float>(ws, pp.raw), sc, at<void>(ws, pp.x16), s);
        if (e != cudaSuccess) DSPARK_FAIL(DSPARK_ERR_CUDA, std::string("context K/V projection launch: ") + cudaGetErrorString(e));
    }
    return DSPARK_OK;
}

}  // namespace
}  // namespace dspark

using namespace dspark;

extern "C" {

const char* dspark_last_error(void) { return g_error.c_str(); }

int32_t dspark_kv_dtype(const dspark_config* cfg) {
    std::string why;
    if (validate_config(cfg, &why) != DSPARK_OK) return -1;
    return make_dims(cfg).kv_dtype;
}

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
        R.o = make_ref(lw.o_proj, d.H, (int64_t)d.nH * d.hd, q);
        R.down = make_ref(lw.down_proj, d.H, d.I, q);
        if (!q && d.dtype == DSPARK_DTYPE_F32) {
            // fp32: stacked copies for the CUDA-core GEMM
            e = copy_rows(d, mq, qkw, qks, qkb, 0, s);
            if (e == cudaSuccess) e = copy_rows(d, mk, qkw, qks, qkb, (int64_t)d.nH * d.hd, s);
            if (e == cudaSuccess) e = copy_rows(d, mg, guw, gus, gub, 0, s);
            if (e == cudaSuccess) e = copy_rows(d, mu, guw, gus, gub, d.I, s);
            if (e == cudaSuccess)
                e = copy_rows(d, mk, base + L.wk, at<bf16>(base, L.wk_s), at<bf16>(base, L.wk_b), (int64_t)l * d.nKv * d.hd, s);
            R.qk = stacked_ref(d, qkw, qks, qkb, Nqk, d.H);
            R.gu = stacked_ref(d, guw, gus, gub, 2 * (int64_t)d.I, d.H);
        } else if (!q) {
            // bf16: fp16 copies for the tensor-core GEMMs (exact inside fp16's range; a weight
            // outside it fails the model's creation), stacked where the GEMM is; the all-layer
            // k_proj stays bf16 for the context projection of the caller's bf16 rows
            int32_t* ovf = m->ws.status + 1;
            const size_t qrow = (size_t)d.H * 2;
            char* qk16 = static_cast<char*>(qkw);
            char* gu16 = static_cast<char*>(guw);
            void* o16 = base + L.h_o + L.h_o_b * l;
            void* dn16 = base + L.h_down + L.h_down_b * l;
            e = tc::f16_copy(mq.w, mq.n * d.H, qk16, ovf, s);
            if (e == cudaSuccess) e = tc::f16_copy(mk.w, mk.n * d.H, qk16 + (size_t)mq.n * qrow, ovf, s);
            if (e == cudaSuccess) e = tc::f16_copy(mg.w, mg.n * d.H, gu16, ovf, s);
            if (e == cudaSuccess) e = tc::f16_copy(mu.w, mu.n * d.H, gu16 + (size_t)mg.n * qrow, ovf, s);
            if (e == cudaSuccess) e = tc::f16_copy(R.o.w, R.o.n * R.o.k, o16, ovf, s);
            if (e == cudaSuccess) e = tc::f16_copy(R.down.w, R.down.n * R.down.k, dn16, ovf, s);
            if (e == cudaSuccess)
                e = copy_rows(d, mk, base + L.wk, at<bf16>(base, L.wk_s), at<bf16>(base, L.wk_b), (int64_t)l * d.nKv * d.hd, s);
            R.qk = stacked_ref(d, nullptr, nullptr, nullptr, Nqk, d.H);
            R.gu = stacked_ref(d, nullptr, nullptr, nullptr, 2 * (int64_t)d.I, d.H);
            R.qk.w16 = qkw; R.gu.w16 = guw; R.o.w16 = o16; R.down.w16 = dn16;
        } else {
            // the packed copies the tensor-core GEMM streams (stacked where the GEMM is)
            auto piece = [](const MatRef& r, int64_t row0) {
                tc::Q4Piece pc{};
                pc.w = static_cast<const uint32_t*>(r.w); pc.s = r.scales; pc.b = r.biases; pc.row0 = row0; pc.rows = r.n;
                return pc;
            };
            void* pqk = base + L.pk_qk + L.pk_qk_b * l;
            void* po = base + L.pk_o + L.pk_o_b * l;
            void* pgu = base + L.pk_gu + L.pk_gu_b * l;
            void* pdn = base + L.pk_down + L.pk_down_b * l;
            const tc::Q4Piece qk2[2] = {piece(mq, 0), piece(mk, (int64_t)d.nH * d.hd)};
            const tc::Q4Piece gu2[2] = {piece(mg, 0), piece(mu, d.I)};
            const tc::Q4Piece o1 = piece(R.o, 0), d1 = piece(R.down, 0);
            e = tc::q4_pack(qk2, 2, Nqk, d.H, pqk, s);
            if (e == cudaSuccess) e = tc::q4_pack(&o1, 1, d.H, (int64_t)d.nH * d.hd, po, s);
            if (e == cudaSuccess) e = tc::q4_pack(gu2, 2, 2 * (int64_t)d.I, d.H, pgu, s);
            if (e == cudaSuccess) e = tc::q4_pack(&d1, 1, d.H, d.I, pdn, s);
            R.qk = stacked_ref(d, nullptr, nullptr, nullptr, Nqk, d.H);
            R.gu = stacked_ref(d, nullptr, nullptr, nullptr, 2 * (int64_t)d.I, d.H);
            R.qk.packed = pqk; R.gu.packed = pgu; R.o.packed = po; R.down.packed = pdn;
        }
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
    if (!q && d.dtype == DSPARK_DTYPE_BF16) {
        e = tc::f16_copy(m->lm_head.w, (int64_t)d.V * d.H, base + L.h_lm, m->ws.status + 1, s);
        int32_t ovf = 0;
        if (e == cudaSuccess) e = cudaMemcpyAsync(&ovf, m->ws.status + 1, sizeof(int32_t), cudaMemcpyDeviceToHost, s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) {
            delete m;
            DSPARK_FAIL(DSPARK_ERR_CUDA, std::string("fp16 weight copies: ") + cudaGetErrorString(e));
        }
        if (ovf) {
            delete m;
            DSPARK_FAIL(DSPARK_ERR_UNSUPPORTED, "a bf16 weight lies outside fp16's range (|w| > 65504): the tensor-core "
                                                "GEMMs read fp16 copies of the weights");
        }
        m->lm_head.w16 = base + L.h_lm;
    }
    if (q) {
        // packed copies of the lm-head and of all layers' k_proj (one context projection GEMM)
        std::vector<tc::Q4Piece> kp(d.Lyr);
        for (int l = 0; l < d.Lyr; ++l) {
            const MatRef mk = make_ref(w->layers[l].k_proj, (int64_t)d.nKv * d.hd, d.H, q);
            kp[l].w = static_cast<const uint32_t*>(mk.w); kp[l].s = mk.scales; kp[l].b = mk.biases;
            kp[l].row0 = (int64_t)l * d.nKv * d.hd; kp[l].rows = mk.n;
        }
        tc::Q4Piece lm{};
        lm.w = static_cast<const uint32_t*>(m->lm_head.w); lm.s = m->lm_head.scales; lm.b = m->lm_head.biases;
        lm.row0 = 0; lm.rows = d.V;
        e = tc::q4_pack(kp.data(), d.Lyr, (int64_t)d.Lyr * d.nKv * d.hd, d.H, base + L.pk_k, s);
        if (e == cudaSuccess) e = tc::q4_pack(&lm, 1, d.V, d.H, base + L.pk_lm, s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) {
            delete m;
            DSPARK_FAIL(DSPARK_ERR_CUDA, std::string("4-bit weight packing: ") + cudaGetErrorString(e));
        }
        m->wk_all.packed = base + L.pk_k;
        m->lm_head.packed = base + L.pk_lm;
    }
    if (d.r > 0) m->w2 = make_ref(w->markov_w2, d.V, d.r, q);
    if (d.conf_head) m->conf_proj = make_ref(w->confidence_proj, 1, d.conf_in, q);
    m->w1 = w->markov_w1;
    m->final_norm = w->norm;
    m->conf_bias = w->confidence_bias;
    // norm bounds of the pruned walk: once per model, from the weights as given
    if (walk_prune_model_supported(d)) {
        m->ws.w2norm = reinterpret_cast<float*>(base + L.w2norm);
        m->ws.w1max_bits = reinterpret_cast<uint32_t*>(base + L.w1max);
        e = launch_markov_norms(m, s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) {
            delete m;
            DSPARK_FAIL(DSPARK_ERR_CUDA, std::string("markov norm bounds: ") + cudaGetErrorString(e));
        }
    }
    *out = m;
    return DSPARK_OK;
}

int dspark_model_destroy(dspark_model* m) {
    if (!m) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "model is NULL");
    delete m;
    return DSPARK_OK;
}

size_t dspark_project_workspace_bytes(const dspark_model* m, int64_t rows) {
    if (!m || rows < 0) return 0;
    return plan_project(m, rows).total;
}

int dspark_prune_lengths(const float* conf, int32_t A, int32_t gamma, const float* thresholds, int32_t* lengths,
                         void* stream) {
    if (A < 0 || A > (1 << 30)) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "A must be in [0, 2^30]");
    if (gamma < 1) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "gamma must be >= 1");
    if (A == 0) return DSPARK_OK;
    if (!conf || !thresholds || !lengths) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "conf, thresholds and lengths must be non-NULL");
    cudaError_t e = launch_prune_lengths(conf, A, gamma, thresholds, lengths, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) DSPARK_FAIL(DSPARK_ERR_CUDA, std::string("prune lengths launch: ") + cudaGetErrorString(e));
    return DSPARK_OK;
}

size_t dspark_context_features_workspace_bytes(const dspark_model* m, int32_t taps, int64_t rows) {
    if (!m || taps < 1 || rows < 0) return 0;
    return plan_features(m, taps, rows).total;
}

int dspark_project_context_features(const dspark_model* m, const dspark_matrix* fc, const void* hidden_norm,
                                    int32_t taps, const void* target_hiddens, int32_t B, int32_t L, void* out,
                                    void* ws, size_t ws_bytes, void* stream) {
    if (!m || !fc) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "model and fc must be non-NULL");
    const Dims& d = m->d;
    if (taps < 1) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "taps must be >= 1");
    if ((int64_t)taps * d.H > (int64_t)1 << 24) DSPARK_FAIL(DSPARK_ERR_UNSUPPORTED, "taps * hidden above 2^24");
    const bool q4 = fc->scales || fc->biases;          // a 4-bit affine fc
    if (q4 && !(fc->scales && fc->biases)) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "a 4-bit fc needs both scales and biases");
    if (q4 && ((int64_t)taps * d.H) % d.group != 0)
        DSPARK_FAIL(DSPARK_ERR_UNSUPPORTED, "taps * hidden must be a multiple of the quantization group");
    if (B < 0 || L < 0) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "B and L must be >= 0");
    if ((int64_t)B * L == 0) return DSPARK_OK;
    if ((int64_t)B * L > (int64_t)1 << 30) DSPARK_FAIL(DSPARK_ERR_UNSUPPORTED, "B * L above 2^30 rows");
    if (!fc->w || !hidden_norm || !target_hiddens || !out || !ws)
        DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "fc.w, hidden_norm, target_hiddens, out and ws must be non-NULL");
    if (!aligned16(fc->w) || !aligned16(target_hiddens) || !aligned16(out) || !aligned16(ws))
        DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "fc.w, target_hiddens, out and ws must be 16-byte aligned");
    const int K = taps * d.H;
    if (use_tensor_cores(m) && K % 64 != 0) DSPARK_FAIL(DSPARK_ERR_UNSUPPORTED, "taps * hidden must be a multiple of 64");
    const int64_t rows = (int64_t)B * L;
    const FeaturePlan pp = plan_features(m, taps, rows);
    if (ws_bytes < pp.total)
        DSPARK_FAIL(DSPARK_ERR_WORKSPACE, "ws smaller than dspark_context_features_workspace_bytes(): " + std::to_string(pp.total));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    MatRef fr;
    fr.w = fc->w; fr.n = d.H; fr.k = K; fr.quant = q4;
    fr.scales = static_cast<const bf16*>(fc->scales); fr.biases = static_cast<const bf16*>(fc->biases);
    const size_t es = esize(d.dtype);
    const GemmScratch sc = gemm_scratch_at(at<void>(ws, pp.gscr), pp.gscr_bytes);
    for (int64_t r0 = 0; r0 < rows; r0 += pp.chunk_rows) {
        const int nr = (int)std::min<int64_t>(pp.chunk_rows, rows - r0);
        const void* X = static_cast<const char*>(target_hiddens) + (size_t)r0 * K * es;
        PartView view;
        cudaError_t e = run_context_features(m, X, nr, fr, at<float>(ws, pp.raw), sc, &view, s);
        if (e == cudaSuccess)
            e = launch_context_norm(m, view, nr, hidden_norm, static_cast<char*>(out) + (size_t)r0 * d.H * es, s);
        if (e != cudaSuccess) DSPARK_FAIL(DSPARK_ERR_CUDA, std::string("context feature projection launch: ") + cudaGetErrorString(e));
    }
    return DSPARK_OK;
}

int dspark_project_context_kv(const dspark_model* m, const void* hidden, int32_t B, int32_t L, int32_t static_pos,
                              const int32_t* pos0, void* k_out, void* v_out, void* ws, size_t ws_bytes, void* stream) {
    if (!m) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "model is NULL");
    if (B < 0 || L < 0) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "B and L must be >= 0");
    if ((int64_t)B * L == 0) return DSPARK_OK;
    if ((int64_t)B * L > (int64_t)1 << 30) DSPARK_FAIL(DSPARK_ERR_UNSUPPORTED, "B * L above 2^30 rows");
    if (!hidden || !v_out || !ws) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "hidden, v_out and ws must be non-NULL");
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
    if (!n_new || !pos0 || !cache->len || !cache->v)
        DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "n_new, pos0 and the cache's v, len must be non-NULL");
    if (!cache->k && !tc::vonly_attention_supported(m))
        DSPARK_FAIL(DSPARK_ERR_UNSUPPORTED, "a V-only cache (k = NULL) needs the tensor-core attention (bf16 model)");
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

// allow_vonly: the call can read a V-only cache (k = NULL, K rebuilt from v at pos0[b] + t)
static int check_cache(const dspark_model* m, const dspark_kv_cache* c, int A, int maxL, std::string* why,
                       bool allow_vonly) {
    if (!c || !c->v || !c->len) { *why = "cache and its v, len must be non-NULL"; return DSPARK_ERR_INVALID_ARGUMENT; }
    if (!c->k) {
        if (!allow_vonly) { *why = "the attend seam takes explicit keys: a V-only cache (k = NULL) is refused"; return DSPARK_ERR_INVALID_ARGUMENT; }
        if (!tc::vonly_attention_supported(m)) {
            *why = "a V-only cache (k = NULL) needs the tensor-core attention (bf16 model)";
            return DSPARK_ERR_UNSUPPORTED;
        }
        if (!c->pos0) { *why = "a V-only cache (k = NULL) needs pos0"; return DSPARK_ERR_INVALID_ARGUMENT; }
    }
    if (A <= 0 || A > c->batch) { *why = "A must be in [1, cache.batch]"; return DSPARK_ERR_INVALID_ARGUMENT; }
    if (maxL < 0 || maxL > c->capacity) { *why = "max_ctx_len must be in [0, cache.capacity]"; return DSPARK_ERR_INVALID_ARGUMENT; }
    if (!aligned16(c->k) || !aligned16(c->v)) { *why = "cache k / v must be 16-byte aligned"; return DSPARK_ERR_INVALID_ARGUMENT; }
    return DSPARK_OK;
}

static AttnArgs attn_args(const dspark_model* m, const DraftPlan& p, void* ws, const dspark_kv_cache* c, int layer, int A,
                          const void* q, const void* kb, const void* vb, void* out, int q_dtype, int out_dtype) {
    const Dims& d = m->d;
    const size_t es = esize(d.kv_dtype);
    const size_t layer_bytes = (size_t)c->batch * c->capacity * d.nKv * d.hd * es;
    AttnArgs a{};
    a.q = q; a.kb = kb; a.vb = vb; a.out = out;
    a.q_dtype = q_dtype; a.out_dtype = out_dtype;
    a.kc = c->k ? static_cast<const char*>(c->k) + layer_bytes * layer : nullptr;   // NULL: V-only
    a.vc = static_cast<const char*>(c->v) + layer_bytes * layer;
    a.len = c->len; a.capacity = c->capacity; a.batch = c->batch;
    a.part_o = at<float>(ws, p.part_o); a.part_ml = at<float>(ws, p.part_ml);
    a.item_slots = p.attn_tc_grid ? at<int>(ws, p.attn_items) : nullptr; a.tc_grid = p.attn_tc_grid;
    a.A = A; a.n_splits = p.attn_splits; a.chunk = p.attn_chunk;
    a.status = m->ws.status;
    // algorithmic work: every valid context row's K and V once, the block K/V, q and out
    double keys = (double)A * d.gamma;
    if (c->len_host)
        for (int b = 0; b < A; ++b) keys += c->len_host[b];
    else
        keys += (double)A * c->capacity;
    const double qo = (double)A * d.gamma * d.nH * d.hd * (esize(q_dtype) + esize(out_dtype));
    a.kv_bytes = keys * d.nKv * d.hd * (c->k ? 2.0 : 1.0) * es + qo;   // a V-only cache streams v alone
    a.flops = 4.0 * (double)d.nH * d.gamma * d.hd * keys;
    return a;
}

int dspark_attend(const dspark_model* m, int32_t layer, const dspark_kv_cache* cache, const void* q, const void* k_blk,
                  const void* v_blk, void* out, int32_t A, int32_t max_ctx_len, void* ws, size_t ws_bytes, void* stream) {
    if (!m) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "model is NULL");
    std::string why;
    int rc = check_cache(m, cache, A, max_ctx_len, &why, false);
    if (rc) DSPARK_FAIL(rc, why);
    if (layer < 0 || layer >= m->d.Lyr) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "layer out of range");
    if (!q || !k_blk || !v_blk || !out || !ws) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "q, k_blk, v_blk, out and ws must be non-NULL");
    if (!aligned16(q) || !aligned16(k_blk) || !aligned16(v_blk) || !aligned16(out) || !aligned16(ws))
        DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "q, k_blk, v_blk, out and ws must be 16-byte aligned");
    const DraftPlan p = plan_draft(m, A, max_ctx_len);
    if (ws_bytes < p.total) DSPARK_FAIL(DSPARK_ERR_WORKSPACE, "ws smaller than dspark_draft_workspace_bytes(): " + std::to_string(p.total));
    const AttnArgs a = attn_args(m, p, ws, cache, layer, A, q, k_blk, v_blk, out, m->d.kv_dtype, m->d.kv_dtype);
    cudaError_t e = run_attention(m, a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) DSPARK_FAIL(DSPARK_ERR_CUDA, std::string("attention launch: ") + cudaGetErrorString(e));
    return DSPARK_OK;
}

int dspark_draft_rows(const dspark_model* m, const dspark_kv_cache* cache, const int32_t* anchors,
                      const int32_t* block_pos, int32_t A, int32_t max_ctx_len, int32_t* tokens, float* conf,
                      int32_t* lengths, float* base_logits, void* ws, size_t ws_bytes, void* stream) {
    if (!m) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "model is NULL");
    std::string why;
    int rc = check_cache(m, cache, A, max_ctx_len, &why, true);
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
    if (m->logit_dump && m->logit_dump_bytes < (size_t)A * d.gamma * sizeof(LogitRowStat))
        DSPARK_FAIL(DSPARK_ERR_WORKSPACE, "logit statistics dump smaller than A * gamma * 16 bytes");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int M = p.M;
    float* h = at<float>(ws, p.h);
    float* part = at<float>(ws, p.part);
    void* q = at<void>(ws, p.q); void* kb = at<void>(ws, p.kb); void* vb = at<void>(ws, p.vb);
    float* U = base_logits ? base_logits : at<float>(ws, p.U);
    ActBuf x, ao, act;
    x.f32 = at<float>(ws, p.x); ao.f32 = at<float>(ws, p.attn_out); act.f32 = at<float>(ws, p.act);
    if (p.tc) {
        x.hi = at<__half>(ws, p.x_hi); ao.hi = at<__half>(ws, p.ao_hi); act.hi = at<__half>(ws, p.act_hi);
    }
    if (p.pairs) {
        x.lo = at<__half>(ws, p.x_lo); ao.lo = at<__half>(ws, p.ao_lo); act.lo = at<__half>(ws, p.act_lo);
    }
    const int Nqk = (d.nH + d.nKv) * d.hd;
    PartView pv;
    const GemmScratch sc = gemm_scratch_at(at<void>(ws, p.gscr), p.gscr_bytes);
    // the persistent walk's grid-barrier counter
    cudaError_t e = cudaMemsetAsync(at<uint32_t>(ws, p.ticket), 0, sizeof(uint32_t), s);
    if (e == cudaSuccess) e = cudaMemsetAsync(at<void>(ws, p.walk_keys), 0, (size_t)d.gamma * A * 8, s);
    ActBuf x_emb = x;
    if (p.tc) x_emb.f32 = nullptr;                  // the first layer's GEMM reads the fp16 form
    if (e == cudaSuccess) e = launch_embed(m, anchors, A, h, x_emb, m->ws.status, s);
    for (int l = 0; l < d.Lyr && e == cudaSuccess; ++l) {
        const LayerRef& L = m->layers[l];
        e = run_gemm(m, x, L.qk, M, Nqk, d.H, part, sc, &pv, DSPARK_TIMER_GEMM_QK, s);
        if (e == cudaSuccess) e = launch_qk_epilogue(m, l, pv, A, block_pos, q, kb, vb, s);
        if (e == cudaSuccess) {
            AttnArgs a = attn_args(m, p, ws, cache, l, A, q, kb, vb, ao.f32, d.kv_dtype, DSPARK_DTYPE_F32);
            a.out_hi = ao.hi; a.out_lo = ao.lo;
            a.pos0 = cache->pos0; a.block_pos = block_pos; a.k_norm = L.k_norm;
            if (p.tc && !m->attn_dump) a.out = nullptr;    // the o GEMM reads the fp16 form only
            e = run_attention(m, a, s);
        }
        if (e == cudaSuccess && m->attn_dump)
            e = cudaMemcpyAsync(reinterpret_cast<char*>(m->attn_dump) + dump_layer * l, ao.f32, dump_layer,
                                cudaMemcpyDeviceToDevice, s);
        if (e == cudaSuccess) e = run_gemm(m, ao, L.o, M, d.H, d.nH * d.hd, part, sc, &pv, DSPARK_TIMER_GEMM_O, s);
        // on tensor cores the next GEMM reads only the fp16 forms: the fp32 ones are
        // written only for the last layer's normed hidden (the confidence head reads it)
        ActBuf x_out = x, act_out = act;
        if (p.tc) act_out.f32 = nullptr;
        if (p.tc && l + 1 < d.Lyr) x_out.f32 = nullptr;
        ActBuf x_mid = x;
        if (p.tc) x_mid.f32 = nullptr;
        if (e == cudaSuccess) e = launch_o_epilogue(m, l, pv, M, h, x_mid, s);
        if (e == cudaSuccess) e = run_gemm(m, x, L.gu, M, 2 * d.I, d.H, part, sc, &pv, DSPARK_TIMER_GEMM_GU, s);
        if (e == cudaSuccess) e = launch_gu_epilogue(m, pv, M, act_out, s);
        if (e == cudaSuccess) e = run_gemm(m, act, L.down, M, d.H, d.I, part, sc, &pv, DSPARK_TIMER_GEMM_DOWN, s);
        if (e == cudaSuccess) e = launch_down_epilogue(m, l, pv, M, h, x_out, s);
    }
    TileStats ts;
    ts.mx = at<float>(ws, p.st_mx); ts.arg = at<int>(ws, p.st_arg); ts.se = at<float>(ws, p.st_se);
    if (d.r > 0) { ts.lo = at<float>(ws, p.st_lo); ts.hi = at<float>(ws, p.st_hi); }
    ts.M = M; ts.n_tiles = p.n_vt;
    if (e == cudaSuccess) e = run_lm_head(m, x, M, U, ts, s);
    if (e == cudaSuccess) {
        // exact pruning: candidate lists from the tile statistics, then the walk over them
        PruneScratch ps;
        ps.cnt = at<int>(ws, p.prune_cnt); ps.fail = at<int>(ws, p.prune_fail); ps.list = at<int>(ws, p.prune_list);
        LogitRowStat* row_out = static_cast<LogitRowStat*>(m->logit_dump);
        {
            // algorithmic bytes: the tile statistics (the candidate tiles' U rows depend on the data)
            KernelTimer t(DSPARK_TIMER_WALK, s, (double)p.n_vt * M * (d.r > 0 ? 20.0 : 12.0), 0.0);
            e = launch_walk_prune(m, U, ts, anchors, tokens, A, ps, row_out, s);
        }
        if (e == cudaSuccess && d.r > 0) {
            // the full walk runs only when a candidate list overflowed (it returns at once
            // otherwise), so its work is not counted
            const int* skip = ps.fail;
            KernelTimer t(DSPARK_TIMER_WALK, s, 0.0, 0.0);
            WalkArgs wa{};
            wa.U = U; wa.tokens = tokens; wa.prev = at<int32_t>(ws, p.prev);
            wa.part_val = at<float>(ws, p.walk_val); wa.part_idx = at<int32_t>(ws, p.walk_idx);
            wa.ticket = at<uint32_t>(ws, p.ticket); wa.A = A; wa.nblk = p.walk_blocks; wa.status = m->ws.status;
            wa.skip = skip;
            if (tc::walk_tc_supported(m, A)) {
                e = tc::launch_walk_tc(m, U, anchors, tokens, at<unsigned long long>(ws, p.walk_keys), wa.ticket, skip,
                                       A, s);
            } else if (walk_persistent_supported(m, A)) {
                e = launch_walk_persistent(m, U, anchors, tokens, wa.part_val, wa.part_idx, wa.ticket, skip, A, s);
            } else {
                e = launch_walk_init(anchors, wa.prev, wa.ticket, A, d.V, m->ws.status, skip, s);
                for (int k = 0; k < d.gamma && e == cudaSuccess; ++k) {
                    wa.step = k;
                    e = launch_walk_step(m, wa, s);
                }
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

int dspark_debug_logit_stats(dspark_model* m, void* dst, size_t bytes) {
    if (!m) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "model is NULL");
    if (dst && (reinterpret_cast<uintptr_t>(dst) & 15u)) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "dst must be 16-byte aligned");
    m->logit_dump = dst;
    m->logit_dump_bytes = dst ? bytes : 0;
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
