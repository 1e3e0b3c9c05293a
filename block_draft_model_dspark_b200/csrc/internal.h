// Internal declarations of libdspark (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>
#include <stddef.h>
#include <string>
#include <vector>

#include "../../include/dspark.h"
#include "gemm_tc.h"
#include "logit_stats.cuh"

namespace dspark {

using bf16 = __nv_bfloat16;

// ---------------------------------------------------------------- errors
void set_error(const std::string& msg);
#define DSPARK_FAIL(code, msg)                 \
    do {                                       \
        ::dspark::set_error(msg);              \
        return (code);                         \
    } while (0)
#define DSPARK_CUDA_CHECK(expr)                                                           \
    do {                                                                                  \
        cudaError_t e_ = (expr);                                                          \
        if (e_ != cudaSuccess)                                                            \
            DSPARK_FAIL(DSPARK_ERR_CUDA, std::string(#expr) + ": " + cudaGetErrorString(e_)); \
    } while (0)

// A weight matrix as the kernels see it: dense T [n, k] (row stride k), or
// affine 4-bit words [n, k/8] + bf16 scales/biases [n, k/group].
struct MatRef {
    const void* w = nullptr;
    const bf16* scales = nullptr;
    const bf16* biases = nullptr;
    int64_t n = 0, k = 0;
    bool quant = false;
    const void* packed = nullptr;   // 4-bit GEMM weights: the packed copy the tensor-core GEMM reads
    const void* w16 = nullptr;      // dense bf16 GEMM weights: the fp16 copy the tensor-core GEMM reads
};

// Device layout of everything dspark_model_create places in model_ws.
struct ModelWs {
    int32_t* status = nullptr;      // device status word (+ padding; status[1]: fp16-copy overflow flag)
    double* inv_freq = nullptr;     // [hd/2] RoPE inverse frequencies (0 = identity lane)
    void* wqk = nullptr;            // per layer [(nH+nKv)*hd, H] (dense) or words
    void* wgu = nullptr;            // per layer [2I, H]
    void* wk_all = nullptr;         // [Lyr*nKv*hd, H]
    bf16* wqk_s = nullptr; bf16* wqk_b = nullptr;   // quantized scales / biases of the stacks
    bf16* wgu_s = nullptr; bf16* wgu_b = nullptr;
    bf16* wk_all_s = nullptr; bf16* wk_all_b = nullptr;
    float* w2norm = nullptr;        // [V] |markov_w2[v]| upper bounds (pruned walk; NULL when not eligible)
    uint32_t* w1max_bits = nullptr; // max_p |markov_w1[p]| upper bound, as float bits
};

constexpr int kMaxPartials = 8;    // partials a consumer keeps in flight per element

// A GEMM result as its consumers read it. mode 0: out[m][n] is the sum, in
// slice order, of S split-K slices [S][M][ld] (S = 1: a plain result).
// mode 1: the tensor-core GEMM's stream-K partial tiles [tile][P][BN][128]
// (tile = (n / 128) * n_mt + m / BN); the tile's cnt partials come from
// consecutive CTAs and are summed in CTA order. load() issues every partial
// load of one element, finish() adds them: callers load all their elements
// first, so one round of memory latency covers a row.
struct PartView {
    const float* p = nullptr;
    int mode = 0;
    int S = 1; int64_t stride = 0, ld = 0;     // mode 0
    int BN = 16, n_mt = 1, kb = 1, P = 1;      // mode 1
    int T = 1, G = 1;                          // mode 1: stream-K partition (K blocks, CTAs)
    int wide = 0;                              // mode 1: T * G needs 64-bit arithmetic
    int pair = 0;                              // mode 1: CTA-pair tiles (256 weight rows, two 128-row halves)
    // mode 1: division by T as a multiply (Granlund-Montgomery round-up method):
    // x / T = (t + ((x - t) >> sh1)) >> sh2 with t = umulhi(x, magic), exact for every
    // 32-bit x (set_divisor)
    uint32_t magic = 1; int sh1 = 0, sh2 = 0;
    void set_divisor(uint32_t d) {
        int l = 0;
        while (l < 32 && ((uint64_t)1 << l) < d) ++l;
        magic = (uint32_t)((((uint64_t)1 << 32) * (((uint64_t)1 << l) - d)) / d + 1);
        sh1 = l < 1 ? l : 1;
        sh2 = l > 1 ? l - 1 : 0;
    }
    struct Pending {
        float x[kMaxPartials];
        int cnt;
        const float* rest;                     // partials beyond kMaxPartials (rare)
    };
    // the CTA whose K range holds global K block g (32-bit division unless T * G >= 2^32)
    __device__ __forceinline__ int cta_of(int g) const {
        if (wide) return (int)((((int64_t)g + 1) * G - 1) / T);
        const uint32_t x = ((uint32_t)g + 1u) * (uint32_t)G - 1u;
        const uint32_t t = __umulhi(x, magic);
        return (int)((t + ((x - t) >> sh1)) >> sh2);
    }
    __device__ __forceinline__ Pending load(int64_t m, int64_t n) const {
        Pending q;
        if (mode == 0) {
#pragma unroll
            for (int s = 0; s < kMaxPartials; ++s) q.x[s] = s < S ? p[s * stride + m * ld + n] : 0.f;
            q.cnt = S; q.rest = p + m * ld + n;
            return q;
        }
        const int mi = (int)m, ni = (int)n;
        const int mt = mi / BN, ml = mi - mt * BN, nt = ni >> 7, nl = ni & 127;
        const int tile = (pair ? nt >> 1 : nt) * n_mt + mt;      // the work unit's tile
        const int store = pair ? 2 * tile + (nt & 1) : tile;     // its 128-row half
        q.cnt = cta_of(tile * kb + kb - 1) - cta_of(tile * kb) + 1;
        const float* base = p + (((int64_t)store * P) * BN + ml) * 128 + nl;
#pragma unroll
        for (int s = 0; s < kMaxPartials; ++s) q.x[s] = s < q.cnt ? base[(int64_t)s * BN * 128] : 0.f;
        q.rest = base;
        return q;
    }
    __device__ __forceinline__ float finish(const Pending& q) const {
        float v = q.x[0];
#pragma unroll
        for (int s = 1; s < kMaxPartials; ++s) v += q.x[s];      // in slot order; absent slots are +0
        const int64_t step = mode == 0 ? stride : (int64_t)BN * 128;
        for (int s = kMaxPartials; s < q.cnt; ++s) v += q.rest[s * step];
        return v;
    }
    __device__ __forceinline__ float sum(int64_t m, int64_t n) const { return finish(load(m, n)); }

    // Four consecutive columns n .. n + 3 of row m (n % 4 == 0; mode 1: within one
    // 128-column block, so they share a tile), each the sum of its partials in order.
    // KMAX: partials load4 keeps in flight (more are read in finish4); a kernel with
    // few columns per thread and many partials per tile raises it, one with many
    // columns lowers it to keep its registers.
    template <int KMAX>
    struct Pending4T {
        float4 x[KMAX];
        int cnt;
        const float* rest;
        int64_t step;
    };
    static constexpr int kMax4 = 4;
    using Pending4 = Pending4T<kMax4>;
    template <int KMAX = kMax4>
    __device__ __forceinline__ Pending4T<KMAX> load4(int m, int64_t n) const {
        Pending4T<KMAX> q;
        const float* base;
        if (mode == 0) {
            q.cnt = S; q.step = stride;
            base = p + (int64_t)m * ld + n;
        } else {
            const int mt = m / BN, ml = m - mt * BN, nt = (int)(n >> 7), nl = (int)(n & 127);
            const int tile = (pair ? nt >> 1 : nt) * n_mt + mt;
            const int store = pair ? 2 * tile + (nt & 1) : tile;
            q.cnt = cta_of(tile * kb + kb - 1) - cta_of(tile * kb) + 1;
            q.step = (int64_t)BN * 128;
            base = p + (((int64_t)store * P) * BN + ml) * 128 + nl;
        }
#pragma unroll
        for (int s = 0; s < KMAX; ++s)
            q.x[s] = s < q.cnt ? *reinterpret_cast<const float4*>(base + s * q.step) : make_float4(0.f, 0.f, 0.f, 0.f);
        q.rest = base;
        return q;
    }
    template <int KMAX>
    __device__ __forceinline__ float4 finish4(const Pending4T<KMAX>& q) const {
        float4 v = q.x[0];
#pragma unroll
        for (int s = 1; s < KMAX; ++s) { v.x += q.x[s].x; v.y += q.x[s].y; v.z += q.x[s].z; v.w += q.x[s].w; }
        for (int s = KMAX; s < q.cnt; ++s) {
            const float4 t = *reinterpret_cast<const float4*>(q.rest + s * q.step);
            v.x += t.x; v.y += t.y; v.z += t.z; v.w += t.w;
        }
        return v;
    }
};

// An fp32 activation and the fp16 form its tensor-core GEMM reads: hi =
// fp16(x), and for the pair form also lo = fp16(x - hi) (dense weights at up
// to 128 activation rows, where both parts go through one MMA and the pair
// costs nothing); with more rows (the MMAs bound the GEMM) and with 4-bit
// weights, hi alone. hi and lo are one [2][M][K] block (lo right after hi).
struct ActBuf {
    float* f32 = nullptr;
    __half* hi = nullptr;
    __half* lo = nullptr;
};

constexpr int kMaxLayers = 64;
struct LayerPtrs { const void* p[kMaxLayers]; };

struct LayerRef {
    MatRef qk, o, gu, down;   // qk = [Wq; Wk], gu = [Wg; Wu]
    const void *q_norm, *k_norm, *in_norm, *post_attn_norm, *pre_ff_norm, *post_ff_norm, *layer_scalar;
};

struct Dims {
    int H, Lyr, nH, nKv, hd, grp, I, V, gamma, mask_id, r;
    int dtype;          // DSPARK_DTYPE_* of the weights and gains
    int kv_dtype;       // DSPARK_DTYPE_* of the context and block K/V (fp16 for bf16 models)
    bool quant;
    int group;
    float eps, cap, conf_thr;
    bool conf_head, conf_markov;
    int conf_in;        // H (+ r)
};

}  // namespace dspark

struct dspark_model {
    dspark_config cfg;
    dspark::Dims d;
    dspark::ModelWs ws;
    std::vector<dspark::LayerRef> layers;
    dspark::MatRef embed, lm_head, w2, conf_proj, wk_all;
    const void* w1 = nullptr;
    const void* final_norm = nullptr;
    const void* conf_bias = nullptr;
    int device = 0;
    int num_sms = 148;
    float* attn_dump = nullptr;      // test-facing per-layer attention dump (dspark_debug_attention_dump)
    size_t attn_dump_bytes = 0;
    void* logit_dump = nullptr;      // test-facing per-position logit statistics (dspark_debug_logit_stats)
    size_t logit_dump_bytes = 0;
};

namespace dspark {

// ---------------------------------------------------------------- launch helpers
// Each returns cudaGetLastError() of its launch.

// SIMT GEMM: out[z][m][n] = sum_{k in split z} X[m,k] * W[n,k]  (fp32 partials),
// or with softcap (splits must be 1): out[m][n] = cap*tanh(acc/cap) (cap > 0) or acc.
cudaError_t launch_simt_gemm(const void* X, int64_t ldx, int x_dtype, int w_dtype, const MatRef& W, int group,
                             int M, int N, int K, int splits, float* out, int64_t ldo, int64_t split_stride,
                             bool softcap, float cap, cudaStream_t s);

// Context K/V epilogue: the K/V GEMM's result [rows, Lyr*nKv*hd] -> cache rows.
// Row r = b*Lrows + t is valid when t < n_b.
struct KvDest {
    void* k; void* v;        // k NULL: a V-only cache (v written alone)
    int64_t batch_stride;    // elements between batch rows   (= cap * nKv * hd)
    int64_t layer_stride;    // elements between layers       (= batch * cap * nKv * hd)
    int capacity;
};
struct RowsPlan {
    int B, Lrows;            // rows are b*Lrows + t
    int row0;                // first global row index (b*Lrows+t) held by this chunk
    int nrows;               // rows in this chunk
    const int32_t* n_valid;  // device [B] or null (all Lrows valid)
    const int32_t* dst_row0; // device [B] cache row of t = 0, or null (0)
    const int32_t* pos0;     // device [B] position of t = 0, or null (static_pos)
    int static_pos;
};
// Alg 1 draft-length pruning: lengths[b] = first k >= 1 with conf[b, k] < thr[k], else gamma.
cudaError_t launch_prune_lengths(const float* conf, int A, int gamma, const float* thr, int32_t* lengths,
                                 cudaStream_t s);
// Context features (deepspec.ts #projectContext): out[r] = rms(raw[r], gain) for `nrows` rows of H,
// in the model's dtype.
cudaError_t launch_context_norm(const dspark_model* m, const PartView& raw, int nrows, const void* gain, void* out,
                                cudaStream_t s);
cudaError_t launch_kv_epilogue(const dspark_model* m, const PartView& raw, const RowsPlan& rp, const KvDest& dst,
                               cudaStream_t s);
// Validates an append's device counts (0 <= n_new[b] <= Lnew_max, len[b] + n_new[b] <= capacity);
// writes the counts to use (all 0 when any row fails, with DSPARK_DEV_CAPACITY set) and a
// snapshot of len as each row's first destination row.
cudaError_t launch_append_check(const int32_t* n_new, const int32_t* len, int B, int Lnew_max, int capacity,
                                int32_t* nvalid, int32_t* row0, int32_t* status, cudaStream_t s);
cudaError_t launch_commit_len(int32_t* len, const int32_t* n_new, int B, cudaStream_t s);

// Activations of the round (x, q, attention output, gelu*up) are fp32 in the
// workspace for both model dtypes; only the K/V cache and the block K/V are
// stored in the model dtype.
// Block embedding: h = embed[ids]*sqrt(H) (fp32 [M,H]); x = rms(h, w_in0) (fp32 [M,H]).
cudaError_t launch_embed(const dspark_model* m, const int32_t* anchors, int A, float* h, const ActBuf& x,
                         int32_t* status, cudaStream_t s);
// q and block k/v heads (all in the KV dtype) from the [Wq;Wk] GEMM partials.
cudaError_t launch_qk_epilogue(const dspark_model* m, int layer, const PartView& part, int A,
                               const int32_t* block_pos, void* q, void* kb, void* vb, cudaStream_t s);
// h += rms(o_proj partials, post_attn); x = rms(h, pre_ff).
cudaError_t launch_o_epilogue(const dspark_model* m, int layer, const PartView& part, int M, float* h,
                              const ActBuf& x, cudaStream_t s);
// act = gelu_tanh(g) * u  (fp32 [M, I]).
cudaError_t launch_gu_epilogue(const dspark_model* m, const PartView& part, int M, const ActBuf& act,
                               cudaStream_t s);
// h = (h + rms(down partials, post_ff)) * layer_scalar; then x = rms(h, next gain)
// (next gain = next layer's input norm, or the final norm).
cudaError_t launch_down_epilogue(const dspark_model* m, int layer, const PartView& part, int M, float* h,
                                 const ActBuf& x, cudaStream_t s);

// Attention: partial pass over context chunks + block keys, then merge.
struct AttnArgs {
    const void* q;  const void* kb; const void* vb;  // [A, G, nH, hd] / [A, G, nKv, hd]
    int q_dtype, out_dtype;                          // DSPARK_DTYPE_* of q and out (kb, vb, cache: the KV dtype)
    const void* kc; const void* vc;                  // cache of this layer: [batch, cap, nKv, hd]
    const int32_t* len; int capacity, batch;         // cache lengths [batch], capacity, batch rows
    void* out;                                       // [A, G, nH, hd]
    __half* out_hi; __half* out_lo;                  // optional fp16 form of out (fp32 out only; lo may be NULL)
    float* part_o; float* part_ml;                   // workspace
    int* item_slots; int tc_grid;                    // tensor cores: per-item (first slot, slots) and the CTAs
    int A, n_splits, chunk;                          // CUDA cores: context splits of `chunk` keys
    int S1;                                          // partial slots per (b, h): set by the kernel path
    int32_t* status;
    double kv_bytes, flops;                          // algorithmic work (for the timers)
    // V-only cache (kc == NULL): K rebuilt in the kernel as rope(v * k_norm) at the
    // positions pos0[b] + t (context row t) and block_pos[b] + i (block row i)
    const int32_t* pos0; const int32_t* block_pos;
    const void* k_norm;                              // this layer's k_norm gain [hd]
};

// Markov walk step k: tokens[:,k] from U[:,k,:] + w2 . w1[prev]; prev updated.
struct WalkArgs {
    const float* U;            // [A, G, V]
    int32_t* tokens;           // [A, G]
    int32_t* prev;             // [A]
    float* part_val; int32_t* part_idx;  // [nblk, A]
    uint32_t* ticket;          // one counter, zero at entry
    int A, nblk, step;
    int32_t* status;
    const int* skip;           // non-NULL: the step returns at once when *skip == 0
};
cudaError_t launch_walk_step(const dspark_model* m, const WalkArgs& a, cudaStream_t s);
// The whole walk in one cooperative launch (one CTA per SM, bounded grid barriers).
namespace tc {
// Markov walk with the bias on tensor cores (walk_tc.cu). With `skip` non-NULL the
// kernel returns at once when *skip == 0 (the pruned walk already wrote the tokens).
bool walk_tc_supported(const dspark_model* m, int A);
cudaError_t launch_walk_tc(const dspark_model* m, const float* U, const int32_t* anchors, int32_t* tokens,
                           unsigned long long* keys, uint32_t* arrivals, const int* skip, int A, cudaStream_t s);
}  // namespace tc
// Exact pruning of the walk (walk_prune.cu): candidate lists from norm bounds and the
// lm-head's tile statistics, then the walk over the candidates; *fail = 1 hands the
// round to the full walk.
constexpr int kPruneCap = 1024;     // candidates a position may keep
struct PruneScratch {
    int* cnt = nullptr;             // [M] candidate counts
    int* fail = nullptr;            // one word (cleared by the candidate kernel)
    int* list = nullptr;            // [M][kPruneCap]
};
// Per-position logit telemetry (dspark_debug_logit_stats): 16 bytes.
struct LogitRowStat {
    float max;
    float lse;
    int32_t argmax;
    int32_t candidates;
};
bool walk_prune_model_supported(const Dims& d);
cudaError_t launch_markov_norms(const dspark_model* m, cudaStream_t s);
// The tile statistics of U by a scan (lm-heads that do not produce them in their epilogue).
cudaError_t launch_tile_stats(const dspark_model* m, const float* U, int M, const TileStats& ts, cudaStream_t s);
// Candidate lists (and with markov_rank 0 the tokens), then the pruned walk.
cudaError_t launch_walk_prune(const dspark_model* m, const float* U, const TileStats& ts, const int32_t* anchors,
                              int32_t* tokens, int A, const PruneScratch& ps, LogitRowStat* row_out, cudaStream_t s);
bool walk_persistent_supported(const dspark_model* m, int A);
int walk_persistent_blocks(const dspark_model* m);
// With `skip` non-NULL the kernel returns at once when *skip == 0 (the pruned walk wrote the tokens).
cudaError_t launch_walk_persistent(const dspark_model* m, const float* U, const int32_t* anchors, int32_t* tokens,
                                   float* cand_val, int32_t* cand_idx, uint32_t* arrivals, const int* skip, int A,
                                   cudaStream_t s);
// Vocabulary slices (grid.x) of a walk step.
int walk_vocab_blocks(int num_sms, int V, int r, int dtype, bool quant);
cudaError_t launch_walk_init(const int32_t* anchors, int32_t* prev, uint32_t* ticket, int A, int V,
                             int32_t* status, const int* skip, cudaStream_t s);
// Confidence + lengths (hf = the final-normed hidden, fp32 [M, H]).
cudaError_t launch_confidence(const dspark_model* m, const float* hf32, const int32_t* anchors, const int32_t* tokens,
                              int A, float* conf, int32_t* lengths, cudaStream_t s);

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Launches a kernel with programmatic stream serialization (it may begin
// before its predecessor in the stream ends; see pdl_wait in common.cuh) and
// counts it.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void count_launches(int n);
    count_launches(1);
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// launch_pdl with clusters of `cluster_x` CTAs along x (gridDim.x a multiple of it).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, int cluster_x, size_t smem,
                               cudaStream_t s, Args&&... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)cluster_x;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    void count_launches(int n);
    count_launches(1);
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Launch accounting (timing.cu): count_launches after each launch; a
// KernelTimer in scope around a launch brackets it with events when timing is on.
void count_launches(int n);
class KernelTimer {
  public:
    KernelTimer(int kind, cudaStream_t s, double bytes, double flops);
    ~KernelTimer();
    KernelTimer(const KernelTimer&) = delete;
    KernelTimer& operator=(const KernelTimer&) = delete;
  private:
    int kind_;
    cudaStream_t s_;
    double bytes_, flops_;
    cudaEvent_t a_ = nullptr, b_ = nullptr;
};

}  // namespace dspark
