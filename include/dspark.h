/*
 * dspark.h -- C ABI of libdspark, the DSpark draft round on one B200 (sm_100a).
 *
 * The round is the one the "@mlx-bun/inference 0.0.0-stage -> 1.0.0" page
 * defines in package/src/models/speculative/deepspec.ts (class
 * DeepspecDrafter): context K/V projection (#projectContextKVRows), the
 * backbone over the noise block with KV-injection attention
 * (#forwardBackbone and the DeepspecContextAttention.attend seam of the
 * "mlx-bun 0.2.0 -> 0.4.0" page 75), logits with softcap (#computeLogits),
 * the VanillaMarkov walk (#markovStepBias / #selectStep), the confidence
 * head (#confidence) and the confident-prefix truncation (draftRows).
 *
 * Conventions shared by every entry point:
 *  - Every pointer argument named "device" is CUDA device memory the caller
 *    allocated and owns; the library never allocates device memory. Pointers
 *    named "host" are host memory, read during the call only.
 *  - Row-major layouts; dims listed outermost first. "T" is the model's
 *    storage dtype (dspark_config.dtype: fp32 or bf16).
 *  - All work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream); calls return once enqueued. Results are valid after the stream
 *    reaches them.
 *  - Return value: DSPARK_OK or a negative DSPARK_ERR_*; on error nothing was
 *    enqueued and no output or cache was modified, and dspark_last_error()
 *    (per host thread) says why. Arguments are validated before any launch.
 *  - Device-side checks (token ids, cache lengths, bounded waits) record a
 *    nonzero code in the model's device status word instead of faulting;
 *    dspark_read_device_status() fetches and clears it.
 */
#ifndef DSPARK_H
#define DSPARK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DSPARK_OK                    0
#define DSPARK_ERR_INVALID_ARGUMENT (-1) /* null pointer, bad size, misaligned buffer */
#define DSPARK_ERR_UNSUPPORTED      (-2) /* a config the drafter page refuses, or outside this build's shapes */
#define DSPARK_ERR_CAPACITY         (-3) /* reserved: appends are validated on the device (DSPARK_DEV_CAPACITY) */
#define DSPARK_ERR_WORKSPACE        (-4) /* workspace smaller than the matching *_workspace_bytes() */
#define DSPARK_ERR_CUDA             (-5) /* a CUDA runtime call or launch failed */
#define DSPARK_ERR_DEVICE           (-6) /* a device-side check failed (see dspark_read_device_status) */

/* Device status codes (bit flags, OR-ed by kernels). */
#define DSPARK_DEV_BAD_TOKEN     1  /* an anchor or walked token outside [0, vocab) was clamped */
#define DSPARK_DEV_BAD_LENGTH    2  /* a cache length above capacity was clamped */
#define DSPARK_DEV_WAIT_TIMEOUT  4  /* a bounded device wait gave up */
#define DSPARK_DEV_CAPACITY      8  /* an append was refused on the device (a count outside [0, Lnew_max] or past capacity) */
#define DSPARK_DEV_RANGE        16  /* a 4-bit model's context row held a value outside fp16's range (|x| > 65504) */

#define DSPARK_DTYPE_F32  0
#define DSPARK_DTYPE_BF16 1
#define DSPARK_DTYPE_F16  2   /* the context K/V of bf16 models (dspark_kv_dtype) */

/*
 * Model configuration: the drafter's config.json keys (deepspec.ts,
 * DeepspecConfig / readConfig), one int or float each. The three variants
 * readConfig refuses are refused here too (DSPARK_ERR_UNSUPPORTED):
 * attention_k_eq_v = 0, a non-vanilla Markov head with markov_rank > 0, and
 * an activation other than gelu_pytorch_tanh.
 */
typedef struct dspark_config {
    int32_t hidden_size;
    int32_t num_hidden_layers;
    int32_t num_attention_heads;
    int32_t global_head_dim;               /* 64, 128, 192 or 256 */
    int32_t num_global_key_value_heads;    /* divides num_attention_heads */
    int32_t intermediate_size;
    int32_t vocab_size;
    int32_t block_size;                    /* gamma */
    int32_t mask_token_id;
    int32_t markov_rank;                   /* 0 = no Markov head (plain argmax); else a power of two in [8, 256] */
    int32_t attention_k_eq_v;              /* must be 1 */
    int32_t markov_head_vanilla;           /* must be 1 when markov_rank > 0 */
    int32_t hidden_activation_gelu_tanh;   /* must be 1 */
    int32_t enable_confidence_head;
    int32_t confidence_head_with_markov;
    int32_t dtype;                         /* DSPARK_DTYPE_F32 or DSPARK_DTYPE_BF16 */
    int32_t quant_bits;                    /* 0 = dense T weights; 4 = affine 4-bit (bf16 only) */
    int32_t quant_group_size;              /* 64 when quant_bits == 4 */
    float   rope_theta;
    float   partial_rotary_factor;
    float   rms_norm_eps;
    float   final_logit_softcapping;       /* 0 = none (config null) */
    float   confidence_threshold;          /* <= 0: no truncation, full gamma */
} dspark_config;

/*
 * A matmul weight W [out, in] used as x @ W^T (deepspec.ts MatW), or a
 * gather table [rows, dim] (TableW). Dense: `w` is T [out, in] and
 * `scales`/`biases` are NULL. Affine 4-bit (MLX QuantizedLinear layout): `w`
 * is uint32 [out, in/8] with input column 8*j + i in bits 4i..4i+3 of word
 * j; `scales` and `biases` are bf16 [out, in/group]; weight = scale*code + bias.
 * All device pointers, 16-byte aligned.
 */
typedef struct dspark_matrix {
    const void* w;
    const void* scales;
    const void* biases;
} dspark_matrix;

/* One decoder layer's weights (deepspec.ts, interface Layer). Gains are T
 * [hidden] or [head_dim]; layer_scalar is T [1]. */
typedef struct dspark_layer_weights {
    dspark_matrix q_proj;     /* [nH*hd, H] */
    dspark_matrix k_proj;     /* [nKv*hd, H] */
    dspark_matrix o_proj;     /* [H, nH*hd] */
    dspark_matrix gate_proj;  /* [I, H] */
    dspark_matrix up_proj;    /* [I, H] */
    dspark_matrix down_proj;  /* [H, I] */
    const void* q_norm;                      /* [hd] */
    const void* k_norm;                      /* [hd] */
    const void* input_layernorm;             /* [H] */
    const void* post_attention_layernorm;    /* [H] */
    const void* pre_feedforward_layernorm;   /* [H] */
    const void* post_feedforward_layernorm;  /* [H] */
    const void* layer_scalar;                /* [1] */
} dspark_layer_weights;

/* All weights (device pointers, caller-owned, read-only to the library). */
typedef struct dspark_weights {
    dspark_matrix embed_tokens;      /* table [V, H] */
    dspark_matrix lm_head;           /* [V, H] */
    dspark_matrix markov_w2;         /* [V, r] (unused when markov_rank == 0) */
    dspark_matrix confidence_proj;   /* [1, H (+ r)] (unused without the confidence head) */
    const void* markov_w1;           /* dense T table [V, r] */
    const void* norm;                /* final norm gain, T [H] */
    const void* confidence_bias;     /* T [1] */
    const dspark_layer_weights* layers;  /* HOST array of num_hidden_layers entries */
} dspark_weights;

/*
 * Element type "KV" of the context K/V (caches, the projection's outputs, the
 * attention seam's tensors): DSPARK_DTYPE_F16 for a bf16 model, DSPARK_DTYPE_F32
 * for an fp32 one; -1 for an invalid config. The drafter page keeps ContextKV
 * rows in the model dtype; here a bf16 model's rows are fp16 instead (same two
 * bytes per element): the keys and values are RMS-normed (|x| <= sqrt(head_dim)
 * times the k_norm gain), where fp16's 11-bit significand holds them more
 * precisely than bf16's 8 bits, and the tensor cores multiply fp16 queries and
 * probabilities with them without converting any cache tile.
 */
int32_t dspark_kv_dtype(const dspark_config* cfg);

/*
 * Per-request context K/V storage, owned by the caller (the drafter page's
 * seam: "storage owns context validity"; deepspec.ts draftRows doc: the
 * caller owns the cache's lifetime and the crop after the round).
 * k, v: device KV [num_hidden_layers][batch][capacity][nKv][hd]; row t of
 * batch row b holds the K (normed, roped) / V (scale-less normed, unroped)
 * of context row t. len: device int32 [batch], the valid rows per batch row;
 * the caller sets it when it builds or crops a cache (a crop is a smaller
 * len: rows past len are never read), dspark_append_context_kv advances it.
 * len_host: optional host int32 [batch] (may be NULL), the caller's own
 * host copy of len when it keeps one. The library never writes it and reads
 * it only to count the attention's algorithmic bytes for the instrumentation
 * timers below.
 * V-only cache: k = NULL. With attention_k_eq_v the keys and values come from
 * one projection and one normalisation, so k[l,b,t] = rope(v[l,b,t] * k_norm_l,
 * position of row t) (dspark_project_context_kv below); a V-only cache stores v
 * alone and the attention rebuilds k from it, which halves the cache's memory
 * and the bytes every round reads (the rebuild costs SM time: with every RoPE
 * pair rotated, a round's attention is slower than on a K+V cache, so V-only
 * trades speed for memory). It needs pos0 (device int32 [batch], the
 * absolute position of cache row 0 of each batch row, so row t sits at
 * pos0[b] + t: the positions the rows were projected at) and a bf16 model on
 * the tensor-core attention (head_dim a multiple of 64, at most 256), and is
 * read by dspark_draft_rows and written by
 * dspark_append_context_kv; dspark_attend and dspark_attend_no_alloc take
 * the seam's explicit block keys and refuse it (DSPARK_ERR_INVALID_ARGUMENT).
 * Other calls refuse k = NULL where V-only is unsupported
 * (DSPARK_ERR_UNSUPPORTED). pos0 is ignored when k != NULL.
 */
typedef struct dspark_kv_cache {
    void*    k;
    void*    v;
    int32_t* len;
    int32_t* len_host;
    int32_t  batch;
    int32_t  capacity;
    const int32_t* pos0;
} dspark_kv_cache;

typedef struct dspark_model dspark_model;

/* Bytes of device memory dspark_model_create needs for its stacked weight
 * copies, RoPE table, status word and (bf16, markov_rank 64) the Markov norm
 * bounds; 0 for an invalid config. */
size_t dspark_model_workspace_bytes(const dspark_config* cfg);

/*
 * Builds a model handle: validates `cfg` (readConfig's guards plus this
 * build's shape limits), records the weight pointers, and writes into
 * `model_ws` (device, >= dspark_model_workspace_bytes, 256-byte aligned,
 * caller-owned, must outlive the model) the RoPE inverse-frequency table and
 * the stacked [q_proj; k_proj], [gate_proj; up_proj] and all-layer k_proj
 * copies the kernels read, and for bf16 weights with markov_rank 64 the
 * bounds |markov_w2[v]| and max_p |markov_w1[p]| that let dspark_draft_rows
 * prune the walk exactly. Enqueues this work on `stream` and waits for it. The
 * weights must stay valid and unchanged for the model's lifetime.
 */
int dspark_model_create(const dspark_config* cfg, const dspark_weights* weights,
                        void* model_ws, size_t model_ws_bytes, void* stream,
                        dspark_model** out_model);

/* Frees the host-side handle (device memory stays the caller's). */
int dspark_model_destroy(dspark_model* model);

/* Scratch bytes dspark_project_context_kv / dspark_append_context_kv need
 * for `rows` = B * L projected rows. */
size_t dspark_project_workspace_bytes(const dspark_model* model, int64_t rows);

/*
 * Confidence-scheduled draft-length pruning (Alg 1 of the DFlash generator's
 * forwardInfer, "@mlx-bun/inference 0.0.0-stage -> 1.0.0": calibrated
 * per-position thresholds, or one minConf for every position): for row b,
 *   lengths[b] = the first k >= 1 with conf[b, k] < thresholds[k], else gamma
 * (position 0 always survives, unlike dspark_draft_rows' confidence_threshold
 * rule, which can keep none; a NaN confidence is not below any threshold).
 *   conf        device float [A, gamma] (the confidences dspark_draft_rows wrote)
 *   thresholds  device float [gamma] (entry 0 unused)
 *   lengths     device int32 [A]
 * Enqueued on `stream`; argument errors return before any launch.
 */
int dspark_prune_lengths(const float* conf, int32_t A, int32_t gamma, const float* thresholds, int32_t* lengths,
                         void* stream);

/*
 * Context feature projection (deepspec.ts #projectContext): the context hidden
 * the projections below read, from the target model's tap hiddens. The caller
 * concatenates, per context row, the target's hiddens at the taps
 * (extract_context_feature: the post-layer output of every target_layer_ids
 * entry, in that order) into target_hiddens; then for every row
 *   out[b,t] = rms(target_hiddens[b,t] @ fc^T, hidden_norm)
 * with rms the Gemma4RMSNorm of the config's eps (computed in fp32).
 *   fc              [hidden, taps * hidden] stored [out, in]: dense in the model
 *                   dtype (.w only; a bf16 model runs it on the tensor cores), or
 *                   4-bit affine (.w the packed words [hidden, taps*hidden/8],
 *                   .scales / .biases bf16 [hidden, taps*hidden/group], group the
 *                   model's quant_group_size, 64 for a dense model: dequantized on
 *                   load by the CUDA-core GEMM; both or neither of scales and
 *                   biases, else DSPARK_ERR_INVALID_ARGUMENT)
 *   hidden_norm     device T [hidden]
 *   target_hiddens  device T [B, L, taps * hidden]
 *   out             device T [B, L, hidden]: the `hidden` of
 *                   dspark_project_context_kv / dspark_append_context_kv
 *   ws              >= dspark_context_features_workspace_bytes(model, taps, B * L)
 * fc.w, target_hiddens, out and ws must be 16-byte aligned; on a bf16 model
 * taps * hidden must be a multiple of 64. Argument errors return before any
 * launch. The weights are the caller's (not part of dspark_weights): the
 * projection runs once per context row, outside the draft round.
 */
size_t dspark_context_features_workspace_bytes(const dspark_model* model, int32_t taps, int64_t rows);
int dspark_project_context_features(const dspark_model* model, const dspark_matrix* fc, const void* hidden_norm,
                                    int32_t taps, const void* target_hiddens, int32_t B, int32_t L, void* out,
                                    void* ws, size_t ws_bytes, void* stream);

/*
 * Context K/V projection (deepspec.ts #projectContextKVRows; page 75
 * projectContextKV). For every layer l, batch row b < B and context row
 * t < L, with k_raw = hidden[b,t,:] @ k_proj_l^T viewed [nKv, hd]:
 *   v[l,b,t] = k_raw / sqrt(mean(k_raw^2) + eps)            (v_norm, no rope)
 *   k[l,b,t] = rope(v[l,b,t] * k_norm_l, position p)        (k_norm then rope)
 * where p = static_pos + t when pos0 == NULL, else pos0[b] + t.
 *   hidden  device T [B, L, H]
 *   pos0    device int32 [B] or NULL
 *   k_out, v_out  device KV [num_hidden_layers][B][L][nKv][hd]
 * (the dspark_kv_cache layout with capacity = L). k_out = NULL writes v alone
 * (the rows of a V-only cache).
 */
int dspark_project_context_kv(const dspark_model* model, const void* hidden, int32_t B, int32_t L,
                              int32_t static_pos, const int32_t* pos0,
                              void* k_out, void* v_out, void* ws, size_t ws_bytes, void* stream);

/*
 * Incremental context append (the drafter page's incremental cache:
 * post-norm, post-rope context rows are per-row, so caching them equals
 * recomputing them inside every round's concat; deepspec.ts draftRows doc:
 * the caller owns the cache and its crop). For batch row b, projects
 * hidden[b, 0:n_new[b]] as above and writes cache rows [len_b, len_b +
 * n_new[b]) at positions pos0[b] + len_b + t, then sets len[b] += n_new[b],
 * all on the device (the accepted-row counts come out of verification on the
 * device; no host round trip is needed between verifying and appending).
 *   hidden     device T [cache.batch, Lnew_max, H] (rows past n_new[b] are ignored)
 *   n_new      device int32 [cache.batch]
 *   Lnew_max   host: the largest count the caller may pass, in [0, capacity]
 *   pos0       device int32 [cache.batch]: absolute position of cache row 0
 * The counts are validated on the device before any row is written: if any
 * row has n_new[b] outside [0, Lnew_max] or len[b] + n_new[b] > capacity,
 * the whole append is refused -- no cache row and no len changes -- and
 * DSPARK_DEV_CAPACITY is set in the device status word (read it with
 * dspark_read_device_status). Host-side argument errors return before any
 * launch. cache.batch <= 4096. On a V-only cache (cache.k = NULL) only v rows
 * are written (their values do not depend on the position).
 */
int dspark_append_context_kv(const dspark_model* model, const void* hidden, int32_t Lnew_max,
                             const int32_t* n_new, const int32_t* pos0, dspark_kv_cache* cache,
                             void* ws, size_t ws_bytes, void* stream);

/* Scratch bytes dspark_draft_rows / dspark_attend need for A rows whose
 * context is at most max_ctx_len rows. */
size_t dspark_draft_workspace_bytes(const dspark_model* model, int32_t A, int32_t max_ctx_len);

/*
 * One draft round for A rows (deepspec.ts draftRows). Row b drafts the block
 * [anchors[b], mask x (gamma-1)] at positions block_pos[b] + t against its
 * cached context rows [0, cache.len[b]) (cache batch row b; A <= cache.batch):
 * backbone -> final norm -> U = softcap(lm_head(h)) -> for k = 0..gamma-1:
 * tokens[b,k] = argmax_v(U[b,k,v] + markov_w2(markov_w1[prev])[v]) with prev =
 * anchor then the previous token (lowest index on ties) -> conf[b,k] =
 * sigmoid(proj([h_k ; markov_w1[prev_k]]) + bias) -> lengths[b] = first k with
 * conf < threshold (threshold > 0), else gamma.
 *   anchors    device int32 [A]       block_pos device int32 [A]
 *   max_ctx_len  host upper bound of cache.len[b] over the A rows (<= capacity)
 *   tokens     device int32 [A, gamma] (all gamma walked tokens; lengths says how many to keep)
 *   conf       device float [A, gamma] or NULL (needs the confidence head)
 *   lengths    device int32 [A]
 *   base_logits device float [A, gamma, V] or NULL (the page's collectLogits)
 */
int dspark_draft_rows(const dspark_model* model, const dspark_kv_cache* cache,
                      const int32_t* anchors, const int32_t* block_pos, int32_t A, int32_t max_ctx_len,
                      int32_t* tokens, float* conf, int32_t* lengths, float* base_logits,
                      void* ws, size_t ws_bytes, void* stream);

/*
 * The attention seam alone (page 75, DeepspecContextAttention.attend and
 * plainDeepspecContext): for batch row b < A and query head h, attends
 * q[b,:,h,:] over keys [cache.k[layer,b,0:len_b,g] ++ k_blk[b,:,g]] and
 * values [cache.v[layer,b,0:len_b,g] ++ v_blk[b,:,g]], g = h / (nH/nKv),
 * non-causal, scale 1.0, softmax in fp32.
 *   q   device KV [A, gamma, nH, hd]    k_blk, v_blk device KV [A, gamma, nKv, hd]
 *   out device KV [A, gamma, nH, hd]      (KV: dspark_kv_dtype)
 * q, k_blk, v_blk, out and ws must be 16-byte aligned (DSPARK_ERR_INVALID_ARGUMENT
 * otherwise, before any launch); the same holds for dspark_attend_no_alloc.
 */
int dspark_attend(const dspark_model* model, int32_t layer, const dspark_kv_cache* cache,
                  const void* q, const void* k_blk, const void* v_blk, void* out,
                  int32_t A, int32_t max_ctx_len, void* ws, size_t ws_bytes, void* stream);

/*
 * dspark_attend without a workspace argument: it computes what dspark_attend
 * computes, with the same kernels (a bf16 model's call may split the keys
 * over fewer CTAs, so results can differ in the last bits), for callers that
 * cannot provide device scratch memory -- a plugin whose host program owns
 * the whole device pool and hands it only the tensors above, or a path that
 * must not call cudaMalloc (which may synchronise the device). The pages have
 * no counterpart to this entry point.
 * Its scratch (the per-split softmax state and, for a bf16 model, the
 * per-item slot records) is a 16 MiB static device array inside libdspark, allocated on
 * every GPU that loads the library and held until the process exits. A bf16
 * model's call uses at most as many CTAs as that array holds partial states
 * of 128 x (hd + 2) floats (at hd = 256, 126; fewer CTAs only lengthen the
 * call), and is refused with DSPARK_ERR_WORKSPACE before any launch when A *
 * nKv exceeds that; an fp32 model's call needs A * nH * (context splits + 1)
 * * gamma * (hd + 2) * 4 bytes and is refused above 16 MiB. It allocates nothing. The first
 * call on each device looks up the array's device address (a one-time
 * runtime call) and keeps it for the process: make that first call, with the
 * model's device current, before any stream capture, and do not use this entry
 * point on a device whose context the process has reset (cudaDeviceReset)
 * since then: the kept address would not belong to the new context. Every
 * call on a device shares the one array, so
 * calls that overlap on the GPU (different streams or threads) race: issue
 * them in order on one stream per device. No part of the array needs to
 * start at zero: each call writes every slot before reading it.
 */
int dspark_attend_no_alloc(const dspark_model* model, int32_t layer, const dspark_kv_cache* cache,
                           const void* q, const void* k_blk, const void* v_blk, void* out,
                           int32_t A, int32_t max_ctx_len, void* stream);

/*
 * Test-facing dump of every layer's attention output (the parity check of the
 * DeepspecContextAttention.attend seam inside a round, page 75). While `dst`
 * is non-NULL, every later dspark_draft_rows call on `model` also copies each
 * layer's attention output, fp32 [num_hidden_layers][A][gamma][nH][hd], into
 * `dst` (device, at least `bytes`; a round whose A needs more fails with
 * DSPARK_ERR_WORKSPACE before any launch). dst = NULL turns the dump off. The
 * copies run on the round's stream; they slow the round down.
 */
int dspark_debug_attention_dump(dspark_model* model, float* dst, size_t bytes);

/*
 * Test-facing dump of the per-position statistics of the logits U (the
 * lm-head epilogue's per-tile max / argmax / sum of exponentials, merged per
 * position; deepspec.ts #computeLogits). While `dst` is non-NULL, every later
 * dspark_draft_rows call on `model` writes, for each position (row b, step k)
 * in [A][gamma] order, 16 bytes: float max_v U[b,k,v]; float logsumexp_v
 * U[b,k,v]; int32 lowest argmax; int32 candidates the Markov walk's exact
 * pruning kept (above 1024: the full walk decided). `dst` is device memory of
 * at least `bytes` (a round needing more than A * gamma * 16 bytes fails with
 * DSPARK_ERR_WORKSPACE before any launch); dst = NULL turns the dump off.
 */
int dspark_debug_logit_stats(dspark_model* model, void* dst, size_t bytes);

/*
 * Test-facing probe of the device-side failure detection (no counterpart on
 * the pages). Every wait inside the library's kernels is bounded: when it runs
 * out it records DSPARK_DEV_WAIT_TIMEOUT in the model's status word and the
 * kernel returns instead of hanging. This enqueues one small kernel that runs
 * the same bounded wait on an mbarrier nothing ever arrives on, giving up after
 * `limit_us` microseconds (1 .. 2,000,000), so a test can read the status and
 * check that the next call runs normally. Faults nothing.
 */
int dspark_debug_wait_probe(const dspark_model* model, int32_t limit_us, void* stream);

/* Synchronises `stream`, returns the device status bits in *status and
 * clears them. */
int dspark_read_device_status(const dspark_model* model, void* stream, int32_t* status);

/* Last error message of the calling host thread ("" if none). */
const char* dspark_last_error(void);

/*
 * Instrumentation (no counterpart on the pages; used by the benchmark).
 * dspark_kernel_launches: number of CUDA kernels this library has launched in
 * this process. dspark_timer_enable(1): from now on each launch of a kernel
 * class below is bracketed by CUDA events on its stream (a few microseconds of
 * host work per launch) and tagged with its algorithmic bytes and flops.
 * dspark_timer_read: waits for the recorded events of `kind`, returns their
 * summed device milliseconds, launch count, bytes and flops (either of the
 * last two may be NULL), and forgets them.
 */
#define DSPARK_TIMER_GEMM_QK     0  /* per layer: x @ [q_proj; k_proj]^T */
#define DSPARK_TIMER_LM_HEAD     1  /* lm-head GEMM with softcap */
#define DSPARK_TIMER_ATTENTION   2  /* KV-injection attention (partials + merge) */
#define DSPARK_TIMER_WALK        3  /* Markov walk */
#define DSPARK_TIMER_KV_PROJECT  4  /* context K/V projection GEMM + epilogue */
#define DSPARK_TIMER_ROWS        5  /* embedding, norms/RoPE/residual epilogues, confidence */
#define DSPARK_TIMER_GEMM_O      6  /* per layer: attention out @ o_proj^T */
#define DSPARK_TIMER_GEMM_GU     7  /* per layer: x @ [gate; up]^T */
#define DSPARK_TIMER_GEMM_DOWN   8  /* per layer: gelu(gate) * up @ down^T */
#define DSPARK_TIMER_KINDS       9
uint64_t dspark_kernel_launches(void);
int dspark_timer_enable(int enable);
int dspark_timer_read(int kind, double* total_ms, int64_t* launches, double* bytes, double* flops);

#ifdef __cplusplus
}
#endif

#endif /* DSPARK_H */
