// dspark_attend_no_alloc: the attention seam with its scratch in a static
// device array, for callers that cannot hand the library any device memory
// beyond the tensors they already own -- a plugin whose host program owns
// the whole device pool, or a code path that must not call cudaMalloc
// because of the device-wide synchronisation it can imply.
//
// The scratch is the per-split softmax state of the split-KV attention (the
// unnormalised outputs and the (max, sum) pair of every context chunk and of
// the block keys). It lives in g_attend_scratch below: a file-scope
// __device__ array of kNoAllocScratchBytes, allocated once per GPU when the
// library's code is loaded there and held until the process exits.
#include <algorithm>
#include <mutex>
#include <string>

#include "internal.h"
#include "gemm.h"

namespace dspark {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;   // 16 MiB per GPU
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_attend_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_attend_scratch on the current device, looked up once per
// device. In host code the symbol is only a host-side stand-in: kernels must be
// given this address, never the symbol itself.
int scratch_address(int device, void** out) {
    std::lock_guard<std::mutex> lk(g_setup_mu);
    if (!g_scratch_addr[device]) {
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_attend_scratch);
        if (e != cudaSuccess)
            DSPARK_FAIL(DSPARK_ERR_CUDA, std::string("cudaGetSymbolAddress(attention scratch): ") + cudaGetErrorString(e));
        g_scratch_addr[device] = p;
    }
    *out = g_scratch_addr[device];
    return DSPARK_OK;
}

}  // namespace
}  // namespace dspark

using namespace dspark;

extern "C" int dspark_attend_no_alloc(const dspark_model* m, int32_t layer, const dspark_kv_cache* c, const void* q,
                                      const void* k_blk, const void* v_blk, void* out, int32_t A, int32_t max_ctx_len,
                                      void* stream) {
    if (!m) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "model is NULL");
    if (!c || !c->k || !c->v || !c->len) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "cache and its k, v, len must be non-NULL");
    if (A <= 0 || A > c->batch) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "A must be in [1, cache.batch]");
    if (max_ctx_len < 0 || max_ctx_len > c->capacity) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "max_ctx_len must be in [0, cache.capacity]");
    if (layer < 0 || layer >= m->d.Lyr) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "layer out of range");
    if (!q || !k_blk || !v_blk || !out) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "q, k_blk, v_blk and out must be non-NULL");
    if ((reinterpret_cast<uintptr_t>(c->k) | reinterpret_cast<uintptr_t>(c->v)) & 15u)
        DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "cache k / v must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k_blk) | reinterpret_cast<uintptr_t>(v_blk) |
         reinterpret_cast<uintptr_t>(out)) & 15u)
        DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "q, k_blk, v_blk and out must be 16-byte aligned");
    const Dims& d = m->d;

    // The split plan of dspark_attend; on tensor cores with at most as many CTAs (one
    // partial slot each) as the scratch holds.
    const bool tcore = tc::attention_tc_supported(m);
    const int chunk = attention_key_chunk(m, A, max_ctx_len);
    const int splits = max_ctx_len > 0 ? (max_ctx_len + chunk - 1) / chunk : 0;
    int grid = 0;
    size_t o_bytes, ml_bytes, items_bytes = 0;
    if (tcore) {
        const size_t slot_bytes = (size_t)128 * (d.hd + 2) * sizeof(float);
        grid = tc::attention_tc_grid(m, A);
        const size_t fixed = align_up(tc::attention_tc_item_ints(m, A) * 4, 256) + 512;
        const int fit = (int)((kNoAllocScratchBytes - std::min(fixed, kNoAllocScratchBytes)) / slot_bytes);
        grid = std::min(grid, fit);
        if (grid < A * d.nKv)
            DSPARK_FAIL(DSPARK_ERR_WORKSPACE, "attention state of " + std::to_string(A * d.nKv) + " CTAs needs more than "
                                              "the 16 MiB static scratch of dspark_attend_no_alloc; use dspark_attend "
                                              "with a caller workspace");
        o_bytes = align_up((size_t)grid * 128 * d.hd * sizeof(float), 256);
        ml_bytes = align_up((size_t)grid * 128 * 2 * sizeof(float), 256);
        items_bytes = align_up(tc::attention_tc_item_ints(m, A) * 4, 256);
    } else {
        const size_t parts = (size_t)A * d.nH * (size_t)(splits + 1) * d.gamma;
        o_bytes = align_up(parts * d.hd * sizeof(float), 256);
        ml_bytes = align_up(parts * 2 * sizeof(float), 256);
    }
    if (o_bytes + ml_bytes + items_bytes > kNoAllocScratchBytes)
        DSPARK_FAIL(DSPARK_ERR_WORKSPACE, "attention state needs " + std::to_string(o_bytes + ml_bytes + items_bytes) +
                                              " bytes, above the 16 MiB static scratch of dspark_attend_no_alloc; "
                                              "use dspark_attend with a caller workspace");

    int dev = -1;
    DSPARK_CUDA_CHECK(cudaGetDevice(&dev));
    if (dev != m->device) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "the model's device must be current");
    if (dev < 0 || dev >= kMaxDevices) DSPARK_FAIL(DSPARK_ERR_UNSUPPORTED, "device index above 63");
    void* scratch = nullptr;
    int rc = scratch_address(dev, &scratch);
    if (rc != DSPARK_OK) return rc;

    const size_t es = d.kv_dtype == DSPARK_DTYPE_F32 ? 4 : 2;
    const size_t layer_bytes = (size_t)c->batch * c->capacity * d.nKv * d.hd * es;
    AttnArgs a{};
    a.q = q; a.kb = k_blk; a.vb = v_blk; a.out = out;
    a.q_dtype = d.kv_dtype; a.out_dtype = d.kv_dtype;
    a.kc = static_cast<const char*>(c->k) + layer_bytes * layer;
    a.vc = static_cast<const char*>(c->v) + layer_bytes * layer;
    a.len = c->len; a.capacity = c->capacity; a.batch = c->batch;
    // Every slot (and per-item record) a merge reads is written earlier in the same
    // call, so nothing here needs clearing between calls.
    a.part_o = static_cast<float*>(scratch);
    a.part_ml = reinterpret_cast<float*>(static_cast<char*>(scratch) + o_bytes);
    a.item_slots = tcore ? reinterpret_cast<int*>(static_cast<char*>(scratch) + o_bytes + ml_bytes) : nullptr;
    a.tc_grid = grid;
    a.A = A; a.n_splits = splits; a.chunk = chunk;
    a.status = m->ws.status;
    double keys = (double)A * d.gamma;
    if (c->len_host)
        for (int b = 0; b < A; ++b) keys += c->len_host[b];
    a.kv_bytes = keys * d.nKv * d.hd * 2.0 * es + 2.0 * A * d.gamma * d.nH * d.hd * es;
    a.flops = 4.0 * (double)d.nH * d.gamma * d.hd * keys;
    cudaError_t e = run_attention(m, a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) DSPARK_FAIL(DSPARK_ERR_CUDA, std::string("attention launch: ") + cudaGetErrorString(e));
    return DSPARK_OK;
}
