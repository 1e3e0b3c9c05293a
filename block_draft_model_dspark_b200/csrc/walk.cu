// The VanillaMarkov walk at temperature 0 (deepspec.ts #markovStepBias,
// #selectStep and the sequential loop of draftRows): for step k,
//   bias_b[v] = markov_w2[v] . markov_w1[prev_b]        (rank-r GEMV over the vocabulary)
//   tok_{b,k} = argmax_v (U[b,k,v] + bias_b[v])          (lowest index on ties)
//   prev_b    = tok_{b,k}
// The sum is taken in fp32. One launch per step. A CTA owns a slice of the
// vocabulary and up to kRowsPerCta batch rows: r/8 lanes share one W2 row
// (each lane holds 8 of its values in registers, loaded once with 16-byte
// coalesced loads) and apply it to every row's markov_w1[prev] (from shared
// memory), so W2 streams once per step per kRowsPerCta rows. Each CTA writes
// its (value, index) candidates; the last CTA to finish (a ticket counter,
// not a value atomic) reduces them in CTA order and commits the step's
// tokens, so the result does not depend on scheduling.
#include <math.h>

#include <algorithm>

#include "internal.h"
#include "common.cuh"
#include "tc_ptx.cuh"

namespace dspark {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRowsPerCta = 8;       // batch rows per CTA (grid.y covers the rest)
constexpr int kMaxRank = 256;
constexpr int kChunkRows = 128;      // rows per bulk copy of the staged markov_w2 slice
constexpr int kMaxChunks = 16;
constexpr int kStageBytes = 96 * 1024;

__global__ void walk_init_kernel(const int32_t* anchors, int32_t* prev, uint32_t* ticket, int A, int V,
                                 int32_t* status, const int* skip) {
    pdl_trigger();
    pdl_wait();
    if (skip && *skip == 0) return;      // the pruned walk wrote the tokens
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b == 0) *ticket = 0u;
    if (b < A) {
        int t = anchors[b];
        if (t < 0 || t >= V) {
            atomicOr(status, DSPARK_DEV_BAD_TOKEN);
            t = min(max(t, 0), V - 1);
        }
        prev[b] = t;
    }
}

// Eight consecutive markov_w2 values W2[v, c8 .. c8+7] as fp32.
__device__ __forceinline__ void load_w2_8(const MatRef& W, int dtype, int group, int64_t v, int c8, int r,
                                          float w[8]) {
    if (W.quant) {
        dequant8(static_cast<const uint32_t*>(W.w), W.scales, W.biases, v, c8, r, group, w);
    } else if (dtype == DSPARK_DTYPE_F32) {
        const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(W.w) + v * r + c8);
        const float4 a = p[0], b = p[1];
        w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w; w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    } else {
        const uint4 u = *reinterpret_cast<const uint4*>(static_cast<const bf16*>(W.w) + v * r + c8);
        const uint32_t q[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) { w[2 * j] = __uint_as_float(q[j] << 16); w[2 * j + 1] = __uint_as_float(q[j] & 0xffff0000u); }
    }
}

// grid (vocabulary slices, ceil(A / kRowsPerCta)). With STAGED, the CTA's
// slice of a dense markov_w2 (contiguous rows) is requested at entry with 1-D
// bulk copies into shared memory, in chunks of kChunkRows rows with one
// mbarrier each, so the whole table is in flight at once; rows are then read
// from shared memory chunk by chunk.
template <bool STAGED>
__global__ void __launch_bounds__(kThreads)
walk_step_kernel(WalkArgs a, MatRef W2, const void* __restrict__ w1, int dtype, int group, int G, int V, int r,
                 int per) {
    extern __shared__ __align__(128) uint8_t wsm[];
    __shared__ float e[kRowsPerCta][kMaxRank];
    __shared__ float rv[kWarps][kRowsPerCta];
    __shared__ int ri[kWarps][kRowsPerCta];
    __shared__ bool last;
    __shared__ uint64_t bars[kMaxChunks];
    __shared__ int abort_flag;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int b0 = blockIdx.y * kRowsPerCta;
    const int nb = min(kRowsPerCta, a.A - b0);
    const int v0 = blockIdx.x * per, v1 = min(V, v0 + per);
    const int es = dtype == DSPARK_DTYPE_F32 ? 4 : 2;
    const int row_bytes = r * es;
    const int nchunks = v1 > v0 ? (v1 - v0 + kChunkRows - 1) / kChunkRows : 0;
    pdl_trigger();

    if (STAGED && tid == 0) {
        abort_flag = 0;
        for (int c = 0; c < nchunks; ++c) tc::mbar_init(&bars[c], 1);
        tc::mbar_fence_init();
        for (int c = 0; c < nchunks; ++c) {
            const int rows = min(kChunkRows, v1 - v0 - c * kChunkRows);
            const uint32_t bytes = (uint32_t)rows * row_bytes;
            tc::mbar_arrive_expect_tx(&bars[c], bytes);
            tc::bulk_load(wsm + (size_t)c * kChunkRows * row_bytes,
                          static_cast<const uint8_t*>(W2.w) + ((int64_t)v0 + (int64_t)c * kChunkRows) * row_bytes,
                          bytes, &bars[c]);
        }
    }
    pdl_wait();          // markov_w2 is requested above; prev comes from the previous step
    if (a.skip && *a.skip == 0) {
        // the pruned walk wrote the tokens: only the copies in flight must land before exit (bounded)
        if (STAGED && tid == 0) {
            const uint64_t deadline = tc::global_timer_ns() + tc::kWaitLimitNs;
            for (int c = 0; c < nchunks; ++c)
                if (!tc::mbar_wait_until(&bars[c], 0u, deadline)) { atomicOr(a.status, DSPARK_DEV_WAIT_TIMEOUT); break; }
        }
        return;
    }
    for (int i = tid; i < nb * r; i += kThreads) {
        const int bb = i / r, j = i % r;
        e[bb][j] = load_any(w1, (int64_t)a.prev[b0 + bb] * r + j, dtype);
    }
    __syncthreads();

    // lanes per W2 row (r/8, a power of two <= 32) and rows per warp step
    const int lpr = r > 0 ? r / 8 : 1;
    const int rpw = 32 / lpr;
    const int c8 = (lane % lpr) * 8;
    const bool leader = (lane % lpr) == 0;
    float best[kRowsPerCta];
    int bidx[kRowsPerCta];
#pragma unroll
    for (int bb = 0; bb < kRowsPerCta; ++bb) { best[bb] = -INFINITY; bidx[bb] = 0x7fffffff; }

    constexpr int U = 4;                                   // row groups in flight per lane
    const int stride = kWarps * rpw;
    bool ok = true;
    for (int c = 0; c < (STAGED ? nchunks : 1) && ok; ++c) {
        const int cv0 = STAGED ? v0 + c * kChunkRows : v0;
        const int cv1 = STAGED ? min(v1, cv0 + kChunkRows) : v1;
        if (STAGED && !tc::mbar_wait(&bars[c], 0u, &abort_flag, a.status)) { ok = false; break; }
        for (int vbase = cv0 + wid * rpw; vbase < cv1; vbase += U * stride) {     // warp-uniform
            int vv[U];
            float w[U][8];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                vv[u] = vbase + u * stride + lane / lpr;
                if (r > 0 && vv[u] < cv1) {
                    if (STAGED) {
                        const uint8_t* rowp = wsm + (size_t)(vv[u] - v0) * row_bytes;
                        if (dtype == DSPARK_DTYPE_F32) {
                            const float4 x0 = *reinterpret_cast<const float4*>(rowp + c8 * 4);
                            const float4 x1 = *reinterpret_cast<const float4*>(rowp + c8 * 4 + 16);
                            w[u][0] = x0.x; w[u][1] = x0.y; w[u][2] = x0.z; w[u][3] = x0.w;
                            w[u][4] = x1.x; w[u][5] = x1.y; w[u][6] = x1.z; w[u][7] = x1.w;
                        } else {
                            const uint4 q4 = *reinterpret_cast<const uint4*>(rowp + c8 * 2);
                            const uint32_t q[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
                            for (int j = 0; j < 4; ++j) { w[u][2 * j] = __uint_as_float(q[j] << 16); w[u][2 * j + 1] = __uint_as_float(q[j] & 0xffff0000u); }
                        }
                    } else {
                        load_w2_8(W2, dtype, group, vv[u], c8, r, w[u]);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j) w[u][j] = 0.f;
                }
            }
#pragma unroll
            for (int bb = 0; bb < kRowsPerCta; ++bb) {
                if (bb >= nb) break;
                const float* Urow = a.U + ((int64_t)(b0 + bb) * G + a.step) * V;
                float uv[U];
#pragma unroll
                for (int u = 0; u < U; ++u) uv[u] = (leader && vv[u] < cv1) ? Urow[vv[u]] : 0.f;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    float part = 0.f;
                    if (r > 0) {
#pragma unroll
                        for (int j = 0; j < 8; ++j) part = fmaf(w[u][j], e[bb][c8 + j], part);
                        for (int o = lpr / 2; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
                    }
                    if (leader && vv[u] < cv1) argmax_merge(best[bb], bidx[bb], uv[u] + part, vv[u]);
                }
            }
        }
    }
#pragma unroll
    for (int bb = 0; bb < kRowsPerCta; ++bb) {
        if (bb >= nb) break;
        float bv = best[bb];
        int bi = bidx[bb];
        warp_argmax(bv, bi);
        if (lane == 0) { rv[wid][bb] = bv; ri[wid][bb] = bi; }
    }
    __syncthreads();
    if (tid < nb) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
        for (int w = 0; w < kWarps; ++w) argmax_merge(bv, bi, rv[w][tid], ri[w][tid]);
        a.part_val[(int64_t)blockIdx.x * a.A + b0 + tid] = bv;
        a.part_idx[(int64_t)blockIdx.x * a.A + b0 + tid] = bi;
    }

    // ticket: the last CTA reduces all candidates in CTA order
    __threadfence();
    __syncthreads();
    if (tid == 0) last = atomicAdd(a.ticket, 1u) == gridDim.x * gridDim.y - 1;
    __syncthreads();
    if (!last) return;
    __threadfence();
    for (int b = wid; b < a.A; b += kWarps) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
        for (int c = lane; c < (int)gridDim.x; c += 32)
            argmax_merge(bv, bi, a.part_val[(int64_t)c * a.A + b], a.part_idx[(int64_t)c * a.A + b]);
        warp_argmax(bv, bi);
        if (lane == 0) {
            if (bi < 0 || bi >= V) {            // only if a row was all NaN
                atomicOr(a.status, DSPARK_DEV_BAD_TOKEN);
                bi = 0;
            }
            a.tokens[b * G + a.step] = bi;
            a.prev[b] = bi;
        }
    }
    if (tid == 0) *a.ticket = 0u;
}

}  // namespace

// Vocabulary slices of a step: dense tables are staged in shared memory
// (at most kStageBytes and kMaxChunks chunks a slice); 4-bit tables are read
// directly, about 2 slices per SM.
int walk_vocab_blocks(int num_sms, int V, int r, int dtype, bool quant) {
    if (!quant && r > 0) {
        const int row_bytes = r * (dtype == DSPARK_DTYPE_F32 ? 4 : 2);
        int rows = std::min(kStageBytes / row_bytes, kMaxChunks * kChunkRows);
        rows = std::max(kChunkRows, rows / kChunkRows * kChunkRows);
        int nblk = (V + rows - 1) / rows;
        return std::max(nblk, std::min(2 * num_sms, (V + kChunkRows - 1) / kChunkRows));
    }
    const int rpw = r > 0 ? 32 / (r / 8) : 32;
    const int rows_per_iter = kWarps * rpw;
    const int cap = (V + rows_per_iter * 4 - 1) / (rows_per_iter * 4);   // >= 4 warp steps per CTA
    return std::max(1, std::min(2 * num_sms, cap));
}

cudaError_t launch_walk_init(const int32_t* anchors, int32_t* prev, uint32_t* ticket, int A, int V, int32_t* status,
                             const int* skip, cudaStream_t s) {
    return launch_pdl(walk_init_kernel, dim3((A + 127) / 128), dim3(128), 0, s, anchors, prev, ticket, A, V, status,
                      skip);
}

cudaError_t launch_walk_step(const dspark_model* m, const WalkArgs& a, cudaStream_t s) {
    const Dims& d = m->d;
    const int per = (d.V + a.nblk - 1) / a.nblk;
    dim3 grid(a.nblk, (a.A + kRowsPerCta - 1) / kRowsPerCta);
    const bool staged = !d.quant && d.r > 0;
    if (staged) {
        const int row_bytes = d.r * (d.dtype == DSPARK_DTYPE_F32 ? 4 : 2);
        const size_t smem = (size_t)per * row_bytes;
        if (per > kMaxChunks * kChunkRows || smem > (size_t)kStageBytes) return cudaErrorInvalidValue;
        cudaError_t e = cudaFuncSetAttribute(walk_step_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kStageBytes);
        if (e != cudaSuccess) return e;
        return launch_pdl(walk_step_kernel<true>, grid, dim3(kThreads), smem, s, a, m->w2, m->w1, d.dtype, d.group,
                          d.gamma, d.V, d.r, per);
    }
    return launch_pdl(walk_step_kernel<false>, grid, dim3(kThreads), 0, s, a, m->w2, m->w1, d.dtype, d.group, d.gamma,
                      d.V, d.r, per);
}

}  // namespace dspark
