// The whole temperature-0 VanillaMarkov walk of a round in one launch
// (deepspec.ts #markovStepBias / #selectStep and the sequential loop of
// draftRows): for k = 0 .. gamma-1,
//   bias_b[v] = markov_w2[v] . markov_w1[prev_b];  tok_{b,k} = argmax_v(U[b,k,v] + bias_b[v]);  prev_b = tok_{b,k}
// (fp32 sum, lowest index on ties).
//
// One CTA per SM, launched cooperatively (all CTAs resident). Each CTA owns
// a fixed slice of the vocabulary. Per step every CTA scans its slice for all
// rows, writes one (value, index) candidate per row, and arrives on a grid
// barrier (a global arrival counter; the wait is bounded: past kWaitLimitNs
// it records DSPARK_DEV_WAIT_TIMEOUT and the kernel returns). After the
// barrier every CTA reduces all candidates in CTA order -- the same
// arithmetic in every CTA, so all agree on the step's token without a second
// barrier -- and takes markov_w1 of the new token for the next step.
// Candidates are double-buffered by step parity. The arrival counter is
// zeroed by the caller before the round's first kernel.
//
// Staged variant (dense markov_w2, at most kStagedRows batch rows): the step
// is latency-bound unless the slice sits on chip. markov_w2 does not change
// during the walk, so as much of the CTA's slice as shared memory holds is
// bulk-copied in once ("resident" rows) and the rest streams through a ring
// of kRing chunks that runs ahead across steps; the U rows of each step are
// bulk-copied into a double buffer one step ahead. The scan then reads only
// shared memory.
#include <math.h>

#include <algorithm>

#include "internal.h"
#include "common.cuh"
#include "tc_ptx.cuh"

namespace dspark {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxRows = 64;         // batch rows per launch
constexpr int kMaxRank = 256;
constexpr int kStagedRows = 8;       // batch rows of the staged variant (one register group)
constexpr int kRing = 4;             // ring slots of streamed markov_w2 rows
constexpr int kChunkRows = 64;       // markov_w2 rows per ring slot
constexpr int kSmemLimit = 225 * 1024;      // dynamic shared memory: 227 KB less the static arrays
constexpr int kPieceBytes = 32 * 1024;   // resident rows are requested in pieces of this size

struct PWalkArgs {
    const float* U;            // [A, G, V]
    const int32_t* anchors;    // [A]
    int32_t* tokens;           // [A, G]
    float* cand_val;           // [2][grid][A]
    int32_t* cand_idx;         // [2][grid][A]
    uint32_t* arrivals;        // one counter, zero at entry
    int A, G, V, r, dtype, group;
    int per;                   // vocabulary rows per CTA
    // staged variant: shared-memory layout (byte offsets) and resident rows
    int staged, R, off_u, off_res, off_ring, off_bars;
    int32_t* status;
    const int* skip;           // non-NULL: return at once when *skip == 0 (tokens already written)
};

__device__ __forceinline__ void w2_load8(const MatRef& W, int dtype, int group, int64_t v, int c8, int r, float w[8]) {
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

// Eight markov_w2 values of a row held in shared memory.
__device__ __forceinline__ void w2_smem8(const uint8_t* row, int dtype, int c8, float w[8]) {
    if (dtype == DSPARK_DTYPE_F32) {
        const float4* p = reinterpret_cast<const float4*>(row + c8 * 4);
        const float4 a = p[0], b = p[1];
        w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w; w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    } else {
        const uint4 u = *reinterpret_cast<const uint4*>(row + c8 * 2);
        const uint32_t q[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) { w[2 * j] = __uint_as_float(q[j] << 16); w[2 * j + 1] = __uint_as_float(q[j] & 0xffff0000u); }
    }
}

__device__ __forceinline__ void red_release_add(uint32_t* p, uint32_t v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Grid barrier of step `step`: arrive, then wait (bounded) until every CTA
// has arrived. Returns false after a timeout.
__device__ __forceinline__ bool grid_barrier(uint32_t* arrivals, int step, int nblk, int32_t* status, int* s_fail) {
    __syncthreads();
    if (threadIdx.x == 0) {
        red_release_add(arrivals, 1u);
        const uint32_t target = (uint32_t)(step + 1) * (uint32_t)nblk;
        const uint64_t t0 = tc::global_timer_ns();
        while (ld_acquire(arrivals) < target) {
            if (tc::global_timer_ns() - t0 > tc::kWaitLimitNs) {
                atomicOr(status, DSPARK_DEV_WAIT_TIMEOUT);
                *s_fail = 1;
                break;
            }
        }
    }
    __syncthreads();
    return *s_fail == 0;
}

// Every CTA reduces all candidates of this step in CTA order into prev[].
__device__ __forceinline__ void reduce_candidates(const PWalkArgs& a, const float* cval, const int32_t* cidx,
                                                  int step, int* prev) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nblk = gridDim.x;
    for (int b = wid; b < a.A; b += kWarps) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
        for (int c = lane; c < nblk; c += 32)
            argmax_merge(bv, bi, __ldcg(&cval[(size_t)c * a.A + b]), __ldcg(&cidx[(size_t)c * a.A + b]));
        warp_argmax(bv, bi);
        if (lane == 0) {
            if (bi < 0 || bi >= a.V) {        // only if a row was all NaN
                if (blockIdx.x == 0) atomicOr(a.status, DSPARK_DEV_BAD_TOKEN);
                bi = 0;
            }
            prev[b] = bi;
            if (blockIdx.x == 0) a.tokens[b * a.G + step] = bi;
        }
    }
    __syncthreads();
}

// The per-lane bests of rows [b0, b0 + nb) merged over the CTA and written as
// this CTA's candidates.
__device__ __forceinline__ void write_candidates(const PWalkArgs& a, float (&best)[8], int (&bidx)[8], int b0, int nb,
                                                 float* cval, int32_t* cidx, float (*rv)[8], int (*ri)[8]) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, tid = threadIdx.x;
#pragma unroll
    for (int bb = 0; bb < 8; ++bb) {
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
        cval[(size_t)blockIdx.x * a.A + b0 + tid] = bv;
        cidx[(size_t)blockIdx.x * a.A + b0 + tid] = bi;
        __threadfence();
    }
}

__global__ void __launch_bounds__(kThreads, 1)
walk_persistent_kernel(PWalkArgs a, MatRef W2, const void* __restrict__ w1) {
    extern __shared__ __align__(128) uint8_t wdyn[];
    float* e_dyn = reinterpret_cast<float*>(wdyn);    // [A][r + 4]: markov_w1 of each row's previous token
    __shared__ int prev[kMaxRows];
    __shared__ float rv[kWarps][8];
    __shared__ int ri[kWarps][8];
    __shared__ int s_fail;
    if (a.skip && *a.skip == 0) return;   // uniform: every CTA reads the same word
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int G = a.G, V = a.V, r = a.r, A = a.A;
    const int nblk = gridDim.x;
    const int per = a.per;
    const int v0 = min(V, blockIdx.x * per), v1 = min(V, v0 + per);
    const int lpr = r > 0 ? r / 8 : 1;      // lanes per markov_w2 row
    const int rpw = 32 / lpr;               // rows per warp step
    const int c8 = (lane % lpr) * 8;
    const bool leader = (lane % lpr) == 0;
    const int ep = r + 4;
    auto e = [&](int b, int j) -> float& { return e_dyn[b * ep + j]; };
    constexpr int U4 = 4;
    const int stride = kWarps * rpw;

    // ---- staged layout
    const bool staged = a.staged != 0;
    const int es = a.dtype == DSPARK_DTYPE_F32 ? 4 : 2;
    const int row_bytes = r * es;
    const int nrows = v1 - v0;
    const int n_res = min(a.R, nrows);                                            // resident rows of this CTA
    const int nck = staged ? (nrows - n_res + kChunkRows - 1) / kChunkRows : 0;   // streamed chunks per step
    const int total_ck = nck * G;
    float* ustage = reinterpret_cast<float*>(wdyn + a.off_u);            // [2][A][per]
    uint8_t* res = wdyn + a.off_res;
    uint8_t* ring = wdyn + a.off_ring;
    uint64_t* bars = reinterpret_cast<uint64_t*>(wdyn + a.off_bars);     // res, full[kRing], u[2]
    uint64_t* bar_res = bars;
    uint64_t* full = bars + 1;
    uint64_t* bar_u = bars + 1 + kRing;
    const uint8_t* w2b = static_cast<const uint8_t*>(W2.w);

    int q_next = 0, u_next = 0;            // thread 0: ring chunks and U steps issued so far
    auto issue_chunk = [&](int q) {        // ring chunk q (counted over all steps) into slot q % kRing
        q_next = q + 1;
        const int cc = q % nck;
        const int row = n_res + cc * kChunkRows;
        const int rows = min(kChunkRows, nrows - row);
        uint64_t* bar = &full[q % kRing];
        tc::mbar_arrive_expect_tx(bar, (uint32_t)(rows * row_bytes));
        tc::bulk_load(ring + (size_t)(q % kRing) * kChunkRows * row_bytes, w2b + ((int64_t)v0 + row) * row_bytes,
                      (uint32_t)(rows * row_bytes), bar);
    };
    auto issue_u = [&](int step) {         // U rows of `step` into buffer step & 1
        u_next = step + 1;
        uint64_t* bar = &bar_u[step & 1];
        tc::mbar_arrive_expect_tx(bar, (uint32_t)(A * nrows * 4));
        if (nrows > 0)
            for (int b = 0; b < A; ++b)
                tc::bulk_load(ustage + ((size_t)(step & 1) * A + b) * per, a.U + ((int64_t)b * G + step) * V + v0,
                              (uint32_t)(nrows * 4), bar);
    };

    if (tid == 0) {
        s_fail = 0;
        if (staged) {
            tc::mbar_init(bar_res, 1);
            for (int i = 0; i < kRing; ++i) tc::mbar_init(&full[i], 1);
            tc::mbar_init(&bar_u[0], 1);
            tc::mbar_init(&bar_u[1], 1);
            tc::mbar_fence_init();
            // markov_w2 is a weight: requested before waiting on the previous kernel
            const int64_t bytes = (int64_t)n_res * row_bytes;
            tc::mbar_arrive_expect_tx(bar_res, (uint32_t)bytes);
            for (int64_t o = 0; o < bytes; o += kPieceBytes)
                tc::bulk_load(res + o, w2b + (int64_t)v0 * row_bytes + o,
                              (uint32_t)(bytes - o < kPieceBytes ? bytes - o : kPieceBytes), bar_res);
            for (int q = 0; q < kRing && q < total_ck; ++q) issue_chunk(q);
        }
    }
    pdl_trigger();
    pdl_wait();
    if (tid == 0 && staged) {
        issue_u(0);
        if (G > 1) issue_u(1);
    }
    for (int b = tid; b < A; b += kThreads) {
        int t = a.anchors[b];
        if (t < 0 || t >= V) {
            if (blockIdx.x == 0) atomicOr(a.status, DSPARK_DEV_BAD_TOKEN);
            t = min(max(t, 0), V - 1);
        }
        prev[b] = t;
    }
    __syncthreads();

    bool ok = true;
    for (int step = 0; step < G && ok; ++step) {
        // markov_w1 of each row's previous token
        for (int i = tid; i < A * r; i += kThreads) {
            const int b = i / r, j = i % r;
            e(b, j) = load_any(w1, (int64_t)prev[b] * r + j, a.dtype);
        }
        __syncthreads();
        float* cval = a.cand_val + (size_t)(step & 1) * nblk * A;
        int32_t* cidx = a.cand_idx + (size_t)(step & 1) * nblk * A;

        if (staged) {
            // ---------------------------------------------------- shared-memory scan
            const int nb = A;                       // <= kStagedRows
            if (!tc::mbar_wait(&bar_u[step & 1], (uint32_t)(step >> 1) & 1u, &s_fail, a.status) ||
                !tc::mbar_wait(bar_res, 0u, &s_fail, a.status)) { ok = false; break; }
            const float* us = ustage + (size_t)(step & 1) * A * per;
            float best[8];
            int bidx[8];
#pragma unroll
            for (int bb = 0; bb < 8; ++bb) { best[bb] = -INFINITY; bidx[bb] = 0x7fffffff; }
            // rows [base_row, base_row + n) of the slice, held at `src` (row_bytes apart)
            auto scan = [&](const uint8_t* src, int base_row, int n) {
                for (int i0 = wid * rpw; i0 < n; i0 += U4 * stride) {      // warp-uniform
                    int il[U4];
                    float w[U4][8];
#pragma unroll
                    for (int u = 0; u < U4; ++u) {
                        il[u] = i0 + u * stride + lane / lpr;
                        if (il[u] < n) w2_smem8(src + (size_t)il[u] * row_bytes, a.dtype, c8, w[u]);
                        else {
#pragma unroll
                            for (int j = 0; j < 8; ++j) w[u][j] = 0.f;
                        }
                    }
#pragma unroll
                    for (int bb = 0; bb < 8; ++bb) {
                        if (bb >= nb) break;
#pragma unroll
                        for (int u = 0; u < U4; ++u) {
                            float part = 0.f;
#pragma unroll
                            for (int j = 0; j < 8; ++j) part = fmaf(w[u][j], e(bb, c8 + j), part);
                            for (int o = lpr / 2; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
                            if (leader && il[u] < n) {
                                const int vl = base_row + il[u];
                                argmax_merge(best[bb], bidx[bb], us[(size_t)bb * per + vl] + part, v0 + vl);
                            }
                        }
                    }
                }
            };
            scan(res, 0, n_res);
            for (int c = 0; c < nck; ++c) {
                const int q = step * nck + c;
                if (!tc::mbar_wait(&full[q % kRing], (uint32_t)(q / kRing) & 1u, &s_fail, a.status)) { ok = false; break; }
                const int row = n_res + c * kChunkRows;
                scan(ring + (size_t)(q % kRing) * kChunkRows * row_bytes, row, min(kChunkRows, nrows - row));
                __syncthreads();                                   // the slot is free again
                if (tid == 0 && q + kRing < total_ck) issue_chunk(q + kRing);
            }
            if (!ok) break;
            write_candidates(a, best, bidx, 0, nb, cval, cidx, rv, ri);
            __syncthreads();                                       // this step's U buffer is consumed
            if (tid == 0 && step + 2 < G) issue_u(step + 2);
        } else {
            // ---------------------------------------------------- global-memory scan, rows in groups of 8
            for (int b0 = 0; b0 < A; b0 += 8) {
                const int nb = min(8, A - b0);
                float best[8];
                int bidx[8];
#pragma unroll
                for (int bb = 0; bb < 8; ++bb) { best[bb] = -INFINITY; bidx[bb] = 0x7fffffff; }
                for (int vbase = v0 + wid * rpw; vbase < v1; vbase += U4 * stride) {       // warp-uniform
                    int vv[U4];
                    float w[U4][8];
#pragma unroll
                    for (int u = 0; u < U4; ++u) {
                        vv[u] = vbase + u * stride + lane / lpr;
                        if (r > 0 && vv[u] < v1) w2_load8(W2, a.dtype, a.group, vv[u], c8, r, w[u]);
                        else {
#pragma unroll
                            for (int j = 0; j < 8; ++j) w[u][j] = 0.f;
                        }
                    }
#pragma unroll
                    for (int bb = 0; bb < 8; ++bb) {
                        if (bb >= nb) break;
                        const float* Urow = a.U + ((int64_t)(b0 + bb) * G + step) * V;
                        float uv[U4];
#pragma unroll
                        for (int u = 0; u < U4; ++u) uv[u] = (leader && vv[u] < v1) ? Urow[vv[u]] : 0.f;
#pragma unroll
                        for (int u = 0; u < U4; ++u) {
                            float part = 0.f;
                            if (r > 0) {
#pragma unroll
                                for (int j = 0; j < 8; ++j) part = fmaf(w[u][j], e(b0 + bb, c8 + j), part);
                                for (int o = lpr / 2; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
                            }
                            if (leader && vv[u] < v1) argmax_merge(best[bb], bidx[bb], uv[u] + part, vv[u]);
                        }
                    }
                }
                write_candidates(a, best, bidx, b0, nb, cval, cidx, rv, ri);
                __syncthreads();
            }
        }
        if (!grid_barrier(a.arrivals, step, nblk, a.status, &s_fail)) { ok = false; break; }
        reduce_candidates(a, cval, cidx, step, prev);
    }

    // copies still in flight land before the CTA exits (bounded)
    if (staged && tid == 0) {
        const uint64_t deadline = tc::global_timer_ns() + tc::kWaitLimitNs;
        bool drained = tc::mbar_wait_until(bar_res, 0u, deadline);
        for (int q = max(0, q_next - kRing); q < q_next && drained; ++q)
            drained = tc::mbar_wait_until(&full[q % kRing], (uint32_t)(q / kRing) & 1u, deadline);
        for (int st = max(0, u_next - 2); st < u_next && drained; ++st)
            drained = tc::mbar_wait_until(&bar_u[st & 1], (uint32_t)(st >> 1) & 1u, deadline);
        if (!drained) atomicOr(a.status, DSPARK_DEV_WAIT_TIMEOUT);
    }
}

struct Layout {
    bool staged = false;
    int R = 0, off_u = 0, off_res = 0, off_ring = 0, off_bars = 0;
    size_t smem = 0;
};

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

Layout plan_layout(const dspark_model* m, int A, int per, const float* U) {
    const Dims& d = m->d;
    Layout L;
    const size_t e_bytes = round_up((size_t)A * (d.r + 4) * sizeof(float), 128);
    L.smem = std::max<size_t>(e_bytes, 16);
    const int es = d.dtype == DSPARK_DTYPE_F32 ? 4 : 2;
    const size_t row_bytes = (size_t)d.r * es;
    // bulk copies need 16-byte aligned addresses and sizes
    const bool can = !d.quant && d.r >= 8 && A <= kStagedRows && d.V % 4 == 0 && per % 4 == 0 &&
                     row_bytes % 16 == 0 && reinterpret_cast<uintptr_t>(U) % 16 == 0 &&
                     reinterpret_cast<uintptr_t>(m->w2.w) % 16 == 0;
    if (!can) return L;
    const size_t u_bytes = round_up((size_t)2 * A * per * sizeof(float), 128);
    const size_t ring_bytes = (size_t)kRing * kChunkRows * row_bytes;
    const size_t bar_bytes = 8 * (1 + kRing + 2);
    const size_t fixed = e_bytes + u_bytes + ring_bytes + bar_bytes + 256;   // + alignment of the ring and bars
    if (fixed + row_bytes > (size_t)kSmemLimit) return L;
    const size_t R = std::min<size_t>((size_t)per, ((size_t)kSmemLimit - fixed) / row_bytes);
    Layout S;
    S.staged = true;
    S.R = (int)R;
    S.off_u = (int)e_bytes;
    S.off_res = (int)(e_bytes + u_bytes);
    S.off_ring = (int)round_up(S.off_res + R * row_bytes, 128);
    S.off_bars = (int)round_up(S.off_ring + ring_bytes, 8);
    S.smem = S.off_bars + bar_bytes;
    return S.smem <= (size_t)kSmemLimit ? S : L;
}

}  // namespace

bool walk_persistent_supported(const dspark_model* m, int A) {
    return A <= kMaxRows && m->d.r <= kMaxRank;
}

int walk_persistent_blocks(const dspark_model* m) { return m->num_sms; }

cudaError_t launch_walk_persistent(const dspark_model* m, const float* U, const int32_t* anchors, int32_t* tokens,
                                   float* cand_val, int32_t* cand_idx, uint32_t* arrivals, const int* skip, int A,
                                   cudaStream_t s) {
    const Dims& d = m->d;
    const int nblk = walk_persistent_blocks(m);
    PWalkArgs pa{};
    pa.U = U; pa.anchors = anchors; pa.tokens = tokens; pa.cand_val = cand_val; pa.cand_idx = cand_idx;
    pa.arrivals = arrivals; pa.A = A; pa.G = d.gamma; pa.V = d.V; pa.r = d.r; pa.dtype = d.dtype; pa.group = d.group;
    pa.per = (int)round_up((size_t)(d.V + nblk - 1) / nblk, 4);
    pa.status = m->ws.status;
    pa.skip = skip;
    const Layout L = plan_layout(m, A, pa.per, U);
    pa.staged = L.staged ? 1 : 0;
    pa.R = L.R; pa.off_u = L.off_u; pa.off_res = L.off_res; pa.off_ring = L.off_ring; pa.off_bars = L.off_bars;
    MatRef w2 = m->w2;
    const void* w1 = m->w1;
    void* args[] = {&pa, &w2, &w1};
    cudaError_t e = cudaFuncSetAttribute((const void*)walk_persistent_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.smem);
    if (e != cudaSuccess) return e;
    // cooperative: all CTAs co-resident, which the grid barrier needs
    e = cudaLaunchCooperativeKernel((const void*)walk_persistent_kernel, dim3(nblk), dim3(kThreads), args, L.smem, s);
    count_launches(1);
    return e;
}

}  // namespace dspark
