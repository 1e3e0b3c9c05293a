// The VanillaMarkov walk at temperature 0 (deepspec.ts #markovStepBias,
// #selectStep and the sequential loop of draftRows): for step k,
//   bias_b[v] = markov_w2[v] . markov_w1[prev_b]        (rank-r GEMV over the vocabulary)
//   tok_{b,k} = argmax_v (U[b,k,v] + bias_b[v])          (lowest index on ties)
//   prev_b    = tok_{b,k}
// The sum is taken in fp32. One launch per step: every CTA scans a slice of
// the vocabulary for all rows and writes its (value, index) candidates; the
// last CTA to finish (a ticket counter, not a value atomic) reduces the
// candidates in CTA order and commits the step's tokens, so the result does
// not depend on scheduling.
#include <math.h>

#include "internal.h"
#include "common.cuh"

namespace dspark {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxRank = 256;

__device__ __forceinline__ float w2_at(const MatRef& W, int dtype, int group, int64_t v, int j) {
    if (!W.quant) return load_any(W.w, v * W.k + j, dtype);
    const uint32_t w = static_cast<const uint32_t*>(W.w)[v * (W.k / 8) + j / 8];
    const int64_t g = v * (W.k / group) + j / group;
    return fmaf(__bfloat162float(W.scales[g]), (float)((w >> (4 * (j % 8))) & 0xFu), __bfloat162float(W.biases[g]));
}

__global__ void walk_init_kernel(const int32_t* anchors, int32_t* prev, uint32_t* ticket, int A, int V,
                                 int32_t* status) {
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

__global__ void __launch_bounds__(kThreads)
walk_step_kernel(WalkArgs a, MatRef W2, const void* __restrict__ w1, int dtype, int group, int G, int V, int r) {
    __shared__ float e[kMaxRank];
    __shared__ float rv[32];
    __shared__ int ri[32];
    __shared__ bool last;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int per = (V + gridDim.x - 1) / gridDim.x;
    const int v0 = blockIdx.x * per, v1 = min(V, v0 + per);

    for (int b = 0; b < a.A; ++b) {
        const int pb = a.prev[b];
        for (int j = tid; j < r; j += kThreads) e[j] = load_any(w1, (int64_t)pb * r + j, dtype);
        __syncthreads();
        float best = -INFINITY;
        int bi = 0x7fffffff;
        const float* Urow = a.U + ((int64_t)b * G + a.step) * V;
        for (int v = v0 + tid; v < v1; v += kThreads) {
            float s = Urow[v];
            float bias = 0.f;
            for (int j = 0; j < r; ++j) bias = fmaf(e[j], w2_at(W2, dtype, group, v, j), bias);
            s += bias;
            argmax_merge(best, bi, s, v);
        }
        warp_argmax(best, bi);
        if (lane == 0) { rv[wid] = best; ri[wid] = bi; }
        __syncthreads();
        if (wid == 0) {
            best = lane < kThreads / 32 ? rv[lane] : -INFINITY;
            bi = lane < kThreads / 32 ? ri[lane] : 0x7fffffff;
            warp_argmax(best, bi);
            if (lane == 0) {
                a.part_val[(int64_t)blockIdx.x * a.A + b] = best;
                a.part_idx[(int64_t)blockIdx.x * a.A + b] = bi;
            }
        }
        __syncthreads();
    }

    // ticket: the last CTA reduces all candidates in CTA order
    __threadfence();
    if (tid == 0) last = atomicAdd(a.ticket, 1u) == gridDim.x - 1;
    __syncthreads();
    if (!last) return;
    __threadfence();
    for (int b = wid; b < a.A; b += kThreads / 32) {
        float best = -INFINITY;
        int bi = 0x7fffffff;
        for (int c = lane; c < (int)gridDim.x; c += 32)
            argmax_merge(best, bi, a.part_val[(int64_t)c * a.A + b], a.part_idx[(int64_t)c * a.A + b]);
        warp_argmax(best, bi);
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

cudaError_t launch_walk_init(const int32_t* anchors, int32_t* prev, uint32_t* ticket, int A, int V, int32_t* status,
                             cudaStream_t s) {
    walk_init_kernel<<<(A + 127) / 128, 128, 0, s>>>(anchors, prev, ticket, A, V, status);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_walk_step(const dspark_model* m, const WalkArgs& a, cudaStream_t s) {
    const Dims& d = m->d;
    walk_step_kernel<<<a.nblk, kThreads, 0, s>>>(a, m->w2, m->w1, d.dtype, d.group, d.gamma, d.V, d.r);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace dspark
