// The whole temperature-0 VanillaMarkov walk of a round in one launch
// (deepspec.ts #markovStepBias / #selectStep and the sequential loop of
// draftRows): for k = 0 .. gamma-1,
//   bias_b[v] = markov_w2[v] . markov_w1[prev_b];  tok_{b,k} = argmax_v(U[b,k,v] + bias_b[v]);  prev_b = tok_{b,k}
// (fp32 sum, lowest index on ties).
//
// One CTA per SM, launched cooperatively (all CTAs resident). Each CTA owns
// a fixed slice of the vocabulary. Per step every CTA scans its slice for all
// rows (markov_w2 stays in L2 across steps), writes one (value, index)
// candidate per row, and arrives on a grid barrier (a global arrival counter;
// the wait is bounded: past kWaitLimitNs it records DSPARK_DEV_WAIT_TIMEOUT
// and the kernel returns). After the barrier every CTA reduces all
// candidates in CTA order -- the same arithmetic in every CTA, so all agree
// on the step's token without a second barrier -- and takes markov_w1 of the
// new token for the next step. Candidates are double-buffered by step parity.
// The arrival counter is zeroed by the caller before the round's first kernel.
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

struct PWalkArgs {
    const float* U;            // [A, G, V]
    const int32_t* anchors;    // [A]
    int32_t* tokens;           // [A, G]
    float* cand_val;           // [2][grid][A]
    int32_t* cand_idx;         // [2][grid][A]
    uint32_t* arrivals;        // one counter, zero at entry
    int A, G, V, r, dtype, group;
    int32_t* status;
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

__global__ void __launch_bounds__(kThreads, 1)
walk_persistent_kernel(PWalkArgs a, MatRef W2, const void* __restrict__ w1) {
    extern __shared__ float e_dyn[];             // [A][r + 4]: markov_w1 of each row's previous token
    __shared__ int prev[kMaxRows];
    __shared__ float rv[kWarps][8];
    __shared__ int ri[kWarps][8];
    __shared__ int s_fail;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int G = a.G, V = a.V, r = a.r, A = a.A;
    const int nblk = gridDim.x;
    const int per = (V + nblk - 1) / nblk;
    const int v0 = blockIdx.x * per, v1 = min(V, v0 + per);
    const int lpr = r > 0 ? r / 8 : 1;      // lanes per markov_w2 row
    const int rpw = 32 / lpr;               // rows per warp step
    const int c8 = (lane % lpr) * 8;
    const bool leader = (lane % lpr) == 0;
    const int ep = r + 4;
    auto e = [&](int b, int j) -> float& { return e_dyn[b * ep + j]; };

    if (tid == 0) s_fail = 0;
    pdl_trigger();
    pdl_wait();
    for (int b = tid; b < A; b += kThreads) {
        int t = a.anchors[b];
        if (t < 0 || t >= V) {
            if (blockIdx.x == 0) atomicOr(a.status, DSPARK_DEV_BAD_TOKEN);
            t = min(max(t, 0), V - 1);
        }
        prev[b] = t;
    }
    __syncthreads();

    for (int step = 0; step < G; ++step) {
        // markov_w1 of each row's previous token
        for (int i = tid; i < A * r; i += kThreads) {
            const int b = i / r, j = i % r;
            e(b, j) = load_any(w1, (int64_t)prev[b] * r + j, a.dtype);
        }
        __syncthreads();
        float* cval = a.cand_val + (size_t)(step & 1) * nblk * A;
        int32_t* cidx = a.cand_idx + (size_t)(step & 1) * nblk * A;
        // rows in groups of 8 (registers hold the running best of each)
        for (int b0 = 0; b0 < A; b0 += 8) {
            const int nb = min(8, A - b0);
            float best[8];
            int bidx[8];
#pragma unroll
            for (int bb = 0; bb < 8; ++bb) { best[bb] = -INFINITY; bidx[bb] = 0x7fffffff; }
            constexpr int U4 = 4;
            const int stride = kWarps * rpw;
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
                cval[(size_t)blockIdx.x * A + b0 + tid] = bv;
                cidx[(size_t)blockIdx.x * A + b0 + tid] = bi;
                __threadfence();
            }
            __syncthreads();
        }
        // grid barrier: arrive, then wait (bounded) for every CTA of this step
        if (tid == 0) {
            atomicAdd(a.arrivals, 1u);
            const uint32_t target = (uint32_t)(step + 1) * (uint32_t)nblk;
            const uint64_t t0 = tc::global_timer_ns();
            while (atomicAdd(a.arrivals, 0u) < target) {
                if (tc::global_timer_ns() - t0 > tc::kWaitLimitNs) {
                    atomicOr(a.status, DSPARK_DEV_WAIT_TIMEOUT);
                    s_fail = 1;
                    break;
                }
                __nanosleep(64);
            }
            __threadfence();
        }
        __syncthreads();
        if (s_fail) return;
        // every CTA reduces all candidates in CTA order (identical result everywhere)
        for (int b = wid; b < A; b += kWarps) {
            float bv = -INFINITY;
            int bi = 0x7fffffff;
            for (int c = lane; c < nblk; c += 32) {
                const float cv = __ldcg(&cval[(size_t)c * A + b]);
                const int ci = __ldcg(&cidx[(size_t)c * A + b]);
                argmax_merge(bv, bi, cv, ci);
            }
            warp_argmax(bv, bi);
            if (lane == 0) {
                if (bi < 0 || bi >= V) {        // only if a row was all NaN
                    if (blockIdx.x == 0) atomicOr(a.status, DSPARK_DEV_BAD_TOKEN);
                    bi = 0;
                }
                prev[b] = bi;
                if (blockIdx.x == 0) a.tokens[b * G + step] = bi;
            }
        }
        __syncthreads();
    }
}

}  // namespace

bool walk_persistent_supported(const dspark_model* m, int A) {
    return A <= kMaxRows && m->d.r <= kMaxRank;
}

int walk_persistent_blocks(const dspark_model* m) { return m->num_sms; }

cudaError_t launch_walk_persistent(const dspark_model* m, const float* U, const int32_t* anchors, int32_t* tokens,
                                   float* cand_val, int32_t* cand_idx, uint32_t* arrivals, int A, cudaStream_t s) {
    const Dims& d = m->d;
    PWalkArgs pa{};
    pa.U = U; pa.anchors = anchors; pa.tokens = tokens; pa.cand_val = cand_val; pa.cand_idx = cand_idx;
    pa.arrivals = arrivals; pa.A = A; pa.G = d.gamma; pa.V = d.V; pa.r = d.r; pa.dtype = d.dtype; pa.group = d.group;
    pa.status = m->ws.status;
    MatRef w2 = m->w2;
    const void* w1 = m->w1;
    void* args[] = {&pa, &w2, &w1};
    const size_t smem = (size_t)A * (d.r + 4) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute((const void*)walk_persistent_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)std::max<size_t>(smem, 1));
    if (e != cudaSuccess) return e;
    // cooperative: all CTAs co-resident, which the grid barrier needs
    e = cudaLaunchCooperativeKernel((const void*)walk_persistent_kernel, dim3(walk_persistent_blocks(m)),
                                    dim3(kThreads), args, smem, s);
    count_launches(1);
    return e;
}

}  // namespace dspark
