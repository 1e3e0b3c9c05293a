// Exact pruning of the VanillaMarkov walk (DSpark draft head, "draftRows":
// tok_k = argmax_v (U[k, v] + markov_w2[v] . markov_w1[prev])).
//
// For every vocabulary entry v and every previous token p, Cauchy-Schwarz bounds
// the transition bias: |w2[v] . w1[p]| <= |w2[v]| * B with B = max_p |w1[p]|.
// So at position k the winner's value is at least T_k = max_u (U[k, u] - B |w2[u]|),
// and no v with U[k, v] + B |w2[v]| < T_k can win, whatever the previous token.
// Those bounds do not depend on the walk's sequential state, so the candidate
// list of every position is built in parallel after the lm-head; the walk itself
// then evaluates the bias of the few candidates only, one CTA per request row.
// A position whose list is empty or longer than kPruneCap hands the round to the
// full walk (walk_tc.cu), which then runs instead: the tokens are the full
// walk's argmax under either path (the list keeps a slack far above fp32
// rounding of the bias, so every entry that could win survives).
#include <math.h>

#include "internal.h"
#include "common.cuh"

namespace dspark {
namespace {

constexpr int kNormThreads = 256;              // 8 warps: one markov row each
constexpr int kScanThreads = 256;
constexpr int kScanPer = 8;                     // vocabulary entries per thread in a scan CTA
constexpr int kScanChunk = kScanThreads * kScanPer;

// Order-preserving float <-> uint32 (larger float, larger code); code 0 lies
// below every float, so a zeroed word is the identity of the maximum.
__device__ __forceinline__ uint32_t f2ord(float f) {
    const uint32_t b = __float_as_uint(f);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float ord2f(uint32_t c) {
    return __uint_as_float((c & 0x80000000u) ? (c & 0x7fffffffu) : ~c);
}

// |markov_w2[v]| for every v (times 1 + 1e-4: an upper bound of the exact norm
// despite fp32 rounding) and max_p |markov_w1[p]| (same margin), r = 64.
__global__ void __launch_bounds__(kNormThreads) markov_norms_kernel(const bf16* __restrict__ w1,
                                                                    const bf16* __restrict__ w2, int V,
                                                                    float* __restrict__ w2norm,
                                                                    uint32_t* __restrict__ w1max_bits) {
    pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int v = blockIdx.x * (kNormThreads / 32) + (threadIdx.x >> 5);
    if (v >= V) return;
    const __nv_bfloat162 a2 = reinterpret_cast<const __nv_bfloat162*>(w2 + (int64_t)v * 64)[lane];
    const __nv_bfloat162 b2 = reinterpret_cast<const __nv_bfloat162*>(w1 + (int64_t)v * 64)[lane];
    const float a0 = __low2float(a2), a1 = __high2float(a2), b0 = __low2float(b2), b1 = __high2float(b2);
    const float s2 = warp_sum(fmaf(a0, a0, a1 * a1));
    const float s1 = warp_sum(fmaf(b0, b0, b1 * b1));
    if (lane == 0) {
        w2norm[v] = sqrtf(s2) * (1.f + 1e-4f);
        atomicMax(w1max_bits, __float_as_uint(sqrtf(s1) * (1.f + 1e-4f)));   // non-negative: bits order as floats
    }
}

// T[m] = max_v (U[m, v] - B |w2[v]|): grid (vocabulary chunks, M).
__global__ void __launch_bounds__(kScanThreads) prune_max_kernel(const float* __restrict__ U,
                                                                 const float* __restrict__ w2norm,
                                                                 const uint32_t* __restrict__ w1max_bits, int V,
                                                                 uint32_t* __restrict__ T) {
    __shared__ float red[32];
    const float B = __uint_as_float(*w1max_bits);   // model constant: written at model creation
    pdl_trigger();
    pdl_wait();
    const int m = blockIdx.y;
    const int64_t row = (int64_t)m * V;
    float t = -INFINITY;
#pragma unroll
    for (int j = 0; j < kScanPer; ++j) {
        const int v = blockIdx.x * kScanChunk + j * kScanThreads + threadIdx.x;
        if (v < V) t = fmaxf(t, U[row + v] - B * w2norm[v]);
    }
    for (int o = 16; o > 0; o >>= 1) t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = t;
    __syncthreads();
    if (threadIdx.x < 32) {
        t = threadIdx.x < kScanThreads / 32 ? red[threadIdx.x] : -INFINITY;
        for (int o = 16; o > 0; o >>= 1) t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, o));
        if (threadIdx.x == 0 && t > -INFINITY) atomicMax(&T[m], f2ord(t));
    }
}

// Candidates of row m: every v with U[m, v] + B |w2[v]| >= T[m] - slack, in
// list[m][0, cap) (order arbitrary); cnt[m] counts all of them, also past cap.
__global__ void __launch_bounds__(kScanThreads) prune_select_kernel(const float* __restrict__ U,
                                                                    const float* __restrict__ w2norm,
                                                                    const uint32_t* __restrict__ w1max_bits, int V,
                                                                    const uint32_t* __restrict__ T,
                                                                    int* __restrict__ cnt, int* __restrict__ list,
                                                                    int cap) {
    const float B = __uint_as_float(*w1max_bits);
    pdl_trigger();
    pdl_wait();
    const int m = blockIdx.y;
    const uint32_t tc = T[m];
    if (tc == 0u) return;                            // no finite value in the row: the full walk decides
    float thr = ord2f(tc);
    thr -= 1e-3f + 1e-3f * fabsf(thr);               // far above the fp32 rounding of U + bias
    const int64_t row = (int64_t)m * V;
#pragma unroll
    for (int j = 0; j < kScanPer; ++j) {
        const int v = blockIdx.x * kScanChunk + j * kScanThreads + threadIdx.x;
        if (v < V && U[row + v] + B * w2norm[v] >= thr) {
            const int i = atomicAdd(&cnt[m], 1);
            if (i < cap) list[(int64_t)m * cap + i] = v;
        }
    }
}

// The walk over the candidate lists: one CTA per request row b, one thread per
// candidate. Step k: e = w1[prev]; value of candidate v = U[b, k, v] + w2[v] . e
// (fp32, j ascending); argmax with the lowest index on ties. A list that is
// empty or overflowed sets *fail and stops this row: the full walk then runs.
__global__ void __launch_bounds__(kPruneCap) prune_walk_kernel(const float* __restrict__ U,
                                                              const bf16* __restrict__ w1,
                                                              const bf16* __restrict__ w2,
                                                              const int32_t* __restrict__ anchors,
                                                              const int* __restrict__ cnt,
                                                              const int* __restrict__ list, int G, int V,
                                                              int32_t* __restrict__ tokens, int* __restrict__ fail) {
    __shared__ float e[64];
    __shared__ float rv[kPruneCap / 32];
    __shared__ int ri[kPruneCap / 32];
    __shared__ int s_prev;
    pdl_trigger();
    pdl_wait();
    const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) s_prev = min(max(anchors[b], 0), V - 1);
    __syncthreads();
    for (int k = 0; k < G; ++k) {
        const int m = b * G + k;
        const int c = cnt[m];                         // uniform over the CTA
        if (c <= 0 || c > kPruneCap) {
            if (tid == 0) atomicOr(fail, 1);
            return;
        }
        const int prev = s_prev;
        if (tid < 64) e[tid] = __bfloat162float(w1[(int64_t)prev * 64 + tid]);
        __syncthreads();
        float val = -INFINITY;
        int idx = 0x7fffffff;
        if (tid < c) {
            const int v = list[(int64_t)m * kPruneCap + tid];
            if (v >= 0 && v < V) {
                const bf16* wr = w2 + (int64_t)v * 64;
                float acc = 0.f;
#pragma unroll 16
                for (int j = 0; j < 64; ++j) acc = fmaf(__bfloat162float(wr[j]), e[j], acc);
                val = U[(int64_t)m * V + v] + acc;
                idx = v;
            }
        }
        warp_argmax(val, idx);
        if (lane == 0) { rv[warp] = val; ri[warp] = idx; }
        __syncthreads();
        if (warp == 0) {
            val = lane < kPruneCap / 32 ? rv[lane] : -INFINITY;
            idx = lane < kPruneCap / 32 ? ri[lane] : 0x7fffffff;
            warp_argmax(val, idx);
            if (lane == 0) {
                if (idx == 0x7fffffff) {
                    atomicOr(fail, 1);
                    s_prev = -1;
                } else {
                    tokens[m] = idx;
                    s_prev = idx;
                }
            }
        }
        __syncthreads();
        if (s_prev < 0) return;                       // uniform: read after the barrier
    }
}

}  // namespace

bool walk_prune_model_supported(const Dims& d) { return d.dtype == DSPARK_DTYPE_BF16 && !d.quant && d.r == 64; }

cudaError_t launch_markov_norms(const dspark_model* m, cudaStream_t s) {
    const Dims& d = m->d;
    cudaError_t e = cudaMemsetAsync(m->ws.w1max_bits, 0, sizeof(uint32_t), s);
    if (e != cudaSuccess) return e;
    const int blocks = (d.V + kNormThreads / 32 - 1) / (kNormThreads / 32);
    return launch_pdl(markov_norms_kernel, dim3(blocks), dim3(kNormThreads), 0, s, static_cast<const bf16*>(m->w1),
                      static_cast<const bf16*>(m->w2.w), d.V, m->ws.w2norm, m->ws.w1max_bits);
}

cudaError_t launch_walk_prune(const dspark_model* m, const float* U, const int32_t* anchors, int32_t* tokens, int A,
                              const PruneScratch& ps, cudaStream_t s) {
    const Dims& d = m->d;
    const int M = A * d.gamma;
    const dim3 grid((d.V + kScanChunk - 1) / kScanChunk, M);
    cudaError_t e = launch_pdl(prune_max_kernel, grid, dim3(kScanThreads), 0, s, U, m->ws.w2norm,
                               m->ws.w1max_bits, d.V, ps.T);
    if (e == cudaSuccess)
        e = launch_pdl(prune_select_kernel, grid, dim3(kScanThreads), 0, s, U, m->ws.w2norm, m->ws.w1max_bits, d.V,
                       ps.T, ps.cnt, ps.list, kPruneCap);
    if (e == cudaSuccess)
        e = launch_pdl(prune_walk_kernel, dim3(A), dim3(kPruneCap), 0, s, U, static_cast<const bf16*>(m->w1),
                       static_cast<const bf16*>(m->w2.w), anchors, ps.cnt, ps.list, d.gamma, d.V, tokens, ps.fail);
    return e;
}

}  // namespace dspark
