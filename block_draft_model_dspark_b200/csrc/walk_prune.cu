// Exact pruning of the VanillaMarkov walk (DSpark draft head, "draftRows":
// tok_k = argmax_v (U[k, v] + markov_w2[v] . markov_w1[prev])).
//
// For every vocabulary entry v and every previous token p, Cauchy-Schwarz bounds
// the transition bias: |w2[v] . w1[p]| <= |w2[v]| * B with B = max_p |w1[p]|.
// So at position k the winner's value is at least T_k = max_u (U[k, u] - B |w2[u]|),
// and no v with U[k, v] + B |w2[v]| < T_k can win, whatever the previous token.
// Those bounds do not depend on the walk's sequential state, so the candidate
// list of every position is built in parallel after the lm-head, and the walk
// then evaluates the bias of the few candidates only, one CTA per request row.
//
// The lists come from per-(128-entry vocabulary tile, position) statistics
// of U (logit_stats.cuh), which the tensor-core lm-head writes in its
// epilogue (tile_stats_kernel computes the same from U for the CUDA-core
// lm-heads): T_k is the maximum of the tiles' lo values, and only tiles whose
// hi value reaches T_k are scanned for candidates. The same statistics give
// every position's maximum, argmax and logsumexp of U (telemetry; with
// markov_rank 0 the argmax is the token).
//
// A position whose list is empty or longer than kPruneCap hands the round to
// the full walk (walk_tc.cu, walk_persistent.cu or walk.cu), which then runs
// instead: the tokens are the full walk's argmax under either path (the list
// keeps a slack far above fp32 rounding of the bias, so every entry that could
// win survives).
#include <math.h>

#include "internal.h"
#include "common.cuh"
#include "logit_stats.cuh"

namespace dspark {
namespace {

constexpr int kNormThreads = 256;              // 8 warps: one markov row each
constexpr int kStatRows = 16;                  // positions per CTA of the statistics scan
constexpr int kCandThreads = 256;
constexpr int kMaxCandTiles = 256;             // tiles a position may scan (more: the full walk decides)
constexpr int kWalkThreads = 256;
constexpr int kPerThread = kPruneCap / kWalkThreads;

// Eight consecutive values W[v, c8 .. c8+7] of a dense (T) or 4-bit table with rows of r.
__device__ __forceinline__ void row8(const MatRef& W, int dtype, int group, int64_t v, int c8, int r, float w[8]) {
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

// |markov_w2[v]| for every v (times 1 + 1e-4: an upper bound of the exact norm
// despite fp32 rounding) and max_p |markov_w1[p]| (same margin). One warp per
// row; lane i holds the row's 8-wide chunk i (r <= 256).
__global__ void __launch_bounds__(kNormThreads) markov_norms_kernel(MatRef w1, MatRef w2, int dtype, int group, int V,
                                                                    int r, float* __restrict__ w2norm,
                                                                    uint32_t* __restrict__ w1max_bits) {
    pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int v = blockIdx.x * (kNormThreads / 32) + (threadIdx.x >> 5);
    if (v >= V) return;
    float s2 = 0.f, s1 = 0.f;
    if (lane * 8 < r) {
        float a[8], b[8];
        row8(w2, dtype, group, v, lane * 8, r, a);
        row8(w1, dtype, group, v, lane * 8, r, b);
#pragma unroll
        for (int j = 0; j < 8; ++j) { s2 = fmaf(a[j], a[j], s2); s1 = fmaf(b[j], b[j], s1); }
    }
    s2 = warp_sum(s2);
    s1 = warp_sum(s1);
    if (lane == 0) {
        w2norm[v] = sqrtf(s2) * (1.f + 1e-4f);
        atomicMax(w1max_bits, __float_as_uint(sqrtf(s1) * (1.f + 1e-4f)));   // non-negative: bits order as floats
    }
}

// The tile statistics of U by a scan (for lm-heads without the tensor-core
// epilogue): grid (tiles, ceil(M / kStatRows)), 128 threads = the tile's entries.
__global__ void __launch_bounds__(128) tile_stats_kernel(const float* __restrict__ U, int V, int M, TileStats ts,
                                                          const float* __restrict__ w2norm,
                                                          const uint32_t* __restrict__ w1max_bits) {
    __shared__ WarpStat q4[4][kStatRows];
    const bool bounds = w2norm != nullptr;
    const float B = bounds ? __uint_as_float(*w1max_bits) : 0.f;   // model constant (written at model creation)
    pdl_trigger();
    pdl_wait();
    const int t = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int v = t * 128 + threadIdx.x;
    const float bw = bounds && v < V ? B * w2norm[v] : 0.f;
    // the epilogue's reduction: 16 positions at once
    const int m0 = blockIdx.y * kStatRows;
    float u[kStatRows];
#pragma unroll
    for (int j = 0; j < kStatRows; ++j) {
        const int m = m0 + j;
        u[j] = (v < V && m < M) ? U[(int64_t)m * V + v] : -INFINITY;
    }
    const float bwmax = bounds ? __uint_as_float(warp_max_u32(__float_as_uint(bw))) : 0.f;
    const WarpStat w = warp_logit_stat16(u, v, bwmax, bounds);
    if ((lane & 1) == 0) q4[warp][warp_stat16_col(lane)] = w;
    __syncthreads();
    if (threadIdx.x < kStatRows && m0 + threadIdx.x < M) {
        const WarpStat q[4] = {q4[0][threadIdx.x], q4[1][threadIdx.x], q4[2][threadIdx.x], q4[3][threadIdx.x]};
        store_tile_stat(ts, t, m0 + threadIdx.x, q);
    }
}

// One position m per CTA: the row's maximum, argmax and logsumexp from the tile
// statistics; with the Markov head, T_m and the candidate list (every v with
// U[m, v] + B |w2[v]| >= T_m - slack, order arbitrary; cnt[m] counts them all,
// also past cap); without it, the argmax is the token.
__global__ void __launch_bounds__(kCandThreads) prune_candidates_kernel(const float* __restrict__ U, int V, TileStats ts,
                                                                        const float* __restrict__ w2norm,
                                                                        const uint32_t* __restrict__ w1max_bits,
                                                                        int* __restrict__ cnt, int* __restrict__ list,
                                                                        int cap, int* __restrict__ fail,
                                                                        int32_t* __restrict__ tokens,
                                                                        LogitRowStat* __restrict__ row_out) {
    __shared__ uint32_t s_key[kCandThreads / 32];
    __shared__ int s_arg[kCandThreads / 32];
    __shared__ float s_red[32];
    __shared__ int s_tiles[kMaxCandTiles];
    __shared__ int s_nt, s_cnt;
    const bool markov = w2norm != nullptr;
    const float B = markov ? __uint_as_float(*w1max_bits) : 0.f;
    pdl_trigger();
    pdl_wait();
    const int m = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int M = ts.M, nt = ts.n_tiles;
    if (m == 0 && tid == 0) *fail = 0;
    if (tid == 0) { s_nt = 0; s_cnt = 0; }
    // row maximum (lowest index on ties) and T
    uint32_t kbest = 0u, klo = 0u;
    int abest = 0x7fffffff;
    for (int t = tid; t < nt; t += kCandThreads) {
        const float mx = ts.mx[(int64_t)t * M + m];
        const uint32_t k = mx > -INFINITY ? f2ord(mx) : 0u;
        const int a = ts.arg[(int64_t)t * M + m];
        if (k > kbest || (k == kbest && a < abest)) { kbest = k; abest = a; }
        if (markov) {
            const float lo = ts.lo[(int64_t)t * M + m];
            if (lo > -INFINITY) klo = max(klo, f2ord(lo));
        }
    }
    const uint32_t wk = warp_max_u32(kbest);
    int wa = kbest == wk ? abest : 0x7fffffff;
    for (int o = 16; o > 0; o >>= 1) wa = min(wa, __shfl_xor_sync(0xffffffffu, wa, o));
    if (lane == 0) { s_key[warp] = wk; s_arg[warp] = wa; }
    const float Tm_partial = klo ? ord2f(klo) : -INFINITY;
    float Tm = Tm_partial;
    for (int o = 16; o > 0; o >>= 1) Tm = fmaxf(Tm, __shfl_xor_sync(0xffffffffu, Tm, o));
    if (lane == 0) s_red[warp] = Tm;
    __syncthreads();
    uint32_t rk = 0u;
    int ra = 0x7fffffff;
    for (int w = 0; w < kCandThreads / 32; ++w) {
        if (s_key[w] > rk || (s_key[w] == rk && s_arg[w] < ra)) { rk = s_key[w]; ra = s_arg[w]; }
    }
    Tm = -INFINITY;
    for (int w = 0; w < kCandThreads / 32; ++w) Tm = fmaxf(Tm, s_red[w]);
    const float rmax = rk ? ord2f(rk) : -INFINITY;
    __syncthreads();
    // logsumexp: the tiles' sums rescaled to the row maximum
    float se = 0.f;
    if (rk)
        for (int t = tid; t < nt; t += kCandThreads) {
            const float mx = ts.mx[(int64_t)t * M + m];
            if (mx > -INFINITY) se += ts.se[(int64_t)t * M + m] * __expf(mx - rmax);
        }
    se = block_sum(se, s_red);
    if (!markov) {
        if (tid == 0) {
            tokens[m] = ra == 0x7fffffff ? 0 : ra;
            cnt[m] = ra == 0x7fffffff ? 0 : 1;
            if (row_out) row_out[m] = LogitRowStat{rmax, rmax + logf(se), ra, 1};
        }
        return;
    }
    // candidate tiles, then their entries
    if (!(Tm > -INFINITY)) {               // no finite value in the row: the full walk decides
        if (tid == 0) {
            cnt[m] = 0;
            if (row_out) row_out[m] = LogitRowStat{rmax, rmax + logf(se), ra, 0};
        }
        return;
    }
    const float thr = Tm - (1e-3f + 1e-3f * fabsf(Tm));   // far above the fp32 rounding of U + bias
    for (int t = tid; t < nt; t += kCandThreads) {
        if (ts.hi[(int64_t)t * M + m] >= thr) {
            const int i = atomicAdd(&s_nt, 1);
            if (i < kMaxCandTiles) s_tiles[i] = t;
        }
    }
    __syncthreads();
    const int ntl = s_nt;
    if (ntl <= kMaxCandTiles) {
        for (int idx = tid; idx < ntl * 128; idx += kCandThreads) {
            const int v = s_tiles[idx >> 7] * 128 + (idx & 127);
            if (v < V && U[(int64_t)m * V + v] + B * w2norm[v] >= thr) {
                const int i = atomicAdd(&s_cnt, 1);
                if (i < cap) list[(int64_t)m * cap + i] = v;
            }
        }
    }
    __syncthreads();
    if (tid == 0) {
        const int c = ntl <= kMaxCandTiles ? s_cnt : cap + 1;
        cnt[m] = c;
        if (row_out) row_out[m] = LogitRowStat{rmax, rmax + logf(se), ra, c};
    }
}

// The walk over the candidate lists: one CTA per request row b, each thread
// evaluating up to kPerThread candidates. Step k: e = w1[prev]; value of
// candidate v = U[b, k, v] + w2[v] . e (fp32, j ascending); argmax with the
// lowest index on ties. A list that is empty or overflowed sets *fail and
// stops this row: the full walk then runs.
__global__ void __launch_bounds__(kWalkThreads) prune_walk_kernel(const float* __restrict__ U, MatRef w1, MatRef w2,
                                                                  int dtype, int group, int r,
                                                                  const int32_t* __restrict__ anchors,
                                                                  const int* __restrict__ cnt,
                                                                  const int* __restrict__ list, int G, int V,
                                                                  int32_t* __restrict__ tokens, int* __restrict__ fail,
                                                                  int32_t* __restrict__ status) {
    __shared__ float e[256];
    __shared__ float rv[kWalkThreads / 32];
    __shared__ int ri[kWalkThreads / 32];
    __shared__ int s_prev;
    pdl_trigger();
    pdl_wait();
    const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) {
        int a = anchors[b];
        if (a < 0 || a >= V) {
            atomicOr(status, DSPARK_DEV_BAD_TOKEN);
            a = min(max(a, 0), V - 1);
        }
        s_prev = a;
    }
    __syncthreads();
    for (int k = 0; k < G; ++k) {
        const int m = b * G + k;
        const int c = cnt[m];                         // uniform over the CTA
        if (c <= 0 || c > kPruneCap) {
            if (tid == 0) atomicOr(fail, 1);
            return;
        }
        const int prev = s_prev;
        if (tid * 8 < r) {
            float w[8];
            row8(w1, dtype, group, prev, tid * 8, r, w);
#pragma unroll
            for (int j = 0; j < 8; ++j) e[tid * 8 + j] = w[j];
        }
        __syncthreads();
        float val = -INFINITY;
        int idx = 0x7fffffff;
#pragma unroll
        for (int q = 0; q < kPerThread; ++q) {
            const int i = tid + q * kWalkThreads;
            if (i < c) {
                const int v = list[(int64_t)m * kPruneCap + i];
                if (v >= 0 && v < V) {
                    float acc = 0.f;
                    for (int c8 = 0; c8 < r; c8 += 8) {
                        float w[8];
                        row8(w2, dtype, group, v, c8, r, w);
#pragma unroll
                        for (int j = 0; j < 8; ++j) acc = fmaf(w[j], e[c8 + j], acc);
                    }
                    argmax_merge(val, idx, U[(int64_t)m * V + v] + acc, v);
                }
            }
        }
        warp_argmax(val, idx);
        if (lane == 0) { rv[warp] = val; ri[warp] = idx; }
        __syncthreads();
        if (warp == 0) {
            val = lane < kWalkThreads / 32 ? rv[lane] : -INFINITY;
            idx = lane < kWalkThreads / 32 ? ri[lane] : 0x7fffffff;
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

bool walk_prune_model_supported(const Dims& d) { return d.r > 0 && d.r <= 256; }

cudaError_t launch_markov_norms(const dspark_model* m, cudaStream_t s) {
    const Dims& d = m->d;
    cudaError_t e = cudaMemsetAsync(m->ws.w1max_bits, 0, sizeof(uint32_t), s);
    if (e != cudaSuccess) return e;
    MatRef w1{};
    w1.w = m->w1; w1.n = d.V; w1.k = d.r;
    const int blocks = (d.V + kNormThreads / 32 - 1) / (kNormThreads / 32);
    return launch_pdl(markov_norms_kernel, dim3(blocks), dim3(kNormThreads), 0, s, w1, m->w2, d.dtype, d.group, d.V,
                      d.r, m->ws.w2norm, m->ws.w1max_bits);
}

cudaError_t launch_tile_stats(const dspark_model* m, const float* U, int M, const TileStats& ts, cudaStream_t s) {
    const Dims& d = m->d;
    const dim3 grid(ts.n_tiles, (M + kStatRows - 1) / kStatRows);
    return launch_pdl(tile_stats_kernel, grid, dim3(128), 0, s, U, d.V, M, ts, d.r > 0 ? m->ws.w2norm : nullptr,
                      m->ws.w1max_bits);
}

cudaError_t launch_walk_prune(const dspark_model* m, const float* U, const TileStats& ts, const int32_t* anchors,
                              int32_t* tokens, int A, const PruneScratch& ps, LogitRowStat* row_out, cudaStream_t s) {
    const Dims& d = m->d;
    const int M = A * d.gamma;
    const bool markov = d.r > 0;
    cudaError_t e = launch_pdl(prune_candidates_kernel, dim3(M), dim3(kCandThreads), 0, s, U, d.V, ts,
                               markov ? m->ws.w2norm : nullptr, m->ws.w1max_bits, ps.cnt, ps.list, kPruneCap,
                               ps.fail, tokens, row_out);
    if (e != cudaSuccess || !markov) return e;
    MatRef w1{};
    w1.w = m->w1; w1.n = d.V; w1.k = d.r;
    return launch_pdl(prune_walk_kernel, dim3(A), dim3(kWalkThreads), 0, s, U, w1, m->w2, d.dtype, d.group, d.r,
                      anchors, ps.cnt, ps.list, d.gamma, d.V, tokens, ps.fail, m->ws.status);
}

}  // namespace dspark
