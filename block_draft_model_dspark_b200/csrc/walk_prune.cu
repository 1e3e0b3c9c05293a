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

#include <algorithm>

#include "internal.h"
#include "common.cuh"
#include "logit_stats.cuh"

namespace dspark {
namespace {

constexpr int kNormThreads = 256;              // 8 warps: one markov row each
constexpr int kStatRows = 16;                  // positions per CTA of the statistics scan
constexpr int kCandThreads = 256;
constexpr int kMaxCandTiles = 256;             // tiles a position may scan (more: the full walk decides)
constexpr int kHiKeep = 8;                     // tiles' hi values a candidate thread keeps in registers
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
    // one pass over the tiles: row maximum (lowest index on ties), T, the logsumexp
    // (tiles' sums merged online to the running maximum) and the tiles' hi kept for
    // the candidate test (up to kHiKeep per thread; more are read again)
    uint32_t kbest = 0u, klo = 0u;
    int abest = 0x7fffffff;
    float sm = -INFINITY, ss = 0.f;
    float hi_keep[kHiKeep];
#pragma unroll
    for (int q = 0; q < kHiKeep; ++q) hi_keep[q] = -INFINITY;
    for (int t = tid, q = 0; t < nt; t += kCandThreads, ++q) {
        const int64_t o = (int64_t)t * M + m;
        const float mx = ts.mx[o];
        const int a = ts.arg[o];
        const float se_t = ts.se[o];
        const float lo = markov ? ts.lo[o] : -INFINITY;
        const float hi = markov ? ts.hi[o] : -INFINITY;
        const uint32_t k = mx > -INFINITY ? f2ord(mx) : 0u;
        if (k > kbest || (k == kbest && a < abest)) { kbest = k; abest = a; }
        if (lo > -INFINITY) klo = max(klo, f2ord(lo));
        if (mx > -INFINITY) {
            if (mx > sm) { ss = ss * __expf(sm - mx) + se_t; sm = mx; }
            else ss += se_t * __expf(mx - sm);
        }
#pragma unroll
        for (int qq = 0; qq < kHiKeep; ++qq) if (qq == q) hi_keep[qq] = hi;
    }
    // the CTA's maximum / argmax, T and logsumexp: warps, then warp 0 over the warps
    const uint32_t wk = warp_max_u32(kbest);
    int wa = kbest == wk ? abest : 0x7fffffff;
    for (int o = 16; o > 0; o >>= 1) wa = min(wa, __shfl_xor_sync(0xffffffffu, wa, o));
    float Tm = klo ? ord2f(klo) : -INFINITY;
    for (int o = 16; o > 0; o >>= 1) Tm = fmaxf(Tm, __shfl_xor_sync(0xffffffffu, Tm, o));
    const float wmax = wk ? ord2f(wk) : -INFINITY;
    float wsum = sm > -INFINITY ? ss * __expf(sm - wmax) : 0.f;
    for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
    if (lane == 0) { s_key[warp] = wk; s_arg[warp] = wa; s_red[warp] = Tm; s_red[16 + warp] = wsum; }
    __syncthreads();
    uint32_t rk = 0u;
    int ra = 0x7fffffff;
    for (int w = 0; w < kCandThreads / 32; ++w) {
        if (s_key[w] > rk || (s_key[w] == rk && s_arg[w] < ra)) { rk = s_key[w]; ra = s_arg[w]; }
    }
    Tm = -INFINITY;
    for (int w = 0; w < kCandThreads / 32; ++w) Tm = fmaxf(Tm, s_red[w]);
    const float rmax = rk ? ord2f(rk) : -INFINITY;
    float se = 0.f;
    for (int w = 0; w < kCandThreads / 32; ++w)
        if (s_key[w]) se += s_red[16 + w] * __expf(ord2f(s_key[w]) - rmax);
    __syncthreads();
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
    for (int t = tid, q = 0; t < nt; t += kCandThreads, ++q) {
        float hi = -INFINITY;
#pragma unroll
        for (int qq = 0; qq < kHiKeep; ++qq) if (qq == q) hi = hi_keep[qq];
        if (q >= kHiKeep) hi = ts.hi[(int64_t)t * M + m];
        if (hi >= thr) {
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

// ------------------------------------------------------------------ the walk on one warp
// The same walk for dense bf16 Markov tables, on one warp per request row: the
// lists are short (a handful of candidates per position once the norm bound
// has pruned the vocabulary), so every position's count and list are read once
// and, when all of a row's candidates fit (at most `cap`), their w2 rows, w1
// rows and U values are copied into shared memory before the first step; a step
// is then warp-synchronous (lane i evaluates candidates i, i + 32, ...; a warp
// argmax; the winner's w1 row becomes the next e), with no block barrier. Rows
// whose lists do not fit read the tables from global memory at each step.
// Values and the summation order (fp32, j ascending) are those of
// prune_walk_kernel.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(smem))),
                 "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async4(void* smem, const void* gmem) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(smem))),
                 "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

template <int R>
__global__ void __launch_bounds__(32) prune_walk_warp_kernel(const float* __restrict__ U, const bf16* __restrict__ w1,
                                                             const bf16* __restrict__ w2, int r,
                                                             const int32_t* __restrict__ anchors,
                                                             const int* __restrict__ cnt, const int* __restrict__ list,
                                                             int G, int V, int cap, int32_t* __restrict__ tokens,
                                                             int* __restrict__ fail, int32_t* __restrict__ status) {
    extern __shared__ __align__(16) uint8_t wsm[];
    constexpr int chunks = R / 8;                   // 16-byte chunks of a row (r == R)
    const int rowb = R * 2;
    const int sstride = 2 * rowb;                   // a slot: w2 row, w1 row
    int* s_cnt = reinterpret_cast<int*>(wsm);       // [G]
    int* s_off = s_cnt + 64;                        // [G + 1] exclusive prefix of the counts
    int* s_v = s_off + 72;                          // [cap]
    uint8_t* s_rows = reinterpret_cast<uint8_t*>(s_v + cap);     // [cap] slots
    float* s_u = reinterpret_cast<float*>(s_rows + (size_t)cap * sstride);   // [cap]
    float* s_e = s_u + cap;                         // [r]
    pdl_trigger();
    pdl_wait();
    const int b = blockIdx.x, lane = threadIdx.x;
    int prev = anchors[b];
    if (prev < 0 || prev >= V) {
        if (lane == 0) atomicOr(status, DSPARK_DEV_BAD_TOKEN);
        prev = min(max(prev, 0), V - 1);
    }
    // counts and their prefix (G <= 64: two per lane)
    bool bad = false;
    int c0 = 0, c1 = 0;
    if (lane < G) { c0 = cnt[b * G + lane]; bad |= c0 <= 0 || c0 > kPruneCap; }
    if (lane + 32 < G) { c1 = cnt[b * G + lane + 32]; bad |= c1 <= 0 || c1 > kPruneCap; }
    if (__any_sync(0xffffffffu, bad)) {             // a list empty or too long: the full walk decides
        if (lane == 0) atomicOr(fail, 1);
        return;
    }
    int x0 = c0, x1 = c1;                           // inclusive scans of the two halves
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y0 = __shfl_up_sync(0xffffffffu, x0, o), y1 = __shfl_up_sync(0xffffffffu, x1, o);
        if (lane >= o) { x0 += y0; x1 += y1; }
    }
    const int tot0 = __shfl_sync(0xffffffffu, x0, 31);
    if (lane < G) { s_cnt[lane] = c0; s_off[lane] = x0 - c0; }
    if (lane + 32 < G) { s_cnt[lane + 32] = c1; s_off[lane + 32] = tot0 + x1 - c1; }
    const int total = tot0 + __shfl_sync(0xffffffffu, x1, 31);
    if (lane == 0) s_off[G] = total;
    __syncwarp();
    const bool resident = total <= cap;
    if (resident) {
        // every candidate of the row, flattened (slot t = offset of its position + its list index):
        // lane l takes slots l, l + 32, ..., so all list reads go out at once; then its rows and U
        // value by cp.async
        for (int t = lane; t < total; t += 32) {
            int k = 0;
            while (k + 1 < G && s_off[k + 1] <= t) ++k;     // the position holding slot t
            const int i = t - s_off[k], m = b * G + k;
            const int v = min(max(list[(int64_t)m * kPruneCap + i], 0), V - 1);   // (in range; clamped for safety)
            s_v[t] = v;
            uint8_t* slot = s_rows + (size_t)t * sstride;
            const uint4* g2 = reinterpret_cast<const uint4*>(w2 + (int64_t)v * R);
            const uint4* g1 = reinterpret_cast<const uint4*>(w1 + (int64_t)v * R);
#pragma unroll
            for (int ch = 0; ch < chunks; ++ch) {
                cp_async16(slot + ch * 16, g2 + ch);
                cp_async16(slot + rowb + ch * 16, g1 + ch);
            }
            cp_async4(s_u + t, U + (int64_t)m * V + v);
        }
    }
    // e = w1[anchor]
#pragma unroll
    for (int j = lane; j < R; j += 32) s_e[j] = __bfloat162float(w1[(int64_t)prev * R + j]);
    cp_async_wait_all();
    __syncwarp();
    for (int k = 0; k < G; ++k) {
        const int m = b * G + k;
        const int c = s_cnt[k], off = s_off[k];
        float val = -INFINITY;
        int idx = 0x7fffffff, slot_of = -1;
        if (resident && c == 1) {
            // one candidate: it is the step's argmax whatever its bias (the list keeps every entry
            // that could win; a single valid entry wins)
            const int v = s_v[off];
            const float u = s_u[off];
            if (v >= 0 && v < V && u == u) { idx = v; slot_of = off; val = 0.f; }   // (a NaN value never wins)
        } else {
        float ev[R];                                 // e in registers for the dot products
#pragma unroll
        for (int j4 = 0; j4 < R / 4; ++j4) {
            const float4 q = reinterpret_cast<const float4*>(s_e)[j4];
            ev[4 * j4] = q.x; ev[4 * j4 + 1] = q.y; ev[4 * j4 + 2] = q.z; ev[4 * j4 + 3] = q.w;
        }
        for (int i = lane; i < c; i += 32) {
            const int v = resident ? s_v[off + i] : list[(int64_t)m * kPruneCap + i];
            if (v < 0 || v >= V) continue;
            const uint4* row = resident ? reinterpret_cast<const uint4*>(s_rows + (size_t)(off + i) * sstride)
                                        : reinterpret_cast<const uint4*>(w2 + (int64_t)v * r);
            uint4 q[chunks];
#pragma unroll
            for (int ch = 0; ch < chunks; ++ch) q[ch] = row[ch];
            float acc = 0.f;
#pragma unroll
            for (int ch = 0; ch < chunks; ++ch) {
                const uint32_t w[4] = {q[ch].x, q[ch].y, q[ch].z, q[ch].w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc = fmaf(__uint_as_float(w[j] << 16), ev[ch * 8 + 2 * j], acc);
                    acc = fmaf(__uint_as_float(w[j] & 0xffff0000u), ev[ch * 8 + 2 * j + 1], acc);
                }
            }
            const float x = (resident ? s_u[off + i] : U[(int64_t)m * V + v]) + acc;
            if (x > val || (x == val && v < idx)) { val = x; idx = v; slot_of = off + i; }
        }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, val, o);
            const int oi = __shfl_xor_sync(0xffffffffu, idx, o);
            const int os = __shfl_xor_sync(0xffffffffu, slot_of, o);
            if (ov > val || (ov == val && oi < idx)) { val = ov; idx = oi; slot_of = os; }
        }
        if (idx == 0x7fffffff) {                     // uniform over the warp
            if (lane == 0) atomicOr(fail, 1);
            return;
        }
        if (lane == 0) tokens[m] = idx;
        if (k + 1 < G) {
            __syncwarp();                            // every lane is done reading e
            if (resident) {
                const __nv_bfloat16* row1 = reinterpret_cast<const __nv_bfloat16*>(s_rows + (size_t)slot_of * sstride + rowb);
                for (int j = lane; j < R; j += 32) s_e[j] = __bfloat162float(row1[j]);
            } else {
                for (int j = lane; j < R; j += 32) s_e[j] = __bfloat162float(w1[(int64_t)idx * R + j]);
            }
            __syncwarp();
        }
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
    // dense bf16 tables: the walk with prefetched rows (a position's candidates in shared
    // memory when there are at most `cap` of them)
    const bool warp_walk = !m->w2.quant && d.dtype == DSPARK_DTYPE_BF16 && d.gamma <= 64 &&
                           (d.r == 16 || d.r == 32 || d.r == 64 || d.r == 128);
    if (warp_walk) {
        // a row's candidates stay in shared memory when at most `cap` of them: 64 KB of rows
        const size_t sstride = 4 * (size_t)d.r;
        const int cap = std::max(32, (int)((64 * 1024) / (sstride + 8)) / 32 * 32);
        const size_t smem = (64 + 72) * 4 + (size_t)cap * (4 + sstride + 4) + 4 * (size_t)d.r;
        auto kern = d.r == 16 ? prune_walk_warp_kernel<16> : d.r == 32 ? prune_walk_warp_kernel<32>
                  : d.r == 64 ? prune_walk_warp_kernel<64> : prune_walk_warp_kernel<128>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        return launch_pdl(kern, dim3(A), dim3(32), smem, s, U, static_cast<const bf16*>(m->w1),
                          static_cast<const bf16*>(m->w2.w), d.r, anchors, ps.cnt, ps.list, d.gamma, d.V, cap, tokens,
                          ps.fail, m->ws.status);
    }
    return launch_pdl(prune_walk_kernel, dim3(A), dim3(kWalkThreads), 0, s, U, w1, m->w2, d.dtype, d.group, d.r,
                      anchors, ps.cnt, ps.list, d.gamma, d.V, tokens, ps.fail, m->ws.status);
}

}  // namespace dspark
