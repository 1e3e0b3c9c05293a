// Per-(vocabulary tile, position) statistics of the logits U, computed where U
// is produced (the lm-head GEMM's epilogue) or by a scan of U: over the tile's
// 128 vocabulary entries v and for each position m,
//   mx  = max_v U[m, v]                      arg = its lowest v
//   se  = sum_v exp(U[m, v] - mx)            (the tile's share of the logsumexp)
//   lo  = max_g (mx_g - B max_{v in g} |w2[v]|)   hi = max_g (mx_g + B max_{v in g} |w2[v]|)
// over the tile's four 32-entry groups g (mx_g: the group's maximum), where B
// |w2[v]| bounds the Markov transition bias |w2[v] . w1[p]| over every
// previous token p (Cauchy-Schwarz). lo is at most max_v (U[m, v] - B |w2[v]|)
// and hi at least max_v (U[m, v] + B |w2[v]|), so the walk's exact pruning,
// which skips every tile whose hi is below some lo, stays exact; derived from
// the group maxima, they add nothing to the per-position reduction. A warp
// holds 32 entries of a tile (one per lane) and reduces them per position; the
// four warps of a tile then merge in warp order, so both producers give
// identical results.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>
#include <math.h>

namespace dspark {

// Order-preserving float <-> uint32 (larger float, larger code); code 0 lies
// below every float, so a zero word is the identity of the maximum.
__device__ __forceinline__ uint32_t f2ord(float f) {
    const uint32_t b = __float_as_uint(f);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float ord2f(uint32_t c) {
    return __uint_as_float((c & 0x80000000u) ? (c & 0x7fffffffu) : ~c);
}
__device__ __forceinline__ uint32_t warp_max_u32(uint32_t v) {
    uint32_t r;
    asm volatile("redux.sync.max.u32 %0, %1, 0xffffffff;" : "=r"(r) : "r"(v));
    return r;
}

struct TileStats {
    float* mx = nullptr;   // [n_tiles][M]
    int* arg = nullptr;    // [n_tiles][M]
    float* se = nullptr;   // [n_tiles][M]
    float* lo = nullptr;   // [n_tiles][M] (only with the bounds)
    float* hi = nullptr;   // [n_tiles][M]
    int M = 0, n_tiles = 0;
};

// One warp's part of a tile for one position: `u` is this lane's U value
// (-inf for an entry past the vocabulary), `v` its vocabulary index and `bwmax`
// the group bound B max |w2| over the warp's 32 entries (0 without bounds). Returns the warp's results in every
// lane: keys of mx / lo / hi (0 = no entry), the lowest arg, and se relative
// to the warp's mx.
struct WarpStat {
    uint32_t kmx, klo, khi;
    int arg;
    float se;
};
__device__ __forceinline__ WarpStat warp_logit_stat(float u, int v, float bwmax, bool bounds) {
    WarpStat w;
    const bool valid = u > -INFINITY;
    w.kmx = warp_max_u32(valid ? f2ord(u) : 0u);
    const unsigned ties = __ballot_sync(0xffffffffu, valid && f2ord(u) == w.kmx);
    w.arg = ties ? __shfl_sync(0xffffffffu, v, __ffs(ties) - 1) : 0x7fffffff;
    float e = 0.f;
    if (w.kmx) e = valid ? __expf(u - ord2f(w.kmx)) : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) e += __shfl_xor_sync(0xffffffffu, e, o);
    w.se = e;
    if (bounds && w.kmx) {
        w.klo = f2ord(ord2f(w.kmx) - bwmax);
        w.khi = f2ord(ord2f(w.kmx) + bwmax);
    } else {
        w.klo = w.khi = 0u;
    }
    return w;
}

// The same reduction for 16 positions at once: this lane's values u[j] of
// positions j = 0..15 (entry v, bound bw). A transposing butterfly halves the
// positions a lane carries at each step (8, 4, 2, 1) while doubling the lanes
// they are reduced over, and a last exchange completes the warp: 16 transfers
// in 5 dependent steps instead of a full butterfly per position. Lane L ends
// with position warp_stat16_col(L) (lanes L and L ^ 1 agree).
__device__ __forceinline__ int warp_stat16_col(int lane) {
    return ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 + ((lane >> 1) & 1);
}
struct StatAcc {
    float m;     // maximum (-inf: no entry)
    int a;       // its lowest index
    float s;     // sum of exp(u - m)
};
__device__ __forceinline__ StatAcc stat_merge(const StatAcc& x, const StatAcc& y) {
    StatAcc r;
    const bool y_wins = y.m > x.m || (y.m == x.m && y.a < x.a);
    r.m = y_wins ? y.m : x.m;
    r.a = y_wins ? y.a : x.a;
    const float small = y_wins ? x.m : y.m;
    const float s_big = y_wins ? y.s : x.s, s_small = y_wins ? x.s : y.s;
    r.s = small == -INFINITY ? s_big : s_big + s_small * __expf(small - r.m);
    return r;
}
__device__ __forceinline__ StatAcc stat_shfl(const StatAcc& x, int mask) {
    StatAcc r;
    r.m = __shfl_xor_sync(0xffffffffu, x.m, mask);
    r.a = __shfl_xor_sync(0xffffffffu, x.a, mask);
    r.s = __shfl_xor_sync(0xffffffffu, x.s, mask);
    return r;
}
// With `cap` > 0 the values are softcapped logits, |u| <= cap: then exp(u - cap)
// lies in [exp(-2 cap), 1] and the sums need no rescaling (plain adds, one
// exponential per value), and each warp result is turned into a sum relative to
// its maximum once at the end. cap must stay below ~43 for exp(-2 cap) to be a
// normal fp32; larger caps (and cap = 0) take the rescaling merge.
__device__ __forceinline__ StatAcc stat_merge_fixed(const StatAcc& x, const StatAcc& y) {
    StatAcc r;
    const bool y_wins = y.m > x.m || (y.m == x.m && y.a < x.a);
    r.m = y_wins ? y.m : x.m;
    r.a = y_wins ? y.a : x.a;
    r.s = x.s + y.s;
    return r;
}
__device__ __forceinline__ WarpStat warp_logit_stat16(const float (&u)[16], int v, float bwmax, bool bounds,
                                                      float cap = 0.f) {
    const int lane = threadIdx.x & 31;
    const bool fixed = cap > 0.f && cap < 43.f;
    StatAcc x[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const bool valid = u[j] > -INFINITY;
        x[j].m = u[j];
        x[j].a = valid ? v : 0x7fffffff;
        x[j].s = valid ? (fixed ? __expf(u[j] - cap) : 1.f) : 0.f;
    }
    StatAcc f;
    if (fixed) {
#pragma unroll
        for (int half = 8, bit = 16; half >= 1; half >>= 1, bit >>= 1) {
            const bool upper = (lane & bit) != 0;
#pragma unroll
            for (int j = 0; j < half; ++j) {
                const StatAcc give = upper ? x[j] : x[j + half];
                const StatAcc keep = upper ? x[j + half] : x[j];
                x[j] = stat_merge_fixed(keep, stat_shfl(give, bit));
            }
        }
        f = stat_merge_fixed(x[0], stat_shfl(x[0], 1));
        if (f.m > -INFINITY) f.s *= __expf(cap - f.m);          // relative to the warp's maximum
    } else {
#pragma unroll
        for (int half = 8, bit = 16; half >= 1; half >>= 1, bit >>= 1) {
            const bool upper = (lane & bit) != 0;
#pragma unroll
            for (int j = 0; j < half; ++j) {
                const StatAcc give = upper ? x[j] : x[j + half];
                const StatAcc keep = upper ? x[j + half] : x[j];
                x[j] = stat_merge(keep, stat_shfl(give, bit));
            }
        }
        f = stat_merge(x[0], stat_shfl(x[0], 1));
    }
    WarpStat w;
    w.kmx = f.m > -INFINITY ? f2ord(f.m) : 0u;
    w.arg = f.m > -INFINITY ? f.a : 0x7fffffff;
    w.se = f.m > -INFINITY ? f.s : 0.f;
    w.klo = bounds && f.m > -INFINITY ? f2ord(f.m - bwmax) : 0u;
    w.khi = bounds && f.m > -INFINITY ? f2ord(f.m + bwmax) : 0u;
    return w;
}

// Merges the four warps' results of a tile (in warp order) and stores the
// tile's statistics for position m.
__device__ __forceinline__ void store_tile_stat(const TileStats& ts, int tile, int m, const WarpStat* q4) {
    uint32_t kmx = 0, klo = 0, khi = 0;
    int arg = 0x7fffffff;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        if (q4[q].kmx > kmx) { kmx = q4[q].kmx; arg = q4[q].arg; }   // strict: the lower warp keeps a tie
        klo = max(klo, q4[q].klo);
        khi = max(khi, q4[q].khi);
    }
    float se = 0.f;
    if (kmx) {
        const float mx = ord2f(kmx);
#pragma unroll
        for (int q = 0; q < 4; ++q)
            if (q4[q].kmx) se += q4[q].se * __expf(ord2f(q4[q].kmx) - mx);
    }
    const int64_t i = (int64_t)tile * ts.M + m;
    ts.mx[i] = kmx ? ord2f(kmx) : -INFINITY;
    ts.arg[i] = arg;
    ts.se[i] = se;
    if (ts.lo) {
        ts.lo[i] = klo ? ord2f(klo) : -INFINITY;
        ts.hi[i] = khi ? ord2f(khi) : -INFINITY;
    }
}

}  // namespace dspark
