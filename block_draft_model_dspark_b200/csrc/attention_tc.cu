// KV-injection attention on tcgen05 tensor cores: the
// DeepspecContextAttention.attend seam ("mlx-bun 0.2.0 -> 0.4.0" page 75,
// plainDeepspecContext): the block queries of one row attend, non-causally
// and at scale 1.0, over the row's cached context keys followed by the
// block's own keys; GQA maps query head h to kv head h / (nH / nKv).
//
// One CTA = a range of key tiles of one item (row b, kv head g), as the work
// plan assigns them from the device-side lengths (ragged rows get CTAs in
// proportion to their tiles; every CTA runs in one wave); every CTA computes
// the plan itself from the lengths, so no plan kernel precedes it. Its query tile is the
// 128-row MMA side: the grp * gamma queries of the heads that share kv head g
// (row r = query i * grp + head-in-group), in tensor memory as the S product's
// A operand (two fp16 values per 32-bit column). Key tiles of KT = 64 rows are
// TMA-loaded from the fp16 cache (4-D maps pick kv head g out of [rows, nKv,
// hd]) and multiplied as they land: both MMAs run as kind::f16 with fp16
// operands (q and the probabilities P keep an 11-bit significand).
//   S = Q K^T  -> TMEM, two 64-column buffers (tile t in buffer t % 2)
//   softmax    -> one thread per query row (TMEM lane = row); the running max
//                 is raised only when a tile's max exceeds it by more than
//                 kRescale, so O is rarely rescaled in TMEM
//   O += P V   -> TMEM (hd columns), P fp16 from shared memory (K-major,
//                 128-byte swizzle), V as an MN-major operand
// TMEM columns: S buffers [0, 128), O [128, 128 + hd), Q [384, 384 + hd / 2).
// K and V tiles have 3 shared-memory slots each, so three tiles' loads are in
// flight; per 64 keys at hd = 256 the tensor cores run 16 (S) + 4 (P V) MMAs.
//
// Warp roles (224 threads): warps 0-3 run the softmax, one thread per query
// row (TMEM lane), all 64 columns of a tile, no exchange between threads; warp 4
// issues the S products and K loads, warp 5 the P V products and V loads, and
// warp 6 zeroes the V rows past the last key of a partial tile before its
// product (stale cache rows may hold any bits, and P = 0 times NaN still
// poisons the accumulator; K needs no fix: those S columns are masked to
// -inf). Tile t + 1's S product and tile t - 1's P V product overlap tile t's
// softmax; the softmax waits for P V of tile t - 1 only to rescale O (rare).
// Every wait is bounded. Shared memory at hd = 256: K, V 3 x 32 KB each, P 2 x 16 KB.
//
// V-only cache (attention_k_eq_v: k and v come from one k_proj row and one
// normalisation, so k = rope(v * k_norm) row by row, and the cache can hold v
// alone): only V tiles are loaded, half the bytes, and eight more warps (6-13,
// 448 threads) rebuild each tile's K into a K slot as it lands, in fp16:
// x = v * k_norm, k1 = x1 cos - x2 sin, k2 = x2 cos + x1 sin for every RoPE pair
// (i, i + hd / 2) at the key's position (pos0[b] + t for context row t,
// block_pos[b] + i for block row i), the products and the rotation on packed
// fp16 (the keys are rounded to fp16 anyway), the angles in fp32. A builder
// thread owns 8 pairs of 4 keys; it starts from the angle of its first key's
// position (reduced in double) and turns it by theta per key and by 64 theta
// per tile (one complex product each, so the rounding of a tile's angles grows
// with the tiles a CTA walks, a few 1e-7 per tile, far below fp16's 2^-11). The
// V rows past the last key are zeroed by the same threads. The S product then
// reads the rebuilt K tile as it would a loaded one. A rebuilt K tile lives
// only from its build to its S product, so the six tile slots split 4 V + 2 K
// (four V loads in flight, where a K+V cache keeps three of each).
//
// An item on one CTA writes its output straight from tensor memory. Otherwise
// each CTA writes its normalised O / l (fp16) with (max, sum) per query row into
// its own slot, and the merge kernel (one or two warps per output row, over the
// whole GPU) combines the item's slots in slot order. The last range of each (b, g) also
// takes the block's own keys, as one more tile.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <mutex>
#include <type_traits>

#include "internal.h"
#include "common.cuh"
#include "tc_ptx.cuh"

namespace dspark {

namespace tc {
namespace {

// threads: warps 0-6; a V-only cache adds the K builders, warps 6-9 (warp 6 then builds too)
constexpr int kBuildWarps = 8;       // V-only: warps 6 .. 13 rebuild K from the V tiles
constexpr int kBuildKeys = 4;        // keys per builder thread and tile
template <bool VONLY> struct AttnThreads { static constexpr int n = VONLY ? 192 + 32 * kBuildWarps : 224; };
constexpr int kSoftThreads = 128;    // warps 0-3: one thread per query row
constexpr int kIssuerWarp = 4;       // S products and K loads; warp 5: P V products and V loads
constexpr int kFixWarp = 6;          // zeroes the V rows past the last key of a partial tile
constexpr int KT = 64;               // keys per tile
// Shared-memory tile slots (6 tiles in all): a K+V cache loads both, 3 K and 3 V
// slots; a V-only cache loads V alone and rebuilds each K tile just before its S
// product, so 4 V slots keep four loads in flight and 2 K slots suffice.
constexpr int kSlotsMax = 4;
template <bool VONLY> struct AttnSlots { static constexpr int k = VONLY ? 2 : 3, v = VONLY ? 4 : 3; };
constexpr int kQCol = 2 * KT + 256;  // TMEM columns: S buffers [0, 2 KT), O [2 KT, 2 KT + hd), Q from 384
constexpr int QROWS = 128;           // MMA M
// Natural-log headroom before the running max is raised: P = exp(s - m_run) stays
// below e^10 = 22026, inside fp16's range (65504) at fp16's relative precision.
constexpr float kRescale = 10.0f;

struct AttnTcParams {
    int A, G, nH, nKv, grp, hd, capacity, q_dtype, grid;
    const void* q;                   // [A, G, nH, hd] fp16
    const int32_t* len;
    __half* part_o; float* part_ml;  // one slot per CTA: [CTA][128 rows][hd] (O / l) and [CTA][128 rows][2] (m, l)
    int* item_slots;                 // [A * nKv][2]: the item's first slot and its number of slots
    void* out; int out_dtype;        // [A, G, nH, hd] fp32 or fp16
    __half* out_hi; __half* out_lo;  // optional fp16 pair of the output (the next GEMM's input)
    int32_t* status;
    // V-only cache: K rebuilt from the V tiles at the keys' positions
    const int32_t* pos0;             // [A] position of cache row 0
    const int32_t* block_pos;        // [A] position of block row 0
    const __nv_bfloat16* k_norm;     // [hd]
    const double* inv_freq;          // [hd / 2]
};

// The work plan (device lengths): item i = (row b, kv head g) has n_i =
// ceil(len_b / KT) context tiles plus the block tile. The smallest q >= 2 with
// sum_i ceil(n_i / q) <= grid splits item i into k_i = ceil(n_i / q) equal
// tile ranges, one CTA each (all CTAs in one wave, none above q tiles; a CTA
// also builds its query tile and writes a 128-row state, so q = 1 does not
// pay); the CTAs of item i are the exclusive prefix sum of k_i onwards.
__device__ __forceinline__ int plan_tiles(const int32_t* len, int b, int capacity) {
    const int L = min(max(len[b], 0), capacity);
    return (L + KT - 1) / KT + 1;
}
// Sum (or maximum) over the block of NW warps; `buf` holds NW ints and callers
// alternate two buffers, so one barrier per reduction suffices.
template <int NW>
__device__ __forceinline__ int block_reduce_int(int v, int* buf, bool is_max) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const int y = __shfl_xor_sync(0xffffffffu, v, o);
        v = is_max ? max(v, y) : v + y;
    }
    if (lane == 0) buf[wid] = v;
    __syncthreads();
    int t = is_max ? buf[0] : 0;
    for (int w = is_max ? 1 : 0; w < NW; ++w) t = is_max ? max(t, buf[w]) : t + buf[w];
    return t;
}
struct CtaWork {
    int item;        // -1: idle
    int t0, t1;      // tile range within the item
    int s0, k;       // the item's first CTA (slot) and its number of CTAs
};
// ceil(n / q) for 0 <= n, 1 <= q below 2^20, from a float reciprocal of q
// (off by at most one before the correction).
__device__ __forceinline__ int ceil_div_small(int n, int q, float rq) {
    const int a = n + q - 1;
    int c = __float2int_rz((float)a * rq);
    if (c * q > a) --c;
    else if ((c + 1) * q <= a) ++c;
    return c;
}
// This CTA's share of the plan, by all threads of the block (every CTA computes
// the same plan). Items (b, g) of one row b have the same n_b, so the plan works
// on rows: n_b cached in `ncache` (A ints of shared memory), the smallest
// feasible q found by testing up to kThreads candidates at once (each thread
// sums nKv * ceil(n_b / q) over the rows for its candidate; two rounds at most
// for n up to kThreads^2), then a scan of k_b over the rows places the CTA.
// `sh` holds 2 kWarps + 5 ints. kThreads: the block's threads.
template <int kThreads>
__device__ CtaWork cta_work(const int32_t* __restrict__ len, int A, int nKv, int capacity, int grid, int slot,
                            int* sh, int* ncache) {
    constexpr int kWarps = kThreads / 32;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    int* res = sh + 2 * kWarps;                      // item, index within the item, n, k, first slot
    if (tid == 0) res[0] = -1;                       // ordered before the scan by the barriers below
    int nb = 0;
    int mx = 1;
    for (int b = tid; b < A; b += kThreads) {
        const int n = plan_tiles(len, b, capacity);
        ncache[b] = n;
        mx = max(mx, n);
    }
    mx = block_reduce_int<kWarps>(mx, sh + (nb++ & 1) * kWarps, true);   // also publishes ncache
    int q = mx;                                      // q = mx is feasible: A * nKv <= grid
    if (A * nKv < grid) {
        int lo = min(2, mx), hi = mx;                // the answer lies in [lo, hi]; hi is feasible
        while (lo < hi) {
            const int step = (hi - lo + kThreads - 1) / kThreads;
            const int cand = lo + tid * step;
            int best = hi;
            if (cand < hi) {
                const float rq = 1.f / (float)cand;
                int cnt = 0;
                for (int b = 0; b < A; ++b) cnt += ceil_div_small(ncache[b], cand, rq);
                if ((int64_t)cnt * nKv <= grid) best = cand;
            }
            // the smallest feasible candidate; the answer is in (best - step, best]
            best = -block_reduce_int<kWarps>(-best, sh + (nb++ & 1) * kWarps, true);
            hi = best;
            lo = max(lo, best - step + 1);
        }
        q = hi;
    }
    int base = 0;                                    // CTAs of the rows before this chunk
    for (int b0 = 0; b0 < A; b0 += kThreads) {
        const int b = b0 + tid;
        const int n = b < A ? ncache[b] : 0;
        const int k = b < A ? (n + q - 1) / q : 0;
        int x = k * nKv;                             // inclusive scan of the rows' CTAs within the warp
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        int* wb = sh + (nb++ & 1) * kWarps;
        if (lane == 31) wb[wid] = x;
        __syncthreads();
        int wbase = 0, tot = 0;
        for (int w = 0; w < kWarps; ++w) {
            if (w < wid) wbase += wb[w];
            tot += wb[w];
        }
        const int first = base + wbase + x - k * nKv;   // the row's first CTA
        if (b < A && slot >= first && slot < first + k * nKv) {
            const int rel = slot - first, g = rel / k;
            res[0] = b * nKv + g; res[1] = rel - g * k; res[2] = n; res[3] = k; res[4] = first + g * k;
        }
        base += tot;                                 // the same in every thread
        if (base > slot) break;
    }
    __syncthreads();
    CtaWork w{res[0], 0, 0, 0, 0};
    if (w.item >= 0) {
        const int j = res[1], n = res[2], k = res[3];
        w.t0 = (int)((int64_t)j * n / k);
        w.t1 = (int)((int64_t)(j + 1) * n / k);
        w.s0 = res[4];
        w.k = k;
    }
    return w;
}

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// Four consecutive outputs at element o of the output (fp32 or fp16) and of its
// optional fp16 pair hi = fp16(v), lo = fp16(v - hi).
__device__ __forceinline__ void store_out4(const AttnTcParams& P, int64_t o, float4 v) {
    const __half2 h01 = __floats2half2_rn(v.x, v.y), h23 = __floats2half2_rn(v.z, v.w);
    uint2 hv;
    hv.x = *reinterpret_cast<const uint32_t*>(&h01);
    hv.y = *reinterpret_cast<const uint32_t*>(&h23);
    if (!P.out) {
    } else if (P.out_dtype == DSPARK_DTYPE_F32) {
        *reinterpret_cast<float4*>(static_cast<float*>(P.out) + o) = v;
    } else {
        *reinterpret_cast<uint2*>(static_cast<__half*>(P.out) + o) = hv;
    }
    if (P.out_hi) {
        *reinterpret_cast<uint2*>(P.out_hi + o) = hv;
        if (P.out_lo) {
            const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
            uint2 lv;
            lv.x = pack_half2(v.x - f01.x, v.y - f01.y);
            lv.y = pack_half2(v.z - f23.x, v.w - f23.y);
            *reinterpret_cast<uint2*>(P.out_lo + o) = lv;
        }
    }
}

// Row r of item (b, g) combined over the item's k slots s0 .. s0 + k - 1 by one
// warp, lane l owning the CPL columns c0 + CPL l .. + CPL - 1: out = sum_s w_s l_s
// O_s / sum_s w_s l_s with w_s = exp(m_s - M) and O_s the slot's normalised output
// (fp16). BATCH slots' loads per lane are in flight at once. Items of many slots (a
// short call's few items) take CPL = 4 and two warps per row, with twice the loads
// in flight; items of a few slots take CPL = 8 (each warp's fixed work then counts).
template <int CPL, int BATCH>
__device__ __forceinline__ void merge_row(const AttnTcParams& P, int s0, int k, int r, int64_t out_row, int c0) {
    using Vec = typename std::conditional<CPL == 8, uint4, uint2>::type;
    const int lane = threadIdx.x & 31, col = c0 + CPL * lane;
    const bool mine = col < P.hd;
    float num[CPL];
#pragma unroll
    for (int e = 0; e < CPL; ++e) num[e] = 0.f;
    float den = 0.f, M = -INFINITY;
    for (int sb = 0; sb < k; sb += 32) {
        const int cnt = min(32, k - sb);
        // the first batch of rows and this chunk's (max, sum) pairs go out together: the rows'
        // loads do not depend on the maxima
        Vec v[BATCH];
        auto load_rows = [&](int t0) {
#pragma unroll
            for (int u = 0; u < BATCH; ++u) {
                const __half* o = P.part_o + ((int64_t)(s0 + sb + t0 + u) * QROWS + r) * P.hd + col;
                Vec z{};
                v[u] = (t0 + u < cnt && mine) ? *reinterpret_cast<const Vec*>(o) : z;
            }
        };
        load_rows(0);
        float2 ml = make_float2(-INFINITY, 0.f);
        if (lane < cnt) ml = reinterpret_cast<const float2*>(P.part_ml)[(int64_t)(s0 + sb + lane) * QROWS + r];
        float mc = ml.x;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mc = fmaxf(mc, __shfl_xor_sync(0xffffffffu, mc, o));
        // a later chunk with a larger maximum rescales what the earlier ones summed
        const float Mn = fmaxf(M, mc);
        if (Mn > M && M > -INFINITY) {
            const float f = __expf(M - Mn);
            den *= f;
#pragma unroll
            for (int e = 0; e < CPL; ++e) num[e] *= f;
        }
        M = Mn;
        const float wl = ml.x == -INFINITY ? 0.f : __expf(ml.x - M) * ml.y;   // w_s l_s
        for (int t0 = 0; t0 < cnt; t0 += BATCH) {
            if (t0 > 0) load_rows(t0);
#pragma unroll
            for (int u = 0; u < BATCH; ++u) {
                const float w = __shfl_sync(0xffffffffu, wl, (t0 + u) & 31);
                if (t0 + u >= cnt) break;
                den += w;
                if (w == 0.f) continue;                // uniform: an empty range
                const __half2* h = reinterpret_cast<const __half2*>(&v[u]);
#pragma unroll
                for (int e = 0; e < CPL / 2; ++e) {
                    const float2 f = __half22float2(h[e]);
                    num[2 * e] += w * f.x;
                    num[2 * e + 1] += w * f.y;
                }
            }
        }
    }
    const float inv = 1.f / den;
    if (mine) {
#pragma unroll
        for (int e = 0; e < CPL; e += 4)
            store_out4(P, out_row + col + e, make_float4(num[e] * inv, num[e + 1] * inv, num[e + 2] * inv, num[e + 3] * inv));
    }
}

// Zeroes rows [nvalid, KT) of a V tile of `nsub` sub-tiles [KT rows x 128 B] (one warp).
__device__ __forceinline__ void zero_tail(uint8_t* tile, int nsub, int nvalid, int lane) {
    const int per_sub = (KT - nvalid) * 8;          // 16-byte chunks past the last key, per sub-tile
    for (int c = lane; c < nsub * per_sub; c += 32) {
        const int sub = c / per_sub, r = c % per_sub;
        reinterpret_cast<uint4*>(tile + sub * KT * 128 + nvalid * 128)[r] = make_uint4(0u, 0u, 0u, 0u);
    }
}

// Bounded mbarrier wait by polling (no suspension): for the short waits on the
// softmax's critical path, where a wake-up delay would add to every tile.
__device__ __forceinline__ bool mbar_wait_spin(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int32_t* status) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 0) {
            if (*abort_flag) return false;
            if (global_timer_ns() - t0 > kWaitLimitNs) {
                *abort_flag = 1;
                atomicOr(status, DSPARK_DEV_WAIT_TIMEOUT);
                return false;
            }
        }
    }
}

// A bounded mbarrier wait whose outcome is the same in every lane of the warp
// (the softmax warps run warp-collective tcgen05.ld and votes after it).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int32_t* status) {
    const bool w = mbar_wait(bar, parity, abort_flag, status);
    return __all_sync(0xffffffffu, w);
}
__device__ __forceinline__ bool warp_wait_spin(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int32_t* status) {
    const bool w = mbar_wait_spin(bar, parity, abort_flag, status);
    return __all_sync(0xffffffffu, w);
}

// (sin, cos) of pos * inv_freq for the K rebuild: the angle reduced to [-pi, pi] in
// double, then the fast single-precision intrinsic (absolute error a few 1e-7 there,
// far below the fp16 rounding of the rebuilt keys).
__device__ __forceinline__ void rope_angle_fast(int pos, double inv_freq, float* s, float* c) {
    const double two_pi = 6.283185307179586476925286766559;
    const double inv_two_pi = 0.15915494309189533576888376337251;
    double a = (double)pos * inv_freq;
    a -= rint(a * inv_two_pi) * two_pi;
    __sincosf((float)a, s, c);
}

template <bool VONLY>
__global__ void __launch_bounds__(AttnThreads<VONLY>::n, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
               const __grid_constant__ CUtensorMap tmKb, const __grid_constant__ CUtensorMap tmVb,
               const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmQ, AttnTcParams P) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const int hd = P.hd, nsub = hd / 64;
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tile_sz = nsub * KT * 128;                  // one K or V tile: nsub x [64 keys x 128 B]
    constexpr int kSK = AttnSlots<VONLY>::k, kSV = AttnSlots<VONLY>::v;
    uint8_t* sK = base;                                   // kSK x tile
    uint8_t* sV = sK + kSK * tile_sz;                     // kSV x tile
    uint8_t* sP = sV + kSV * tile_sz;                     // 2 slots x [128 rows x 128 B]
    int* red = reinterpret_cast<int*>(sP + 2 * QROWS * 128);      // plan scratch (2 kWarps + 5 ints), last-CTA flag
    uint64_t* bars = reinterpret_cast<uint64_t*>(red + 2 * QROWS);
    uint64_t* kfull = bars + 0;                // [kSK] K tile landed in the slot (TMA)
    uint64_t* vfull = kfull + kSlotsMax;       // [kSV] V tile landed in the slot (TMA)
    uint64_t* vready = vfull + kSlotsMax;      // [kSV] V tile ready (V-only: and K rebuilt): 1 / kBuildWarps arrivals
    uint64_t* kfree = vready + kSlotsMax;      // [kSK] the S product that read the K slot is done
    uint64_t* vfree = kfree + kSlotsMax;       // [kSV] the P V product that read the V slot is done
    uint64_t* sdone = vfree + kSlotsMax;       // [2] S product of the tile in that buffer done
    uint64_t* sfree = sdone + 2;               // [2] softmax has read the S buffer (256 arrivals)
    uint64_t* pready = sfree + 2;              // [2] P slot written (256 arrivals)
    uint64_t* odone = pready + 2;              // [2] P V product of the tile in that P slot done (O settled)
    uint64_t* spare = odone + 2;               // teardown: MMAs in flight after an abort
    uint64_t* spare2 = spare + 1;              // teardown of the P V issuer
    uint64_t* qfull = spare2 + 1;              // the query tile landed in shared memory (TMA)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(qfull + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nq = P.grp * P.G;

    if (tid == 0) {
        for (int i = 0; i < kSlotsMax; ++i) {
            mbar_init(&kfull[i], 1); mbar_init(&vfull[i], 1); mbar_init(&vready[i], VONLY ? kBuildWarps : 1);
            mbar_init(&kfree[i], 1); mbar_init(&vfree[i], 1);
        }
        mbar_init(&sdone[0], 1); mbar_init(&sdone[1], 1);
        mbar_init(&sfree[0], kSoftThreads); mbar_init(&sfree[1], kSoftThreads);
        mbar_init(&pready[0], kSoftThreads); mbar_init(&pready[1], kSoftThreads);
        mbar_init(&odone[0], 1); mbar_init(&odone[1], 1); mbar_init(spare, 1); mbar_init(spare2, 1);
        mbar_init(qfull, 1);
        *abort_flag = 0;
        mbar_fence_init();
        prefetch_tmap(&tmK); prefetch_tmap(&tmV); prefetch_tmap(&tmKb); prefetch_tmap(&tmVb); prefetch_tmap(&tmO);
        prefetch_tmap(&tmQ);
    }
    if (warp == kIssuerWarp) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // q, the lengths and the caches come from earlier kernels. No
    // pdl_trigger: the next kernel launches as these CTAs exit (see gemm_tc.cu)
    pdl_wait();

    // this CTA's work: tiles [t_lo, t_hi) of item (b, g); an idle CTA has none
    const int slot = blockIdx.x;
    const CtaWork W = cta_work<AttnThreads<VONLY>::n>(P.len, P.A, P.nKv, P.capacity, P.grid, slot, red, reinterpret_cast<int*>(sK));
    const int item = W.item;
    const int b = item >= 0 ? item / P.nKv : 0, g = item >= 0 ? item % P.nKv : 0;
    const int t_lo = W.t0, t_hi = W.t1;
    int len = P.len[b];
    if (len < 0 || len > P.capacity) {
        if (tid == 0) atomicOr(P.status, DSPARK_DEV_BAD_LENGTH);
        len = min(max(len, 0), P.capacity);
    }
    // the item's tiles: ceil(len / KT) context tiles of KT keys, then the block's G keys
    const int n_ctx_all = (len + KT - 1) / KT;
    const int nt = t_hi - t_lo;
    auto tile_rows = [&](int t, int* row, int* nvalid, bool* blk) {
        const int u = t_lo + t;
        if (u < n_ctx_all) { *row = b * P.capacity + u * KT; *nvalid = min(KT, len - u * KT); *blk = false; }
        else { *row = b * P.G; *nvalid = P.G; *blk = true; }
    };

    // Q tile in tensor memory (the S product's A operand): TMEM lane r holds query
    // row r, two fp16 values per 32-bit column from column kQCol; rows past the
    // queries are zero. The tile comes by TMA, one request per 64 head dimensions
    // ([nq rows x 128 B], 128-byte swizzle), into V slots 1 and 2 (free until it is
    // in tensor memory; their V tiles are requested after it), while K tiles 0..2
    // and V tile 0 load. Softmax thread r then copies its row to tensor memory.
    const uint32_t tile_bytes = (uint32_t)nsub * KT * 128;
    // V-only: the K slots are free until the builders start (after the query tile is in
    // tensor memory), so the query tile goes there and V tiles 0..2 load at once
    uint8_t* sQ = VONLY ? sK : sV + tile_sz;              // nsub x [nq rows x 128 B] <= 2 tiles
    const int qstride = (nq * 128 + 1023) & ~1023;        // chunks 1 KB aligned (the swizzle's period)
    if (warp == kIssuerWarp && lane == 0 && item >= 0) {
        mbar_arrive_expect_tx(qfull, (uint32_t)(nsub * nq * 128));
        for (int c = 0; c < nsub; ++c) tma_load_5d(sQ + c * qstride, &tmQ, qfull, 0, 0, g, b * P.G, c);
    }
    if ((warp == kIssuerWarp || warp == kIssuerWarp + 1) && lane == 0) {
        const bool v_tile = warp != kIssuerWarp;
        const int n0 = v_tile ? (VONLY ? kSV : 1) : (VONLY ? 0 : kSK);
        for (int t = 0; t < n0 && t < nt; ++t) {
            int row, nvalid; bool blk;
            tile_rows(t, &row, &nvalid, &blk);
            const CUtensorMap* m = blk ? (v_tile ? &tmVb : &tmKb) : (v_tile ? &tmV : &tmK);
            uint64_t* bar = v_tile ? &vfull[t] : &kfull[t];
            mbar_arrive_expect_tx(bar, tile_bytes);
            tma_load_4d((v_tile ? sV : sK) + t * tile_sz, m, bar, 0, row, g, 0);
        }
    }
    bool ok = true;
    if (tid < kSoftThreads) {
        const int r = tid;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        if (item >= 0 && !warp_wait(qfull, 0u, abort_flag, P.status)) ok = false;
        for (int c = 0; c < nsub; ++c) {
            const uint8_t* line = sQ + c * qstride + r * 128;
#pragma unroll
            for (int j0 = 0; j0 < 8; j0 += 4) {               // 4 pieces of 16 bytes = 16 columns per tcgen05.st
                uint32_t w[16];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint4 u = make_uint4(0u, 0u, 0u, 0u);
                    if (r < nq && ok) u = *reinterpret_cast<const uint4*>(line + (((j0 + j) ^ (r & 7)) * 16));
                    w[4 * j] = u.x; w[4 * j + 1] = u.y; w[4 * j + 2] = u.z; w[4 * j + 3] = u.w;
                }
                tmem_st_x16(tmem + (uint32_t)(kQCol + c * 32 + j0 * 4) + lane_off, w);
            }
        }
        tmem_st_wait();
        fence_async_shared();                             // reads done before V tiles 1, 2 overwrite the area
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kIssuerWarp + 1 && lane == 0 && !VONLY) {
        for (int t = 1; t < kSV && t < nt; ++t) {
            int row, nvalid; bool blk;
            tile_rows(t, &row, &nvalid, &blk);
            mbar_arrive_expect_tx(&vfull[t], tile_bytes);
            tma_load_4d(sV + t * tile_sz, blk ? &tmVb : &tmV, &vfull[t], 0, row, g, 0);
        }
    }

    const uint32_t tO = tmem + 2 * KT;                    // O: columns [128, 128 + hd); S buffers at 0 and 64

    if (warp == kIssuerWarp || warp == kIssuerWarp + 1) {
        // ------------------------------------------------------------ issuers
        // warp 8: S = Q K^T and the K loads; warp 9: O += P V and the V loads.
        // Each waits only for what its own products need; a load waits only for its
        // slot to be free, and every wait keeps issuing the loads that can go.
        if (lane == 0) {
            const bool is_qk = warp == kIssuerWarp;
            auto load = [&](uint8_t* dst, uint64_t* bar, bool v_tile, int t) {
                int row, nvalid; bool blk;
                tile_rows(t, &row, &nvalid, &blk);
                const CUtensorMap* m = blk ? (v_tile ? &tmVb : &tmKb) : (v_tile ? &tmV : &tmK);
                mbar_arrive_expect_tx(bar, tile_bytes);
                tma_load_4d(dst, m, bar, 0, row, g, 0);     // the whole tile in one request
            };
            uint8_t* buf = is_qk ? sK : sV;
            uint64_t* fullb = is_qk ? kfull : vfull;
            uint64_t* freeb = is_qk ? kfree : vfree;          // completion of the product that read a slot
            const int ns = is_qk ? kSK : kSV;                 // this issuer's slots
            int nl[kSlotsMax] = {};                           // loads issued per slot
            const bool loads = !(VONLY && is_qk);             // V-only: the S issuer loads nothing
            if (loads)
                for (int t = 0; t < ns && t < nt; ++t) ++nl[t];   // issued before the loop
            int ln = loads ? min(ns, nt) : nt;                // next tile to load
            int issued = 0;                                   // products issued
            // tile ln goes into slot ln % ns once the product of tile ln - ns (the slot's
            // previous tile, phase (ln - ns) / ns of its barrier) is done
            auto service = [&]() {
                while (ln < nt && ln - ns < issued &&
                       mbar_try_wait(&freeb[ln % ns], (uint32_t)((ln - ns) / ns) & 1u)) {
                    load(buf + (ln % ns) * tile_sz, &fullb[ln % ns], !is_qk, ln);
                    ++nl[ln % ns];
                    ++ln;
                }
            };
            // a waiting issuer sleeps in the barrier (woken by its completion) instead of
            // spinning, so it takes no issue slots from the softmax and the K builders;
            // while a load waits for its slot it looks again within 200 ns
            auto wait_serving = [&](uint64_t* bar, uint32_t parity) -> bool {
                const uint64_t t0w = global_timer_ns();
                while (!mbar_try_wait_hint(bar, parity, ln < nt ? 200u : 2000u)) {
                    service();
                    if (*abort_flag) return false;
                    if (global_timer_ns() - t0w > kWaitLimitNs) {
                        *abort_flag = 1;
                        atomicOr(P.status, DSPARK_DEV_WAIT_TIMEOUT);
                        return false;
                    }
                }
                return true;
            };
            const uint32_t idesc_qk = idesc_f16(QROWS, KT, 0);
            const uint32_t idesc_pv = idesc_f16(QROWS, hd, 1);
            const uint32_t qa = tmem + (uint32_t)kQCol;      // Q in tensor memory: 8 columns per 16-wide K slice
            for (int t = 0; t < nt && ok; ++t) {
                const int sl = t & 1;                             // S buffer / P slot
                const int tk = t % kSK, tv = t % kSV;             // K slot, V slot
                const uint32_t kph = (uint32_t)(t / kSK) & 1u, vph = (uint32_t)(t / kSV) & 1u;
                if (is_qk) {
                    // S(t) = Q K(t)^T into buffer t % 2
                    // V-only: the K tile is rebuilt from the V tile (vready), not loaded
                    if (!(VONLY ? wait_serving(&vready[tv], vph) : wait_serving(&kfull[tk], kph))) { ok = false; break; }
                    if (t >= 2 && !wait_serving(&sfree[sl], (uint32_t)((t - 2) >> 1) & 1u)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t d = tmem + (uint32_t)(sl * KT);
                    // descriptors advance by address / 16: constants per unrolled slice
                    const uint64_t bd0 = sdesc_k_sw128(smem_u32(sK + tk * tile_sz));
                    mma_f16_ts(d, qa, bd0, idesc_qk, 0u);
#pragma unroll
                    for (int j = 1; j < 16; ++j) {
                        if (j >= hd / 16) break;
                        const uint64_t boff = (uint64_t)(((j >> 2) * KT * 128 + (j & 3) * 32) >> 4);
                        mma_f16_ts(d, qa + (uint32_t)(8 * j), bd0 + boff, idesc_qk, 1u);
                    }
                    mma_commit(&sdone[sl]);
                    mma_commit(&kfree[tk]);                         // V-only: the builders wait on it
                } else {
                    // O += P(t) V(t)
                    if (!wait_serving(&pready[sl], (uint32_t)(t >> 1) & 1u) || !wait_serving(&vready[tv], vph)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad0 = sdesc_k_sw128(smem_u32(sP + sl * QROWS * 128));
                    const uint64_t bd0 = sdesc_mn_sw128(smem_u32(sV + tv * tile_sz), KT * 128);
#pragma unroll
                    for (int j = 0; j < KT / 16; ++j)
                        mma_bf16(tO, ad0 + (uint64_t)((j * 32) >> 4), bd0 + (uint64_t)((j * 2048) >> 4), idesc_pv,
                                 (t > 0 || j > 0) ? 1u : 0u);
                    mma_commit(&odone[sl]);
                    mma_commit(&vfree[tv]);
                }
                issued = t + 1;
                service();
            }
            // teardown after an abort: copies and MMAs in flight land first (bounded)
            if (!ok) {
                const uint64_t deadline = global_timer_ns() + kWaitLimitNs;
                bool drained = true;
                for (int i = 0; i < ns; ++i)
                    if (drained && nl[i] > 0) drained = mbar_wait_until(&fullb[i], (uint32_t)(nl[i] - 1) & 1u, deadline);
                uint64_t* sp = is_qk ? spare : spare2;
                mma_commit(sp);
                if (drained) drained = mbar_wait_until(sp, 0u, deadline);
                if (!drained) atomicOr(P.status, DSPARK_DEV_WAIT_TIMEOUT);
            }
        }
    } else if (VONLY && warp >= kFixWarp) {
        // ------------------------------------------------------------ K from V (V-only cache)
        // builder thread bt owns RoPE pairs [8 pg, 8 pg + 8) of keys [4 kr, 4 kr + 4) of
        // every tile: dimensions d1 + m and d2 + m (d2 = d1 + hd / 2), two 16-byte
        // pieces of each key row, read from the V slot and written to the K slot (same
        // 128-byte swizzled layout); rows past the last key are zeroed in the V slot
        const int bt = tid - kFixWarp * 32;
        const int npg = hd / 16, half = hd / 2;
        const int pg = bt % npg, kr = bt / npg;
        const bool active = kr < KT / kBuildKeys;
        const int d1 = pg * 8, d2 = pg * 8 + half;
        const int o1 = (d1 / 64) * KT * 128, c1 = (d1 % 64) / 8;
        const int o2 = (d2 / 64) * KT * 128, c2 = (d2 % 64) / 8;
        // gains as fp16 pairs (the products and the rotation run on packed fp16: each
        // key's k is rounded to fp16 anyway); the angles stay in fp32
        __half2 w1h[4], w2h[4];
        float cs[8], sn[8], cs1[8], sn1[8], cs64[8], sn64[8];
        if (active) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                w1h[e] = __floats2half2_rn(__bfloat162float(P.k_norm[d1 + 2 * e]), __bfloat162float(P.k_norm[d1 + 2 * e + 1]));
                w2h[e] = __floats2half2_rn(__bfloat162float(P.k_norm[d2 + 2 * e]), __bfloat162float(P.k_norm[d2 + 2 * e + 1]));
            }
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const double f = P.inv_freq[d1 + m];
                rope_angle_fast(1, f, &sn1[m], &cs1[m]);      // one key further
                rope_angle_fast(KT, f, &sn64[m], &cs64[m]);   // one tile further
                cs[m] = 1.f; sn[m] = 0.f;
            }
        }
        bool anchored = false;                             // cs, sn: angles of this thread's first key of tile t
        for (int t = 0; t < nt && ok; ++t) {
            int row, nvalid; bool blk;
            tile_rows(t, &row, &nvalid, &blk);
            const int tv = t % kSV, tk = t % kSK;
            if (!warp_wait(&vfull[tv], (uint32_t)(t / kSV) & 1u, abort_flag, P.status)) { ok = false; break; }
            // the K slot's previous tile, t - kSK, must have had its S product
            if (t >= kSK && !warp_wait(&kfree[tk], (uint32_t)((t - kSK) / kSK) & 1u, abort_flag, P.status)) {
                ok = false;
                break;
            }
            if (active) {
                if (blk || !anchored) {                        // exact angles at the first context tile and the block
                    const int p = (blk ? P.block_pos[b] : P.pos0[b] + (t_lo + t) * KT) + kr * kBuildKeys;
#pragma unroll
                    for (int m = 0; m < 8; ++m) rope_angle_fast(p, P.inv_freq[d1 + m], &sn[m], &cs[m]);
                    anchored = true;
                }
                uint8_t* vt = sV + tv * tile_sz;
                uint8_t* kt = sK + tk * tile_sz;
                float c[8], sv_[8];
#pragma unroll
                for (int m = 0; m < 8; ++m) { c[m] = cs[m]; sv_[m] = sn[m]; }
#pragma unroll
                for (int kk = 0; kk < kBuildKeys; ++kk) {
                    const int j = kr * kBuildKeys + kk;
                    const int a1 = o1 + j * 128 + ((c1 ^ (j & 7)) * 16), a2 = o2 + j * 128 + ((c2 ^ (j & 7)) * 16);
                    if (j < nvalid) {
                        const uint4 x4 = *reinterpret_cast<const uint4*>(vt + a1);
                        const uint4 y4 = *reinterpret_cast<const uint4*>(vt + a2);
                        const __half2* xh = reinterpret_cast<const __half2*>(&x4);
                        const __half2* yh = reinterpret_cast<const __half2*>(&y4);
                        uint32_t k1[4], k2[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const __half2 xw = __hmul2(xh[e], w1h[e]), yw = __hmul2(yh[e], w2h[e]);
                            const __half2 ch = __floats2half2_rn(c[2 * e], c[2 * e + 1]);
                            const __half2 sh = __floats2half2_rn(sv_[2 * e], sv_[2 * e + 1]);
                            const __half2 r1 = __hfma2(xw, ch, __hneg2(__hmul2(yw, sh)));   // x cos - y sin
                            const __half2 r2 = __hfma2(yw, ch, __hmul2(xw, sh));            // y cos + x sin
                            k1[e] = *reinterpret_cast<const uint32_t*>(&r1);
                            k2[e] = *reinterpret_cast<const uint32_t*>(&r2);
                        }
                        *reinterpret_cast<uint4*>(kt + a1) = make_uint4(k1[0], k1[1], k1[2], k1[3]);
                        *reinterpret_cast<uint4*>(kt + a2) = make_uint4(k2[0], k2[1], k2[2], k2[3]);
                    } else {
                        // past the last key: the P V product must not meet stale bits (S masks these keys)
                        *reinterpret_cast<uint4*>(vt + a1) = make_uint4(0u, 0u, 0u, 0u);
                        *reinterpret_cast<uint4*>(vt + a2) = make_uint4(0u, 0u, 0u, 0u);
                    }
#pragma unroll
                    for (int m = 0; m < 8; ++m) {              // the next key: angle + theta
                        const float cn = c[m] * cs1[m] - sv_[m] * sn1[m];
                        sv_[m] = sv_[m] * cs1[m] + c[m] * sn1[m];
                        c[m] = cn;
                    }
                }
#pragma unroll
                for (int m = 0; m < 8; ++m) {                  // the next context tile: angle + 64 theta
                    const float cn = cs[m] * cs64[m] - sn[m] * sn64[m];
                    sn[m] = sn[m] * cs64[m] + cs[m] * sn64[m];
                    cs[m] = cn;
                }
            }
            fence_async_shared();                           // both tiles are read through the async proxy
            __syncwarp();
            if (lane == 0) mbar_arrive(&vready[tv]);
        }
    } else if (warp == kFixWarp) {
        // ------------------------------------------------------------ V tails
        for (int t = 0; t < nt && ok; ++t) {
            int row, nvalid; bool blk;
            tile_rows(t, &row, &nvalid, &blk);
            const int ks = t % kSV;
            if (!warp_wait(&vfull[ks], (uint32_t)(t / kSV) & 1u, abort_flag, P.status)) { ok = false; break; }
            if (nvalid < KT) {
                zero_tail(sV + ks * tile_sz, nsub, nvalid, lane);
                fence_async_shared();               // the P V product reads the tile through the async proxy
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&vready[ks]);
        }
    } else {
        // ------------------------------------------------------------ softmax (one thread per query row)
        const int r = tid;                                 // query row = TMEM lane
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        float m_run = -INFINITY, l_run = 0.f;
        for (int t = 0; t < nt && ok; ++t) {
            int row, nvalid; bool blk;
            tile_rows(t, &row, &nvalid, &blk);
            const int sl = t & 1;
            const uint32_t tS = tmem + (uint32_t)(sl * KT) + lane_off;
            // S(t) is on the critical path: poll (no suspension)
            // (V-only: the wait is long, behind the K rebuild, so the warp sleeps in it)
            if (!(VONLY ? warp_wait(&sdone[sl], (uint32_t)(t >> 1) & 1u, abort_flag, P.status)
                        : warp_wait_spin(&sdone[sl], (uint32_t)(t >> 1) & 1u, abort_flag, P.status))) { ok = false; break; }
            tc_fence_after();
            uint32_t u[4][16];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld_x16(tS + (uint32_t)(16 * c), u[c]);
            tmem_ld_wait();
            float sv[KT];
#pragma unroll
            for (int j = 0; j < KT; ++j) sv[j] = __uint_as_float(u[j >> 4][j & 15]);
            if (nvalid < KT) {
#pragma unroll
                for (int j = 0; j < KT; ++j) if (j >= nvalid) sv[j] = -INFINITY;
            }
            float mt[32];                                   // tree maximum: 6 dependent steps, not 64
#pragma unroll
            for (int j = 0; j < 32; ++j) mt[j] = fmaxf(sv[j], sv[32 + j]);
#pragma unroll
            for (int w = 16; w > 0; w >>= 1) {
#pragma unroll
                for (int j = 0; j < w; ++j) mt[j] = fmaxf(mt[j], mt[j + w]);
            }
            const float mx = mt[0];
            const bool need = t > 0 && mx > m_run + kRescale;
            if (t == 0) m_run = mx;
            if (__any_sync(0xffffffffu, need)) {
                // O holds tiles up to t - 1 at the old max: P(t-1) V(t-1) must have landed
                if (t >= 1 && !warp_wait(&odone[(t - 1) & 1], (uint32_t)((t - 1) >> 1) & 1u, abort_flag, P.status)) { ok = false; break; }
                tc_fence_after();
                const float f = need ? __expf(m_run - mx) : 1.f;
                if (need) { l_run *= f; m_run = mx; }
                for (int c = 0; c < hd; c += 32) {            // 32 columns per TMEM round trip
                    uint32_t o[2][16];
                    tmem_ld_x16(tO + lane_off + (uint32_t)c, o[0]);
                    tmem_ld_x16(tO + lane_off + (uint32_t)(c + 16), o[1]);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j) o[j >> 4][j & 15] = __float_as_uint(__uint_as_float(o[j >> 4][j & 15]) * f);
                    tmem_st_x16(tO + lane_off + (uint32_t)c, o[0]);
                    tmem_st_x16(tO + lane_off + (uint32_t)(c + 16), o[1]);
                }
                tmem_st_wait();
            }
            // P slot t % 2 was last read by P(t-2) V(t-2)
            if (t >= 2 && !(VONLY ? warp_wait(&odone[sl], (uint32_t)((t - 2) >> 1) & 1u, abort_flag, P.status)
                                  : warp_wait_spin(&odone[sl], (uint32_t)((t - 2) >> 1) & 1u, abort_flag, P.status))) {
                ok = false;
                break;
            }
            float ls[8];                                    // sums in 8 independent chains
#pragma unroll
            for (int j = 0; j < 8; ++j) ls[j] = 0.f;
            uint8_t* pslot = sP + sl * QROWS * 128;
#pragma unroll
            for (int q = 0; q < 8; ++q) {                  // eight 16-byte chunks of 8 keys
                float p[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) { p[j] = __expf(sv[q * 8 + j] - m_run); ls[j] += p[j]; }
                *reinterpret_cast<uint4*>(pslot + r * 128 + ((q ^ (r & 7)) * 16)) =
                    make_uint4(pack_half2(p[0], p[1]), pack_half2(p[2], p[3]), pack_half2(p[4], p[5]), pack_half2(p[6], p[7]));
            }
            l_run += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
            tc_fence_before();
            mbar_arrive(&sfree[sl]);                           // S buffer read
            fence_async_shared();
            mbar_arrive(&pready[sl]);                          // P written
        }
        // ---- this range's result
        const bool any = nt > 0;
        if (any && ok && !warp_wait(&odone[(nt - 1) & 1], (uint32_t)((nt - 1) >> 1) & 1u, abort_flag, P.status)) ok = false;
        tc_fence_after();
        if (W.k == 1) {
            // the item's only CTA: the normalised output straight from tensor memory
            if (tid == 0) { P.item_slots[2 * item] = W.s0; P.item_slots[2 * item + 1] = 1; }
            const int64_t out_row = (((int64_t)b * P.G + r / P.grp) * P.nH + g * P.grp + r % P.grp) * hd;
            if (any && ok) {
                const float inv = 1.f / l_run;
                for (int c = 0; c < hd; c += 32) {
                    uint32_t o[2][16];
                    tmem_ld_x16(tO + lane_off + (uint32_t)c, o[0]);
                    tmem_ld_x16(tO + lane_off + (uint32_t)(c + 16), o[1]);
                    tmem_ld_wait();
                    if (r < nq) {
#pragma unroll
                        for (int j = 0; j < 32; j += 4)
                            store_out4(P, out_row + c + j,
                                       make_float4(__uint_as_float(o[j >> 4][j & 15]) * inv,
                                                   __uint_as_float(o[j >> 4][(j & 15) + 1]) * inv,
                                                   __uint_as_float(o[j >> 4][(j & 15) + 2]) * inv,
                                                   __uint_as_float(o[j >> 4][(j & 15) + 3]) * inv));
                    }
                }
            }
        } else if (item >= 0) {
            // O / l and (max, sum) per query row into this CTA's slot
            if (tid == 0 && W.t0 == 0) {                      // the item's first CTA tells the merge its slots
                P.item_slots[2 * item] = W.s0;
                P.item_slots[2 * item + 1] = W.k;
            }
            if (r < nq) {
                const int64_t prow = (int64_t)slot * QROWS + r;
                P.part_ml[prow * 2] = any ? m_run : -INFINITY;
                P.part_ml[prow * 2 + 1] = any ? l_run : 0.f;
            }
            // The normalised O = O / l (|O / l| <= max |v|: inside fp16, at fp16's relative
            // precision; half the bytes of the fp32 sums) goes through shared memory (the K / V
            // slots are free: every product has completed): hd / 64 slices of [128 rows x
            // 128 B], 16-byte chunks swizzled by row (the 128-byte TMA swizzle), then one TMA
            // store per slice writes whole 128-byte lines instead of scattered 16-byte pieces.
            const bool stage_ok = any && ok;
            if (stage_ok) {
                const float inv = 1.f / l_run;
                for (int c = 0; c < hd; c += 64) {
                    uint32_t o[4][16];
#pragma unroll
                    for (int q = 0; q < 4; ++q) tmem_ld_x16(tO + lane_off + (uint32_t)(c + 16 * q), o[q]);
                    tmem_ld_wait();
                    uint8_t* line = sK + (c / 64) * (QROWS * 128) + r * 128;
#pragma unroll
                    for (int j8 = 0; j8 < 8; ++j8) {               // 16-byte chunk j8: columns c + 8 j8 .. + 7
                        uint32_t h[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int x = 8 * j8 + 2 * e;
                            h[e] = pack_half2(__uint_as_float(o[x >> 4][x & 15]) * inv,
                                              __uint_as_float(o[(x + 1) >> 4][(x + 1) & 15]) * inv);
                        }
                        *reinterpret_cast<uint4*>(line + ((j8 ^ (r & 7)) * 16)) = make_uint4(h[0], h[1], h[2], h[3]);
                    }
                }
                fence_async_shared();                         // visible to the TMA
            }
            named_barrier_sync(2, kSoftThreads);
            if (tid == 0 && stage_ok) {
                for (int c = 0; c < hd; c += 64) tma_store_2d(&tmO, sK + (c / 64) * (QROWS * 128), c, slot * QROWS);
                bulk_commit_group();
                bulk_wait_all();                              // written before this CTA's shared memory goes
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kIssuerWarp) tmem_dealloc(tmem, 512);
}

PFN_cuTensorMapEncodeTiled_v12000 g_enc = nullptr;
std::once_flag g_enc_once;

// Map over a bf16 [rows, nKv, hd] tensor; 128-byte swizzle.
bool make_kv_map(CUtensorMap* tm, const void* ptr, int64_t rows, int nKv, int hd) {
    std::call_once(g_enc_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    if (!g_enc) return false;
    // 4-D view {64 dims, rows, kv heads, hd / 64 chunks (128 bytes apart)}: one request brings a whole
    // tile, laid out [chunk][key][64] = nsub K-major sub-tiles of KT rows (one 32 KB request
    // measured faster than eight of 8 keys each)
    cuuint64_t dims[4] = {64, (cuuint64_t)rows, (cuuint64_t)nKv, (cuuint64_t)(hd / 64)};
    cuuint64_t strides[3] = {(cuuint64_t)nKv * hd * 2, (cuuint64_t)hd * 2, 128};
    cuuint32_t box[4] = {64, (cuuint32_t)KT, 1, (cuuint32_t)(hd / 64)};   // KT <= 256
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return g_enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Map over the partial outputs [rows = CTAs x 128][hd] fp16: boxes of 64 columns
// (128 bytes, 128-byte swizzle) x 128 rows, for the TMA stores of the epilogue.
bool make_part_map(CUtensorMap* tm, __half* ptr, int64_t rows, int hd) {
    if (!g_enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)hd, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)hd * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)QROWS};
    cuuint32_t estr[2] = {1, 1};
    return g_enc(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, ptr, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                 CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// Map over the queries [A * G][nKv][grp][hd] (fp16) with the head dimension split
// into 64-element chunks: 5-D view {64 dims, grp heads, nKv, A * G rows, hd / 64
// chunks}; a box is one chunk of one item's query tile, [G][grp][64] = [nq rows x
// 128 B] with the 128-byte swizzle (query row r = i * grp + head-in-group).
bool make_q_map(CUtensorMap* tm, const void* ptr, int64_t rows, int nKv, int grp, int G, int hd) {
    if (!g_enc) return false;
    cuuint64_t dims[5] = {64, (cuuint64_t)grp, (cuuint64_t)nKv, (cuuint64_t)rows, (cuuint64_t)(hd / 64)};
    cuuint64_t strides[4] = {(cuuint64_t)hd * 2, (cuuint64_t)grp * hd * 2, (cuuint64_t)nKv * grp * hd * 2, 128};
    cuuint32_t box[5] = {64, (cuuint32_t)grp, 1, (cuuint32_t)G, 1};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    return g_enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(ptr), dims, strides, box, estr,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t attn_tc_smem(int hd) {
    const int nsub = hd / 64;
    // six K / V tiles, P (2 slots), the plan scratch, then the barriers
    // (5 kSlotsMax + 11), the TMEM slot and the abort flag; 1 KB alignment slack
    return 6 * (size_t)nsub * KT * 128 + 2 * QROWS * 128 + 2 * QROWS * 4 + 8 * (5 * kSlotsMax + 11) + 16 + 1024;
}


// One warp per output row (b, h, i) of the items on more than one CTA (an item
// on one CTA wrote its output itself).
constexpr int kMergeWarps = 8;
// wpr warps per output row, 32 CPL columns each
template <int CPL>
__global__ void __launch_bounds__(kMergeWarps * 32) attn_tc_merge_kernel(AttnTcParams P, int rows, int wpr) {
    pdl_trigger();
    pdl_wait();
    const int gw = blockIdx.x * kMergeWarps + (threadIdx.x >> 5);
    const int row = gw / wpr, part = gw % wpr;                      // row = ((b * nH) + h) * G + i
    if (row >= rows) return;
    const int i = row % P.G, bh = row / P.G;
    const int b = bh / P.nH, h = bh % P.nH;
    const int item = b * P.nKv + h / P.grp;
    const int k = P.item_slots[2 * item + 1];
    if (k <= 1) return;
    merge_row<CPL, CPL == 4 ? 16 : 8>(P, P.item_slots[2 * item], k, i * P.grp + h % P.grp,
                                      (((int64_t)b * P.G + i) * P.nH + h) * P.hd, part * 32 * CPL);
}

}  // namespace

bool attention_tc_supported(const dspark_model* m) {
    const Dims& d = m->d;
    return d.dtype == DSPARK_DTYPE_BF16 && d.grp * d.gamma <= QROWS && d.hd % 64 == 0 && d.hd <= 256;
}

// The V-only cache: the tensor-core attention, which rebuilds K from the V tiles.
bool vonly_attention_supported(const dspark_model* m) { return attention_tc_supported(m); }

int attention_tc_key_tile() { return KT; }

int attention_tc_grid(const dspark_model* m, int A) { return std::max(m->num_sms, A * m->d.nKv); }

size_t attention_tc_item_ints(const dspark_model* m, int A) { return 2 * (size_t)A * m->d.nKv; }

size_t attention_tc_partial_floats(const dspark_model* m, int grid) { return (size_t)grid * QROWS * (m->d.hd + 2); }

cudaError_t launch_attention_tc(const dspark_model* m, const AttnArgs& a, cudaStream_t s) {
    const Dims& d = m->d;
    if (!a.item_slots || a.tc_grid < std::max(1, a.A * d.nKv) || a.q_dtype != DSPARK_DTYPE_F16 ||
        (a.out_dtype != DSPARK_DTYPE_F32 && a.out_dtype != DSPARK_DTYPE_F16))
        return cudaErrorInvalidValue;
    // V-only cache: K is rebuilt from the V tiles (the K maps repeat the V ones, unused)
    const bool vonly = a.kc == nullptr;
    if (vonly && (!vonly_attention_supported(m) || !a.pos0 || !a.block_pos || !a.k_norm)) return cudaErrorInvalidValue;
    CUtensorMap tk, tv, tkb, tvb, to, tq;
    const int64_t cache_rows = (int64_t)a.batch * a.capacity;   // all rows of this layer's cache
    if (!make_kv_map(&tk, vonly ? a.vc : a.kc, cache_rows, d.nKv, d.hd) ||
        !make_kv_map(&tv, a.vc, cache_rows, d.nKv, d.hd) ||
        !make_kv_map(&tkb, vonly ? a.vb : a.kb, (int64_t)a.A * d.gamma, d.nKv, d.hd) ||
        !make_kv_map(&tvb, a.vb, (int64_t)a.A * d.gamma, d.nKv, d.hd) ||
        !make_part_map(&to, reinterpret_cast<__half*>(a.part_o), (int64_t)a.tc_grid * QROWS, d.hd) ||
        !make_q_map(&tq, a.q, (int64_t)a.A * d.gamma, d.nKv, d.grp, d.gamma, d.hd))
        return cudaErrorInvalidValue;
    AttnTcParams P{};
    P.A = a.A; P.G = d.gamma; P.nH = d.nH; P.nKv = d.nKv; P.grp = d.grp; P.hd = d.hd; P.capacity = a.capacity;
    P.q_dtype = a.q_dtype; P.grid = a.tc_grid; P.q = a.q; P.len = a.len;
    P.part_o = reinterpret_cast<__half*>(a.part_o);   // the fp32 workspace holds the fp16 slots
    P.part_ml = a.part_ml; P.item_slots = a.item_slots; P.status = a.status;
    P.out = a.out; P.out_dtype = a.out_dtype; P.out_hi = a.out_hi; P.out_lo = a.out_lo;
    P.pos0 = a.pos0; P.block_pos = a.block_pos;
    P.k_norm = static_cast<const __nv_bfloat16*>(a.k_norm); P.inv_freq = m->ws.inv_freq;
    const size_t smem = attn_tc_smem(d.hd);
    auto kern = vonly ? attn_tc_kernel<true> : attn_tc_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kern, dim3(a.tc_grid), dim3(vonly ? AttnThreads<true>::n : AttnThreads<false>::n), smem, s, tk, tv,
                   tkb, tvb, to, tq, P);
    if (e != cudaSuccess) return e;
    // with at least as many items as CTAs every item is on one CTA: nothing to merge
    if (a.A * d.nKv >= a.tc_grid) return cudaSuccess;
    const int rows = a.A * d.nH * d.gamma;
    // items of 8 or more slots on average: two warps per row (a few items, many slots each)
    const bool wide = a.tc_grid >= 8 * a.A * d.nKv;
    const int wpr = wide ? (d.hd + 127) / 128 : 1;
    const int64_t warps = (int64_t)rows * wpr;
    return launch_pdl(wide ? attn_tc_merge_kernel<4> : attn_tc_merge_kernel<8>,
                      dim3((unsigned)((warps + kMergeWarps - 1) / kMergeWarps)), dim3(kMergeWarps * 32), 0, s, P, rows,
                      wpr);
}

}  // namespace tc
}  // namespace dspark
