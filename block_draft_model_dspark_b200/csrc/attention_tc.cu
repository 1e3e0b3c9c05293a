// KV-injection attention on tcgen05 tensor cores: the
// DeepspecContextAttention.attend seam ("mlx-bun 0.2.0 -> 0.4.0" page 75,
// plainDeepspecContext): the block queries of one row attend, non-causally
// and at scale 1.0, over the row's cached context keys followed by the
// block's own keys; GQA maps query head h to kv head h / (nH / nKv).
//
// One CTA = a range of key tiles of one item (row b, kv head g), as the plan
// kernel assigns them from the device-side lengths (ragged rows get CTAs in
// proportion to their tiles; every CTA runs in one wave). Its query tile is the 128-row MMA
// side: the grp * gamma queries of the heads that share kv head g (row r =
// query i * grp + head-in-group). Key tiles of KT = 64 rows are TMA-loaded
// from the fp16 cache (4-D maps pick kv head g out of [rows, nKv, hd]) and
// multiplied as they land: both MMAs run as kind::f16 with fp16 operands (q
// and the probabilities P keep an 11-bit significand; the cache holds fp16).
//   S = Q K^T  -> TMEM, two 64-column buffers (tile t in buffer t % 2)
//   softmax    -> one thread per query row (TMEM lane = row); the running max
//                 is raised only when a tile's max exceeds it by more than
//                 kRescale, so O is rarely rescaled in TMEM
//   O += P V   -> TMEM (hd columns), P fp16 from shared memory (K-major,
//                 128-byte swizzle), V as an MN-major operand
// K and V tiles have two shared-memory slots each, so the loads of tile t + 2
// are in flight while tile t is multiplied; per 64 keys at hd = 256 the
// tensor cores run 16 (S) + 4 (P V) MMAs.
//
// Warp roles (352 threads): warps 0-7 run the softmax, two threads per query
// row (warps w and w + 4 share TMEM lanes 32 (w % 4) ..; each takes 32 of the
// tile's 64 columns and half of O's columns; the row max is exchanged through
// shared memory), warp 8 issues the S products and K loads, warp 9 the P V
// products and V loads, and warp 10 zeroes the V rows past the last key of a
// partial tile before its product (stale cache rows may hold any bits, and
// P = 0 times NaN still poisons the accumulator; K needs no fix: those S
// columns are masked to -inf). K, V and P have two slots each and S two TMEM
// buffers, so tile t + 1's load and S product and tile t - 1's P V product all
// overlap tile t's softmax; the softmax waits for P V of tile t - 1 only to
// rescale O (rare). Every wait is bounded. Shared memory at hd = 256: Q 64 KB,
// K, V 2 x 32 KB each, P 2 x 16 KB.
//
// The CTA writes its unnormalised O with (max, sum) per query row into its own
// slot, which the merge kernel combines per item. The last range of each (b, g) also takes the
// block's own keys, as one more tile.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <mutex>

#include "internal.h"
#include "common.cuh"
#include "tc_ptx.cuh"

namespace dspark {

namespace tc {
namespace {

constexpr int kThreads = 352;
constexpr int kSoftThreads = 256;    // warps 0-7
constexpr int kIssuerWarp = 8;       // S products and K loads; warp 9: P V products and V loads
constexpr int kFixWarp = 10;         // zeroes the V rows past the last key of a partial tile
constexpr int KT = 64;               // keys per tile
constexpr int kSlots = 3;            // shared-memory slots of K tiles, and of V tiles (loads in flight)
constexpr int kQCol = 2 * KT + 256;  // TMEM columns: S buffers [0, 2 KT), O [2 KT, 2 KT + hd), Q from 384
constexpr int QROWS = 128;           // MMA M
constexpr float kRescale = 5.0f;     // natural-log headroom before the running max is raised

struct AttnTcParams {
    int A, G, nH, nKv, grp, hd, capacity, q_dtype;
    const void* q;                   // [A, G, nH, hd] (fp32 or fp16)
    const int32_t* len;
    float* part_o; float* part_ml;   // one slot per CTA: [CTA][128 rows][hd] and [CTA][128 rows][2]
    const int* cta_item;             // [grid] the (row, kv head) item of each CTA (-1: idle)
    const int* cta_t0; const int* cta_t1;   // [grid] its tile range within the item
    int32_t* status;
};

// The work plan (one CTA, device lengths): item i = (row b, kv head g) has n_i =
// ceil(len_b / KT) context tiles plus the block tile. The smallest q with
// sum_i ceil(n_i / q) <= grid splits item i into k_i = ceil(n_i / q) equal
// tile ranges, one CTA each (all CTAs in one wave, none above q tiles);
// item_cta0 is the exclusive prefix sum of k_i (the CTAs, and partial slots,
// of item i are item_cta0[i] .. item_cta0[i + 1] - 1).
constexpr int kPlanThreads = 1024;
__device__ __forceinline__ int plan_tiles(const int32_t* len, int b, int capacity) {
    const int L = min(max(len[b], 0), capacity);
    return (L + KT - 1) / KT + 1;
}
__device__ __forceinline__ int block_sum_int(int v, int* red) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();
    if (lane == 0) red[wid] = v;
    __syncthreads();
    int t = 0;
    for (int w = 0; w < kPlanThreads / 32; ++w) t += red[w];
    return t;
}
__global__ void __launch_bounds__(kPlanThreads) attn_plan_kernel(const int32_t* __restrict__ len, int A, int nKv,
                                                                 int capacity, int grid, int* __restrict__ cta_item,
                                                                 int* __restrict__ cta_t0, int* __restrict__ cta_t1,
                                                                 int* __restrict__ item_cta0) {
    __shared__ int red[kPlanThreads / 32];
    __shared__ int s_base;
    pdl_trigger();
    pdl_wait();
    const int tid = threadIdx.x, n_items = A * nKv;
    int mx = 1;
    for (int i = tid; i < n_items; i += kPlanThreads) mx = max(mx, plan_tiles(len, i / nKv, capacity));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    __syncthreads();
    if ((tid & 31) == 0) red[tid >> 5] = mx;
    __syncthreads();
    mx = 1;
    for (int w = 0; w < kPlanThreads / 32; ++w) mx = max(mx, red[w]);
    // the smallest q (tiles per CTA) whose splits fit the grid (q = mx needs n_items <= grid
    // CTAs), at least 2: a CTA also builds its query tile and writes a 128-row partial
    // state, and one tile per CTA measured slower at a single 4096-key row
    int lo = min(2, mx), hi = mx;
    while (lo < hi) {
        const int mid = (lo + hi) / 2;
        int cnt = 0;
        for (int i = tid; i < n_items; i += kPlanThreads) cnt += (plan_tiles(len, i / nKv, capacity) + mid - 1) / mid;
        cnt = block_sum_int(cnt, red);
        if (cnt <= grid) hi = mid; else lo = mid + 1;
    }
    const int q = lo;
    // exclusive scan of k_i over the items, in chunks of kPlanThreads
    if (tid == 0) s_base = 0;
    __syncthreads();
    for (int i0 = 0; i0 < n_items; i0 += kPlanThreads) {
        const int i = i0 + tid;
        const int n = i < n_items ? plan_tiles(len, i / nKv, capacity) : 0;
        const int k = i < n_items ? (n + q - 1) / q : 0;
        int x = k;                                        // inclusive scan within the warp
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if ((tid & 31) >= o) x += y;
        }
        __syncthreads();
        if ((tid & 31) == 31) red[tid >> 5] = x;
        __syncthreads();
        int wbase = 0;
        for (int w = 0; w < (tid >> 5); ++w) wbase += red[w];
        const int excl = s_base + wbase + x - k;
        if (i < n_items) {
            item_cta0[i] = excl;
            // the item's k ranges of n tiles: range j is [j n / k, (j + 1) n / k)
            for (int j = 0; j < k; ++j) {
                cta_item[excl + j] = i;
                cta_t0[excl + j] = (int)((int64_t)j * n / k);
                cta_t1[excl + j] = (int)((int64_t)(j + 1) * n / k);
            }
        }
        __syncthreads();
        if (tid == kPlanThreads - 1) s_base = excl + k;
        __syncthreads();
    }
    const int total = s_base;
    if (tid == 0) item_cta0[n_items] = total;
    for (int c = total + tid; c < grid; c += kPlanThreads) { cta_item[c] = -1; cta_t0[c] = 0; cta_t1[c] = 0; }
}

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
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

__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
               const __grid_constant__ CUtensorMap tmKb, const __grid_constant__ CUtensorMap tmVb, AttnTcParams P) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const int hd = P.hd, nsub = hd / 64;
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tile_sz = nsub * KT * 128;                  // one K or V tile: nsub x [64 keys x 128 B]
    uint8_t* sK = base;                                   // kSlots x tile
    uint8_t* sV = sK + kSlots * tile_sz;                  // kSlots x tile
    uint8_t* sP = sV + kSlots * tile_sz;                  // 2 slots x [128 rows x 128 B]
    float* red = reinterpret_cast<float*>(sP + 2 * QROWS * 128);   // [2 halves][128 rows] row maxima / sums
    uint64_t* bars = reinterpret_cast<uint64_t*>(red + 2 * QROWS);
    uint64_t* kfull = bars + 0;                // [kSlots] K tile landed in the slot (TMA)
    uint64_t* vfull = kfull + kSlots;          // [kSlots] V tile landed in the slot (TMA)
    uint64_t* vready = vfull + kSlots;         // [kSlots] V tile of the slot ready for its product (1 arrival)
    uint64_t* kfree = vready + kSlots;         // [kSlots] the S product that read the K slot is done
    uint64_t* vfree = kfree + kSlots;          // [kSlots] the P V product that read the V slot is done
    uint64_t* sdone = vfree + kSlots;          // [2] S product of the tile in that buffer done
    uint64_t* sfree = sdone + 2;               // [2] softmax has read the S buffer (256 arrivals)
    uint64_t* pready = sfree + 2;              // [2] P slot written (256 arrivals)
    uint64_t* odone = pready + 2;              // [2] P V product of the tile in that P slot done (O settled)
    uint64_t* spare = odone + 2;               // teardown: MMAs in flight after an abort
    uint64_t* xw = spare + 1;                  // row-max exchange: both halves wrote (256 arrivals)
    uint64_t* xr = xw + 1;                     // row-max exchange: both halves read (256 arrivals)
    uint64_t* spare2 = xr + 1;                 // teardown of the P V issuer
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(spare2 + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nq = P.grp * P.G;

    if (tid == 0) {
        for (int i = 0; i < kSlots; ++i) {
            mbar_init(&kfull[i], 1); mbar_init(&vfull[i], 1); mbar_init(&vready[i], 1);
            mbar_init(&kfree[i], 1); mbar_init(&vfree[i], 1);
        }
        mbar_init(&sdone[0], 1); mbar_init(&sdone[1], 1);
        mbar_init(&sfree[0], kSoftThreads); mbar_init(&sfree[1], kSoftThreads);
        mbar_init(&pready[0], kSoftThreads); mbar_init(&pready[1], kSoftThreads);
        mbar_init(&odone[0], 1); mbar_init(&odone[1], 1); mbar_init(spare, 1);
        mbar_init(xw, kSoftThreads); mbar_init(xr, kSoftThreads); mbar_init(spare2, 1);
        *abort_flag = 0;
        mbar_fence_init();
        prefetch_tmap(&tmK); prefetch_tmap(&tmV); prefetch_tmap(&tmKb); prefetch_tmap(&tmVb);
    }
    if (warp == kIssuerWarp) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // q, the lengths and the caches come from earlier kernels. No
    // pdl_trigger: the merge launches as these CTAs exit (see gemm_tc.cu)
    pdl_wait();

    // this CTA's work: tiles [t_lo, t_hi) of item (b, g) (the plan's); an idle CTA has none
    const int slot = blockIdx.x;
    const int item = P.cta_item[slot];
    const int b = item >= 0 ? item / P.nKv : 0, g = item >= 0 ? item % P.nKv : 0;
    const int t_lo = item >= 0 ? P.cta_t0[slot] : 0, t_hi = item >= 0 ? P.cta_t1[slot] : 0;
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

    // The first kSlots K and V tiles do not depend on Q: their loads go out
    // before the Q tile is built, so they land while it is.
    const uint32_t tile_bytes = (uint32_t)nsub * KT * 128;
    if ((warp == kIssuerWarp || warp == kIssuerWarp + 1) && lane == 0) {
        const bool v_tile = warp != kIssuerWarp;
        for (int t = 0; t < kSlots && t < nt; ++t) {
            int row, nvalid; bool blk;
            tile_rows(t, &row, &nvalid, &blk);
            const CUtensorMap* m = blk ? (v_tile ? &tmVb : &tmKb) : (v_tile ? &tmV : &tmK);
            uint64_t* bar = v_tile ? &vfull[t] : &kfull[t];
            mbar_arrive_expect_tx(bar, tile_bytes);
            tma_load_4d((v_tile ? sV : sK) + t * tile_sz, m, bar, 0, row, g, 0);
        }
    }

    // Q tile in tensor memory (the S product's A operand): TMEM lane r holds query
    // row r, two fp16 values per 32-bit column from column kQCol; rows past the
    // queries are zero. The softmax threads write it, thread (r, half) the row's
    // half of the head dimensions, 16 columns per tcgen05.st.
    if (tid < kSoftThreads) {
        const int r = tid & (QROWS - 1), half = tid >> 7;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const int d0 = half * (hd / 2);
        const int i = r / P.grp, h = g * P.grp + r % P.grp;
        const int64_t off = (((int64_t)b * P.G + i) * P.nH + h) * hd + d0;
        for (int c0 = 0; c0 < hd / 4; c0 += 16) {           // 16 columns = 32 dimensions
            uint32_t w[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                float x0 = 0.f, x1 = 0.f;
                if (r < nq) {
                    const int d = 2 * (c0 + j);
                    if (P.q_dtype == DSPARK_DTYPE_F32) {
                        const float2 f = *reinterpret_cast<const float2*>(static_cast<const float*>(P.q) + off + d);
                        x0 = f.x; x1 = f.y;
                    } else {
                        // fp16 queries (the attention seam)
                        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(static_cast<const __half*>(P.q) + off + d));
                        x0 = f.x; x1 = f.y;
                    }
                }
                w[j] = pack_half2(x0, x1);
            }
            tmem_st_x16(tmem + (uint32_t)(kQCol + half * (hd / 4) + c0) + lane_off, w);
        }
        tmem_st_wait();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tO = tmem + 2 * KT;                    // O: columns [128, 128 + hd); S buffers at 0 and 64
    bool ok = true;

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
            int nl[kSlots] = {};                              // loads issued per slot
            for (int t = 0; t < kSlots && t < nt; ++t) ++nl[t];   // issued before the Q tile
            int ln = min(kSlots, nt);                         // next tile to load
            int issued = 0;                                   // products issued
            // tile ln goes into slot ln % kSlots once the product of tile ln - kSlots (the
            // slot's previous tile, phase (ln - kSlots) / kSlots of its barrier) is done
            auto service = [&]() {
                while (ln < nt && ln - kSlots < issued &&
                       mbar_try_wait(&freeb[ln % kSlots], (uint32_t)((ln - kSlots) / kSlots) & 1u)) {
                    load(buf + (ln % kSlots) * tile_sz, &fullb[ln % kSlots], !is_qk, ln);
                    ++nl[ln % kSlots];
                    ++ln;
                }
            };
            auto wait_serving = [&](uint64_t* bar, uint32_t parity) -> bool {
                const uint64_t t0w = global_timer_ns();
                while (!mbar_try_wait(bar, parity)) {
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
                const int ks = t % kSlots;                        // K / V slot
                const uint32_t kph = (uint32_t)(t / kSlots) & 1u;
                if (is_qk) {
                    // S(t) = Q K(t)^T into buffer t % 2
                    if (!wait_serving(&kfull[ks], kph)) { ok = false; break; }
                    if (t >= 2 && !wait_serving(&sfree[sl], (uint32_t)((t - 2) >> 1) & 1u)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t d = tmem + (uint32_t)(sl * KT);
                    // descriptors advance by address / 16: constants per unrolled slice
                    const uint64_t bd0 = sdesc_k_sw128(smem_u32(sK + ks * tile_sz));
                    mma_f16_ts(d, qa, bd0, idesc_qk, 0u);
#pragma unroll
                    for (int j = 1; j < 16; ++j) {
                        if (j >= hd / 16) break;
                        const uint64_t boff = (uint64_t)(((j >> 2) * KT * 128 + (j & 3) * 32) >> 4);
                        mma_f16_ts(d, qa + (uint32_t)(8 * j), bd0 + boff, idesc_qk, 1u);
                    }
                    mma_commit(&sdone[sl]);
                    mma_commit(&kfree[ks]);
                } else {
                    // O += P(t) V(t)
                    if (!wait_serving(&pready[sl], (uint32_t)(t >> 1) & 1u) || !wait_serving(&vready[ks], kph)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad0 = sdesc_k_sw128(smem_u32(sP + sl * QROWS * 128));
                    const uint64_t bd0 = sdesc_mn_sw128(smem_u32(sV + ks * tile_sz), KT * 128);
#pragma unroll
                    for (int j = 0; j < KT / 16; ++j)
                        mma_bf16(tO, ad0 + (uint64_t)((j * 32) >> 4), bd0 + (uint64_t)((j * 2048) >> 4), idesc_pv,
                                 (t > 0 || j > 0) ? 1u : 0u);
                    mma_commit(&odone[sl]);
                    mma_commit(&vfree[ks]);
                }
                issued = t + 1;
                service();
            }
            // teardown after an abort: copies and MMAs in flight land first (bounded)
            if (!ok) {
                const uint64_t deadline = global_timer_ns() + kWaitLimitNs;
                bool drained = true;
                for (int i = 0; i < kSlots; ++i)
                    if (drained && nl[i] > 0) drained = mbar_wait_until(&fullb[i], (uint32_t)(nl[i] - 1) & 1u, deadline);
                uint64_t* sp = is_qk ? spare : spare2;
                mma_commit(sp);
                if (drained) drained = mbar_wait_until(sp, 0u, deadline);
                if (!drained) atomicOr(P.status, DSPARK_DEV_WAIT_TIMEOUT);
            }
        }
    } else if (warp == kFixWarp) {
        // ------------------------------------------------------------ V tails
        for (int t = 0; t < nt && ok; ++t) {
            int row, nvalid; bool blk;
            tile_rows(t, &row, &nvalid, &blk);
            const int ks = t % kSlots;
            if (!warp_wait(&vfull[ks], (uint32_t)(t / kSlots) & 1u, abort_flag, P.status)) { ok = false; break; }
            if (nvalid < KT) {
                zero_tail(sV + ks * tile_sz, nsub, nvalid, lane);
                fence_async_shared();               // the P V product reads the tile through the async proxy
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&vready[ks]);
        }
    } else {
        // ------------------------------------------------------------ softmax (two threads per query row)
        const int r = tid & (QROWS - 1);                   // query row = TMEM lane
        const int half = tid >> 7;                         // S columns [32 half, +32), O columns [hd/2 half, +hd/2)
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const int oc0 = half * (hd / 2);
        float m_run = -INFINITY, l_run = 0.f;              // l_run: this half's columns
        for (int t = 0; t < nt && ok; ++t) {
            int row, nvalid; bool blk;
            tile_rows(t, &row, &nvalid, &blk);
            const int sl = t & 1;
            const uint32_t tS = tmem + (uint32_t)(sl * KT) + lane_off + (uint32_t)(half * 32);
            const int cbase = half * 32;                   // first key of this thread's columns
            if (!warp_wait(&sdone[sl], (uint32_t)(t >> 1) & 1u, abort_flag, P.status)) { ok = false; break; }
            tc_fence_after();
            uint32_t u0[16], u1[16];
            tmem_ld_x16(tS, u0);
            tmem_ld_x16(tS + 16, u1);
            tmem_ld_wait();
            float sv[32];
#pragma unroll
            for (int j = 0; j < 16; ++j) { sv[j] = __uint_as_float(u0[j]); sv[16 + j] = __uint_as_float(u1[j]); }
            if (nvalid < KT) {
#pragma unroll
                for (int j = 0; j < 32; ++j) if (cbase + j >= nvalid) sv[j] = -INFINITY;
            }
            float mt[16];                                   // tree maximum: 5 dependent steps, not 32
#pragma unroll
            for (int j = 0; j < 16; ++j) mt[j] = fmaxf(sv[j], sv[16 + j]);
#pragma unroll
            for (int w = 8; w > 0; w >>= 1) {
#pragma unroll
                for (int j = 0; j < w; ++j) mt[j] = fmaxf(mt[j], mt[j + w]);
            }
            float mx = mt[0];
            // exchange with the other half of the row (mbarriers: every wait stays bounded)
            if (t >= 1 && !warp_wait_spin(xr, (uint32_t)(t - 1) & 1u, abort_flag, P.status)) { ok = false; break; }
            red[half * QROWS + r] = mx;
            mbar_arrive(xw);
            if (!warp_wait_spin(xw, (uint32_t)t & 1u, abort_flag, P.status)) { ok = false; break; }
            mx = fmaxf(mx, red[(half ^ 1) * QROWS + r]);
            mbar_arrive(xr);
            const bool need = t > 0 && mx > m_run + kRescale;
            if (t == 0) m_run = mx;
            if (__any_sync(0xffffffffu, need)) {
                // O holds tiles up to t - 1 at the old max: P(t-1) V(t-1) must have landed
                if (t >= 1 && !warp_wait(&odone[(t - 1) & 1], (uint32_t)((t - 1) >> 1) & 1u, abort_flag, P.status)) { ok = false; break; }
                tc_fence_after();
                const float f = need ? __expf(m_run - mx) : 1.f;
                if (need) { l_run *= f; m_run = mx; }
                for (int c = 0; c < hd / 2; c += 16) {
                    uint32_t u[16];
                    tmem_ld_x16(tO + lane_off + (uint32_t)(oc0 + c), u);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 16; ++j) u[j] = __float_as_uint(__uint_as_float(u[j]) * f);
                    tmem_st_x16(tO + lane_off + (uint32_t)(oc0 + c), u);
                }
                tmem_st_wait();
            }
            // P slot t % 2 was last read by P(t-2) V(t-2)
            if (t >= 2 && !warp_wait(&odone[sl], (uint32_t)((t - 2) >> 1) & 1u, abort_flag, P.status)) { ok = false; break; }
            float ls[8];                                    // sums in 8 independent chains
#pragma unroll
            for (int j = 0; j < 8; ++j) ls[j] = 0.f;
            uint8_t* pslot = sP + sl * QROWS * 128;
#pragma unroll
            for (int q = 0; q < 4; ++q) {                  // four 16-byte chunks of 8 keys
                float p[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) { p[j] = __expf(sv[q * 8 + j] - m_run); ls[j] += p[j]; }
                const int chunk = (cbase >> 3) + q;
                *reinterpret_cast<uint4*>(pslot + r * 128 + ((chunk ^ (r & 7)) * 16)) =
                    make_uint4(pack_half2(p[0], p[1]), pack_half2(p[2], p[3]), pack_half2(p[4], p[5]), pack_half2(p[6], p[7]));
            }
            const float lsum = ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
            l_run += lsum;
            tc_fence_before();
            mbar_arrive(&sfree[sl]);                           // S buffer read
            fence_async_shared();
            mbar_arrive(&pready[sl]);                          // P written
        }
        // ---- this range's state: unnormalised O and (max, sum) per query row
        const bool any = nt > 0;
        if (any && ok && !warp_wait(&odone[(nt - 1) & 1], (uint32_t)((nt - 1) >> 1) & 1u, abort_flag, P.status)) ok = false;
        tc_fence_after();
        // the row's sum = both halves' sums (same running max): one more exchange
        float l_tot = l_run;
        if (any && ok) {
            if (!warp_wait(xr, (uint32_t)(nt - 1) & 1u, abort_flag, P.status)) ok = false;
            if (ok) {
                red[half * QROWS + r] = l_run;
                mbar_arrive(xw);
                if (!warp_wait(xw, (uint32_t)nt & 1u, abort_flag, P.status)) ok = false;
                else l_tot = l_run + red[(half ^ 1) * QROWS + r];
            }
        }
        if (r < nq && half == 0) {
            const int64_t prow = (int64_t)slot * QROWS + r;
            P.part_ml[prow * 2] = any ? m_run : -INFINITY;
            P.part_ml[prow * 2 + 1] = any ? l_tot : 0.f;
        }
        if (any && ok) {
            float* dst = P.part_o + ((int64_t)slot * QROWS + r) * hd + oc0;
            // 32 columns per TMEM wait: half the waits, stores of 128 contiguous bytes
            for (int c = 0; c < hd / 2; c += 32) {
                uint32_t u[2][16];
                tmem_ld_x16(tO + lane_off + (uint32_t)(oc0 + c), u[0]);
                tmem_ld_x16(tO + lane_off + (uint32_t)(oc0 + c + 16), u[1]);
                tmem_ld_wait();
                if (r < nq) {
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        *reinterpret_cast<float4*>(dst + c + j) =
                            make_float4(__uint_as_float(u[j >> 4][j & 15]), __uint_as_float(u[j >> 4][(j & 15) + 1]),
                                        __uint_as_float(u[j >> 4][(j & 15) + 2]), __uint_as_float(u[j >> 4][(j & 15) + 3]));
                }
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
    // tile, laid out [chunk][key][64] = nsub K-major sub-tiles of KT rows
    cuuint64_t dims[4] = {64, (cuuint64_t)rows, (cuuint64_t)nKv, (cuuint64_t)(hd / 64)};
    cuuint64_t strides[3] = {(cuuint64_t)nKv * hd * 2, (cuuint64_t)hd * 2, 128};
    cuuint32_t box[4] = {64, (cuuint32_t)KT, 1, (cuuint32_t)(hd / 64)};   // KT <= 256
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return g_enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t attn_tc_smem(int hd) {
    const int nsub = hd / 64;
    // K and V (kSlots each), P (2 slots), row maxima, then the barriers (5 kSlots + 12),
    // the TMEM slot and the abort flag; 1 KB alignment slack
    return 2 * (size_t)kSlots * nsub * KT * 128 + 2 * QROWS * 128 + 2 * QROWS * 4 + 8 * (5 * kSlots + 12) + 16 + 1024;
}

}  // namespace

// One warp per output row (b, h, i): the item's slots item_cta0[item] ..
// item_cta0[item + 1] - 1, row r = i * grp + h % grp of each; the weights
// w_s = exp(m_s - M) combine the unnormalised outputs (lane l owns the 4-column
// groups l, l + 32 of the row). Slots of empty ranges (m = -inf) weigh nothing.
constexpr int kMergeWarps = 8;
constexpr int kMergeBatch = 16;      // slots a merge lane loads at once
__global__ void __launch_bounds__(kMergeWarps * 32) attn_tc_merge_kernel(AttnArgs a, const int* __restrict__ item_cta0,
                                                                         int G, int nH, int nKv, int hd, int rows) {
    pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * kMergeWarps + (threadIdx.x >> 5);   // ((b * nH) + h) * G + i
    if (row >= rows) return;
    const int i = row % G, bh = row / G;
    const int b = bh / nH, h = bh % nH;
    const int grp = nH / nKv;
    const int item = b * nKv + h / grp, r = i * grp + h % grp;
    const int s0 = item_cta0[item], s1 = item_cta0[item + 1];
    float M = -INFINITY;
    for (int s = s0 + lane; s < s1; s += 32) M = fmaxf(M, a.part_ml[((int64_t)s * QROWS + r) * 2]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const int ng = hd / 4;
    float4 num[2] = {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};
    float den = 0.f;
    for (int sb = s0; sb < s1; sb += 32) {
        float ws = 0.f, ls = 0.f;
        if (sb + lane < s1) {
            const int64_t base = (int64_t)(sb + lane) * QROWS + r;
            const float m = a.part_ml[base * 2];
            ls = a.part_ml[base * 2 + 1];
            ws = m == -INFINITY ? 0.f : __expf(m - M);
        }
        const int cnt = min(32, s1 - sb);
        // kMergeBatch slots' loads in flight at once, then their weighted sum in slot order
        for (int t0 = 0; t0 < cnt; t0 += kMergeBatch) {
            float4 v[kMergeBatch][2];
#pragma unroll
            for (int u = 0; u < kMergeBatch; ++u) {
                const float* o = a.part_o + ((int64_t)(sb + t0 + u) * QROWS + r) * hd;
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int g4 = lane + q * 32;
                    v[u][q] = (t0 + u < cnt && g4 < ng) ? reinterpret_cast<const float4*>(o)[g4]
                                                         : make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
#pragma unroll
            for (int u = 0; u < kMergeBatch; ++u) {
                const float w = __shfl_sync(0xffffffffu, ws, (t0 + u) & 31);
                const float l = __shfl_sync(0xffffffffu, ls, (t0 + u) & 31);
                if (t0 + u >= cnt) break;
                den += w * l;
                if (w == 0.f) continue;                // uniform: an empty range (its O slot is not written)
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    num[q].x += w * v[u][q].x; num[q].y += w * v[u][q].y;
                    num[q].z += w * v[u][q].z; num[q].w += w * v[u][q].w;
                }
            }
        }
    }
    const float inv = 1.f / den;
    const int64_t ob = (((int64_t)b * G + i) * nH + h) * hd;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        const int g4 = lane + q * 32;
        if (g4 >= ng) continue;
        const float v[4] = {num[q].x * inv, num[q].y * inv, num[q].z * inv, num[q].w * inv};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int64_t o = ob + g4 * 4 + c;
            store_any(a.out, o, a.out_dtype, v[c]);
            if (a.out_hi) {
                const __half hv = __float2half_rn(v[c]);
                a.out_hi[o] = hv;
                if (a.out_lo) a.out_lo[o] = __float2half_rn(v[c] - __half2float(hv));
            }
        }
    }
}

bool attention_tc_supported(const dspark_model* m) {
    const Dims& d = m->d;
    return d.dtype == DSPARK_DTYPE_BF16 && d.grp * d.gamma <= QROWS && d.hd % 64 == 0 && d.hd <= 256;
}

int attention_tc_key_tile() { return KT; }

int attention_tc_grid(const dspark_model* m, int A) { return std::max(m->num_sms, A * m->d.nKv); }

size_t attention_tc_plan_ints(const dspark_model* m, int A, int grid) {
    return 3 * (size_t)grid + (size_t)A * m->d.nKv + 1;
}

size_t attention_tc_partial_floats(const dspark_model* m, int grid) { return (size_t)grid * QROWS * (m->d.hd + 2); }

cudaError_t launch_attention_tc(const dspark_model* m, const AttnArgs& a, cudaStream_t s) {
    const Dims& d = m->d;
    if (!a.plan || a.tc_grid < std::max(1, a.A * d.nKv)) return cudaErrorInvalidValue;
    CUtensorMap tk, tv, tkb, tvb;
    const int64_t cache_rows = (int64_t)a.batch * a.capacity;   // all rows of this layer's cache
    if (!make_kv_map(&tk, a.kc, cache_rows, d.nKv, d.hd) || !make_kv_map(&tv, a.vc, cache_rows, d.nKv, d.hd) ||
        !make_kv_map(&tkb, a.kb, (int64_t)a.A * d.gamma, d.nKv, d.hd) ||
        !make_kv_map(&tvb, a.vb, (int64_t)a.A * d.gamma, d.nKv, d.hd))
        return cudaErrorInvalidValue;
    const int grid = a.tc_grid;
    int* cta_item = a.plan;
    int* cta_t0 = cta_item + grid;
    int* cta_t1 = cta_t0 + grid;
    int* item_cta0 = cta_t1 + grid;
    cudaError_t e = cudaSuccess;
    if (!a.plan_ready)      // the plan depends only on the lengths: a round computes it for its first layer
        e = launch_pdl(attn_plan_kernel, dim3(1), dim3(kPlanThreads), 0, s, a.len, a.A, d.nKv, a.capacity, grid,
                       cta_item, cta_t0, cta_t1, item_cta0);
    if (e != cudaSuccess) return e;
    AttnTcParams P{};
    P.A = a.A; P.G = d.gamma; P.nH = d.nH; P.nKv = d.nKv; P.grp = d.grp; P.hd = d.hd; P.capacity = a.capacity;
    P.q_dtype = a.q_dtype; P.q = a.q; P.len = a.len;
    P.part_o = a.part_o; P.part_ml = a.part_ml; P.status = a.status;
    P.cta_item = cta_item; P.cta_t0 = cta_t0; P.cta_t1 = cta_t1;
    const size_t smem = attn_tc_smem(d.hd);
    e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(attn_tc_kernel, dim3(grid), dim3(kThreads), smem, s, tk, tv, tkb, tvb, P);
    if (e != cudaSuccess) return e;
    const int rows = a.A * d.nH * d.gamma;
    return launch_pdl(attn_tc_merge_kernel, dim3((rows + kMergeWarps - 1) / kMergeWarps), dim3(kMergeWarps * 32), 0, s,
                      a, item_cta0, d.gamma, d.nH, d.nKv, d.hd, rows);
}

}  // namespace tc
}  // namespace dspark
