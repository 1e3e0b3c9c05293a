// KV-injection attention on tcgen05 tensor cores: the
// DeepspecContextAttention.attend seam ("mlx-bun 0.2.0 -> 0.4.0" page 75,
// plainDeepspecContext): the block queries of one row attend, non-causally
// and at scale 1.0, over the row's cached context keys followed by the
// block's own keys; GQA maps query head h to kv head h / (nH / nKv).
//
// One CTA = (row b, kv head g, key split). Its query tile is the 128-row MMA
// side: the grp * gamma queries of the heads that share kv head g (row r =
// query i * grp + head-in-group). Key tiles of KT = 64 rows are TMA-loaded
// from the bf16 cache (3-D maps pick kv head g out of [rows, nKv, hd]) and
// converted in place to fp16, so both MMAs run as kind::f16 with fp16
// operands: q and the probabilities P keep an 11-bit mantissa (bf16 has 8)
// and the bf16 keys and values convert exactly.
//   S = Q K^T  -> TMEM, two 64-column buffers (tile t in buffer t % 2)
//   softmax    -> one thread per query row (TMEM lane = row); the running max
//                 is raised only when a tile's max exceeds it by more than
//                 kRescale, so O is rarely rescaled in TMEM
//   O += P V   -> TMEM (hd columns), P fp16 from shared memory (K-major,
//                 128-byte swizzle), V as an MN-major operand
// K and V tiles have two shared-memory slots each, so the loads of tile t + 2
// are in flight while tile t is converted and multiplied; per 64 keys at
// hd = 256 the tensor cores run 16 (S) + 4 (P V) MMAs.
//
// Warp roles (576 threads): warps 0-7 run the softmax, two threads per query
// row (warps w and w + 4 share TMEM lanes 32 (w % 4) ..; each takes 32 of the
// tile's 64 columns and half of O's columns; the row max is exchanged through
// shared memory), warps 8-15 convert K and V tiles (and zero the rows past the
// last key: stale cache bytes could be NaN, and P = 0 times NaN still poisons
// the accumulator), warp 16 issues the S products and K loads, warp 17 the
// P V products and V loads. K, V and P have two
// slots each and S two TMEM buffers, so tile t + 1's load, conversion and S
// product and tile t - 1's P V product all overlap tile t's softmax; the
// softmax waits for P V of tile t - 1 only to rescale O (rare). Every wait is
// bounded. Shared memory at hd = 256: Q 64 KB, K, V 2 x 32 KB each, P 2 x 16 KB.
//
// The CTA writes its unnormalised O with (max, sum) per query row: the split
// layout the merge kernel reads. The last split of each (b, g) also takes the
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

cudaError_t launch_attention_merge(const dspark_model* m, const AttnArgs& a, cudaStream_t s);

namespace tc {
namespace {

constexpr int kThreads = 576;
constexpr int kSoftThreads = 256;    // warps 0-7
constexpr int kConvThreads = 256;    // warps 8-15
constexpr int kIssuerWarp = 16;      // S products and K loads; warp 17: P V products and V loads
constexpr int KT = 64;               // keys per tile
constexpr int QROWS = 128;           // MMA M
constexpr float kRescale = 5.0f;     // natural-log headroom before the running max is raised

struct AttnTcParams {
    int A, G, nH, nKv, grp, hd, capacity, S1, chunk, q_dtype;
    const void* q;                   // [A, G, nH, hd] (fp32 or bf16)
    const int32_t* len;
    float* part_o; float* part_ml;
    int32_t* status;
};

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// bf16 -> fp16 in place over a tile of `nsub` sub-tiles [KT rows x 128 B] by
// the converter threads; rows >= nvalid become zeros.
// Each thread owns 16-byte chunks ct, ct + kConvThreads, ...; all its loads
// are issued before the first conversion (one round of shared-memory latency).
__device__ __forceinline__ void convert_tile(uint8_t* tile, int nsub, int nvalid, int ct) {
    constexpr int kPer = 4 * KT * 8 / kConvThreads;    // chunks per thread at nsub = 4
    const int n16 = nsub * KT * 8;
    uint4* p = reinterpret_cast<uint4*>(tile);
    uint4 u[kPer];
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
        const int i = ct + k * kConvThreads;
        u[k] = i < n16 ? p[i] : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
        const int i = ct + k * kConvThreads;
        if (i >= n16) break;
        const int row = (i >> 3) % KT;
        if (row >= nvalid) { p[i] = make_uint4(0u, 0u, 0u, 0u); continue; }
        const uint32_t w[4] = {u[k].x, u[k].y, u[k].z, u[k].w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) o[j] = pack_half2(__uint_as_float(w[j] << 16), __uint_as_float(w[j] & 0xffff0000u));
        p[i] = make_uint4(o[0], o[1], o[2], o[3]);
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
    uint8_t* sQ = base;                                   // nsub x [128 rows x 128 B] fp16
    uint8_t* sK = sQ + nsub * QROWS * 128;                // 2 slots x tile
    uint8_t* sV = sK + 2 * tile_sz;                       // 2 slots x tile
    uint8_t* sP = sV + 2 * tile_sz;                       // 2 slots x [128 rows x 128 B]
    float* red = reinterpret_cast<float*>(sP + 2 * QROWS * 128);   // [2 halves][128 rows] row maxima / sums
    uint64_t* bars = reinterpret_cast<uint64_t*>(red + 2 * QROWS);
    uint64_t* kfull = bars + 0;      // [2] K tile landed in the slot (TMA)
    uint64_t* vfull = bars + 2;      // [2] V tile landed in the slot (TMA)
    uint64_t* kready = bars + 4;     // [2] K tile of the slot converted (128 arrivals)
    uint64_t* vready = bars + 6;     // [2] V tile of the slot converted (128 arrivals)
    uint64_t* sdone = bars + 8;      // [2] S product of the tile in that buffer done (its K slot free)
    uint64_t* sfree = bars + 10;     // [2] softmax has read the S buffer (128 arrivals)
    uint64_t* pready = bars + 12;    // [2] P slot written (256 arrivals)
    uint64_t* odone = bars + 14;     // [2] P V product of the tile in that P slot done (its V slot free, O settled)
    uint64_t* spare = bars + 16;     // teardown: MMAs in flight after an abort
    uint64_t* xw = bars + 17;        // row-max exchange: both halves wrote (256 arrivals)
    uint64_t* xr = bars + 18;        // row-max exchange: both halves read (256 arrivals)
    uint64_t* spare2 = bars + 19;    // teardown of the P V issuer
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 20);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x;                            // b * nKv + g
    const int b = bh / P.nKv, g = bh % P.nKv;
    const int split = blockIdx.y;
    const int nq = P.grp * P.G;

    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&kfull[i], 1); mbar_init(&vfull[i], 1);
            mbar_init(&kready[i], kConvThreads); mbar_init(&vready[i], kConvThreads);
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

    int len = P.len[b];
    if (len < 0 || len > P.capacity) {
        if (tid == 0) atomicOr(P.status, DSPARK_DEV_BAD_LENGTH);
        len = min(max(len, 0), P.capacity);
    }
    // this split's context keys [c0, c1), then (last split) the block's G keys
    const int c0 = min(len, split * P.chunk), c1 = min(len, c0 + P.chunk);
    const bool has_blk = split == P.S1 - 1;
    const int n_ctx = (c1 - c0 + KT - 1) / KT;
    const int nt = n_ctx + (has_blk ? 1 : 0);
    auto tile_rows = [&](int t, int* row, int* nvalid, bool* blk) {
        if (t < n_ctx) { *row = b * P.capacity + c0 + t * KT; *nvalid = min(KT, c1 - (c0 + t * KT)); *blk = false; }
        else { *row = b * P.G; *nvalid = P.G; *blk = true; }
    };

    // The first two K and V tiles do not depend on Q: their loads go out
    // before the Q tile is built, so they land while it is.
    const uint32_t tile_bytes = (uint32_t)nsub * KT * 128;
    if ((warp == kIssuerWarp || warp == kIssuerWarp + 1) && lane == 0) {
        const bool v_tile = warp != kIssuerWarp;
        for (int t = 0; t < 2 && t < nt; ++t) {
            int row, nvalid; bool blk;
            tile_rows(t, &row, &nvalid, &blk);
            const CUtensorMap* m = blk ? (v_tile ? &tmVb : &tmKb) : (v_tile ? &tmV : &tmK);
            uint64_t* bar = v_tile ? &vfull[t] : &kfull[t];
            mbar_arrive_expect_tx(bar, tile_bytes);
            tma_load_4d((v_tile ? sV : sK) + t * tile_sz, m, bar, 0, row, g, 0);
        }
    }

    // Q tile (all warps): fp16, 128-byte swizzle; rows past the queries are zero.
    // Each thread's rows are loaded kQBatch at a time before any is converted:
    // a few rounds of memory latency instead of one per row.
    constexpr int kQBatch = 4;
    for (int cd = 0; cd < hd; cd += 256) {
        const int d = cd + lane * 8;
        const int sub = d / 64, chunk = (d % 64) / 8;
        for (int row0 = warp; row0 < QROWS; row0 += kQBatch * (kThreads / 32)) {
            float v[kQBatch][8];
#pragma unroll
            for (int k = 0; k < kQBatch; ++k) {
                const int row = row0 + k * (kThreads / 32);
#pragma unroll
                for (int j = 0; j < 8; ++j) v[k][j] = 0.f;
                if (row < nq && d < hd) {
                    const int i = row / P.grp, h = g * P.grp + row % P.grp;
                    const int64_t off = (((int64_t)b * P.G + i) * P.nH + h) * hd + d;
                    if (P.q_dtype == DSPARK_DTYPE_F32) {
                        const float4 a0 = *reinterpret_cast<const float4*>(static_cast<const float*>(P.q) + off);
                        const float4 a1 = *reinterpret_cast<const float4*>(static_cast<const float*>(P.q) + off + 4);
                        v[k][0] = a0.x; v[k][1] = a0.y; v[k][2] = a0.z; v[k][3] = a0.w;
                        v[k][4] = a1.x; v[k][5] = a1.y; v[k][6] = a1.z; v[k][7] = a1.w;
                    } else {
                        const uint4 u = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(P.q) + off);
                        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            v[k][2 * j] = __uint_as_float(w[j] << 16);
                            v[k][2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
                        }
                    }
                }
            }
#pragma unroll
            for (int k = 0; k < kQBatch; ++k) {
                const int row = row0 + k * (kThreads / 32);
                if (row < QROWS && d < hd)
                    *reinterpret_cast<uint4*>(sQ + sub * QROWS * 128 + row * 128 + ((chunk ^ (row & 7)) * 16)) =
                        make_uint4(pack_half2(v[k][0], v[k][1]), pack_half2(v[k][2], v[k][3]),
                                   pack_half2(v[k][4], v[k][5]), pack_half2(v[k][6], v[k][7]));
            }
        }
    }
    fence_async_shared();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tO = tmem + 2 * KT;                    // O: columns [128, 128 + hd); S buffers at 0 and 64
    bool ok = true;

    if (warp >= kIssuerWarp) {
        // ------------------------------------------------------------ issuers
        // warp 16: S = Q K^T and the K loads; warp 17: O += P V and the V loads.
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
            uint64_t* doneb = is_qk ? sdone : odone;          // completion of the product that read a slot
            int nl[2] = {0, 0};                               // loads issued per slot
            for (int t = 0; t < 2 && t < nt; ++t) ++nl[t];    // tiles 0 and 1: issued before the Q tile
            int ln = min(2, nt);                              // next tile to load
            int issued = 0;                                   // products issued
            auto service = [&]() {
                while (ln < nt && ln - 2 < issued && mbar_try_wait(&doneb[ln & 1], (uint32_t)((ln - 2) >> 1) & 1u)) {
                    load(buf + (ln & 1) * tile_sz, &fullb[ln & 1], !is_qk, ln); ++nl[ln & 1]; ++ln;
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
            const uint32_t qa = smem_u32(sQ);
            for (int t = 0; t < nt && ok; ++t) {
                const int sl = t & 1;
                if (is_qk) {
                    // S(t) = Q K(t)^T into buffer t % 2
                    if (!wait_serving(&kready[sl], (uint32_t)(t >> 1) & 1u)) { ok = false; break; }
                    if (t >= 2 && !wait_serving(&sfree[sl], (uint32_t)((t - 2) >> 1) & 1u)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t d = tmem + (uint32_t)(sl * KT);
                    // descriptors advance by address / 16: constants per unrolled slice
                    const uint64_t ad0 = sdesc_k_sw128(qa);
                    const uint64_t bd0 = sdesc_k_sw128(smem_u32(sK + sl * tile_sz));
                    mma_bf16(d, ad0, bd0, idesc_qk, 0u);
#pragma unroll
                    for (int j = 1; j < 16; ++j) {
                        if (j >= hd / 16) break;
                        const uint64_t aoff = (uint64_t)(((j >> 2) * QROWS * 128 + (j & 3) * 32) >> 4);
                        const uint64_t boff = (uint64_t)(((j >> 2) * KT * 128 + (j & 3) * 32) >> 4);
                        mma_bf16(d, ad0 + aoff, bd0 + boff, idesc_qk, 1u);
                    }
                    mma_commit(&sdone[sl]);
                } else {
                    // O += P(t) V(t)
                    if (!wait_serving(&pready[sl], (uint32_t)(t >> 1) & 1u) ||
                        !wait_serving(&vready[sl], (uint32_t)(t >> 1) & 1u)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t ad0 = sdesc_k_sw128(smem_u32(sP + sl * QROWS * 128));
                    const uint64_t bd0 = sdesc_mn_sw128(smem_u32(sV + sl * tile_sz), KT * 128);
#pragma unroll
                    for (int j = 0; j < KT / 16; ++j)
                        mma_bf16(tO, ad0 + (uint64_t)((j * 32) >> 4), bd0 + (uint64_t)((j * 2048) >> 4), idesc_pv,
                                 (t > 0 || j > 0) ? 1u : 0u);
                    mma_commit(&odone[sl]);
                }
                issued = t + 1;
                service();
            }
            // teardown after an abort: copies and MMAs in flight land first (bounded)
            if (!ok) {
                const uint64_t deadline = global_timer_ns() + kWaitLimitNs;
                bool drained = true;
                for (int i = 0; i < 2; ++i)
                    if (drained && nl[i] > 0) drained = mbar_wait_until(&fullb[i], (uint32_t)(nl[i] - 1) & 1u, deadline);
                uint64_t* sp = is_qk ? spare : spare2;
                mma_commit(sp);
                if (drained) drained = mbar_wait_until(sp, 0u, deadline);
                if (!drained) atomicOr(P.status, DSPARK_DEV_WAIT_TIMEOUT);
            }
        }
    } else if (warp >= kSoftThreads / 32) {
        // ------------------------------------------------------------ converters
        const int ct = tid - kSoftThreads;
        for (int t = 0; t < nt && ok; ++t) {
            int row, nvalid; bool blk;
            tile_rows(t, &row, &nvalid, &blk);
            const int sl = t & 1;
            const uint32_t ph = (uint32_t)(t >> 1) & 1u;
            if (!mbar_wait(&kfull[sl], ph, abort_flag, P.status)) { ok = false; break; }
            convert_tile(sK + sl * tile_sz, nsub, nvalid, ct);
            fence_async_shared();
            mbar_arrive(&kready[sl]);
            if (!mbar_wait(&vfull[sl], ph, abort_flag, P.status)) { ok = false; break; }
            convert_tile(sV + sl * tile_sz, nsub, nvalid, ct);
            fence_async_shared();
            mbar_arrive(&vready[sl]);
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
        // ---- this split's state: unnormalised O and (max, sum) per query row
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
            const int i = r / P.grp, h = g * P.grp + r % P.grp;
            const int64_t prow = ((int64_t)(b * P.nH + h) * P.S1 + split) * P.G + i;
            P.part_ml[prow * 2] = any ? m_run : -INFINITY;
            P.part_ml[prow * 2 + 1] = any ? l_tot : 0.f;
        }
        if (any && ok) {
            const int i = r / P.grp, h = g * P.grp + r % P.grp;
            float* dst = P.part_o + (((int64_t)(b * P.nH + h) * P.S1 + split) * P.G + i) * hd + oc0;
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
    // Q, K (2 slots), V (2 slots), P (2 slots), row maxima, then 20 barriers + TMEM slot + abort
    // flag; 1 KB alignment slack
    return (size_t)nsub * QROWS * 128 + 4 * (size_t)nsub * KT * 128 + 2 * QROWS * 128 + 2 * QROWS * 4 + 192 + 1024;
}

}  // namespace

bool attention_tc_supported(const dspark_model* m) {
    const Dims& d = m->d;
    return d.dtype == DSPARK_DTYPE_BF16 && d.grp * d.gamma <= QROWS && d.hd % 64 == 0 && d.hd <= 256;
}

int attention_tc_key_tile() { return KT; }

cudaError_t launch_attention_tc(const dspark_model* m, const AttnArgs& a_in, cudaStream_t s) {
    AttnArgs a = a_in;
    a.S1 = std::max(1, a.n_splits);             // the last context split also takes the block keys
    const Dims& d = m->d;
    CUtensorMap tk, tv, tkb, tvb;
    const int64_t cache_rows = (int64_t)a.batch * a.capacity;   // all rows of this layer's cache
    if (!make_kv_map(&tk, a.kc, cache_rows, d.nKv, d.hd) || !make_kv_map(&tv, a.vc, cache_rows, d.nKv, d.hd) ||
        !make_kv_map(&tkb, a.kb, (int64_t)a.A * d.gamma, d.nKv, d.hd) ||
        !make_kv_map(&tvb, a.vb, (int64_t)a.A * d.gamma, d.nKv, d.hd))
        return cudaErrorInvalidValue;
    AttnTcParams P{};
    P.A = a.A; P.G = d.gamma; P.nH = d.nH; P.nKv = d.nKv; P.grp = d.grp; P.hd = d.hd; P.capacity = a.capacity;
    P.S1 = a.S1; P.chunk = a.chunk; P.q_dtype = a.q_dtype; P.q = a.q; P.len = a.len;
    P.part_o = a.part_o; P.part_ml = a.part_ml; P.status = a.status;
    const size_t smem = attn_tc_smem(d.hd);
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(a.A * d.nKv, a.S1);
    e = launch_pdl(attn_tc_kernel, grid, dim3(kThreads), smem, s, tk, tv, tkb, tvb, P);
    if (e != cudaSuccess) return e;
    return launch_attention_merge(m, a, s);
}

}  // namespace tc
}  // namespace dspark
