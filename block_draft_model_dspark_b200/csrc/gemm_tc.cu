// Tensor-core GEMM for sm_100a: out = X @ W^T with bf16 operands and fp32
// accumulation in TMEM (deepspec.ts `matmulW`: x @ W^T for a Linear weight
// stored [out, in]).
//
// Orientation ("swap-AB"): the weight supplies the MMA's 128-row A operand
// (128 output features per tile) and the activation rows supply its N side
// (BN = 16..256 columns), so a round with 16 activation rows still runs full
// 128-row MMAs and streams each weight tile exactly once.
//
// Operands are staged by TMA with the 128-byte swizzle into a ring of
// shared-memory stages. An fp32 activation enters as a bf16 pair (hi, lo =
// x - hi), stored as one [2][M][K] block: when 2 BN <= 256 the pair is one B
// operand of 2 BN rows and one MMA per K slice produces both products in
// adjacent accumulator columns (summed in the epilogue), else two MMAs per
// slice accumulate into the same columns. The activation keeps ~16
// significant bits while the weight streams once.
//
// A stage spans KSUB = 2 K blocks of 64 when K allows: one TMA request brings
// the stage's 2 x 16 KB of weights (a 3-D map whose third dimension steps
// 128 bytes along K) and one brings its activation rows (hi and lo, both K
// blocks). A single producer thread issues every request, and its issue
// rate, not HBM, bounded the weight stream at one request per 4 KB of X or
// 16 KB of W.
//
// Roles (448 threads): warp 0 issues TMA loads, warp 1 owns TMEM and issues
// MMAs, warps 2-13 drain accumulators (TMEM lane quadrant = warp % 4; warps w,
// w + 4 and w + 8 take every third 16-column chunk); with 4-bit weights (320
// threads) warps 2-5 drain and warps 6-9 dequantize the weight tiles.
// Accumulators are double-buffered in TMEM so the epilogue of one tile
// overlaps the MMAs of the next.
//
// Work split: the grid is persistent (at most one CTA per SM). In stream-K
// mode the tiles' K-blocks form one sequence cut into equal contiguous
// ranges, one per CTA; a CTA writes one fp32 partial tile per tile it
// touches, and the consuming kernel sums a tile's partials in CTA order (no
// atomics, no wait between CTAs: deterministic). In tile mode each CTA owns
// whole tiles (round-robin) and the epilogue writes the result directly,
// optionally with the final-logit softcap.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <string>

#include "internal.h"
#include "common.cuh"
#include "gemm_tc.h"
#include "tmap.h"
#include "tc_ptx.cuh"
#include "logit_stats.cuh"

namespace dspark {
namespace tc {
namespace {

constexpr int BM = 128;            // weight rows per tile (MMA M)
constexpr int BK = 64;             // K elements per K block: one 128-byte swizzle row
constexpr int kThreads = 192;      // TMA, MMA and four epilogue warps
constexpr int kConvThreads = 128;  // the weight-transform warps (one weight row each)
// Epilogue warps: twelve (three per TMEM lane quadrant, taking every third
// 16-column chunk) for the 16-bit weight formats, whose drain of softcapped
// logits and their statistics otherwise outlasts a tile's MMAs (eight measured
// 4% slower at the lm-head of 512 positions; 448 threads leave 146 registers a
// thread); four beside the 4-bit dequantizing warps.
__host__ __device__ constexpr int epi_warps_for(int wfmt) { return wfmt == kWQ4AsF16 ? 4 : 12; }
constexpr int kABytes = BM * BK * 2;   // one K block of weights (16 KB)
// threads of a launch: the weight-transform formats add the converter warps (warps 6-9)
__host__ __device__ constexpr int threads_for(int wfmt) {
    return 64 + 32 * epi_warps_for(wfmt) + (wfmt == kWQ4AsF16 ? kConvThreads : 0);
}
constexpr int kMaxStages = 12;
constexpr int kSmemLimit = 227 * 1024;   // dynamic shared memory a CTA may opt into
// alignment slack + full/empty barriers per stage + 4 accumulator barriers,
// the TMEM slot and the abort flag (plus one spare word)
constexpr int kSmemExtra(int stages) { return 1024 + 24 * stages + 32 + 16 + 64; }
// shared memory of the epilogue's logit statistics: [4 warps][BN] WarpStat
constexpr int kStatBytes(int BN) { return 4 * BN * (int)sizeof(WarpStat); }

struct KParams {
    GemmPlan p;
    float* out;        // result rows out[m * ldo + n]
    int64_t ldo;
    float cap;         // softcap of the result (0 = none)
    float cap_inv;     // 1 / cap
    float* part;       // stream-K partial tiles [tile][P][BN][128]
    int32_t* status;
    TileStats stats;               // tile mode: per (128-row weight tile, activation row) logit statistics
    const float* w2norm;           // with stats: |markov_w2[n]| bounds (NULL: no lo / hi)
    const uint32_t* w1max_bits;    // max_p |markov_w1[p]| as float bits
    const void* wq4;               // kWQ4*: the packed 4-bit blocks [tile][K block]
};

struct Q4Pieces {
    Q4Piece p[kMaxQ4Pieces];
    int n;
};

// Iterates the (tile, k-range) segments of one work unit (a CTA, or a CTA pair),
// identically in every role.
struct SegIter {
    const GemmPlan& p;
    int c;
    int g, g1;      // stream-K: this CTA's remaining global K-block range
    int t;          // tile mode: next tile
    __device__ SegIter(const GemmPlan& p_, int c_) : p(p_), c(c_) {
        g = p.streamk ? p.range_lo(c) : 0;
        g1 = p.streamk ? p.range_lo(c + 1) : 0;
        t = c;
    }
    __device__ bool next(int& tile, int& k0, int& k1, int& slot) {
        if (p.streamk) {
            if (g >= g1) return false;
            tile = g / p.kb;
            k0 = g - tile * p.kb;
            k1 = min(p.kb, k0 + (g1 - g));
            slot = c - p.cta_of(tile * p.kb);
            g += k1 - k0;
            return true;
        }
        if (t >= p.tiles) return false;
        tile = t; k0 = 0; k1 = p.kb; slot = 0;
        t += p.units;
        return true;
    }
};

// Eight 4-bit codes of one 32-bit word (code j in bits 4j..4j+3) dequantized to
// scale * code + bias with one rounding, as 8 fp16 in element order. Each code
// becomes the exact fp16 value 1024 + code by OR-ing it under a fixed exponent;
// subtracting 1024 is exact, and the fused multiply-add rounds once.
__device__ __forceinline__ uint4 q4x8_dequant(uint32_t w, uint32_t s2, uint32_t b2) {
    const uint32_t magic = 0x64006400u;     // 1024.0 in both halves
    uint32_t v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t t = ((w >> (4 * k)) & 0x000F000Fu) | magic;   // codes k (low half) and k + 4 (high half)
        const __half2 c = __hsub2(*reinterpret_cast<const __half2*>(&t), *reinterpret_cast<const __half2*>(&magic));
        const __half2 r = __hfma2(c, *reinterpret_cast<const __half2*>(&s2), *reinterpret_cast<const __half2*>(&b2));
        v[k] = *reinterpret_cast<const uint32_t*>(&r);
    }
    // v[k] holds elements (k, k + 4): regroup to (0,1) (2,3) (4,5) (6,7)
    return make_uint4(__byte_perm(v[0], v[1], 0x5410), __byte_perm(v[2], v[3], 0x5410),
                      __byte_perm(v[0], v[1], 0x7632), __byte_perm(v[2], v[3], 0x7632));
}

// tanh by the hardware's approximation (relative error about 2^-11): the
// final-logit softcap cap * tanh(x / cap) then stays within 5e-4 |U| of the exact
// value, far inside the logits' 2e-2 relative bar, at one instruction per logit.
__device__ __forceinline__ float tanh_fast(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// KSUB K blocks per stage; stage layout [KSUB x W block][KSUB x (NP x BN rows of X)]
// [the packed 4-bit blocks, for WFMT kWQ4*]. WFMT: the weight format and the MMA's
// operand type (gemm_tc.h).
// PAIR: the CTAs of a cluster of two form one work unit (cta_group::2): CTA rank
// r holds weight rows [128 r, 128 r + 128) of the unit's 256-row tile and
// activation rows [r BN / 2, (r + 1) BN / 2) of its BN, at the same shared-memory
// offsets, and half of the accumulator (its TMEM lanes). The even CTA issues the
// MMAs (M = 256) and commits to both CTAs' barriers; both CTAs' TMA loads count
// on its stage barriers (the 4-bit format: each CTA's converters tell it), and
// both CTAs' epilogues free its accumulator buffers.
template <int NP, int KSUB, int WFMT, bool PAIR>
__global__ void __launch_bounds__(threads_for(WFMT), 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX, KParams kp) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    constexpr bool kQ4 = WFMT == kWQ4AsF16;
    constexpr bool kConv = kQ4;                     // the 4-bit formats have the dequantizing warps
    constexpr int kEpi = epi_warps_for(WFMT);       // epilogue warps 2 .. 2 + kEpi - 1
    const GemmPlan& p = kp.p;
    const int BN = p.BN;
    const int stages = p.stages;
    const int rank = PAIR ? (int)cluster_ctarank() : 0;
    const int unit = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
    const int xrows = PAIR ? BN / 2 : BN;           // activation rows this CTA holds
    const int b_bytes = xrows * BK * 2;             // one K block of one activation part
    const int x_bytes = NP * b_bytes;               // one K block of the activation (hi and lo)
    const int raw_off = KSUB * (kABytes + x_bytes); // packed 4-bit blocks of the stage
    const int stage_bytes = raw_off + (kQ4 ? q4_raw_bytes(KSUB) : 0);
    // bytes the TMA / bulk copies of one stage bring
    const uint32_t tx_bytes = (uint32_t)(KSUB * ((kQ4 ? kQ4BlockBytes : kABytes) + x_bytes));

    // carve: [stages x (W blocks, X blocks)] then barriers
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(base + stages * stage_bytes);
    uint64_t* empty = full + stages;
    uint64_t* acc_full = empty + stages;      // [2]
    uint64_t* acc_empty = acc_full + 2;       // [2]
    uint64_t* conv = acc_empty + 2;           // [stages] the stage's weights are in MMA operand form
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(conv + stages);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);   // set when a wait gives up
    WarpStat* stat_sm = reinterpret_cast<WarpStat*>(tmem_slot + 16);              // [4 warps][BN] (with stats)

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t tmem_cols = p.tmem_cols;

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full[s], 1); mbar_init(&empty[s], 1);
            if (kConv) mbar_init(&conv[s], (PAIR ? 2 : 1) * kConvThreads);
        }
        for (int a = 0; a < 2; ++a) { mbar_init(&acc_full[a], 1); mbar_init(&acc_empty[a], (PAIR ? 2 : 1) * 32 * kEpi); }
        *abort_flag = 0;
        mbar_fence_init();
        if (!kQ4) prefetch_tmap(&tmW);       // packed 4-bit weights come by bulk copy (no weight map)
        prefetch_tmap(&tmX);
    }
    if (warp == 1) {
        if (PAIR) tmem_alloc_pair(tmem_slot, tmem_cols);
        else tmem_alloc(tmem_slot, tmem_cols);
    }
    tc_fence_before();
    __syncthreads();
    if (PAIR) cluster_sync();                        // the peer's barriers exist before any remote arrival
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // PAIR: the even CTA's barriers, as shared::cluster addresses (stage s at + 8 s)
    const uint32_t full0 = PAIR ? mapa_shared(&full[0], 0) : 0u;
    const uint32_t conv0 = PAIR ? mapa_shared(&conv[0], 0) : 0u;
    const uint32_t acc_empty0 = PAIR ? mapa_shared(&acc_empty[0], 0) : 0u;
    // stage loads counted on the even CTA's barrier (not for the 4-bit format, whose
    // converters wait for their own CTA's loads)
    constexpr bool kRemoteFull = PAIR && !kQ4;
    // No pdl_trigger: the consumer is launched as these CTAs exit. CTAs of a
    // consumer launched at the GEMM's start would sit in griddepcontrol.wait
    // for the whole GEMM, and kernels running beside such waiting CTAs were
    // measured to take ~3x longer over their memory phase.

    if (warp == 0) {
        // ---------------------------------------------------------- TMA producer
        if (lane == 0) {
            // one request per stage for the weights, one for the activation
            auto load_w = [&](uint8_t* dst, uint64_t* bar, int kk, int nt) {
                if (kRemoteFull) {
                    const uint32_t fb = full0 + 8u * (uint32_t)(bar - full);
                    if (KSUB == 1) tma_load_2d_pair(dst, &tmW, fb, kk * BK, nt * BM);
                    else tma_load_3d_pair(dst, &tmW, fb, 0, nt * BM, kk * KSUB);
                } else if (kQ4) {
                    // the tile's packed blocks [nt][K block] are contiguous: one bulk copy per stage
                    const uint8_t* src = static_cast<const uint8_t*>(kp.wq4) +
                                         ((int64_t)nt * (p.kb * KSUB) + (int64_t)kk * KSUB) * kQ4BlockBytes;
                    bulk_load(dst + raw_off, src, (uint32_t)(KSUB * kQ4BlockBytes), bar);
                } else if (KSUB == 1) {
                    tma_load_2d(dst, &tmW, bar, kk * BK, nt * BM);
                } else {
                    tma_load_3d(dst, &tmW, bar, 0, nt * BM, kk * KSUB);
                }
            };
            auto load_x = [&](uint8_t* dst, uint64_t* bar, int kk, int mt) {
                const int xr = mt * BN + rank * xrows;         // this CTA's activation rows
                if (kRemoteFull) {
                    const uint32_t fb = full0 + 8u * (uint32_t)(bar - full);
                    if (KSUB == 1) tma_load_2d_pair(dst, &tmX, fb, kk * BK, xr);
                    else tma_load_3d_pair(dst, &tmX, fb, 0, xr, kk * KSUB);
                } else if (NP == 1 && KSUB == 1) tma_load_2d(dst, &tmX, bar, kk * BK, xr);
                else if (NP == 1) tma_load_3d(dst, &tmX, bar, 0, xr, kk * KSUB);
                else if (KSUB == 1) tma_load_3d(dst, &tmX, bar, kk * BK, mt * BN, 0);
                else tma_load_4d(dst, &tmX, bar, 0, mt * BN, 0, kk * KSUB);
            };
            // The weights do not depend on the previous kernel: the first
            // `stages` weight tiles are requested before waiting for it, so
            // the weight stream starts while the producer of X drains.
            auto expect = [&](uint64_t* bar) {
                if (!kRemoteFull) mbar_arrive_expect_tx(bar, tx_bytes);
                else if (rank == 0) mbar_arrive_expect_tx(bar, 2 * tx_bytes);
            };
            // the 128-row weight tile of this CTA in a unit's tile
            auto wtile = [&](int tile) { return PAIR ? (tile / p.n_mt) * 2 + rank : tile / p.n_mt; };
            int n_pre = 0;
            {
                SegIter it(p, unit);
                int tile, k0, k1, slot;
                while (n_pre < stages && it.next(tile, k0, k1, slot)) {
                    const int nt = wtile(tile);
                    for (int kk = k0; kk < k1 && n_pre < stages; ++kk, ++n_pre) {
                        expect(&full[n_pre]);
                        load_w(base + n_pre * stage_bytes, &full[n_pre], kk, nt);
                    }
                }
            }
            pdl_wait();
            SegIter it(p, unit);
            int tile, k0, k1, slot, n = 0;
            bool ok = true;
            while (ok && it.next(tile, k0, k1, slot)) {
                const int nt = wtile(tile), mt = tile % p.n_mt;
                for (int kk = k0; kk < k1; ++kk, ++n) {
                    const int s = n % stages;
                    uint8_t* st = base + s * stage_bytes;
                    if (n >= n_pre) {
                        const uint32_t ph = (uint32_t)(n / stages) & 1u;
                        if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, kp.status)) { ok = false; break; }
                        expect(&full[s]);
                        load_w(st, &full[s], kk, nt);
                    }
                    load_x(st + KSUB * kABytes, &full[s], kk, mt);
                }
            }
            // drain: the loads of the last `stages` slots (every issued slot
            // has its X loads too, since no wait precedes them) complete
            // before teardown, also after an abort (bounded)
            // (the odd CTA of a pair whose loads count on the even CTA's barriers waits
            // for the MMAs that read them instead: the commits reach its own empty barriers)
            const uint64_t deadline = global_timer_ns() + kWaitLimitNs;
            const bool own_full = !kRemoteFull || rank == 0;
            for (int d = 0; d < stages && d < n; ++d) {
                const int m = n - 1 - d;
                uint64_t* bar = own_full ? &full[m % stages] : &empty[m % stages];
                if (!mbar_wait_until(bar, (uint32_t)(m / stages) & 1u, deadline)) {
                    atomicOr(kp.status, DSPARK_DEV_WAIT_TIMEOUT);
                    break;
                }
            }
        } else {
            pdl_wait();
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        pdl_wait();
        if (lane == 0 && (!PAIR || rank == 0)) {
            // hi and lo in one MMA when both fit in N <= 256: the X_lo rows sit right
            // after the X_hi rows in the stage, so [X_hi; X_lo] is one B operand of
            // 2 BN rows and the two products land in adjacent accumulator columns
            const bool fused = NP == 2 && p.acc_cols == 2 * BN;
            constexpr bool kF16 = WFMT == kWF16 || WFMT == kWQ4AsF16;
            constexpr int kM = PAIR ? 2 * BM : BM;         // the pair's MMA spans both CTAs' weight rows
            const uint32_t idesc = kF16 ? idesc_f16(kM, fused ? 2 * BN : BN, 0) : idesc_bf16(kM, fused ? 2 * BN : BN);
            uint64_t* ready = kConv ? conv : full;          // the converters' barrier when they transform W
            SegIter it(p, unit);
            int tile, k0, k1, slot, n = 0, seg = 0;
            bool ok = true;
            while (ok && it.next(tile, k0, k1, slot)) {
                const int acc = seg & 1;
                const uint32_t aph = (uint32_t)(seg >> 1) & 1u;
                if (!mbar_wait(&acc_empty[acc], aph ^ 1u, abort_flag, kp.status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * p.acc_cols);
                for (int kk = k0; kk < k1; ++kk, ++n) {
                    const int s = n % stages;
                    const uint32_t ph = (uint32_t)(n / stages) & 1u;
                    if (!mbar_wait(&ready[s], ph, abort_flag, kp.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t st_addr = smem_u32(base + s * stage_bytes);
#pragma unroll
                    for (int sub = 0; sub < KSUB; ++sub) {
                        const uint64_t adesc = sdesc_k_sw128(st_addr + sub * kABytes);
                        const uint32_t x_addr = st_addr + KSUB * kABytes + sub * x_bytes;
#pragma unroll
                        for (int part = 0; part < (fused ? 1 : NP); ++part) {
                            const uint64_t bdesc = sdesc_k_sw128(x_addr + part * b_bytes);
#pragma unroll
                            for (int j = 0; j < BK / 16; ++j) {
                                const uint32_t accum = (kk > k0 || sub > 0 || part > 0 || j > 0) ? 1u : 0u;
                                if (PAIR) mma_pair(d_tmem, adesc + (uint64_t)(2 * j), bdesc + (uint64_t)(2 * j), idesc, accum);
                                else mma_bf16(d_tmem, adesc + (uint64_t)(2 * j), bdesc + (uint64_t)(2 * j), idesc, accum);
                            }
                        }
                    }
                    // frees the stage (in both CTAs of a pair) once these MMAs have read it
                    if (PAIR) mma_commit_pair(&empty[s], 3);
                    else mma_commit(&empty[s]);
                }
                if (!ok) break;
                // the tile's accumulator is complete (both halves of a pair's)
                if (PAIR) mma_commit_pair(&acc_full[acc], 3);
                else mma_commit(&acc_full[acc]);
                ++seg;
            }
        }
    } else if (kConv && warp >= 2 + kEpi) {
        // ---------------------------------------------------------- weight dequantization (warps 6-9)
        // Thread i owns weight row i of the tile: per K block it turns the packed
        // 4-bit codes into the MMA operand (128 bytes, 128-byte swizzle: 16-byte chunk c
        // of row i at chunk c ^ (i & 7)), then the stage's barrier counts it.
        pdl_wait();
        const int i = threadIdx.x - (64 + 32 * kEpi);
        SegIter it(p, unit);
        int tile, k0, k1, slot, n = 0;
        bool ok = true;
        while (ok && it.next(tile, k0, k1, slot)) {
            for (int kk = k0; kk < k1; ++kk, ++n) {
                const int s = n % stages;
                if (!mbar_wait(&full[s], (uint32_t)(n / stages) & 1u, abort_flag, kp.status)) { ok = false; break; }
                uint8_t* st = base + s * stage_bytes;
#pragma unroll
                for (int sub = 0; sub < KSUB; ++sub) {
                    uint8_t* wrow = st + sub * kABytes + i * 128;
                    {
                        // packed block: words [128 rows][8], scales [128], biases [128] (bf16)
                        const uint8_t* blk = st + raw_off + sub * kQ4BlockBytes;
                        const uint4 w0 = reinterpret_cast<const uint4*>(blk + i * 32)[0];
                        const uint4 w1 = reinterpret_cast<const uint4*>(blk + i * 32)[1];
                        const uint16_t sb = reinterpret_cast<const uint16_t*>(blk + BM * 32)[i];
                        const uint16_t bb = reinterpret_cast<const uint16_t*>(blk + BM * 32 + BM * 2)[i];
                        // bf16 scale and bias as fp16 (exact inside fp16's normal range)
                        const __half hs = __float2half_rn(__uint_as_float((uint32_t)sb << 16));
                        const __half hb = __float2half_rn(__uint_as_float((uint32_t)bb << 16));
                        const uint16_t us = *reinterpret_cast<const uint16_t*>(&hs);
                        const uint16_t ub = *reinterpret_cast<const uint16_t*>(&hb);
                        const uint32_t s2 = (uint32_t)us | ((uint32_t)us << 16);
                        const uint32_t b2 = (uint32_t)ub | ((uint32_t)ub << 16);
                        const uint32_t ws[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            reinterpret_cast<uint4*>(wrow)[c ^ (i & 7)] = q4x8_dequant(ws[c], s2, b2);
                    }
                }
                fence_async_shared();            // the MMA reads these through the async proxy
                if (PAIR) mbar_arrive_cluster(conv0 + 8u * (uint32_t)s);   // the even CTA's MMAs read both halves
                else mbar_arrive(&conv[s]);
            }
        }
    } else {
        // ---------------------------------------------------------- epilogue (warps 2-5)
        // Tile mode: the result goes straight to `out` (with the softcap). Stream-K:
        // each CTA writes its partial of every tile it touches into that tile's slot
        // (slot = CTA - first CTA of the tile); the consumer kernel sums a tile's
        // partials in slot order (PartView), so no CTA waits for another and the
        // GEMM ends as soon as its last MMA has drained.
        pdl_wait();
        const int quad = warp & 3;
        const int n_local = quad * 32 + lane;
        const int grp = (warp - 2) >> 2;                  // column group: chunks grp, grp + kEpi / 4, ...
        const bool with_stats = kp.stats.mx != nullptr && !p.streamk;
        const bool bounds = with_stats && kp.w2norm != nullptr;
        const float Bw1 = bounds ? __uint_as_float(*kp.w1max_bits) : 0.f;
        SegIter it(p, unit);
        int tile, k0, k1, slot, seg = 0;
        while (it.next(tile, k0, k1, slot)) {
            const int acc = seg & 1;
            const uint32_t aph = (uint32_t)(seg >> 1) & 1u;
            const bool got = mbar_wait(&acc_full[acc], aph, abort_flag, kp.status);
            // the group leaves together if any wait gave up
            if (named_barrier_or(1, 32 * kEpi, !got || *abort_flag != 0)) break;
            tc_fence_after();
            // this CTA's 128-row weight tile (a pair's CTA r holds rows 128 r .. of the unit's 256)
            const int nt = PAIR ? (tile / p.n_mt) * 2 + rank : tile / p.n_mt, mt = tile % p.n_mt;
            const int n = nt * BM + n_local;
            const uint32_t tbase = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * p.acc_cols);
            const int64_t store = PAIR ? 2 * (int64_t)tile + rank : tile;     // the partial tiles' 128-row half
            float* part_tile = kp.part + (store * p.P * BN) * BM + n_local;
            const bool split_acc = p.acc_cols == 2 * BN;       // X_hi and X_lo products in separate columns
            // B max |w2| over this warp's 32 entries (the group bound of the tile statistics)
            float bwmax = 0.f;
            if (with_stats && bounds) {
                const float bw = n < p.N ? Bw1 * kp.w2norm[n] : 0.f;
                bwmax = __uint_as_float(warp_max_u32(__float_as_uint(bw)));   // >= 0: bits order as floats
            }
            for (int c0 = 16 * grp; c0 < BN; c0 += 16 * (kEpi / 4)) {
                uint32_t r[16];
                tmem_ld_x16(tbase + (uint32_t)c0, r);
                if (split_acc) {
                    uint32_t r2[16];
                    tmem_ld_x16(tbase + (uint32_t)(BN + c0), r2);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 16; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) + __uint_as_float(r2[j]));
                } else {
                    tmem_ld_wait();
                }
                if (!p.streamk) {
                    float u[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int m = mt * BN + c0 + j;
                        float v = __uint_as_float(r[j]);
                        if (kp.cap > 0.f) v = kp.cap * tanh_fast(v * kp.cap_inv);
                        u[j] = n < p.N ? v : -INFINITY;
                        if (m < p.M && n < p.N) kp.out[(int64_t)m * kp.ldo + n] = v;
                    }
                    if (with_stats) {
                        // the 16 positions (columns) over this warp's 32 entries at once
                        const WarpStat w = warp_logit_stat16(u, n, bwmax, bounds, kp.cap);
                        if ((lane & 1) == 0) stat_sm[quad * BN + c0 + warp_stat16_col(lane)] = w;
                    }
                } else {
                    float* dst = part_tile + ((int64_t)slot * BN + c0) * BM;
#pragma unroll
                    for (int j = 0; j < 16; ++j) dst[(int64_t)j * BM] = __uint_as_float(r[j]);
                }
            }
            tc_fence_before();
            if (PAIR) mbar_arrive_cluster(acc_empty0 + 8u * (uint32_t)acc);   // the even CTA's MMAs reuse it
            else mbar_arrive(&acc_empty[acc]);
            if (with_stats) {
                // the four warps' results of every position of the tile, merged in warp order
                asm volatile("bar.sync 2, %0;" ::"r"(32 * kEpi) : "memory");
                const int tid_e = threadIdx.x - 64;
                for (int c = tid_e; c < BN; c += 32 * kEpi) {
                    const int m = mt * BN + c;
                    if (m < p.M) {
                        const WarpStat q4[4] = {stat_sm[c], stat_sm[BN + c], stat_sm[2 * BN + c], stat_sm[3 * BN + c]};
                        store_tile_stat(kp.stats, nt, m, q4);
                    }
                }
            }
            ++seg;
        }
    }

    tc_fence_before();
    __syncthreads();
    // a pair's CTAs leave together: neither frees shared memory the other's MMAs,
    // loads or arrivals may still reach
    if (PAIR) cluster_sync();
    tc_fence_after();
    if (warp == 1) {
        if (PAIR) tmem_dealloc_pair(tmem_base, tmem_cols);
        else tmem_dealloc(tmem_base, tmem_cols);
    }
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool get_encoder() {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode != nullptr;
}

}  // namespace

// Row-major bf16 [rows, cols] matrix, box of box_rows x 64 columns, 128-byte swizzle.
bool make_tmap(CUtensorMap* tm, const void* ptr, int64_t rows, int64_t cols, int box_rows) {
    if (!get_encoder()) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

namespace {

bool encode(CUtensorMap* tm, int rank, const void* ptr, const cuuint64_t* dims, const cuuint64_t* strides,
            const cuuint32_t* box) {
    if (!get_encoder()) return false;
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return g_encode(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Weights [rows, K]: KSUB = 1 -> 2-D box {64, 128}; KSUB = 2 -> 3-D view
// {64, rows, K / 64} (the third dimension steps 128 bytes along K), box
// {64, 128, 2}: shared layout [K block][row][64].
bool make_wmap(CUtensorMap* tm, const void* W, int64_t rows, int64_t K, int ksub) {
    if (ksub == 1) return make_tmap(tm, W, rows, K, BM);
    const cuuint64_t dims[3] = {(cuuint64_t)BK, (cuuint64_t)rows, (cuuint64_t)(K / BK)};
    const cuuint64_t strides[2] = {(cuuint64_t)K * 2, (cuuint64_t)BK * 2};
    const cuuint32_t box[3] = {(cuuint32_t)BK, (cuuint32_t)BM, (cuuint32_t)ksub};
    return encode(tm, 3, W, dims, strides, box);
}

// Activation [np][M][K] (np = 2: hi then lo, adjacent): shared layout
// [K block][part][row][64] for a box of BN rows.
bool make_xmap(CUtensorMap* tm, const void* X, int64_t M, int64_t K, int BN, int np, int ksub) {
    if (np == 1 && ksub == 1) return make_tmap(tm, X, M, K, BN);
    if (np == 1) {
        const cuuint64_t dims[3] = {(cuuint64_t)BK, (cuuint64_t)M, (cuuint64_t)(K / BK)};
        const cuuint64_t strides[2] = {(cuuint64_t)K * 2, (cuuint64_t)BK * 2};
        const cuuint32_t box[3] = {(cuuint32_t)BK, (cuuint32_t)BN, (cuuint32_t)ksub};
        return encode(tm, 3, X, dims, strides, box);
    }
    if (ksub == 1) {
        const cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)M, 2};
        const cuuint64_t strides[2] = {(cuuint64_t)K * 2, (cuuint64_t)M * K * 2};
        const cuuint32_t box[3] = {(cuuint32_t)BK, (cuuint32_t)BN, 2};
        return encode(tm, 3, X, dims, strides, box);
    }
    const cuuint64_t dims[4] = {(cuuint64_t)BK, (cuuint64_t)M, 2, (cuuint64_t)(K / BK)};
    const cuuint64_t strides[3] = {(cuuint64_t)K * 2, (cuuint64_t)M * K * 2, (cuuint64_t)BK * 2};
    const cuuint32_t box[4] = {(cuuint32_t)BK, (cuuint32_t)BN, 2, (cuuint32_t)ksub};
    return encode(tm, 4, X, dims, strides, box);
}

// Two accumulator buffers of acc_cols columns each.
int tmem_cols_for(int acc_cols) {
    int c = 32;
    while (c < 2 * acc_cols) c <<= 1;
    return c;
}

}  // namespace

int pair_clusters_max(int wfmt, int ksub, size_t smem, int num_sms);

GemmPlan plan_gemm(int num_sms, int M, int N, int K, int np, bool force_tiles, bool stats, int wfmt) {
    GemmPlan p{};
    p.M = M; p.N = N; p.K = K; p.np = np; p.stats = stats ? 1 : 0; p.wfmt = wfmt;
    const bool q4 = wfmt == kWQ4AsF16;
    const int m_pad = (M + 15) / 16 * 16;
    p.BN = m_pad <= 256 ? m_pad : 256;
    p.n_mt = (M + p.BN - 1) / p.BN;
    // CTA pairs (cta_group::2) when the shared-memory traffic of the MMAs bounds the
    // GEMM: one activation part and >= 128 activation rows per tile. Each CTA then
    // stages 128 weight rows and BN / 2 activation rows per K block, for an MMA of
    // 256 x BN: a third less shared-memory traffic per flop than 128 x BN alone.
    // (not for 4-bit weights: their converters' hand-off to the other CTA's MMAs
    // measured slower than one CTA per tile)
    p.pair = (np == 1 && !q4 && p.BN >= 128 && N > BM && num_sms >= 2) ? 1 : 0;
    const int xrows = p.pair ? p.BN / 2 : p.BN;
    p.n_nt = (N + BM * (p.pair ? 2 : 1) - 1) / (BM * (p.pair ? 2 : 1));
    p.tiles = p.n_mt * p.n_nt;
    // as many stages as shared memory holds: the bytes in flight per SM are
    // what sustains the weight stream at HBM latency under load; two K blocks
    // per stage (half the TMA requests) when K allows and >= 3 stages still fit
    auto stage_bytes_for = [&](int ksub) {
        return ksub * (kABytes + np * xrows * BK * 2) + (q4 ? q4_raw_bytes(ksub) : 0);
    };
    const int avail = kSmemLimit - kSmemExtra(kMaxStages) - (stats ? kStatBytes(p.BN) : 0);
    p.ksub = (K % (2 * BK) == 0 && avail / stage_bytes_for(2) >= 3) ? 2 : 1;
    p.kb = K / (BK * p.ksub);
    p.stages = std::max(2, std::min(kMaxStages, avail / stage_bytes_for(p.ksub)));
    // the tensor core takes as long for an MMA of N = 16 as for N = 256: with a
    // bf16 pair activation, hi and lo go through one MMA of N = 2 BN when it fits
    p.acc_cols = (np == 2 && 2 * p.BN <= 256) ? 2 * p.BN : p.BN;
    p.tmem_cols = tmem_cols_for(p.acc_cols);
    // work units: CTAs, or as many CTA pairs as can be resident at once
    int units_max = num_sms;
    if (p.pair) units_max = pair_clusters_max(wfmt, p.ksub, gemm_smem_bytes(p), num_sms);
    // tile mode when whole tiles balance the units to >= 90%, else stream-K
    const int waves = (p.tiles + units_max - 1) / units_max;
    const bool tiles_ok = force_tiles || (p.tiles >= units_max && 10 * p.tiles >= 9 * waves * units_max);
    if (tiles_ok) {
        p.mode = kModeTiles; p.streamk = 0;
        p.units = std::min(p.tiles, units_max);
        p.T = p.tiles * p.kb; p.G = p.units; p.P = 1;
    } else {
        p.mode = kModePartials; p.streamk = 1;
        p.T = p.tiles * p.kb;
        p.G = std::min(p.T, units_max);
        p.units = p.G;
        int P = 1;
        for (int t = 0; t < p.tiles; ++t) P = std::max(P, p.cta_of((t + 1) * p.kb - 1) - p.cta_of(t * p.kb) + 1);
        p.P = P;
    }
    p.grid = p.units * (p.pair ? 2 : 1);
    return p;
}

size_t gemm_partial_elems(const GemmPlan& p) {
    return p.streamk ? (size_t)p.tiles * (p.pair ? 2 : 1) * p.P * p.BN * BM : 0;
}

size_t gemm_smem_bytes(const GemmPlan& p) {
    const bool q4 = p.wfmt == kWQ4AsF16;
    const int xrows = p.pair ? p.BN / 2 : p.BN;
    const int stage_bytes = p.ksub * (kABytes + p.np * xrows * BK * 2) + (q4 ? q4_raw_bytes(p.ksub) : 0);
    return (size_t)p.stages * stage_bytes + kSmemExtra(p.stages) + (p.stats ? kStatBytes(p.BN) : 0);
}

namespace {

template <int NP, int KSUB, bool PAIR>
void* pick_kernel(int wfmt) {
    switch (wfmt) {
        case kWF16: return (void*)gemm_tc_kernel<NP, KSUB, kWF16, PAIR>;
        case kWQ4AsF16: return (void*)gemm_tc_kernel<NP, KSUB, kWQ4AsF16, PAIR>;
        default: return (void*)gemm_tc_kernel<NP, KSUB, kWBf16, PAIR>;
    }
}

void* kernel_for(int np, int ksub, int pair, int wfmt) {
    if (pair) return ksub == 2 ? pick_kernel<1, 2, true>(wfmt) : pick_kernel<1, 1, true>(wfmt);
    return np == 2 ? (ksub == 2 ? pick_kernel<2, 2, false>(wfmt) : pick_kernel<2, 1, false>(wfmt))
                   : (ksub == 2 ? pick_kernel<1, 2, false>(wfmt) : pick_kernel<1, 1, false>(wfmt));
}

// Packs one 128-row tile x one K block per CTA; thread i copies row i.
__global__ void __launch_bounds__(128) q4_pack_kernel(Q4Pieces pcs, int64_t n, int64_t k, uint8_t* __restrict__ dst) {
    pdl_trigger();
    pdl_wait();
    const int64_t t = blockIdx.x;
    const int kb = blockIdx.y, KB = (int)(k / 64), i = threadIdx.x;
    const int64_t row = t * 128 + i;
    uint8_t* blk = dst + ((int64_t)t * KB + kb) * kQ4BlockBytes;
    uint4 w0 = make_uint4(0u, 0u, 0u, 0u), w1 = w0;
    uint16_t sv = 0, bv = 0;
    if (row < n) {
        for (int q = 0; q < pcs.n; ++q) {
            const Q4Piece& pc = pcs.p[q];
            if (row >= pc.row0 && row < pc.row0 + pc.rows) {
                const int64_t r = row - pc.row0;
                const uint4* src = reinterpret_cast<const uint4*>(pc.w + r * (k / 8) + (int64_t)kb * 8);
                w0 = src[0];
                w1 = src[1];
                sv = reinterpret_cast<const uint16_t*>(pc.s)[r * KB + kb];
                bv = reinterpret_cast<const uint16_t*>(pc.b)[r * KB + kb];
                break;
            }
        }
    }
    reinterpret_cast<uint4*>(blk + i * 32)[0] = w0;
    reinterpret_cast<uint4*>(blk + i * 32)[1] = w1;
    reinterpret_cast<uint16_t*>(blk + 128 * 32)[i] = sv;
    reinterpret_cast<uint16_t*>(blk + 128 * 32 + 128 * 2)[i] = bv;
}

}  // namespace

namespace {

// bf16 -> fp16, eight values per thread (n a multiple of 8); flags values outside fp16's range.
__global__ void f16_copy_kernel(const uint4* __restrict__ src, int64_t n8, uint4* __restrict__ dst,
                                int32_t* __restrict__ overflow, int32_t bits) {
    pdl_trigger();
    pdl_wait();
    bool bad = false;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
        const uint4 u = src[i];
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float a = __uint_as_float(w[j] << 16), b = __uint_as_float(w[j] & 0xffff0000u);
            bad |= !(fabsf(a) <= 65504.f) || !(fabsf(b) <= 65504.f);
            const __half2 h = __floats2half2_rn(a, b);
            o[j] = *reinterpret_cast<const uint32_t*>(&h);
        }
        dst[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    if (bad) atomicOr(overflow, bits);
}

}  // namespace

cudaError_t f16_copy(const void* src, int64_t n, void* dst, int32_t* overflow, cudaStream_t s, int32_t bits) {
    if (n % 8 || (reinterpret_cast<uintptr_t>(src) & 15u) || (reinterpret_cast<uintptr_t>(dst) & 15u))
        return cudaErrorInvalidValue;
    const int64_t n8 = n / 8;
    const int blocks = (int)std::min<int64_t>((n8 + 255) / 256, 148 * 8);
    return launch_pdl(f16_copy_kernel, dim3(std::max(blocks, 1)), dim3(256), 0, s, static_cast<const uint4*>(src), n8,
                      static_cast<uint4*>(dst), overflow, bits);
}

cudaError_t q4_pack(const Q4Piece* pieces, int npieces, int64_t n, int64_t k, void* dst, cudaStream_t s) {
    if (npieces < 1 || npieces > kMaxQ4Pieces || k % 64 != 0 || n <= 0) return cudaErrorInvalidValue;
    Q4Pieces pcs{};
    pcs.n = npieces;
    for (int q = 0; q < npieces; ++q) pcs.p[q] = pieces[q];
    const dim3 grid((unsigned)((n + 127) / 128), (unsigned)(k / 64));
    return launch_pdl(q4_pack_kernel, grid, dim3(128), 0, s, pcs, n, k, static_cast<uint8_t*>(dst));
}

// CTA pairs resident at once on this device for the pair kernel of (wfmt, ksub)
// with `smem` bytes of shared memory (clusters of two need two SMs of one GPC, so
// this can be below num_sms / 2); cached per (device, kernel, smem).
int pair_clusters_max(int wfmt, int ksub, size_t smem, int num_sms) {
    static std::mutex mu;
    struct Key { int dev; void* k; size_t smem; int v; };
    static Key cache[32];
    static int n_cache = 0;
    int dev = 0;
    cudaGetDevice(&dev);
    void* kern = kernel_for(1, ksub, 1, wfmt);
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n_cache; ++i)
        if (cache[i].dev == dev && cache[i].k == kern && cache[i].smem == smem) return cache[i].v;
    int v = num_sms / 2;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) == cudaSuccess) {
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3((unsigned)(2 * v));
        cfg.blockDim = dim3((unsigned)threads_for(wfmt));
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2; attr[0].val.clusterDim.y = 1; attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int c = 0;
        if (cudaOccupancyMaxActiveClusters(&c, kern, &cfg) == cudaSuccess && c > 0) v = std::min(v, c);
    }
    cudaGetLastError();                               // a failed query leaves no sticky error
    if (n_cache < 32) cache[n_cache++] = Key{dev, kern, smem, v};
    return std::max(v, 1);
}

cudaError_t launch_gemm_tc(const GemmPlan& p, const void* W, int64_t w_rows, const void* X0, const void* X1,
                           float* out, int64_t ldo, float cap, float* part, int32_t* status, cudaStream_t s,
                           const TileStats* stats, const float* w2norm, const uint32_t* w1max_bits) {
    if (stats && (p.streamk || !p.stats)) return cudaErrorInvalidValue;
    if (p.streamk && !part) return cudaErrorInvalidValue;
    const bool q4 = p.wfmt == kWQ4AsF16;
    if (q4 && p.np != 1) return cudaErrorInvalidValue;
    // the bf16 pair must be one [2][M][K] block (lo right after hi)
    if (p.np == 2 && static_cast<const char*>(X1) != static_cast<const char*>(X0) + (size_t)p.M * p.K * 2)
        return cudaErrorInvalidValue;
    if (q4 && (reinterpret_cast<uintptr_t>(W) & 15u)) return cudaErrorInvalidValue;
    CUtensorMap tw, tx;
    memset(&tw, 0, sizeof(tw));
    // packed 4-bit weights come by bulk copy: the weight map is unused
    if (!q4 && !make_wmap(&tw, W, w_rows, p.K, p.ksub)) return cudaErrorInvalidValue;
    if (p.pair && (p.np != 1 || p.BN % 16)) return cudaErrorInvalidValue;
    if (!make_xmap(&tx, X0, p.M, p.K, p.pair ? p.BN / 2 : p.BN, p.np, p.ksub)) return cudaErrorInvalidValue;
    KParams kp{};
    kp.p = p; kp.out = out; kp.ldo = ldo; kp.cap = cap; kp.cap_inv = cap > 0.f ? 1.f / cap : 0.f;
    kp.status = status; kp.part = part;
    kp.wq4 = q4 ? W : nullptr;
    if (stats) { kp.stats = *stats; kp.w2norm = w2norm; kp.w1max_bits = w1max_bits; }
    const size_t smem = gemm_smem_bytes(p);
    void* kern = kernel_for(p.np, p.ksub, p.pair, p.wfmt);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (p.pair)
        return launch_pdl_cluster(reinterpret_cast<void (*)(CUtensorMap, CUtensorMap, KParams)>(kern), dim3(p.grid),
                                  dim3(threads_for(p.wfmt)), 2, smem, s, tw, tx, kp);
    return launch_pdl(reinterpret_cast<void (*)(CUtensorMap, CUtensorMap, KParams)>(kern), dim3(p.grid),
                      dim3(threads_for(p.wfmt)), smem, s, tw, tx, kp);
}

}  // namespace tc
}  // namespace dspark
