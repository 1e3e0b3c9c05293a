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
// Roles (192 threads): warp 0 issues TMA loads, warp 1 owns TMEM and issues
// MMAs, warps 2-5 drain accumulators (TMEM lane quadrant = warp % 4).
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

#include <algorithm>
#include <mutex>
#include <string>

#include "internal.h"
#include "common.cuh"
#include "gemm_tc.h"
#include "tmap.h"
#include "tc_ptx.cuh"

namespace dspark {
namespace tc {
namespace {

constexpr int BM = 128;            // weight rows per tile (MMA M)
constexpr int BK = 64;             // K elements per K block: one 128-byte swizzle row
constexpr int kThreads = 192;
constexpr int kABytes = BM * BK * 2;   // one K block of weights (16 KB)
constexpr int kMaxStages = 12;
constexpr int kSmemLimit = 227 * 1024;   // dynamic shared memory a CTA may opt into
// alignment slack + full/empty barriers per stage + 4 accumulator barriers,
// the TMEM slot and the abort flag (plus one spare word)
constexpr int kSmemExtra(int stages) { return 1024 + 16 * stages + 32 + 16 + 64; }

struct KParams {
    GemmPlan p;
    float* out;        // result rows out[m * ldo + n]
    int64_t ldo;
    float cap;         // softcap of the result (0 = none)
    float* part;       // stream-K partial tiles [tile][P][BN][128]
    int32_t* status;
};

// Iterates the (tile, k-range) segments of one CTA, identically in every role.
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
        t += p.grid;
        return true;
    }
};

// KSUB K blocks per stage; stage layout [KSUB x W block][KSUB x (NP x BN rows of X)].
template <int NP, int KSUB>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX, KParams kp) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const GemmPlan& p = kp.p;
    const int BN = p.BN;
    const int stages = p.stages;
    const int b_bytes = BN * BK * 2;                // one K block of one activation part
    const int x_bytes = NP * b_bytes;               // one K block of the activation (hi and lo)
    const int stage_bytes = KSUB * (kABytes + x_bytes);

    // carve: [stages x (W blocks, X blocks)] then barriers
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(base + stages * stage_bytes);
    uint64_t* empty = full + stages;
    uint64_t* acc_full = empty + stages;      // [2]
    uint64_t* acc_empty = acc_full + 2;       // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);   // set when a wait gives up

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t tmem_cols = p.tmem_cols;

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        for (int a = 0; a < 2; ++a) { mbar_init(&acc_full[a], 1); mbar_init(&acc_empty[a], 128); }
        *abort_flag = 0;
        mbar_fence_init();
        prefetch_tmap(&tmW); prefetch_tmap(&tmX);
    }
    if (warp == 1) tmem_alloc(tmem_slot, tmem_cols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // No pdl_trigger: the consumer is launched as these CTAs exit. CTAs of a
    // consumer launched at the GEMM's start would sit in griddepcontrol.wait
    // for the whole GEMM, and kernels running beside such waiting CTAs were
    // measured to take ~3x longer over their memory phase.

    if (warp == 0) {
        // ---------------------------------------------------------- TMA producer
        if (lane == 0) {
            // one request per stage for the weights, one for the activation
            auto load_w = [&](uint8_t* dst, uint64_t* bar, int kk, int nt) {
                if (KSUB == 1) tma_load_2d(dst, &tmW, bar, kk * BK, nt * BM);
                else tma_load_3d(dst, &tmW, bar, 0, nt * BM, kk * KSUB);
            };
            auto load_x = [&](uint8_t* dst, uint64_t* bar, int kk, int mt) {
                if (NP == 1 && KSUB == 1) tma_load_2d(dst, &tmX, bar, kk * BK, mt * BN);
                else if (NP == 1) tma_load_3d(dst, &tmX, bar, 0, mt * BN, kk * KSUB);
                else if (KSUB == 1) tma_load_3d(dst, &tmX, bar, kk * BK, mt * BN, 0);
                else tma_load_4d(dst, &tmX, bar, 0, mt * BN, 0, kk * KSUB);
            };
            // The weights do not depend on the previous kernel: the first
            // `stages` weight tiles are requested before waiting for it, so
            // the weight stream starts while the producer of X drains.
            int n_pre = 0;
            {
                SegIter it(p, blockIdx.x);
                int tile, k0, k1, slot;
                while (n_pre < stages && it.next(tile, k0, k1, slot)) {
                    const int nt = tile / p.n_mt;
                    for (int kk = k0; kk < k1 && n_pre < stages; ++kk, ++n_pre) {
                        mbar_arrive_expect_tx(&full[n_pre], stage_bytes);
                        load_w(base + n_pre * stage_bytes, &full[n_pre], kk, nt);
                    }
                }
            }
            pdl_wait();
            SegIter it(p, blockIdx.x);
            int tile, k0, k1, slot, n = 0;
            bool ok = true;
            while (ok && it.next(tile, k0, k1, slot)) {
                const int nt = tile / p.n_mt, mt = tile % p.n_mt;
                for (int kk = k0; kk < k1; ++kk, ++n) {
                    const int s = n % stages;
                    uint8_t* st = base + s * stage_bytes;
                    if (n >= n_pre) {
                        const uint32_t ph = (uint32_t)(n / stages) & 1u;
                        if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, kp.status)) { ok = false; break; }
                        mbar_arrive_expect_tx(&full[s], stage_bytes);
                        load_w(st, &full[s], kk, nt);
                    }
                    load_x(st + KSUB * kABytes, &full[s], kk, mt);
                }
            }
            // drain: the loads of the last `stages` slots (every issued slot
            // has its X loads too, since no wait precedes them) complete
            // before teardown, also after an abort (bounded)
            const uint64_t deadline = global_timer_ns() + kWaitLimitNs;
            for (int d = 0; d < stages && d < n; ++d) {
                const int m = n - 1 - d;
                if (!mbar_wait_until(&full[m % stages], (uint32_t)(m / stages) & 1u, deadline)) {
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
        if (lane == 0) {
            // hi and lo in one MMA when both fit in N <= 256: the X_lo rows sit right
            // after the X_hi rows in the stage, so [X_hi; X_lo] is one B operand of
            // 2 BN rows and the two products land in adjacent accumulator columns
            const bool fused = NP == 2 && p.acc_cols == 2 * BN;
            const uint32_t idesc = idesc_bf16(BM, fused ? 2 * BN : BN);
            SegIter it(p, blockIdx.x);
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
                    if (!mbar_wait(&full[s], ph, abort_flag, kp.status)) { ok = false; break; }
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
                                mma_bf16(d_tmem, adesc + (uint64_t)(2 * j), bdesc + (uint64_t)(2 * j), idesc, accum);
                            }
                        }
                    }
                    mma_commit(&empty[s]);          // frees the stage once these MMAs have read it
                }
                if (!ok) break;
                mma_commit(&acc_full[acc]);         // the tile's accumulator is complete
                ++seg;
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
        SegIter it(p, blockIdx.x);
        int tile, k0, k1, slot, seg = 0;
        while (it.next(tile, k0, k1, slot)) {
            const int acc = seg & 1;
            const uint32_t aph = (uint32_t)(seg >> 1) & 1u;
            mbar_wait(&acc_full[acc], aph, abort_flag, kp.status);
            asm volatile("bar.sync 1, 128;" ::: "memory");   // the group leaves together if any wait gave up
            if (*abort_flag) break;
            tc_fence_after();
            const int nt = tile / p.n_mt, mt = tile % p.n_mt;
            const int n = nt * BM + n_local;
            const uint32_t tbase = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * p.acc_cols);
            float* part_tile = kp.part + ((int64_t)tile * p.P * BN) * BM + n_local;
            const bool split_acc = p.acc_cols == 2 * BN;       // X_hi and X_lo products in separate columns
            for (int c0 = 0; c0 < BN; c0 += 16) {
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
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int m = mt * BN + c0 + j;
                        if (m < p.M && n < p.N) {
                            float v = __uint_as_float(r[j]);
                            if (kp.cap > 0.f) v = kp.cap * tanhf(v / kp.cap);
                            kp.out[(int64_t)m * kp.ldo + n] = v;
                        }
                    }
                } else {
                    float* dst = part_tile + ((int64_t)slot * BN + c0) * BM;
#pragma unroll
                    for (int j = 0; j < 16; ++j) dst[(int64_t)j * BM] = __uint_as_float(r[j]);
                }
            }
            tc_fence_before();
            mbar_arrive(&acc_empty[acc]);
            ++seg;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, tmem_cols);
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

GemmPlan plan_gemm(int num_sms, int M, int N, int K, int np, bool force_tiles) {
    GemmPlan p{};
    p.M = M; p.N = N; p.K = K; p.np = np;
    const int m_pad = (M + 15) / 16 * 16;
    p.BN = m_pad <= 256 ? m_pad : 256;
    p.n_mt = (M + p.BN - 1) / p.BN;
    p.n_nt = (N + BM - 1) / BM;
    p.tiles = p.n_mt * p.n_nt;
    // as many stages as shared memory holds: the bytes in flight per SM are
    // what sustains the weight stream at HBM latency under load; two K blocks
    // per stage (half the TMA requests) when K allows and >= 3 stages still fit
    auto stage_bytes_for = [&](int ksub) { return ksub * (kABytes + np * p.BN * BK * 2); };
    const int avail = kSmemLimit - kSmemExtra(kMaxStages);
    p.ksub = (K % (2 * BK) == 0 && avail / stage_bytes_for(2) >= 3) ? 2 : 1;
    p.kb = K / (BK * p.ksub);
    p.stages = std::max(2, std::min(kMaxStages, avail / stage_bytes_for(p.ksub)));
    // the tensor core takes as long for an MMA of N = 16 as for N = 256: with a
    // bf16 pair activation, hi and lo go through one MMA of N = 2 BN when it fits
    p.acc_cols = (np == 2 && 2 * p.BN <= 256) ? 2 * p.BN : p.BN;
    p.tmem_cols = tmem_cols_for(p.acc_cols);
    // tile mode when whole tiles balance the SMs to >= 90%, else stream-K
    const int waves = (p.tiles + num_sms - 1) / num_sms;
    const bool tiles_ok = force_tiles || (p.tiles >= num_sms && 10 * p.tiles >= 9 * waves * num_sms);
    if (tiles_ok) {
        p.mode = kModeTiles; p.streamk = 0;
        p.grid = std::min(p.tiles, num_sms);
        p.T = p.tiles * p.kb; p.G = p.grid; p.P = 1;
    } else {
        p.mode = kModePartials; p.streamk = 1;
        p.T = p.tiles * p.kb;
        p.G = std::min(p.T, num_sms);
        p.grid = p.G;
        int P = 1;
        for (int t = 0; t < p.tiles; ++t) P = std::max(P, p.cta_of((t + 1) * p.kb - 1) - p.cta_of(t * p.kb) + 1);
        p.P = P;
    }
    return p;
}

size_t gemm_partial_elems(const GemmPlan& p) {
    return p.streamk ? (size_t)p.tiles * p.P * p.BN * BM : 0;
}

size_t gemm_smem_bytes(const GemmPlan& p) {
    const int stage_bytes = p.ksub * (kABytes + p.np * p.BN * BK * 2);
    return (size_t)p.stages * stage_bytes + kSmemExtra(p.stages);
}

cudaError_t launch_gemm_tc(const GemmPlan& p, const void* W, int64_t w_rows, const void* X0, const void* X1,
                           float* out, int64_t ldo, float cap, float* part, int32_t* status, cudaStream_t s) {
    if (p.streamk && !part) return cudaErrorInvalidValue;
    // the bf16 pair must be one [2][M][K] block (lo right after hi)
    if (p.np == 2 && static_cast<const char*>(X1) != static_cast<const char*>(X0) + (size_t)p.M * p.K * 2)
        return cudaErrorInvalidValue;
    CUtensorMap tw, tx;
    if (!make_wmap(&tw, W, w_rows, p.K, p.ksub)) return cudaErrorInvalidValue;
    if (!make_xmap(&tx, X0, p.M, p.K, p.BN, p.np, p.ksub)) return cudaErrorInvalidValue;
    KParams kp{};
    kp.p = p; kp.out = out; kp.ldo = ldo; kp.cap = cap; kp.status = status; kp.part = part;
    const size_t smem = gemm_smem_bytes(p);
    void (*kern)(CUtensorMap, CUtensorMap, KParams) =
        p.np == 2 ? (p.ksub == 2 ? gemm_tc_kernel<2, 2> : gemm_tc_kernel<2, 1>)
                  : (p.ksub == 2 ? gemm_tc_kernel<1, 2> : gemm_tc_kernel<1, 1>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3(p.grid), dim3(kThreads), smem, s, tw, tx, kp);
}

}  // namespace tc
}  // namespace dspark
