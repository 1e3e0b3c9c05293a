// The temperature-0 VanillaMarkov walk with the rank-r bias on tensor cores
// (deepspec.ts #markovStepBias / #selectStep and the sequential loop of
// draftRows): for k = 0 .. gamma-1,
//   bias_b[v] = markov_w2[v] . markov_w1[prev_b];  tok_{b,k} = argmax_v(U[b,k,v] + bias_b[v]);  prev_b = tok_{b,k}
// (fp32 sum, lowest index on ties).
//
// Per step the bias over the whole vocabulary is a [V x r] by [r x A] product:
// each CTA (one per SM, cooperative launch) owns a slice of 128-row vocabulary
// tiles and computes them as tcgen05 MMAs, M = 128 vocabulary rows of
// markov_w2 (bf16, K-major, r = 64 = one 128-byte swizzle row), N = 16 columns
// holding markov_w1[prev_b] for the batch rows b < A (zeros beyond), fp32
// accumulators in TMEM (one 16-column group per tile). bf16 times bf16
// products are exact in fp32, so the bias differs from a CUDA-core sum only
// in the order of its fp32 additions. Then one thread per (tile row, b)
// adds U[b, k, v] and keeps a running argmax; warp and CTA reductions give
// one candidate per row b, folded into one 64-bit key per (step, row) with an
// atomic maximum (the value's bits made order-preserving, then the
// complemented index: the largest value, lowest index on ties), and after a
// grid barrier (bounded wait) every CTA reads the step's token from it.
//
// markov_w2 does not change during the walk: most of the CTA's tiles are
// TMA-loaded once and stay in shared memory; the rest (at most 2 * kSlots)
// cycle through kSlots slots, reloaded as soon as their MMAs have read them.
#include <math.h>

#include <algorithm>

#include "internal.h"
#include "common.cuh"
#include "tc_ptx.cuh"
#include "tmap.h"

namespace dspark {
namespace tc {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kRows = 8;             // batch rows (candidate registers per thread)
constexpr int kN = 16;               // MMA N: batch rows padded
constexpr int kTileBytes = 128 * 128;  // 128 vocabulary rows x 64 bf16
constexpr int kSlots = 2;
constexpr int kDynLimit = 225 * 1024;  // dynamic shared memory (227 KB less the static arrays)
constexpr int kTmemCols = 256;

struct WtcArgs {
    const float* U;            // [A, G, V] fp32
    const int32_t* anchors;    // [A]
    const bf16* w1;            // markov_w1 [V, 64]
    int32_t* tokens;           // [A, G]
    uint32_t* arrivals;        // grid-barrier counter, zero at entry
    unsigned long long* keys;  // [G][A] packed (value, index) maxima of each step, zero at entry
    int A, G, V;
    int tiles_total;           // ceil(V / 128)
    int res_max;               // resident tiles a CTA may hold
    int32_t* status;
    const int* skip;           // non-NULL: return at once when *skip == 0 (tokens already written)
};

__device__ __forceinline__ void red_release_add(uint32_t* p, uint32_t v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// (value, index) as one 64-bit key whose unsigned maximum is the largest
// value with the lowest index: the value's bits made order-preserving, then
// the complemented index. NaN maps to 0 and never wins.
__device__ __forceinline__ unsigned long long pack_key(float v, int idx) {
    const uint32_t u = __float_as_uint(v);
    uint32_t ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    if (v != v) ord = 0u;
    return ((unsigned long long)ord << 32) | (unsigned long long)(~(uint32_t)idx);
}

__global__ void __launch_bounds__(kThreads, 1)
walk_tc_kernel(const __grid_constant__ CUtensorMap tmW2, WtcArgs a) {
    extern __shared__ __align__(1024) uint8_t dyn[];
    __shared__ int prev[kRows];
    __shared__ float rv[kWarps][kRows];
    __shared__ int ri[kWarps][kRows];
    __shared__ uint64_t bars[2 + 2 * kSlots];         // res, mma, full[kSlots], freed[kSlots]
    __shared__ uint32_t tmem_slot;
    __shared__ int s_fail;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // the pruned walk has written this round's tokens: every CTA reads the same
    // word (its writer completed before this stream-ordered launch) and leaves
    // before touching TMEM, barriers or memory
    if (a.skip && *a.skip == 0) return;
    const int A = a.A, G = a.G, V = a.V;
    const int nblk = gridDim.x;
    // this CTA's tiles [t0, t1) of the vocabulary
    const int t0 = (int)(((int64_t)blockIdx.x * a.tiles_total) / nblk);
    const int t1 = (int)(((int64_t)(blockIdx.x + 1) * a.tiles_total) / nblk);
    const int nt = t1 - t0;
    const int nres = min(nt, a.res_max);
    const int ns = nt - nres;                          // streamed tiles, <= 2 * kSlots
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn) + 1023) & ~uintptr_t(1023));
    uint8_t* sE = base;                                // [16 rows x 128 B]: markov_w1[prev_b] (K-major, swizzled)
    uint8_t* sSlot = base + 2048;                      // kSlots x tile (1 KB aligned: 2048 + k * 16 KB)
    uint8_t* sRes = sSlot + kSlots * kTileBytes;       // nres x tile
    uint64_t* bar_res = &bars[0];
    uint64_t* bar_mma = &bars[1];
    uint64_t* full = &bars[2];
    uint64_t* freed = &bars[2 + kSlots];
    volatile int* abort_flag = &s_fail;

    if (tid == 0) {
        s_fail = 0;
        for (int i = 0; i < 2 + 2 * kSlots; ++i) mbar_init(&bars[i], i == 1 ? 2 : 1);   // bar_mma: two issuers
        mbar_fence_init();
        prefetch_tmap(&tmW2);
        // markov_w2 is a weight: requested before waiting on the previous kernel
        mbar_arrive_expect_tx(bar_res, (uint32_t)(nres * kTileBytes));
        for (int t = 0; t < nres; ++t) tma_load_2d(sRes + t * kTileBytes, &tmW2, bar_res, 0, (t0 + t) * 128);
    }
    if (warp == 0) tmem_alloc(&tmem_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    // no pdl_trigger: the confidence kernel launches as the walk exits
    pdl_wait();

    // streamed tiles: load q (counted over all steps) goes to slot q % kSlots
    int q_load = 0;                                    // thread 0: loads issued
    auto load_q = [&](int q) {
        const int s = q % kSlots;
        mbar_arrive_expect_tx(&full[s], (uint32_t)kTileBytes);
        tma_load_2d(sSlot + s * kTileBytes, &tmW2, &full[s], 0, (t0 + nres + q % ns) * 128);
    };
    if (tid == 0)
        for (; q_load < kSlots && q_load < G * ns; ++q_load) load_q(q_load);
    for (int b = tid; b < A; b += kThreads) {
        int t = a.anchors[b];
        if (t < 0 || t >= V) {
            if (blockIdx.x == 0) atomicOr(a.status, DSPARK_DEV_BAD_TOKEN);
            t = min(max(t, 0), V - 1);
        }
        prev[b] = t;
    }
    __syncthreads();

    const uint32_t idesc = idesc_bf16(128, kN);
    const int group = warp >> 2;                       // tiles group, group + 4, ...
    const int quad = warp & 3;                         // TMEM lanes 32 quad .. 32 quad + 31
    const int row = quad * 32 + lane;                  // vocabulary row within a tile
    bool ok = true;
    for (int step = 0; step < G && ok; ++step) {
        // ---- the N operand: markov_w1[prev_b] as bf16 rows, 128-byte swizzle
        if (tid < kN * 8) {
            const int b = tid >> 3, c = tid & 7;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (b < A) v = *reinterpret_cast<const uint4*>(a.w1 + (int64_t)prev[b] * 64 + c * 8);
            *reinterpret_cast<uint4*>(sE + b * 128 + ((c ^ (b & 7)) * 16)) = v;
        }
        fence_async_shared();
        tc_fence_before();
        __syncthreads();
        // ---- U of this step for this thread's rows, in flight during the MMAs
        float uval[4][kRows];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int t = group + 4 * i;
            const int v = (t0 + t) * 128 + row;
#pragma unroll
            for (int b = 0; b < kRows; ++b)
                uval[i][b] = (t < nt && b < A && v < V) ? __ldcs(a.U + ((int64_t)b * G + step) * V + v) : 0.f;
        }
        // ---- bias tiles on the tensor cores: two issuing threads. Thread 32 runs every
        // resident tile while thread 0 runs the streamed ones, whose mid-step reload
        // latency then hides behind thread 32's MMAs.
        auto mma_tile = [&](const uint8_t* src, int t) {
            const uint64_t adesc = sdesc_k_sw128(smem_u32(src));
            const uint64_t bdesc = sdesc_k_sw128(smem_u32(sE));
            const uint32_t d = tmem + (uint32_t)(t * kN);
#pragma unroll
            for (int j = 0; j < 4; ++j) mma_bf16(d, adesc + (uint64_t)(2 * j), bdesc + (uint64_t)(2 * j), idesc, j > 0 ? 1u : 0u);
        };
        if (tid == 32) {
            tc_fence_after();
            if (step == 0 && !mbar_wait(bar_res, 0u, abort_flag, a.status)) ok = false;
            if (ok) {
                tc_fence_after();
                for (int t = 0; t < nres; ++t) mma_tile(sRes + t * kTileBytes, t);
                mma_commit(bar_mma);
            }
        }
        if (tid == 0) {
            tc_fence_after();
            const int q0 = step * ns, q1 = q0 + ns;
            const int q_pre = min(q_load, q1);         // streamed tiles already requested
            for (int q = q0; q < q_pre && ok; ++q) {
                if (!mbar_wait(&full[q % kSlots], (uint32_t)(q / kSlots) & 1u, abort_flag, a.status)) { ok = false; break; }
                tc_fence_after();
                mma_tile(sSlot + (q % kSlots) * kTileBytes, nres + q % ns);
                mma_commit(&freed[q % kSlots]);
            }
            // this step's other streamed tiles: their slots free up as the MMAs above finish
            for (; ok && q_load < q1; ++q_load) {
                const int qp = q_load - kSlots;        // the previous use of the slot
                if (!mbar_wait(&freed[qp % kSlots], (uint32_t)(qp / kSlots) & 1u, abort_flag, a.status)) { ok = false; break; }
                load_q(q_load);
            }
            for (int q = q_pre; ok && q < q1; ++q) {
                if (!mbar_wait(&full[q % kSlots], (uint32_t)(q / kSlots) & 1u, abort_flag, a.status)) { ok = false; break; }
                tc_fence_after();
                mma_tile(sSlot + (q % kSlots) * kTileBytes, nres + q % ns);
                mma_commit(&freed[q % kSlots]);
            }
            if (ok) mma_commit(bar_mma);
            // the next step's first streamed tiles
            for (; ok && q_load < min(q1 + kSlots, G * ns); ++q_load) {
                const int qp = q_load - kSlots;
                if (!mbar_wait(&freed[qp % kSlots], (uint32_t)(qp / kSlots) & 1u, abort_flag, a.status)) { ok = false; break; }
                load_q(q_load);
            }
        }
        if (!mbar_wait(bar_mma, (uint32_t)step & 1u, abort_flag, a.status)) { ok = false; break; }
        tc_fence_after();
        // ---- U + bias, running argmax per batch row
        float best[kRows];
        int bidx[kRows];
#pragma unroll
        for (int b = 0; b < kRows; ++b) { best[b] = -INFINITY; bidx[b] = 0x7fffffff; }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int t = group + 4 * i;
            if (t >= nt) break;                        // warp-uniform
            uint32_t r[16];
            tmem_ld_x16(tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(t * kN), r);
            tmem_ld_wait();
            const int v = (t0 + t) * 128 + row;
#pragma unroll
            for (int b = 0; b < kRows; ++b)
                if (b < A && v < V) argmax_merge(best[b], bidx[b], uval[i][b] + __uint_as_float(r[b]), v);
        }
        tc_fence_before();
        // the next step's U rows of this thread into L2 while the step's reduction runs
        if (step + 1 < G) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = group + 4 * i;
                const int v = (t0 + t) * 128 + row;
                if (t < nt && v < V)
                    for (int b = 0; b < A; ++b)
                        asm volatile("prefetch.global.L2 [%0];" ::"l"(a.U + ((int64_t)b * G + step + 1) * V + v));
            }
        }
        // ---- candidates of this CTA
#pragma unroll
        for (int b = 0; b < kRows; ++b) {
            if (b >= A) break;
            float bv = best[b];
            int bi = bidx[b];
            warp_argmax(bv, bi);
            if (lane == 0) { rv[warp][b] = bv; ri[warp][b] = bi; }
        }
        __syncthreads();
        if (tid < A) {
            float bv = -INFINITY;
            int bi = 0x7fffffff;
            for (int w = 0; w < kWarps; ++w) argmax_merge(bv, bi, rv[w][tid], ri[w][tid]);
            if (bi != 0x7fffffff) {
                atomicMax(&a.keys[(size_t)step * A + tid], pack_key(bv, bi));
                // the winner's markov_w1 row is the next step's operand: have it in L2
                asm volatile("prefetch.global.L2 [%0];" ::"l"(a.w1 + (int64_t)bi * 64));
            }
        }
        __syncthreads();
        // ---- grid barrier (bounded), then every CTA reduces all candidates in CTA order
        if (tid == 0) {
            red_release_add(a.arrivals, 1u);
            const uint32_t target = (uint32_t)(step + 1) * (uint32_t)nblk;
            const uint64_t tw = global_timer_ns();
            while (ld_acquire(a.arrivals) < target) {
                if (global_timer_ns() - tw > kWaitLimitNs) {
                    atomicOr(a.status, DSPARK_DEV_WAIT_TIMEOUT);
                    s_fail = 1;
                    break;
                }
            }
        }
        __syncthreads();
        if (s_fail) { ok = false; break; }
        // the step's maximum over all CTAs is one 64-bit word per row
        if (tid < A) {
            const unsigned long long key = __ldcg(&a.keys[(size_t)step * A + tid]);
            int bi = (int)~(uint32_t)(key & 0xffffffffull);
            if ((key >> 32) == 0ull || bi < 0 || bi >= V) {   // only if a row was all NaN
                if (blockIdx.x == 0) atomicOr(a.status, DSPARK_DEV_BAD_TOKEN);
                bi = 0;
            }
            prev[tid] = bi;
            if (blockIdx.x == 0) a.tokens[tid * G + step] = bi;
        }
        __syncthreads();
    }

    // copies and MMAs still in flight finish before teardown (bounded)
    if (tid == 0) {
        const uint64_t deadline = global_timer_ns() + kWaitLimitNs;
        bool drained = mbar_wait_until(bar_res, 0u, deadline);
        for (int q = max(0, q_load - kSlots); q < q_load && drained; ++q)
            drained = mbar_wait_until(&full[q % kSlots], (uint32_t)(q / kSlots) & 1u, deadline);
        if (!drained) atomicOr(a.status, DSPARK_DEV_WAIT_TIMEOUT);
        if (!ok && drained) {
            // MMAs issued in a step that did not finish complete before TMEM is released
            mma_commit(bar_res);
            if (!mbar_wait_until(bar_res, 1u, deadline)) atomicOr(a.status, DSPARK_DEV_WAIT_TIMEOUT);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

int resident_tiles() {
    // dynamic: 1 KB alignment slack + the N operand (2 KB) + kSlots slots + resident tiles
    return (kDynLimit - 1024 - 2048 - kSlots * kTileBytes) / kTileBytes;
}

}  // namespace

// Tensor-core walk: bf16 dense markov_w2 with rank 64, at most kRows batch
// rows, and every CTA's tiles within the resident tiles plus 2 * kSlots.
bool walk_tc_supported(const dspark_model* m, int A) {
    const Dims& d = m->d;
    if (d.dtype != DSPARK_DTYPE_BF16 || d.quant || d.r != 64 || A < 1 || A > kRows) return false;
    if (reinterpret_cast<uintptr_t>(m->w2.w) % 16 != 0 || reinterpret_cast<uintptr_t>(m->w1) % 16 != 0) return false;
    const int tiles = (d.V + 127) / 128;
    const int per = (tiles + m->num_sms - 1) / m->num_sms;
    return per <= resident_tiles() + 2 * kSlots;
}

cudaError_t launch_walk_tc(const dspark_model* m, const float* U, const int32_t* anchors, int32_t* tokens,
                           unsigned long long* keys, uint32_t* arrivals, const int* skip, int A, cudaStream_t s) {
    const Dims& d = m->d;
    CUtensorMap tw;
    if (!make_tmap(&tw, m->w2.w, d.V, 64, 128)) return cudaErrorInvalidValue;
    WtcArgs wa{};
    wa.U = U; wa.anchors = anchors; wa.w1 = static_cast<const bf16*>(m->w1); wa.tokens = tokens;
    wa.keys = keys; wa.arrivals = arrivals;
    wa.A = A; wa.G = d.gamma; wa.V = d.V;
    wa.tiles_total = (d.V + 127) / 128;
    wa.res_max = resident_tiles();
    wa.status = m->ws.status;
    wa.skip = skip;
    const int nblk = m->num_sms;
    const int per = (wa.tiles_total + nblk - 1) / nblk;
    const int nres = std::min(per, wa.res_max);
    const size_t smem = 1024 + 2048 + (size_t)kSlots * kTileBytes + (size_t)nres * kTileBytes;
    cudaError_t e = cudaFuncSetAttribute((const void*)walk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    void* args[] = {&tw, &wa};
    // cooperative: all CTAs co-resident, which the grid barrier needs
    e = cudaLaunchCooperativeKernel((const void*)walk_tc_kernel, dim3(nblk), dim3(kThreads), args, smem, s);
    count_launches(1);
    return e;
}

}  // namespace tc
}  // namespace dspark
