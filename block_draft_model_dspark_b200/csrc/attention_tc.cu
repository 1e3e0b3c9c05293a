// KV-injection attention on tcgen05 tensor cores: the
// DeepspecContextAttention.attend seam ("mlx-bun 0.2.0 -> 0.4.0" page 75,
// plainDeepspecContext): the block queries of one row attend, non-causally
// and at scale 1.0, over the row's cached context keys followed by the
// block's own keys; GQA maps query head h to kv head h / (nH / nKv).
//
// One CTA = (row b, kv head g, key split). Its query tile is the 128-row MMA
// side: the grp * gamma queries of the heads that share kv head g (row r =
// query i * grp + head-in-group). Key tiles of 64 rows are TMA-loaded from the
// bf16 cache as they are stored (3-D maps pick kv head g out of
// [rows, nKv, hd]) and used directly as bf16 MMA operands. The fp32 side of
// each product enters as a bf16 pair (hi, lo = x - hi) and takes two MMAs
// into the same fp32 accumulator, so q and the probabilities P keep ~16
// significant bits while K and V are read exactly once:
//   S  = Qhi K^T + Qlo K^T        -> TMEM (64 columns), fp32
//   softmax                       -> one thread per query row (TMEM lane =
//                                    row); the running max is raised only when
//                                    a tile's max exceeds it by more than
//                                    kRescale, so O is rarely rescaled in TMEM
//   O += Phi V + Plo V            -> TMEM (hd columns); P from shared memory
//                                    (K-major, 128-byte swizzle), V as an
//                                    MN-major operand
// K and V have one buffer each and are reloaded as soon as their MMAs have
// read them: the next K tile streams in during the softmax and the P V
// product, the next V tile during the next S product and softmax.
// The CTA writes its unnormalised O with (max, sum) per query row: the split
// layout the merge kernel reads. The last split of each (b, g) takes the
// block's own keys.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "internal.h"
#include "common.cuh"
#include "tc_ptx.cuh"

namespace dspark {

cudaError_t launch_attention_merge(const dspark_model* m, const AttnArgs& a, cudaStream_t s);

namespace tc {
namespace {

constexpr int kThreads = 128;
constexpr int KT = 64;               // keys per tile
constexpr int QROWS = 128;           // MMA M
constexpr float kRescale = 5.0f;     // natural-log headroom before the running max is raised

struct AttnTcParams {
    int A, G, nH, nKv, grp, hd, capacity, n_splits, chunk, q_dtype;
    const void* q;                   // [A, G, nH, hd] (fp32 or bf16)
    const int32_t* len;
    float* part_o; float* part_ml;
    int32_t* status;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// Eight fp32 values as a bf16 pair: hi = bf16(v), lo = bf16(v - hi).
__device__ __forceinline__ void split8(const float v[8], uint4& hi, uint4& lo) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float a = v[2 * j], b = v[2 * j + 1];
        const float ah = __bfloat162float(__float2bfloat16_rn(a)), bh = __bfloat162float(__float2bfloat16_rn(b));
        h[j] = pack_bf16x2(ah, bh);
        l[j] = pack_bf16x2(a - ah, b - bh);
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// Zeroes rows [nvalid, KT) of a tile of `nsub` sub-tiles [KT rows x 128 B]
// (the swizzle permutes 16-byte chunks within a row, so rows stay whole):
// past a row's length the cache may hold stale or never-written bytes, and
// P = 0 times a NaN would still poison the accumulator.
__device__ __forceinline__ void zero_rows(uint8_t* tile, int nsub, int nvalid) {
    const int per_sub = (KT - nvalid) * 8;
    for (int i = threadIdx.x; i < nsub * per_sub; i += kThreads) {
        const int sub = i / per_sub, k = i % per_sub;
        reinterpret_cast<uint4*>(tile + sub * KT * 128 + nvalid * 128)[k] = make_uint4(0u, 0u, 0u, 0u);
    }
}

// Operations thread 0 issued on one mbarrier and the phases it has waited
// for; what is outstanding at exit is drained (bounded) before teardown.
struct Issued {
    int n = 0, done = 0;
};

__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
               const __grid_constant__ CUtensorMap tmKb, const __grid_constant__ CUtensorMap tmVb, AttnTcParams P) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const int hd = P.hd, nsub = hd / 64;
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQh = base;                                  // nsub x [128 rows x 128 B]
    uint8_t* sQl = sQh + nsub * QROWS * 128;              // nsub x [128 rows x 128 B]
    uint8_t* sK = sQl + nsub * QROWS * 128;               // nsub x [64 keys x 128 B]
    uint8_t* sV = sK + nsub * KT * 128;                   // nsub x [64 keys x 128 B]
    uint8_t* sPh = sV + nsub * KT * 128;                  // [128 rows x 128 B]
    uint8_t* sPl = sPh + QROWS * 128;                     // [128 rows x 128 B]
    uint64_t* bars = reinterpret_cast<uint64_t*>(sPl + QROWS * 128);
    uint64_t* bar_k = bars;                               // K tile landed
    uint64_t* bar_v = bars + 1;                           // V tile landed
    uint64_t* bar_s = bars + 2;                           // S MMAs done (K buffer free)
    uint64_t* bar_o = bars + 3;                           // P V MMAs done (V and P buffers free)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = threadIdx.x;                            // query row = TMEM lane
    const int bh = blockIdx.x;                            // b * nKv + g
    const int b = bh / P.nKv, g = bh % P.nKv;
    const int split = blockIdx.y;
    const int nq = P.grp * P.G;
    const uint32_t tmem_cols = hd + KT <= 256 ? 256u : 512u;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(&bars[i], 1);
        *abort_flag = 0;
        mbar_fence_init();
        prefetch_tmap(&tmK); prefetch_tmap(&tmV); prefetch_tmap(&tmKb); prefetch_tmap(&tmVb);
    }
    if (warp == 0) tmem_alloc(tmem_slot, tmem_cols);
    __syncthreads();
    // TMEM is held: the next kernel may begin launching; q, the lengths and
    // the caches come from earlier kernels
    pdl_trigger();
    pdl_wait();

    int len = P.len[b];
    if (len < 0 || len > P.capacity) {
        if (threadIdx.x == 0) atomicOr(P.status, DSPARK_DEV_BAD_LENGTH);
        len = min(max(len, 0), P.capacity);
    }
    const bool blk = split == P.n_splits;
    const int k0 = blk ? 0 : split * P.chunk;
    const int k1 = blk ? P.G : min(len, k0 + P.chunk);
    const int row0 = blk ? b * P.G : b * P.capacity;      // first tensor-map row of this (b, g)
    const CUtensorMap* mK = blk ? &tmKb : &tmK;
    const CUtensorMap* mV = blk ? &tmVb : &tmV;
    const uint32_t kv_bytes = (uint32_t)nsub * KT * 128;
    const bool q_lo = P.q_dtype == DSPARK_DTYPE_F32;      // a bf16 q has no low part

    Issued ik, iv, is, io;                                // meaningful in thread 0
    if (threadIdx.x == 0 && k0 < k1) {
        mbar_arrive_expect_tx(bar_k, kv_bytes);
        for (int sub = 0; sub < nsub; ++sub) tma_load_3d(sK + sub * KT * 128, mK, bar_k, sub * 64, g, row0 + k0);
        mbar_arrive_expect_tx(bar_v, kv_bytes);
        for (int sub = 0; sub < nsub; ++sub) tma_load_3d(sV + sub * KT * 128, mV, bar_v, sub * 64, g, row0 + k0);
        ik.n = iv.n = 1;
    }

    // Q tile as a bf16 pair: warp w loads rows w, w+4, ...; a lane owns 8 head dims.
    for (int row = warp; row < QROWS; row += kThreads / 32) {
        for (int c0 = 0; c0 < hd; c0 += 256) {
            const int d = c0 + lane * 8;
            float v[8];
            if (row < nq && d < hd) {
                const int i = row / P.grp, h = g * P.grp + row % P.grp;
                const int64_t off = (((int64_t)b * P.G + i) * P.nH + h) * hd + d;
                if (q_lo) {
                    const float4 a0 = *reinterpret_cast<const float4*>(static_cast<const float*>(P.q) + off);
                    const float4 a1 = *reinterpret_cast<const float4*>(static_cast<const float*>(P.q) + off + 4);
                    v[0] = a0.x; v[1] = a0.y; v[2] = a0.z; v[3] = a0.w; v[4] = a1.x; v[5] = a1.y; v[6] = a1.z; v[7] = a1.w;
                } else {
                    const uint4 u = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(P.q) + off);
                    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) { v[2 * j] = __uint_as_float(w[j] << 16); v[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u); }
                }
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) v[j] = 0.f;
            }
            if (d < hd) {
                const int sub = d / 64, chunk = (d % 64) / 8;
                const int off = sub * QROWS * 128 + row * 128 + ((chunk ^ (row & 7)) * 16);
                uint4 hi, lo;
                split8(v, hi, lo);
                *reinterpret_cast<uint4*>(sQh + off) = hi;
                *reinterpret_cast<uint4*>(sQl + off) = lo;
            }
        }
    }
    fence_async_shared();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const uint32_t tS = tmem_base;                        // columns [0, 64)
    const uint32_t tO = tmem_base + KT;                   // columns [64, 64 + hd)
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;

    const uint32_t idesc_qk = idesc_bf16(QROWS, KT);
    const uint32_t idesc_pv = idesc_bf16(QROWS, hd) | (1u << 16);   // B (V) MN-major

    float m_run = -INFINITY, l_run = 0.f;
    bool first = true, ok = true;
    int it = 0;
    for (int t0 = k0; t0 < k1 && ok; t0 += KT, ++it) {
        const int nvalid = min(KT, k1 - t0);
        const bool has_next = t0 + KT < k1;
        const uint32_t ph = (uint32_t)it & 1u;
        // ---- S = Q K^T
        if (threadIdx.x == 0) {
            if (!mbar_wait(bar_k, ph, abort_flag, P.status)) { ok = false; }
            else {
                ++ik.done;
                tc_fence_after();
                const uint32_t ka = smem_u32(sK);
                for (int part = 0; part < (q_lo ? 2 : 1); ++part) {
                    const uint32_t qa = smem_u32(part ? sQl : sQh);
                    for (int j = 0; j < hd / 16; ++j) {
                        const uint64_t ad = sdesc_k_sw128(qa + (j >> 2) * QROWS * 128 + (j & 3) * 32);
                        const uint64_t bd = sdesc_k_sw128(ka + (j >> 2) * KT * 128 + (j & 3) * 32);
                        mma_bf16(tS, ad, bd, idesc_qk, (part > 0 || j > 0) ? 1u : 0u);
                    }
                }
                mma_commit(bar_s);
                ++is.n;
            }
        }
        if (!mbar_wait(bar_s, ph, abort_flag, P.status)) { ok = false; break; }
        tc_fence_after();
        if (threadIdx.x == 0) {
            ++is.done;
            if (has_next) {                               // the K buffer is free again
                mbar_arrive_expect_tx(bar_k, kv_bytes);
                for (int sub = 0; sub < nsub; ++sub)
                    tma_load_3d(sK + sub * KT * 128, mK, bar_k, sub * 64, g, row0 + t0 + KT);
                ++ik.n;
            }
        }
        // ---- softmax of row r over this tile
        float s[KT];
#pragma unroll
        for (int c = 0; c < KT; c += 16) {
            uint32_t u[16];
            tmem_ld_x16(tS + lane_off + c, u);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j) s[c + j] = c + j < nvalid ? __uint_as_float(u[j]) : -INFINITY;
        }
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < KT; ++j) mx = fmaxf(mx, s[j]);
        const bool need = !first && mx > m_run + kRescale;
        if (first) m_run = mx;
        if (__any_sync(0xffffffffu, need)) {
            const float f = need ? expf(m_run - mx) : 1.f;
            if (need) { l_run *= f; m_run = mx; }
            for (int c = 0; c < hd; c += 16) {
                uint32_t u[16];
                tmem_ld_x16(tO + lane_off + c, u);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 16; ++j) u[j] = __float_as_uint(__uint_as_float(u[j]) * f);
                tmem_st_x16(tO + lane_off + c, u);
            }
            tmem_st_wait();
        }
        float lsum = 0.f;
#pragma unroll
        for (int c = 0; c < KT; c += 8) {
            float p[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) { p[j] = expf(s[c + j] - m_run); lsum += p[j]; }
            const int off = r * 128 + (((c / 8) ^ (r & 7)) * 16);
            uint4 hi, lo;
            split8(p, hi, lo);
            *reinterpret_cast<uint4*>(sPh + off) = hi;
            *reinterpret_cast<uint4*>(sPl + off) = lo;
        }
        l_run += lsum;
        // ---- V tile (rows past the keys zeroed)
        if (!mbar_wait(bar_v, ph, abort_flag, P.status)) { ok = false; break; }
        if (threadIdx.x == 0) ++iv.done;
        if (nvalid < KT) zero_rows(sV, nsub, nvalid);
        fence_async_shared();
        tc_fence_before();
        __syncthreads();
        // ---- O += P V
        if (threadIdx.x == 0) {
            tc_fence_after();
            const uint32_t va = smem_u32(sV);
            for (int part = 0; part < 2; ++part) {
                const uint32_t pa = smem_u32(part ? sPl : sPh);
                for (int j = 0; j < KT / 16; ++j) {
                    const uint64_t ad = sdesc_k_sw128(pa + j * 32);
                    const uint64_t bd = sdesc_mn_sw128(va + j * 2048, KT * 128);
                    mma_bf16(tO, ad, bd, idesc_pv, (!first || part > 0 || j > 0) ? 1u : 0u);
                }
            }
            mma_commit(bar_o);
            ++io.n;
        }
        if (!mbar_wait(bar_o, ph, abort_flag, P.status)) { ok = false; break; }
        tc_fence_after();
        if (threadIdx.x == 0) {
            ++io.done;
            if (has_next) {                               // the V buffer is free again
                mbar_arrive_expect_tx(bar_v, kv_bytes);
                for (int sub = 0; sub < nsub; ++sub)
                    tma_load_3d(sV + sub * KT * 128, mV, bar_v, sub * 64, g, row0 + t0 + KT);
                ++iv.n;
            }
        }
        first = false;
    }

    // ---- write this split's state: unnormalised O and (max, sum) per query row
    if (r < nq) {
        const int i = r / P.grp, h = g * P.grp + r % P.grp;
        const int S1 = P.n_splits + 1;
        const int64_t row = ((int64_t)(b * P.nH + h) * S1 + split) * P.G + i;
        P.part_ml[row * 2] = first ? -INFINITY : m_run;
        P.part_ml[row * 2 + 1] = first ? 0.f : l_run;
    }
    if (!first && ok) {
        const int i = r / P.grp, h = g * P.grp + r % P.grp;
        const int S1 = P.n_splits + 1;
        float* dst = P.part_o + (((int64_t)(b * P.nH + h) * S1 + split) * P.G + i) * hd;
        for (int c = 0; c < hd; c += 16) {
            uint32_t u[16];
            tmem_ld_x16(tO + lane_off + c, u);
            tmem_ld_wait();
            if (r < nq) {
#pragma unroll
                for (int j = 0; j < 16; j += 4)
                    *reinterpret_cast<float4*>(dst + c + j) = make_float4(__uint_as_float(u[j]), __uint_as_float(u[j + 1]),
                                                                          __uint_as_float(u[j + 2]), __uint_as_float(u[j + 3]));
            }
        }
    }
    // after an abort, copies and MMAs still in flight land before teardown (bounded)
    if (threadIdx.x == 0 && !ok) {
        const uint64_t deadline = global_timer_ns() + kWaitLimitNs;
        Issued* all[4] = {&ik, &iv, &is, &io};
        for (int i = 0; i < 4; ++i)
            if (all[i]->n > all[i]->done && !mbar_wait_until(&bars[i], (uint32_t)(all[i]->n - 1) & 1u, deadline))
                atomicOr(P.status, DSPARK_DEV_WAIT_TIMEOUT);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem_base, tmem_cols);
}

PFN_cuTensorMapEncodeTiled_v12000 g_enc = nullptr;
std::once_flag g_enc_once;

// 3-D map over a bf16 [rows, nKv, hd] tensor; box {64, 1, KT}, 128-byte swizzle.
bool make_kv_map(CUtensorMap* tm, const void* ptr, int64_t rows, int nKv, int hd) {
    std::call_once(g_enc_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    if (!g_enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)hd, (cuuint64_t)nKv, (cuuint64_t)rows};
    cuuint64_t strides[2] = {(cuuint64_t)hd * 2, (cuuint64_t)nKv * hd * 2};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)KT};
    cuuint32_t estr[3] = {1, 1, 1};
    return g_enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t attn_tc_smem(int hd) {
    const int nsub = hd / 64;
    // Q pair, K, V, P pair, then 4 barriers + TMEM slot + abort flag; 1 KB alignment slack
    return 2 * (size_t)nsub * QROWS * 128 + 2 * (size_t)nsub * KT * 128 + 2 * QROWS * 128 + 64 + 1024;
}

}  // namespace

bool attention_tc_supported(const dspark_model* m) {
    const Dims& d = m->d;
    return d.dtype == DSPARK_DTYPE_BF16 && d.grp * d.gamma <= QROWS && d.hd % 64 == 0 && d.hd <= 256;
}

int attention_tc_key_tile() { return KT; }

cudaError_t launch_attention_tc(const dspark_model* m, const AttnArgs& a, cudaStream_t s) {
    const Dims& d = m->d;
    CUtensorMap tk, tv, tkb, tvb;
    const int64_t cache_rows = (int64_t)a.batch * a.capacity;   // all rows of this layer's cache
    if (!make_kv_map(&tk, a.kc, cache_rows, d.nKv, d.hd) || !make_kv_map(&tv, a.vc, cache_rows, d.nKv, d.hd) ||
        !make_kv_map(&tkb, a.kb, (int64_t)a.A * d.gamma, d.nKv, d.hd) ||
        !make_kv_map(&tvb, a.vb, (int64_t)a.A * d.gamma, d.nKv, d.hd))
        return cudaErrorInvalidValue;
    AttnTcParams P{};
    P.A = a.A; P.G = d.gamma; P.nH = d.nH; P.nKv = d.nKv; P.grp = d.grp; P.hd = d.hd; P.capacity = a.capacity;
    P.n_splits = a.n_splits; P.chunk = a.chunk; P.q_dtype = a.q_dtype; P.q = a.q; P.len = a.len;
    P.part_o = a.part_o; P.part_ml = a.part_ml; P.status = a.status;
    const size_t smem = attn_tc_smem(d.hd);
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(a.A * d.nKv, a.n_splits + 1);
    e = launch_pdl(attn_tc_kernel, grid, dim3(kThreads), smem, s, tk, tv, tkb, tvb, P);
    if (e != cudaSuccess) return e;
    return launch_attention_merge(m, a, s);
}

}  // namespace tc
}  // namespace dspark
