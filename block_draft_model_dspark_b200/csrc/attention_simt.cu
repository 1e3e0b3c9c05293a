// KV-injection attention on CUDA cores: the DeepspecContextAttention.attend
// seam ("mlx-bun 0.2.0 -> 0.4.0" page 75): block queries attend, non-causally
// and at scale 1.0, over the row's cached context keys followed by the
// block's own keys. The storage-side split: context keys in chunks plus the
// block keys as one more part, each reduced to (max, sum, weighted values),
// then merged by the online-softmax rule.
//
// This is the path of the fp32 workload (no tensor cores at its 1e-4 bar).
#include <float.h>
#include <math.h>

#include "internal.h"
#include "common.cuh"

namespace dspark {
namespace {

constexpr int KT = 16;            // keys per tile
constexpr int kMaxO = 16;         // O elements per thread (G * hd <= 16 * 256)
constexpr int kThreads = 256;

// grid (A * nH, n_splits + 1); one CTA = one query head of one row over one key range.
__global__ void __launch_bounds__(kThreads)
attn_partial_kernel(AttnArgs a, int G, int nH, int nKv, int hd, int dtype) {
    extern __shared__ float sm[];
    float* qs = sm;                       // [G][hd]
    float* ks = qs + G * hd;              // [KT][hd]
    float* vs = ks + KT * hd;             // [KT][hd]
    float* ps = vs + KT * hd;             // [G][KT]
    float* mrow = ps + G * KT;            // [G]
    float* lrow = mrow + G;               // [G]
    float* alpha = lrow + G;              // [G]

    pdl_trigger();
    pdl_wait();
    const int b = blockIdx.x / nH, h = blockIdx.x % nH;
    const int g = h / (nH / nKv);
    const int split = blockIdx.y;
    const int tid = threadIdx.x;

    int len = a.len[b];
    if (len < 0 || len > a.capacity) {
        if (tid == 0) atomicOr(a.status, DSPARK_DEV_BAD_LENGTH);
        len = min(max(len, 0), a.capacity);
    }
    int k0, k1;
    const bool blk = split == a.n_splits;
    if (blk) { k0 = 0; k1 = G; }
    else { k0 = split * a.chunk; k1 = min(len, k0 + a.chunk); }

    for (int e = tid; e < G * hd; e += kThreads) {
        const int i = e / hd, d = e % hd;
        qs[e] = load_any(a.q, (((int64_t)b * G + i) * nH + h) * hd + d, a.q_dtype);
    }
    for (int i = tid; i < G; i += kThreads) { mrow[i] = -INFINITY; lrow[i] = 0.f; }
    float o[kMaxO];
#pragma unroll
    for (int c = 0; c < kMaxO; ++c) o[c] = 0.f;
    __syncthreads();

    for (int t0 = k0; t0 < k1; t0 += KT) {
        const int nt = min(KT, k1 - t0);
        for (int e = tid; e < KT * hd; e += kThreads) {
            const int j = e / hd, d = e % hd;
            float kv = 0.f, vv = 0.f;
            if (j < nt) {
                int64_t idx;
                if (blk) {
                    idx = (((int64_t)b * G + t0 + j) * nKv + g) * hd + d;
                    kv = load_any(a.kb, idx, dtype); vv = load_any(a.vb, idx, dtype);
                } else {
                    idx = (((int64_t)b * a.capacity + t0 + j) * nKv + g) * hd + d;
                    kv = load_any(a.kc, idx, dtype); vv = load_any(a.vc, idx, dtype);
                }
            }
            ks[e] = kv; vs[e] = vv;
        }
        __syncthreads();
        // scores
        for (int e = tid; e < G * KT; e += kThreads) {
            const int i = e / KT, j = e % KT;
            float s = -INFINITY;
            if (j < nt) {
                s = 0.f;
                for (int d = 0; d < hd; ++d) s = fmaf(qs[i * hd + d], ks[j * hd + d], s);
            }
            ps[e] = s;
        }
        __syncthreads();
        // online softmax per query row
        for (int i = tid; i < G; i += kThreads) {
            float mx = mrow[i];
            for (int j = 0; j < nt; ++j) mx = fmaxf(mx, ps[i * KT + j]);
            const float al = expf(mrow[i] - mx);        // mrow = -inf on the first tile: 0
            float l = lrow[i] * al;
            for (int j = 0; j < KT; ++j) {
                const float p = j < nt ? expf(ps[i * KT + j] - mx) : 0.f;
                ps[i * KT + j] = p;
                l += p;
            }
            mrow[i] = mx; lrow[i] = l; alpha[i] = al;
        }
        __syncthreads();
#pragma unroll
        for (int c = 0; c < kMaxO; ++c) {
            const int e = tid + c * kThreads;
            if (e < G * hd) {
                const int i = e / hd, d = e % hd;
                float acc = o[c] * alpha[i];
                for (int j = 0; j < nt; ++j) acc = fmaf(ps[i * KT + j], vs[j * hd + d], acc);
                o[c] = acc;
            }
        }
        __syncthreads();
    }

    const int S1 = a.n_splits + 1;
    const int64_t base = ((int64_t)blockIdx.x * S1 + split) * G;   // (b, h, split) major
#pragma unroll
    for (int c = 0; c < kMaxO; ++c) {
        const int e = tid + c * kThreads;
        if (e < G * hd) a.part_o[base * hd + e] = o[c];
    }
    for (int i = tid; i < G; i += kThreads) {
        a.part_ml[(base + i) * 2] = mrow[i];
        a.part_ml[(base + i) * 2 + 1] = lrow[i];
    }
}

constexpr int kMergeWarps = 8;       // query rows per merge CTA (one warp each)

// One warp per query row (b, h, i): the splits' (max, sum) pairs are read by
// lane s (loops over 32 splits at a time), the weights w_s = exp(m_s - M)
// combine the unnormalised outputs, lane l owning the 4-column groups l, l + 32,
// ... of the row (float4 loads). Empty splits (m = -inf) weigh nothing.
__global__ void __launch_bounds__(kMergeWarps * 32) attn_merge_kernel(AttnArgs a, int G, int nH, int hd, int rows) {
    pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * kMergeWarps + (threadIdx.x >> 5);   // ((b * nH) + h) * G + i
    if (row >= rows) return;
    const int i = row % G, bh = row / G;
    const int b = bh / nH, h = bh % nH;
    const int S1 = a.S1;
    // the row maximum over the splits
    float M = -INFINITY;
    for (int s = lane; s < S1; s += 32) M = fmaxf(M, a.part_ml[(((int64_t)bh * S1 + s) * G + i) * 2]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const int ng = hd / 4;                      // float4 groups of the row
    float4 num[2] = {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};
    float den = 0.f;
    for (int s0 = 0; s0 < S1; s0 += 32) {
        float ws = 0.f, ls = 0.f;
        if (s0 + lane < S1) {
            const int64_t base = ((int64_t)bh * S1 + s0 + lane) * G + i;
            const float m = a.part_ml[base * 2];
            ls = a.part_ml[base * 2 + 1];
            ws = m == -INFINITY ? 0.f : __expf(m - M);
        }
        const int cnt = min(32, S1 - s0);
        for (int t = 0; t < cnt; ++t) {
            const float w = __shfl_sync(0xffffffffu, ws, t);
            den += w * __shfl_sync(0xffffffffu, ls, t);
            if (w == 0.f) continue;                 // uniform: an empty split
            const float* o = a.part_o + (((int64_t)bh * S1 + s0 + t) * G + i) * hd;
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int g4 = lane + q * 32;
                if (g4 < ng) {
                    const float4 v = reinterpret_cast<const float4*>(o)[g4];
                    num[q].x += w * v.x; num[q].y += w * v.y; num[q].z += w * v.z; num[q].w += w * v.w;
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

}  // namespace

cudaError_t launch_attention_merge(const dspark_model* m, const AttnArgs& a, cudaStream_t s);

size_t attn_simt_smem(int G, int hd) {
    return sizeof(float) * ((size_t)G * hd + 2 * (size_t)KT * hd + (size_t)G * KT + 3 * (size_t)G);
}

cudaError_t launch_attention_simt(const dspark_model* m, const AttnArgs& a_in, cudaStream_t s) {
    AttnArgs a = a_in;
    a.S1 = a.n_splits + 1;                      // context splits + the block split
    const Dims& d = m->d;
    const size_t smem = attn_simt_smem(d.gamma, d.hd);
    static thread_local int configured_dev = -1;
    if (configured_dev != m->device) {
        cudaFuncSetAttribute(attn_partial_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 96 * 1024);
        configured_dev = m->device;
    }
    dim3 grid(a.A * d.nH, a.n_splits + 1);
    cudaError_t e = launch_pdl(attn_partial_kernel, grid, dim3(kThreads), smem, s, a, d.gamma, d.nH, d.nKv, d.hd,
                               d.kv_dtype);
    if (e != cudaSuccess) return e;
    return launch_attention_merge(m, a, s);
}

cudaError_t launch_attention_merge(const dspark_model* m, const AttnArgs& a, cudaStream_t s) {
    const Dims& d = m->d;
    const int rows = a.A * d.nH * d.gamma;
    return launch_pdl(attn_merge_kernel, dim3((rows + kMergeWarps - 1) / kMergeWarps), dim3(kMergeWarps * 32), 0, s, a,
                      d.gamma, d.nH, d.hd, rows);
}

}  // namespace dspark
