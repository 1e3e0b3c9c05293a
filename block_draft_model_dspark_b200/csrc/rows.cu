// Row-wise kernels of the round: the block embedding, the fused epilogues
// that follow each GEMM (norms, RoPE, residual adds, gelu, layer scalar),
// the context K/V epilogue, and the confidence head with truncation.
//
// Each epilogue reads its GEMM's result through a PartView, which sums the
// GEMM's partial tiles in a fixed order (results do not depend on
// scheduling). Activations that feed the next GEMM are written in fp32 and,
// for the tensor-core GEMMs of a bf16 model, also in fp16 (hi = fp16(v), and
// for the pair form lo = fp16(v - hi)).
#include <math.h>

#include <algorithm>

#include "internal.h"
#include "common.cuh"

namespace dspark {
namespace {

constexpr int kMaxPer = 16;   // columns per thread in the full-row kernels

// The fp32 form is written only where a consumer reads it (f32 != NULL).
__device__ __forceinline__ void store_act(const ActBuf& a, int64_t i, float v) {
    if (a.f32) a.f32[i] = v;
    if (a.hi) {
        const __half h = __float2half_rn(v);
        a.hi[i] = h;
        if (a.lo) a.lo[i] = __float2half_rn(v - __half2float(h));
    }
}

// Four consecutive activation values at i .. i + 3 (i % 4 == 0).
__device__ __forceinline__ void store_act4(const ActBuf& a, int64_t i, float4 v) {
    if (a.f32) *reinterpret_cast<float4*>(a.f32 + i) = v;
    if (a.hi) {
        const __half2 h01 = __floats2half2_rn(v.x, v.y), h23 = __floats2half2_rn(v.z, v.w);
        uint2 hv;
        hv.x = *reinterpret_cast<const uint32_t*>(&h01);
        hv.y = *reinterpret_cast<const uint32_t*>(&h23);
        *reinterpret_cast<uint2*>(a.hi + i) = hv;
        if (a.lo) {
            const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
            const __half2 l01 = __floats2half2_rn(v.x - f01.x, v.y - f01.y), l23 = __floats2half2_rn(v.z - f23.x, v.w - f23.y);
            uint2 lv;
            lv.x = *reinterpret_cast<const uint32_t*>(&l01);
            lv.y = *reinterpret_cast<const uint32_t*>(&l23);
            *reinterpret_cast<uint2*>(a.lo + i) = lv;
        }
    }
}

// One element W[n, j] of a (possibly 4-bit) matrix.
__device__ __forceinline__ float mat_at(const MatRef& W, int dtype, int group, int64_t n, int64_t j) {
    if (!W.quant) return load_any(W.w, n * W.k + j, dtype);
    const uint32_t w = static_cast<const uint32_t*>(W.w)[n * (W.k / 8) + j / 8];
    const int64_t g = n * (W.k / group) + j / group;
    return fmaf(__bfloat162float(W.scales[g]), (float)((w >> (4 * (j % 8))) & 0xFu), __bfloat162float(W.biases[g]));
}

// ------------------------------------------------------------------ context K/V
// grid (rows, Lyr*nKv), block hd/2: thread i owns the RoPE pair (i, i + hd/2).
__global__ void kv_epilogue_kernel(PartView raw, RowsPlan rp, KvDest dst, const double* __restrict__ inv_freq,
                                   LayerPtrs k_norms, int nKv, int hd, float eps, int dtype, int kv_dtype,
                                   int32_t* status) {
    __shared__ float red[32];
    pdl_trigger();
    pdl_wait();
    const int r = blockIdx.x;
    const int rg = rp.row0 + r;
    const int b = rg / rp.Lrows, t = rg % rp.Lrows;
    if (rp.n_valid && t >= rp.n_valid[b]) return;
    const int dst_row = (rp.dst_row0 ? rp.dst_row0[b] : 0) + t;
    if (dst_row < 0 || dst_row >= dst.capacity) {
        if (threadIdx.x == 0) atomicOr(status, DSPARK_DEV_BAD_LENGTH);
        return;
    }
    const int pos = (rp.pos0 ? rp.pos0[b] : rp.static_pos) + dst_row;
    const int l = blockIdx.y / nKv, g = blockIdx.y % nKv;
    const int half = hd / 2, i = threadIdx.x;
    const int64_t col = (int64_t)blockIdx.y * hd;
    const PartView::Pending q1 = raw.load(r, col + i), q2 = raw.load(r, col + i + half);
    const float x1 = raw.finish(q1), x2 = raw.finish(q2);
    const float ss = block_sum(x1 * x1 + x2 * x2, red);
    const float rinv = rsqrtf(ss / (float)hd + eps);
    const float v1 = x1 * rinv, v2 = x2 * rinv;
    const int64_t o = (int64_t)l * dst.layer_stride + (int64_t)b * dst.batch_stride + ((int64_t)dst_row * nKv + g) * hd;
    store_any(dst.v, o + i, kv_dtype, v1);
    store_any(dst.v, o + i + half, kv_dtype, v2);
    if (!dst.k) return;                                    // a V-only cache
    const void* wk = k_norms.p[l];
    const float k1 = v1 * load_any(wk, i, dtype), k2 = v2 * load_any(wk, i + half, dtype);
    float sn, cs;
    rope_sincos(pos, inv_freq[i], &sn, &cs);
    store_any(dst.k, o + i, kv_dtype, k1 * cs - k2 * sn);
    store_any(dst.k, o + i + half, kv_dtype, k2 * cs + k1 * sn);
}

// ------------------------------------------------------------------ context features
// deepspec.ts #projectContext: out[r] = rms(raw[r], hidden_norm), raw = the taps' hiddens @ fc^T.
// grid rows, block 256; the row's H values in shared memory between the two passes.
__global__ void context_norm_kernel(PartView raw, int H, const void* __restrict__ gain, float eps, int dtype,
                                    void* __restrict__ out) {
    extern __shared__ float ctx_row[];
    __shared__ float red[32];
    pdl_trigger();
    pdl_wait();
    const int r = blockIdx.x;
    float ss = 0.f;
    for (int j = threadIdx.x; j < H; j += blockDim.x) {
        const float x = raw.sum(r, j);
        ctx_row[j] = x;                                   // each thread reads back only its own columns
        ss += x * x;
    }
    ss = block_sum(ss, red);
    const float rinv = rsqrtf(ss / (float)H + eps);
    for (int j = threadIdx.x; j < H; j += blockDim.x)
        store_any(out, (int64_t)r * H + j, dtype, ctx_row[j] * rinv * load_any(gain, j, dtype));
}

// The append's device-side validation (the accepted-row counts come from the
// caller's device memory, so the host cannot check them): every row must have
// 0 <= n_new[b] <= Lnew_max and len[b] + n_new[b] <= capacity. If any row
// fails, the whole append is refused -- every count becomes 0, so the
// epilogue writes no cache row and the commit adds nothing -- and
// DSPARK_DEV_CAPACITY is recorded. One CTA; row0[b] snapshots len[b], the
// cache row where row b's new rows start.
constexpr int kCheckThreads = 1024;
__global__ void __launch_bounds__(kCheckThreads) append_check_kernel(const int32_t* __restrict__ n_new,
                                                                     const int32_t* __restrict__ len, int B,
                                                                     int Lnew_max, int capacity,
                                                                     int32_t* __restrict__ nvalid,
                                                                     int32_t* __restrict__ row0,
                                                                     int32_t* __restrict__ status) {
    pdl_trigger();
    pdl_wait();
    int bad = 0;
    for (int b = threadIdx.x; b < B; b += kCheckThreads) {
        const int n = n_new[b], l = len[b];
        if (n < 0 || n > Lnew_max || l < 0 || (int64_t)l + n > capacity) bad = 1;
    }
    bad = __syncthreads_or(bad);
    for (int b = threadIdx.x; b < B; b += kCheckThreads) {
        nvalid[b] = bad ? 0 : n_new[b];
        row0[b] = len[b];
    }
    if (bad && threadIdx.x == 0) atomicOr(status, DSPARK_DEV_CAPACITY);
}

__global__ void commit_len_kernel(int32_t* len, const int32_t* n_new, int B) {
    pdl_trigger();
    pdl_wait();
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b < B) len[b] += n_new[b];
}

// ------------------------------------------------------------------ block embedding
__global__ void __launch_bounds__(1024) embed_kernel(MatRef E, int dtype, int group, const int32_t* __restrict__ anchors, int gamma,
                             int mask_id, int V, int H, float scale, const void* __restrict__ w_in,
                             float eps, float* __restrict__ h, ActBuf x, int32_t* status) {
    __shared__ float red[32];
    pdl_trigger();
    pdl_wait();
    const int m = blockIdx.x;
    const int b = m / gamma, t = m % gamma;
    int id = t == 0 ? anchors[b] : mask_id;
    if (id < 0 || id >= V) {
        if (threadIdx.x == 0) atomicOr(status, DSPARK_DEV_BAD_TOKEN);
        id = min(max(id, 0), V - 1);
    }
    float vals[kMaxPer];
    float ss = 0.f;
    if (!E.quant && dtype == DSPARK_DTYPE_BF16 && (H & 7) == 0) {
        // bf16 rows: 8 consecutive values (16 bytes) per load, groups tid, tid + blockDim.x
        const uint4* row = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(E.w) + (int64_t)id * E.k);
#pragma unroll
        for (int c8 = 0; c8 < kMaxPer / 8; ++c8) {
            const int gi = threadIdx.x + c8 * blockDim.x;
            uint4 u = make_uint4(0u, 0u, 0u, 0u);
            if (gi * 8 < H) u = row[gi];
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                vals[c8 * 8 + 2 * k] = __uint_as_float(w[k] << 16) * scale;
                vals[c8 * 8 + 2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u) * scale;
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) ss += vals[c8 * 8 + k] * vals[c8 * 8 + k];
        }
        ss = block_sum(ss, red);
        const float rinv = rsqrtf(ss / (float)H + eps);
#pragma unroll
        for (int c8 = 0; c8 < kMaxPer / 8; ++c8) {
            const int j = (threadIdx.x + c8 * blockDim.x) * 8;
            if (j >= H) continue;
            float4* hp = reinterpret_cast<float4*>(h + (int64_t)m * H + j);
            hp[0] = make_float4(vals[c8 * 8], vals[c8 * 8 + 1], vals[c8 * 8 + 2], vals[c8 * 8 + 3]);
            hp[1] = make_float4(vals[c8 * 8 + 4], vals[c8 * 8 + 5], vals[c8 * 8 + 6], vals[c8 * 8 + 7]);
            float y[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) y[k] = vals[c8 * 8 + k] * rinv * load_any(w_in, j + k, dtype);
            store_act4(x, (int64_t)m * H + j, make_float4(y[0], y[1], y[2], y[3]));
            store_act4(x, (int64_t)m * H + j + 4, make_float4(y[4], y[5], y[6], y[7]));
        }
        return;
    }
#pragma unroll
    for (int c = 0; c < kMaxPer; ++c) {
        const int j = threadIdx.x + c * blockDim.x;
        vals[c] = 0.f;
        if (j < H) {
            vals[c] = mat_at(E, dtype, group, id, j) * scale;
            ss += vals[c] * vals[c];
        }
    }
    ss = block_sum(ss, red);
    const float rinv = rsqrtf(ss / (float)H + eps);
#pragma unroll
    for (int c = 0; c < kMaxPer; ++c) {
        const int j = threadIdx.x + c * blockDim.x;
        if (j < H) {
            h[(int64_t)m * H + j] = vals[c];
            store_act(x, (int64_t)m * H + j, vals[c] * rinv * load_any(w_in, j, dtype));
        }
    }
}

// ------------------------------------------------------------------ q / k / v heads
// grid (M, ceil((nH + nKv) / kQkWarps)), block kQkWarps warps: the row's RoPE
// angles (hd/2 of them, one position) go into shared memory first, one per
// thread, then one warp per head.
constexpr int kQkWarps = 4;
// Four consecutive values at i .. i + 3 of an fp32 or fp16 tensor (i % 4 == 0).
__device__ __forceinline__ void store4_any(void* p, int64_t i, int dtype, float4 v) {
    if (dtype == DSPARK_DTYPE_F32) {
        *reinterpret_cast<float4*>(static_cast<float*>(p) + i) = v;
    } else if (dtype == DSPARK_DTYPE_F16) {
        const __half2 a = __floats2half2_rn(v.x, v.y), c = __floats2half2_rn(v.z, v.w);
        uint2 u;
        u.x = *reinterpret_cast<const uint32_t*>(&a);
        u.y = *reinterpret_cast<const uint32_t*>(&c);
        *reinterpret_cast<uint2*>(static_cast<__half*>(p) + i) = u;
    } else {
        store_any(p, i, dtype, v.x); store_any(p, i + 1, dtype, v.y);
        store_any(p, i + 2, dtype, v.z); store_any(p, i + 3, dtype, v.w);
    }
}
__global__ void __launch_bounds__(32 * kQkWarps)
qk_epilogue_kernel(PartView part, int gamma, int nH, int nKv, int hd, const int32_t* __restrict__ block_pos,
                   const double* __restrict__ inv_freq, const void* __restrict__ q_norm,
                   const void* __restrict__ k_norm, float eps, int dtype, int kv_dtype, void* __restrict__ q,
                   void* __restrict__ kb, void* __restrict__ vb) {
    __shared__ float s_sin[128], s_cos[128];
    pdl_trigger();
    pdl_wait();
    const int m = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int b = m / gamma, t = m % gamma;
    const int pos = block_pos[b] + t;
    const int half = hd / 2;
    for (int i = threadIdx.x; i < half; i += blockDim.x) rope_sincos(pos, inv_freq[i], &s_sin[i], &s_cos[i]);
    __syncthreads();
    const int hh = blockIdx.y * kQkWarps + warp;
    if (hh >= nH + nKv) return;
    // lane l: the RoPE pairs (i, i + hd/2) for the four i = 4l .. 4l + 3 (lanes past hd/8 idle)
    const int i0 = 4 * lane;
    const bool act = i0 < half;
    const int64_t col = (int64_t)hh * hd;
    float4 x1 = make_float4(0.f, 0.f, 0.f, 0.f), x2 = x1;
    if (act) {
        const PartView::Pending4 p1 = part.load4(m, col + i0), p2 = part.load4(m, col + i0 + half);
        x1 = part.finish4(p1);
        x2 = part.finish4(p2);
    }
    float ss = x1.x * x1.x + x1.y * x1.y + x1.z * x1.z + x1.w * x1.w + x2.x * x2.x + x2.y * x2.y + x2.z * x2.z +
               x2.w * x2.w;
    ss = warp_sum(ss);
    if (!act) return;
    const float rinv = rsqrtf(ss / (float)hd + eps);
    const float a1[4] = {x1.x * rinv, x1.y * rinv, x1.z * rinv, x1.w * rinv};
    const float a2[4] = {x2.x * rinv, x2.y * rinv, x2.z * rinv, x2.w * rinv};
    float r1[4], r2[4];
    if (hh < nH) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = i0 + j;
            const float y1 = a1[j] * load_any(q_norm, i, dtype), y2 = a2[j] * load_any(q_norm, i + half, dtype);
            r1[j] = y1 * s_cos[i] - y2 * s_sin[i];
            r2[j] = y2 * s_cos[i] + y1 * s_sin[i];
        }
        const int64_t o = ((int64_t)m * nH + hh) * hd;                // the attention's query type
        store4_any(q, o + i0, kv_dtype, make_float4(r1[0], r1[1], r1[2], r1[3]));
        store4_any(q, o + i0 + half, kv_dtype, make_float4(r2[0], r2[1], r2[2], r2[3]));
    } else {
        const int g = hh - nH;
        const int64_t o = ((int64_t)m * nKv + g) * hd;
        store4_any(vb, o + i0, kv_dtype, make_float4(a1[0], a1[1], a1[2], a1[3]));
        store4_any(vb, o + i0 + half, kv_dtype, make_float4(a2[0], a2[1], a2[2], a2[3]));
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = i0 + j;
            const float k1 = a1[j] * load_any(k_norm, i, dtype), k2 = a2[j] * load_any(k_norm, i + half, dtype);
            r1[j] = k1 * s_cos[i] - k2 * s_sin[i];
            r2[j] = k2 * s_cos[i] + k1 * s_sin[i];
        }
        store4_any(kb, o + i0, kv_dtype, make_float4(r1[0], r1[1], r1[2], r1[3]));
        store4_any(kb, o + i0 + half, kv_dtype, make_float4(r2[0], r2[1], r2[2], r2[3]));
    }
}

// ------------------------------------------------------------------ o_proj / down epilogues
// mode 0 (o_proj):  h += rms(sum, g1);            x = rms(h, g2)
// mode 1 (down):    h = (h + rms(sum, g1)) * s;   x = rms(h, g2)
//
// grid (C, M) with clusters of C CTAs along x: the C CTAs of a row split its
// columns (CTA c owns [c * span, (c + 1) * span), span = blockDim.x * PER) and
// add up the row's two sums of squares through distributed shared memory, in
// rank order, so every CTA gets the same totals. Few rows (a draft block)
// thereby still spread over many SMs.

// Sum of v over the block, then over the cluster's C CTAs (rank order). `slot`
// is this CTA's shared word for the exchange; callers end with cluster_sync()
// before exiting so no CTA leaves while another still reads its slot.
__device__ __forceinline__ float cluster_row_sum(float v, float* red, float* slot, int C) {
    v = block_sum(v, red);
    if (C == 1) return v;
    if (threadIdx.x == 0) *slot = v;
    cluster_sync();
    float t = 0.f;
    for (int r = 0; r < C; ++r) t += ld_cluster_f32(slot, r);
    return t;
}

template <int PER>
__global__ void __launch_bounds__(512) residual_epilogue_kernel(PartView part, int H, const void* __restrict__ g1,
                                         const void* __restrict__ g2, const void* __restrict__ scalar, int mode,
                                         float eps, int dtype, float* __restrict__ h, ActBuf x) {
    constexpr int G4 = PER / 4;                  // float4 groups per thread
    __shared__ float red[32];
    __shared__ float xch[2];
    pdl_trigger();
    const int C = gridDim.x;
    const int m = blockIdx.y;
    // this thread's columns: 4 consecutive ones per group, groups blockDim.x * 4 apart
    const int j0 = blockIdx.x * blockDim.x * PER + threadIdx.x * 4;
    float a[PER], hv[PER], w1v[PER], w2v[PER];
    // the gains are weights: loaded while the producing GEMM drains
#pragma unroll
    for (int g = 0; g < G4; ++g) {
        const int j = j0 + g * blockDim.x * 4;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const bool in = j + c < H;
            w1v[g * 4 + c] = in ? load_any(g1, j + c, dtype) : 0.f;
            w2v[g * 4 + c] = in ? load_any(g2, j + c, dtype) : 0.f;
        }
    }
    const float s = mode == 1 ? load_any(scalar, 0, dtype) : 1.f;
    pdl_wait();
    // the activation loads go out two groups at a time (each with all its partials):
    // a round of memory latency per two groups at bounded registers
    constexpr int kBatch = G4 < 2 ? G4 : 2;
#pragma unroll
    for (int g0 = 0; g0 < G4; g0 += kBatch) {
        PartView::Pending4T<(PER == 4 ? 8 : 4)> q[kBatch];   // few columns a thread (small M): the many partials at once
#pragma unroll
        for (int gb = 0; gb < kBatch; ++gb) {
            const int g = g0 + gb;
            const int j = j0 + g * blockDim.x * 4;
            const bool in = j < H;
            q[gb] = part.load4<(PER == 4 ? 8 : 4)>(m, in ? j : 0);
            const float4 hh = in ? *reinterpret_cast<const float4*>(h + (int64_t)m * H + j) : make_float4(0.f, 0.f, 0.f, 0.f);
            hv[g * 4] = hh.x; hv[g * 4 + 1] = hh.y; hv[g * 4 + 2] = hh.z; hv[g * 4 + 3] = hh.w;
        }
#pragma unroll
        for (int gb = 0; gb < kBatch; ++gb) {
            const int g = g0 + gb;
            const int j = j0 + g * blockDim.x * 4;
            const float4 v = j < H ? part.finish4(q[gb]) : make_float4(0.f, 0.f, 0.f, 0.f);
            a[g * 4] = v.x; a[g * 4 + 1] = v.y; a[g * 4 + 2] = v.z; a[g * 4 + 3] = v.w;
        }
    }
    float ss = 0.f;
#pragma unroll
    for (int c = 0; c < PER; ++c) ss += a[c] * a[c];
    ss = cluster_row_sum(ss, red, &xch[0], C);
    const float r1 = rsqrtf(ss / (float)H + eps);
    float ss2 = 0.f;
#pragma unroll
    for (int c = 0; c < PER; ++c) {
        hv[c] = (hv[c] + a[c] * r1 * w1v[c]) * s;
        ss2 += hv[c] * hv[c];
    }
    ss2 = cluster_row_sum(ss2, red, &xch[1], C);
    const float r2 = rsqrtf(ss2 / (float)H + eps);
#pragma unroll
    for (int g = 0; g < G4; ++g) {
        const int j = j0 + g * blockDim.x * 4;
        if (j < H) {
            const int64_t o = (int64_t)m * H + j;
            *reinterpret_cast<float4*>(h + o) = make_float4(hv[g * 4], hv[g * 4 + 1], hv[g * 4 + 2], hv[g * 4 + 3]);
            store_act4(x, o, make_float4(hv[g * 4] * r2 * w2v[g * 4], hv[g * 4 + 1] * r2 * w2v[g * 4 + 1],
                                         hv[g * 4 + 2] * r2 * w2v[g * 4 + 2], hv[g * 4 + 3] * r2 * w2v[g * 4 + 3]));
        }
    }
    if (C > 1) cluster_sync();
}

// The same epilogue with one CTA of kResThreads per row and the row's GEMM
// result in shared memory (H / 4 float4, one per 4-column group; a thread owns
// groups tid, tid + kResThreads, ...): few registers, so several rows share an
// SM, for M well above the SM count. Three passes over the thread's groups:
// the partial sums (two groups' loads in flight) and their sum of squares; h
// and its sum of squares; x.
constexpr int kResThreads = 256;
__global__ void __launch_bounds__(kResThreads, 4) residual_row_kernel(PartView part, int H, const void* __restrict__ g1,
                                                                   const void* __restrict__ g2,
                                                                   const void* __restrict__ scalar, int mode, float eps,
                                                                   int dtype, float* __restrict__ h, ActBuf x) {
    extern __shared__ float4 srow[];                // [H / 4]
    __shared__ float red[32];
    pdl_trigger();
    const float s = mode == 1 ? load_any(scalar, 0, dtype) : 1.f;
    pdl_wait();
    const int m = blockIdx.x, ng = H / 4;
    float ss = 0.f;
    for (int g0 = threadIdx.x; g0 < ng; g0 += 2 * kResThreads) {
        const int ga = g0, gb = g0 + kResThreads;
        PartView::Pending4 qa, qb;
        qa = part.load4(m, 4 * (int64_t)ga);
        if (gb < ng) qb = part.load4(m, 4 * (int64_t)gb);
        const float4 va = part.finish4(qa);
        srow[ga] = va;
        ss += va.x * va.x + va.y * va.y + va.z * va.z + va.w * va.w;
        if (gb < ng) {
            const float4 vb = part.finish4(qb);
            srow[gb] = vb;
            ss += vb.x * vb.x + vb.y * vb.y + vb.z * vb.z + vb.w * vb.w;
        }
    }
    ss = block_sum(ss, red);
    const float r1 = rsqrtf(ss / (float)H + eps);
    float4* hrow = reinterpret_cast<float4*>(h + (int64_t)m * H);
    float ss2 = 0.f;
    for (int gi = threadIdx.x; gi < ng; gi += kResThreads) {
        const float4 a = srow[gi], hh = hrow[gi];
        const int j = 4 * gi;
        float4 v;
        v.x = (hh.x + a.x * r1 * load_any(g1, j, dtype)) * s;
        v.y = (hh.y + a.y * r1 * load_any(g1, j + 1, dtype)) * s;
        v.z = (hh.z + a.z * r1 * load_any(g1, j + 2, dtype)) * s;
        v.w = (hh.w + a.w * r1 * load_any(g1, j + 3, dtype)) * s;
        hrow[gi] = v;
        srow[gi] = v;
        ss2 += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
    }
    ss2 = block_sum(ss2, red);
    const float r2 = rsqrtf(ss2 / (float)H + eps);
    for (int gi = threadIdx.x; gi < ng; gi += kResThreads) {
        const float4 v = srow[gi];
        const int j = 4 * gi;
        store_act4(x, (int64_t)m * H + j,
                   make_float4(v.x * r2 * load_any(g2, j, dtype), v.y * r2 * load_any(g2, j + 1, dtype),
                               v.z * r2 * load_any(g2, j + 2, dtype), v.w * r2 * load_any(g2, j + 3, dtype)));
    }
}

// grid (ceil(I / (4 kGuGroups * 256)), M), 256 threads: thread t of CTA x owns the
// kGuGroups 4-column groups x * 256 kGuGroups + t + 256 j; all their gate and up
// loads go out before the first is used (two groups per thread, with two or four
// partials in flight each, measured no faster at 512 rows and slower at 16).
constexpr int kGuGroups = 1;
constexpr int kGuPartials = 4;      // partials in flight per load
__global__ void __launch_bounds__(256) gu_epilogue_kernel(PartView part, int M, int I, ActBuf act) {
    pdl_trigger();
    pdl_wait();
    const int m = blockIdx.y;
    const int64_t g0 = (int64_t)blockIdx.x * blockDim.x * kGuGroups + threadIdx.x;
    PartView::Pending4T<kGuPartials> qg[kGuGroups], qu[kGuGroups];
#pragma unroll
    for (int j = 0; j < kGuGroups; ++j) {
        const int64_t i = (g0 + (int64_t)j * blockDim.x) * 4;
        if (i < I) {
            qg[j] = part.load4<kGuPartials>(m, i);
            qu[j] = part.load4<kGuPartials>(m, I + i);
        }
    }
#pragma unroll
    for (int j = 0; j < kGuGroups; ++j) {
        const int64_t i = (g0 + (int64_t)j * blockDim.x) * 4;
        if (i >= I) continue;
        const float4 g = part.finish4(qg[j]), u = part.finish4(qu[j]);
        store_act4(act, (int64_t)m * I + i,
                   make_float4(gelu_tanh(g.x) * u.x, gelu_tanh(g.y) * u.y, gelu_tanh(g.z) * u.z, gelu_tanh(g.w) * u.w));
    }
}

// ------------------------------------------------------------------ confidence + truncation
// grid A * gamma, block 256: c[b,k] = sigmoid(proj . [hf(b,k) ; w1[prev_k]] + bias),
// prev_0 = anchor, prev_k = tokens[b, k-1].
__global__ void confidence_kernel(const float* __restrict__ hf32, MatRef P, int dtype, int group,
                                  const void* __restrict__ w1, const void* __restrict__ bias,
                                  const int32_t* __restrict__ anchors, const int32_t* __restrict__ tokens,
                                  int gamma, int H, int r, int with_markov, int V, float* __restrict__ conf) {
    __shared__ float red[32];
    pdl_trigger();
    pdl_wait();
    const int m = blockIdx.x;
    const int b = m / gamma, k = m % gamma;
    int prev = k == 0 ? anchors[b] : tokens[b * gamma + k - 1];
    prev = min(max(prev, 0), V - 1);
    float z = 0.f;
    for (int j = threadIdx.x; j < H; j += blockDim.x) z += hf32[(int64_t)m * H + j] * mat_at(P, dtype, group, 0, j);
    if (with_markov)
        for (int j = threadIdx.x; j < r; j += blockDim.x)
            z += load_any(w1, (int64_t)prev * r + j, dtype) * mat_at(P, dtype, group, 0, H + j);
    z = block_sum(z, red) + load_any(bias, 0, dtype);
    if (threadIdx.x == 0) conf[m] = 1.f / (1.f + expf(-z));
}

// lengths[b] = first k with conf < thr (thr > 0), else gamma (no head: gamma).
__global__ void lengths_kernel(const float* __restrict__ conf, int A, int gamma, float thr, int has_head,
                               int32_t* __restrict__ lengths) {
    pdl_trigger();
    pdl_wait();
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= A) return;
    int len = gamma;
    if (has_head && thr > 0.f)
        for (int k = 0; k < gamma; ++k)
            if (conf[(int64_t)b * gamma + k] < thr) { len = k; break; }
    lengths[b] = len;
}

// Alg 1 (the DFlash generator's confidence-scheduled draft-length pruning):
// lengths[b] = first k >= 1 with conf[b, k] < thr[k], else gamma (position 0
// always survives; a NaN confidence is not below any threshold).
__global__ void prune_lengths_kernel(const float* __restrict__ conf, int A, int gamma, const float* __restrict__ thr,
                                     int32_t* __restrict__ lengths) {
    pdl_trigger();
    pdl_wait();
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= A) return;
    int len = gamma;
    for (int k = 1; k < gamma; ++k)
        if (conf[(int64_t)b * gamma + k] < thr[k]) { len = k; break; }
    lengths[b] = len;
}

// Threads of a full-row kernel: enough that each holds at most kMaxPer
// columns, about 8 columns per thread, and at most 512 (the kernels use up
// to ~80 registers a thread; 512 x 80 fits a block's register file).
// Columns per thread (template argument of the full-row kernels) for a row
// of H spread over row_threads(H) threads.
int row_per(int H, int threads) {
    const int per = (H + threads - 1) / threads;
    return per <= 4 ? 4 : per <= 8 ? 8 : kMaxPer;
}

template <int PER>
cudaError_t launch_residual(const PartView& part, int M, int H, const void* g1, const void* g2, const void* scalar,
                            int mode, float eps, int dtype, float* h, const ActBuf& x, int C, int threads,
                            cudaStream_t s) {
    return launch_pdl_cluster(residual_epilogue_kernel<PER>, dim3(C, M), dim3(threads), C, 0, s, part, H, g1, g2,
                              scalar, mode, eps, dtype, h, x);
}

int row_threads(int H) {
    int t = (H + 7) / 8;
    const int need = (H + kMaxPer - 1) / kMaxPer;
    if (t > 512) t = 512;
    if (t < need) t = need;
    t = (t + 31) / 32 * 32;
    return t < 32 ? 32 : t;
}

// Rows of a full-row epilogue spread over a cluster of C CTAs (C a power of
// two, at most 8) while M * C stays under about one CTA per SM and each CTA
// keeps >= 256 columns.
int residual_cluster(int M, int H, int num_sms) {
    int C = 1;
    while (C < 8 && M * C * 2 <= num_sms && H / (C * 2) >= 256) C *= 2;
    return C;
}

cudaError_t launch_residual_any(const PartView& part, int M, int H, const void* g1, const void* g2,
                                const void* scalar, int mode, float eps, int dtype, float* h, const ActBuf& x,
                                int num_sms, cudaStream_t s) {
    const int C = residual_cluster(M, H, num_sms);
    if (C == 1 && M >= num_sms && H % 4 == 0) {      // rows enough to fill the SMs: a CTA per row
        const size_t smem = (size_t)H * sizeof(float);
        if (smem > 48 * 1024) {
            const cudaError_t e = cudaFuncSetAttribute(residual_row_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                       (int)smem);
            if (e != cudaSuccess) return e;
        }
        return launch_pdl(residual_row_kernel, dim3(M), dim3(kResThreads), smem, s, part, H, g1, g2, scalar, mode, eps,
                          dtype, h, x);
    }
    const int Hc = (H + C - 1) / C;                 // columns per CTA
    // split rows: ~4 columns a thread (each load group of 4 covers the CTA's columns)
    const int t = C > 1 ? std::min(512, std::max(32, ((Hc + 3) / 4 + 31) / 32 * 32)) : row_threads(Hc);
    switch (row_per(Hc, t)) {
        case 4: return launch_residual<4>(part, M, H, g1, g2, scalar, mode, eps, dtype, h, x, C, t, s);
        case 8: return launch_residual<8>(part, M, H, g1, g2, scalar, mode, eps, dtype, h, x, C, t, s);
        default: return launch_residual<kMaxPer>(part, M, H, g1, g2, scalar, mode, eps, dtype, h, x, C, t, s);
    }
}

}  // namespace

cudaError_t launch_kv_epilogue(const dspark_model* m, const PartView& raw, const RowsPlan& rp, const KvDest& dst,
                               cudaStream_t s) {
    const Dims& d = m->d;
    if (rp.nrows <= 0) return cudaSuccess;
    LayerPtrs kn{};
    for (int l = 0; l < d.Lyr; ++l) kn.p[l] = m->layers[l].k_norm;
    dim3 grid(rp.nrows, d.Lyr * d.nKv);
    return launch_pdl(kv_epilogue_kernel, grid, dim3(d.hd / 2), 0, s, raw, rp, dst, m->ws.inv_freq, kn, d.nKv, d.hd,
                      d.eps, d.dtype, d.kv_dtype, m->ws.status);
}

cudaError_t launch_context_norm(const dspark_model* m, const PartView& raw, int nrows, const void* gain, void* out,
                                cudaStream_t s) {
    const Dims& d = m->d;
    if (nrows <= 0) return cudaSuccess;
    return launch_pdl(context_norm_kernel, dim3(nrows), dim3(256), (size_t)d.H * sizeof(float), s, raw, d.H, gain,
                      d.eps, d.dtype, out);
}

cudaError_t launch_prune_lengths(const float* conf, int A, int gamma, const float* thr, int32_t* lengths,
                                 cudaStream_t s) {
    if (A <= 0) return cudaSuccess;
    return launch_pdl(prune_lengths_kernel, dim3((A + 127) / 128), dim3(128), 0, s, conf, A, gamma, thr, lengths);
}

cudaError_t launch_append_check(const int32_t* n_new, const int32_t* len, int B, int Lnew_max, int capacity,
                                int32_t* nvalid, int32_t* row0, int32_t* status, cudaStream_t s) {
    return launch_pdl(append_check_kernel, dim3(1), dim3(kCheckThreads), 0, s, n_new, len, B, Lnew_max, capacity,
                      nvalid, row0, status);
}

cudaError_t launch_commit_len(int32_t* len, const int32_t* n_new, int B, cudaStream_t s) {
    return launch_pdl(commit_len_kernel, dim3((B + 127) / 128), dim3(128), 0, s, len, n_new, B);
}

cudaError_t launch_embed(const dspark_model* m, const int32_t* anchors, int A, float* h, const ActBuf& x,
                         int32_t* status, cudaStream_t s) {
    const Dims& d = m->d;
    KernelTimer t(DSPARK_TIMER_ROWS, s, 0.0, 0.0);
    // the bf16 path reads 8 values per load: H / 8 threads (two groups each above 1024 threads)
    const bool vec = !m->embed.quant && d.dtype == DSPARK_DTYPE_BF16 && d.H % 8 == 0;
    const int threads = vec ? ((std::min(d.H / 8, 1024) + 31) / 32 * 32) : row_threads(d.H);
    if (vec && threads * kMaxPer < d.H) return cudaErrorInvalidValue;
    return launch_pdl(embed_kernel, dim3(A * d.gamma), dim3(threads), 0, s, m->embed, d.dtype, d.group, anchors,
                      d.gamma, d.mask_id, d.V, d.H, sqrtf((float)d.H), m->layers[0].in_norm, d.eps, h, x, status);
}

cudaError_t launch_qk_epilogue(const dspark_model* m, int layer, const PartView& part, int A,
                               const int32_t* block_pos, void* q, void* kb, void* vb, cudaStream_t s) {
    const Dims& d = m->d;
    KernelTimer t(DSPARK_TIMER_ROWS, s, 0.0, 0.0);
    const dim3 grid((unsigned)(A * d.gamma), (unsigned)((d.nH + d.nKv + kQkWarps - 1) / kQkWarps));
    return launch_pdl(qk_epilogue_kernel, grid, dim3(32 * kQkWarps), 0, s, part, d.gamma, d.nH, d.nKv, d.hd,
                      block_pos, m->ws.inv_freq, m->layers[layer].q_norm, m->layers[layer].k_norm, d.eps, d.dtype,
                      d.kv_dtype, q, kb, vb);
}

cudaError_t launch_o_epilogue(const dspark_model* m, int layer, const PartView& part, int M, float* h,
                              const ActBuf& x, cudaStream_t s) {
    const Dims& d = m->d;
    KernelTimer t(DSPARK_TIMER_ROWS, s, 0.0, 0.0);
    const LayerRef& L = m->layers[layer];
    return launch_residual_any(part, M, d.H, L.post_attn_norm, L.pre_ff_norm, nullptr, 0, d.eps, d.dtype, h, x, m->num_sms, s);
}

cudaError_t launch_gu_epilogue(const dspark_model* m, const PartView& part, int M, const ActBuf& act,
                               cudaStream_t s) {
    const Dims& d = m->d;
    KernelTimer t(DSPARK_TIMER_ROWS, s, 0.0, 0.0);
    const dim3 grid((unsigned)((d.I / 4 + 256 * kGuGroups - 1) / (256 * kGuGroups)), (unsigned)M);
    return launch_pdl(gu_epilogue_kernel, grid, dim3(256), 0, s, part, M, d.I, act);
}

cudaError_t launch_down_epilogue(const dspark_model* m, int layer, const PartView& part, int M, float* h,
                                 const ActBuf& x, cudaStream_t s) {
    const Dims& d = m->d;
    KernelTimer t(DSPARK_TIMER_ROWS, s, 0.0, 0.0);
    const LayerRef& L = m->layers[layer];
    const bool last = layer + 1 == d.Lyr;
    const void* next = last ? m->final_norm : m->layers[layer + 1].in_norm;
    return launch_residual_any(part, M, d.H, L.post_ff_norm, next, L.layer_scalar, 1, d.eps, d.dtype, h, x, m->num_sms, s);
}

cudaError_t launch_confidence(const dspark_model* m, const float* hf32, const int32_t* anchors, const int32_t* tokens,
                              int A, float* conf, int32_t* lengths, cudaStream_t s) {
    const Dims& d = m->d;
    KernelTimer t(DSPARK_TIMER_ROWS, s, 0.0, 0.0);
    if (d.conf_head) {
        cudaError_t e = launch_pdl(confidence_kernel, dim3(A * d.gamma), dim3(256), 0, s, hf32, m->conf_proj, d.dtype,
                                   d.group, m->w1, m->conf_bias, anchors, tokens, d.gamma, d.H, d.r,
                                   d.conf_markov ? 1 : 0, d.V, conf);
        if (e != cudaSuccess) return e;
    }
    return launch_pdl(lengths_kernel, dim3((A + 127) / 128), dim3(128), 0, s, conf, A, d.gamma, d.conf_thr,
                      d.conf_head ? 1 : 0, lengths);
}

}  // namespace dspark
