// CUDA-core GEMM  out = X @ W^T  with fp32 FFMA accumulation.
//
// This is the contraction of deepspec.ts `matmulW` (x @ W^T for a Linear
// weight stored [out, in]; quantized weights dequantize on load, MLX
// QuantizedLinear semantics). It is the path of the fp32 workload, whose
// 1e-4 relative bar rules out TF32 tensor cores, and of any shape the
// tcgen05 GEMM does not take.
//
// Tiles: 64 X-rows x 64 W-rows x 32 k per step, 256 threads, 4x4 outputs per
// thread. Split-K over grid.z writes fp32 partials out[z][m][n]; a row
// epilogue sums the splits in order (deterministic, no atomics).
#include "internal.h"
#include "common.cuh"

namespace dspark {
namespace {

constexpr int BM = 64, BN = 64, BK = 32;

template <typename T>
__device__ __forceinline__ void load8(const T* p, float out[8]);
template <>
__device__ __forceinline__ void load8<float>(const float* p, float out[8]) {
    const float4 a = reinterpret_cast<const float4*>(p)[0];
    const float4 b = reinterpret_cast<const float4*>(p)[1];
    out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
    out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
}
template <>
__device__ __forceinline__ void load8<bf16>(const bf16* p, float out[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        out[2 * j] = __uint_as_float(w[j] << 16);
        out[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
    }
}

template <typename TX, typename TW, bool QUANT>
__global__ void __launch_bounds__(256)
simt_gemm_kernel(const TX* __restrict__ X, int64_t ldx, const void* __restrict__ Wv,
                 const bf16* __restrict__ scales, const bf16* __restrict__ biases, int group,
                 int M, int N, int K, int k_per_split, float* __restrict__ out, int64_t ldo,
                 int64_t split_stride, int softcap, float cap) {
    __shared__ float Xs[BK][BM + 4];
    __shared__ float Ws[BK][BN + 4];
    pdl_trigger();
    pdl_wait();
    const int tid = threadIdx.x;
    const int tx = tid & 15, ty = tid >> 4;
    const int n0 = blockIdx.x * BN, m0 = blockIdx.y * BM;
    const int kb = blockIdx.z * k_per_split;
    const int ke = min(K, kb + k_per_split);

    // loader coordinates: 64 rows x 4 groups of 8 k
    const int lrow = tid >> 2, lk = (tid & 3) * 8;

    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

    for (int k0 = kb; k0 < ke; k0 += BK) {
        float xv[8], wv[8];
        const int k = k0 + lk;
        const int m = m0 + lrow, n = n0 + lrow;
        if (m < M && k < ke) load8<TX>(X + (int64_t)m * ldx + k, xv);
        else {
#pragma unroll
            for (int j = 0; j < 8; ++j) xv[j] = 0.f;
        }
        if (n < N && k < ke) {
            if constexpr (QUANT) dequant8(static_cast<const uint32_t*>(Wv), scales, biases, n, k, K, group, wv);
            else load8<TW>(static_cast<const TW*>(Wv) + (int64_t)n * K + k, wv);
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) wv[j] = 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            Xs[lk + j][lrow] = xv[j];
            Ws[lk + j][lrow] = wv[j];
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < BK; ++kk) {
            const float4 a = *reinterpret_cast<const float4*>(&Xs[kk][ty * 4]);
            const float4 b = *reinterpret_cast<const float4*>(&Ws[kk][tx * 4]);
            const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
    }

    float* o = out + (int64_t)blockIdx.z * split_stride;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + ty * 4 + i;
        if (m >= M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx * 4 + j;
            if (n >= N) continue;
            float v = acc[i][j];
            if (softcap && cap > 0.f) v = cap * tanhf(v / cap);
            o[(int64_t)m * ldo + n] = v;
        }
    }
}

}  // namespace

cudaError_t launch_simt_gemm(const void* X, int64_t ldx, int x_dtype, int w_dtype, const MatRef& W, int group,
                             int M, int N, int K, int splits, float* out, int64_t ldo, int64_t split_stride,
                             bool softcap, float cap, cudaStream_t s) {
    if (M <= 0 || N <= 0) return cudaSuccess;
    int kps = (K + splits - 1) / splits;
    kps = (kps + BK - 1) / BK * BK;
    const int z = (K + kps - 1) / kps;
    dim3 grid((N + BN - 1) / BN, (M + BM - 1) / BM, z);
#define DSPARK_SIMT_LAUNCH(TX, TW, Q)                                                                     \
    e = launch_pdl(simt_gemm_kernel<TX, TW, Q>, grid, dim3(256), 0, s, static_cast<const TX*>(X), ldx, W.w,   \
                   W.scales, W.biases, group, M, N, K, kps, out, ldo, split_stride, (int)softcap, cap)
    const bool xf = x_dtype == DSPARK_DTYPE_F32;
    cudaError_t e;
    if (W.quant) {
        if (xf) DSPARK_SIMT_LAUNCH(float, bf16, true); else DSPARK_SIMT_LAUNCH(bf16, bf16, true);
    } else if (w_dtype == DSPARK_DTYPE_F32) {
        if (xf) DSPARK_SIMT_LAUNCH(float, float, false); else DSPARK_SIMT_LAUNCH(bf16, float, false);
    } else {
        if (xf) DSPARK_SIMT_LAUNCH(float, bf16, false); else DSPARK_SIMT_LAUNCH(bf16, bf16, false);
    }
#undef DSPARK_SIMT_LAUNCH
    return e;
}

}  // namespace dspark
