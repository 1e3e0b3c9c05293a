// Device helpers shared by the kernels: dtype conversion, block reductions,
// RoPE angles, 4-bit affine dequantization.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace dspark {

// Programmatic dependent launch: every kernel of the library is launched so
// that it may start while its predecessor in the stream is still running.
// pdl_trigger lets the next kernel start launching; pdl_wait blocks until the
// predecessor grid has completed and its memory is visible. A kernel reads
// nothing its predecessors wrote (and writes nothing they read) before
// pdl_wait; only constant data (weights) may be touched earlier. The short
// row kernels trigger at once (the GEMM after them then streams its first
// weight tiles early); the long kernels (GEMMs, attention, walk) do not
// trigger, so their consumers launch as they exit instead of waiting beside them.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Thread-block cluster: all threads of every CTA of the cluster meet (release /
// acquire), and a 32-bit shared-memory word of CTA `rank` of the cluster.
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float ld_cluster_f32(const float* local, int rank) {
    uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(local)), ra;
    float v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(ra) : "memory");
    return v;
}

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Loads element i of an array whose dtype (DSPARK_DTYPE_F32 0, BF16 1, F16 2)
// is chosen at run time.
__device__ __forceinline__ float load_any(const void* p, int64_t i, int dtype) {
    if (dtype == 0) return static_cast<const float*>(p)[i];
    if (dtype == 2) return __half2float(static_cast<const __half*>(p)[i]);
    return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
}
__device__ __forceinline__ void store_any(void* p, int64_t i, int dtype, float v) {
    if (dtype == 0) static_cast<float*>(p)[i] = v;
    else if (dtype == 2) static_cast<__half*>(p)[i] = __float2half_rn(v);
    else static_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Sum over the block; every thread gets the result. `red` holds >= 32 floats.
__device__ __forceinline__ float block_sum(float v, float* red) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
    v = warp_sum(v);
    __syncthreads();
    if (lane == 0) red[wid] = v;
    __syncthreads();
    float t = lane < nw ? red[lane] : 0.f;
    t = warp_sum(t);
    return t;
}

// (value, index) max with the lowest index on ties.
__device__ __forceinline__ void argmax_merge(float& v, int& i, float ov, int oi) {
    if (ov > v || (ov == v && oi < i)) { v = ov; i = oi; }
}
__device__ __forceinline__ void warp_argmax(float& v, int& i) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        float ov = __shfl_xor_sync(0xffffffffu, v, o);
        int oi = __shfl_xor_sync(0xffffffffu, i, o);
        argmax_merge(v, i, ov, oi);
    }
}

// RoPE angle pos * inv_freq reduced to [0, 2pi) in double, then sin/cos in fp32.
__device__ __forceinline__ void rope_sincos(int pos, double inv_freq, float* s, float* c) {
    if (inv_freq == 0.0) { *s = 0.f; *c = 1.f; return; }
    const double two_pi = 6.283185307179586476925286766559;
    const double inv_two_pi = 0.15915494309189533576888376337251;
    double a = (double)pos * inv_freq;
    a -= floor(a * inv_two_pi) * two_pi;        // within an ulp of [0, 2 pi) either way the turn count rounds
    sincosf((float)a, s, c);
}

// gelu_pytorch_tanh.
// gelu with the tanh approximation, 0.5 x (1 + tanh(u)), u = sqrt(2/pi) (x + 0.044715 x^3),
// written as x sigmoid(2u) = x / (1 + exp(-2u)) (the same function): one exponential
// and one approximate division (x / inf -> 0 for very negative x).
__device__ __forceinline__ float gelu_tanh(float x) {
    const float k2 = 2.f * 0.7978845608028654f;   // 2 sqrt(2/pi)
    const float u2 = k2 * fmaf(0.044715f * x, x * x, x);
    return __fdividef(x, 1.f + __expf(-u2));
}

// Eight consecutive weights W[n, k0 .. k0+7] of an affine 4-bit matrix
// (k0 a multiple of 8): one 32-bit word, one scale and one bias.
__device__ __forceinline__ void dequant8(const uint32_t* words, const __nv_bfloat16* scales,
                                         const __nv_bfloat16* biases, int64_t n, int64_t k0, int64_t K,
                                         int group, float out[8]) {
    const uint32_t w = words[n * (K / 8) + k0 / 8];
    const int64_t g = n * (K / group) + k0 / group;
    const float sc = __bfloat162float(scales[g]);
    const float bi = __bfloat162float(biases[g]);
#pragma unroll
    for (int j = 0; j < 8; ++j) out[j] = fmaf(sc, (float)((w >> (4 * j)) & 0xFu), bi);
}

}  // namespace dspark
