// Plan and launch interface of the tcgen05 GEMM (gemm_tc.cu), and the view
// the row epilogues use to sum its partial tiles.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>
#include <stddef.h>

namespace dspark {
namespace tc {

constexpr int kModeTiles = 0;      // whole tiles per CTA; result written directly
constexpr int kModePartials = 1;   // stream-K; fp32 partial tiles [tile][P][BN][128]

struct GemmPlan {
    int M, N, K, np;       // out [M, N] = X [M, K] @ W [N, K]^T; np = 1 (bf16 X) or 2 (X as bf16 hi + lo)
    int BN;                // activation rows per tile (MMA N)
    int n_mt, n_nt;        // tiles along the activation rows and along the 128 weight rows
    int ksub;              // 64-wide K blocks per stage (1 or 2)
    int kb;                // stages along K: K / (64 ksub)
    int tiles;             // n_mt * n_nt; tile index t = nt * n_mt + mt
    int stages, tmem_cols;
    int acc_cols;          // TMEM columns per accumulator: 2 BN when X_hi and X_lo products share one MMA
    int mode, streamk;
    int grid;              // CTAs launched
    int T, G, P;           // stream-K: K blocks in all tiles, CTAs, most CTAs touching one tile
    // First global K block of CTA c (stream-K partition of T blocks over G CTAs).
    __host__ __device__ int range_lo(int c) const { return (int)(((int64_t)c * T) / G); }
    // The CTA whose range holds global K block g.
    __host__ __device__ int cta_of(int g) const { return (int)((((int64_t)g + 1) * G - 1) / T); }
};

GemmPlan plan_gemm(int num_sms, int M, int N, int K, int np, bool force_tiles);
// fp32 scratch elements of the stream-K partial tiles (0 in tile mode).
size_t gemm_partial_elems(const GemmPlan& p);
size_t gemm_smem_bytes(const GemmPlan& p);
// W: bf16 [w_rows >= N, K]; X0 (and X1 when np == 2): bf16 [M, K].
// Writes the fp32 result out[m * ldo + n] for m < M, n < N, with the softcap
// cap * tanh(v / cap) when cap > 0, in tile mode. A stream-K plan writes
// its partial tiles to `part` (gemm_partial_elems floats) instead, and the
// consumer sums them (PartView mode 1); `out` is then untouched.
cudaError_t launch_gemm_tc(const GemmPlan& p, const void* W, int64_t w_rows, const void* X0, const void* X1,
                           float* out, int64_t ldo, float cap, float* part, int32_t* status, cudaStream_t s);

}  // namespace tc
}  // namespace dspark
