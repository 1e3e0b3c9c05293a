// Plan and launch interface of the tcgen05 GEMM (gemm_tc.cu), and the view
// the row epilogues use to sum its partial tiles.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stddef.h>

namespace dspark {
struct TileStats;
namespace tc {

constexpr int kModeTiles = 0;      // whole tiles per CTA; result written directly
constexpr int kModePartials = 1;   // stream-K; fp32 partial tiles [tile][P][BN][128] ([tile][2][P][BN][128] for pairs)

// Weight formats (and MMA operand types) of the GEMM:
constexpr int kWBf16 = 0;       // bf16 weights straight from TMA; bf16 activation (the caller's context rows)
constexpr int kWF16 = 1;        // fp16 weights (the model's fp16 copy) straight from TMA; fp16 activation,
                                // one part or an fp16 pair hi + lo
constexpr int kWQ4AsF16 = 2;    // packed 4-bit weights dequantized to fp16 in shared memory; fp16 activation
// A packed 4-bit block: 128 weight rows x 64 K (one group): words [128][8] uint32,
// then scales [128] and biases [128] bf16; a matrix's blocks are [128-row tile][K block].
constexpr int kQ4BlockBytes = 128 * 32 + 128 * 2 * 2;
__host__ __device__ constexpr int q4_raw_bytes(int ksub) { return (ksub * kQ4BlockBytes + 1023) / 1024 * 1024; }
// Bytes of the packed copy of an [n, k] matrix.
inline size_t q4_packed_bytes(int64_t n, int64_t k) { return (size_t)((n + 127) / 128) * (size_t)(k / 64) * kQ4BlockBytes; }

struct GemmPlan {
    int M, N, K, np;       // out [M, N] = X [M, K] @ W [N, K]^T; np = 1 (bf16 X) or 2 (X as bf16 hi + lo)
    int wfmt;              // weight format (kW*)
    int stats;             // tile mode: shared memory reserved for the epilogue's logit statistics
    int BN;                // activation rows per tile (MMA N)
    int n_mt, n_nt;        // tiles along the activation rows and along the weight rows (128, or 256 for pairs)
    int ksub;              // 64-wide K blocks per stage (1 or 2)
    int kb;                // stages along K: K / (64 ksub)
    int tiles;             // n_mt * n_nt; tile index t = nt * n_mt + mt
    int stages, tmem_cols;
    int acc_cols;          // TMEM columns per accumulator: 2 BN when X_hi and X_lo products share one MMA
    int mode, streamk;
    int pair;              // CTA pairs (cta_group::2): a work unit is a 256-row weight tile on two CTAs
    int units;             // work units: CTAs, or CTA pairs (grid = 2 units)
    int grid;              // CTAs launched
    int T, G, P;           // stream-K: K blocks in all tiles, work units, most units touching one tile
    // First global K block of CTA c (stream-K partition of T blocks over G CTAs).
    __host__ __device__ int range_lo(int c) const { return (int)(((int64_t)c * T) / G); }
    // The CTA whose range holds global K block g.
    __host__ __device__ int cta_of(int g) const { return (int)((((int64_t)g + 1) * G - 1) / T); }
};

GemmPlan plan_gemm(int num_sms, int M, int N, int K, int np, bool force_tiles, bool stats = false,
                   int wfmt = kWBf16);
// fp32 scratch elements of the stream-K partial tiles (0 in tile mode).
size_t gemm_partial_elems(const GemmPlan& p);
size_t gemm_smem_bytes(const GemmPlan& p);
// W: 16-bit [w_rows >= N, K] (bf16 for kWBf16, fp16 for kWF16), or the packed 4-bit
// copy of the matrix (kWQ4*: q4_pack); X0 (and X1 when np == 2): 16-bit [M, K]
// (fp16 for the fp16 formats).
// Writes the fp32 result out[m * ldo + n] for m < M, n < N, with the softcap
// cap * tanh(v / cap) when cap > 0, in tile mode. A stream-K plan writes
// its partial tiles to `part` (gemm_partial_elems floats) instead, and the
// consumer sums them (PartView mode 1); `out` is then untouched.
// With `stats` (tile mode, a plan made with stats = true) the epilogue also
// writes the per-(128-row weight tile, activation row) logit statistics of
// logit_stats.cuh, with the Markov bounds when w2norm is non-NULL.
cudaError_t launch_gemm_tc(const GemmPlan& p, const void* W, int64_t w_rows, const void* X0, const void* X1,
                           float* out, int64_t ldo, float cap, float* part, int32_t* status, cudaStream_t s,
                           const TileStats* stats = nullptr, const float* w2norm = nullptr,
                           const uint32_t* w1max_bits = nullptr);

// One source of a packed copy: rows [row0, row0 + rows) of the destination are the
// rows of an MLX 4-bit matrix (words [rows, k/8], scales / biases [rows, k/64]).
struct Q4Piece {
    const uint32_t* w;
    const __nv_bfloat16* s;
    const __nv_bfloat16* b;
    int64_t row0, rows;
};
constexpr int kMaxQ4Pieces = 64;
// Converts n bf16 values to fp16 (exact inside fp16's range); ORs `bits` into
// *overflow when a value lies outside it (or is not finite).
cudaError_t f16_copy(const void* src, int64_t n, void* dst, int32_t* overflow, cudaStream_t s, int32_t bits = 1);
// Writes the packed 4-bit copy (q4_packed_bytes(n, k) bytes at `dst`) of an [n, k]
// matrix stacked from `pieces` (rows not covered are zero); group size 64.
cudaError_t q4_pack(const Q4Piece* pieces, int npieces, int64_t n, int64_t k, void* dst, cudaStream_t s);

}  // namespace tc
}  // namespace dspark
