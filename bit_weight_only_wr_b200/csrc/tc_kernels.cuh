// Launch interface of the tcgen05 GEMV/GEMM kernels (internal to libwr).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace wr {

struct TcArgs {
  const uint8_t* packed;     // packed units, tile-major
  const uint16_t* scales;    // fp16 [N, K/256] (Q2/Q3), or fp16 [N] row scales d with scale_q
  const int8_t* scale_q;     // int8 [N, K/256] block multipliers (s = d q), or null: fp16 scales
  const uint16_t* alpha;     // fp16 [N] (ternary)
  float* y;                  // fp32 [M, N]
  float* partial;            // pieces of tiles cut by range ends [grid][2][TOK][128]
  int* counter;              // [RG*MT] arrival counters, zero between calls
  int* err;                  // device error word (bounded waits)
  const int* tok_ex;         // ternary: per-token exponent of the scaled R x planes (y *= 2^tok_ex)
  int M, N, K;
  int B;                     // 256-code (or 320-trit) blocks per row
  int RG;                    // 128-row groups
  int MT;                    // token tiles
  int64_t total;             // RG * MT * B (tile, block) pairs, cut into one range per CTA
};

// Batched decode GEMV (M <= 32): one launch over up to kMaxDecodeProblems independent problems.
constexpr int kMaxDecodeProblems = 256;

struct DecProblem {
  const uint16_t* x;         // bf16 [M, K] activations (read by the preparation pass)
  uint8_t* xt;               // prepared activation tiles of this problem (workspace), one per block
  const uint8_t* packed;     // packed units, tile-major
  const uint16_t* scales;    // fp16 [N, K/256] (Q2/Q3) or alpha [N] (ternary); d [N] with scale_q
  const int8_t* scale_q;     // int8 [N, K/256] block multipliers (s = d q), or null: fp16 scales
  float* y;                  // fp32 [M, N]
  const uint32_t* signs;     // ternary: random-sign mask of the rotation
  int64_t block_base;        // first block of this problem in the batch's block sequence
  int64_t cost_base;         // cost (block_cost units) of the batch's blocks before this problem
  int N, K, Kp;              // Kp: padded K (ternary: a multiple of the 320-trit unit)
  int B, RG, bits;           // blocks per row, 128-row groups, 2/3/T2 (ternary: 1)
  int xblk_base;             // first block (K unit) of this problem in the preparation pass
  int counter_base;          // first arrival counter (row group) of this problem
};

// Relative decode-GEMV time of one 128 x 256 block, by format and token count: a 3-bit (or
// trellis) block takes about 1.3 times a 2-bit one at M <= 2 and 1.2 times at M = 8 (its weights
// are 1.5 times the bytes and its decode is longer; the per-block work that does not depend on
// the format grows with M). The block ranges of the CTAs are cut by this cost so that they
// finish together; the ratios are the best of a sweep on the 36-layer body.
__host__ __device__ inline int64_t block_cost(int bits, int M) {
  return bits == 2 ? 20 : (bits == 1 ? 32 : (M <= 2 ? 26 : (M <= 4 ? 25 : 24)));
}

// The batch's blocks (problem by problem, row group by row group, K block by K block) are cut
// into gridDim.x contiguous ranges, one per CTA: CTA c takes the blocks whose cost before them
// (in block_cost units) lies in [c C / G, (c+1) C / G). A row group cut by a range boundary is
// finished through per-CTA partial slots (two per CTA: the row group that started before the
// range, and the one that ends after it). A batch is all ternary or all 2/3-bit.
constexpr int kMaxDecodeGrid = 444;   // CTAs of one decode launch, at most (3 per SM of a 148-SM part)

struct DecArgs {
  int count, M;
  int64_t total;             // blocks of the batch (T)
  int64_t total_cost;        // their summed block_cost (C)
  int32_t rs[kMaxDecodeGrid + 1];   // first block of CTA c's range (range_start, computed on the host)
  uint16_t rp[kMaxDecodeGrid];      // problem that holds that first block
  float* partial;
  int* counter;
  int* err;
  DecProblem prob[kMaxDecodeProblems];
};
static_assert(sizeof(DecArgs) <= 32764, "kernel parameter space");

// Block ranges of the 2/3-bit decode GEMV, used by the kernel (G = gridDim.x) and by the host
// planner: CTA c of G starts at cost position c C / G (block_cost units, C = total_cost), at the
// first block whose cost before it is at least that. The host sizes G so that every range holds
// at least one block (C / G is at least the largest block cost in the batch).
__host__ __device__ inline int64_t range_cost_start(const DecArgs& a, int G, int c) {
  return (int64_t)c * a.total_cost / G;
}
// First block at or after cost position cs, for a cs inside problem pr (or at its end)
__host__ __device__ inline int64_t range_start_in(const DecProblem& pr, int M, int64_t cs) {
  const int64_t w = block_cost(pr.bits, M), d = cs - pr.cost_base;
  return pr.block_base + (d > 0 ? (d + w - 1) / w : 0);
}
// First block of CTA c's range (c = G: the end of the batch)
__host__ __device__ inline int64_t range_start(const DecArgs& a, int G, int c) {
  const int64_t cs = range_cost_start(a, G, c);
  int lo = 0, hi = a.count - 1;
  while (lo < hi) {  // last problem whose first block's cost position is <= cs
    const int mid = (lo + hi + 1) >> 1;
    if (a.prob[mid].cost_base <= cs) lo = mid;
    else hi = mid - 1;
  }
  return range_start_in(a.prob[lo], a.M, cs);
}
// CTA whose range holds global block g of problem pr: the largest c with
// range_cost_start(c) <= the cost before g
__host__ __device__ inline int range_cta_of(const DecArgs& a, int G, const DecProblem& pr, int64_t g) {
  const int64_t x = pr.cost_base + (g - pr.block_base) * block_cost(pr.bits, a.M);
  return (int)(((x + 1) * G - 1) / a.total_cost);
}

// Decode GEMV: the preparation pass writes the B tiles (for a ternary batch it applies the
// rotation first), then the GEMV kernel.
cudaError_t launch_prep_x(const DecArgs& a, int total_blocks, cudaStream_t stream);
cudaError_t launch_gemv_q(const DecArgs& a, int grid, cudaStream_t stream);
// CTAs that one SM holds of the decode GEMV kernel for this kind of batch.
int decode_ctas_per_sm(bool ternary, int M, int64_t total_blocks);

// One prepared activation tile per block, stored as the exact image of a shared-memory B stage
// so that one bulk copy moves it (128-byte swizzle: 16-byte chunk c of a row r at c ^ (r % 8)):
// atoms of 128 K positions x xrows rows of int8, limb j of token slot m in row 4m + j (two atoms
// for a 256-code block, three for a 320-trit unit, the last half used), then a 256-byte
// correction record (per slot: 2/3-bit {C, f, f2, 0}; ternary {4 limb corrections}, {f, f2, 0, 0}).
// xrows = 8, 16, 32, 64 or 128 for M <= 2, 4, 8, 16, 32 (the MMA's N; the ternary form takes M
// <= 8). The record holds 16 bytes per token slot (2/3-bit) or 32 (ternary), at least 256.
constexpr int kMaxDecodeTokens = 32;          // 2/3-bit and trellis formats
constexpr int kMaxTernaryDecodeTokens = 8;
__host__ __device__ inline int decode_xrows(int M) {
  return M <= 2 ? 8 : (M <= 4 ? 16 : (M <= 8 ? 32 : (M <= 16 ? 64 : 128)));
}
__host__ __device__ inline int decode_rec_bytes(bool ternary, int M) {
  const int r = (ternary ? 32 : 16) * (decode_xrows(M) / 4);
  return r < 256 ? 256 : r;
}
__host__ __device__ inline int64_t xtile_bytes(bool ternary, int M) {
  return (int64_t)(ternary ? 3 : 2) * decode_xrows(M) * 128 + decode_rec_bytes(ternary, M);
}
// The 128-column (17..32 token) form of the 2/3-bit decode GEMV runs with one accumulator at two
// CTAs per SM when the batch holds at least 8 blocks per such CTA (the 36-layer body at M = 32:
// 1.09 -> 0.89 ms); below that, where the ranges are short and split row groups three or four
// ways, with two accumulators at one CTA per SM (a 9728 x 2560 linear at M = 32: 21.6 vs 25.0 us).
constexpr int64_t kOneAccBlocks = 8 * 2 * 148;
__host__ __device__ inline bool decode_one_acc(int M, int64_t total_blocks) {
  return decode_xrows(M) == 128 && total_blocks >= kOneAccBlocks;
}

cudaError_t launch_tc_kernel(int fmt, int bn, const TcArgs& a, const void* x_act, int64_t x_rows, int64_t x_k,
                             int grid, cudaStream_t stream);
// R x as two bf16 planes [2][M][Kp] (hi, lo) in the decoded K order, for the prefill GEMM.
// Token m is scaled by 2^-tok_ex[m] (tok_ex [M] int, written first by a per-token pass: the
// exponent of the token's largest |x|), so that tiny and huge tokens keep full precision.
cudaError_t launch_rotate_planes(const uint16_t* x, const uint32_t* signs, uint8_t* planes, int M, int K, int64_t Kp,
                                 int* tok_ex, cudaStream_t stream);
// Device quantizer + packer for the 2/3-bit odd grid (quantize.cu). scale_q null: fp16 block
// scales [N, K/256] in `scales`; else the int8 form: fp16 row scales d [N] in `scales` and the
// int8 multipliers [N, K/256] in scale_q.
cudaError_t launch_quantize_pack(int bits, const float* w, int N, int K, uint8_t* packed, uint16_t* scales,
                                 int8_t* scale_q, cudaStream_t stream);
// Failure-path self-test: a bounded wait on a barrier that never completes (see wr.h).
cudaError_t launch_selftest_wait_timeout(int* err_word, cudaStream_t stream);
// scales: fp16 [N, K/256] (alpha [N] for ternary), or the fp16 row scales d when scale_q (int8
// [N, K/256] multipliers) is not null.
cudaError_t launch_unpack_bf16(int fmt, const uint8_t* packed, const uint16_t* scales, const int8_t* scale_q, int N,
                               int K, int units, uint16_t* w, cudaStream_t stream);

}  // namespace wr
