// C ABI of libwr: argument checks, workspace layout and launch configuration.
//
// Every entry point validates its arguments on the host and returns before any launch when
// they are wrong; device work is enqueued on the caller's stream and never synchronized.
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cstdint>
#include <mutex>

#include "tc_kernels.cuh"
#include "wr.h"
#include "wr_internal.h"

namespace {

constexpr int64_t kMaxDim = (int64_t)1 << 30;

__device__ int g_device_error = 0;

inline bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

int* device_error_word() {
  static std::mutex mu;
  static int* cache[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) == cudaSuccess) cache[dev] = static_cast<int*>(p);
  }
  return cache[dev];
}

wr_status check_dims(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || N < 1 || K < 1 || M > kMaxDim || N > kMaxDim || K > kMaxDim) return WR_ERR_INVALID_ARG;
  if ((double)N * (double)K > 9.0e15) return WR_ERR_INVALID_ARG;
  return WR_OK;
}

// The format argument of the 2/3-bit calls: a base format, optionally | WR_SCALES_I8.
struct QFmt {
  int base;
  bool s8;
};
inline bool split_fmt(int fmt, bool allow_t2, QFmt* f) {
  f->s8 = (fmt & WR_SCALES_I8) != 0;
  f->base = fmt & ~WR_SCALES_I8;
  return f->base == WR_FMT_Q2 || f->base == WR_FMT_Q3 || (allow_t2 && (f->base == WR_FMT_T2 || f->base == WR_FMT_T8));
}
// The int8 multipliers of an int8 scale record (null for fp16 scales).
inline const int8_t* scale_q_of(const QFmt& f, const uint16_t* scales, int64_t N) {
  return f.s8 ? reinterpret_cast<const int8_t*>(reinterpret_cast<const uint8_t*>(scales) + wr::s8_q_offset(N))
              : nullptr;
}

constexpr int kPlanSMs = 148;   // split heuristics are sized for a 148-SM part (device-independent)
// Token counts the integer decode kernel takes (4 activation limbs per token: up to 128 MMA
// columns for the 2/3-bit formats, 32 for ternary); larger M goes to the tensor-core GEMM.
constexpr int kDecodeTokens = wr::kMaxDecodeTokens;
constexpr int kTernaryDecodeTokens = wr::kMaxTernaryDecodeTokens;

// ---- decode kernel (M <= 32; ternary M <= 8) and workspace [counters: one int per row group of every problem]
// [partials][prepared activation tiles: one per block of every problem]. The batch's blocks are
// cut into one contiguous range of equal cost per CTA, and the partials are two 128-row slots per
// CTA for the row groups that several ranges share. A batch is all 2/3-bit or all ternary.
struct DecodePlan {
  wr::DecArgs args;
  int total_blocks = 0;   // K blocks of all problems (work of the preparation pass, per token slot)
  int grid = 0;           // CTAs (block ranges) of the decode launch
  size_t counter_off = 0, partial_off = 0, xt_off = 0, total = 0;
  int64_t xt_rel[wr::kMaxDecodeProblems];
};

struct ProblemShape {
  int64_t N, K;
  int fmt;
};

void plan_decode(int64_t M, int count, const ProblemShape* shapes, DecodePlan* dp) {
  wr::DecArgs& a = dp->args;
  a.count = count;
  a.M = (int)M;
  const bool ternary = count > 0 && shapes[0].fmt == WR_FMT_TERNARY;
  int counters = 0, blocks = 0;
  int64_t xt_bytes = 0, block_base = 0, cost_base = 0, max_cost = 1;
  for (int i = 0; i < count; ++i) {
    int64_t ub = 0, units = 0, tiles = 0;
    wr::packed_geometry(shapes[i].fmt, shapes[i].N, shapes[i].K, &ub, &units, &tiles);
    wr::DecProblem& pr = a.prob[i];
    pr = wr::DecProblem{};
    pr.N = (int)shapes[i].N;
    pr.K = (int)shapes[i].K;
    pr.B = (int)units;
    pr.Kp = ternary ? (int)(units * 320) : (int)shapes[i].K;
    pr.RG = (int)((shapes[i].N + 127) / 128);
    pr.bits = ternary ? 1 : shapes[i].fmt;
    pr.counter_base = counters;
    pr.xblk_base = blocks;
    pr.block_base = block_base;
    pr.cost_base = cost_base;
    counters += pr.RG;
    blocks += pr.B;
    block_base += (int64_t)pr.RG * pr.B;
    cost_base += (int64_t)pr.RG * pr.B * wr::block_cost(pr.bits, (int)M);
    max_cost = std::max(max_cost, wr::block_cost(pr.bits, (int)M));
    dp->xt_rel[i] = xt_bytes;
    xt_bytes += (int64_t)pr.B * wr::xtile_bytes(ternary, (int)M);
  }
  a.total = block_base;
  a.total_cost = cost_base;
  // ranges of at least the largest block cost in the batch, so that each holds a block (one
  // block per CTA for a small single-format batch), at most one wave of CTAs; two partial slots
  // per CTA of the launch (see DecArgs)
  const int64_t wave = (int64_t)wr::decode_ctas_per_sm(ternary, (int)M, block_base) * kPlanSMs;
  dp->grid = (int)std::max<int64_t>(1, std::min<int64_t>(wave, cost_base / max_cost));
  // each CTA's first block and the problem that holds it
  for (int c = 0, pi = 0; c <= dp->grid; ++c) {
    const int64_t g = wr::range_start(a, dp->grid, c);
    a.rs[c] = (int32_t)g;
    if (c == dp->grid) break;
    while (pi + 1 < count && a.prob[pi + 1].block_base <= g) ++pi;
    a.rp[c] = (uint16_t)pi;
  }
  const int64_t partials = 2 * (int64_t)dp->grid * M * 128;
  dp->total_blocks = blocks;
  dp->counter_off = 0;
  dp->partial_off = align256((size_t)counters * sizeof(int));
  dp->xt_off = dp->partial_off + align256((size_t)partials * sizeof(float));
  dp->total = dp->xt_off + align256((size_t)xt_bytes);
}

// Fills the workspace pointers of a plan (the activation tiles of problem i start at
// xt_off + xt_rel[i]).
void bind_workspace(DecodePlan& dp, void* workspace) {
  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  dp.args.counter = reinterpret_cast<int*>(wsb + dp.counter_off);
  dp.args.partial = reinterpret_cast<float*>(wsb + dp.partial_off);
  for (int i = 0; i < dp.args.count; ++i) dp.args.prob[i].xt = wsb + dp.xt_off + dp.xt_rel[i];
  dp.args.err = device_error_word();
}

// The preparation pass (for ternary, with the rotation), then the decode kernel over one
// contiguous block range per CTA (the partial slots were sized for this grid).
//
// Problems that read the same activations (same x pointer and K; for ternary the same sign mask)
// through the same tile layout (Q2, Q3, T2 and ternary order and scale K positions differently)
// share one set of prepared tiles: the preparation pass writes it once, for the first of them
// (looked up among the last few distinct sets, which is where q/k/v or gate/up sit in a batch).
wr_status run_decode(DecodePlan& dp, cudaStream_t stream) {
  if (dp.args.total > INT32_MAX) return WR_ERR_INVALID_ARG;   // block indices are 32-bit in the kernel
  static thread_local wr::DecArgs prep;
  wr::DecArgs& a = dp.args;
  prep.count = 0;
  prep.M = a.M;
  int blocks = 0;
  constexpr int kLook = 8;
  for (int i = 0; i < a.count; ++i) {
    wr::DecProblem& pi = a.prob[i];
    int owner = -1;
    for (int j = prep.count - 1; j >= 0 && j >= prep.count - kLook; --j) {
      const wr::DecProblem& pj = prep.prob[j];
      if (pj.x == pi.x && pj.K == pi.K && pj.bits == pi.bits && pj.signs == pi.signs) {
        owner = j;
        break;
      }
    }
    if (owner >= 0) {
      pi.xt = prep.prob[owner].xt;
    } else {
      prep.prob[prep.count] = pi;
      prep.prob[prep.count].xblk_base = blocks;
      blocks += pi.B;
      ++prep.count;
    }
  }
  if (wr::launch_prep_x(prep, blocks, stream) != cudaSuccess) return WR_ERR_CUDA;
  return wr::launch_gemv_q(a, dp.grid, stream) == cudaSuccess ? WR_OK : WR_ERR_CUDA;
}

// ---- prefill GEMM kernel (M > 32; ternary M > 8): 128-row groups x token tiles x K blocks, cut "stream-K" into
// one contiguous range of (tile, block) pairs per CTA; workspace [counters: one int per tile]
// [two partial tiles per CTA, for the pieces of tiles cut by range ends].
struct GemmPlan {
  int B = 0, RG = 0, MT = 0, grid = 0;
  int64_t total = 0, Kp = 0;
  size_t counter_off = 0, partial_off = 0, planes_off = 0, tokex_off = 0, total_bytes = 0;
};

// tok: tokens per tile (128; 64 for ternary, whose R x hi and lo planes fill 128 MMA columns);
// unit_k: K per block (256; 320 trits for ternary).
GemmPlan plan_gemm(int64_t M, int64_t N, int64_t K, int tok, int unit_k) {
  GemmPlan p;
  p.B = (int)((K + unit_k - 1) / unit_k);
  p.Kp = (int64_t)p.B * unit_k;
  p.RG = (int)((N + 127) / 128);
  p.MT = (int)((M + tok - 1) / tok);
  p.total = (int64_t)p.RG * p.MT * p.B;
  p.grid = (int)std::min<int64_t>(p.total, kPlanSMs);
  p.counter_off = 0;
  p.partial_off = align256((size_t)p.RG * p.MT * sizeof(int));
  p.planes_off = p.partial_off + align256((size_t)p.grid * 2 * tok * 128 * sizeof(float));
  p.total_bytes = p.planes_off;
  return p;
}

wr::TcArgs gemm_args(const GemmPlan& p, int64_t M, int64_t N, int64_t K, void* workspace) {
  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  wr::TcArgs a{};
  a.partial = reinterpret_cast<float*>(wsb + p.partial_off);
  a.counter = reinterpret_cast<int*>(wsb + p.counter_off);
  a.err = device_error_word();
  a.M = (int)M;
  a.N = (int)N;
  a.K = (int)K;
  a.B = p.B;
  a.RG = p.RG;
  a.MT = p.MT;
  a.total = p.total;
  return a;
}

wr_status run_gemm(int bits, int M, int N, int K, const uint16_t* x, const uint8_t* packed, const uint16_t* scales,
                   const int8_t* scale_q, float* y, void* workspace, cudaStream_t stream) {
  const GemmPlan p = plan_gemm(M, N, K, 128, 256);
  wr::TcArgs a = gemm_args(p, M, N, K, workspace);
  a.packed = packed;
  a.scales = scales;
  a.scale_q = scale_q;
  a.y = y;
  return wr::launch_tc_kernel(bits, 128, a, x, M, K, p.grid, stream) == cudaSuccess ? WR_OK : WR_ERR_CUDA;
}

// Which kernel a 2/3-bit call of M tokens runs. wr_gemv always takes the integer decode kernel
// (M <= 32). wr_gemm takes it for M <= 8, and for M <= 32 when K <= 4096: there a row group has
// few K blocks and the decode kernel measured faster than the tensor-core GEMM (gate 2560 -> 9728:
// 17.8-21.8 against 24.5-28.2 us at M = 9..32); for long K (down 9728 -> 2560) the GEMM is faster
// at M <= 16, since four int8 limbs per token make the activation tile twice the weights' bytes
// and a long row group is split over many CTAs.
bool decode_route(bool gemm, int64_t M, int64_t K) {
  if (!gemm) return M <= kDecodeTokens;
  return M <= 8 || (M <= kDecodeTokens && K <= 4096);
}

// One Q2/Q3 call of any M.
size_t q_workspace(int bits, int64_t M, int64_t N, int64_t K, bool gemm) {
  if (decode_route(gemm, M, K)) {
    static thread_local DecodePlan dp;
    const ProblemShape sh{N, K, bits};
    plan_decode(M, 1, &sh, &dp);
    return dp.total;
  }
  return plan_gemm(M, N, K, 128, 256).total_bytes;
}

wr_status run_q(int bits, int64_t M, int64_t N, int64_t K, const uint16_t* x, const void* packed,
                const uint16_t* scales, const int8_t* scale_q, float* y, void* workspace, cudaStream_t stream,
                bool gemm) {
  if (decode_route(gemm, M, K)) {
    static thread_local DecodePlan dp;
    const ProblemShape sh{N, K, bits};
    plan_decode(M, 1, &sh, &dp);
    dp.args.prob[0].x = x;
    dp.args.prob[0].packed = static_cast<const uint8_t*>(packed);
    dp.args.prob[0].scales = scales;
    dp.args.prob[0].scale_q = scale_q;
    dp.args.prob[0].y = y;
    bind_workspace(dp, workspace);
    return run_decode(dp, stream);
  }
  return run_gemm(bits, (int)M, (int)N, (int)K, x, static_cast<const uint8_t*>(packed), scales, scale_q, y, workspace,
                  stream);
}

// Ternary. M <= 8: the decode kernel (its preparation pass applies the rotation). M > 8: the
// prefill GEMM over 64-token tiles (the hi and lo planes of R x make the 128 MMA columns); its
// workspace adds the R x planes [2][M][Kp] bf16 and the per-token exponents after the GEMM's own.
constexpr int kTernaryTok = 64;   // tokens per GEMM tile

GemmPlan plan_gemm_t(int64_t M, int64_t N, int64_t K) {
  GemmPlan p = plan_gemm(M, N, K, kTernaryTok, 320);
  p.tokex_off = p.planes_off + align256((size_t)2 * M * p.Kp * sizeof(uint16_t));
  p.total_bytes = p.tokex_off + align256((size_t)M * sizeof(int));
  return p;
}

size_t t_workspace(int64_t M, int64_t N, int64_t K) {
  if (M > kTernaryDecodeTokens) return plan_gemm_t(M, N, K).total_bytes;
  static thread_local DecodePlan dp;
  const ProblemShape sh{N, K, WR_FMT_TERNARY};
  plan_decode(M, 1, &sh, &dp);
  return dp.total;
}

wr_status run_t(int64_t M, int64_t N, int64_t K, const uint16_t* x, const void* packed, const uint16_t* alpha,
                const uint32_t* signs, float* y, void* workspace, cudaStream_t stream) {
  if (M <= kTernaryDecodeTokens) {
    static thread_local DecodePlan dp;
    const ProblemShape sh{N, K, WR_FMT_TERNARY};
    plan_decode(M, 1, &sh, &dp);
    bind_workspace(dp, workspace);
    dp.args.prob[0].x = x;
    dp.args.prob[0].signs = signs;
    dp.args.prob[0].packed = static_cast<const uint8_t*>(packed);
    dp.args.prob[0].scales = alpha;
    dp.args.prob[0].y = y;
    return run_decode(dp, stream);
  }
  const GemmPlan p = plan_gemm_t(M, N, K);
  uint8_t* planes = static_cast<uint8_t*>(workspace) + p.planes_off;
  int* tok_ex = reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) + p.tokex_off);
  if (wr::launch_rotate_planes(x, signs, planes, (int)M, (int)K, p.Kp, tok_ex, stream) != cudaSuccess)
    return WR_ERR_CUDA;
  wr::TcArgs a = gemm_args(p, M, N, K, workspace);
  a.tok_ex = tok_ex;
  a.packed = static_cast<const uint8_t*>(packed);
  a.alpha = alpha;
  a.y = y;
  return wr::launch_tc_kernel(WR_FMT_TERNARY, 128, a, planes, M, p.Kp, p.grid, stream) == cudaSuccess ? WR_OK
                                                                                                  : WR_ERR_CUDA;
}

}  // namespace

// Scratch of wr_gemv_noalloc: a fixed device array (one per device, zero at module load), so
// that the entry point needs no allocation and no workspace argument.
static __device__ __align__(256) uint8_t g_noalloc_scratch[WR_GEMV_NOALLOC_SCRATCH_BYTES];

namespace {

// Device address of the current device's scratch array. Looked up once per device, with that
// device current (the one-time set-up, which may load the module: keep it outside stream
// capture); later calls read the cached pointer.
void* noalloc_scratch(wr_status* st) {
  static std::mutex mu;
  static void* cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    *st = WR_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      *st = WR_ERR_CUDA;
      return nullptr;
    }
    cache[dev] = p;
  }
  return cache[dev];
}

}  // namespace

extern "C" {

int wr_abi_version(void) { return 1; }

const char* wr_status_string(wr_status st) {
  switch (st) {
    case WR_OK: return "ok";
    case WR_ERR_INVALID_ARG: return "invalid argument";
    case WR_ERR_UNSUPPORTED: return "unsupported configuration";
    case WR_ERR_CUDA: return "CUDA error";
    case WR_ERR_TIMEOUT: return "device-side wait timed out";
    case WR_ERR_TOO_LARGE: return "problem needs more than the fixed scratch of wr_gemv_noalloc";
  }
  return "unknown status";
}

wr_status wr_unpack_bf16(int fmt, int64_t N, int64_t K, const void* packed, const uint16_t* scales,
                         int group, uint16_t* w_bf16, void* stream) {
  QFmt f{};
  if (!split_fmt(fmt, true, &f) && fmt != WR_FMT_TERNARY) return WR_ERR_UNSUPPORTED;
  if (fmt == WR_FMT_TERNARY) f = QFmt{WR_FMT_TERNARY, false};
  fmt = f.base;
  if (check_dims(1, N, K) != WR_OK) return WR_ERR_INVALID_ARG;
  if (fmt != WR_FMT_TERNARY && group != 256) return WR_ERR_UNSUPPORTED;
  int64_t ub = 0, units = 0, tiles = 0;
  if (!wr::packed_geometry(fmt, N, K, &ub, &units, &tiles)) return WR_ERR_INVALID_ARG;
  if (!aligned16(packed) || !aligned16(scales) || !aligned16(w_bf16)) return WR_ERR_INVALID_ARG;
  const cudaError_t e = wr::launch_unpack_bf16(fmt, static_cast<const uint8_t*>(packed), scales,
                                               scale_q_of(f, scales, N), (int)N, (int)K, (int)units, w_bf16,
                                               static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? WR_OK : WR_ERR_CUDA;
}

size_t wr_gemv_workspace_bytes(int64_t M, int64_t N, int64_t K, int bits) {
  QFmt f{};
  if (!split_fmt(bits, true, &f)) return 0;
  if (M < 1 || M > kDecodeTokens || check_dims(M, N, K) != WR_OK || K % 256 != 0) return 0;
  return q_workspace(f.base, M, N, K, false);
}

wr_status wr_gemv(int64_t M, int64_t N, int64_t K, const uint16_t* x, const void* packed,
                  const uint16_t* scales, int bits, int group, float* y, void* workspace,
                  size_t workspace_bytes, void* stream) {
  QFmt f{};
  if (!split_fmt(bits, true, &f)) return WR_ERR_UNSUPPORTED;
  if (group != 256) return WR_ERR_UNSUPPORTED;
  if (M < 1 || M > kDecodeTokens || check_dims(M, N, K) != WR_OK || K % 256 != 0) return WR_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(packed) || !aligned16(scales) || !aligned16(y) || !aligned16(workspace))
    return WR_ERR_INVALID_ARG;
  if (workspace_bytes < q_workspace(f.base, M, N, K, false)) return WR_ERR_INVALID_ARG;
  return run_q(f.base, M, N, K, x, packed, scales, scale_q_of(f, scales, N), y, workspace,
               static_cast<cudaStream_t>(stream), false);
}

wr_status wr_gemv_noalloc(int64_t M, int64_t N, int64_t K, const uint16_t* x, const void* packed,
                          const uint16_t* scales, int bits, int group, float* y, void* stream) {
  QFmt f{};
  if (!split_fmt(bits, true, &f)) return WR_ERR_UNSUPPORTED;
  bits = f.base;
  if (group != 256) return WR_ERR_UNSUPPORTED;
  if (M < 1 || M > kDecodeTokens || check_dims(M, N, K) != WR_OK || K % 256 != 0) return WR_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(packed) || !aligned16(scales) || !aligned16(y)) return WR_ERR_INVALID_ARG;
  const int8_t* scale_q = scale_q_of(f, scales, N);
  if (q_workspace(bits, M, N, K, false) > WR_GEMV_NOALLOC_SCRATCH_BYTES) return WR_ERR_TOO_LARGE;
  wr_status st = WR_OK;
  void* scratch = noalloc_scratch(&st);
  if (scratch == nullptr) return st;
  // the arrival counters (the first bytes of the plan) must start at zero
  static thread_local DecodePlan dp;
  const ProblemShape sh{N, K, bits};
  plan_decode(M, 1, &sh, &dp);
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dp.partial_off > 0 && cudaMemsetAsync(scratch, 0, dp.partial_off, s) != cudaSuccess) return WR_ERR_CUDA;
  return run_q(bits, M, N, K, x, packed, scales, scale_q, y, scratch, s, false);
}

// Shape and format of one batched problem (what the plan reads); the batched call also checks
// its pointers.
static wr_status problem_shape_ok(int64_t M, const wr_gemv_problem& pr) {
  QFmt f{};
  if (!split_fmt(pr.bits, true, &f)) return WR_ERR_UNSUPPORTED;
  if (pr.reserved != 0 || check_dims(M, pr.N, pr.K) != WR_OK || pr.K % 256 != 0) return WR_ERR_INVALID_ARG;
  return WR_OK;
}

static bool batch_ok(int64_t M, int32_t count, const wr_gemv_problem* pr) {
  if (M < 1 || M > kDecodeTokens || count < 1 || !pr) return false;
  for (int i = 0; i < count; ++i) {
    if (problem_shape_ok(M, pr[i]) != WR_OK) return false;
    if (!aligned16(pr[i].x) || !aligned16(pr[i].packed) || !aligned16(pr[i].scales) || !aligned16(pr[i].y))
      return false;
  }
  return true;
}

wr_status wr_gemv_batched_plan(int64_t M, int32_t count, const wr_gemv_problem* problems, int32_t* grid,
                               int64_t* range_starts, int32_t range_starts_len, int64_t* block_costs) {
  if (M < 1 || M > kDecodeTokens || count < 1 || count > wr::kMaxDecodeProblems || !problems || !grid)
    return WR_ERR_INVALID_ARG;
  ProblemShape sh[wr::kMaxDecodeProblems];
  for (int i = 0; i < count; ++i) {
    const wr_status st = problem_shape_ok(M, problems[i]);
    if (st != WR_OK) return st;
    sh[i] = ProblemShape{problems[i].N, problems[i].K, problems[i].bits & ~WR_SCALES_I8};
  }
  static thread_local DecodePlan dp;
  plan_decode(M, count, sh, &dp);
  *grid = dp.grid;
  if (range_starts) {
    if (range_starts_len < dp.grid + 1) return WR_ERR_INVALID_ARG;
    for (int c = 0; c <= dp.grid; ++c) range_starts[c] = wr::range_start(dp.args, dp.grid, c);
  }
  if (block_costs)
    for (int i = 0; i < count; ++i) block_costs[i] = wr::block_cost(dp.args.prob[i].bits, (int)M);
  return WR_OK;
}

size_t wr_gemv_batched_workspace_bytes(int64_t M, int32_t count, const wr_gemv_problem* problems) {
  if (!batch_ok(M, count, problems)) return 0;
  size_t total = 0;
  static thread_local DecodePlan dp;
  ProblemShape sh[wr::kMaxDecodeProblems];
  for (int c0 = 0; c0 < count; c0 += wr::kMaxDecodeProblems) {
    const int n = std::min(count - c0, wr::kMaxDecodeProblems);
    for (int i = 0; i < n; ++i)
      sh[i] = ProblemShape{problems[c0 + i].N, problems[c0 + i].K, problems[c0 + i].bits & ~WR_SCALES_I8};
    plan_decode(M, n, sh, &dp);
    total = std::max(total, dp.total);
  }
  return total;
}

wr_status wr_gemv_batched(int64_t M, int32_t count, const wr_gemv_problem* problems, void* workspace,
                          size_t workspace_bytes, void* stream) {
  if (!batch_ok(M, count, problems) || !aligned16(workspace)) return WR_ERR_INVALID_ARG;
  if (workspace_bytes < wr_gemv_batched_workspace_bytes(M, count, problems)) return WR_ERR_INVALID_ARG;
  static thread_local DecodePlan dp;
  ProblemShape sh[wr::kMaxDecodeProblems];
  for (int c0 = 0; c0 < count; c0 += wr::kMaxDecodeProblems) {
    const int n = std::min(count - c0, wr::kMaxDecodeProblems);
    for (int i = 0; i < n; ++i)
      sh[i] = ProblemShape{problems[c0 + i].N, problems[c0 + i].K, problems[c0 + i].bits & ~WR_SCALES_I8};
    plan_decode(M, n, sh, &dp);
    for (int i = 0; i < n; ++i) {
      const wr_gemv_problem& pi = problems[c0 + i];
      QFmt f{};
      split_fmt(pi.bits, true, &f);
      dp.args.prob[i].x = pi.x;
      dp.args.prob[i].packed = static_cast<const uint8_t*>(pi.packed);
      dp.args.prob[i].scales = pi.scales;
      dp.args.prob[i].scale_q = scale_q_of(f, pi.scales, pi.N);
      dp.args.prob[i].y = problems[c0 + i].y;
    }
    bind_workspace(dp, workspace);
    const wr_status st = run_decode(dp, static_cast<cudaStream_t>(stream));
    if (st != WR_OK) return st;
  }
  return WR_OK;
}

static bool group_ok(int64_t M, int64_t K, int32_t count, const wr_gemv_group_item* it) {
  if (M < 1 || M > kDecodeTokens || count < 1 || count > wr::kMaxDecodeProblems || !it) return false;
  for (int i = 0; i < count; ++i) {
    QFmt f{};
    if (!split_fmt(it[i].bits, true, &f)) return false;
    if (it[i].reserved != 0 || check_dims(M, it[i].N, K) != WR_OK || K % 256 != 0) return false;
    if (!aligned16(it[i].packed) || !aligned16(it[i].scales) || !aligned16(it[i].y)) return false;
  }
  return true;
}

size_t wr_gemv_grouped_workspace_bytes(int64_t M, int64_t K, int32_t count, const wr_gemv_group_item* items) {
  if (!group_ok(M, K, count, items)) return 0;
  static thread_local DecodePlan dp;
  ProblemShape sh[wr::kMaxDecodeProblems];
  for (int i = 0; i < count; ++i) sh[i] = ProblemShape{items[i].N, K, items[i].bits & ~WR_SCALES_I8};
  plan_decode(M, count, sh, &dp);
  return dp.total;
}

wr_status wr_gemv_grouped(int64_t M, int64_t K, const uint16_t* x, int32_t count, const wr_gemv_group_item* items,
                          void* workspace, size_t workspace_bytes, void* stream) {
  if (!group_ok(M, K, count, items) || !aligned16(x) || !aligned16(workspace)) return WR_ERR_INVALID_ARG;
  if (workspace_bytes < wr_gemv_grouped_workspace_bytes(M, K, count, items)) return WR_ERR_INVALID_ARG;
  static thread_local DecodePlan dp;
  ProblemShape sh[wr::kMaxDecodeProblems];
  for (int i = 0; i < count; ++i) sh[i] = ProblemShape{items[i].N, K, items[i].bits & ~WR_SCALES_I8};
  plan_decode(M, count, sh, &dp);
  for (int i = 0; i < count; ++i) {
    QFmt f{};
    split_fmt(items[i].bits, true, &f);
    dp.args.prob[i].x = x;
    dp.args.prob[i].packed = static_cast<const uint8_t*>(items[i].packed);
    dp.args.prob[i].scales = items[i].scales;
    dp.args.prob[i].scale_q = scale_q_of(f, items[i].scales, items[i].N);
    dp.args.prob[i].y = items[i].y;
  }
  bind_workspace(dp, workspace);
  return run_decode(dp, static_cast<cudaStream_t>(stream));
}

static bool tbatch_ok(int64_t M, int32_t count, const wr_gemv_ternary_problem* pr) {
  if (M < 1 || M > kTernaryDecodeTokens || count < 1 || !pr) return false;
  for (int i = 0; i < count; ++i) {
    if (check_dims(M, pr[i].N, pr[i].K) != WR_OK || pr[i].K % 128 != 0) return false;
    if (!aligned16(pr[i].x) || !aligned16(pr[i].packed) || !aligned16(pr[i].alpha) || !aligned16(pr[i].sign_bits) ||
        !aligned16(pr[i].y))
      return false;
  }
  return true;
}

size_t wr_gemv_ternary_batched_workspace_bytes(int64_t M, int32_t count, const wr_gemv_ternary_problem* problems) {
  if (!tbatch_ok(M, count, problems)) return 0;
  size_t total = 0;
  static thread_local DecodePlan dp;
  ProblemShape sh[wr::kMaxDecodeProblems];
  for (int c0 = 0; c0 < count; c0 += wr::kMaxDecodeProblems) {
    const int n = std::min(count - c0, wr::kMaxDecodeProblems);
    for (int i = 0; i < n; ++i) sh[i] = ProblemShape{problems[c0 + i].N, problems[c0 + i].K, WR_FMT_TERNARY};
    plan_decode(M, n, sh, &dp);
    total = std::max(total, dp.total);
  }
  return total;
}

wr_status wr_gemv_ternary_batched(int64_t M, int32_t count, const wr_gemv_ternary_problem* problems,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  if (!tbatch_ok(M, count, problems) || !aligned16(workspace)) return WR_ERR_INVALID_ARG;
  if (workspace_bytes < wr_gemv_ternary_batched_workspace_bytes(M, count, problems)) return WR_ERR_INVALID_ARG;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  static thread_local DecodePlan dp;
  ProblemShape sh[wr::kMaxDecodeProblems];
  for (int c0 = 0; c0 < count; c0 += wr::kMaxDecodeProblems) {
    const int n = std::min(count - c0, wr::kMaxDecodeProblems);
    for (int i = 0; i < n; ++i) sh[i] = ProblemShape{problems[c0 + i].N, problems[c0 + i].K, WR_FMT_TERNARY};
    plan_decode(M, n, sh, &dp);
    for (int i = 0; i < n; ++i) {
      wr::DecProblem& pr = dp.args.prob[i];
      pr.x = problems[c0 + i].x;
      pr.packed = static_cast<const uint8_t*>(problems[c0 + i].packed);
      pr.scales = problems[c0 + i].alpha;
      pr.signs = problems[c0 + i].sign_bits;
      pr.y = problems[c0 + i].y;
    }
    bind_workspace(dp, workspace);
    const wr_status st = run_decode(dp, s);
    if (st != WR_OK) return st;
  }
  return WR_OK;
}

size_t wr_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int bits) {
  QFmt f{};
  if (!split_fmt(bits, false, &f)) return 0;
  if (check_dims(M, N, K) != WR_OK || K % 256 != 0) return 0;
  return q_workspace(f.base, M, N, K, true);
}

wr_status wr_gemm(int64_t M, int64_t N, int64_t K, const uint16_t* x, const void* packed,
                  const uint16_t* scales, int bits, int group, float* y, void* workspace,
                  size_t workspace_bytes, void* stream) {
  QFmt f{};
  if (!split_fmt(bits, false, &f)) return WR_ERR_UNSUPPORTED;
  if (group != 256) return WR_ERR_UNSUPPORTED;
  if (check_dims(M, N, K) != WR_OK || K % 256 != 0) return WR_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(packed) || !aligned16(scales) || !aligned16(y) || !aligned16(workspace))
    return WR_ERR_INVALID_ARG;
  if (workspace_bytes < q_workspace(f.base, M, N, K, true)) return WR_ERR_INVALID_ARG;
  return run_q(f.base, M, N, K, x, packed, scales, scale_q_of(f, scales, N), y, workspace,
               static_cast<cudaStream_t>(stream), true);
}

size_t wr_gemm_ternary_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (check_dims(M, N, K) != WR_OK || K % 128 != 0) return 0;
  return t_workspace(M, N, K);
}

wr_status wr_gemm_ternary(int64_t M, int64_t N, int64_t K, const uint16_t* x, const void* packed,
                          const uint16_t* alpha, const uint32_t* sign_bits, float* y, void* workspace,
                          size_t workspace_bytes, void* stream) {
  if (check_dims(M, N, K) != WR_OK || K % 128 != 0) return WR_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(packed) || !aligned16(alpha) || !aligned16(sign_bits) || !aligned16(y) ||
      !aligned16(workspace))
    return WR_ERR_INVALID_ARG;
  if (workspace_bytes < t_workspace(M, N, K)) return WR_ERR_INVALID_ARG;
  return run_t(M, N, K, x, packed, alpha, sign_bits, y, workspace, static_cast<cudaStream_t>(stream));
}

wr_status wr_quantize_pack(int bits, int64_t N, int64_t K, const float* w, void* packed, uint16_t* scales,
                           void* stream) {
  QFmt f{};
  if (!split_fmt(bits, false, &f)) return WR_ERR_UNSUPPORTED;
  if (check_dims(1, N, K) != WR_OK || K % 256 != 0) return WR_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(packed) || !aligned16(scales)) return WR_ERR_INVALID_ARG;
  int8_t* scale_q = const_cast<int8_t*>(scale_q_of(f, scales, N));
  return wr::launch_quantize_pack(f.base, w, (int)N, (int)K, static_cast<uint8_t*>(packed), scales, scale_q,
                                  static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? WR_OK
             : WR_ERR_CUDA;
}

wr_status wr_selftest_wait_timeout(void* stream) {
  if (wr::launch_selftest_wait_timeout(device_error_word(), static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return WR_ERR_CUDA;
  return WR_OK;
}

wr_status wr_get_device_error(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return WR_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)) != cudaSuccess) return WR_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) return WR_ERR_CUDA;
    return WR_ERR_TIMEOUT;
  }
  return WR_OK;
}

}  // extern "C"
