// Decode GEMV (M <= 8 tokens) for 2/3-bit weights on integer tensor cores, for one problem or a
// batch of independent problems.
//
// Decoding a token reads every weight once ("How We Shrank an AI Model by 85%...", section
// "Results": generating a token is mostly reading the weights from memory), so the kernel is a
// weight stream: each CTA walks a list of work items (problem, 128-row group, range of
// 256-code blocks) and keeps its copy rings full across item and problem boundaries.
//
//   y[m,n] = sum_b s[n,b] sum_{k in b} g[n,k] x[m,k],   g = 2c - L  (L = 3 or 7)
//
// The weights go to tensor memory as their unsigned codes c (one byte each; kind::i8, K = 32
// per MMA). The activations of a (token, block) are the integers n_k = x_k / 2^E, with
// E = exponent(max |x|) - 29, written as four balanced signed bytes d_j (n = sum_j 256^j d_j);
// limb j of token m is B row 4m + j. Every product and block sum is an exact integer,
//   D_j[n] = sum_k c[n,k] d_j[k],   sum_k g x = 2^E sum_j 256^j (2 D_j - L S_j),
// with S_j = sum_k d_j[k]; the last step runs in fp32. Values below 2^E (more than 2^29 under
// the block maximum) round to a multiple of 2^E: at most 2^-30 max|x| per element.
//
// Warp roles (320 threads, two CTAs per SM):
//   warps 0-7  consumers. Thread = weight row (TMEM lane); warps w and w+4 share a lane quarter.
//              Per block they decode their half of the codes into an A buffer (one 32-column
//              tensor-memory store per thread) and, two blocks behind, turn the integer
//              accumulator of an earlier block into fp32 partial dot products times s[n,b]
//              (warp group g takes tokens g*T .. g*T+T-1 of the T = N/8 per group). Doing both in
//              the same warps keeps cross-warp handoffs off the critical loop: a handoff costs
//              a few hundred cycles, a block of a 2-bit row group about seven hundred.
//   warp 8     producer: per block one bulk copy for the 8 packed units of the row group, one
//              for the B tile and one for its per-token corrections.
//   warp 9     allocates tensor memory and issues the MMAs (8 per block) and one commit per
//              block: the whole warp walks the blocks, one elected lane issues.
// Tensor memory (256 columns): A ring of 2 x 64 columns, accumulator ring of 3 x 32 columns.
// Every wait is bounded.
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "tc_common.cuh"
#include "tc_kernels.cuh"
#include "wr.h"

namespace wr {
namespace {

using namespace tc;

constexpr int kThreads = 320;
constexpr int kSP = 5;   // packed stages: 8 units of up to 1.5 KB
constexpr int kSX = 4;   // B tiles: up to 2 atoms x 32 rows x 128 bytes; also the MMA-done ring
constexpr int kSC = 8;   // correction records, 256 bytes
constexpr int kPStage = 8 * 1536;
constexpr int kXStage = 8 * 1024;
constexpr int kXOff = 0;                          // 1024-byte aligned (128-byte swizzle atoms)
constexpr int kPOff = kXOff + kSX * kXStage;
constexpr int kCOff = kPOff + kSP * kPStage;
constexpr int kBarOff = kCOff + kSC * 256;
constexpr int kBaseOff = kBarOff + 512;           // first work item of every problem (int[256])
constexpr int kSmem = kBaseOff + 4 * kMaxDecodeProblems + 1024;   // + alignment slack
static_assert(3 * kSmem > 228 * 1024, "at most two CTAs per SM (each holds 256 TMEM columns)");
static_assert(2 * kSmem <= 227 * 1024, "two CTAs per SM");
constexpr int kACols = 64;                        // one block of codes: 256 bytes per lane
constexpr int kDCol = 2 * kACols;                 // accumulators after the A ring
constexpr int kDCols = 32;
constexpr int kTmemCols = 256;
static_assert(kDCol + 3 * kDCols <= kTmemCols, "tensor memory budget");
constexpr int kLag = 2;                           // epilogue runs this many blocks behind decode
constexpr uint32_t kMagic = 0x4B400000u;          // 1.5 * 2^23: int -> float by an add

struct Bars {
  uint64_t pk_full[kSP], pk_empty[kSP], x_full[kSX], c_full[kSC], c_empty[kSC];
  uint64_t a_full[2];
  uint64_t mma_done[kSX];   // block j's MMAs complete: frees B stage j % kSX, A and accumulator of j
  uint64_t group;           // the 8 consumer warps meet here (bounded, unlike bar.sync)
  uint32_t tmem_base;
  int abort_flag;
  int last_flag;
};
static_assert(sizeof(Bars) <= 512, "barrier area");

// Position in this CTA's sequence of (item, block) (items blockIdx.x, +gridDim.x, ...), with
// the per-block fields of the item's problem held in registers: the problem table lives in the
// kernel parameters, whose constant-cache misses cost hundreds of cycles, so it is read once
// per item (and once more by the epilogue when the item ends).
struct Cursor {
  int it, b, b1, rg, p, pi;
  int N, B, P, bits;
  const uint8_t* packed;
  const uint8_t* xt;
  const uint16_t* scales;
};

__device__ __forceinline__ void cursor_load(Cursor& c, const DecArgs& a, const int* base) {
  if (c.it >= a.items) return;
  int lo = 0, hi = a.count - 1;
  while (lo < hi) {  // last problem with item_base <= it
    const int mid = (lo + hi + 1) >> 1;
    if (base[mid] <= c.it) lo = mid;
    else hi = mid - 1;
  }
  const DecProblem& pr = a.prob[lo];
  c.pi = lo;
  c.N = pr.N;
  c.B = pr.B;
  c.P = pr.P;
  c.bits = pr.bits;
  c.packed = pr.packed;
  c.xt = pr.xt;
  c.scales = pr.scales;
  const int local = c.it - base[lo];
  c.p = local % c.P;
  c.rg = local / c.P;
  c.b = (int)((int64_t)c.B * c.p / c.P);
  c.b1 = (int)((int64_t)c.B * (c.p + 1) / c.P);
}
__device__ __forceinline__ Cursor cursor_start(const DecArgs& a, const int* base) {
  Cursor c{};
  c.it = blockIdx.x;
  cursor_load(c, a, base);
  return c;
}
__device__ __forceinline__ void cursor_next(Cursor& c, const DecArgs& a, const int* base) {
  if (++c.b >= c.b1) {
    c.it += gridDim.x;
    cursor_load(c, a, base);
  }
}

// One thread's two quarters (128 codes) of a 16-row tile unit, as bytes in logical K order;
// see the packed layout in include/wr.h.
__device__ __forceinline__ void q2_half_i8(const uint8_t* unit, int r0, int half, int g, uint32_t v[32]) {
#pragma unroll
  for (int qq = 0; qq < 2; ++qq) {
    const uint4 c = *reinterpret_cast<const uint4*>(unit + (32 * half + 4 * r0 + 2 * g + qq) * 16);
    decode_q2_word_i8(c.x, v + 16 * qq + 0);
    decode_q2_word_i8(c.y, v + 16 * qq + 4);
    decode_q2_word_i8(c.z, v + 16 * qq + 8);
    decode_q2_word_i8(c.w, v + 16 * qq + 12);
  }
}

__device__ __forceinline__ void q3_half_i8(const uint8_t* unit, int r0, int half, int g, uint32_t v[32]) {
#pragma unroll
  for (int qq = 0; qq < 2; ++qq) {
    const int l = 4 * r0 + 2 * g + qq;
    uint32_t w[6];
    if (half == 0) {
      const uint4 c0 = *reinterpret_cast<const uint4*>(unit + l * 16);
      const uint2 c1 = *reinterpret_cast<const uint2*>(unit + (32 + l) * 16);
      w[0] = c0.x; w[1] = c0.y; w[2] = c0.z; w[3] = c0.w; w[4] = c1.x; w[5] = c1.y;
    } else {
      const uint2 c1 = *reinterpret_cast<const uint2*>(unit + (32 + l) * 16 + 8);
      const uint4 c2 = *reinterpret_cast<const uint4*>(unit + (64 + l) * 16);
      w[0] = c1.x; w[1] = c1.y; w[2] = c2.x; w[3] = c2.y; w[4] = c2.z; w[5] = c2.w;
    }
    decode_q3_group_i8(w, v + 16 * qq);
    decode_q3_group_i8(w + 3, v + 16 * qq + 8);
  }
}

// tcgen05.ld of 16 raw 32-bit columns; the values are valid after tmem_wait_ld16 on the same array.
__device__ __forceinline__ void tmem_ld16_raw(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
// tcgen05.wait::ld that also names the loaded registers, so that no use of them is scheduled
// before the wait.
__device__ __forceinline__ void tmem_wait_ld16(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
               :
               : "memory");
}

__global__ void __launch_bounds__(kThreads, 2) gemv_q_kernel(const __grid_constant__ DecArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* xs = smem + kXOff;
  uint8_t* ps = smem + kPOff;
  uint8_t* cs = smem + kCOff;
  Bars* bars = reinterpret_cast<Bars*>(smem + kBarOff);
  int* base = reinterpret_cast<int*>(smem + kBaseOff);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &bars->abort_flag;
  const int M = a.M;
  const int xrows = decode_xrows(M);   // MMA N: 4 limb rows per token slot

  for (int i = threadIdx.x; i < a.count; i += kThreads) base[i] = a.prob[i].item_base;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kSP; ++i) {
      mbar_init(&bars->pk_full[i], 1);
      mbar_init(&bars->pk_empty[i], 8);
    }
    for (int i = 0; i < kSX; ++i) {
      mbar_init(&bars->x_full[i], 1);
      mbar_init(&bars->mma_done[i], 1);
    }
    for (int i = 0; i < kSC; ++i) {
      mbar_init(&bars->c_full[i], 1);
      mbar_init(&bars->c_empty[i], 8);
    }
    for (int i = 0; i < 2; ++i) mbar_init(&bars->a_full[i], 8);
    mbar_init(&bars->group, 8);
    bars->abort_flag = 0;
    bars->last_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) tmem_alloc(&bars->tmem_base, kTmemCols);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 8) {
    // ------------------------------------------------------------ producer (one thread)
    if (lane == 0) {
      const uint32_t xtb = (uint32_t)xtile_bytes(false, M);
      const uint32_t bbytes = 256u * xrows;
      uint32_t nx = 0, nc = 0, np = 0;   // copies issued per ring
      bool ok = true;
      for (Cursor c = cursor_start(a, base); c.it < a.items && ok; cursor_next(c, a, base)) {
        const uint8_t* xsrc = c.xt + (int64_t)c.b * xtb;
        const int sx = nx % kSX;
        if (!(ok = mbar_wait_bg(&bars->mma_done[sx], ((nx / kSX) & 1) ^ 1, abort_flag, a.err, 101))) break;
        mbar_arrive_expect_tx(&bars->x_full[sx], bbytes);
        bulk_load(xs + sx * kXStage, xsrc, bbytes, &bars->x_full[sx]);
        ++nx;
        const int sc = nc % kSC;
        if (!(ok = mbar_wait_bg(&bars->c_empty[sc], ((nc / kSC) & 1) ^ 1, abort_flag, a.err, 102))) break;
        mbar_arrive_expect_tx(&bars->c_full[sc], 256);
        bulk_load(cs + sc * 256, xsrc + bbytes, 256, &bars->c_full[sc]);
        ++nc;
        // the ntile units of this row group and block are adjacent: one copy
        const int ub = c.bits == 2 ? 1024 : 1536;
        const int ntile = min(8, (c.N + 15) / 16 - c.rg * 8);
        const int sp = np % kSP;
        if (!(ok = mbar_wait_bg(&bars->pk_empty[sp], ((np / kSP) & 1) ^ 1, abort_flag, a.err, 103))) break;
        mbar_arrive_expect_tx(&bars->pk_full[sp], ntile * ub);
        bulk_load(ps + sp * kPStage, c.packed + ((int64_t)c.rg * 8 * c.B + (int64_t)c.b * ntile) * ub, ntile * ub,
                  &bars->pk_full[sp]);
        ++np;
      }
      if (!ok) {
        // aborted: let the copies in flight land before the CTA exits
        for (uint32_t k = np > kSP ? np - kSP : 0; k < np; ++k) mbar_wait_drain(&bars->pk_full[k % kSP], (k / kSP) & 1);
        for (uint32_t k = nx > kSX ? nx - kSX : 0; k < nx; ++k) mbar_wait_drain(&bars->x_full[k % kSX], (k / kSX) & 1);
        for (uint32_t k = nc > kSC ? nc - kSC : 0; k < nc; ++k) mbar_wait_drain(&bars->c_full[k % kSC], (k / kSC) & 1);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer (whole warp, one lane issues)
    const uint64_t bdesc0 = smem_desc_sw128(xs);
    const uint32_t idesc = idesc_i8_m128(xrows);
    const uint32_t atom16 = (uint32_t)(xrows * 128) >> 4;
    uint32_t gm = 0;
    bool ok = true;
    for (Cursor c = cursor_start(a, base); c.it < a.items; cursor_next(c, a, base), ++gm) {
      const int sx = gm % kSX;
      if (!(ok = mbar_wait_bg(&bars->a_full[gm & 1], (gm >> 1) & 1, abort_flag, a.err, 201))) break;
      if (!(ok = mbar_wait_bg(&bars->x_full[sx], (gm / kSX) & 1, abort_flag, a.err, 202))) break;
      fence_after_sync();
      const uint32_t dcol = tmem + kDCol + (gm % 3) * kDCols;
      const uint32_t acol = tmem + (gm & 1) * kACols;
      const uint64_t bd = bdesc0 + (uint64_t)((sx * kXStage) >> 4);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        // K slice j: B atom j / 4 (128 K positions x xrows rows), 32-byte step inside it
        const uint64_t off = (uint64_t)((j >> 2) * atom16 + (((j & 3) * 32) >> 4));
        mma_ts_i8_elect(dcol, acol + 8 * j, bd + off, idesc, j != 0);
      }
      mma_commit_elect(&bars->mma_done[sx]);
    }
    // the MMAs already issued finish before tensor memory is released
    if (!ok && gm > 0) mbar_wait_drain(&bars->mma_done[(gm - 1) % kSX], ((gm - 1) / kSX) & 1);
  } else {
    // ------------------------------------------------------------ consumers (warps 0-7)
    // One iteration: decode block gd and finish block ge = gd - 2. The tensor-memory store of the
    // codes and the load of the accumulator are both in flight before either is waited for.
    const int g = warp >> 2, lq = warp & 3;
    const int t = 32 * lq + lane;                       // row in the row group = TMEM lane
    const int tile = t >> 4, r = t & 15, r0 = r & 7, half = r >> 3;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * lq) << 16);
    const int tpg = xrows >> 3;                         // token slots per warp group: 1, 2, 4
    const int m0 = tpg * g;                             // first token slot of this group
    Cursor dc = cursor_start(a, base), ec = dc;
    uint32_t gd = 0, ge = 0, ng = 0;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    auto group_sync = [&](int code) {
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->group);
      return mbar_wait(&bars->group, (ng++) & 1, abort_flag, a.err, code);
    };
    // scale of the next block to finish, loaded one iteration ahead
    auto scale_of = [&](const Cursor& c) -> uint16_t {
      const int n = c.rg * 128 + t;
      return (c.it < a.items && n < c.N) ? __ldg(c.scales + (int64_t)n * c.B + c.b) : (uint16_t)0;
    };
    uint16_t sraw = scale_of(ec);
    bool ok = true;
    for (;;) {
      const bool do_d = dc.it < a.items;
      const bool do_e = ec.it < a.items && (!do_d || gd >= ge + kLag);
      if (!do_d && !do_e) break;
      const int sp = gd % kSP, sc = ge % kSC;
      if (do_d) {
        // A buffer gd % 2 is free once block gd - 2 (= ge when both run) has been multiplied
        if (gd >= 2 && !(ok = mbar_wait(&bars->mma_done[(gd - 2) % kSX], ((gd - 2) / kSX) & 1, abort_flag, a.err, 301)))
          break;
        if (!(ok = mbar_wait(&bars->pk_full[sp], (gd / kSP) & 1, abort_flag, a.err, 302))) break;
      } else if (!(ok = mbar_wait(&bars->mma_done[ge % kSX], (ge / kSX) & 1, abort_flag, a.err, 303))) {
        break;
      }
      if (do_e && !(ok = mbar_wait(&bars->c_full[sc], (ge / kSC) & 1, abort_flag, a.err, 304))) break;
      fence_after_sync();
      if (do_d) {
        uint32_t v[32];
        if (dc.bits == 2) q2_half_i8(ps + sp * kPStage + tile * 1024, r0, half, g, v);
        else q3_half_i8(ps + sp * kPStage + tile * 1536, r0, half, g, v);
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->pk_empty[sp]);
        tmem_st32(lane_base + (gd & 1) * kACols + 32 * g, v);
      }
      uint32_t d[16];
      if (do_e) tmem_ld16_raw(lane_base + kDCol + (ge % 3) * kDCols + 4 * m0, d);
      if (do_d) tmem_wait_st();
      if (do_e) tmem_wait_ld16(d);
      fence_before_sync();
      if (do_d) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->a_full[gd & 1]);
        cursor_next(dc, a, base);
        ++gd;
      }
      if (do_e) {
        // corrections of the block: per token slot the factor 2^E, then per limb
        // C = magic - L S_j
        const uint8_t* cst = cs + sc * 256;
        const float s = half_bits_to_float(sraw);
#pragma unroll
        for (int ml = 0; ml < 4; ++ml) {
          if (ml < tpg && m0 + ml < M) {
            // limb j: 2 D_j - L S_j is an exact integer below 2^22 in magnitude; the add of
            // the magic constant makes it a float exactly
            const int4 c4 = reinterpret_cast<const int4*>(cst + 32)[m0 + ml];
            const float fm = reinterpret_cast<const float*>(cst)[m0 + ml];
            const int cj[4] = {c4.x, c4.y, c4.z, c4.w};
            float v = 0.f;
#pragma unroll
            for (int j = 3; j >= 0; --j)
              v = fmaf(v, 256.f, __int_as_float(2 * (int)d[4 * ml + j] + cj[j]) - 12582912.f);
            acc[ml] = fmaf(s * fm, v, acc[ml]);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->c_empty[sc]);
        if (ec.b + 1 == ec.b1) {
          // last block of the item: y, or the split-K combine through the workspace
          const int n = ec.rg * 128 + t;
          float* y = a.prob[ec.pi].y;
          if (ec.P == 1) {
            if (n < ec.N) {
#pragma unroll
              for (int ml = 0; ml < 4; ++ml)
                if (ml < tpg && m0 + ml < M) y[(int64_t)(m0 + ml) * ec.N + n] = acc[ml];
            }
          } else {
            const int cid = a.prob[ec.pi].counter_base + ec.rg;
            const int64_t pbase = a.prob[ec.pi].partial_base;
            float* part = a.partial + pbase + ((int64_t)ec.rg * ec.P + ec.p) * M * 128;
#pragma unroll
            for (int ml = 0; ml < 4; ++ml)
              if (ml < tpg && m0 + ml < M) part[(m0 + ml) * 128 + t] = acc[ml];
            __threadfence();
            if (!(ok = group_sync(305))) break;
            if (threadIdx.x == 0) bars->last_flag = (atomicAdd(a.counter + cid, 1) == ec.P - 1);
            if (!(ok = group_sync(306))) break;
            if (bars->last_flag) {
              __threadfence();
              float sum[4] = {0.f, 0.f, 0.f, 0.f};
              for (int pp = 0; pp < ec.P; ++pp) {
                const float* src = a.partial + pbase + ((int64_t)ec.rg * ec.P + pp) * M * 128;
#pragma unroll
                for (int ml = 0; ml < 4; ++ml)
                  if (ml < tpg && m0 + ml < M) sum[ml] += __ldcg(src + (m0 + ml) * 128 + t);
              }
              if (n < ec.N) {
#pragma unroll
                for (int ml = 0; ml < 4; ++ml)
                  if (ml < tpg && m0 + ml < M) y[(int64_t)(m0 + ml) * ec.N + n] = sum[ml];
              }
              if (threadIdx.x == 0) a.counter[cid] = 0;
            }
          }
#pragma unroll
          for (int ml = 0; ml < 4; ++ml) acc[ml] = 0.f;
        }
        cursor_next(ec, a, base);
        ++ge;
        sraw = scale_of(ec);
      }
    }
    (void)ok;
  }

  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 9) tmem_dealloc(tmem, kTmemCols);
}

// Preparation pass: one warp per (problem, block, token slot m < N/4). The block's activations
// of token m become integers n_k = x_k / 2^E (E = exponent of the block maximum - 29; values
// that are not multiples of 2^E round to the nearest, ties to even), split into four balanced
// signed bytes d_j (n = sum_j 256^j d_j, d_j in [-128, 127]). Limb j goes to B row 4m + j (two
// atoms of 128 K positions x N rows, 128-byte swizzle) at the logical K position whose A byte
// holds code k. After the atoms: the factor 2^E per slot (8 floats) and, per slot and limb,
// C = 0x4B400000 - L S_j with S_j = sum_k d_j[k] (8 x 4 int32). Slots m >= M hold zeros.
__global__ void __launch_bounds__(256) prep_x_kernel(const __grid_constant__ DecArgs a, int total_blocks) {
  const int lane = threadIdx.x & 31;
  const int M = a.M;
  const int xrows = decode_xrows(M), slots = xrows >> 2;
  const int w = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (w >= total_blocks * slots) return;
  const int gblk = w / slots, m = w - gblk * slots;
  int lo = 0, hi = a.count - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a.prob[mid].xblk_base <= gblk) lo = mid;
    else hi = mid - 1;
  }
  const DecProblem& pr = a.prob[lo];
  const int b = gblk - pr.xblk_base;
  uint8_t* dst = pr.xt + (int64_t)b * xtile_bytes(false, M);
  // lane l holds logical K positions 8l .. 8l+7 of the decoded block
  float xv[8];
  float amax = 0.f;
  if (m < M) {
    const uint16_t* xrow = pr.x + (int64_t)m * pr.K + (int64_t)b * 256;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int kl = 8 * lane + e;
      const int k = pr.bits == 2 ? q2_code_at(kl) : q3_code_at(kl);
      xv[e] = __bfloat162float(__ushort_as_bfloat16(__ldg(xrow + k)));
      amax = fmaxf(amax, fabsf(xv[e]));
    }
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) xv[e] = 0.f;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  int ex = 0;
  if (amax > 0.f) frexpf(amax, &ex);   // amax in [2^(ex-1), 2^ex)
  const int E = ex - 30;                // |n| < 2^30
  uint32_t lw[4][2] = {{0u, 0u}, {0u, 0u}, {0u, 0u}, {0u, 0u}};
  int s[4] = {0, 0, 0, 0};
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int n = amax > 0.f ? __float2int_rn(ldexpf(xv[e], -E)) : 0;
    int rest = n;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int d = j < 3 ? (int)(int8_t)(rest & 0xFF) : rest;
      rest = (rest - d) >> 8;
      s[j] += d;
      lw[j][e >> 2] |= ((uint32_t)d & 0xFFu) << (8 * (e & 3));
    }
  }
  const int atom = lane >> 4, chunk = (lane & 15) >> 1, off = (lane & 1) * 8;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int row = 4 * m + j;
    *reinterpret_cast<uint2*>(dst + atom * xrows * 128 + row * 128 + ((chunk ^ (row & 7)) << 4) + off) =
        make_uint2(lw[j][0], lw[j][1]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
    for (int j = 0; j < 4; ++j) s[j] += __shfl_xor_sync(0xffffffffu, s[j], o);
  }
  if (lane == 0) {
    const int L = pr.bits == 2 ? 3 : 7;
    float* fct = reinterpret_cast<float*>(dst + 256 * xrows);
    int* cc = reinterpret_cast<int*>(dst + 256 * xrows + 32);
    fct[m] = (m < M && amax > 0.f) ? ldexpf(1.f, E) : 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) cc[4 * m + j] = (int)kMagic - L * s[j];
  }
}

}  // namespace

cudaError_t launch_prep_x(const DecArgs& a, int total_blocks, cudaStream_t stream) {
  const int warps = total_blocks * (decode_xrows(a.M) >> 2);
  prep_x_kernel<<<(warps + 7) / 8, 256, 0, stream>>>(a, total_blocks);
  return cudaGetLastError();
}

cudaError_t launch_gemv_q(const DecArgs& a, int grid, cudaStream_t stream) {
  static bool set = false;
  if (!set) {
    const cudaError_t e = cudaFuncSetAttribute(gemv_q_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    set = true;
  }
  gemv_q_kernel<<<grid, kThreads, kSmem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace wr
