// Decode GEMV (M <= 8 tokens) for 2/3-bit weights on integer tensor cores, for one problem or a
// batch of independent problems.
//
// Decoding a token reads every weight once ("How We Shrank an AI Model by 85%...", section
// "Results": generating a token is mostly reading the weights from memory), so the kernel is a
// weight stream: the batch's blocks (problem by problem, 128-row group by row group, 256-code
// block by block) are cut into one contiguous range per CTA, of equal cost (a 3-bit block weighs
// more than a 2-bit one: block_cost), so that the CTAs finish together, each keeping its copy
// rings full across row-group and problem boundaries.
//
//   y[m,n] = sum_b s[n,b] sum_{k in b} g[n,k] x[m,k],   g = 2c - L  (L = 3 or 7)
//
// The weights go to tensor memory as their unsigned codes c, one byte each (kind::i8, K = 32 per
// MMA), each cut out of the packed words by a mask and left in place in its byte: the byte at
// K position k holds c_k 2^e_k for a fixed position exponent e_k <= 6. The activations of a
// (token, block) become the integers n_k = x_k / 2^(E + e_k), E = exponent(max |x|) - 30, written
// as four balanced signed bytes d_j (n = sum_j 256^j d_j); limb j of token m is B row 4m + j.
// Every product and limb sum is an exact integer,
//   D_j[n] = sum_k c[n,k] 2^e_k d_j[k],   sum_k g x = 2^E (sum_j 256^j (2 D_j - L S_j)),
// with S_j = sum_k 2^e_k d_j[k]; the limbs are combined in fp32. Activations below 2^(E + e_k)
// (more than 2^24 under the block maximum) round to that step: at most 2^-25 max |x| per
// element, and the fp32 combination adds a few units of 2^-24 of sum |x| per block.
//
// The 2-bit trellis-coded format (WR_FMT_T2) runs through the same kernel: its symbols are
// stored like Q2 codes, and the decode warps turn each into the level index 2 u + p (p = the
// low bit of the previous symbol in the row, carried word by word) before the MMA, so the
// MMA sees 8 levels (L = 7), as for Q3.
//
// A CTA is one small pipeline; three run on every SM so that their latency chains overlap
// (warp roles, 320 threads):
//   warps 0-3  decode, thread = weight row (TMEM lane 32 w + lane): per block, the row's 256
//              codes into the A buffer (two 32-column tensor-memory stores), then hand it to
//              the MMA warp.
//   warps 4-7  epilogue, thread = row: per block, once its MMAs are done, the integer
//              accumulator becomes fp32 partial dot products times s[n,b] for all tokens of
//              the row. Decode and epilogue run in separate warps so that a block costs the
//              longer of the two chains, not their sum.
//   warp 8     copies: the packed weights (one bulk copy per block, a ring of kSP blocks), the
//              prepared B tiles and their correction records (a ring of kSX blocks).
//   warp 9     allocates tensor memory and issues the 8 MMAs and one commit per block (the
//              whole warp walks the blocks, one elected lane issues).
// Tensor memory (128 columns): one A buffer (64 columns) and two accumulators (32 columns). The
// store of block i waits for the MMAs of block i - 1; block i's MMAs write accumulator i % 2
// once the epilogue has read block i - 2 from it. Every wait is bounded.
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
constexpr int kCtasPerSm = 3;
constexpr int kSP = 4;   // packed stages: 8 units of up to 1.5 KB
constexpr int kSX = 3;   // B tiles (up to 2 atoms x 32 rows x 128 bytes); also the MMA-done ring
constexpr int kSC = 4;   // correction records, 256 bytes
constexpr int kPStage = 8 * 1536;
constexpr int kXStage = 8 * 1024;
constexpr int kXOff = 0;                          // 1024-byte aligned (128-byte swizzle atoms)
constexpr int kPOff = kXOff + kSX * kXStage;
constexpr int kCOff = kPOff + kSP * kPStage;
constexpr int kBarOff = kCOff + kSC * 256;
constexpr int kSmem = kBarOff + 256 + 1024;        // + alignment slack
static_assert(kCtasPerSm * (kSmem + 1024) <= 228 * 1024, "three CTAs per SM");
constexpr int kACol = 0;                          // one block of codes: 256 bytes per lane
constexpr int kDCol = 64;                         // two accumulators of N <= 32 columns
constexpr int kDCols = 32;
constexpr int kTmemCols = 128;
static_assert(kCtasPerSm * kTmemCols <= 512, "tensor memory of an SM");

struct Bars {
  uint64_t pk_full[kSP], pk_empty[kSP], x_full[kSX], c_full[kSC], c_empty[kSC];
  uint64_t mma_done[kSX];   // block j's MMAs complete: frees B stage j % kSX, A; accumulator holds j
  uint64_t a_full;          // the decode warps have stored block j's codes
  uint64_t d_empty[2];      // the epilogue warps have read accumulator j % 2
  uint64_t group;           // the 4 consumer warps meet here (bounded, unlike bar.sync)
  uint32_t tmem_base;
  int abort_flag;
  int last_flag;
};
static_assert(sizeof(Bars) <= 256, "barrier area");

// Position in this CTA's contiguous range of the batch's blocks (problem by problem, row group
// by row group, K block by K block), with the fields of the current problem in registers: the
// problem table lives in the kernel parameters, whose constant-cache misses cost hundreds of
// cycles, so it is read only when the range crosses into the next problem.
struct Pos {
  int64_t g;            // global block
  int left;             // blocks left in the range, this one included
  int pi, rg, b;        // problem, row group, K block
  int grg;              // global row group (arrival counter index)
  int N, B, RG, bits;
  const uint8_t* packed;
  const uint8_t* xt;
  const uint16_t* scales;
  const int8_t* scale_q;
  float* y;
};

__device__ __forceinline__ void pos_load(Pos& p, const DecArgs& a) {
  const DecProblem& pr = a.prob[p.pi];
  p.N = pr.N;
  p.B = pr.B;
  p.RG = pr.RG;
  p.bits = pr.bits;
  p.packed = pr.packed;
  p.xt = pr.xt;
  p.scales = pr.scales;
  p.scale_q = pr.scale_q;
  p.y = pr.y;
}
__device__ __forceinline__ Pos pos_start(const DecArgs& a) {
  Pos p{};
  const int G = (int)gridDim.x;   // the block ranges: range_start in tc_kernels.cuh
  p.g = range_start(a, G, blockIdx.x);
  p.left = (int)(range_start(a, G, blockIdx.x + 1) - p.g);
  if (p.left <= 0) return p;
  int lo = 0, hi = a.count - 1;
  while (lo < hi) {  // last problem whose first block is <= g
    const int mid = (lo + hi + 1) >> 1;
    if (a.prob[mid].block_base <= p.g) lo = mid;
    else hi = mid - 1;
  }
  p.pi = lo;
  pos_load(p, a);
  const int64_t local = p.g - a.prob[lo].block_base;
  p.rg = (int)(local / p.B);
  p.b = (int)(local - (int64_t)p.rg * p.B);
  p.grg = a.prob[lo].counter_base + p.rg;
  return p;
}
__device__ __forceinline__ void pos_next(Pos& p, const DecArgs& a) {
  ++p.g;
  if (--p.left <= 0) return;
  if (++p.b == p.B) {
    p.b = 0;
    ++p.grg;
    if (++p.rg == p.RG) {
      p.rg = 0;
      ++p.pi;
      pos_load(p, a);
    }
  }
}

// The decode side of the consumers needs only the block's format: a lighter position.
struct Lite {
  int left, pi, rg, b, B, RG, bits;
};
__device__ __forceinline__ Lite lite_of(const Pos& p) { return Lite{p.left, p.pi, p.rg, p.b, p.B, p.RG, p.bits}; }
__device__ __forceinline__ void lite_next(Lite& p, const DecArgs& a) {
  if (--p.left <= 0) return;
  if (++p.b == p.B) {
    p.b = 0;
    if (++p.rg == p.RG) {
      p.rg = 0;
      ++p.pi;
      p.B = a.prob[p.pi].B;
      p.RG = a.prob[p.pi].RG;
      p.bits = a.prob[p.pi].bits;
    }
  }
}

// Half h (codes 128 h .. 128 h + 127 of the row: quarters 2h, 2h+1) of a 16-row tile unit, as
// bytes in logical K order; see the packed layout in include/wr.h.
__device__ __forceinline__ void q2_half_i8(const uint8_t* unit, int r0, int half, int h, uint32_t v[32]) {
#pragma unroll
  for (int qq = 0; qq < 2; ++qq) {
    const uint4 c = *reinterpret_cast<const uint4*>(unit + (32 * half + lane_pos(r0, 2 * h + qq)) * 16);
    decode_q2_word_i8(c.x, v + 16 * qq + 0);
    decode_q2_word_i8(c.y, v + 16 * qq + 4);
    decode_q2_word_i8(c.z, v + 16 * qq + 8);
    decode_q2_word_i8(c.w, v + 16 * qq + 12);
  }
}

// The trellis-coded format: the Q2 words, with the low bit of the previous symbol carried
// through the row in code order (quarter by quarter, word by word).
__device__ __forceinline__ void t2_half_i8(const uint8_t* unit, int r0, int half, int h, uint32_t v[32],
                                           uint32_t& carry) {
#pragma unroll
  for (int qq = 0; qq < 2; ++qq) {
    const uint4 c = *reinterpret_cast<const uint4*>(unit + (32 * half + lane_pos(r0, 2 * h + qq)) * 16);
    decode_t2_word_i8(c.x, carry, v + 16 * qq + 0);
    decode_t2_word_i8(c.y, carry, v + 16 * qq + 4);
    decode_t2_word_i8(c.z, carry, v + 16 * qq + 8);
    decode_t2_word_i8(c.w, carry, v + 16 * qq + 12);
  }
}

__device__ __forceinline__ void q3_half_i8(const uint8_t* unit, int r0, int half, int h, uint32_t v[32]) {
#pragma unroll
  for (int qq = 0; qq < 2; ++qq) {
    const int l = lane_pos(r0, 2 * h + qq);
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

// tcgen05.ld of NC (8, 16 or 32) raw 32-bit columns; the values are valid after
// tmem_wait_ld_regs on the same array, which names them so that no use is scheduled earlier.
template <int NC>
__device__ __forceinline__ void tmem_ld_raw(uint32_t taddr, uint32_t (&r)[NC]) {
  if constexpr (NC == 8) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr)
                 : "memory");
  } else if constexpr (NC == 16) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
  } else {
    static_assert(NC == 32, "8, 16 or 32 columns");
    tmem_ld32(taddr, r);
  }
}
template <int NC>
__device__ __forceinline__ void tmem_wait_ld_regs(uint32_t (&r)[NC]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
  // the empty asm below ties every loaded register to a point after the wait
#pragma unroll
  for (int i = 0; i < NC; ++i) asm volatile("" : "+r"(r[i]));
}

// XR: MMA N, 4 limb rows per token slot (8, 16 or 32 for M <= 2, 4, 8). kAll: the batch holds
// trellis-coded problems or int8 block scales; without them the decode and epilogue warps keep
// only the Q2/Q3 branches and the fp16 scale load.
template <int XR, bool kAll>
__global__ void __launch_bounds__(kThreads, kCtasPerSm) gemv_q_kernel(const __grid_constant__ DecArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* xs = smem + kXOff;
  uint8_t* ps = smem + kPOff;
  uint8_t* cs = smem + kCOff;
  Bars* bars = reinterpret_cast<Bars*>(smem + kBarOff);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &bars->abort_flag;
  constexpr int kSlots = XR / 4;       // token slots
  const int M = a.M;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSP; ++i) {
      mbar_init(&bars->pk_full[i], 1);
      mbar_init(&bars->pk_empty[i], 4);
    }
    for (int i = 0; i < kSX; ++i) {
      mbar_init(&bars->x_full[i], 1);
      mbar_init(&bars->mma_done[i], 1);
    }
    for (int i = 0; i < kSC; ++i) {
      mbar_init(&bars->c_full[i], 1);
      mbar_init(&bars->c_empty[i], 4);
    }
    mbar_init(&bars->a_full, 4);
    for (int i = 0; i < 2; ++i) mbar_init(&bars->d_empty[i], 4);
    mbar_init(&bars->group, 4);
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
    // ------------------------------------------------------------ copy warp (whole warp walks the
    // blocks, one elected lane issues): packed weights (a ring of kSP blocks), prepared B tiles
    // and their correction records (a ring of kSX blocks)
    constexpr uint32_t bbytes = 256u * XR;
    constexpr uint32_t xtb = bbytes + 256u;   // prepared tile: B atoms, then corrections
    Pos cp = pos_start(a), cx = cp;            // next block to copy: weights, activations
    const uint32_t nblocks = cp.left > 0 ? (uint32_t)cp.left : 0u;
    uint32_t np = 0, nx = 0;                   // weight copies, activation copies issued
    bool ok = true;
    while (ok && (np < nblocks || nx < nblocks)) {
      if (np < nblocks) {
        // weight stage np % kSP: free once the decode warps have read block np - kSP
        const int sp = np % kSP;
        if (!(ok = mbar_wait_bg(&bars->pk_empty[sp], ((np / kSP) & 1) ^ 1, abort_flag, a.err, 101))) break;
        const int ub = cp.bits == 3 ? 1536 : 1024;
        const int ntile = min(8, (cp.N + 15) / 16 - cp.rg * 8);
        if (elect_one()) {
          mbar_arrive_expect_tx(&bars->pk_full[sp], ntile * ub);
          bulk_load(ps + sp * kPStage, cp.packed + ((int64_t)cp.rg * 8 * cp.B + (int64_t)cp.b * ntile) * ub,
                    ntile * ub, &bars->pk_full[sp]);
        }
        __syncwarp();
        pos_next(cp, a);
        ++np;
      }
      if (nx < nblocks) {
        // activation stage nx % kSX: free once block nx - kSX's MMAs are done; correction slot
        // nx % kSC once the epilogue has read block nx - kSC
        const int sx = nx % kSX, sc = nx % kSC;
        if (!(ok = mbar_wait_bg(&bars->mma_done[sx], ((nx / kSX) & 1) ^ 1, abort_flag, a.err, 102))) break;
        if (!(ok = mbar_wait_bg(&bars->c_empty[sc], ((nx / kSC) & 1) ^ 1, abort_flag, a.err, 103))) break;
        const uint8_t* xsrc = cx.xt + (int64_t)cx.b * xtb;
        if (elect_one()) {
          mbar_arrive_expect_tx(&bars->x_full[sx], bbytes);
          bulk_load(xs + sx * kXStage, xsrc, bbytes, &bars->x_full[sx]);
          mbar_arrive_expect_tx(&bars->c_full[sc], 256);
          bulk_load(cs + sc * 256, xsrc + bbytes, 256, &bars->c_full[sc]);
        }
        __syncwarp();
        pos_next(cx, a);
        ++nx;
      }
    }
    if (!ok) {
      // aborted: let the copies in flight land before the CTA exits
      for (uint32_t k = np > kSP ? np - kSP : 0; k < np; ++k) mbar_wait_drain(&bars->pk_full[k % kSP], (k / kSP) & 1);
      for (uint32_t k = nx > kSX ? nx - kSX : 0; k < nx; ++k) mbar_wait_drain(&bars->x_full[k % kSX], (k / kSX) & 1);
      for (uint32_t k = nx > kSC ? nx - kSC : 0; k < nx; ++k) mbar_wait_drain(&bars->c_full[k % kSC], (k / kSC) & 1);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA warp (whole warp, one lane issues)
    const uint64_t bdesc0 = smem_desc_sw128(xs);
    constexpr uint32_t idesc = idesc_i8_m128(XR);
    constexpr uint32_t atom16 = (uint32_t)(XR * 128) >> 4;
    const int G = (int)gridDim.x;
    const int64_t span = range_start(a, G, blockIdx.x + 1) - range_start(a, G, blockIdx.x);
    const uint32_t nblocks = span > 0 ? (uint32_t)span : 0u;
    uint32_t gm = 0;
    bool ok = true;
    for (; gm < nblocks; ++gm) {
      const int sx = gm % kSX;
      // the B tile and the accumulator are normally ready long before the codes: wait for them
      // first, so that the wait for the A handoff is the last one before the MMAs
      if (!(ok = mbar_wait(&bars->x_full[sx], (gm / kSX) & 1, abort_flag, a.err, 202))) break;
      // accumulator gm % 2 was read by the epilogue warps (block gm - 2)
      if (!(ok = mbar_wait(&bars->d_empty[gm & 1], ((gm >> 1) & 1) ^ 1, abort_flag, a.err, 203))) break;
      if (!(ok = mbar_wait(&bars->a_full, gm & 1, abort_flag, a.err, 201))) break;
      fence_after_sync();
      mma8_i8_commit_elect(tmem + kDCol + (gm & 1) * kDCols, tmem + kACol,
                           bdesc0 + (uint64_t)((sx * kXStage) >> 4), atom16, idesc, &bars->mma_done[sx]);
    }
    // the MMAs already issued finish before tensor memory is released
    if (!ok && gm > 0) mbar_wait_drain(&bars->mma_done[(gm - 1) % kSX], ((gm - 1) / kSX) & 1);
  } else if (warp < 4) {
    // ------------------------------------------------------------ decode (warps 0-3, thread = row)
    const int t = threadIdx.x;                          // row in the row group = TMEM lane
    const int tile = t >> 4, r = t & 15, r0 = r & 7, half = r >> 3;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * warp) << 16);
    Lite dc = lite_of(pos_start(a));
    for (uint32_t gd = 0; dc.left > 0; ++gd) {
      const int sp = gd % kSP;
      if (!mbar_wait(&bars->pk_full[sp], (gd / kSP) & 1, abort_flag, a.err, 301)) break;
      const uint8_t* unit = ps + sp * kPStage + tile * (dc.bits == 3 ? 1536 : 1024);
      uint32_t v[32];
      uint32_t carry = 0;   // trellis state at the block start
      if (dc.bits == 2) q2_half_i8(unit, r0, half, 0, v);
      else if (!kAll || dc.bits == 3) q3_half_i8(unit, r0, half, 0, v);
      else t2_half_i8(unit, r0, half, 0, v, carry);
      // the A buffer is free once block gd - 1's MMAs are done
      if (gd > 0 && !mbar_wait(&bars->mma_done[(gd - 1) % kSX], ((gd - 1) / kSX) & 1, abort_flag, a.err, 302)) break;
      fence_after_sync();
      tmem_st32(lane_base + kACol, v);
      if (dc.bits == 2) q2_half_i8(unit, r0, half, 1, v);
      else if (!kAll || dc.bits == 3) q3_half_i8(unit, r0, half, 1, v);
      else t2_half_i8(unit, r0, half, 1, v, carry);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->pk_empty[sp]);
      tmem_st32(lane_base + kACol + 32, v);
      tmem_wait_st();
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->a_full);
      lite_next(dc, a);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 4-7, thread = row)
    // Per block, once its MMAs are done: the integer accumulator becomes fp32 partial dot
    // products times s[n,b] (all tokens of the row), summed in registers over the row group.
    const int t = threadIdx.x - 128;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * (warp - 4)) << 16);
    float acc[kSlots];
#pragma unroll
    for (int m = 0; m < kSlots; ++m) acc[m] = 0.f;
    uint32_t ng = 0;
    auto group_sync = [&](int code) {
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->group);
      return mbar_wait(&bars->group, (ng++) & 1, abort_flag, a.err, code);
    };
    // the scale of the block being finished is loaded one block ahead (its latency is an L2
    // round trip, longer than the work it would wait for): the fp16 scale with multiplier 1,
    // or the row scale d and the int8 multiplier q (s = d q, exact in fp32)
    auto scale_of = [&](const Pos& c, int& qv) -> uint16_t {
      const int n = c.rg * 128 + t;
      qv = 0;
      if (c.left <= 0 || n >= c.N) return (uint16_t)0;
      if (!kAll || c.scale_q == nullptr) {
        qv = 1;
        return __ldg(c.scales + (int64_t)n * c.B + c.b);
      }
      qv = __ldg(c.scale_q + (int64_t)n * c.B + c.b);
      return __ldg(c.scales + n);
    };
    Pos ec = pos_start(a);
    int qnext = 0;
    uint16_t snext = scale_of(ec, qnext);
    for (uint32_t ge = 0; ec.left > 0; ++ge) {
      const int n = ec.rg * 128 + t;
      const uint16_t sraw = snext;
      const int qraw = qnext;
      const int sc = ge % kSC;
      if (!mbar_wait(&bars->mma_done[ge % kSX], (ge / kSX) & 1, abort_flag, a.err, 303)) break;
      if (!mbar_wait(&bars->c_full[sc], (ge / kSC) & 1, abort_flag, a.err, 304)) break;
      fence_after_sync();
      const int4* rec = reinterpret_cast<const int4*>(cs + sc * 256);
      const float s = kAll ? half_bits_to_float(sraw) * (float)qraw : half_bits_to_float(sraw);
      // 2^E = f f2 with f a normal fp32 power of two and f2 = 2^-j (0 <= j <= 36): s f2 is exact
      // and normal, (s f2) v rounds once, and the last multiply by f rounds once more, gradually
      // into the subnormal range where the block's activations are that small
      constexpr int kChunk = XR < 16 ? XR : 16;   // columns per load
#pragma unroll
      for (int c0 = 0; c0 < XR; c0 += kChunk) {
        if (c0 / 4 >= M) break;
        uint32_t d[kChunk];
        tmem_ld_raw<kChunk>(lane_base + kDCol + (ge & 1) * kDCols + c0, d);
        tmem_wait_ld_regs<kChunk>(d);
#pragma unroll
        for (int mm = 0; mm < kChunk / 4; ++mm) {
          const int m = c0 / 4 + mm;
          if (m < M) {
            const int4 c = rec[m];
            // 2 sum_j 256^j D_j + C in fp32 (each D_j is exact in fp32: |D_j| < 2^23)
            float v = fmaf((float)(int)d[4 * mm], 2.f, __int_as_float(c.x));
            v = fmaf((float)(int)d[4 * mm + 1], 512.f, v);
            v = fmaf((float)(int)d[4 * mm + 2], 131072.f, v);
            v = fmaf((float)(int)d[4 * mm + 3], 33554432.f, v);
            acc[m] = fmaf((s * __int_as_float(c.z)) * v, __int_as_float(c.y), acc[m]);
          }
        }
      }
      fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars->d_empty[ge & 1]);
        mbar_arrive(&bars->c_empty[sc]);
      }
      if (ec.b + 1 == ec.B || ec.left == 1) {
        // the row group ends here (or this range does): y, or, for a row group that several
        // CTA ranges share, the combine through the partial slots (the last range to arrive
        // adds the pieces in range order)
        const DecProblem& pr = a.prob[ec.pi];
        const int64_t g0 = ec.g - ec.b;                     // first block of the row group
        const int G = (int)gridDim.x;
        const int c0 = range_cta_of(a, G, pr, g0), c1 = range_cta_of(a, G, pr, g0 + ec.B - 1);
        if (c0 == c1) {
          if (n < ec.N) {
#pragma unroll
            for (int m = 0; m < kSlots; ++m)
              if (m < M) ec.y[(int64_t)m * ec.N + n] = acc[m];
          }
        } else {
          // slot 0: the row group began before this range; slot 1: it continues after it
          const int slot = g0 < range_start_in(pr, M, range_cost_start(a, G, blockIdx.x)) ? 0 : 1;
          float* part = a.partial + ((int64_t)2 * blockIdx.x + slot) * M * 128;
#pragma unroll
          for (int m = 0; m < kSlots; ++m)
            if (m < M) part[m * 128 + t] = acc[m];
          __threadfence();
          if (!group_sync(305)) break;
          if (t == 0) bars->last_flag = (atomicAdd(a.counter + ec.grg, 1) == c1 - c0);
          if (!group_sync(306)) break;
          if (bars->last_flag) {
            __threadfence();
#pragma unroll
            for (int m = 0; m < kSlots; ++m) acc[m] = 0.f;
            for (int c = c0; c <= c1; ++c) {
              const int sl = g0 < range_start_in(pr, M, range_cost_start(a, G, c)) ? 0 : 1;
              const float* src = a.partial + ((int64_t)2 * c + sl) * M * 128;
#pragma unroll
              for (int m = 0; m < kSlots; ++m)
                if (m < M) acc[m] += __ldcg(src + m * 128 + t);
            }
            if (n < ec.N) {
#pragma unroll
              for (int m = 0; m < kSlots; ++m)
                if (m < M) ec.y[(int64_t)m * ec.N + n] = acc[m];
            }
            if (t == 0) a.counter[ec.grg] = 0;
          }
        }
#pragma unroll
        for (int m = 0; m < kSlots; ++m) acc[m] = 0.f;
      }
      pos_next(ec, a);
      snext = scale_of(ec, qnext);
    }
  }

  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 9) tmem_dealloc(tmem, kTmemCols);
}

// Preparation pass: one warp per (problem, block, token slot m < N/4). At the logical K position
// whose A byte holds c_k * 2^e (code k, position exponent e), the activation of token m becomes
// the integer n = x_k / 2^(E + e) (E = exponent of the block maximum - 30; values that are not
// multiples of 2^(E + e) round to the nearest, ties to even), split into four balanced signed
// bytes d_j (n = sum_j 256^j d_j, d_j in [-128, 127]). Limb j goes to B row 4m + j (two atoms of
// 128 K positions x N rows, 128-byte swizzle). After the atoms, one 16-byte correction record
// per slot: {C, bits of 2^E, 0, 0} with S_j = sum_k 2^e_k d_j[k] and C = -L sum_j 256^j S_j in
// fp32. The factor 2^E is stored as two powers of two, f = 2^max(E, -126) (normal) and
// f2 = 2^(E - max(E, -126)) >= 2^-36, so that no product in the epilogue leaves the normal range
// before its last multiply (E reaches -162 for subnormal bf16 activations). Slots m >= M hold zero
// limbs and a zero factor.
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
  int pe[8];   // position exponents: the A byte there holds c * 2^pe
  float amax = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int kl = 8 * lane + e;
    pe[e] = pr.bits == 2 ? q2_exp_at(kl) : (pr.bits == 3 ? q3_exp_at(kl) : t2_exp_at(kl));
    xv[e] = 0.f;
    if (m < M) {
      const int k = pr.bits == 3 ? q3_code_at(kl) : q2_code_at(kl);
      xv[e] = __bfloat162float(__ushort_as_bfloat16(__ldg(pr.x + (int64_t)m * pr.K + (int64_t)b * 256 + k)));
      amax = fmaxf(amax, fabsf(xv[e]));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  int ex = 0;
  if (amax > 0.f) frexpf(amax, &ex);   // amax in [2^(ex-1), 2^ex)
  const int E = ex - 30;                // |n| < 2^30
  uint32_t lw[4][2] = {{0u, 0u}, {0u, 0u}, {0u, 0u}, {0u, 0u}};
  int s[4] = {0, 0, 0, 0};                // S_j = sum_k 2^pe_k d_j[k]
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int n = amax > 0.f ? __float2int_rn(ldexpf(xv[e], -(E + pe[e]))) : 0;
    int rest = n;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int d = j < 3 ? (int)(int8_t)(rest & 0xFF) : rest;
      rest = (rest - d) >> 8;
      s[j] += d * (1 << pe[e]);
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
    // correction record of slot m: C = -L sum_j 256^j S_j (exact in fp64, one rounding to
    // fp32), then 2^E as the two factors f and f2
    const int L = pr.bits == 2 ? 3 : 7;
    const int Ehi = max(E, -126);
    const float f = (m < M && amax > 0.f) ? ldexpf(1.f, Ehi) : 0.f;
    const float f2 = ldexpf(1.f, E - Ehi);
    const double S = (double)s[0] + 256.0 * s[1] + 65536.0 * s[2] + 16777216.0 * s[3];
    reinterpret_cast<int4*>(dst + 256 * xrows)[m] =
        make_int4(__float_as_int((float)(-L * S)), __float_as_int(f), __float_as_int(f2), 0);
  }
}

}  // namespace

cudaError_t launch_prep_x(const DecArgs& a, int total_blocks, cudaStream_t stream) {
  const int warps = total_blocks * (decode_xrows(a.M) >> 2);
  prep_x_kernel<<<(warps + 7) / 8, 256, 0, stream>>>(a, total_blocks);
  return cudaGetLastError();
}

namespace {
template <int XR, bool kAll>
cudaError_t launch_xr(const DecArgs& a, int grid, cudaStream_t stream) {
  static bool set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!set[dev]) {
    cudaError_t e =
        cudaFuncSetAttribute(gemv_q_kernel<XR, kAll>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    // all of the unified L1/shared array as shared memory, so that three CTAs fit
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gemv_q_kernel<XR, kAll>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    set[dev] = true;
  }
  gemv_q_kernel<XR, kAll><<<grid, kThreads, kSmem, stream>>>(a);
  return cudaGetLastError();
}

template <bool kAll>
cudaError_t launch_feat(const DecArgs& a, int grid, cudaStream_t stream) {
  switch (decode_xrows(a.M)) {
    case 8: return launch_xr<8, kAll>(a, grid, stream);
    case 16: return launch_xr<16, kAll>(a, grid, stream);
    default: return launch_xr<32, kAll>(a, grid, stream);
  }
}
}  // namespace

cudaError_t launch_gemv_q(const DecArgs& a, int grid, cudaStream_t stream) {
  bool all = false;
  for (int i = 0; i < a.count; ++i) all = all || a.prob[i].bits == WR_FMT_T2 || a.prob[i].scale_q != nullptr;
  return all ? launch_feat<true>(a, grid, stream) : launch_feat<false>(a, grid, stream);
}

}  // namespace wr
