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
// once the epilogue has read block i - 2 from it (the 32-token form keeps one accumulator, see
// Cfg). Every wait is bounded.
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
constexpr int kSP = 4;   // packed stages: the 8 units of a row group's block (Cfg::kSPn may be fewer)
constexpr int kSX = 3;   // B tiles; also the MMA-done ring (Cfg::kSXn may be fewer)
constexpr int kSC = 4;   // correction records, 256 bytes

// The three forms of the kernel: a batch of Q2/Q3 problems with fp16 scales (the lean form), a
// batch that also holds trellis-coded problems or int8 block scales, and a ternary batch.
enum { kModeLean = 0, kModeAll = 1, kModeTern = 2 };

// Shared-memory and tensor-memory layout of one form. Q2/Q3: a block is 256 codes (A: 64 columns,
// B: two atoms of 128 K positions). Ternary: a block is one 320-trit unit (A: 80 columns, B: three
// atoms, the last half used), plus a 243-entry decode table replicated per lane (31 KB), so a CTA
// needs more room; at MMA N = 16 or 32 two CTAs share an SM.
// At MMA N = 64 or 128 (16 or 32 token slots, 2/3-bit forms only) the accumulators and B tiles
// grow: two CTAs per SM at N = 64 (256 tensor-memory columns), one at N = 128 (512). For a batch
// of many blocks the N = 128 form instead keeps one accumulator (ONE: 192 columns, in an
// allocation of 256) and shallower rings, so that two CTAs share an SM; block i + 1's MMAs then
// wait for the epilogue to read block i (decode_one_acc picks the form).
template <int XR, int MODE, bool ONE = false>
struct Cfg {
  static constexpr bool kT = MODE == kModeTern;
  static constexpr bool kOneAcc = ONE && !kT && XR == 128;
  static constexpr int kCtas = kT ? (XR > 8 ? 2 : 3) : (XR <= 32 ? 3 : (XR == 64 || kOneAcc ? 2 : 1));
  static constexpr int kSXn = kOneAcc ? 2 : kSX;   // B-tile stages (and the MMA-done ring)
  static constexpr int kSPn = kOneAcc ? 3 : kSP;   // weight stages
  static constexpr int kDBufs = kOneAcc ? 1 : 2;   // accumulators
  // accumulator of block g, and the parity of the epilogue's read that frees it for block g
  __device__ static constexpr int dbuf(uint32_t g) { return kDBufs == 2 ? (int)(g & 1u) : 0; }
  __device__ static constexpr uint32_t dfree_parity(uint32_t g) {
    return kDBufs == 2 ? (((g >> 1) & 1u) ^ 1u) : ((g & 1u) ^ 1u);
  }
  static constexpr int kPStage = 8 * (kT ? 1024 : 1536);
  static constexpr int kXStage = kT ? 3 * XR * 128 : (XR <= 32 ? 8 * 1024 : 2 * XR * 128);   // 1024-byte multiples
  static constexpr int kRec = kT ? 256 : (XR <= 64 ? 256 : 4 * XR);   // correction record per block
  static constexpr int kXOff = 0;
  static constexpr int kPOff = kXOff + kSXn * kXStage;
  static constexpr int kCOff = kPOff + kSPn * kPStage;
  static constexpr int kBarOff = kCOff + kSC * kRec;
  static constexpr int kSmem = kBarOff + 256 + 1024;   // + alignment slack
  static constexpr int kLutWords = kT ? 243 * 32 : 1;
  static constexpr int kACol = 0;
  static constexpr int kDCol = kT ? 96 : 64;           // two accumulators after the A buffer
  static constexpr int kDCols = kT ? XR : (XR < 32 ? 32 : XR);
  static constexpr int kTmemCols =
      kDCol + kDBufs * kDCols <= 128 ? 128 : (kDCol + kDBufs * kDCols <= 256 ? 256 : 512);
  static_assert(kCtas * (kSmem + 4 * kLutWords + 1024) <= 228 * 1024, "CTAs per SM by shared memory");
  static_assert(kCtas * kTmemCols <= 512, "tensor memory of an SM");
};

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
  // the block ranges (range_start in tc_kernels.cuh) and the problem of each range's first block
  // come computed from the host, so no role searches the problem table on the way in
  p.g = a.rs[blockIdx.x];
  p.left = (int)(a.rs[blockIdx.x + 1] - p.g);
  if (p.left <= 0) return p;
  const int lo = a.rp[blockIdx.x];
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

// The 8-state trellis format: the Q2 words, with the last three symbols' low bits carried
// through the row in code order.
__device__ __forceinline__ void t8_half_i8(const uint8_t* unit, int r0, int half, int h, uint32_t v[32],
                                           uint32_t& carry) {
#pragma unroll
  for (int qq = 0; qq < 2; ++qq) {
    const uint4 c = *reinterpret_cast<const uint4*>(unit + (32 * half + lane_pos(r0, 2 * h + qq)) * 16);
    decode_t8_word_i8(c.x, carry, v + 16 * qq + 0);
    decode_t8_word_i8(c.y, carry, v + 16 * qq + 4);
    decode_t8_word_i8(c.z, carry, v + 16 * qq + 8);
    decode_t8_word_i8(c.w, carry, v + 16 * qq + 12);
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

// Ternary quarter q (80 trits: 16 base-3 bytes v = sum_d c_d 3^d) of a row, as 20 A registers of
// signed bytes. The 4 packed words themselves, each byte flipped to v - 128 (one XOR), fill A
// columns 4q .. 4q+3; the first four digits of each byte, as t_d = c_d - 1, come from a 243-entry
// table (one copy per lane, so the 32 lookups of a warp hit 32 different banks) and fill columns
// 16 + 16q + j (byte j). With the activations arranged to match (the preparation pass), byte j
// contributes (v - 128) n_v + sum_{d<4} t_d (n_d - 3^d n_v) = sum_{d<4} t_d n_d + 81 t_4 n_v - 7 n_v,
// since v - 128 = sum_{d<=4} 3^d t_d - 7: its fifth trit through n_v, the activation of that trit
// divided by 81, and a constant 7 n_v that the correction record adds back in integers.
__device__ __forceinline__ void tern_quarter_i8(const uint8_t* unit, int r0, int half, int q, const uint32_t* lut,
                                                int lane, uint32_t raw[4], uint32_t lv[16]) {
  const uint4 c = *reinterpret_cast<const uint4*>(unit + (32 * half + lane_pos(r0, q)) * 16);
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) raw[i] = w[i] ^ 0x80808080u;
#pragma unroll
  for (int j = 0; j < 16; ++j) lv[j] = lut[(((w[j >> 2] >> (8 * (j & 3))) & 0xFFu) << 5) | (uint32_t)lane];
}

// The 10 K slices of one 320-trit block and their commit, issued by one elected lane: A slice j is
// the 8 columns at a_tmem + 8 j; B slice j is at byte 32 (j % 4) of atom j / 4 (atom16 = the atom
// size in 16-byte units); the first slice overwrites D.
__device__ __forceinline__ void mma10_i8_commit_elect(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                                      uint32_t atom16, uint32_t idesc, uint64_t* bar) {
  const uint64_t b4 = b_desc + atom16, b8 = b_desc + 2 * atom16;
  asm volatile(
      "{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n"
      " @e tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, 0;\n"
      " @e tcgen05.mma.cta_group::1.kind::i8 [%0], [%4], %5, %3, 1;\n"
      " @e tcgen05.mma.cta_group::1.kind::i8 [%0], [%6], %7, %3, 1;\n"
      " @e tcgen05.mma.cta_group::1.kind::i8 [%0], [%8], %9, %3, 1;\n"
      " @e tcgen05.mma.cta_group::1.kind::i8 [%0], [%10], %11, %3, 1;\n"
      " @e tcgen05.mma.cta_group::1.kind::i8 [%0], [%12], %13, %3, 1;\n"
      " @e tcgen05.mma.cta_group::1.kind::i8 [%0], [%14], %15, %3, 1;\n"
      " @e tcgen05.mma.cta_group::1.kind::i8 [%0], [%16], %17, %3, 1;\n"
      " @e tcgen05.mma.cta_group::1.kind::i8 [%0], [%18], %19, %3, 1;\n"
      " @e tcgen05.mma.cta_group::1.kind::i8 [%0], [%20], %21, %3, 1;\n"
      " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%22];\n}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(a_tmem + 8), "l"(b_desc + 2), "r"(a_tmem + 16), "l"(b_desc + 4),
      "r"(a_tmem + 24), "l"(b_desc + 6), "r"(a_tmem + 32), "l"(b4), "r"(a_tmem + 40), "l"(b4 + 2), "r"(a_tmem + 48),
      "l"(b4 + 4), "r"(a_tmem + 56), "l"(b4 + 6), "r"(a_tmem + 64), "l"(b8), "r"(a_tmem + 72), "l"(b8 + 2),
      "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tmem_st4(uint32_t taddr, const uint32_t* v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(v[0]), "r"(v[1]),
               "r"(v[2]), "r"(v[3])
               : "memory");
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

// XR: MMA N, 4 limb rows per token slot (8, 16 or 32 for M <= 2, 4, 8). MODE: kModeLean keeps
// only the Q2/Q3 decode branches and the fp16 scale load; kModeAll adds the trellis decode and
// int8 block scales; kModeTern is the ternary batch (its decode table, 320-trit blocks, signed A).
template <int XR, int MODE, bool ONE>
__global__ void __launch_bounds__(kThreads, Cfg<XR, MODE, ONE>::kCtas)
    gemv_q_kernel(const __grid_constant__ DecArgs a) {
  using C = Cfg<XR, MODE, ONE>;
  constexpr bool kAll = MODE == kModeAll;
  constexpr bool kT = C::kT;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t tlut[C::kLutWords];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* xs = smem + C::kXOff;
  uint8_t* ps = smem + C::kPOff;
  uint8_t* cs = smem + C::kCOff;
  Bars* bars = reinterpret_cast<Bars*>(smem + C::kBarOff);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &bars->abort_flag;
  constexpr int kSlots = XR / 4;       // token slots
  const int M = a.M;

  if constexpr (kT) {
    // decode table: entry v holds t_d = c_d - 1 (d = 0..3) of the base-3 byte v as signed bytes,
    // one copy per lane (word 32 v + lane)
    for (int i = threadIdx.x; i < 243 * 32; i += kThreads) {
      int v = i >> 5;
      uint32_t e = 0;
#pragma unroll
      for (int d = 0; d < 4; ++d) {
        e |= (uint32_t)(uint8_t)(int8_t)(v % 3 - 1) << (8 * d);
        v /= 3;
      }
      tlut[i] = e;
    }
  }

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kSPn; ++i) {
      mbar_init(&bars->pk_full[i], 1);
      mbar_init(&bars->pk_empty[i], 4);
    }
    for (int i = 0; i < C::kSXn; ++i) {
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
  if (warp == 9) tmem_alloc(&bars->tmem_base, C::kTmemCols);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 8) {
    // ------------------------------------------------------------ copy warp (whole warp walks the
    // blocks, one elected lane issues): packed weights (a ring of kSPn blocks), prepared B tiles
    // and their correction records (a ring of kSXn blocks)
    constexpr uint32_t bbytes = (kT ? 384u : 256u) * XR;
    constexpr uint32_t xtb = bbytes + (uint32_t)C::kRec;   // prepared tile: B atoms, then corrections
    Pos cp = pos_start(a), cx = cp;            // next block to copy: weights, activations
    const uint32_t nblocks = cp.left > 0 ? (uint32_t)cp.left : 0u;
    uint32_t np = 0, nx = 0;                   // weight copies, activation copies issued
    // the weights are read once and the activation tiles by every row group of their problem:
    // keep the tiles in L2 ahead of the weights streaming through it
    const uint64_t pol_w = l2_policy_evict_first(), pol_x = l2_policy_evict_last();
    bool ok = true;
    while (ok && (np < nblocks || nx < nblocks)) {
      if (np < nblocks) {
        // weight stage np % kSPn: free once the decode warps have read block np - kSPn
        const int sp = np % C::kSPn;
        if (!(ok = mbar_wait_bg(&bars->pk_empty[sp], ((np / C::kSPn) & 1) ^ 1, abort_flag, a.err, 101))) break;
        const int ub = cp.bits == 3 ? 1536 : 1024;
        const int ntile = min(8, (cp.N + 15) / 16 - cp.rg * 8);
        if (elect_one()) {
          mbar_arrive_expect_tx(&bars->pk_full[sp], ntile * ub);
          bulk_load_hint(ps + sp * C::kPStage, cp.packed + ((int64_t)cp.rg * 8 * cp.B + (int64_t)cp.b * ntile) * ub,
                         ntile * ub, &bars->pk_full[sp], pol_w);
        }
        __syncwarp();
        pos_next(cp, a);
        ++np;
      }
      if (nx < nblocks && np >= min(nblocks, (uint32_t)C::kSPn)) {
        // the activation tiles come from the preparation pass, which may still be running (the
        // kernel is launched as its programmatic dependent): the first weight copies above are
        // issued before waiting for it
        if (nx == 0) grid_dependency_wait();
        // activation stage nx % kSXn: free once block nx - kSXn's MMAs are done; correction slot
        // nx % kSC once the epilogue has read block nx - kSC
        const int sx = nx % C::kSXn, sc = nx % kSC;
        if (!(ok = mbar_wait_bg(&bars->mma_done[sx], ((nx / C::kSXn) & 1) ^ 1, abort_flag, a.err, 102))) break;
        if (!(ok = mbar_wait_bg(&bars->c_empty[sc], ((nx / kSC) & 1) ^ 1, abort_flag, a.err, 103))) break;
        const uint8_t* xsrc = cx.xt + (int64_t)cx.b * xtb;
        if (elect_one()) {
          mbar_arrive_expect_tx(&bars->x_full[sx], bbytes);
          bulk_load_hint(xs + sx * C::kXStage, xsrc, bbytes, &bars->x_full[sx], pol_x);
          mbar_arrive_expect_tx(&bars->c_full[sc], C::kRec);
          bulk_load_hint(cs + sc * C::kRec, xsrc + bbytes, C::kRec, &bars->c_full[sc], pol_x);
        }
        __syncwarp();
        pos_next(cx, a);
        ++nx;
      }
    }
    if (!ok) {
      // aborted: let the copies in flight land before the CTA exits
      for (uint32_t k = np > C::kSPn ? np - C::kSPn : 0; k < np; ++k)
        mbar_wait_drain(&bars->pk_full[k % C::kSPn], (k / C::kSPn) & 1);
      for (uint32_t k = nx > C::kSXn ? nx - C::kSXn : 0; k < nx; ++k)
        mbar_wait_drain(&bars->x_full[k % C::kSXn], (k / C::kSXn) & 1);
      for (uint32_t k = nx > kSC ? nx - kSC : 0; k < nx; ++k) mbar_wait_drain(&bars->c_full[k % kSC], (k / kSC) & 1);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA warp (whole warp, one lane issues)
    const uint64_t bdesc0 = smem_desc_sw128(xs);
    constexpr uint32_t idesc = kT ? idesc_i8s_m128(XR) : idesc_i8_m128(XR);
    constexpr uint32_t atom16 = (uint32_t)(XR * 128) >> 4;
    const int64_t span = (int64_t)a.rs[blockIdx.x + 1] - a.rs[blockIdx.x];
    const uint32_t nblocks = span > 0 ? (uint32_t)span : 0u;
    uint32_t gm = 0;
    bool ok = true;
    for (; gm < nblocks; ++gm) {
      const int sx = gm % C::kSXn;
      // the B tile and the accumulator are normally ready long before the codes: wait for them
      // first, so that the wait for the A handoff is the last one before the MMAs
      if (!(ok = mbar_wait(&bars->x_full[sx], (gm / C::kSXn) & 1, abort_flag, a.err, 202))) break;
      // the accumulator of block gm was read by the epilogue warps (block gm - 2, or gm - 1 with one accumulator)
      if (!(ok = mbar_wait(&bars->d_empty[C::dbuf(gm)], C::dfree_parity(gm), abort_flag, a.err, 203))) break;
      if (!(ok = mbar_wait(&bars->a_full, gm & 1, abort_flag, a.err, 201))) break;
      fence_after_sync();
      if constexpr (kT)
        mma10_i8_commit_elect(tmem + C::kDCol + C::dbuf(gm) * C::kDCols, tmem + C::kACol,
                              bdesc0 + (uint64_t)((sx * C::kXStage) >> 4), atom16, idesc, &bars->mma_done[sx]);
      else
        mma8_i8_commit_elect(tmem + C::kDCol + C::dbuf(gm) * C::kDCols, tmem + C::kACol,
                             bdesc0 + (uint64_t)((sx * C::kXStage) >> 4), atom16, idesc, &bars->mma_done[sx]);
    }
    // the MMAs already issued finish before tensor memory is released
    if (!ok && gm > 0) mbar_wait_drain(&bars->mma_done[(gm - 1) % C::kSXn], ((gm - 1) / C::kSXn) & 1);
  } else if (warp < 4) {
    // ------------------------------------------------------------ decode (warps 0-3, thread = row)
    const int t = threadIdx.x;                          // row in the row group = TMEM lane
    const int tile = t >> 4, r = t & 15, r0 = r & 7, half = r >> 3;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * warp) << 16);
    Lite dc = lite_of(pos_start(a));
    for (uint32_t gd = 0; dc.left > 0; ++gd) {
      const int sp = gd % C::kSPn;
      if (!mbar_wait(&bars->pk_full[sp], (gd / C::kSPn) & 1, abort_flag, a.err, 301)) break;
      if constexpr (kT) {
        // ternary: four quarters of 20 columns (4 packed words, then 16 table entries), each
        // stored as soon as it is decoded
        const uint8_t* unit = ps + sp * C::kPStage + tile * 1024;
        uint32_t raw[4], lv[16];
        tern_quarter_i8(unit, r0, half, 0, tlut, lane, raw, lv);
        // the A buffer is free once block gd - 1's MMAs are done
        if (gd > 0 &&
            !mbar_wait(&bars->mma_done[(gd - 1) % C::kSXn], ((gd - 1) / C::kSXn) & 1, abort_flag, a.err, 302))
          break;
        fence_after_sync();
        tmem_st4(lane_base + C::kACol, raw);
        tmem_st16(lane_base + C::kACol + 16, lv);
#pragma unroll
        for (int q = 1; q < 4; ++q) {
          tern_quarter_i8(unit, r0, half, q, tlut, lane, raw, lv);
          tmem_st4(lane_base + C::kACol + 4 * q, raw);
          tmem_st16(lane_base + C::kACol + 16 + 16 * q, lv);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->pk_empty[sp]);
      } else {
        const uint8_t* unit = ps + sp * C::kPStage + tile * (dc.bits == 3 ? 1536 : 1024);
        uint32_t v[32];
        uint32_t carry = 0;   // trellis state at the block start (both trellis formats)
        if (dc.bits == 2) q2_half_i8(unit, r0, half, 0, v);
        else if (!kAll || dc.bits == 3) q3_half_i8(unit, r0, half, 0, v);
        else if (dc.bits == WR_FMT_T2) t2_half_i8(unit, r0, half, 0, v, carry);
        else t8_half_i8(unit, r0, half, 0, v, carry);
        // the A buffer is free once block gd - 1's MMAs are done
        if (gd > 0 &&
            !mbar_wait(&bars->mma_done[(gd - 1) % C::kSXn], ((gd - 1) / C::kSXn) & 1, abort_flag, a.err, 302))
          break;
        fence_after_sync();
        tmem_st32(lane_base + C::kACol, v);
        if (dc.bits == 2) q2_half_i8(unit, r0, half, 1, v);
        else if (!kAll || dc.bits == 3) q3_half_i8(unit, r0, half, 1, v);
        else if (dc.bits == WR_FMT_T2) t2_half_i8(unit, r0, half, 1, v, carry);
        else t8_half_i8(unit, r0, half, 1, v, carry);
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->pk_empty[sp]);
        tmem_st32(lane_base + C::kACol + 32, v);
      }
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
      if (kT) {   // ternary: alpha, one scale per row
        qv = 1;
        return __ldg(c.scales + n);
      }
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
      if (!mbar_wait(&bars->mma_done[ge % C::kSXn], (ge / C::kSXn) & 1, abort_flag, a.err, 303)) break;
      if (!mbar_wait(&bars->c_full[sc], (ge / kSC) & 1, abort_flag, a.err, 304)) break;
      fence_after_sync();
      const int4* rec = reinterpret_cast<const int4*>(cs + sc * C::kRec);
      const float s = kAll ? half_bits_to_float(sraw) * (float)qraw : half_bits_to_float(sraw);
      // 2^E = f f2 with f a normal fp32 power of two and f2 = 2^-j (0 <= j <= 36): s f2 is exact
      // and normal, (s f2) v rounds once, and the last multiply by f rounds once more, gradually
      // into the subnormal range where the block's activations are that small
      constexpr int kChunk = XR < 16 ? XR : 16;   // columns per load
#pragma unroll
      for (int c0 = 0; c0 < XR; c0 += kChunk) {
        if (c0 / 4 >= M) break;
        uint32_t d[kChunk];
        tmem_ld_raw<kChunk>(lane_base + C::kDCol + C::dbuf(ge) * C::kDCols + c0, d);
        tmem_wait_ld_regs<kChunk>(d);
#pragma unroll
        for (int mm = 0; mm < kChunk / 4; ++mm) {
          const int m = c0 / 4 + mm;
          if (kT && m < M) {
            // ternary: each limb sum plus its integer correction is exact; sum_j 256^j of those
            // is sum_k t_k n_k, zero when every t of the block is zero
            const int4 cr = rec[2 * m], ff = rec[2 * m + 1];
            float v = (float)((int)d[4 * mm] + cr.x);
            v = fmaf((float)((int)d[4 * mm + 1] + cr.y), 256.f, v);
            v = fmaf((float)((int)d[4 * mm + 2] + cr.z), 65536.f, v);
            v = fmaf((float)((int)d[4 * mm + 3] + cr.w), 16777216.f, v);
            acc[m] = fmaf((s * __int_as_float(ff.y)) * v, __int_as_float(ff.x), acc[m]);
          } else if (m < M) {
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
        mbar_arrive(&bars->d_empty[C::dbuf(ge)]);
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
          const int slot = g0 < a.rs[blockIdx.x] ? 0 : 1;
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
              const int sl = g0 < a.rs[c] ? 0 : 1;
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
  if (warp == 9) tmem_dealloc(tmem, C::kTmemCols);
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
  grid_launch_dependents();   // the GEMV may start its prologue and weight copies now
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

// Ternary preparation pass, with the rotation fused in: one warp per (problem, 320-trit unit b,
// token slot m < N/4). The warp applies R = (1/sqrt(128)) H D to x (fp32, the sign mask first,
// then a Walsh-Hadamard butterfly: lane l holds positions 4l .. 4l+3 of a 128-block) on the three
// 128-blocks that the unit overlaps, keeps x' = R x in shared memory, and writes the B tile of the
// unit in the K order of the decoded A columns (tern_quarter_i8): with E = exponent(max |x'| over
// the unit) - 30 and n_k = x'_k / 2^E rounded to the nearest integer (|n| < 2^30),
//   A column 4q + r, byte p        (v-slot of byte j = 4r + p of quarter q):  n_v = x'_(80q+5j+4) / (81 2^E), rounded
//   A column 16 + 16q + j, byte d  (digit d of byte j of quarter q):           n_(80q+5j+d) - 3^d n_v(j)
// each as four balanced signed limbs (B rows 4m + limb). Then the correction record of slot m:
// {7 S_0, 7 S_1, 7 S_2, 7 S_3} (S_j = sum over the v-slots of limb j of n_v), then the two factors
// of 2^E as in the 2/3-bit record. Every t_k x'_k then reaches the MMA exactly, up to the rounding
// of n_k (half a unit of 2^E) and, for the fifth trit of a byte, of 81 n_v (40.5 units).
__global__ void __launch_bounds__(256) prep_t_kernel(const __grid_constant__ DecArgs a, int total_blocks) {
  grid_launch_dependents();   // the GEMV may start its prologue and weight copies now
  __shared__ float xbuf[8][384];
  const int lane = threadIdx.x & 31, wi = threadIdx.x >> 5;
  const int M = a.M;
  const int xrows = decode_xrows(M), slots = xrows >> 2;
  const int w = blockIdx.x * 8 + wi;
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
  uint8_t* dst = pr.xt + (int64_t)b * xtile_bytes(true, M);
  float* xb = xbuf[wi];
  const int64_t k0 = (int64_t)320 * b;
  const int64_t hb0 = k0 / 128;   // first 128-block the unit overlaps; the unit starts 0 or 64 into it
  const float inv = 0.08838834764831845f;   // 1/sqrt(128)
#pragma unroll
  for (int h = 0; h < 3; ++h) {
    const int64_t kb = (hb0 + h) * 128;
    float v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t k = kb + 4 * lane + i;
      float xv = 0.f;
      if (m < M && k < pr.K) {   // K is a multiple of 128: a 128-block is all in or all out
        xv = __bfloat162float(__ushort_as_bfloat16(__ldg(pr.x + (int64_t)m * pr.K + k)));
        if ((__ldg(pr.signs + (k >> 5)) >> (k & 31)) & 1u) xv = -xv;
      }
      v[i] = xv;
    }
    float t0 = v[0] + v[1], t1 = v[0] - v[1], t2 = v[2] + v[3], t3 = v[2] - v[3];
    v[0] = t0 + t2; v[2] = t0 - t2; v[1] = t1 + t3; v[3] = t1 - t3;
#pragma unroll
    for (int sft = 1; sft < 32; sft <<= 1) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float o = __shfl_xor_sync(0xffffffffu, v[i], sft);
        v[i] = (lane & sft) ? o - v[i] : v[i] + o;
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) xb[h * 128 + 4 * lane + i] = v[i] * inv;
  }
  __syncwarp();
  const float* xu = xb + (int)(k0 - hb0 * 128);   // x' of unit position u = xu[u], u < 320
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 10; ++i) amax = fmaxf(amax, fabsf(xu[lane + 32 * i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  int ex = 0;
  if (amax > 0.f) frexpf(amax, &ex);
  const int E = ex - 30;
  const bool live = amax > 0.f;
  auto n_of = [&](int u) -> int { return live ? __float2int_rn(ldexpf(xu[u], -E)) : 0; };
  auto nv_of = [&](int u) -> int { return live ? __double2int_rn(ldexp((double)xu[u], -E) / 81.0) : 0; };
  int sv[4] = {0, 0, 0, 0};
  for (int g = lane; g < 40; g += 32) {   // 8 consecutive K positions 8g .. 8g+7 of the tile
    uint32_t lw[4][2] = {{0u, 0u}, {0u, 0u}, {0u, 0u}, {0u, 0u}};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int kl = 8 * g + e, col = kl >> 2, p = kl & 3;
      int bv;
      bool vslot;
      if (col < 16) {
        const int q = col >> 2, j = 4 * (col & 3) + p;
        bv = nv_of(80 * q + 5 * j + 4);
        vslot = true;
      } else {
        const int q = (col - 16) >> 4, j = (col - 16) & 15;
        const int pw = p == 0 ? 1 : (p == 1 ? 3 : (p == 2 ? 9 : 27));
        bv = n_of(80 * q + 5 * j + p) - pw * nv_of(80 * q + 5 * j + 4);
        vslot = false;
      }
      int rest = bv;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int d = j < 3 ? (int)(int8_t)(rest & 0xFF) : rest;
        rest = (rest - d) >> 8;
        if (vslot) sv[j] += d;
        lw[j][e >> 2] |= ((uint32_t)d & 0xFFu) << (8 * (e & 3));
      }
    }
    const int atom = (8 * g) >> 7, within = (8 * g) & 127, chunk = within >> 4, off = within & 15;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int row = 4 * m + j;
      *reinterpret_cast<uint2*>(dst + atom * xrows * 128 + row * 128 + ((chunk ^ (row & 7)) << 4) + off) =
          make_uint2(lw[j][0], lw[j][1]);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
    for (int j = 0; j < 4; ++j) sv[j] += __shfl_xor_sync(0xffffffffu, sv[j], o);
  }
  if (lane == 0) {
    const int Ehi = max(E, -126);
    const float f = (m < M && live) ? ldexpf(1.f, Ehi) : 0.f;
    const float f2 = ldexpf(1.f, E - Ehi);
    int4* rec = reinterpret_cast<int4*>(dst + 3 * xrows * 128);
    rec[2 * m] = make_int4(7 * sv[0], 7 * sv[1], 7 * sv[2], 7 * sv[3]);
    rec[2 * m + 1] = make_int4(__float_as_int(f), __float_as_int(f2), 0, 0);
  }
}

}  // namespace

cudaError_t launch_prep_x(const DecArgs& a, int total_blocks, cudaStream_t stream) {
  const int warps = total_blocks * (decode_xrows(a.M) >> 2);
  if (a.count > 0 && a.prob[0].bits == 1)
    prep_t_kernel<<<(warps + 7) / 8, 256, 0, stream>>>(a, total_blocks);
  else
    prep_x_kernel<<<(warps + 7) / 8, 256, 0, stream>>>(a, total_blocks);
  return cudaGetLastError();
}

namespace {
template <int XR, int MODE, bool ONE = false>
cudaError_t launch_xr(const DecArgs& a, int grid, cudaStream_t stream) {
  using C = Cfg<XR, MODE, ONE>;
  static bool set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(gemv_q_kernel<XR, MODE, ONE>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    // all of the unified L1/shared array as shared memory, so that the CTAs fit
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gemv_q_kernel<XR, MODE, ONE>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    set[dev] = true;
  }
  // a programmatic dependent of the preparation pass launched just before it on the stream
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemv_q_kernel<XR, MODE, ONE>, a);
}

template <int MODE>
cudaError_t launch_mode(const DecArgs& a, int grid, cudaStream_t stream) {
  switch (decode_xrows(a.M)) {
    case 8: return launch_xr<8, MODE>(a, grid, stream);
    case 16: return launch_xr<16, MODE>(a, grid, stream);
    case 32: return launch_xr<32, MODE>(a, grid, stream);
    case 64:
      if constexpr (MODE != kModeTern) return launch_xr<64, MODE>(a, grid, stream);
      return cudaErrorInvalidValue;
    default:
      if constexpr (MODE != kModeTern) {
        if (decode_one_acc(a.M, a.total)) return launch_xr<128, MODE, true>(a, grid, stream);
        return launch_xr<128, MODE>(a, grid, stream);
      }
      return cudaErrorInvalidValue;
  }
}
}  // namespace

// A batch is either ternary (every problem) or 2/3-bit; the 2/3-bit form is chosen by whether
// any problem is trellis-coded or has int8 block scales.
cudaError_t launch_gemv_q(const DecArgs& a, int grid, cudaStream_t stream) {
  if (a.count > 0 && a.prob[0].bits == 1) return launch_mode<kModeTern>(a, grid, stream);
  bool all = false;
  for (int i = 0; i < a.count; ++i)
    all = all || a.prob[i].bits == WR_FMT_T2 || a.prob[i].bits == WR_FMT_T8 || a.prob[i].scale_q != nullptr;
  return all ? launch_mode<kModeAll>(a, grid, stream) : launch_mode<kModeLean>(a, grid, stream);
}

// CTAs of one wave of the decode kernel for a batch of this kind on a 148-SM part.
int decode_ctas_per_sm(bool ternary, int M, int64_t total_blocks) {
  const int xr = decode_xrows(M);
  if (ternary) return xr > 8 ? 2 : 3;
  if (xr <= 32) return 3;
  return xr == 64 || decode_one_acc(M, total_blocks) ? 2 : 1;
}

}  // namespace wr
