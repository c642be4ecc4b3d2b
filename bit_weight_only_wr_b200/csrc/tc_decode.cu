// Decode GEMV (M <= 8 tokens) on tcgen05, for one problem or a batch of independent problems.
//
// Decoding a token reads every weight once ("How We Shrank an AI Model by 85%...", section
// "Results": generating a token is mostly reading the weights from memory), so the kernel is a
// weight stream: each CTA walks a list of work items (problem, 128-row group, range of
// 256-code blocks) and keeps its rings full across item and problem boundaries, so the fixed
// latency of one small GEMV hides behind the loads of the next.
//
//   y[m,n] = sum_b s[n,b] sum_{k in b} g[n,k] x[m,k]      (2/3-bit odd grid, fp16 scales)
//   y[m,n] = alpha[n] sum_k t[n,k] (R x[m,:])[k]          (ternary, rotated basis)
//
// 2/3-bit path: integer tensor cores. The weights go to tensor memory as their unsigned codes
// c (one byte each; kind::i8, K = 32 per MMA). The activations of a (token, block) are the
// integers n_k = x_k / 2^E for a per-(token, block) exponent E = exponent(max |x|) - 29,
// written as four balanced signed bytes (limbs) d_j, n = sum_j 256^j d_j; limb j of token m is
// B row (N/4) j + m, with N = 8, 16 or 32 MMA columns for M <= 2, 4 or 8 tokens. Every product and every block sum is an exact integer,
//   D_j[n] = sum_k c[n,k] d_j[k],   and with g = 2c - L:
//   sum_k g x = 2^E sum_j 256^j (2 D_j - L S_j),   S_j = sum_k d_j[k],
// the last step in fp32. Values below 2^E (more than 2^29 under the block maximum) round to a
// multiple of 2^E: an error of at most 2^-30 max|x| per element.
// Ternary path: bf16 tensor cores, t exact in bf16, R x as hi + lo bf16 in B rows m and 8 + m.
//
// Warp roles (448 threads, two CTAs per SM):
//   warps 0-7  decode: thread = weight row (TMEM lane); warps w and w+4 share a lane quarter and
//              take the two halves of each block. Codes leave shared memory as bytes (for 2-bit,
//              one shift and one AND per 4 codes) and are stored to tensor memory.
//   warp 12    producer: per block one bulk copy for the 8 packed units of the row group, one
//              for the B part of the prepared activation tile and one for its per-token
//              corrections (a separate, deeper ring, read by the epilogue).
//   warp 13    allocates TMEM and issues the MMAs from one thread.
//   warps 8-11 epilogue: per block, the integer partials turned into the block's fp32 dot
//              products and multiplied by s[n,b] (ternary: hi + lo columns once per item, times
//              alpha), summed in registers; then y, or a split-K combine through the workspace
//              (the last of the P pieces to arrive adds them in order p = 0..P-1).
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

constexpr int kThreads = 448;  // 8 decode, 4 epilogue, producer, MMA warps
constexpr int kSP = 5;         // packed stages
constexpr int kSX = 6;         // activation stages
constexpr int kSC = 8;         // correction stages (2/3-bit): 256 bytes each

template <bool T>
struct DL {  // decode-kernel layout
  static constexpr int kUnitK = T ? 320 : 256;
  static constexpr int kBN = T ? 16 : 32;                       // accumulator columns (MMA N <= kBN)
  static constexpr int kXStage = T ? 10 * 1024 : 8 * 1024;     // B part of one prepared tile
  static constexpr int kPStage = T ? 8 * 1024 : 8 * 1536;       // 8 units of the widest format
  static constexpr int kXOff = 0;
  static constexpr int kPOff = kSX * kXStage;
  static constexpr int kCOff = kPOff + kSP * kPStage;
  static constexpr int kBarOff = kCOff + kSC * 256;
  // + barriers and alignment slack, padded so that at most two CTAs share an SM (each holds
  // 256 of the SM's 512 TMEM columns)
  static constexpr int kSmemRaw = kBarOff + 1024 + 1024;
  static constexpr int kSmem = kSmemRaw < 80 * 1024 ? 80 * 1024 : kSmemRaw;
  // tensor memory: A buffers, then two accumulators
  static constexpr int kQuarterCols = T ? 40 : 16;
  static constexpr int kABuf = T ? 2 * kQuarterCols : 4 * kQuarterCols;   // T: half block; Q: block
  static constexpr int kDCol = 2 * kABuf;
  static constexpr int kTmemCols = 256;
  static_assert(kDCol + 2 * kBN <= kTmemCols, "tensor memory budget");
};

struct Bars {
  uint64_t pk_full[kSP], pk_empty[kSP], x_full[kSX], x_empty[kSX];
  uint64_t a_full[2], a_empty[2], d_full[2], d_empty[2];
  uint64_t c_full[kSC], c_empty[kSC];
  uint32_t tmem_base;
  int abort_flag;
  int last_flag;
};

struct Item {
  int pi, rg, p, b0, b1;
};

__device__ __forceinline__ Item find_item(const DecArgs& a, int it) {
  int lo = 0, hi = a.count - 1;
  while (lo < hi) {  // last problem with item_base <= it
    const int mid = (lo + hi + 1) >> 1;
    if (a.prob[mid].item_base <= it) lo = mid;
    else hi = mid - 1;
  }
  const DecProblem& pr = a.prob[lo];
  Item r;
  r.pi = lo;
  const int local = it - pr.item_base;
  r.p = local % pr.P;
  r.rg = local / pr.P;
  r.b0 = (int)((int64_t)pr.B * r.p / pr.P);
  r.b1 = (int)((int64_t)pr.B * (r.p + 1) / pr.P);
  return r;
}

// Row-of-a-quarter decoders (thread = row); see the packed layout in include/wr.h.
__device__ __forceinline__ void q2_quarter_i8(const uint8_t* unit, int r0, int half, int q, uint32_t v[16]) {
  const uint4 c = *reinterpret_cast<const uint4*>(unit + (32 * half + 4 * r0 + q) * 16);
  decode_q2_word_i8(c.x, v + 0);
  decode_q2_word_i8(c.y, v + 4);
  decode_q2_word_i8(c.z, v + 8);
  decode_q2_word_i8(c.w, v + 12);
}

__device__ __forceinline__ void q3_quarter_i8(const uint8_t* unit, int r0, int half, int q, uint32_t v[16]) {
  const int l = 4 * r0 + q;
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
  decode_q3_group_i8(w, v);
  decode_q3_group_i8(w + 3, v + 8);
}

__device__ __forceinline__ void t_quarter(const uint8_t* unit, int r0, int half, int q, const uint32_t* lut_lo,
                                          const uint32_t* lut_hi, uint32_t v[40]) {
  const uint4 c = *reinterpret_cast<const uint4*>(unit + (32 * half + 4 * r0 + q) * 16);
  const uint32_t wv[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
  for (int w = 0; w < 4; ++w) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t e = lut_lo[(wv[w] >> (16 * h)) & 0xFFu] | lut_hi[(wv[w] >> (16 * h + 8)) & 0xFFu];
      decode_trit_pairs(e, v + 5 * (2 * w + h));
    }
  }
}

__device__ __forceinline__ uint32_t trit_entry(int v) {
  const int slot[5] = {1, 3, 5, 9, 11};
  uint32_t e = 0;
  for (int d = 0; d < 5; ++d) {
    e |= (uint32_t)(v % 3) << slot[d];
    v /= 3;
  }
  return e;
}

template <bool T>
__global__ void __launch_bounds__(kThreads, 2) decode_kernel(const __grid_constant__ DecArgs a) {
  using L = DL<T>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* xs = smem + L::kXOff;
  uint8_t* ps = smem + L::kPOff;
  uint8_t* cs = smem + L::kCOff;
  Bars* bars = reinterpret_cast<Bars*>(smem + L::kBarOff);
  __shared__ uint32_t lut_lo[T ? 256 : 1], lut_hi[T ? 256 : 1];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &bars->abort_flag;
  const int M = a.M;
  const int xrows = decode_xrows(M);   // 2/3-bit: MMA N and rows per B atom

  if (T) {
    for (int i = threadIdx.x; i < 256; i += kThreads) {
      const uint32_t e = i < 243 ? trit_entry(i) : 0u;
      lut_lo[i] = e;
      lut_hi[i] = e << 16;
    }
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < kSP; ++i) {
      mbar_init(&bars->pk_full[i], 1);
      mbar_init(&bars->pk_empty[i], 8);
    }
    for (int i = 0; i < kSX; ++i) {
      mbar_init(&bars->x_full[i], 1);
      mbar_init(&bars->x_empty[i], 1);   // released by the MMA
    }
    for (int i = 0; i < kSC; ++i) {
      mbar_init(&bars->c_full[i], 1);
      mbar_init(&bars->c_empty[i], 4);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->a_full[i], T ? 4 : 8);
      mbar_init(&bars->a_empty[i], 1);
      mbar_init(&bars->d_full[i], 1);
      mbar_init(&bars->d_empty[i], 4);
    }
    bars->abort_flag = 0;
    bars->last_flag = 0;
    fence_barrier_init();
  }
  if (warp == 13) tmem_alloc(&bars->tmem_base, L::kTmemCols);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 12) {
    // ------------------------------------------------------------ producer (one thread)
    if (lane == 0) {
      uint32_t gb = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < a.items && ok && !*abort_flag; it += gridDim.x) {
        const Item im = find_item(a, it);
        const DecProblem& pr = a.prob[im.pi];
        const int ub = T ? 1024 : (pr.bits == 2 ? 1024 : 1536);
        const int ntile = min(8, (pr.N + 15) / 16 - im.rg * 8);
        const uint32_t xtb = (uint32_t)xtile_bytes(T, M);
        for (int b = im.b0; b < im.b1; ++b, ++gb) {
          const int sx = gb % kSX;
          if (!(ok = mbar_wait(&bars->x_empty[sx], ((gb / kSX) & 1) ^ 1, abort_flag, a.err, 101))) break;
          const uint8_t* xsrc = pr.xt + (int64_t)b * xtb;
          if (T) {
            mbar_arrive_expect_tx(&bars->x_full[sx], xtb);
            bulk_load(xs + sx * L::kXStage, xsrc, xtb, &bars->x_full[sx]);
          } else {
            const uint32_t bbytes = 2u * xrows * 128u;
            mbar_arrive_expect_tx(&bars->x_full[sx], bbytes);
            bulk_load(xs + sx * L::kXStage, xsrc, bbytes, &bars->x_full[sx]);
            const int sc = gb % kSC;
            if (!(ok = mbar_wait(&bars->c_empty[sc], ((gb / kSC) & 1) ^ 1, abort_flag, a.err, 103))) break;
            mbar_arrive_expect_tx(&bars->c_full[sc], 256);
            bulk_load(cs + sc * 256, xsrc + bbytes, 256, &bars->c_full[sc]);
          }
          // the ntile units of this row group and block are adjacent: one copy
          const int sp = gb % kSP;
          if (!(ok = mbar_wait(&bars->pk_empty[sp], ((gb / kSP) & 1) ^ 1, abort_flag, a.err, 102))) break;
          mbar_arrive_expect_tx(&bars->pk_full[sp], ntile * ub);
          bulk_load(ps + sp * L::kPStage, pr.packed + ((int64_t)im.rg * 8 * pr.B + (int64_t)b * ntile) * ub,
                    ntile * ub, &bars->pk_full[sp]);
        }
      }
    }
  } else if (warp == 13) {
    // ------------------------------------------------------------ MMA issuer (one thread)
    if (lane == 0) {
      const uint64_t bdesc0 = smem_desc_sw128(xs);
      uint32_t gb = 0, gi = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < a.items && ok && !*abort_flag; it += gridDim.x, ++gi) {
        const Item im = find_item(a, it);
        uint32_t dbuf = 0;
        if (T) {
          dbuf = gi & 1;
          ok = mbar_wait(&bars->d_empty[dbuf], ((gi >> 1) & 1) ^ 1, abort_flag, a.err, 201);
        }
        for (int b = im.b0; b < im.b1 && ok; ++b, ++gb) {
          if (!T) {
            dbuf = gb & 1;
            if (!(ok = mbar_wait(&bars->d_empty[dbuf], ((gb >> 1) & 1) ^ 1, abort_flag, a.err, 202))) break;
          }
          const int sx = gb % kSX;
          if (!(ok = mbar_wait(&bars->x_full[sx], (gb / kSX) & 1, abort_flag, a.err, 203))) break;
          const uint32_t dcol = tmem + L::kDCol + dbuf * L::kBN;
          const uint64_t bd = bdesc0 + (uint64_t)((sx * L::kXStage) >> 4);
          if (!T) {
            // 2/3-bit: one A buffer per block (by parity), 8 integer MMAs of K = 32; the B tile is
            // two atoms of 128 K positions x 32 rows (4 KB each)
            const uint32_t abuf = gb & 1;
            if (!(ok = mbar_wait(&bars->a_full[abuf], (gb >> 1) & 1, abort_flag, a.err, 204))) break;
            fence_after_sync();
            const uint32_t idesc = idesc_i8_m128(xrows);
            const uint32_t atom16 = (uint32_t)(xrows * 128) >> 4;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const uint64_t off = (uint64_t)((j >> 2) * atom16 + (((j & 3) * 32) >> 4));
              mma_ts_i8(dcol, tmem + abuf * L::kABuf + 8 * j, bd + off, idesc, j != 0);
            }
            mma_commit(&bars->a_empty[abuf]);
            mma_commit(&bars->x_empty[sx]);
            mma_commit(&bars->d_full[dbuf]);
          } else {
            // ternary: two half-block A buffers, bf16 MMAs of K = 16 over 5 atoms of 16 rows
            constexpr uint32_t idesc = idesc_bf16_m128(16);
            const bool first_of_item = b == im.b0;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              if (!(ok = mbar_wait(&bars->a_full[c], gb & 1, abort_flag, a.err, 205))) break;
              fence_after_sync();
#pragma unroll
              for (int j = 0; j < 10; ++j) {
                const int kk = c * 160 + 16 * j;
                const uint64_t off = (uint64_t)(((kk / 64) * 2048 + (kk % 64) * 2) >> 4);
                mma_ts(dcol, tmem + c * L::kABuf + 8 * j, bd + off, idesc,
                       (uint32_t)(!first_of_item || c != 0 || j != 0));
              }
              mma_commit(&bars->a_empty[c]);
            }
            if (!ok) break;
            mma_commit(&bars->x_empty[sx]);
          }
        }
        if (T && ok) mma_commit(&bars->d_full[dbuf]);
      }
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ decode (thread = row)
    // warp w: lane quarter w % 4 (rows 32*(w%4) .. +31); group g = w / 4 decodes quarters 2g and
    // 2g+1 of every block.
    const int g = warp >> 2, lq = warp & 3;
    const int t = 32 * lq + lane;
    const int tile = t >> 4, r = t & 15, r0 = r & 7, half = r >> 3;
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * lq) << 16);
    uint32_t gb = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < a.items && ok && !*abort_flag; it += gridDim.x) {
      const Item im = find_item(a, it);
      const int bits = a.prob[im.pi].bits;
      const int ub = T ? 1024 : (bits == 2 ? 1024 : 1536);
      for (int b = im.b0; b < im.b1; ++b, ++gb) {
        const int sp = gb % kSP;
        if (!(ok = mbar_wait(&bars->pk_full[sp], (gb / kSP) & 1, abort_flag, a.err, 301))) break;
        const uint8_t* unit = ps + sp * L::kPStage + tile * ub;
        // 2/3-bit: A buffer = block parity (both groups fill it); ternary: A buffer = group
        const int abuf = T ? g : (int)(gb & 1);
        const uint32_t aphase = T ? ((gb & 1) ^ 1) : (((gb >> 1) & 1) ^ 1);
        if (!(ok = mbar_wait(&bars->a_empty[abuf], aphase, abort_flag, a.err, 302))) break;
        fence_after_sync();
#pragma unroll
        for (int qq = 0; qq < 2; ++qq) {
          const int q = 2 * g + qq;
          if (T) {
            uint32_t v[40];
            t_quarter(unit, r0, half, q, lut_lo, lut_hi, v);
            const uint32_t col = lane_addr + abuf * L::kABuf + qq * L::kQuarterCols;
            tmem_st32(col, v);
            tmem_st8(col + 32, v + 32);
          } else {
            uint32_t v[16];
            if (bits == 2) q2_quarter_i8(unit, r0, half, q, v);
            else q3_quarter_i8(unit, r0, half, q, v);
            tmem_st16(lane_addr + abuf * L::kABuf + q * L::kQuarterCols, v);
          }
        }
        tmem_wait_st();
        fence_before_sync();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bars->a_full[abuf]);
          mbar_arrive(&bars->pk_empty[sp]);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 8-11, thread = row)
    const int t = threadIdx.x - 256;
    const uint32_t lane_addr = (uint32_t)(32 * (warp - 8)) << 16;
    uint32_t gb = 0, gi = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < a.items && ok && !*abort_flag; it += gridDim.x, ++gi) {
      const Item im = find_item(a, it);
      const DecProblem& pr = a.prob[im.pi];
      const int n = im.rg * 128 + t;
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
      if (T) {
        const uint32_t dbuf = gi & 1;
        gb += im.b1 - im.b0;
        if (!(ok = mbar_wait(&bars->d_full[dbuf], (gi >> 1) & 1, abort_flag, a.err, 401))) break;
        fence_after_sync();
        float d[16];
        tmem_ld16(tmem + lane_addr + L::kDCol + dbuf * L::kBN, d);
        tmem_wait_ld();
        fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->d_empty[dbuf]);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = d[i] + d[i + 8];
      } else {
        const int lcode = pr.bits == 2 ? 3 : 7;
        const uint16_t* srow = pr.scales + (int64_t)(n < pr.N ? n : 0) * pr.B;
        uint16_t s_next = __ldg(srow + im.b0);
        for (int b = im.b0; b < im.b1; ++b, ++gb) {
          const uint32_t dbuf = gb & 1;
          const float s = n < pr.N ? half_bits_to_float(s_next) : 0.f;
          if (b + 1 < im.b1) s_next = __ldg(srow + b + 1);   // one block ahead
          if (!(ok = mbar_wait(&bars->d_full[dbuf], (gb >> 1) & 1, abort_flag, a.err, 402))) break;
          fence_after_sync();
          uint32_t d[32];
          tmem_ld32(tmem + lane_addr + L::kDCol + dbuf * L::kBN, d);
          tmem_wait_ld();
          fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->d_empty[dbuf]);
          // corrections of this block: per token m the factor 2^E and the limb sums S_j
          const int sc = gb % kSC;
          if (!(ok = mbar_wait(&bars->c_full[sc], (gb / kSC) & 1, abort_flag, a.err, 403))) break;
          const uint8_t* cst = cs + sc * 256;
          const float* fct = reinterpret_cast<const float*>(cst);
          const int* ssum = reinterpret_cast<const int*>(cst + 32);
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            if (m < M) {
              // limb j: sum_k (2c - L) d_j = 2 D_j - L S_j, exact in int32; limbs combined in fp32
              float v = 0.f;
#pragma unroll
              for (int j = 3; j >= 0; --j)
                v = fmaf(v, 256.f, (float)(2 * (int)d[(xrows >> 2) * j + m] - lcode * ssum[4 * m + j]));
              acc[m] = fmaf(s * fct[m], v, acc[m]);
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->c_empty[sc]);
        }
        if (!ok) break;
      }
      const float rs = (T && n < pr.N) ? half_bits_to_float(__ldg(pr.scales + n)) : 1.f;
      if (pr.P == 1) {
        if (n < pr.N) {
#pragma unroll
          for (int i = 0; i < 8; ++i)
            if (i < M) pr.y[(int64_t)i * pr.N + n] = rs * acc[i];
        }
      } else {
        const int cid = pr.counter_base + im.rg;
        float* part = a.partial + pr.partial_base + ((int64_t)im.rg * pr.P + im.p) * M * 128;
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (i < M) part[i * 128 + t] = acc[i];
        __threadfence();
        named_bar_sync(1, 128);
        if (t == 0) bars->last_flag = (atomicAdd(a.counter + cid, 1) == pr.P - 1);
        named_bar_sync(1, 128);
        if (bars->last_flag) {
          __threadfence();
          float sum[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) sum[i] = 0.f;
          for (int pp = 0; pp < pr.P; ++pp) {
            const float* src = a.partial + pr.partial_base + ((int64_t)im.rg * pr.P + pp) * M * 128;
#pragma unroll
            for (int i = 0; i < 8; ++i)
              if (i < M) sum[i] += __ldcg(src + i * 128 + t);
          }
          if (n < pr.N) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              if (i < M) pr.y[(int64_t)i * pr.N + n] = rs * sum[i];
          }
          if (t == 0) a.counter[cid] = 0;
        }
        named_bar_sync(1, 128);
      }
    }
  }

  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 13) tmem_dealloc(tmem, L::kTmemCols);
}

// Preparation pass for 2/3-bit problems: one warp per (problem, block). For each token m the
// block's activations become integers n_k = x_k / 2^E (E = exponent of the block maximum - 29;
// values that are not multiples of 2^E round to the nearest, ties to even), split into four
// balanced signed bytes d_j (n = sum_j 256^j d_j, d_j in [-128, 127]). Limb j of token m goes to
// row (xrows/4) j + m of the B tile (two atoms of 128 K positions x xrows rows, 128-byte
// swizzle) at the logical K position whose A byte holds code k. After the atoms: the factor 2^E per token
// (8 floats) and the limb sums S_j (8 x 4 int32). Rows, factors and sums of tokens >= M are 0.
__global__ void __launch_bounds__(256) prep_x_kernel(const __grid_constant__ DecArgs a, int total_blocks) {
  const int lane = threadIdx.x & 31;
  const int g = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (g >= total_blocks) return;
  int lo = 0, hi = a.count - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a.prob[mid].xblk_base <= g) lo = mid;
    else hi = mid - 1;
  }
  const DecProblem& pr = a.prob[lo];
  const int b = g - pr.xblk_base;
  const int M = a.M;
  const int xrows = decode_xrows(M), rstep = xrows >> 2;
  uint8_t* dst = pr.xt + (int64_t)b * xtile_bytes(false, M);
  float* fct = reinterpret_cast<float*>(dst + 2 * xrows * 128);
  int* ssum = reinterpret_cast<int*>(dst + 2 * xrows * 128 + 32);
  for (int i = lane; i < 2 * xrows * 128 / 16; i += 32) reinterpret_cast<uint4*>(dst)[i] = make_uint4(0, 0, 0, 0);
  if (lane < 8) fct[lane] = 0.f;
  ssum[lane] = 0;
  __syncwarp();
  for (int m = 0; m < M; ++m) {
    // lane l holds logical K positions 8l .. 8l+7 of the decoded block
    float xv[8];
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int kl = 8 * lane + e;
      const int k = pr.bits == 2 ? q2_code_at(kl) : q3_code_at(kl);
      xv[e] = __bfloat162float(__ushort_as_bfloat16(pr.x[(int64_t)m * pr.K + (int64_t)b * 256 + k]));
      amax = fmaxf(amax, fabsf(xv[e]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    int ex = 0;
    if (amax > 0.f) frexpf(amax, &ex);   // amax in [2^(ex-1), 2^ex)
    const int E = ex - 1 - 29;            // |n| < 2^30
    int s0 = 0, s1 = 0, s2 = 0, s3 = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int kl = 8 * lane + e;
      const int n = amax > 0.f ? __float2int_rn(ldexpf(xv[e], -E)) : 0;
      const int d0 = (int)(int8_t)(n & 0xFF);
      const int n1 = (n - d0) >> 8;
      const int d1 = (int)(int8_t)(n1 & 0xFF);
      const int n2 = (n1 - d1) >> 8;
      const int d2 = (int)(int8_t)(n2 & 0xFF);
      const int d3 = (n2 - d2) >> 8;
      s0 += d0;
      s1 += d1;
      s2 += d2;
      s3 += d3;
      const int atom = kl >> 7, kb = kl & 127;
      const int dl[4] = {d0, d1, d2, d3};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int row = rstep * j + m;
        dst[atom * xrows * 128 + row * 128 + ((((kb >> 4) ^ (row & 7)) << 4) | (kb & 15))] = (uint8_t)(int8_t)dl[j];
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      s0 += __shfl_xor_sync(0xffffffffu, s0, o);
      s1 += __shfl_xor_sync(0xffffffffu, s1, o);
      s2 += __shfl_xor_sync(0xffffffffu, s2, o);
      s3 += __shfl_xor_sync(0xffffffffu, s3, o);
    }
    if (lane == 0) {
      fct[m] = amax > 0.f ? ldexpf(1.f, E) : 0.f;
      ssum[4 * m + 0] = s0;
      ssum[4 * m + 1] = s1;
      ssum[4 * m + 2] = s2;
      ssum[4 * m + 3] = s3;
    }
  }
}

}  // namespace

cudaError_t launch_prep_x(const DecArgs& a, int total_blocks, cudaStream_t stream) {
  prep_x_kernel<<<(total_blocks + 7) / 8, 256, 0, stream>>>(a, total_blocks);
  return cudaGetLastError();
}

cudaError_t launch_decode(bool ternary, const DecArgs& a, int grid, cudaStream_t stream) {
  if (ternary) {
    static bool set = false;
    if (!set) {
      const cudaError_t e = cudaFuncSetAttribute(decode_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 DL<true>::kSmem);
      if (e != cudaSuccess) return e;
      set = true;
    }
    decode_kernel<true><<<grid, kThreads, DL<true>::kSmem, stream>>>(a);
  } else {
    static bool set = false;
    if (!set) {
      const cudaError_t e = cudaFuncSetAttribute(decode_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 DL<false>::kSmem);
      if (e != cudaSuccess) return e;
      set = true;
    }
    decode_kernel<false><<<grid, kThreads, DL<false>::kSmem, stream>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace wr
