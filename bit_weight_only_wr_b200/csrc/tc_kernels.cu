// Packed-code GEMV/GEMM on tcgen05 tensor cores (sm_100a).
//
//   y[m,n] = sum_b s[n,b] sum_{k in b} g[n,k] x[m,k]         (2/3-bit odd grid, fp16 or int8 scales)
//   y[m,n] = alpha[n] sum_k t[n,k] (R x[m,:])[k]             (ternary, rotated basis)
//
// One CTA owns 128 weight rows ("row group") at a time; the MMA is D[128 x BN] += A[128 x 16]
// * B[16 x BN] with the weights as A and BN token columns as B ("swap-AB"), so every TMEM lane
// is one output row and the per-block scale is a single scalar per lane.
//
// Warp roles (576 threads):
//   warps 0-7  decode: warps w and w + 4 own rows 32 (w % 4) .. + 31 of the group (TMEM lanes)
//              and take alternate quarters of each half-block chunk. A thread reads its row's
//              packed codes from shared memory, turns them into exact bf16 values (g/2, or t
//              for ternary) in registers and writes them into tensor memory with tcgen05.st:
//              A is consumed from TMEM, so the decoded weights never touch shared memory.
//   warp 16    producer: bulk-copies the packed units of each 256-block (8 x 16-row units) and
//              TMA-loads the activation tile (128-byte swizzle) into shared-memory rings.
//   warp 17    allocates TMEM and issues the MMAs (whole warp, one elected lane), committing to the barriers
//              that recycle A buffers, activation stages and accumulators.
//   warps 8-15 epilogue (two per lane quarter, half of the token tile each): per 256-block,
//              load the fp32 partial from TMEM, multiply by 2*s[n,b] in fp32 and add it to a
//              register running sum (ternary: one accumulator per piece of a tile); at the end
//              of a tile (or of the CTA's range), write y, or, for a tile that several ranges
//              share, leave the piece in a partial slot (the last piece to arrive adds them in
//              range order and writes y).
// Work: the (tile, block) pairs are cut into one contiguous range per CTA ("stream-K"), so that
// every CTA streams the same number of blocks whatever the tile count.
// Every wait is bounded: a stuck pipeline records an error code and the CTA unwinds.
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "tc_common.cuh"
#include "tc_kernels.cuh"
#include "wr.h"

namespace wr {
namespace {

using namespace tc;

constexpr int kThreads = 576;
constexpr int kSP = 4;  // packed-unit stages
constexpr int kSX = 2;  // activation stages (per block)
constexpr int kSA = 3;  // A buffers in tensor memory (half-block chunks)

template <int FMT>
struct Fmt {
  static constexpr int kUnitK = FMT == WR_FMT_TERNARY ? 320 : 256;       // K per block
  static constexpr int kUnitBytes = FMT == WR_FMT_Q3 ? 1536 : 1024;      // bytes per 16-row unit
  static constexpr int kQuarterCols = FMT == WR_FMT_TERNARY ? 40 : 32;   // TMEM columns per quarter
  static constexpr int kChunkCols = 2 * kQuarterCols;                   // A buffer (half block)
  static constexpr int kChunkSteps = kChunkCols / 8;                    // K-steps of 16 per chunk
};

template <int FMT, int BN>
struct Layout {
  static constexpr int kXStage = BN * Fmt<FMT>::kUnitK * 2;              // bytes per activation stage
  static constexpr int kXAtom = BN * 128;                                // bytes per 64-wide K atom
  static constexpr int kPStage = 8 * Fmt<FMT>::kUnitBytes;
  static constexpr int kXOff = 0;
  static constexpr int kPOff = kXOff + kSX * kXStage;
  static constexpr int kBarOff = kPOff + kSP * kPStage;
  static constexpr int kSmem = kBarOff + 256 + 1024;   // + barriers and alignment slack
  static constexpr int kACols = Fmt<FMT>::kChunkCols;
  static constexpr int kDCol = kSA * kACols;
  static constexpr int kTmemCols = (kDCol + 2 * BN) <= 256 ? 256 : 512;
  static_assert(kDCol + 2 * BN <= 512, "tensor memory of the SM");
  static constexpr int kTok = FMT == WR_FMT_TERNARY ? BN / 2 : BN;      // tokens per tile
};

struct Bars {
  uint64_t pk_full[kSP], pk_empty[kSP], x_full[kSX], x_empty[kSX];
  uint64_t a_full[kSA], a_empty[kSA], d_full[2], d_empty[2];
  uint64_t group;   // the 8 epilogue warps meet here (bounded, unlike a named barrier)
  uint32_t tmem_base;
  int abort_flag;
  int last_flag;
};
static_assert(sizeof(Bars) <= 256, "barrier area");

// Work is split "stream-K": the batch of (tile, block) pairs, tile-major (tile t = rg * MT + mt,
// token tiles innermost so that a range reuses one row group's weights from L2), is cut into one
// contiguous range of blocks per CTA. A tile cut by a range boundary is finished from pieces.
__device__ __forceinline__ int64_t sk_start(int64_t T, int c) { return (int64_t)c * T / gridDim.x; }
// CTA whose range holds global block g: the largest c with sk_start(c) <= g
__device__ __forceinline__ int sk_cta_of(int64_t T, int64_t g) { return (int)(((g + 1) * gridDim.x - 1) / T); }

// Position in this CTA's range, advanced block by block without divisions.
struct SkPos {
  int64_t g, g1;      // current global block, end of the range
  int t;              // tile
  int b;              // block inside the tile
  int rg, mt;
  bool first, last;   // the first / last block of this CTA's piece of the tile
};
__device__ __forceinline__ void sk_flags(const TcArgs& a, SkPos& p, bool start) {
  p.first = start || p.b == 0;
  p.last = p.b == a.B - 1 || p.g == p.g1 - 1;
}
__device__ __forceinline__ SkPos sk_begin(const TcArgs& a) {
  SkPos p;
  p.g = sk_start(a.total, blockIdx.x);
  p.g1 = sk_start(a.total, blockIdx.x + 1);
  const int64_t t = p.g / a.B;
  p.t = (int)t;
  p.b = (int)(p.g - t * a.B);
  p.rg = p.t / a.MT;
  p.mt = p.t - p.rg * a.MT;
  sk_flags(a, p, true);
  return p;
}
__device__ __forceinline__ void sk_next(const TcArgs& a, SkPos& p) {
  ++p.g;
  if (++p.b == a.B) {
    p.b = 0;
    ++p.t;
    if (++p.mt == a.MT) {
      p.mt = 0;
      ++p.rg;
    }
  }
  sk_flags(a, p, false);
}

// ---------------------------------------------------------------- decode helpers (thread = row)

// Q2: the row's quarter q of a unit is 16 bytes at chunk (32*half + lane_pos(r0, q)).
__device__ __forceinline__ void decode_q2_quarter(const uint8_t* unit, int r0, int half, int q, uint32_t v[32]) {
  const uint4 c = *reinterpret_cast<const uint4*>(unit + (32 * half + lane_pos(r0, q)) * 16);
  decode_q2_word(c.x, v + 0);
  decode_q2_word(c.y, v + 8);
  decode_q2_word(c.z, v + 16);
  decode_q2_word(c.w, v + 24);
}

// Q3: lane 4*r0 + q holds 48 bytes in chunks (32c + lane_pos(r0, q))*16; row half h uses lane
// bytes 24h .. 24h+23, i.e. two 12-byte groups of 3 words.
__device__ __forceinline__ void decode_q3_quarter(const uint8_t* unit, int r0, int half, int q, uint32_t v[32]) {
  const int l = lane_pos(r0, q);
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
  decode_q3_group(w, v);
  decode_q3_group(w + 3, v + 16);
}

// Ternary: a quarter is 16 bytes = 80 trits; byte pair (2b', 2b'+1) gives pair registers
// 5b'..5b'+4, pair i = (trit i of byte 2b', trit i of byte 2b'+1).
__device__ __forceinline__ void decode_t_quarter(const uint8_t* unit, int r0, int half, int q,
                                                 const uint32_t* lut_lo, const uint32_t* lut_hi, uint32_t v[40]) {
  const uint4 c = *reinterpret_cast<const uint4*>(unit + (32 * half + lane_pos(r0, q)) * 16);
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

// Output value of token m: the ternary planes hold token m scaled by 2^-tok_ex[m], undone here
// (one rounding, gradual into fp32's subnormal range); the 2/3-bit forms read x unscaled.
template <int FMT>
__device__ __forceinline__ float out_value(const TcArgs& a, float v, int m) {
  if constexpr (FMT == WR_FMT_TERNARY) return ldexpf(v, a.tok_ex[m]);
  else return v;
}

// ---------------------------------------------------------------- the kernel

template <int FMT, int BN>
__global__ void __launch_bounds__(kThreads, 1) tc_kernel(const TcArgs a, const __grid_constant__ CUtensorMap xmap) {
  using F = Fmt<FMT>;
  using Ly = Layout<FMT, BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* xs = smem + Ly::kXOff;
  uint8_t* ps = smem + Ly::kPOff;
  Bars* bars = reinterpret_cast<Bars*>(smem + Ly::kBarOff);
  __shared__ uint32_t lut_lo[FMT == WR_FMT_TERNARY ? 256 : 1], lut_hi[FMT == WR_FMT_TERNARY ? 256 : 1];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &bars->abort_flag;

  if (FMT == WR_FMT_TERNARY) {
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
      mbar_init(&bars->x_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->d_full[i], 1);
      mbar_init(&bars->d_empty[i], 8);
    }
    for (int i = 0; i < kSA; ++i) {
      mbar_init(&bars->a_full[i], 8);
      mbar_init(&bars->a_empty[i], 1);
    }
    mbar_init(&bars->group, 8);
    bars->abort_flag = 0;
    bars->last_flag = 0;
    fence_barrier_init();
  }
  if (warp == 17) tmem_alloc(&bars->tmem_base, Ly::kTmemCols);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 16) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&xmap);
      uint32_t gb = 0;
      const int tiles = (a.N + 15) / 16;
      for (SkPos ps_ = sk_begin(a); ps_.g < ps_.g1 && !*abort_flag; sk_next(a, ps_), ++gb) {
        const int b = ps_.b, rg = ps_.rg, mt = ps_.mt;
        const int sx = gb % kSX;
        if (!mbar_wait_bg(&bars->x_empty[sx], ((gb / kSX) & 1) ^ 1, abort_flag, a.err, 101)) break;
        mbar_arrive_expect_tx(&bars->x_full[sx], Ly::kXStage);
#pragma unroll
        for (int at = 0; at < F::kUnitK / 64; ++at) {
          uint8_t* dst = xs + sx * Ly::kXStage + at * Ly::kXAtom;
          const int k = b * F::kUnitK + 64 * at;
          if (FMT == WR_FMT_TERNARY) {
            // two boxes of kTok tokens: the hi plane of R x into rows 0 .. kTok - 1, the lo
            // plane into rows kTok .. 2 kTok - 1
            tma_load_3d(dst, &xmap, k, mt * Ly::kTok, 0, &bars->x_full[sx]);
            tma_load_3d(dst + Ly::kTok * 128, &xmap, k, mt * Ly::kTok, 1, &bars->x_full[sx]);
          } else {
            tma_load_2d(dst, &xmap, k, mt * BN, &bars->x_full[sx]);
          }
        }
        const int sp = gb % kSP;
        if (!mbar_wait_bg(&bars->pk_empty[sp], ((gb / kSP) & 1) ^ 1, abort_flag, a.err, 102)) break;
        const int ntile = min(8, tiles - rg * 8);
        mbar_arrive_expect_tx(&bars->pk_full[sp], ntile * F::kUnitBytes);
        bulk_load(ps + sp * Ly::kPStage, a.packed + ((int64_t)rg * 8 * a.B + (int64_t)b * ntile) * F::kUnitBytes,
                  ntile * F::kUnitBytes, &bars->pk_full[sp]);
      }
    }
  } else if (warp == 17) {
    // ------------------------------------------------------------ MMA issuer (whole warp, one lane issues)
    constexpr uint32_t idesc = idesc_bf16_m128(BN);
    uint32_t gb = 0, gc = 0, gp = 0;   // blocks, half-block chunks, pieces (ternary accumulators)
    bool ok = true;
    uint32_t dbuf = 0;
    for (SkPos ps_ = sk_begin(a); ps_.g < ps_.g1 && ok && !*abort_flag; sk_next(a, ps_), ++gb) {
      if (FMT == WR_FMT_TERNARY) {
        // one accumulator per piece: all its blocks add into it
        if (ps_.first) {
          dbuf = gp & 1;
          if (!(ok = mbar_wait_bg(&bars->d_empty[dbuf], ((gp >> 1) & 1) ^ 1, abort_flag, a.err, 201))) break;
        }
      } else {
        // one accumulator per block (its scale is applied in the epilogue)
        dbuf = gb & 1;
        if (!(ok = mbar_wait_bg(&bars->d_empty[dbuf], ((gb >> 1) & 1) ^ 1, abort_flag, a.err, 202))) break;
      }
      const int sx = gb % kSX;
      if (!(ok = mbar_wait_bg(&bars->x_full[sx], (gb / kSX) & 1, abort_flag, a.err, 203))) break;
      const uint8_t* xst = xs + sx * Ly::kXStage;
      for (int c = 0; c < 2; ++c, ++gc) {
        const int sa = gc % kSA;
        if (!(ok = mbar_wait_bg(&bars->a_full[sa], (gc / kSA) & 1, abort_flag, a.err, 204))) break;
        fence_after_sync();
#pragma unroll
        for (int j = 0; j < F::kChunkSteps; ++j) {
          const int kk = c * (F::kUnitK / 2) + 16 * j;     // K offset inside the block
          const uint64_t bdesc = smem_desc_sw128(xst + (kk / 64) * Ly::kXAtom + (kk % 64) * 2);
          const uint32_t acc = (FMT == WR_FMT_TERNARY) ? (uint32_t)(!ps_.first || c != 0 || j != 0)
                                                       : (uint32_t)(c != 0 || j != 0);
          mma_ts_elect(tmem + Ly::kDCol + dbuf * BN, tmem + sa * Ly::kACols + 8 * j, bdesc, idesc, acc);
        }
        mma_commit_elect(&bars->a_empty[sa]);
      }
      if (!ok) break;
      mma_commit_elect(&bars->x_empty[sx]);
      if (FMT != WR_FMT_TERNARY) {
        mma_commit_elect(&bars->d_full[dbuf]);
      } else if (ps_.last) {
        mma_commit_elect(&bars->d_full[dbuf]);
        ++gp;
      }
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ decode (thread = row)
    // warps w and w + 4 share lane quarter w % 4 (rows 32 (w % 4) ..); group g = w / 4 decodes
    // quarter g of each half-block chunk, so each row's decode chain is split in two
    const int g = warp >> 2, lq = warp & 3;
    const int t = 32 * lq + lane;
    const int tile = t >> 4, r = t & 15, r0 = r & 7, half = r >> 3;
    const uint32_t lane_addr = (uint32_t)(32 * lq) << 16;
    uint32_t gb = 0, gc = 0;
    bool ok = true;
    const int64_t nblk = sk_start(a.total, blockIdx.x + 1) - sk_start(a.total, blockIdx.x);
    for (int64_t gg = 0; gg < nblk && ok && !*abort_flag; ++gg, ++gb) {
      {
        const int sp = gb % kSP;
        if (!(ok = mbar_wait(&bars->pk_full[sp], (gb / kSP) & 1, abort_flag, a.err, 301))) break;
        const uint8_t* unit = ps + sp * Ly::kPStage + tile * F::kUnitBytes;
        for (int c = 0; c < 2; ++c, ++gc) {
          const int sa = gc % kSA;
          if (!(ok = mbar_wait(&bars->a_empty[sa], ((gc / kSA) & 1) ^ 1, abort_flag, a.err, 302))) break;
          fence_after_sync();
          const int q = 2 * c + g;
          const uint32_t col = tmem + lane_addr + sa * Ly::kACols + g * F::kQuarterCols;
          if (FMT == WR_FMT_TERNARY) {
            uint32_t v[40];
            decode_t_quarter(unit, r0, half, q, lut_lo, lut_hi, v);
            tmem_st32(col, v);
            tmem_st8(col + 32, v + 32);
          } else {
            uint32_t v[32];
            if (FMT == WR_FMT_Q2) decode_q2_quarter(unit, r0, half, q, v);
            else decode_q3_quarter(unit, r0, half, q, v);
            tmem_st32(col, v);
          }
          tmem_wait_st();
          fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->a_full[sa]);
        }
        if (!ok) break;
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->pk_empty[sp]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 8-15, thread = row)
    // warps 8 + w and 12 + w share lane quarter w; group e takes tokens e*TH .. e*TH + TH - 1
    constexpr int TOK = Ly::kTok, TH = TOK / 2;
    static_assert(TH % 16 == 0, "tokens per epilogue group: a multiple of 16");
    const int e = (warp - 8) >> 2, lq = (warp - 8) & 3;
    uint32_t ng = 0;   // group barrier phases used
    auto group_sync = [&](int code) {
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->group);
      return mbar_wait(&bars->group, (ng++) & 1, abort_flag, a.err, code);
    };
    const int t = 32 * lq + lane;
    const uint32_t lane_addr = (uint32_t)(32 * lq) << 16;
    uint32_t gb = 0, gp = 0;   // blocks, pieces (ternary accumulators)
    const int64_t g0 = sk_start(a.total, blockIdx.x);
    float acc[TH];
    bool ok = true;
    for (SkPos ps_ = sk_begin(a); ps_.g < ps_.g1 && ok; sk_next(a, ps_), ++gb) {
      const int n = ps_.rg * 128 + t;
      if (ps_.first) {
#pragma unroll
        for (int i = 0; i < TH; ++i) acc[i] = 0.f;
      }
      if (FMT == WR_FMT_TERNARY) {
        if (!ps_.last) continue;
        // the piece's accumulator: column j < TOK holds token j against the hi plane of R x,
        // column TOK + j against the lo plane
        const uint32_t dbuf = gp & 1;
        ok = mbar_wait(&bars->d_full[dbuf], (gp >> 1) & 1, abort_flag, a.err, 401);
        ++gp;
        if (!ok) break;
        fence_after_sync();
#pragma unroll
        for (int c0 = 0; c0 < TH; c0 += 16) {
          float dh[16], dl[16];
          tmem_ld16(tmem + lane_addr + Ly::kDCol + dbuf * BN + e * TH + c0, dh);
          tmem_ld16(tmem + lane_addr + Ly::kDCol + dbuf * BN + TOK + e * TH + c0, dl);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) acc[c0 + i] = dh[i] + dl[i];
        }
        fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->d_empty[dbuf]);
      } else {
        const uint32_t dbuf = gb & 1;
        // 2 s: the fp16 block scale, or d_n q[n,b] (exact in fp32)
        const float s2 = n >= a.N ? 0.f
                         : a.scale_q == nullptr
                             ? 2.f * half_bits_to_float(__ldg(a.scales + (int64_t)n * a.B + ps_.b))
                             : 2.f * half_bits_to_float(__ldg(a.scales + n)) *
                                   (float)__ldg(a.scale_q + (int64_t)n * a.B + ps_.b);
        if (!(ok = mbar_wait(&bars->d_full[dbuf], (gb >> 1) & 1, abort_flag, a.err, 402))) break;
        fence_after_sync();
#pragma unroll
        for (int c0 = 0; c0 < TH; c0 += 16) {
          float d[16];
          tmem_ld16(tmem + lane_addr + Ly::kDCol + dbuf * BN + e * TH + c0, d);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) acc[c0 + i] = fmaf(s2, d[i], acc[c0 + i]);
        }
        fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->d_empty[dbuf]);
      }
      if (!ps_.last) continue;
      // ---- output: y directly, or, for a tile that several CTA ranges share, the combine
      // through the partial slots (the last range to arrive adds the pieces in range order)
      const int m0 = ps_.mt * TOK + e * TH;
      const int mcount = max(0, min(TH, a.M - m0));
      const float rs = (FMT == WR_FMT_TERNARY && n < a.N) ? half_bits_to_float(__ldg(a.alpha + n)) : 1.f;
      const int64_t tb = (int64_t)ps_.t * a.B;   // first block of the tile
      const int c0 = sk_cta_of(a.total, tb), c1 = sk_cta_of(a.total, tb + a.B - 1);
      if (c0 == c1) {
        if (n < a.N) {
#pragma unroll
          for (int i = 0; i < TH; ++i)
            if (i < mcount) a.y[(int64_t)(m0 + i) * a.N + n] = out_value<FMT>(a, rs * acc[i], m0 + i);
        }
      } else {
        // slot 0: the tile began before this range; slot 1: it continues after it
        const int slot = tb < g0 ? 0 : 1;
        float* part = a.partial + ((int64_t)blockIdx.x * 2 + slot) * (TOK * 128) + (int64_t)e * TH * 128;
#pragma unroll
        for (int i = 0; i < TH; ++i)
          if (i < mcount) part[i * 128 + t] = acc[i];
        __threadfence();
        if (!(ok = group_sync(403))) break;
        if (threadIdx.x == 256) bars->last_flag = (atomicAdd(a.counter + ps_.t, 1) == c1 - c0);
        if (!(ok = group_sync(404))) break;
        if (bars->last_flag) {
          __threadfence();
#pragma unroll
          for (int i = 0; i < TH; ++i) acc[i] = 0.f;
          for (int c = c0; c <= c1; ++c) {
            const int sl = tb < sk_start(a.total, c) ? 0 : 1;
            const float* src = a.partial + ((int64_t)c * 2 + sl) * (TOK * 128) + (int64_t)e * TH * 128;
#pragma unroll
            for (int i = 0; i < TH; ++i)
              if (i < mcount) acc[i] += __ldcg(src + i * 128 + t);
          }
          if (n < a.N) {
#pragma unroll
            for (int i = 0; i < TH; ++i)
              if (i < mcount) a.y[(int64_t)(m0 + i) * a.N + n] = out_value<FMT>(a, rs * acc[i], m0 + i);
          }
          if (threadIdx.x == 256) a.counter[ps_.t] = 0;
        }
        if (!(ok = group_sync(405))) break;
      }
    }
  }

  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 17) tmem_dealloc(tmem, Ly::kTmemCols);
}

// ---------------------------------------------------------------- host side

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

template <int FMT, int BN>
cudaError_t launch_tc(const TcArgs& a, const void* x_act, int64_t x_rows, int64_t x_k, int grid, cudaStream_t stream) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap map;
  CUresult r;
  if (FMT == WR_FMT_TERNARY) {
    // R x planes: [2][M][Kp] bf16 -> dims (Kp, M, 2), box (64 positions, kTok tokens, 1 plane)
    const cuuint64_t dims[3] = {(cuuint64_t)x_k, (cuuint64_t)x_rows, 2};
    const cuuint64_t strides[2] = {(cuuint64_t)x_k * 2, (cuuint64_t)x_k * 2 * x_rows};
    const cuuint32_t box[3] = {64, (cuuint32_t)Layout<FMT, BN>::kTok, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(x_act), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  } else {
    const cuuint64_t dims[2] = {(cuuint64_t)x_k, (cuuint64_t)x_rows};
    const cuuint64_t strides[1] = {(cuuint64_t)x_k * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)BN};
    const cuuint32_t estr[2] = {1, 1};
    r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x_act), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  }
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  using Ly = Layout<FMT, BN>;
  auto kern = tc_kernel<FMT, BN>;
  static bool attr_set = false;
  if (!attr_set) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Ly::kSmem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  kern<<<grid, kThreads, Ly::kSmem, stream>>>(a, map);
  return cudaGetLastError();
}

// R x for the ternary prefill GEMM: one warp per (token, 128-block). x' = (1/sqrt(128)) H (d * x)
// in fp32, token m scaled first by 2^-tok_ex[m] (exact) so that its hi and lo parts stay in bf16's
// normal range whatever the magnitude of x (the GEMM epilogue multiplies the token's results by
// 2^tok_ex[m]); then split into hi = bf16(x') and lo = bf16(x' - hi). Inside each 320-trit unit,
// position 80q + 2P + h holds trit 80q + 5*(2*(P/5) + h) + P%5 (pair P of byte pair P/5; h
// selects the byte): the K order of the decoded A columns. Pad trits get 0. The planes are
// [2][M][Kp] bf16 row-major, hi then lo, read by TMA. Lane l holds K positions 4l .. 4l+3.
__global__ void rotate_planes_kernel(const uint16_t* __restrict__ x, const uint32_t* __restrict__ signs,
                                     uint8_t* __restrict__ planes, int M, int K, int64_t Kp,
                                     const int* __restrict__ tok_ex) {
  const int lane = threadIdx.x & 31;
  const int64_t item = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t nblk = (Kp + 127) / 128;
  if (item >= (int64_t)M * nblk) return;
  const int m = (int)(item / nblk);
  const int64_t k0 = (item % nblk) * 128;
  const int scale_ex = tok_ex[m];
  float v[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t k = k0 + 4 * lane + i;
    float xv = 0.f;
    if (k < K) {
      xv = __bfloat162float(__ushort_as_bfloat16(x[(int64_t)m * K + k]));
      if ((signs[k >> 5] >> (k & 31)) & 1u) xv = -xv;
      xv = ldexpf(xv, -scale_ex);
    }
    v[i] = xv;
  }
  float t0 = v[0] + v[1], t1 = v[0] - v[1], t2 = v[2] + v[3], t3 = v[2] - v[3];
  v[0] = t0 + t2; v[2] = t0 - t2; v[1] = t1 + t3; v[3] = t1 - t3;
#pragma unroll
  for (int s = 1; s < 32; s <<= 1) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float o = __shfl_xor_sync(0xffffffffu, v[i], s);
      v[i] = (lane & s) ? o - v[i] : v[i] + o;
    }
  }
  const float inv = 0.08838834764831845f;  // 1/sqrt(128)
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t k = k0 + 4 * lane + i;
    if (k >= Kp) continue;
    const float xp = v[i] * inv;
    const __nv_bfloat16 hi = __float2bfloat16_rn(xp);
    const __nv_bfloat16 lo = __float2bfloat16_rn(xp - __bfloat162float(hi));
    const int64_t u = k / 320;
    const int kk = (int)(k % 320), q = kk / 80, i80 = kk % 80, beta = i80 / 5, dig = i80 % 5;
    const int P = 5 * (beta >> 1) + dig;
    const int kp = 80 * q + 2 * P + (beta & 1);
    uint16_t* pl = reinterpret_cast<uint16_t*>(planes);
    const int64_t off = (int64_t)m * Kp + u * 320 + kp;
    pl[off] = __bfloat16_as_ushort(hi);
    pl[(int64_t)M * Kp + off] = __bfloat16_as_ushort(lo);
  }
}

// Per-token exponent of the ternary prefill GEMM: tok_ex[m] = e with max_k |x[m,k]| in
// [2^(e-1), 2^e) (0 for an all-zero token). One CTA of 256 threads per token, 16-byte loads of 8
// activations (K is a multiple of 128, so rows are 256-byte aligned).
__global__ void __launch_bounds__(256) token_exponent_kernel(const uint16_t* __restrict__ x, int M, int K,
                                                            int* __restrict__ tok_ex) {
  __shared__ float wmax[8];
  const int m = blockIdx.x;
  const uint4* row = reinterpret_cast<const uint4*>(x + (int64_t)m * K);
  float amax = 0.f;
  for (int i = threadIdx.x; i < K / 8; i += 256) {
    const uint4 v = __ldg(row + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      amax = fmaxf(amax, fabsf(__uint_as_float(w[j] << 16)));
      amax = fmaxf(amax, fabsf(__uint_as_float(w[j] & 0xFFFF0000u)));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = amax;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 1; i < 8; ++i) amax = fmaxf(amax, wmax[i]);
    amax = fmaxf(amax, wmax[0]);
    int ex = 0;
    if (amax > 0.f) frexpf(amax, &ex);
    tok_ex[m] = ex;
  }
}

// Failure-path self-test: warp 0 waits on a barrier nobody arrives on until the bounded wait
// gives up (error code 901, abort flag raised); warp 1 waits on another such barrier and
// leaves on the abort flag (code 902 only if it ran out of time on its own first).
__global__ void __launch_bounds__(64) selftest_wait_timeout_kernel(int* err_word) {
  __shared__ __align__(8) uint64_t bar[2];
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  if (warp == 0) {
    mbar_wait(&bar[0], 0, &abort_flag, err_word, 901);
  } else {
    mbar_wait(&bar[1], 0, &abort_flag, err_word, 902);
  }
}

}  // namespace

cudaError_t launch_selftest_wait_timeout(int* err_word, cudaStream_t stream) {
  selftest_wait_timeout_kernel<<<1, 64, 0, stream>>>(err_word);
  return cudaGetLastError();
}

cudaError_t launch_tc_kernel(int fmt, int bn, const TcArgs& a, const void* x_act, int64_t x_rows, int64_t x_k,
                             int grid, cudaStream_t stream) {
  if (fmt == WR_FMT_Q2 && bn == 128) return launch_tc<WR_FMT_Q2, 128>(a, x_act, x_rows, x_k, grid, stream);
  if (fmt == WR_FMT_Q3 && bn == 128) return launch_tc<WR_FMT_Q3, 128>(a, x_act, x_rows, x_k, grid, stream);
  if (fmt == WR_FMT_TERNARY && bn == 128) return launch_tc<WR_FMT_TERNARY, 128>(a, x_act, x_rows, x_k, grid, stream);
  return cudaErrorNotSupported;
}

cudaError_t launch_rotate_planes(const uint16_t* x, const uint32_t* signs, uint8_t* planes, int M, int K, int64_t Kp,
                                 int* tok_ex, cudaStream_t stream) {
  const int warps = 8;
  token_exponent_kernel<<<(unsigned)M, 256, 0, stream>>>(x, M, K, tok_ex);
  const int64_t items = (int64_t)M * ((Kp + 127) / 128);
  rotate_planes_kernel<<<(unsigned)((items + warps - 1) / warps), warps * 32, 0, stream>>>(x, signs, planes, M, K, Kp,
                                                                                         tok_ex);
  return cudaGetLastError();
}

}  // namespace wr
