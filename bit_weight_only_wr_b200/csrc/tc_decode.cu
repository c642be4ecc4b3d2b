// Decode GEMV (M <= 16 tokens) on tcgen05, for one problem or a batch of independent problems.
//
// Decoding a token reads every weight once ("How We Shrank an AI Model by 85%...", section
// "Results": generating a token is mostly reading the weights from memory), so the kernel is a
// weight stream: each CTA walks a list of work items (problem, 128-row group, range of
// 256-code blocks) and keeps its rings full across item and problem boundaries, so the latency
// of one small GEMV hides behind the loads of the next.
//
//   y[m,n] = sum_b s[n,b] sum_{k in b} g[n,k] x[m,k]         (2/3-bit odd grid, fp16 scales)
//   y[m,n] = alpha[n] sum_k t[n,k] (R x[m,:])[k]             (ternary: x = R x planes hi, lo)
//
// MMA: D[128 rows x 16 cols] += A[128 x 16] (weights, tensor memory) * B[16 x 16] (tokens,
// shared memory). Warp roles (448 threads, two CTAs per SM):
//   warps 0-7  decode: thread = row (TMEM lane); warps w and w+4 share a lane quarter and take
//              the two halves of each block. The packed codes become bf16 values in registers
//              (one LOP3 per pair) and are stored to tensor memory (tcgen05.st).
//   warp 12    producer: bulk-copies the 16-row packed units of each block into a 4-deep ring
//              and copies the x rows of the block (cp.async, 128-byte swizzled layout) into a
//              4-deep ring; an x stage is released to the MMA one block later, after the
//              copies have landed and a proxy fence has made them visible to the tensor core.
//   warp 13    allocates TMEM and issues the MMAs from one thread.
//   warps 8-11 epilogue: per block, the fp32 partial times 2*s[n,b] into a register sum
//              (ternary: hi + lo columns once per item, times alpha); then y, or a split-K
//              combine through the workspace (last of the P pieces adds them in order).
// Rows M..15 of the B tile are zero for the whole launch. Every wait is bounded.
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "tc_common.cuh"
#include "tc_kernels.cuh"
#include "wr.h"

namespace wr {
namespace {

using namespace tc;

constexpr int kThreads = 448;   // 8 decode, 4 epilogue, producer, MMA warps
constexpr int kSP = 4;       // packed stages
constexpr int kSX = 4;       // activation stages
constexpr int kBN = 16;      // MMA N (token columns)
constexpr int kXAtom = kBN * 128;

template <bool T>
struct DL {  // decode-kernel layout
  static constexpr int kUnitK = T ? 320 : 256;
  static constexpr int kXStage = T ? 10 * 1024 : 9 * 1024;    // 4 atoms + corrections (Q) / 5 atoms (T)
  static constexpr int kPStage = T ? 8 * 1024 : 8 * 1536;     // room for 8 units of the widest format
  static constexpr int kXOff = 0;
  static constexpr int kPOff = kSX * kXStage;
  static constexpr int kBarOff = kPOff + kSP * kPStage;
  // + barriers and alignment slack, padded so that at most two CTAs share an SM (each
  // holds 256 of the SM's 512 TMEM columns)
  static constexpr int kSmemRaw = kBarOff + 1024 + 1024;
  static constexpr int kSmem = kSmemRaw < 80 * 1024 ? 80 * 1024 : kSmemRaw;
  static constexpr int kQuarterCols = T ? 40 : 32;
  static constexpr int kACols = 2 * kQuarterCols;             // A buffer = half block
  static constexpr int kDCol = 2 * kACols;
  static constexpr int kTmemCols = 256;
};

struct Bars {
  uint64_t pk_full[kSP], pk_empty[kSP], x_full[kSX], x_empty[kSX];
  uint64_t a_full[2], a_empty[2], d_full[2], d_empty[2];
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
__device__ __forceinline__ void q2_quarter(const uint8_t* unit, int r0, int half, int q, uint32_t v[32]) {
  const uint4 c = *reinterpret_cast<const uint4*>(unit + (32 * half + 4 * r0 + q) * 16);
  decode_q2_word_raw(c.x, v + 0);
  decode_q2_word_raw(c.y, v + 8);
  decode_q2_word_raw(c.z, v + 16);
  decode_q2_word_raw(c.w, v + 24);
}

__device__ __forceinline__ void q3_quarter(const uint8_t* unit, int r0, int half, int q, uint32_t v[32]) {
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
  decode_q3_group_raw(w, v);
  decode_q3_group_raw(w + 3, v + 16);
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
  Bars* bars = reinterpret_cast<Bars*>(smem + L::kBarOff);
  __shared__ uint32_t lut_lo[T ? 256 : 1], lut_hi[T ? 256 : 1];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &bars->abort_flag;
  const int M = a.M;

  // zero the activation ring once: rows >= M of every stage stay zero for the whole launch
  for (int i = threadIdx.x; i < kSX * L::kXStage / 16; i += kThreads)
    reinterpret_cast<uint4*>(xs)[i] = make_uint4(0, 0, 0, 0);
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
      // Q2/Q3: the epilogue releases a stage once it has read the corrections; ternary: the MMA
      mbar_init(&bars->x_empty[i], T ? 1 : 4);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->a_full[i], 4);
      mbar_init(&bars->a_empty[i], 1);
      mbar_init(&bars->d_full[i], 1);
      mbar_init(&bars->d_empty[i], 4);
    }
    bars->abort_flag = 0;
    bars->last_flag = 0;
    fence_barrier_init();
  }
  if (warp == 13) tmem_alloc(&bars->tmem_base, L::kTmemCols);
  fence_proxy_async_smem();
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
        const int64_t xtb = xtile_bytes(T, M);
        for (int b = im.b0; b < im.b1; ++b, ++gb) {
          // activation tile (and, for Q2/Q3, its corrections) of block b
          const int sx = gb % kSX;
          if (!(ok = mbar_wait(&bars->x_empty[sx], ((gb / kSX) & 1) ^ 1, abort_flag, a.err, 101))) break;
          mbar_arrive_expect_tx(&bars->x_full[sx], (uint32_t)xtb);
          bulk_load(xs + sx * L::kXStage, pr.xt + (int64_t)b * xtb, (uint32_t)xtb, &bars->x_full[sx]);
          // packed units of block b
          const int sp = gb % kSP;
          if (!(ok = mbar_wait(&bars->pk_empty[sp], ((gb / kSP) & 1) ^ 1, abort_flag, a.err, 102))) break;
          // the ntile units of this row group and block are adjacent: one copy
          mbar_arrive_expect_tx(&bars->pk_full[sp], ntile * ub);
          bulk_load(ps + sp * L::kPStage, pr.packed + ((int64_t)im.rg * 8 * pr.B + (int64_t)b * ntile) * ub,
                    ntile * ub, &bars->pk_full[sp]);
        }
      }
    }
  } else if (warp == 13) {
    // ------------------------------------------------------------ MMA issuer (one thread)
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_m128(kBN);
      constexpr int kChunkSteps = L::kACols / 8;
      // B descriptors of every activation stage, precomputed; MMA j of chunk c adds the byte
      // offset of K position c*(unit/2) + 16 j (>> 4 in the descriptor's address field)
      const uint64_t bdesc0 = smem_desc_sw128(xs);
      const int astr = xatom_stride(T, M);
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
          const uint32_t dcol = tmem + L::kDCol + dbuf * kBN;
          const uint64_t bd = bdesc0 + (uint64_t)((sx * L::kXStage) >> 4);
          const bool first_of_item = b == im.b0;
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            if (!(ok = mbar_wait(&bars->a_full[c], gb & 1, abort_flag, a.err, 204))) break;
            fence_after_sync();
#pragma unroll
            for (int j = 0; j < kChunkSteps; ++j) {
              constexpr int kHalf = L::kUnitK / 2;
              const int kk = c * kHalf + 16 * j;
              const uint64_t off = (uint64_t)(((kk / 64) * astr + (kk % 64) * 2) >> 4);
              const uint32_t acc = T ? (uint32_t)(!first_of_item || c != 0 || j != 0) : (uint32_t)(c != 0 || j != 0);
              mma_ts(dcol, tmem + c * L::kACols + 8 * j, bd + off, idesc, acc);
            }
            mma_commit(&bars->a_empty[c]);
          }
          if (!ok) break;
          if (T) mma_commit(&bars->x_empty[sx]);
          else mma_commit(&bars->d_full[dbuf]);
        }
        if (T && ok) mma_commit(&bars->d_full[dbuf]);
      }
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ decode (thread = row)
    // warp w: lane quarter w % 4 (rows 32*(w%4) .. +31), group w / 4 decodes chunk (w / 4) of
    // every block, i.e. quarters 2g and 2g+1, into A buffer g.
    const int g = warp >> 2, lq = warp & 3;
    const int t = 32 * lq + lane;
    const int tile = t >> 4, r = t & 15, r0 = r & 7, half = r >> 3;
    const uint32_t abase = tmem + ((uint32_t)(32 * lq) << 16) + g * L::kACols;
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
        if (!(ok = mbar_wait(&bars->a_empty[g], (gb & 1) ^ 1, abort_flag, a.err, 302))) break;
        fence_after_sync();
#pragma unroll
        for (int qq = 0; qq < 2; ++qq) {
          const int q = 2 * g + qq;
          const uint32_t col = abase + qq * L::kQuarterCols;
          if (T) {
            uint32_t v[40];
            t_quarter(unit, r0, half, q, lut_lo, lut_hi, v);
            tmem_st32(col, v);
            tmem_st8(col + 32, v + 32);
          } else {
            uint32_t v[32];
            if (bits == 2) q2_quarter(unit, r0, half, q, v);
            else q3_quarter(unit, r0, half, q, v);
            tmem_st32(col, v);
          }
        }
        tmem_wait_st();
        fence_before_sync();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bars->a_full[g]);
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
      float acc[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) acc[i] = 0.f;
      if (T) {
        const uint32_t dbuf = gi & 1;
        gb += im.b1 - im.b0;
        if (!(ok = mbar_wait(&bars->d_full[dbuf], (gi >> 1) & 1, abort_flag, a.err, 401))) break;
        fence_after_sync();
        float d[16];
        tmem_ld16(tmem + lane_addr + L::kDCol + dbuf * kBN, d);
        tmem_wait_ld();
        fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->d_empty[dbuf]);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = d[i] + d[i + 8];
      } else {
        const uint16_t* srow = pr.scales + (int64_t)(n < pr.N ? n : 0) * pr.B;
        uint16_t s_next = __ldg(srow + im.b0);
        for (int b = im.b0; b < im.b1; ++b, ++gb) {
          const uint32_t dbuf = gb & 1;
          const float s2 = n < pr.N ? 2.f * half_bits_to_float(s_next) : 0.f;
          if (b + 1 < im.b1) s_next = __ldg(srow + b + 1);   // one block ahead
          if (!(ok = mbar_wait(&bars->d_full[dbuf], (gb >> 1) & 1, abort_flag, a.err, 402))) break;
          fence_after_sync();
          float d[16];
          tmem_ld16(tmem + lane_addr + L::kDCol + dbuf * kBN, d);
          tmem_wait_ld();
          fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->d_empty[dbuf]);
          // corrections of this block sit after the atoms of its activation stage
          const int sx = gb % kSX;
          if (!(ok = mbar_wait(&bars->x_full[sx], (gb / kSX) & 1, abort_flag, a.err, 403))) break;
          float cr[16];
          const float* cs = reinterpret_cast<const float*>(xs + sx * L::kXStage + 4 * xatom_stride(false, M));
#pragma unroll
          for (int i = 0; i < 16; ++i) cr[i] = cs[i];
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->x_empty[sx]);
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (i < M) acc[i] = fmaf(s2, d[i] - cr[i], acc[i]);
        }
        if (!ok) break;
      }
      const float rs = (T && n < pr.N) ? half_bits_to_float(__ldg(pr.scales + n)) : 1.f;
      if (pr.P == 1) {
        if (n < pr.N) {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (i < M) pr.y[(int64_t)i * pr.N + n] = rs * acc[i];
        }
      } else {
        const int cid = pr.counter_base + im.rg;
        float* part = a.partial + pr.partial_base + ((int64_t)im.rg * pr.P + im.p) * M * 128;
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (i < M) part[i * 128 + t] = acc[i];
        __threadfence();
        named_bar_sync(1, 128);
        if (t == 0) bars->last_flag = (atomicAdd(a.counter + cid, 1) == pr.P - 1);
        named_bar_sync(1, 128);
        if (bars->last_flag) {
          __threadfence();
          float sum[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) sum[i] = 0.f;
          for (int pp = 0; pp < pr.P; ++pp) {
            const float* src = a.partial + pr.partial_base + ((int64_t)im.rg * pr.P + pp) * M * 128;
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (i < M) sum[i] += __ldcg(src + i * 128 + t);
          }
          if (n < pr.N) {
#pragma unroll
            for (int i = 0; i < 16; ++i)
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

// Preparation pass for Q2/Q3 problems: one warp per (problem, block). Writes the block's
// activations pre-scaled by 2^(7-p_k) (exact) as the image of the B stage (atom a = k/64 at
// a * xatom_stride, row m, 16-byte chunk c at position c ^ (m % 8)), followed by
// C_m = sum_k x'_k + (L/2) sum_k x_k for each token (fp32, 16 slots).
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
  uint8_t* dst = pr.xt + (int64_t)b * xtile_bytes(false, M);
  const int astr = xatom_stride(false, M);
  float* corr = reinterpret_cast<float*>(dst + 4 * astr);
  const float half_l = pr.bits == 2 ? 1.5f : 3.5f;
  for (int m = 0; m < M; ++m) {
    const uint4 v = *reinterpret_cast<const uint4*>(pr.x + (int64_t)m * pr.K + (int64_t)b * 256 + 8 * lane);
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float sx = 0.f, sxp = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int k = 8 * lane + 2 * e;
      const int sh = pr.bits == 2 ? q2_shift(k) : q3_shift(k);
      const float f = __int_as_float((127 + sh) << 23);
      float l0 = __uint_as_float(w[e] << 16), h0 = __uint_as_float(w[e] & 0xFFFF0000u);
      sx += l0 + h0;
      l0 *= f;
      h0 *= f;
      sxp += l0 + h0;
      w[e] = (__float_as_uint(h0) & 0xFFFF0000u) | (__float_as_uint(l0) >> 16);
    }
    *reinterpret_cast<uint4*>(dst + (lane >> 3) * astr + m * 128 + (((lane & 7) ^ (m & 7)) << 4)) =
        make_uint4(w[0], w[1], w[2], w[3]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sx += __shfl_xor_sync(0xffffffffu, sx, o);
      sxp += __shfl_xor_sync(0xffffffffu, sxp, o);
    }
    if (lane == 0) corr[m] = sxp + half_l * sx;
  }
  if (lane < 16 && lane >= M) corr[lane] = 0.f;
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
