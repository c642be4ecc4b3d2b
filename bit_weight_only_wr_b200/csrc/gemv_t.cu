// Decode GEMV (M <= 8 tokens) for ternary weights on bf16 tensor cores, for one problem or a
// batch of independent problems.
//
// The weights are ternary (the news item on ternarizing Qwen3-4B to W1.58A16) in a rotated
// basis ("How We Shrank an AI Model by 85%...", "Trick 1: rotate the weights first": store W R^T,
// apply R to x): y[m,n] = alpha[n] sum_k t[n,k] (R x[m,:])[k]. The rotation pass has already
// written, per 320-trit block, R x as hi + lo bf16 parts in B rows m and 8 + m; t is exact in
// bf16, so the tensor cores see the exact product of t with hi + lo.
//
// Each CTA walks a list of work items (problem, 128-row group, range of 320-trit blocks);
// the accumulator of an item collects all its blocks (alpha is per row), so the epilogue runs
// once per item.
// Warp roles (448 threads, two CTAs per SM):
//   warps 0-7  decode: thread = weight row (TMEM lane); warp group g = w / 4 decodes half g of
//              every block (two quarters of 80 trits) through a 5-trits-per-byte table and
//              stores the bf16 values to A buffer g.
//   warp 12    producer: per block one bulk copy for the 8 packed units of the row group and
//              one for the activation tile.
//   warp 13    allocates TMEM and issues the MMAs (10 per half block; the whole warp walks the
//              blocks and one elected lane issues).
//   warps 8-11 epilogue: hi + lo columns summed, times alpha; then y, or a split-K combine
//              through the workspace (the last of the P pieces to arrive adds them in order).
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

constexpr int kThreads = 448;   // 8 decode, 4 epilogue, producer, MMA warps
constexpr int kSP = 5;          // packed stages
constexpr int kSX = 6;          // activation stages
constexpr int kBN = 16;         // accumulator columns: hi rows 0-7, lo rows 8-15
constexpr int kXStage = 10 * 1024;
constexpr int kPStage = 8 * 1024;
constexpr int kXOff = 0;
constexpr int kPOff = kSX * kXStage;
constexpr int kBarOff = kPOff + kSP * kPStage;
// + barriers and alignment slack; at most two CTAs per SM (each holds 256 TMEM columns)
constexpr int kSmem = kBarOff + 1024 + 1024;
static_assert(3 * kSmem > 228 * 1024, "at most two CTAs per SM");
constexpr int kQuarterCols = 40;                // 80 trits as bf16 pairs
constexpr int kABuf = 2 * kQuarterCols;         // half block
constexpr int kDCol = 2 * kABuf;
constexpr int kTmemCols = 256;
static_assert(kDCol + 2 * kBN <= kTmemCols, "tensor memory budget");

struct Bars {
  uint64_t pk_full[kSP], pk_empty[kSP], x_full[kSX], x_empty[kSX];
  uint64_t a_full[2], a_empty[2], d_full[2], d_empty[2];
  uint64_t group;   // the 4 epilogue warps meet here (bounded, unlike bar.sync)
  uint64_t drain;   // MMA completion on the way out of an aborted CTA
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

// One thread's quarter (80 trits) of a 16-row tile unit as bf16 pairs; see the packed layout
// in include/wr.h.
__device__ __forceinline__ void t_quarter(const uint8_t* unit, int r0, int half, int q, const uint32_t* lut_lo,
                                          const uint32_t* lut_hi, uint32_t v[40]) {
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

// Table entry of a base-3 byte: its five trits at the bit slots decode_trit_pairs reads.
__device__ __forceinline__ uint32_t trit_entry(int v) {
  const int slot[5] = {1, 3, 5, 9, 11};
  uint32_t e = 0;
  for (int d = 0; d < 5; ++d) {
    e |= (uint32_t)(v % 3) << slot[d];
    v /= 3;
  }
  return e;
}

__global__ void __launch_bounds__(kThreads, 2) gemv_t_kernel(const __grid_constant__ DecArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* xs = smem + kXOff;
  uint8_t* ps = smem + kPOff;
  Bars* bars = reinterpret_cast<Bars*>(smem + kBarOff);
  __shared__ uint32_t lut_lo[256], lut_hi[256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &bars->abort_flag;
  const int M = a.M;

  for (int i = threadIdx.x; i < 256; i += kThreads) {
    const uint32_t e = i < 243 ? trit_entry(i) : 0u;
    lut_lo[i] = e;
    lut_hi[i] = e << 16;
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
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->a_full[i], 4);
      mbar_init(&bars->a_empty[i], 1);
      mbar_init(&bars->d_full[i], 1);
      mbar_init(&bars->d_empty[i], 4);
    }
    mbar_init(&bars->group, 4);
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    bars->last_flag = 0;
    fence_barrier_init();
  }
  if (warp == 13) tmem_alloc(&bars->tmem_base, kTmemCols);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 12) {
    // ------------------------------------------------------------ producer (one thread)
    if (lane == 0) {
      uint32_t gb = 0, nx = 0, np = 0;
      bool ok = true;
      const uint32_t xtb = (uint32_t)xtile_bytes(true, M);
      for (int it = blockIdx.x; it < a.items && ok; it += gridDim.x) {
        const Item im = find_item(a, it);
        const DecProblem& pr = a.prob[im.pi];
        const int ntile = min(8, (pr.N + 15) / 16 - im.rg * 8);
        for (int b = im.b0; b < im.b1; ++b, ++gb) {
          const int sx = gb % kSX;
          if (!(ok = mbar_wait_bg(&bars->x_empty[sx], ((gb / kSX) & 1) ^ 1, abort_flag, a.err, 101))) break;
          mbar_arrive_expect_tx(&bars->x_full[sx], xtb);
          bulk_load(xs + sx * kXStage, pr.xt + (int64_t)b * xtb, xtb, &bars->x_full[sx]);
          ++nx;
          // the ntile units of this row group and block are adjacent: one copy
          const int sp = gb % kSP;
          if (!(ok = mbar_wait_bg(&bars->pk_empty[sp], ((gb / kSP) & 1) ^ 1, abort_flag, a.err, 102))) break;
          mbar_arrive_expect_tx(&bars->pk_full[sp], ntile * 1024);
          bulk_load(ps + sp * kPStage, pr.packed + ((int64_t)im.rg * 8 * pr.B + (int64_t)b * ntile) * 1024,
                    ntile * 1024, &bars->pk_full[sp]);
          ++np;
        }
      }
      if (!ok) {
        // aborted: let the copies in flight land before the CTA exits
        for (uint32_t k = np > kSP ? np - kSP : 0; k < np; ++k) mbar_wait_drain(&bars->pk_full[k % kSP], (k / kSP) & 1);
        for (uint32_t k = nx > kSX ? nx - kSX : 0; k < nx; ++k) mbar_wait_drain(&bars->x_full[k % kSX], (k / kSX) & 1);
      }
    }
  } else if (warp == 13) {
    // ------------------------------------------------------------ MMA issuer (whole warp, one lane issues)
    const uint64_t bdesc0 = smem_desc_sw128(xs);
    constexpr uint32_t idesc = idesc_bf16_m128(16);
    uint32_t gb = 0, gi = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < a.items && ok; it += gridDim.x, ++gi) {
      const Item im = find_item(a, it);
      const uint32_t dbuf = gi & 1;
      if (!(ok = mbar_wait_bg(&bars->d_empty[dbuf], ((gi >> 1) & 1) ^ 1, abort_flag, a.err, 201))) break;
      const uint32_t dcol = tmem + kDCol + dbuf * kBN;
      for (int b = im.b0; b < im.b1 && ok; ++b, ++gb) {
        const int sx = gb % kSX;
        if (!(ok = mbar_wait_bg(&bars->x_full[sx], (gb / kSX) & 1, abort_flag, a.err, 202))) break;
        const uint64_t bd = bdesc0 + (uint64_t)((sx * kXStage) >> 4);
        // two half-block A buffers, bf16 MMAs of K = 16 over 5 atoms of 16 rows
        const bool first_of_item = b == im.b0;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          if (!(ok = mbar_wait_bg(&bars->a_full[c], gb & 1, abort_flag, a.err, 203))) break;
          fence_after_sync();
#pragma unroll
          for (int j = 0; j < 10; ++j) {
            const int kk = c * 160 + 16 * j;
            const uint64_t off = (uint64_t)(((kk / 64) * 2048 + (kk % 64) * 2) >> 4);
            mma_ts_elect(dcol, tmem + c * kABuf + 8 * j, bd + off, idesc,
                   (uint32_t)(!first_of_item || c != 0 || j != 0));
          }
          mma_commit_elect(&bars->a_empty[c]);
        }
        if (!ok) break;
        mma_commit_elect(&bars->x_empty[sx]);
      }
      if (ok) mma_commit_elect(&bars->d_full[dbuf]);
    }
    // the MMAs already issued finish before tensor memory is released
    if (!ok) {
      mma_commit_elect(&bars->drain);
      mbar_wait_drain(&bars->drain, 0);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ decode (thread = row)
    // warp w: lane quarter w % 4 (rows 32*(w%4) .. +31); group g = w / 4 decodes quarters 2g and
    // 2g+1 of every block into A buffer g.
    const int g = warp >> 2, lq = warp & 3;
    const int t = 32 * lq + lane;
    const int tile = t >> 4, r = t & 15, r0 = r & 7, half = r >> 3;
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * lq) << 16);
    uint32_t gb = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < a.items && ok; it += gridDim.x) {
      const Item im = find_item(a, it);
      for (int b = im.b0; b < im.b1; ++b, ++gb) {
        const int sp = gb % kSP;
        if (!(ok = mbar_wait(&bars->pk_full[sp], (gb / kSP) & 1, abort_flag, a.err, 301))) break;
        const uint8_t* unit = ps + sp * kPStage + tile * 1024;
        if (!(ok = mbar_wait(&bars->a_empty[g], (gb & 1) ^ 1, abort_flag, a.err, 302))) break;
        fence_after_sync();
#pragma unroll
        for (int qq = 0; qq < 2; ++qq) {
          uint32_t v[40];
          t_quarter(unit, r0, half, 2 * g + qq, lut_lo, lut_hi, v);
          const uint32_t col = lane_addr + g * kABuf + qq * kQuarterCols;
          tmem_st32(col, v);
          tmem_st8(col + 32, v + 32);
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
    uint32_t gi = 0, ng = 0;
    bool ok = true;
    auto group_sync = [&](int code) {
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->group);
      return mbar_wait(&bars->group, (ng++) & 1, abort_flag, a.err, code);
    };
    for (int it = blockIdx.x; it < a.items && ok; it += gridDim.x, ++gi) {
      const Item im = find_item(a, it);
      const DecProblem& pr = a.prob[im.pi];
      const int n = im.rg * 128 + t;
      const uint32_t dbuf = gi & 1;
      if (!(ok = mbar_wait(&bars->d_full[dbuf], (gi >> 1) & 1, abort_flag, a.err, 401))) break;
      fence_after_sync();
      float d[16];
      tmem_ld16(tmem + lane_addr + kDCol + dbuf * kBN, d);
      tmem_wait_ld();
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->d_empty[dbuf]);
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = d[i] + d[i + 8];
      const float rs = n < pr.N ? half_bits_to_float(__ldg(pr.scales + n)) : 1.f;
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
        if (!(ok = group_sync(402))) break;
        if (t == 0) bars->last_flag = (atomicAdd(a.counter + cid, 1) == pr.P - 1);
        if (!(ok = group_sync(403))) break;
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
      }
    }
  }

  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 13) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

cudaError_t launch_gemv_t(const DecArgs& a, int grid, cudaStream_t stream) {
  static bool set = false;
  if (!set) {
    const cudaError_t e = cudaFuncSetAttribute(gemv_t_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    set = true;
  }
  gemv_t_kernel<<<grid, kThreads, kSmem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace wr
