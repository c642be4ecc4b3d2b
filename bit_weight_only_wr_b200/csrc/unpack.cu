// Materializer: packed codes + scales -> bf16 weights, bit-exact.
//
// The "Qwen3-4B-Wringer-Q2.6" card ("What is in this repo") describes a materializer that
// expands the container into a bf16 checkpoint, bit-identical across independent re-runs.
// Here W[n,k] = bf16_RNE(s * g): the fp32 product of an fp16 scale (11 significant bits; 18 for
// the int8 form d q) and a grid integer (at most 3 bits) is exact, so the one rounding to bf16
// is the only one.
// One warp per packed unit; each lane expands its 64 codes (80 trits) of two rows into shared
// memory, and the warp writes the unit out in whole-row segments. The kernel is bound by the
// 2 bytes/weight it writes.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "tc_kernels.cuh"
#include "wr.h"

namespace wr {
namespace {

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const uint32_t a = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
  const uint32_t b = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
  return a | (b << 16);
}

constexpr int kUnpackWarps = 4;   // one packed unit per warp

template <int FMT>
struct UnpackGeom {
  static constexpr int kUnitK = FMT == WR_FMT_TERNARY ? 320 : 256;    // K positions per unit
  static constexpr int kRowBytes = 2 * kUnitK;                          // one staged row of bf16
  static constexpr int kStride = kRowBytes + 16;                        // padded: rows 4 banks apart
  static constexpr int kChunks = kRowBytes / 16;                        // 16-byte chunks per row
};

// One warp per packed unit (16 rows x 256 codes, or x 320 trits). Each lane expands the 64 codes
// (80 trits) of its two rows into shared memory; the warp then writes the unit row by row, 32
// lanes x 16 bytes = 512 contiguous bytes per store, so that every global store covers whole
// 128-byte lines.
template <int FMT>
__global__ void __launch_bounds__(32 * kUnpackWarps) unpack_kernel(const uint8_t* __restrict__ packed,
                                                                  const uint16_t* __restrict__ scales,
                                                                  const int8_t* __restrict__ scale_q, int N,
                                                                  int K, int B, int64_t U,
                                                                  uint16_t* __restrict__ out) {
  using G = UnpackGeom<FMT>;
  __shared__ __align__(16) uint8_t stage[kUnpackWarps][16 * G::kStride];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t u = (int64_t)blockIdx.x * kUnpackWarps + warp;
  if (u >= U) return;
  uint8_t* st = stage[warp];
  constexpr int UB = FMT == WR_FMT_Q3 ? 1536 : 1024;
  constexpr int kChunks = FMT == WR_FMT_Q3 ? 3 : 2;
  const uint8_t* base = packed + u * UB;
  uint32_t wd[4 * kChunks];
#pragma unroll
  for (int c = 0; c < kChunks; ++c) {
    const uint4 v = ld_stream_v4(base + (32 * c + lane) * 16);
    wd[4 * c + 0] = v.x;
    wd[4 * c + 1] = v.y;
    wd[4 * c + 2] = v.z;
    wd[4 * c + 3] = v.w;
  }
  // unit u -> (tile, block): groups of 8 tiles, each group's units block by block
  const int64_t tiles = (N + 15) / 16;
  const int64_t grp = u / (8 * (int64_t)B);
  const int64_t tg = min((int64_t)8, tiles - 8 * grp);
  const int64_t rem = u - grp * 8 * (int64_t)B;
  const int64_t ub = rem / tg, tn = 8 * grp + rem % tg;
  // this thread read the chunks at position `lane`, which belong to lane lane ^ ((lane >> 3) & 3)
  const int ll = lane ^ ((lane >> 3) & 3);
  const int r0 = ll >> 2, q = ll & 3;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int r = r0 + 8 * h;
    const int64_t n = tn * 16 + r;
    uint4* srow = reinterpret_cast<uint4*>(st + r * G::kStride);
    if (FMT == WR_FMT_TERNARY) {
      const float al = n < N ? half_bits_to_float(scales[n]) : 0.f;
      float v[80];
#pragma unroll
      for (int beta = 0; beta < 16; ++beta) {
        uint32_t byte = (wd[4 * h + beta / 4] >> (8 * (beta % 4))) & 0xFFu;
#pragma unroll
        for (int d = 0; d < 5; ++d) {
          v[5 * beta + d] = al * (float)((int)(byte % 3u) - 1);
          byte /= 3u;
        }
      }
#pragma unroll
      for (int i = 0; i < 10; ++i) {
        uint4 w;
        w.x = pack_bf16x2(v[8 * i + 0], v[8 * i + 1]);
        w.y = pack_bf16x2(v[8 * i + 2], v[8 * i + 3]);
        w.z = pack_bf16x2(v[8 * i + 4], v[8 * i + 5]);
        w.w = pack_bf16x2(v[8 * i + 6], v[8 * i + 7]);
        srow[10 * q + i] = w;
      }
    } else {
      // the fp16 block scale, or d_n q[n,b]: exact in fp32, so s * g stays exact
      const float s = n >= N ? 0.f
                      : scale_q == nullptr ? half_bits_to_float(scales[n * B + ub])
                                           : half_bits_to_float(scales[n]) * (float)scale_q[n * B + ub];
      const int L = FMT == WR_FMT_Q2 ? 3 : 7;
      int c[64];
      if (FMT == WR_FMT_Q2 || FMT == WR_FMT_T2 || FMT == WR_FMT_T8) {
#pragma unroll
        for (int w = 0; w < 4; ++w)
#pragma unroll
          for (int e = 0; e < 16; ++e) c[16 * w + e] = (wd[4 * h + w] >> (16 * (e & 1) + 2 * (e >> 1))) & 3;
      } else {
        const uint32_t* rw = wd + 6 * h;
#pragma unroll
        for (int g = 0; g < 2; ++g) {
#pragma unroll
          for (int uu = 0; uu < 3; ++uu)
#pragma unroll
            for (int f = 0; f < 10; ++f)
              c[32 * g + 10 * uu + f] = (rw[3 * g + uu] >> (16 * (f & 1) + 3 * (f >> 1))) & 7;
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            int cc = 0;
#pragma unroll
            for (int uu = 0; uu < 3; ++uu) cc |= ((rw[3 * g + uu] >> (16 * hh + 15)) & 1) << uu;
            c[32 * g + 30 + hh] = cc;
          }
        }
      }
      if (FMT == WR_FMT_T2) {
        // trellis: level index 2u + (low bit of the previous symbol); the previous symbol of
        // this quarter's first code is the last of quarter q - 1 of the same row (another
        // lane), and 0 at the block start
        const uint32_t prev = __shfl_sync(0xffffffffu, (uint32_t)c[63] & 1u, lane_pos(r0, (q + 3) & 3));
        int p = q == 0 ? 0 : (int)prev;
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const int u = c[i];
          c[i] = 2 * u + p;
          p = u & 1;
        }
      }
      if (FMT == WR_FMT_T8) {
        // 8-state trellis: the state entering this quarter is the low bits of the last codes of
        // quarter q - 1's last three symbols (codes 55, 59, 63 of that lane), 0 at the block start
        const uint32_t es = (((uint32_t)c[55] & 1u) << 2) | (((uint32_t)c[59] & 1u) << 1) | ((uint32_t)c[63] & 1u);
        const uint32_t prev = __shfl_sync(0xffffffffu, es, lane_pos(r0, (q + 3) & 3));
        int st = q == 0 ? 0 : (int)prev;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int p0 = st & 1, p1 = (st >> 1) & 1, p2 = (st >> 2) & 1;
          const int z = c[4 * j + 3] & 1;
          c[4 * j + 0] = 2 * c[4 * j + 0] + p0;
          c[4 * j + 1] = 2 * c[4 * j + 1] + p1;
          c[4 * j + 2] = 2 * c[4 * j + 2] + p2;
          c[4 * j + 3] = 2 * c[4 * j + 3] + (p0 ^ p1 ^ p2);
          st = ((st << 1) | z) & 7;
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        uint4 w;
        w.x = pack_bf16x2(s * (float)(2 * c[8 * i + 0] - L), s * (float)(2 * c[8 * i + 1] - L));
        w.y = pack_bf16x2(s * (float)(2 * c[8 * i + 2] - L), s * (float)(2 * c[8 * i + 3] - L));
        w.z = pack_bf16x2(s * (float)(2 * c[8 * i + 4] - L), s * (float)(2 * c[8 * i + 5] - L));
        w.w = pack_bf16x2(s * (float)(2 * c[8 * i + 6] - L), s * (float)(2 * c[8 * i + 7] - L));
        srow[8 * q + i] = w;
      }
    }
  }
  __syncwarp();
  // row by row: chunk j of row r is K positions k0 + 8j .. k0 + 8j + 7
  const int64_t k0 = ub * G::kUnitK;
  const bool vec = (K & 7) == 0;   // rows start 16-byte aligned
  for (int r = 0; r < 16; ++r) {
    const int64_t n = tn * 16 + r;
    if (n >= N) break;
    uint16_t* orow = out + n * (int64_t)K;
    const uint4* srow = reinterpret_cast<const uint4*>(st + r * G::kStride);
    for (int j = lane; j < G::kChunks; j += 32) {
      const int64_t k = k0 + 8 * j;
      if (k >= K) break;
      const uint4 w = srow[j];
      if (vec && k + 8 <= K) {
        *reinterpret_cast<uint4*>(orow + k) = w;
      } else {
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
        for (int e = 0; e < 8 && k + e < K; ++e) orow[k + e] = (uint16_t)(ww[e >> 1] >> (16 * (e & 1)));
      }
    }
  }
}

}  // namespace

cudaError_t launch_unpack_bf16(int fmt, const uint8_t* packed, const uint16_t* scales, const int8_t* scale_q, int N,
                               int K, int units, uint16_t* w, cudaStream_t stream) {
  const int64_t tiles = (N + 15) / 16;
  const int64_t U = tiles * units;
  const unsigned ctas = (unsigned)((U + kUnpackWarps - 1) / kUnpackWarps);
  constexpr int th = 32 * kUnpackWarps;
  if (fmt == WR_FMT_Q2) unpack_kernel<WR_FMT_Q2><<<ctas, th, 0, stream>>>(packed, scales, scale_q, N, K, units, U, w);
  else if (fmt == WR_FMT_Q3) unpack_kernel<WR_FMT_Q3><<<ctas, th, 0, stream>>>(packed, scales, scale_q, N, K, units, U, w);
  else if (fmt == WR_FMT_T2) unpack_kernel<WR_FMT_T2><<<ctas, th, 0, stream>>>(packed, scales, scale_q, N, K, units, U, w);
  else if (fmt == WR_FMT_T8) unpack_kernel<WR_FMT_T8><<<ctas, th, 0, stream>>>(packed, scales, scale_q, N, K, units, U, w);
  else unpack_kernel<WR_FMT_TERNARY><<<ctas, th, 0, stream>>>(packed, scales, nullptr, N, K, units, U, w);
  return cudaGetLastError();
}

}  // namespace wr
