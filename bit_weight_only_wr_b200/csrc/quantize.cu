// Device quantizer and packer for the 2/3-bit odd grid: fp32 weights -> fp16 block scales and
// packed codes, in one pass over W.
//
// Per 256-weight block of a row: s = fp16(absmax / L), the division in fp64 and one rounding to
// fp16, so the scale is fixed before the codes are chosen ("Agents-A1-4B-Wringer-Q2.6" card,
// "Honest caveats"); then each weight takes the nearest odd level of w / s, clamped to
// [-L, L], an exact even quotient going up ("Qwen3-4B-Wringer-Q2.6" card, "Recipe":
// nearest-point codes). s = 0 (and s = inf) give level +1.
//
// The level is decided without a division. The nearest odd level of q = w / s is
// 2 floor(q / 2) + 1, so its code c = (g + L) / 2 is the number of even boundaries m in
// {-L+1, -L+3, ..., L-1} with q >= m, and with s > 0 that is w >= m s. m s is exact in fp32
// (|m| <= 6 times an 11-bit significand), so every comparison is exact: the same decision as
// the fp64 quotient, whose rounding cannot cross an even boundary (a w that is not m s differs
// from it by at least 2^-24 relative, far above the quotient's 2^-53).
//
// One warp per packed unit (16 rows x 256 codes). Lane l = 4 r0 + q holds the 64 weights of
// quarter q of rows r0 and r0 + 8, the 4 lanes of a row find the block's absmax by two
// shuffles, and each lane writes its own 16-byte chunks of the unit (see the packed layout in
// include/wr.h). W is read once, with 16-byte loads.
//
// Int8 block scales (the "Agents-A1-4B-Wringer-Q2.6" card, "What is in this repo": fp16 / int8
// block scales): a first pass finds each row's absmax A and writes d = fp16(A / (127 L))
// (fp64 division, one rounding, saturated to 65504); the pack pass then takes
// q = rint(absmax / (L d)) in fp64 (ties to even), clamped to [0, 127], and chooses the codes
// against s = d q, exact in fp32 (at most 18 significant bits, so m s stays exact too). W is
// read twice on this path.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "tc_kernels.cuh"
#include "wr.h"

namespace wr {
namespace {

constexpr int kQWarps = 8;   // units (rows, for the row pass) per CTA

// Row pass of the int8 form: d[n] = fp16(max_k |w[n,k]| / (127 L)), saturated to 65504.
__global__ void __launch_bounds__(32 * kQWarps) row_scale_kernel(const float* __restrict__ w, int N, int K, int L,
                                                                 uint16_t* __restrict__ d) {
  const int lane = threadIdx.x & 31;
  const int64_t n = (int64_t)blockIdx.x * kQWarps + (threadIdx.x >> 5);
  if (n >= N) return;   // whole warps leave together
  const float4* src = reinterpret_cast<const float4*>(w + n * (int64_t)K);
  float am = 0.f;
  for (int i = lane; i < K / 4; i += 32) {
    const float4 f = __ldg(src + i);
    am = fmaxf(am, fmaxf(fmaxf(fabsf(f.x), fabsf(f.y)), fmaxf(fabsf(f.z), fabsf(f.w))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
  if (lane == 0) {
    uint16_t h = __half_as_ushort(__double2half((double)am / (double)(127 * L)));
    if ((h & 0x7FFFu) >= 0x7C00u) h = 0x7BFFu;
    d[n] = h;
  }
}

template <int BITS, bool S8>
__global__ void __launch_bounds__(32 * kQWarps) quantize_pack_kernel(const float* __restrict__ w, int N, int K,
                                                                    int B, int64_t U, uint8_t* __restrict__ packed,
                                                                    uint16_t* __restrict__ scales,
                                                                    int8_t* __restrict__ scale_q) {
  constexpr int L = (1 << BITS) - 1;
  constexpr int UB = BITS == 2 ? 1024 : 1536;
  const int lane = threadIdx.x & 31;
  const int64_t u = (int64_t)blockIdx.x * kQWarps + (threadIdx.x >> 5);
  if (u >= U) return;   // whole warps leave together: U is counted in warps
  // unit u -> (tile, block): groups of 8 tiles, each group's units block by block
  const int64_t tiles = (N + 15) / 16;
  const int64_t grp = u / (8 * (int64_t)B);
  const int64_t tg = min((int64_t)8, tiles - 8 * grp);
  const int64_t rem = u - grp * 8 * (int64_t)B;
  const int64_t ub = rem / tg, tn = 8 * grp + rem % tg;
  const int r0 = lane >> 2, q = lane & 3;
  uint8_t* unit = packed + u * UB;
  const int pos = lane_pos(r0, q);
#pragma unroll 1
  for (int h = 0; h < 2; ++h) {
    const int64_t n = tn * 16 + r0 + 8 * h;
    const bool real = n < N;
    float v[64];
    if (real) {
      const float4* src = reinterpret_cast<const float4*>(w + n * (int64_t)K + ub * 256 + 64 * q);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float4 f = __ldg(src + i);
        v[4 * i] = f.x;
        v[4 * i + 1] = f.y;
        v[4 * i + 2] = f.z;
        v[4 * i + 3] = f.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 64; ++i) v[i] = 0.f;
    }
    float am = 0.f;
#pragma unroll
    for (int i = 0; i < 64; ++i) am = fmaxf(am, fabsf(v[i]));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
    float s;
    if (S8) {
      // d was written by the row pass (an earlier launch on the same stream)
      const double d = real ? (double)__half2float(__ushort_as_half(scales[n])) : 0.0;
      double qv = d > 0.0 ? rint((double)am / ((double)L * d)) : 0.0;
      qv = fmin(127.0, fmax(0.0, qv));
      if (real && q == 0) scale_q[n * (int64_t)B + ub] = (int8_t)qv;
      s = (float)(d * qv);
    } else {
      const __half sh = __double2half((double)am / (double)L);
      s = __half2float(sh);
      if (real && q == 0) scales[n * (int64_t)B + ub] = __half_as_ushort(sh);
    }
    const bool unit_level = !(s > 0.f) || isinf(s);   // s = 0 or inf: level +1
    // code of weight i (pad rows: code 0)
    auto code = [&](int i) -> uint32_t {
      uint32_t k = 0;
#pragma unroll
      for (int m = -L + 1; m < L; m += 2) k += v[i] >= (float)m * s ? 1u : 0u;
      return !real ? 0u : (unit_level ? (uint32_t)((L + 1) / 2) : k);
    };
    if (BITS == 2) {
      // 4 words of 16 codes: code e of a word at bits 16 (e & 1) + 2 (e >> 1); row half h is
      // chunk h of the lane
      uint32_t wd[4];
#pragma unroll
      for (int ww = 0; ww < 4; ++ww) {
        uint32_t x = 0;
#pragma unroll
        for (int e = 0; e < 16; ++e) x |= code(16 * ww + e) << (16 * (e & 1) + 2 * (e >> 1));
        wd[ww] = x;
      }
      *reinterpret_cast<uint4*>(unit + (32 * h + pos) * 16) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
    } else {
      // 2 groups of 3 words of 32 codes: code 10 u + f at bits 16 (f & 1) + 3 (f >> 1) of word
      // u; bit u of codes 30 + hh at bit 16 hh + 15 of word u. Row half h is lane bytes
      // 24 h .. 24 h + 23.
      uint32_t wd[6];
#pragma unroll
      for (int g = 0; g < 2; ++g) {
#pragma unroll
        for (int uu = 0; uu < 3; ++uu) {
          uint32_t x = 0;
#pragma unroll
          for (int f = 0; f < 10; ++f) x |= code(32 * g + 10 * uu + f) << (16 * (f & 1) + 3 * (f >> 1));
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) x |= ((code(32 * g + 30 + hh) >> uu) & 1u) << (16 * hh + 15);
          wd[3 * g + uu] = x;
        }
      }
      if (h == 0) {
        *reinterpret_cast<uint4*>(unit + pos * 16) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
        *reinterpret_cast<uint2*>(unit + (32 + pos) * 16) = make_uint2(wd[4], wd[5]);
      } else {
        *reinterpret_cast<uint2*>(unit + (32 + pos) * 16 + 8) = make_uint2(wd[0], wd[1]);
        *reinterpret_cast<uint4*>(unit + (64 + pos) * 16) = make_uint4(wd[2], wd[3], wd[4], wd[5]);
      }
    }
  }
}

}  // namespace

cudaError_t launch_quantize_pack(int bits, const float* w, int N, int K, uint8_t* packed, uint16_t* scales,
                                 int8_t* scale_q, cudaStream_t stream) {
  const int B = K / 256;
  const int64_t U = (int64_t)((N + 15) / 16) * B;
  const unsigned ctas = (unsigned)((U + kQWarps - 1) / kQWarps);
  constexpr int th = 32 * kQWarps;
  if (scale_q != nullptr) {
    row_scale_kernel<<<(unsigned)((N + kQWarps - 1) / kQWarps), th, 0, stream>>>(w, N, K, (1 << bits) - 1, scales);
    if (bits == 2) quantize_pack_kernel<2, true><<<ctas, th, 0, stream>>>(w, N, K, B, U, packed, scales, scale_q);
    else quantize_pack_kernel<3, true><<<ctas, th, 0, stream>>>(w, N, K, B, U, packed, scales, scale_q);
  } else {
    if (bits == 2) quantize_pack_kernel<2, false><<<ctas, th, 0, stream>>>(w, N, K, B, U, packed, scales, nullptr);
    else quantize_pack_kernel<3, false><<<ctas, th, 0, stream>>>(w, N, K, B, U, packed, scales, nullptr);
  }
  return cudaGetLastError();
}

}  // namespace wr
