// Decode GEMV (M <= 8) on packed codes: y[m,n] = sum_b s[n,b] sum_{k in b} g[n,k] x[m,k].
//
// Decoding one token means reading every weight once ("How We Shrank an AI Model by 85%...",
// "Results": generating a token is mostly reading the weights from memory), so this kernel is
// built to stream the packed buffer at HBM speed:
//  * the buffer is a sequence of 16-row x 256-code units (1 KB for Q2, 1.5 KB for Q3); a warp
//    reads a unit with 2-3 coalesced 16-byte loads per lane that bypass L1;
//  * each lane decodes its codes in registers into exact bf16 values g/2 (LOP3 + one bf16x2
//    FMA per pair) laid out directly as the A fragments of m16n8k16 MMAs; the B fragments are
//    the activations of up to 8 tokens, read through L1 from x in natural order;
//  * the 16 MMAs of a unit accumulate the 256-block partial in fp32; the lane then applies
//    2*s[n,b] in fp32 to the running sum of its two rows;
//  * the unit sequence is split evenly over all warps of a persistent grid; a row tile shared
//    by several warps is combined through the workspace: each contributor stores its partial,
//    the last to arrive (per-tile counter) adds all partials in warp order and writes y, then
//    resets the counter to zero.
// The ternary variant reads 16-row x 320-trit units, decodes five trits per byte through a
// shared-memory table, and contracts with R x that a small pre-pass writes (split into
// hi + lo bf16, permuted into fragment order) into the workspace.
#include <cuda_runtime.h>

#include "common.cuh"
#include "gemv.cuh"
#include "wr.h"

namespace wr {

namespace {

constexpr int kWarpsPerCta = 4;

__device__ __forceinline__ int64_t range_begin(int64_t U, int Wt, int w) { return U * w / Wt; }
// Warp whose unit range contains unit u (every warp owns at least one unit).
__device__ __forceinline__ int warp_of_unit(int64_t U, int Wt, int64_t u) {
  return (int)(((u + 1) * Wt - 1) / U);
}

struct TileFrag {
  float c[4];  // rows r0, r0 (cols 2q, 2q+1); rows r0+8 (cols 2q, 2q+1)
};

// Store the finished tile (or its share of it). `rowscale` multiplies the final value
// (alpha for ternary, 1 otherwise) and is applied once, when y is written.
template <bool kTernaryCombine>
__device__ __forceinline__ void finish_tile(const GemvArgs& a, int w, int64_t tn, bool complete,
                                            TileFrag f, int lane) {
  const int r0 = lane >> 2, q = lane & 3;
  const int64_t n0 = tn * 16;
  if (kTernaryCombine) {
    // columns 0..3 carry R x rounded to bf16 (hi), columns 4..7 the remainder (lo)
#pragma unroll
    for (int i = 0; i < 4; ++i) f.c[i] += __shfl_down_sync(0xffffffffu, f.c[i], 2);
  }
  if (!complete) {
    const int64_t first_tile = range_begin(a.U, a.Wt, w) / a.B;
    float* slot = a.partial + (size_t)(2 * w + (tn == first_tile ? 0 : 1)) * 128;
    *reinterpret_cast<float2*>(slot + r0 * 8 + 2 * q) = make_float2(f.c[0], f.c[1]);
    *reinterpret_cast<float2*>(slot + (r0 + 8) * 8 + 2 * q) = make_float2(f.c[2], f.c[3]);
    __threadfence();
    __syncwarp();
    int last = 0;
    const int wa = warp_of_unit(a.U, a.Wt, tn * a.B);
    const int wb = warp_of_unit(a.U, a.Wt, (tn + 1) * a.B - 1);
    if (lane == 0) last = (atomicAdd(a.counter + tn, 1) == wb - wa);
    last = __shfl_sync(0xffffffffu, last, 0);
    if (!last) return;
    __threadfence();
    f.c[0] = f.c[1] = f.c[2] = f.c[3] = 0.f;
    for (int v = wa; v <= wb; ++v) {
      const int64_t ft = range_begin(a.U, a.Wt, v) / a.B;
      const float* s = a.partial + (size_t)(2 * v + (tn == ft ? 0 : 1)) * 128;
      const float2 lo = __ldcg(reinterpret_cast<const float2*>(s + r0 * 8 + 2 * q));
      const float2 hi = __ldcg(reinterpret_cast<const float2*>(s + (r0 + 8) * 8 + 2 * q));
      f.c[0] += lo.x;
      f.c[1] += lo.y;
      f.c[2] += hi.x;
      f.c[3] += hi.y;
    }
    if (lane == 0) a.counter[tn] = 0;
  }
  const int ncols = kTernaryCombine ? 4 : 8;
  const int c0 = 2 * q;
  if (c0 >= ncols) return;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int64_t n = n0 + r0 + 8 * h;
    if (n >= a.N) continue;
    float rs = 1.f;
    if (a.row_scale) rs = half_bits_to_float(a.row_scale[n]);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int m = c0 + e;
      if (m < a.M) a.y[(int64_t)m * a.N + n] = rs * f.c[2 * h + e];
    }
  }
}

// -------------------------------------------------------------------- Q2 / Q3

template <int BITS>
struct UnitRegs {
  static constexpr int kChunks = BITS == 2 ? 2 : 3;
  uint4 c[kChunks];
  float s0, s1;  // 2 * s[n, b] for rows r0 and r0 + 8
};

template <int BITS>
__device__ __forceinline__ void load_unit(const GemvArgs& a, int64_t u, int lane, UnitRegs<BITS>& r) {
  constexpr int UB = BITS == 2 ? 1024 : 1536;
  const uint8_t* base = a.packed + u * UB;
#pragma unroll
  for (int c = 0; c < UnitRegs<BITS>::kChunks; ++c) r.c[c] = ld_stream_v4(base + (32 * c + lane) * 16);
  const int64_t tn = u / a.B, b = u % a.B;
  const int64_t n = tn * 16 + (lane >> 2);
  r.s0 = n < a.N ? 2.f * half_bits_to_float(__ldg(a.scales + n * a.B + b)) : 0.f;
  r.s1 = n + 8 < a.N ? 2.f * half_bits_to_float(__ldg(a.scales + (n + 8) * a.B + b)) : 0.f;
}

template <int BITS>
__device__ __forceinline__ void compute_unit(const GemvArgs& a, int64_t u, int lane,
                                             const UnitRegs<BITS>& r, float acc[4]) {
  const int r0 = lane >> 2, q = lane & 3;
  const int64_t b = u % a.B;
  // B fragments: token r0, k = 256 b + 64 q + 4 j .. +3 for MMA j (8 bytes per MMA)
  uint4 xv[8];
  if (r0 < a.M) {
    const uint16_t* xp = a.x + (int64_t)r0 * a.K + b * 256 + 64 * q;
#pragma unroll
    for (int i = 0; i < 8; ++i) xv[i] = ld_ro_v4(xp + 8 * i);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) xv[i] = make_uint4(0, 0, 0, 0);
  }
  float d[4] = {0.f, 0.f, 0.f, 0.f};
  if (BITS == 2) {
    const uint32_t w0[4] = {r.c[0].x, r.c[0].y, r.c[0].z, r.c[0].w};
    const uint32_t w1[4] = {r.c[1].x, r.c[1].y, r.c[1].z, r.c[1].w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      uint32_t p0[8], p1[8];
      decode_q2_word(w0[w], p0);
      decode_q2_word(w1[w], p1);
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int j = 4 * w + jj;  // MMA index; B words of MMA j are xv[j/2] halves
        const uint32_t b0 = (j & 1) ? xv[j >> 1].z : xv[j >> 1].x;
        const uint32_t b1 = (j & 1) ? xv[j >> 1].w : xv[j >> 1].y;
        mma_bf16_16816(d, p0[2 * jj], p1[2 * jj], p0[2 * jj + 1], p1[2 * jj + 1], b0, b1);
      }
    }
  } else {
    const uint32_t wl[12] = {r.c[0].x, r.c[0].y, r.c[0].z, r.c[0].w, r.c[1].x, r.c[1].y,
                             r.c[1].z, r.c[1].w, r.c[2].x, r.c[2].y, r.c[2].z, r.c[2].w};
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      uint32_t p0[16], p1[16];
      decode_q3_group(wl + 3 * g, p0);
      decode_q3_group(wl + 6 + 3 * g, p1);
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        const int j = 8 * g + jj;
        const uint32_t b0 = (j & 1) ? xv[j >> 1].z : xv[j >> 1].x;
        const uint32_t b1 = (j & 1) ? xv[j >> 1].w : xv[j >> 1].y;
        mma_bf16_16816(d, p0[2 * jj], p1[2 * jj], p0[2 * jj + 1], p1[2 * jj + 1], b0, b1);
      }
    }
  }
  acc[0] = fmaf(r.s0, d[0], acc[0]);
  acc[1] = fmaf(r.s0, d[1], acc[1]);
  acc[2] = fmaf(r.s1, d[2], acc[2]);
  acc[3] = fmaf(r.s1, d[3], acc[3]);
}

template <int BITS>
__global__ void __launch_bounds__(kWarpsPerCta * 32) gemv_q_kernel(GemvArgs a) {
  const int lane = threadIdx.x & 31;
  const int w = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  if (w >= a.Wt) return;
  const int64_t u0 = range_begin(a.U, a.Wt, w), u1 = range_begin(a.U, a.Wt, w + 1);
  UnitRegs<BITS> cur, nxt;
  load_unit<BITS>(a, u0, lane, cur);
  TileFrag f = {{0.f, 0.f, 0.f, 0.f}};
  int64_t tile_first = u0;
  for (int64_t u = u0; u < u1; ++u) {
    if (u + 1 < u1) load_unit<BITS>(a, u + 1, lane, nxt);
    compute_unit<BITS>(a, u, lane, cur, f.c);
    const int64_t tn = u / a.B;
    if (u + 1 == u1 || (u + 1) % a.B == 0) {
      const bool complete = tile_first == tn * a.B && u + 1 == (tn + 1) * a.B;
      finish_tile<false>(a, w, tn, complete, f, lane);
      f.c[0] = f.c[1] = f.c[2] = f.c[3] = 0.f;
      tile_first = u + 1;
    }
    cur = nxt;
  }
}

// -------------------------------------------------------------------- ternary

// Table of the 243 byte values: five trits (little-endian base 3) as 2-bit codes at bits
// 1, 3, 5, 9, 11; the high-half table is the same shifted by 16.
__device__ __forceinline__ uint32_t trit_entry(int v) {
  const int slot[5] = {1, 3, 5, 9, 11};
  uint32_t e = 0;
  for (int d = 0; d < 5; ++d) {
    e |= (uint32_t)(v % 3) << slot[d];
    v /= 3;
  }
  return e;
}

struct TritRegs {
  uint4 c[2];  // row r0, row r0 + 8: 16 bytes = 80 trits each
};

__device__ __forceinline__ void load_trit_unit(const GemvArgs& a, int64_t u, int lane, TritRegs& r) {
  const uint8_t* base = a.packed + u * 1024;
  r.c[0] = ld_stream_v4(base + lane * 16);
  r.c[1] = ld_stream_v4(base + (32 + lane) * 16);
}

// One row's 16 bytes -> 40 pair registers: byte pair (2b', 2b'+1) gives pairs 5b'..5b'+4,
// pair i = (trit i of byte 2b', trit i of byte 2b'+1).
__device__ __forceinline__ void decode_trit_row(const uint4& c, const uint32_t* lut_lo,
                                                const uint32_t* lut_hi, uint32_t p[40]) {
  const uint32_t wv[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
  for (int w = 0; w < 4; ++w) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t bA = (wv[w] >> (16 * h)) & 0xFFu, bB = (wv[w] >> (16 * h + 8)) & 0xFFu;
      const uint32_t e = lut_lo[bA] | lut_hi[bB];
      decode_trit_pairs(e, p + 5 * (2 * w + h));
    }
  }
}

__global__ void __launch_bounds__(kWarpsPerCta * 32) gemv_ternary_kernel(GemvArgs a) {
  __shared__ uint32_t lut_lo[256], lut_hi[256];
  for (int i = threadIdx.x; i < 256; i += blockDim.x) {
    const uint32_t e = i < 243 ? trit_entry(i) : 0u;
    lut_lo[i] = e;
    lut_hi[i] = e << 16;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int w = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  if (w >= a.Wt) return;
  const int r0 = lane >> 2, q = lane & 3;
  // B operand: for M <= 4 one pass, columns 0..3 = hi of tokens 0..3, 4..7 = lo;
  // for M > 4 two passes (hi, then lo), column = token.
  const bool split_cols = a.M <= 4;
  const int passes = split_cols ? 1 : 2;
  const int64_t Kp = (int64_t)a.B * 320;
  const int64_t u0 = range_begin(a.U, a.Wt, w), u1 = range_begin(a.U, a.Wt, w + 1);
  TritRegs cur, nxt;
  load_trit_unit(a, u0, lane, cur);
  TileFrag f = {{0.f, 0.f, 0.f, 0.f}};
  int64_t tile_first = u0;
  for (int64_t u = u0; u < u1; ++u) {
    if (u + 1 < u1) load_trit_unit(a, u + 1, lane, nxt);
    const int64_t ub = u % a.B;
    uint32_t p0[40], p1[40];
    decode_trit_row(cur.c[0], lut_lo, lut_hi, p0);
    decode_trit_row(cur.c[1], lut_lo, lut_hi, p1);
    for (int pass = 0; pass < passes; ++pass) {
      int plane, tok;
      if (split_cols) {
        plane = r0 >> 2;
        tok = r0 & 3;
      } else {
        plane = pass;
        tok = r0;
      }
      uint4 xv[10];
      if (tok < a.M) {
        const uint16_t* xp = a.xr + ((int64_t)plane * a.M + tok) * Kp + ub * 320 + 80 * q;
#pragma unroll
        for (int i = 0; i < 10; ++i) xv[i] = ld_ro_v4(xp + 8 * i);
      } else {
#pragma unroll
        for (int i = 0; i < 10; ++i) xv[i] = make_uint4(0, 0, 0, 0);
      }
      float* dst = f.c;
      float dl[4] = {0.f, 0.f, 0.f, 0.f};
      if (pass == 1) dst = dl;
#pragma unroll
      for (int j = 0; j < 20; ++j) {
        const uint32_t b0 = (j & 1) ? xv[j >> 1].z : xv[j >> 1].x;
        const uint32_t b1 = (j & 1) ? xv[j >> 1].w : xv[j >> 1].y;
        mma_bf16_16816(dst, p0[2 * j], p1[2 * j], p0[2 * j + 1], p1[2 * j + 1], b0, b1);
      }
      if (pass == 1) {
#pragma unroll
        for (int i = 0; i < 4; ++i) f.c[i] += dl[i];
      }
    }
    const int64_t tn = u / a.B;
    if (u + 1 == u1 || (u + 1) % a.B == 0) {
      const bool complete = tile_first == tn * a.B && u + 1 == (tn + 1) * a.B;
      if (split_cols) finish_tile<true>(a, w, tn, complete, f, lane);
      else finish_tile<false>(a, w, tn, complete, f, lane);
      f.c[0] = f.c[1] = f.c[2] = f.c[3] = 0.f;
      tile_first = u + 1;
    }
    cur = nxt;
  }
}

// R x for the ternary GEMV: one warp per (token, 128-block). x' = (1/sqrt(128)) H (d * x) in
// fp32, split into hi = bf16(x') and lo = bf16(x' - hi), and written in the order the GEMV
// reads its B fragments: position u*320 + 80q + 4j + e holds trit k with q = (k%320)/80,
// byte beta = (k%80)/5, digit i = k%5, pair P = 5*(beta/2) + i, j = P/2,
// e = 2*(P%2) + beta%2. Positions of pad trits hold zero.
__global__ void rotate_x_kernel(const uint16_t* __restrict__ x, const uint32_t* __restrict__ signs,
                                uint16_t* __restrict__ xr, int M, int K, int64_t Kp) {
  const int lane = threadIdx.x & 31;
  const int64_t item = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t nblk = (Kp + 127) / 128;   // includes pad blocks, written as zero
  if (item >= (int64_t)M * nblk) return;
  const int m = (int)(item / nblk);
  const int64_t k0 = (item % nblk) * 128;
  float v[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t k = k0 + 4 * lane + i;
    float xv = 0.f;
    if (k < K) {
      xv = __bfloat162float(__ushort_as_bfloat16(x[(int64_t)m * K + k]));
      if ((signs[k >> 5] >> (k & 31)) & 1u) xv = -xv;
    }
    v[i] = xv;
  }
  // butterflies of distance 1 and 2 inside the lane, 4..64 across lanes
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
    const int kk = (int)(k % 320), qq = kk / 80, i80 = kk % 80, beta = i80 / 5, dig = i80 % 5;
    const int P = 5 * (beta >> 1) + dig, j = P >> 1, e = 2 * (P & 1) + (beta & 1);
    const int64_t pos = u * 320 + 80 * qq + 4 * j + e;
    xr[(int64_t)m * Kp + pos] = __bfloat16_as_ushort(hi);
    xr[((int64_t)M + m) * Kp + pos] = __bfloat16_as_ushort(lo);
  }
}

}  // namespace

cudaError_t launch_gemv(int fmt, const GemvArgs& a, int ctas, cudaStream_t stream) {
  if (fmt == WR_FMT_Q2) gemv_q_kernel<2><<<ctas, kWarpsPerCta * 32, 0, stream>>>(a);
  else if (fmt == WR_FMT_Q3) gemv_q_kernel<3><<<ctas, kWarpsPerCta * 32, 0, stream>>>(a);
  else gemv_ternary_kernel<<<ctas, kWarpsPerCta * 32, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_rotate_x(const uint16_t* x, const uint32_t* signs, uint16_t* xr, int M, int K,
                            int64_t Kp, cudaStream_t stream) {
  const int64_t items = (int64_t)M * ((Kp + 127) / 128);
  const int warps = 8;
  const int64_t ctas = (items + warps - 1) / warps;
  rotate_x_kernel<<<(unsigned)ctas, warps * 32, 0, stream>>>(x, signs, xr, M, K, Kp);
  return cudaGetLastError();
}

int gemv_warps_per_cta() { return kWarpsPerCta; }

}  // namespace wr
