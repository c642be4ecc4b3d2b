// Device helpers shared by the libwr kernels: loads and the register decoders that turn
// packed codes into exact bf16 grid values or integer codes.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace wr {

// ---------------------------------------------------------------- loads

// Streaming 16-byte load: read once, do not keep in L1 (the weights are touched once).
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// ---------------------------------------------------------------- exact code decoders
//
// A pair register holds two bf16 weights (low half: even code, high half: odd code).
// A code field c of width w placed at mantissa bits p..p+w-1 of bf16 1.0 (0x3F80) reads as
// 1 + c*2^(p-7). One fused multiply-add with power-of-two scale 2^(7-p) and offset
// -(2^(7-p) + o) yields c - o exactly (the result is a small multiple of 1/2 and the
// offset has at most 8 significant bits). With o = L/2 the result is g/2 = c - L/2, the
// grid level halved; with o = 1 (ternary) it is t = c - 1.

constexpr uint32_t kOneBf16x2 = 0x3F803F80u;

__device__ __forceinline__ uint32_t bf16x2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// bf16x2 constants (both halves equal).
constexpr uint32_t kB64 = 0x42804280u, kB16 = 0x41804180u, kB4 = 0x40804080u, kB8 = 0x41004100u;
constexpr uint32_t kBm65_5 = 0xC283C283u, kBm17_5 = 0xC18CC18Cu, kBm5_5 = 0xC0B0C0B0u;  // Q2: o = 1.5
constexpr uint32_t kBm67_5 = 0xC287C287u, kBm11_5 = 0xC138C138u;                      // Q3: o = 3.5
constexpr uint32_t kBm65 = 0xC282C282u, kBm17 = 0xC188C188u, kBm5 = 0xC0A0C0A0u;      // ternary: o = 1

// Q2 word -> 8 pair registers of g/2 values. Pair j = codes (2j, 2j+1) at bits 2j, 16+2j.
__device__ __forceinline__ void decode_q2_word(uint32_t w, uint32_t p[8]) {
  const uint32_t t0 = w << 1, t1 = w >> 5, t2 = w >> 11;
  p[0] = bf16x2_fma((t0 & 0x00060006u) | kOneBf16x2, kB64, kBm65_5);
  p[1] = bf16x2_fma((t0 & 0x00180018u) | kOneBf16x2, kB16, kBm17_5);
  p[2] = bf16x2_fma((t0 & 0x00600060u) | kOneBf16x2, kB4, kBm5_5);
  p[3] = bf16x2_fma((t1 & 0x00060006u) | kOneBf16x2, kB64, kBm65_5);
  p[4] = bf16x2_fma((t1 & 0x00180018u) | kOneBf16x2, kB16, kBm17_5);
  p[5] = bf16x2_fma((t1 & 0x00600060u) | kOneBf16x2, kB4, kBm5_5);
  p[6] = bf16x2_fma((t2 & 0x00060006u) | kOneBf16x2, kB64, kBm65_5);
  p[7] = bf16x2_fma((t2 & 0x00180018u) | kOneBf16x2, kB16, kBm17_5);
}

// Q3 group (3 words, 32 codes) -> 16 pair registers of g/2 values. Word u holds pairs
// 5u..5u+4 as 3-bit fields at bits 3j (low half) and 16+3j (high half); pair 15 is spread
// over bit 15 / bit 31 of the three words.
__device__ __forceinline__ void decode_q3_group(const uint32_t w[3], uint32_t p[16]) {
#pragma unroll
  for (int u = 0; u < 3; ++u) {
    const uint32_t t0 = w[u] << 1, t1 = w[u] >> 5, t2 = w[u] >> 11;
    p[5 * u + 0] = bf16x2_fma((t0 & 0x000E000Eu) | kOneBf16x2, kB64, kBm67_5);
    p[5 * u + 1] = bf16x2_fma((t0 & 0x00700070u) | kOneBf16x2, kB8, kBm11_5);
    p[5 * u + 2] = bf16x2_fma((t1 & 0x000E000Eu) | kOneBf16x2, kB64, kBm67_5);
    p[5 * u + 3] = bf16x2_fma((t1 & 0x00700070u) | kOneBf16x2, kB8, kBm11_5);
    p[5 * u + 4] = bf16x2_fma((t2 & 0x000E000Eu) | kOneBf16x2, kB64, kBm67_5);
  }
  const uint32_t s = ((w[0] >> 14) & 0x00020002u) | ((w[1] >> 13) & 0x00040004u) |
                     ((w[2] >> 12) & 0x00080008u) | kOneBf16x2;
  p[15] = bf16x2_fma(s, kB64, kBm67_5);
}

// Ternary: a table entry holds the five trits of one byte as 2-bit codes at bits 1, 3, 5,
// 9, 11 (entry for the low half) or those +16 (high half). OR-ing a low entry and a high
// entry gives five pair registers' worth of fields: slots 1, 3, 5 directly, 9 and 11 after
// a shift by 8.
__device__ __forceinline__ void decode_trit_pairs(uint32_t e, uint32_t p[5]) {
  const uint32_t t1 = e >> 8;
  p[0] = bf16x2_fma((e & 0x00060006u) | kOneBf16x2, kB64, kBm65);
  p[1] = bf16x2_fma((e & 0x00180018u) | kOneBf16x2, kB16, kBm17);
  p[2] = bf16x2_fma((e & 0x00600060u) | kOneBf16x2, kB4, kBm5);
  p[3] = bf16x2_fma((t1 & 0x00060006u) | kOneBf16x2, kB64, kBm65);
  p[4] = bf16x2_fma((t1 & 0x00180018u) | kOneBf16x2, kB16, kBm17);
}

// Position of lane l = 4 r0 + q's chunks inside a 32-chunk row of a packed unit (the swizzle
// of the layout in include/wr.h).
__host__ __device__ __forceinline__ int lane_pos(int r0, int q) { return 4 * r0 + (q ^ ((r0 >> 1) & 3)); }

// ---------------------------------------------------------------- int8 code decoders
//
// The integer tensor-core path keeps weights as their unsigned codes c, one byte each; a 32-bit
// TMEM column holds 4 consecutive K positions of the MMA. Each byte is cut out of the packed
// words by a mask and left where the mask finds it, so byte b of a register holds c * 2^e for a
// position exponent e (the code sits at bits e .. e + bits - 1 of its byte); the activation of
// that position is divided by 2^e instead (see the preparation pass of the decode GEMV). The
// K order inside a register is a fixed permutation of the code order, and the activation tile
// is written in the same order (q2_code_at / q3_code_at, q2_exp_at / q3_exp_at).
//
// Q2 word (codes e = 0..15, code e at bits 16*(e&1) + 2*(e>>1)): register s = w & (3 << 2s in
// every byte) holds codes [2s, 2s+8, 2s+1, 2s+9] in bytes 0..3, each times 4^s. One AND each.
__host__ __device__ __forceinline__ void decode_q2_word_i8(uint32_t w, uint32_t r[4]) {
  r[0] = w & 0x03030303u;
  r[1] = w & 0x0C0C0C0Cu;
  r[2] = w & 0x30303030u;
  r[3] = w & 0xC0C0C0C0u;
}

// Q3 group (3 words, codes 10u + 2j + h at bits 16h + 3j of word u; codes 30 + h have their
// bit j in bit 16h + 15 of word j) -> 8 registers (code, exponent per byte):
//   2u:   [10u,   10u+6, 10u+1, 10u+7]  e = 0,1,0,1   (fields j = 0 and j = 3 of word u)
//   2u+1: [10u+2, 10u+8, 10u+3, 10u+9]  e = 3,4,3,4   (fields j = 1 and j = 4)
//   6:    [4, 14, 5, 15]                e = 5         (field j = 2 of words 0 and 1: it
//   7:    [24, 30, 25, 31]              e = 5          crosses a byte, so it is shifted)
// Six registers are one AND each; the two others gather the byte-crossing fields and the
// spread codes 30 and 31 with a few shifts.
__host__ __device__ __forceinline__ void decode_q3_group_i8(const uint32_t w[3], uint32_t r[8]) {
#pragma unroll
  for (int u = 0; u < 3; ++u) {
    r[2 * u] = w[u] & 0x0E070E07u;
    r[2 * u + 1] = w[u] & 0x70387038u;
  }
  r[6] = ((w[0] >> 1) & 0x00E000E0u) | ((w[1] << 7) & 0xE000E000u);
  r[7] = ((w[2] >> 1) & 0x00E000E0u) | ((w[0] >> 2) & 0x20002000u) | ((w[1] >> 1) & 0x40004000u) |
         (w[2] & 0x80008000u);
}

// 2-bit trellis-coded word (the Q2 word layout holding symbols u, code e at bits
// 16*(e&1) + 2*(e>>1)): the level index of code e is c3 = 2 u_e + p_e, with p_e the low bit of
// the previous symbol (of code e - 1; of the previous word's code 15 for e = 0, given in
// `carry`, which returns this word's code-15 low bit). P holds p_e at each field's low bit:
// odd codes take the low bit of the even code in the same slot, even codes that of the odd
// code one slot down. Register s holds codes [2s, 2s+8, 2s+1, 2s+9] as (2 u + p) * 2^e,
// e = 0, 1, 3, 5 for s = 0..3 (u stays in place; p is masked in one bit below it).
__host__ __device__ __forceinline__ void decode_t2_word_i8(uint32_t w, uint32_t& carry, uint32_t r[4]) {
  const uint32_t P = ((w << 16) & 0x55550000u) | ((w >> 14) & 0x00005554u) | carry;
  carry = (w >> 30) & 1u;
  const uint32_t P1 = P >> 1;
  r[0] = ((w & 0x03030303u) << 1) | (P & 0x01010101u);
  r[1] = (w & 0x0C0C0C0Cu) | (P1 & 0x02020202u);
  r[2] = (w & 0x30303030u) | (P1 & 0x08080808u);
  r[3] = (w & 0xC0C0C0C0u) | (P1 & 0x20202020u);
}

// 8-state trellis word (WR_FMT_T8; the Q2 word layout, code e at bits 16*(e&1) + 2*(e>>1)): its
// 16 codes are symbols j = 0..3 of 4 codes each, and code 4j + i has level index 2 u + p_i with
// (p_0, p_1, p_2, p_3) = (z_(j-1), z_(j-2), z_(j-3), z_(j-1) ^ z_(j-2) ^ z_(j-3)), z_k the low bit of
// symbol k's last code (the state is the last three z). `carry` holds the previous word's z_0..z_3
// at bits 2, 6, 10, 14 (0 at the block start) and returns this word's. With X = (this word's z
// at bits 18 + 4j) | carry, z_k sits at bit 18 + 4k for k = -4..3, and P (each code's parity at
// its field's low bit) is four shifted copies of X; the registers then come out as for T2.
__host__ __device__ __forceinline__ void decode_t8_word_i8(uint32_t w, uint32_t& carry, uint32_t r[4]) {
  const uint32_t zl = (w >> 16) & 0x4444u;
  const uint32_t X = (zl << 16) | carry;
  carry = zl;
  const uint32_t P = ((X >> 14) & 0x1111u) | ((X << 6) & 0x11110000u) | ((X >> 4) & 0x4444u) |
                     (((X << 4) ^ (X << 8) ^ (X << 12)) & 0x44440000u);
  const uint32_t P1 = P >> 1;
  r[0] = ((w & 0x03030303u) << 1) | (P & 0x01010101u);
  r[1] = (w & 0x0C0C0C0Cu) | (P1 & 0x02020202u);
  r[2] = (w & 0x30303030u) | (P1 & 0x08080808u);
  r[3] = (w & 0xC0C0C0C0u) | (P1 & 0x20202020u);
}

// Code index (within a 256-code block) held at logical K position kl of the decoded block, and
// the exponent e of its byte, for the register orders above. Rows of a block are 4 quarters of
// 64 codes; a quarter is 16 registers (Q2: 4 words x 4; Q3: 2 groups x 8).
__host__ __device__ inline int q2_code_at(int kl) {
  const int q = kl >> 6, w = (kl >> 4) & 3, sp = (kl >> 2) & 3, byte = kl & 3;
  const int p = 2 * sp + ((byte & 1) ? 8 : 0) + (byte >> 1);
  return 64 * q + 16 * w + p;
}
__host__ __device__ inline int q2_exp_at(int kl) { return 2 * ((kl >> 2) & 3); }
// The trellis formats use the Q2 K order; their bytes hold (2u + p) * 2^e, e = 0, 1, 3, 5.
__host__ __device__ inline int t2_exp_at(int kl) {
  const int sp = (kl >> 2) & 3;
  return sp == 0 ? 0 : 2 * sp - 1;
}
__host__ __device__ inline int q3_code_at(int kl) {
  const int q = kl >> 6, g = (kl >> 5) & 1, reg = (kl >> 2) & 7, byte = kl & 3;
  int c;
  if (reg < 6) {
    const int u = reg >> 1;
    const int lo[4] = {0, 6, 1, 7}, hi[4] = {2, 8, 3, 9};
    c = 10 * u + ((reg & 1) ? hi[byte] : lo[byte]);
  } else if (reg == 6) {
    const int t[4] = {4, 14, 5, 15};
    c = t[byte];
  } else {
    const int t[4] = {24, 30, 25, 31};
    c = t[byte];
  }
  return 64 * q + 32 * g + c;
}
__host__ __device__ inline int q3_exp_at(int kl) {
  const int reg = (kl >> 2) & 7, byte = kl & 3;
  if (reg >= 6) return 5;
  return ((reg & 1) ? 3 : 0) + (byte & 1);
}

__device__ __forceinline__ float half_bits_to_float(uint16_t h) {
  return __half2float(__ushort_as_half(h));
}

}  // namespace wr
