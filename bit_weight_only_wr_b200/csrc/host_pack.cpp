// Host side of libwr: packed-layout writer/reader and the synthetic quantizers.
//
// The byte layout is specified in include/wr.h. Here it is produced word by word: each
// lane's 16-byte chunks are assembled from the code matrix and stored at
// (32*chunk + lane)*16 inside their unit, and units are placed group by group. The quantizers prepare inputs (codes and fp16
// scales) from fp32 weights; they are not part of the device path.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <vector>

#include "wr.h"
#include "wr_internal.h"

namespace {

constexpr int kTileRows = 16;

inline bool fmt_ok(int fmt) {
  return fmt == WR_FMT_Q2 || fmt == WR_FMT_Q3 || fmt == WR_FMT_TERNARY || fmt == WR_FMT_T2 || fmt == WR_FMT_T8;
}
// 2-bit symbol formats share the Q2 words: Q2 codes and the trellis formats' codes.
inline bool two_bit(int fmt) { return fmt == WR_FMT_Q2 || fmt == WR_FMT_T2 || fmt == WR_FMT_T8; }

struct Geometry {
  int64_t unit_k;      // codes per unit along K
  int64_t unit_bytes;  // bytes per unit
  int64_t tiles;       // ceil(N/16)
  int64_t units;       // units per tile row
};

bool geometry(int fmt, int64_t N, int64_t K, Geometry* g) {
  if (!fmt_ok(fmt) || N <= 0 || K <= 0) return false;
  if (fmt == WR_FMT_TERNARY) {
    g->unit_k = 320;   // any K: the last unit is padded with trit 1 (t = 0)
    g->unit_bytes = 1024;
  } else {
    if (K % 256 != 0) return false;
    g->unit_k = 256;
    g->unit_bytes = fmt == WR_FMT_Q3 ? 1536 : 1024;
  }
  g->tiles = (N + kTileRows - 1) / kTileRows;
  g->units = (K + g->unit_k - 1) / g->unit_k;
  return true;
}

// Index of unit (tile tn, block u): tiles come in groups of 8; a group's units are stored
// block by block and, within a block, tile by tile.
inline int64_t unit_index(const Geometry& g, int64_t tn, int64_t u) {
  const int64_t grp = tn / 8;
  const int64_t tg = std::min<int64_t>(8, g.tiles - 8 * grp);
  return 8 * grp * g.units + u * tg + tn % 8;
}

// Byte offset inside a unit of lane-byte `lb` of lane `lane`: chunk lb / 16 of the lane sits at
// position lane ^ ((lane >> 3) & 3) of its 32-chunk row, so that the 8 lanes r0 = 0..7 of one
// quarter land on 8 different 16-byte bank groups.
inline int64_t unit_offset(int lane, int lb) {
  return (int64_t)(32 * (lb / 16) + (lane ^ ((lane >> 3) & 3))) * 16 + lb % 16;
}

inline void put_word(uint8_t* unit, int lane, int lb, uint32_t w) {
  const int64_t off = unit_offset(lane, lb);   // lb is a multiple of 4: never crosses a chunk
  unit[off + 0] = (uint8_t)(w);
  unit[off + 1] = (uint8_t)(w >> 8);
  unit[off + 2] = (uint8_t)(w >> 16);
  unit[off + 3] = (uint8_t)(w >> 24);
}

inline uint32_t get_word(const uint8_t* unit, int lane, int lb) {
  const int64_t off = unit_offset(lane, lb);
  return (uint32_t)unit[off] | ((uint32_t)unit[off + 1] << 8) | ((uint32_t)unit[off + 2] << 16) |
         ((uint32_t)unit[off + 3] << 24);
}

// Q2: one row quarter = 4 words of 16 codes; code e of a word at bits 16*(e&1) + 2*(e>>1).
uint32_t q2_word(const uint8_t* c16) {
  uint32_t w = 0;
  for (int e = 0; e < 16; ++e) w |= (uint32_t)(c16[e] & 3u) << (16 * (e & 1) + 2 * (e >> 1));
  return w;
}
void q2_unword(uint32_t w, uint8_t* c16) {
  for (int e = 0; e < 16; ++e) c16[e] = (uint8_t)((w >> (16 * (e & 1) + 2 * (e >> 1))) & 3u);
}

// Q3: one 12-byte group = 3 words holding 32 codes. Codes 10u + 2j + h (j = 0..4) of word u
// at bits 16h + 3j; code 30 + h spread over bit 16h + 15 of words 0, 1, 2.
void q3_group(const uint8_t* c32, uint32_t w[3]) {
  for (int u = 0; u < 3; ++u) {
    uint32_t v = 0;
    for (int f = 0; f < 10; ++f) v |= (uint32_t)(c32[10 * u + f] & 7u) << (16 * (f & 1) + 3 * (f >> 1));
    for (int h = 0; h < 2; ++h) v |= (uint32_t)((c32[30 + h] >> u) & 1u) << (16 * h + 15);
    w[u] = v;
  }
}
void q3_ungroup(const uint32_t w[3], uint8_t* c32) {
  for (int u = 0; u < 3; ++u)
    for (int f = 0; f < 10; ++f) c32[10 * u + f] = (uint8_t)((w[u] >> (16 * (f & 1) + 3 * (f >> 1))) & 7u);
  for (int h = 0; h < 2; ++h) {
    uint8_t c = 0;
    for (int u = 0; u < 3; ++u) c |= (uint8_t)(((w[u] >> (16 * h + 15)) & 1u) << u);
    c32[30 + h] = c;
  }
}

// fp16 helpers (host): decode bits exactly; encode a double with one RNE rounding.
double half_to_double(uint16_t h) {
  const int e = (h >> 10) & 31, m = h & 1023;
  double v;
  if (e == 0) v = std::ldexp((double)m, -24);
  else if (e == 31) v = m ? NAN : INFINITY;
  else v = std::ldexp((double)(m + 1024), e - 25);
  return (h & 0x8000) ? -v : v;
}

uint16_t double_to_half(double v) {
  const uint16_t sign = std::signbit(v) ? 0x8000 : 0;
  const double a = std::fabs(v);
  if (std::isnan(v)) return 0x7E00;
  if (a == 0.0) return sign;
  int ex;
  std::frexp(a, &ex);          // a = f * 2^ex, f in [0.5, 1)
  int E = ex - 1;              // a in [2^E, 2^(E+1))
  if (E < -14) E = -14;        // subnormal range shares the 2^-24 step
  const double q = std::ldexp(a, 10 - E);   // a / ulp, exact
  double fl = std::floor(q);
  const double rem = q - fl;
  if (rem > 0.5 || (rem == 0.5 && std::fmod(fl, 2.0) == 1.0)) fl += 1.0;
  int64_t mant = (int64_t)fl;
  if (mant == 2048) { mant = 1024; E += 1; }
  if (mant < 1024) return (uint16_t)(sign | mant);            // subnormal (E == -14)
  if (E + 15 >= 31) return (uint16_t)(sign | 0x7C00);        // overflow to infinity
  return (uint16_t)(sign | ((E + 15) << 10) | (mant - 1024));
}

}  // namespace

namespace wr {
bool packed_geometry(int fmt, int64_t N, int64_t K, int64_t* unit_bytes, int64_t* units, int64_t* tiles) {
  Geometry g;
  if (!geometry(fmt, N, K, &g)) return false;
  if (unit_bytes) *unit_bytes = g.unit_bytes;
  if (units) *units = g.units;
  if (tiles) *tiles = g.tiles;
  return true;
}
uint16_t host_double_to_half(double v) { return double_to_half(v); }
double host_half_to_double(uint16_t h) { return half_to_double(h); }
}  // namespace wr

extern "C" {

size_t wr_packed_bytes(int fmt, int64_t N, int64_t K) {
  Geometry g;
  if (!geometry(fmt, N, K, &g)) return 0;
  return (size_t)(g.tiles * g.units * g.unit_bytes);
}

wr_status wr_pack(int fmt, int64_t N, int64_t K, const uint8_t* codes, uint8_t* packed) {
  Geometry g;
  if (!geometry(fmt, N, K, &g) || !codes || !packed) return WR_ERR_INVALID_ARG;
  const uint8_t cmax = two_bit(fmt) ? 3 : fmt == WR_FMT_Q3 ? 7 : 2;
  bool bad = false;
#pragma omp parallel for reduction(|| : bad)
  for (int64_t i = 0; i < N * K; ++i) bad = bad || codes[i] > cmax;
  if (bad) return WR_ERR_INVALID_ARG;

#pragma omp parallel for collapse(2) schedule(static)
  for (int64_t tn = 0; tn < g.tiles; ++tn) {
    for (int64_t u = 0; u < g.units; ++u) {
      uint8_t* unit = packed + unit_index(g, tn, u) * g.unit_bytes;
      for (int lane = 0; lane < 32; ++lane) {
        const int r0 = lane / 4, q = lane % 4;
        for (int half = 0; half < 2; ++half) {
          const int64_t n = tn * kTileRows + r0 + 8 * half;
          if (fmt == WR_FMT_TERNARY) {
            for (int beta = 0; beta < 16; ++beta) {
              int v = 0, p3 = 1;
              for (int d = 0; d < 5; ++d) {
                const int64_t k = u * 320 + 80 * q + 5 * beta + d;
                const int c = (n < N && k < K) ? codes[n * K + k] : 1;
                v += c * p3;
                p3 *= 3;
              }
              unit[unit_offset(lane, 16 * half + beta)] = (uint8_t)v;
            }
          } else {
            uint8_t c64[64];
            for (int i = 0; i < 64; ++i) c64[i] = n < N ? codes[n * K + u * 256 + 64 * q + i] : 0;
            if (two_bit(fmt)) {
              for (int w = 0; w < 4; ++w) put_word(unit, lane, 16 * half + 4 * w, q2_word(c64 + 16 * w));
            } else {
              for (int grp = 0; grp < 2; ++grp) {
                uint32_t w3[3];
                q3_group(c64 + 32 * grp, w3);
                for (int uu = 0; uu < 3; ++uu) put_word(unit, lane, 24 * half + 12 * grp + 4 * uu, w3[uu]);
              }
            }
          }
        }
      }
    }
  }
  return WR_OK;
}

wr_status wr_unpack_codes(int fmt, int64_t N, int64_t K, const uint8_t* packed, uint8_t* codes) {
  Geometry g;
  if (!geometry(fmt, N, K, &g) || !codes || !packed) return WR_ERR_INVALID_ARG;
#pragma omp parallel for collapse(2) schedule(static)
  for (int64_t tn = 0; tn < g.tiles; ++tn) {
    for (int64_t u = 0; u < g.units; ++u) {
      const uint8_t* unit = packed + unit_index(g, tn, u) * g.unit_bytes;
      for (int lane = 0; lane < 32; ++lane) {
        const int r0 = lane / 4, q = lane % 4;
        for (int half = 0; half < 2; ++half) {
          const int64_t n = tn * kTileRows + r0 + 8 * half;
          if (n >= N) continue;
          if (fmt == WR_FMT_TERNARY) {
            for (int beta = 0; beta < 16; ++beta) {
              int v = unit[unit_offset(lane, 16 * half + beta)];
              for (int d = 0; d < 5; ++d) {
                const int64_t k = u * 320 + 80 * q + 5 * beta + d;
                if (k < K) codes[n * K + k] = (uint8_t)(v % 3);
                v /= 3;
              }
            }
          } else {
            uint8_t c64[64];
            if (two_bit(fmt)) {
              for (int w = 0; w < 4; ++w) q2_unword(get_word(unit, lane, 16 * half + 4 * w), c64 + 16 * w);
            } else {
              for (int grp = 0; grp < 2; ++grp) {
                uint32_t w3[3];
                for (int uu = 0; uu < 3; ++uu) w3[uu] = get_word(unit, lane, 24 * half + 12 * grp + 4 * uu);
                q3_ungroup(w3, c64 + 32 * grp);
              }
            }
            std::memcpy(codes + n * K + u * 256 + 64 * q, c64, 64);
          }
        }
      }
    }
  }
  return WR_OK;
}

size_t wr_scales_bytes(int fmt, int64_t N, int64_t K) {
  const bool s8 = (fmt & WR_SCALES_I8) != 0;
  const int base = fmt & ~WR_SCALES_I8;
  Geometry g;
  if (!geometry(base, N, K, &g)) return 0;
  if (base == WR_FMT_TERNARY) return s8 ? 0 : (size_t)(2 * N);
  const int64_t nb = K / 256;
  return s8 ? (size_t)(wr::s8_q_offset(N) + N * nb) : (size_t)(2 * N * nb);
}

wr_status wr_quantize(int bits, int64_t N, int64_t K, const float* w, uint8_t* codes, uint16_t* scales) {
  const bool s8 = (bits & WR_SCALES_I8) != 0;
  bits &= ~WR_SCALES_I8;
  if (bits != 2 && bits != 3) return WR_ERR_UNSUPPORTED;
  if (N <= 0 || K <= 0 || K % 256 != 0 || !w || !codes || !scales) return WR_ERR_INVALID_ARG;
  const int L = (1 << bits) - 1;
  const int64_t nb = K / 256;
  // int8 scale record: d fp16 [N] at byte 0, q int8 [N, nb] from byte s8_q_offset(N)
  int8_t* qrec = s8 ? reinterpret_cast<int8_t*>(reinterpret_cast<uint8_t*>(scales) + wr::s8_q_offset(N)) : nullptr;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    double d = 0.0;
    if (s8) {
      // d_n = fp16(A_n / (127 L)), saturated to the largest finite fp16
      double A = 0.0;
      for (int64_t k = 0; k < K; ++k) A = std::fmax(A, std::fabs((double)w[n * K + k]));
      uint16_t dh = double_to_half(A / (double)(127 * L));
      if ((dh & 0x7FFFu) >= 0x7C00u) dh = 0x7BFFu;
      scales[n] = dh;
      d = half_to_double(dh);
    }
    for (int64_t b = 0; b < nb; ++b) {
      const float* wb = w + n * K + b * 256;
      double amax = 0.0;
      for (int i = 0; i < 256; ++i) amax = std::fmax(amax, std::fabs((double)wb[i]));
      double s;
      if (s8) {
        // q = nearest integer to amax / (L d) (ties to even under the default rounding mode)
        double qv = d > 0.0 ? std::nearbyint(amax / ((double)L * d)) : 0.0;
        qv = std::min(127.0, std::max(0.0, qv));
        qrec[n * nb + b] = (int8_t)qv;
        s = d * qv;
      } else {
        const uint16_t sh = double_to_half(amax / (double)L);
        scales[n * nb + b] = sh;
        s = half_to_double(sh);
      }
      for (int i = 0; i < 256; ++i) {
        int g = 1;
        if (s > 0.0) {
          const double qv = (double)wb[i] / s;
          double gd = 2.0 * std::floor(qv * 0.5) + 1.0;
          if (gd > L) gd = L;
          if (gd < -L) gd = -L;
          g = (int)gd;
        }
        codes[n * K + b * 256 + i] = (uint8_t)((g + L) / 2);
      }
    }
  }
  return WR_OK;
}

// The 2-bit trellis-coded format: per 256-block, s = fp16(absmax / 7), levels s * {-7..7 odd};
// state s may use level index 2u + s (u in [0, 4)) and the next state is u & 1; the Viterbi
// search (state 0 at the block start) keeps, for each state, the cheapest path ending there.
// Ties go to the lower (state, symbol) pair and, at the end, the lower final state.
wr_status wr_quantize_trellis(int64_t N, int64_t K, const float* w, uint8_t* codes, uint16_t* scales) {
  if (N <= 0 || K <= 0 || K % 256 != 0 || !w || !codes || !scales) return WR_ERR_INVALID_ARG;
  const int64_t nb = K / 256;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    std::vector<uint8_t> bs(256 * 2), bu(256 * 2);
    for (int64_t b = 0; b < nb; ++b) {
      const float* wb = w + n * K + b * 256;
      double amax = 0.0;
      for (int i = 0; i < 256; ++i) amax = std::fmax(amax, std::fabs((double)wb[i]));
      const uint16_t sh = double_to_half(amax / 7.0);
      scales[n * nb + b] = sh;
      const double s = half_to_double(sh);
      double val[8];
      for (int l = 0; l < 8; ++l) val[l] = s * (double)(2 * l - 7);
      const double inf = std::numeric_limits<double>::infinity();
      double cost[2] = {0.0, inf};
      for (int i = 0; i < 256; ++i) {
        const double t = (double)wb[i];
        double nc[2] = {inf, inf};
        uint8_t ns[2] = {0, 0}, nu[2] = {0, 0};
        for (int st = 0; st < 2; ++st) {
          for (int u = 0; u < 4; ++u) {
            const double d = t - val[2 * u + st];
            const double c = cost[st] + d * d;
            const int nx = u & 1;
            if (c < nc[nx]) {
              nc[nx] = c;
              ns[nx] = (uint8_t)st;
              nu[nx] = (uint8_t)u;
            }
          }
        }
        cost[0] = nc[0];
        cost[1] = nc[1];
        bs[2 * i] = ns[0];
        bs[2 * i + 1] = ns[1];
        bu[2 * i] = nu[0];
        bu[2 * i + 1] = nu[1];
      }
      int st = cost[1] < cost[0] ? 1 : 0;
      for (int i = 255; i >= 0; --i) {
        codes[n * K + b * 256 + i] = bu[2 * i + st];
        st = bs[2 * i + st];
      }
    }
  }
  return WR_OK;
}

// The 8-state trellis over 4-weight symbols: per 256-block s = fp16(absmax / 7), levels
// s * {-7..7 odd}; state (s0, s1, s2) selects the parity pattern (s0, s1, s2, s0^s1^s2), code u_i
// of the symbol's weight i gives level index 2 u_i + p_i, and the next state is
// ((s << 1) | (u_3 & 1)) & 7. Viterbi from state 0: for each next state, its two predecessors
// (the lower first), each with its nearest allowed symbol (per weight the nearest level, a tie
// to the lower code; u_3 restricted to the low bit the next state needs); a tie keeps the
// earlier candidate; the path ends in the cheapest state (a tie to the lower). The branch cost
// is summed as cost + e_0 + e_1 + e_2 + e_3, in that order.
wr_status wr_quantize_trellis8(int64_t N, int64_t K, const float* w, uint8_t* codes, uint16_t* scales) {
  if (N <= 0 || K <= 0 || K % 256 != 0 || !w || !codes || !scales) return WR_ERR_INVALID_ARG;
  const int64_t nb = K / 256;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    std::vector<uint8_t> bs(64 * 8), bu(64 * 8 * 4);
    for (int64_t b = 0; b < nb; ++b) {
      const float* wb = w + n * K + b * 256;
      double amax = 0.0;
      for (int i = 0; i < 256; ++i) amax = std::fmax(amax, std::fabs((double)wb[i]));
      const uint16_t sh = double_to_half(amax / 7.0);
      scales[n * nb + b] = sh;
      const double s = half_to_double(sh);
      double val[8];
      for (int l = 0; l < 8; ++l) val[l] = s * (double)(2 * l - 7);
      const double inf = std::numeric_limits<double>::infinity();
      double cost[8];
      for (int st = 0; st < 8; ++st) cost[st] = st == 0 ? 0.0 : inf;
      for (int j = 0; j < 64; ++j) {
        double t[4];
        for (int i = 0; i < 4; ++i) t[i] = (double)wb[4 * j + i];
        double nc[8];
        for (int st = 0; st < 8; ++st) nc[st] = inf;
        for (int nx = 0; nx < 8; ++nx) {
          const int z = nx & 1;
          for (int pass = 0; pass < 2; ++pass) {
            const int st = pass ? ((nx >> 1) | 4) : (nx >> 1);
            const int p[4] = {st & 1, (st >> 1) & 1, (st >> 2) & 1, (st ^ (st >> 1) ^ (st >> 2)) & 1};
            double e[4];
            int u[4];
            for (int i = 0; i < 4; ++i) {
              e[i] = inf;
              u[i] = 0;
              for (int uu = 0; uu < 4; ++uu) {
                if (i == 3 && (uu & 1) != z) continue;
                const double d = t[i] - val[2 * uu + p[i]];
                const double ee = d * d;
                if (ee < e[i]) {
                  e[i] = ee;
                  u[i] = uu;
                }
              }
            }
            const double c = cost[st] + e[0] + e[1] + e[2] + e[3];
            if (c < nc[nx]) {
              nc[nx] = c;
              bs[8 * j + nx] = (uint8_t)st;
              for (int i = 0; i < 4; ++i) bu[32 * j + 4 * nx + i] = (uint8_t)u[i];
            }
          }
        }
        for (int st = 0; st < 8; ++st) cost[st] = nc[st];
      }
      int st = 0;
      for (int k = 1; k < 8; ++k)
        if (cost[k] < cost[st]) st = k;
      for (int j = 63; j >= 0; --j) {
        for (int i = 0; i < 4; ++i) codes[n * K + b * 256 + 4 * j + i] = bu[32 * j + 4 * st + i];
        st = bs[8 * j + st];
      }
    }
  }
  return WR_OK;
}

wr_status wr_quantize_ternary(int64_t N, int64_t K, const float* w, const uint32_t* sign_bits,
                              uint8_t* codes, uint16_t* alpha) {
  if (N <= 0 || K <= 0 || K % 128 != 0 || !w || !sign_bits || !codes || !alpha) return WR_ERR_INVALID_ARG;
  const double inv = 1.0 / std::sqrt(128.0);
#pragma omp parallel
  {
    std::vector<double> row((size_t)K);
#pragma omp for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
      // row n of W R^T is R applied to row n of W: signs, then the butterfly, then 1/sqrt(128)
      for (int64_t k = 0; k < K; ++k) {
        const bool neg = (sign_bits[k >> 5] >> (k & 31)) & 1u;
        row[k] = neg ? -(double)w[n * K + k] : (double)w[n * K + k];
      }
      for (int64_t b0 = 0; b0 < K; b0 += 128) {
        double* v = row.data() + b0;
        for (int h = 1; h < 128; h *= 2)
          for (int i = 0; i < 128; i += 2 * h)
            for (int j = i; j < i + h; ++j) {
              const double a = v[j], c = v[j + h];
              v[j] = a + c;
              v[j + h] = a - c;
            }
        for (int i = 0; i < 128; ++i) v[i] *= inv;
      }
      double sum = 0.0;
      for (int64_t k = 0; k < K; ++k) sum += std::fabs(row[k]);
      const double delta = 0.7 * (sum / (double)K);
      double kept = 0.0;
      int64_t cnt = 0;
      for (int64_t k = 0; k < K; ++k) {
        const double a = std::fabs(row[k]);
        int t = 0;
        if (a > delta) {
          t = row[k] > 0 ? 1 : -1;
          kept += a;
          ++cnt;
        }
        codes[n * K + k] = (uint8_t)(t + 1);
      }
      alpha[n] = double_to_half(cnt > 0 ? kept / (double)cnt : 0.0);
    }
  }
  return WR_OK;
}

}  // extern "C"
