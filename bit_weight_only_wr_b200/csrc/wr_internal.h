// Internal declarations shared by the translation units of libwr (not part of the ABI).
#pragma once
#include <cstdint>

#include "wr.h"

namespace wr {

bool packed_geometry(int fmt, int64_t N, int64_t K, int64_t* unit_bytes, int64_t* units, int64_t* tiles);
uint16_t host_double_to_half(double v);
double host_half_to_double(uint16_t h);
// Byte offset of the int8 multipliers in an int8 scale record (after the fp16 row scales).
inline int64_t s8_q_offset(int64_t N) { return (2 * N + 15) / 16 * 16; }


}  // namespace wr
