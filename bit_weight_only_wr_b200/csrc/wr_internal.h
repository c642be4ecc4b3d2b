// Internal declarations shared by the translation units of libwr (not part of the ABI).
#pragma once
#include <cstdint>

#include "wr.h"

namespace wr {

bool packed_geometry(int fmt, int64_t N, int64_t K, int64_t* unit_bytes, int64_t* units, int64_t* tiles);
uint16_t host_double_to_half(double v);
double host_half_to_double(uint16_t h);


}  // namespace wr
