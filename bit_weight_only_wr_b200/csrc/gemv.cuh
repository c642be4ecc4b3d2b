// Launch interface of the decode GEMV kernels (internal to libwr).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace wr {

struct GemvArgs {
  const uint16_t* x;          // bf16 [M, K] (Q2/Q3)
  const uint16_t* xr;         // ternary: R x as [2][M][Kp] bf16 planes (hi, lo), fragment order
  const uint8_t* packed;      // packed units
  const uint16_t* scales;     // fp16 [N, K/256] (Q2/Q3)
  const uint16_t* row_scale;  // fp16 [N] applied when y is written (ternary alpha), or null
  float* y;                   // fp32 [M, N]
  float* partial;             // [2 * Wt][16 * 8] fp32 partial tiles
  int* counter;               // [ceil(N/16)] arrival counters, zero between calls
  int M, N, K;
  int B;                      // units per tile row
  int64_t U;                  // units in total (tiles * B)
  int Wt;                     // warps of the grid that own units (Wt <= U)
};

cudaError_t launch_gemv(int fmt, const GemvArgs& a, int ctas, cudaStream_t stream);
cudaError_t launch_rotate_x(const uint16_t* x, const uint32_t* signs, uint16_t* xr, int M, int K,
                            int64_t Kp, cudaStream_t stream);
int gemv_warps_per_cta();

cudaError_t launch_unpack_bf16(int fmt, const uint8_t* packed, const uint16_t* scales, int N, int K,
                               int units, uint16_t* w, cudaStream_t stream);

}  // namespace wr
