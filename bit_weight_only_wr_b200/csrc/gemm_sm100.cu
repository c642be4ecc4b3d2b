// Prefill GEMM on tcgen05 (sm_100a): placeholder until the tensor-memory kernel lands.
#include "gemm.cuh"

namespace wr {

size_t gemm_workspace_bytes(int64_t, int64_t, int64_t, int) { return 0; }
cudaError_t launch_gemm(int, int, int, int, const uint16_t*, const uint8_t*, const uint16_t*, float*, void*,
                        cudaStream_t) {
  return cudaErrorNotSupported;
}
size_t gemm_ternary_workspace_bytes(int64_t, int64_t, int64_t) { return 0; }
cudaError_t launch_gemm_ternary(int, int, int, const uint16_t*, const uint8_t*, const uint16_t*,
                                const uint32_t*, float*, void*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace wr
