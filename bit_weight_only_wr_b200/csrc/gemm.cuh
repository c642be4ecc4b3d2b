// Launch interface of the prefill GEMM kernels (internal to libwr).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace wr {

size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int bits);
cudaError_t launch_gemm(int bits, int M, int N, int K, const uint16_t* x, const uint8_t* packed,
                        const uint16_t* scales, float* y, void* workspace, cudaStream_t stream);

size_t gemm_ternary_workspace_bytes(int64_t M, int64_t N, int64_t K);
cudaError_t launch_gemm_ternary(int M, int N, int K, const uint16_t* x, const uint8_t* packed,
                                const uint16_t* alpha, const uint32_t* signs, float* y, void* workspace,
                                cudaStream_t stream);

}  // namespace wr
