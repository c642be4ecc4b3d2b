// C ABI of libwr: argument checks, workspace layout and launch configuration.
//
// Every entry point validates its arguments on the host and returns before any launch when
// they are wrong; device work is enqueued on the caller's stream and never synchronized.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <mutex>

#include "gemm.cuh"
#include "gemv.cuh"
#include "wr.h"
#include "wr_internal.h"

namespace {

constexpr int64_t kMaxDim = (int64_t)1 << 30;

__device__ int g_device_error = 0;

inline bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

int sm_count() {
  static std::mutex mu;
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    cache[dev] = v;
  }
  return cache[dev];
}

// Workspace of the decode GEMV: [counters: one int per 16-row tile][partials: 2 per warp,
// 16 x 8 fp32 each][ternary only: R x as two bf16 planes of M x Kp].
struct GemvWorkspace {
  size_t counter_off, partial_off, xr_off, total;
};

GemvWorkspace gemv_workspace(int fmt, int64_t M, int64_t N, int64_t K) {
  int64_t unit_bytes = 0, units = 0, tiles = 0;
  wr::packed_geometry(fmt, N, K, &unit_bytes, &units, &tiles);
  const int64_t U = tiles * units;
  const int64_t wt = std::min<int64_t>(U, wr::kGemvMaxWarps);
  GemvWorkspace w;
  w.counter_off = 0;
  w.partial_off = align256((size_t)tiles * sizeof(int));
  w.xr_off = w.partial_off + align256((size_t)(2 * wt) * 128 * sizeof(float));
  w.total = w.xr_off;
  if (fmt == WR_FMT_TERNARY) w.total += align256((size_t)(2 * M) * (size_t)(units * 320) * 2);
  return w;
}

wr_status check_dims(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || N < 1 || K < 1 || M > kMaxDim || N > kMaxDim || K > kMaxDim) return WR_ERR_INVALID_ARG;
  if ((double)N * (double)K > 9.0e15) return WR_ERR_INVALID_ARG;
  return WR_OK;
}

// Launch the GEMV on tokens [0, M) (M <= 8) of already validated operands.
wr_status run_gemv(int fmt, int M, int N, int K, const uint16_t* x, const uint8_t* packed,
                   const uint16_t* scales, const uint16_t* alpha, const uint32_t* signs, float* y,
                   void* workspace, cudaStream_t stream) {
  int64_t unit_bytes = 0, units = 0, tiles = 0;
  wr::packed_geometry(fmt, N, K, &unit_bytes, &units, &tiles);
  const GemvWorkspace ws = gemv_workspace(fmt, M, N, K);
  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  wr::GemvArgs a{};
  a.x = x;
  a.packed = packed;
  a.scales = scales;
  a.row_scale = alpha;
  a.y = y;
  a.counter = reinterpret_cast<int*>(wsb + ws.counter_off);
  a.partial = reinterpret_cast<float*>(wsb + ws.partial_off);
  a.M = M;
  a.N = N;
  a.K = K;
  a.B = (int)units;
  a.U = tiles * units;
  const int64_t wt_cap = std::min<int64_t>((int64_t)sm_count() * wr::kGemvWarpsPerSM, wr::kGemvMaxWarps);
  a.Wt = (int)std::min<int64_t>(a.U, wt_cap);
  if (fmt == WR_FMT_TERNARY) {
    uint16_t* xr = reinterpret_cast<uint16_t*>(wsb + ws.xr_off);
    a.xr = xr;
    if (wr::launch_rotate_x(x, signs, xr, M, K, units * 320, stream) != cudaSuccess) return WR_ERR_CUDA;
  }
  const int wpc = wr::gemv_warps_per_cta();
  const int ctas = (a.Wt + wpc - 1) / wpc;
  if (wr::launch_gemv(fmt, a, ctas, stream) != cudaSuccess) return WR_ERR_CUDA;
  return WR_OK;
}

}  // namespace

extern "C" {

int wr_abi_version(void) { return 1; }

const char* wr_status_string(wr_status st) {
  switch (st) {
    case WR_OK: return "ok";
    case WR_ERR_INVALID_ARG: return "invalid argument";
    case WR_ERR_UNSUPPORTED: return "unsupported configuration";
    case WR_ERR_CUDA: return "CUDA error";
    case WR_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

wr_status wr_unpack_bf16(int fmt, int64_t N, int64_t K, const void* packed, const uint16_t* scales,
                         int group, uint16_t* w_bf16, void* stream) {
  if (fmt != WR_FMT_Q2 && fmt != WR_FMT_Q3 && fmt != WR_FMT_TERNARY) return WR_ERR_UNSUPPORTED;
  if (check_dims(1, N, K) != WR_OK) return WR_ERR_INVALID_ARG;
  if (fmt != WR_FMT_TERNARY && group != 256) return WR_ERR_UNSUPPORTED;
  int64_t ub = 0, units = 0, tiles = 0;
  if (!wr::packed_geometry(fmt, N, K, &ub, &units, &tiles)) return WR_ERR_INVALID_ARG;
  if (!aligned16(packed) || !aligned16(scales) || !aligned16(w_bf16)) return WR_ERR_INVALID_ARG;
  const cudaError_t e = wr::launch_unpack_bf16(fmt, static_cast<const uint8_t*>(packed), scales, (int)N,
                                               (int)K, (int)units, w_bf16, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? WR_OK : WR_ERR_CUDA;
}

size_t wr_gemv_workspace_bytes(int64_t M, int64_t N, int64_t K, int bits) {
  if (bits != 2 && bits != 3) return 0;
  if (M < 1 || M > 8 || check_dims(M, N, K) != WR_OK || K % 256 != 0) return 0;
  return gemv_workspace(bits, M, N, K).total;
}

wr_status wr_gemv(int64_t M, int64_t N, int64_t K, const uint16_t* x, const void* packed,
                  const uint16_t* scales, int bits, int group, float* y, void* workspace,
                  size_t workspace_bytes, void* stream) {
  if (bits != 2 && bits != 3) return WR_ERR_UNSUPPORTED;
  if (group != 256) return WR_ERR_UNSUPPORTED;
  if (M < 1 || M > 8 || check_dims(M, N, K) != WR_OK || K % 256 != 0) return WR_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(packed) || !aligned16(scales) || !aligned16(y) || !aligned16(workspace))
    return WR_ERR_INVALID_ARG;
  if (workspace_bytes < gemv_workspace(bits, M, N, K).total) return WR_ERR_INVALID_ARG;
  return run_gemv(bits, (int)M, (int)N, (int)K, x, static_cast<const uint8_t*>(packed), scales, nullptr,
                  nullptr, y, workspace, static_cast<cudaStream_t>(stream));
}

size_t wr_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int bits) {
  if (bits != 2 && bits != 3) return 0;
  if (check_dims(M, N, K) != WR_OK || K % 256 != 0) return 0;
  return std::max(wr::gemm_workspace_bytes(M, N, K, bits), gemv_workspace(bits, 8, N, K).total);
}

wr_status wr_gemm(int64_t M, int64_t N, int64_t K, const uint16_t* x, const void* packed,
                  const uint16_t* scales, int bits, int group, float* y, void* workspace,
                  size_t workspace_bytes, void* stream) {
  if (bits != 2 && bits != 3) return WR_ERR_UNSUPPORTED;
  if (group != 256) return WR_ERR_UNSUPPORTED;
  if (check_dims(M, N, K) != WR_OK || K % 256 != 0) return WR_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(packed) || !aligned16(scales) || !aligned16(y) || !aligned16(workspace))
    return WR_ERR_INVALID_ARG;
  if (workspace_bytes < wr_gemm_workspace_bytes(M, N, K, bits)) return WR_ERR_INVALID_ARG;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (M <= 8)
    return run_gemv(bits, (int)M, (int)N, (int)K, x, static_cast<const uint8_t*>(packed), scales, nullptr,
                    nullptr, y, workspace, s);
  const cudaError_t e = wr::launch_gemm(bits, (int)M, (int)N, (int)K, x, static_cast<const uint8_t*>(packed),
                                        scales, y, workspace, s);
  if (e == cudaErrorNotSupported) {
    // interim path until the tensor-memory kernel covers this shape: 8-token GEMV slices
    for (int64_t m0 = 0; m0 < M; m0 += 8) {
      const int mm = (int)std::min<int64_t>(8, M - m0);
      const wr_status st = run_gemv(bits, mm, (int)N, (int)K, x + m0 * K, static_cast<const uint8_t*>(packed),
                                    scales, nullptr, nullptr, y + m0 * N, workspace, s);
      if (st != WR_OK) return st;
    }
    return WR_OK;
  }
  return e == cudaSuccess ? WR_OK : WR_ERR_CUDA;
}

size_t wr_gemm_ternary_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (check_dims(M, N, K) != WR_OK || K % 128 != 0) return 0;
  return std::max(gemv_workspace(WR_FMT_TERNARY, std::min<int64_t>(M, 8), N, K).total,
                  wr::gemm_ternary_workspace_bytes(M, N, K));
}

wr_status wr_gemm_ternary(int64_t M, int64_t N, int64_t K, const uint16_t* x, const void* packed,
                          const uint16_t* alpha, const uint32_t* sign_bits, float* y, void* workspace,
                          size_t workspace_bytes, void* stream) {
  if (check_dims(M, N, K) != WR_OK || K % 128 != 0) return WR_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(packed) || !aligned16(alpha) || !aligned16(sign_bits) || !aligned16(y) ||
      !aligned16(workspace))
    return WR_ERR_INVALID_ARG;
  if (workspace_bytes < wr_gemm_ternary_workspace_bytes(M, N, K)) return WR_ERR_INVALID_ARG;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (M <= 8)
    return run_gemv(WR_FMT_TERNARY, (int)M, (int)N, (int)K, x, static_cast<const uint8_t*>(packed), nullptr,
                    alpha, sign_bits, y, workspace, s);
  const cudaError_t e = wr::launch_gemm_ternary((int)M, (int)N, (int)K, x, static_cast<const uint8_t*>(packed),
                                                alpha, sign_bits, y, workspace, s);
  if (e == cudaErrorNotSupported) {
    for (int64_t m0 = 0; m0 < M; m0 += 8) {
      const int mm = (int)std::min<int64_t>(8, M - m0);
      const wr_status st = run_gemv(WR_FMT_TERNARY, mm, (int)N, (int)K, x + m0 * K,
                                    static_cast<const uint8_t*>(packed), nullptr, alpha, sign_bits, y + m0 * N,
                                    workspace, s);
      if (st != WR_OK) return st;
    }
    return WR_OK;
  }
  return e == cudaSuccess ? WR_OK : WR_ERR_CUDA;
}

wr_status wr_get_device_error(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return WR_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)) != cudaSuccess) return WR_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) return WR_ERR_CUDA;
    return WR_ERR_TIMEOUT;
  }
  return WR_OK;
}

}  // extern "C"
