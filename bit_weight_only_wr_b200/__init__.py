"""Python binding of libwr (packed low-bit weight-only GEMV/GEMM for B200).

Argument marshalling only: every function forwards to the C entry point of the same name in
``libwr.so`` (declared in ``include/wr.h``). Device operands are torch CUDA tensors (or raw
device addresses as ints); torch supplies device memory and the current stream, nothing else.
Importing this module fails loudly when the shared library has not been built.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

__all__ = [
    "WR_FMT_TERNARY", "WR_FMT_Q2", "WR_FMT_Q3", "WrError", "LIB_PATH",
    "wr_abi_version", "wr_status_string", "wr_packed_bytes", "wr_pack", "wr_unpack_codes",
    "wr_quantize", "wr_quantize_ternary", "wr_unpack_bf16", "wr_gemv_workspace_bytes", "wr_gemv",
    "wr_gemm_workspace_bytes", "wr_gemm", "wr_gemm_ternary_workspace_bytes", "wr_gemm_ternary",
    "wr_get_device_error", "exported_symbols", "WrGemvProblem", "wr_gemv_batched_workspace_bytes",
    "wr_gemv_batched", "wr_gemv_noalloc", "WR_GEMV_NOALLOC_SCRATCH_BYTES", "WrGemvTernaryProblem",
    "wr_gemv_ternary_batched_workspace_bytes", "wr_gemv_ternary_batched", "wr_selftest_wait_timeout",
    "wr_quantize_pack", "wr_quantize_trellis", "WR_FMT_T2", "WR_FMT_T8", "wr_quantize_trellis8", "WR_SCALES_I8", "wr_scales_bytes",
    "wr_gemv_batched_plan", "WrGemvGroupItem", "wr_gemv_grouped_workspace_bytes", "wr_gemv_grouped",
]

WR_FMT_TERNARY, WR_FMT_Q2, WR_FMT_Q3, WR_FMT_T2, WR_FMT_T8 = 1, 2, 3, 4, 5
WR_SCALES_I8 = 0x100   # OR'd into a format code: int8 block scales (the scale record of include/wr.h)
WR_GEMV_NOALLOC_SCRATCH_BYTES = 4 << 20   # mirrors the macro in include/wr.h
LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libwr.so")

_c_i64, _c_int, _c_size, _vp = ctypes.c_int64, ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p

class WrGemvProblem(ctypes.Structure):
    """Mirror of the C struct wr_gemv_problem."""
    _fields_ = [("x", ctypes.c_void_p), ("packed", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("y", ctypes.c_void_p), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("bits", ctypes.c_int32), ("reserved", ctypes.c_int32)]


_PROBLEMS = ctypes.POINTER(WrGemvProblem)


class WrGemvTernaryProblem(ctypes.Structure):
    """Mirror of the C struct wr_gemv_ternary_problem."""
    _fields_ = [("x", ctypes.c_void_p), ("packed", ctypes.c_void_p), ("alpha", ctypes.c_void_p),
                ("sign_bits", ctypes.c_void_p), ("y", ctypes.c_void_p), ("N", ctypes.c_int64),
                ("K", ctypes.c_int64)]


_TPROBLEMS = ctypes.POINTER(WrGemvTernaryProblem)


class WrGemvGroupItem(ctypes.Structure):
    """Mirror of the C struct wr_gemv_group_item."""
    _fields_ = [("packed", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("y", ctypes.c_void_p),
                ("N", ctypes.c_int64), ("bits", ctypes.c_int32), ("reserved", ctypes.c_int32)]


_GITEMS = ctypes.POINTER(WrGemvGroupItem)

_SIGNATURES = {
    "wr_abi_version": (_c_int, []),
    "wr_status_string": (ctypes.c_char_p, [_c_int]),
    "wr_packed_bytes": (_c_size, [_c_int, _c_i64, _c_i64]),
    "wr_scales_bytes": (_c_size, [_c_int, _c_i64, _c_i64]),
    "wr_pack": (_c_int, [_c_int, _c_i64, _c_i64, _vp, _vp]),
    "wr_unpack_codes": (_c_int, [_c_int, _c_i64, _c_i64, _vp, _vp]),
    "wr_quantize": (_c_int, [_c_int, _c_i64, _c_i64, _vp, _vp, _vp]),
    "wr_quantize_trellis": (_c_int, [_c_i64, _c_i64, _vp, _vp, _vp]),
    "wr_quantize_trellis8": (_c_int, [_c_i64, _c_i64, _vp, _vp, _vp]),
    "wr_quantize_ternary": (_c_int, [_c_i64, _c_i64, _vp, _vp, _vp, _vp]),
    "wr_unpack_bf16": (_c_int, [_c_int, _c_i64, _c_i64, _vp, _vp, _c_int, _vp, _vp]),
    "wr_gemv_workspace_bytes": (_c_size, [_c_i64, _c_i64, _c_i64, _c_int]),
    "wr_gemv": (_c_int, [_c_i64, _c_i64, _c_i64, _vp, _vp, _vp, _c_int, _c_int, _vp, _vp, _c_size, _vp]),
    "wr_gemv_batched_workspace_bytes": (_c_size, [_c_i64, ctypes.c_int32, _PROBLEMS]),
    "wr_gemv_batched": (_c_int, [_c_i64, ctypes.c_int32, _PROBLEMS, _vp, _c_size, _vp]),
    "wr_gemv_batched_plan": (_c_int, [_c_i64, ctypes.c_int32, _PROBLEMS, _vp, _vp, ctypes.c_int32, _vp]),
    "wr_gemm_workspace_bytes": (_c_size, [_c_i64, _c_i64, _c_i64, _c_int]),
    "wr_gemm": (_c_int, [_c_i64, _c_i64, _c_i64, _vp, _vp, _vp, _c_int, _c_int, _vp, _vp, _c_size, _vp]),
    "wr_gemm_ternary_workspace_bytes": (_c_size, [_c_i64, _c_i64, _c_i64]),
    "wr_gemm_ternary": (_c_int, [_c_i64, _c_i64, _c_i64, _vp, _vp, _vp, _vp, _vp, _vp, _c_size, _vp]),
    "wr_get_device_error": (_c_int, [_vp]),
    "wr_gemv_grouped_workspace_bytes": (_c_size, [_c_i64, _c_i64, ctypes.c_int32, _GITEMS]),
    "wr_gemv_grouped": (_c_int, [_c_i64, _c_i64, _vp, ctypes.c_int32, _GITEMS, _vp, _c_size, _vp]),
    "wr_selftest_wait_timeout": (_c_int, [_vp]),
    "wr_quantize_pack": (_c_int, [_c_int, _c_i64, _c_i64, _vp, _vp, _vp, _vp]),
    "wr_gemv_noalloc": (_c_int, [_c_i64, _c_i64, _c_i64, _vp, _vp, _vp, _c_int, _c_int, _vp, _vp]),
    "wr_gemv_ternary_batched_workspace_bytes": (_c_size, [_c_i64, ctypes.c_int32, _TPROBLEMS]),
    "wr_gemv_ternary_batched": (_c_int, [_c_i64, ctypes.c_int32, _TPROBLEMS, _vp, _c_size, _vp]),
}


def exported_symbols():
    """Names of the C entry points this binding expects libwr.so to export."""
    return sorted(_SIGNATURES)


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libwr.so not found at {LIB_PATH}; build it with "
                          "`python bit_weight_only_wr_b200/build.py` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    return lib


_lib = _load()


class WrError(RuntimeError):
    def __init__(self, func: str, status: int):
        super().__init__(f"{func}: {wr_status_string(status)} (status {status})")
        self.status = status


def _check(func: str, st: int) -> None:
    if st != 0:
        raise WrError(func, st)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def wr_abi_version() -> int:
    return _lib.wr_abi_version()


def wr_status_string(st: int) -> str:
    return _lib.wr_status_string(st).decode()


def wr_packed_bytes(fmt: int, N: int, K: int) -> int:
    return _lib.wr_packed_bytes(fmt, N, K)


def wr_scales_bytes(fmt: int, N: int, K: int) -> int:
    return _lib.wr_scales_bytes(fmt, N, K)


def wr_pack(fmt: int, codes: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    N, K = codes.shape
    nb = wr_packed_bytes(fmt, N, K)
    if nb == 0:
        raise WrError("wr_pack", 1)
    out = np.empty(nb, dtype=np.uint8)
    _check("wr_pack", _lib.wr_pack(fmt, N, K, _ptr(codes), _ptr(out)))
    return out


def wr_unpack_codes(fmt: int, packed: np.ndarray, N: int, K: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    if packed.size < wr_packed_bytes(fmt, N, K):
        raise WrError("wr_unpack_codes", 1)
    out = np.empty((N, K), dtype=np.uint8)
    _check("wr_unpack_codes", _lib.wr_unpack_codes(fmt, N, K, _ptr(packed), _ptr(out)))
    return out


def wr_quantize(bits: int, W: np.ndarray):
    """fp32 [N, K] -> (codes uint8 [N, K], fp16 scale bits uint16 [N, K/256]); with
    bits | WR_SCALES_I8 the scales are the int8 scale record (uint8 [wr_scales_bytes])."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    codes = np.empty((N, K), dtype=np.uint8)
    if bits & WR_SCALES_I8:
        scales = np.zeros(max(wr_scales_bytes(bits, N, K), 16), dtype=np.uint8)
    else:
        scales = np.empty((N, max(K // 256, 1)), dtype=np.uint16)
    _check("wr_quantize", _lib.wr_quantize(bits, N, K, _ptr(W), _ptr(codes), _ptr(scales)))
    return codes, scales


def wr_quantize_trellis(W: np.ndarray):
    """fp32 [N, K] -> (symbols uint8 [N, K] of the 2-bit trellis format, fp16 scale bits
    uint16 [N, K/256]); pack the symbols with wr_pack(WR_FMT_T2, ...)."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    codes = np.empty((N, K), dtype=np.uint8)
    scales = np.empty((N, max(K // 256, 1)), dtype=np.uint16)
    _check("wr_quantize_trellis", _lib.wr_quantize_trellis(N, K, _ptr(W), _ptr(codes), _ptr(scales)))
    return codes, scales


def wr_quantize_trellis8(W: np.ndarray):
    """fp32 [N, K] -> (codes uint8 [N, K] of the 8-state trellis format, fp16 scale bits
    uint16 [N, K/256]); pack the codes with wr_pack(WR_FMT_T8, ...)."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    codes = np.empty((N, K), dtype=np.uint8)
    scales = np.empty((N, max(K // 256, 1)), dtype=np.uint16)
    _check("wr_quantize_trellis8", _lib.wr_quantize_trellis8(N, K, _ptr(W), _ptr(codes), _ptr(scales)))
    return codes, scales


def wr_quantize_ternary(W: np.ndarray, sign_bits: np.ndarray):
    """fp32 [N, K] and uint32 sign mask -> (codes uint8 [N, K], fp16 alpha bits uint16 [N])."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    sign_bits = np.ascontiguousarray(sign_bits, dtype=np.uint32)
    N, K = W.shape
    codes = np.empty((N, K), dtype=np.uint8)
    alpha = np.empty(N, dtype=np.uint16)
    _check("wr_quantize_ternary",
           _lib.wr_quantize_ternary(N, K, _ptr(W), _ptr(sign_bits), _ptr(codes), _ptr(alpha)))
    return codes, alpha


def wr_unpack_bf16(fmt: int, N: int, K: int, packed, scales, out, group: int = 256, stream=None) -> None:
    _check("wr_unpack_bf16", _lib.wr_unpack_bf16(fmt, N, K, _ptr(packed), _ptr(scales), group,
                                                 _ptr(out), _stream(stream)))


def wr_gemv_workspace_bytes(M: int, N: int, K: int, bits: int) -> int:
    return _lib.wr_gemv_workspace_bytes(M, N, K, bits)


def wr_gemv(M: int, N: int, K: int, x, packed, scales, bits: int, y, workspace, workspace_bytes: int,
            group: int = 256, stream=None) -> None:
    _check("wr_gemv", _lib.wr_gemv(M, N, K, _ptr(x), _ptr(packed), _ptr(scales), bits, group, _ptr(y),
                                   _ptr(workspace), workspace_bytes, _stream(stream)))


def wr_gemv_noalloc(M: int, N: int, K: int, x, packed, scales, bits: int, y, group: int = 256,
                    stream=None) -> None:
    """wr_gemv without a workspace (fixed scratch inside libwr; see include/wr.h)."""
    _check("wr_gemv_noalloc", _lib.wr_gemv_noalloc(M, N, K, _ptr(x), _ptr(packed), _ptr(scales), bits, group,
                                                   _ptr(y), _stream(stream)))


def _problems(problems):
    """problems: sequence of (x, packed, scales, y, N, K, bits) -> ctypes array."""
    arr = (WrGemvProblem * len(problems))()
    for i, (x, packed, scales, y, N, K, bits) in enumerate(problems):
        arr[i] = WrGemvProblem(_ptr(x), _ptr(packed), _ptr(scales), _ptr(y), N, K, bits, 0)
    return arr


def wr_gemv_batched_workspace_bytes(M: int, problems) -> int:
    arr = problems if isinstance(problems, ctypes.Array) else _problems(problems)
    return _lib.wr_gemv_batched_workspace_bytes(M, len(arr), arr)


def wr_gemv_batched_plan(M: int, problems):
    """(grid, range_starts int64 [grid + 1], block_costs int64 [count]): the CTA block ranges of
    one batched decode launch and the per-problem block cost they were cut by (problems as for
    wr_gemv_batched; only their shapes and formats are read)."""
    arr = problems if isinstance(problems, ctypes.Array) else _problems(problems)
    grid = ctypes.c_int32(0)
    _check("wr_gemv_batched_plan", _lib.wr_gemv_batched_plan(M, len(arr), arr, ctypes.addressof(grid), None, 0, None))
    starts = np.zeros(grid.value + 1, dtype=np.int64)
    costs = np.zeros(len(arr), dtype=np.int64)
    _check("wr_gemv_batched_plan", _lib.wr_gemv_batched_plan(M, len(arr), arr, ctypes.addressof(grid),
                                                             _ptr(starts), grid.value + 1, _ptr(costs)))
    return grid.value, starts, costs


def wr_gemv_batched(M: int, problems, workspace, workspace_bytes: int, stream=None) -> None:
    """problems: sequence of (x, packed, scales, y, N, K, bits), or a prepared ctypes array."""
    arr = problems if isinstance(problems, ctypes.Array) else _problems(problems)
    _check("wr_gemv_batched", _lib.wr_gemv_batched(M, len(arr), arr, _ptr(workspace), workspace_bytes,
                                                   _stream(stream)))


def _gitems(items):
    """items: sequence of (packed, scales, y, N, bits) -> ctypes array."""
    arr = (WrGemvGroupItem * len(items))()
    for i, (packed, scales, y, N, bits) in enumerate(items):
        arr[i] = WrGemvGroupItem(_ptr(packed), _ptr(scales), _ptr(y), N, bits, 0)
    return arr


def wr_gemv_grouped_workspace_bytes(M: int, K: int, items) -> int:
    arr = items if isinstance(items, ctypes.Array) else _gitems(items)
    return _lib.wr_gemv_grouped_workspace_bytes(M, K, len(arr), arr)


def wr_gemv_grouped(M: int, K: int, x, items, workspace, workspace_bytes: int, stream=None) -> None:
    """items: sequence of (packed, scales, y, N, bits), or a prepared ctypes array; all read x."""
    arr = items if isinstance(items, ctypes.Array) else _gitems(items)
    _check("wr_gemv_grouped", _lib.wr_gemv_grouped(M, K, _ptr(x), len(arr), arr, _ptr(workspace),
                                                   workspace_bytes, _stream(stream)))


def _tproblems(problems):
    """problems: sequence of (x, packed, alpha, sign_bits, y, N, K) -> ctypes array."""
    arr = (WrGemvTernaryProblem * len(problems))()
    for i, (x, packed, alpha, signs, y, N, K) in enumerate(problems):
        arr[i] = WrGemvTernaryProblem(_ptr(x), _ptr(packed), _ptr(alpha), _ptr(signs), _ptr(y), N, K)
    return arr


def wr_gemv_ternary_batched_workspace_bytes(M: int, problems) -> int:
    arr = problems if isinstance(problems, ctypes.Array) else _tproblems(problems)
    return _lib.wr_gemv_ternary_batched_workspace_bytes(M, len(arr), arr)


def wr_gemv_ternary_batched(M: int, problems, workspace, workspace_bytes: int, stream=None) -> None:
    """problems: sequence of (x, packed, alpha, sign_bits, y, N, K), or a prepared ctypes array."""
    arr = problems if isinstance(problems, ctypes.Array) else _tproblems(problems)
    _check("wr_gemv_ternary_batched", _lib.wr_gemv_ternary_batched(M, len(arr), arr, _ptr(workspace),
                                                                   workspace_bytes, _stream(stream)))


def wr_gemm_workspace_bytes(M: int, N: int, K: int, bits: int) -> int:
    return _lib.wr_gemm_workspace_bytes(M, N, K, bits)


def wr_gemm(M: int, N: int, K: int, x, packed, scales, bits: int, y, workspace, workspace_bytes: int,
            group: int = 256, stream=None) -> None:
    _check("wr_gemm", _lib.wr_gemm(M, N, K, _ptr(x), _ptr(packed), _ptr(scales), bits, group, _ptr(y),
                                   _ptr(workspace), workspace_bytes, _stream(stream)))


def wr_gemm_ternary_workspace_bytes(M: int, N: int, K: int) -> int:
    return _lib.wr_gemm_ternary_workspace_bytes(M, N, K)


def wr_gemm_ternary(M: int, N: int, K: int, x, packed, alpha, sign_bits, y, workspace,
                    workspace_bytes: int, stream=None) -> None:
    _check("wr_gemm_ternary", _lib.wr_gemm_ternary(M, N, K, _ptr(x), _ptr(packed), _ptr(alpha),
                                                   _ptr(sign_bits), _ptr(y), _ptr(workspace),
                                                   workspace_bytes, _stream(stream)))


def wr_get_device_error(stream=None) -> int:
    return _lib.wr_get_device_error(_stream(stream))


def wr_quantize_pack(bits: int, N: int, K: int, w, packed, scales, stream=None) -> None:
    """Device quantizer + packer: fp32 W [N, K] (device) -> packed codes and fp16 block scales
    (device), bit-identical with wr_quantize + wr_pack; with bits | WR_SCALES_I8, `scales` is
    the int8 scale record (wr_scales_bytes bytes)."""
    _check("wr_quantize_pack", _lib.wr_quantize_pack(bits, N, K, _ptr(w), _ptr(packed), _ptr(scales),
                                                     _stream(stream)))


def wr_selftest_wait_timeout(stream=None) -> None:
    """Launch the failure-path self-test (a bounded wait that runs out after one second)."""
    _check("wr_selftest_wait_timeout", _lib.wr_selftest_wait_timeout(_stream(stream)))
