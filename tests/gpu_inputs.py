"""Shared set-up of the GPU parity tests: both sides start from the same seeded fp32
weights and bf16 activations (wr_synth); the library quantizes and packs for the CUDA
path, the oracle quantizes for itself, and the two code sets are checked to agree."""
import numpy as np

import wr_synth
from oracle import wr_oracle as o


def torch_mod():
    import torch
    return torch


def dev(a: np.ndarray):
    """numpy array -> CUDA tensor with the same bytes (uint16 bit patterns travel as int16)."""
    torch = torch_mod()
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    elif a.dtype == np.uint32:
        a = a.view(np.int32)
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def q_case(wr, bits, N, K, seed):
    W = wr_synth.weights_fp32(seed, N, K)
    codes, scales = wr.wr_quantize(bits, W)
    codes_o, scales_o = o.quantize_odd_grid(W, bits)
    assert np.array_equal(codes, codes_o) and np.array_equal(scales, scales_o.view(np.uint16))
    packed = wr.wr_pack(bits, codes)
    return codes_o, scales_o, dev(packed), dev(scales)


def t_case(wr, N, K, seed):
    signs = wr_synth.sign_bits(seed + 1, K)
    W = wr_synth.weights_fp32(seed, N, K)
    codes, alpha = wr.wr_quantize_ternary(W, signs)
    codes_o, alpha_o, _ = o.quantize_ternary(W, signs)
    assert np.array_equal(codes, codes_o) and np.array_equal(alpha, alpha_o.view(np.uint16))
    packed = wr.wr_pack(1, codes)
    return codes_o, alpha_o, signs, dev(packed), dev(alpha), dev(signs)


def s8_record(d, q):
    """Int8 scale record of include/wr.h from d (fp16 [N]) and q (int8 [N, B]): d at byte 0,
    q from byte 16 * ceil(2N / 16)."""
    d = np.asarray(d, dtype=np.float16)
    q = np.ascontiguousarray(q, dtype=np.int8)
    N = d.shape[0]
    off = (2 * N + 15) // 16 * 16
    rec = np.zeros(max(off + q.size, 16), dtype=np.uint8)
    rec[:2 * N] = d.view(np.uint8)
    rec[off:off + q.size] = q.reshape(-1).view(np.uint8)
    return rec


def s8_case(wr, bits, N, K, seed, W=None):
    """Codes with int8 block scales: the library's quantizer checked against the oracle's;
    returns (codes, d, q, packed on the device, scale record on the device)."""
    if W is None:
        W = wr_synth.weights_fp32(seed, N, K)
    fmt = bits | wr.WR_SCALES_I8
    codes, rec = wr.wr_quantize(fmt, W)
    codes_o, d_o, q_o = o.quantize_odd_grid_s8(W, bits)
    nrec = wr.wr_scales_bytes(fmt, N, K)
    assert np.array_equal(codes, codes_o) and np.array_equal(rec[:nrec], s8_record(d_o, q_o)[:nrec])
    return codes_o, d_o, q_o, dev(wr.wr_pack(bits, codes)), dev(rec)


def fp32_floor(K: int) -> float:
    """Absolute slack for results below fp32's normal range: one half spacing of fp32's
    subnormals (2^-150) per accumulated term of a K-long sum. It matters only where
    1e-4 * sum_k |w x| is itself below about 2^-130; everywhere else the relative bound rules."""
    return K * 2.0 ** -150


def check_close(y_gpu: np.ndarray, y_ref: np.ndarray, bound: np.ndarray, rel: float = 1e-4,
                floor: float = 0.0):
    """Per element |y_gpu - y_ref| <= rel * sum_k |w x| (+ floor, for subnormal results); exact
    zero where the bound is zero."""
    err = np.abs(y_gpu.astype(np.float64) - y_ref)
    bad = err > rel * bound + floor
    assert not bad.any(), (f"{bad.sum()} of {bad.size} elements out of tolerance; "
                           f"worst err/bound {np.max(err / np.maximum(bound, 1e-300)):.3e}")
    assert np.all(y_gpu[bound == 0] == 0)
