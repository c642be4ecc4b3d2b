"""Pins for the oracle: facts fixed by the pages or by mathematics, checked without a GPU.

Each test ties one part of ``oracle.wr_oracle`` to something other than itself: a worked
example printed on the pages, a closed form, an invariant, a brute-force computation on a
tiny input, or an independent library routine.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import wr_oracle as o
import wr_synth


# ---------------------------------------------------------------- pages' worked examples

def test_hadamard_4x4_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "hadamard_4x4.json")))
    H = o.hadamard(4)
    assert np.array_equal(H, np.array(g["matrix_times_2"], dtype=np.float64))
    v = np.array(g["input"])
    out = (H / 2.0) @ v
    assert np.allclose(out, g["output"], atol=1e-12)
    assert math.isclose(float(v @ v), g["sum_of_squares"], rel_tol=1e-12)
    assert math.isclose(float(out @ out), g["sum_of_squares"], rel_tol=1e-12)
    small = np.abs(v[1:])
    assert g["max_ratio_before_min"] <= 3.0 / small.max() + 1e-9
    assert 3.0 / small.min() <= g["max_ratio_before_max"] + 1e-9
    # after the rotation the largest value is close to the others
    assert out.max() / out.min() < 1.3


def test_grid_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "grid_example.json")))
    W = np.zeros((1, 256), dtype=np.float32)
    W[0, :4] = g["group"]
    codes, s = o.quantize_odd_grid(W, 2)
    assert float(s[0, 0]) == 1.0
    levels = o.code_to_level(codes[0, :4], 2)
    assert list(levels) == g["expected_levels"]
    assert set(o.code_to_level(np.arange(4), 2)) == set(g["levels"])
    # the small values are off by about 1 each, larger than the values themselves
    err = np.abs(levels[1:] * 1.0 - np.array(g["group"][1:]))
    assert np.all(err > np.abs(g["group"][1:]))


def test_ledger(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "ledger.json")))
    mods = wr_synth.QWEN3_4B_LAYER
    assert len(mods) * wr_synth.QWEN3_4B_LAYERS == g["modules"]
    weights = sum(K * N for _, K, N, _ in mods)
    assert round(weights * wr_synth.QWEN3_4B_LAYERS / 1e9, 2) == g["body_weights_billions"]
    code_bits = sum(K * N * b for _, K, N, b in mods) / weights
    assert abs(code_bits - g["code_bits_per_weight"]) < 1e-3      # 2.5195 vs the printed 2.520
    # packed sizes of the layout match the code ledger exactly (N multiple of 16)
    packed = sum(o.packed_bytes(b, N, K) for _, K, N, b in mods)
    assert packed * 8 == sum(K * N * b for _, K, N, b in mods)


def test_ternary_bits_per_weight():
    # 5 trits per byte: 1.6 bits per weight when K is a multiple of 320 (K = 2560)
    assert o.packed_bytes(o.FMT_TERNARY, 16, 2560) * 8 / (16 * 2560) == pytest.approx(1.6)
    # K = 4096 pads to 4160 trits: 1.625 bits per weight
    assert o.packed_bytes(o.FMT_TERNARY, 16, 4096) * 8 / (16 * 4096) == pytest.approx(1.625)


# ---------------------------------------------------------------- Hadamard and rotation

def _fwht_python(v):
    """Textbook in-place butterfly, pure Python, unnormalized."""
    v = list(v)
    h = 1
    while h < len(v):
        for i in range(0, len(v), 2 * h):
            for j in range(i, i + h):
                a, b = v[j], v[j + h]
                v[j], v[j + h] = a + b, a - b
        h *= 2
    return v


@pytest.mark.parametrize("n", [2, 4, 8, 16, 32, 64, 128])
def test_hadamard_orthogonal(n):
    H = o.hadamard(n)
    assert np.array_equal(H @ H.T, n * np.eye(n))


def test_rotation_is_orthogonal_and_matches_butterfly():
    K = 384
    signs = wr_synth.sign_bits(7, K)
    R = o.rotate(np.eye(K), signs).T          # column k = R e_k
    assert np.allclose(R.T @ R, np.eye(K), atol=1e-13)
    d = [(-1.0 if (int(signs[k // 32]) >> (k % 32)) & 1 else 1.0) for k in range(K)]
    rng = np.random.default_rng(3)
    v = rng.standard_normal(K)
    ref = []
    for b in range(K // 128):
        blk = [v[k] * d[k] for k in range(128 * b, 128 * b + 128)]
        ref += [t / math.sqrt(128) for t in _fwht_python(blk)]
    assert np.allclose(o.rotate(v, signs), ref, atol=1e-13)


def test_rotation_preserves_products():
    # W x = (W R^T)(R x): the stored weights are rotated, the input is rotated in-kernel
    K, N, M = 512, 24, 3
    signs = wr_synth.sign_bits(11, K)
    W = wr_synth.weights_fp32(5, N, K).astype(np.float64)
    x = wr_synth.bf16_bits_to_f32(wr_synth.activations_bf16(6, M, K)).astype(np.float64)
    y = x @ W.T
    yr = o.rotate(x, signs) @ o.rotate(W, signs).T
    assert np.allclose(y, yr, rtol=1e-12, atol=1e-13)


def test_sign_vector_bits():
    w = np.array([0b1011, 0x80000000], dtype=np.uint32)
    d = o.sign_vector(w, 64)
    assert list(d[:5]) == [-1, -1, 1, -1, 1]
    assert d[63] == -1 and d[62] == 1


# ---------------------------------------------------------------- scalar conversions

def _fp16_exact_rne(x: Fraction) -> Fraction:
    """Round a positive rational to fp16 by exact arithmetic (normal and subnormal)."""
    if x == 0:
        return Fraction(0)
    e = math.floor(math.log2(x))
    while Fraction(2) ** e > x:
        e -= 1
    while Fraction(2) ** (e + 1) <= x:
        e += 1
    e = max(e, -14)
    ulp = Fraction(2) ** (e - 10)
    q = x / ulp
    fl = math.floor(q)
    rem = q - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return fl * ulp


def test_fp16_round_matches_exact_rounding():
    rng = np.random.default_rng(0)
    vals = list(rng.uniform(1e-6, 1.0, 200)) + [1 + 2 ** -11, 1 + 2 ** -11 + 2 ** -40,
                                                 3 * 2 ** -20, 0.0612 / 3, 0.02 / 7]
    for v in vals:
        exact = _fp16_exact_rne(Fraction(v))
        assert Fraction(float(o.fp16_round(np.float64(v)))) == exact, v


def test_bf16_conversions_match_torch():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(1)
    s = rng.uniform(1e-3, 0.1, 4096).astype(np.float16).astype(np.float64)
    g = rng.integers(-3, 4, 4096) * 2 + 1
    w = s * g
    mine = o.f64_to_bf16_bits(w)
    ref = torch.from_numpy(w).to(torch.float32).to(torch.bfloat16).view(torch.int16).numpy()
    assert np.array_equal(mine, ref.view(np.uint16))
    back = o.bf16_bits_to_f64(mine)
    ref_back = torch.from_numpy(ref).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(back, ref_back)


# ---------------------------------------------------------------- quantizer

@pytest.mark.parametrize("bits", [2, 3])
def test_nearest_point_against_brute_force(bits):
    L = o.grid_L(bits)
    W = wr_synth.weights_fp32(21 + bits, 8, 512)
    codes, s = o.quantize_odd_grid(W, bits)
    levels = np.arange(-L, L + 1, 2)
    for n in range(8):
        for k in range(0, 512, 7):
            sc = float(s[n, k // 256])
            absmax = float(np.abs(W[n, (k // 256) * 256:(k // 256 + 1) * 256]).max())
            assert Fraction(sc) == _fp16_exact_rne(Fraction(absmax) / L)
            q = float(W[n, k]) / sc
            dist = np.abs(levels - q)
            best = levels[dist == dist.min()].max()    # ties go to the larger level
            assert o.code_to_level(codes[n, k], bits) == best


def test_quantizer_special_blocks():
    W = np.zeros((2, 512), dtype=np.float32)
    W[1, 256:] = -0.5
    W[1, 300] = 0.25
    codes, s = o.quantize_odd_grid(W, 2)
    assert float(s[0, 0]) == 0.0 and np.all(o.code_to_level(codes[0], 2) == 1)
    # block of constant -0.5: s = 0.5/3 rounded to fp16, all codes at -3
    assert float(s[1, 1]) == float(np.float16(0.5 / 3))
    assert o.code_to_level(codes[1, 257], 2) == -3
    assert o.code_to_level(codes[1, 300], 2) == 1     # 0.25/s = 1.5 -> nearest odd is 1


# ---------------------------------------------------------------- two-level int8 block scales

def _nearest_int_ties_even(x: Fraction, lo: int, hi: int) -> int:
    """Brute force over the integers lo..hi: the nearest to x, ties to the even one."""
    best = None
    for j in range(lo, hi + 1):
        dist = abs(Fraction(j) - x)
        if best is None or dist < best[0] or (dist == best[0] and j % 2 == 0):
            best = (dist, j)
    return best[1]


@pytest.mark.parametrize("bits", [2, 3])
def test_s8_scales_against_exact_arithmetic(bits):
    L = o.grid_L(bits)
    W = wr_synth.weights_fp32(31 + bits, 6, 1024)
    W[2] *= np.linspace(0.05, 1.0, 1024, dtype=np.float32)   # blocks of very different absmax
    codes, d, q = o.quantize_odd_grid_s8(W, bits)
    assert d.dtype == np.float16 and q.dtype == np.int8 and q.shape == (6, 4)
    levels = np.arange(-L, L + 1, 2)
    for n in range(6):
        A = max(Fraction(float(v)) for v in np.abs(W[n]))
        assert Fraction(float(d[n])) == _fp16_exact_rne(A / (127 * L))
        dn = Fraction(float(d[n]))
        for b in range(4):
            a = max(Fraction(float(v)) for v in np.abs(W[n, 256 * b:256 * (b + 1)]))
            assert int(q[n, b]) == _nearest_int_ties_even(a / (L * dn), 0, 127)
        # the block that holds the row maximum gets the full multiplier
        assert q[n].max() == 127
        s = o.s8_block_scales(d, q)
        for k in range(0, 1024, 11):
            r = float(W[n, k]) / float(s[n, k // 256])
            dist = np.abs(levels - r)
            assert o.code_to_level(codes[n, k], bits) == levels[dist == dist.min()].max()


def test_s8_closed_form_row():
    # Q2 (L = 3). Block 0's absmax 127*3*2^-8 makes d = 2^-8 exactly; blocks 1 and 2 have
    # absmax 3*2^-8 times 10.5 and 11.5, exact ties that go to the even multipliers 10 and 12;
    # block 3's absmax is 0.4 * 3 * 2^-8, whose multiplier rounds to 0 (s = 0, all codes +1).
    u = 2.0 ** -8
    W = np.zeros((3, 1024), dtype=np.float32)
    W[0, 0] = 127 * 3 * u
    W[0, 256] = 3 * u * 10.5
    W[0, 257] = -0.05
    W[0, 512] = -3 * u * 11.5
    W[0, 768] = 0.4 * 3 * u
    W[2, 5] = 1.0e9                      # d saturates at the largest finite fp16
    codes, d, q = o.quantize_odd_grid_s8(W, 2)
    assert float(d[0]) == u
    assert q[0].tolist() == [127, 10, 12, 0]
    g = o.code_to_level(codes[0], 2)
    assert g[0] == 3 and g[256] == 3     # 0.123046875 / (10 u) = 3.15 -> level 3
    assert g[257] == -1                  # -0.05 / (10 u) = -1.28 -> level -1
    assert g[512] == -3 and np.all(g[768:] == 1)
    # all-zero row: d = 0, q = 0, every code at level +1
    assert float(d[1]) == 0.0 and np.all(q[1] == 0) and np.all(o.code_to_level(codes[1], 2) == 1)
    assert float(d[2]) == 65504.0 and q[2, 0] == 127 and o.code_to_level(codes[2, 5], 2) == 3
    assert q[2, 1] == 0


def test_s8_dequant_hand_examples():
    codes = np.zeros((2, 512), dtype=np.uint8)
    codes[0, :2] = [0, 3]
    codes[1, 256:258] = [7, 2]
    d = np.array([0.5, 2.0 ** -10], dtype=np.float16)
    q = np.array([[3, 1], [0, 100]], dtype=np.int8)
    W2 = o.dequant_s8(codes, d, q, 2)
    assert W2[0, 0] == -4.5 and W2[0, 1] == 4.5 and W2[0, 256] == -1.5 and np.all(W2[1, :256] == 0)
    W3 = o.dequant_s8(codes, d, q, 3)
    assert W3[1, 256] == 7 * 100 * 2.0 ** -10 and W3[1, 257] == -3 * 100 * 2.0 ** -10
    # bf16 of 700 * 2^-10 = 0.68359375 is exact (8 significant bits)
    bits = o.unpack_bf16_s8(codes, d, q, 3)
    assert o.bf16_bits_to_f64(bits[1, 256]) == 0.68359375
    # trellis symbols with two-level scales match the fp16-scale definition when d q is the scale
    sym = np.random.default_rng(5).integers(0, 4, size=(2, 512)).astype(np.uint8)
    dd = np.array([1.0, 0.25], dtype=np.float16)
    qq = np.array([[5, 7], [9, 127]], dtype=np.int8)
    ref = o.dequant_trellis2(sym, o.s8_block_scales(dd, qq))
    assert np.array_equal(o.dequant_trellis2_s8(sym, dd, qq), ref)


def test_dequant_hand_examples():
    codes = np.array([[0, 3] + [1] * 254, [7, 4] + [0] * 254], dtype=np.uint8)
    s2 = np.array([[0.5]], dtype=np.float16)
    W = o.dequant(codes[:1, :256] & 3, s2, 2)
    assert W[0, 0] == -1.5 and W[0, 1] == 1.5 and W[0, 2] == -0.5
    s3 = np.array([[2.0]], dtype=np.float16)
    W3 = o.dequant(codes[1:, :256], s3, 3)
    assert W3[0, 0] == 14.0 and W3[0, 1] == 2.0 and W3[0, 2] == -14.0
    tiny = np.array([[2.0 ** -24]], dtype=np.float16)       # smallest fp16 subnormal
    assert o.dequant(codes[1:, :256], tiny, 3)[0, 0] == 7 * 2.0 ** -24
    assert np.all(o.dequant(codes[1:, :256], np.zeros((1, 1), np.float16), 3) == 0)


def test_ternary_quantizer_rules():
    K, N = 512, 16
    signs = wr_synth.sign_bits(3, K)
    W = wr_synth.weights_fp32(4, N, K)
    codes, alpha, Wr = o.quantize_ternary(W, signs)
    t = codes.astype(np.int64) - 1
    for n in range(N):
        a = np.abs(Wr[n])
        delta = 0.7 * a.mean()
        assert np.array_equal(t[n] != 0, a > delta)
        assert np.array_equal(np.sign(Wr[n])[t[n] != 0], t[n][t[n] != 0])
        # alpha is the least-squares scale for fixed t (then rounded to fp16)
        best = float(np.dot(np.abs(Wr[n]), np.abs(t[n])) / np.abs(t[n]).sum())
        f = lambda al: float(((Wr[n] - al * t[n]) ** 2).sum())
        assert f(best) <= min(f(best * 1.001), f(best * 0.999))
        assert float(alpha[n]) == float(np.float16(best))


# ---------------------------------------------------------------- contraction

def _brute(x_bits, codes, scales, bits):
    """Exact rational y[m, n] = sum_k s g x and bound[m, n] = sum_k |s g x|, term by term."""
    M, K = x_bits.shape
    N = codes.shape[0]
    L = (1 << bits) - 1
    xf = [[float(v) for v in row] for row in wr_synth.bf16_bits_to_f32(x_bits)]
    y = [[0.0] * N for _ in range(M)]
    bound = [[Fraction(0)] * N for _ in range(M)]
    for m in range(M):
        for n in range(N):
            acc, mag = Fraction(0), Fraction(0)
            for k in range(K):
                g = 2 * int(codes[n, k]) - L
                term = Fraction(float(scales[n, k // 256])) * g * Fraction(xf[m][k])
                acc += term
                mag += abs(term)
            y[m][n] = float(acc)
            bound[m][n] = mag
    return np.array(y), bound


@pytest.mark.parametrize("bits", [2, 3])
def test_gemm_against_exact_brute_force(bits):
    M, N, K = 2, 5, 512
    W = wr_synth.weights_fp32(31, N, K)
    codes, s = o.quantize_odd_grid(W, bits)
    x = wr_synth.activations_bf16(32, M, K)
    y, B = o.gemm_codes(x, codes, s, bits)
    ref, ref_bound = _brute(x, codes, s, bits)
    assert np.allclose(y, ref, rtol=1e-13, atol=1e-14)
    # the tolerance bound is exactly sum_k |w x| of the same (m, n): not a looser product of
    # norms, not summed over another axis
    for m in range(M):
        for n in range(N):
            assert math.isclose(float(B[m, n]), float(ref_bound[m][n]), rel_tol=1e-13)
    assert np.all(B >= np.abs(y))


def test_gemm_bound_hand_example():
    # one 256-block, 2-bit: s = 0.5, codes 0, 3, 1, 2 (g = -3, 3, -1, 1) on x = 1, 2, -4, 8
    # y = 0.5 (-3 + 6 + 4 + 8) = 7.5 ;  bound = 0.5 (3 + 6 + 4 + 8) = 10.5 ; a second row with
    # all codes 3 on the same x gives 0.5 * 3 * 7 = 10.5 and bound 0.5 * 3 * 15 = 22.5
    codes = np.full((2, 256), 1, dtype=np.uint8)
    codes[0, :4] = [0, 3, 1, 2]
    codes[1, :4] = [3, 3, 3, 3]
    codes[:, 4:] = 1
    s = np.full((2, 1), 0.5, dtype=np.float16)
    xv = np.zeros((1, 256), dtype=np.float32)
    xv[0, :4] = [1, 2, -4, 8]
    x = wr_synth.f32_to_bf16_bits(xv)
    y, B = o.gemm_codes(x, codes, s, 2)
    assert y[0, 0] == 7.5 and B[0, 0] == 10.5
    assert y[0, 1] == 10.5 and B[0, 1] == 22.5


def test_gemm_special_cases():
    K, N = 512, 4
    codes = np.full((N, K), 3, dtype=np.uint8)        # level +3 everywhere (2-bit)
    s = np.full((N, 2), 0.25, dtype=np.float16)
    x = wr_synth.activations_bf16(9, 1, K)
    xf = wr_synth.bf16_bits_to_f32(x).astype(np.float64)
    y, _ = o.gemm_codes(x, codes, s, 2)
    assert np.allclose(y, 3 * 0.25 * xf.sum(), rtol=1e-14)
    # one-hot x picks a column of W
    W = wr_synth.weights_fp32(10, N, K)
    codes, s = o.quantize_odd_grid(W, 3)
    onehot = np.zeros((1, K), dtype=np.uint16)
    onehot[0, 300] = 0x3F80                             # bf16 1.0
    y, _ = o.gemm_codes(onehot, codes, s, 3)
    assert np.array_equal(y[0], o.dequant(codes, s, 3)[:, 300])


def test_dequant_ternary_hand_example():
    # N = 2 rows, K = 3 positions (N != K, so a broadcast along the wrong axis shows):
    # codes 0, 1, 2 stand for t = -1, 0, +1 and alpha is one scale per ROW
    codes = np.array([[0, 1, 2], [2, 2, 0]], dtype=np.uint8)
    alpha = np.array([0.5, 3.0], dtype=np.float16)
    W = o.dequant_ternary(codes, alpha)
    assert W.shape == (2, 3)
    assert W.tolist() == [[-0.5, 0.0, 0.5], [3.0, 3.0, -3.0]]


def _hadamard_entry(a, b):
    """Sylvester Hadamard entry in closed form: (-1)^popcount(a & b)."""
    return -1.0 if bin(a & b).count("1") % 2 else 1.0


def test_ternary_gemm_against_closed_form_brute_force():
    # (R x)[k] = (1/sqrt(128)) sum_{j in k's block} (-1)^popcount(k%128 & j%128) d_j x_j, with
    # d_j = -1 where bit j of the sign mask is set; y = alpha_n sum_k (c - 1) (R x)[k] and
    # bound = sum_k |alpha_n (c - 1)| |(R x)[k]|, written out element by element
    K, N, M = 256, 3, 2
    signs = wr_synth.sign_bits(40, K)
    rng = np.random.default_rng(41)
    codes = rng.integers(0, 3, size=(N, K)).astype(np.uint8)
    alpha = np.array([0.25, 1.5, 0.0625], dtype=np.float16)
    x = wr_synth.activations_bf16(42, M, K)
    xf = wr_synth.bf16_bits_to_f32(x).astype(np.float64)
    d = [(-1.0 if (int(signs[j // 32]) >> (j % 32)) & 1 else 1.0) for j in range(K)]
    xr = np.zeros((M, K))
    for m in range(M):
        for k in range(K):
            b0 = (k // 128) * 128
            xr[m, k] = sum(_hadamard_entry(k - b0, j - b0) * d[j] * xf[m, j]
                           for j in range(b0, b0 + 128)) / math.sqrt(128)
    y, B = o.gemm_ternary(x, codes, alpha, signs)
    for m in range(M):
        for n in range(N):
            a = float(alpha[n])
            ref = sum(a * (int(codes[n, k]) - 1) * xr[m, k] for k in range(K))
            mag = sum(abs(a * (int(codes[n, k]) - 1)) * abs(xr[m, k]) for k in range(K))
            assert math.isclose(y[m, n], ref, rel_tol=1e-12, abs_tol=1e-12)
            assert math.isclose(B[m, n], mag, rel_tol=1e-12)


def test_ternary_gemm_matches_rotation_identity():
    K, N, M = 640, 16, 2
    signs = wr_synth.sign_bits(12, K)
    W = wr_synth.weights_fp32(13, N, K)
    codes, alpha, _ = o.quantize_ternary(W, signs)
    x = wr_synth.activations_bf16(14, M, K)
    y, B = o.gemm_ternary(x, codes, alpha, signs)
    # same result from the unrotated dense weight R^T (alpha t) applied to plain x
    Wt = o.dequant_ternary(codes, alpha)
    R = o.rotate(np.eye(K), signs).T       # column k is R e_k
    dense = Wt @ R                         # (alpha t) R: the weights in the unrotated basis
    xf = wr_synth.bf16_bits_to_f32(x).astype(np.float64)
    assert np.allclose(y, xf @ dense.T, rtol=1e-11, atol=1e-12)
    assert np.all(B >= np.abs(y) - 1e-12)


# ---------------------------------------------------------------- packed layout

def test_pack_golden_vectors(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "pack_vectors.json")))
    for case in g["cases"]:
        fmt, N, K = case["fmt"], case["N"], case["K"]
        codes = np.full((N, K), case["fill"], dtype=np.uint8)
        for n, k, c in case["set"]:
            codes[n, k] = c
        p = o.pack(fmt, codes)
        assert p.size == o.packed_bytes(fmt, N, K)
        for idx, val in case["expect"].items():
            assert int(p[int(idx)]) == val, (case["fmt"], idx)
        # every byte not listed holds the fill pattern
        fillbyte = 121 if fmt == o.FMT_TERNARY else 0
        listed = {int(i) for i in case["expect"]}
        others = np.array([i for i in range(p.size) if i not in listed])
        nz = others[p[others] != fillbyte]
        assert nz.size == 0, (fmt, nz[:10])
        assert np.array_equal(o.unpack_codes(fmt, p, N, K), codes)


@pytest.mark.parametrize("fmt,levels,N,K", [(2, 4, 48, 768), (3, 8, 40, 512), (1, 3, 35, 700),
                                             (1, 3, 16, 2560), (2, 4, 1, 256)])
def test_pack_round_trip(fmt, levels, N, K):
    rng = np.random.default_rng(fmt * 100 + N)
    codes = rng.integers(0, levels, (N, K)).astype(np.uint8)
    p = o.pack(fmt, codes)
    assert np.array_equal(o.unpack_codes(fmt, p, N, K), codes)


def test_pack_is_a_bijection_on_bytes():
    # Q2/Q3 with N % 16 == 0 use every bit exactly once: distinct code arrays give
    # distinct byte arrays and the byte count equals the bit count / 8
    for fmt, b in ((2, 2), (3, 3)):
        N, K = 16, 256
        byte, bit = o.code_bit_positions(fmt, N, K)
        flat = (byte.astype(np.int64) * 8 + bit).ravel()
        assert np.unique(flat).size == flat.size == N * K * b
        assert flat.max() < o.packed_bytes(fmt, N, K) * 8


# ---------------------------------------------------------------- trellis coding

def test_trellis_toy_matches_the_page(golden_dir):
    """The page's 1-bit toy: greedy and best-path picks, states and squared errors, and the
    plain 1-bit rounding it is compared with."""
    g = json.load(open(os.path.join(golden_dir, "trellis_toy.json")))
    vals, t, k = np.array(g["values"]), np.array(g["targets"]), g["bits"]
    u_g, e_g = o.trellis_greedy(t, vals, k)
    idx_g = o.trellis_level_index(u_g)
    assert np.allclose(vals[idx_g], g["greedy"]["picks"])
    assert list(idx_g & 1) == g["greedy"]["states"]           # the level's coset is the state
    assert abs(e_g - g["greedy"]["squared_error"]) < 1e-9
    u_v, e_v = o.trellis_viterbi(t, vals, k)
    idx_v = o.trellis_level_index(u_v)
    assert np.allclose(vals[idx_v], g["best_path"]["picks"])
    assert list(idx_v & 1) == g["best_path"]["states"]
    assert abs(float(e_v) - g["best_path"]["squared_error"]) < 1e-9
    lv = np.array(g["plain_one_bit_rounding"]["levels"])
    plain = ((t[:, None] - lv[None, :]) ** 2).min(axis=1).sum()
    assert abs(plain - g["plain_one_bit_rounding"]["squared_error"]) < 1e-9


@pytest.mark.parametrize("k", [1, 2])
def test_trellis_viterbi_is_the_brute_force_optimum(k):
    """On short random sequences the Viterbi path costs exactly the minimum over all U^n
    symbol sequences, and its symbols reach that cost."""
    import itertools
    rng = np.random.default_rng(11 + k)
    U = 1 << k
    for _ in range(40):
        n = int(rng.integers(1, 6))
        vals = np.sort(rng.normal(size=2 * U))
        t = rng.normal(size=n)
        best = min(
            sum((t[i] - vals[idx]) ** 2 for i, idx in enumerate(o.trellis_level_index(np.array(seq))))
            for seq in itertools.product(range(U), repeat=n))
        u, c = o.trellis_viterbi(t, vals, k)
        idx = o.trellis_level_index(u)
        assert abs(float(c) - best) < 1e-12
        assert abs(float(((t - vals[idx]) ** 2).sum()) - best) < 1e-12
        _, cg = o.trellis_greedy(t, vals, k)
        assert float(c) <= cg + 1e-12


def test_trellis2_quantizer_invariants():
    """The 2-bit trellis format: symbols in [0, 4), the level index 2u + state restarts at
    every block, the weights lie on s * {-7..7 odd}, its squared error is never above the
    greedy encoding of the same block, and over the matrix it is below that of the 4-level
    nearest-point grid, which stores the same 2 bits per weight."""
    W = wr_synth.weights_fp32(5, 8, 512)
    u, s = o.quantize_trellis2(W)
    assert u.dtype == np.uint8 and u.max() <= 3
    Wd = o.dequant_trellis2(u, s)
    sb = np.repeat(s.astype(np.float64), 256, axis=1)
    lv = Wd / np.where(sb > 0, sb, 1.0)
    assert np.all(np.isin(np.round(lv), np.arange(-7, 8, 2))) and np.allclose(lv, np.round(lv))
    # block restart: the first weight of every block takes an even level index (state 0)
    c3 = (np.round(lv).astype(int) + 7) // 2
    assert np.all(c3[:, ::256] % 2 == 0)
    err_t = ((W.astype(np.float64) - Wd) ** 2).reshape(8, 2, 256).sum(axis=2)
    levels = np.arange(-7, 8, 2, dtype=np.float64)
    for n in range(8):
        for b in range(2):
            vals = float(s[n, b]) * levels
            _, eg = o.trellis_greedy(W[n, 256 * b:256 * (b + 1)].astype(np.float64), vals, 2)
            assert err_t[n, b] <= eg + 1e-12
    c2, s2 = o.quantize_odd_grid(W, 2)
    err_q2 = ((W.astype(np.float64) - o.dequant(c2, s2, 2)) ** 2).sum()
    assert err_t.sum() < err_q2


# ---------------------------------------------------------------- 8-state trellis (4-weight symbols)

def test_trellis8_state_machine_hand_example():
    # two symbols: codes [1, 2, 3, 1] from state 0 (parity pattern 0000) give level indices
    # [2, 4, 6, 2]; the last code's low bit (1) makes the next state 1, whose pattern is
    # (1, 0, 0, 1): codes [0, 3, 2, 2] give [1, 6, 4, 5]; the next state is (1 << 1 | 0) = 2
    c = o.trellis8_level_index(np.array([1, 2, 3, 1, 0, 3, 2, 2]))
    assert c.tolist() == [2, 4, 6, 2, 1, 6, 4, 5]
    assert o.trellis8_next(1, 2) == 2 and o.trellis8_next(5, 3) == 3 and o.trellis8_next(7, 1) == 7
    assert [o.trellis8_parity(s) for s in range(8)] == [
        (0, 0, 0, 0), (1, 0, 0, 1), (0, 1, 0, 1), (1, 1, 0, 0),
        (0, 0, 1, 1), (1, 0, 1, 0), (0, 1, 1, 0), (1, 1, 1, 1)]


def test_trellis8_cosets_are_a_set_partition_of_the_even_parity_vectors():
    # every state's coset holds 256 points, the 8 cosets are disjoint, and together they are
    # exactly the 2048 level-index 4-vectors whose parities sum to an even number
    seen = set()
    for s in range(8):
        p = o.trellis8_parity(s)
        pts = {tuple(2 * u + p[i] for i, u in enumerate(us))
               for us in np.ndindex(4, 4, 4, 4)}
        assert len(pts) == 256 and not (pts & seen)
        seen |= pts
    even = {v for v in np.ndindex(8, 8, 8, 8) if sum(x & 1 for x in v) % 2 == 0}
    assert seen == even


def _trellis8_cost(t, vals, codes):
    c = o.trellis8_level_index(codes)
    return float(((t - vals[c]) ** 2).sum())


@pytest.mark.parametrize("nsym", [1, 2])
def test_trellis8_viterbi_is_the_brute_force_optimum(nsym):
    rng = np.random.default_rng(50 + nsym)
    vals = np.arange(-7, 8, 2, dtype=np.float64) * 0.31
    all_codes = np.array(list(np.ndindex(*([4] * (4 * nsym)))), dtype=np.int64)   # 256^nsym paths
    lvl = o.trellis8_level_index(all_codes)
    for _ in range(4):
        t = rng.normal(0, 1.0, 4 * nsym)
        brute = ((t[None, :] - vals[lvl]) ** 2).sum(axis=1).min()
        codes, cost = o.trellis8_viterbi(t, vals)
        assert math.isclose(float(cost), float(brute), rel_tol=1e-12, abs_tol=1e-12)
        assert math.isclose(_trellis8_cost(t, vals, codes), float(brute), rel_tol=1e-12, abs_tol=1e-12)


def test_trellis8_error_below_the_two_state_trellis_and_the_grid():
    # on Gaussian weights at the same 2 bits per weight: 8-state < 2-state < 4-level grid
    W = wr_synth.weights_fp32(55, 8, 1024)
    codes8, s8 = o.quantize_trellis8(W)
    sym2, s2 = o.quantize_trellis2(W)
    q, sq = o.quantize_odd_grid(W, 2)
    W64 = W.astype(np.float64)
    e8 = ((W64 - o.dequant_trellis8(codes8, s8)) ** 2).sum()
    e2 = ((W64 - o.dequant_trellis2(sym2, s2)) ** 2).sum()
    eq = ((W64 - o.dequant(q, sq, 2)) ** 2).sum()
    assert e8 < e2 < eq
    assert codes8.max() <= 3 and np.array_equal(s8, s2)   # same scale rule as the 2-state format
    # the decoded level indices of each symbol have even parity sum
    c = o.trellis8_level_index(codes8.reshape(8, 4, 256).astype(np.int64)).reshape(-1, 4)
    assert np.all((c & 1).sum(axis=1) % 2 == 0)


def test_trellis8_dequant_and_s8_form():
    codes = np.zeros((2, 256), dtype=np.uint8)
    codes[0, :8] = [1, 2, 3, 1, 0, 3, 2, 2]
    s = np.array([[0.5], [2.0]], dtype=np.float16)
    W = o.dequant_trellis8(codes, s)
    assert W[0, :8].tolist() == [0.5 * (2 * c - 7) for c in (2, 4, 6, 2, 1, 6, 4, 5)]
    # all-zero codes stay in state 0 (the low bit of u_3 is 0): level index 0 everywhere
    assert np.all(W[1] == -14.0)
    d = np.array([0.25, 1.0], dtype=np.float16)
    qm = np.array([[2], [2]], dtype=np.int8)
    assert np.array_equal(o.dequant_trellis8_s8(codes, d, qm), o.dequant_trellis8(codes, s))
