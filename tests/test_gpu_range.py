"""GPU parity on the activation dynamic range: every GEMV/GEMM path against the fp64 oracle when
the activations of a row, or of single 256-blocks, are far from N(0, 1).

The decode GEMV turns each (token, block) of x into integers relative to the block's largest
element, so these cases reach the corners of that encoding: blocks scaled by 2^-90 .. 2^-120 and
into bf16's subnormal range, blocks scaled by 2^+100, rows whose blocks alternate between tiny
and N(0, 1), and the worst case of the rounding argument (one element sets the block's exponent
and every other element sits on a half step of the coarsest position). Tolerance as everywhere:
|err| <= 1e-4 * sum_k |w x| per element, plus one half subnormal spacing per accumulated term
where the result itself is below fp32's normal range (gpu_inputs.fp32_floor)."""
import numpy as np
import pytest

import wr_synth
from oracle import wr_oracle as o
from gpu_inputs import check_close, dev, fp32_floor, q_case, s8_case, t_case, torch_mod

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wr():
    torch = torch_mod()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_weight_only_wr_b200 as lib
    return lib


def scaled_x(seed, M, K, pattern):
    """bf16 activations: N(0, 1) drawn in fp32, scaled per 256-block by a power of two (in
    fp64, exact), then rounded once to bf16 (values below 2^-126 become bf16 subnormals)."""
    x = wr_synth.bf16_bits_to_f32(wr_synth.activations_bf16(seed, M, K)).astype(np.float64)
    nb = K // 256
    if pattern == "mixed":        # blocks alternate between 2^-120 and 1, token by token
        e = np.array([[(-120 if (b + m) % 2 == 0 else 0) for b in range(nb)] for m in range(M)])
    elif pattern == "subnormal":  # every block in bf16's subnormal range (2^-133 .. 2^-126)
        e = np.full((M, nb), -131)
    else:
        e = np.full((M, nb), int(pattern))
    x = x * np.repeat(np.exp2(e.astype(np.float64)), 256, axis=1)
    return wr_synth.f32_to_bf16_bits(x.astype(np.float32))


PATTERNS = ["-90", "-110", "-120", "subnormal", "100", "mixed"]


def _ws(nb):
    torch = torch_mod()
    return torch.zeros(max(nb, 256), dtype=torch.uint8, device="cuda")


def _gemv(wr, fmt, x_bits, packed, scales, N, K):
    torch = torch_mod()
    M = x_bits.shape[0]
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    nb = wr.wr_gemv_workspace_bytes(M, N, K, fmt)
    wr.wr_gemv(M, N, K, dev(x_bits), packed, scales, fmt, y, _ws(nb), nb)
    torch.cuda.synchronize()
    return y.cpu().numpy()


@pytest.mark.parametrize("pattern", PATTERNS)
@pytest.mark.parametrize("bits,M", [(2, 1), (3, 3), (2, 8)])
def test_gemv_activation_range(wr, bits, M, pattern):
    N, K = 300, 1024
    codes, scales, packed, s_d = q_case(wr, bits, N, K, seed=1100 + bits)
    x = scaled_x(1200 + M, M, K, pattern)
    y = _gemv(wr, bits, x, packed, s_d, N, K)
    ref, B = o.gemm_codes(x, codes, scales, bits)
    check_close(y, ref, B, floor=fp32_floor(K))
    assert wr.wr_get_device_error() == 0


@pytest.mark.parametrize("pattern", ["-120", "subnormal", "mixed"])
def test_gemv_activation_range_trellis_and_int8_scales(wr, pattern):
    N, K, M = 130, 768, 2
    x = scaled_x(1300, M, K, pattern)
    W = wr_synth.weights_fp32(1301, N, K)
    sym, sc = wr.wr_quantize_trellis(W)
    y = _gemv(wr, wr.WR_FMT_T2, x, dev(wr.wr_pack(wr.WR_FMT_T2, sym)), dev(sc), N, K)
    ref, B = o.gemm_trellis2(x, sym, sc.view(np.float16))
    check_close(y, ref, B, floor=fp32_floor(K))
    c8, sc8 = wr.wr_quantize_trellis8(W)
    y = _gemv(wr, wr.WR_FMT_T8, x, dev(wr.wr_pack(wr.WR_FMT_T8, c8)), dev(sc8), N, K)
    ref, B = o.gemm_trellis8(x, c8, sc8.view(np.float16))
    check_close(y, ref, B, floor=fp32_floor(K))
    codes, d, q, packed, rec = s8_case(wr, 3, N, K, seed=1302)
    y = _gemv(wr, 3 | wr.WR_SCALES_I8, x, packed, rec, N, K)
    ref, B = o.gemm_codes_s8(x, codes, d, q, 3)
    check_close(y, ref, B, floor=fp32_floor(K))


def test_gemv_batched_and_noalloc_activation_range(wr):
    torch = torch_mod()
    M = 4
    problems, refs = [], []
    for i, (N, K, bits, pattern) in enumerate([(64, 512, 2, "subnormal"), (200, 2560, 3, "mixed"),
                                               (40, 256, 2, "100"), (129, 768, 3, "-110")]):
        codes, scales, packed, s_d = q_case(wr, bits, N, K, seed=1400 + i)
        x = scaled_x(1410 + i, M, K, pattern)
        refs.append((o.gemm_codes(x, codes, scales, bits), K))
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        problems.append((dev(x), packed, s_d, y, N, K, bits))
    nb = wr.wr_gemv_batched_workspace_bytes(M, problems)
    wr.wr_gemv_batched(M, problems, _ws(nb), nb)
    torch.cuda.synchronize()
    for (_, _, _, y, _, _, _), ((ref, B), K) in zip(problems, refs):
        check_close(y.cpu().numpy(), ref, B, floor=fp32_floor(K))
    # the no-allocation entry point on the same inputs
    for (x, packed, s_d, _, N, K, bits), ((ref, B), _) in zip(problems, refs):
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        wr.wr_gemv_noalloc(M, N, K, x, packed, s_d, bits, y)
        torch.cuda.synchronize()
        check_close(y.cpu().numpy(), ref, B, floor=fp32_floor(K))


@pytest.mark.parametrize("bits", [2, 3])
def test_gemv_worst_case_rounding(wr, bits):
    """One element per block (value 1.0, level +-1) sets the block exponent; every other element
    is a positive odd multiple of half the coarsest position step, 2^(E + e_max - 1), with level
    +L, so that every element at a coarsest position rounds by half a step (ties go to even: all
    multiples 4j + 1 round down, the errors add up) and carries the largest level."""
    N, K, M = 64, 1024, 1
    L = (1 << bits) - 1
    E = 1 - 30                                    # max |x| = 1.0: exponent 1
    e_max = 6 if bits == 2 else 5                 # largest position exponent of the format
    step = 2.0 ** (E + e_max - 1)
    rng = np.random.default_rng(1500 + bits)
    xv = ((4 * rng.integers(0, 32, size=(M, K)) + 1) * step).astype(np.float64)
    xv[:, ::256] = 1.0
    x = wr_synth.f32_to_bf16_bits(xv.astype(np.float32))
    assert np.array_equal(wr_synth.bf16_bits_to_f32(x).astype(np.float64), xv)   # exact in bf16
    codes = np.full((N, K), L, dtype=np.uint8)    # code L: level +L
    codes[:, ::256] = (L + 1) // 2                # level +1 at the element that sets E
    scales = np.full((N, K // 256), 0.01, dtype=np.float16)
    packed = dev(wr.wr_pack(bits, codes))
    y = _gemv(wr, bits, x, packed, dev(scales.view(np.uint16)), N, K)
    ref, B = o.gemm_codes(x, codes, scales, bits)
    check_close(y, ref, B)


@pytest.mark.parametrize("pattern", ["-120", "subnormal", "100", "mixed"])
@pytest.mark.parametrize("bits,M", [(2, 16), (3, 129)])
def test_gemm_activation_range(wr, bits, M, pattern):
    torch = torch_mod()
    N, K = 256, 1024
    codes, scales, packed, s_d = q_case(wr, bits, N, K, seed=1600 + bits)
    x = scaled_x(1700 + M, M, K, pattern)
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    nb = wr.wr_gemm_workspace_bytes(M, N, K, bits)
    wr.wr_gemm(M, N, K, dev(x), packed, s_d, bits, y, _ws(nb), nb)
    torch.cuda.synchronize()
    ref, B = o.gemm_codes(x, codes, scales, bits)
    check_close(y.cpu().numpy(), ref, B, floor=fp32_floor(K))


@pytest.mark.parametrize("pattern", ["-110", "-120", "subnormal", "100", "mixed"])
@pytest.mark.parametrize("M", [1, 5, 64, 129])
def test_ternary_activation_range(wr, M, pattern):
    torch = torch_mod()
    N, K = 200, 1280
    codes, alpha, signs, packed, a_d, s_d = t_case(wr, N, K, seed=1800)
    x = scaled_x(1900 + M, M, K, pattern)
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    nb = wr.wr_gemm_ternary_workspace_bytes(M, N, K)
    wr.wr_gemm_ternary(M, N, K, dev(x), packed, a_d, s_d, y, _ws(nb), nb)
    torch.cuda.synchronize()
    ref, B = o.gemm_ternary(x, codes, alpha, signs)
    check_close(y.cpu().numpy(), ref, B, floor=fp32_floor(K))
