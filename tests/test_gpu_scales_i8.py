"""GPU parity of the int8 block-scale form (s[n,b] = d_n q[n,b], the scale record of
include/wr.h) against the fp64 oracle, through the C ABI: the materializer bit for bit, the
decode GEMV (single, no-allocation and batched, mixed with fp16-scale problems), the prefill
GEMM and the device quantizer. Same tolerance as every other GEMV/GEMM test."""
import numpy as np
import pytest

import wr_synth
from oracle import wr_oracle as o
from gpu_inputs import check_close, dev, q_case, s8_case, s8_record, torch_mod

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wr():
    torch = torch_mod()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_weight_only_wr_b200 as lib
    return lib


def _zeros_ws(nbytes):
    torch = torch_mod()
    return torch.zeros(max(nbytes, 256), dtype=torch.uint8, device="cuda")


def _weights_with_edges(N, K, seed):
    """Seeded weights with rows whose blocks differ in absmax by orders of magnitude (small
    multipliers, q = 0 blocks), an all-zero row and an all-zero block."""
    W = wr_synth.weights_fp32(seed, N, K).copy()
    if N >= 4 and K >= 512:
        W[0, :256] *= np.float32(1e-3)          # q rounds to 0 for this block
        W[1, 256:512] *= np.float32(0.02)       # a small multiplier
        W[2] = 0.0                              # d = 0: the whole row is zero
        W[3, :256] = 0.0
    return W


def _trellis_s8(wr, N, K, seed):
    """Trellis symbols with an int8 scale record: the symbols of the trellis encoder and the
    two-level scales the odd-grid quantizer finds for the same weights at 3 bits."""
    W = wr_synth.weights_fp32(seed, N, K)
    sym, _ = wr.wr_quantize_trellis(W)
    _, d, q = o.quantize_odd_grid_s8(W, 3)
    return sym, d, q, dev(wr.wr_pack(wr.WR_FMT_T2, sym)), dev(s8_record(d, q))


@pytest.mark.parametrize("bits,N,K", [(2, 40, 512), (3, 33, 768), (2, 2560, 2560), (3, 1024, 9728)])
def test_s8_unpack_bf16_bit_exact(wr, bits, N, K):
    torch = torch_mod()
    W = _weights_with_edges(N, K, seed=N + K)
    codes, d, q, packed, rec = s8_case(wr, bits, N, K, 0, W=W)
    out = torch.zeros((N, K), dtype=torch.int16, device="cuda")
    wr.wr_unpack_bf16(bits | wr.WR_SCALES_I8, N, K, packed, rec, out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy().view(np.uint16), o.unpack_bf16_s8(codes, d, q, bits))


def test_s8_trellis_unpack_bf16_bit_exact(wr):
    torch = torch_mod()
    N, K = 45, 768
    sym, d, q, packed, rec = _trellis_s8(wr, N, K, seed=17)
    out = torch.zeros((N, K), dtype=torch.int16, device="cuda")
    wr.wr_unpack_bf16(wr.WR_FMT_T2 | wr.WR_SCALES_I8, N, K, packed, rec, out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy().view(np.uint16), o.f64_to_bf16_bits(o.dequant_trellis2_s8(sym, d, q)))


@pytest.mark.parametrize("M", [1, 3, 8])
@pytest.mark.parametrize("bits,N,K", [(2, 40, 512), (3, 129, 768), (2, 4096, 2560), (3, 2560, 9728)])
def test_s8_gemv(wr, bits, N, K, M):
    torch = torch_mod()
    W = _weights_with_edges(N, K, seed=3 * N + K + M)
    codes, d, q, packed, rec = s8_case(wr, bits, N, K, 0, W=W)
    x = wr_synth.activations_bf16(1000 + M, M, K)
    fmt = bits | wr.WR_SCALES_I8
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    nb = wr.wr_gemv_workspace_bytes(M, N, K, fmt)
    ws = _zeros_ws(nb)
    wr.wr_gemv(M, N, K, dev(x), packed, rec, fmt, y, ws, nb)
    torch.cuda.synchronize()
    rows = np.arange(N) if N <= 512 else np.random.default_rng(M).choice(N, 384, replace=False)
    ref, B = o.gemm_codes_s8(x, codes[rows], d[rows], q[rows], bits)
    check_close(y.cpu().numpy()[:, rows], ref, B)
    if N > 2 and K >= 512:
        assert np.all(y.cpu().numpy()[:, 2] == 0)     # the all-zero row (d = 0)
    assert wr.wr_get_device_error() == 0


def test_s8_gemv_noalloc_and_trellis(wr):
    torch = torch_mod()
    M, N, K = 2, 300, 2560
    sym, d, q, packed, rec = _trellis_s8(wr, N, K, seed=23)
    x = wr_synth.activations_bf16(1100, M, K)
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    wr.wr_gemv_noalloc(M, N, K, dev(x), packed, rec, wr.WR_FMT_T2 | wr.WR_SCALES_I8, y)
    torch.cuda.synchronize()
    ref, B = o.gemm(x, o.dequant_trellis2_s8(sym, d, q))
    check_close(y.cpu().numpy(), ref, B)


def test_s8_in_a_mixed_batch(wr):
    """fp16-scale and int8-scale problems of Q2, Q3 and the trellis format in one launch."""
    torch = torch_mod()
    M = 5
    problems, refs = [], []
    cases = [(64, 512, 2, True), (100, 768, 3, False), (40, 256, 3, True), (200, 2560, 4, True),
             (130, 1024, 2, False), (256, 2560, 3, True)]
    for i, (N, K, fmt, s8) in enumerate(cases):
        x = wr_synth.activations_bf16(1200 + i, M, K)
        if fmt == 4:
            sym, d, q, packed, rec = _trellis_s8(wr, N, K, seed=80 + i)
            refs.append(o.gemm(x, o.dequant_trellis2_s8(sym, d, q)))
            scales = rec
        elif s8:
            codes, d, q, packed, scales = s8_case(wr, fmt, N, K, seed=80 + i)
            refs.append(o.gemm_codes_s8(x, codes, d, q, fmt))
        else:
            codes, sc, packed, scales = q_case(wr, fmt, N, K, seed=80 + i)
            refs.append(o.gemm_codes(x, codes, sc, fmt))
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        problems.append((dev(x), packed, scales, y, N, K, fmt | (wr.WR_SCALES_I8 if s8 else 0)))
    nb = wr.wr_gemv_batched_workspace_bytes(M, problems)
    ws = _zeros_ws(nb)
    for _ in range(2):
        wr.wr_gemv_batched(M, problems, ws, nb)
        torch.cuda.synchronize()
        for (_, _, _, y, _, _, _), (ref, B) in zip(problems, refs):
            check_close(y.cpu().numpy(), ref, B)


@pytest.mark.parametrize("bits,N,K,M", [(2, 200, 1024, 16), (3, 200, 1024, 129), (2, 9728, 2560, 512),
                                        (3, 2560, 9728, 300)])
def test_s8_gemm(wr, bits, N, K, M):
    torch = torch_mod()
    W = _weights_with_edges(N, K, seed=5 * N + K + M)
    codes, d, q, packed, rec = s8_case(wr, bits, N, K, 0, W=W)
    x = wr_synth.activations_bf16(1300 + M, M, K)
    fmt = bits | wr.WR_SCALES_I8
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    nb = wr.wr_gemm_workspace_bytes(M, N, K, fmt)
    ws = _zeros_ws(nb)
    wr.wr_gemm(M, N, K, dev(x), packed, rec, fmt, y, ws, nb)
    torch.cuda.synchronize()
    rows = np.arange(N) if N <= 512 else np.random.default_rng(M).choice(N, 256, replace=False)
    ref, B = o.gemm_codes_s8(x, codes[rows], d[rows], q[rows], bits)
    check_close(y.cpu().numpy()[:, rows], ref, B)
    assert wr.wr_get_device_error() == 0


@pytest.mark.filterwarnings("ignore:overflow encountered in cast")
@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("N,K", [(16, 256), (37, 768), (130, 2560), (9, 9728)])
def test_s8_quantize_pack_bit_exact(wr, bits, N, K):
    """wr_quantize_pack with int8 block scales: the oracle's d, q and codes, packed, byte for
    byte, and the same bytes as the host quantizer."""
    torch = torch_mod()
    W = _weights_with_edges(N, K, seed=90 + N + bits)
    if N >= 9:
        W[5] *= np.float32(1e-3)               # d is an fp16 subnormal
        W[6, 3] = np.float32(4.0e9)            # d saturates at 65504; other blocks get q = 0
        W[7, 0:256] = np.float32(0.125) * np.array([3, -3, 2, -2] * 64, np.float32)   # ties on m s
    fmt = bits | wr.WR_SCALES_I8
    nrec = wr.wr_scales_bytes(fmt, N, K)
    pk = torch.zeros(wr.wr_packed_bytes(bits, N, K), dtype=torch.uint8, device="cuda")
    rec = torch.zeros(max(nrec, 16), dtype=torch.uint8, device="cuda")
    wr.wr_quantize_pack(fmt, N, K, dev(W), pk, rec)
    torch.cuda.synchronize()
    codes_o, d_o, q_o = o.quantize_odd_grid_s8(W, bits)
    assert np.array_equal(rec.cpu().numpy()[:nrec], s8_record(d_o, q_o)[:nrec])
    assert np.array_equal(pk.cpu().numpy(), o.pack(bits, codes_o))
    codes_h, rec_h = wr.wr_quantize(fmt, W)
    assert np.array_equal(rec.cpu().numpy()[:nrec], rec_h[:nrec])
    assert wr.wr_get_device_error() == 0
