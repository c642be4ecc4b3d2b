"""GPU parity of the 8-state trellis format (WR_FMT_T8, 4-weight symbols): the decode GEMV (single,
batched among the other formats, int8 block scales) against the oracle's decode of the same codes,
|err| <= 1e-4 * sum_k |w x| per element, and the bf16 materializer bit for bit."""
import numpy as np
import pytest

import wr_synth
from oracle import wr_oracle as o
from gpu_inputs import check_close, dev, q_case, s8_record, torch_mod

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wr():
    torch = torch_mod()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_weight_only_wr_b200 as lib
    return lib


def _ws(nb):
    torch = torch_mod()
    return torch.zeros(max(nb, 256), dtype=torch.uint8, device="cuda")


def t8_case(wr, N, K, seed):
    W = wr_synth.weights_fp32(seed, N, K)
    codes, sc = wr.wr_quantize_trellis8(W)
    codes_o, sc_o = o.quantize_trellis8(W)
    assert np.array_equal(codes, codes_o) and np.array_equal(sc, sc_o.view(np.uint16))
    return codes_o, sc_o, dev(wr.wr_pack(wr.WR_FMT_T8, codes)), dev(sc)


@pytest.mark.parametrize("M", [1, 3, 8])
@pytest.mark.parametrize("N,K", [(40, 512), (129, 768), (300, 2560), (2560, 9728)])
def test_trellis8_gemv(wr, M, N, K):
    torch = torch_mod()
    codes, sc, packed, s_d = t8_case(wr, N, K, seed=N + K + M)
    x = wr_synth.activations_bf16(810 + M, M, K)
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    nb = wr.wr_gemv_workspace_bytes(M, N, K, wr.WR_FMT_T8)
    wr.wr_gemv(M, N, K, dev(x), packed, s_d, wr.WR_FMT_T8, y, _ws(nb), nb)
    torch.cuda.synchronize()
    ref, B = o.gemm_trellis8(x, codes, sc)
    check_close(y.cpu().numpy(), ref, B)
    assert wr.wr_get_device_error() == 0


def test_trellis8_in_a_mixed_batch_with_int8_scales(wr):
    torch = torch_mod()
    M = 4
    problems, refs = [], []
    spec = [(64, 512, "t8"), (100, 768, "q2"), (40, 256, "t2"), (200, 2560, "t8i8"), (33, 1024, "q3")]
    for i, (N, K, kind) in enumerate(spec):
        x = wr_synth.activations_bf16(910 + i, M, K)
        if kind == "t8":
            codes, sc, packed, s_d = t8_case(wr, N, K, seed=80 + i)
            fmt, ref = wr.WR_FMT_T8, o.gemm_trellis8(x, codes, sc)
        elif kind == "t8i8":
            codes, sc, packed, _ = t8_case(wr, N, K, seed=80 + i)
            rng = np.random.default_rng(i)
            d = np.float16(0.01) * (1 + rng.random(N)).astype(np.float16)
            q = rng.integers(0, 128, (N, K // 256)).astype(np.int8)
            s_d = dev(s8_record(d, q))
            fmt, ref = wr.WR_FMT_T8 | wr.WR_SCALES_I8, o.gemm(x, o.dequant_trellis8_s8(codes, d, q))
        elif kind == "t2":
            W = wr_synth.weights_fp32(80 + i, N, K)
            sym, sc = wr.wr_quantize_trellis(W)
            packed, s_d = dev(wr.wr_pack(wr.WR_FMT_T2, sym)), dev(sc)
            fmt, ref = wr.WR_FMT_T2, o.gemm_trellis2(x, sym, sc.view(np.float16))
        else:
            bits = int(kind[1])
            codes, scales, packed, s_d = q_case(wr, bits, N, K, seed=80 + i)
            fmt, ref = bits, o.gemm_codes(x, codes, scales, bits)
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        problems.append((dev(x), packed, s_d, y, N, K, fmt))
        refs.append(ref)
    nb = wr.wr_gemv_batched_workspace_bytes(M, problems)
    wr.wr_gemv_batched(M, problems, _ws(nb), nb)
    torch.cuda.synchronize()
    for p, (ref, B) in zip(problems, refs):
        check_close(p[3].cpu().numpy(), ref, B)


@pytest.mark.parametrize("N,K", [(16, 256), (45, 768), (130, 2560)])
def test_trellis8_unpack_bf16_bit_exact(wr, N, K):
    torch = torch_mod()
    codes, sc, packed, s_d = t8_case(wr, N, K, seed=N * K)
    w = torch.empty(N, K, dtype=torch.int16, device="cuda")
    wr.wr_unpack_bf16(wr.WR_FMT_T8, N, K, packed, s_d, w)
    torch.cuda.synchronize()
    ref = o.f64_to_bf16_bits(o.dequant_trellis8(codes, sc))
    assert np.array_equal(w.cpu().numpy().view(np.uint16), ref)


def test_trellis8_gemm_is_unsupported(wr):
    torch = torch_mod()
    with pytest.raises(wr.WrError) as e:
        wr.wr_gemm(16, 16, 256, 16, 16, 16, wr.WR_FMT_T8, 16, 16, 1 << 20)
    assert e.value.status == 2
