"""wr_gemv_noalloc: the decode GEMV with its scratch in a fixed device array inside libwr.

Collected last on purpose (file name): it must also pass after every other test has run in the
same process. Each case runs wr_gemv (caller workspace) once and wr_gemv_noalloc twice in a row
on the same inputs; both no-allocation results must agree with the workspace result and with
the fp64 oracle within the GEMV tolerance (|err| <= 1e-4 * sum_k |w x|, exact zero where that
sum is zero). The second call checks that the scratch (its counters in particular) is left
ready for the next call."""
import numpy as np
import pytest

import wr_synth
from oracle import wr_oracle as o
from gpu_inputs import check_close, dev, q_case, s8_case, torch_mod


def test_too_large_rejected_before_device_work():
    import bit_weight_only_wr_b200 as wr
    M, N, K, bits = 8, 65536, 65536, 2
    assert wr.wr_gemv_workspace_bytes(M, N, K, bits) > wr.WR_GEMV_NOALLOC_SCRATCH_BYTES
    fake = 4096   # aligned, never dereferenced: the size check comes first
    with pytest.raises(wr.WrError) as e:
        wr.wr_gemv_noalloc(M, N, K, fake, fake, fake, bits, fake, stream=0)
    assert e.value.status == 5
    with pytest.raises(wr.WrError) as e:
        wr.wr_gemv_noalloc(M, 256, 300, fake, fake, fake, bits, fake, stream=0)   # K % 256 != 0
    assert e.value.status == 1


@pytest.mark.gpu
@pytest.mark.parametrize("bits,N,K,M", [
    (2, 4096, 2560, 1),      # q projection, split K
    (3, 2560, 9728, 5),      # down projection, deep split K
    (2, 300, 768, 8),        # ragged N, every token slot
    (3, 9728, 2560, 3),      # up projection
])
def test_noalloc_matches_workspace_path(bits, N, K, M):
    torch = torch_mod()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_weight_only_wr_b200 as wr
    assert wr.wr_gemv_workspace_bytes(M, N, K, bits) <= wr.WR_GEMV_NOALLOC_SCRATCH_BYTES
    seed = 7000 + 10 * bits + M
    codes, scales_h, packed, scales = q_case(wr, bits, N, K, seed)
    x_bits = wr_synth.activations_bf16(seed + 1, M, K)
    x = dev(x_bits)

    y_ws = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    nb = wr.wr_gemv_workspace_bytes(M, N, K, bits)
    ws = torch.zeros(max(nb, 256), dtype=torch.uint8, device="cuda")
    wr.wr_gemv(M, N, K, x, packed, scales, bits, y_ws, ws, nb)

    outs = []
    for _ in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        wr.wr_gemv_noalloc(M, N, K, x, packed, scales, bits, y)
        torch.cuda.synchronize()
        outs.append(y.cpu().numpy())
    torch.cuda.synchronize()
    assert wr.wr_get_device_error() == 0

    y_ref, bound = o.gemm_codes(x_bits, codes, scales_h, bits)
    y_ws = y_ws.cpu().numpy()
    check_close(y_ws, y_ref, bound)
    for y in outs:
        check_close(y, y_ref, bound)
        assert np.all(np.abs(y.astype(np.float64) - y_ws) <= 1e-4 * bound)


@pytest.mark.gpu
@pytest.mark.parametrize("fmt_name,N,K,M", [
    ("t2", 300, 2560, 1),        # trellis-coded 2-bit symbols
    ("q3_i8", 1024, 2560, 4),    # 3-bit codes with int8 block scales
    ("q2_i8", 129, 768, 8),      # 2-bit codes with int8 block scales, ragged N
    ("t8", 200, 1024, 2),        # 8-state trellis codes
])
def test_noalloc_trellis_and_int8_scales(fmt_name, N, K, M):
    """The formats wr_gemv accepts besides plain Q2/Q3 (WR_FMT_T2, | WR_SCALES_I8), through the
    no-allocation entry point: agreement with wr_gemv and with the oracle on two calls in a row."""
    torch = torch_mod()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_weight_only_wr_b200 as wr
    seed = 7100 + N + M
    x_bits = wr_synth.activations_bf16(seed + 1, M, K)
    x = dev(x_bits)
    if fmt_name == "t8":
        fmt = wr.WR_FMT_T8
        c8, sc = wr.wr_quantize_trellis8(wr_synth.weights_fp32(seed, N, K))
        packed, scales = dev(wr.wr_pack(fmt, c8)), dev(sc)
        y_ref, bound = o.gemm_trellis8(x_bits, c8, sc.view(np.float16))
    elif fmt_name == "t2":
        fmt = wr.WR_FMT_T2
        sym, sc = wr.wr_quantize_trellis(wr_synth.weights_fp32(seed, N, K))
        packed, scales = dev(wr.wr_pack(fmt, sym)), dev(sc)
        y_ref, bound = o.gemm_trellis2(x_bits, sym, sc.view(np.float16))
    else:
        bits = 3 if fmt_name == "q3_i8" else 2
        fmt = bits | wr.WR_SCALES_I8
        codes, d, q, packed, scales = s8_case(wr, bits, N, K, seed)
        y_ref, bound = o.gemm_codes_s8(x_bits, codes, d, q, bits)
    assert wr.wr_gemv_workspace_bytes(M, N, K, fmt) <= wr.WR_GEMV_NOALLOC_SCRATCH_BYTES

    y_ws = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    nb = wr.wr_gemv_workspace_bytes(M, N, K, fmt)
    ws = torch.zeros(max(nb, 256), dtype=torch.uint8, device="cuda")
    wr.wr_gemv(M, N, K, x, packed, scales, fmt, y_ws, ws, nb)
    outs = []
    for _ in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        wr.wr_gemv_noalloc(M, N, K, x, packed, scales, fmt, y)
        torch.cuda.synchronize()
        outs.append(y.cpu().numpy())
    assert wr.wr_get_device_error() == 0
    y_ws = y_ws.cpu().numpy()
    check_close(y_ws, y_ref, bound)
    for y in outs:
        check_close(y, y_ref, bound)
        assert np.all(np.abs(y.astype(np.float64) - y_ws) <= 1e-4 * bound)
