"""GPU parity of the grouped decode GEMV (one x, several weight matrices, one launch pair) and of
batched calls whose problems share an x (their activation tiles are prepared once): every output
against the fp64 oracle, |err| <= 1e-4 * sum_k |w x| per element."""
import numpy as np
import pytest

import wr_synth
from oracle import wr_oracle as o
from gpu_inputs import check_close, dev, q_case, s8_case, torch_mod

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


def _item(wr, kind, N, K, seed):
    """(packed, scales, fmt, reference function of x) for one weight matrix."""
    if kind == "t8":
        codes, sc = wr.wr_quantize_trellis8(wr_synth.weights_fp32(seed, N, K))
        return dev(wr.wr_pack(wr.WR_FMT_T8, codes)), dev(sc), wr.WR_FMT_T8, \
            (lambda x: o.gemm_trellis8(x, codes, sc.view(np.float16)))
    if kind == "t2":
        sym, sc = wr.wr_quantize_trellis(wr_synth.weights_fp32(seed, N, K))
        return dev(wr.wr_pack(wr.WR_FMT_T2, sym)), dev(sc), wr.WR_FMT_T2, \
            (lambda x: o.gemm_trellis2(x, sym, sc.view(np.float16)))
    if kind.endswith("i8"):
        bits = int(kind[1])
        codes, d, q, packed, rec = s8_case(wr, bits, N, K, seed)
        return packed, rec, bits | wr.WR_SCALES_I8, (lambda x: o.gemm_codes_s8(x, codes, d, q, bits))
    bits = int(kind[1])
    codes, scales, packed, s_d = q_case(wr, bits, N, K, seed)
    return packed, s_d, bits, (lambda x: o.gemm_codes(x, codes, scales, bits))


@pytest.mark.parametrize("M", [1, 4, 8])
@pytest.mark.parametrize("group", [
    ("qkv", 2560, [("q2", 4096), ("q2", 1024), ("q3", 1024)]),
    ("gate_up", 2560, [("q2", 9728), ("q3", 9728)]),
    ("ragged_mixed", 768, [("q3", 129), ("t2", 40), ("q2i8", 300), ("q2", 16), ("q3i8", 200), ("t8", 77)]),
])
def test_grouped_matches_oracle(wr, M, group):
    torch = torch_mod()
    name, K, kinds = group
    x_bits = wr_synth.activations_bf16(2000 + M + K, M, K)
    items, refs = [], []
    for i, (kind, N) in enumerate(kinds):
        packed, scales, fmt, ref = _item(wr, kind, N, K, seed=2100 + 10 * i + N)
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        items.append((packed, scales, y, N, fmt))
        refs.append(ref(x_bits))
    nb = wr.wr_gemv_grouped_workspace_bytes(M, K, items)
    ws = _ws(nb)
    x = dev(x_bits)
    for _ in range(2):   # twice in a row: the workspace is left ready for the next call
        for it in items:
            it[2].fill_(float("nan"))
        wr.wr_gemv_grouped(M, K, x, items, ws, nb)
        torch.cuda.synchronize()
        for (_, _, y, _, _), (ref, B) in zip(items, refs):
            check_close(y.cpu().numpy(), ref, B)
    assert wr.wr_get_device_error() == 0


def test_batched_problems_sharing_x(wr):
    """A batched call in which several problems read the same x tensor (and others their own):
    the shared activation tiles are prepared once and every output still matches the oracle."""
    torch = torch_mod()
    M, K = 3, 1024
    xa_bits, xb_bits = wr_synth.activations_bf16(2201, M, K), wr_synth.activations_bf16(2202, M, K)
    xa, xb = dev(xa_bits), dev(xb_bits)
    spec = [("q2", 256, xa, xa_bits), ("q3", 130, xa, xa_bits), ("q2", 64, xb, xb_bits), ("q2", 512, xa, xa_bits),
            ("t2", 100, xa, xa_bits), ("q3", 70, xb, xb_bits)]
    problems, refs = [], []
    for i, (kind, N, x, xbits) in enumerate(spec):
        packed, scales, fmt, ref = _item(wr, kind, N, K, seed=2300 + i)
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        problems.append((x, packed, scales, y, N, K, fmt))
        refs.append(ref(xbits))
    nb = wr.wr_gemv_batched_workspace_bytes(M, problems)
    ws = _ws(nb)
    wr.wr_gemv_batched(M, problems, ws, nb)
    torch.cuda.synchronize()
    for p, (ref, B) in zip(problems, refs):
        check_close(p[3].cpu().numpy(), ref, B)


def test_grouped_rejects_bad_items(wr):
    torch = torch_mod()
    M, K = 1, 512
    y = torch.zeros(1, 16, device="cuda")
    ok = [(16, 16, y, 16, 2)]
    assert wr.wr_gemv_grouped_workspace_bytes(M, K, ok) > 0
    for bad in ([(16, 16, y, 16, 6)], [(16, 16, y, 0, 2)]):
        assert wr.wr_gemv_grouped_workspace_bytes(M, K, bad) == 0
    assert wr.wr_gemv_grouped_workspace_bytes(M, 300, ok) == 0     # K % 256 != 0
    assert wr.wr_gemv_grouped_workspace_bytes(33, K, ok) == 0      # M > 32
