"""GPU parity: the CUDA path against the fp64 oracle, element by element, through the C ABI.

Unpack must be bit-exact; every GEMV/GEMM output must satisfy
|y_gpu - y_ref| <= 1e-4 * sum_k |w[n,k] x[m,k]| (the bound in the oracle's fp64), and be
exactly zero where that sum is zero. Shapes span several tiles, ragged N, every M from 1 to 8
for the decode path, and the Qwen3-4B layer shapes at full size."""
import numpy as np
import pytest

import wr_synth
from oracle import wr_oracle as o
from gpu_inputs import check_close, dev, q_case, t_case, torch_mod

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


def _run_gemv(wr, bits, x_bits, packed, scales, N, K):
    torch = torch_mod()
    M = x_bits.shape[0]
    x = dev(x_bits)
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    nb = wr.wr_gemv_workspace_bytes(M, N, K, bits)
    ws = _zeros_ws(nb)
    wr.wr_gemv(M, N, K, x, packed, scales, bits, y, ws, nb)
    torch.cuda.synchronize()
    return y.cpu().numpy(), ws


# ---------------------------------------------------------------- unpack (bit-exact)

@pytest.mark.parametrize("bits,N,K", [(2, 40, 512), (2, 2560, 2560), (3, 33, 768), (3, 1024, 2560)])
def test_unpack_bf16_bit_exact(wr, bits, N, K):
    torch = torch_mod()
    codes, scales, packed, s_d = q_case(wr, bits, N, K, seed=N + K + bits)
    out = torch.zeros((N, K), dtype=torch.int16, device="cuda")
    wr.wr_unpack_bf16(bits, N, K, packed, s_d, out)
    torch.cuda.synchronize()
    ref = o.unpack_bf16(codes, scales, bits)
    assert np.array_equal(out.cpu().numpy().view(np.uint16), ref)


@pytest.mark.parametrize("N,K", [(35, 640), (48, 4096), (16, 9728)])
def test_unpack_bf16_ternary_bit_exact(wr, N, K):
    torch = torch_mod()
    codes, alpha, signs, packed, a_d, _ = t_case(wr, N, K, seed=N + K)
    out = torch.zeros((N, K), dtype=torch.int16, device="cuda")
    wr.wr_unpack_bf16(1, N, K, packed, a_d, out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy().view(np.uint16), o.unpack_bf16_ternary(codes, alpha))


# ---------------------------------------------------------------- decode GEMV

@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 6, 7, 8])
def test_gemv_every_m_ragged(wr, bits, M):
    N, K = 40, 768
    codes, scales, packed, s_d = q_case(wr, bits, N, K, seed=11 * M + bits)
    x = wr_synth.activations_bf16(200 + M, M, K)
    y, _ = _run_gemv(wr, bits, x, packed, s_d, N, K)
    ref, B = o.gemm_codes(x, codes, scales, bits)
    check_close(y, ref, B)


@pytest.mark.parametrize("bits,N,K,M", [(2, 2560, 2560, 1), (2, 4096, 2560, 8), (3, 1024, 2560, 1),
                                        (3, 2560, 9728, 1), (3, 2560, 9728, 8), (2, 9728, 2560, 3)])
def test_gemv_layer_shapes(wr, bits, N, K, M):
    codes, scales, packed, s_d = q_case(wr, bits, N, K, seed=N * 3 + K + M)
    x = wr_synth.activations_bf16(300 + M, M, K)
    y, ws = _run_gemv(wr, bits, x, packed, s_d, N, K)
    ref, B = o.gemm_codes(x, codes, scales, bits)
    check_close(y, ref, B)
    # the same workspace serves further calls (its counters were left at zero)
    torch = torch_mod()
    y2 = torch.empty_like(torch.from_numpy(y)).cuda()
    nb = wr.wr_gemv_workspace_bytes(M, N, K, bits)
    for _ in range(2):
        wr.wr_gemv(M, N, K, dev(x), packed, s_d, bits, y2, ws, nb)
    torch.cuda.synchronize()
    assert np.array_equal(y2.cpu().numpy().view(np.uint32), y.view(np.uint32))


def test_gemv_deterministic(wr):
    N, K, M = 2560, 9728, 2
    codes, scales, packed, s_d = q_case(wr, 3, N, K, seed=77)
    x = wr_synth.activations_bf16(78, M, K)
    y1, _ = _run_gemv(wr, 3, x, packed, s_d, N, K)
    y2, _ = _run_gemv(wr, 3, x, packed, s_d, N, K)
    assert np.array_equal(y1.view(np.uint32), y2.view(np.uint32))


def test_gemv_zero_cases(wr):
    N, K, M = 48, 512, 3
    codes, scales, packed, s_d = q_case(wr, 2, N, K, seed=5)
    x = wr_synth.activations_bf16(6, M, K)
    x[1] = 0                                   # an all-zero token
    y, _ = _run_gemv(wr, 2, x, packed, s_d, N, K)
    ref, B = o.gemm_codes(x, codes, scales, 2)
    check_close(y, ref, B)
    assert np.all(y[1] == 0)
    zs = dev(np.zeros_like(scales.view(np.uint16)))   # all scales zero -> y exactly 0
    y0, _ = _run_gemv(wr, 2, x, packed, zs, N, K)
    assert np.all(y0 == 0)


# ---------------------------------------------------------------- ternary

@pytest.mark.parametrize("M", [1, 2, 4, 5, 8, 9, 20])
@pytest.mark.parametrize("N,K", [(40, 640), (64, 4096)])
def test_ternary_gemv(wr, M, N, K):
    torch = torch_mod()
    codes, alpha, signs, packed, a_d, s_d = t_case(wr, N, K, seed=N + K + M)
    x = wr_synth.activations_bf16(400 + M, M, K)
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    nb = wr.wr_gemm_ternary_workspace_bytes(M, N, K)
    ws = _zeros_ws(nb)
    wr.wr_gemm_ternary(M, N, K, dev(x), packed, a_d, s_d, y, ws, nb)
    torch.cuda.synchronize()
    ref, B = o.gemm_ternary(x, codes, alpha, signs)
    check_close(y.cpu().numpy(), ref, B)


@pytest.mark.parametrize("N,K", [(2560, 9728), (9728, 2560)])
def test_ternary_gemv_layer_shapes(wr, N, K):
    torch = torch_mod()
    codes, alpha, signs, packed, a_d, s_d = t_case(wr, N, K, seed=N + 2 * K)
    M = 1
    x = wr_synth.activations_bf16(500, M, K)
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    nb = wr.wr_gemm_ternary_workspace_bytes(M, N, K)
    ws = _zeros_ws(nb)
    wr.wr_gemm_ternary(M, N, K, dev(x), packed, a_d, s_d, y, ws, nb)
    torch.cuda.synchronize()
    ref, B = o.gemm_ternary(x, codes, alpha, signs)
    check_close(y.cpu().numpy(), ref, B)


# ---------------------------------------------------------------- prefill GEMM (tcgen05)

def _run_gemm(wr, bits, x_bits, packed, scales, N, K):
    torch = torch_mod()
    M = x_bits.shape[0]
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    nb = wr.wr_gemm_workspace_bytes(M, N, K, bits)
    ws = _zeros_ws(nb)
    wr.wr_gemm(M, N, K, dev(x_bits), packed, scales, bits, y, ws, nb)
    torch.cuda.synchronize()
    return y.cpu().numpy()


@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("M", [9, 16, 17, 100, 128, 129, 300])
def test_gemm_ragged(wr, bits, M):
    N, K = 200, 1024
    codes, scales, packed, s_d = q_case(wr, bits, N, K, seed=13 * M + bits)
    x = wr_synth.activations_bf16(600 + M, M, K)
    y = _run_gemm(wr, bits, x, packed, s_d, N, K)
    ref, B = o.gemm_codes(x, codes, scales, bits)
    check_close(y, ref, B)


@pytest.mark.parametrize("bits,N,K,M", [(2, 9728, 2560, 512), (3, 2560, 9728, 512), (3, 9728, 2560, 16)])
def test_gemm_layer_shapes(wr, bits, N, K, M):
    codes, scales, packed, s_d = q_case(wr, bits, N, K, seed=N + K + M + bits)
    x = wr_synth.activations_bf16(700 + M, M, K)
    y = _run_gemm(wr, bits, x, packed, s_d, N, K)
    rows = np.random.default_rng(M).choice(N, 256, replace=False)
    ref, B = o.gemm_codes(x, codes[rows], scales[rows], bits)
    check_close(y[:, rows], ref, B)


@pytest.mark.parametrize("bits,N,K", [(2, 9728, 2560), (3, 2560, 9728)])
def test_gemm_full_size_sampled(wr, bits, N, K):
    """M = 4096 (the largest prefill size): every column of y for 64 sampled rows."""
    M = 4096
    codes, scales, packed, s_d = q_case(wr, bits, N, K, seed=N * 7 + K)
    x = wr_synth.activations_bf16(800, M, K)
    y = _run_gemm(wr, bits, x, packed, s_d, N, K)
    rows = np.random.default_rng(1).choice(N, 64, replace=False)
    ref, B = o.gemm_codes(x, codes[rows], scales[rows], bits)
    check_close(y[:, rows], ref, B)


def test_no_device_error_after_calls(wr):
    assert wr.wr_get_device_error() == 0


# ---------------------------------------------------------------- batched decode GEMV

@pytest.mark.parametrize("M", [1, 3, 8])
def test_gemv_batched_layer(wr, M):
    """The 7 linears of one Qwen3-4B layer (mixed 2/3-bit) in one batched launch, twice."""
    torch = torch_mod()
    cases, problems, ys = [], [], []
    for idx, (name, K, N, bits) in enumerate(wr_synth.QWEN3_4B_LAYER):
        codes, scales, packed, s_d = q_case(wr, bits, N, K, seed=wr_synth.module_seed(0, idx))
        x = wr_synth.activations_bf16(900 + idx, M, K)
        xd = dev(x)
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        cases.append((codes, scales, bits, x, xd, packed, s_d))
        ys.append(y)
        problems.append((xd, packed, s_d, y, N, K, bits))
    nb = wr.wr_gemv_batched_workspace_bytes(M, problems)
    ws = _zeros_ws(nb)
    for rep in range(2):
        wr.wr_gemv_batched(M, problems, ws, nb)
        torch.cuda.synchronize()
        for (codes, scales, bits, x, *_), y in zip(cases, ys):
            ref, B = o.gemm_codes(x, codes, scales, bits)
            check_close(y.cpu().numpy(), ref, B)


def test_gemv_batched_ragged_mixed(wr):
    torch = torch_mod()
    M = 5
    shapes = [(40, 512, 2), (300, 768, 3), (16, 256, 2), (129, 2560, 3), (1, 256, 3)]
    cases, problems = [], []
    for i, (N, K, bits) in enumerate(shapes):
        codes, scales, packed, s_d = q_case(wr, bits, N, K, seed=1000 + i)
        x = wr_synth.activations_bf16(1100 + i, M, K)
        xd = dev(x)
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        cases.append((codes, scales, bits, x, y))
        problems.append((xd, packed, s_d, y, N, K, bits))
    nb = wr.wr_gemv_batched_workspace_bytes(M, problems)
    ws = _zeros_ws(nb)
    wr.wr_gemv_batched(M, problems, ws, nb)
    torch.cuda.synchronize()
    for codes, scales, bits, x, y in cases:
        ref, B = o.gemm_codes(x, codes, scales, bits)
        check_close(y.cpu().numpy(), ref, B)


@pytest.mark.parametrize("M", [1, 3, 8])
def test_gemv_row_group_shared_by_many_ranges(wr, M):
    """Long rows: one 128-row group of 600 blocks (2-bit) and one of 400 blocks (3-bit) in one
    batch, so that the cost-cut block ranges give every CTA one or two blocks and a single row
    group is finished by hundreds of ranges through the partial slots (the last to arrive adds
    them in range order); then a ragged 3-bit problem after them. Run twice (the arrival
    counters must be back at zero)."""
    torch = torch_mod()
    shapes = [(100, 256 * 600, 2), (128, 256 * 400, 3), (37, 768, 3)]
    cases, problems = [], []
    for i, (N, K, bits) in enumerate(shapes):
        codes, scales, packed, s_d = q_case(wr, bits, N, K, seed=1500 + i)
        x = wr_synth.activations_bf16(1600 + i, M, K)
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        cases.append((codes, scales, bits, x, y))
        problems.append((dev(x), packed, s_d, y, N, K, bits))
    nb = wr.wr_gemv_batched_workspace_bytes(M, problems)
    ws = _zeros_ws(nb)
    for _ in range(2):
        wr.wr_gemv_batched(M, problems, ws, nb)
        torch.cuda.synchronize()
        for codes, scales, bits, x, y in cases:
            ref, B = o.gemm_codes(x, codes, scales, bits)
            check_close(y.cpu().numpy(), ref, B)
    assert wr.wr_get_device_error() == 0


@pytest.mark.parametrize("M", [64, 65, 129])
@pytest.mark.parametrize("N,K", [(200, 640), (1024, 2560), (256, 4096)])
def test_ternary_gemm_prefill(wr, M, N, K):
    """M > 8 runs the tensor-core prefill GEMM: 64-token tiles, ragged N and M, K splits."""
    torch = torch_mod()
    codes, alpha, signs, packed, a_d, s_d = t_case(wr, N, K, seed=7 * N + K + M)
    x = wr_synth.activations_bf16(600 + M, M, K)
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    nb = wr.wr_gemm_ternary_workspace_bytes(M, N, K)
    ws = _zeros_ws(nb)
    for _ in range(2):   # the counters left at zero serve a second call
        y.fill_(float("nan"))
        wr.wr_gemm_ternary(M, N, K, dev(x), packed, a_d, s_d, y, ws, nb)
        torch.cuda.synchronize()
        ref, B = o.gemm_ternary(x, codes, alpha, signs)
        check_close(y.cpu().numpy(), ref, B)


@pytest.mark.parametrize("N,K", [(9728, 2560), (2560, 9728)])
def test_ternary_gemm_prefill_m512(wr, N, K):
    """The bench's M = 512 ternary prefill shapes, every output element against the oracle."""
    torch = torch_mod()
    M = 512
    codes, alpha, signs, packed, a_d, s_d = t_case(wr, N, K, seed=N + 3 * K)
    x = wr_synth.activations_bf16(700, M, K)
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    nb = wr.wr_gemm_ternary_workspace_bytes(M, N, K)
    ws = _zeros_ws(nb)
    wr.wr_gemm_ternary(M, N, K, dev(x), packed, a_d, s_d, y, ws, nb)
    torch.cuda.synchronize()
    ref, B = o.gemm_ternary(x, codes, alpha, signs)
    check_close(y.cpu().numpy(), ref, B)


def test_gemv_batched_more_problems_than_one_launch(wr):
    """300 small mixed 2/3-bit problems in one call: the batch is split over two launches of at
    most 256 problems, and every problem still matches the oracle."""
    torch = torch_mod()
    rng = np.random.default_rng(4242)
    M = 2
    problems, refs, keep = [], [], []
    for i in range(300):
        N = int(rng.integers(1, 80))
        K = 256 * int(rng.integers(1, 4))
        bits = int(rng.integers(2, 4))
        codes, scales, packed, s_d = q_case(wr, bits, N, K, seed=20000 + i)
        x = wr_synth.activations_bf16(30000 + i, M, K)
        xd = dev(x)
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        keep += [xd, packed, s_d]
        problems.append((xd, packed, s_d, y, N, K, bits))
        refs.append(o.gemm_codes(x, codes, scales, bits))
    nb = wr.wr_gemv_batched_workspace_bytes(M, problems)
    ws = _zeros_ws(nb)
    wr.wr_gemv_batched(M, problems, ws, nb)
    torch.cuda.synchronize()
    for (_, _, _, y, _, _, _), (ref, B) in zip(problems, refs):
        check_close(y.cpu().numpy(), ref, B)
    assert wr.wr_get_device_error() == 0


def test_ternary_gemv_batched_more_problems_than_one_launch(wr):
    """270 small ternary problems in one batched call (two launches of at most 256)."""
    torch = torch_mod()
    rng = np.random.default_rng(4343)
    M = 3
    problems, refs = [], []
    for i in range(270):
        N = int(rng.integers(1, 48))
        K = 128 * int(rng.integers(1, 6))
        codes, alpha, signs, packed, a_d, s_d = t_case(wr, N, K, seed=40000 + i)
        x = wr_synth.activations_bf16(50000 + i, M, K)
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        problems.append((dev(x), packed, a_d, s_d, y, N, K))
        refs.append(o.gemm_ternary(x, codes, alpha, signs))
    nb = wr.wr_gemv_ternary_batched_workspace_bytes(M, problems)
    ws = _zeros_ws(nb)
    wr.wr_gemv_ternary_batched(M, problems, ws, nb)
    torch.cuda.synchronize()
    for (_, _, _, _, y, _, _), (ref, B) in zip(problems, refs):
        check_close(y.cpu().numpy(), ref, B)
    assert wr.wr_get_device_error() == 0


# ---------------------------------------------------------------- trellis-coded 2-bit format

def tr_case(wr, N, K, seed):
    W = wr_synth.weights_fp32(seed, N, K)
    sym, sc = wr.wr_quantize_trellis(W)
    sym_o, sc_o = o.quantize_trellis2(W)
    assert np.array_equal(sym, sym_o) and np.array_equal(sc, sc_o.view(np.uint16))
    return sym_o, sc_o, dev(wr.wr_pack(wr.WR_FMT_T2, sym)), dev(sc)


@pytest.mark.parametrize("M", [1, 3, 8])
@pytest.mark.parametrize("N,K", [(40, 512), (129, 768), (300, 2560)])
def test_trellis_gemv(wr, M, N, K):
    """Decode GEMV on the 2-bit trellis-coded format (bits = WR_FMT_T2) against the oracle's
    decode of the same symbols."""
    torch = torch_mod()
    sym, sc, packed, s_d = tr_case(wr, N, K, seed=N + K + M)
    x = wr_synth.activations_bf16(800 + M, M, K)
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    nb = wr.wr_gemv_workspace_bytes(M, N, K, wr.WR_FMT_T2)
    ws = _zeros_ws(nb)
    wr.wr_gemv(M, N, K, dev(x), packed, s_d, wr.WR_FMT_T2, y, ws, nb)
    torch.cuda.synchronize()
    ref, B = o.gemm_trellis2(x, sym, sc)
    check_close(y.cpu().numpy(), ref, B)
    assert wr.wr_get_device_error() == 0


def test_trellis_in_a_mixed_batch(wr):
    """Q2, Q3 and trellis problems in one batched launch."""
    torch = torch_mod()
    M = 4
    problems, refs = [], []
    for i, (N, K, fmt) in enumerate([(64, 512, 4), (100, 768, 2), (40, 256, 3), (200, 2560, 4)]):
        x = wr_synth.activations_bf16(900 + i, M, K)
        if fmt == 4:
            sym, sc, packed, s_d = tr_case(wr, N, K, seed=70 + i)
            refs.append(o.gemm_trellis2(x, sym, sc))
        else:
            codes, scales, packed, s_d = q_case(wr, fmt, N, K, seed=70 + i)
            refs.append(o.gemm_codes(x, codes, scales, fmt))
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        problems.append((dev(x), packed, s_d, y, N, K, fmt))
    nb = wr.wr_gemv_batched_workspace_bytes(M, problems)
    ws = _zeros_ws(nb)
    wr.wr_gemv_batched(M, problems, ws, nb)
    torch.cuda.synchronize()
    for (_, _, _, y, _, _, _), (ref, B) in zip(problems, refs):
        check_close(y.cpu().numpy(), ref, B)


@pytest.mark.parametrize("N,K", [(16, 256), (45, 768)])
def test_trellis_unpack_bf16_bit_exact(wr, N, K):
    torch = torch_mod()
    sym, sc, packed, s_d = tr_case(wr, N, K, seed=3 * N + K)
    out = torch.empty(N, K, dtype=torch.int16, device="cuda")
    wr.wr_unpack_bf16(wr.WR_FMT_T2, N, K, packed, s_d, out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy().view(np.uint16), o.f64_to_bf16_bits(o.dequant_trellis2(sym, sc)))


# ---------------------------------------------------------------- device quantizer + packer

def _edge_weights(N, K, seed):
    """Seeded N(0, 0.02) weights with edge blocks planted: all zeros, ties on the even
    boundaries (w = m s exactly), negative zeros, tiny blocks whose scale underflows to 0 in
    fp16, and huge blocks whose scale overflows to inf."""
    W = wr_synth.weights_fp32(seed, N, K).copy()
    if N >= 6 and K >= 512:
        W[0, 0:256] = 0.0
        s = np.float32(0.125)                     # absmax 3 s -> s exact in fp16 for both grids
        W[1, 0:256] = np.float32(0.0)
        W[1, 0:8] = np.array([3, -3, 2, -2, 0, 1, -1, 2], np.float32) * s
        W[1, 256:512] = np.float32(7.0) * s * np.sign(np.arange(256) - 127.5).astype(np.float32)
        W[1, 256:262] = np.array([4, -4, 6, -6, 2, -2], np.float32) * s
        W[2, 0:256] = np.float32(-0.0)
        W[2, 0] = np.float32(1e-3)
        W[3, 0:256] = np.float32(1e-9)             # absmax / L underflows fp16 -> s = 0
        W[4, 0:256] = np.float32(3e5)              # absmax / L overflows fp16 -> s = inf
        W[5, 256:512] *= np.float32(1e-4)
    return W


@pytest.mark.filterwarnings("ignore:overflow encountered in cast")   # the planted fp16 overflow
@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("N,K", [(16, 256), (37, 768), (130, 2560), (6, 512)])
def test_quantize_pack_bit_exact(wr, bits, N, K):
    """wr_quantize_pack on the GPU gives the oracle's codes and scales, packed, byte for byte,
    and the same bytes as the host quantizer and packer."""
    torch = torch_mod()
    W = _edge_weights(N, K, seed=60 + N + bits)
    pk = torch.zeros(wr.wr_packed_bytes(bits, N, K), dtype=torch.uint8, device="cuda")
    sc = torch.zeros(N * (K // 256), dtype=torch.int16, device="cuda")
    wr.wr_quantize_pack(bits, N, K, dev(W), pk, sc)
    torch.cuda.synchronize()
    codes_o, s_o = o.quantize_odd_grid(W, bits)
    assert np.array_equal(sc.cpu().numpy().view(np.uint16).reshape(N, K // 256), s_o.view(np.uint16))
    assert np.array_equal(pk.cpu().numpy(), o.pack(bits, codes_o))
    codes_h, s_h = wr.wr_quantize(bits, W)
    assert np.array_equal(pk.cpu().numpy(), wr.wr_pack(bits, codes_h))
    assert wr.wr_get_device_error() == 0


# ---------------------------------------------------------------- batched ternary decode GEMV

@pytest.mark.parametrize("M", [1, 6])
def test_ternary_gemv_batched_layer_and_ragged(wr, M):
    """The 7 Qwen3-4B layer shapes plus ragged ones, ternary, in one batched call, twice."""
    torch = torch_mod()
    shapes = [(N, K) for (_, K, N, _) in wr_synth.QWEN3_4B_LAYER] + [(40, 640), (300, 128), (17, 384)]
    cases, problems = [], []
    for i, (N, K) in enumerate(shapes):
        codes, alpha, signs, packed, a_d, s_d = t_case(wr, N, K, seed=2000 + i)
        x = wr_synth.activations_bf16(2100 + i, M, K)
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        cases.append((codes, alpha, signs, x, y))
        problems.append((dev(x), packed, a_d, s_d, y, N, K))
    nb = wr.wr_gemv_ternary_batched_workspace_bytes(M, problems)
    assert nb > 0
    ws = _zeros_ws(nb)
    for rep in range(2):
        for *_, y in cases:
            y.fill_(float("nan"))
        wr.wr_gemv_ternary_batched(M, problems, ws, nb)
        torch.cuda.synchronize()
        for codes, alpha, signs, x, y in cases:
            ref, B = o.gemm_ternary(x, codes, alpha, signs)
            check_close(y.cpu().numpy(), ref, B)
    assert wr.wr_get_device_error() == 0


# ---------------------------------------------------------------- small-M prefill on the decode kernel

@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("M", [9, 12, 16, 17, 24, 32])
def test_decode_kernel_up_to_32_tokens(wr, bits, M):
    """wr_gemv and wr_gemm at 9 <= M <= 32 run the integer decode kernel with 64 or 128 MMA
    columns; ragged N and several K blocks, against the oracle, both entry points."""
    torch = torch_mod()
    N, K = 300, 1280
    codes, scales, packed, s_d = q_case(wr, bits, N, K, seed=3000 + M + bits)
    x = wr_synth.activations_bf16(3100 + M, M, K)
    ref, B = o.gemm_codes(x, codes, scales, bits)
    y, _ = _run_gemv(wr, bits, x, packed, s_d, N, K)
    check_close(y, ref, B)
    check_close(_run_gemm(wr, bits, x, packed, s_d, N, K), ref, B)


@pytest.mark.parametrize("bits,N,K,M", [(2, 9728, 2560, 16), (3, 2560, 9728, 32), (3, 9728, 2560, 24)])
def test_decode_kernel_layer_shapes_small_prefill(wr, bits, N, K, M):
    codes, scales, packed, s_d = q_case(wr, bits, N, K, seed=3200 + M)
    x = wr_synth.activations_bf16(3300 + M, M, K)
    ref, B = o.gemm_codes(x, codes, scales, bits)
    check_close(_run_gemm(wr, bits, x, packed, s_d, N, K), ref, B)


def test_batched_at_16_tokens(wr):
    torch = torch_mod()
    M = 16
    problems, refs = [], []
    for i, (N, K, bits) in enumerate([(64, 512, 2), (200, 2560, 3), (40, 256, 2), (1024, 2560, 3)]):
        codes, scales, packed, s_d = q_case(wr, bits, N, K, seed=3400 + i)
        x = wr_synth.activations_bf16(3410 + i, M, K)
        refs.append(o.gemm_codes(x, codes, scales, bits))
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        problems.append((dev(x), packed, s_d, y, N, K, bits))
    nb = wr.wr_gemv_batched_workspace_bytes(M, problems)
    ws = _zeros_ws(nb)
    for _ in range(2):
        wr.wr_gemv_batched(M, problems, ws, nb)
        torch.cuda.synchronize()
        for p, (ref, B) in zip(problems, refs):
            check_close(p[3].cpu().numpy(), ref, B)


@pytest.mark.parametrize("M", [24, 32])
def test_batched_32_token_form_with_one_accumulator(wr, M):
    """A batch of at least 8 blocks per CTA at 17..32 tokens runs the 128-column form with one
    accumulator at two CTAs per SM (the plan's grid shows which form runs); all of y against the
    oracle, twice on one workspace."""
    torch = torch_mod()
    shapes = [(9728, 2560, 2), (9728, 2560, 3), (2560, 9728, 3), (4096, 2560, 2)]
    problems, refs = [], []
    for i, (N, K, bits) in enumerate(shapes):
        codes, scales, packed, s_d = q_case(wr, bits, N, K, seed=3500 + i)
        x = wr_synth.activations_bf16(3510 + i + M, M, K)
        refs.append(o.gemm_codes(x, codes, scales, bits))
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        problems.append((dev(x), packed, s_d, y, N, K, bits))
    G, _, _ = wr.wr_gemv_batched_plan(M, problems)
    assert G == 296
    nb = wr.wr_gemv_batched_workspace_bytes(M, problems)
    ws = _zeros_ws(nb)
    for _ in range(2):
        wr.wr_gemv_batched(M, problems, ws, nb)
        torch.cuda.synchronize()
        for p, (ref, B) in zip(problems, refs):
            check_close(p[3].cpu().numpy(), ref, B)
    assert wr.wr_get_device_error() == 0


def test_single_32_token_call_keeps_two_accumulators(wr):
    """A single linear at 32 tokens has too few blocks for the one-accumulator form: one CTA per
    SM (grid at most 148)."""
    probs = [(None, None, None, None, 9728, 2560, 2)]
    G, _, _ = wr.wr_gemv_batched_plan(32, probs)
    assert G <= 148


def test_batched_32_token_form_with_one_accumulator_all_formats(wr):
    """The same one-accumulator form in the kernel build that also decodes trellis codes and int8
    block scales: a batch of random codes in every 2-bit and 3-bit format, large enough for two
    CTAs per SM at M = 24, all of y against the oracle."""
    from gpu_inputs import s8_record
    torch = torch_mod()
    M = 24
    rng = np.random.default_rng(3600)
    spec = [(9728, 2560, "q3i8"), (9728, 2560, "q2"), (2560, 9728, "q3"), (1024, 2560, "q2i8"),
            (256, 1024, "t8"), (512, 2560, "t2")]
    problems, refs = [], []
    for i, (N, K, kind) in enumerate(spec):
        x = wr_synth.activations_bf16(3610 + i, M, K)
        bits = 3 if kind.startswith("q3") else 2
        codes = rng.integers(0, 1 << bits, (N, K)).astype(np.uint8)
        if kind.endswith("i8"):
            d = (np.float16(0.01) * (1 + rng.random(N))).astype(np.float16)
            q = rng.integers(0, 128, (N, K // 256)).astype(np.int8)
            fmt, s_d = bits | wr.WR_SCALES_I8, dev(s8_record(d, q))
            ref = o.gemm_codes_s8(x, codes, d, q, bits)
        else:
            sc = (np.float16(0.01) * (1 + rng.random((N, K // 256)))).astype(np.float16)
            s_d = dev(sc.view(np.uint16))
            if kind == "t8":
                fmt, ref = wr.WR_FMT_T8, o.gemm_trellis8(x, codes, sc)
            elif kind == "t2":
                fmt, ref = wr.WR_FMT_T2, o.gemm_trellis2(x, codes, sc)
            else:
                fmt, ref = bits, o.gemm_codes(x, codes, sc, bits)
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        problems.append((dev(x), dev(wr.wr_pack(fmt & 0xFF, codes)), s_d, y, N, K, fmt))
        refs.append(ref)
    G, _, _ = wr.wr_gemv_batched_plan(M, problems)
    assert G == 296
    nb = wr.wr_gemv_batched_workspace_bytes(M, problems)
    ws = _zeros_ws(nb)
    wr.wr_gemv_batched(M, problems, ws, nb)
    torch.cuda.synchronize()
    for p, (r, B) in zip(problems, refs):
        check_close(p[3].cpu().numpy(), r, B)
    assert wr.wr_get_device_error() == 0
