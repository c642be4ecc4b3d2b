"""Host-side checks of libwr (no GPU): exported symbols, the packer against the oracle's
independent implementation of the layout, the synthetic quantizers against the oracle's,
and argument validation that must return before any device work."""
import json
import os
import re

import numpy as np
import pytest

import bit_weight_only_wr_b200 as wr
import wr_synth
from oracle import wr_oracle as o
from gpu_inputs import s8_record

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    text = open(os.path.join(ROOT, "include", "wr.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(wr_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    declared = _header_functions()
    assert declared == wr.exported_symbols()
    out = os.popen(f"nm -D --defined-only {wr.LIB_PATH}").read()
    exported = set(re.findall(r" T (wr_[a-z0-9_]+)", out))
    missing = [f for f in declared if f not in exported]
    assert not missing, missing
    assert wr.wr_abi_version() == 1
    assert wr.wr_status_string(0) == "ok"


@pytest.mark.parametrize("fmt", [2, 3, 1])
@pytest.mark.parametrize("N,K", [(16, 256), (40, 512), (1, 768), (33, 2560)])
def test_pack_matches_oracle(fmt, N, K):
    if fmt == 1 and K % 128:
        pytest.skip()
    levels = {1: 3, 2: 4, 3: 8}[fmt]
    rng = np.random.default_rng(N * 7 + K + fmt)
    codes = rng.integers(0, levels, (N, K)).astype(np.uint8)
    assert wr.wr_packed_bytes(fmt, N, K) == o.packed_bytes(fmt, N, K)
    mine = wr.wr_pack(fmt, codes)
    ref = o.pack(fmt, codes)
    assert np.array_equal(mine, ref)
    assert np.array_equal(wr.wr_unpack_codes(fmt, mine, N, K), codes)


def test_pack_golden_vectors_through_library(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "pack_vectors.json")))
    for case in g["cases"]:
        codes = np.full((case["N"], case["K"]), case["fill"], dtype=np.uint8)
        for n, k, c in case["set"]:
            codes[n, k] = c
        p = wr.wr_pack(case["fmt"], codes)
        for idx, val in case["expect"].items():
            assert int(p[int(idx)]) == val


def test_pack_rejects_bad_codes_and_shapes():
    with pytest.raises(wr.WrError):
        wr.wr_pack(2, np.full((16, 256), 4, dtype=np.uint8))
    with pytest.raises(wr.WrError):
        wr.wr_pack(1, np.full((16, 256), 3, dtype=np.uint8))
    assert wr.wr_packed_bytes(2, 16, 100) == 0           # K not a multiple of 256
    assert wr.wr_packed_bytes(1, 16, 100) == 1024        # ternary: any K, padded to 320 trits
    assert wr.wr_packed_bytes(7, 16, 256) == 0


@pytest.mark.parametrize("bits", [2, 3])
def test_quantizer_matches_oracle(bits):
    W = wr_synth.weights_fp32(100 + bits, 64, 1024)
    W[3, :256] = 0.0                                      # an all-zero block (s = 0)
    W[5, 300] = 1e-9                                      # tiny values, tiny scale
    c1, s1 = wr.wr_quantize(bits, W)
    c2, s2 = o.quantize_odd_grid(W, bits)
    assert np.array_equal(s1, s2.view(np.uint16))
    assert np.array_equal(c1, c2)


@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("N,K", [(64, 1024), (7, 256), (33, 2560)])
def test_s8_quantizer_matches_oracle(bits, N, K):
    """Int8 block scales: the library's quantizer writes the oracle's d, q and codes, bit for bit."""
    W = wr_synth.weights_fp32(200 + bits + N, N, K)
    W[min(3, N - 1), :256] = 0.0                          # an all-zero block (q = 0)
    if N > 5:
        W[5] *= np.float32(1e-30)                         # d subnormal in fp16 (or zero)
        W[4, 7] = 3.0e9                                   # d saturates at 65504
    fmt = bits | wr.WR_SCALES_I8
    assert wr.wr_scales_bytes(fmt, N, K) == (2 * N + 15) // 16 * 16 + N * (K // 256)
    c1, rec = wr.wr_quantize(fmt, W)
    c2, d, q = o.quantize_odd_grid_s8(W, bits)
    assert np.array_equal(rec[:wr.wr_scales_bytes(fmt, N, K)], s8_record(d, q)[:wr.wr_scales_bytes(fmt, N, K)])
    assert np.array_equal(c1, c2)


def test_scales_bytes():
    assert wr.wr_scales_bytes(2, 16, 512) == 2 * 16 * 2
    assert wr.wr_scales_bytes(3 | wr.WR_SCALES_I8, 16, 512) == 32 + 16 * 2
    assert wr.wr_scales_bytes(wr.WR_FMT_T2 | wr.WR_SCALES_I8, 9, 256) == 32 + 9
    assert wr.wr_scales_bytes(1, 10, 300) == 20                 # ternary alpha [N]
    assert wr.wr_scales_bytes(1 | wr.WR_SCALES_I8, 10, 300) == 0
    assert wr.wr_scales_bytes(2, 16, 100) == 0
    # packed codes do not depend on the scale form: the packer takes the base format
    assert wr.wr_packed_bytes(2 | wr.WR_SCALES_I8, 16, 256) == 0


def test_trellis_quantizer_matches_oracle():
    """The library's Viterbi encoder for the 2-bit trellis format picks the oracle's symbols
    and scales, bit for bit (same fp64 arithmetic, same tie order)."""
    W = wr_synth.weights_fp32(321, 48, 1024)
    W[3, :256] = 0.0                                      # an all-zero block (s = 0)
    W[5, 256:512] *= np.float32(1e-6)                     # a tiny block
    c1, s1 = wr.wr_quantize_trellis(W)
    c2, s2 = o.quantize_trellis2(W)
    assert np.array_equal(s1, s2.view(np.uint16))
    assert np.array_equal(c1, c2)


def test_trellis8_quantizer_matches_oracle():
    """The library's Viterbi encoder for the 8-state trellis format picks the oracle's codes and
    scales, bit for bit (same fp64 arithmetic, same tie order), including all-zero blocks (every
    branch ties) and blocks built from exact level values."""
    W = wr_synth.weights_fp32(322, 24, 1024)
    W[3, :256] = 0.0
    W[5, 256:512] *= np.float32(1e-6)
    W[7, :256] = np.float32(0.25) * np.arange(256, dtype=np.float32) % 3 - 1   # many exact ties
    c1, s1 = wr.wr_quantize_trellis8(W)
    c2, s2 = o.quantize_trellis8(W)
    assert np.array_equal(s1, s2.view(np.uint16))
    assert np.array_equal(c1, c2)


def test_trellis8_word_decoder_matches_the_state_machine():
    """The GEMV's word decoder for the 8-state format, written out here from its definition in
    include/wr.h as host arithmetic on one packed word at a time, is checked against the oracle's
    state machine: every code's level index through the parity-bit positions of the word."""
    rng = np.random.default_rng(9)
    for trial in range(20):
        u = rng.integers(0, 4, 64)
        lvl = o.trellis8_level_index(u)
        # the 4 words of a 64-code quarter, code e of word t at bits 16*(e&1) + 2*(e>>1)
        words = [sum(int(u[16 * t + e]) << (16 * (e & 1) + 2 * (e >> 1)) for e in range(16)) for t in range(4)]
        carry = 0
        for t, w in enumerate(words):
            zl = (w >> 16) & 0x4444
            X = ((zl << 16) | carry) & 0xFFFFFFFF
            carry = zl
            P = (((X >> 14) & 0x1111) | ((X << 6) & 0x11110000) | ((X >> 4) & 0x4444)
                 | (((X << 4) ^ (X << 8) ^ (X << 12)) & 0x44440000))
            for e in range(16):
                pos = 16 * (e & 1) + 2 * (e >> 1)
                c = 2 * ((w >> pos) & 3) + ((P >> pos) & 1)
                assert c == lvl[16 * t + e], (trial, t, e)


@pytest.mark.parametrize("N,K", [(16, 256), (37, 768)])
@pytest.mark.parametrize("fmt", [4, 5])
def test_trellis_format_packs_like_q2(N, K, fmt):
    """WR_FMT_T2 and WR_FMT_T8 store their 2-bit codes in the Q2 layout: same size, same bytes."""
    rng = np.random.default_rng(N + K)
    sym = rng.integers(0, 4, (N, K)).astype(np.uint8)
    assert wr.wr_packed_bytes(fmt, N, K) == wr.wr_packed_bytes(2, N, K)
    p = wr.wr_pack(fmt, sym)
    assert np.array_equal(p, o.pack(o.FMT_Q2, sym))
    assert np.array_equal(wr.wr_unpack_codes(fmt, p, N, K), sym)


def test_ternary_quantizer_matches_oracle():
    K = 1280
    signs = wr_synth.sign_bits(5, K)
    W = wr_synth.weights_fp32(6, 48, K)
    c1, a1 = wr.wr_quantize_ternary(W, signs)
    c2, a2, Wr = o.quantize_ternary(W, signs)
    assert np.array_equal(a1, a2.view(np.uint16))
    diff = c1 != c2
    # the two sides rotate with different summation orders; a code may differ only where
    # |W'| sits on the threshold to within rounding
    if diff.any():
        a = np.abs(Wr)
        delta = 0.7 * a.mean(axis=1, keepdims=True)
        assert np.all(np.abs(a - delta)[diff] < 1e-12 * delta.repeat(K, 1)[diff])
    assert diff.sum() == 0


def test_device_calls_reject_bad_arguments_before_launch():
    # misaligned / null pointers and unsupported configurations return before any CUDA call
    st = wr._lib.wr_gemv(1, 16, 256, 8, 16, 16, 2, 256, 16, 16, 1 << 20, None)
    assert st == 1
    st = wr._lib.wr_gemv(33, 16, 256, 16, 16, 16, 2, 256, 16, 16, 1 << 20, None)   # M > 32
    assert st == 1
    st = wr._lib.wr_gemv(1, 16, 256, 16, 16, 16, 6, 256, 16, 16, 1 << 20, None)   # bits
    assert st == 2
    st = wr._lib.wr_gemm(16, 16, 256, 16, 16, 16, 4, 256, 16, 16, 1 << 20, None)  # trellis, M > 8
    assert st == 2
    st = wr._lib.wr_gemv(1, 16, 256, 16, 16, 16, 2, 128, 16, 16, 1 << 20, None)   # group
    assert st == 2
    st = wr._lib.wr_gemv(1, 16, 300, 16, 16, 16, 2, 256, 16, 16, 1 << 20, None)   # K % 256
    assert st == 1
    st = wr._lib.wr_gemv(1, 16, 256, 16, 16, 16, 2, 256, 16, 16, 0, None)         # workspace
    assert st == 1
    st = wr._lib.wr_gemm(4, 16, 256, 16, 0, 16, 2, 256, 16, 16, 1 << 20, None)    # null packed
    assert st == 1
    st = wr._lib.wr_gemm_ternary(4, 16, 200, 16, 16, 16, 16, 16, 16, 1 << 20, None)  # K % 128
    assert st == 1
    st = wr._lib.wr_unpack_bf16(2, 16, 256, 16, 16, 64, 16, None)                 # group
    assert st == 2
    i8 = wr.WR_SCALES_I8
    st = wr._lib.wr_gemv(1, 16, 256, 16, 16, 16, 6 | i8, 256, 16, 16, 1 << 20, None)   # bits
    assert st == 2
    st = wr._lib.wr_gemm(16, 16, 256, 16, 16, 16, 4 | i8, 256, 16, 16, 1 << 20, None)  # trellis, M > 8
    assert st == 2
    st = wr._lib.wr_gemv(1, 16, 256, 16, 16, 8, 2 | i8, 256, 16, 16, 1 << 20, None)    # misaligned record
    assert st == 1
    st = wr._lib.wr_unpack_bf16(1 | i8, 16, 320, 16, 16, 256, 16, None)           # ternary has no int8 form
    assert st == 2
    st = wr._lib.wr_quantize_pack(wr.WR_FMT_T2 | i8, 16, 256, 16, 16, 16, None)
    assert st == 2
    assert wr.wr_gemv_workspace_bytes(1, 16, 256, 3 | i8) == wr.wr_gemv_workspace_bytes(1, 16, 256, 3)
    assert wr.wr_gemm_workspace_bytes(64, 16, 256, 2 | i8) == wr.wr_gemm_workspace_bytes(64, 16, 256, 2)
    assert wr.wr_gemv_workspace_bytes(33, 16, 256, 2) == 0
    assert wr.wr_gemv_workspace_bytes(1, 16, 256, 2) > 0


def _check_plan(M, shapes):
    """The ranges partition the batch's blocks, none is empty, and each range's cost (in the
    per-problem block costs the library reports) is within one block of C / G."""
    probs = [(None, None, None, None, N, K, fmt) for (N, K, fmt) in shapes]
    G, starts, pcost = wr.wr_gemv_batched_plan(M, probs)
    assert np.all(pcost > 0)
    costs = []
    for (N, K, fmt), c in zip(shapes, pcost):
        costs += [int(c)] * (((N + 127) // 128) * (K // 256))
    T = len(costs)
    assert 1 <= G <= 444 and starts[0] == 0 and starts[G] == T
    assert np.all(np.diff(starts) >= 1), "every CTA range holds at least one block"
    cum = np.concatenate([[0], np.cumsum(costs)])
    rc = cum[starts[1:]] - cum[starts[:-1]]
    C, wmax = cum[-1], max(costs)
    assert np.all(rc <= C / G + wmax) and np.all(rc >= C / G - wmax)
    return G, starts


def test_decode_plan_block_costs_order():
    # a 3-bit or trellis block is the longer one to decode; int8 scales do not change the cost
    probs = [(None, None, None, None, 128, 256, f) for f in (2, 3, wr.WR_FMT_T2, 2 | wr.WR_SCALES_I8)]
    for M in (1, 4, 8):
        _, _, c = wr.wr_gemv_batched_plan(M, probs)
        assert c[1] > c[0] and c[2] == c[1] and c[3] == c[0]


def test_decode_plan_rejects_what_the_batched_call_rejects():
    bad = wr._problems([(16, 16, 16, 16, 16, 256, 2)])
    bad[0].reserved = 1
    with pytest.raises(wr.WrError) as e:
        wr.wr_gemv_batched_plan(1, bad)
    assert e.value.status == 1
    assert wr._lib.wr_gemv_batched(1, 1, bad, 16, 1 << 20, None) == 1
    for fields, status in (((16, 300, 2), 1), ((16, 256, 6), 2), ((0, 256, 2), 1)):
        N, K, fmt = fields
        p = wr._problems([(16, 16, 16, 16, N, K, fmt)])
        with pytest.raises(wr.WrError) as e:
            wr.wr_gemv_batched_plan(1, p)
        assert e.value.status == status
        assert wr._lib.wr_gemv_batched(1, 1, p, 16, 1 << 20, None) != 0


def test_decode_plan_of_the_qwen3_body():
    import wr_synth
    shapes = [(N, K, bits) for _ in range(36) for (_, K, N, bits) in wr_synth.QWEN3_4B_LAYER]
    for M in (1, 3, 8):
        G, _ = _check_plan(M, shapes)
        assert G == 444      # three CTAs per SM of a 148-SM part
    for M in (9, 16, 17, 32):
        G, _ = _check_plan(M, shapes)
        assert G == 296      # the 64- and 128-column forms: two CTAs per SM
    # a lone 17..32-token linear keeps the two-accumulator form at one CTA per SM
    G, _ = _check_plan(32, [(9728, 2560, 2)])
    assert G == 148


def test_decode_plan_switches_the_32_token_form_at_8_blocks_per_cta():
    # 2368 blocks (8 per CTA at two CTAs per SM of 148) take the one-accumulator form, 2367 not
    for M in (17, 32):
        G, _ = _check_plan(M, [(128, 256 * 2368, 2)])
        assert G == 296
        G, _ = _check_plan(M, [(128, 256 * 2367, 2)])
        assert G == 148
    # the 16-token form is two CTAs per SM whatever the batch
    G, _ = _check_plan(16, [(128, 256 * 2367, 2)])
    assert G == 296
    # a small single-format batch runs one block per CTA
    G, starts = _check_plan(1, [(2560, 2560, 2)])
    assert G == 200 and np.array_equal(starts, np.arange(201))


def test_decode_plan_random_batches():
    rng = np.random.default_rng(7)
    fmts = [2, 3, wr.WR_FMT_T2, 2 | wr.WR_SCALES_I8, 3 | wr.WR_SCALES_I8]
    for _ in range(300):
        n = int(rng.integers(1, 24))
        shapes = [(int(rng.integers(1, 3000)), 256 * int(rng.integers(1, 48)), int(rng.choice(fmts)))
                  for _ in range(n)]
        _check_plan(int(rng.integers(1, 9)), shapes)
    with pytest.raises(wr.WrError):
        wr.wr_gemv_batched_plan(33, [(None, None, None, None, 16, 256, 2)])


def test_grouped_argument_checks():
    items = [(16, 16, 16, 16, 2), (16, 16, 16, 1024, 3)]
    assert wr.wr_gemv_grouped_workspace_bytes(1, 512, items) > 0
    assert wr.wr_gemv_grouped_workspace_bytes(1, 300, items) == 0          # K % 256
    assert wr.wr_gemv_grouped_workspace_bytes(33, 512, items) == 0         # M > 32
    assert wr.wr_gemv_grouped_workspace_bytes(1, 512, [(16, 16, 16, 16, 7)]) == 0
    arr = wr._gitems(items)
    arr[1].reserved = 3
    assert wr.wr_gemv_grouped_workspace_bytes(1, 512, arr) == 0
    # misaligned x, and a workspace smaller than asked for, are rejected before any launch
    nb = wr.wr_gemv_grouped_workspace_bytes(1, 512, items)
    assert wr._lib.wr_gemv_grouped(1, 512, 8, 2, wr._gitems(items), 16, nb, None) == 1
    assert wr._lib.wr_gemv_grouped(1, 512, 16, 2, wr._gitems(items), 16, nb - 1, None) == 1


def test_decode_token_limits():
    # the 2/3-bit decode path takes up to 32 tokens (128 MMA columns), the ternary one up to 8;
    # wr_gemm takes any M (the decode kernel up to 32, the tensor-core GEMM above)
    for M in (1, 8, 9, 16, 17, 32):
        assert wr.wr_gemv_workspace_bytes(M, 256, 512, 2) > 0
        # wr_gemm runs the decode kernel (same workspace) for M <= 8, and up to 32 when K <= 4096
        assert wr.wr_gemm_workspace_bytes(M, 256, 512, 3) == wr.wr_gemv_workspace_bytes(M, 256, 512, 3)
        if M > 8:
            assert wr.wr_gemm_workspace_bytes(M, 256, 9728, 3) != wr.wr_gemv_workspace_bytes(M, 256, 9728, 3)
    assert wr.wr_gemv_workspace_bytes(33, 256, 512, 2) == 0
    assert wr.wr_gemm_workspace_bytes(33, 256, 512, 2) > 0
    t = wr._tproblems([(16, 16, 16, 16, 16, 256, 512)])
    assert wr.wr_gemv_ternary_batched_workspace_bytes(8, t) > 0
    assert wr.wr_gemv_ternary_batched_workspace_bytes(9, t) == 0
