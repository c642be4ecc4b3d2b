"""Oracle for the packed-code weight-only GEMM: a plain, slow, fp64 CPU definition.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import or run
anything in this package. The library (``libwr.so`` and its Python binding)
never calls it, and this file imports nothing from the library.

What it defines (citations are to the source pages by title and section):

* Weights live on a signed odd grid: with b bits, code c in [0, 2^b) stands for
  the level g = 2c - (2^b - 1), e.g. {-3, -1, 1, 3} at 2 bits
  ("How We Shrank an AI Model by 85%...", "Why 2 bits is hard"), and
  W = s * g with one fp16 scale s per 256 weights along K ("Qwen3-4B-Wringer-Q2.6",
  "What is in this repo": packed codes + fp16 block scales).
* Synthetic quantization: scale s = fp16(absmax / L), projected to fp16 before the
  codes are chosen ("Agents-A1-4B-Wringer-Q2.6", "Honest caveats": the solver
  projects scales to fp16 at solve time), then nearest-point codes
  ("Qwen3-4B-Wringer-Q2.6", "Recipe": nearest-point rounding onto the grid).
* Ternary W1.58A16 ({-1, 0, +1}, per-row fp16 scale) in a basis rotated by a
  block-128 random-sign Hadamard R: W x = (W R^T)(R x)
  ("How We Shrank...", "Trick 1: rotate the weights first"; the Qwen3-4B
  ternarization article for W1.58A16).
* A 2-bit trellis-coded format ("How We Shrank...", "Trick 3: trellis coding"): the
  encoder carries a state from one weight to the next, the state picks a coset of the
  levels, the written bits pick a value inside it and set the next state, and a Viterbi
  search finds the cheapest path. The pages give the 2-state, 1-bit toy in full; the
  format here is its 2-bit form: 8 odd levels, state = low bit of the previous symbol.
* Two-level int8 block scales ("Agents-A1-4B-Wringer-Q2.6", "What is in this repo":
  packed codes with fp16 or int8 block scales): s[n, b] = d_n q[n, b], an fp16 scale per
  row times an int8 multiplier 0..127 per 256-block.
* The contraction y[m, n] = sum_k W[n, k] x[m, k] in fp64, and the bound
  B[m, n] = sum_k |W[n, k] x[m, k]| used for the per-element tolerance.
* The packed byte layout (defined in ``include/wr.h``), re-implemented here from
  its written specification through explicit per-code index arithmetic.

Where the pages are silent, the plainest reading is taken; each reading that changes
numbers is stated next to the code below.
"""
from __future__ import annotations

import numpy as np

BLOCK = 256          # weights per fp16 scale along K
HBLOCK = 128         # Hadamard block length of the ternary rotation
TERNARY_UNIT = 320   # trits per 16-row tile unit along K (4 lanes x 80 trits)
TILE_ROWS = 16

FMT_TERNARY = 1
FMT_Q2 = 2
FMT_Q3 = 3
FMT_T2 = 4   # 2-bit trellis-coded: 2-bit symbols in the Q2 layout, 8 odd levels
FMT_T8 = 5   # 8-state trellis over 4-weight symbols: 2-bit codes in the Q2 layout, 8 odd levels


# --------------------------------------------------------------------------------------
# Grid and scalar conversions
# --------------------------------------------------------------------------------------

def grid_L(bits: int) -> int:
    """Largest level of the b-bit odd grid, L = 2^b - 1 (3 at 2 bits, 7 at 3 bits)."""
    return (1 << bits) - 1


def code_to_level(codes: np.ndarray, bits: int) -> np.ndarray:
    """g = 2c - L: code 0 is the most negative level ("Why 2 bits is hard": {-3,-1,1,3})."""
    return 2 * np.asarray(codes, dtype=np.int64) - grid_L(bits)


def fp16_round(a: np.ndarray) -> np.ndarray:
    """Round fp64 values to fp16 once (numpy converts float64 -> float16 directly, RNE)."""
    return np.asarray(a, dtype=np.float64).astype(np.float16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns: the 16 bits are the top half of an fp32."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def f64_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp64 to bf16 (nearest, ties to even) and return the uint16 patterns.

    Used only for values that are exact in fp32 (s * g has at most 11 + 3 significant
    bits), so narrowing to fp32 first is exact and a single RNE step to bf16 follows."""
    f = np.asarray(a, dtype=np.float64).astype(np.float32)
    assert np.array_equal(f.astype(np.float64), np.asarray(a, dtype=np.float64)), \
        "value not exact in fp32"
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return r.astype(np.uint16)


# --------------------------------------------------------------------------------------
# Synthetic quantizers (data generation; not on the timed path)
# --------------------------------------------------------------------------------------

def quantize_odd_grid(W: np.ndarray, bits: int):
    """Nearest-point codes on the b-bit odd grid with fp16 absmax block scales.

    Per 256-weight block along K: s = fp16(absmax / L) (the division in fp64, one
    rounding to fp16); q = w / s in fp64; g = clamp(2*floor(q/2) + 1, -L, L), the
    nearest odd level (an exact even q goes up); s == 0 gives g = +1.
    Returns (codes uint8 [N, K], scales float16 [N, K/256])."""
    W = np.asarray(W, dtype=np.float32)
    N, K = W.shape
    assert K % BLOCK == 0
    L = grid_L(bits)
    Wb = W.astype(np.float64).reshape(N, K // BLOCK, BLOCK)
    absmax = np.abs(Wb).max(axis=2)
    s16 = fp16_round(absmax / L)
    s = s16.astype(np.float64)[:, :, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.where(s > 0, Wb / np.where(s > 0, s, 1.0), 0.0)
    g = 2.0 * np.floor(q / 2.0) + 1.0
    g = np.clip(g, -L, L).astype(np.int64)
    codes = ((g + L) // 2).astype(np.uint8).reshape(N, K)
    return codes, s16


S8_QMAX = 127   # int8 block multipliers of the two-level scales take the values 0..127


def quantize_odd_grid_s8(W: np.ndarray, bits: int):
    """Nearest-point codes on the b-bit odd grid with int8 block scales.

    The "Agents-A1-4B-Wringer-Q2.6" card ("What is in this repo") lists a container of
    packed codes with fp16 or int8 block scales and says no more about the int8 form.
    Reading: an int8 block scale is a multiplier of a wider per-row scale. Per row n:
    A_n = max_k |w[n, k]|; d_n = fp16(A_n / (127 L)) (fp64 division, one rounding,
    saturated to the largest finite fp16). Per 256-block b with absmax a_b:
    q[n, b] = the integer nearest to a_b / (L d_n) (ties to even), clamped to [0, 127]
    (0 when d_n = 0). The block scale is s[n, b] = d_n q[n, b] (exact in fp32: at most
    11 + 7 significant bits), and the codes are the nearest odd levels of w / s exactly
    as in quantize_odd_grid (an exact even quotient goes up, s == 0 gives g = +1).
    Returns (codes uint8 [N, K], d float16 [N], q int8 [N, K/256])."""
    W = np.asarray(W, dtype=np.float32)
    N, K = W.shape
    assert K % BLOCK == 0
    L = grid_L(bits)
    Wb = W.astype(np.float64).reshape(N, K // BLOCK, BLOCK)
    absmax = np.abs(Wb).max(axis=2)                      # a_b * L, per block
    A = absmax.max(axis=1)                               # row absmax
    with np.errstate(over="ignore"):
        d16 = fp16_round(A / (S8_QMAX * L))
    d16 = np.minimum(d16, np.float16(np.finfo(np.float16).max))
    d = d16.astype(np.float64)[:, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        qf = np.where(d > 0, np.rint(absmax / (L * np.where(d > 0, d, 1.0))), 0.0)
    q = np.clip(qf, 0, S8_QMAX).astype(np.int8)
    s = (d * q.astype(np.float64))[:, :, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.where(s > 0, Wb / np.where(s > 0, s, 1.0), 0.0)
    g = 2.0 * np.floor(r / 2.0) + 1.0
    g = np.clip(g, -L, L).astype(np.int64)
    codes = ((g + L) // 2).astype(np.uint8).reshape(N, K)
    return codes, d16, q


def s8_block_scales(d: np.ndarray, q: np.ndarray) -> np.ndarray:
    """s[n, b] = d_n * q[n, b] in fp64 (exact)."""
    return np.asarray(d, dtype=np.float16).astype(np.float64)[:, None] * np.asarray(q, dtype=np.int64)


# --------------------------------------------------------------------------------------
# Trellis coding ("How We Shrank...", "Trick 3: trellis coding")
# --------------------------------------------------------------------------------------
#
# The toy on that page: four levels in two cosets, state 0 may use {-1.5, 0.5} and state 1
# {-0.5, 1.5}; bit 0 picks the lower value, bit 1 the higher, and the bit written becomes the
# next state. In general form, with `values` the 2^(k+1) levels in ascending order and k bits
# written per weight: state s may use values[2u + s] for u in [0, 2^k), and the next state is
# the low bit of u. At k = 1 this is the toy exactly. The 2-bit format below is k = 2 over the
# 8 odd levels {-7, ..., 7} * s, with the state reset to 0 at the start of every 256-block so
# that blocks decode on their own. (Reading: the pages also name an 8-state set-partitioned
# trellis over 4-weight symbols but give no tables for it; the 2-state scalar trellis is the
# one they specify completely.)

def trellis_level_index(symbols: np.ndarray, state0: int = 0) -> np.ndarray:
    """Level index 2 u_i + state_i of each step (last axis), state_{i+1} = u_i & 1."""
    u = np.asarray(symbols, dtype=np.int64)
    state = np.empty_like(u)
    state[..., 0] = state0
    state[..., 1:] = u[..., :-1] & 1
    return 2 * u + state


def trellis_greedy(targets, values, k: int, state0: int = 0):
    """Greedy encoding: at each step the nearest value the current state allows (a tie takes
    the lower symbol). Returns (symbols, squared error)."""
    values = np.asarray(values, dtype=np.float64)
    state, out, err = state0, [], 0.0
    for t in np.asarray(targets, dtype=np.float64):
        cand = [(float(t - values[2 * u + state]) ** 2, u) for u in range(1 << k)]
        e, u = min(cand)
        out.append(u)
        err += e
        state = u & 1
    return np.array(out, dtype=np.int64), err


def trellis_viterbi(targets: np.ndarray, values: np.ndarray, k: int, state0: int = 0):
    """Minimum squared-error path (the Viterbi algorithm: for every state, the cheapest path
    ending there). targets [..., n] (several independent sequences along the leading axes),
    values [..., 2^(k+1)] ascending (broadcast against the leading axes). Ties go to the
    lower (state, symbol) pair and, at the end, the lower final state.
    Returns (symbols int64 [..., n], cost float64 [...])."""
    t = np.asarray(targets, dtype=np.float64)
    v = np.asarray(values, dtype=np.float64)
    lead, n = t.shape[:-1], t.shape[-1]
    v = np.broadcast_to(v, lead + v.shape[-1:])
    U = 1 << k
    inf = np.inf
    cost = np.full(lead + (2,), inf)
    cost[..., state0] = 0.0
    back_s = np.zeros(lead + (n, 2), dtype=np.int64)
    back_u = np.zeros(lead + (n, 2), dtype=np.int64)
    for i in range(n):
        ti = t[..., i]
        new = np.full(lead + (2,), inf)
        bs = np.zeros(lead + (2,), dtype=np.int64)
        bu = np.zeros(lead + (2,), dtype=np.int64)
        for s in range(2):
            for u in range(U):
                d = ti - v[..., 2 * u + s]
                c = cost[..., s] + d * d
                nxt = u & 1
                better = c < new[..., nxt]
                new[..., nxt] = np.where(better, c, new[..., nxt])
                bs[..., nxt] = np.where(better, s, bs[..., nxt])
                bu[..., nxt] = np.where(better, u, bu[..., nxt])
        cost = new
        back_s[..., i, :] = bs
        back_u[..., i, :] = bu
    final = np.argmin(cost, axis=-1)
    best = np.take_along_axis(cost, final[..., None], axis=-1)[..., 0]
    sym = np.zeros(lead + (n,), dtype=np.int64)
    st = final
    for i in range(n - 1, -1, -1):
        sym[..., i] = np.take_along_axis(back_u[..., i, :], st[..., None], axis=-1)[..., 0]
        st = np.take_along_axis(back_s[..., i, :], st[..., None], axis=-1)[..., 0]
    return sym, best


def quantize_trellis2(W: np.ndarray):
    """The 2-bit trellis-coded format: per 256-block, s = fp16(absmax / 7) (fp64 division,
    one rounding), levels s * {-7, -5, ..., 7}, symbols u in [0, 4) by the Viterbi search
    (state 0 at the block start), so the level index is c3 = 2 u + state and the weight
    s * (2 c3 - 7). Returns (symbols uint8 [N, K], scales float16 [N, K/256])."""
    W = np.asarray(W, dtype=np.float32)
    N, K = W.shape
    assert K % BLOCK == 0
    Wb = W.astype(np.float64).reshape(N, K // BLOCK, BLOCK)
    s16 = fp16_round(np.abs(Wb).max(axis=2) / 7.0)
    levels = np.arange(-7, 8, 2, dtype=np.float64)
    vals = s16.astype(np.float64)[:, :, None] * levels
    sym, _ = trellis_viterbi(Wb, vals, 2)
    return sym.reshape(N, K).astype(np.uint8), s16


def dequant_trellis2(symbols: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """W = s * (2 c3 - 7) with c3 = 2 u + state, the state restarting at every 256-block."""
    u = np.asarray(symbols, dtype=np.int64)
    N, K = u.shape
    c3 = trellis_level_index(u.reshape(N, K // BLOCK, BLOCK)).reshape(N, K)
    s = np.repeat(np.asarray(scales, dtype=np.float64), BLOCK, axis=1)
    return s * (2 * c3 - 7).astype(np.float64)


def gemm_trellis2(x_bits, symbols, scales):
    return gemm(x_bits, dequant_trellis2(symbols, scales))


def rotate(v: np.ndarray, sign_words: np.ndarray) -> np.ndarray:
    """Apply R = blockdiag((1/sqrt(128)) * H_128 * D_b) to the last axis, in fp64.

    H_128 is the Sylvester Hadamard matrix in natural order (the 4x4 example of
    "Trick 1: rotate the weights first" is H_4 / 2); D_b = diag(d) over the block,
    d_k = -1 where bit k of the sign mask is set. Written as a plain matrix product."""
    v = np.asarray(v, dtype=np.float64)
    K = v.shape[-1]
    assert K % HBLOCK == 0
    d = sign_vector(sign_words, K)
    H = hadamard(HBLOCK)
    vb = (v * d).reshape(v.shape[:-1] + (K // HBLOCK, HBLOCK))
    out = np.matmul(vb, H.T) / np.sqrt(HBLOCK)
    return out.reshape(v.shape)


def quantize_ternary(W: np.ndarray, sign_words: np.ndarray):
    """Ternary codes in the rotated basis, with a per-row fp16 scale.

    W' = W R^T (row n of W' is R applied to row n of W), in fp64.
    Delta_n = 0.7 * mean_k |W'[n, k]|; t = sign(W') where |W'| > Delta_n, else 0.
    alpha_n = fp16(mean of |W'[n, k]| over t != 0), the least-squares scale for fixed t
    (0 for a row with no nonzero t). Codes are c = t + 1.
    Returns (codes uint8 [N, K], alpha float16 [N], W' float64 [N, K])."""
    W = np.asarray(W, dtype=np.float32).astype(np.float64)
    Wr = rotate(W, sign_words)
    a = np.abs(Wr)
    delta = 0.7 * a.mean(axis=1, keepdims=True)
    keep = a > delta
    t = np.where(keep, np.sign(Wr), 0.0).astype(np.int64)
    cnt = keep.sum(axis=1)
    tot = np.where(keep, a, 0.0).sum(axis=1)
    alpha = fp16_round(np.where(cnt > 0, tot / np.maximum(cnt, 1), 0.0))
    return (t + 1).astype(np.uint8), alpha, Wr


# --------------------------------------------------------------------------------------
# Dequantization and contraction (the definition the GPU path must reproduce)
# --------------------------------------------------------------------------------------

def dequant(codes: np.ndarray, scales: np.ndarray, bits: int) -> np.ndarray:
    """W[n, k] = s[n, k // 256] * g(c[n, k]) in fp64."""
    codes = np.asarray(codes)
    N, K = codes.shape
    g = code_to_level(codes, bits).astype(np.float64)
    s = np.asarray(scales, dtype=np.float16).astype(np.float64)
    return (g.reshape(N, K // BLOCK, BLOCK) * s[:, :, None]).reshape(N, K)


def dequant_s8(codes: np.ndarray, d: np.ndarray, q: np.ndarray, bits: int) -> np.ndarray:
    """W[n, k] = d_n q[n, k // 256] g(c[n, k]) in fp64 (two-level scales)."""
    codes = np.asarray(codes)
    N, K = codes.shape
    g = code_to_level(codes, bits).astype(np.float64)
    s = s8_block_scales(d, q)
    return (g.reshape(N, K // BLOCK, BLOCK) * s[:, :, None]).reshape(N, K)


def dequant_trellis2_s8(symbols: np.ndarray, d: np.ndarray, q: np.ndarray) -> np.ndarray:
    """The trellis format with two-level scales: W = d_n q[n, b] (2 c3 - 7)."""
    symbols = np.asarray(symbols)
    N, K = symbols.shape
    c3 = trellis_level_index(symbols.reshape(N * (K // BLOCK), BLOCK)).reshape(N, K)
    g = code_to_level(c3, 3).astype(np.float64)
    return (g.reshape(N, K // BLOCK, BLOCK) * s8_block_scales(d, q)[:, :, None]).reshape(N, K)


def unpack_bf16_s8(codes: np.ndarray, d: np.ndarray, q: np.ndarray, bits: int) -> np.ndarray:
    """The bf16 materialization with two-level scales: bf16_RNE(d q g), one rounding."""
    return f64_to_bf16_bits(dequant_s8(codes, d, q, bits))


def gemm_codes_s8(x_bits, codes, d, q, bits):
    """y[m, n] = sum_b d_n q[n, b] sum_{k in b} g[n, k] x[m, k]."""
    return gemm(x_bits, dequant_s8(codes, d, q, bits))


def dequant_ternary(codes: np.ndarray, alpha: np.ndarray) -> np.ndarray:
    """W'[n, k] = alpha_n * (c[n, k] - 1) in fp64 (rotated basis)."""
    t = np.asarray(codes, dtype=np.int64) - 1
    return np.asarray(alpha, dtype=np.float16).astype(np.float64)[:, None] * t


def unpack_bf16(codes: np.ndarray, scales: np.ndarray, bits: int) -> np.ndarray:
    """The bf16 materialization: bf16_RNE(s * g), as uint16 bit patterns [N, K]."""
    return f64_to_bf16_bits(dequant(codes, scales, bits))


def unpack_bf16_ternary(codes: np.ndarray, alpha: np.ndarray) -> np.ndarray:
    return f64_to_bf16_bits(dequant_ternary(codes, alpha))


def gemm(x_bits: np.ndarray, W: np.ndarray):
    """y = x W^T and B = |x| |W|^T in fp64; x given as bf16 bits [M, K], W fp64 [N, K]."""
    x = bf16_bits_to_f64(x_bits)
    W = np.asarray(W, dtype=np.float64)
    return x @ W.T, np.abs(x) @ np.abs(W).T


def gemm_codes(x_bits, codes, scales, bits):
    """The packed-code GEMM/GEMV: y[m, n] = sum_b s[n, b] sum_{k in b} g[n, k] x[m, k]."""
    return gemm(x_bits, dequant(codes, scales, bits))


def gemm_ternary(x_bits, codes, alpha, sign_words):
    """Ternary GEMM: y = alpha_n * sum_k t[n, k] (R x)[m, k], with R x in fp64.
    The bound uses w' = alpha * t and x' = R x."""
    xr = rotate(bf16_bits_to_f64(x_bits), sign_words)
    Wt = dequant_ternary(codes, alpha)
    return xr @ Wt.T, np.abs(xr) @ np.abs(Wt).T


# --------------------------------------------------------------------------------------
# The 8-state trellis over 4-weight symbols ("How We Shrank...", "Trick 3: trellis coding")
# --------------------------------------------------------------------------------------
#
# The page names an 8-state set-partitioned trellis over symbols of 4 weights at about 2 bits
# per weight, without tables. Reading taken here (the plainest one that keeps the toy's
# mechanism): the signal set is the 4-vectors of level indices c in [0, 8) on the 8 odd levels
# {-7..7} * s whose parities sum to an even number (a checkerboard set), partitioned by parity
# pattern into 8 cosets of 256 points. State s = (s0, s1, s2) selects the coset whose parity
# pattern is p = (s0, s1, s2, s0 ^ s1 ^ s2); the 8 written bits, four 2-bit codes u_i, pick the
# point c_i = 2 u_i + p_i; and, as in the toy, a written bit sets the next state: the low bit of
# u_3 shifts into the state, s' = ((s << 1) | (u_3 & 1)) & 7. The state restarts at 0 at every
# 256-block. Storage: the codes u are packed exactly like 2-bit codes (2 bits per weight).

def trellis8_parity(state: int):
    """Parity pattern (p_0, p_1, p_2, p_3) of the coset that state s selects."""
    s0, s1, s2 = state & 1, (state >> 1) & 1, (state >> 2) & 1
    return (s0, s1, s2, s0 ^ s1 ^ s2)


def trellis8_next(state: int, u3: int) -> int:
    """The next state: the low bit of the symbol's last code shifted into the state."""
    return ((state << 1) | (int(u3) & 1)) & 7


def trellis8_level_index(codes: np.ndarray, state0: int = 0) -> np.ndarray:
    """Level indices c = 2 u + p of each weight along the last axis (a multiple of 4 long),
    running the state machine from state0 symbol by symbol."""
    u = np.asarray(codes, dtype=np.int64)
    n = u.shape[-1]
    assert n % 4 == 0
    flat = u.reshape(-1, n)
    out = np.empty_like(flat)
    for r in range(flat.shape[0]):
        st = state0
        for j in range(n // 4):
            p = trellis8_parity(st)
            for i in range(4):
                out[r, 4 * j + i] = 2 * flat[r, 4 * j + i] + p[i]
            st = trellis8_next(st, flat[r, 4 * j + 3])
    return out.reshape(u.shape)


def trellis8_viterbi(targets: np.ndarray, values: np.ndarray, state0: int = 0):
    """Minimum squared-error path through the 8-state trellis: targets [..., n] (n a multiple
    of 4; independent sequences along the leading axes), values [..., 8] ascending (the levels
    of index 0..7). For each state and the low bit z of the last code, the branch's symbol is the
    nearest allowed level per weight (u_0..u_2 free, u_3 with u_3 & 1 = z; a tie takes the lower
    code); each new state keeps the cheaper of its two predecessors (a tie keeps the lower one),
    and the path ends in the cheapest state (a tie takes the lower). Returns (codes int64
    [..., n], cost float64 [...])."""
    t = np.asarray(targets, dtype=np.float64)
    v = np.asarray(values, dtype=np.float64)
    lead, n = t.shape[:-1], t.shape[-1]
    assert n % 4 == 0
    v = np.broadcast_to(v, lead + v.shape[-1:])
    nsym = n // 4
    inf = np.inf
    cost = np.full(lead + (8,), inf)
    cost[..., state0] = 0.0
    back_s = np.zeros(lead + (nsym, 8), dtype=np.int64)
    back_u = np.zeros(lead + (nsym, 8, 4), dtype=np.int64)
    for j in range(nsym):
        tj = t[..., 4 * j:4 * j + 4]
        # best code and its error for weight i, parity p, optionally restricted to u & 1 = z
        def best(i, p, z=None):
            us = [u for u in range(4) if z is None or (u & 1) == z]
            be = np.full(lead, inf)
            bu = np.zeros(lead, dtype=np.int64)
            for u in us:
                d = tj[..., i] - v[..., 2 * u + p]
                e = d * d
                better = e < be
                be = np.where(better, e, be)
                bu = np.where(better, u, bu)
            return be, bu
        new = np.full(lead + (8,), inf)
        bs = np.zeros(lead + (8,), dtype=np.int64)
        bu = np.zeros(lead + (8, 4), dtype=np.int64)
        for nxt in range(8):
            z = nxt & 1
            for s in (nxt >> 1, (nxt >> 1) | 4):       # the two predecessors, lower first
                p = trellis8_parity(s)
                e0, u0 = best(0, p[0])
                e1, u1 = best(1, p[1])
                e2, u2 = best(2, p[2])
                e3, u3 = best(3, p[3], z)
                c = cost[..., s] + e0 + e1 + e2 + e3
                better = c < new[..., nxt]
                new[..., nxt] = np.where(better, c, new[..., nxt])
                bs[..., nxt] = np.where(better, s, bs[..., nxt])
                for i, ui in enumerate((u0, u1, u2, u3)):
                    bu[..., nxt, i] = np.where(better, ui, bu[..., nxt, i])
        cost = new
        back_s[..., j, :] = bs
        back_u[..., j, :, :] = bu
    final = np.argmin(cost, axis=-1)
    total = np.take_along_axis(cost, final[..., None], axis=-1)[..., 0]
    codes = np.zeros(lead + (n,), dtype=np.int64)
    st = final
    for j in range(nsym - 1, -1, -1):
        for i in range(4):
            codes[..., 4 * j + i] = np.take_along_axis(back_u[..., j, :, i], st[..., None], axis=-1)[..., 0]
        st = np.take_along_axis(back_s[..., j, :], st[..., None], axis=-1)[..., 0]
    return codes, total


def quantize_trellis8(W: np.ndarray):
    """The 8-state trellis format: per 256-block s = fp16(absmax / 7) (fp64 division, one
    rounding), levels s * {-7, ..., 7}, codes by trellis8_viterbi from state 0.
    Returns (codes uint8 [N, K] in [0, 4), scales float16 [N, K/256])."""
    W = np.asarray(W, dtype=np.float32)
    N, K = W.shape
    assert K % BLOCK == 0
    Wb = W.astype(np.float64).reshape(N, K // BLOCK, BLOCK)
    s16 = fp16_round(np.abs(Wb).max(axis=2) / 7.0)
    levels = np.arange(-7, 8, 2, dtype=np.float64)
    vals = s16.astype(np.float64)[:, :, None] * levels
    codes, _ = trellis8_viterbi(Wb, vals)
    return codes.reshape(N, K).astype(np.uint8), s16


def dequant_trellis8(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """W = s * (2 c - 7) with c the level indices of the 8-state trellis (state 0 at every
    256-block)."""
    u = np.asarray(codes, dtype=np.int64)
    N, K = u.shape
    c = trellis8_level_index(u.reshape(N, K // BLOCK, BLOCK)).reshape(N, K)
    s = np.repeat(np.asarray(scales, dtype=np.float16).astype(np.float64), BLOCK, axis=1)
    return s * (2 * c - 7).astype(np.float64)


def dequant_trellis8_s8(codes: np.ndarray, d: np.ndarray, q: np.ndarray) -> np.ndarray:
    """The 8-state trellis format with two-level scales: W = d_n q[n, b] (2 c - 7)."""
    u = np.asarray(codes, dtype=np.int64)
    N, K = u.shape
    c = trellis8_level_index(u.reshape(N, K // BLOCK, BLOCK)).reshape(N, K)
    g = (2 * c - 7).astype(np.float64)
    return (g.reshape(N, K // BLOCK, BLOCK) * s8_block_scales(d, q)[:, :, None]).reshape(N, K)


def gemm_trellis8(x_bits, codes, scales):
    return gemm(x_bits, dequant_trellis8(codes, scales))


# --------------------------------------------------------------------------------------
# Hadamard / sign helpers
# --------------------------------------------------------------------------------------

def hadamard(n: int) -> np.ndarray:
    """Sylvester Hadamard matrix of order n (a power of two), entries +-1."""
    assert n >= 1 and n & (n - 1) == 0
    H = np.ones((1, 1), dtype=np.float64)
    while H.shape[0] < n:
        H = np.block([[H, H], [H, -H]])
    return H


def sign_vector(sign_words: np.ndarray, K: int) -> np.ndarray:
    """d_k = -1 if bit (k % 32) of word k // 32 is set, else +1."""
    w = np.asarray(sign_words, dtype=np.uint32)
    k = np.arange(K)
    bit = (w[k // 32] >> (k % 32).astype(np.uint32)) & np.uint32(1)
    return np.where(bit == 1, -1.0, 1.0)


# --------------------------------------------------------------------------------------
# Packed layout, re-implemented from the written specification
# --------------------------------------------------------------------------------------
#
# Common frame (2-bit, 3-bit and ternary): rows are grouped in tiles of 16 (the last
# tile padded) and tiles in groups of 8 (the last group may hold fewer); the K axis is
# cut in units (256 codes for Q2/Q3, 320 trits for ternary, the last ternary unit
# padded). Each unit is a contiguous byte block; a group's units are stored block by
# block and, within a block, tile by tile: unit (tile t, block b) has index
# 8*(t//8)*B + b*T_g + t%8, with B units per tile row and T_g = min(8, tiles - 8*(t//8)).
# Inside a unit, "lane"
# l = 4*r0 + q (r0 = 0..7, q = 0..3) owns rows r0 and r0 + 8 of the tile and the
# q-th quarter of the unit's K range; a lane's bytes (row r0's data, then row
# r0+8's) are cut in 16-byte chunks, and chunk c of lane l sits at unit byte
# (32 * c + (l XOR ((l >> 3) & 3))) * 16.

def _unit_geometry(fmt: int):
    if fmt == FMT_Q2:
        return BLOCK, 1024, 16      # k per unit, unit bytes, lane bytes per row
    if fmt == FMT_Q3:
        return BLOCK, 1536, 24
    if fmt == FMT_TERNARY:
        return TERNARY_UNIT, 1024, 16
    raise ValueError(fmt)


def packed_bytes(fmt: int, N: int, K: int) -> int:
    ku, ub, _ = _unit_geometry(fmt)
    tiles = -(-N // TILE_ROWS)
    units = -(-K // ku)
    return tiles * units * ub


def _lane_byte_to_unit_byte(lane: np.ndarray, lane_byte: np.ndarray) -> np.ndarray:
    position = lane ^ ((lane >> 3) & 3)
    return (32 * (lane_byte // 16) + position) * 16 + lane_byte % 16


def _frame(fmt: int, N: int, K: int):
    """Per code (n, k): unit base byte, lane, row half (0: row r0, 1: row r0+8) and
    the index i of the code inside the lane's quarter."""
    ku, ub, _ = _unit_geometry(fmt)
    n = np.arange(N)[:, None]
    k = np.arange(K)[None, :]
    units = -(-K // ku)
    tiles = -(-N // TILE_ROWS)
    tn, r = n // TILE_ROWS, n % TILE_ROWS
    u, kk = k // ku, k % ku
    qlen = ku // 4
    q, i = kk // qlen, kk % qlen
    lane = 4 * (r % 8) + q
    half = r // 8
    grp = tn // 8
    tg = np.minimum(8, tiles - 8 * grp)
    base = (8 * grp * units + u * tg + tn % 8) * ub
    return base, lane, half, i


def code_bit_positions(fmt: int, N: int, K: int):
    """For Q2/Q3: arrays byte[N, K, b], bit[N, K, b] giving where bit j of code (n, k) lives.

    Q2 (one 16-byte chunk per row per lane = 4 little-endian uint32 words w, 64 codes):
    code i of the lane's quarter is in word w = i // 16; with e = i % 16, it sits in
    half h = e % 2 at bits 16*h + 2*(e // 2) .. +1 (even codes in the low half).
    Q3 (24 bytes per row per lane = two 12-byte groups of 3 words, 32 codes each):
    code i is in group i // 32; with e = i % 32: for e < 30, word u = e // 10,
    f = e % 10, half h = f % 2, slot j = f // 2, bits 16*h + 3*j .. +2; for e = 30 + h,
    bit j of the code is bit 16*h + 15 of word j."""
    base, lane, half, i = _frame(fmt, N, K)
    shape = np.broadcast(base, i).shape
    if fmt == FMT_Q2:
        w = i // 16
        e = i % 16
        h = e % 2
        wbit0 = 16 * h + 2 * (e // 2)
        lane_bit0 = half * 16 * 8 + w * 32 + wbit0
        nb = 2
        lane_bits = np.stack([lane_bit0 + j for j in range(nb)], axis=-1)
    elif fmt == FMT_Q3:
        grp = i // 32
        e = i % 32
        u = np.where(e < 30, e // 10, 0)
        f = e % 10
        h = np.where(e < 30, f % 2, e - 30)
        j = f // 2
        gbase = half * 24 * 8 + grp * 12 * 8
        bits = []
        for jb in range(3):
            reg = gbase + u * 32 + 16 * h + 3 * j + jb
            spare = gbase + jb * 32 + 16 * h + 15
            bits.append(np.where(e < 30, reg, spare))
        lane_bits = np.stack(bits, axis=-1)
    else:
        raise ValueError(fmt)
    lane_bits = np.broadcast_to(lane_bits, shape + (lane_bits.shape[-1],))
    lane_b = lane_bits // 8
    byte = np.broadcast_to(base, shape)[..., None] + \
        _lane_byte_to_unit_byte(np.broadcast_to(lane, shape)[..., None], lane_b)
    return byte, lane_bits % 8


def trit_positions(N: int, K: int):
    """Ternary: byte[N, K] and base-3 digit index[N, K] of trit (n, k).

    Each lane quarter is 80 trits in 16 bytes; trit i is digit i % 5 of byte i // 5,
    and the byte value is sum_d c_d * 3^d."""
    base, lane, half, i = _frame(FMT_TERNARY, N, K)
    shape = np.broadcast(base, i).shape
    lane_byte = half * 16 + i // 5
    byte = np.broadcast_to(base, shape) + _lane_byte_to_unit_byte(np.broadcast_to(lane, shape), lane_byte)
    return byte, np.broadcast_to(i % 5, shape)


def pack(fmt: int, codes: np.ndarray) -> np.ndarray:
    """Codes [N, K] -> packed bytes. Pad rows and pad trits: Q2/Q3 pad codes are 0,
    ternary pad trits are 1 (t = 0)."""
    codes = np.asarray(codes, dtype=np.uint8)
    N, K = codes.shape
    out = np.zeros(packed_bytes(fmt, N, K), dtype=np.int64)
    if fmt == FMT_TERNARY:
        ku = TERNARY_UNIT
        Kp = -(-K // ku) * ku
        Np = -(-N // TILE_ROWS) * TILE_ROWS
        full = np.ones((Np, Kp), dtype=np.int64)
        full[:N, :K] = codes
        byte, digit = trit_positions(Np, Kp)
        np.add.at(out, byte.ravel(), (full * (3 ** digit)).ravel())
    else:
        bits = 2 if fmt == FMT_Q2 else 3
        Np = -(-N // TILE_ROWS) * TILE_ROWS
        full = np.zeros((Np, K), dtype=np.int64)
        full[:N] = codes
        byte, bit = code_bit_positions(fmt, Np, K)
        for j in range(bits):
            v = ((full >> j) & 1) << bit[..., j]
            np.add.at(out, byte[..., j].ravel(), v.ravel())
    assert out.max(initial=0) < 256
    return out.astype(np.uint8)


def unpack_codes(fmt: int, packed: np.ndarray, N: int, K: int) -> np.ndarray:
    """Packed bytes -> codes [N, K] (inverse of ``pack`` on the real rows and columns)."""
    p = np.asarray(packed, dtype=np.uint8).astype(np.int64)
    if fmt == FMT_TERNARY:
        byte, digit = trit_positions(N, K)
        return ((p[byte] // (3 ** digit)) % 3).astype(np.uint8)
    bits = 2 if fmt == FMT_Q2 else 3
    byte, bit = code_bit_positions(fmt, N, K)
    c = np.zeros((N, K), dtype=np.int64)
    for j in range(bits):
        c |= ((p[byte[..., j]] >> bit[..., j]) & 1) << j
    return c.astype(np.uint8)
