/*
 * wr.h -- C ABI of libwr: packed low-bit weight-only GEMV/GEMM for B200 (sm_100a).
 *
 * What is computed
 * ----------------
 * Weights are stored as integer codes on a signed odd grid with one fp16 scale per
 * 256 weights along K:  W[n,k] = s[n, k/256] * g(c[n,k]),  g(c) = 2c - (2^b - 1),
 * i.e. {-3,-1,1,3} at b = 2 and {-7,-5,...,5,7} at b = 3.  The 2-bit grid and the
 * reason it has no zero level are the worked example in "How We Shrank an AI Model by
 * 85% and Kept 90% of Its Smarts" (section "Why 2 bits is hard"); the container of
 * "packed codes + fp16 block scales" is described on the "Qwen3-4B-Wringer-Q2.6" model
 * card ("What is in this repo"), which also states that no kernel consumes it.
 *
 * The ternary format (W1.58A16, the Qwen3-4B post-training ternarization article) stores
 * t in {-1,0,+1} as c = t + 1, five trits per byte, with one fp16 scale alpha per row, in
 * a basis rotated along K by R = blockdiag((1/sqrt(128)) H_128 D): W x = (W R^T)(R x)
 * ("How We Shrank...", "Trick 1: rotate the weights first"). H_128 is the Sylvester
 * Hadamard matrix in natural order, D = diag(d), d_k = -1 where bit k%32 of word k/32 of
 * the sign mask is set. The library applies R to x inside the call.
 *
 * Every GEMV/GEMM computes, for m < M and n < N,
 *     y[m,n] = sum_b s[n,b] * sum_{k in block b} g[n,k] * x[m,k]          (Q2, Q3)
 *     y[m,n] = alpha[n] * sum_k t[n,k] * (R x[m,:])[k]                      (ternary)
 * with x bf16 [M,K] row-major and y fp32 [M,N] row-major (overwritten). Products of the
 * exact grid integers and x are formed exactly and accumulated in fp32; each 256-block
 * partial is multiplied by its scale in fp32. R x is kept in fp32 (split into two bf16
 * terms where tensor cores consume it).
 *
 * Packed layout (shared by every kernel; the bytes are what wr_pack writes)
 * -------------------------------------------------------------------------
 * Rows are grouped in tiles of 16 (the last tile padded) and tiles in groups of 8 (the last
 * group may hold fewer). K is cut in units: 256 codes for Q2/Q3 (K must be a multiple of 256),
 * 320 trits for ternary (any K, the last unit padded; the ternary GEMM needs K to be a multiple
 * of 128 for the rotation). A unit is UB contiguous bytes: UB = 1024 (Q2), 1536 (Q3), 1024
 * (ternary). A group's units are stored block by block and, within a block, tile by tile:
 * unit (tile t, block b) is number 8*(t/8)*B + b*Tg + t%8, with B units per row of tiles and
 * Tg = min(8, tiles - 8*(t/8)), so the 8 units that cover 128 rows of one block are adjacent.
 * Inside a unit, lane l = 4*r0 + q (r0 = 0..7, q = 0..3) owns rows r0 and r0+8 of the
 * tile and the q-th quarter (64 codes, or 80 trits) of the unit's K range. A lane's bytes
 * are its row-r0 bytes followed by its row-(r0+8) bytes (16 + 16 for Q2, 24 + 24 for Q3,
 * 16 + 16 for ternary), cut in 16-byte chunks; chunk c of lane l is stored at unit byte
 * (32*c + (l ^ ((l >> 3) & 3)))*16: the swizzle puts the 8 rows r0 of one quarter in 8
 * different shared-memory bank groups when one thread reads one row. Multi-byte words below
 * are little-endian uint32.
 *   Q2: a row quarter is 4 words; code i (0..63) is in word i/16; with e = i%16 it sits
 *       at bits 16*(e%2) + 2*(e/2) .. +1 (even codes in the low 16 bits, odd in the high).
 *   Q3: a row quarter is two 12-byte groups (codes 0..31, 32..63), 3 words each. With
 *       e = i%32: for e < 30, word e/10, f = e%10, bits 16*(f%2) + 3*(f/2) .. +2; code
 *       30+h (h = 0,1) has its bit j in bit 16*h + 15 of word j.
 *   Ternary: a row quarter is 16 bytes; trit i is digit i%5 of byte i/5, whose value is
 *       sum_d c_d * 3^d. Pad trits are c = 1 (t = 0).
 * Pad rows of Q2/Q3 hold code 0. packed bytes = ceil(N/16) * ceil(K/unit) * UB.
 *
 * Conventions
 * -----------
 * - Pointers: device pointers unless the name ends in _host. The caller owns every
 *   buffer; the library allocates nothing and keeps no per-call state.
 * - Alignment: every pointer must be 16-byte aligned (WR_ERR_INVALID_ARG otherwise).
 * - stream: a cudaStream_t passed as void* (NULL = legacy default stream). Device calls
 *   are asynchronous on that stream and never synchronize.
 * - Errors: arguments are checked synchronously and the call returns before any launch;
 *   launch failures return WR_ERR_CUDA. Nothing aborts and no exception crosses the ABI.
 * - Workspace: where a call takes one, it must be at least *_workspace_bytes(...) bytes
 *   and zero-filled before its first use. Each successful call leaves the parts that must
 *   start at zero (arrival counters) zero again, so one zeroed buffer serves any number of
 *   calls issued in stream order. Calls that may run concurrently (different streams) need
 *   different workspaces.
 */
#ifndef WR_H
#define WR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  WR_OK = 0,
  WR_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size or code value */
  WR_ERR_UNSUPPORTED = 2,   /* valid but unsupported: group != 256, bits not 2/3, ... */
  WR_ERR_CUDA = 3,          /* a CUDA launch or runtime call failed */
  WR_ERR_TIMEOUT = 4,       /* a bounded device-side wait gave up (see wr_get_device_error) */
  WR_ERR_TOO_LARGE = 5      /* the problem needs more than the fixed scratch of wr_gemv_noalloc */
} wr_status;

enum { WR_FMT_TERNARY = 1, WR_FMT_Q2 = 2, WR_FMT_Q3 = 3, WR_FMT_T2 = 4, WR_FMT_T8 = 5 };

/* WR_FMT_T2, the 2-bit trellis-coded format ("How We Shrank...", "Trick 3: trellis coding"):
 * symbols u in [0, 4) are stored exactly like Q2 codes (same packed layout, same bytes), with
 * fp16 scales per 256-block, but they select among the 8 odd levels {-7..7} * s through a
 * 2-state trellis: at step i of a block the state is the low bit of u_(i-1) (0 at the block
 * start), the level index is c3 = 2 u_i + state and the weight is s * (2 c3 - 7). This is the
 * pages' 1-bit toy (two cosets of four levels, the written bit is the next state) written
 * with 2 bits per weight. The codes come from wr_quantize_trellis (a Viterbi search). The
 * decode GEMV (wr_gemv, wr_gemv_batched, wr_gemv_noalloc with bits = WR_FMT_T2) and
 * wr_unpack_bf16 accept it; wr_gemm does not (WR_ERR_UNSUPPORTED). */

/* WR_FMT_T8, the 8-state trellis over symbols of 4 weights at 2 bits per weight ("How We
 * Shrank...", "Trick 3: trellis coding", which names an 8-state set-partitioned trellis over
 * 4-weight symbols and gives no tables; this is the reading taken). The codes u in [0, 4) are stored
 * exactly like Q2 codes (same packed layout and bytes) with fp16 scales per 256-block (or
 * | WR_SCALES_I8). Consecutive groups of 4 codes along K are symbols. The state (s0, s1, s2), 0 at
 * every 256-block start, selects the parity pattern p = (s0, s1, s2, s0 ^ s1 ^ s2): weight i of
 * the symbol has level index c = 2 u_i + p_i and weight s * (2c - 7) on the 8 odd levels; the next
 * state is ((s << 1) | (u_3 & 1)) & 7. The reachable 4-vectors of level indices are those whose
 * parities sum to an even number, split by parity pattern into the 8 cosets the states select.
 * Codes come from wr_quantize_trellis8 (a Viterbi search). Accepted where WR_FMT_T2 is. */

/* Int8 block scales (the "Agents-A1-4B-Wringer-Q2.6" card, "What is in this repo": a container
 * of packed codes with fp16 or int8 block scales). WR_SCALES_I8 is OR'd into the format code
 * (the `bits` or `fmt` argument, or wr_gemv_problem.bits) of Q2, Q3 and T2; the codes and their
 * packed bytes are unchanged, only the `scales` argument changes meaning: it points to a scale
 * record of wr_scales_bytes() bytes,
 *     bytes [0, 2N)          d: fp16 [N], one scale per row,
 *     bytes [R, R + N*K/256) q: int8 [N, K/256] row-major, values 0..127, R = 16*ceil(2N/16),
 * and the block scale is s[n,b] = d[n] * q[n,b], formed exactly in fp32 (at most 11 + 7
 * significant bits), after which every call computes what it computes with fp16 scales s.
 * wr_quantize(bits | WR_SCALES_I8, ...) writes such a record: d_n = fp16(max_k |w[n,k]| /
 * (127 L)) (fp64 division, one rounding, saturated to 65504), q = the integer nearest to
 * absmax_b / (L d_n) (ties to even) clamped to [0, 127] (0 where d_n = 0). Accepted by
 * wr_quantize, wr_quantize_pack, wr_unpack_bf16, wr_gemv, wr_gemv_noalloc, wr_gemv_batched,
 * wr_gemm and their *_workspace_bytes; wr_packed_bytes, wr_pack and wr_unpack_codes take the
 * format without it. Scales: 8 bits per 256 weights plus 16 bits per row, instead of 16 per
 * 256 weights. */
enum { WR_SCALES_I8 = 0x100 };

/* Bytes of the scale buffer of an N x K matrix: fp16 [N, K/256] for Q2/Q3/T2, fp16 [N] for
 * ternary, the record above with WR_SCALES_I8; 0 on bad arguments. */
size_t wr_scales_bytes(int fmt, int64_t N, int64_t K);

/* Version of this ABI (incremented on any incompatible change). */
int wr_abi_version(void);

/* Static description of a status code. */
const char* wr_status_string(wr_status st);

/* Bytes of the packed buffer for an N x K code matrix in format fmt; 0 on bad arguments. */
size_t wr_packed_bytes(int fmt, int64_t N, int64_t K);

/* Host packer: codes_host [N,K] uint8 (Q2: 0..3, Q3: 0..7, ternary: 0..2) ->
 * packed_host (wr_packed_bytes bytes, caller-allocated). Pad bytes are written too.
 * WR_ERR_INVALID_ARG on a code out of range (nothing is guaranteed about packed_host). */
wr_status wr_pack(int fmt, int64_t N, int64_t K, const uint8_t* codes_host, uint8_t* packed_host);

/* Host inverse of wr_pack on the real rows and columns: packed_host -> codes_host [N,K]. */
wr_status wr_unpack_codes(int fmt, int64_t N, int64_t K, const uint8_t* packed_host,
                          uint8_t* codes_host);

/* Host synthetic quantizer for the odd grid (data preparation, not on the device path).
 * Per 256-block along K: s = fp16(absmax / L) (L = 2^bits - 1; the division in fp64 and
 * one rounding to fp16, so the scale is fixed before the codes are chosen, as on the
 * "Agents-A1-4B-Wringer-Q2.6" card, "Honest caveats"), then the nearest odd level of
 * w/s (fp64), clamped to [-L, L]; an exact even quotient goes up; s = 0 gives level +1
 * (nearest-point codes: "Qwen3-4B-Wringer-Q2.6", "Recipe").
 * w_host fp32 [N,K]; codes_host uint8 [N,K]; scales_host fp16 bits [N, K/256]. */
wr_status wr_quantize(int bits, int64_t N, int64_t K, const float* w_host, uint8_t* codes_host,
                      uint16_t* scales_host);
/* (With bits | WR_SCALES_I8, scales_host receives the int8 scale record described above and
 * the codes are chosen against s = d q.) */

/* Device quantizer + packer for the 2/3-bit odd grid: computes on the GPU exactly what
 * wr_quantize followed by wr_pack computes on the host (bit-identical scales and packed bytes),
 * in one pass over W. w [N,K] fp32 row-major, packed (wr_packed_bytes(bits, N, K) bytes) and
 * scales fp16 bits [N, K/256] are device pointers (16-byte aligned); K % 256 == 0. The code of
 * each weight is decided by exact comparisons of w with m*s for the even m between the levels,
 * which is the decision of the fp64 quotient. Asynchronous on `stream`. */
wr_status wr_quantize_pack(int bits, int64_t N, int64_t K, const float* w, void* packed, uint16_t* scales,
                           void* stream);

/* Host trellis encoder for WR_FMT_T2: per 256-block s = fp16(absmax / 7) (fp64 division, one
 * rounding), then the symbol sequence of least squared error under the trellis (Viterbi; ties
 * go to the lower state and symbol). w_host fp32 [N,K]; codes_host uint8 [N,K] (symbols
 * 0..3, packed with wr_pack(WR_FMT_T2, ...)); scales_host fp16 bits [N, K/256]; K % 256 == 0. */
wr_status wr_quantize_trellis(int64_t N, int64_t K, const float* w_host, uint8_t* codes_host,
                              uint16_t* scales_host);

/* Host encoder for WR_FMT_T8: per 256-block s = fp16(absmax / 7) (fp64 division, one rounding),
 * then the code sequence of least squared error under the 8-state trellis (Viterbi from state 0;
 * per weight the nearest allowed level, a tie to the lower code; each state keeps the cheaper of
 * its two predecessors, a tie to the lower; the path ends in the cheapest state, a tie to the
 * lower). w_host fp32 [N,K]; codes_host uint8 [N,K] (0..3, packed with wr_pack(WR_FMT_T8, ...));
 * scales_host fp16 bits [N, K/256]; K % 256 == 0. */
wr_status wr_quantize_trellis8(int64_t N, int64_t K, const float* w_host, uint8_t* codes_host,
                               uint16_t* scales_host);

/* Host synthetic ternary quantizer: W' = W R^T (fp64, per 128-block fast Walsh-Hadamard
 * transform with the sign mask), Delta_n = 0.7 * mean_k |W'[n,k]|, t = sign(W') where
 * |W'| > Delta_n else 0, alpha_n = fp16(mean |W'| over t != 0) (0 if none); codes c = t+1.
 * K % 128 == 0. sign_bits_host uint32 [ceil(K/32)]; alpha_host fp16 bits [N]. */
wr_status wr_quantize_ternary(int64_t N, int64_t K, const float* w_host,
                              const uint32_t* sign_bits_host, uint8_t* codes_host,
                              uint16_t* alpha_host);

/* Device materializer: w_bf16 [N,K] = bf16_RNE(s * g) for Q2, Q3, T2 and T8, optionally
 * | WR_SCALES_I8 (group must be 256), or bf16_RNE(alpha_n * t) for ternary (scales = alpha [N],
 * group ignored; the result is in the rotated basis). Bit-exact; the bf16 checkpoint the
 * "Qwen3-4B-Wringer-Q2.6" card's materializer produces from the container. */
wr_status wr_unpack_bf16(int fmt, int64_t N, int64_t K, const void* packed, const uint16_t* scales,
                         int group, uint16_t* w_bf16, void* stream);

/* Decode GEMV for 1 <= M <= 32 (bits = 2, 3, WR_FMT_T2 or WR_FMT_T8, optionally | WR_SCALES_I8; group 256):
 * streams the packed codes once, decodes them in registers and contracts them on tensor cores
 * (kind::i8: four int8 limbs per token, so M <= 2, 4, 8, 16, 32 take 8, 16, 32, 64, 128 MMA columns).
 * The 128-row x 256-code blocks are cut into one contiguous range per CTA; a row group that
 * several ranges share is combined through the workspace in range order, so the result is the
 * same bits on every run. */
size_t wr_gemv_workspace_bytes(int64_t M, int64_t N, int64_t K, int bits);
wr_status wr_gemv(int64_t M, int64_t N, int64_t K, const uint16_t* x, const void* packed,
                  const uint16_t* scales, int bits, int group, float* y, void* workspace,
                  size_t workspace_bytes, void* stream);

/* One problem of a batched decode GEMV (all fields are read on the host during the call). */
typedef struct {
  const uint16_t* x;       /* bf16 [M, K] activations (device) */
  const void* packed;      /* packed codes (device), format Q2 or Q3 as given by bits */
  const uint16_t* scales;  /* fp16 [N, K/256] block scales, or the int8 scale record (device) */
  float* y;                /* fp32 [M, N] output (device, overwritten) */
  int64_t N, K;            /* K % 256 == 0 */
  int32_t bits;            /* 2, 3, WR_FMT_T2 or WR_FMT_T8, optionally | WR_SCALES_I8 */
  int32_t reserved;        /* must be 0 */
} wr_gemv_problem;

/* Batched decode GEMV: `count` independent problems (2- and 3-bit may be mixed) sharing one
 * token count 1 <= M <= 32, computed by one persistent launch that streams all their packed
 * weights back to back, so the fixed latency of a small GEMV is paid once per batch instead
 * of once per problem (the 252 linears of a 36-layer decoder body fit in one batch of at most
 * 256 problems; larger batches are split into several launches). Each problem computes what
 * wr_gemv computes. problems_host is a host array read during the call. */
size_t wr_gemv_batched_workspace_bytes(int64_t M, int32_t count, const wr_gemv_problem* problems_host);
/* The work split of one batched decode launch (count <= 256 problems), computed on the host
 * with the launch's own arithmetic, for inspection and tests: *grid receives the number of CTAs;
 * if range_starts is not NULL it receives grid + 1 entries (range_starts_len at least that), the
 * first block of each CTA's range in the batch's block sequence (problem by problem, 128-row
 * group by row group, 256-code block by block), then the total block count. Ranges are cut by
 * an estimated cost per block (a 3-bit or trellis block weighs more than a 2-bit one) and each
 * holds at least one block; if block_costs is not NULL it receives that cost for each problem
 * (count entries, in the units the split uses). Only the shapes and formats of problems_host are
 * read (pointers may be NULL); a problem that wr_gemv_batched would reject for its shape, format
 * or reserved field is rejected with the same status. */
wr_status wr_gemv_batched_plan(int64_t M, int32_t count, const wr_gemv_problem* problems_host, int32_t* grid,
                               int64_t* range_starts, int32_t range_starts_len, int64_t* block_costs);
wr_status wr_gemv_batched(int64_t M, int32_t count, const wr_gemv_problem* problems_host, void* workspace,
                          size_t workspace_bytes, void* stream);

/* One weight matrix of a grouped decode GEMV (fields read on the host during the call). */
typedef struct {
  const void* packed;      /* packed codes (device) */
  const uint16_t* scales;  /* fp16 [N, K/256] block scales, or the int8 scale record (device) */
  float* y;                /* fp32 [M, N] output (device, overwritten) */
  int64_t N;
  int32_t bits;            /* 2, 3, WR_FMT_T2 or WR_FMT_T8, optionally | WR_SCALES_I8 */
  int32_t reserved;        /* must be 0 */
} wr_gemv_group_item;

/* Grouped decode GEMV: `count` (1..256) weight matrices applied to the same activations x
 * (bf16 [M, K], 1 <= M <= 32, K % 256 == 0), as the linears of a decoder layer that read one input
 * do: q, k and v read the attention input, gate and up the MLP input ("Qwen3-4B-Wringer-Q2.6",
 * "Recipe": each layer's seven linears, quantized alike). One preparation pass turns x into
 * activation tiles once per tile layout (Q2, Q3, T2), then one persistent launch streams all the
 * weights; each item computes y_i = what wr_gemv computes for (x, packed_i, scales_i). This is the
 * grouping a decoder whose layers depend on each other can use: layer i+1's inputs exist only
 * after layer i. items_host is a host array read during the call; the workspace rules are those
 * of the other calls (wr_gemv_grouped_workspace_bytes, zero-filled before first use). */
size_t wr_gemv_grouped_workspace_bytes(int64_t M, int64_t K, int32_t count, const wr_gemv_group_item* items_host);
wr_status wr_gemv_grouped(int64_t M, int64_t K, const uint16_t* x, int32_t count, const wr_gemv_group_item* items_host,
                          void* workspace, size_t workspace_bytes, void* stream);

/* Prefill GEMM, any M >= 1 (bits = 2 or 3, optionally | WR_SCALES_I8; group 256). M <= 8, and
 * M <= 32 when K <= 4096, run the decode GEMV's integer kernel, which measured faster there; the
 * workspace size follows the same choice (wr_gemm_workspace_bytes). Otherwise: packed tiles are staged in shared memory, decoded to exact bf16 grid
 * integers and contracted by tcgen05 MMAs into TMEM, one fp32 partial per 256-block, scaled in
 * fp32 by the epilogue. */
size_t wr_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int bits);
wr_status wr_gemm(int64_t M, int64_t N, int64_t K, const uint16_t* x, const void* packed,
                  const uint16_t* scales, int bits, int group, float* y, void* workspace,
                  size_t workspace_bytes, void* stream);

/* Ternary GEMV/GEMM, any M >= 1: applies the block-128 random-sign Hadamard to x and
 * contracts with the packed trits; alpha fp16 [N]; sign_bits uint32 [ceil(K/32)]. */
size_t wr_gemm_ternary_workspace_bytes(int64_t M, int64_t N, int64_t K);
wr_status wr_gemm_ternary(int64_t M, int64_t N, int64_t K, const uint16_t* x, const void* packed,
                          const uint16_t* alpha, const uint32_t* sign_bits, float* y,
                          void* workspace, size_t workspace_bytes, void* stream);

/* Decode GEMV that allocates nothing and takes no workspace (no counterpart in the paper: a
 * deployment convenience). For callers that may not allocate device memory or pass a
 * workspace while they run: code recorded into a CUDA graph whose memory was planned up front,
 * allocator-free serving loops, and callers that hold no handle to a caching allocator. The
 * scratch that wr_gemv takes as `workspace` is instead a fixed device array of
 * WR_GEMV_NOALLOC_SCRATCH_BYTES (4 MiB) inside libwr, one per device.
 *
 * Computes exactly what wr_gemv computes (same arguments without workspace/workspace_bytes;
 * 1 <= M <= 32, bits 2, 3, WR_FMT_T2 or WR_FMT_T8, each optionally | WR_SCALES_I8, group 256, K % 256 == 0,
 * 16-byte aligned device pointers).
 * Returns WR_ERR_TOO_LARGE, before touching the device, when the problem's scratch need
 * (wr_gemv_workspace_bytes) exceeds WR_GEMV_NOALLOC_SCRATCH_BYTES; then nothing is launched.
 *
 * The first call on a device does a one-time set-up with that device current (it looks up the
 * address of the scratch array): make that first call before any stream capture begins. Each
 * call clears the scratch's arrival counters on `stream` (cudaMemsetAsync) and then launches
 * the same kernels as wr_gemv. All calls on one device share the one scratch array, so calls
 * that overlap in time (on different streams, or from several host threads) race on it and
 * give undefined results: serialize them. */
#define WR_GEMV_NOALLOC_SCRATCH_BYTES ((size_t)4 << 20)
wr_status wr_gemv_noalloc(int64_t M, int64_t N, int64_t K, const uint16_t* x, const void* packed,
                          const uint16_t* scales, int bits, int group, float* y, void* stream);

/* One problem of a batched ternary decode GEMV (fields read on the host during the call). */
typedef struct {
  const uint16_t* x;           /* bf16 [M, K] activations (device) */
  const void* packed;          /* packed trits (device) */
  const uint16_t* alpha;       /* fp16 [N] row scales (device) */
  const uint32_t* sign_bits;   /* uint32 [ceil(K/32)] random-sign mask of the rotation (device) */
  float* y;                    /* fp32 [M, N] output (device, overwritten) */
  int64_t N, K;                /* K % 128 == 0 */
} wr_gemv_ternary_problem;

/* Batched ternary decode GEMV: `count` independent problems sharing one token count
 * 1 <= M <= 8. One launch applies the block-128 random-sign Hadamard to every problem's x,
 * one persistent launch contracts them all (at most 256 problems per launch; larger batches
 * are split). Each problem computes what wr_gemm_ternary computes. problems_host is read
 * during the call. */
size_t wr_gemv_ternary_batched_workspace_bytes(int64_t M, int32_t count,
                                               const wr_gemv_ternary_problem* problems_host);
wr_status wr_gemv_ternary_batched(int64_t M, int32_t count, const wr_gemv_ternary_problem* problems_host,
                                  void* workspace, size_t workspace_bytes, void* stream);

/* Reads and clears the device error word that bounded waits set when they give up
 * (synchronizes the stream). WR_OK when no wait timed out since the last call. */
wr_status wr_get_device_error(void* stream);

/* Self-test of the failure path that every kernel uses (no counterpart in the pages). Launches
 * one CTA of two warps on `stream`. Warp 0 waits, through the same bounded wait as the
 * kernels, on an mbarrier that nothing arrives on. After the wait limit (one second) it
 * records its code in the device error word and raises the CTA's abort flag. Warp 1 waits on
 * a second such barrier and leaves when it sees the flag. The kernel then returns normally:
 * nothing faults, traps or hangs, and the context stays usable. Returns WR_OK once launched;
 * wr_get_device_error(stream) then returns WR_ERR_TIMEOUT (and clears the word). */
wr_status wr_selftest_wait_timeout(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* WR_H */
