/*
 * trellis_moe.h -- C ABI of the B200 (sm_100a) library for the routed-expert matrix
 * multiply of a trellis-coded quantised mixture-of-experts layer.
 *
 * The method (web pages on T16 / TrellisMX / exlr8 trellis-coded DeepSeek experts):
 *   "DeepSeek-V4.1-Flash-1017 · dsx T16", section "How T16 works":
 *     - experts quantised with a QTIP-style bitshift trellis and 128-wide Hadamard
 *       rotations (section intro);
 *     - item 1, the T16 codebook: a weight's value comes from its 16-bit window of the
 *       bit stream, multiplied by 0x3A2F (16 bits), plus the product's two bytes;
 *     - item 2: column-major positions inside each 16 x 16 tile;
 *     - item 4: each output channel's stored scale.
 *   same card, "October 25 runtime checkpoint": warp Hadamard transforms, fixed-bit
 *     weight expansion, fused gate/up post-processing of the routed experts;
 *   "DeepSeek-V4.1-Flash-1017 TrellisMX K2 Mix", "What is stored": one tensor group per
 *     width present in a layer, each with its ascending global expert ids; "Status":
 *     each width's routes bit-identical to the single-width kernels, full CUDA-graph
 *     replay with changing routes.
 *
 * Stored format (readings where the pages are silent):
 *   - A matrix of R x C weights (R = output channels, C = inputs; both multiples of 16)
 *     is (R/16) x (C/16) tiles in row-major tile order; tile (i, j) holds rows
 *     16i..16i+15 and columns 16j..16j+15 and is 8*K little-endian uint32 words
 *     (exactly 256*K bits, K = 2, 3 or 4 bits per weight).
 *   - Stream bit b of a tile is bit (b mod 32) of its word b/32.  The weight at tile
 *     position p (row p mod 16, column p div 16) takes the 16-bit window whose bit i is
 *     stream bit (p*K + i) mod 256K (tail-biting inside the tile).
 *   - t = lo + hi, the two unsigned bytes of (window * 0x3A2F) mod 2^16; code c = t - 255.
 *   - W[r][col] = s[r] * 2^-12 * c[r][col], s the fp16 per-output-channel scale.
 *   - A projection's input is rotated first: x' = (1/sqrt(128)) * H_128 x on every
 *     contiguous 128-chunk, H_128 the natural-order Sylvester matrix.
 *
 * Conventions for every entry point:
 *   - All array arguments are DEVICE pointers to memory the caller owns (e.g. PyTorch
 *     tensors), unless stated otherwise.  The library allocates nothing, keeps no
 *     pointer after the call returns, and never synchronises the host: work is enqueued
 *     on `stream` (a cudaStream_t; NULL means the legacy default stream).
 *   - fp16 / bf16 buffers are passed as uint16_t bit patterns.
 *   - Return value: TQ_OK, or a tq_status error.  Argument errors are detected on the
 *     host before anything is enqueued; TQ_ERR_CUDA reports a launch error.  Device-side
 *     anomalies (an out-of-range id met by a kernel, a bounded wait that gave up) never
 *     trap: the kernel skips the work and raises a flag readable by tq_device_status().
 *   - No C++ exception crosses this ABI.  Every entry point is usable inside CUDA-graph
 *     capture: none reads device data on the host or synchronises.
 *   - Sizes of zero (T = 0, rows = 0) are valid no-ops returning TQ_OK.
 *   - Kernels run on the current device.  The first call of an entry point on a device
 *     sets its kernels' launch attributes (shared-memory limits) and reads the SM count
 *     for that device; later calls there reuse them.  Calls from several host threads
 *     are safe once each device in use has had one call of each entry point.
 */
#ifndef TRELLIS_MOE_H
#define TRELLIS_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TQ_ABI_VERSION 3

typedef enum {
    TQ_OK = 0,
    TQ_ERR_INVALID_ARG = 1,     /* a size, width, count or pointer is invalid        */
    TQ_ERR_UNSUPPORTED = 2,     /* valid but outside what this build implements      */
    TQ_ERR_ALIGNMENT = 3,       /* a pointer is not aligned as documented            */
    TQ_ERR_WORKSPACE = 4,       /* workspace missing or smaller than required         */
    TQ_ERR_CUDA = 5,            /* a CUDA launch or runtime call failed               */
    TQ_ERR_DEVICE_TIMEOUT = 6   /* a kernel's bounded wait gave up (device flag)      */
} tq_status;

typedef enum { TQ_DTYPE_F16 = 0, TQ_DTYPE_BF16 = 1, TQ_DTYPE_F32 = 2 } tq_dtype;

/* Codebook of a layer's bit streams (every width group of a layer shares it: "All
 * encodes of a layer share its signs and its codebook", exlr8 card, "Stores"). */
typedef enum {
    TQ_CODEBOOK_T16 = 0,        /* T16: one weight per 16-bit window (dsx T16 card)       */
    TQ_CODEBOOK_PAIR_E4M3 = 1   /* pair trellis decoded to FP8 E4M3 (exlr8 card, pmcgx)   */
} tq_codebook;

typedef void *tq_stream; /* cudaStream_t */

/* Human-readable name of a status code (static string; never NULL). */
const char *tq_status_string(int status);

/* TQ_ABI_VERSION of the loaded library. */
int tq_abi_version(void);

/* Text of the most recent CUDA failure behind a TQ_ERR_CUDA return (static buffer,
 * overwritten by the next failure; "" if none).  Host-only, not thread-safe. */
const char *tq_last_error_string(void);

/*
 * Device-side anomaly flags of the current device, OR-ed since the last clear:
 *   bit 0: a kernel met an expert id outside [0, E) or a route index outside [0, T*k)
 *          and skipped that work;
 *   bit 1: a bounded wait inside a kernel gave up (the kernel returned early).
 * Reads the flag word with a synchronous copy (not for use inside graph capture);
 * `clear` != 0 resets it.  Writes the flags to *flags_out (host pointer).
 */
int tq_device_status(int32_t *flags_out, int clear);

/*
 * Launch accounting and per-stage timing of the library's own kernels (tracing; no
 * counterpart on the pages).  Every kernel launch increments a host counter.  While
 * profiling is enabled, each launch is bracketed by two CUDA events recorded on its
 * stream and tagged with its stage:
 *   0 route_topk, 1 route_permute, 2 hadamard128 of the input, 3 MoE GEMV (the fused
 *   launch: gate/up, SwiGLU with the rotation of h, and down; or, for the smallest
 *   batches, the gate/up launch), 4 rotation (and, GEMV, quantisation) of h, 5 MoE GEMV
 *   down launch of the smallest batches, 6 route_unpermute, 7 trellis_decode, 8 trellis_gemv,
 *   9 GEMM gate/up+SiLU, 10 GEMM down, 11 GEMM preparation (tile list, route-ordered
 *   activation rows), 12 GEMV activation quantisation (x' rows to 16-bit fixed point),
 *   13 trellis_encode, 14 route_gather_rows.
 * tq_profile_enable creates 2*max_launches events (host-side CUDA resources; call it
 * outside graph capture); launches beyond max_launches are not recorded.  A launch made
 * during stream capture records its events as external event-record nodes of the graph,
 * re-recorded at every replay, so a collect after replays reads the last replay.
 * tq_profile_collect waits for the recorded events, writes per-stage summed
 * milliseconds and launch counts into the host arrays stage_ms[n_stages] /
 * stage_launches[n_stages] (skipping events never recorded), and clears the record.
 * tq_profile_stages restricts recording to the stages whose bit is set in stage_mask
 * (bit i = stage i; all stages after tq_profile_enable), so that a timed run can carry
 * the events of one kernel only; TQ_ERR_INVALID_ARG while profiling is off.
 */
/*
 * tq_selftest_bounded_wait -- failure-detection check (no counterpart on the pages):
 * one warp runs the library's bounded mbarrier wait on a barrier that nothing arrives
 * on.  After limit_us microseconds (1 .. 10,000,000) the wait gives up, raises device
 * flag bit 1 (read it with tq_device_status) and the kernel returns; nothing traps and
 * the context stays usable.  Asynchronous on `stream`, like every entry point.
 */
int tq_selftest_bounded_wait(uint32_t limit_us, tq_stream stream);

unsigned long long tq_launch_count(void);
int tq_profile_enable(int max_launches);
int tq_profile_stages(uint32_t stage_mask);
int tq_profile_disable(void);
int tq_profile_collect(double *stage_ms, int32_t *stage_launches, int n_stages);

/*
 * trellis_decode -- standalone T16 decode to dense codes ("fixed-bit weight
 * expansion", dsx T16 card, "October 25 runtime checkpoint"; codebook and tile order
 * from "How T16 works", items 1 and 2).
 *   bits : [rows/16][cols/16][8K] uint32, 16-byte aligned.
 *   out  : [rows][cols] fp16, row-major, 16-byte aligned; out[r][c] = c_rc = t - 255
 *          (an integer in [-255, 255], exact in fp16).  Scales are not applied.
 *   rows, cols: multiples of 16.  K in {2, 3, 4}.
 */
int trellis_decode(const uint32_t *bits, int K, int rows, int cols, uint16_t *out,
                   tq_stream stream);

/*
 * trellis_decode_e4m3 -- standalone decode of a pair-trellis matrix to its FP8 E4M3 codes
 * (the pmcgx codebook of the "deepseek-v4.1-flash-exlr8" card, "Stores": two weights share
 * one 20-bit state; each is the sum of the two fp16 halves of the state's product with its
 * multiplier, rounded to E4M3).  Readings: the stream layout is T16's (same tiles, words
 * and bit order); pair q of a tile reads stream bits 2Kq .. 2Kq + 19 (tail-biting) and
 * holds tile positions 2q (product with 0xCBAC1FED) and 2q + 1 (0xBCA14C51); bit 14 of each
 * 16-bit half is cleared before it is read as binary16; the halves are added in binary16
 * (nearest even) and the sum rounded to E4M3 (nearest even).  W[r][c] = s[r] * 2^-5 * w.
 *   bits : [rows/16][cols/16][8K] uint32, 16-byte aligned.
 *   out  : [rows][cols] E4M3 bytes, row-major, 16-byte aligned (scales not applied).
 *   rows, cols: multiples of 16.  K in {2, 3, 4}.
 */
int trellis_decode_e4m3(const uint32_t *bits, int K, int rows, int cols, uint8_t *out, tq_stream stream);

/*
 * hadamard128 -- x' = (1/sqrt(128)) * H_128 x on every contiguous 128-chunk of each
 * row ("128-wide Hadamard rotations", dsx T16 card "How T16 works"; "warp Hadamard
 * transforms", its "October 25 runtime checkpoint").  Computed in fp32, rounded to fp16.
 *   x    : [rows][cols] of x_dtype (F16, BF16 or F32), row-major, 16-byte aligned.
 *   out  : [rows][cols] fp16, row-major, 16-byte aligned.  May not alias x.
 *   cols : a multiple of 128.
 */
int hadamard128(const void *x, int x_dtype, int64_t rows, int64_t cols, uint16_t *out,
                tq_stream stream);

/*
 * hadamard128_signed -- the input side of the two-sided transform: out = rotate(signs * x)
 * (signs: device int8 [cols] of +1/-1, 4-byte aligned); otherwise as hadamard128.
 */
int hadamard128_signed(const void *x, int x_dtype, int64_t rows, int64_t cols, const int8_t *signs,
                       uint16_t *out, tq_stream stream);

/*
 * trellis_gemv -- one trellis-coded matrix times a small batch of rotated activations:
 *   y[b][r] = s[r] * 2^-12 * sum_c code[r][c] * x_rot[b][c]
 * (the projection of "How T16 works", items 1, 2 and 4, on decode-sized batches).
 *   bits   : [rows/16][cols/16][8K] uint32, 16-byte aligned.
 *   scales : [rows] fp16.
 *   x_rot  : [batch][cols] fp16 (already rotated, e.g. by hadamard128), 16-byte aligned.
 *   y      : [batch][rows] fp32.
 *   ws     : device workspace of at least trellis_gemv_workspace_size(rows, cols, batch)
 *            bytes, 16-byte aligned (TQ_ERR_WORKSPACE otherwise).
 *   rows % 16 == 0, cols % 128 == 0, cols <= 16384, K in {2, 3, 4}.
 * Numerics: each row of x_rot enters the tensor-core contraction as 16-bit fixed point
 * x_q = rint(x / 2^e) with one power-of-two scale per row (|x_q| <= 32639), codes exactly;
 * sums are exact in int32 and the scales are applied in double.  A row whose rounding
 * step is coarse for its mass (2^(e-1) * cols > 2^-12 * sum |x|) also carries its residual
 * as a second 16-bit word at 2^(e-15), i.e. it is 32-bit fixed point.  Error per element:
 * at most 2^(e-1) (one word) or 2^(e-16) (two words).
 */
size_t trellis_gemv_workspace_size(int rows, int cols, int batch);
int trellis_gemv(const uint32_t *bits, const uint16_t *scales, int K, int rows, int cols,
                 const uint16_t *x_rot, int batch, float *y, void *ws, size_t ws_bytes,
                 tq_stream stream);

/*
 * route_topk -- top-k experts of every token and their route weights ("top-8 softmax
 * routing"): ids sorted by decreasing logit, ties to the lower expert id; weights are
 * the softmax of the k kept logits (fp32, expf).  NaN logits are not supported.
 *   logits   : [T][E] fp32.   topk_ids : [T][k] int32.   topk_w : [T][k] fp32.
 *   1 <= k <= 32, k <= E <= 1024.
 */
int route_topk(const float *logits, int T, int E, int k, int32_t *topk_ids, float *topk_w,
               tq_stream stream);

/*
 * route_permute -- group the T*k (token, slot) routes by expert ("per-width tensor
 * groups, each with its ascending global expert_ids", TrellisMX K2 Mix card, "What is
 * stored"; grouping is stable in route order).  Route index i = t*k + s.
 *   topk_ids  : [T*k] int32, each in [0, E) (out-of-range ids: flag bit 0, route dropped).
 *   counts    : [E] int32     routes per expert.
 *   offsets   : [E+1] int32   exclusive prefix sum of counts.
 *   perm      : [T*k] int32   route indices sorted by (expert, route index).
 *   inv       : [T*k] int32   inv[perm[j]] = j.
 *   active_ids: [E] int32     experts with counts > 0, ascending (rest untouched).
 *   n_active  : [1] int32     number of such experts.
 *   1 <= E <= 1024.  Deterministic; one CTA.
 */
int route_permute(const int32_t *topk_ids, int T, int k, int E, int32_t *counts,
                  int32_t *offsets, int32_t *perm, int32_t *inv, int32_t *active_ids,
                  int32_t *n_active, tq_stream stream);

/*
 * route_gather_rows -- out[j][:] = src[index[j] / divisor][:] for j < rows: the row moves
 * of expert parallelism (no counterpart on the pages, which run on one GPU).  With
 * index = perm and divisor = k it lays the tokens' rotated rows out in expert-grouped
 * route order (the rows one rank sends to the owners of its routes' experts); with
 * index = inv and divisor = 1 it puts expert-grouped results back into arrival order.
 *   src   : [src_rows][cols] of dtype (TQ_DTYPE_F16 / BF16 / F32), 16-byte aligned.
 *   index : [rows] int32 (device).  out : [rows][cols], 16-byte aligned, caller-owned.
 *   cols * element size must be a multiple of 16 bytes (TQ_ERR_INVALID_ARG otherwise).
 *   An index outside [0, src_rows * divisor) raises device flag bit 0 and yields a zero
 *   row.  The rows are copied bit for bit.
 */
int route_gather_rows(const void *src, int dtype, long long src_rows, int cols, const int32_t *index,
                      int divisor, long long rows, void *out, tq_stream stream);

/*
 * route_topk_permute -- route_topk followed by route_permute, with the same arguments
 * and results (topk_ids / topk_w as route_topk writes them, the grouping arrays as
 * route_permute writes them).  Up to T*k = 4096 routes it is one single-CTA launch (the
 * CTA's warps take the tokens' top-k in turn, then the CTA groups the routes from a
 * shared-memory copy of the ids), recorded under profiling stage 0; larger batches run
 * the two calls.  1 <= k <= 32, k <= E <= 1024.
 */
int route_topk_permute(const float *logits, int T, int E, int k, int32_t *topk_ids, float *topk_w,
                       int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *inv,
                       int32_t *active_ids, int32_t *n_active, tq_stream stream);

/*
 * route_unpermute -- combine: out[t][d] = sum_{s=0..k-1} topk_w[t][s] * y_perm[inv[t*k+s]][d],
 * summed in slot order in fp32 (deterministic, no atomics).
 *   y_perm : [T*k][D] fp32 in expert-grouped order.  inv, topk_w : [T*k].
 *   out    : [T][D] fp32.  D % 4 == 0; y_perm and out 16-byte aligned.
 */
int route_unpermute(const float *y_perm, const int32_t *inv, const float *topk_w, int T, int k,
                    int D, float *out, tq_stream stream);

/*
 * route_unpermute_signed -- combine plus the output side of the down projection's
 * two-sided transform: out[t] = signs_y * rotate(sum_s topk_w[t][s] * y_perm[inv[t*k+s]]),
 * summed in slot order in fp32 (the rotation is linear, so it is applied once, after the
 * weighted sum).  D % 128 == 0; signs_y: device int8 [D], 4-byte aligned.
 */
int route_unpermute_signed(const float *y_perm, const int32_t *inv, const float *topk_w, int T, int k,
                           int D, const int8_t *signs_y, float *out, tq_stream stream);

/*
 * trellis_encode -- T16 bit streams for a target matrix by a tail-biting Viterbi search
 * ("How T16 works": a QTIP-style bitshift trellis found by a Viterbi search, item 1's
 * codebook, item 2's column-major tile positions, item 4: a quantizer minimising squared
 * error).  For every 16x16 tile it minimises sum_p (tau_p - 4 c_p)^2, tau_p =
 * rint(4 * target_p) clamped to [-1276, 1276] (quarter code units), c_p = t - 255 the
 * centred code of window p, over tail-biting streams of 256*K bits; the search is one
 * free pass and, unless its best path already closes, two passes closed on the closure
 * bits of that path's last and first windows (the cheaper wins; ties to the first, to
 * the smaller dropped bits, to the smaller final window), so the result is deterministic.
 *   target : device fp32 [rows][cols], row-major, in code units (the caller divides the
 *            weights by scale * 2^-12); 4-byte aligned.
 *   bits   : device [rows/16][cols/16][8K] uint32, the layout trellis_decode and the
 *            MoE kernels read.
 *   tile_cost : device uint32 [rows/16][cols/16], each tile's objective, or NULL.
 *   ws     : device workspace of trellis_encode_workspace_size(K, rows, cols) bytes
 *            (255 rows of 2^(16-K) backpointer bytes per resident CTA), 16-byte aligned.
 * rows, cols multiples of 16; K in 2..4.  Integer arithmetic throughout.  Returns
 * TQ_ERR_INVALID_ARG / TQ_ERR_ALIGNMENT / TQ_ERR_WORKSPACE before launching anything.
 */
size_t trellis_encode_workspace_size(int K, int rows, int cols);
int trellis_encode(const float *target, int K, int rows, int cols, uint32_t *bits,
                   uint32_t *tile_cost, void *ws, size_t ws_bytes, tq_stream stream);

/* One width group of a layer: experts of one K, concatenated in ascending global id. */
typedef struct {
    int K;                       /* 2, 3 or 4 bits per weight                          */
    int n_experts;               /* experts in the group                               */
    const int32_t *expert_ids;   /* device [n_experts], ascending global ids           */
    const uint32_t *gate;        /* device [n_experts][F/16][D/16][8K] words           */
    const uint32_t *up;          /* device [n_experts][F/16][D/16][8K] words           */
    const uint32_t *down;        /* device [n_experts][D/16][F/16][8K] words           */
    const uint16_t *s_gate;      /* device fp16 [n_experts][F]                         */
    const uint16_t *s_up;        /* device fp16 [n_experts][F]                         */
    const uint16_t *s_down;      /* device fp16 [n_experts][D]                         */
} tq_width_group;

/*
 * A trellis-coded MoE layer: E experts of hidden size D and intermediate size F.
 * Optional two-sided transform (the exlr8 layout's "128 x 128 Hadamard on both sides"
 * and layer signs shared by every expert): with the four sign vectors set, every
 * projection is s_out * rotate(W * rotate(s_in * input)), i.e.
 *   x' = rotate(sign_x * x)          (the caller: hadamard128_signed)
 *   g  = sign_gu * rotate(W_gate x'),  u = sign_gu * rotate(W_up x'),  h = silu(g) * u
 *   h' = rotate(sign_h * h),           y = sign_y * rotate(W_down h')
 * moe_trellis_gemv / _gemm apply sign_gu and sign_h; their y_perm holds W_down h' before
 * the output rotation, which route_unpermute_signed applies after the combine.  All four
 * NULL: the input-side-only layer (x' = rotate(x), h' = rotate(h), y = W_down h').
 */
typedef struct {
    int E, D, F;                 /* D % 128 == 0, F % 128 == 0                         */
    int n_groups;                /* 1..3 width groups                                  */
    tq_width_group groups[3];
    const int32_t *expert_slot;  /* device [E]: (group << 16) | index in group, or -1  */
    const int8_t *sign_x;        /* device [D] +1/-1, 4-byte aligned, or NULL          */
    const int8_t *sign_gu;       /* device [F]                                         */
    const int8_t *sign_h;        /* device [F]                                         */
    const int8_t *sign_y;        /* device [D]                                         */
    int codebook;                /* tq_codebook of every group (0: T16)                */
} tq_moe_layer;

/*
 * Workspace bytes moe_trellis_gemv and moe_trellis_gemm need for T tokens and k routes
 * (the larger of the two).  GEMV: the gate and up results of every route ([T*k][S][2][F]
 * fp32, S column splits), the rotated SwiGLU activations h' and the rotated tokens x' as
 * fixed point (four half-word planes per value, 16 bytes per row) and the counters of its
 * work queue.  GEMM: route-ordered activation rows and their sums or scales, h, h' with
 * its sums and scales, and the tile list.  The split count S depends on the device's SM
 * count, so query the size on the device that runs the call.  Returns 0 on invalid
 * arguments.
 */
size_t moe_trellis_workspace_size(const tq_moe_layer *layer, int T, int k);

/*
 * moe_trellis_gemv -- the routed experts of one MoE layer for decode-sized batches
 * (the SwiGLU expert with fused gate/up post-processing, "October 25 runtime
 * checkpoint" of the dsx T16 card, on T16 weights, "How T16 works"):
 *   for every route i (expert e = expert of route i, token t = perm[i] / k):
 *     g = W_gate[e] x'_t,  u = W_up[e] x'_t,  h = silu(g) * u,
 *     h' = rotate128(h),   y_perm[i] = W_down[e] h'
 *   x_rot    : [T][D] fp16 rotated tokens (hadamard128 of the layer input).
 *   offsets, perm, active_ids, n_active : from route_permute (device).
 *   y_perm   : [T*k][D] fp32, expert-grouped route order.
 *   ws       : device workspace of at least moe_trellis_workspace_size() bytes.
 *   From 32 routes (T*k): two launches, the fixed-point quantisation of x', then one
 *   persistent kernel that takes gate/up items and then down items from a work queue; the
 *   CTA finishing an expert's last gate/up item computes that expert's h' (SwiGLU,
 *   rotation, quantisation) and its down items wait for it.  Below 32 routes: four
 *   launches (x' quantisation, gate/up, h', down) with the same arithmetic.  Mixed
 *   widths run in the same launches; routes of an
 *   expert are processed together, each weight decoded once per 4 (or 8) of its routes.
 *   x' and h' enter the tensor-core contraction as fixed point with one power-of-two
 *   scale per row (as in trellis_gemv: 16 bits, 32 for a row whose rounding step is
 *   coarse for its mass); h' is rotated from fp32 h without an fp16 rounding.
 *   D, F <= 16384.
 */
int moe_trellis_gemv(const tq_moe_layer *layer, const uint16_t *x_rot, const int32_t *offsets,
                     const int32_t *perm, const int32_t *active_ids, const int32_t *n_active,
                     int T, int k, float *y_perm, void *ws, size_t ws_bytes, tq_stream stream);

/*
 * moe_trellis_gemv_noalloc -- moe_trellis_gemv without a caller-provided workspace, for
 * callers that cannot allocate device memory when they run the layer (a serving
 * runtime whose memory is one pool carved up at start-up, a plugin or sandboxed engine
 * that only receives the call's own tensors, a latency-critical path where an
 * allocation and the synchronisation it may imply are not allowed).  The pages have no
 * counterpart: this is a packaging of the same computation.
 *   Same arguments and result as moe_trellis_gemv, minus ws / ws_bytes.  The workspace
 *   is a 4 MiB array compiled into the library (a __device__ array every GPU that loads
 *   the library holds until exit), so the GEMV workspace -- 8 * S * T * k * F (gate/up
 *   results, S = 1..8 column splits for small batches) + 8 * T * k * F + 8 * T * D bytes
 *   (fixed-point h' and x', two words each) plus 16 bytes per row and 4 * (1 + 2E) bytes
 *   of work-queue counters, each part rounded up to 256 bytes; T <= 25 at k = 8, E = 384,
 *   D = 4096, F = 1024 -- must fit in it; larger calls return TQ_ERR_WORKSPACE without
 *   doing anything.
 *   Allocates nothing: no cudaMalloc, no cudaFree, no allocating library routine.
 *   Arguments are checked first, with the same statuses as moe_trellis_gemv; then a call
 *   whose workspace would not fit returns TQ_ERR_WORKSPACE.
 *   The first call on a device looks up the array's device address (cudaGetSymbolAddress,
 *   once per device, with that device current) and keeps it for the life of the
 *   context: make that first call before any stream capture, and reload the library
 *   after a cudaDeviceReset.  Every call on a device shares the one array and it keeps
 *   the last call's contents; each call writes every workspace byte it reads before
 *   reading it, so nothing needs clearing, but calls that overlap on the GPU (other
 *   streams, other threads) race on the array and must be serialised by the caller.
 *   The results are those of moe_trellis_gemv bit for bit.
 */
int moe_trellis_gemv_noalloc(const tq_moe_layer *layer, const uint16_t *x_rot,
                             const int32_t *offsets, const int32_t *perm, const int32_t *active_ids,
                             const int32_t *n_active, int T, int k, float *y_perm, tq_stream stream);

/*
 * moe_trellis_gemm -- same result as moe_trellis_gemv for prefill-sized batches: the
 * bit streams are decoded to tensor-core operands of tcgen05 MMAs (accumulating in
 * tensor memory), each weight decoded once per block of up to 256 routes of its
 * expert.  Same arguments as moe_trellis_gemv; the workspace must hold
 * moe_trellis_workspace_size() bytes; D must be a multiple of 256 (TQ_ERR_UNSUPPORTED
 * otherwise).
 *   T16 layers: fp16 operands (codes exact as fp16 subnormals t * 2^-24, activations
 *   fp16), kind::f16 MMAs.  The rotated h' rows are stored as fp16 h' / 2^e with the
 *   row's largest magnitude in [2^14, 2^15), so no finite h overflows.
 *   Pair-trellis layers (codebook TQ_CODEBOOK_PAIR_E4M3, the exlr8 card's FP8 decode):
 *   E4M3 weights and E4M3 activations, kind::f8f6f4 MMAs at twice the fp16 rate.  Each
 *   route row of x' and of h' is scaled by the power of two 2^-e that puts its largest
 *   magnitude in (224, 448] and rounded to E4M3 (nearest even), so the activations carry
 *   E4M3's 2^-4 relative rounding; y = s * 2^-5 * 2^e * sum_j w_j * v8_j.
 * moe_trellis_gemv and moe_trellis_gemv_noalloc run T16 layers only
 * (TQ_ERR_UNSUPPORTED for a pair-trellis layer).
 */
int moe_trellis_gemm(const tq_moe_layer *layer, const uint16_t *x_rot, const int32_t *offsets,
                     const int32_t *perm, const int32_t *active_ids, const int32_t *n_active,
                     int T, int k, float *y_perm, void *ws, size_t ws_bytes, tq_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* TRELLIS_MOE_H */
