/*
 * stq.h -- C ABI of the quantized linear-attention state library (B200, sm_100a).
 *
 * What it computes. Linear-attention models with the gated delta rule keep one fixed-size
 * recurrent state per request and head ("线性注意力状态量化难题" (aitest123.com/news/n1kj09),
 * introduction); serving many requests makes that state pool the memory bottleneck ("K1 論文詳解"
 * (k1-news.pages.dev/paper/2026-10-09), section 背景). Each decode step reads the previous
 * state, updates it, requantizes it and stores it back (aitest123 page, section
 * 直接量化为什么会翻车). The state of a head is kept as low-bit integer codes with one scale per
 * key row and one per value column whose product sets the step (k1 page, section 方法;
 * aitest123 page, section 空间维度); widths come per head from a few discrete candidates and the
 * highest-risk heads stay FP16 (k1 page, section 方法; aitest123 page, section 时间维度). The
 * pages print no formula; this library fixes them as follows (d_k x d_v state S per head):
 *
 *   dequantize   S_ij = r_i c_j Q_ij,  Q_ij in [-qmax, qmax], qmax = 2^(b-1) - 1, b in {4,6,8}
 *   update       u = k^T S;  S' = alpha (S - beta k u^T) + beta k v^T
 *   readout      o = S'^T q               (after the update, before requantization)
 *   column scale c'_j = sqrt( sum_i w_i S'_ij^2 / sum_i w_i )   (w: per-head key-row impact)
 *   row scale    r'_i = max_j |S'_ij / c'_j| / qmax
 *   requantize   Q'_ij = round_half_even(S'_ij / (r'_i c'_j)); a zero scale is replaced by 1
 * Scales are stored as fp32 (or, with scale_dtype = STQ_BF16, as bf16 rounded half to even: the
 * 16-bit scales that bring a 6-bit 128 x 128 head to 5.12x compression, the figure the k1 page's
 * section 實驗結果 reports as ~5.03x with pivots) and codes are computed from the stored scales,
 * column scales first, then the row scales from the stored column scales. A layout may ask for
 * scale_fit_rounds rounds of joint refinement after that fit (the pages fit the two scales jointly,
 * weighting high-impact rows more: "线性注意力状态量化难题", section 空间维度): each round refits
 * every column scale by impact-weighted least squares, c_j = sum_i w_i a_ij S_ij / sum_i w_i a_ij^2
 * with a_ij = r_i Q_ij, then every row scale by least squares, r_i = sum_j b_ij S_ij / sum_j b_ij^2
 * with b_ij = c_j Q_ij (new c, same Q), then recomputes the codes; a refit value that is not finite
 * and positive keeps the old one. A pivot head (b = 16)
 * stores S' as fp16 (round to nearest even) and has no scales. With the channel gate alpha is a
 * vector over key rows: STQ_GATE_CHANNEL substitutes it literally,
 * S'_ij = alpha_i (S_ij - beta k_i u_j) + beta k_i v_j; STQ_GATE_CHANNEL_DECAY_FIRST decays first,
 * u = k^T diag(alpha) S, S'_ij = alpha_i S_ij - beta k_i u_j + beta k_i v_j.
 *
 * Byte layout of the pool. A request block is the concatenation of its head blocks (in head
 * order) padded to 128 bytes; request `slot` starts at pool + slot * bytes_per_request. A quantized
 * head block holds the codes as a little-endian bitstream (code (i,j) at bit b*(i*d_v + j), bit k
 * of the stream = bit k%8 of byte k/8, stored offset-binary Q + 2^(b-1)), zero padding to 16 bytes,
 * r[d_k], c[d_v] (fp32, or bf16 in the 16-bit scale format), zero padding to 128 bytes. A pivot
 * head block is S as fp16 row-major,
 * padded to 128 bytes. The pool is its own checkpoint: its bytes plus the layout descriptor.
 *
 * Conventions for every call below.
 *   - All pointers named "device" point to memory of the current CUDA device; the caller owns and
 *     allocates every buffer. The library allocates no device memory and never synchronizes.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream). All work is
 *     enqueued on it; results are ready when the stream reaches that point.
 *   - Arguments are checked before anything is enqueued; a failed check returns
 *     STQ_ERR_INVALID_ARG / STQ_ERR_UNSUPPORTED and enqueues nothing. A failed launch returns
 *     STQ_ERR_CUDA.
 *   - Conditions found on the device are OR-ed into *dev_status (a device int32 the caller zeroes;
 *     may be NULL) as the bit (1 << code): STQ_ERR_NONFINITE when an updated state, scale or output
 *     is not finite (or a pivot overflows fp16; the tile's bytes are then unspecified),
 *     STQ_ERR_BOUNDS when a slot is outside [0, pool_slots) (that tile is skipped),
 *     STQ_ERR_TIMEOUT when a bounded wait for a staged copy gave up (the thread block that timed
 *     out skips its remaining tiles, whose bytes are then unspecified; other thread blocks of the
 *     call carry on). Kernels never trap.
 *   - Slots within one call must be distinct. Calls on different streams must not touch the same
 *     slots concurrently.
 *   - Supported on the device: d_k == d_v == d in {16, 32, 64, 128}; widths {4, 6, 8, 16};
 *     q/k/v in fp32 or bf16; all three gates, for decode and for prefill.
 */
#ifndef STQ_H
#define STQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define STQ_ABI_VERSION 4

typedef enum {
    STQ_OK = 0,
    STQ_ERR_INVALID_ARG = 1,
    STQ_ERR_UNSUPPORTED = 2,
    STQ_ERR_CUDA = 3,
    STQ_ERR_NONFINITE = 4,
    STQ_ERR_TIMEOUT = 5,
    STQ_ERR_BOUNDS = 6
} stq_status;

typedef enum { STQ_F32 = 0, STQ_BF16 = 1 } stq_dtype;

typedef enum {
    STQ_GATE_SCALAR = 0,             /* alpha [B][H]        */
    STQ_GATE_CHANNEL = 1,            /* alpha [B][H][d_k]   */
    STQ_GATE_CHANNEL_DECAY_FIRST = 2 /* alpha [B][H][d_k]   */
} stq_gate;

/* How the 4/6/8-bit heads of a layout are scaled. STQ_SCALES_UNIFORM is the baseline the pages
 * compare the method with ("线性注意力状态量化难题", sections 直接量化为什么会翻车 / 数据说话): one
 * symmetric scale per head, s = max_ij |S_ij| / qmax (0 -> 1), stored fp32, codes
 * Q_ij = round_half_even(S_ij / s); its head block is the codes bitstream, zero padding to 16
 * bytes, s, zero padding to 128 bytes. Uniform layouts run on the plain (untuned) kernels. */
typedef enum { STQ_SCALES_ROW_COLUMN = 0, STQ_SCALES_UNIFORM = 1 } stq_scale_mode;

/* Static description of one model's state: fixed across requests and steps. */
typedef struct {
    int32_t num_heads;         /* H >= 1 (all layers' heads of one request, in pool order)   */
    int32_t d_k;               /* key dimension (rows of a head's state)                     */
    int32_t d_v;               /* value dimension (columns)                                  */
    const uint8_t *head_bits;  /* host [H]: 4, 6, 8, or 16 (FP16 pivot head); copied         */
    int32_t gate;              /* stq_gate                                                   */
    int32_t in_dtype;          /* stq_dtype of q, k, v                                       */
    int32_t scale_mode;        /* stq_scale_mode (0: the method's row x column scales)       */
    int32_t scale_dtype;       /* stq_dtype of the stored row and column scales: STQ_F32 (0) */
                               /* or STQ_BF16 (16-bit scales; row x column mode only)        */
    int32_t scale_fit_rounds;  /* 0: the one-pass fit above. 1..8: that many rounds of the    */
                               /* impact-weighted joint refinement (row x column mode only)  */
} stq_layout_desc;

typedef struct stq_layout stq_layout; /* opaque, host-only, immutable after creation */

/* Version of this ABI (STQ_ABI_VERSION of the built library). */
int32_t stq_abi_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char *stq_status_string(int32_t status);

/* Build a layout from `desc` (host only; no CUDA call). Returns STQ_ERR_INVALID_ARG for NULL
 * pointers, non-positive sizes, an unknown gate, input dtype, scale mode or scale dtype, or
 * scale_fit_rounds outside 0..8; STQ_ERR_UNSUPPORTED for widths other than {4,6,8,16}, shapes the
 * device path does not support, or bf16 scales / refinement rounds with the uniform mode. On success *out owns a new layout, released with
 * stq_layout_destroy. The layout may be shared between threads. */
stq_status stq_layout_create(const stq_layout_desc *desc, stq_layout **out);
void stq_layout_destroy(stq_layout *layout);

/* Bytes of one request block (a multiple of 128), and the byte offset / size / width of head h
 * inside it (0 for an invalid head). */
size_t stq_layout_bytes_per_request(const stq_layout *layout);
size_t stq_layout_head_offset(const stq_layout *layout, int32_t head);
size_t stq_layout_head_bytes(const stq_layout *layout, int32_t head);
int32_t stq_layout_head_bits(const stq_layout *layout, int32_t head);

/* Quantize given fp32 states into the pool: the column / row scale fit and requantization above
 * applied to S0 (or the fp16 conversion for pivot heads).
 *   pool        device, >= pool_slots * bytes_per_request bytes, 128-byte aligned
 *   slots       device int32 [B], the pool slot of each request
 *   S0          device fp32 [B][H][d_k][d_v], row-major, 4-byte aligned (with a 16-byte aligned
 *               S0 and w, 128 x 128 row x column heads stream through TMA tensor copies; else
 *               4-byte loads)
 *   w           device fp32 [H][d_k], impact weights, finite and > 0
 * B == 0 is a no-op. */
stq_status stq_init_state(const stq_layout *layout, void *pool, int32_t pool_slots,
                          const int32_t *slots, int32_t B, const float *S0, const float *w,
                          int32_t *dev_status, void *stream);

/* One decode step, in place, for heads [head_begin, head_begin + head_count) of B requests:
 * dequantize, update, read out, refit the scales, requantize, store. Per-head arrays below are
 * indexed by (request b, head h - head_begin), i.e. they hold only the heads of this call:
 *   q, k        device [B][head_count][d_k] of in_dtype, 16-byte aligned
 *   v           device [B][head_count][d_v] of in_dtype, 16-byte aligned
 *   beta        device fp32 [B][head_count]
 *   alpha       device fp32 [B][head_count] (scalar gate) or [B][head_count][d_k], 16-byte aligned
 *   w           device fp32 [head_count][d_k], finite and > 0, 16-byte aligned
 *   o           device fp32 [B][head_count][d_v], written
 * B == 0 or head_count == 0 is a no-op. */
stq_status stq_decode_step(const stq_layout *layout, void *pool, int32_t pool_slots,
                           const int32_t *slots, int32_t B, int32_t head_begin, int32_t head_count,
                           const void *q, const void *k, const void *v, const float *beta,
                           const float *alpha, const float *w, float *o, int32_t *dev_status,
                           void *stream);

/* Workspace bytes stq_prefill_chunk can use for B requests and T tokens in chunks of `chunk`.
 * Nonzero only for the shapes that take the tensor-core chunk form with one plain
 * requantization per chunk end (128 x 128 heads, bf16 inputs, the scalar gate, chunk == 64, row x
 * column scales, no refit round): one record of 116736 bytes per request, head (FP16 pivot heads
 * included) and chunk of a segment, where the call is cut into segments of at most 32 chunks, so
 * at most B x H x 32 records whatever T. Host only. */
size_t stq_prefill_workspace_bytes(const stq_layout *layout, int32_t B, int32_t T, int32_t chunk);

/* Chunked prefill of T tokens for all H heads of B requests, in place. Tokens are cut into
 * chunks [0,chunk), [chunk,2chunk), ... of this call (the last may be short); inside a chunk
 * the state is carried unquantized, o_t = S_t^T q_t is emitted for every token, and the state is
 * requantized at the end of every chunk exactly as a decode step requantizes it; the pool holds
 * the requantized state after the last chunk (a multi-chunk call equals the same chunks issued one
 * call each). chunk == 1 is the decode step token by token.
 *   q, k        device [B][H][T][d_k] of in_dtype;  v device [B][H][T][d_v] of in_dtype
 *   beta        device fp32 [B][H][T]
 *   alpha       device fp32 [B][H][T] (scalar gate) or [B][H][T][d_k] (channel gates)
 * 128 x 128 heads with bf16 inputs, the scalar gate and chunk == 64 run the tensor-core chunk
 * form (with a workspace for every head, FP16 pivots included; without one for the 4/6/8-bit
 * heads); the other heads, shapes, gates and chunks run token by token with the same
 * chunk-boundary requantization (128 x 128 heads with the state held on chip).
 *   w           device fp32 [H][d_k]
 *   o           device fp32 [B][H][T][d_v], written
 *   workspace   device scratch of >= stq_prefill_workspace_bytes(...) bytes, 256-byte aligned, or
 *               NULL. With a workspace the chunk form runs as three kernels per segment: the
 *               state-free parts of every chunk in parallel, the state recurrence chunk after
 *               chunk, then every chunk's readout in parallel; without one it runs as a single
 *               kernel that keeps everything on chip (slower). The two agree up to the rounding
 *               order of fp32 sums. A workspace that is given but too small or misaligned is
 *               STQ_ERR_INVALID_ARG. It is the caller's memory, used on `stream` only and free again
 *               when the call's work on `stream` is done: calls in flight at the same time need
 *               separate workspaces.
 * T == 0 or B == 0 is a no-op. */
stq_status stq_prefill_chunk(const stq_layout *layout, void *pool, int32_t pool_slots,
                             const int32_t *slots, int32_t B, int32_t T, int32_t chunk,
                             const void *q, const void *k, const void *v, const float *beta,
                             const float *alpha, const float *w, float *o, void *workspace,
                             size_t workspace_bytes, int32_t *dev_status, void *stream);

/* stq_prefill_chunk for callers that cannot allocate device memory, with the workspace in memory
 * the library owns. It has no counterpart in the paper: the method says nothing about where
 * scratch memory comes from; this call only moves the workspace into the library.
 * Who needs it: a caller that may not allocate on this path - a serving loop whose device memory
 * is fixed at start-up and handed out by its own pool, a plug-in or embedding host that gives this
 * library no allocator, or code that must not call cudaMalloc / cudaFree because they can block
 * until the whole device is idle and so stall every other stream.
 * The records live in one fixed device array of 33554432 bytes (32 MiB), defined in the library
 * and created with it on each device; the call allocates nothing, on the device or the host. It
 * fits the segments to the array: segments of min(32, 32 MiB / (B * m * 116736)) chunks, where m
 * is the largest number of heads of one width (FP16 pivots are a width); if one chunk of one width does not fit
 * (B * m * 116736 > 32 MiB, for example more than 287 requests of one 4-bit head) the call returns
 * STQ_ERR_UNSUPPORTED before any device work (use stq_prefill_chunk with a workspace instead).
 * Nothing in the array has to start at zero: every record a call reads is written earlier in the
 * same call. All calls on a device share the one array, so calls whose device work overlaps (on
 * different streams, or from different host threads) race on it and give wrong results; keep
 * them on one stream or order them. The first call on each device looks up the array's device
 * address (cudaGetSymbolAddress) and keeps it for later calls. Shapes without a workspace form
 * run exactly as stq_prefill_chunk with workspace == NULL. Arguments, results and errors are
 * otherwise those of stq_prefill_chunk; results equal stq_prefill_chunk with a workspace bit for
 * bit (segment length changes no arithmetic). */
stq_status stq_prefill_chunk_noalloc(const stq_layout *layout, void *pool, int32_t pool_slots,
                                     const int32_t *slots, int32_t B, int32_t T, int32_t chunk,
                                     const void *q, const void *k, const void *v, const float *beta,
                                     const float *alpha, const float *w, float *o, int32_t *dev_status,
                                     void *stream);

/* Dequantize the pool into fp32: S_out[b][h][i][j] = fp32(r_i c_j) * Q_ij (the fp16 value for a
 * pivot head).  S_out device fp32 [B][H][d_k][d_v]. */
stq_status stq_dequantize(const stq_layout *layout, const void *pool, int32_t pool_slots,
                          const int32_t *slots, int32_t B, float *S_out, int32_t *dev_status,
                          void *stream);

/* Lifetime-aware width allocation (host only; no device work). The time dimension of the method
 * ("线性注意力状态量化难题" (aitest123.com/news/n1kj09), section 时间维度; "K1 論文詳解", section
 * 方法): a state unit's quantization error lives as long as its memory, so under a fixed budget
 * the heads with large error and long lifetime get the higher precision, and the few
 * highest-risk heads stay FP16 pivots. The pages fix no formula; this library uses, per head h:
 *   lifetime weight  lam_h = 1 / max(1 - exp(l_h), 1e-12),  l_h = mean log-retention of the gate
 *   risk             R_h(b) = lam_h * D_h(b),  D_h(b) = calibration distortion at width b
 *   pivots           the num_pivots heads of largest R_h(8) (ties: lower head index)
 *   the rest start at 4 bits; repeatedly the step 4 -> 6 or 6 -> 8 of largest risk reduction per
 *   extra byte (ties: lower head index) is taken if the request's head-block bytes stay within
 *   budget_bytes, otherwise that head keeps its width; until no step fits.
 *   distortion          host double [H][3]: D_h at widths 4, 6, 8 (finite, >= 0)
 *   mean_log_retention  host double [H] (finite, <= 0)
 *   d                   d_k = d_v of the heads (16, 32, 64 or 128), sets the head-block bytes
 *   widths_out          host uint8 [H], written: 4, 6, 8 or 16
 * Returns STQ_ERR_INVALID_ARG for bad arguments or a budget below the smallest allocation (pivots
 * at 16 bits, every other head at 4 bits). Deterministic; thread-safe. */
stq_status stq_allocate_widths(int32_t num_heads, int32_t d, const double *distortion,
                               const double *mean_log_retention, int32_t num_pivots,
                               uint64_t budget_bytes, uint8_t *widths_out);

/* Key-row impact scores from calibration tokens ("线性注意力状态量化难题", section 空间维度): the
 * readout error is a sum over key rows of the row's state error times a weight set by the current
 * key, query and gate; the score is that weight's mean square, the w the quantizer takes. With
 * one update E -> E' of a state error, the next readout error is E'^T q = E^T g, where
 *   STQ_GATE_SCALAR               g = a (q - b (k.q) k)
 *   STQ_GATE_CHANNEL              g = a*q - b (k.(a*q)) k
 *   STQ_GATE_CHANNEL_DECAY_FIRST  g = a * (q - b (k.q) k)
 *   q, k    device [T][H][d] of in_dtype (calibration tokens of H heads)
 *   beta    device fp32 [T][H];  alpha device fp32 [T][H] (scalar gate) or [T][H][d]
 *   w_out   device fp32 [H][d], written: w_i = mean over the T tokens of g_i^2
 * d in {16, 32, 64, 128}. Enqueued on `stream`; allocates nothing. */
stq_status stq_row_impact(int32_t T, int32_t H, int32_t d, int32_t gate, int32_t in_dtype, const void *q,
                          const void *k, const float *beta, const float *alpha, float *w_out, void *stream);

/* Self-test of the bounded wait every kernel of this library uses on its copies: one CTA waits on
 * a barrier that nothing completes, gives up after the library's cap (about 4e9 SM clock cycles,
 * ~2 s), ORs the STQ_ERR_TIMEOUT bit into *dev_status and exits, leaving the context usable. It
 * shows how a stalled copy is reported, without a fault or a hang.
 *   dev_status  device int32 status word (required)
 * Enqueued on `stream`; returns STQ_ERR_INVALID_ARG for a null status word. */
stq_status stq_selftest_wait_timeout(int32_t *dev_status, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* STQ_H */
