/*
 * sq.h -- C ABI of libsq: the per-token decode step of gated delta-rule linear attention over
 * a pool of per-request recurrent states held in a packed, mixed-width, dual-axis-scaled
 * format, on NVIDIA B200 (sm_100a).
 *
 * Sources (prose web pages; no formulas or code are printed there):
 *   [SQ-E] STEPQuant explainer (blog.ontle.kr/blog/302)
 *   [SQ-N] STEPQuant news, "STEPQuant、推論メモリを最大68.7%削減", section 研究の概要
 *   [LQ-N] LeapQuant news, "LeapQuant、線形注意の推論を1.47倍高速化", section 研究の概要
 *
 * Conventions for every call
 *   - Pointers marked (device) are CUDA device pointers; (host) are ordinary host pointers.
 *     Device pointers must be 16-byte aligned; the pool buffer must be 256-byte aligned.
 *   - The caller owns every buffer it passes. The pool handle owns only its host metadata, a
 *     few small device tables (offset tables and a status word, allocated at create; the row
 *     impact table, allocated by sq_pool_set_row_impact) and, after its first split step, two
 *     CUDA events; destroy frees them all.
 *   - `stream` is a cudaStream_t passed as void*; NULL means the legacy default stream. Calls
 *     that take a stream only enqueue work and return; they do not synchronize.
 *   - Every call returns an sq_status. Nothing aborts, traps or prints. Argument errors are
 *     found on the host before anything is enqueued. Problems only the GPU can see (a slot
 *     index out of range, a non-finite input, a state too large for fp16 scales) set a sticky
 *     device status word, and the affected (request, head) is skipped: its slot bytes stay as
 *     they were and its output row is filled with NaN. sq_pool_status() reads and clears it.
 *   - Within one call every slot index must be distinct; duplicates are not detected and give
 *     an undefined result. Calls on one pool must not overlap in time on different streams
 *     (the second stream of sq_decode_step_split is ordered by the pool itself).
 *   - A pool lives on the device that was current when it was created, and every later call
 *     on it must be made with that device current: the library never switches devices, and
 *     every pointer passed with a pool must be memory of that device.
 *   - State layout: S[i][j] with i the key channel ("key row", [SQ-E] fitting paragraph) and
 *     j the value channel ("value column", [SQ-N]). Dense fp32 states are row-major
 *     [n][n_heads][d_k][d_v].
 */
#ifndef SQ_H
#define SQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SQ_API __attribute__((visibility("default")))
#else
#define SQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SQ_OK = 0,
  SQ_ERR_INVALID_ARG = 1, /* bad layout, bit map, pointer, alignment or size */
  SQ_ERR_UNSUPPORTED = 2, /* a valid request this build does not handle (e.g. no sm_100 GPU) */
  SQ_ERR_CUDA = 3,        /* a CUDA runtime call failed */
  SQ_ERR_OOM = 4,         /* the pool's small device tables could not be allocated */
  SQ_ERR_DEVICE_FLAG = 5, /* sq_pool_status: the GPU flagged a slot, a value or a range */
  SQ_ERR_TIMEOUT = 6      /* sq_pool_status: a kernel gave up waiting on a copy */
} sq_status;

typedef enum { SQ_GATE_SCALAR = 0 /* GDN: one alpha per head */,
               SQ_GATE_DIAG = 1 /* KDA: one alpha per key channel */ } sq_gate;
typedef enum { SQ_UNIT_HEAD = 0 /* one width per head */,
               SQ_UNIT_KEY_ROW = 1 /* one width per key row */ } sq_unit;
typedef enum { SQ_IO_F32 = 0, SQ_IO_BF16 = 1 } sq_io_dtype; /* dtype of q, k, v */

/* Bits of the device status word returned by sq_pool_status(). */
#define SQ_FLAG_BAD_SLOT 1  /* a slot index outside [0, n_slots) */
#define SQ_FLAG_NONFINITE 2 /* a non-finite q, k, v, alpha, beta or state value */
#define SQ_FLAG_RANGE 4     /* a scale or fp16 value above the fp16 range */
#define SQ_FLAG_TIMEOUT 8   /* a kernel stopped waiting for a bulk copy */

/*
 * Layout of one pool. [SQ-E] lifetime-aware allocation paragraph: a unit is a whole head
 * (Qwen / GDN) or one key row (Kimi / KDA), and its width is fixed offline; the pool holds
 * one state per concurrent request plus spare slots ([SQ-E], state-pool paragraph).
 *   d_k, d_v     multiples of 16, at most 128.
 *   fit_iters    alternations of the row/column max-abs scale fit, 1..8 (2 by default).
 *   window       1: requantize after every token. W > 1: requantize after every W tokens,
 *                holding the update at full precision in between ([LQ-N]).
 *   n_outliers   per head, the entries of largest |S| kept in fp16 at each requantization
 *                ([LQ-N], "compensation tokens"); 0..64, only with window > 1.
 */
typedef struct {
  int32_t n_slots, n_heads, d_k, d_v;
  int32_t unit;     /* sq_unit */
  int32_t gate;     /* sq_gate */
  int32_t io_dtype; /* sq_io_dtype */
  int32_t fit_iters;
  int32_t window;
  int32_t n_outliers;
} sq_layout;

typedef struct sq_pool sq_pool;

/*
 * Packed format ([SQ-E] limitations paragraph: compressed values packed densely; efficiency
 * paragraph: the compression ratio follows from the storage format).
 *   bits_map (host): [n_heads] for SQ_UNIT_HEAD, [n_heads][d_k] for SQ_UNIT_KEY_ROW; values
 *     2, 4, 6 or 8, or 16 for an FP16 pivot unit ([SQ-E]: a few high-risk units stay FP16).
 *   pivot_mask (host, may be NULL): same shape; nonzero exactly where bits_map is 16.
 * A quantized head block is r16[d_k] | c16[d_v] | rows | outliers: fp16 row and column
 * scales, then row i as a little-endian bit stream in which element j holds the offset code
 * code + 2^(b-1) (code in [-(2^(b-1)-1), 2^(b-1)-1]) at bits [j*b, (j+1)*b); a pivot row is
 * the same stream of fp16 bit patterns. A pivot head (head units) is its fp16 matrix. Each
 * head block is padded to 16 bytes; a slot is the heads in order. With window > 1 a side
 * region follows the slots (per slot: the token count of the open window and the
 * full-precision update held as low-rank factors).
 *
 * sq_pool_required_bytes: size in bytes of the device buffer a pool with this layout needs.
 */
SQ_API sq_status sq_pool_required_bytes(const sq_layout* layout, const uint8_t* bits_map,
                                 const uint8_t* pivot_mask, size_t* bytes);

/* Create a pool over a caller-owned device buffer (at least sq_pool_required_bytes, 256-byte
 * aligned; contents are not touched until a quantize or step call). bits_map and pivot_mask
 * are copied. On success *out receives the handle. Must be called with the buffer's device
 * current. */
SQ_API sq_status sq_state_pool_create(const sq_layout* layout, const uint8_t* bits_map,
                               const uint8_t* pivot_mask, void* device_buf,
                               size_t device_buf_bytes, sq_pool** out);

/* Free the handle and its device tables (not the caller's buffer). NULL is accepted. */
SQ_API sq_status sq_state_pool_destroy(sq_pool* pool);

/* Geometry of a pool: bytes per slot, byte offset of each head block within a slot
 * (head_offsets: host array of n_heads, may be NULL), and bytes per slot of the windowed side
 * region (0 when window == 1; it starts at n_slots * slot_bytes). */
SQ_API sq_status sq_pool_info(const sq_pool* pool, size_t* slot_bytes, size_t* head_offsets,
                       size_t* side_bytes_per_slot);

/* Quantize dense fp32 states into slots (cold start; [SQ-E] experimental setup uses the FP32
 * state as baseline, so a pool is filled from fp32 states).
 *   slot_idx (device) [n]; S (device) fp32 [n][n_heads][d_k][d_v].
 * Fits the dual-axis scales, rounds pivots and outliers to fp16, packs, and (window > 1)
 * closes the slot's window. */
SQ_API sq_status sq_quantize_fp32_state(sq_pool* pool, const int32_t* slot_idx, int32_t n,
                                 const float* S, void* stream);

/* Dequantize slots to dense fp32: S_out[i][j] = fl32(code * r16_i * c16_j); pivots and
 * outliers as their fp16 values. With window > 1 this is the frozen state (the open window's
 * update is not included).
 *   slot_idx (device) [n]; S_out (device) fp32 [n][n_heads][d_k][d_v]. */
SQ_API sq_status sq_dequantize_state(sq_pool* pool, const int32_t* slot_idx, int32_t n,
                              float* S_out, void* stream);

/*
 * One decode step for `batch` requests ([SQ-E] experimental-setup paragraph: the state is
 * unpacked, updated and written back by one fused kernel at every decode step, and the two
 * scales are refit on the updated state at every step; [SQ-E] paragraph introducing the gated
 * Delta rule). For request b, head h, with M the state of slot slot_idx[b]:
 *   S' = D M  (D = alpha I, or diag(alpha_i) for SQ_GATE_DIAG);  u = S'^T k;
 *   b = beta (v - u);  M_new = S' + k b^T;  out = M_new^T q;
 * then M_new's row and column scales are refit and it is requantized in place.
 *   slot_idx (device) int32 [batch]
 *   q, k (device) [batch][n_heads][d_k], v (device) [batch][n_heads][d_v], in io_dtype
 *   alpha (device) fp32 [batch][n_heads] (scalar gate) or [batch][n_heads][d_k] (diagonal)
 *   beta (device) fp32 [batch][n_heads]
 *   out (device) fp32 [batch][n_heads][d_v]
 * With window > 1 the frozen block is only read; the update goes to the side region, and the
 * block is requantized after the W-th token of the window ([LQ-N]).
 */
SQ_API sq_status sq_decode_step(sq_pool* pool, const int32_t* slot_idx, int32_t batch, const void* q,
                         const void* k, const void* v, const float* alpha, const float* beta,
                         float* out, void* stream);

/*
 * The decode step split over two streams, for comparison with the fused sq_decode_step ([SQ-E]
 * experimental-setup paragraph: the scale fit and compression run on a side stream). On
 * `stream` one kernel unpacks, updates and writes out (as sq_decode_step) and writes the updated
 * fp32 state to `staging`; on `side_stream`, after it, the fit and requantization of
 * sq_quantize_fp32_state turn `staging` back into the slots. Every later call on this pool
 * (any entry point, any stream) first waits for that requantization on the GPU.
 *   staging (device, caller-owned scratch) fp32 [batch][n_heads][d_k][d_v], 16-byte aligned;
 *   the caller must not touch it until the side stream's work has finished.
 * Other arguments as sq_decode_step; window == 1 pools only (SQ_ERR_UNSUPPORTED otherwise).
 * A request-head with a non-finite input keeps its bytes (SQ_FLAG_NONFINITE). */
SQ_API sq_status sq_decode_step_split(sq_pool* pool, const int32_t* slot_idx, int32_t batch,
                                      const void* q, const void* k, const void* v,
                                      const float* alpha, const float* beta, float* out,
                                      float* staging, void* stream, void* side_stream);

/*
 * sq_decode_step_split for callers that cannot allocate device memory (a serving engine that
 * hands all device memory to its own allocator at start-up, a host whose memory plan is fixed
 * before the first request): the staging state lives in a static device array that libsq
 * owns, 32 MiB on every GPU that loads the library, held until the process exits. This entry
 * point allocates nothing. The pages have no counterpart: it only serves such callers.
 *   batch * n_heads * d_k * d_v * 4 bytes must fit in 32 MiB (512 request-heads at
 *   d = 128); larger batches return SQ_ERR_INVALID_ARG.
 * Both halves (update, then refit + requantize) run on `stream`. Every call looks up the
 * array's device address on the current device (no address is cached, so a context torn down
 * and created again is harmless); the first call on a device may load the library's module
 * there, so make that first call before any stream capture. All calls in the process share
 * the one array and it keeps the last call's contents (nothing in it needs to start at zero:
 * each call writes every tile it reads back); calls that can run at the same time on the GPU
 * (different streams, different pools) race on it and must be ordered by the caller. Other
 * arguments and errors as sq_decode_step_split. */
SQ_API sq_status sq_decode_step_split_static(sq_pool* pool, const int32_t* slot_idx,
                                             int32_t batch, const void* q, const void* k,
                                             const void* v, const float* alpha,
                                             const float* beta, float* out, void* stream);

/*
 * n_tokens consecutive tokens of each request in one call (prefill, or speculative decode into a
 * quantized state): the state is read from the pool once, advanced through the tokens in fp32 on
 * chip, and refit and requantized once, after the last token. Each token's update and output
 * are those of sq_decode_step ([SQ-E] gated Delta rule paragraph); quantizing only after the
 * last of them is the window-end requantization of [LQ-N] with W = n_tokens and no
 * compensation entries. n_tokens == 1 is sq_decode_step. Pools with window == 1 only
 * (SQ_ERR_UNSUPPORTED otherwise); 1 <= n_tokens <= 16 (SQ_ERR_INVALID_ARG otherwise).
 *   slot_idx (device) int32 [batch]
 *   q, k (device) [batch][n_heads][n_tokens][d_k], v (device) [batch][n_heads][n_tokens][d_v]
 *   alpha (device) fp32 [batch][n_heads][n_tokens] or [batch][n_heads][n_tokens][d_k]
 *   beta (device) fp32 [batch][n_heads][n_tokens]
 *   out (device) fp32 [batch][n_heads][n_tokens][d_v]
 * Pointers 16-byte aligned. A request with a non-finite input is skipped (its slot unchanged,
 * its outputs NaN, SQ_FLAG_NONFINITE set). */
SQ_API sq_status sq_decode_chunk(sq_pool* pool, const int32_t* slot_idx, int32_t batch,
                                 int32_t n_tokens, const void* q, const void* k, const void* v,
                                 const float* alpha, const float* beta, float* out, void* stream);

/* Windowed pools: fold each listed slot's open window into its quantized block now and close
 * the window (no-op for a closed window). slot_idx (device) [n]. */
SQ_API sq_status sq_window_flush(sq_pool* pool, const int32_t* slot_idx, int32_t n, void* stream);

/*
 * Row-impact weighting of the dual-axis fit ([SQ-E] experimental-setup paragraph: the row scale
 * weighs the row's current size together with its impact score, and the column scale
 * penalizes reconstruction error more in high-impact rows; the impact scores are fixed
 * offline, [SQ-E] row-impact score paragraph). impact (host) fp32 [n_heads][d_k], every entry
 * > 0 and finite, or NULL to remove the weighting. Reading taken (the pages print no
 * formula): row i of head h counts in the column passes of every refit of the pool (decode
 * step, chunk, window end, quantize, flush) with the weight omega_i = min(1, sqrt(impact_i /
 * mean impact of head h)) (double precision, rounded to fp32), i.e. w_i = omega_i / (r_i Q_i),
 * so the column scales follow the high-impact rows; after the last alternation every row with
 * omega_i < 1 widens its scale to fit the final column scales, so no code leaves [-Q, Q].
 * Each row scale otherwise follows the row's own size. Equal impacts give the plain fit.
 * Synchronizes the device; allocates a small device table on first use. SQ_ERR_INVALID_ARG for
 * a bad entry (the previous weighting stays). */
SQ_API sq_status sq_pool_set_row_impact(sq_pool* pool, const float* impact);

/* Synchronize the device, read and clear the status word (*device_flag, may be NULL).
 * Returns SQ_OK, SQ_ERR_DEVICE_FLAG or SQ_ERR_TIMEOUT. */
SQ_API sq_status sq_pool_status(sq_pool* pool, int32_t* device_flag);

/*
 * Offline width allocation (host; no device work). [SQ-E] lifetime-aware allocation paragraph:
 * under a fixed average bit budget, units whose error is large and long-lived get more bits,
 * chosen from a score combining each unit's reconstruction distortion with the mean lifetime of
 * its memory; a few high-risk units stay FP16 (pivots). The Block-GTQ page's greedy rule (the
 * next bits to the unit whose error they reduce most) decides the widths.
 *   n_units           units (heads for SQ_UNIT_HEAD, H * d_k key rows for SQ_UNIT_KEY_ROW)
 *   variance (host)   [n_units] variance of the unit's state entries, >= 0, finite
 *   lifetime (host)   [n_units] mean lifetime of the unit's memory in steps, >= 0, finite
 *                     (1 / (1 - mean gate) for a gate keeping a fraction alpha per step)
 *   avg_bits          mean width of the non-pivot units, in [2, 8]
 *   n_pivots          units kept FP16: the largest risks lifetime * variance (ties: lower index)
 *   bits_map (host)   [n_units] out: 2, 4, 6, 8, or 16 for a pivot (the pool's bits_map)
 *   pivot_mask (host) [n_units] out, may be NULL: 1 where bits_map is 16
 * Non-pivot units start at 2 bits and receive floor((avg_bits - 2) n' / 2) steps of 2 bits
 * (n' non-pivot units; widths at most 8), each to the unit with the largest reduction of
 * lifetime * variance * 2^(-2 b) (ties: lower index); this minimizes the total of that score.
 * Returns SQ_ERR_INVALID_ARG for a bad count, budget or statistic (nothing written). */
SQ_API sq_status sq_allocate_bits(int32_t n_units, const float* variance, const float* lifetime,
                                  float avg_bits, int32_t n_pivots, uint8_t* bits_map,
                                  uint8_t* pivot_mask);

/* Text of a status code (static storage). */
SQ_API const char* sq_status_string(sq_status status);

/* As sq_decode_step (window == 1 only), and also writes the fp32 state after the update and
 * before requantization to s_new (device) fp32 [batch][n_heads][d_k][d_v]. For tests. */
SQ_API sq_status sq_debug_decode_step_fp32(sq_pool* pool, const int32_t* slot_idx, int32_t batch,
                                    const void* q, const void* k, const void* v,
                                    const float* alpha, const float* beta, float* out,
                                    float* s_new, void* stream);

/*
 * Test hook for the bounded waits (the pages have no counterpart: it exists so that the
 * timeout path can be exercised without faulting anything). Every later sq_decode_step (the
 * per-step and the windowed kernel), sq_decode_chunk and sq_debug_decode_step_fp32 on this pool
 * gives up a wait on a bulk copy after
 * wait_limit_ns nanoseconds of the GPU's global timer (0 restores the default, 1 s), and, with
 * extra_expected_bytes > 0 (at most 4096), has each copy's barrier expect that many bytes more
 * than the copies bring, so that every wait runs out. A kernel whose wait runs out sets
 * SQ_FLAG_TIMEOUT (sq_pool_status then returns SQ_ERR_TIMEOUT), lets its own copies land, frees
 * its tensor memory and returns; the items it did not reach keep their slot bytes (and their
 * window side state) and their output rows are not written. Host only; nothing is enqueued. Call with 0, 0 to restore normal
 * operation. SQ_ERR_INVALID_ARG for a NULL pool or more than 4096 extra bytes. */
SQ_API sq_status sq_debug_set_wait(sq_pool* pool, uint64_t wait_limit_ns,
                                   uint32_t extra_expected_bytes);

/*
 * Test hook of the decode step's last column pass (the pages have no counterpart: it exists to
 * check an exactness claim). The decode kernel skips the last column pass of the scale fit
 * when a bound proves it cannot change any fp16 column scale (the multipliers of the last row
 * pass moved less than every column scale's distance to an fp16 rounding boundary allows); the
 * stored bytes are then exactly those of the full pass. full_fit = 1 makes every later decode
 * step of this pool run the full pass, so a test can compare the two bit for bit; 0 restores
 * the default. Host only. SQ_ERR_INVALID_ARG for a NULL pool or another value. */
SQ_API sq_status sq_debug_set_full_fit(sq_pool* pool, int32_t full_fit);

#ifdef __cplusplus
}
#endif
#endif /* SQ_H */
