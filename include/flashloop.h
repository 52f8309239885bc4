/*
 * flashloop.h -- C ABI of libflashloop_b200.so, the B200 (sm_100a) decode path of
 * FlashLoop: single-query attention over a cross-loop INT4 KV cache with
 * loop-aware sparse attention in late loops.
 *
 * Sources (page title, then section):
 *   [PyPI]    "flashloop 0.1.0" project description, "Configuration and supported scope":
 *             four loops, dense loops 1-2, 25 % / 10 % token retention in loops 3-4,
 *             10 % key retention in sparse late loops, 4-bit K/V with group size 64,
 *             a 64-token BF16 tail; head dimension 128, equal query/KV head counts.
 *   [Project] "FlashLoop: Fast and Memory-Efficient Looped Transformers via Lazy
 *             Updates" project page, "The Method": Step 01 (inactive tokens reuse the
 *             preceding loop's KV), Step 02 (recompute a few columns chosen from the
 *             preceding loop and keep their global probability mass), Step 03 (a
 *             quantised loop-1 base plus per-loop residuals against the reconstructed
 *             preceding state), and the closing paragraph on compact gather buffers and
 *             fusing KV updates into the attention kernel.
 *   [Guide]   flozi.net "FlashLoop: store changes between repeated passes", section 3:
 *             per-channel (post-RoPE) key groups, per-token value groups, residuals of
 *             active tokens only; sparse loops are a rank-K correction of the previous
 *             loop's output.  Section 4: the "Per-loop KIVI4" ablation (full KV states
 *             quantised per loop instead of residuals) and the 2-bit residual row of
 *             Figure 5; the project page's "Experiments" caption of Figure 5 (residual
 *             precision varied).
 *
 * Conventions for every entry point
 *   - All data pointers are DEVICE pointers owned by the caller.  The library never
 *     allocates or frees device memory.  Its only process-wide state is (a) per-device
 *     caches filled on a device's first call (its SM count, the kernels' shared-memory
 *     attributes, the address of the array below, and the stream fl_decode_step_io copies
 *     its inputs on), each guarded so that host threads making their first call at once
 *     neither race nor repeat it, and (b) the one static device array of
 *     fl_decode_attn_sparse_noalloc (FL_NOALLOC_SCRATCH_BYTES per device that loads the
 *     library).  The caches do not survive cudaDeviceReset or a context teardown: reload
 *     the library after one.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call only
 *     enqueues work and returns (on `stream`, and for fl_decode_step_io's input copy on
 *     the library's copy stream, ordered after `stream`'s earlier work and before the
 *     readers that need it); calls on one cache must be stream-ordered.
 *   - BF16 tensors are passed as uint16_t bit patterns.
 *   - Arguments are validated on the host before any launch: a bad value returns
 *     FL_ERR_INVALID / FL_ERR_UNSUPPORTED / FL_ERR_WORKSPACE and enqueues nothing.
 *     A failed launch returns FL_ERR_CUDA.  Data errors found on the device (rows
 *     out of order, sets that do not nest, a selected index out of range) are
 *     recorded in the cache's status words, read with fl_read_status(); kernels
 *     never trap, and every wait inside a kernel (the readers' mbarrier hand-offs) is
 *     bounded: after 2 s of device time it records FL_DEV_TIMEOUT and the kernel drains.
 *   - Numbers: codes, scales and zero points are exact (the quantiser below, fp32
 *     with one IEEE rounding per operation); attention runs in fp32 and returns fp32.
 *
 * The 4-bit quantiser (a group of values x):
 *     s = fp16_rn(fp32_rn(max - min) / 15),  z = fp16_rn(min),
 *     code = clamp(rint_even(fp32_rn(x - z) / s), 0, 15)   (0 when s == 0),
 *     x_hat = fma(code, s, z).
 *   Key groups are (64-token block, channel) in the base and (64 consecutive
 *   slots of one encode call, channel) in a residual store; value groups are
 *   (token or slot, 64-channel half).
 *
 * Codecs of the loop r >= 2 stores (fl_dims.codec; the base is always the 4-bit
 * quantiser of loop-1 K/V):
 *   FL_CODEC_RESIDUAL_INT4  the method: store r holds E = X^(r) - X_hat^(r-1) of the
 *                           rows active in loop r, 4-bit; a token's loop-r state is the
 *                           base plus its stores 2 .. min(r, depth), added in loop order.
 *   FL_CODEC_FULL_INT4      per-loop KIVI4: store r holds X^(r) itself, 4-bit, same
 *                           groups; a token's loop-r state is its store min(r, depth)
 *                           alone (the base when that is 1).
 *   FL_CODEC_RESIDUAL_INT2  residuals as in the method with 2-bit codes:
 *                           s = fp16_rn(fp32_rn(max - min) / 3), code = clamp(.., 0, 3),
 *                           in 5120-byte residual records (below).
 *   Every reader and encode entry point serves all three codecs; the fused tail flush
 *   (fl_decode_step_flush) writes FL_CODEC_RESIDUAL_INT4 stores only.
 *
 * Packed cache layout (one buffer of fl_cache_layout().total_bytes; every array
 * starts on a 256-byte boundary; L layers, H heads, C = capacity, T = total slots,
 * R loops; "sz" = a (scale, zero) fp16 pair stored as scale in the low half of a
 * 32-bit word).  Codes and scales live in 9216-byte GROUP RECORDS, one per 64 rows
 * of a store (a 64-token block of the base, or 64 consecutive slots of a residual
 * store):
 *     bytes [0, 8192)     64 rows x 128 B: row i = 64 B of key codes then 64 B of
 *                         value codes; code byte b holds channel 2b (low nibble) and
 *                         2b+1 (high nibble)
 *     bytes [8192, 8704)  64 x 2 value sz: row i, half h (channels 64h..64h+63)
 *     bytes [8704, 9216)  128 key sz: one per channel of the group
 *   With FL_CODEC_RESIDUAL_INT2 the residual records are 5120 bytes:
 *     bytes [0, 4096)     64 rows x 64 B: row i = 32 B of key codes then 32 B of value
 *                         codes; 32-bit word w of a part holds channels 16w .. 16w+15:
 *                         channel 16w+k (k < 8) in bits 4k..4k+1 and channel 16w+8+k in
 *                         bits 4k+2..4k+3 (so word & 0x33333333 and (word >> 2) &
 *                         0x33333333 are the two 8-channel words of the 4-bit layout)
 *     bytes [4096, 4608)  64 x 2 value sz
 *     bytes [4608, 5120)  128 key sz
 *   brec   u8  [L][H][C/64][9216]  base group records (loop 1), block b = tokens 64b..64b+63
 *   rrec   u8  [L][H][T/64][RB]    residual group records of every loop (RB = 9216, or 5120
 *                                   with 2-bit codes); loop r owns slots
 *                                   [slot_base[r], slot_base[r] + res_capacity[r])
 *   mask   u64 [L][R+1][C/64]      bit t of mask[r][b]: token 64b+t has a loop-r residual
 *   first  i32 [L][R+1][C/64]      slot (within loop r's store) of block b's first loop-r row;
 *                                   the block's rows occupy consecutive slots in token order
 *   depth  u8  [L][C]              last loop in which the token was active (1 = base only)
 *   tail_k bf16[L][R][H][64][128]  BF16 tail of loop r at index r-1
 *   tail_v bf16[L][R][H][64][128]
 *   score  f32 [L][H][C]           log2-domain score of each column from the loop that last
 *                                   computed it (tag); log2 p~_j = score_j - offset[tag_j]
 *   tag    u8  [L][H][C]
 *   offset f32 [L][H][33]          per-loop log2 normaliser
 *   sel    i32 [L][H][max_select]  selected columns S, ascending
 *   mass   f32 [L][H]              m = sum over S of p~
 *   unsel  f32 [L][H][128]         u = sum over columns not in S of p~_j * v_j (at loop tag_j)
 *   plan   i32 [L][H][max_select][P] gather plan of S, P = plan_stride = roundup(R + 2, 4):
 *                                   [0] column j, [1] tag_j | (stores << 8) where stores =
 *                                   min(loop, depth_j) for a quantised column and 0 for a tail
 *                                   column, [2] p~_j as fp32 bits, [3 + (r - 2)] the global
 *                                   residual slot of column j in loop r's store, r = 2..stores
 *   status i32 [16]                [0] first device error code (0 = none), [1] its detail,
 *                                   [2] number of device errors
 */
#ifndef FLASHLOOP_H
#define FLASHLOOP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FL_HEAD_DIM 128
#define FL_GROUP 64
#define FL_TAIL 64
#define FL_MAX_LOOPS 32
/* The selector holds every column's key of one (layer, head) in the shared memory of one
 * thread-block cluster of up to 8 CTAs. */
#define FL_MAX_SELECT_COLS 385024

typedef enum fl_status {
  FL_OK = 0,
  FL_ERR_INVALID = -1,     /* null pointer, index out of range, inconsistent sizes */
  FL_ERR_UNSUPPORTED = -2, /* a shape the kernels do not implement (head_dim != 128, group != 64, ...) */
  FL_ERR_CUDA = -3,        /* a CUDA runtime call or kernel launch failed */
  FL_ERR_WORKSPACE = -4,   /* workspace pointer null or smaller than fl_workspace_bytes() */
  FL_ERR_DEVICE = -6       /* fl_read_status: a kernel recorded a data error */
} fl_status;

/* Device error codes recorded in status[0] (status[1] holds the offending index). */
#define FL_DEV_ROWS_ORDER 1   /* encode rows not strictly ascending */
#define FL_DEV_ROWS_RANGE 2   /* encode row outside [row0, row0 + n_span) */
#define FL_DEV_NOT_NESTED 3   /* loop-r row not active in loop r-1 */
#define FL_DEV_SEL_RANGE 4    /* selected column outside [0, N) */
#define FL_DEV_TAG_RANGE 5    /* a column's loop tag outside [1, R] */
#define FL_DEV_TIMEOUT 6      /* a bounded wait for staged data ran out (the kernel returned early) */
#define FL_GROUP_RECORD 9216  /* bytes of one group record */
#define FL_GROUP_RECORD_INT2 5120  /* bytes of one 2-bit residual group record */

/* fl_dims.codec: what the loop r >= 2 stores hold (see the codec notes above). */
#define FL_CODEC_RESIDUAL_INT4 0
#define FL_CODEC_FULL_INT4 1
#define FL_CODEC_RESIDUAL_INT2 2

typedef struct fl_dims {
  int32_t layers;      /* L >= 1 */
  int32_t heads;       /* H >= 1 (MHA: query heads == KV heads) */
  int32_t head_dim;    /* must be 128 */
  int32_t group;       /* must be 64 */
  int32_t loops;       /* R in [1, 32] */
  int32_t capacity;    /* max columns N = quantised + tail; a positive multiple of 64 */
  int32_t max_select;  /* capacity of the selected-column list per (layer, head), >= 1 */
  int32_t res_capacity[FL_MAX_LOOPS + 1]; /* slots of loop r's residual store, r = 2..R, multiples of 64 */
  int32_t codec;       /* FL_CODEC_*: 0 (zero-initialised) is the method's INT4 residuals */
} fl_dims;

typedef struct fl_layout {
  uint64_t total_bytes;
  uint64_t brec, rrec;
  uint64_t mask, first, depth;
  uint64_t tail_k, tail_v;
  uint64_t score, tag, offset;
  uint64_t sel, mass, unsel, plan;
  uint64_t status;
  /* bytes from one layer to the next inside each array above (same order) */
  uint64_t layer_stride[14];
  int32_t plan_stride;                 /* int32 words per plan entry */
  int32_t slot_base[FL_MAX_LOOPS + 1]; /* first global slot of loop r's residual store */
  int32_t total_slots;                 /* T */
} fl_layout;

/* Library version string. */
const char* fl_version(void);

/* Human-readable name of a status code (static storage). */
const char* fl_status_string(fl_status st);

/* Byte offsets of every cache array for `dims` (host-only, no CUDA call).
 * Returns FL_ERR_INVALID / FL_ERR_UNSUPPORTED for bad dims. */
fl_status fl_cache_layout(const fl_dims* dims, fl_layout* out);

/* Zero the whole cache buffer (`cache` has fl_cache_layout().total_bytes) on `stream`. */
fl_status fl_cache_init(const fl_dims* dims, void* cache, void* stream);

/* Workspace the readers need for split-K partials and their completion counters: room for
 * every dense launch and for every sparse launch with k_sel <= max_select (a sparse CTA
 * holds at most 1024 / plan_stride selected columns, so large k_sel at many loops takes
 * more than the usual 256 partials per head). */
size_t fl_workspace_bytes(const fl_dims* dims);

/* Host-only (no CUDA call): the number of split-K partitions per head the sparse reader
 * of loop `loop` (2..R) uses for k_sel (1..max_select) selected columns on a device with
 * `sm_count` SMs, into *splits; *capacity (may be NULL) receives the partials per head
 * a workspace of fl_workspace_bytes(dims) holds.  *splits <= *capacity for every valid
 * k_sel, and every CTA's share of the gather plan fits its shared-memory copy.
 * FL_ERR_INVALID for out-of-range arguments. */
fl_status fl_sparse_splits(const fl_dims* dims, int32_t loop, int32_t k_sel, int32_t sm_count, int32_t* splits,
                           int32_t* capacity);

/* Zero the workspace counters; required once before the first reader call. */
fl_status fl_workspace_init(const fl_dims* dims, void* ws, size_t ws_bytes, void* stream);

/* Copy `n_rows` BF16 rows [H][n_rows][128] (head stride `head_stride` elements) into
 * rows [row0, row0 + n_rows) of layer `layer`'s loop-`loop` tail.  Used to load the
 * prompt's last 1..64 columns.  0 <= row0, row0 + n_rows <= 64. */
fl_status fl_write_tail(const fl_dims* dims, void* cache, int32_t layer, int32_t loop,
                        int32_t row0, int32_t n_rows, const uint16_t* k, const uint16_t* v,
                        int64_t head_stride, void* stream);

/* [Project] Step 03 base; [Guide] section 3.  Quantise loop-1 keys/values of tokens
 * [row0, row0 + n_rows) (both multiples of 64) into the base.  k, v: BF16
 * [H][n_rows][128] with `head_stride` elements between heads (row i = token row0 + i).
 * Sets depth = 1 and clears every loop's residual mask/first entries for those blocks. */
fl_status fl_encode_base(const fl_dims* dims, void* cache, int32_t layer, int32_t row0,
                         int32_t n_rows, const uint16_t* k, const uint16_t* v,
                         int64_t head_stride, void* stream);

/* [Project] Step 01 + Step 03; [Guide] section 3.  Store loop-`loop` (2..R) residuals
 * of the active tokens `rows` (device int32, strictly ascending, inside
 * [row0, row0 + n_span), each active in loop `loop`-1 as well: the sets nest) against the reconstructed
 * loop-(loop-1) state.  row0 and n_span are multiples of 64 and cover whole blocks that
 * are already in the base; the call owns those blocks' loop-`loop` metadata (cleared,
 * then rebuilt).  Rows go to slots [slot0, slot0 + n_rows) of the loop's store; slot0
 * is a multiple of 64 and slot0 + n_rows <= res_capacity[loop].  Inputs are BF16
 * [H][.][128]: with `compact` = 1 row i of k/v is token rows[i]; with `compact` = 0
 * it is token row0 + i.  n_rows may be 0 (clears the blocks' metadata only).
 * Codecs (fl_dims.codec): FL_CODEC_FULL_INT4 stores X^(loop) itself instead of the
 * residual; FL_CODEC_RESIDUAL_INT2 quantises the residual to 2-bit codes in the 5120-byte
 * records. */
fl_status fl_encode_residual(const fl_dims* dims, void* cache, int32_t layer, int32_t loop,
                             int32_t row0, int32_t n_span, int32_t slot0,
                             const int32_t* rows, int32_t n_rows,
                             const uint16_t* k, const uint16_t* v, int64_t head_stride,
                             int32_t compact, void* stream);

/* [Project] Step 02 (dense loops); [PyPI] "dense loops 1-2".  Full single-query
 * attention of loop `loop` over N = n_q + n_tail columns (n_q a multiple of 64,
 * n_tail in [1, 64]): keys/values are the base plus the column's residuals of loops
 * 2..loop, or the loop's BF16 tail row.  q: BF16 [H][128]; o: fp32 [H][128]
 * (softmax(q K^T / sqrt(128)) V).  If k_new/v_new (BF16 [H][128]) are non-NULL they
 * are the current token's loop-`loop` key/value: they are used as column N-1 and
 * stored into tail row n_tail-1.  With keep_scores != 0 every column's score and tag
 * (and the loop's offset) are written for the selector. */
fl_status fl_decode_attn_dense(const fl_dims* dims, void* cache, int32_t layer, int32_t loop,
                               int32_t n_q, int32_t n_tail, const uint16_t* q,
                               const uint16_t* k_new, const uint16_t* v_new, float* o,
                               int32_t keep_scores, void* ws, size_t ws_bytes, void* stream);

/* [Project] Step 02; [Guide] section 3.  Prepares sparse loop `loop` for layers
 * [layer0, layer0 + n_layers) and every head: S = the k_sel columns of largest p~ (the
 * distribution the preceding loop left: scores/tags/offsets), ties to the smaller
 * index, written ascending; the selected mass m = sum over S of p~; and the gather
 * plan of S (its layout is above).  N = n_q + n_tail <= FL_MAX_SELECT_COLS and
 * 1 <= k_sel <= min(N, max_select); 2 <= loop <= R. */
fl_status fl_select_topk(const fl_dims* dims, void* cache, int32_t layer0, int32_t n_layers,
                         int32_t loop, int32_t n_q, int32_t n_tail, int32_t k_sel, void* stream);

/* [Project] Step 02; [Guide] section 3.  Sparse attention of loop `loop` over the
 * columns fl_select_topk chose for this loop (same k_sel, n_q, n_tail):
 *   o = u + m * softmax_S(q K_S^T / sqrt(128)) V_S,
 *   u = o_prev - sum over S of p~_j v_j   (v_j at the loop that last computed column j),
 * i.e. u is the unselected columns' contribution to the preceding loop's output o_prev
 * (fp32 [H][128]).  Keys/values are those of loop `loop`.  The pass also records m and u
 * in the cache and splices the state: score/tag of j in S become this loop's, and
 * offset[loop] makes p~_j = m * softmax_S(.)_j.  q, k_new, v_new, o as in
 * fl_decode_attn_dense. */
fl_status fl_decode_attn_sparse(const fl_dims* dims, void* cache, int32_t layer, int32_t loop,
                                int32_t n_q, int32_t n_tail, int32_t k_sel, const uint16_t* q,
                                const uint16_t* k_new, const uint16_t* v_new, const float* o_prev,
                                float* o, void* ws, size_t ws_bytes, void* stream);

/* Largest scratch of fl_decode_attn_sparse_noalloc, in bytes (a static device array of
 * the library). */
#define FL_NOALLOC_SCRATCH_BYTES (1u << 20)

/* fl_decode_attn_sparse for callers that cannot allocate device memory -- an engine
 * whose allocator is frozen after start-up, or a host ABI with no way to hand over a
 * workspace.  Same arguments, validation and results as fl_decode_attn_sparse except
 * that there is no ws/ws_bytes: the reader's scratch (one ticket per head, which this
 * call clears on `stream` before the launch, and heads x splits x 1040 bytes of split
 * partials) lives in a file-scope device array of FL_NOALLOC_SCRATCH_BYTES owned by the
 * library.  Nothing is allocated by this call.
 *   - The first call on a device looks the array's address up (cudaGetSymbolAddress,
 *     with that device current) and caches it; make that first call before any stream
 *     capture that is to contain this call.
 *   - The array keeps its contents between calls and is shared by every caller in the
 *     process on that device: calls that can overlap (different streams, threads)
 *     race on it and must be serialised by the caller.
 *   - FL_ERR_UNSUPPORTED when the scratch would exceed FL_NOALLOC_SCRATCH_BYTES (many
 *     heads or a large k_sel); use fl_decode_attn_sparse with a workspace then.  The
 *     scratch is sized from the split count this very call launches with
 *     (fl_sparse_splits with the device's SM count).
 *   - The cached address does not survive cudaDeviceReset or a context teardown.
 * The FlashLoop pages have no counterpart: this is a deployment convenience of this
 * library, not a step of the method. */
fl_status fl_decode_attn_sparse_noalloc(const fl_dims* dims, void* cache, int32_t layer, int32_t loop,
                                        int32_t n_q, int32_t n_tail, int32_t k_sel, const uint16_t* q,
                                        const uint16_t* k_new, const uint16_t* v_new,
                                        const float* o_prev, float* o, void* stream);

/* Native executor of one decode step for layers [0, L) in loop-major order (every
 * layer runs loop r before any layer runs loop r+1), for loops loop_first..loop_last:
 * loops up to dense_loops call the dense reader (the last dense loop keeps scores);
 * every later loop first selects k_sel columns for all layers in one launch
 * (fl_select_topk) and then runs each layer's sparse reader with o_prev = that
 * layer's output of the previous loop (for the 4-bit residual codec and loops <= 8,
 * one persistent launch covers every layer, then one combine launch).  Same arguments
 * and semantics as the individual calls; validated once.
 *   q, k_new, v_new: BF16 [R+1][L][H][128] (slice r = loop r, slice 0 unused;
 *                    k_new/v_new may be NULL)
 *   o: fp32 [R+1][L][H][128]   (o[r] = loop r's outputs; o[loop_first-1] must hold the
 *                               previous loop's outputs when loop_first is sparse)
 *   events: NULL, or 2*R+1 cudaEvent_t; events[0] is recorded before loop_first, and
 *           for each loop r in range events[2r-1] after its selection (right away for a
 *           dense loop) and events[2r] after its readers. */
fl_status fl_decode_step(const fl_dims* dims, void* cache, int32_t n_q, int32_t n_tail,
                         int32_t dense_loops, int32_t k_sel, int32_t loop_first, int32_t loop_last,
                         const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new, float* o,
                         void* ws, size_t ws_bytes, void* const* events, void* stream);

/* [Project] "The Method", closing paragraph (KV updates and quantisation fused into the
 * attention kernel); Step 03; Step 01.  The 64-row tail group that a decode step
 * quantises while it attends over it (fl_decode_step_flush). */
typedef struct fl_flush {
  /* active[r], r = 2..R: bit i set when tail row i (token n_q + i) enters loop r's
   * residual store.  Must nest: active[r] is a subset of active[r-1], and every row is in
   * the base (entries 0 and 1 are ignored). */
  uint64_t active[FL_MAX_LOOPS + 1];
  /* HOST int32 [layers][FL_MAX_LOOPS + 1]: slot0[l * (FL_MAX_LOOPS + 1) + r] is the first
   * slot of loop r's residual store that layer l's group takes (a multiple of 64, with
   * slot0 + popcount(active[r]) <= res_capacity[r]; unused when active[r] is 0). */
  const int32_t* slot0;
} fl_flush;

/* fl_decode_step that also moves a full BF16 tail (n_tail == 64, n_q + 64 <= capacity)
 * into the INT4 stores as the step runs, with no encode launches.  flush == NULL is
 * exactly fl_decode_step.  Each reader of a loop r in loop_first..loop_last, dense or
 * sparse, first attends over the tail as BF16 (the
 * outputs are those of fl_decode_step) and then writes, for every head, store r of the
 * 64 tail rows [n_q, n_q + 64): for r = 1 the base group record (depth 1, the block's
 * residual mask/first entries cleared), for r >= 2 the residual record of the rows in
 * active[r] at slot0[l][r] (mask = active[r], first = slot0 or -1, depth = r).  The bytes
 * equal those of fl_encode_base / fl_encode_residual on the same rows after the step;
 * the new token (tail row 63) is taken from k_new / v_new when they are given.  A step
 * split over several calls (loop ranges) passes the same `flush` to each and must run
 * its loops in order.  After loop R the caller's timeline moves on: n_q += 64, n_tail
 * = 0.  Validated on the host (nesting, slot alignment and capacity per layer). */
fl_status fl_decode_step_flush(const fl_dims* dims, void* cache, int32_t n_q, int32_t n_tail,
                               int32_t dense_loops, int32_t k_sel, int32_t loop_first,
                               int32_t loop_last, const uint16_t* q, const uint16_t* k_new,
                               const uint16_t* v_new, float* o, void* ws, size_t ws_bytes,
                               void* const* events, const fl_flush* flush, void* stream);

/* fl_decode_step_flush fed from and returning to HOST memory in one call, for callers whose
 * step inputs arrive on the host: copies q, k_new, v_new of loops loop_first..loop_last from
 * host_qkv (BF16 [3][loop_last - loop_first + 1][L][H][128]: q, then k_new, then v_new) into
 * the device array qkv (BF16 [3][R+1][L][H][128], the same three arrays fl_decode_step takes
 * as q, k_new, v_new) with one 2-D copy, runs those loops, and copies o of those loops
 * (fp32 [loop_last - loop_first + 1][L][H][128]) from the device array o ([R+1][L][H][128])
 * to host_o -- nothing waited for on the host.  The input copy runs on a stream the library
 * creates once per device, after all work enqueued on `stream` before the call and beside
 * the first loop's selection (which reads no query); the first reader waits for it, and the
 * output copy follows the last loop on `stream`.  Host buffers should be pinned
 * (page-locked) for the copies to be asynchronous; read host_o after synchronising
 * `stream`.  Calls from several host threads share the copy stream (their copies run one
 * after another).  flush as in fl_decode_step_flush (NULL: none).  Arguments are validated
 * before anything is enqueued. */
fl_status fl_decode_step_io(const fl_dims* dims, void* cache, int32_t n_q, int32_t n_tail, int32_t dense_loops,
                            int32_t k_sel, int32_t loop_first, int32_t loop_last, uint16_t* qkv, const uint16_t* host_qkv,
                            float* o, float* host_o, void* ws, size_t ws_bytes, void* const* events,
                            const fl_flush* flush, void* stream);

/* [Project] Step 01; [Guide] section 3 (cross-loop token-sparse updates: after the dense
 * early loops each loop ranks the tokens updated in the previous loop by normalized
 * hidden-state change and keeps a top-k subset, so the active sets nest).  A_r from
 * A_{r-1}: for the n_rows candidate tokens `rows` (device int32, strictly ascending:
 * A_{r-1}) compute
 *     keys[i] = ||h_cur[j] - h_prev[j]||^2 / ||h_prev[j]||^2,   j = rows[i]
 * (fp64 sums of the exactly widened BF16 values; 0 when both norms are 0, +inf when only
 * the previous state is 0), and write the k candidates with the largest key -- ties to
 * the lower token -- to rows_out in ascending token order (A_r, ready to be the `rows` of
 * fl_encode_residual).  Ranking by the squared ratio is ranking by the ratio.
 *   h_prev: the state entering loop r-1 (h^(r-2)); h_cur: the state leaving it (h^(r-1));
 *           BF16 [n_tokens][d_model], rows `row_stride` elements apart; 16-byte aligned,
 *           d_model and row_stride multiples of 8, d_model <= row_stride.
 *   keys: device fp64 [n_rows], caller-owned: receives every candidate's key (it is also
 *         the selector's scratch).  rows_out: device int32 [k].  0 <= k <= n_rows.
 *   status: NULL or device int32[3] (first error code, detail, count) receiving
 *           FL_DEV_ROWS_RANGE for a candidate outside [0, n_tokens) -- its key is NaN and
 *           it ranks below every valid one -- or FL_DEV_ROWS_ORDER for a candidate not
 *           above its predecessor (still ranked).
 * Two launches on `stream` (per-token change, HBM-bound; one-CTA radix select); nothing
 * is allocated. */
fl_status fl_select_active(const uint16_t* h_prev, const uint16_t* h_cur, int32_t n_tokens,
                           int32_t d_model, int64_t row_stride, const int32_t* rows, int32_t n_rows,
                           int32_t k, int32_t* rows_out, double* keys, int32_t* status, void* stream);

/* [Project] "The Method", Step 01 (only the active tokens are recomputed in a
 * token-sparse loop) and the closing paragraph (selected tokens gathered into compact
 * buffers so the work stays a regular GEMM).  Sparse prefill attention of one loop: the
 * n_act active tokens' queries attend causally over every token's key and value,
 *     o[h][i] = softmax_{j <= pos[i]}(q[h][i] . k[h][j] / sqrt(128)) v[h][j],
 * on the tensor cores (BF16 operands, fp32 accumulation; the probabilities reach the
 * value product as two BF16 terms P_hi + P_lo, about 16 significant bits, and the row sum
 * is taken in fp32).
 *   q: BF16 [heads][n_act][128] (compact, in token order; head stride q_head_stride
 *      elements); pos: device int32 [n_act], strictly ascending, in [0, n_tokens);
 *   k, v: BF16 [heads][n_tokens][128] (head stride kv_head_stride): each token's key and
 *      value in this loop (an inactive token's reused from the previous loop);
 *   o: fp32 [heads][n_act][128] (head stride o_head_stride), written for every row.
 * Rows are 128 elements apart; pointers 16-byte aligned; head strides multiples of 8.
 * status: NULL or device int32[3] receiving FL_DEV_ROWS_RANGE / FL_DEV_ROWS_ORDER for a
 * bad position (that row attends over nothing and is left unwritten) or FL_DEV_TIMEOUT
 * (a bounded wait for the tensor cores ran out).  One launch; nothing is allocated. */
fl_status fl_prefill_attn_sparse(const uint16_t* q, const int32_t* pos, int32_t n_act, const uint16_t* k,
                                 const uint16_t* v, int32_t n_tokens, int32_t heads, int64_t q_head_stride,
                                 int64_t kv_head_stride, float* o, int64_t o_head_stride, int32_t* status,
                                 void* stream);

/* Synchronise `stream`, copy the cache's status words to host `out[0..2]`, and return
 * FL_ERR_DEVICE if a kernel recorded an error (FL_OK otherwise).  With `clear` != 0
 * the words are zeroed afterwards. */
fl_status fl_read_status(const fl_dims* dims, void* cache, int32_t* out, int32_t clear,
                         void* stream);

#ifdef __cplusplus
}
#endif
#endif /* FLASHLOOP_H */
