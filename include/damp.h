/*
 * damp.h -- C ABI of libdamp: the decode step of a DAMP-style mixed-precision
 * recurrent state for Gated DeltaNet (GDN) and Kimi Delta Attention (KDA)
 * layers, on NVIDIA B200 (sm_100a).
 *
 * What the operation is (web pages, cited by title and section):
 *   - "DAMP: Decay-Aware Mixed-Precision Recurrent-State Quantization",
 *     arXiv 2608.27513v1 abstract: GDN/KDA recurrent states are FP32 by
 *     default, their update is memory-bandwidth bound; DAMP keeps high-risk
 *     channels at higher precision and the rest in INT8 (9.9 bits/value,
 *     69.1 % less state storage).  The later abstract (mlsanity.com index
 *     page) names the high-risk *key channels* and FP16, chosen offline under
 *     a fixed storage budget.
 *   - "STEPQuant: When and Where Errors Matter in Delta-Rule Recurrent State
 *     Quantization", Appendix Table C2 (one persistent decode step): (1)
 *     reconstruct the state from codes and scales or FP16 values, (2)
 *     X = D S^ + beta k (v^T - k^T D S^) with D = alpha I (GDN) or
 *     Diag(alpha) (KDA), (3) emit X^T q before requantization, (6) pack codes
 *     and scales, store the FP16 rows, keeping the old representation valid
 *     until its readers finish.
 *
 * Arithmetic (one reading each where the pages are silent):
 *   S^_ij   = fp16 value (FP16 row) | fl(code_ij * scale_i) (INT8 row)
 *   S'_ij   = fl(alpha_i * S^_ij)
 *   u_j     = sum_i fl(k_i * S'_ij), recursive pairwise order over rows
 *   delta_j = fl(v_j - u_j);  b_i = fl(beta * k_i)
 *   X_ij    = fma(b_i, delta_j, S'_ij)           (all of the above in FP32)
 *   out_j   = X^T q read out before requantization, computed through the
 *             identity X^T q = S'^T q + (q^T b) delta:  w = S'^T q and
 *             c = q^T b (FP32, any order), out_j = fma(c, delta_j, w_j).  It
 *             differs from sum_i q_i X_ij only by FP32 rounding (checked
 *             against the FP64 readout of X within 1e-4 relative / 1e-5
 *             absolute).
 *   FP16 rows: X rounded to binary16, nearest-even.
 *   INT8 rows: a = max_j |X_ij|; scale = fl(a/127); inv = fl(127/a);
 *              code = nearest integer to the exact X*inv, ties to even.
 *              a == 0 or inv == +inf -> scale 0, codes 0.
 *   FP8 rows (DAMP_FMT_FP8_ROW, the uniform FP8 baseline the DAMP v1 abstract
 *              names): E4M3 codes as the OCP 8-bit floating point
 *              specification defines them; scale = fl(a/448); inv =
 *              fl(448/a); code = the E4M3 value nearest to the FP32 product
 *              fl(X*inv), ties to even, saturating at 448; dequantized as
 *              fl(value * scale).  Same zero-row rule as INT8 rows.
 *
 * Conventions for every call:
 *   - Device memory is owned by the caller (for example allocated by
 *     PyTorch).  The library allocates no device memory.  The only host
 *     memory it owns is the damp_pool descriptor.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *     that take a stream only enqueue work and return; their results are
 *     visible after the stream is synchronised.
 *   - Arguments are checked on the host before anything is enqueued.  A
 *     negative return means nothing was enqueued (except DAMP_ERR_CUDA, which
 *     reports a failed enqueue).  Device-side conditions that the host cannot
 *     see (a slot index out of range, an internal wait that hit its bound)
 *     set bits in the pool's status word (damp_pool_get_error); kernels never
 *     trap.
 *   - Supported shapes: d_k and d_v multiples of 16 in [16, 256] (d_k may
 *     differ from d_v); 1 <= H; 1 <= n_slots; 0 <= hp_rows <= d_k.  The
 *     square shapes d_k = d_v in {16, 32, 64, 128} run the fastest kernels.
 *   - Device pointers passed for bulk copies (pool buffer, q, k, v, KDA
 *     alpha, out, FP32 states) must be 16-byte aligned.
 */
#ifndef DAMP_H
#define DAMP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes --------------------------------------------------------- */
#define DAMP_OK 0
#define DAMP_ERR_INVALID_ARGUMENT (-1) /* null pointer, bad enum, bad index map */
#define DAMP_ERR_UNSUPPORTED (-2)      /* shape outside the supported set       */
#define DAMP_ERR_MISALIGNED (-3)       /* a pointer is not 16-byte aligned      */
#define DAMP_ERR_BUFFER_TOO_SMALL (-4) /* buf_bytes < damp_pool_bytes(...)      */
#define DAMP_ERR_CUDA (-5)             /* a CUDA runtime call failed            */
#define DAMP_ERR_TIMEOUT (-6)          /* a host wait on the stream hit its limit */

/* ---- device status word bits (damp_pool_get_error) ----------------------- */
#define DAMP_EFLAG_SLOT_RANGE 1u /* a slot_idx entry >= n_slots (entry skipped) */
#define DAMP_EFLAG_TIMEOUT 2u    /* an internal pipeline wait hit its bound     */
#define DAMP_EFLAG_NONFINITE 4u  /* a unit's inputs held a NaN or an infinity
                                    (damp_decode_step_validated; unit skipped) */

/* ---- enums ----------------------------------------------------------------- */
#define DAMP_FMT_FP32 0     /* plain FP32 state (the pages' unquantized baseline)   */
#define DAMP_FMT_INT8_ROW 1 /* every row INT8 + FP32 absmax scale (uniform INT8)   */
#define DAMP_FMT_MIXED 2    /* hp_rows FP16 key rows per head, the rest INT8 (DAMP) */
#define DAMP_FMT_FP8_ROW 3  /* every row FP8 E4M3 + FP32 absmax scale (uniform FP8) */

#define DAMP_GATE_SCALAR 0 /* GDN: alpha is one FP32 per (entry, head)            */
#define DAMP_GATE_VECTOR 1 /* KDA: alpha is d_k FP32 per (entry, head)            */

#define DAMP_DTYPE_BF16 0 /* q, k, v are bfloat16 */
#define DAMP_DTYPE_F32 1  /* q, k, v are float32  */

typedef struct damp_pool damp_pool; /* opaque host-side descriptor */

/* Human-readable text of a status code.  Never NULL; static storage. */
const char* damp_status_string(int status);

/*
 * Byte layout of one (slot, head) state block.
 *   *block_bytes  : bytes the format must hold (the algorithmic size:
 *                   FP32 d_k*d_v*4; quantized 2*hp*d_v + r*d_v + 4*r with
 *                   r = d_k - hp).  27 FP16 rows at d = 128 give 20,244 B,
 *                   9.885 bits per value, 69.1 % below FP32 (the pages'
 *                   "9.9 bits" and "69.1 %", DAMP v1 abstract).
 *   *block_stride : bytes between consecutive blocks in a pool (block_bytes
 *                   rounded up to 16 for bulk copies).
 * Quantized block byte order: r FP32 scales (INT8 rows in increasing key
 * index) padded to 16 B, then the hp FP16 rows in increasing key index, then
 * the r INT8 rows in increasing key index.  FP32 blocks: row-major [d_k][d_v].
 * FP8 blocks have the INT8-row layout with E4M3 bytes in place of INT8 codes.
 * Either output pointer may be NULL.
 */
int damp_layout(int format, int d_k, int d_v, int hp_rows, size_t* block_bytes,
                size_t* block_stride);

/*
 * Bytes the caller must allocate for a pool of n_slots x H blocks: a header
 * (device status word, per-head FP16-row masks, row directory and block
 * table, 256 B aligned) followed by the slots.  With one FP16-row count for
 * every head, block (slot, h) is at header + (slot*H + h)*stride.
 */
int damp_pool_bytes(int format, int n_slots, int H, int d_k, int d_v, int hp_rows,
                    size_t* bytes);

/*
 * Bind a descriptor to a caller-owned device buffer and write its header.
 *   hp_row_idx : host array [H][hp_rows] of the FP16 key rows of each head
 *                (the frozen precision map from offline calibration).  Each
 *                head's entries must be distinct and < d_k; any order.  NULL
 *                allowed when hp_rows == 0.  Copied; the caller keeps it.
 *   dev_buf    : device buffer of buf_bytes >= damp_pool_bytes(...), 16-byte
 *                aligned; stays owned by the caller and must outlive the pool.
 * The block contents are left as they are (pack them, or restore raw bytes).
 * Synchronous (writes the header with a blocking copy).  On success *out
 * receives a descriptor to release with damp_pool_destroy.
 */
int damp_pool_create(int format, int n_slots, int H, int d_k, int d_v, int hp_rows,
                     const uint16_t* hp_row_idx, void* dev_buf, size_t buf_bytes,
                     damp_pool** out);

/*
 * Mixed pool whose heads hold different numbers of FP16 rows: the "fixed
 * storage budget" of the DAMP later abstract (mlsanity.com index page) spent
 * unevenly, e.g. as damp_calib_select_budget picks it.
 *   is_fp16 : host array [H][d_k] of 0/1 bytes, 1 = FP16 key row.  Copied.
 * Head h's block has the layout of damp_layout(DAMP_FMT_MIXED, d_k, d_v,
 * hp_h) with hp_h the head's FP16-row count; a slot holds the H blocks one
 * after another (damp_pool_head_layout gives each head's offset and size).
 * Every other call treats such a pool like any DAMP_FMT_MIXED pool; a map
 * with the same count in every head gives the pool damp_pool_create makes.
 */
int damp_pool_bytes_map(int n_slots, int H, int d_k, int d_v, const uint8_t* is_fp16,
                        size_t* bytes);
int damp_pool_create_map(int n_slots, int H, int d_k, int d_v, const uint8_t* is_fp16,
                         void* dev_buf, size_t buf_bytes, damp_pool** out);

/* Head h's block: algorithmic size, stride and byte offset inside a slot.
 * Any output pointer may be NULL. */
int damp_pool_head_layout(const damp_pool* pool, int h, size_t* block_bytes,
                          size_t* block_stride, size_t* offset_in_slot);

/* Release the descriptor (never the caller's device buffer).  NULL is a no-op. */
int damp_pool_destroy(damp_pool* pool);

/* Byte offset of block (slot, h) from the start of the caller's buffer. */
int damp_pool_block_offset(const damp_pool* pool, int slot, int h, size_t* offset);

/*
 * Compress FP32 states into pool slots (prefill hand-off, restore).
 *   slot_idx : device int32 [n]; entry b < 0 is skipped; >= n_slots sets
 *              DAMP_EFLAG_SLOT_RANGE and is skipped.
 *   state    : device float32 [n][H][d_k][d_v].
 * Entries of slot_idx must be distinct (each block has one writer).
 */
int damp_pool_pack(const damp_pool* pool, int n, const int32_t* slot_idx, const float* state,
                   void* stream);

/*
 * Reconstruct FP32 states from pool slots (Table C2 step 1: FP16 rows
 * exactly, INT8 rows as fl(code * scale)).  state: device float32
 * [n][H][d_k][d_v]; entries with slot_idx < 0 or out of range are zeroed.
 */
int damp_pool_unpack(const damp_pool* pool, int n, const int32_t* slot_idx, float* state,
                     void* stream);

/*
 * One decode step for every (entry b, head h): read block (slot_idx[b], h),
 * apply the gated delta rule, write out[b][h][:] = X^T q, requantize the
 * block in place.
 *   slot_idx : device int32 [n].  < 0: padding, out row zeroed, block
 *              untouched.  >= n_slots: DAMP_EFLAG_SLOT_RANGE, out row zeroed.
 *              Entries must be distinct.
 *   in_dtype : DAMP_DTYPE_BF16 | DAMP_DTYPE_F32 for q, k, v.
 *   q, k     : device [n][H][d_k];  v : device [n][H][d_v]  (final values: the
 *              step applies no scaling or normalisation).
 *   gate     : DAMP_GATE_SCALAR (alpha device float32 [n][H]) or
 *              DAMP_GATE_VECTOR (alpha device float32 [n][H][d_k]).
 *   beta     : device float32 [n][H].
 *   out      : device float32 [n][H][d_v].
 * n == 0 is a no-op.  Inputs and out must not alias the pool buffer.
 */
int damp_decode_step(const damp_pool* pool, int n, const int32_t* slot_idx, int in_dtype,
                     const void* q, const void* k, const void* v, int gate,
                     const float* alpha, const float* beta, float* out, void* stream);

/*
 * damp_decode_step with the inputs of every unit checked on the device: a
 * unit whose q, k, v, alpha or beta holds a NaN or an infinity is skipped
 * (its out row is zeroed, its block is neither updated nor stored) and
 * DAMP_EFLAG_NONFINITE is set in the pool's status word.  Nothing traps.
 * The pages leave non-finite inputs undefined (the oracle does not model
 * them); this variant is for callers that want them caught instead of
 * propagated into the stored state.  Same arguments and results otherwise.
 */
int damp_decode_step_validated(const damp_pool* pool, int n, const int32_t* slot_idx,
                               int in_dtype, const void* q, const void* k, const void* v,
                               int gate, const float* alpha, const float* beta, float* out,
                               void* stream);

/*
 * Test hooks of the failure path (for tests of the library; not for serving).
 *   wait_limit_ns : bound of every internal pipeline wait of the decode step;
 *                   0 restores the default (2 s).  A wait that runs out sets
 *                   DAMP_EFLAG_TIMEOUT in the pool's status word; the kernel
 *                   then waits (bounded) for its copies in flight and returns,
 *                   so the CUDA context stays usable.
 *   hooks         : 0, or DAMP_HOOK_HOLD_FIRST_ITEM: every CTA of the decode
 *                   step leaves the loads of its first work item unissued, so
 *                   the wait for them runs out; no unit of the call is
 *                   updated or stored and the out rows are left as they were.
 * Process-wide, for the launches enqueued after the call.
 */
#define DAMP_HOOK_HOLD_FIRST_ITEM 1u
int damp_set_test_hooks(uint64_t wait_limit_ns, uint32_t hooks);

/*
 * Host-side check of a batch's slot indices (host int32 array [n]), for
 * callers that want it before a step: every non-negative entry must be below
 * n_slots and appear once.  Duplicates would give one block two writers in
 * the same call (the in-place update of "STEPQuant ...", Appendix Table C2
 * step 6, keeps one reader and one writer per block).  Returns DAMP_OK, or
 * DAMP_ERR_INVALID_ARGUMENT with *bad_entry (may be NULL) set to the first
 * offending batch position.  Reads host memory only; launches nothing.
 */
int damp_validate_slots(const int32_t* slot_idx, int n, int n_slots, int* bad_entry);

/*
 * Read the device status word (DAMP_EFLAG_* bits accumulated since the last
 * clear) into *flags; clear it when `clear` is non-zero.  Waits for the work
 * already queued on `stream` by polling, for at most 10 s: DAMP_ERR_TIMEOUT
 * (nothing read, nothing cleared) if it has not finished by then.
 */
int damp_pool_get_error(const damp_pool* pool, uint32_t* flags, int clear, void* stream);

/*
 * Host-only conversion between one raw block (block_stride bytes, as stored
 * in the pool) of head h and the logical per-row form, rows in key-channel
 * order: scale[d_k] (0 for FP16 rows), half[d_k][d_v] (binary16 bits, 0 for
 * INT8 rows), code[d_k][d_v] (0 for FP16 rows); FP32 format: f32[d_k][d_v].
 * Pointers a format does not use may be NULL.  No CUDA call is made.
 */
int damp_block_to_logical(const damp_pool* pool, int h, const void* block, float* scale,
                          uint16_t* half, int8_t* code, float* f32);
int damp_block_from_logical(const damp_pool* pool, int h, const float* scale,
                            const uint16_t* half, const int8_t* code, const float* f32,
                            void* block);

/*
 * Block (slot, h) of a pool in its logical per-row form, read from the device
 * into host memory (for tests and inspection, not the serving path: a
 * blocking device-to-host copy on the legacy default stream).  host_out
 * receives, rows in key-channel order:
 *   FP32 pools:      f32[d_k][d_v]                                    (4*d_k*d_v bytes)
 *   quantized pools: scale[d_k] (float), then half[d_k][d_v] (uint16),
 *                    then code[d_k][d_v] (int8), as damp_block_to_logical
 *                    fills them                             (4*d_k + 3*d_k*d_v bytes)
 * The caller owns host_out.  DAMP_ERR_INVALID_ARGUMENT for a host-only
 * descriptor or an index out of range; DAMP_ERR_CUDA if the copy fails.
 */
int damp_pool_read_raw(const damp_pool* pool, int slot, int h, void* host_out);

/* ---- offline calibration of the FP16 key rows ------------------------------
 *
 * Picks, per head, the key rows to keep in FP16 from a calibration run of the
 * unquantized recurrence.  The pages ("DAMP: Decay-Aware Mixed-Precision
 * Recurrent-State Quantization", both abstracts) select high-risk key channels
 * offline from two signals, quantization-error energy and decay-based error
 * retention, under a fixed storage budget; they give no formula.  Readings:
 *   energy_i    += sum_j (X_ij - fl(c_ij * s_i))^2     (double)
 *                  for the FP32 state X after a step, with c, s the decode
 *                  step's own INT8 quantizer applied to row i;
 *   retention_i += alpha_i^2                           (double; GDN: the
 *                  scalar decay of the (entry, head), KDA: channel i);
 *   count       += 1 per recorded (entry, head);
 *   score_i      = (energy_i / count) / max(1 - retention_i / count, 2^-30)
 *                  (error injected every step and multiplied by alpha_i^2 per
 *                  step accumulates as a geometric series).
 * Selection: per head the hp_rows largest scores (ties: lower row), or the
 * `budget` largest over all heads (ties: lower head, then lower row).
 *
 * Accumulator: caller-owned device memory of damp_calib_bytes(H, d_k) bytes,
 * 8-byte aligned, zeroed by the caller before the first accumulate; layout
 * double energy[H][d_k], retention[H][d_k], count[H].  Accumulation is
 * deterministic: each (head, row) total is owned by one warp that adds the
 * batch entries in order.
 */
size_t damp_calib_bytes(int H, int d_k);

/*
 * Add one step's records.  `pool` must be a DAMP_FMT_FP32 pool holding the
 * states after the step (for example right after damp_decode_step on it);
 * slot_idx [n] (device int32) names the entries stepped, negative entries are
 * skipped, entries >= n_slots set DAMP_EFLAG_SLOT_RANGE and are skipped;
 * alpha is the step's decay, [n][H] (gate DAMP_GATE_SCALAR) or [n][H][d_k]
 * (DAMP_GATE_VECTOR) FP32 on the device.
 */
int damp_calib_accumulate(const damp_pool* pool, int n, const int32_t* slot_idx, int gate,
                          const float* alpha, double* acc, void* stream);

/*
 * Scores and per-head selection.  score [H][d_k] (device double, may be NULL)
 * receives every score; hp_row_idx [H][hp_rows] (device uint16) receives the
 * selected rows of each head in increasing order, ready for
 * damp_pool_create.  0 <= hp_rows <= d_k.
 */
int damp_calib_select(int H, int d_k, int hp_rows, const double* acc, double* score,
                      uint16_t* hp_row_idx, void* stream);

/*
 * Selection under one budget shared by the H heads: is_fp16 [H][d_k] (device
 * uint8, 1 = FP16 row) and hp_per_head [H] (device int32).  score [H][d_k]
 * (device double) is required here: it holds the scores the ranking reads.
 * 0 <= budget <= H*d_k.
 */
int damp_calib_select_budget(int H, int d_k, int budget, const double* acc, double* score,
                             uint8_t* is_fp16, int32_t* hp_per_head, void* stream);

/*
 * damp_calib_select_budget without the caller's score buffer, for callers that
 * cannot allocate device memory when they select: a serving process whose
 * memory plan hands all free HBM to the state pools up front, or a C host
 * with no allocator of its own that only holds buffers it was given.  (The
 * pages have no counterpart: this is an interface convenience, not part of
 * the method.)
 *
 * The scores go to a scratch array inside the library instead: one static
 * device array of DAMP_SELECT_BUDGET_STATIC_MAX doubles (128 KiB), which every
 * GPU that loads the library holds until the process exits.  The call
 * allocates and frees nothing.  Results (is_fp16, hp_per_head) are the same
 * as damp_calib_select_budget's; no scores are returned.
 *   - H * d_k > DAMP_SELECT_BUDGET_STATIC_MAX: DAMP_ERR_UNSUPPORTED, nothing
 *     enqueued.  Other arguments as for damp_calib_select_budget.
 *   - The first call on a device looks up the array's device address (with
 *     that device current) and caches it; make that first call before any
 *     stream capture.
 *   - Every call on a device shares the one array, and it keeps the last
 *     call's scores (each call writes every entry it reads first).  Calls
 *     whose work overlaps on the GPU (different streams, no ordering between
 *     them) race on it: order them on one stream or with events.
 */
#define DAMP_SELECT_BUDGET_STATIC_MAX 16384
int damp_calib_select_budget_static(int H, int d_k, int budget, const double* acc,
                                    uint8_t* is_fp16, int32_t* hp_per_head, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* DAMP_H */
