/*
 * lores.h -- C ABI of the LoReS quantized recurrent-state decode step (B200, sm_100a).
 *
 * One decode step of a linear-recurrence layer, for every sequence and head of a
 * batch, fused into one read and one write of the quantized state:
 *
 *   dequantize  S_hat = code * scale                       (value-axis groups)
 *   update      S_t = S_hat diag(alpha_t) (I - delta beta_t k_t k_t^T) + beta_t v_t k_t^T
 *   readout     o_t = S_t q_t                              (from the fp32 S_t)
 *   requantize  per group of G key entries of one value row: s = max|S_t| / r,
 *               r = 2^(b-1) - 1, stochastic rounding (or round to nearest)
 *
 * Sources: "Quantizing Recurrent Language Models Is Easier Than You Think"
 * (summary page): General recurrence form (Introduction); Key properties item 3
 * (dequantize -> update -> requantize each step); Proposition 1 (absmax scale,
 * value-axis grouping); Table 5 text (decay-based mixed precision per head);
 * Proposition 3 / Table 6 (stochastic rounding).
 *
 * Conventions for every call:
 *  - Every function returns a lores_status; nothing aborts, throws or traps.
 *  - Device pointers are plain CUDA device addresses (for example a torch tensor's
 *    data_ptr()).  Unless a call says otherwise they are owned by the caller, must be
 *    fp32, contiguous, row-major with the shapes given, and stay valid until the
 *    stream has executed the call.  Vector inputs q, k, v, alpha (per column) and the
 *    outputs of dequant/load must be 16-byte aligned; misaligned or NULL pointers
 *    return LORES_ERR_INVALID_ARG before anything is launched.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *    Calls that launch work are asynchronous unless stated.
 *  - A handle is not thread-safe: two calls on one handle that overlap on the GPU
 *    (different streams, no ordering) race on the state.
 *  - CUDA failures map to LORES_ERR_CUDA.  Values that the device finds non-finite
 *    raise a sticky flag that lores_check_errors reports.
 *
 * Shapes: B = batch, H = heads, d_k = key dim (16, 32, 64, 128 or 256), d_v = value
 * dim (multiple of 4, at most 4096), G = group_size (multiple of 16 dividing d_k).
 */
#ifndef LORES_H
#define LORES_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LORES_OK = 0,
    LORES_ERR_INVALID_ARG = 1,   /* bad shape, value, NULL or misaligned pointer          */
    LORES_ERR_OOM = 2,           /* a device or host allocation failed                   */
    LORES_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed                 */
    LORES_ERR_NONFINITE = 4,     /* a state row became non-finite (inf or NaN)            */
    LORES_ERR_UNSUPPORTED = 5,   /* well-formed but not supported (bits, d_k, device)     */
    LORES_ERR_TIMEOUT = 6,       /* a kernel gave up waiting on its own copies            */
    LORES_ERR_CORRUPT = 7,       /* the guard bands around the state were overwritten      */
    LORES_ERR_INDEX = 8          /* index-checked build: an access fell outside its buffer */
} lores_status;

typedef struct lores_handle lores_handle;

/* Create-time description of one recurrent layer's state for a batch. */
typedef struct {
    int32_t batch;          /* B >= 1 sequences                                              */
    int32_t heads;          /* H >= 1                                                        */
    int32_t d_k;            /* key dim: 16, 32, 64, 128 or 256                               */
    int32_t d_v;            /* value dim: multiple of 4, 4..4096                             */
    int32_t group_size;     /* G: key entries per scale; 0 means d_k (one scale per row)     */
    int32_t delta;          /* 1: delta-rule correction (GDN, KDA); 0: none (Mamba-2)        */
    int32_t decay_diag;     /* 0: alpha is one scalar per (seq, head); 1: one per key column */
    const int32_t *head_bits; /* host [H], each 4..8 (b-bit codes, r = 2^(b-1) - 1) or 32  */
                              /* (fp32, unquantized); NULL: all 8.  4-bit codes are stored */
                              /* as nibbles, 5- to 8-bit codes one per byte               */
    int32_t stochastic;     /* 1: stochastic rounding (LoReS); 0: round to nearest           */
    uint64_t seed;          /* key of the rounding dither                                    */
    int32_t device;         /* CUDA device ordinal                                           */
    int32_t scale_axis;     /* 0: value-axis groups (LoReS: one scale per value row, or per  */
                            /* G key entries of a row); 1: key axis, one scale per key       */
                            /* column of a tile (the comparator of the Scale Grouping        */
                            /* paragraph; needs G = d_k; a whole tile is processed by one    */
                            /* CTA, so d_v * d_k is limited by shared memory)                 */
    const int32_t *group_bits; /* NULL, or host [H][d_k/G] bits (4..8) of every key group of   */
                            /* every head: per-channel precision (the abstract's decay-based  */
                            /* mixed precision over channels).  A row stores its key groups   */
                            /* back to back, group g in G*storage(b_g)/8 bytes (4 bits as     */
                            /* nibbles, 5..8 bits one byte per code); each group is scaled    */
                            /* with its own r = 2^(b_g-1)-1.  Needs head_bits = NULL and      */
                            /* scale_axis = 0; not taken by lores_decode_step_noalloc.        */
    int32_t dense_codes;    /* 0: 5- to 7-bit codes one per byte (two's complement);         */
                            /* 1: dense, b bits per code (layout below).  Per-head bits only  */
                            /* (group_bits NULL, scale_axis 0); not taken by                   */
                            /* lores_decode_step_noalloc.                                      */
} lores_config;

/* Dense b-bit codes (dense_codes = 1, b = 5, 6, 7).  A code c is stored in offset binary,
 * u = c + 2^(b-1) (1 .. 2^b - 1), split into bit planes laid out one after another in
 * each row of the tile, the row padded to a multiple of 8 bytes:
 *   4-bit plane, d_k/2 bytes: u & 15 of column j in byte j/2, the low nibble for even j;
 *   2-bit plane, d_k/4 bytes (b >= 6): (u >> 4) & 3.  The 16-column block l (columns
 *     16l .. 16l+15) owns bytes 4l .. 4l+3; with m = j - 16l, byte 4l + p (p = 0..3)
 *     holds m = 8+2p in bits 0-1, m = 9+2p in bits 2-3, m = 2p in bits 4-5 and
 *     m = 2p+1 in bits 6-7;
 *   1-bit plane, d_k/8 bytes (b odd): bit b-1 of u.  Block l owns bytes 2l, 2l+1; byte
 *     2l holds m = 0, 2, 4, 6 in bits 0-3 and m = 1, 3, 5, 7 in bits 4-7, byte 2l+1
 *     likewise m = 8, 10, 12, 14 in bits 0-3 and m = 9, 11, 13, 15 in bits 4-7.
 * (A 16-column block's fields sit so that one lane holding the block rebuilds its 16
 * offset-binary bytes with a few shifts and masks per 4 codes.) */

/* Sizes of the handle's state, for export/import buffers, and its device buffers. */
typedef struct {
    int64_t code_bytes;        /* bytes of the whole code pool = batch * seq_code_bytes      */
    int64_t seq_code_bytes;    /* bytes of one sequence: all heads' tiles back to back       */
    int64_t scale_count;       /* fp32 scales: batch * heads * d_v * n_groups (value axis)   */
                               /* or batch * heads * d_k (key axis)                          */
    int32_t n_groups;          /* d_k / G scales per value row; 0 in key-axis mode           */
    int32_t units_per_step;    /* work units (sequence, head, row block) of one step         */
    int32_t grid;              /* CTAs of the decode kernel                                  */
    int32_t smem_bytes;        /* dynamic shared memory per CTA of the decode kernel         */
    void *codes_dev;           /* the handle's code pool and scales in device memory (owned  */
    float *scales_dev;         /* by the handle, valid until lores_destroy): for zero-copy    */
                               /* readers; writes through them must stay inside code_bytes   */
                               /* and scale_count * 4 bytes                                   */
    int32_t step_kernel;       /* single-token decode kernel: 3 tensor-core contractions     */
                               /* (heads of one byte or one nibble per code, one scale per     */
                               /* row, d_k <= 128), 1 two rows per lane (such heads with       */
                               /* several scales per row, full row blocks), 0 the general      */
                               /* one, 2 the key-axis one                                      */
} lores_layout;

/* Create a handle: validate `cfg`, allocate the code pool, the scales and the
 * handle's bookkeeping on cfg->device, and zero the state (the zero state has
 * scale 0 and code 0 everywhere).  The head precision map is fixed for the life of
 * the handle (Table 5 text: precision follows the head's decay).  On success
 * *out receives the handle; on failure *out is NULL.  Errors: INVALID_ARG
 * (shapes, bits, group size), UNSUPPORTED (device without sm_100), OOM, CUDA. */
lores_status lores_create(const lores_config *cfg, lores_handle **out);

/* Release every allocation of the handle.  NULL is accepted and returns LORES_OK.
 * The caller must make sure no work on the handle is still queued. */
lores_status lores_destroy(lores_handle *h);

/* One decode step for all B*H (sequence, head) pairs, in place on the handle's
 * state (General recurrence form; dequantize -> update -> requantize).
 *   q, k   [B, H, d_k] unit-norm fp32 (not renormalised here)
 *   v      [B, H, d_v]
 *   alpha  [B, H] (decay_diag = 0) or [B, H, d_k] (decay_diag = 1), in (0, 1]
 *   beta   [B, H], in (0, 2)
 *   o      [B, H, d_v] output, o_t = S_t q_t from the updated fp32 state
 *   step   the rounding counter: the dither of step t is a pure function of
 *          (seed, step, sequence, head, row, column), so replaying the same steps
 *          from the same state reproduces the state bit for bit.
 * A row whose updated state holds inf or NaN is stored as zero (scales 0, codes 0)
 * and raises the sticky NONFINITE flag.  Asynchronous on `stream`. */
lores_status lores_decode_step(lores_handle *h, const float *q, const float *k, const float *v,
                               const float *alpha, const float *beta, float *o,
                               uint64_t step, void *stream);

/* The decode step with its step counter in DEVICE memory (`step`: a uint64_t, 8-byte
 * aligned, read when the kernel runs), so that a sequence of steps captured once into a
 * CUDA graph replays with a fresh dither each time; lores_advance_step moves the counter
 * on the device (also capturable).  Otherwise identical to lores_decode_step: with
 * *step = t the result equals lores_decode_step(..., t, ...) bit for bit.  Launch-only
 * (no host synchronisation, no allocation), hence legal inside stream capture.
 * Errors: INVALID_ARG (as lores_decode_step; NULL or misaligned `step`), CUDA. */
lores_status lores_decode_step_dev(lores_handle *h, const float *q, const float *k,
                                   const float *v, const float *alpha, const float *beta,
                                   float *o, const uint64_t *step, void *stream);

/* *step += n on the device, ordered on `stream`.  Errors: INVALID_ARG, CUDA. */
lores_status lores_advance_step(uint64_t *step, uint64_t n, void *stream);

/* T consecutive decode steps in one call (a chunk of tokens of each sequence: the
 * decode side of a prefill -> decode handoff, or several tokens per scheduling step).
 * Token t in [0, T) reads q + t*B*H*d_k, k + t*B*H*d_k, v + t*B*H*d_v, alpha + t*B*H
 * (or + t*B*H*d_k with decay_diag), beta + t*B*H, writes o + t*B*H*d_v, and uses the
 * dither of step step0 + t: the result (state, scales, every o_t, flags) is bit for
 * bit that of T calls of lores_decode_step with steps step0 .. step0+T-1.  Inputs are
 * token-major [T, B, H, ...] with the per-token layouts of lores_decode_step.  The
 * recurrence (General recurrence form) is applied token by token with requantization
 * after every token (Key properties item 3); the state stays on chip between tokens
 * and is read from and written to HBM once per call.  Key-axis handles run one step
 * launch per token.  Errors: INVALID_ARG (T < 1, NULL or misaligned pointers), CUDA.
 * Asynchronous on `stream`. */
lores_status lores_decode_steps(lores_handle *h, int32_t T, const float *q, const float *k,
                                const float *v, const float *alpha, const float *beta,
                                float *o, uint64_t step0, void *stream);

/* The same step with HOST buffers of the same shapes (pinned or pageable).  The
 * call copies the inputs to device staging buffers owned by the handle (allocated
 * on first use), runs the step, copies o back, and returns after `stream` has
 * finished, so `o` is valid on return. */
lores_status lores_decode_step_host(lores_handle *h, const float *q, const float *k,
                                    const float *v, const float *alpha, const float *beta,
                                    float *o, uint64_t step, void *stream);

/* lores_decode_step_host without the final wait: the copies and the step are only
 * enqueued on `stream` (o is valid once the stream reaches the call).  For true overlap
 * the host buffers must be pinned (page-locked); they must stay untouched until then.
 * Steps of different handles on different streams overlap one handle's host<->device
 * copies with another handle's kernel.  Errors: as lores_decode_step_host. */
lores_status lores_decode_step_host_async(lores_handle *h, const float *q, const float *k,
                                          const float *v, const float *alpha,
                                          const float *beta, float *o, uint64_t step,
                                          void *stream);

/* The decode step for callers that must not let this library allocate device memory:
 * for example a serving engine that hands out every buffer from its own pre-planned
 * pool (a cudaMalloc inside a step can stall the device and fragment that pool), or an
 * application held to a fixed device-memory budget.  The paper has no counterpart to
 * this call; it only changes who owns the memory.
 *
 * There is no handle: cfg describes the layer (as for lores_create), and the caller
 * owns the state as two device buffers, updated in place:
 *   codes   the code pool in the handle's export layout: per sequence, the heads'
 *           tiles back to back in head order (int8 tile d_v*d_k bytes, int4 d_v*d_k/2,
 *           fp32 4*d_v*d_k), 16-byte aligned; all zero for a zero state
 *   scales  [B, H, d_v, d_k/G] fp32, 16-byte aligned
 * q, k, v, alpha, beta, o, step as for lores_decode_step.  flags_out (may be NULL):
 * host or device address that receives this call's error bits (1 = a row became
 * non-finite, 2 = the kernel gave up a wait) when the stream reaches the copy.
 * Results are the same as lores_decode_step's on a handle whose state equals these
 * buffers.
 *
 * The call allocates nothing: it never calls cudaMalloc, cudaFree or any allocating
 * library routine.  The kernel's bookkeeping (its work-unit table and error word) lives
 * in one fixed array of 64 KB + 256 B compiled into the library, which every GPU that
 * loads the library holds until the process exits.  That fixes a limit: one sequence
 * may span at most 2048 work units (a unit is up to 4 KB of one head's state, so e.g.
 * 32 heads of 128 x 128 int8 use 128); beyond it the call returns
 * LORES_ERR_UNSUPPORTED before launching anything.  The array is shared by every call
 * and keeps the last call's contents; each call rewrites the table and clears the
 * error word on its own stream, so calls that overlap on the GPU (different streams,
 * no ordering between them) race on it.  The first call on each device looks up the
 * array's device address; make that first call before any stream capture.
 * Asynchronous on `stream` (the table upload from host memory may wait for the
 * stream's earlier work).  Value-axis groups only.  Errors: INVALID_ARG (shapes, NULL
 * or misaligned pointers), UNSUPPORTED (too many units, key-axis scales, device
 * ordinal >= 64), CUDA. */
lores_status lores_decode_step_noalloc(const lores_config *cfg, void *codes, float *scales,
                                       const float *q, const float *k, const float *v,
                                       const float *alpha, const float *beta, float *o,
                                       uint64_t step, uint32_t *flags_out, void *stream);

/* Write the dequantized state, out[B, H, d_v, d_k] = code * scale (fp32 heads:
 * the state itself), to device memory `out`.  Asynchronous. */
lores_status lores_dequant_state(lores_handle *h, float *out, void *stream);

/* Replace the state by the quantization of the fp32 state S[B, H, d_v, d_k]
 * (device memory), with the decode step's own quantizer and the dither of `step`
 * (fp32 heads copy S).  Used to start from a warmed-up fp32 state.  Asynchronous. */
lores_status lores_load_state(lores_handle *h, const float *S, uint64_t step, void *stream);

/* Copy the raw state out: codes (layout_.code_bytes bytes; per sequence the heads'
 * tiles back to back in head order; a tile is row-major [d_v][d_k] bytes of 5- to
 * 8-bit codes (two's complement), or [d_v][d_k/2] bytes of 4-bit codes with the even
 * column in the low nibble, or [d_v][d_k] fp32) and scales [B, H, d_v, n_groups] fp32.  Either pointer may be
 * host or device memory (unified addressing); either may be NULL to skip it.
 * Returns after the copies have finished on `stream`. */
lores_status lores_export_codes(lores_handle *h, void *codes, float *scales, void *stream);

/* Inverse of lores_export_codes: overwrite the state with the given codes and
 * scales (host or device memory).  Returns after the copies have finished. */
lores_status lores_load_codes(lores_handle *h, const void *codes, const float *scales,
                              void *stream);

/* Fill *out with the handle's sizes.  head_offsets (may be NULL) receives H int64
 * byte offsets of each head's tile inside one sequence's block. */
lores_status lores_get_layout(const lores_handle *h, lores_layout *out, int64_t *head_offsets);

/* Wait for `stream`, then read and clear the handle's sticky device flag and verify
 * the 256-byte guard bands written around the code pool and the scales at creation.
 * Returns LORES_ERR_INDEX if (index-checked build only, see lores_index_checked) a
 * kernel skipped an access outside its buffer, else LORES_ERR_TIMEOUT if a kernel gave
 * up waiting on its own copies (its outputs for that call are incomplete), else
 * LORES_ERR_CORRUPT if a guard band was
 * overwritten (a write outside the state: a library defect, or a caller's write
 * through a pointer derived from the state), else LORES_ERR_NONFINITE if any row
 * became non-finite since the last check, else LORES_OK. */
lores_status lores_check_errors(lores_handle *h, void *stream);

/* Testing hook for the kernels' failure path (no counterpart on the pages).  Every
 * wait of a decode kernel on its own bulk copies is bounded: it gives up after a limit of
 * GPU time (one second by default), sets the handle's TIMEOUT flag, lets its other copy
 * in flight land and leaves, so the call's outputs are incomplete but the GPU context
 * stays usable.  This call makes that path run on purpose: on every later decode step of
 * h, the bulk copies of work unit `unit` (0 .. units_per_step / batch - 1, see
 * lores_get_layout) of sequence `seq` are announced to the unit's barrier but never
 * issued, so the warp that owns the unit waits out the limit; and every bounded wait of
 * the handle gives up after `wait_us` microseconds (0: the default).  Nothing is left in
 * flight: the withheld unit has no copies.  seq = -1 withholds nothing (wait_us still
 * sets the limit); lores_set_fault_injection(h, -1, 0, 0) restores normal operation.
 * Errors: INVALID_ARG (NULL, seq outside -1 .. B-1, unit outside the table),
 * UNSUPPORTED (withholding on a key-axis handle). */
lores_status lores_set_fault_injection(lores_handle *h, int32_t seq, int32_t unit,
                                       uint32_t wait_us);

/* Index-checked build (no counterpart on the pages; a stand-in for a memory sanitizer).
 * liblores_checked.so is this library compiled with LORES_INDEX_CHECKS: every global
 * access of the decode, loader and dequantizer kernels (bulk copies, their shared-memory
 * destinations, loads, stores) is first checked against the extent of the buffer it
 * belongs to, as the host declares it for the launch:
 *   0 code pool (B * seq_code_bytes)   1 scales (scale_count floats)
 *   2 q, 3 k (T*B*H*d_k floats)        4 v (T*B*H*d_v)     5 alpha (T*B*H, d_k if diagonal)
 *   6 beta (T*B*H)                     7 o (T*B*H*d_v)     8 the fp32 state of
 *   lores_load_state / lores_dequant_state (B*H*d_v*d_k floats)
 * An access outside its buffer is skipped and raises the handle's INDEX flag together
 * with bit 8 + the buffer's number (bit 17: a copy outside the launch's shared memory);
 * a skipped copy leaves its barrier short, so that warp's wait runs out as well.  Outputs
 * are bit-identical to the ordinary build's when nothing is out of range.
 *
 * lores_index_checked: 1 in the index-checked build, 0 in the ordinary one.
 * lores_debug_trim_range: declare buffer `which` (0..8 above) `bytes` shorter than it is
 * on every later launch of h, so that the checks see accesses at its end as out of range
 * (the memory itself is untouched, so nothing can fault); bytes = 0 restores it.  Errors:
 * INVALID_ARG (NULL, which outside 0..8); UNSUPPORTED in the ordinary build.
 * lores_debug_last_flags: the raw error word the last lores_check_errors on h read
 * (bit 0 NONFINITE, bit 1 TIMEOUT, bit 2 INDEX, bits 8.. the buffers).  Errors:
 * INVALID_ARG (NULL). */
int32_t lores_index_checked(void);
lores_status lores_debug_trim_range(lores_handle *h, int32_t which, uint64_t bytes);
lores_status lores_debug_last_flags(lores_handle *h, uint32_t *flags);

/* Decay-based mixed precision (Table 5 text): the round(frac_high * H) heads with
 * the largest mean decay (slowest to forget) get bits_high, the others bits_low;
 * equal decays go to the lower head index.  Host only; mean_decay and out_bits
 * are host arrays of H entries.  Errors: INVALID_ARG for NULL, H < 1, frac outside
 * [0, 1] or bits outside 4..8 and 32. */
lores_status lores_assign_bits_by_decay(const float *mean_decay, int32_t H, float frac_high,
                                        int32_t bits_high, int32_t bits_low, int32_t *out_bits);

/* Static English name of a status code. */
const char *lores_status_string(lores_status s);

#ifdef __cplusplus
}
#endif

#endif /* LORES_H */
