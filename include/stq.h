/*
 * stq.h -- C ABI of the quantized gated delta-rule decode library (libstq.so).
 *
 * The library keeps the recurrent state of Gated DeltaNet (GDN) and Kimi
 * Delta Attention (KDA) heads as bit-packed integer codes with per-row
 * scales, and advances it one decode token at a time on an NVIDIA B200
 * (sm_100a).  Method: "STEPQuant: When and Where Errors Matter in Delta-Rule
 * Recurrent State Quantization" (paper.rainbus.top/paper/2609.38169);
 * sections of that page are cited by name below.
 *
 * Conventions for every call:
 *   - All entry points return an stq_status and never throw.  On a non-OK
 *     return stq_last_error() gives a message (thread-local).
 *   - Argument errors (null pointers, bad sizes, bad bit widths) are found
 *     on the host, before anything is enqueued, and return STQ_ERR_ARG or
 *     STQ_ERR_UNSUPPORTED; nothing is launched in that case.
 *   - Work is asynchronous on the caller's CUDA stream, passed as a plain
 *     pointer (a cudaStream_t / CUstream; NULL is the legacy default
 *     stream).  Tensors named "device" must be device memory of the device
 *     that was current when the pool was created, contiguous, row-major,
 *     fp32 unless stated.  The caller owns every input and output buffer
 *     and the stream; the pool owns its device memory and its copies of the
 *     tables it was created from.
 *   - Errors only the device can see (an out-of-range request or slot
 *     index, a non-finite value) set a sticky error word in the pool; the
 *     affected tile is skipped (index) or its content is unspecified
 *     (non-finite).  stq_pool_check() reports and clears it.  No device
 *     trap is ever raised.
 *   - A call that names the same (request, slot) twice in its index lists
 *     has undefined results (tiles are updated in place, one CTA each).
 *     With the environment variable STQ_DEBUG_CHECKS=1 set when the pool is
 *     created, every call that writes pages first runs a check kernel that
 *     marks each in-range (request, slot) of the call in a bitmap the pool
 *     owns; a pair seen twice sets the error word, and stq_pool_check then
 *     returns STQ_ERR_INDEX.  The decode still runs (its results stay
 *     undefined); the check costs a memset and a launch per call.
 *   - Setting the environment variable STQ_FAULT=alloc makes
 *     stq_pool_create fail with STQ_ERR_OOM, STQ_FAULT=launch makes every
 *     launching call fail with STQ_ERR_CUDA, both before any CUDA call
 *     (host-side fault injection for tests).  STQ_FAULT=timeout exercises the
 *     decode kernel's bounded waits: calls made while it is set shorten the
 *     wait limit from 1 s to 2 ms and make the first stage of the first CTA
 *     expect 16 bytes more than its copies deliver, so that every copy lands
 *     and that wait runs out; the kernel then waits (bounded) for its copies,
 *     returns, and stq_pool_check reports STQ_ERR_TIMEOUT.  The step's
 *     results are then undefined for the tiles that CTA did not finish.
 */
#ifndef STQ_H
#define STQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    STQ_OK = 0,
    STQ_ERR_ARG = 1,         /* bad argument, found on the host */
    STQ_ERR_OOM = 2,         /* device allocation failed */
    STQ_ERR_CUDA = 3,        /* a CUDA runtime call failed */
    STQ_ERR_INDEX = 4,       /* device saw a request or slot index out of range */
    STQ_ERR_NONFINITE = 5,   /* device saw a NaN or infinity */
    STQ_ERR_UNSUPPORTED = 6, /* valid but not implemented (e.g. d_k != 128) */
    STQ_ERR_TIMEOUT = 7      /* a bounded device-side wait gave up */
} stq_status;

typedef enum { STQ_GDN = 0, STQ_KDA = 1 } stq_kind;

/* Opaque pool of packed states, owned by the library. */
typedef struct stq_pool stq_pool;

/*
 * Pool description ("SGLang state pool" section: pool = concurrency x slots
 * x per-request state).  A unit of precision ("core method" section: a whole
 * head for GDN, one key row for KDA) carries a bit width b in {4, 6, 8}
 * (quantized codes) or 16: an FP16 pivot unit ("method steps", step 1, and
 * offline step (3): the riskiest units are kept in FP16, 32 of 2304 GDN heads
 * and 512 of 81920 KDA rows in the page's setting).  A pivot row keeps its
 * scale slot, which holds 1, and stores mu_ij = X_ij / (r_i c_j) rounded once
 * to binary16 (the state itself when r = c = 1; X_ij / r_i with
 * STQ_FIT_COLUMNS).  A KDA head's page (its scales, a fitted page's 512 bytes
 * of column factors, 16 b_i bytes per row with pivot rows at b = 16, padded
 * to 128 bytes) must fit the decode kernel's 17408-byte staging buffer: with
 * fp32 scales, rows averaging at most 8.25 bits (8 when fitted); else
 * STQ_ERR_UNSUPPORTED.
 * Raw pools hold the state values themselves: every unit at 16 (IEEE
 * binary16, no scales, r and c unused) or every unit at 32 (fp32, the
 * unquantized control the page's state-update timings compare against); fp32
 * units mixed with others return STQ_ERR_UNSUPPORTED.
 */
#define STQ_SCALE_F16 1u /* flags: per-row scales stored as IEEE binary16 ("method steps", step 6) */
/* flags: every page carries its own column factors c_j, refitted at each
 * quantisation ("core method" dual-axis fit; "method steps", steps 4-5):
 * the codes are taken with the page's current factors, then
 *   c_j <- sum_i w_i^2 v_ij X_ij / sum_i w_i^2 v_ij^2,  v_ij = s_i r_i z_ij,
 * over the head's non-pivot rows ("core innovation": c_j is fitted "across
 * non-pivot rows") with the frozen row weights w_i (row_weight); a column
 * whose codes are all zero keeps its factor.  col_factor gives the factors
 * the first quantisation starts from.  An FP16 pivot row of a fitted page
 * stores mu_ij = X_ij / r_i (no column factor, so that refitting does not
 * move it) and reconstructs as r_i mu_ij; a GDN pivot head's page keeps an
 * unused factor section.  Not with raw pools. */
#define STQ_FIT_COLUMNS 2u

typedef struct {
    int32_t kind;         /* stq_kind */
    int32_t num_requests; /* R >= 1 */
    int32_t num_slots;    /* S >= 1 (five per request on the page's serving setup) */
    int32_t num_heads;    /* H >= 1 */
    int32_t d_k;          /* must be 128 ("linear attention and recurrent state": d_k = d_v = 128) */
    int32_t d_v;          /* must be 128 */
    const uint8_t *unit_bits;  /* host; GDN: [H] one width per head; KDA: [H * d_k] one per key row */
    const float *row_factor;   /* host; [H * d_k] r_i, finite and > 0; NULL means all 1 */
    const float *col_factor;   /* host; [H * d_v] c_j, finite and > 0; NULL means all 1 */
    uint32_t flags;            /* STQ_SCALE_F16 | STQ_FIT_COLUMNS, or 0; must be 0 for a raw pool */
    const float *row_weight;   /* host; [H * d_k] w_i > 0, finite: row influence weights of the
                                  column fit ("core method": w_i, the gamma = 0.25 power of the
                                  calibrated influence omega_i, geometric-mean normalised);
                                  NULL means all 1; read only with STQ_FIT_COLUMNS */
} stq_pool_desc;

/*
 * Packed page of one (request, slot, head) state, in device memory:
 *   bytes [0, 512)   128 fp32 scales s_i, one per key row ([0, 256): 128
 *                    binary16 scales with STQ_SCALE_F16; codes are then
 *                    rounded from mu / s16 so that s16 z reconstructs them,
 *                    and a scale beyond the binary16 range is reported as
 *                    STQ_ERR_NONFINITE)
 *   with STQ_FIT_COLUMNS: then 128 fp32 column factors c_j of this page
 *   then rows i = 0..127 in order, row i holding 128 codes of b_i bits
 *   (16 * b_i bytes), each a b_i-bit two's complement integer in
 *   [-q_b, q_b], q_b = 2^(b_i - 1) - 1, placed in the row's little-endian
 *   bit string (bit p is bit p % 8 of byte p / 8):
 *     4 and 8 bits: code j at bits [j b_i, (j+1) b_i);
 *     6 bits: codes in 16 groups of eight; group g's 48-bit string (code
 *     8g + p at its bits [6p, 6p + 6)) is split into a 32-bit word at
 *     bytes [4g, 4g + 4) and a 16-bit half at bytes [64 + 2g, 66 + 2g)
 *   zero padding up to a multiple of 128 bytes.
 * The pages of heads 0..H-1 follow each other inside a slot; slots are
 * ordered [request][slot].  The state the page stands for is
 *   S^_ij = s_i * r_i * c_j * z_ij          ("core method": X^ = r c z),
 * with c_j the pool's column factors, or the page's own with STQ_FIT_COLUMNS.
 * A raw page (units of 16 or 32 bits) is the row-major 128 x 128 state in
 * binary16 or fp32 (32 KiB or 64 KiB), with no scales; r and c do not apply,
 * and every step rounds X once (to nearest even) into it.
 */

/* Allocate a pool (device memory, all states zero) for the current device.
 * With STQ_FIT_COLUMNS every page's column factors start as col_factor. */
stq_status stq_pool_create(const stq_pool_desc *desc, stq_pool **out);
stq_status stq_pool_destroy(stq_pool *pool);

/* Bytes of the whole packed pool and of one slot (all heads of one
 * (request, slot)). */
stq_status stq_pool_bytes(const stq_pool *pool, size_t *packed_bytes, size_t *per_slot_bytes);

/* The same figures for a description, computed on the host without
 * allocating anything (no device needed). */
stq_status stq_desc_bytes(const stq_pool_desc *desc, size_t *packed_bytes, size_t *per_slot_bytes);

/* Where head `head`'s page sits inside a slot, and its size in bytes. */
stq_status stq_page_layout(const stq_pool *pool, int32_t head, size_t *offset_in_slot,
                           size_t *page_bytes);

/*
 * Quantize fp32 states into the pool ("PTQ" section: Q(x) = s clip(round(x/s),
 * -q_b, q_b), one absmax scale per key row of X / (r c)).
 *   req_idx, slot_idx: device int32 [n]; entry e names the (request, slot)
 *                      that state e is written to.
 *   state:             device fp32 [n][H][128][128], S[i][j] with i the key row,
 *                      16-byte aligned.
 * n == 0 is a no-op.
 */
stq_status stq_quantize_state(stq_pool *pool, const int32_t *req_idx, const int32_t *slot_idx,
                              int32_t n, const float *state, void *stream);

/* Reconstruct fp32 states fl32(s_i r_i c_j z_ij) from the pool into
 * state_out (device fp32 [n][H][128][128], 16-byte aligned). */
stq_status stq_dequantize_state(stq_pool *pool, const int32_t *req_idx, const int32_t *slot_idx,
                                int32_t n, float *state_out, void *stream);

/*
 * One decode token for n (request, slot) entries and all H heads
 * ("method steps", online decode, steps 1-7), updating the packed pages in
 * place with no fp32 copy of the state kept anywhere:
 *   S^  = reconstruct(page)                        step 1
 *   X   = D S^ + beta k (v^T - k^T D S^)           step 2 ("gated delta rule")
 *   y   = X^T q                                     step 3, before requantisation
 *   page = pack(quantize_rows(X))                   steps 4-6
 *   D = alpha I (GDN) or diag(d) (KDA).
 *   q, k, v: device fp32 [n][H][128], 16-byte aligned; beta: device fp32 [n][H];
 *   gate:    device fp32, GDN [n][H] (alpha), KDA [n][H][128] (d_i per key row,
 *            16-byte aligned);
 *   y:       device fp32 [n][H][128], written.
 * n == 0 is a no-op.
 */
stq_status stq_decode_step(stq_pool *pool, const int32_t *req_idx, const int32_t *slot_idx,
                           int32_t n, const float *q, const float *k, const float *v,
                           const float *beta, const float *gate, float *y, void *stream);

/*
 * The same step split in two ("method steps", steps 3-7, and "technical
 * novelty" (4): the readout is produced first so that later layers can go
 * on, while requantisation and write-back run on a separate CUDA stream and
 * finish before the next step reads the state).  The arithmetic is that of
 * stq_decode_step, so y, codes and scales are bit-identical to it.
 *
 * stq_decode_readout    steps 1-3.  Writes y and u_tilde = u / c, where
 *                       u = beta (v - k^T D S^), as device fp32 [n][H][128]
 *                       (16-byte aligned scratch owned by the caller); the
 *                       pages are only read.
 * stq_decode_writeback  steps 4-7 with the pool's frozen factors: re-reads
 *                       the pages of the same entries, forms
 *                       X = D S^ + k (c u_tilde)^T, requantises and packs it
 *                       in place.  Reads k, gate and u_tilde (q, v, beta are
 *                       not read and may be NULL).  The caller orders it after
 *                       the readout of the same entries and before any other
 *                       access to their pages.
 * stq_decode_step_split both halves: the readout on `stream`, the write-back
 *                       on `side_stream` after an event recorded behind the
 *                       readout.  The pool then holds a pending write-back:
 *                       its next asynchronous call makes its own stream wait
 *                       for it, its synchronous calls (export, import, check)
 *                       wait for it on the host, and stq_pool_join makes a
 *                       given stream wait for it.  Before capturing a CUDA
 *                       graph, join or synchronize any write-back issued
 *                       outside the capture.
 * GDN pivot heads are advanced completely by the readout (their own kernel
 * stores the new binary16 values); every other unit as described.
 * Raw pools (units of 16 or 32 bits) return STQ_ERR_UNSUPPORTED.  Argument
 * rules are those of stq_decode_step; u_tilde must not be NULL for n > 0.
 */
stq_status stq_decode_readout(stq_pool *pool, const int32_t *req_idx, const int32_t *slot_idx,
                              int32_t n, const float *q, const float *k, const float *v,
                              const float *beta, const float *gate, float *y, float *u_tilde,
                              void *stream);
stq_status stq_decode_writeback(stq_pool *pool, const int32_t *req_idx, const int32_t *slot_idx,
                                int32_t n, const float *k, const float *gate,
                                const float *u_tilde, void *stream);
stq_status stq_decode_step_split(stq_pool *pool, const int32_t *req_idx,
                                 const int32_t *slot_idx, int32_t n, const float *q,
                                 const float *k, const float *v, const float *beta,
                                 const float *gate, float *y, float *u_tilde, void *stream,
                                 void *side_stream);

/*
 * The split step with scratch the library owns: no counterpart in the paper.
 * For callers that must not allocate device memory while they run, such as a
 * serving engine that reserved all of its device memory at start-up, or one
 * that cannot risk an allocation failing under memory pressure or stalling
 * the device inside its latency budget.  Same arguments and results as
 * stq_decode_step; it runs stq_decode_readout and stq_decode_writeback one
 * after the other on `stream`, with u_tilde kept in a fixed 4 MiB device array
 * built into the library (every GPU that loads the library holds it until the
 * process exits).  It never allocates or frees memory.
 *   - n * H may be at most 8192 tiles (n * H * 128 floats <= 2^20);
 *     larger calls return STQ_ERR_ARG before anything is enqueued.
 *   - The first call on a device looks up the array's device address on
 *     that device; make that first call before any stream capture.  Later
 *     calls look it up again (so a context re-created after a device reset
 *     is served from its own copy).
 *   - All calls on a device share the one array: calls that may overlap on the
 *     GPU (other streams, other threads) race on it and must be serialized by
 *     the caller.  Each call writes the array in full before reading it, so
 *     nothing has to be cleared between calls.
 * Raw pools return STQ_ERR_UNSUPPORTED.
 */
stq_status stq_decode_step_static(stq_pool *pool, const int32_t *req_idx, const int32_t *slot_idx,
                                  int32_t n, const float *q, const float *k, const float *v,
                                  const float *beta, const float *gate, float *y, void *stream);

/*
 * stq_decode_step with every per-token buffer in HOST memory: no counterpart
 * in the paper, for callers that hold their inputs and want y on the host.
 * Arguments, results and rules are those of stq_decode_step, except that
 * req_idx, slot_idx, q, k, v, beta, gate and y are host pointers (no
 * alignment rule).  On `stream`, after the work already queued there, the
 * library copies the inputs into a device staging buffer that the pool owns,
 * runs the step (the same kernels, so the results are those of
 * stq_decode_step bit for bit) and delivers y; y may be read once `stream` is
 * synchronized.
 *   - Page-locked host memory (cudaHostAlloc, cudaHostRegister) makes the
 *     copies asynchronous; pageable memory works, with copies that block the
 *     host.
 *   - A page-locked y that the device can address (every page-locked
 *     allocation on a system with unified addressing) is written by the
 *     decode kernels directly, across the bus, with no copy back; any other y
 *     is written to the staging buffer and copied back.  A page-locked y must
 *     therefore be writable by the device: memory registered with
 *     cudaHostRegisterReadOnly is not a valid y.
 *   - The inputs must stay unchanged, and y unread, until `stream` has
 *     passed the step.
 *   - The first call, and any call with more entries than every earlier
 *     one, allocates the staging buffer (n * H * 2 KiB, and 512 B more per
 *     tile for a KDA gate), after waiting on the host for the previous
 *     host-buffer step of the pool; it is not meant for stream capture.
 *   - A call on another stream than the pool's previous host-buffer step
 *     waits for that step (the staging buffer is shared).  Calls on one pool
 *     from several host threads must be serialized.
 * Host pointers that are not host memory make a copy fail with STQ_ERR_CUDA.
 */
stq_status stq_decode_step_host(stq_pool *pool, const int32_t *req_idx, const int32_t *slot_idx,
                                int32_t n, const float *q, const float *k, const float *v,
                                const float *beta, const float *gate, float *y, void *stream);

/*
 * The host-buffer step with every input in ONE host block, so that the inputs
 * cross the bus in a single copy (no counterpart in the paper).
 *
 * stq_host_block_layout: for n entries of `pool`, the byte offsets inside
 * the block of req_idx, slot_idx, q, k, v, beta and gate, in that order, in
 * offsets[0..6] (each a multiple of 256, arrays as stq_decode_step lays them
 * out: int32 [n], int32 [n], fp32 [n][H][128] x 3, fp32 [n][H], gate fp32
 * [n][H] (GDN) or [n][H][128] (KDA)), and the block size in *bytes (the end
 * of the gate array).  The bytes between arrays are never read.  STQ_ERR_ARG
 * for a NULL pool or output, or n < 0.
 *
 * stq_decode_step_host_block: stq_decode_step_host with the inputs read
 * from `block` (host memory of at least `bytes` bytes, as laid out above for
 * this n; `bytes` must equal the layout's size, else STQ_ERR_ARG) and y
 * written to the host array y (fp32 [n][H][128]).  One host-to-device copy
 * of the block and the step, all on `stream`, with y delivered as by
 * stq_decode_step_host (written by the kernels when page-locked, else one
 * device-to-host copy); the results equal stq_decode_step's bit for bit, and
 * the staging rules (shared buffer, first-call allocation, page-locked memory
 * for asynchronous copies) are those of stq_decode_step_host.
 */
stq_status stq_host_block_layout(const stq_pool *pool, int32_t n, size_t offsets[7], size_t *bytes);
stq_status stq_decode_step_host_block(stq_pool *pool, int32_t n, const void *block, size_t bytes, float *y,
                                      void *stream);

/* Make `stream` wait for the pool's pending split write-back (no-op if none). */
stq_status stq_pool_join(stq_pool *pool, void *stream);

/*
 * Lifetime-aware mixed-precision bit allocation (host computation; "core
 * innovation", first point, and "method steps", offline calibration steps
 * (1)-(3)).  Produces the unit_bits of a pool description from per-unit
 * calibration statistics.
 *
 * stq_lifetime_weight: L_u = sum_{j=0}^{horizon-1} exp(2 j l_u) for each
 *   unit's mean log retention l_u = E[log r_{t,u}] (<= 0): the factor by which
 *   the squared error injected at one step is summed over the horizon.  The
 *   page leaves the horizon open; it is an argument here.
 * stq_allocate_bits: minimises sum_u L_u d_u(b_u) subject to
 *   sum_u n_u b_u <= mean_bits * sum_u n_u (Eq. 8) over b_u in `choices`
 *   (strictly increasing widths), with
 *     unit_values n_u [U]   values per unit (a GDN head: 16384; a KDA row: 128),
 *     distortion d_u(b) [U][C] (row-major, >= 0), weight L_u [U] (>= 0),
 *     method STQ_ALLOC_DP       exact multiple-choice dynamic programme
 *                               (integer n_u; STQ_ERR_UNSUPPORTED if the
 *                               table would exceed 4e8 cells),
 *            STQ_ALLOC_LAGRANGE per-unit minimiser of L d + lambda n b at the
 *                               smallest multiplier that fits the budget
 *                               (optimal for the bits it uses).
 *   Afterwards the num_pivots units of largest remaining risk L_u d_u(b_u)
 *   get pivot_bits (the page's FP16 pivots: 16); pivots are outside the
 *   budget.  bits_out [U] receives the widths, objective_out (may be NULL)
 *   the minimised sum before pivots.  Ties go to the smaller width.
 *   STQ_ERR_ARG: bad sizes, non-finite or negative inputs, a budget below the
 *   smallest width.
 */
typedef enum { STQ_ALLOC_DP = 0, STQ_ALLOC_LAGRANGE = 1 } stq_alloc_method;
stq_status stq_lifetime_weight(int32_t num_units, const double *log_retention, int32_t horizon,
                               double *weight_out);
stq_status stq_allocate_bits(int32_t num_units, const double *unit_values, int32_t num_choices,
                             const uint8_t *choices, const double *distortion, const double *weight,
                             double mean_bits, int32_t method, int32_t num_pivots, uint8_t pivot_bits,
                             uint8_t *bits_out, double *objective_out);

/* Copy one slot's raw pages (per_slot_bytes bytes) to / from host memory.
 * Synchronous (device-wide ordering with the legacy default stream). */
stq_status stq_export_slot(const stq_pool *pool, int32_t req, int32_t slot, void *host_dst,
                           size_t bytes);
stq_status stq_import_slot(stq_pool *pool, int32_t req, int32_t slot, const void *host_src,
                           size_t bytes);

/* Synchronize `stream` (and any pending split write-back), then return and clear the pool's device error word
 * (STQ_ERR_INDEX, STQ_ERR_NONFINITE or STQ_ERR_TIMEOUT; STQ_OK if clear). */
stq_status stq_pool_check(stq_pool *pool, void *stream);

/* Number of kernel launches this library has issued in this process. */
uint64_t stq_launch_count(void);

const char *stq_status_str(stq_status status);
const char *stq_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* STQ_H */
