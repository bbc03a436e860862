/*
 * spear_w4ec.h -- C ABI of the W4 + per-token-gated low-rank Error
 * Compensator (EC) linear layer for NVIDIA B200 (sm_100a).
 *
 * The layer (SPEAR, "A System for Post-Quantization Error-Adaptive Recovery
 * Enabling Efficient Low-Bit LLM Serving", Abstract): weights quantised to
 * 4 bits per output channel, and a lightweight Error Compensator whose
 * strength a per-token gate sets, with the correction fused into the low-bit
 * GEMM and an adaptive choice between fused and unfused kernels.  The pages
 * give no equations; this library computes
 *
 *   y[t,n] = sum_k x[t,k] * s[n]*(q[n,k] - z[n])  +  g_t * sum_j u[t,j] * B[j,n]
 *   u[t,j] = sum_k x[t,k] * A[k,j]
 *   g_t    = 1 / (1 + exp(-(sum_k x[t,k] * w_g[k] + b_g)))
 *
 * with q in {0..15} packed eight per uint32 (code of k = 8j+i in bits
 * [4i, 4i+3] of word j of row n), s[n] = fp32(max_k |W[n,k]|) / 7,
 * q = clamp(round_half_even(fp32(W/s)), -8, 7) + 8 and z[n] = 8.
 *
 * Conventions for every call:
 *  - All matrices are row-major and dense (leading dimension = row length).
 *  - bf16 means IEEE bfloat16 bit patterns (uint16); "dev" pointers are CUDA
 *    device pointers on the handle's device, "host" pointers are host memory.
 *  - `stream` is a cudaStream_t passed as an opaque pointer (NULL = the
 *    legacy default stream).  Device work is enqueued on it; calls return
 *    before it completes unless stated otherwise.
 *  - Every call returns a spear_status; nothing throws across the ABI.
 *    Argument errors are reported synchronously and leave all state
 *    unchanged.  Errors raised by kernels while they run (non-finite
 *    weights, a device-side wait that ran out of time) are sticky in a
 *    device status word that spear_w4ec_sync_status() returns and clears.
 *  - The caller owns every buffer it passes; the library keeps no pointer
 *    to a caller buffer after the call's stream work completes.
 *  - A handle may be used from one host thread at a time.  Its workspace is
 *    shared by its forward calls, so forward calls on one handle must be
 *    ordered (issue them on one stream, or synchronise between streams);
 *    calls that overlap on the GPU race on the workspace.
 */
#ifndef SPEAR_W4EC_H
#define SPEAR_W4EC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct spear_w4ec spear_w4ec; /* opaque, owned by the library */

typedef enum spear_status {
    SPEAR_OK = 0,
    SPEAR_ERR_INVALID = -1,     /* bad argument: shape, NULL, alignment, M > max_M */
    SPEAR_ERR_UNSUPPORTED = -2, /* valid arguments, but no kernel for this case */
    SPEAR_ERR_NOMEM = -3,       /* a device or host allocation failed */
    SPEAR_ERR_CUDA = -4,        /* a CUDA runtime call or kernel launch failed */
    SPEAR_ERR_TIMEOUT = -5,     /* a device-side wait gave up (sticky) */
    SPEAR_ERR_DEVICE = -6,      /* a kernel flagged bad data, e.g. non-finite W (sticky) */
    SPEAR_ERR_STATE = -7        /* call out of order, e.g. forward before pack */
} spear_status;

/* Flags of spear_w4ec_forward.  Path flags force one kernel family instead of
 * the dispatch table's choice and return SPEAR_ERR_UNSUPPORTED if it cannot
 * run the shape. */
enum {
    SPEAR_EC_OFF = 1u,        /* drop the EC: the plain W4 GEMM, y = x.W^T */
    SPEAR_FORCE_FUSED = 2u,   /* EC applied inside the GEMM's epilogue / accumulator */
    SPEAR_FORCE_SPLIT = 4u,   /* EC applied by a separate kernel after the GEMM */
    SPEAR_FORCE_DECODE = 8u,  /* decode kernels, mma.sync on register-dequantised codes (small M):
                                 one CTA per 16 weight rows over all of K (up to 16 tokens, K a
                                 multiple of 64 and at most 8192, one wave of CTAs), else the
                                 split-K streaming kernel (up to 32 tokens per launch) */
    SPEAR_FORCE_TC = 16u,     /* tcgen05 / TMEM tile kernel (larger M) */
    SPEAR_STACK_PERSISTENT = 32u /* spear_w4ec_stack_forward only: run the whole stack as one
                                 persistent kernel (up to 16 tokens; see the stack section) */
};

typedef struct spear_w4ec_opts {
    int64_t max_M;   /* largest M forward will be called with (workspace size); <= 0: 4096 */
    int32_t device;  /* CUDA device ordinal; < 0: the current device */
} spear_w4ec_opts;

/* Create a layer of K input features, N output features and EC rank r.
 * K and N must be positive multiples of 8; 0 <= r <= 128 (r = 0: no EC).
 * Allocates the packed weights and the workspace on the device (about
 * N*K/2 bytes of codes plus small buffers); no data is packed yet.
 * opts may be NULL.  On success *out receives the handle. */
int spear_w4ec_create(spear_w4ec **out, int64_t K, int64_t N, int32_t r,
                      const spear_w4ec_opts *opts);

/* Quantise and pack the layer (SPEAR, Abstract: per-channel 4-bit weights).
 *   W    dev bf16 [N][K]  full-precision weights, 16-byte aligned, finite
 *   A    dev bf16 [K][r]  EC down-projection (ignored if r == 0; may be NULL)
 *   B    dev bf16 [r][N]  EC up-projection   (ignored if r == 0; may be NULL)
 *   w_g  dev bf16 [K]     gate weights       (ignored if r == 0; may be NULL)
 *   b_g                   gate bias
 * The codes and scales are bit-identical to the definition above.  The inputs
 * may be freed once the stream work of this call has completed.  A
 * non-finite W is reported as SPEAR_ERR_DEVICE by spear_w4ec_sync_status. */
int spear_w4ec_pack(spear_w4ec *h, const void *W, const void *A, const void *B,
                    const void *w_g, float b_g, void *stream);

/* The same as spear_w4ec_pack with the asymmetric (min-max) per-channel
 * rule and a stored zero point, the form that the abstract's "state-of-the-art
 * 4-bit quantizers" commonly use per channel (the pages give no rule; this is
 * the library's reading):
 *   lo = min(0, min_k W[n,k]),  hi = max(0, max_k W[n,k])
 *   s[n] = fp32(fp32(hi - lo) / 15)
 *   z[n] = clamp(round_half_even(fp32(-lo / s[n])), 0, 15)
 *   q    = clamp(round_half_even(fp32(W[n,k] / s[n])) + z[n], 0, 15)
 *   an all-zero row has s = 0, z = 8 and every code 8.
 * Codes, scales and zero points are bit-identical to this definition. */
int spear_w4ec_pack_asym(spear_w4ec *h, const void *W, const void *A, const void *B,
                         const void *w_g, float b_g, void *stream);

/* Import a layer quantised by any per-channel 4-bit quantiser (SPEAR,
 * Abstract: the Error Compensators sit on top of existing 4-bit quantizers):
 *   codes dev uint32 [N][K/8]  the exported layout (code of k = 8j+i in bits
 *                              [4i, 4i+3] of word j of row n)
 *   s     dev float [N]        per-channel scale
 *   z     dev uint8 [N]        per-channel zero point, 0..15
 * so that w^[n,k] = s[n] * (q[n,k] - z[n]); A, B, w_g and b_g as in
 * spear_w4ec_pack.  spear_w4ec_get_packed returns the three arrays bit for
 * bit.  A zero point above 15 or a non-finite scale is reported as
 * SPEAR_ERR_DEVICE by spear_w4ec_sync_status.  The inputs may be freed once
 * the stream work of this call has completed. */
int spear_w4ec_import(spear_w4ec *h, const void *codes, const float *s, const uint8_t *z,
                      const void *A, const void *B, const void *w_g, float b_g, void *stream);

/* y = x.W^T + g.(x.A).B for M tokens.
 *   x  dev bf16 [M][K], 16-byte aligned;  y  dev bf16 [M][N], 16-byte aligned.
 * 0 <= M <= max_M (M = 0 is a no-op).  flags: SPEAR_* above (0 = dispatch).
 * The result is rounded once to bf16 (round to nearest even) from an fp32
 * accumulation.  Kernels of one call are ordered on `stream`. */
int spear_w4ec_forward(const spear_w4ec *h, const void *x, void *y, int64_t M,
                       uint32_t flags, void *stream);

/* The same as spear_w4ec_forward, with x and y in HOST memory: copies x to a
 * device staging buffer, runs the forward and copies y back, all on `stream`,
 * then synchronises the stream.  Pinned host memory gives the fastest copies.
 * The staging buffers are allocated on the first call (max_M rows). */
int spear_w4ec_forward_host(spear_w4ec *h, const void *x_host, void *y_host, int64_t M,
                            uint32_t flags, void *stream);

/* Free everything the handle owns (synchronises the device first). NULL is a no-op. */
int spear_w4ec_destroy(spear_w4ec *h);

/* Copy the packed layer out, in the exported layout:
 *   codes dev uint32 [N][K/8], s dev float [N], z dev uint8 [N].
 * Any of the three may be NULL to skip it. */
int spear_w4ec_get_packed(const spear_w4ec *h, void *codes, float *s, uint8_t *z, void *stream);

/* Per-token gate g_t for M tokens of x (dev bf16 [M][K]) into g (dev float [M]).
 * Uses the same kernel as the forward pass's gate. Requires r > 0. */
int spear_w4ec_get_gate(const spear_w4ec *h, const void *x, float *g, int64_t M, void *stream);

/* Synchronise `stream`, then return and clear the sticky device status
 * (SPEAR_OK, SPEAR_ERR_TIMEOUT or SPEAR_ERR_DEVICE). */
int spear_w4ec_sync_status(spear_w4ec *h, void *stream);

/* Adaptive kernel-fusion dispatch (SPEAR, Abstract): time every legal
 * {kernel family} x {fused, split} choice for M tokens on the caller's x and
 * y buffers (dev, shapes as in forward; y is overwritten), record the fastest
 * in the handle's table for M's bucket (1,2,4,...,128, 256+) and return its
 * flags in *choice (may be NULL).  Synchronises `stream`. */
int spear_w4ec_tune(spear_w4ec *h, const void *x, void *y, int64_t M, void *stream,
                    uint32_t *choice);

/* The flags (path | fused/split) that forward would use for M tokens now:
 * the tuned choice of M's bucket if spear_w4ec_tune has filled it, else the
 * default rule (fused EC; the decode kernels up to 32 tokens; beyond, the
 * tcgen05 kernel, which splits K for up to 128 tokens on layers whose 128-row
 * tiles fill at most half of the SMs). */
int spear_w4ec_dispatch(const spear_w4ec *h, int64_t M, uint32_t *choice);

/* Cost model for an EC-aware scheduler (SPEAR, Abstract: an SLO-constrained
 * EC-aware scheduler keeps serving predictable; the scheduler itself is not
 * part of this library).  After spear_w4ec_tune has run for M's bucket, *us
 * receives the measured median time in microseconds of one forward with
 *   flags = SPEAR_FORCE_DECODE or SPEAR_FORCE_TC,
 *         | SPEAR_FORCE_FUSED or SPEAR_FORCE_SPLIT (EC placement),
 *         | SPEAR_EC_OFF optionally (the same path without the EC; the
 *           placement flag is then ignored),
 * so that a scheduler can weigh the EC's price per batch size.  Returns
 * SPEAR_ERR_STATE if that choice was not measured (not tuned, or the path
 * cannot run this layer), SPEAR_ERR_INVALID for flags that name no single
 * choice.  Host-only; no device work. */
int spear_w4ec_cost(const spear_w4ec *h, int64_t M, uint32_t flags, float *us);

/* Save the handle's dispatch table (the tuned choice and measured costs of
 * every bucket tuned so far) as JSON text into buf (cap bytes, including the
 * terminating NUL); *len receives the text's length without the NUL.  If buf
 * is NULL or too small, returns SPEAR_ERR_INVALID with *len set, so a caller
 * can size the buffer and call again.  Host-only.  The text records K, N and r
 * and, per bucket: {"bucket": b, "M_max": 2^b (-1 for the last), "choice":
 * "decode+fused" | "decode+split" | "tcgen05+fused" | "tcgen05+split" | null,
 * "us": {name: microseconds, ...}}. */
int spear_w4ec_table_save(const spear_w4ec *h, char *buf, size_t cap, size_t *len);

/* Load a table saved by spear_w4ec_table_save (NUL-terminated JSON) into a
 * handle of the same K, N and r, replacing the buckets it lists; forward then
 * follows the loaded choices as if spear_w4ec_tune had chosen them.
 * SPEAR_ERR_INVALID for text that does not parse, another layer shape or a
 * malformed entry; SPEAR_ERR_UNSUPPORTED for a choice whose path cannot run
 * this layer on this device.  Nothing changes unless the whole table is
 * accepted.  Host-only. */
int spear_w4ec_table_load(spear_w4ec *h, const char *json);

/* Cross-layer weight prefetch, a hint for serving loops that run a fixed
 * sequence of layers (the SPEAR pages do not describe one).  `next` names the
 * layer whose forward follows h's forward on the same stream (h itself is
 * allowed; NULL clears the hint).  While h's decode-size kernel computes, its
 * CTAs read next's int4 codes from HBM into the L2 cache once their own codes
 * have landed, so that next's kernel finds its weights in L2: the weight
 * stream of one layer overlaps the compute of the layer before.  Results are
 * identical with or without the hint; a wrong `next` only costs HBM
 * bandwidth.  The tcgen05 path (more than 32 tokens) ignores it.
 *   h, next  handles on the same device (SPEAR_ERR_INVALID otherwise)
 * Destroying `next` clears the hints of every handle that names it.  Not
 * thread-safe with respect to concurrent calls on the same handles; takes
 * effect at the next forward (a captured CUDA graph keeps the hint it was
 * captured with). */
int spear_w4ec_set_next(spear_w4ec *h, spear_w4ec *next);

/* Per-token gate with no allocation at all, for callers that may not call
 * cudaMalloc (code inside a CUDA graph capture, a real-time serving loop with
 * a fixed memory budget, a host framework whose pool owns every allocation):
 *   g[t] = 1 / (1 + exp(-(x[t,:] . w_g + b_g)))   for t < M,
 * the same gate as spear_w4ec_get_gate, from the caller's own buffers and
 * without a handle.  (The SPEAR pages have no counterpart of this call; it
 * exists for those callers.)
 *   x    dev bf16 [M][K], 16-byte aligned;  w_g  dev bf16 [K], 16-byte aligned
 *   g    dev float [M]
 * K must be a positive multiple of 8 and 0 <= M <= 4096; a larger M returns
 * SPEAR_ERR_INVALID (the scratch is sized for 4096 tokens).  Runs on the
 * current device and `stream`.
 * Scratch: one static device array of 65,536 + 1,024 bytes inside the
 * library, which every GPU that loads the library holds until the process
 * exits.  All calls share it and each call clears the part that must start
 * at zero, so calls that overlap on the GPU (different streams without
 * ordering between them) race and must be avoided.  The first call on a
 * device looks up the array's device address (cudaGetSymbolAddress); make
 * that first call before any stream capture. */
int spear_w4ec_gate_noalloc(const void *x, int64_t M, int64_t K, const void *w_g, float b_g, float *g,
                            void *stream);

/* ---- Layer stack with a caller-given EC placement.
 *
 * SPEAR, Abstract: Error Compensators are placed only at the most
 * error-sensitive layers (its diagnostic that picks them is not part of this
 * library; the placement is an input here).  A stack runs a fixed sequence
 * of packed layers on one stream, each op reading one activation buffer and
 * writing another, so a decoder's projections (q, k, v from h; o from q;
 * gate and up from o; down from up) or a plain chain of layers run as one
 * call, with the EC of each op switched on or off by the placement.
 *
 * Buffers are numbered: 0 is the stack's input x (read only), 1 its output
 * y (written by the last op and no other), 2 and up are intermediates the
 * stack allocates (max_M rows of the widest activation written there).
 * Every buffer holds [M][width] bf16, row-major and dense. */
typedef struct spear_w4ec_stack spear_w4ec_stack; /* opaque, owned by the library */

typedef struct spear_w4ec_stack_op {
    spear_w4ec *layer; /* the packed layer this op runs (not owned by the stack) */
    int32_t in;        /* buffer it reads: 0 (the input x) or an intermediate >= 2 */
    int32_t out;       /* buffer it writes: 1 (the output y, last op only) or an intermediate >= 2 */
    int32_t ec;        /* EC placement: 1 applies the layer's EC (if it has one), 0 runs the
                          plain W4 GEMM (as SPEAR_EC_OFF) */
} spear_w4ec_stack_op;

/* Build a stack of n_ops ops (1 <= n_ops <= 4096) for up to max_M tokens.
 * Checked here, all SPEAR_ERR_INVALID: every layer non-NULL, on one device
 * and created with max_M at least this max_M; SPEAR_ERR_STATE if a layer is
 * not packed.  Buffer rules: intermediates are numbered 2 .. n_ops + 1; an op
 * reads 0 or an intermediate that an earlier op wrote, with the width (N)
 * that op wrote equal to its own K; every op that reads 0 has the same K;
 * only the last op writes 1; no op reads the buffer it writes.  The ops are
 * copied; the layers must outlive the stack.  Allocates the intermediates
 * and host-call staging buffers (max_M rows each) on the layers' device, and
 * names each op's layer's successor in the sequence (the last names the
 * first) as its prefetch hint (spear_w4ec_set_next), replacing earlier hints. */
int spear_w4ec_stack_create(spear_w4ec_stack **out, const spear_w4ec_stack_op *ops, int32_t n_ops,
                            int64_t max_M);

/* Run the ops in order on `stream` for M tokens (0 <= M <= max_M; M = 0 is a
 * no-op): x dev bf16 [M][K of the ops reading 0], y dev bf16 [M][N of the
 * last op], both 16-byte aligned.  Each op's output equals that of
 * spear_w4ec_forward on the same input with flags 0 (EC placed) or
 * SPEAR_EC_OFF (EC not placed), bit for bit.  `flags` (0 for the placement
 * as given) may add SPEAR_FORCE_* path flags or SPEAR_EC_OFF, which then
 * apply to every op.
 *
 * With SPEAR_STACK_PERSISTENT (and optionally SPEAR_EC_OFF, no path flag)
 * the ops run instead as ONE kernel launch of one CTA per SM that stays
 * resident for the whole stack (plus a clear of its counters before it): the
 * weights of later ops stream into shared memory while earlier ops compute,
 * and an op waits (bounded, on device counters) only for the earlier op it
 * depends on.  For M <= 16 on stacks whose layers all have K a multiple of 8
 * and r <= 64; otherwise SPEAR_ERR_UNSUPPORTED.  Its results match the same
 * definition within the same fp32-accumulation bounds, not bit for bit: the
 * EC down-projection of an op that reads the previous op's output is summed
 * from that op's epilogues with fp32 atomic adds (order may vary run to run).
 * A wait that runs out sets the timeout bit of the status word of the layer
 * of the op that waited (spear_w4ec_sync_status). */
int spear_w4ec_stack_forward(spear_w4ec_stack *s, const void *x, void *y, int64_t M, uint32_t flags,
                             void *stream);

/* The same with x and y in HOST memory: copies x to the stack's device
 * staging buffer, runs the ops, copies y back, all on `stream`, then
 * synchronises the stream.  Pinned host memory gives the fastest copies. */
int spear_w4ec_stack_forward_host(spear_w4ec_stack *s, const void *x_host, void *y_host, int64_t M,
                                  uint32_t flags, void *stream);

/* Device address of intermediate buffer `index` (>= 2) in *ptr: after a
 * forward on M tokens it holds the [M][width] output of the last op that
 * wrote it (for inspection and tests). */
int spear_w4ec_stack_buffer(const spear_w4ec_stack *s, int32_t index, void **ptr);

/* Free the stack's buffers (synchronises the device first); the layers are
 * left as they are.  NULL is a no-op. */
int spear_w4ec_stack_destroy(spear_w4ec_stack *s);

/* ---- Row-parallel tensor parallelism: a layer split along K over ranks.
 *
 * SPEAR, Abstract: with the EC in a tensor-parallel layer the input-dependent
 * gate forces a synchronisation between ranks; the pages answer it with a
 * peer-reduction kernel integrated with the epilogue and a P2P dual write.
 * This library's reading, for `world` ranks (one per GPU, one process each):
 * rank p holds the input features [k0_p, k1_p) of the layer, that is
 *   codes[:, k0_p/8 : k1_p/8] of the exported layout with the per-channel
 *   s and z of the whole rows, A[k0_p:k1_p, :], w_g[k0_p:k1_p], all of B and b_g,
 * as an ordinary handle of K = k1_p - k0_p made with spear_w4ec_import (the
 * scales must be those of the whole row, so do not pack the slice anew), and
 * receives x_p = x[:, k0_p:k1_p].  Then
 *   y = sum_p x_p.W^_p^T + g . ((sum_p x_p.A_p) . B),
 *   g = sigmoid(sum_p x_p.w_g,p + b_g),
 * where the gate needs the complete [M][r + 1] sum of the partials before the
 * sigmoid.  One call runs, on each rank's stream:
 *   partial: waits (bounded) until every rank has finished reading this
 *            rank's buffers of the previous call, runs the shard's forward
 *            with the EC off into this rank's partial-output buffer, and
 *            writes the raw fp32 partials x_p.[w_g,p, A_p] into slot p of
 *            EVERY rank's exchange buffer (peer stores: the dual write),
 *            then raises this rank's ready word in every rank's buffer;
 *   reduce:  waits (bounded) for every rank's ready word, sums the u slots
 *            in rank order (every rank gets the same u, hence the same gate),
 *            sums the ranks' partial outputs in rank order (peer loads), adds
 *            g . (u . B) once and writes the complete y on this rank (an
 *            all-reduce: every rank holds all of y).  Then it tells every
 *            rank that it has finished reading their buffers.
 * Rounding: each rank's partial output is rounded to bf16 once before the
 * sum, so an element of y is within the single-GPU bound plus about 2^-9 of
 * the sum over ranks of the partials' magnitudes.
 * The words that order the ranks count calls on the device, so a sequence of
 * calls may be captured in a CUDA graph and replayed.  Every rank must make
 * the same calls with the same M and the same SPEAR_EC_OFF flag.  A wait that
 * runs out (about a second) sets the timeout bit of the shard handle's
 * status word (spear_w4ec_sync_status); the group is then out of step and
 * must be destroyed and created again. */
typedef struct spear_w4ec_tp spear_w4ec_tp; /* opaque, owned by the library */

/* Largest number of ranks. */
#define SPEAR_TP_MAX_WORLD 8
/* Bytes of an exchange buffer's inter-process handle (cudaIpcMemHandle_t). */
#define SPEAR_TP_IPC_HANDLE_BYTES 64

/* Create rank `rank` (0 <= rank < world <= SPEAR_TP_MAX_WORLD) of a group
 * over the packed shard handle `shard` (not owned; must outlive the group;
 * created with max_M at least this max_M) and allocate its exchange buffer
 * on the shard's device, zeroed: a 256-byte control block, the u slots
 * [world][max_M][R1] fp32 (R1 = r + 1 rounded up to 16) and the partial
 * output [max_M][N] bf16.  Every rank of a group must give the same world,
 * max_M, N and r.  SPEAR_ERR_INVALID for bad arguments, SPEAR_ERR_STATE if
 * the shard is not packed. */
int spear_w4ec_tp_create(spear_w4ec_tp **out, spear_w4ec *shard, int32_t rank, int32_t world, int64_t max_M);

/* The exchange buffer of this rank: its device address, its size in bytes
 * and the byte offsets of the u slots and of the partial output in it (any
 * of the pointers may be NULL). */
int spear_w4ec_tp_buffer(const spear_w4ec_tp *t, void **base, size_t *bytes, size_t *u_offset,
                         size_t *y_offset);

/* The inter-process handle of this rank's exchange buffer, written to
 * `handle` (SPEAR_TP_IPC_HANDLE_BYTES bytes), to be gathered by every rank. */
int spear_w4ec_tp_ipc_handle(const spear_w4ec_tp *t, void *handle);

/* Connect the group from the handles of all ranks, `handles` holding world
 * consecutive SPEAR_TP_IPC_HANDLE_BYTES-byte handles in rank order (this
 * rank's own entry must be its own handle and is not opened; its buffer is
 * used directly).  Opens the other ranks' buffers with peer access and
 * checks each one's control block (rank, world, max_M, N, r):
 * SPEAR_ERR_INVALID on a mismatch or a handle that cannot be opened,
 * SPEAR_ERR_UNSUPPORTED if a peer's device cannot be reached, SPEAR_ERR_CUDA
 * for another failure of the runtime.  On any failure nothing stays open. */
int spear_w4ec_tp_connect_ipc(spear_w4ec_tp *t, const void *handles);

/* Connect the group from device addresses that this process can already use
 * (world entries in rank order, the entry of this rank being its own buffer):
 * the buffers of other groups' ranks in the same process, on this device or
 * on a peer device (peer access is enabled here when needed).  The same
 * checks as spear_w4ec_tp_connect_ipc. */
int spear_w4ec_tp_connect(spear_w4ec_tp *t, void *const *buffers);

/* The first phase of a call on M tokens (1 <= M <= max_M):
 *   x   dev bf16 [M][K of the shard] (this rank's columns of the input), 16-byte aligned.
 * flags: SPEAR_EC_OFF (the plain W4 GEMM on every rank; all ranks must
 * agree) and SPEAR_FORCE_DECODE / SPEAR_FORCE_TC for the shard's forward.
 * SPEAR_ERR_STATE before a connect. */
int spear_w4ec_tp_partial(spear_w4ec_tp *t, const void *x, int64_t M, uint32_t flags, void *stream);

/* The second phase: y dev bf16 [M][N], 16-byte aligned, receives the whole
 * layer's output.  M and SPEAR_EC_OFF as in the partial phase before it. */
int spear_w4ec_tp_reduce(spear_w4ec_tp *t, void *y, int64_t M, uint32_t flags, void *stream);

/* Both phases of one call, in order on `stream`. */
int spear_w4ec_tp_forward(spear_w4ec_tp *t, const void *x, void *y, int64_t M, uint32_t flags,
                          void *stream);

/* Close the other ranks' buffers and free this rank's (synchronises the
 * device first).  Every rank must have finished its calls (a barrier of the
 * caller's) before any rank destroys its group.  NULL is a no-op. */
int spear_w4ec_tp_destroy(spear_w4ec_tp *t);

/* Human-readable name of a status code (static storage). */
const char *spear_w4ec_strerror(int status);

#ifdef __cplusplus
}
#endif

#endif /* SPEAR_W4EC_H */
