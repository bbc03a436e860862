// Launch interfaces of the kernels behind the C ABI (library-internal).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace spear {

// Raise a kernel's dynamic shared-memory limit once per process (the call is
// not a stream operation, and is skipped while a stream is being captured).
cudaError_t raise_smem_limit(const void *func, size_t bytes);

// Whether `blocks` CTAs of `func` (in clusters of `cs`, 1 for none) with
// `threads` threads and `smem` bytes of dynamic shared memory can all be
// resident at once on the current device (the occupancy calculator's answer,
// cached per kernel, cluster size, shared memory and device).  The decode
// kernels' CTAs wait on one another with bounded waits, so a grid that is not
// one wave would only run into those limits.
bool grid_is_one_wave(const void *func, int threads, size_t smem, int cs, int64_t blocks, int num_sms);

// Library-owned packed layout (all device memory, zero/neutral padded):
//   codes tiled [Np/64][Kp/256][64][32] uint32: the word holding codes k = 8j..8j+7
//                             of row n (code of k = 8j+i at bit nibble_shift(i), i.e.
//                             even k in nibbles 0..3, odd k in nibbles 4..7) sits at
//                             ((n/64 * Kp/256 + j/32) * 64 + n%64) * 32 + j%32, so every
//                             64-row x 256-k block is 8 KB of contiguous memory;
//                             padding words hold code 8 (weight 0)
//   s     [Np] float          per-channel scale (0 on padding rows)
//   z     [Np] uint8          per-channel zero point (8)
//   G     [R1p][Kp] bf16      row 0 = w_g, rows 1..r = A^T, other rows 0
//   Bt    [Np][rp] bf16       B transposed (Bt[n][j] = B[j][n]), zero padded
//   Bts   [Np][rp] fp32       Bt[n][j] / e[n] rounded to tf32, e[n] = s[n] (1 where
//                             s[n] = 0): the EC operand of the tcgen05 kernel, which
//                             accumulates sum_k x (q - z) unscaled and applies e[n] once
// Np = N rounded up to 128, Kp = K rounded up to 256, rp = r rounded up to 16,
// R1p = (r + 1) rounded up to 16.
struct Packed {
    int64_t K, N, Kp, Np;
    int r, rp, R1p;
    uint32_t *codes;
    float *s;
    uint8_t *z;
    uint16_t *G;
    uint16_t *Bt;
    float *Bts;
    float b_g;
};

// ---- pack: per-channel RTN int4 of W (symmetric, z = 8, or asymmetric
// min-max with a stored zero point), plus the EC operand layouts
cudaError_t launch_pack(const Packed &pk, const void *W, const void *A, const void *B,
                        const void *wg, int *status, cudaStream_t st, bool asym);
// codes quantised elsewhere ([N][K/8], exported nibble order), s [N], z [N]
// into the device layout, plus the EC operand layouts
cudaError_t launch_import(const Packed &pk, const void *codes, const float *s, const uint8_t *z, const void *A,
                          const void *B, const void *wg, int *status, cudaStream_t st);
// codes in the exported layout [N][K/8] (row-major, no padding)
cudaError_t launch_untile_codes(const Packed &pk, uint32_t *dst, cudaStream_t st);

// Every forward-pass kernel is launched with programmatic dependent launch:
// it lets its own dependents start at once and waits for its predecessor
// (griddepcontrol.wait) before reading anything a previous kernel wrote.

// ---- prepass: per-token gate and EC down-projection
//   g[t] = sigmoid(x[t].w_g + b_g),  v[t][j] = g[t] * x[t].A[:,j]  (v is fp32 [M][rp],
//   rounded to tf32 when `tf32` is set: the operand of the tcgen05 kernel's EC k-steps)
struct PrepassWork {
    float *part;          // split-K partials
    size_t part_floats;
    unsigned *counters;   // one per 16-token tile, zero between calls
    int n_counters;
};
// `ready` (may be null): counted (release) once per 16-token tile when its v is
// written, ceil(M / 16) counts in all.  `slim`: the register-capped form, whose
// CTAs fit beside those of a tcgen05 kernel with 64-token tiles.
cudaError_t launch_prepass(const Packed &pk, const void *x, int64_t M, float *v, bool tf32, float *g,
                           const PrepassWork &w, cudaStream_t st, int num_sms, unsigned *ready, bool slim);
size_t prepass_part_floats(const Packed &pk, int64_t max_M, int num_sms);
int prepass_counters(int64_t max_M);

// ---- decode kernel: clusters of CTAs split K over 64 weight rows, mma.sync
// on exact int4 codes, EC down-projection on extra clusters of the same grid
// and EC up-projection in the epilogue (when `ec` is set).
struct DecodeWork {
    void *maps;           // tensor maps of the packed operands (host memory)
    float *ws_u;          // [9][R1p][32] published partials of the EC down-projection, then their sum
    unsigned *flags;      // kDecodeFlags counters, zero between calls: [0] groups of G published,
                          // [1] row clusters done, [2 + g] EC CTAs of group g done
    // codes of the layer that runs next (prefetched into L2 by the decode
    // kernels once their own codes have landed), null for none
    const void *pf;
    size_t pf_bytes;
    // cluster-split decode kernel (decode_stream.cu): partials of the EC
    // down-projection and u (decode_stream_ws_floats), and its counters
    // (kDecodeStreamCounters, zero between calls)
    float *ws_stream;
    unsigned *cnt_stream;
};
constexpr int kDecodeMaxTokens = 32;   // tokens per launch
constexpr int kDecodeFlags = 2 + 16;
bool decode_supported(const Packed &pk, int num_sms);
cudaError_t decode_prepare(const Packed &pk, DecodeWork &w);
void decode_free(DecodeWork &w);
size_t decode_u_floats(const Packed &pk);
cudaError_t launch_decode(const Packed &pk, const void *x, void *y, int64_t M, bool ec, const DecodeWork &w,
                          int *status, cudaStream_t st, int num_sms);

// ---- decode kernel with one CTA per 16 weight rows over the whole of K (up to
// 16 tokens, K a multiple of 64 and at most 8192, a grid of one wave of two
// CTAs per SM); launch_decode takes it when it fits.  `maps` is filled by
// decode_rows_prepare; it uses the DecodeWork buffers and prefetch hint.
bool decode_rows_shape(const Packed &pk);
bool decode_rows_fits(const Packed &pk, int64_t M, int num_sms);
cudaError_t decode_rows_prepare(const Packed &pk, void **maps);
void decode_rows_free(void *maps);
cudaError_t launch_decode_rows(const Packed &pk, const void *maps, const void *x, void *y, int64_t M, bool ec,
                               const DecodeWork &w, int *status, cudaStream_t st, int num_sms);

// ---- decode kernel for up to 16 tokens with K split over a thread-block
// cluster (each CTA stages only its slice of x; partial tiles summed over
// distributed shared memory; EC down-projection in small units with a
// last-arriver reduction).  launch_decode takes it when it fits.
constexpr int kDecodeStreamCounters = 2 + 9;
bool decode_stream_shape(const Packed &pk);
bool decode_stream_fits(const Packed &pk, int64_t M, int num_sms);
size_t decode_stream_ws_floats(const Packed &pk);
cudaError_t decode_stream_prepare(const Packed &pk, void **maps);
void decode_stream_free(void *maps);
cudaError_t launch_decode_stream(const Packed &pk, const void *maps, const void *x, void *y, int64_t M, bool ec,
                                 const DecodeWork &w, int *status, cudaStream_t st, int num_sms);

// ---- persistent decode kernel over a whole layer stack (up to 16 tokens, one
// CTA per SM for the whole stack; see stack_decode.cu).  The stack builds one
// StackOpDev per op (device memory) and two tensor maps per op.
constexpr int kStackMaxTokens = 16;
constexpr int kStackMaxRp = 64;
constexpr int kStackMaxR1p = 80;
struct StackOpDev {
    const float *s;
    const uint8_t *z;
    const uint16_t *Bt;
    const uint16_t *Gnext;   // G of the next op (its u is formed in this op's epilogue), or null
    const uint16_t *xbuf;    // input buffer (null: the call's x)
    uint16_t *ybuf;          // output buffer (null: the call's y)
    int *status;             // status word of the op's layer
    int K, N, nch, rp, R1p;
    int R1p_next, Kp_next;
    float b_g;
    int ec;                  // EC placed (and the layer has one)
    int u_mode;              // 0 no EC; 1 u from this op's EC units; 2 u from the previous op's epilogues
    int fuse_next;           // this op's epilogues form the next op's u
    int wait_op;             // the latest earlier op this one conflicts with (-1: none)
    int base;                // CTA that takes this op's item 0
    int n_g, n_tiles;        // EC units (u_mode 1) and 16-row tiles
    int u_off;               // float offset of the op's u accumulator [R1p][16]
};
bool stack_decode_layer_ok(const Packed &pk);
bool stack_decode_fits(int num_sms);
cudaError_t stack_decode_maps(const Packed &pk, CUtensorMap *codes, CUtensorMap *g);
// done: [2 n_ops] counters followed by the u accumulators, ws_bytes in all
// (cleared on the stream before the kernel); fault: make the first wait run
// out (fault injection of the timeout path).
cudaError_t launch_stack_decode(const StackOpDev *ops, const CUtensorMap *maps, int n_ops, const void *x, void *y,
                                int64_t M, bool ec_on, unsigned *done, float *uacc, size_t ws_bytes, bool fault,
                                cudaStream_t st, int num_sms);

// ---- split EC: y[t][n] = bf16(y[t][n] + sum_j v[t][j] * Bt[n][j]), v in fp32
cudaError_t launch_ec_apply(const Packed &pk, const float *vf, void *y, int64_t M, cudaStream_t st);

}  // namespace spear
