// Launch interfaces of the kernels behind the C ABI (library-internal).
#pragma once
#include <cuda_runtime.h>
#include <cstdint>

namespace spear {

// Raise a kernel's dynamic shared-memory limit once per process (the call is
// not a stream operation, and is skipped while a stream is being captured).
cudaError_t raise_smem_limit(const void *func, size_t bytes);

// Library-owned packed layout (all device memory, zero/neutral padded):
//   codes [Np][Kp/8] uint32   code of k = 8j+i in bits [4i,4i+3] of word j;
//                             padding words hold code 8 (weight 0)
//   s     [Np] float          per-channel scale (0 on padding rows)
//   z     [Np] uint8          per-channel zero point (8)
//   G     [R1p][Kp] bf16      row 0 = w_g, rows 1..r = A^T, other rows 0
//   Bt    [Np][rp] bf16       B transposed (Bt[n][j] = B[j][n]), zero padded
// Np = N rounded up to 128, Kp = K rounded up to 128, rp = r rounded up to 16,
// R1p = (r + 1) rounded up to 16.
struct Packed {
    int64_t K, N, Kp, Np;
    int r, rp, R1p;
    uint32_t *codes;
    float *s;
    uint8_t *z;
    uint16_t *G;
    uint16_t *Bt;
    float b_g;
};

// ---- pack: per-channel RTN int4 of W, plus the EC operand layouts
cudaError_t launch_pack(const Packed &pk, const void *W, const void *A, const void *B,
                        const void *wg, int *status, cudaStream_t st);

// Every forward-pass kernel is launched with programmatic dependent launch:
// it lets its own dependents start at once and waits for its predecessor
// (griddepcontrol.wait) before reading anything a previous kernel wrote.

// ---- prepass: per-token gate and EC down-projection
//   g[t] = sigmoid(x[t].w_g + b_g),  v[t][j] = bf16(g[t] * x[t].A[:,j])  (v is [M][rp])
struct PrepassWork {
    float *part;          // split-K partials
    size_t part_floats;
    unsigned *counters;   // one per 16-token tile, zero between calls
    int n_counters;
};
cudaError_t launch_prepass(const Packed &pk, const void *x, int64_t M, uint16_t *v, float *g,
                           const PrepassWork &w, cudaStream_t st, int num_sms);
size_t prepass_part_floats(const Packed &pk, int64_t max_M, int num_sms);
int prepass_counters(int64_t max_M);

// ---- decode main kernel: tensor-core (mma.sync) split-K W4 GEMM, tokens on
// the narrow side, EC applied in the epilogue when `ec` is set.
struct DecodeWork {
    float *part;
    size_t part_floats;
    unsigned *counters;   // one per 64-row block, zero between calls
    int n_counters;
};
constexpr int kDecodeMaxTokens = 32;   // tokens per launch
cudaError_t launch_decode(const Packed &pk, const void *x, void *y, int64_t M, const uint16_t *v,
                          bool ec, const DecodeWork &w, cudaStream_t st, int num_sms);
size_t decode_part_floats(const Packed &pk, int num_sms);
int decode_counters(const Packed &pk);

// ---- split EC: y[t][n] = bf16(y[t][n] + sum_j v[t][j] * Bt[n][j])
cudaError_t launch_ec_apply(const Packed &pk, const uint16_t *v, void *y, int64_t M, cudaStream_t st);

}  // namespace spear
