// Per-output-channel round-to-nearest int4 packing of a bf16 weight matrix,
// and the operand layouts of the Error Compensator.
//
// SPEAR, "A System for Post-Quantization Error-Adaptive Recovery Enabling
// Efficient Low-Bit LLM Serving", Abstract: weights are held at 4 bits per
// output channel.  The rounding rule and bit layout are this library's
// reading (the pages give neither):
//   s[n] = fp32(max_k |W[n,k]|) / 7        (IEEE fp32 division)
//   q    = clamp(rint(fp32(W[n,k] / s[n])), -8, 7) + 8    (ties to even)
//   z[n] = 8;  an all-zero row has s = 0 and every code 8
// or, with a stored zero point (the asymmetric min-max form that the
// abstract's "state-of-the-art 4-bit quantizers" commonly use per channel):
//   lo = min(0, min_k W[n,k]),  hi = max(0, max_k W[n,k])
//   s[n] = fp32(fp32(hi - lo) / 15)
//   z[n] = clamp(rint(fp32(-lo / s[n])), 0, 15)
//   q    = clamp(rint(fp32(W[n,k] / s[n])) + z[n], 0, 15)
//   an all-zero row has s = 0, z = 8 and every code 8
// and codes quantised elsewhere can be imported in the exported layout;
//   code of k = 8j+i in bits [4i, 4i+3] of word j of row n in the exported
//   layout [N][K/8]; on the device the words are stored tiled in 8 KB blocks
//   of 64 rows x 256 k (see kernels.h) with their nibbles in the order of
//   nibble_shift (device_utils.cuh), which the dequantisers unpack as
//   consecutive k pairs.
#include "device_utils.cuh"
#include "kernels.h"

namespace spear {
namespace {

constexpr int kPackWarps = 8;

// Padding word of a row with zero point zp: every code equals zp (weight 0).
__device__ __forceinline__ uint32_t pad_word(uint32_t zp) { return zp * 0x11111111u; }

template <bool ASYM>
__global__ void __launch_bounds__(kPackWarps * 32)
pack_w4_kernel(const uint16_t *__restrict__ W, int64_t N, int64_t K, int64_t Np, int64_t Kp,
               uint32_t *__restrict__ codes, float *__restrict__ s, uint8_t *__restrict__ z,
               int *status)
{
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * kPackWarps + (threadIdx.x >> 5);
    if (row >= Np)
        return;
    const int64_t words = Kp / 8, valid_words = K / 8;
    // tiled layout: word j of row n at ((n/64 * Kp/256 + j/32) * 64 + n%64) * 32 + j%32
    uint32_t *crow = codes + ((row >> 6) * (Kp / 256) * 64 + (row & 63)) * 32;
    auto word_at = [&](int64_t j) -> uint32_t & { return crow[(j >> 5) * 64 * 32 + (j & 31)]; };
    if (row >= N) {
        for (int64_t j = lane; j < words; j += 32)
            word_at(j) = 0x88888888u;
        if (lane == 0) {
            s[row] = 0.0f;
            z[row] = 8;
        }
        return;
    }
    const uint16_t *wrow = W + row * K;

    // pass 1: amax (symmetric) or min and max with 0 (asymmetric) of the row
    // (bf16 -> fp32 is exact), and a non-finite check
    uint32_t amax_bits = 0;  // |w| as bits: ordered like the values for finite inputs
    float lo = 0.0f, hi = 0.0f;
    for (int64_t j = lane; j < valid_words; j += 32) {
        const uint4 v = ld_nc(wrow + 8 * j);
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            amax_bits = max(amax_bits, (w4[i] & 0x7FFFu) << 16);
            amax_bits = max(amax_bits, w4[i] & 0x7FFF0000u);
            if (ASYM) {
                const float a = bf16_lo(w4[i]), b = bf16_hi(w4[i]);
                lo = fminf(lo, fminf(a, b));
                hi = fmaxf(hi, fmaxf(a, b));
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        amax_bits = max(amax_bits, __shfl_xor_sync(0xFFFFFFFFu, amax_bits, o));
        if (ASYM) {
            lo = fminf(lo, __shfl_xor_sync(0xFFFFFFFFu, lo, o));
            hi = fmaxf(hi, __shfl_xor_sync(0xFFFFFFFFu, hi, o));
        }
    }
    if (amax_bits >= 0x7F800000u && lane == 0)
        atomicOr(status, kStatusNonFinite);
    float sn;
    uint32_t zp = 8;
    if (ASYM) {
        sn = __fdiv_rn(__fsub_rn(hi, lo), 15.0f);
        if (sn != 0.0f)
            zp = (uint32_t)fminf(fmaxf(rintf(__fdiv_rn(-lo, sn)), 0.0f), 15.0f);
    } else {
        sn = __fdiv_rn(__uint_as_float(amax_bits), 7.0f);
    }

    // pass 2: quantise and pack eight codes per word
    for (int64_t j = lane; j < words; j += 32) {
        uint32_t word = pad_word(zp);
        if (j < valid_words && sn != 0.0f) {
            const uint4 v = ld_nc(wrow + 8 * j);
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
            word = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t h = (i & 1) ? (w4[i >> 1] & 0xFFFF0000u) : (w4[i >> 1] << 16);
                float c = rintf(__fdiv_rn(__uint_as_float(h), sn));
                if (ASYM)
                    c = fminf(fmaxf(c + (float)zp, 0.0f), 15.0f);
                else
                    c = fminf(fmaxf(c, -8.0f), 7.0f) + 8.0f;
                word |= (uint32_t)c << nibble_shift(i);
            }
        }
        word_at(j) = word;
    }
    if (lane == 0) {
        s[row] = sn;
        z[row] = (uint8_t)zp;
    }
}

// Codes quantised elsewhere, in the exported layout (code of k = 8j + i in
// bits [4i, 4i + 3] of word j of row n, [N][K/8]), with their scales and zero
// points: tiled into the device layout, nibbles in the order of nibble_shift,
// padding codes equal to the row's zero point (weight 0).  A zero point above
// 15 or a non-finite scale is flagged.
__global__ void import_codes_kernel(const uint32_t *__restrict__ src, const float *__restrict__ s_src,
                                    const uint8_t *__restrict__ z_src, int64_t N, int64_t K, int64_t Np,
                                    int64_t Kp, uint32_t *__restrict__ codes, float *__restrict__ s,
                                    uint8_t *__restrict__ z, int *status)
{
    const int64_t words = Kp / 8, valid_words = K / 8;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < Np * words;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = i / words, j = i - n * words;
        uint32_t zp = 8;
        if (n < N) {
            zp = z_src[n];
            if (j == 0) {
                const float sn = s_src[n];
                if (zp > 15u || !isfinite(sn))
                    atomicOr(status, kStatusNonFinite);
                s[n] = sn;
                z[n] = (uint8_t)zp;
            }
        } else if (j == 0) {
            s[n] = 0.0f;
            z[n] = 8;
        }
        uint32_t word = pad_word(zp & 15u);
        if (n < N && j < valid_words) {
            const uint32_t w = src[n * valid_words + j];
            word = 0;
#pragma unroll
            for (int t = 0; t < 8; ++t)
                word |= ((w >> (4 * t)) & 0xFu) << nibble_shift(t);
        }
        codes[(((n >> 6) * (Kp / 256) + (j >> 5)) * 64 + (n & 63)) * 32 + (j & 31)] = word;
    }
}

// G [R1p][Kp]: row 0 = w_g, rows 1..r = A^T;  Bt [Np][rp] = B^T; zeros elsewhere.
// Bts = Bt / e[n], e[n] = s[n] (1 where s[n] = 0): fp32 quotient rounded to tf32.
__global__ void pack_ec_kernel(const uint16_t *__restrict__ A, const uint16_t *__restrict__ B,
                               const uint16_t *__restrict__ wg, const float *__restrict__ s, int64_t K,
                               int64_t N, int r, int64_t Kp, int64_t Np, int R1p, int rp,
                               uint16_t *__restrict__ G, uint16_t *__restrict__ Bt, float *__restrict__ Bts,
                               int *status)
{
    const int64_t nG = (int64_t)R1p * Kp, nB = Np * rp;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nG + nB;
         i += (int64_t)gridDim.x * blockDim.x) {
        if (i < nG) {
            const int64_t j = i / Kp, k = i - j * Kp;
            uint16_t v = 0;
            if (k < K) {
                if (j == 0)
                    v = wg[k];
                else if (j - 1 < r)
                    v = A[k * r + (j - 1)];
            }
            G[i] = v;
        } else {
            const int64_t e = i - nG, n = e / rp, j = e - n * rp;
            const uint16_t b = (n < N && j < r) ? B[j * N + n] : (uint16_t)0;
            Bt[e] = b;
            const float sn = s[n];
            const float q = to_tf32(__fdiv_rn(__uint_as_float((uint32_t)b << 16), sn != 0.0f ? sn : 1.0f));
            if (!isfinite(q))
                atomicOr(status, kStatusNonFinite);
            Bts[e] = q;
        }
    }
}

// Back to the documented order: code of k = 8j + i in bits [4i, 4i + 3].
__device__ __forceinline__ uint32_t natural_nibble_order(uint32_t w)
{
    uint32_t out = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i)
        out |= ((w >> nibble_shift(i)) & 0xFu) << (4 * i);
    return out;
}

__global__ void untile_codes_kernel(const uint32_t *__restrict__ tiled, uint32_t *__restrict__ dst, int64_t N,
                                    int64_t K, int64_t Kp)
{
    const int64_t words = K / 8;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < N * words;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = i / words, j = i - n * words;
        dst[i] = natural_nibble_order(tiled[(((n >> 6) * (Kp / 256) + (j >> 5)) * 64 + (n & 63)) * 32 + (j & 31)]);
    }
}

}  // namespace

cudaError_t launch_untile_codes(const Packed &pk, uint32_t *dst, cudaStream_t st)
{
    untile_codes_kernel<<<1024, 256, 0, st>>>(pk.codes, dst, pk.N, pk.K, pk.Kp);
    return cudaGetLastError();
}

namespace {

cudaError_t launch_pack_ec(const Packed &pk, const void *A, const void *B, const void *wg, int *status,
                           cudaStream_t st)
{
    if (pk.r == 0)
        return cudaSuccess;
    pack_ec_kernel<<<1024, 256, 0, st>>>(static_cast<const uint16_t *>(A), static_cast<const uint16_t *>(B),
                                         static_cast<const uint16_t *>(wg), pk.s, pk.K, pk.N, pk.r, pk.Kp,
                                         pk.Np, pk.R1p, pk.rp, pk.G, pk.Bt, pk.Bts, status);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pack(const Packed &pk, const void *W, const void *A, const void *B,
                        const void *wg, int *status, cudaStream_t st, bool asym)
{
    const int blocks = (int)((pk.Np + kPackWarps - 1) / kPackWarps);
    if (asym)
        pack_w4_kernel<true><<<blocks, kPackWarps * 32, 0, st>>>(static_cast<const uint16_t *>(W), pk.N, pk.K,
                                                                 pk.Np, pk.Kp, pk.codes, pk.s, pk.z, status);
    else
        pack_w4_kernel<false><<<blocks, kPackWarps * 32, 0, st>>>(static_cast<const uint16_t *>(W), pk.N, pk.K,
                                                                  pk.Np, pk.Kp, pk.codes, pk.s, pk.z, status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return e;
    return launch_pack_ec(pk, A, B, wg, status, st);
}

cudaError_t launch_import(const Packed &pk, const void *codes, const float *s, const uint8_t *z, const void *A,
                          const void *B, const void *wg, int *status, cudaStream_t st)
{
    import_codes_kernel<<<1024, 256, 0, st>>>(static_cast<const uint32_t *>(codes), s, z, pk.N, pk.K, pk.Np,
                                              pk.Kp, pk.codes, pk.s, pk.z, status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return e;
    return launch_pack_ec(pk, A, B, wg, status, st);
}

}  // namespace spear
