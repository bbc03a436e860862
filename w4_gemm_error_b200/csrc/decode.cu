// Decode-size W4 GEMM with the Error Compensator fused into its epilogue.
//
// SPEAR, "A System for Post-Quantization Error-Adaptive Recovery Enabling
// Efficient Low-Bit LLM Serving", Abstract: the post-EC computation is fused
// into the low-bit GEMM.  For a few tokens the GEMM is bound by reading the
// int4 codes from HBM, so this kernel is built around streaming them:
//
//  * weight rows sit on the 16-row side of mma.sync m16n8k16 and tokens on
//    the 8-column side (up to 32 tokens per launch), so one code is read
//    once however many tokens there are;
//  * each lane loads 16 bytes (32 codes) of two rows per 128-wide k block
//    straight from the exported [N][K/8] layout into registers, four blocks
//    ahead, and dequantises them in registers: two nibbles 16 bits apart
//    become a bf16x2 pair (q - z) exactly, so the tensor cores see exact
//    integer weights and the per-channel scale is applied once at the end;
//  * the k order inside the MMA is permuted so that those register pairs
//    (codes k and k+4) line up with the activations, which are staged once
//    per CTA in shared memory (XOR-swizzled, conflict-free) and paired with
//    one byte-permute per register;
//  * the K range is split over CTAs; the last CTA of each 64-row block to
//    finish sums the partial tiles in a fixed order (run-to-run identical)
//    and runs the epilogue
//        y[t,n] = bf16( s[n] * acc[t,n] + sum_j v[t,j] * B[j,n] )
//    where v = g * (x . A) comes from the prepass kernel;
//  * kernels are chained with programmatic dependent launch: the first code
//    blocks are requested before waiting for the previous kernel (which
//    writes x, and v), so the weight stream overlaps the previous kernel's
//    tail and the prepass.
#include <algorithm>

#include "device_utils.cuh"
#include "kernels.h"

namespace spear {
namespace {

constexpr int kRows = 64;      // weight rows per CTA (four warps x 16)
constexpr int kPrefetch = 4;   // 128-wide k blocks in flight per warp
constexpr int kMaxBps = 8;     // k blocks per CTA at most (shared-memory bound)

struct DecodeParams {
    const uint32_t *codes;
    const float *s;
    const uint8_t *z;
    const uint16_t *x;
    uint16_t *y;
    const uint16_t *v;
    const uint16_t *Bt;
    float *part;
    unsigned *counters;
    int64_t M, K, Kp, N;
    int S, bps, rp;
    int ec;
};

__device__ __forceinline__ int swz(int t, int c, int q)
{
    // physical 16-byte chunk of logical chunk (lane group c, word q) of token t
    return 4 * c + (q ^ (2 * (c >> 1)) ^ (t & 1));
}

template <int T>
__global__ void __launch_bounds__(128) decode_w4ec_kernel(DecodeParams p)
{
    constexpr int TOK = 8 * T;
    extern __shared__ uint4 smem_u4[];
    __shared__ int s_last;

    pdl_launch_dependents();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gid = lane >> 2, c = lane & 3;
    const int nb = blockIdx.x / p.S, ks = blockIdx.x - nb * p.S;
    const int nkb = (int)(p.Kp / 128);
    const int kb0 = ks * p.bps, kb1 = min(kb0 + p.bps, nkb);
    const int nblk = kb1 - kb0;
    const int64_t words = p.Kp / 8;

    // ---- start the code stream first: rows (gid) and (gid + 8) of this warp
    const int64_t row_g = (int64_t)nb * kRows + warp * 16 + gid;
    const uint32_t *cg = p.codes + row_g * words + 16 * kb0 + 4 * c;
    const uint32_t *ch = cg + 8 * words;
    uint4 wg[kPrefetch], wh[kPrefetch];
#pragma unroll
    for (int i = 0; i < kPrefetch; ++i) {
        if (i < nblk) {
            wg[i] = ld_stream(cg + 16 * i);
            wh[i] = ld_stream(ch + 16 * i);
        }
    }
    const uint32_t zg = 128u + p.z[row_g], zh = 128u + p.z[row_g + 8];
    // bf16 of -(128 + z): exact (an integer below 256)
    const uint32_t nbg = __bfloat16_as_ushort(__float2bfloat16_rn(-(float)zg));
    const uint32_t nbh = __bfloat16_as_ushort(__float2bfloat16_rn(-(float)zh));
    const uint32_t negg = nbg | (nbg << 16), negh = nbh | (nbh << 16);

    // x (and v) are written by the kernels before this one in the stream:
    // everything above only touched the packed weights.
    pdl_wait();

    // ---- stage the activations of this k range: [TOK][nblk][16 chunks]
    uint4 *xs = smem_u4;
    const int cpt = nblk * 16;
    for (int i = tid; i < TOK * cpt; i += 128) {
        const int t = i / cpt, rem = i - t * cpt, b = rem >> 4, chk = rem & 15;
        const int64_t k = (int64_t)(kb0 + b) * 128 + 8 * chk;
        uint4 val = make_uint4(0, 0, 0, 0);
        if (t < p.M && k < p.K)
            val = ld_nc(p.x + (int64_t)t * p.K + k);
        xs[(t * nblk + b) * 16 + swz(t, chk >> 2, chk & 3)] = val;
    }
    __syncthreads();

    float acc[T][4];
#pragma unroll
    for (int n = 0; n < T; ++n)
#pragma unroll
        for (int i = 0; i < 4; ++i)
            acc[n][i] = 0.f;

    for (int b0 = 0; b0 < nblk; b0 += kPrefetch) {
#pragma unroll
        for (int i = 0; i < kPrefetch; ++i) {
            const int b = b0 + i;
            if (b < nblk) {
                const uint4 cw = wg[i], hw = wh[i];
                if (b + kPrefetch < nblk) {
                    wg[i] = ld_stream(cg + 16 * (b + kPrefetch));
                    wh[i] = ld_stream(ch + 16 * (b + kPrefetch));
                }
                const uint32_t cgw[4] = {cw.x, cw.y, cw.z, cw.w};
                const uint32_t chw[4] = {hw.x, hw.y, hw.z, hw.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    // codes k = 32c + 8j + {0..7}: pairs (0,4) (1,5) (2,6) (3,7)
                    const uint32_t g0 = dequant_pair(cgw[j], negg), g1 = dequant_pair(cgw[j] >> 4, negg);
                    const uint32_t g2 = dequant_pair(cgw[j] >> 8, negg), g3 = dequant_pair(cgw[j] >> 12, negg);
                    const uint32_t h0 = dequant_pair(chw[j], negh), h1 = dequant_pair(chw[j] >> 4, negh);
                    const uint32_t h2 = dequant_pair(chw[j] >> 8, negh), h3 = dequant_pair(chw[j] >> 12, negh);
#pragma unroll
                    for (int n = 0; n < T; ++n) {
                        const int t = 8 * n + gid;
                        const uint4 xv = xs[(t * nblk + b) * 16 + swz(t, c, j)];
                        const uint32_t b00 = prmt(xv.x, xv.z, 0x5410), b01 = prmt(xv.x, xv.z, 0x7632);
                        const uint32_t b10 = prmt(xv.y, xv.w, 0x5410), b11 = prmt(xv.y, xv.w, 0x7632);
                        mma_bf16_16816(acc[n], g0, h0, g1, h1, b00, b01);
                        mma_bf16_16816(acc[n], g2, h2, g3, h3, b10, b11);
                    }
                }
            }
        }
    }

    // ---- partial tile [64 rows][TOK] to shared memory
    __syncthreads();  // every warp is done reading xs
    float *red = reinterpret_cast<float *>(smem_u4);
#pragma unroll
    for (int n = 0; n < T; ++n) {
        const int r0 = warp * 16 + gid, col = 8 * n + 2 * c;
        red[r0 * TOK + col] = acc[n][0];
        red[r0 * TOK + col + 1] = acc[n][1];
        red[(r0 + 8) * TOK + col] = acc[n][2];
        red[(r0 + 8) * TOK + col + 1] = acc[n][3];
    }
    __syncthreads();

    constexpr int kTile = kRows * TOK;
    if (p.S > 1) {
        float *mine = p.part + ((size_t)nb * p.S + ks) * kTile;
        for (int e = tid; e < kTile; e += 128)
            mine[e] = red[e];
        __threadfence();
        __syncthreads();
        if (tid == 0)
            s_last = (atomicAdd(&p.counters[nb], 1u) == (unsigned)(p.S - 1));
        __syncthreads();
        if (!s_last)
            return;
        __threadfence();
        const float *all = p.part + (size_t)nb * p.S * kTile;
        for (int e = tid; e < kTile; e += 128) {
            float sum = 0.f;
            for (int q = 0; q < p.S; ++q)
                sum += __ldcg(all + (size_t)q * kTile + e);
            red[e] = sum;
        }
        if (tid == 0)
            p.counters[nb] = 0u;
        __syncthreads();
    }

    // ---- epilogue: scale, EC up-projection, one rounding to bf16
    const int row = tid & (kRows - 1), th = tid >> 6;  // two token phases
    const int64_t n = (int64_t)nb * kRows + row;
    const float sn = p.s[n];
    float out[TOK / 2];
#pragma unroll
    for (int i = 0; i < TOK / 2; ++i)
        out[i] = sn * red[row * TOK + th + 2 * i];
    if (p.ec) {
        const uint16_t *bt = p.Bt + n * p.rp;
        for (int j = 0; j < p.rp; j += 8) {
            const uint4 bv = ld_nc(bt + j);
            const float bj[8] = {bf16_lo(bv.x), bf16_hi(bv.x), bf16_lo(bv.y), bf16_hi(bv.y),
                                 bf16_lo(bv.z), bf16_hi(bv.z), bf16_lo(bv.w), bf16_hi(bv.w)};
#pragma unroll
            for (int i = 0; i < TOK / 2; ++i) {
                const int t = th + 2 * i;
                if (t < p.M) {
                    const uint4 vv = __ldcg(reinterpret_cast<const uint4 *>(p.v + (int64_t)t * p.rp + j));
                    out[i] += bf16_lo(vv.x) * bj[0] + bf16_hi(vv.x) * bj[1] + bf16_lo(vv.y) * bj[2] +
                              bf16_hi(vv.y) * bj[3] + bf16_lo(vv.z) * bj[4] + bf16_hi(vv.z) * bj[5] +
                              bf16_lo(vv.w) * bj[6] + bf16_hi(vv.w) * bj[7];
                }
            }
        }
    }
    if (n < p.N) {
#pragma unroll
        for (int i = 0; i < TOK / 2; ++i) {
            const int t = th + 2 * i;
            if (t < p.M)
                p.y[(int64_t)t * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(out[i]));
        }
    }
}

void pick_split(const Packed &pk, int num_sms, int &S, int &bps)
{
    const int nkb = (int)(pk.Kp / 128);
    const int nblocks = (int)(pk.Np / kRows);
    // aim for about four CTAs per SM, at most kMaxBps k blocks per CTA
    int target = std::max(1, (4 * num_sms + nblocks - 1) / nblocks);
    S = std::min(target, nkb);
    bps = (nkb + S - 1) / S;
    if (bps > kMaxBps)
        bps = kMaxBps;
    S = (nkb + bps - 1) / bps;
}

}  // namespace

size_t decode_part_floats(const Packed &pk, int num_sms)
{
    int S, bps;
    pick_split(pk, num_sms, S, bps);
    return S > 1 ? (size_t)(pk.Np / kRows) * S * kRows * kDecodeMaxTokens : 0;
}

int decode_counters(const Packed &pk) { return (int)(pk.Np / kRows); }

cudaError_t launch_decode(const Packed &pk, const void *x, void *y, int64_t M, const uint16_t *v,
                          bool ec, const DecodeWork &w, cudaStream_t st,
                          int num_sms)
{
    if (M <= 0)
        return cudaSuccess;
    if (M > kDecodeMaxTokens)
        return cudaErrorInvalidValue;
    DecodeParams p;
    p.codes = pk.codes;
    p.s = pk.s;
    p.z = pk.z;
    p.x = static_cast<const uint16_t *>(x);
    p.y = static_cast<uint16_t *>(y);
    p.v = v;
    p.Bt = pk.Bt;
    p.part = w.part;
    p.counters = w.counters;
    p.M = M;
    p.K = pk.K;
    p.Kp = pk.Kp;
    p.N = pk.N;
    p.rp = pk.rp;
    p.ec = (ec && pk.r > 0) ? 1 : 0;
    pick_split(pk, num_sms, p.S, p.bps);
    const int T = M <= 8 ? 1 : (M <= 16 ? 2 : 4);
    const int nblocks = (int)(pk.Np / kRows);
    if (nblocks > w.n_counters || (p.S > 1 && (size_t)nblocks * p.S * kRows * 8 * T > w.part_floats))
        return cudaErrorInvalidValue;
    const size_t smem = std::max((size_t)8 * T * p.bps * 256, (size_t)kRows * 8 * T * sizeof(float));

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(nblocks * p.S));
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void (*fn)(DecodeParams) = T == 1 ? decode_w4ec_kernel<1> : (T == 2 ? decode_w4ec_kernel<2> : decode_w4ec_kernel<4>);
    if (smem > 48 * 1024) {
        cudaError_t e = raise_smem_limit(reinterpret_cast<const void *>(fn), smem);
        if (e != cudaSuccess)
            return e;
    }
    return cudaLaunchKernelEx(&cfg, fn, p);
}

}  // namespace spear
