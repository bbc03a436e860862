// Decode-size W4 GEMM with the Error Compensator fused in, one CTA per 16
// weight rows over the whole of K.
//
// SPEAR, "A System for Post-Quantization Error-Adaptive Recovery Enabling
// Efficient Low-Bit LLM Serving", Abstract: the post-EC computation is fused
// into the low-bit GEMM.  For a few tokens (at most 16) on a layer whose
// 16-row slice of codes fits in shared memory (K up to 8192), the layer's
// critical path "previous layer done -> this layer done" is kept free of any
// exchange between CTAs for the main product:
//
//  * a row CTA owns 16 weight rows and all of K.  Before waiting for the
//    previous kernel (programmatic dependent launch) it requests all its
//    codes (TMA boxes of 16 rows x up to eight 256-k chunks): they do not
//    depend on earlier kernels;
//  * each consumer warp takes a contiguous range of 64-k sub-blocks, reads
//    its activations straight from global memory (one sub-block ahead),
//    dequantises the codes in registers to exact (q - z) bf16 pairs and runs
//    mma.sync m16n8k16 with the weight rows on the 16-row side and the tokens
//    on the 8-column side (the same fragment layout as the split-K decode
//    kernel);
//  * the warps' partial tiles are summed in shared memory in warp order and
//    the CTA writes its 16 rows of y;
//  * with the EC, R1p/16 x 4 extra CTAs (the first ones of the grid) compute
//    partials of u = x . [w_g, A] (16 rows of G over a quarter of K each) and
//    publish them behind a release increment.  In every row CTA the spare
//    warp waits for the count while the others compute, sums the four
//    partials in order into shared memory, and the epilogue forms
//        y[t,n] = bf16( s[n] * acc[t,n] + g_t * sum_j u[t,1+j] B[j,n] ),
//        g_t = 1 / (1 + exp(-(u[t,0] + b_g))),
//    every wait bounded (about a second, then a timeout in the status word).
#include <algorithm>
#include <new>

#include "async_utils.cuh"
#include "kernels.h"
#include "tensor_map.h"

namespace spear {
namespace {

constexpr int kRowsPerCta = 16;   // weight rows of a row CTA (one MMA row tile)
constexpr int kECSplit = 4;       // EC CTAs per 16 rows of G (quarters of K)
constexpr int kUStrideR = 32;     // token stride of the published u rows (as the split-K kernel)
constexpr int kMaxBoxes = 4;      // TMA boxes per CTA (K <= 8192)
constexpr int kRowsMaxK = 8192;
constexpr int kRowsMaxTokens = 16;
constexpr size_t kRowsSmemPerCta = 112 * 1024;   // two CTAs per SM

struct RowsMaps {
    CUtensorMap codes;   // tiled codes seen as [blocks][64 rows][32 words]: box 32 x 16 rows x cb blocks
    CUtensorMap g;       // [R1p][Kp] bf16 seen as [Kp/64][R1p][64]: box 64 x 16 rows x gkb k-blocks
    int cb, gkb;
};

struct RowsParams {
    const uint16_t *x;
    const uint16_t *Bt;   // [Np][rp]
    const float *s;
    const uint8_t *z;
    uint16_t *y;
    float *ws_u;          // [kECSplit][R1p][kUStrideR]
    unsigned *flags;      // [0] EC CTAs published, [1] row CTAs done with u
    int *status;
    int64_t M, N, K;
    int nsb, nch;         // 64-k sub-blocks and 256-k chunks of Kp
    int cb, nbox;         // chunks per code box, code boxes per row CTA
    int gkb, ngbox;       // k-blocks per G box, G boxes per EC CTA
    int JB, NR;           // 16-row groups of G (0 without the EC), row CTAs
    int r, rp, R1p;
    uint32_t region;      // bytes of the codes / G region of shared memory
    uint32_t xs_off;      // byte offset of the staged activations
    int xstage;           // the activations are staged in shared memory (a few tokens)
    float b_g;
    const void *pf;       // codes of the next layer, prefetched into L2 (null for none)
    uint64_t pf_bytes;
};

__device__ __forceinline__ void named_bar_sync(int id, int n)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Bounded wait (one thread) until `expected` EC CTAs have published.
__device__ __forceinline__ bool wait_count(const unsigned *flag, unsigned expected, int *status)
{
    const long long t0 = clock64();
    while (ld_acquire_gpu(flag) < expected) {
        if (clock64() - t0 > kWaitBudgetCycles) {
            atomicOr(status, kStatusTimeout);
            return false;
        }
        __nanosleep(64);
    }
    return true;
}

// Shared memory after the codes / G region: the warps' partial tiles
// [W][TOK][16] fp32, the B^T rows of the CTA [16][rp] bf16, u0 [TOK] and
// uT [TOK][rp] fp32.
template <int TOK>
__host__ __device__ constexpr uint32_t rows_tail_bytes(int W, int rp)
{
    return (uint32_t)(W * TOK * kRowsPerCta * 4 + 32 * rp + 4 * TOK * (1 + rp));
}

// Register budget: MINB CTAs per SM.
template <int T, int W, int MINB>
__global__ void __launch_bounds__(32 * W + 32, MINB)
decode_rows_kernel(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_g,
                   RowsParams p)
{
    constexpr int TOK = 8 * T;
    constexpr int kConsumers = 32 * W;
    constexpr int kEpi = kRowsPerCta * TOK;   // epilogue threads: (row, token) pairs
    static_assert(kEpi <= kConsumers, "one epilogue thread per output of the CTA");
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t bars[kMaxBoxes + 1];   // code / G boxes, then "u is in shared memory"

    pdl_launch_dependents();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gid = lane >> 2, cl = lane & 3;
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *const bp = smem_raw + (base - raw);
    float *const red = reinterpret_cast<float *>(bp + p.region);
    uint16_t *const bts = reinterpret_cast<uint16_t *>(bp + p.region + W * TOK * kRowsPerCta * 4);
    float *const u0 = reinterpret_cast<float *>(bp + p.region + W * TOK * kRowsPerCta * 4 + 32 * p.rp);
    float *const uT = u0 + TOK;

    const int nec = p.JB * kECSplit;
    const bool is_u = (int)blockIdx.x < nec;
    const int grp = is_u ? (int)blockIdx.x / kECSplit : 0;   // G rows 16 grp .. + 15
    const int qk = is_u ? (int)blockIdx.x % kECSplit : 0;    // quarter of K
    const int n0 = is_u ? 0 : ((int)blockIdx.x - nec) * kRowsPerCta;
    const int nbox = is_u ? p.ngbox : p.nbox;
    const int nsb_cta = is_u ? p.nsb / kECSplit : p.nsb;     // 64-k sub-blocks of this CTA
    const int spb = is_u ? p.gkb : 4 * p.cb;                 // sub-blocks per box

    if (warp == W && lane == 0) {
        for (int b = 0; b < nbox; ++b)
            mbar_init(smem_addr(&bars[b]), 1);
        mbar_init(smem_addr(&bars[kMaxBoxes]), 1);
        fence_mbarrier_init_cluster();
        // the weights do not depend on earlier kernels: request them all now
        for (int b = 0; b < nbox; ++b) {
            const uint32_t bar = smem_addr(&bars[b]);
            if (is_u) {
                mbar_expect_tx(bar, (uint32_t)p.gkb * 2048u);
                tma_load_3d(base + (uint32_t)(b * p.gkb) * 2048u, &tm_g, 0, kRowsPerCta * grp,
                            qk * nsb_cta + b * p.gkb, bar);
            } else {
                mbar_expect_tx(bar, (uint32_t)p.cb * 2048u);
                tma_load_3d(base + (uint32_t)(b * p.cb) * 2048u, &tm_codes, 0, n0 % 64,
                            (n0 / 64) * p.nch + b * p.cb, bar);
            }
        }
    }
    if (warp == W && !is_u && p.JB > 0) {
        // B^T rows of the epilogue, also independent of earlier kernels
        const int per_row = p.rp / 8;
        for (int i = lane; i < kRowsPerCta * per_row; i += 32) {
            const int row = i / per_row, c8 = i - row * per_row;
            reinterpret_cast<uint4 *>(bts)[i] = ld_nc(p.Bt + (int64_t)(n0 + row) * p.rp + 8 * c8);
        }
    }
    __syncthreads();   // the barriers are initialised

    if (warp < W) {
        // ---- main product: warp w owns sub-blocks [sb0, sb1) of this CTA
        uint32_t negg = 0, negh = 0;
        float s_epi = 0.f;
        if (!is_u) {
            const uint32_t zg = __ldg(p.z + n0 + gid), zh = __ldg(p.z + n0 + gid + 8);
            const uint32_t nbg = __bfloat16_as_ushort(__float2bfloat16_rn(-(float)(128u + zg)));
            const uint32_t nbh = __bfloat16_as_ushort(__float2bfloat16_rn(-(float)(128u + zh)));
            negg = nbg | (nbg << 16);
            negh = nbh | (nbh << 16);
            if (tid < kEpi)
                s_epi = __ldg(p.s + n0 + (tid & (kRowsPerCta - 1)));
        }
        const int64_t kbase = is_u ? (int64_t)qk * nsb_cta * 64 : 0;
        float acc[T][4], acc2[T][4];
#pragma unroll
        for (int n = 0; n < T; ++n)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                acc[n][i] = acc2[n][i] = 0.f;

        // one 64-k sub-block of the product, activations in xv
        auto product = [&](int sb, const uint4 (&xv)[T][2]) {
            if (!is_u) {
                // codes k = 64 sb + 16 cl + {0..15} of rows gid and gid + 8 (8 bytes
                // each) in chunk sb / 4, a [16 rows][128 B] tile with the 128B swizzle
                const uint8_t *ct = bp + (sb >> 2) * 2048;
                const int unit = ((2 * (sb & 3) + (cl >> 1)) ^ gid) * 16 + (cl & 1) * 8;
                const uint2 wgv = *reinterpret_cast<const uint2 *>(ct + gid * 128 + unit);
                const uint2 whv = *reinterpret_cast<const uint2 *>(ct + (gid + 8) * 128 + unit);
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const uint32_t wgw = j ? wgv.y : wgv.x, whw = j ? whv.y : whv.x;
                    // codes k = 8j + {0..7}: nibbles (m, m + 4) hold the pair k = 2m, 2m + 1,
                    // the order of the activations in one uint4
                    const uint32_t g0 = dequant_pair(wgw, negg), g1 = dequant_pair(wgw >> 4, negg);
                    const uint32_t g2 = dequant_pair(wgw >> 8, negg), g3 = dequant_pair(wgw >> 12, negg);
                    const uint32_t h0 = dequant_pair(whw, negh), h1 = dequant_pair(whw >> 4, negh);
                    const uint32_t h2 = dequant_pair(whw >> 8, negh), h3 = dequant_pair(whw >> 12, negh);
#pragma unroll
                    for (int n = 0; n < T; ++n) {
                        const uint4 v = xv[n][j];
                        float (&a)[4] = j ? acc2[n] : acc[n];
                        mma_bf16_16816(a, g0, h0, g1, h1, v.x, v.y);
                        mma_bf16_16816(a, g2, h2, g3, h3, v.z, v.w);
                    }
                }
            } else {
                // 16 rows of G, k = 64 sb + 16 cl + {0..15}: natural pairs, step s
                // covering k = 16 cl + 4s + {0,1} and + {2,3}
                const uint8_t *gt = bp + sb * 2048;
                const uint4 a0 = *reinterpret_cast<const uint4 *>(gt + gid * 128 + (((2 * cl) ^ gid) << 4));
                const uint4 a1 = *reinterpret_cast<const uint4 *>(gt + gid * 128 + (((2 * cl + 1) ^ gid) << 4));
                const uint4 b0 = *reinterpret_cast<const uint4 *>(gt + (gid + 8) * 128 + (((2 * cl) ^ gid) << 4));
                const uint4 b1 =
                    *reinterpret_cast<const uint4 *>(gt + (gid + 8) * 128 + (((2 * cl + 1) ^ gid) << 4));
                const uint32_t ga[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                const uint32_t ha[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                for (int n = 0; n < T; ++n) {
                    const uint32_t xa[8] = {xv[n][0].x, xv[n][0].y, xv[n][0].z, xv[n][0].w,
                                            xv[n][1].x, xv[n][1].y, xv[n][1].z, xv[n][1].w};
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        mma_bf16_16816((s & 1) ? acc2[n] : acc[n], ga[2 * s], ha[2 * s], ga[2 * s + 1],
                                       ha[2 * s + 1], xa[2 * s], xa[2 * s + 1]);
                }
            }
        };
        const int sb0 = warp * nsb_cta / W, sb1 = (warp + 1) * nsb_cta / W;
        pdl_wait();
        bool ok = true;
        if (p.xstage && !is_u) {
            // A few tokens: the row CTA's activations x[t][0 .. K) are staged in
            // shared memory first, one round trip for all of them (rows padded by
            // 16 bytes to spread them over the banks).  A CTA of u (one sub-block
            // per warp) reads its own directly and saves the staging barrier.
            const int xst = nsb_cta * 64 + 8;
            uint16_t *const xs = reinterpret_cast<uint16_t *>(bp + p.xs_off);
            const int mrows = p.M < TOK ? (int)p.M : TOK;
            const int per_row = nsb_cta * 8;
            for (int c = tid; c < mrows * per_row; c += kConsumers) {
                const int t = c / per_row, c8 = c - t * per_row;
                const int64_t k = kbase + 8 * c8;
                const uint4 v = k < p.K ? ld_nc(p.x + (int64_t)t * p.K + k) : make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4 *>(xs + t * xst + 8 * c8) = v;
            }
            named_bar_sync(2, kConsumers);
            if (sb0 < sb1) {
                for (int b = sb0 / spb; b <= (sb1 - 1) / spb && ok; ++b)
                    ok = mbar_wait_bounded(smem_addr(&bars[b]), 0);
                for (int sb = sb0; sb < sb1 && ok; ++sb) {
                    uint4 xv[T][2];
#pragma unroll
                    for (int n = 0; n < T; ++n) {
                        const int t = 8 * n + gid;
                        if (t < p.M) {
                            const uint16_t *src = xs + t * xst + sb * 64 + 16 * cl;
                            xv[n][0] = *reinterpret_cast<const uint4 *>(src);
                            xv[n][1] = *reinterpret_cast<const uint4 *>(src + 8);
                        } else {
                            xv[n][0] = make_uint4(0, 0, 0, 0);
                            xv[n][1] = xv[n][0];
                        }
                    }
                    product(sb, xv);
                }
            }
        } else if (sb0 < sb1) {
            // More tokens: every CTA staging all of x would multiply the traffic
            // from L2; each warp reads its own activations from global memory,
            // one sub-block ahead.
            auto load_x = [&](int sb, uint4 (&dst)[T][2]) {
                const int64_t k = kbase + (int64_t)sb * 64 + 16 * cl;
#pragma unroll
                for (int n = 0; n < T; ++n) {
                    const int64_t t = 8 * n + gid;
                    if (t < p.M && k < p.K) {
                        const uint16_t *src = p.x + t * p.K + k;
                        dst[n][0] = ld_nc(src);
                        dst[n][1] = ld_nc(src + 8);
                    } else {
                        dst[n][0] = make_uint4(0, 0, 0, 0);
                        dst[n][1] = dst[n][0];
                    }
                }
            };
            uint4 xv[T][2], xn[T][2];
            load_x(sb0, xv);
            for (int b = sb0 / spb; b <= (sb1 - 1) / spb && ok; ++b)
                ok = mbar_wait_bounded(smem_addr(&bars[b]), 0);
            for (int sb = sb0; sb < sb1 && ok; ++sb) {
                if (sb + 1 < sb1)
                    load_x(sb + 1, xn);
                product(sb, xv);
                if (sb + 1 < sb1) {
#pragma unroll
                    for (int n = 0; n < T; ++n) {
                        xv[n][0] = xn[n][0];
                        xv[n][1] = xn[n][1];
                    }
                }
            }
        }
        if (!ok)
            atomicOr(p.status, kStatusTimeout);
        // partial tile of this warp: red[warp][token][row]
        float *mine = red + warp * TOK * kRowsPerCta;
#pragma unroll
        for (int n = 0; n < T; ++n) {
            const int col = 8 * n + 2 * cl;
            mine[col * kRowsPerCta + gid] = acc[n][0] + acc2[n][0];
            mine[(col + 1) * kRowsPerCta + gid] = acc[n][1] + acc2[n][1];
            mine[col * kRowsPerCta + gid + 8] = acc[n][2] + acc2[n][2];
            mine[(col + 1) * kRowsPerCta + gid + 8] = acc[n][3] + acc2[n][3];
        }
        named_bar_sync(2, kConsumers);

        if (is_u) {
            // ---- publish this CTA's partial of u rows 16 grp .. + 15 (sum over the
            // warps in warp order); the row CTAs sum the quarters in order
            for (int e = tid; e < kEpi; e += kConsumers) {
                float sum = red[e];
                for (int w = 1; w < W; ++w)
                    sum += red[w * TOK * kRowsPerCta + e];
                const int t = e / kRowsPerCta, row = e - t * kRowsPerCta;
                p.ws_u[((int64_t)qk * p.R1p + kRowsPerCta * grp + row) * kUStrideR + t] = sum;
            }
            named_bar_sync(2, kConsumers);
            if (tid == 0)
                red_release_gpu_add(&p.flags[0], 1u);
        } else {
            // ---- epilogue: thread = (row tid mod 16, token tid / 16)
            if (tid < kEpi) {
                const int row = tid & (kRowsPerCta - 1), t = tid / kRowsPerCta;
                float sum = red[tid];
                for (int w = 1; w < W; ++w)
                    sum += red[w * TOK * kRowsPerCta + tid];
                float out = s_epi * sum;
                // u is in shared memory (tokens below M) once the spare warp has
                // arrived on this barrier (bounded wait)
                if (p.JB > 0 && !mbar_wait_bounded(smem_addr(&bars[kMaxBoxes]), 0))
                    atomicOr(p.status, kStatusTimeout);
                if (p.JB > 0 && t < p.M) {
                    const uint16_t *btrow = bts + row * p.rp;
                    const float *ut = uT + t * p.rp;
                    float corr = 0.f;
                    for (int j0 = 0; j0 < p.rp; j0 += 8) {
                        const uint4 bv = *reinterpret_cast<const uint4 *>(btrow + j0);
                        const float4 v0 = *reinterpret_cast<const float4 *>(ut + j0);
                        const float4 v1 = *reinterpret_cast<const float4 *>(ut + j0 + 4);
                        corr += v0.x * bf16_lo(bv.x) + v0.y * bf16_hi(bv.x) + v0.z * bf16_lo(bv.y) +
                                v0.w * bf16_hi(bv.y) + v1.x * bf16_lo(bv.z) + v1.y * bf16_hi(bv.z) +
                                v1.z * bf16_lo(bv.w) + v1.w * bf16_hi(bv.w);
                    }
                    const float g = 1.0f / (1.0f + expf(-(u0[t] + p.b_g)));
                    out += g * corr;
                }
                const int64_t n = n0 + row;
                if (t < p.M && n < p.N)
                    p.y[(int64_t)t * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(out));
            }
            if (p.JB > 0 && tid == 0 && atomicAdd(&p.flags[1], 1u) == (unsigned)(p.NR - 1)) {
                // every row CTA has read u: reset for the next forward
                p.flags[1] = 0u;
                p.flags[0] = 0u;
            }
        }
    } else {
        // ---- spare warp: once this CTA's codes have landed, its share of the next
        // layer's codes goes from HBM into L2 (the copies no longer compete with
        // this layer's own); no copy may still be landing when the CTA leaves
        if (lane == 0) {
            for (int b = 0; b < nbox; ++b)
                mbar_wait_bounded(smem_addr(&bars[b]), 0);
            prefetch_l2_share(p.pf, p.pf_bytes);
        }
        __syncwarp();
        // then, in a row CTA, fetch u while the others compute
        if (!is_u && p.JB > 0) {
            pdl_wait();   // the previous forward has reset the counters
            int good = 1;
            if (lane == 0)
                good = wait_count(&p.flags[0], (unsigned)(p.JB * kECSplit), p.status) ? 1 : 0;
            good = __shfl_sync(0xffffffffu, good, 0);
            // u[row][4 t4 .. 4 t4 + 3] for rows 0..r and the groups of four tokens
            // that hold the M real ones, the four quarters summed in order.  This
            // warp shares its SM with the busy consumer warps, so the loop is kept
            // short: 16-byte loads, two (row, group) pairs 32 apart per lane in flight.
            const int mt4 = ((p.M < TOK ? (int)p.M : TOK) + 3) / 4;
            const int npair = (1 + p.r) * mt4;
            for (int p0 = lane; p0 < npair; p0 += 64) {
                float4 v[2][kECSplit];
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int pr = p0 + 32 * i, row = pr / mt4, t4 = pr - row * mt4;
#pragma unroll
                    for (int q = 0; q < kECSplit; ++q)
                        v[i][q] = (good && pr < npair)
                                      ? __ldcg(reinterpret_cast<const float4 *>(
                                            p.ws_u + ((int64_t)q * p.R1p + row) * kUStrideR + 4 * t4))
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int pr = p0 + 32 * i, row = pr / mt4, t4 = pr - row * mt4;
                    if (pr >= npair)
                        continue;
                    float4 u = v[i][0];
#pragma unroll
                    for (int q = 1; q < kECSplit; ++q) {
                        u.x += v[i][q].x;
                        u.y += v[i][q].y;
                        u.z += v[i][q].z;
                        u.w += v[i][q].w;
                    }
                    const float uu[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        if (row == 0)
                            u0[4 * t4 + c] = uu[c];
                        else
                            uT[(4 * t4 + c) * p.rp + row - 1] = uu[c];
                    }
                }
            }
            for (int e = lane; e < TOK * (p.rp - p.r); e += 32) {
                const int t = e / (p.rp - p.r), j = p.r + e - t * (p.rp - p.r);
                uT[t * p.rp + j] = 0.f;
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_addr(&bars[kMaxBoxes]));   // release: the warp's writes of u come first
        }
    }
    // no warp leaves before the others are done
    __syncthreads();
}

template <int T, int W, int MINB>
const void *rows_ptr()
{
    return reinterpret_cast<const void *>(decode_rows_kernel<T, W, MINB>);
}

// Consumer warps per CTA: sixteen for one token group, eight for two.
int rows_warps(int T) { return T == 1 ? 16 : 8; }

uint32_t rows_region(const Packed &pk, int cb, int gkb)
{
    const int nch = (int)(pk.Kp / 256);
    const int code_bytes = (nch + cb - 1) / cb * cb * 2048;
    const int g_bytes = pk.r > 0 ? (nch + gkb - 1) / gkb * gkb * 2048 : 0;
    return (uint32_t)std::max(code_bytes, g_bytes);
}

struct RowsPlan {
    int T, W, cb, gkb, xstage;
    uint32_t region, xs_off;
    size_t smem;
};

// Token groups, warps and shared-memory layout.  Up to 8 tokens the
// activations of all of K are staged in shared memory when two CTAs still fit
// on an SM; for more, staging them in every CTA would cost more L2 traffic
// than it saves in latency.
void rows_plan(const Packed &pk, int64_t M, RowsPlan &pl)
{
    const int nch = (int)(pk.Kp / 256);
    pl.T = M <= 8 ? 1 : 2;
    pl.W = rows_warps(pl.T);
    pl.cb = std::min(8, nch);
    pl.gkb = std::min(16, nch);
    pl.region = rows_region(pk, pl.cb, pl.gkb);
    const size_t tail = pl.T == 1 ? rows_tail_bytes<8>(pl.W, pk.rp) : rows_tail_bytes<16>(pl.W, pk.rp);
    pl.xs_off = (uint32_t)((pl.region + tail + 15) / 16 * 16);
    const size_t xs_bytes = (size_t)std::min<int64_t>(M, 8) * (pk.Kp + 8) * 2;
    pl.xstage = pl.T == 1 && pl.xs_off + xs_bytes + 1024 <= kRowsSmemPerCta ? 1 : 0;
    pl.smem = pl.xs_off + (pl.xstage ? xs_bytes : 0) + 1024;
}

}  // namespace

bool decode_rows_shape(const Packed &pk)
{
    return pk.K % 64 == 0 && pk.Kp <= kRowsMaxK && pk.rp <= 128;
}

// The grid (row CTAs and, with the EC, the CTAs of u) must be one wave of two
// CTAs per SM: a second wave would wait for a whole first one.
bool decode_rows_fits(const Packed &pk, int64_t M, int num_sms)
{
    const int64_t ctas = pk.Np / kRowsPerCta + (pk.r > 0 ? (int64_t)pk.R1p / kRowsPerCta * kECSplit : 0);
    if (!(M >= 1 && M <= kRowsMaxTokens && decode_rows_shape(pk) && ctas <= 2LL * num_sms))
        return false;
    // the occupancy calculator must agree that the grid is one wave (the row
    // CTAs wait, bounded, for the CTAs of u)
    RowsPlan pl;
    rows_plan(pk, M, pl);
    const void *fn = pl.T == 1 ? rows_ptr<1, 16, 2>() : rows_ptr<2, 8, 2>();
    return grid_is_one_wave(fn, 32 * pl.W + 32, pl.smem, 1, ctas, num_sms);
}

cudaError_t decode_rows_prepare(const Packed &pk, void **maps)
{
    RowsMaps *m = static_cast<RowsMaps *>(*maps);
    if (!m) {
        m = new (std::nothrow) RowsMaps();
        if (!m)
            return cudaErrorMemoryAllocation;
        *maps = m;
    }
    const int nch = (int)(pk.Kp / 256);
    m->cb = std::min(8, nch);
    m->gkb = std::min(16, nch);
    // the split-K kernel's view of the tiled codes, boxes of 16 rows x cb blocks
    const uint64_t dims[3] = {32, 64, (uint64_t)(pk.Np / 64) * (uint64_t)nch};
    const uint64_t strides[2] = {128, 8192};
    const uint32_t box[3] = {32, (uint32_t)kRowsPerCta, (uint32_t)m->cb};
    cudaError_t e = make_map_nd(&m->codes, pk.codes, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, dims, strides, box,
                                CU_TENSOR_MAP_SWIZZLE_128B);
    if (e == cudaSuccess && pk.r > 0) {
        const uint64_t gd[3] = {64, (uint64_t)pk.R1p, (uint64_t)(pk.Kp / 64)};
        const uint64_t gs[2] = {(uint64_t)pk.Kp * 2, 128};
        const uint32_t gb[3] = {64, (uint32_t)kRowsPerCta, (uint32_t)m->gkb};
        e = make_map_nd(&m->g, pk.G, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, gd, gs, gb, CU_TENSOR_MAP_SWIZZLE_128B);
    } else if (e == cudaSuccess) {
        m->g = m->codes;
    }
    return e;
}

void decode_rows_free(void *maps) { delete static_cast<RowsMaps *>(maps); }

cudaError_t launch_decode_rows(const Packed &pk, const void *maps, const void *x, void *y, int64_t M, bool ec,
                               const DecodeWork &w, int *status, cudaStream_t st, int num_sms)
{
    if (!decode_rows_fits(pk, M, num_sms) || !maps)
        return cudaErrorInvalidValue;
    const RowsMaps *m = static_cast<const RowsMaps *>(maps);
    const bool use_ec = ec && pk.r > 0;
    RowsParams p;
    p.x = static_cast<const uint16_t *>(x);
    p.Bt = pk.Bt;
    p.s = pk.s;
    p.z = pk.z;
    p.y = static_cast<uint16_t *>(y);
    p.ws_u = w.ws_u;
    p.flags = w.flags;
    p.status = status;
    p.M = M;
    p.N = pk.N;
    p.K = pk.K;
    p.nsb = (int)(pk.Kp / 64);
    p.nch = (int)(pk.Kp / 256);
    p.cb = m->cb;
    p.nbox = (p.nch + p.cb - 1) / p.cb;
    p.gkb = m->gkb;
    p.ngbox = (p.nch + p.gkb - 1) / p.gkb;
    p.JB = use_ec ? pk.R1p / kRowsPerCta : 0;
    p.NR = (int)(pk.Np / kRowsPerCta);
    p.r = pk.r;
    p.rp = pk.rp;
    p.R1p = pk.R1p;
    RowsPlan pl;
    rows_plan(pk, M, pl);
    if (pl.cb != m->cb || pl.gkb != m->gkb)
        return cudaErrorInvalidValue;
    p.region = pl.region;
    p.xs_off = pl.xs_off;
    p.xstage = pl.xstage;
    p.b_g = pk.b_g;
    p.pf = w.pf;
    p.pf_bytes = w.pf_bytes;
    if (p.nbox > kMaxBoxes || p.ngbox > kMaxBoxes)
        return cudaErrorInvalidValue;
    const int T = pl.T;
    const int W = pl.W;
    const size_t smem = pl.smem;
    const void *fn = T == 1 ? rows_ptr<1, 16, 2>() : rows_ptr<2, 8, 2>();
    cudaError_t e = raise_smem_limit(fn, smem);
    if (e != cudaSuccess)
        return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(p.JB * kECSplit + p.NR));
    cfg.blockDim = dim3((unsigned)(32 * W + 32));
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (T == 1)
        return cudaLaunchKernelEx(&cfg, decode_rows_kernel<1, 16, 2>, m->codes, m->g, p);
    return cudaLaunchKernelEx(&cfg, decode_rows_kernel<2, 8, 2>, m->codes, m->g, p);
}

}  // namespace spear
