// Decode-size W4 GEMM (a few tokens) with the Error Compensator fused in.
//
// SPEAR, "A System for Post-Quantization Error-Adaptive Recovery Enabling
// Efficient Low-Bit LLM Serving", Abstract: the post-EC computation is fused
// into the low-bit GEMM.  For a few tokens the layer is bound by reading the
// int4 codes from HBM, and in a decode pass its critical path is the chain
// "previous layer done -> this layer done", so the kernel is built to stream
// the weights before that chain starts and to keep the chain short:
//
//  * one kernel per forward; a cluster of CS CTAs owns 64 weight rows, each
//    CTA one K/CS slice of them;
//  * before waiting for the previous kernel (programmatic dependent launch)
//    every CTA starts TMA copies of its whole slice of codes (and the
//    cluster's first CTA those of the B^T rows of its epilogue), so the
//    weight stream overlaps the previous layer; only the activations are
//    fetched after the wait;
//  * eight warps per CTA, two per 16-row group splitting the 64-wide
//    sub-blocks, so the dequantise-MMA chains of one warp hide another's;
//  * weight rows sit on the 16-row side of mma.sync m16n8k16 and tokens on
//    the 8-column side, so a code is read once for up to 32 tokens; the
//    codes are dequantised in registers to exact (q - z) bf16 pairs (two
//    nibbles 16 bits apart per register, set into the mantissa of 128.0 and
//    offset by one bf16 fma), and the activations are paired to match with
//    one byte permute per register, the k order inside the MMA being
//    permuted accordingly;
//  * the K split is summed inside the cluster, in rank order
//    (deterministic), with no global round trip: the other CTAs push their
//    partial tiles into receive slots of the first CTA (st.async, counted on
//    one mbarrier whose cluster handshake happens before the wait for the
//    previous kernel); where the slots do not fit in shared memory the first
//    CTA pulls the tiles over distributed shared memory between two cluster
//    barriers instead;
//  * the EC down-projection u = x . [w_g, A] runs on R1p/16 extra clusters
//    of the same grid (the first ones) with the same slicing; each of their
//    CTAs publishes its partial of u in global memory and counts it with a
//    release increment, and the first CTA of each 64-row cluster, once the
//    count is complete, sums the partials in rank order for its epilogue
//        y[t,n] = bf16( s[n] * acc[t,n] + g_t * sum_j u[t,1+j] B[j,n] ),
//        g_t = 1 / (1 + exp(-(u[t,0] + b_g))),
//    with a bounded wait (about a second) that records a timeout in the
//    handle's status word instead of hanging.
#include <algorithm>
#include <new>

#include "async_utils.cuh"
#include "kernels.h"
#include "tensor_map.h"

namespace spear {
namespace {

constexpr int kRows = 64;       // weight rows per cluster (four warps x 16)
constexpr int kChunk = 256;     // k per code chunk (one 8 KB TMA box of 64 rows)
constexpr int kMaxChunks = 8;   // so K/CS <= 2048
constexpr int kUStride = 32;    // token stride of the published u rows

struct Maps {
    CUtensorMap codes;    // tiled codes, one box = one 8 KB block (64 rows x 256 k), 128B swizzle
    CUtensorMap g;        // [R1p][Kp] bf16, boxes of 64 x 16, 128B swizzle
    CUtensorMap bt;       // [Np][rp] bf16, boxes of rp x 64
};

struct DecodeParams {
    const uint16_t *Bt;   // [Np][rp]
    const float *s;
    const uint8_t *z;
    uint16_t *y;
    float *ws_u;          // [CS][R1p][kUStride] fp32: one partial of u per rank
    unsigned *flags;      // [0] EC CTAs published, [1] row clusters done with u
    int *status;
    int64_t M, N, Kp;
    int KS, nch;          // k per CTA (a multiple of 256), code chunks per CTA
    int JB, NC;           // EC clusters, 64-row clusters
    int r, rp, R1p;
    int push;             // partial tiles pushed into receive slots of the first CTA
    float b_g;
};

struct Smem {
    uint32_t codes, x, bt, red, u, recv;   // byte offsets from the 1024-aligned base
    uint32_t total;
};

// nslots receive slots of one partial tile (64 rows x TOK fp32) each.
template <int TOK>
__host__ __device__ inline Smem smem_layout(int KS, int rp, int R1p, int nslots)
{
    Smem m;
    m.codes = 0;                                   // 32*KS bytes: codes (64 rows) or G (16 rows bf16)
    m.x = m.codes + 32 * KS;                       // 2*TOK*KS bytes: activation sub-tiles
    m.bt = m.x + 2 * TOK * KS;                     // 128*rp bytes: B^T rows of the cluster
    m.red = m.bt + 128 * rp;                       // 512*TOK bytes: partial tiles
    m.u = m.red + 512 * TOK;                       // u0 [TOK], uT [TOK][rp] (fp32)
    m.recv = (m.u + 4 * TOK * (rp + 1) + 15) & ~15u;
    m.total = m.recv + nslots * 256 * TOK;
    return m;
}

__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity) { return mbar_wait_bounded(bar, parity); }

constexpr int kThreads = 256;   // 8 warps: two per 16-row group, splitting the sub-blocks
constexpr int kEcWarp = kThreads / 32 - 1;

// Bounded wait (one thread) until every CTA of the EC clusters has published
// its partial u; false if it ran out (the timeout is recorded in the status).
__device__ __forceinline__ bool wait_u_published(const DecodeParams &p, unsigned expected)
{
    const long long t0 = clock64();
    while (ld_acquire_gpu(&p.flags[0]) < expected) {
        if (clock64() - t0 > kWaitBudgetCycles) {
            atomicOr(p.status, kStatusTimeout);
            return false;
        }
        __nanosleep(32);
    }
    return true;
}

template <int T>
__global__ void __launch_bounds__(kThreads)
decode_w4ec_kernel(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_g,
                   const __grid_constant__ CUtensorMap tm_bt, const __grid_constant__ CUtensorMap tm_x,
                   DecodeParams p, int CS)
{
    constexpr int TOK = 8 * T;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t bars[kMaxChunks + 3];

    pdl_launch_dependents();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gid = lane >> 2, cl = lane & 3;
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *const bp = smem_raw + (base - raw);
    const bool push = p.push != 0;
    const Smem L = smem_layout<TOK>(p.KS, p.rp, p.R1p, push ? CS - 1 : 0);
    const uint32_t rank = cluster_ctarank();
    const int cluster = blockIdx.x / CS;
    const bool is_u = cluster < p.JB;
    const int k0 = (int)rank * p.KS;
    // the last ranks may hold a shorter (or empty) slice when K/256 is not a multiple of CS
    const int nch = max(0, min(p.nch, (int)((p.Kp - k0) / kChunk)));
    const int nsub = 4 * nch;
    const uint32_t bar_chunk = smem_addr(&bars[0]);
    const uint32_t bar_x = smem_addr(&bars[kMaxChunks]);
    const uint32_t bar_bt = smem_addr(&bars[kMaxChunks + 1]);
    const uint32_t bar_recv = smem_addr(&bars[kMaxChunks + 2]);
    const int n0 = is_u ? 0 : (cluster - p.JB) * kRows;

    // loads that do not depend on earlier kernels are issued before waiting
    // for them: the epilogue scale of this thread's row and the zero points
    // of its two MMA rows
    const float s_epi = (!is_u && rank == 0) ? __ldg(p.s + n0 + (tid & (kRows - 1))) : 0.f;
    const int rg = 16 * (warp & 3) + gid;  // MMA rows rg and rg + 8 (64-row clusters)
    const uint32_t zg_raw = is_u ? 0u : (uint32_t)__ldg(p.z + n0 + rg);
    const uint32_t zh_raw = is_u ? 0u : (uint32_t)__ldg(p.z + n0 + rg + 8);
    if (tid == 0) {
        for (int c = 0; c < kMaxChunks + 3; ++c)
            mbar_init(bar_chunk + 8 * c, 1);
        fence_mbarrier_init_cluster();
        if (push && !is_u && rank == 0 && CS > 1)
            mbar_expect_tx(bar_recv, (uint32_t)((CS - 1) * kRows * TOK * 4));
        // the weights do not depend on earlier kernels: start them now
        for (int c = 0; c < nch; ++c) {
            const uint32_t bar = bar_chunk + 8 * c;
            mbar_expect_tx(bar, 8192);
            if (is_u) {
                for (int i = 0; i < 4; ++i)
                    tma_load_2d(base + L.codes + c * 8192 + i * 2048, &tm_g, k0 + c * kChunk + i * 64, 16 * cluster,
                                bar);
            } else {
                tma_load_3d(base + L.codes + c * 8192, &tm_codes, 0, 0,
                            (n0 / kRows) * (int)(p.Kp / kChunk) + (k0 / kChunk) + c, bar);
            }
        }
        if (!is_u && rank == 0 && p.rp > 0) {
            mbar_expect_tx(bar_bt, 128 * p.rp);   // B^T rows of the cluster, for the epilogue
            tma_load_2d(base + L.bt, &tm_bt, 0, n0, bar_bt);
        }
    }
    __syncthreads();
    if (push)
        cluster_arrive_relaxed();   // the receive barrier of the first CTA is initialised
    __shared__ int s_xok;
    if (tid == 0) {
        // the activations are written by the previous kernel in the stream
        pdl_wait();
        mbar_expect_tx(bar_x, 2 * TOK * kChunk * nch);
        for (int i = 0; i < nsub; ++i)
            tma_load_2d(base + L.x + i * (TOK * 128), &tm_x, k0 + 64 * i, 0, bar_x);
        s_xok = wait_bounded(bar_x, 0) ? 1 : 0;
    }
    // the other threads sleep in this barrier instead of polling (they would
    // take issue slots from the previous layer's CTAs on the same SM); their
    // own wait below then returns at once and orders their reads after the copy
    __syncthreads();
    bool ok = s_xok != 0 && wait_bounded(bar_x, 0);

    // two accumulator sets (even / odd code word) halve the MMA dependency chains
    float acc[T][4], acc2[T][4];
#pragma unroll
    for (int n = 0; n < T; ++n)
#pragma unroll
        for (int i = 0; i < 4; ++i)
            acc[n][i] = acc2[n][i] = 0.f;

    float *red = reinterpret_cast<float *>(bp + L.red);
    if (!is_u) {
        // ---- 64 weight rows: warps w and w+4 own rows 16w .. 16w+15, sub-blocks of parity w>>2
        const int kpar = warp >> 2;
        const uint32_t nbg = __bfloat16_as_ushort(__float2bfloat16_rn(-(float)(128u + zg_raw)));
        const uint32_t nbh = __bfloat16_as_ushort(__float2bfloat16_rn(-(float)(128u + zh_raw)));
        const uint32_t negg = nbg | (nbg << 16), negh = nbh | (nbh << 16);
        // the codes were requested before the wait for the previous kernel and
        // have normally landed: one wait for all, so that no compiler barrier
        // sits inside the loop
        for (int c = 0; c < nch; ++c)
            ok = ok && wait_bounded(bar_chunk + 8 * c, 0);
#pragma unroll 2
        for (int c = 0; c < (ok ? nch : 0); ++c) {
            const uint8_t *ctile = bp + L.codes + c * 8192;
#pragma unroll
            for (int sb2 = 0; sb2 < 2; ++sb2) {
                const int sb = 2 * sb2 + kpar;
                // codes k = 64 sb + 16 cl + {0..15} of rows rg and rg + 8 (8 bytes each)
                const int chunk = ((2 * sb + (cl >> 1)) ^ (rg & 7)) * 16 + (cl & 1) * 8;
                const uint2 wgv = *reinterpret_cast<const uint2 *>(ctile + rg * 128 + chunk);
                const uint2 whv = *reinterpret_cast<const uint2 *>(ctile + (rg + 8) * 128 + chunk);
                const uint8_t *xt = bp + L.x + (4 * c + sb) * (TOK * 128);
                uint4 xv[T][2];
#pragma unroll
                for (int n = 0; n < T; ++n) {
                    const int t = 8 * n + gid;
                    xv[n][0] = *reinterpret_cast<const uint4 *>(xt + t * 128 + (((2 * cl) ^ (t & 7)) << 4));
                    xv[n][1] = *reinterpret_cast<const uint4 *>(xt + t * 128 + (((2 * cl + 1) ^ (t & 7)) << 4));
                }
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const uint32_t wgw = j ? wgv.y : wgv.x, whw = j ? whv.y : whv.x;
                    // codes k = 8j + {0..7}: pairs (0,4) (1,5) (2,6) (3,7)
                    const uint32_t g0 = dequant_pair(wgw, negg), g1 = dequant_pair(wgw >> 4, negg);
                    const uint32_t g2 = dequant_pair(wgw >> 8, negg), g3 = dequant_pair(wgw >> 12, negg);
                    const uint32_t h0 = dequant_pair(whw, negh), h1 = dequant_pair(whw >> 4, negh);
                    const uint32_t h2 = dequant_pair(whw >> 8, negh), h3 = dequant_pair(whw >> 12, negh);
#pragma unroll
                    for (int n = 0; n < T; ++n) {
                        const uint4 v = xv[n][j];
                        const uint32_t b0 = prmt(v.x, v.z, 0x5410), b1 = prmt(v.x, v.z, 0x7632);
                        const uint32_t b2 = prmt(v.y, v.w, 0x5410), b3 = prmt(v.y, v.w, 0x7632);
                        float (&a)[4] = j ? acc2[n] : acc[n];
                        mma_bf16_16816(a, g0, h0, g1, h1, b0, b1);
                        mma_bf16_16816(a, g2, h2, g3, h3, b2, b3);
                    }
                }
            }
        }
#pragma unroll
        for (int n = 0; n < T; ++n)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                acc[n][i] += acc2[n][i];
        float *mine = red + kpar * kRows * TOK;   // [2][64][TOK]
#pragma unroll
        for (int n = 0; n < T; ++n) {
            const int col = 8 * n + 2 * cl;
            mine[rg * TOK + col] = acc[n][0];
            mine[rg * TOK + col + 1] = acc[n][1];
            mine[(rg + 8) * TOK + col] = acc[n][2];
            mine[(rg + 8) * TOK + col + 1] = acc[n][3];
        }
        __syncthreads();
#pragma unroll
        for (int i = 0; i < TOK / 4; ++i) {
            const int e = tid + kThreads * i;   // row e / TOK, token e % TOK
            red[e] = red[e] + red[kRows * TOK + e];
        }
    } else {
        // ---- 16 rows of G = [w_g; A^T]: warp w takes the 64-wide sub-tiles i = w (mod 8)
        for (int i = warp; i < nsub && ok; i += 8) {
            ok = wait_bounded(bar_chunk + 8 * (i >> 2), 0);
            const uint8_t *gt = bp + L.codes + i * 2048;
            const uint8_t *xt = bp + L.x + i * (TOK * 128);
            const int ra = gid, rb = gid + 8;
            const uint4 a0 = *reinterpret_cast<const uint4 *>(gt + ra * 128 + (((2 * cl) ^ (ra & 7)) << 4));
            const uint4 a1 = *reinterpret_cast<const uint4 *>(gt + ra * 128 + (((2 * cl + 1) ^ (ra & 7)) << 4));
            const uint4 b0 = *reinterpret_cast<const uint4 *>(gt + rb * 128 + (((2 * cl) ^ (rb & 7)) << 4));
            const uint4 b1 = *reinterpret_cast<const uint4 *>(gt + rb * 128 + (((2 * cl + 1) ^ (rb & 7)) << 4));
            const uint32_t ga[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const uint32_t ha[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int n = 0; n < T; ++n) {
                const int t = 8 * n + gid;
                const uint4 x0 = *reinterpret_cast<const uint4 *>(xt + t * 128 + (((2 * cl) ^ (t & 7)) << 4));
                const uint4 x1 = *reinterpret_cast<const uint4 *>(xt + t * 128 + (((2 * cl + 1) ^ (t & 7)) << 4));
                const uint32_t xa[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                // natural pairs: step s covers k = 16 cl + 4s + {0,1} and + {2,3}
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_bf16_16816((s & 1) ? acc2[n] : acc[n], ga[2 * s], ha[2 * s], ga[2 * s + 1], ha[2 * s + 1],
                                   xa[2 * s], xa[2 * s + 1]);
            }
        }
#pragma unroll
        for (int n = 0; n < T; ++n)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                acc[n][i] += acc2[n][i];
        float *mine = red + warp * 16 * TOK;  // [8 warps][16][TOK]
#pragma unroll
        for (int n = 0; n < T; ++n) {
            const int col = 8 * n + 2 * cl;
            mine[gid * TOK + col] = acc[n][0];
            mine[gid * TOK + col + 1] = acc[n][1];
            mine[(gid + 8) * TOK + col] = acc[n][2];
            mine[(gid + 8) * TOK + col + 1] = acc[n][3];
        }
        __syncthreads();
        for (int e = tid; e < 16 * TOK; e += kThreads) {
            float s = red[e];
#pragma unroll
            for (int w = 1; w < 8; ++w)
                s += red[w * 16 * TOK + e];
            red[e] = s;
        }
    }
    if (!ok)
        atomicOr(p.status, kStatusTimeout);
    __syncthreads();
    if (tid == 0) {
        // no copy of this CTA may still be landing when it goes on (bounded;
        // immediate unless a wait above gave up)
        for (int c = 0; c < nch; ++c)
            wait_bounded(bar_chunk + 8 * c, 0);
        wait_bounded(bar_x, 0);
        if (!is_u && rank == 0 && p.rp > 0)
            wait_bounded(bar_bt, 0);
    }

    if (is_u) {
        // ---- publish this CTA's partial of u rows 16*cluster .. +15 (all TOK
        // columns); the 64-row clusters sum the CS partials in rank order
        float *dst = p.ws_u + ((int64_t)rank * p.R1p + 16 * cluster) * kUStride;
        for (int e = tid; e < 16 * TOK; e += kThreads) {
            const int row = e / TOK, t = e - row * TOK;
            dst[row * kUStride + t] = red[e];
        }
        __syncthreads();
        if (tid == 0)
            red_release_gpu_add(&p.flags[0], 1u);
        if (push)
            cluster_wait();   // pairs with the arrive after the barrier set-up
        return;
    }

    // ---- sum the K split over the cluster, in rank order, in the first CTA.
    // With an EC, the last warp of the first CTA meanwhile waits until u is
    // published.
    const bool ec_warp = rank == 0 && p.JB > 0 && warp == kEcWarp;
    const int nsum = p.JB > 0 ? kThreads - 32 : kThreads;
    constexpr int tile4 = kRows * TOK / 4;
    __shared__ int s_good;
    if (push) {
        cluster_wait();   // every receive barrier of the cluster is initialised
        if (rank != 0) {
            const uint32_t dst = map_to_rank(base + L.recv + (rank - 1) * (kRows * TOK * 4), 0);
            const uint32_t rbar = map_to_rank(bar_recv, 0);
            for (int e4 = tid; e4 < tile4; e4 += kThreads)
                st_async_f4(dst + 16 * e4, reinterpret_cast<const float4 *>(red)[e4], rbar);
            cluster_arrive();
            cluster_wait();   // the first CTA has received every tile
            return;
        }
        if (ec_warp) {
            if (lane == 0)
                s_good = wait_u_published(p, (unsigned)(p.JB * CS)) ? 1 : 0;
        } else if (CS > 1 && !wait_bounded(bar_recv, 0) && tid == 0) {
            atomicOr(p.status, kStatusTimeout);
        }
        cluster_arrive();     // the tiles have landed: the other CTAs may leave
        const float4 *slots = reinterpret_cast<const float4 *>(bp + L.recv);
        if (!ec_warp)
            for (int e4 = tid; e4 < tile4; e4 += nsum) {
                float4 s = reinterpret_cast<const float4 *>(red)[e4];
                for (int q = 0; q < CS - 1; ++q) {
                    const float4 o = slots[q * tile4 + e4];
                    s.x += o.x;
                    s.y += o.y;
                    s.z += o.z;
                    s.w += o.w;
                }
                reinterpret_cast<float4 *>(red)[e4] = s;
            }
    } else {
        __syncthreads();
        cluster_sync();
        if (ec_warp) {
            if (lane == 0)
                s_good = wait_u_published(p, (unsigned)(p.JB * CS)) ? 1 : 0;
        } else if (rank == 0) {
            const uint32_t red_addr = base + L.red;
            for (int e4 = tid; e4 < tile4; e4 += nsum) {
                // issue every remote load before summing (in rank order)
                float4 o[8];
#pragma unroll
                for (int q = 1; q < 8; ++q)
                    if (q < CS)
                        o[q] = ld_dsmem_f4(map_to_rank(red_addr + 16 * e4, (uint32_t)q));
                float4 s = reinterpret_cast<const float4 *>(red)[e4];
#pragma unroll
                for (int q = 1; q < 8; ++q)
                    if (q < CS) {
                        s.x += o[q].x;
                        s.y += o[q].y;
                        s.z += o[q].z;
                        s.w += o[q].w;
                    }
                reinterpret_cast<float4 *>(red)[e4] = s;
            }
        }
        cluster_sync();  // the other CTAs' shared memory is no longer read
        if (rank != 0)
            return;
    }
    __syncthreads();

    // ---- EC: u = sum over the CS published partials (rank order), as u0 [TOK]
    // (gate logits) and uT [TOK][rp] (u[1 + j][t] transposed, zero for j >= r)
    float *u0 = reinterpret_cast<float *>(bp + L.u);
    float *uT = u0 + TOK;
    if (p.JB > 0) {
        const bool good = s_good != 0;
        for (int e = tid; e < (1 + p.r) * TOK; e += kThreads) {
            const int row = e / TOK, t = e - row * TOK;
            float v[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
                v[q] = (q < CS && good) ? __ldcg(p.ws_u + ((int64_t)q * p.R1p + row) * kUStride + t) : 0.f;
            float u = v[0];
#pragma unroll
            for (int q = 1; q < 8; ++q)
                if (q < CS)
                    u += v[q];
            if (row == 0)
                u0[t] = u;
            else
                uT[t * p.rp + row - 1] = u;
        }
        for (int e = tid; e < TOK * (p.rp - p.r); e += kThreads) {
            const int t = e / (p.rp - p.r), j = p.r + e - t * (p.rp - p.r);
            uT[t * p.rp + j] = 0.f;
        }
        __syncthreads();
        if (tid == 0 && atomicAdd(&p.flags[1], 1u) == (unsigned)(p.NC - 1)) {
            // every 64-row cluster has read u: reset for the next forward
            p.flags[1] = 0u;
            p.flags[0] = 0u;
        }
    }

    // ---- epilogue of a 64-row cluster
    if (p.JB > 0 && !wait_bounded(bar_bt, 0))
        atomicOr(p.status, kStatusTimeout);
    const int row = tid & (kRows - 1), th = tid >> 6;  // four token phases
    const int64_t n = n0 + row;
    float out[TOK / 4];
#pragma unroll
    for (int i = 0; i < TOK / 4; ++i)
        out[i] = s_epi * red[row * TOK + th + 4 * i];
    if (p.JB > 0) {
        // corr = g_t * sum_j u[1 + j][t] * B^T[n][j]: the B^T row in 16-byte pieces,
        // u broadcast, both from shared memory
        float corr[TOK / 4];
#pragma unroll
        for (int i = 0; i < TOK / 4; ++i)
            corr[i] = 0.f;
        const uint16_t *btrow = reinterpret_cast<const uint16_t *>(bp + L.bt) + row * p.rp;
        for (int j0 = 0; j0 < p.rp; j0 += 8) {
            const uint4 bv = *reinterpret_cast<const uint4 *>(btrow + j0);
            const float bj[8] = {bf16_lo(bv.x), bf16_hi(bv.x), bf16_lo(bv.y), bf16_hi(bv.y),
                                 bf16_lo(bv.z), bf16_hi(bv.z), bf16_lo(bv.w), bf16_hi(bv.w)};
#pragma unroll
            for (int i = 0; i < TOK / 4; ++i) {
                const float4 *ut = reinterpret_cast<const float4 *>(uT + (th + 4 * i) * p.rp + j0);
                const float4 v0 = ut[0], v1 = ut[1];
                corr[i] += v0.x * bj[0] + v0.y * bj[1] + v0.z * bj[2] + v0.w * bj[3] + v1.x * bj[4] +
                           v1.y * bj[5] + v1.z * bj[6] + v1.w * bj[7];
            }
        }
#pragma unroll
        for (int i = 0; i < TOK / 4; ++i) {
            const float g = 1.0f / (1.0f + expf(-(u0[th + 4 * i] + p.b_g)));
            out[i] += g * corr[i];
        }
    }
#pragma unroll
    for (int i = 0; i < TOK / 4; ++i) {
        const int t = th + 4 * i;
        if (t < p.M && n < p.N)
            p.y[(int64_t)t * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(out[i]));
    }
    if (push)
        cluster_wait();
}

// Cluster size CS (CTAs splitting K) and the k per CTA, or 0 if a slice would
// not fit in shared memory.  Preferably the grid takes about two CTAs per SM,
// so that the next layer's kernel (launched early) finds room to start its
// weight copies while this one runs; layers too large for that take up to 8
// CTAs per SM.  No rank is left without a chunk.
int pick_cluster(const Packed &pk, int num_sms, int JB, int *KS_out)
{
    const int NC = (int)(pk.Np / kRows);
    const int chunks = (int)(pk.Kp / kChunk);
    for (int limit : {2, 8}) {
        for (int CS = std::min(8, chunks); CS >= 1; --CS) {
            const int per = (chunks + CS - 1) / CS;
            if (per > kMaxChunks || (CS - 1) * per >= chunks)
                continue;
            if ((int64_t)(NC + JB) * CS <= (int64_t)limit * num_sms) {
                *KS_out = per * kChunk;
                return CS;
            }
        }
    }
    // otherwise the fewest chunks per CTA that fit
    for (int CS = std::min(8, chunks); CS >= 1; --CS) {
        const int per = (chunks + CS - 1) / CS;
        if (per <= kMaxChunks && (CS == 1 || (CS - 1) * per < chunks)) {
            *KS_out = per * kChunk;
            return CS;
        }
    }
    return 0;
}

template <int T>
const void *kernel_ptr()
{
    return reinterpret_cast<const void *>(decode_w4ec_kernel<T>);
}

}  // namespace

bool decode_supported(const Packed &pk, int num_sms)
{
    if (pk.rp > 128)
        return false;
    int KS = 0;
    const int CS = pick_cluster(pk, num_sms, pk.r > 0 ? pk.R1p / 16 : 0, &KS);
    if (CS == 0)
        return false;
    return smem_layout<32>(KS, pk.rp, pk.R1p, 0).total + 1024 <= 227 * 1024;
}

cudaError_t decode_prepare(const Packed &pk, DecodeWork &w)
{
    Maps *m = static_cast<Maps *>(w.maps);
    if (!m) {
        m = new (std::nothrow) Maps();
        if (!m)
            return cudaErrorMemoryAllocation;
        w.maps = m;
    }
    // [blocks][64 rows][32 words]: one box = one contiguous 8 KB block of 64 rows x 256 k
    const uint64_t dims[3] = {32, (uint64_t)kRows, (uint64_t)(pk.Np / kRows) * (uint64_t)(pk.Kp / kChunk)};
    const uint64_t strides[2] = {128, 8192};
    const uint32_t box[3] = {32, (uint32_t)kRows, 1};
    cudaError_t e = make_map_nd(&m->codes, pk.codes, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, dims, strides, box,
                                CU_TENSOR_MAP_SWIZZLE_128B);

    if (e == cudaSuccess && pk.r > 0)
        e = make_map(&m->g, pk.G, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)pk.Kp, (uint64_t)pk.R1p, 64, 16,
                     CU_TENSOR_MAP_SWIZZLE_128B);
    if (e == cudaSuccess && pk.r > 0)
        e = make_map(&m->bt, pk.Bt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)pk.rp, (uint64_t)pk.Np,
                     (uint32_t)pk.rp, kRows, CU_TENSOR_MAP_SWIZZLE_NONE);

    if (e == cudaSuccess && pk.r == 0) {
        m->g = m->codes;
        m->bt = m->codes;
    }
    return e;
}

void decode_free(DecodeWork &w)
{
    delete static_cast<Maps *>(w.maps);
    w.maps = nullptr;
}

// one partial of u per rank of an EC cluster (at most 8 ranks)
size_t decode_u_floats(const Packed &pk) { return (size_t)8 * pk.R1p * kUStride; }

cudaError_t launch_decode(const Packed &pk, const void *x, void *y, int64_t M, bool ec, const DecodeWork &w,
                          int *status, cudaStream_t st, int num_sms)
{
    if (M <= 0)
        return cudaSuccess;
    if (M > kDecodeMaxTokens || !w.maps)
        return cudaErrorInvalidValue;
    const Maps *m = static_cast<const Maps *>(w.maps);
    const bool use_ec = ec && pk.r > 0;
    DecodeParams p;
    p.Bt = pk.Bt;
    p.s = pk.s;
    p.z = pk.z;
    p.y = static_cast<uint16_t *>(y);
    p.ws_u = w.ws_u;
    p.flags = w.flags;
    p.status = status;
    p.M = M;
    p.N = pk.N;
    p.JB = use_ec ? pk.R1p / 16 : 0;
    p.NC = (int)(pk.Np / kRows);
    int KS = 0;
    const int CS = pick_cluster(pk, num_sms, p.JB, &KS);
    if (CS == 0)
        return cudaErrorInvalidValue;
    p.Kp = pk.Kp;
    p.KS = KS;
    p.nch = KS / kChunk;
    p.r = pk.r;
    p.rp = use_ec ? pk.rp : 0;
    p.R1p = use_ec ? pk.R1p : 0;
    p.b_g = pk.b_g;
    const int T = M <= 8 ? 1 : (M <= 16 ? 2 : 4);
    CUtensorMap tm_x;
    cudaError_t e = make_map(&tm_x, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)pk.K, (uint64_t)M, 64,
                             (uint32_t)(8 * T), CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess)
        return e;
    // push the partial tiles when the receive slots fit, else pull them over DSMEM
    auto layout = [&](int nslots) {
        return T == 1 ? smem_layout<8>(p.KS, p.rp, p.R1p, nslots)
                      : (T == 2 ? smem_layout<16>(p.KS, p.rp, p.R1p, nslots)
                                : smem_layout<32>(p.KS, p.rp, p.R1p, nslots));
    };
    p.push = layout(CS - 1).total + 1024 <= 227 * 1024 ? 1 : 0;
    const size_t smem = layout(p.push ? CS - 1 : 0).total + 1024;
    const void *fn = T == 1 ? kernel_ptr<1>() : (T == 2 ? kernel_ptr<2>() : kernel_ptr<4>());
    e = raise_smem_limit(fn, smem);
    if (e != cudaSuccess)
        return e;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((p.JB + p.NC) * CS));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = CS;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    switch (T) {
    case 1: return cudaLaunchKernelEx(&cfg, decode_w4ec_kernel<1>, m->codes, m->g, m->bt, tm_x, p, CS);
    case 2: return cudaLaunchKernelEx(&cfg, decode_w4ec_kernel<2>, m->codes, m->g, m->bt, tm_x, p, CS);
    default: return cudaLaunchKernelEx(&cfg, decode_w4ec_kernel<4>, m->codes, m->g, m->bt, tm_x, p, CS);
    }
}

}  // namespace spear
