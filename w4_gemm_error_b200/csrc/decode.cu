// Decode-size W4 GEMM (a few tokens) with the Error Compensator fused in.
//
// SPEAR, "A System for Post-Quantization Error-Adaptive Recovery Enabling
// Efficient Low-Bit LLM Serving", Abstract: the post-EC computation is fused
// into the low-bit GEMM.  For a few tokens the layer is bound by reading the
// int4 codes from HBM, and in a decode pass its critical path is the chain
// "previous layer done -> this layer done", so the kernel is built to stream
// the weights from the start and to keep that chain short:
//
//  * one kernel per forward; a cluster of CS CTAs owns 64 weight rows, each
//    CTA one K/CS slice of them, sized so that the grid is one wave of about
//    two CTAs per SM;
//  * a producer warp streams the slice through a ring of shared-memory
//    stages (one 8 KB block of codes and the matching activations per
//    256 k), with full and empty mbarriers; before waiting for the previous
//    kernel (programmatic dependent launch) it fills every stage's codes (a
//    short slice is then entirely resident), and the consumers sleep in a CTA
//    barrier until the activations are on their way;
//  * eight consumer warps, two per 16-row group splitting the 64-wide
//    sub-blocks of each stage, or, for one token group on a short slice,
//    sixteen (one per 16-row group and sub-block), so the dequantise-MMA
//    chains of one warp hide another's;
//  * weight rows sit on the 16-row side of mma.sync m16n8k16 and tokens on
//    the 8-column side, so a code is read once for up to 32 tokens; the
//    codes are dequantised in registers to exact (q - z) bf16 pairs (two
//    nibbles 16 bits apart per register, set into the mantissa of 128.0 and
//    offset by one bf16 fma); the stored nibble order makes each pair two
//    consecutive k, so the activations enter the MMA as they lie in shared
//    memory (each thread takes 16 consecutive k of its rows, the k order
//    inside the MMA being permuted accordingly);
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
#include <cstdlib>
#include <mutex>
#include <new>
#include <vector>

#include "async_utils.cuh"
#include "kernels.h"
#include "tensor_map.h"

namespace spear {
namespace {

constexpr int kRows = 64;         // weight rows per cluster (four warps x 16)
constexpr int kChunk = 256;       // k per stage (one 8 KB TMA box of 64 rows of codes)
constexpr int kMaxStages = 8;     // ring depth limit
constexpr int kUStride = 32;      // token stride of the published u rows
constexpr int kUFinal = 8;        // slot of ws_u holding the summed u (slots 0..7: partials)
// A CTA has W consumer warps, W = 16 (one per 16-row group and 64-k
// sub-block of a stage) or W = 8 (two sub-blocks each), then one producer warp.
__host__ __device__ constexpr int block_threads(int W) { return 32 * W + 32; }
// shared memory per CTA that keeps two CTAs per SM resident
constexpr int kSmemPerCta = 110 * 1024;

struct Maps {
    CUtensorMap codes;    // tiled codes, one box = one 8 KB block (64 rows x 256 k), 128B swizzle
    CUtensorMap g;        // [R1p][Kp] bf16 seen as [Kp/64][R1p][64]: one box = 4 x (16 rows x 64 k)
    CUtensorMap bt;       // [Np][rp] bf16, boxes of rp x 64
    int g3;               // g is the 3-D view (else 2-D boxes of 64 k x 16 rows)
    void *rows;           // maps of the row-CTA kernel (decode_rows.cu), null if it does not fit
    void *stream;         // maps of the cluster-split kernel (decode_stream.cu), null if it does not fit
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
    int KS, nch;          // k per CTA (a multiple of 256), chunks of 256 k per CTA
    int S;                // ring stages
    int JB, NC;           // EC clusters, 64-row clusters
    int ES;               // EC clusters per 16 rows of G (each a 1/ES share of K): JB = R1p/16 * ES
    int KSe, nche;        // k per EC CTA (a multiple of 256), its chunks of 256 k
    int r, rp, R1p;
    int push;             // partial tiles pushed into receive slots of the first CTA
    int x3, g3;           // activations / G rows as one 3-D box per stage (else four 2-D boxes)
    float b_g;
    const void *pf;       // codes of the next layer, prefetched into L2 (null for none)
    uint64_t pf_bytes;
};

// Bytes of one ring stage: the codes of 64 rows x 256 k (or 16 G rows x
// 256 k as four 2 KB boxes), then the activations as four 64-k sub-tiles of
// TOK rows x 128 bytes.
template <int TOK>
__host__ __device__ constexpr uint32_t stage_bytes()
{
    return 8192 + 4 * TOK * 128;
}

struct Smem {
    uint32_t ring, bt, red, u, recv;   // byte offsets from the 1024-aligned base
    uint32_t total;
};

// S ring stages; W consumer warps; nslots receive slots of one partial tile
// (64 rows x TOK fp32) each.
template <int TOK>
__host__ __device__ inline Smem smem_layout(int S, int rp, int nslots, int W)
{
    Smem m;
    m.ring = 0;
    m.bt = m.ring + S * stage_bytes<TOK>();        // 128*rp bytes: B^T rows of the cluster
    m.red = m.bt + 128 * rp;                       // partial tiles: 64*W*TOK bytes
    m.u = m.red + 64 * W * TOK;                    // u0 [TOK], uT [TOK][rp] (fp32)
    m.recv = (m.u + 4 * TOK * (rp + 1) + 15) & ~15u;
    m.total = m.recv + nslots * 256 * TOK;
    return m;
}

__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity) { return mbar_wait_bounded(bar, parity); }

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

// Register budget: with 16 consumer warps two CTAs per SM; with 8, three
// CTAs per SM up to 16 tokens (the grid is about two per SM, and the next
// layer's kernel starts beside it) and two at 32 tokens.
template <int T, int W>
__global__ void __launch_bounds__(block_threads(W), (W == 16 || T == 4) ? 2 : 3)
decode_w4ec_kernel(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_g,
                   const __grid_constant__ CUtensorMap tm_bt, const __grid_constant__ CUtensorMap tm_x,
                   DecodeParams p, int CS)
{
    constexpr int TOK = 8 * T;
    constexpr int kConsumers = 32 * W;
    constexpr int kThreads = block_threads(W);
    constexpr int kProducerWarp = W;
    constexpr int KPAR = W / 4;      // consumer warps per 16-row group
    constexpr uint32_t kStage = stage_bytes<TOK>();
    constexpr uint32_t kXBytes = 4 * TOK * 128;
    extern __shared__ uint8_t smem_raw[];
    // per stage: codes landed, activations landed, stage free; then B^T, K-split receive
    __shared__ __align__(8) uint64_t bars[3 * kMaxStages + 2];

    pdl_launch_dependents();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gid = lane >> 2, cl = lane & 3;
    const bool producer = warp == kProducerWarp;
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *const bp = smem_raw + (base - raw);
    const bool push = p.push != 0;
    // a cluster of one CTA sums nothing across CTAs and needs no cluster barrier
    // (a barrier.cluster wait costs microseconds even when it has nothing to wait for)
    const bool solo = CS == 1;
    const Smem L = smem_layout<TOK>(p.S, p.rp, push ? CS - 1 : 0, W);
    const uint32_t rank = cluster_ctarank();
    const int cluster = blockIdx.x / CS;
    const bool is_u = cluster < p.JB;
    // an EC CTA takes rows 16 jg .. + 15 of G over slice sl of K (ES x CS slices)
    const int jg = is_u ? cluster / p.ES : 0;
    const int sl = is_u ? (cluster % p.ES) * CS + (int)rank : (int)rank;
    const int k0 = sl * (is_u ? p.KSe : p.KS);
    // the last ranks may hold a shorter (or empty) slice when K/256 is not a multiple of CS
    const int nch = max(0, min(is_u ? p.nche : p.nch, (int)((p.Kp - k0) / kChunk)));
    const int S = p.S;
    const int first = min(S, nch);   // chunks whose stages are filled before the dependency wait
    const uint32_t bar_full_w = smem_addr(&bars[0]);
    const uint32_t bar_full_x = smem_addr(&bars[kMaxStages]);
    const uint32_t bar_empty = smem_addr(&bars[2 * kMaxStages]);
    const uint32_t bar_bt = smem_addr(&bars[3 * kMaxStages]);
    const uint32_t bar_recv = smem_addr(&bars[3 * kMaxStages + 1]);
    const int n0 = is_u ? 0 : (cluster - p.JB) * kRows;

    // loads that do not depend on earlier kernels are issued first: the
    // epilogue scale of this thread's row and the zero points of its MMA rows
    const float s_epi = (!is_u && rank == 0 && !producer) ? __ldg(p.s + n0 + (tid & (kRows - 1))) : 0.f;
    const int rg = 16 * (warp & 3) + gid;  // MMA rows rg and rg + 8 (64-row clusters)
    const uint32_t zg_raw = (is_u || producer) ? 0u : (uint32_t)__ldg(p.z + n0 + rg);
    const uint32_t zh_raw = (is_u || producer) ? 0u : (uint32_t)__ldg(p.z + n0 + rg + 8);

    // producer: chunk c of this CTA's slice goes to stage st = c % S
    auto issue_codes = [&](int c, int st) {
        const uint32_t dst = base + L.ring + st * kStage;
        const uint32_t bar = bar_full_w + 8 * st;
        mbar_expect_tx(bar, 8192);
        if (is_u) {
            if (p.g3)
                tma_load_3d(dst, &tm_g, 0, 16 * jg, (k0 + c * kChunk) / 64, bar);
            else
                for (int i = 0; i < 4; ++i)
                    tma_load_2d(dst + i * 2048, &tm_g, k0 + c * kChunk + i * 64, 16 * jg, bar);
        } else {
            tma_load_3d(dst, &tm_codes, 0, 0, (n0 / kRows) * (int)(p.Kp / kChunk) + (k0 / kChunk) + c, bar);
        }
    };
    auto issue_x = [&](int c, int st) {
        const uint32_t dst = base + L.ring + st * kStage + 8192;
        const uint32_t bar = bar_full_x + 8 * st;
        mbar_expect_tx(bar, kXBytes);
        if (p.x3)
            tma_load_3d(dst, &tm_x, 0, 0, (k0 + c * kChunk) / 64, bar);
        else
            for (int i = 0; i < 4; ++i)
                tma_load_2d(dst + i * (TOK * 128), &tm_x, k0 + c * kChunk + 64 * i, 0, bar);
    };

    if (producer && lane == 0) {
        for (int i = 0; i < kMaxStages; ++i) {
            mbar_init(bar_full_w + 8 * i, 1);
            mbar_init(bar_full_x + 8 * i, 1);
            mbar_init(bar_empty + 8 * i, W);
        }
        mbar_init(bar_bt, 1);
        mbar_init(bar_recv, 1);
        fence_mbarrier_init_cluster();
        if (push && !is_u && rank == 0 && CS > 1)
            mbar_expect_tx(bar_recv, (uint32_t)((CS - 1) * kRows * TOK * 4));
        // the weights do not depend on earlier kernels: fill every stage now
        for (int c = 0; c < first; ++c)
            issue_codes(c, c);
        if (!is_u && rank == 0 && p.rp > 0) {
            mbar_expect_tx(bar_bt, 128 * p.rp);   // B^T rows of the cluster, for the epilogue
            tma_load_2d(base + L.bt, &tm_bt, 0, n0, bar_bt);
        }
    }
    __syncthreads();
    if (push && !solo)
        cluster_arrive_relaxed();   // the receive barrier of the first CTA is initialised
    int issued = 0;                 // producer: chunks whose codes and activations are requested
    if (producer && lane == 0) {
        // the activations are written by the previous kernel in the stream
        pdl_wait();
        for (int c = 0; c < first; ++c)
            issue_x(c, c);
        issued = first;
    }
    // the consumers sleep in this barrier, rather than poll, while the
    // producer waits for the previous kernel (polling would take issue slots
    // from the previous layer's CTAs on the same SM)
    __syncthreads();

    bool ok = true;
    // two accumulator sets (even / odd code word) halve the MMA dependency chains
    float acc[T][4], acc2[T][4];
#pragma unroll
    for (int n = 0; n < T; ++n)
#pragma unroll
        for (int i = 0; i < 4; ++i)
            acc[n][i] = acc2[n][i] = 0.f;

    constexpr bool kOverlap = W == 16;
    constexpr int kSumThreads = kOverlap ? 128 : kConsumers - 32;
    const bool fetcher = kOverlap && rank == 0 && p.JB > 0 && tid >= kSumThreads && tid < kConsumers;
    const int nsum = (p.JB > 0 && kOverlap) ? kSumThreads : kConsumers;   // summing threads: tid < nsum
    constexpr int tile4 = kRows * TOK / 4;
    float *u0 = reinterpret_cast<float *>(bp + L.u);
    float *uT = u0 + TOK;
    const int nparts = CS * p.ES;   // partials of u, one per slice of K (at most 8)
    // u (the final rows, four tokens per load, every load of a round issued
    // before any is used) into u0 and uT
    auto fetch_u = [&](int ft, int nft, bool good) {
        constexpr int kT4 = TOK / 4;
        const int n4 = (1 + p.r) * kT4;
        const float *fin = p.ws_u + (int64_t)kUFinal * p.R1p * kUStride;
        for (int e0 = ft; e0 < n4; e0 += 4 * nft) {
            float4 v[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int e = e0 + i * nft, row = e / kT4, t4 = e - row * kT4;
                v[i] = (e < n4 && good) ? __ldcg(reinterpret_cast<const float4 *>(fin + row * kUStride + 4 * t4))
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int e = e0 + i * nft, row = e / kT4, t4 = e - row * kT4;
                if (e >= n4)
                    continue;
                const float uu[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    if (row == 0)
                        u0[4 * t4 + c] = uu[c];
                    else
                        uT[(4 * t4 + c) * p.rp + row - 1] = uu[c];
                }
            }
        }
        for (int e = ft; e < TOK * (p.rp - p.r); e += nft) {
            const int t = e / (p.rp - p.r), j = p.r + e - t * (p.rp - p.r);
            uT[t * p.rp + j] = 0.f;
        }
    };
    float *red = reinterpret_cast<float *>(bp + L.red);
    if (producer) {
        if (lane == 0) {
            int st = 0;
            uint32_t prev = 0;   // parity of the stage's previous use
            for (int c = S; c < nch; ++c) {
                // stage st is free once every consumer warp has released chunk c - S
                if (!wait_bounded(bar_empty + 8 * st, prev)) {
                    atomicOr(p.status, kStatusTimeout);
                    break;
                }
                issue_codes(c, st);
                issue_x(c, st);
                issued = c + 1;
                if (++st == S) {
                    st = 0;
                    prev ^= 1u;
                }
            }
            // every chunk of this CTA is requested: its share of the next layer's
            // codes goes from HBM into L2 while the consumers finish
            prefetch_l2_share(p.pf, p.pf_bytes);
        }
        __syncwarp();
        if (!kOverlap && !is_u && rank == 0 && p.JB > 0) {
            // with 8 consumer warps: u (summed over its partials) goes into shared
            // memory while the consumers finish their stages
            int good = 1;
            if (lane == 0)
                good = wait_u_published(p, (unsigned)(p.JB / p.ES)) ? 1 : 0;
            good = __shfl_sync(0xffffffffu, good, 0);
            fetch_u(lane, 32, good != 0);
        }
    } else if (!is_u) {
        // ---- 64 weight rows: warp w owns rows 16(w mod 4) .. +15 and the sub-blocks
        // sb = w/4 (mod KPAR) of each stage
        const int kq = warp >> 2;
        const uint32_t nbg = __bfloat16_as_ushort(__float2bfloat16_rn(-(float)(128u + zg_raw)));
        const uint32_t nbh = __bfloat16_as_ushort(__float2bfloat16_rn(-(float)(128u + zh_raw)));
        const uint32_t negg = nbg | (nbg << 16), negh = nbh | (nbh << 16);
        int s = 0;
        uint32_t par = 0;
        for (int c = 0; c < nch && ok; ++c) {
            ok = wait_bounded(bar_full_w + 8 * s, par) && wait_bounded(bar_full_x + 8 * s, par);
            if (!ok)
                break;
            const uint8_t *ctile = bp + L.ring + s * kStage;
#pragma unroll
            for (int i = 0; i < 4 / KPAR; ++i) {
                const int sb = KPAR * i + kq;
                // codes k = 64 sb + 16 cl + {0..15} of rows rg and rg + 8 (8 bytes each)
                const int chunk = ((2 * sb + (cl >> 1)) ^ (rg & 7)) * 16 + (cl & 1) * 8;
                const uint2 wgv = *reinterpret_cast<const uint2 *>(ctile + rg * 128 + chunk);
                const uint2 whv = *reinterpret_cast<const uint2 *>(ctile + (rg + 8) * 128 + chunk);
                const uint8_t *xt = ctile + 8192 + sb * (TOK * 128);
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
                    // codes k = 8j + {0..7}: nibbles (m, m + 4) hold the pair k = 2m, 2m + 1,
                    // the order of the activations in v
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
            }
            // every lane's shared-memory reads of this stage are done: release it
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar_empty + 8 * s);
            if (++s == S) {
                s = 0;
                par ^= 1u;
            }
        }
#pragma unroll
        for (int n = 0; n < T; ++n)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                acc[n][i] += acc2[n][i];
        float *mine = red + kq * kRows * TOK;   // [KPAR][64][TOK]
#pragma unroll
        for (int n = 0; n < T; ++n) {
            const int col = 8 * n + 2 * cl;
            mine[rg * TOK + col] = acc[n][0];
            mine[rg * TOK + col + 1] = acc[n][1];
            mine[(rg + 8) * TOK + col] = acc[n][2];
            mine[(rg + 8) * TOK + col + 1] = acc[n][3];
        }
    } else {
        // ---- 16 rows of G = [w_g; A^T]: sub-tile i (64 k, global index 4c + j) is warp (i mod W)'s
        int s = 0;
        uint32_t par = 0;
        for (int c = 0; c < nch && ok; ++c) {
            ok = wait_bounded(bar_full_w + 8 * s, par) && wait_bounded(bar_full_x + 8 * s, par);
            if (!ok)
                break;
            const uint8_t *stage = bp + L.ring + s * kStage;
            for (int j = 0; j < 4; ++j) {
                if ((4 * c + j) % W != warp)
                    continue;
                const uint8_t *gt = stage + j * 2048;
                const uint8_t *xt = stage + 8192 + j * (TOK * 128);
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
                    for (int q = 0; q < 4; ++q)
                        mma_bf16_16816((q & 1) ? acc2[n] : acc[n], ga[2 * q], ha[2 * q], ga[2 * q + 1],
                                       ha[2 * q + 1], xa[2 * q], xa[2 * q + 1]);
                }
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar_empty + 8 * s);
            if (++s == S) {
                s = 0;
                par ^= 1u;
            }
        }
#pragma unroll
        for (int n = 0; n < T; ++n)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                acc[n][i] += acc2[n][i];
        float *mine = red + warp * 16 * TOK;  // [W][16][TOK]
#pragma unroll
        for (int n = 0; n < T; ++n) {
            const int col = 8 * n + 2 * cl;
            mine[gid * TOK + col] = acc[n][0];
            mine[gid * TOK + col + 1] = acc[n][1];
            mine[(gid + 8) * TOK + col] = acc[n][2];
            mine[(gid + 8) * TOK + col + 1] = acc[n][3];
        }
    }
    __shared__ int s_gave_up;   // some wait of this CTA ran out
    if (tid == 0)
        s_gave_up = 0;
    __syncthreads();
    if (!ok) {
        atomicOr(p.status, kStatusTimeout);
        s_gave_up = 1;
    }
    __syncthreads();
    if (tid < kConsumers) {
        if (!is_u) {
            for (int e = tid; e < kRows * TOK; e += kConsumers) {   // row e / TOK, token e % TOK
                float s = red[e];
#pragma unroll
                for (int q = 1; q < KPAR; ++q)
                    s += red[q * kRows * TOK + e];
                red[e] = s;
            }
        } else {
            for (int e = tid; e < 16 * TOK; e += kConsumers) {
                float s = red[e];
#pragma unroll
                for (int w = 1; w < W; ++w)
                    s += red[w * 16 * TOK + e];
                red[e] = s;
            }
        }
    } else if (lane == 0) {
        // no copy of this CTA may still be landing when it goes on (bounded).
        // Every stage the producer filled was waited for by the consumers
        // unless one of their waits gave up; only then are the stages waited
        // for here (each mbarrier test costs hundreds of cycles: the 2S tests
        // took about 2.5 us per launch).  B^T is waited for only by an
        // epilogue with the EC, so always here.
        if (s_gave_up) {
            for (int c = max(0, issued - S); c < issued; ++c) {
                wait_bounded(bar_full_w + 8 * (c % S), (uint32_t)(c / S) & 1u);
                wait_bounded(bar_full_x + 8 * (c % S), (uint32_t)(c / S) & 1u);
            }
            for (int c = issued; c < first; ++c)   // codes requested, activations never
                wait_bounded(bar_full_w + 8 * c, 0);
        }
        if (!is_u && rank == 0 && p.rp > 0)
            wait_bounded(bar_bt, 0);
    }
    __syncwarp();
    __syncthreads();

    if (is_u) {
        // ---- publish this CTA's partial of u rows 16 jg .. + 15 (all TOK
        // columns); the EC CTA of the group that arrives last sums the ES x CS
        // partials in slice order into the final rows (slot 8 of ws_u) and
        // counts the group published, so that a row cluster reads u once
        float *dst = p.ws_u + ((int64_t)sl * p.R1p + 16 * jg) * kUStride;
        for (int e = tid; e < 16 * TOK; e += kThreads) {
            const int row = e / TOK, t = e - row * TOK;
            dst[row * kUStride + t] = red[e];
        }
        __shared__ int s_last;
        __syncthreads();
        if (tid == 0) {
            __threadfence();
            s_last = atomicAdd(&p.flags[2 + jg], 1u) == (unsigned)(nparts - 1) ? 1 : 0;
        }
        __syncthreads();
        if (s_last) {
            __threadfence();
            for (int e = tid; e < 16 * TOK; e += kThreads) {
                const int row = e / TOK, t = e - row * TOK;
                float v[8];
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    v[q] = q < nparts ? __ldcg(p.ws_u + ((int64_t)q * p.R1p + 16 * jg + row) * kUStride + t) : 0.f;
                float u = v[0];
#pragma unroll
                for (int q = 1; q < 8; ++q)
                    if (q < nparts)
                        u += v[q];
                p.ws_u[((int64_t)kUFinal * p.R1p + 16 * jg + row) * kUStride + t] = u;
            }
            __syncthreads();
            if (tid == 0) {
                p.flags[2 + jg] = 0u;
                red_release_gpu_add(&p.flags[0], 1u);
            }
        }
        if (push && !solo)
            cluster_wait();   // pairs with the arrive after the barrier set-up
        return;
    }

    // ---- sum the K split over the cluster, in rank order, in the first CTA.
    // With an EC, u is published by the EC CTAs as ES x CS partials (one per
    // slice of K), which are summed (slice order) into u0 [TOK] (gate logits)
    // and uT [TOK][rp] (u[1 + j][t] transposed, zero for j >= r): with 16
    // consumer warps, warps 0-3 sum the K split while the other twelve wait
    // for u and fetch it; with 8, the producer warp has fetched it while the
    // consumers ran their last stages (above).
    if (push) {
        if (!solo)
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
        if (!fetcher && CS > 1 && !wait_bounded(bar_recv, 0) && tid == 0)
            atomicOr(p.status, kStatusTimeout);
        if (!solo)
            cluster_arrive();     // the tiles have landed: the other CTAs may leave
        if (fetcher) {
            int good = 1;
            if (lane == 0)
                good = wait_u_published(p, (unsigned)(p.JB / p.ES)) ? 1 : 0;
            good = __shfl_sync(0xffffffffu, good, 0);
            fetch_u(tid - kSumThreads, kConsumers - kSumThreads, good != 0);
        }
        const float4 *slots = reinterpret_cast<const float4 *>(bp + L.recv);
        if (tid < nsum)
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
        if (!solo)
            cluster_sync();
        if (fetcher) {
            int good = 1;
            if (lane == 0)
                good = wait_u_published(p, (unsigned)(p.JB / p.ES)) ? 1 : 0;
            good = __shfl_sync(0xffffffffu, good, 0);
            fetch_u(tid - kSumThreads, kConsumers - kSumThreads, good != 0);
        } else if (rank == 0 && tid < nsum) {
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
        __syncwarp();
        if (!solo)
            cluster_sync();  // the other CTAs' shared memory is no longer read
        if (rank != 0)
            return;
    }
    __syncthreads();

    if (p.JB > 0 && tid == 0 && atomicAdd(&p.flags[1], 1u) == (unsigned)(p.NC - 1)) {
        // every 64-row cluster has read u: reset for the next forward
        p.flags[1] = 0u;
        p.flags[0] = 0u;
    }

    // ---- epilogue of a 64-row cluster: consumer thread = row (tid mod 64) and
    // the tokens th + kPh * i, th = tid / 64
    constexpr int kPh = kConsumers / 64;
    constexpr int kTokPerThread = TOK / kPh;
    if (tid < kConsumers) {
        if (p.JB > 0 && !wait_bounded(bar_bt, 0))
            atomicOr(p.status, kStatusTimeout);
        const int row = tid & (kRows - 1), th = tid >> 6;
        const int64_t n = n0 + row;
        float out[kTokPerThread];
#pragma unroll
        for (int i = 0; i < kTokPerThread; ++i)
            out[i] = s_epi * red[row * TOK + th + kPh * i];
        if (p.JB > 0) {
            // corr = g_t * sum_j u[1 + j][t] * B^T[n][j]: the B^T row in 16-byte pieces,
            // u from shared memory.  With one token per thread the pieces start at
            // a row-dependent offset, spreading the rows over the banks; with
            // several, all lanes take the same piece and u is a broadcast.
            float corr[kTokPerThread];
#pragma unroll
            for (int i = 0; i < kTokPerThread; ++i)
                corr[i] = 0.f;
            const uint16_t *btrow = reinterpret_cast<const uint16_t *>(bp + L.bt) + row * p.rp;
            const int npiece = p.rp / 8;
            int piece = kTokPerThread == 1 ? (row & (npiece - 1)) : 0;   // start in [0, npiece)
            for (int pc = 0; pc < npiece; ++pc) {
                const int j0 = 8 * piece;
                if (++piece == npiece)
                    piece = 0;
                const uint4 bv = *reinterpret_cast<const uint4 *>(btrow + j0);
                const float bj[8] = {bf16_lo(bv.x), bf16_hi(bv.x), bf16_lo(bv.y), bf16_hi(bv.y),
                                     bf16_lo(bv.z), bf16_hi(bv.z), bf16_lo(bv.w), bf16_hi(bv.w)};
#pragma unroll
                for (int i = 0; i < kTokPerThread; ++i) {
                    const float4 *ut = reinterpret_cast<const float4 *>(uT + (th + kPh * i) * p.rp + j0);
                    const float4 v0 = ut[0], v1 = ut[1];
                    corr[i] += v0.x * bj[0] + v0.y * bj[1] + v0.z * bj[2] + v0.w * bj[3] + v1.x * bj[4] +
                               v1.y * bj[5] + v1.z * bj[6] + v1.w * bj[7];
                }
            }
#pragma unroll
            for (int i = 0; i < kTokPerThread; ++i) {
                const float g = 1.0f / (1.0f + expf(-(u0[th + kPh * i] + p.b_g)));
                out[i] += g * corr[i];
            }
        }
#pragma unroll
        for (int i = 0; i < kTokPerThread; ++i) {
            const int t = th + kPh * i;
            if (t < p.M && n < p.N)
                p.y[(int64_t)t * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(out[i]));
        }
    }
    if (push && !solo)
        cluster_wait();
}

// Cluster size CS (CTAs splitting K) and the k per CTA: the largest CS (at
// most 8) whose grid is one wave of two CTAs per SM (so that the next
// layer's kernel, launched early, also finds room), else CS = 1.  No rank is
// left without a chunk.  The slice is streamed, so its length is not bounded.
int pick_cluster(const Packed &pk, int num_sms, int JB, int *KS_out, int max_cs = 8)
{
    const int NC = (int)(pk.Np / kRows);
    const int chunks = (int)(pk.Kp / kChunk);
    for (int CS = std::min(max_cs, chunks); CS >= 1; --CS) {
        const int per = (chunks + CS - 1) / CS;
        if (CS > 1 && (CS - 1) * per >= chunks)
            continue;
        if (CS == 1 || (int64_t)(NC + JB) * CS <= 2LL * num_sms) {
            *KS_out = per * kChunk;
            return CS;
        }
    }
    return 0;
}

// Ring depth: as many stages as fit in the per-CTA budget beside the other
// regions, at most the chunks of the slice, and two when the slice has two
// chunks or more (then the budget may be exceeded).
template <int TOK>
int pick_stages(int nch, int rp, int nslots, int W)
{
    const int fixed = (int)smem_layout<TOK>(0, rp, nslots, W).total + 1024;
    const int fit = (kSmemPerCta - fixed) / (int)stage_bytes<TOK>();
    return std::max(std::min(2, nch), std::min({fit, nch, kMaxStages}));
}

struct Plan {
    int S, push;
    size_t smem;
};

template <int TOK>
Plan plan_for(int nch, int rp, int CS, int W)
{
    Plan pl;
    // push the partial tiles when the receive slots fit, else pull them over DSMEM
    pl.S = pick_stages<TOK>(nch, rp, CS - 1, W);
    pl.smem = smem_layout<TOK>(pl.S, rp, CS - 1, W).total + 1024;
    pl.push = pl.smem <= 227 * 1024 ? 1 : 0;
    if (!pl.push) {
        pl.S = pick_stages<TOK>(nch, rp, 0, W);
        pl.smem = smem_layout<TOK>(pl.S, rp, 0, W).total + 1024;
    }
    return pl;
}

// Consumer warps: 16 for one token group on a short slice (at most four
// chunks, where hiding latency matters most), else 8, whose per-chunk
// overhead is shared by two sub-blocks.
int pick_warps(int T, int nch) { return (T == 1 && nch <= 4) ? 16 : 8; }

template <int T, int W>
const void *kernel_ptr()
{
    return reinterpret_cast<const void *>(decode_w4ec_kernel<T, W>);
}

}  // namespace

// The cluster-split decode kernel (decode_stream.cu) serves up to 16 tokens
// when SPEAR_DECODE_STREAM=1; otherwise the row-CTA and split-K kernels do.
bool decode_stream_enabled()
{
    const char *v = std::getenv("SPEAR_DECODE_STREAM");
    return v && v[0] == '1';
}

bool grid_is_one_wave(const void *fn, int threads, size_t smem, int cs, int64_t blocks, int num_sms)
{
    struct Entry {
        const void *fn;
        int threads, cs, dev;
        size_t smem;
        int64_t capacity;
    };
    static std::vector<Entry> cache;
    static std::mutex mu;
    int dev = 0;
    cudaGetDevice(&dev);
    {
        std::lock_guard<std::mutex> lock(mu);
        for (const Entry &e : cache)
            if (e.fn == fn && e.threads == threads && e.cs == cs && e.smem == smem && e.dev == dev)
                return blocks <= e.capacity;
    }
    int64_t capacity = 0;
    if (raise_smem_limit(fn, smem) == cudaSuccess) {
        int n = 0;
        if (cs > 1) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3((unsigned)cs);
            cfg.blockDim = dim3((unsigned)threads);
            cfg.dynamicSmemBytes = smem;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = cs;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) == cudaSuccess)
                capacity = (int64_t)n * cs;
        } else if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, threads, smem) == cudaSuccess) {
            capacity = (int64_t)n * num_sms;
        }
    }
    cudaGetLastError();   // a refused query leaves no sticky error
    std::lock_guard<std::mutex> lock(mu);
    cache.push_back({fn, threads, cs, dev, smem, capacity});
    return blocks <= capacity;
}

bool decode_supported(const Packed &pk, int num_sms)
{
    if (pk.rp > 128)
        return false;
    const int JB = pk.r > 0 ? pk.R1p / 16 : 0;
    int KS = 0;
    const int CS = pick_cluster(pk, num_sms, JB, &KS);
    if (CS == 0)
        return false;
    return plan_for<32>(KS / kChunk, pk.rp, CS, 8).smem <= 227 * 1024;
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

    m->g3 = 0;
    if (e == cudaSuccess && pk.r > 0) {
        // one stage of G rows (16 rows x 256 k) as one box: [k block][row][64 k], laid
        // out in shared memory as four 2 KB sub-tiles; the 2-D boxes if the driver
        // does not take this view
        const uint64_t gd[3] = {64, (uint64_t)pk.R1p, (uint64_t)(pk.Kp / 64)};
        const uint64_t gs[2] = {(uint64_t)pk.Kp * 2, 128};
        const uint32_t gb[3] = {64, 16, 4};
        if (make_map_nd(&m->g, pk.G, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, gd, gs, gb, CU_TENSOR_MAP_SWIZZLE_128B) ==
            cudaSuccess)
            m->g3 = 1;
        else
            e = make_map(&m->g, pk.G, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)pk.Kp, (uint64_t)pk.R1p, 64, 16,
                         CU_TENSOR_MAP_SWIZZLE_128B);
    }
    if (e == cudaSuccess && pk.r > 0)
        e = make_map(&m->bt, pk.Bt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)pk.rp, (uint64_t)pk.Np,
                     (uint32_t)pk.rp, kRows, CU_TENSOR_MAP_SWIZZLE_NONE);

    if (e == cudaSuccess && pk.r == 0) {
        m->g = m->codes;
        m->bt = m->codes;
    }
    if (e == cudaSuccess && decode_rows_shape(pk))
        e = decode_rows_prepare(pk, &m->rows);
    if (e == cudaSuccess && decode_stream_shape(pk))
        e = decode_stream_prepare(pk, &m->stream);
    return e;
}

void decode_free(DecodeWork &w)
{
    if (w.maps) {
        decode_rows_free(static_cast<Maps *>(w.maps)->rows);
        decode_stream_free(static_cast<Maps *>(w.maps)->stream);
    }
    delete static_cast<Maps *>(w.maps);
    w.maps = nullptr;
}

// one partial of u per rank of an EC cluster (at most 8 ranks)
size_t decode_u_floats(const Packed &pk) { return (size_t)(kUFinal + 1) * pk.R1p * kUStride; }

cudaError_t launch_decode(const Packed &pk, const void *x, void *y, int64_t M, bool ec, const DecodeWork &w,
                          int *status, cudaStream_t st, int num_sms)
{
    if (M <= 0)
        return cudaSuccess;
    if (M > kDecodeMaxTokens || !w.maps)
        return cudaErrorInvalidValue;
    const Maps *m = static_cast<const Maps *>(w.maps);
    // up to 16 tokens: K split over a cluster, each CTA with its slice of x
    if (m->stream && decode_stream_enabled() && decode_stream_fits(pk, M, num_sms))
        return launch_decode_stream(pk, m->stream, x, y, M, ec, w, status, st, num_sms);
    // up to 16 tokens on a layer whose 16-row slices fit in shared memory: one
    // CTA per 16 rows over the whole of K, no exchange between CTAs
    if (m->rows && decode_rows_fits(pk, M, num_sms))
        return launch_decode_rows(pk, m->rows, x, y, M, ec, w, status, st, num_sms);
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
    const int JG = use_ec ? pk.R1p / 16 : 0;   // 16-row groups of G
    p.JB = JG;
    p.ES = 1;
    p.NC = (int)(pk.Np / kRows);
    p.Kp = pk.Kp;
    p.r = pk.r;
    p.rp = use_ec ? pk.rp : 0;
    p.R1p = use_ec ? pk.R1p : 0;
    p.b_g = pk.b_g;
    p.pf = w.pf;
    p.pf_bytes = w.pf_bytes;
    const int T = M <= 8 ? 1 : (M <= 16 ? 2 : 4);
    // the activations of one stage (TOK rows x 256 k) as one box of the view
    // [k block][token][64 k] when K is a multiple of 64 (then no box reads past
    // the end of a row), else as four 2-D boxes with k >= K filled with zeros
    CUtensorMap tm_x;
    cudaError_t e = cudaErrorInvalidValue;
    p.x3 = 0;
    if (pk.K % 64 == 0) {
        const uint64_t xd[3] = {64, (uint64_t)M, (uint64_t)(pk.K / 64)};
        const uint64_t xs[2] = {(uint64_t)pk.K * 2, 128};
        const uint32_t xb[3] = {64, (uint32_t)(8 * T), 4};
        e = make_map_nd(&tm_x, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, xd, xs, xb, CU_TENSOR_MAP_SWIZZLE_128B);
        p.x3 = e == cudaSuccess ? 1 : 0;
    }
    if (e != cudaSuccess)
        e = make_map(&tm_x, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)pk.K, (uint64_t)M, 64,
                     (uint32_t)(8 * T), CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess)
        return e;
    p.g3 = m->g3;
    // the largest cluster whose grid is one wave when the EC is on (the row
    // clusters then wait, bounded, for the EC clusters' partials of u)
    int CS = 0, W = 0;
    Plan pl{};
    const void *fn = nullptr;
    for (int max_cs = 8; max_cs >= 1;) {
        int KS = 0;
        CS = pick_cluster(pk, num_sms, JG, &KS, max_cs);
        if (CS == 0)
            return cudaErrorInvalidValue;
        p.KS = KS;
        p.nch = KS / kChunk;
        // The EC CTAs stream G (bf16, four times the bytes of a row of codes)
        // and publish u only when their slice is done, so that the rows wait
        // for it.  Without a K split (CS = 1) they take 1/ES of K each, ES the
        // largest (at most 8 partials, no empty slice) that keeps the grid
        // within two CTAs per SM, so that u is ready before the rows' products
        // are (MLP up at one token: 15.7 -> 14.9 us per layer with the EC);
        // with a K split the rows' slices are short already (splitting the EC
        // CTAs further was measured slower there).
        const int chunks = (int)(pk.Kp / kChunk);
        int ES = 1;
        for (int es = 8 / CS; es > 1 && JG > 0 && CS == 1; --es) {
            const int per = (chunks + es * CS - 1) / (es * CS);
            if ((es * CS - 1) * per < chunks && (int64_t)(JG * es + p.NC) * CS <= 2LL * num_sms) {
                ES = es;
                break;
            }
        }
        p.ES = ES;
        p.JB = JG * ES;
        p.nche = (chunks + ES * CS - 1) / (ES * CS);
        p.KSe = p.nche * kChunk;
        W = pick_warps(T, p.nch);
        pl = T == 1 ? plan_for<8>(p.nch, p.rp, CS, W)
                    : (T == 2 ? plan_for<16>(p.nch, p.rp, CS, W) : plan_for<32>(p.nch, p.rp, CS, W));
        if (pl.smem > 227 * 1024)
            return cudaErrorInvalidValue;
        fn = T == 1 ? (W == 16 ? kernel_ptr<1, 16>() : kernel_ptr<1, 8>())
                    : (T == 2 ? kernel_ptr<2, 8>() : kernel_ptr<4, 8>());
        e = raise_smem_limit(fn, pl.smem);
        if (e != cudaSuccess)
            return e;
        if (!use_ec || grid_is_one_wave(fn, block_threads(W), pl.smem, CS, (int64_t)(p.JB + p.NC) * CS, num_sms))
            break;
        if (CS == 1)
            return cudaErrorInvalidConfiguration;
        max_cs = CS - 1;
    }
    p.S = pl.S;
    p.push = pl.push;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((p.JB + p.NC) * CS));
    cfg.blockDim = dim3((unsigned)block_threads(W));
    cfg.dynamicSmemBytes = pl.smem;
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
    case 1:
        if (W == 16)
            return cudaLaunchKernelEx(&cfg, decode_w4ec_kernel<1, 16>, m->codes, m->g, m->bt, tm_x, p, CS);
        return cudaLaunchKernelEx(&cfg, decode_w4ec_kernel<1, 8>, m->codes, m->g, m->bt, tm_x, p, CS);
    case 2: return cudaLaunchKernelEx(&cfg, decode_w4ec_kernel<2, 8>, m->codes, m->g, m->bt, tm_x, p, CS);
    default: return cudaLaunchKernelEx(&cfg, decode_w4ec_kernel<4, 8>, m->codes, m->g, m->bt, tm_x, p, CS);
    }
}

}  // namespace spear
