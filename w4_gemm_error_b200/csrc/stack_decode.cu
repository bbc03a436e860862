// Persistent decode kernel over a whole layer stack: one launch runs every op
// of a spear_w4ec_stack for up to 16 tokens.
//
// SPEAR, "A System for Post-Quantization Error-Adaptive Recovery Enabling
// Efficient Low-Bit LLM Serving", Abstract: the post-EC computation is fused
// into the low-bit GEMM, and ECs sit only at the error-sensitive layers.  At
// decode sizes a layer moves a few MB of int4 codes, about a microsecond of
// HBM time on B200, while a kernel launch that waits for its predecessor
// costs about as much again.  So a stack runs here as one grid of one CTA per
// SM that stays resident for all of its ops:
//
//  * every op's work is cut into items, 16-row tiles of the W4 product (all of
//    K) and, where an op needs it, units of its EC down-projection (16 rows of
//    G = [w_g; A^T] over 256 k); items are dealt round robin over the CTAs,
//    continuing from op to op, so that every CTA streams the same share of
//    the stack's bytes;
//  * a producer warp streams the CTA's items, op after op, through a ring of
//    8 KB shared-memory stages (TMA boxes of 16 code rows x 1024 k, or 16 G
//    rows x 256 k) plus a small ring of per-tile operands (s, z, the tile's
//    B^T rows and, see below, a slice of the next op's G).  Weights do not
//    depend on activations, so it never waits for an earlier op: the next
//    ops' codes are already landing while the current one computes;
//  * sixteen consumer warps run the product as the other decode kernels do
//    (codes dequantised in registers to exact (q - z) bf16 pairs, mma.sync
//    m16n8k16 with the weight rows on the 16-row side and the tokens on the
//    8-column side); warp w takes the 64-k sub-block w of every 1024-k stage
//    and the warps' partial tiles are summed in shared memory in warp order;
//  * an op whose input another op writes waits, before it reads that input
//    or writes its output, until every CTA has counted the conflicting op
//    done (a release increment per CTA, an acquire poll by one thread);
//  * the EC down-projection u = x.[w_g, A] of an op whose input is the output
//    of the op just before it is formed in that op's epilogue: a CTA that
//    has produced y rows n0 .. n0 + 15 of op l adds, for every row j of the
//    next op's G, sum_{i<16} G_{l+1}[j][n0 + i] y[t][n0 + i] into u of op
//    l + 1 (fp32 atomic adds, summed over the CTA's tiles first), so that u
//    is complete when op l is, and op l + 1 reads it together with its x.
//    Any other op with an EC computes u from its input with its G units and
//    counts them done; its epilogue waits (bounded) for that count;
//  * the epilogue thread (row, token) forms
//        y[t,n] = bf16( s[n] acc[t,n] + g_t sum_j u[t,1+j] B[j,n] ),
//        g_t = 1 / (1 + exp(-(u[t,0] + b_g))).
//
// Every wait is bounded (about a second, then a timeout bit in the status
// word of the op's layer and an early, orderly exit of the CTA).  The sums
// of u use fp32 atomic adds, so their order (and the last bits of u) may
// differ from run to run; everything else is summed in a fixed order.
#include <algorithm>
#include <new>
#include <vector>

#include "async_utils.cuh"
#include "kernels.h"
#include "tensor_map.h"

namespace spear {
namespace {

constexpr int kW = 16;                     // consumer warps
constexpr int kConsumers = 32 * kW;
constexpr int kThreads = kConsumers + 32;  // + the producer warp
constexpr int kUnitBytes = 8192;           // one ring stage
constexpr int kStages = 16;
constexpr int kMetaSlots = 8;
constexpr int kMetaBtOff = 128;                                 // s [16] fp32, z [16] u8, then B^T rows
constexpr int kMetaGnOff = kMetaBtOff + 16 * kStackMaxRp * 2;   // then the next op's G slice [R1p][16]
constexpr int kMetaBytes = kMetaGnOff + kStackMaxR1p * 32;
constexpr int kUStride = 16;               // token stride of the u accumulators [R1p][16]

// Tiles in flight per CTA and 1024-k stages of activations held in registers
// (requested ahead), by token groups: both bounded by the registers of 17
// warps per SM.
__host__ __device__ constexpr int tiles_per_group(int) { return 2; }
__host__ __device__ constexpr int x_ahead(int T) { return T == 1 ? 4 : 2; }

struct Layout {
    uint32_t meta, red, us, ybf, total;
};

template <int T>
__host__ __device__ constexpr Layout stack_layout()
{
    Layout L{};
    L.meta = kStages * kUnitBytes;
    L.red = L.meta + kMetaSlots * kMetaBytes;
    L.us = L.red + tiles_per_group(T) * kW * 8 * T * 16 * 4;
    L.ybf = L.us + 8 * T * kStackMaxR1p * 4;
    L.total = L.ybf + tiles_per_group(T) * 8 * T * 16 * 2;
    return L;
}

struct StackParams {
    const StackOpDev *ops;
    const CUtensorMap *maps;   // [n_ops][2]: codes (box 32 x 16 x 4), G (box 64 x 16 x 4)
    const uint16_t *x;         // the call's input (buffer 0)
    uint16_t *y;               // the call's output (buffer 1)
    unsigned *done;            // [n_ops] CTAs done with the op, then [n_ops] EC units done
    float *uacc;               // u accumulators, zero at launch
    int n_ops;
    int M;
    int ec_on;                 // 0: every EC off for this call
    int fault;                 // fault injection: the first op waits for a count nothing reaches
};

__device__ __forceinline__ void bar_consumers() { asm volatile("bar.sync 1, %0;" ::"n"(kConsumers) : "memory"); }

__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

// Bounded acquire poll (one thread) until *ctr reaches target.
__device__ __forceinline__ bool poll_count(const unsigned *ctr, unsigned target, volatile int *abort_flag,
                                           int *status)
{
    const long long t0 = clock64();
    while ((int)(ld_acquire_gpu(ctr) - target) < 0) {
        if (*abort_flag)
            return false;
        if (clock64() - t0 > kWaitBudgetCycles) {
            *abort_flag = 1;
            atomicOr(status, kStatusTimeout);
            return false;
        }
        __nanosleep(32);
    }
    return true;
}

// First item of CTA c in an op whose deal starts at CTA `base`.
__device__ __forceinline__ int first_item(int c, int base, int G) { return (c - base + G) % G; }

__device__ __forceinline__ void zero_x(uint4 &a, uint4 &b)
{
    a = make_uint4(0, 0, 0, 0);
    b = a;
}

template <int T>
__global__ void __launch_bounds__(kThreads, 1) stack_decode_kernel(StackParams p)
{
    constexpr int TOK = 8 * T;
    constexpr int TG = tiles_per_group(T);
    constexpr int XD = x_ahead(T);
    constexpr Layout L = stack_layout<T>();
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full[kStages], empty[kStages], mfull[kMetaSlots], mempty[kMetaSlots];
    __shared__ int abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gid = lane >> 2, cl = lane & 3;
    const int G = gridDim.x, c = blockIdx.x;
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *const bp = smem_raw + (base - raw);
    float *const red = reinterpret_cast<float *>(bp + L.red);
    float *const us = reinterpret_cast<float *>(bp + L.us);
    uint16_t *const ybf = reinterpret_cast<uint16_t *>(bp + L.ybf);
    volatile int *const abrt = &abort_flag;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_addr(&full[s]), 1);
            mbar_init(smem_addr(&empty[s]), kW);
        }
        for (int s = 0; s < kMetaSlots; ++s) {
            mbar_init(smem_addr(&mfull[s]), 1);
            mbar_init(smem_addr(&mempty[s]), 1);
        }
        abort_flag = 0;
        fence_mbarrier_init_cluster();
    }
    __syncthreads();

    if (warp == kW) {
        // ---------------- producer: the CTA's items, op after op, in the order
        // the consumers take them (EC units, then groups of TG tiles: their
        // operands, then stage u of every tile of the group, u = 0, 1, ...)
        uint32_t rseq = 0, mseq = 0;
        for (int l = 0; l < p.n_ops && !*abrt; ++l) {
            const StackOpDev &op = p.ops[l];
            const int n_g = op.n_g, n_items = n_g + op.n_tiles, nch = op.nch, nu = (nch + 3) / 4;
            const CUtensorMap *mc = p.maps + 2 * l, *mg = p.maps + 2 * l + 1;
            const bool ec = p.ec_on && op.ec;
            const bool fuse = p.ec_on && op.fuse_next;
            int i = first_item(c, op.base, G);
            for (; i < n_g && i < n_items && !*abrt; i += G) {
                if (!p.ec_on)
                    continue;
                const int JB = op.R1p / 16, jg = i % JB, ck = i / JB;
                const int s = rseq % kStages;
                if (!mbar_wait(smem_addr(&empty[s]), ((rseq / kStages) & 1) ^ 1, abrt, op.status))
                    break;
                if (lane == 0) {
                    mbar_expect_tx(smem_addr(&full[s]), kUnitBytes);
                    tma_load_3d(base + s * kUnitBytes, mg, 0, 16 * jg, 4 * ck, smem_addr(&full[s]));
                }
                ++rseq;
            }
            while (i < n_items && !*abrt) {
                int n0s[TG];
                int ng = 0;
                for (; ng < TG && i < n_items; ++ng, i += G)
                    n0s[ng] = 16 * (i - n_g);
                for (int tg = 0; tg < ng && !*abrt; ++tg) {
                    // per-tile operands
                    const int n0 = n0s[tg], ms = mseq % kMetaSlots;
                    if (!mbar_wait(smem_addr(&mempty[ms]), ((mseq / kMetaSlots) & 1) ^ 1, abrt, op.status))
                        break;
                    const uint32_t mb = base + L.meta + ms * kMetaBytes, mbar = smem_addr(&mfull[ms]);
                    const uint32_t bt_bytes = ec ? 32u * op.rp : 0u;
                    const uint32_t gn_bytes = fuse ? 32u * op.R1p_next : 0u;
                    if (lane == 0) {
                        mbar_expect_tx(mbar, 64u + 16u + bt_bytes + gn_bytes);
                        bulk_load(mb, op.s + n0, 64u, mbar);
                        bulk_load(mb + 64, op.z + n0, 16u, mbar);
                        if (bt_bytes)
                            bulk_load(mb + kMetaBtOff, op.Bt + (int64_t)n0 * op.rp, bt_bytes, mbar);
                    }
                    __syncwarp();
                    if (gn_bytes)
                        for (int j = lane; j < op.R1p_next; j += 32)
                            bulk_load(mb + kMetaGnOff + 32 * j, op.Gnext + (int64_t)j * op.Kp_next + n0, 32u, mbar);
                    ++mseq;
                }
                // codes: stage u (1024 k) of each tile of the group
                for (int u = 0; u < nu && !*abrt; ++u)
                    for (int tg = 0; tg < ng; ++tg) {
                        const int n0 = n0s[tg], s = rseq % kStages;
                        if (!mbar_wait(smem_addr(&empty[s]), ((rseq / kStages) & 1) ^ 1, abrt, op.status))
                            break;
                        if (lane == 0) {
                            mbar_expect_tx(smem_addr(&full[s]), kUnitBytes);
                            tma_load_3d(base + s * kUnitBytes, mc, 0, n0 % 64, (n0 / 64) * nch + 4 * u,
                                        smem_addr(&full[s]));
                        }
                        ++rseq;
                    }
            }
        }
        // no copy may still be landing when the CTA leaves: the consumers waited
        // for every stage and operand slot issued unless a wait gave up; then the
        // last phase issued on each is waited for here
        if (lane == 0 && *abrt) {
            for (uint32_t q = rseq > (uint32_t)kStages ? rseq - kStages : 0; q < rseq; ++q)
                mbar_wait_final(smem_addr(&full[q % kStages]), (q / kStages) & 1);
            for (uint32_t q = mseq > (uint32_t)kMetaSlots ? mseq - kMetaSlots : 0; q < mseq; ++q)
                mbar_wait_final(smem_addr(&mfull[q % kMetaSlots]), (q / kMetaSlots) & 1);
        }
        __syncwarp();
    } else {
        // ---------------- consumers
        uint32_t rseq = 0, mseq = 0;
        for (int l = 0; l < p.n_ops; ++l) {
            const StackOpDev &op = p.ops[l];
            const int n_g = op.n_g, n_items = n_g + op.n_tiles, nch = op.nch, nsb = 4 * nch, nu = (nch + 3) / 4;
            const int K = op.K, N = op.N, M = p.M;
            const bool ec = p.ec_on && op.ec;
            const bool fuse = p.ec_on && op.fuse_next;
            const uint16_t *x = op.xbuf ? op.xbuf : p.x;
            uint16_t *y = op.ybuf ? op.ybuf : p.y;
            float *const uacc = p.uacc + op.u_off;

            // 1. wait until the op that this one conflicts with is done everywhere
            if (l == 0 && p.fault) {
                if (tid == 0)
                    poll_count(p.done, (unsigned)G + 1u, abrt, op.status);   // never reached: runs out
                bar_consumers();
            }
            if (op.wait_op >= 0) {
                if (tid == 0 && poll_count(p.done + op.wait_op, (unsigned)G, abrt, op.status))
                    __threadfence();
                bar_consumers();
            }
            // 2. u of this op: (j, t) = (e / TOK, e % TOK), e = tid + 512 q; rows
            // past R1p (up to rp, read by the epilogue) are zero
            const int u_rows = op.R1p > op.rp + 1 ? op.R1p : op.rp + 1;
            float uv[3] = {0.f, 0.f, 0.f};
            auto fetch_u = [&]() {
#pragma unroll
                for (int q = 0; q < 3; ++q) {
                    const int e = tid + kConsumers * q, j = e / TOK, t = e - j * TOK;
                    uv[q] = (t < M && j < op.R1p) ? __ldcg(uacc + j * kUStride + t) : 0.f;
                }
            };
            auto store_u = [&]() {
#pragma unroll
                for (int q = 0; q < 3; ++q) {
                    const int e = tid + kConsumers * q, j = e / TOK, t = e - j * TOK;
                    if (j < u_rows)
                        us[t * kStackMaxR1p + j] = uv[q];
                }
            };
            bool u_in_regs = false, u_ready = !ec;
            if (ec && op.u_mode == 2) {
                fetch_u();   // complete: formed by the previous op, which this one waited for
                u_in_regs = true;
            }

            // activations of the 64-k sub-block of stage u that this warp takes (16 k per lane)
            auto load_x = [&](int u, uint4 (&dst)[T][2]) {
                const int64_t k = (int64_t)u * 1024 + 64 * warp + 16 * cl;
#pragma unroll
                for (int n = 0; n < T; ++n) {
                    const int t = 8 * n + gid;
                    if (t < M && k < K) {
                        const uint16_t *src = x + (int64_t)t * K + k;
                        dst[n][0] = __ldcg(reinterpret_cast<const uint4 *>(src));
                        if (k + 8 < K)
                            dst[n][1] = __ldcg(reinterpret_cast<const uint4 *>(src + 8));
                        else
                            dst[n][1] = make_uint4(0, 0, 0, 0);
                    } else {
                        zero_x(dst[n][0], dst[n][1]);
                    }
                }
            };

            float fa[3] = {0.f, 0.f, 0.f};   // this CTA's partials of the next op's u, slots as uv
            int i = first_item(c, op.base, G);
            const bool any_item = i < n_items;
            // ---- EC units: 16 rows of G over 256 k (warps 0..3, one 64-k sub-block each)
            int g_done = 0;
            for (; i < n_g && i < n_items; i += G) {
                if (!p.ec_on)
                    continue;
                const int JB = op.R1p / 16, jg = i % JB, ck = i / JB;
                const int s = rseq % kStages;
                float acc[T][4];
#pragma unroll
                for (int n = 0; n < T; ++n)
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        acc[n][q] = 0.f;
                if (warp < 4) {
                    uint4 xv[T][2];
                    const int64_t k = (int64_t)ck * 256 + 64 * warp + 16 * cl;
#pragma unroll
                    for (int n = 0; n < T; ++n) {
                        const int t = 8 * n + gid;
                        if (t < M && k < K) {
                            const uint16_t *src = x + (int64_t)t * K + k;
                            xv[n][0] = __ldcg(reinterpret_cast<const uint4 *>(src));
                            if (k + 8 < K)
                                xv[n][1] = __ldcg(reinterpret_cast<const uint4 *>(src + 8));
                            else
                                xv[n][1] = make_uint4(0, 0, 0, 0);
                        } else {
                            zero_x(xv[n][0], xv[n][1]);
                        }
                    }
                    if (mbar_wait(smem_addr(&full[s]), (rseq / kStages) & 1, abrt, op.status)) {
                        // 16 rows of G, natural k order, 128B-swizzled [4 k-blocks][16 rows][128 B]
                        const uint8_t *gt = bp + s * kUnitBytes + warp * 2048;
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
                            for (int q = 0; q < 4; ++q)
                                mma_bf16_16816(acc[n], ga[2 * q], ha[2 * q], ga[2 * q + 1], ha[2 * q + 1], xa[2 * q],
                                               xa[2 * q + 1]);
                        }
                    }
                }
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(smem_addr(&empty[s]));
                ++rseq;
                // partial [16 rows][TOK] of the four warps, summed in warp order
                if (warp < 4) {
                    float *mine = red + warp * TOK * 16;
#pragma unroll
                    for (int n = 0; n < T; ++n) {
                        const int col = 8 * n + 2 * cl;
                        mine[col * 16 + gid] = acc[n][0];
                        mine[(col + 1) * 16 + gid] = acc[n][1];
                        mine[col * 16 + gid + 8] = acc[n][2];
                        mine[(col + 1) * 16 + gid + 8] = acc[n][3];
                    }
                }
                bar_consumers();
                if (tid < 16 * TOK) {
                    const int row = tid & 15, t = tid >> 4;
                    const float v = red[tid] + red[TOK * 16 + tid] + red[2 * TOK * 16 + tid] + red[3 * TOK * 16 + tid];
                    if (t < M)
                        atomicAdd(uacc + (16 * jg + row) * kUStride + t, v);
                }
                bar_consumers();   // red is free again; every unit's adds are issued
                ++g_done;
            }
            if (g_done > 0 && tid == 0) {
                __threadfence();
                red_release_gpu_add(p.done + p.n_ops + l, (unsigned)g_done);
            }

            // ---- groups of up to TG tiles (16 weight rows each, all of K)
            uint4 xq[XD][T][2];
            bool xkept = false;
            while (i < n_items) {
                int n0s[TG];
                int ng = 0;
#pragma unroll
                for (int tg = 0; tg < TG; ++tg)
                    if (i < n_items) {
                        n0s[tg] = 16 * (i - n_g);
                        ++ng;
                        i += G;
                    }
                // activations of the first XD stages (all tiles of the group share
                // them; when they are all of K they stay for the op's later groups)
                if (!(xkept && nu <= XD)) {
#pragma unroll
                    for (int q = 0; q < XD; ++q) {
                        if (q < nu)
                            load_x(q, xq[q]);
                        else
#pragma unroll
                            for (int n = 0; n < T; ++n)
                                zero_x(xq[q][n][0], xq[q][n][1]);
                    }
                    xkept = true;
                }
                // operands: the zero points of this lane's two rows in each tile
                bool mok = true;
                uint32_t negg[TG], negh[TG];
#pragma unroll
                for (int tg = 0; tg < TG; ++tg) {
                    negg[tg] = negh[tg] = 0u;
                    if (tg < ng) {
                        const uint32_t ms = (mseq + tg) % kMetaSlots;
                        mok = mok && mbar_wait(smem_addr(&mfull[ms]), ((mseq + tg) / kMetaSlots) & 1, abrt, op.status);
                        const uint8_t *meta = bp + L.meta + ms * kMetaBytes;
                        const uint32_t zg = meta[64 + gid], zh = meta[64 + gid + 8];
                        const uint32_t nbg = __bfloat16_as_ushort(__float2bfloat16_rn(-(float)(128u + zg)));
                        const uint32_t nbh = __bfloat16_as_ushort(__float2bfloat16_rn(-(float)(128u + zh)));
                        negg[tg] = nbg | (nbg << 16);
                        negh[tg] = nbh | (nbh << 16);
                    }
                }
                float acc[TG][T][4];
#pragma unroll
                for (int tg = 0; tg < TG; ++tg)
#pragma unroll
                    for (int n = 0; n < T; ++n)
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            acc[tg][n][q] = 0.f;
                for (int u0 = 0; u0 < nu; u0 += XD) {
#pragma unroll
                    for (int q = 0; q < XD; ++q) {
                        const int u = u0 + q;
                        if (u < nu) {
                            const uint4 (&xv)[T][2] = xq[q];
                            const int sb = 16 * u + warp;   // 64-k sub-block of K
#pragma unroll
                            for (int tg = 0; tg < TG; ++tg) {
                                if (tg < ng) {
                                    const int s = rseq % kStages;
                                    if (mok && sb < nsb &&
                                        mbar_wait(smem_addr(&full[s]), (rseq / kStages) & 1, abrt, op.status)) {
                                        // codes k = 64 sb + 16 cl + {0..15} of rows gid and gid + 8 (8 bytes
                                        // each) in chunk warp / 4 of the stage, [16 rows][128 B], 128B swizzle
                                        const uint8_t *ct = bp + s * kUnitBytes + (warp >> 2) * 2048;
                                        const int unit = ((2 * (warp & 3) + (cl >> 1)) ^ gid) * 16 + (cl & 1) * 8;
                                        const uint2 wgv = *reinterpret_cast<const uint2 *>(ct + gid * 128 + unit);
                                        const uint2 whv = *reinterpret_cast<const uint2 *>(ct + (gid + 8) * 128 + unit);
#pragma unroll
                                        for (int j = 0; j < 2; ++j) {
                                            const uint32_t wgw = j ? wgv.y : wgv.x, whw = j ? whv.y : whv.x;
                                            const uint32_t g0 = dequant_pair(wgw, negg[tg]);
                                            const uint32_t g1 = dequant_pair(wgw >> 4, negg[tg]);
                                            const uint32_t g2 = dequant_pair(wgw >> 8, negg[tg]);
                                            const uint32_t g3 = dequant_pair(wgw >> 12, negg[tg]);
                                            const uint32_t h0 = dequant_pair(whw, negh[tg]);
                                            const uint32_t h1 = dequant_pair(whw >> 4, negh[tg]);
                                            const uint32_t h2 = dequant_pair(whw >> 8, negh[tg]);
                                            const uint32_t h3 = dequant_pair(whw >> 12, negh[tg]);
#pragma unroll
                                            for (int n = 0; n < T; ++n) {
                                                const uint4 v = xv[n][j];
                                                mma_bf16_16816(acc[tg][n], g0, h0, g1, h1, v.x, v.y);
                                                mma_bf16_16816(acc[tg][n], g2, h2, g3, h3, v.z, v.w);
                                            }
                                        }
                                    }
                                    __syncwarp();
                                    if (lane == 0)
                                        mbar_arrive(smem_addr(&empty[s]));
                                    ++rseq;
                                }
                            }
                            // this slot's activations are used: request those of stage u + XD
                            if (u + XD < nu)
                                load_x(u + XD, xq[q]);
                        }
                    }
                }
                // partial tiles of this warp: red[tile][warp][token][row]
#pragma unroll
                for (int tg = 0; tg < TG; ++tg) {
                    if (tg < ng) {
                        float *mine = red + (tg * kW + warp) * TOK * 16;
#pragma unroll
                        for (int n = 0; n < T; ++n) {
                            const int col = 8 * n + 2 * cl;
                            mine[col * 16 + gid] = acc[tg][n][0];
                            mine[(col + 1) * 16 + gid] = acc[tg][n][1];
                            mine[col * 16 + gid + 8] = acc[tg][n][2];
                            mine[(col + 1) * 16 + gid + 8] = acc[tg][n][3];
                        }
                    }
                }
                if (u_in_regs) {
                    store_u();
                    u_in_regs = false;
                    u_ready = true;
                }
                bar_consumers();
                if (!u_ready) {
                    // u of this op comes from its EC units (this and other CTAs)
                    if (tid == 0 && poll_count(p.done + p.n_ops + l, (unsigned)n_g, abrt, op.status))
                        __threadfence();
                    bar_consumers();
                    fetch_u();
                    store_u();
                    bar_consumers();
                    u_ready = true;
                }
                // epilogue: thread = (tile, token, row)
                {
                    const int tg = tid / (16 * TOK), e = tid - tg * 16 * TOK;
                    if (tg < ng) {
                        const int row = e & 15, t = e >> 4;
                        const float *rb = red + tg * kW * TOK * 16;
                        float sum = rb[e];
#pragma unroll
                        for (int w = 1; w < kW; ++w)
                            sum += rb[w * TOK * 16 + e];
                        const uint8_t *meta = bp + L.meta + ((mseq + tg) % kMetaSlots) * kMetaBytes;
                        float out = reinterpret_cast<const float *>(meta)[row] * sum;
                        if (ec && t < M) {
                            const uint16_t *btrow = reinterpret_cast<const uint16_t *>(meta + kMetaBtOff) + row * op.rp;
                            const float *ut = us + t * kStackMaxR1p + 1;
                            float corr = 0.f;
                            for (int j0 = 0; j0 < op.rp; j0 += 8) {
                                const uint4 bv = *reinterpret_cast<const uint4 *>(btrow + j0);
                                corr += ut[j0] * bf16_lo(bv.x) + ut[j0 + 1] * bf16_hi(bv.x) +
                                        ut[j0 + 2] * bf16_lo(bv.y) + ut[j0 + 3] * bf16_hi(bv.y) +
                                        ut[j0 + 4] * bf16_lo(bv.z) + ut[j0 + 5] * bf16_hi(bv.z) +
                                        ut[j0 + 6] * bf16_lo(bv.w) + ut[j0 + 7] * bf16_hi(bv.w);
                            }
                            const float g = 1.0f / (1.0f + expf(-(us[t * kStackMaxR1p] + op.b_g)));
                            out += g * corr;
                        }
                        const uint16_t ob = __bfloat16_as_ushort(__float2bfloat16_rn(out));
                        int n0 = 0;
#pragma unroll
                        for (int q = 0; q < TG; ++q)
                            if (q == tg)
                                n0 = n0s[q];
                        const bool live = t < M && n0 + row < N;
                        if (live)
                            y[(int64_t)t * N + n0 + row] = ob;
                        ybf[(tg * TOK + t) * 16 + row] = live ? ob : (uint16_t)0;
                    }
                }
                if (fuse) {
                    bar_consumers();
                    // the group's share of the next op's u: G_{l+1}[j][n0 .. n0 + 15] . y[t][n0 .. n0 + 15]
#pragma unroll
                    for (int tg = 0; tg < TG; ++tg) {
                        if (tg < ng) {
                            const uint16_t *gn = reinterpret_cast<const uint16_t *>(
                                bp + L.meta + ((mseq + tg) % kMetaSlots) * kMetaBytes + kMetaGnOff);
#pragma unroll
                            for (int q = 0; q < 3; ++q) {
                                const int e = tid + kConsumers * q, j = e / TOK, t = e - j * TOK;
                                if (j < op.R1p_next) {
                                    const uint4 g0 = *reinterpret_cast<const uint4 *>(gn + j * 16);
                                    const uint4 g1 = *reinterpret_cast<const uint4 *>(gn + j * 16 + 8);
                                    const uint16_t *yt = ybf + (tg * TOK + t) * 16;
                                    const uint4 y0 = *reinterpret_cast<const uint4 *>(yt);
                                    const uint4 y1 = *reinterpret_cast<const uint4 *>(yt + 8);
                                    fa[q] += bf16_lo(g0.x) * bf16_lo(y0.x) + bf16_hi(g0.x) * bf16_hi(y0.x) +
                                             bf16_lo(g0.y) * bf16_lo(y0.y) + bf16_hi(g0.y) * bf16_hi(y0.y) +
                                             bf16_lo(g0.z) * bf16_lo(y0.z) + bf16_hi(g0.z) * bf16_hi(y0.z) +
                                             bf16_lo(g0.w) * bf16_lo(y0.w) + bf16_hi(g0.w) * bf16_hi(y0.w) +
                                             bf16_lo(g1.x) * bf16_lo(y1.x) + bf16_hi(g1.x) * bf16_hi(y1.x) +
                                             bf16_lo(g1.y) * bf16_lo(y1.y) + bf16_hi(g1.y) * bf16_hi(y1.y) +
                                             bf16_lo(g1.z) * bf16_lo(y1.z) + bf16_hi(g1.z) * bf16_hi(y1.z) +
                                             bf16_lo(g1.w) * bf16_lo(y1.w) + bf16_hi(g1.w) * bf16_hi(y1.w);
                                }
                            }
                        }
                    }
                }
                // the group's operands, partial tiles and outputs are no longer read
                bar_consumers();
                if (tid == 0)
                    for (int tg = 0; tg < ng; ++tg)
                        mbar_arrive(smem_addr(&mempty[(mseq + tg) % kMetaSlots]));
                mseq += ng;
            }
            if (fuse && any_item) {
                float *const unext = p.uacc + p.ops[l + 1].u_off;
#pragma unroll
                for (int q = 0; q < 3; ++q) {
                    const int e = tid + kConsumers * q, j = e / TOK, t = e - j * TOK;
                    if (j < op.R1p_next && t < M)
                        atomicAdd(unext + j * kUStride + t, fa[q]);
                }
            }
            // the op is done in this CTA: its outputs (and partials of u) go out
            bar_consumers();
            if (tid == 0) {
                __threadfence();
                red_release_gpu_add(p.done + l, 1u);
            }
        }
    }
    __syncthreads();
}

template <int T>
const void *stack_fn()
{
    return reinterpret_cast<const void *>(stack_decode_kernel<T>);
}

}  // namespace

size_t stack_decode_smem(int T)
{
    return (T == 1 ? stack_layout<1>().total : stack_layout<2>().total) + 1024;
}

cudaError_t stack_decode_maps(const Packed &pk, CUtensorMap *codes, CUtensorMap *g)
{
    const int nch = (int)(pk.Kp / 256);
    const uint64_t dims[3] = {32, 64, (uint64_t)(pk.Np / 64) * (uint64_t)nch};
    const uint64_t strides[2] = {128, 8192};
    const uint32_t box[3] = {32, 16, 4};
    cudaError_t e = make_map_nd(codes, pk.codes, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, dims, strides, box,
                                CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess)
        return e;
    if (pk.r > 0) {
        const uint64_t gd[3] = {64, (uint64_t)pk.R1p, (uint64_t)(pk.Kp / 64)};
        const uint64_t gs[2] = {(uint64_t)pk.Kp * 2, 128};
        const uint32_t gb[3] = {64, 16, 4};
        return make_map_nd(g, pk.G, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, gd, gs, gb, CU_TENSOR_MAP_SWIZZLE_128B);
    }
    *g = *codes;
    return cudaSuccess;
}

bool stack_decode_layer_ok(const Packed &pk)
{
    return pk.K % 8 == 0 && pk.rp <= kStackMaxRp && pk.R1p <= kStackMaxR1p;
}

bool stack_decode_fits(int num_sms)
{
    for (int T = 1; T <= 2; ++T) {
        const void *fn = T == 1 ? stack_fn<1>() : stack_fn<2>();
        if (!grid_is_one_wave(fn, kThreads, stack_decode_smem(T), 1, num_sms, num_sms))
            return false;
    }
    return true;
}

cudaError_t launch_stack_decode(const StackOpDev *ops, const CUtensorMap *maps, int n_ops, const void *x, void *y,
                                int64_t M, bool ec_on, unsigned *done, float *uacc, size_t ws_bytes, bool fault,
                                cudaStream_t st, int num_sms)
{
    if (M < 1 || M > kStackMaxTokens || n_ops < 1)
        return cudaErrorInvalidValue;
    const int T = M <= 8 ? 1 : 2;
    const void *fn = T == 1 ? stack_fn<1>() : stack_fn<2>();
    const size_t smem = stack_decode_smem(T);
    cudaError_t e = raise_smem_limit(fn, smem);
    if (e != cudaSuccess)
        return e;
    if (!grid_is_one_wave(fn, kThreads, smem, 1, num_sms, num_sms))
        return cudaErrorInvalidConfiguration;
    // counters and u accumulators start at zero
    e = cudaMemsetAsync(done, 0, ws_bytes, st);
    if (e != cudaSuccess)
        return e;
    StackParams p;
    p.ops = ops;
    p.maps = maps;
    p.x = static_cast<const uint16_t *>(x);
    p.y = static_cast<uint16_t *>(y);
    p.done = done;
    p.uacc = uacc;
    p.n_ops = n_ops;
    p.M = (int)M;
    p.ec_on = ec_on ? 1 : 0;
    p.fault = fault ? 1 : 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)num_sms);
    cfg.blockDim = dim3((unsigned)kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = nullptr;
    cfg.numAttrs = 0;
    if (T == 1)
        return cudaLaunchKernelEx(&cfg, stack_decode_kernel<1>, p);
    return cudaLaunchKernelEx(&cfg, stack_decode_kernel<2>, p);
}

}  // namespace spear
