// Decode-size W4 GEMM (up to 16 tokens) with the Error Compensator fused in:
// a cluster of CTAs splits K, each CTA reads only its slice of the
// activations, and the partial tiles are summed over distributed shared
// memory.
//
// SPEAR, "A System for Post-Quantization Error-Adaptive Recovery Enabling
// Efficient Low-Bit LLM Serving", Abstract: the post-EC computation is fused
// into the low-bit GEMM.  In a decode pass a layer's time is the chain
// "previous layer done -> this layer done"; on B200 the part of that chain
// that grows with the design is not the HBM stream of the codes (8 MB of a
// 4096 x 4096 layer stream in 1.3 us) but what every CTA must do after the
// dependency wait.  Reading all of x in every CTA costs about 2 us per layer
// from L2 at 16 tokens, so:
//
//  * the grid is n_clusters clusters of CS CTAs; cluster c owns a balanced
//    range of 16-row tiles, and CTA rank q of it owns the K slice q (cpr
//    256-k chunks), for all of the cluster's tiles.  A CTA stages only its
//    slice of x in shared memory (one TMA box of TOK tokens x 64 k per
//    sub-block, 128B swizzle), once, after the dependency wait;
//  * the tiles are taken in groups of four; a producer warp streams the
//    group's codes of the slice through a ring of 16 KB stages (4 tiles x
//    512 k), issuing every stage that fits before the dependency wait (the
//    codes do not depend on earlier kernels, and the CTA is small enough for
//    the next layer's CTAs to be resident beside the current layer's);
//  * eight consumer warps (two tile pairs x four sub-block pairs) dequantise
//    the codes in registers to exact (q - z) bf16 pairs and run mma.sync
//    m16n8k16 with weight rows on the 16-row side and tokens on the 8-column
//    side (the same fragment layout as the other decode kernels);
//  * after each group the four sub-block partials of a tile are summed in
//    shared memory in warp order and the tile's slice partial is pushed with
//    st.async into a receive slot of the rank that owns the tile (tile i of a
//    group belongs to rank i mod CS), counted on that rank's mbarrier; the
//    owner sums the CS slices in rank order (deterministic);
//  * the EC down-projection u = x . [w_g, A] is cut into units (16 rows of G
//    x one 256-k chunk) that the CTAs owning the chunk take in turn (G rows
//    arrive by TMA before the dependency wait); a unit's partial goes to
//    global memory and the unit that completes a 16-row group of G (counter,
//    last arriver) sums its chunks in order and counts the group as done.
//    The EC warp of every CTA waits (bounded) for all groups, reads u and
//    g_t = 1 / (1 + exp(-(u_0 + b_g))) into shared memory, and the owner's
//    epilogue forms
//        y[t,n] = bf16( s[n] * acc[t,n] + g_t * sum_j u[t,1+j] B[j,n] )
//    in fp32.  Every wait is bounded (about a second), after which the kernel
//    records a timeout in the handle's status word and returns.
#include <algorithm>
#include <mutex>
#include <new>
#include <vector>

#include "async_utils.cuh"
#include "kernels.h"
#include "tensor_map.h"

namespace spear {
namespace {

constexpr int kTile = 16;                  // weight rows per tile (the MMA's 16-row side)
constexpr int kTG = 4;                     // tiles per group
constexpr int kSubBlocks = 8;             // 64-k sub-blocks of a stage (512 k)
constexpr int kCW = 2 * kSubBlocks;        // consumer warps: (tile pair, sub-block)
constexpr int kThreads = 32 * (kCW + 2);   // + producer warp + EC warp
constexpr int kMaxStageChunks = 4;         // 256-k chunks of a stage (one TMA box per tile)
constexpr int kMaxStages = 16;
constexpr int kMaxGroups = 16;
constexpr int kGSlots = 2;                 // G unit buffers, 8 KB each
constexpr int kUStr = 16;                  // token stride of the G partials and of u
constexpr int kMaxGt = 9;                  // 16-row groups of G (R1p <= 144)
constexpr size_t kSmemPair = 113 * 1024;   // two CTAs per SM (228 KB, 1 KB reserved per CTA)
constexpr size_t kSmemOne = 200 * 1024;

struct StreamMaps {
    CUtensorMap codes;   // tiled codes as [blocks][64 rows][32 words]: box 32 x 16 rows x 2 blocks
    CUtensorMap g;       // [R1p][Kp] bf16 as [Kp/64][R1p][64]: box 64 x 16 rows x 4 k-blocks (8 KB)
};

struct StreamParams {
    const uint16_t *Bt;    // [Np][rp]
    const float *s;
    const uint8_t *z;
    uint16_t *y;
    float *gpart;          // [n_gt][nch][16][kUStr]
    float *ufin;           // [R1p][kUStr]
    unsigned *cnt;         // [0] groups of G done, [1] CTAs done with u, [2 + g] chunks of G group g done
    int *status;
    int64_t M, N;
    int n_tiles, CS, n_clusters;
    int nch, cpr;          // 256-k chunks of Kp, chunks per rank
    int S;                 // ring stages
    int sc;                // chunks per stage (a stage is 4 tiles x sc chunks, one box per tile)
    int r, rp, R1p, n_gt;  // n_gt = R1p / 16, 0 without the EC
    int own_max;           // tiles of a group owned by one rank, at most
    int g_slots;           // G unit buffers in use (1 or 2)
    int btw;               // row stride of the staged B^T rows (bf16 elements)
    int ustr;              // token stride of the staged u (floats)
    int x3;                // tm_x is the 3-D view [K/64][M][64] (K a multiple of 64)
    float b_g;
    uint32_t off_x, off_red, off_recv, off_g, off_bt, off_u, off_zs;
    const void *pf;
    uint64_t pf_bytes;
};

__device__ __forceinline__ void consumers_sync()
{
    asm volatile("bar.sync 1, %0;" ::"r"(kCW * 32) : "memory");
}

__device__ __forceinline__ unsigned atom_add_acq_rel(unsigned *p, unsigned v)
{
    unsigned old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// x fragment of token group n for the 64-k sub-block at `box` (TOK rows x
// 128 B, 128B swizzle): 16 consecutive k of token 8n + gid from k = 16 cl.
__device__ __forceinline__ void load_x(const uint8_t *box, int n, int gid, int cl, uint4 &lo, uint4 &hi)
{
    const int t = 8 * n + gid;
    const uint8_t *row = box + t * 128;
    lo = *reinterpret_cast<const uint4 *>(row + (((2 * cl) ^ (t & 7)) << 4));
    hi = *reinterpret_cast<const uint4 *>(row + (((2 * cl + 1) ^ (t & 7)) << 4));
}

// One token group: two CTAs per SM (the next layer's beside this one's);
// two: one.
template <int T>
__global__ void __launch_bounds__(kThreads, T == 1 ? 2 : 1)
decode_stream_kernel(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_g,
                     const __grid_constant__ CUtensorMap tm_x, StreamParams p)
{
    constexpr int TOK = 8 * T;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full[kMaxStages], empty[kMaxStages], gbar[kGSlots], recvbar[kMaxGroups];
    __shared__ __align__(8) uint64_t xbar, ubar;
    __shared__ int abort_flag;

    pdl_launch_dependents();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gid = lane >> 2, cl = lane & 3;
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    const uint8_t *sm = smem_raw + (base - raw);   // generic view of the aligned base
    const int CS = p.CS;
    const int q = (int)cluster_ctarank();
    const int ci = (int)blockIdx.x / CS;
    const int t_lo = (int)((int64_t)ci * p.n_tiles / p.n_clusters);
    const int t_hi = (int)((int64_t)(ci + 1) * p.n_tiles / p.n_clusters);
    const int ct = t_hi - t_lo;
    const int ngroups = (ct + kTG - 1) / kTG;
    const int c_lo = q * p.cpr;
    const int my_ch = max(0, min(p.nch, c_lo + p.cpr) - c_lo);
    const int nst = (my_ch + p.sc - 1) / p.sc;  // stages per group
    const uint32_t stage_bytes = (uint32_t)kTG * p.sc * 2048u;
    const int total = ngroups * nst;
    const bool ec = p.n_gt > 0;
    // G units of this rank (16 rows of G x one chunk of its slice), split over the clusters
    const int uq = p.n_gt * my_ch;
    const int u_lo = (int)((int64_t)ci * uq / p.n_clusters), u_hi = (int)((int64_t)(ci + 1) * uq / p.n_clusters);
    const int n_units = ec ? u_hi - u_lo : 0;

    auto tiles_of = [&](int g) { return min(kTG, ct - g * kTG); };
    auto owned_in = [&](int g) {   // tiles of group g owned by this rank
        const int tg = tiles_of(g);
        return tg > q ? (tg - q + CS - 1) / CS : 0;
    };

    // zero points (as the dequantiser's bias) and scales of every row of the
    // cluster's tiles: weights, so read before the dependency wait
    uint32_t *nb_s = reinterpret_cast<uint32_t *>(const_cast<uint8_t *>(sm) + p.off_zs);
    float *sc_s = reinterpret_cast<float *>(nb_s + ct * kTile);
    for (int i = tid; i < ct * kTile; i += kThreads) {
        const int64_t n = (int64_t)t_lo * kTile + i;
        const uint32_t nb = __bfloat16_as_ushort(__float2bfloat16_rn(-(float)(128u + __ldg(p.z + n))));
        nb_s[i] = nb | (nb << 16);
        sc_s[i] = __ldg(p.s + n);
    }
    if (tid == 0) {
        abort_flag = 0;
        for (int s = 0; s < p.S; ++s) {
            mbar_init(smem_addr(&full[s]), 1);
            mbar_init(smem_addr(&empty[s]), kCW);
        }
        for (int s = 0; s < kGSlots; ++s)
            mbar_init(smem_addr(&gbar[s]), 1);
        for (int g = 0; g < ngroups; ++g)
            mbar_init(smem_addr(&recvbar[g]), 1);
        mbar_init(smem_addr(&xbar), 1);
        mbar_init(smem_addr(&ubar), 1);
        fence_mbarrier_init_cluster();
        // this rank expects the other ranks' slices of the tiles it owns
        for (int g = 0; g < ngroups; ++g)
            mbar_expect_tx(smem_addr(&recvbar[g]), (uint32_t)((CS - 1) * owned_in(g) * T * 512));
    }
    __syncthreads();
    // every CTA of the cluster has initialised its receive barriers once this
    // barrier completes; each thread waits for it before its first push
    cluster_arrive_relaxed();

    if (warp == kCW) {
        // ---------------- producer
        if (lane == 0) {
            auto issue = [&](int j) {
                const int slot = j % p.S, g = j / nst, st = j - g * nst;
                const int tg = tiles_of(g);
                const uint32_t bar = smem_addr(&full[slot]);
                mbar_expect_tx(bar, (uint32_t)tg * (uint32_t)p.sc * 2048u);
                const uint32_t dst = base + (uint32_t)slot * stage_bytes;
                for (int i = 0; i < tg; ++i) {
                    // tile t: 16 rows x sc chunks of its row block, one box
                    const int t = t_lo + g * kTG + i;
                    tma_load_3d(dst + (uint32_t)(i * p.sc) * 2048u, &tm_codes, 0, (t & 3) * kTile,
                                (t >> 2) * p.nch + c_lo + st * p.sc, bar);
                }
            };
            const int pre = min(total, p.S);
            for (int j = 0; j < pre; ++j)
                issue(j);
            pdl_wait();
            // this rank's slice of x: one 3-D box of 4 cpr sub-blocks x TOK tokens x
            // 64 k (k beyond K and tokens beyond M read as zero), or, when K is not a
            // multiple of 64, one 2-D box of TOK tokens x 64 k per sub-block
            if (p.x3) {
                mbar_expect_tx(smem_addr(&xbar), (uint32_t)(4 * p.cpr * TOK * 128));
                tma_load_3d(base + p.off_x, &tm_x, 0, 0, c_lo * 4, smem_addr(&xbar));
            } else {
                const int nsb = 4 * my_ch;
                mbar_expect_tx(smem_addr(&xbar), (uint32_t)(nsb * TOK * 128));
                for (int b = 0; b < nsb; ++b)
                    tma_load_2d(base + p.off_x + (uint32_t)(b * TOK * 128), &tm_x, (c_lo * 4 + b) * 64, 0,
                                smem_addr(&xbar));
            }
            bool ok = true;
            for (int j = pre; j < total && ok; ++j) {
                const int slot = j % p.S;
                ok = mbar_wait(smem_addr(&empty[slot]), (uint32_t)((j / p.S) - 1) & 1u, &abort_flag, p.status);
                if (ok)
                    issue(j);
            }
            prefetch_l2_share(p.pf, p.pf_bytes);
            // no copy may still be landing when the CTA leaves
            for (int j = max(0, total - p.S); j < total; ++j)
                mbar_wait_final(smem_addr(&full[j % p.S]), (uint32_t)(j / p.S) & 1u);
            mbar_wait_final(smem_addr(&xbar), 0);
        }
        __syncwarp();
        cluster_wait();
    } else if (warp == kCW + 1) {
        // ---------------- EC warp: B^T rows of the owned tiles, G units, then u
        uint16_t *bts = reinterpret_cast<uint16_t *>(const_cast<uint8_t *>(sm) + p.off_bt);
        if (ec) {
            if (lane == 0) {
                for (int i = 0; i < min(n_units, p.g_slots); ++i) {
                    const int u = u_lo + i, gt = u / my_ch, c = c_lo + u % my_ch;
                    mbar_expect_tx(smem_addr(&gbar[i]), 8192u);
                    tma_load_3d(base + p.off_g + (uint32_t)i * 8192u, &tm_g, 0, kTile * gt, 4 * c,
                                smem_addr(&gbar[i]));
                }
            }
            const int per_row = p.rp / 8;
            for (int g = 0; g < ngroups; ++g)
                for (int o = 0; o < owned_in(g); ++o) {
                    const int t = t_lo + g * kTG + o * CS + q;
                    for (int i = lane; i < kTile * per_row; i += 32) {
                        const int row = i / per_row, c8 = i - row * per_row;
                        const uint4 v = ld_nc(p.Bt + ((int64_t)t * kTile + row) * p.rp + 8 * c8);
                        *reinterpret_cast<uint4 *>(bts + ((g * p.own_max + o) * kTile + row) * p.btw + 8 * c8) = v;
                    }
                }
        }
        pdl_wait();   // the previous forward has reset the counters
        float *u_s = reinterpret_cast<float *>(const_cast<uint8_t *>(sm) + p.off_u);   // [TOK][ustr]
        float *g_s = u_s + TOK * p.ustr;                                              // [TOK]
        if (ec) {
            bool ok = mbar_wait(smem_addr(&xbar), 0, &abort_flag, p.status);
            const int mt = p.M < TOK ? (int)p.M : TOK;
            for (int i = 0; i < n_units; ++i) {
                const int u = u_lo + i, gt = u / my_ch, cc = u % my_ch, c = c_lo + cc;
                const int slot = i % p.g_slots;
                if (ok)
                    ok = mbar_wait(smem_addr(&gbar[slot]), (uint32_t)(i / p.g_slots) & 1u, &abort_flag, p.status);
                float acc[T][4];
#pragma unroll
                for (int n = 0; n < T; ++n)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        acc[n][e] = 0.f;
                if (ok) {
                    const uint32_t gb = base + p.off_g + (uint32_t)slot * 8192u;
#pragma unroll
                    for (int kb = 0; kb < 4; ++kb) {
                        // 16 rows of G, k = 64 kb + 16 cl + {0..15}: natural pairs
                        const uint8_t *gt_ = sm + (gb - base) + kb * 2048;
                        const uint4 a0 = *reinterpret_cast<const uint4 *>(gt_ + gid * 128 + (((2 * cl) ^ gid) << 4));
                        const uint4 a1 =
                            *reinterpret_cast<const uint4 *>(gt_ + gid * 128 + (((2 * cl + 1) ^ gid) << 4));
                        const uint4 b0 =
                            *reinterpret_cast<const uint4 *>(gt_ + (gid + 8) * 128 + (((2 * cl) ^ gid) << 4));
                        const uint4 b1 =
                            *reinterpret_cast<const uint4 *>(gt_ + (gid + 8) * 128 + (((2 * cl + 1) ^ gid) << 4));
                        const uint32_t ga[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                        const uint32_t ha[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
                        const uint8_t *xb = sm + p.off_x + (cc * 4 + kb) * TOK * 128;
#pragma unroll
                        for (int n = 0; n < T; ++n) {
                            uint4 xl, xh;
                            load_x(xb, n, gid, cl, xl, xh);
                            const uint32_t xa[8] = {xl.x, xl.y, xl.z, xl.w, xh.x, xh.y, xh.z, xh.w};
#pragma unroll
                            for (int s4 = 0; s4 < 4; ++s4)
                                mma_bf16_16816(acc[n], ga[2 * s4], ha[2 * s4], ga[2 * s4 + 1], ha[2 * s4 + 1],
                                               xa[2 * s4], xa[2 * s4 + 1]);
                        }
                    }
                }
                __syncwarp();
                // the slot is free: the next unit that uses it
                if (lane == 0 && i + p.g_slots < n_units) {
                    const int u2 = u + p.g_slots, gt2 = u2 / my_ch, c2 = c_lo + u2 % my_ch;
                    mbar_expect_tx(smem_addr(&gbar[slot]), 8192u);
                    tma_load_3d(base + p.off_g + (uint32_t)slot * 8192u, &tm_g, 0, kTile * gt2, 4 * c2,
                                smem_addr(&gbar[slot]));
                }
                // publish the unit's partial [16 rows][tokens]
                float *dst = p.gpart + ((size_t)gt * p.nch + c) * kTile * kUStr;
#pragma unroll
                for (int n = 0; n < T; ++n) {
                    const int t0 = 8 * n + 2 * cl;
                    *reinterpret_cast<float2 *>(dst + gid * kUStr + t0) = make_float2(acc[n][0], acc[n][1]);
                    *reinterpret_cast<float2 *>(dst + (gid + 8) * kUStr + t0) = make_float2(acc[n][2], acc[n][3]);
                }
                __syncwarp();
                unsigned last = 0;
                if (lane == 0) {
                    __threadfence();
                    last = atom_add_acq_rel(&p.cnt[2 + gt], 1u) == (unsigned)(p.nch - 1) ? 1u : 0u;
                }
                last = __shfl_sync(0xFFFFFFFFu, last, 0);
                if (last) {
                    // every chunk of G group gt is in: sum them in chunk order
                    __threadfence();
                    for (int e = lane; e < kTile * mt; e += 32) {
                        const int row = e / mt, t = e - row * mt;
                        const float *src = p.gpart + (size_t)gt * p.nch * kTile * kUStr + row * kUStr + t;
                        // eight chunks' loads in flight at a time, added in chunk order
                        float sum = 0.f;
                        int c2 = 0;
                        for (; c2 + 8 <= p.nch; c2 += 8) {
                            float v[8];
#pragma unroll
                            for (int b = 0; b < 8; ++b)
                                v[b] = __ldcg(src + (size_t)(c2 + b) * kTile * kUStr);
#pragma unroll
                            for (int b = 0; b < 8; ++b)
                                sum += v[b];
                        }
                        for (; c2 < p.nch; ++c2)
                            sum += __ldcg(src + (size_t)c2 * kTile * kUStr);
                        p.ufin[(kTile * gt + row) * kUStr + t] = sum;
                    }
                    __syncwarp();
                    if (lane == 0) {
                        p.cnt[2 + gt] = 0u;
                        __threadfence();
                        red_release_gpu_add(&p.cnt[0], 1u);
                    }
                }
            }
            // u for every token, once every group of G is done (bounded wait)
            int good = 1;
            if (lane == 0) {
                const long long t0 = clock64();
                while (ld_acquire_gpu(&p.cnt[0]) < (unsigned)p.n_gt) {
                    if (abort_flag || clock64() - t0 > kWaitBudgetCycles) {
                        abort_flag = 1;
                        atomicOr(p.status, kStatusTimeout);
                        good = 0;
                        break;
                    }
                    __nanosleep(64);
                }
            }
            good = __shfl_sync(0xFFFFFFFFu, good, 0);
            // row 1 + j of u (TOK tokens, 16-byte loads) per lane, all rows in flight
            for (int j = lane; j < p.rp; j += 32) {
                float4 v[T * 2];
#pragma unroll
                for (int c4 = 0; c4 < 2 * T; ++c4)
                    v[c4] = (good && j < p.r) ? __ldcg(reinterpret_cast<const float4 *>(p.ufin + (1 + j) * kUStr) + c4)
                                              : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int c4 = 0; c4 < 2 * T; ++c4) {
                    const float vv[4] = {v[c4].x, v[c4].y, v[c4].z, v[c4].w};
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int t = 4 * c4 + c;
                        u_s[t * p.ustr + j] = t < mt ? vv[c] : 0.f;
                    }
                }
            }
            for (int t = lane; t < TOK; t += 32) {
                const float logit = (good && t < mt) ? __ldcg(p.ufin + t) : 0.f;
                g_s[t] = 1.0f / (1.0f + expf(-(logit + p.b_g)));
            }
            __syncwarp();
            if (lane == 0) {
                if (atomicAdd(&p.cnt[1], 1u) == gridDim.x - 1) {
                    // every CTA has read u: reset for the next forward
                    p.cnt[1] = 0u;
                    p.cnt[0] = 0u;
                }
                mbar_arrive(smem_addr(&ubar));   // release: this warp's writes of u come first
                // no G copy may still be landing when the CTA leaves
                for (int i = max(0, n_units - p.g_slots); i < n_units; ++i)
                    mbar_wait_final(smem_addr(&gbar[i % p.g_slots]), (uint32_t)(i / p.g_slots) & 1u);
            }
        }
        __syncwarp();
        cluster_wait();
    } else {
        // ---------------- consumers: warp (tp, sb) takes tiles {tp, tp + 2} of a
        // group and sub-block sb of each stage, the same work whatever the
        // group's size (a missing tile's product is computed and dropped, a
        // missing sub-block's activations are zero), so that every load and MMA
        // of a stage can be in flight at once
        const int tp = warp & 1, sb = warp >> 1;
        bool ok = mbar_wait(smem_addr(&xbar), 0, &abort_flag, p.status);
        bool cluster_ready = false;
        // two accumulators per tile (the two 32-k halves of a sub-block), so
        // that a warp has four independent MMA chains in flight
        float acc[2][2][T][4];
        for (int g = 0; g < ngroups; ++g) {
            const int tg = tiles_of(g);
            // zero points of the warp's two tiles, rows gid and gid + 8
            uint32_t negg[2], negh[2];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int tl = tp + 2 * i;
                const int r0 = (g * kTG + (tl < tg ? tl : 0)) * kTile;
                negg[i] = nb_s[r0 + gid];
                negh[i] = nb_s[r0 + gid + 8];
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int n = 0; n < T; ++n)
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            acc[h][i][n][e] = 0.f;
            }
            for (int st = 0; st < nst; ++st) {
                const int j = g * nst + st, slot = j % p.S;
                if (ok)
                    ok = mbar_wait(smem_addr(&full[slot]), (uint32_t)(j / p.S) & 1u, &abort_flag, p.status);
                if (ok) {
                    const int nsb = 4 * min(p.sc, my_ch - st * p.sc);   // sub-blocks of this stage
#pragma unroll
                    for (int hh = 0; hh < kMaxStageChunks / 2; ++hh) {
                        const int sbl = sb + kSubBlocks * hh;
                        if (hh * kSubBlocks >= 4 * p.sc)
                            break;
                        const bool live = sbl < nsb;
                        uint4 xv[T][2];
                        const uint8_t *xb = sm + p.off_x + (st * 4 * p.sc + (live ? sbl : 0)) * TOK * 128;
#pragma unroll
                        for (int n = 0; n < T; ++n) {
                            load_x(xb, n, gid, cl, xv[n][0], xv[n][1]);
                            if (!live)
                                xv[n][0] = xv[n][1] = make_uint4(0, 0, 0, 0);
                        }
                        // codes k = 64 sbl + 16 cl + {0..15} of rows gid and gid + 8 of both
                        // tiles, in chunk sbl / 4 of the tile's box: [16 rows][128 B], 128B swizzle
                        const int sbc = live ? sbl : 0;   // a dead sub-block reads valid codes, times zero
                        const int unit = ((2 * (sbc & 3) + (cl >> 1)) ^ gid) * 16 + (cl & 1) * 8;
                        uint2 wgv[2], whv[2];
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            const uint8_t *ct_ = sm + slot * stage_bytes + ((tp + 2 * i) * p.sc + (sbc >> 2)) * 2048;
                            wgv[i] = *reinterpret_cast<const uint2 *>(ct_ + gid * 128 + unit);
                            whv[i] = *reinterpret_cast<const uint2 *>(ct_ + (gid + 8) * 128 + unit);
                        }
#pragma unroll
                        for (int jj = 0; jj < 2; ++jj) {
#pragma unroll
                            for (int i = 0; i < 2; ++i) {
                                const uint32_t wgw = jj ? wgv[i].y : wgv[i].x, whw = jj ? whv[i].y : whv[i].x;
                                const uint32_t g0 = dequant_pair(wgw, negg[i]), g1 = dequant_pair(wgw >> 4, negg[i]);
                                const uint32_t g2 = dequant_pair(wgw >> 8, negg[i]), g3 = dequant_pair(wgw >> 12, negg[i]);
                                const uint32_t h0 = dequant_pair(whw, negh[i]), h1 = dequant_pair(whw >> 4, negh[i]);
                                const uint32_t h2 = dequant_pair(whw >> 8, negh[i]), h3 = dequant_pair(whw >> 12, negh[i]);
#pragma unroll
                                for (int n = 0; n < T; ++n) {
                                    const uint4 v = xv[n][jj];
                                    mma_bf16_16816(acc[jj][i][n], g0, h0, g1, h1, v.x, v.y);
                                    mma_bf16_16816(acc[jj][i][n], g2, h2, g3, h3, v.z, v.w);
                                }
                            }
                        }
                    }
                }
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(smem_addr(&empty[slot]));
            }
            // ---- group done: partials red[sb][tl][n][row][8 tokens], then the sum
            // over sb pushed to the owning rank
            float *red = reinterpret_cast<float *>(const_cast<uint8_t *>(sm) + p.off_red);
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int tl = tp + 2 * i;
#pragma unroll
                for (int n = 0; n < T; ++n) {
                    float *a = red + ((sb * kTG + tl) * T + n) * 128 + gid * 8 + 2 * cl;
                    *reinterpret_cast<float2 *>(a) =
                        make_float2(acc[0][i][n][0] + acc[1][i][n][0], acc[0][i][n][1] + acc[1][i][n][1]);
                    *reinterpret_cast<float2 *>(a + 64) =
                        make_float2(acc[0][i][n][2] + acc[1][i][n][2], acc[0][i][n][3] + acc[1][i][n][3]);
                }
            }
            consumers_sync();
            if (!cluster_ready) {
                cluster_wait();   // every rank's receive barriers are initialised
                cluster_ready = true;
            }
            if (tid < kTG * T * 32) {
                const int e = tid;   // one float4 (tile, n, row, half) per thread
                const int tl = e / (T * 32), rem = e - tl * (T * 32);
                const int n = rem >> 5, row = (rem & 31) >> 1, half = rem & 1;
                if (tl < tg) {
                    float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                    for (int w = 0; w < kSubBlocks; ++w) {
                        const float4 v =
                            *reinterpret_cast<const float4 *>(red + ((w * kTG + tl) * T + n) * 128 + row * 8 + half * 4);
                        sum.x += v.x;
                        sum.y += v.y;
                        sum.z += v.z;
                        sum.w += v.w;
                    }
                    const int owner = tl % CS, o = tl / CS;
                    const uint32_t off = p.off_recv +
                                         (uint32_t)((((((g * CS + q) * p.own_max + o) * T + n) * 128) + row * 8 +
                                                     half * 4) * 4);
                    if (owner == q) {
                        *reinterpret_cast<float4 *>(const_cast<uint8_t *>(sm) + off) = sum;
                    } else {
                        const uint32_t remote = map_to_rank(base + off, (uint32_t)owner);
                        const uint32_t rbar = map_to_rank(smem_addr(&recvbar[g]), (uint32_t)owner);
                        st_async_f4(remote, sum, rbar);
                    }
                }
            }
            consumers_sync();   // red is free for the next group
        }
        if (!cluster_ready)
            cluster_wait();

        // ---- epilogue of the owned tiles: sum the CS slices in rank order, scale,
        // add the gated correction, round to bf16
        const uint16_t *bts = reinterpret_cast<const uint16_t *>(sm + p.off_bt);
        const float *u_s = reinterpret_cast<const float *>(sm + p.off_u);
        const float *g_s = u_s + TOK * p.ustr;
        bool have_u = !ec;
        for (int g = 0; g < ngroups; ++g) {
            const int own = owned_in(g);
            if (own == 0)
                continue;
            if (!mbar_wait(smem_addr(&recvbar[g]), 0, &abort_flag, p.status))
                ok = false;
            if (ec && !have_u) {
                if (!mbar_wait(smem_addr(&ubar), 0, &abort_flag, p.status))
                    ok = false;
                have_u = true;
            }
            for (int e = tid; e < own * kTile * TOK; e += kCW * 32) {
                const int t = e % TOK, row = (e / TOK) % kTile, o = e / (TOK * kTile);
                const int n = t >> 3, t8 = t & 7;
                float acc_sum = 0.f;
                for (int src = 0; src < CS; ++src)
                    acc_sum += reinterpret_cast<const float *>(sm + p.off_recv)
                        [((((g * CS + src) * p.own_max + o) * T + n) * 128) + row * 8 + t8];
                const int tl = o * CS + q;
                const int64_t nn = (int64_t)(t_lo + g * kTG + tl) * kTile + row;
                float out = sc_s[(g * kTG + tl) * kTile + row] * acc_sum;
                if (ec && t < p.M) {
                    const uint16_t *brow = bts + ((g * p.own_max + o) * kTile + row) * p.btw;
                    const float *ut = u_s + t * p.ustr;
                    float corr = 0.f;
                    for (int j0 = 0; j0 < p.rp; j0 += 8) {
                        const uint4 bv = *reinterpret_cast<const uint4 *>(brow + j0);
                        const float4 v0 = *reinterpret_cast<const float4 *>(ut + j0);
                        const float4 v1 = *reinterpret_cast<const float4 *>(ut + j0 + 4);
                        corr += v0.x * bf16_lo(bv.x) + v0.y * bf16_hi(bv.x) + v0.z * bf16_lo(bv.y) +
                                v0.w * bf16_hi(bv.y) + v1.x * bf16_lo(bv.z) + v1.y * bf16_hi(bv.z) +
                                v1.z * bf16_lo(bv.w) + v1.w * bf16_hi(bv.w);
                    }
                    out += g_s[t] * corr;
                }
                if (t < p.M && nn < p.N)
                    p.y[(int64_t)t * p.N + nn] = __bfloat16_as_ushort(__float2bfloat16_rn(out));
            }
        }
        if (!ok)
            atomicOr(p.status, kStatusTimeout);
    }
    // no warp leaves before the others are done (the EC warp's u and the
    // receive slots live in this CTA's shared memory)
    __syncthreads();
}

template <int T>
const void *stream_ptr()
{
    return reinterpret_cast<const void *>(decode_stream_kernel<T>);
}

struct StreamPlan {
    int CS = 0, n_clusters = 0, cpr = 0, S = 0, sc = 1, own_max = 0, btw = 0, ustr = 0, g_slots = 1;
    uint32_t off_x = 0, off_red = 0, off_recv = 0, off_g = 0, off_bt = 0, off_u = 0, off_zs = 0;
    size_t smem = 0;
};

// Shared memory after the ring: x slice, partials, receive slots, G units,
// B^T rows of the owned tiles, u and g.
bool stream_layout(const Packed &pk, int T, int CS, int n_clusters, int S, bool ec, StreamPlan &pl)
{
    const int TOK = 8 * T;
    const int nch = (int)(pk.Kp / 256);
    const int cpr = (nch + CS - 1) / CS;
    const int n_tiles = (int)(pk.Np / kTile);
    const int ct_max = (n_tiles + n_clusters - 1) / n_clusters;
    const int ng_max = (ct_max + kTG - 1) / kTG;
    if (ng_max > kMaxGroups)
        return false;
    pl.CS = CS;
    pl.n_clusters = n_clusters;
    pl.cpr = cpr;
    pl.S = S;
    pl.sc = std::min(cpr, kMaxStageChunks);
    pl.own_max = (kTG + CS - 1) / CS;
    // G units of one CTA at most: 16-row groups of G x chunks of a slice, over the clusters
    const int gu_max = ec ? ((pk.R1p / kTile) * cpr + n_clusters - 1) / n_clusters : 0;
    pl.g_slots = std::max(1, std::min(kGSlots, gu_max));
    pl.btw = pk.rp + 8;
    pl.ustr = pk.rp + 4;
    size_t off = (size_t)S * kTG * pl.sc * 2048;
    pl.off_x = (uint32_t)off;
    off += (size_t)4 * cpr * TOK * 128;
    pl.off_red = (uint32_t)off;
    off += (size_t)kSubBlocks * kTG * T * 512;
    pl.off_recv = (uint32_t)off;
    off += (size_t)ng_max * CS * pl.own_max * T * 512;
    pl.off_g = (uint32_t)off;
    off += ec ? (size_t)pl.g_slots * 8192 : 0;
    pl.off_bt = (uint32_t)off;
    off += ec ? (size_t)ng_max * pl.own_max * kTile * pl.btw * 2 : 0;
    off = (off + 15) / 16 * 16;
    pl.off_u = (uint32_t)off;
    off += ec ? (size_t)TOK * pl.ustr * 4 + TOK * 4 : 0;
    // per row of the CTA's tiles: the dequantiser's bf16x2 bias -(128 + z) and the scale
    pl.off_zs = (uint32_t)off;
    off += (size_t)ct_max * kTile * 8;
    pl.smem = off + 1024;
    return true;
}

// Cluster size (the K split) and ring depth: the split whose slowest cluster
// has the least work (tiles x chunks), its x slice at most 64 KB; two CTAs per
// SM when every stage of a group fits beside the rest, else one.
bool stream_plan(const Packed &pk, int64_t M, bool ec, int num_sms, StreamPlan &best)
{
    const int T = M <= 8 ? 1 : 2;
    const int nch = (int)(pk.Kp / 256);
    const int n_tiles = (int)(pk.Np / kTile);
    long best_cost = -1;
    for (int CS : {4, 8, 2}) {
        const int cpr = (nch + CS - 1) / CS;
        if ((CS - 1) * cpr >= nch)
            continue;   // every rank needs a chunk
        if ((size_t)4 * cpr * 8 * T * 128 > 64 * 1024)
            continue;
        const int n_clusters = std::min(num_sms / CS, n_tiles);
        if (n_clusters < 1)
            continue;
        const int ct_max = (n_tiles + n_clusters - 1) / n_clusters;
        const long cost = (long)ct_max * cpr;
        if (best_cost >= 0 && cost >= best_cost)
            continue;
        const int ng_max = (ct_max + kTG - 1) / kTG;
        const int sc = std::min(cpr, kMaxStageChunks);
        const int total = ng_max * ((cpr + sc - 1) / sc);
        StreamPlan pl;
        int S = std::min(total, kMaxStages);
        bool fit = false;
        for (; T == 1 && S >= 2 && !fit; --S) {
            if (!stream_layout(pk, T, CS, n_clusters, S, ec, pl))
                break;
            fit = pl.smem <= kSmemPair;
        }
        if (!fit) {
            S = std::min(total, kMaxStages);
            for (; S >= 1 && !fit; --S) {
                if (!stream_layout(pk, T, CS, n_clusters, S, ec, pl))
                    break;
                fit = pl.smem <= kSmemOne;
            }
        }
        if (!fit)
            continue;
        best = pl;
        best_cost = cost;
    }
    return best_cost >= 0;
}

// Largest number of clusters of this configuration that are resident at once
// (all must be: the G groups are counted across the grid), once per
// (kernel, cluster size, shared memory).
int max_active_clusters(int T, int CS, size_t smem)
{
    struct Entry {
        int T, CS, dev;
        size_t smem;
        int n;
    };
    static std::vector<Entry> cache;
    static std::mutex mu;
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lock(mu);
    for (const Entry &e : cache)
        if (e.T == T && e.CS == CS && e.smem == smem && e.dev == dev)
            return e.n;
    const void *fn = T == 1 ? stream_ptr<1>() : stream_ptr<2>();
    if (raise_smem_limit(fn, smem) != cudaSuccess)
        return 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)CS);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess)
        n = 0;
    cache.push_back({T, CS, dev, smem, n});
    return n;
}

}  // namespace

bool decode_stream_shape(const Packed &pk)
{
    return pk.rp <= 128 && pk.R1p / kTile <= kMaxGt && pk.Kp >= 512;
}

bool decode_stream_fits(const Packed &pk, int64_t M, int num_sms)
{
    if (M < 1 || M > 16 || !decode_stream_shape(pk))
        return false;
    StreamPlan pl;
    return stream_plan(pk, M, pk.r > 0, num_sms, pl);
}

size_t decode_stream_ws_floats(const Packed &pk)
{
    const size_t n_gt = (size_t)pk.R1p / kTile;
    return n_gt * (size_t)(pk.Kp / 256) * kTile * kUStr + (size_t)pk.R1p * kUStr;
}

cudaError_t decode_stream_prepare(const Packed &pk, void **maps)
{
    StreamMaps *m = static_cast<StreamMaps *>(*maps);
    if (!m) {
        m = new (std::nothrow) StreamMaps();
        if (!m)
            return cudaErrorMemoryAllocation;
        *maps = m;
    }
    const int nch = (int)(pk.Kp / 256);
    const uint64_t dims[3] = {32, 64, (uint64_t)(pk.Np / 64) * (uint64_t)nch};
    const uint64_t strides[2] = {128, 8192};
    const uint32_t box[3] = {32, (uint32_t)kTile, 2};
    cudaError_t e = make_map_nd(&m->codes, pk.codes, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, dims, strides, box,
                                CU_TENSOR_MAP_SWIZZLE_128B);
    if (e == cudaSuccess && pk.r > 0) {
        const uint64_t gd[3] = {64, (uint64_t)pk.R1p, (uint64_t)(pk.Kp / 64)};
        const uint64_t gs[2] = {(uint64_t)pk.Kp * 2, 128};
        const uint32_t gb[3] = {64, (uint32_t)kTile, 4};
        e = make_map_nd(&m->g, pk.G, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, gd, gs, gb, CU_TENSOR_MAP_SWIZZLE_128B);
    } else if (e == cudaSuccess) {
        m->g = m->codes;
    }
    return e;
}

void decode_stream_free(void *maps) { delete static_cast<StreamMaps *>(maps); }

cudaError_t launch_decode_stream(const Packed &pk, const void *maps, const void *x, void *y, int64_t M, bool ec,
                                 const DecodeWork &w, int *status, cudaStream_t st, int num_sms)
{
    if (!maps || M < 1 || M > 16)
        return cudaErrorInvalidValue;
    const StreamMaps *m = static_cast<const StreamMaps *>(maps);
    const bool use_ec = ec && pk.r > 0;
    if (use_ec && (!w.ws_stream || !w.cnt_stream))
        return cudaErrorInvalidValue;
    StreamPlan pl;
    if (!stream_plan(pk, M, use_ec, num_sms, pl))
        return cudaErrorInvalidValue;
    // codes as [blocks][64 rows][32 words]: a box is one tile's 16 rows x sc chunks
    CUtensorMap tm_codes;
    {
        const uint64_t dims[3] = {32, 64, (uint64_t)(pk.Np / 64) * (uint64_t)(pk.Kp / 256)};
        const uint64_t strides[2] = {128, 8192};
        const uint32_t box[3] = {32, (uint32_t)kTile, (uint32_t)pl.sc};
        cudaError_t ec_ = make_map_nd(&tm_codes, pk.codes, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, dims, strides, box,
                                      CU_TENSOR_MAP_SWIZZLE_128B);
        if (ec_ != cudaSuccess)
            return ec_;
    }
    const int T = M <= 8 ? 1 : 2;
    // every cluster must be resident at once
    const int active = max_active_clusters(T, pl.CS, pl.smem);
    if (active < 1)
        return cudaErrorInvalidValue;
    if (pl.n_clusters > active) {
        StreamPlan pl2;
        if (!stream_layout(pk, T, pl.CS, active, pl.S, use_ec, pl2))
            return cudaErrorInvalidValue;
        pl = pl2;
    }
    // x as [K/64][M][64] (a rank's slice is one box) when K is a multiple of 64
    CUtensorMap tm_x;
    cudaError_t e = cudaErrorInvalidValue;
    int x3 = 0;
    if (pk.K % 64 == 0 && 4 * pl.cpr <= 256) {
        const uint64_t xd[3] = {64, (uint64_t)M, (uint64_t)(pk.K / 64)};
        const uint64_t xs[2] = {(uint64_t)pk.K * 2, 128};
        const uint32_t xb[3] = {64, (uint32_t)(8 * T), (uint32_t)(4 * pl.cpr)};
        e = make_map_nd(&tm_x, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, xd, xs, xb, CU_TENSOR_MAP_SWIZZLE_128B);
        x3 = e == cudaSuccess ? 1 : 0;
    }
    if (e != cudaSuccess)
        e = make_map(&tm_x, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)pk.K, (uint64_t)M, 64,
                     (uint32_t)(8 * T), CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess)
        return e;
    StreamParams p;
    p.x3 = x3;
    p.Bt = pk.Bt;
    p.s = pk.s;
    p.z = pk.z;
    p.y = static_cast<uint16_t *>(y);
    const size_t gpart_floats = (size_t)(pk.R1p / kTile) * (size_t)(pk.Kp / 256) * kTile * kUStr;
    p.gpart = w.ws_stream;
    p.ufin = w.ws_stream + gpart_floats;
    p.cnt = w.cnt_stream;
    p.status = status;
    p.M = M;
    p.N = pk.N;
    p.n_tiles = (int)(pk.Np / kTile);
    p.CS = pl.CS;
    p.n_clusters = pl.n_clusters;
    p.nch = (int)(pk.Kp / 256);
    p.cpr = pl.cpr;
    p.S = pl.S;
    p.sc = pl.sc;
    p.r = pk.r;
    p.rp = pk.rp;
    p.R1p = pk.R1p;
    p.n_gt = use_ec ? pk.R1p / kTile : 0;
    p.own_max = pl.own_max;
    p.g_slots = pl.g_slots;
    p.btw = pl.btw;
    p.ustr = pl.ustr;
    p.b_g = pk.b_g;
    p.off_x = pl.off_x;
    p.off_red = pl.off_red;
    p.off_recv = pl.off_recv;
    p.off_g = pl.off_g;
    p.off_bt = pl.off_bt;
    p.off_u = pl.off_u;
    p.off_zs = pl.off_zs;
    p.pf = w.pf;
    p.pf_bytes = w.pf_bytes;
    const void *fn = T == 1 ? stream_ptr<1>() : stream_ptr<2>();
    e = raise_smem_limit(fn, pl.smem);
    if (e != cudaSuccess)
        return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(pl.n_clusters * pl.CS));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = pl.CS;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (T == 1)
        return cudaLaunchKernelEx(&cfg, decode_stream_kernel<1>, tm_codes, m->g, tm_x, p);
    return cudaLaunchKernelEx(&cfg, decode_stream_kernel<2>, tm_codes, m->g, tm_x, p);
}

}  // namespace spear
