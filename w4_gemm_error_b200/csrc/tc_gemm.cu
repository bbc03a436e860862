// W4 GEMM with the Error Compensator as a second accumulation, on the
// Blackwell tensor cores (tcgen05, accumulators in tensor memory, operands
// staged by TMA).
//
// SPEAR, "A System for Post-Quantization Error-Adaptive Recovery Enabling
// Efficient Low-Bit LLM Serving", Abstract: the post-EC computation is fused
// into the low-bit GEMM.  Here the EC is literally part of the same
// accumulation: after the K loop of the main product the tile runs r/8 more
// MMA k-steps, in tf32 (fp32 range, 2^-11 rounding: the EC operands v and
// B^T/s need both), with v = g * (x . A) (from the prepass) against B^T/s,
// into the same TMEM accumulator, so
//     D[n, t] = sum_k (q[n,k] - z[n]) x[t,k] + sum_j (B[j,n] / s[n]) v[t,j]
// and the epilogue writes y[t, n] = bf16(s[n] * D[n, t]).
//
// Layout of one CTA (persistent, one per SM, 22 warps):
//   warp 0      TMA producer: x tile (BN tokens x 64 k, 128B-swizzled) and
//               the int4 code tile (128 rows x 64 k) per stage; for the EC
//               stages the B^T/s tile and the v tile (32 fp32 j each) instead.
//   warp 1      TMEM allocator and the single MMA-issuing thread:
//               tcgen05.mma.cta_group::1.kind::f16, M = 128 weight rows,
//               N = BN tokens (32, 64, 128 or 256: the narrowest that holds
//               the batch), K = 16 per instruction (swap-AB: weights on the
//               M side so one dequantised tile serves BN tokens).
//   warps 2-17  dequantisers, two groups of eight warps taking alternate
//               stages (a stage's wait, code load, conversion, stores and
//               fence form a latency chain; two groups keep two stages in
//               conversion at once): thread (i, h) of a group owns half h of
//               weight row i of the tile (32 k) and writes the exact integers
//               (q - z) as bf16 into the 128B-swizzled K-major A tile of the
//               stage (the layout the MMA descriptor names).
//   warps 18-21 epilogue: tcgen05.ld of the finished accumulator (each warp
//               its 32-lane quarter), times the channel scale s[n], bf16
//               rounding, stores of y[t, n].
// The accumulator holds sum_k x (q - z) exactly up to fp32 summation, so the
// EC stages use B^T / s[n] (prepared at pack time) and one multiplication by
// s[n] in the epilogue scales both terms.
// 4 to 8 stages (about 200 KB) in shared memory; two BN-column accumulators
// in TMEM so the epilogue of one tile overlaps the main loop of the next.
// Every mbarrier wait is bounded (about a second of SM clock cycles); a wait
// that runs out sets the handle's status word and the kernel winds down.
#include <algorithm>
#include <new>

#include "async_utils.cuh"
#include "tc_gemm.h"
#include "tensor_map.h"

namespace spear {
namespace {

constexpr int BM = 128;                       // weight rows per tile (TMEM lanes)
constexpr int BK = 64;                        // k per stage: one 128-byte swizzle atom of bf16
constexpr int A_BYTES = BM * BK * 2;          // 16 KB dequantised weights (or B^T on EC stages)
constexpr int C_BYTES = BM * BK / 2;          // 4 KB int4 codes
constexpr int THREADS = 704;   // 22 warps: TMA, MMA, 2 x 8 dequantisers, 4 epilogue

// Token tile BN (the MMA N: 32, 64, 128 or 256) and what depends on it: the
// activation tile of a stage (BN x 64 bf16, or v on EC stages), the ring depth
// (more stages for narrower tiles, within about 210 KB) and two accumulators of
// BN columns in TMEM.
__host__ __device__ constexpr int tc_b_bytes(int BN) { return BN * BK * 2; }
__host__ __device__ constexpr int tc_stage_bytes(int BN) { return A_BYTES + tc_b_bytes(BN) + C_BYTES; }
__host__ __device__ constexpr int tc_stages(int BN) { return BN >= 256 ? 4 : (BN >= 128 ? 6 : (BN >= 64 ? 7 : 8)); }
__host__ __device__ constexpr int tc_smem_bytes(int BN) { return tc_stages(BN) * tc_stage_bytes(BN) + 1024; }

struct TcParams {
    int64_t M, N;
    int kchunks;       // Kp / 256: tiled code blocks per 64-row block
    int n_main, n_ec, rp;
    int n_ttiles, n_tiles;
    // split K: work unit u = tile * ksplit + ks runs main stages [ks * sps, min((ks + 1) * sps, n_main)),
    // the last split also the EC stages; with ksplit > 1 each unit writes an fp32 partial tile and the
    // last unit of a tile to finish sums them in split order
    int ksplit, sps, n_units;
    float *part;           // [n_tiles][ksplit][BN][128] fp32
    unsigned *counters;    // [n_tiles] finished units of each tile
    const float *s;
    const uint8_t *z;
    uint16_t *y;
    int *status;
    // early start (fused EC after a prepass): the kernel does not wait for its
    // predecessor (the prepass, which starts it only once x is complete) before
    // the main stages; its EC stages wait until v_ready[0] reaches v_expected
    // (the prepass's release increments), and each CTA waits for the prepass to
    // finish before it leaves.  The last CTA resets v_ready[0..1].  Null: the
    // kernel waits for its predecessor first, as usual.
    unsigned *v_ready;
    unsigned v_expected;
};

struct Maps {
    CUtensorMap codes;
    CUtensorMap bt;
    CUtensorMap g;   // G = [w_g; A^T] [R1p][Kp] bf16, boxes of 64 x R1p, 128B swizzle
};

// ---------------------------------------------------------------- EC down-projection for many tokens
//
// D[t, j] = x[t, :] . G[j, :] for a 128-token tile, G = [w_g; A^T] (R1p <= 256
// rows): tcgen05.mma with the tokens on the M = 128 side (TMEM lanes) and the
// R1p rows of G on N, so each epilogue thread owns one token's whole row of D
// and forms g_t = sigmoid(D[t,0] + b_g) and v[t, j] = g_t * D[t, 1+j] alone.
// Warp 0: TMA producer; warp 1: TMEM allocator and MMA issuer; warps 2-5:
// epilogue.  One tile per CTA, 4 stages of x (16 KB) and G (R1p x 128 B).

constexpr int PP_STAGES = 4;
constexpr int PP_THREADS = 192;

struct PrepassTcParams {
    int64_t M;
    int n_k;            // 64-wide k stages
    int R1p, r, rp;
    float b_g;
    float *v;           // [M][rp] fp32
    int tf32;           // round v to tf32
    float *g;           // [M]
    int *status;
    unsigned *ready;    // counted (release) once this CTA's v is written; null for none
};

__global__ void __launch_bounds__(PP_THREADS, 1)
tc_prepass_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_g,
                  PrepassTcParams p)
{
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t bars[2 * PP_STAGES + 2];
    __shared__ uint32_t tmem_base_slot;
    __shared__ volatile int abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t base = (smem_addr(smem_raw) + 1023u) & ~1023u;
    const uint32_t x_bytes = 128 * 128, g_bytes = (uint32_t)p.R1p * 128;
    const uint32_t stage_bytes = x_bytes + ((g_bytes + 1023u) & ~1023u);
    const uint32_t full0 = smem_addr(&bars[0]), empty0 = smem_addr(&bars[PP_STAGES]);
    const uint32_t done = smem_addr(&bars[2 * PP_STAGES]), drain = smem_addr(&bars[2 * PP_STAGES + 1]);
    const int t0 = blockIdx.x * 128;
    uint32_t tmem_cols = 32;
    while (tmem_cols < (uint32_t)p.R1p)
        tmem_cols <<= 1;

    if (tid == 0) {
        abort_flag = 0;
        for (int s = 0; s < PP_STAGES; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 1);
        }
        mbar_init(done, 1);
        mbar_init(drain, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_addr(&tmem_base_slot)),
                     "r"(tmem_cols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_slot;

    if (warp == 0) {
        if (lane == 0) {
            pdl_wait();  // x comes from an earlier kernel in the stream
            // let the next kernel start only now that x is complete (it may read x
            // without waiting) and this CTA holds its tensor memory (a dependent
            // CTA that cannot allocate then waits for a kernel that needs nothing
            // from it)
            pdl_launch_dependents();
            int issued = 0;
            for (int kb = 0; kb < p.n_k; ++kb, ++issued) {
                const uint32_t slot = kb % PP_STAGES, phase = (kb / PP_STAGES) & 1;
                if (!mbar_wait(empty0 + 8 * slot, phase ^ 1, &abort_flag, p.status))
                    break;
                const uint32_t sb = base + slot * stage_bytes;
                mbar_expect_tx(full0 + 8 * slot, x_bytes + g_bytes);
                tma_load_2d(sb, &tm_x, kb * 64, t0, full0 + 8 * slot);
                tma_load_2d(sb + x_bytes, &tm_g, kb * 64, 0, full0 + 8 * slot);
            }
            // (the MMA thread waited for every stage issued unless a wait gave up)
            if (abort_flag)
                for (int k = 0; k < PP_STAGES && k < issued; ++k) {
                    const int kb = issued - 1 - k;
                    mbar_wait_final(full0 + 8 * (kb % PP_STAGES), (kb / PP_STAGES) & 1);
                }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(p.R1p >> 3) << 17) |
                                   ((uint32_t)(128 >> 4) << 24);
            bool ok = true;
            for (int kb = 0; kb < p.n_k && ok; ++kb) {
                const uint32_t slot = kb % PP_STAGES, phase = (kb / PP_STAGES) & 1;
                if (!mbar_wait(full0 + 8 * slot, phase, &abort_flag, p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sb = base + slot * stage_bytes;
                const uint64_t a_desc = smem_desc_sw128(sb), b_desc = smem_desc_sw128(sb + x_bytes);
                for (int k = 0; k < 4; ++k)
                    mma_bf16(tmem, a_desc + 2 * k, b_desc + 2 * k, idesc, (kb > 0 || k > 0) ? 1u : 0u);
                mma_commit(empty0 + 8 * slot);
            }
            if (ok)
                mma_commit(done);
            // every MMA of this thread is complete before TMEM is released
            mma_commit(drain);
            mbar_wait_final(drain, 0);
        }
    } else {
        // epilogue: warp (2..5) & 3 owns TMEM lanes 32q..32q+31 = tokens
        const int q = warp & 3;
        const int64_t t = t0 + 32 * q + lane;
        if (mbar_wait(done, 0, &abort_flag, p.status)) {
            tc_fence_after();
            float gt = 0.f;
            for (int c = 0; c < p.R1p; c += 32) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + c, r);
                if (c == 0)
                    gt = 1.0f / (1.0f + expf(-(__uint_as_float(r[0]) + p.b_g)));
                if (t < p.M) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int j = c + i - 1;   // column c+i holds x . A[:, c+i-1]
                        if (j >= 0 && j < p.rp) {
                            const float val = j < p.r ? gt * __uint_as_float(r[i]) : 0.f;
                            p.v[t * p.rp + j] = p.tf32 ? to_tf32(val) : val;
                        }
                    }
                }
            }
            // v columns past the last column of D (only when r + 1 fills R1p exactly) are zero
            if (t < p.M)
                for (int j = p.R1p - 1; j < p.rp; ++j)
                    p.v[t * p.rp + j] = 0.f;
            if (t < p.M)
                p.g[t] = gt;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (tid == 0 && p.ready)
        red_release_gpu_add(p.ready, 1u);   // this CTA's v and g are written
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(tmem_cols) : "memory");
    }
}

// ---------------------------------------------------------------- the kernel

template <int BN>
__global__ void __launch_bounds__(THREADS, 1)
tc_w4ec_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_codes,
               const __grid_constant__ CUtensorMap tm_bt, const __grid_constant__ CUtensorMap tm_v, TcParams p)
{
    constexpr int STAGES = tc_stages(BN);
    constexpr int B_BYTES = tc_b_bytes(BN);
    constexpr int STAGE_BYTES = tc_stage_bytes(BN);
    constexpr int TMEM_COLS = 2 * BN;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t bars[3 * STAGES + 5];
    __shared__ uint32_t tmem_base_slot;
    __shared__ volatile int abort_flag;
    __shared__ volatile int s_last;   // split K: this unit finished its tile

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t base = (smem_addr(smem_raw) + 1023u) & ~1023u;
    uint8_t *const base_ptr = smem_raw + (base - smem_addr(smem_raw));
    const uint32_t full0 = smem_addr(&bars[0]);
    const uint32_t aready0 = smem_addr(&bars[STAGES]);
    const uint32_t empty0 = smem_addr(&bars[2 * STAGES]);
    const uint32_t tfull0 = smem_addr(&bars[3 * STAGES]);
    const uint32_t tempty0 = smem_addr(&bars[3 * STAGES + 2]);
    const uint32_t drain = smem_addr(&bars[3 * STAGES + 4]);

    if (tid == 0) {
        abort_flag = 0;
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(aready0 + 8 * s, 256);
            mbar_init(empty0 + 8 * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull0 + 8 * b, 1);
            mbar_init(tempty0 + 8 * b, 128);
        }
        mbar_init(drain, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_addr(&tmem_base_slot)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_slot;
    // let the next kernel start only now that this CTA holds its tensor memory
    // (see the prepass kernel)
    pdl_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            if (!p.v_ready)
                pdl_wait();  // x and v come from earlier kernels in the stream
            bool v_seen = p.v_ready == nullptr;
            uint32_t g = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
                const int tile = u / p.ksplit, ks = u - tile * p.ksplit;
                const int t0 = (tile % p.n_ttiles) * BN, n0 = (tile / p.n_ttiles) * BM;
                const int lo = ks * p.sps, nm = min(lo + p.sps, p.n_main) - lo;
                const int nst = nm + (ks == p.ksplit - 1 ? p.n_ec : 0);
                for (int i = 0; i < nst; ++i, ++g) {
                    const int st = i < nm ? lo + i : p.n_main + (i - nm);
                    const uint32_t slot = g % STAGES, phase = (g / STAGES) & 1;
                    if (!mbar_wait(empty0 + 8 * slot, phase ^ 1, &abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    const uint32_t sb = base + slot * STAGE_BYTES;
                    const uint32_t full = full0 + 8 * slot;
                    if (st < p.n_main) {
                        mbar_expect_tx(full, B_BYTES + C_BYTES);
                        tma_load_2d(sb + A_BYTES, &tm_x, st * BK, t0, full);
                        const int blk = (n0 / 64) * p.kchunks + st / 4;
                        tma_load_4d(sb + A_BYTES + B_BYTES, &tm_codes, 0, st & 3, 0, blk, full);
                        tma_load_4d(sb + A_BYTES + B_BYTES + C_BYTES / 2, &tm_codes, 0, st & 3, 0, blk + p.kchunks,
                                    full);
                    } else {
                        if (!v_seen) {
                            // the prepass has written v for every token (bounded wait);
                            // the copies below then read it through the async proxy
                            const long long w0 = clock64();
                            while (ld_acquire_gpu(p.v_ready) < p.v_expected) {
                                if (abort_flag || clock64() - w0 > kWaitBudgetCycles) {
                                    abort_flag = 1;
                                    atomicOr(p.status, kStatusTimeout);
                                    ok = false;
                                    break;
                                }
                                __nanosleep(64);
                            }
                            if (!ok)
                                break;
                            asm volatile("fence.proxy.async;" ::: "memory");
                            v_seen = true;
                        }
                        const int e = st - p.n_main;   // 32 tf32 values of j per EC stage
                        mbar_expect_tx(full, A_BYTES + B_BYTES);
                        tma_load_2d(sb, &tm_bt, e * 32, n0, full);
                        tma_load_2d(sb + A_BYTES, &tm_v, e * 32, t0, full);
                    }
                }
            }
            // do not leave while copies this CTA issued may still land (the
            // consumers waited for every stage unless a wait gave up)
            if (abort_flag)
                for (uint32_t k = 0; k < STAGES && k < g; ++k) {
                    const uint32_t gg = g - 1 - k, slot = gg % STAGES, phase = (gg / STAGES) & 1;
                    mbar_wait_final(full0 + 8 * slot, phase);
                }
            // early start: this grid completes only after its predecessor (the
            // prepass), so that the next kernel's wait still covers both
            if (p.v_ready)
                pdl_wait();
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = (1u << 4)                    // D: f32
                                   | (1u << 7) | (1u << 10)     // A, B: bf16
                                   | ((uint32_t)(BN >> 3) << 17)
                                   | ((uint32_t)(BM >> 4) << 24);
            const uint32_t idesc_tf32 = (1u << 4)               // D: f32
                                        | (2u << 7) | (2u << 10)  // A, B: tf32
                                        | ((uint32_t)(BN >> 3) << 17)
                                        | ((uint32_t)(BM >> 4) << 24);
            uint32_t g = 0;
            int lt = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x, ++lt) {
                const uint32_t buf = lt & 1;
                if (!mbar_wait(tempty0 + 8 * buf, ((lt >> 1) & 1) ^ 1, &abort_flag, p.status))
                    break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + buf * BN;
                const int ks = u % p.ksplit;
                const int lo = ks * p.sps, nm = min(lo + p.sps, p.n_main) - lo;
                const int nst = nm + (ks == p.ksplit - 1 ? p.n_ec : 0);
                for (int i = 0; i < nst; ++i, ++g) {
                    const int st = i < nm ? lo + i : p.n_main + (i - nm);
                    const uint32_t slot = g % STAGES, phase = (g / STAGES) & 1;
                    // one wait per stage: the dequantisers arrive on aready only after
                    // they have waited for the stage's copies (full), so its completion
                    // orders this thread after the copies too (each mbarrier test of
                    // this thread costs about as much as issuing the stage's MMAs: per-
                    // stage stamps put the thread at 0.48 us per 64-k stage with two)
                    if (!mbar_wait(aready0 + 8 * slot, phase, &abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sb = base + slot * STAGE_BYTES;
                    const uint64_t a_desc = smem_desc_sw128(sb), b_desc = smem_desc_sw128(sb + A_BYTES);
                    if (st < p.n_main) {
                        for (int k = 0; k < BK / 16; ++k)
                            mma_bf16(d_tmem, a_desc + 2 * k, b_desc + 2 * k, idesc, (i > 0 || k > 0) ? 1u : 0u);
                    } else {
                        // EC: 32 tf32 values of j per 128-byte row, 8 per instruction
                        const int rem = p.rp - (st - p.n_main) * 32;
                        const int ksteps = (rem < 32 ? rem : 32) / 8;
                        for (int k = 0; k < ksteps; ++k)
                            mma_tf32(d_tmem, a_desc + 2 * k, b_desc + 2 * k, idesc_tf32, 1u);
                    }
                    mma_commit(empty0 + 8 * slot);
                }
                if (ok)
                    mma_commit(tfull0 + 8 * buf);
            }
            // every MMA this thread issued is complete before TMEM is released
            mma_commit(drain);
            mbar_wait_final(drain, 0);
        }
    } else if (warp < 18) {
        // ------------------------------------------------ dequantisers: group `grp` takes the stages
        // g with g % 2 == grp; its thread (i, h) = half h of weight row i
        const int dq = tid - 64;
        const uint32_t grp = (uint32_t)(dq >> 8);
        const int i = dq & 127, half = (dq >> 7) & 1;
        uint32_t g = 0;
        for (int u = blockIdx.x; u < p.n_units; u += gridDim.x) {
            const int tile = u / p.ksplit, ks = u - tile * p.ksplit;
            const int lo = ks * p.sps, nm = min(lo + p.sps, p.n_main) - lo;
            const int nst = nm + (ks == p.ksplit - 1 ? p.n_ec : 0);
            const int n = (tile / p.n_ttiles) * BM + i;
            // the epilogue scales a row whose s is 0 by 1 (its B^T/e operand needs a
            // nonzero e): such a row dequantises to 0, whatever its codes
            const bool live = p.s[n] != 0.0f;
            const uint32_t zb = __bfloat16_as_ushort(__float2bfloat16_rn(-(float)(128u + p.z[n])));
            const uint32_t negz = live ? (zb | (zb << 16)) : 0u;
            const uint32_t mulz = live ? 0x3F803F80u : 0u;
            bool ok = true;
            for (int ii = 0; ii < nst; ++ii, ++g) {
                if ((g & 1u) != grp)
                    continue;
                const int st = ii < nm ? lo + ii : p.n_main + (ii - nm);
                const uint32_t slot = g % STAGES, phase = (g / STAGES) & 1;
                if (!mbar_wait(full0 + 8 * slot, phase, &abort_flag, p.status)) {
                    ok = false;
                    break;
                }
                if (st < p.n_main) {
                    uint8_t *sb = base_ptr + slot * STAGE_BYTES;
                    // code row i: 32 bytes (64 k), its two 16-byte halves swapped in rows
                    // with bit 2 set (32-byte TMA swizzle, conflict-free reads)
                    const uint4 w0 = *reinterpret_cast<const uint4 *>(sb + A_BYTES + B_BYTES + i * 32 +
                                                                      ((half ^ ((i >> 2) & 1)) << 4));
                    const uint32_t words[4] = {w0.x, w0.y, w0.z, w0.w};
                    uint8_t *arow = sb + i * 128;
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const int j = 4 * half + jj;
                        // codes k = 8j + {0..7}: nibbles (m, m + 4) hold k = 2m, 2m + 1
                        uint4 o;
                        o.x = dequant_pair_mul(words[jj], mulz, negz);         // k 0, 1
                        o.y = dequant_pair_mul(words[jj] >> 4, mulz, negz);    // k 2, 3
                        o.z = dequant_pair_mul(words[jj] >> 8, mulz, negz);    // k 4, 5
                        o.w = dequant_pair_mul(words[jj] >> 12, mulz, negz);   // k 6, 7
                        *reinterpret_cast<uint4 *>(arow + ((j ^ (i & 7)) << 4)) = o;
                    }
                    fence_proxy_async_smem();
                }
                mbar_arrive(aready0 + 8 * slot);
            }
            if (!ok)
                break;
        }
    } else {
        // ------------------------------------------------ epilogue: warp quarter q owns TMEM lanes 32q..32q+31
        const int q = warp & 3;
        const int row = 32 * q + lane;
        int lt = 0;
        for (int u = blockIdx.x; u < p.n_units; u += gridDim.x, ++lt) {
            const int tile = u / p.ksplit, ks = u - tile * p.ksplit;
            const uint32_t buf = lt & 1;
            if (!mbar_wait(tfull0 + 8 * buf, (lt >> 1) & 1, &abort_flag, p.status))
                break;
            tc_fence_after();
            const int64_t t0 = (int64_t)(tile % p.n_ttiles) * BN;
            const int64_t n = (int64_t)(tile / p.n_ttiles) * BM + row;
            const float sn = p.s[n];
            const float e_n = sn != 0.0f ? sn : 1.0f;   // the EC operand was divided by it
            if (p.ksplit == 1) {
#pragma unroll 1
                for (int c = 0; c < BN / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(32 * q) << 16) + buf * BN + 32 * c, r);
                    if (n < p.N) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int64_t t = t0 + 32 * c + j;
                            if (t < p.M)
                                p.y[t * p.N + n] =
                                    __bfloat16_as_ushort(__float2bfloat16_rn(e_n * __uint_as_float(r[j])));
                        }
                    }
                }
                tc_fence_before();
                mbar_arrive(tempty0 + 8 * buf);
                continue;
            }
            // ---- split K: this unit's fp32 partial, token-major so that the 128 rows of
            // a token are contiguous; the last unit of the tile to finish sums the
            // partials in split order
            float *tp = p.part + (size_t)tile * p.ksplit * BN * BM;   // [ksplit][BN][128]
            const int jn = (int)min((int64_t)BN, p.M - t0);             // tokens of the tile
#pragma unroll 1
            for (int c = 0; c < BN / 32 && 32 * c < jn; ++c) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(32 * q) << 16) + buf * BN + 32 * c, r);
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (32 * c + j < jn)
                        tp[((size_t)ks * BN + 32 * c + j) * BM + row] = __uint_as_float(r[j]);
            }
            tc_fence_before();
            mbar_arrive(tempty0 + 8 * buf);
            __threadfence();
            asm volatile("bar.sync 1, 128;" ::: "memory");   // the four epilogue warps
            if (q == 0 && lane == 0)
                s_last = atomicAdd(&p.counters[tile], 1u) == (unsigned)(p.ksplit - 1) ? 1 : 0;
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (s_last) {
                __threadfence();
                // eight tokens at a time, so that eight loads per part are in flight
#pragma unroll 1
                for (int j0 = 0; j0 < jn; j0 += 8) {
                    float v[8];
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj)
                        v[jj] = 0.f;
                    for (int k2 = 0; k2 < p.ksplit; ++k2) {
                        float w[8];
#pragma unroll
                        for (int jj = 0; jj < 8; ++jj)
                            w[jj] = j0 + jj < jn ? __ldcg(tp + ((size_t)k2 * BN + j0 + jj) * BM + row) : 0.f;
#pragma unroll
                        for (int jj = 0; jj < 8; ++jj)
                            v[jj] += w[jj];
                    }
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj)
                        if (j0 + jj < jn && n < p.N)
                            p.y[(t0 + j0 + jj) * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(e_n * v[jj]));
                }
                if (q == 0 && lane == 0)
                    p.counters[tile] = 0u;   // for the next forward
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");   // s_last is read before it is rewritten
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                     : "memory");
    }
    if (tid == 0 && p.v_ready && atomicAdd(p.v_ready + 1, 1u) == gridDim.x - 1) {
        // every CTA is past its wait for v and the prepass has finished: reset
        p.v_ready[0] = 0u;
        p.v_ready[1] = 0u;
    }
}

}  // namespace

bool tc_available(const Packed &) { return tensor_maps_available(); }

// Split K for narrow layers: up to 128 tokens, when the 128-row tiles fill at
// most half of the SMs, K is split into as many parts as keep one unit per SM
// (at most 8).  The workspace holds the fp32 partials of every tile at 128
// tokens (part_floats) and one counter per tile.
static int max_ksplit(const Packed &pk, int num_sms)
{
    const int tiles = (int)(pk.Np / BM);
    if (2 * tiles > num_sms)
        return 1;
    return std::min(8, num_sms / tiles);
}

cudaError_t tc_alloc(const Packed &pk, int64_t, int num_sms, TcWork &w)
{
    w.maps = new (std::nothrow) Maps();
    if (!w.maps)
        return cudaErrorMemoryAllocation;
    const int ks = max_ksplit(pk, num_sms);
    if (ks < 2)
        return cudaSuccess;
    w.n_counters = (int)(pk.Np / BM);
    w.part_floats = (size_t)ks * (size_t)pk.Np * 128;
    cudaError_t e = cudaMalloc(&w.part, w.part_floats * sizeof(float));
    if (e == cudaSuccess)
        e = cudaMalloc(&w.counters, (size_t)w.n_counters * sizeof(unsigned));
    if (e == cudaSuccess)
        e = cudaMemset(w.counters, 0, (size_t)w.n_counters * sizeof(unsigned));
    return e;
}

void tc_free(TcWork &w)
{
    delete static_cast<Maps *>(w.maps);
    w.maps = nullptr;
    cudaFree(w.part);
    cudaFree(w.counters);
    w.part = nullptr;
    w.counters = nullptr;
    w.part_floats = 0;
    w.n_counters = 0;
}

cudaError_t tc_prepare(const Packed &pk, TcWork &w)
{
    Maps *m = static_cast<Maps *>(w.maps);
    if (!m)
        return cudaErrorInvalidValue;
    // tiled codes viewed as [blocks][64 rows][4 sub-chunks][8 words]: a box is the 32 bytes
    // (64 k) of one sub-chunk of 64 rows; two boxes (row blocks) make the 128-row stage
    const uint64_t dims[4] = {8, 4, 64, (uint64_t)(pk.Np / 64) * (uint64_t)(pk.Kp / 256)};
    const uint64_t strides[3] = {32, 128, 8192};
    const uint32_t box[4] = {8, 1, 64, 1};
    cudaError_t e = make_map_nd(&m->codes, pk.codes, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, dims, strides, box,
                                CU_TENSOR_MAP_SWIZZLE_32B);
    if (e == cudaSuccess && pk.r > 0)
        e = make_map(&m->g, pk.G, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)pk.Kp, (uint64_t)pk.R1p, 64,
                     (uint32_t)pk.R1p, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e == cudaSuccess && pk.r > 0)
        e = make_map(&m->bt, pk.Bts, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, (uint64_t)pk.rp, (uint64_t)pk.Np, 32, BM,
                     CU_TENSOR_MAP_SWIZZLE_128B);
    return e;
}

cudaError_t launch_tc(const Packed &pk, const void *x, void *y, int64_t M, const float *v, bool ec,
                      const TcWork &w, int *status, bool zero_wait_budget, cudaStream_t st, int num_sms,
                      unsigned *v_ready, unsigned v_expected)
{
    if (M <= 0)
        return cudaSuccess;
    const Maps *m = static_cast<const Maps *>(w.maps);
    if (!m)
        return cudaErrorInvalidValue;
    if (zero_wait_budget) {
        // injected fault: report what a wait that ran out reports, launch nothing
        const int bits = kStatusTimeout;
        return cudaMemcpyAsync(status, &bits, sizeof(int), cudaMemcpyHostToDevice, st);
    }
    // token tile: the narrowest of 32, 64, 128, 256 that holds M (one tile row of tokens
    // up to 256), so that small batches do not run 256-wide MMAs on zero rows
    const int BN = M <= 32 ? 32 : (M <= 64 ? 64 : (M <= 128 ? 128 : 256));
    CUtensorMap tm_x, tm_v;
    cudaError_t e = make_map(&tm_x, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)pk.K, (uint64_t)M, BK,
                             (uint32_t)BN, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess)
        return e;
    const bool use_ec = ec && pk.r > 0;
    if (use_ec) {
        e = make_map(&tm_v, v, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, (uint64_t)pk.rp, (uint64_t)M, 32, (uint32_t)BN,
                     CU_TENSOR_MAP_SWIZZLE_128B);
        if (e != cudaSuccess)
            return e;
    } else {
        tm_v = tm_x;  // unused
    }
    TcParams p;
    p.M = M;
    p.N = pk.N;
    p.kchunks = (int)(pk.Kp / 256);
    p.n_main = (int)(pk.Kp / BK);
    p.n_ec = use_ec ? (pk.rp + 31) / 32 : 0;   // 32 tf32 values per 128-byte row
    p.rp = pk.rp;
    p.n_ttiles = (int)((M + BN - 1) / BN);
    p.n_tiles = p.n_ttiles * (int)(pk.Np / BM);
    // split K (see max_ksplit) with at least 8 stages per part
    int ks = 1;
    if (w.part && M <= 128 && p.n_tiles == w.n_counters)
        ks = std::max(1, std::min(max_ksplit(pk, num_sms), p.n_main / 8));
    p.sps = (p.n_main + ks - 1) / ks;
    p.ksplit = (p.n_main + p.sps - 1) / p.sps;   // no empty part
    p.n_units = p.n_tiles * p.ksplit;
    p.part = w.part;
    p.counters = w.counters;
    p.s = pk.s;
    p.z = pk.z;
    p.y = static_cast<uint16_t *>(y);
    p.status = status;
    p.v_ready = use_ec ? v_ready : nullptr;
    p.v_expected = v_expected;

    const void *fn = BN == 32 ? reinterpret_cast<const void *>(tc_w4ec_kernel<32>)
                   : BN == 64 ? reinterpret_cast<const void *>(tc_w4ec_kernel<64>)
                   : BN == 128 ? reinterpret_cast<const void *>(tc_w4ec_kernel<128>)
                               : reinterpret_cast<const void *>(tc_w4ec_kernel<256>);
    const int smem = tc_smem_bytes(BN);
    e = raise_smem_limit(fn, smem);
    if (e != cudaSuccess)
        return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(p.n_units < num_sms ? p.n_units : num_sms));
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const CUtensorMap &bt = use_ec ? m->bt : m->codes;
    switch (BN) {
    case 32: return cudaLaunchKernelEx(&cfg, tc_w4ec_kernel<32>, tm_x, m->codes, bt, tm_v, p);
    case 64: return cudaLaunchKernelEx(&cfg, tc_w4ec_kernel<64>, tm_x, m->codes, bt, tm_v, p);
    case 128: return cudaLaunchKernelEx(&cfg, tc_w4ec_kernel<128>, tm_x, m->codes, bt, tm_v, p);
    default: return cudaLaunchKernelEx(&cfg, tc_w4ec_kernel<256>, tm_x, m->codes, bt, tm_v, p);
    }
}

}  // namespace spear

namespace spear {

bool tc_prepass_supported(const Packed &pk) { return pk.r > 0 && pk.R1p <= 256 && tensor_maps_available(); }

cudaError_t launch_tc_prepass(const Packed &pk, const void *x, int64_t M, float *v, bool tf32, float *g,
                              const TcWork &w, int *status, cudaStream_t st, unsigned *ready)
{
    if (M <= 0)
        return cudaSuccess;
    const Maps *m = static_cast<const Maps *>(w.maps);
    if (!m || !tc_prepass_supported(pk))
        return cudaErrorInvalidValue;
    CUtensorMap tm_x;
    cudaError_t e = make_map(&tm_x, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)pk.K, (uint64_t)M, 64, 128,
                             CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess)
        return e;
    PrepassTcParams p;
    p.M = M;
    p.n_k = (int)(pk.Kp / 64);
    p.R1p = pk.R1p;
    p.r = pk.r;
    p.rp = pk.rp;
    p.b_g = pk.b_g;
    p.v = v;
    p.tf32 = tf32 ? 1 : 0;
    p.g = g;
    p.status = status;
    p.ready = ready;
    const uint32_t stage = 128 * 128 + (((uint32_t)pk.R1p * 128 + 1023u) & ~1023u);
    const size_t smem = (size_t)PP_STAGES * stage + 1024;
    e = raise_smem_limit(reinterpret_cast<const void *>(tc_prepass_kernel), smem);
    if (e != cudaSuccess)
        return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((M + 127) / 128));
    cfg.blockDim = dim3(PP_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, tc_prepass_kernel, tm_x, m->g, p);
}

}  // namespace spear
