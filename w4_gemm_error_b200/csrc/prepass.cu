// Per-token gate and Error Compensator down-projection.
//
// SPEAR, "A System for Post-Quantization Error-Adaptive Recovery Enabling
// Efficient Low-Bit LLM Serving", Abstract: the EC is "modulated by
// per-token gates".  This library's reading of that gate and of the EC:
//   logit_t = x[t,:] . w_g + b_g,   g_t = 1 / (1 + exp(-logit_t))
//   u[t,j]  = x[t,:] . A[:,j]       v[t,j] = g_t * u[t,j]   (fp32)
// v is the left operand of the EC up-projection that the GEMM kernels add
// to their accumulators (y += v . B).
//
// Both dot products are one small GEMM, D[j][t] = G[j,:] . x[t,:] with
// G = [w_g; A^T] (R1p rows), run on the tensor cores with mma.sync: G rows on
// the 16-row side, 16 tokens per CTA on the 8-column side, the K range split
// over the CTA's four warps and, when few tokens leave SMs idle, over CTAs.
// Split-K partials are summed in a fixed order in two levels (no floating-
// point atomics, run-to-run identical): the last CTA of each group of eight
// splits to arrive sums the group's partials in split order, and the last
// group to arrive sums the groups' sums in group order, so no CTA waits on
// more than eight loads per element.
#include <algorithm>

#include "async_utils.cuh"
#include "device_utils.cuh"
#include "kernels.h"
#include "tp.h"

namespace spear {
namespace {

constexpr int kTok = 16;  // tokens per CTA (two 8-column MMA tiles)
constexpr int kGroup = 8;     // splits per first-level sum
constexpr int kMaxSplits = 32;
constexpr int kMaxGroups = kMaxSplits / kGroup;

struct PrepassParams {
    const uint16_t *G;
    const uint16_t *x;
    int64_t M, K, Kp;
    int R1p, r, rp;
    float b_g;
    int S;       // CTAs per token tile (split-K)
    int bps;     // 64-wide k blocks per split
    float *v;
    int tf32;
    float *g;
    float *part;          // [tiles][S][tile] split partials, then [tiles][kMaxGroups][tile] group sums
    float *gpart;
    unsigned *counters;   // [tiles] groups summed, then [tiles][kMaxGroups] splits of each group
    unsigned *gcounters;
    unsigned *ready;   // counted (release) once per token tile when its v is written; null for none
    TpPush push;       // PUSH form: where the raw partials go (tensor-parallel shard)
};


// MINB = 7 caps the registers at 72 per thread, so that a CTA fits on an SM
// beside a tcgen05 kernel CTA with 64-token tiles (22 warps of 80 registers,
// about 200 KB of shared memory) at the price of some spills; MINB = 1 is the
// fast form for a prepass that runs alone.  PUSH: the tensor-parallel form,
// which writes the raw partial sums of x.G (no bias, no sigmoid) to every
// rank's slot instead of g and v.
template <int MT, int MINB, bool PUSH>
__global__ void __launch_bounds__(128, MINB) prepass_kernel(PrepassParams p)
{
    pdl_wait();  // x is written by the previous kernel in the stream
    // the next kernel may start now: x is complete (a tcgen05 kernel that starts
    // early reads it without waiting)
    pdl_launch_dependents();
    extern __shared__ float4 smem_f4[];
    float *red = reinterpret_cast<float *>(smem_f4);  // [4][R1p][kTok]
    __shared__ int s_last;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gid = lane >> 2, c = lane & 3;
    const int tile = blockIdx.x / p.S, ks = blockIdx.x - tile * p.S;
    const int64_t t0 = (int64_t)tile * kTok;
    const int nkb = (int)(p.Kp / 64);
    const int kb0 = ks * p.bps, kb1 = min(kb0 + p.bps, nkb);

    float acc[MT][2][4];
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                acc[m][n][i] = 0.f;

    for (int kb = kb0 + warp; kb < kb1; kb += 4) {
        const int64_t k = (int64_t)kb * 64 + 16 * c;
        uint32_t xb[2][8];
#pragma unroll
        for (int n = 0; n < 2; ++n) {
            const int64_t t = t0 + 8 * n + gid;
            uint4 a = make_uint4(0, 0, 0, 0), b = a;
            if (t < p.M && k < p.K) {
                const uint16_t *src = p.x + t * p.K + k;
                a = ld_nc(src);
                if (k + 8 < p.K)
                    b = ld_nc(src + 8);
            }
            xb[n][0] = a.x; xb[n][1] = a.y; xb[n][2] = a.z; xb[n][3] = a.w;
            xb[n][4] = b.x; xb[n][5] = b.y; xb[n][6] = b.z; xb[n][7] = b.w;
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            const uint16_t *g0 = p.G + (int64_t)(16 * m + gid) * p.Kp + k;
            const uint16_t *g1 = g0 + 8 * p.Kp;
            const uint4 a0 = ld_nc(g0), a1 = ld_nc(g0 + 8), h0 = ld_nc(g1), h1 = ld_nc(g1 + 8);
            const uint32_t ga[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const uint32_t ha[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
            // step i covers k = 16c + 4i + {0,1} (first pair) and + {2,3} (second pair)
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int n = 0; n < 2; ++n)
                    mma_bf16_16816(acc[m][n], ga[2 * i], ha[2 * i], ga[2 * i + 1], ha[2 * i + 1],
                                   xb[n][2 * i], xb[n][2 * i + 1]);
        }
    }

    // reduce the four warps' partial tiles through shared memory
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int n = 0; n < 2; ++n) {
            float *base = red + ((size_t)warp * p.R1p) * kTok;
            const int r0 = 16 * m + gid, col = 8 * n + 2 * c;
            base[r0 * kTok + col] = acc[m][n][0];
            base[r0 * kTok + col + 1] = acc[m][n][1];
            base[(r0 + 8) * kTok + col] = acc[m][n][2];
            base[(r0 + 8) * kTok + col + 1] = acc[m][n][3];
        }
    __syncthreads();
    const int tile_elems = p.R1p * kTok;
    for (int e = tid; e < tile_elems; e += 128)
        red[e] = red[e] + red[tile_elems + e] + red[2 * tile_elems + e] + red[3 * tile_elems + e];
    __syncthreads();

    if (p.S > 1) {
        float *mine = p.part + ((size_t)tile * p.S + ks) * tile_elems;
        for (int e = tid; e < tile_elems; e += 128)
            mine[e] = red[e];
        __threadfence();
        __syncthreads();
        const int grp = ks / kGroup, g0 = grp * kGroup, gsize = min(kGroup, p.S - g0);
        const int ngroups = (p.S + kGroup - 1) / kGroup;
        if (tid == 0)
            s_last = (atomicAdd(&p.gcounters[tile * kMaxGroups + grp], 1u) == (unsigned)(gsize - 1));
        __syncthreads();
        if (!s_last)
            return;
        __threadfence();
        // first level: this group's partials in split order, four in flight per
        // round; thread tid takes the elements tid + 128 i (the tile is 16 MT x 16)
        auto sum_in_order = [&](const float *src, int n, float (&sum)[2 * MT]) {
#pragma unroll
            for (int i = 0; i < 2 * MT; ++i)
                sum[i] = 0.f;
            for (int q0 = 0; q0 < n; q0 += 4) {
                float w[4][2 * MT];
#pragma unroll
                for (int q = 0; q < 4; ++q)
#pragma unroll
                    for (int i = 0; i < 2 * MT; ++i)
                        w[q][i] = q0 + q < n ? __ldcg(src + (size_t)(q0 + q) * tile_elems + tid + 128 * i) : 0.f;
#pragma unroll
                for (int q = 0; q < 4; ++q)
#pragma unroll
                    for (int i = 0; i < 2 * MT; ++i)
                        sum[i] += w[q][i];
            }
        };
        float sum[2 * MT];
        sum_in_order(p.part + ((size_t)tile * p.S + g0) * tile_elems, gsize, sum);
        if (tid == 0)
            p.gcounters[tile * kMaxGroups + grp] = 0u;
        if (ngroups > 1) {
            // second level: the groups' sums in group order, by the last group
            float *gdst = p.gpart + ((size_t)tile * kMaxGroups + grp) * tile_elems;
#pragma unroll
            for (int i = 0; i < 2 * MT; ++i)
                gdst[tid + 128 * i] = sum[i];
            __threadfence();
            __syncthreads();
            if (tid == 0)
                s_last = (atomicAdd(&p.counters[tile], 1u) == (unsigned)(ngroups - 1));
            __syncthreads();
            if (!s_last)
                return;
            __threadfence();
            sum_in_order(p.gpart + (size_t)tile * kMaxGroups * tile_elems, ngroups, sum);
            if (tid == 0)
                p.counters[tile] = 0u;
        }
#pragma unroll
        for (int i = 0; i < 2 * MT; ++i)
            red[tid + 128 * i] = sum[i];
        __syncthreads();
    }

    if constexpr (PUSH) {
        // the slots this call overwrites are free once every rank has
        // finished the previous call's reduce
        if (tid < p.push.world) {
            const unsigned e = *reinterpret_cast<const volatile unsigned *>(p.push.epoch);
            if (!tp_wait_count(p.push.done + tid, e, p.push.sys))
                atomicOr(p.push.status, kStatusTimeout);
        }
        __syncthreads();
        // rows of x.G for the tile's tokens, to this rank's slot in every
        // rank's buffer (peer stores), consecutive threads on consecutive j
        for (int e = tid; e < kTok * p.R1p; e += 128) {
            const int tt = e / p.R1p, j = e - tt * p.R1p;
            const int64_t t = t0 + tt;
            if (t >= p.M)
                continue;
            const float val = red[j * kTok + tt];
            for (int q = 0; q < p.push.world; ++q)
                p.push.dst[q][t * p.R1p + j] = val;
        }
        __syncthreads();
        if (tid == 0)
            tp_fence(p.push.sys);   // the CTA's stores (before it through the barrier) reach every rank first
        return;
    }

    // epilogue: gate and v for the tile's tokens (row 0 of the tile is the logit)
    __shared__ float s_gate[kTok];
    if (tid < kTok) {
        const float gt = 1.0f / (1.0f + expf(-(red[tid] + p.b_g)));
        s_gate[tid] = gt;
        if (t0 + tid < p.M)
            p.g[t0 + tid] = gt;
    }
    __syncthreads();
    for (int e = tid; e < kTok * p.rp; e += 128) {
        const int tt = e / p.rp, j = e - tt * p.rp;
        const int64_t t = t0 + tt;
        if (t >= p.M)
            continue;
        const float val = (j < p.r) ? s_gate[tt] * red[(1 + j) * kTok + tt] : 0.f;
        p.v[t * p.rp + j] = p.tf32 ? to_tf32(val) : val;
    }
    if (p.ready) {
        __syncthreads();
        if (tid == 0)
            red_release_gpu_add(p.ready, 1u);   // this tile's v and g are written
    }
}

int pick_splits(int64_t M, int64_t Kp, int num_sms)
{
    const int tiles = (int)((M + kTok - 1) / kTok);
    const int nkb = (int)(Kp / 64);
    int S = std::max(1, (2 * num_sms) / std::max(tiles, 1));
    S = std::min(S, std::max(1, nkb / 4));  // at least one k block per warp
    return std::min(S, kMaxSplits);          // summed in groups of eight
}

using PrepassFn = void (*)(PrepassParams);
template <int MINB, bool PUSH>
PrepassFn prepass_fn_b(int MT)
{
    switch (MT) {
    case 1: return prepass_kernel<1, MINB, PUSH>;
    case 2: return prepass_kernel<2, MINB, PUSH>;
    case 3: return prepass_kernel<3, MINB, PUSH>;
    case 4: return prepass_kernel<4, MINB, PUSH>;
    case 5: return prepass_kernel<5, MINB, PUSH>;
    case 6: return prepass_kernel<6, MINB, PUSH>;
    case 7: return prepass_kernel<7, MINB, PUSH>;
    case 8: return prepass_kernel<8, MINB, PUSH>;
    case 9: return prepass_kernel<9, MINB, PUSH>;
    default: return nullptr;
    }
}
PrepassFn prepass_fn(int MT, bool slim) { return slim ? prepass_fn_b<7, false>(MT) : prepass_fn_b<1, false>(MT); }

}  // namespace

size_t prepass_part_floats(const Packed &pk, int64_t max_M, int num_sms)
{
    size_t worst = 0;
    // the split count shrinks as M grows; check every tile count up to max_M
    // (split partials, then kMaxGroups group sums per tile)
    const int64_t tiles_max = (max_M + kTok - 1) / kTok;
    for (int64_t tiles = 1; tiles <= tiles_max; ++tiles) {
        const int S = pick_splits(tiles * kTok, pk.Kp, num_sms);
        if (S > 1)
            worst = std::max(worst, (size_t)tiles * (S + kMaxGroups) * pk.R1p * kTok);
        else
            break;
    }
    return worst;
}

// One counter per token tile for the groups, then kMaxGroups per tile for the splits.
int prepass_counters(int64_t max_M) { return (int)((max_M + kTok - 1) / kTok) * (1 + kMaxGroups); }

namespace {

// push == nullptr: the gate and v (launch_prepass); otherwise the raw
// partials to the ranks' slots (launch_prepass_partial)
cudaError_t launch_any(const Packed &pk, const void *x, int64_t M, float *v, bool tf32, float *g,
                       const PrepassWork &w, cudaStream_t st, int num_sms, unsigned *ready, bool slim,
                       const TpPush *push)
{
    if (M <= 0 || pk.r == 0)
        return cudaSuccess;
    PrepassParams p = {};
    p.G = pk.G;
    p.x = static_cast<const uint16_t *>(x);
    p.M = M;
    p.K = pk.K;
    p.Kp = pk.Kp;
    p.R1p = pk.R1p;
    p.r = pk.r;
    p.rp = pk.rp;
    p.b_g = pk.b_g;
    p.S = pick_splits(M, pk.Kp, num_sms);
    if (push)
        p.S = std::min(p.S, kGroup);   // one level of sums: the push form is on the critical path
    const int nkb = (int)(pk.Kp / 64);
    p.bps = (nkb + p.S - 1) / p.S;
    p.S = (nkb + p.bps - 1) / p.bps;  // drop empty splits
    p.v = v;
    p.tf32 = tf32 ? 1 : 0;
    p.g = g;
    const int tiles = (int)((M + kTok - 1) / kTok);
    const int tiles_cap = w.n_counters / (1 + kMaxGroups);
    p.part = w.part;
    p.gpart = w.part + (size_t)tiles * p.S * pk.R1p * kTok;
    p.counters = w.counters;
    p.gcounters = w.counters + tiles_cap;
    p.ready = ready;
    if (push)
        p.push = *push;
    if (tiles > tiles_cap || (p.S > 1 && (size_t)tiles * (p.S + kMaxGroups) * pk.R1p * kTok > w.part_floats))
        return cudaErrorInvalidValue;
    PrepassFn fn = push ? prepass_fn_b<1, true>(pk.R1p / 16) : prepass_fn(pk.R1p / 16, slim);
    if (!fn)
        return cudaErrorInvalidValue;
    const size_t smem = (size_t)4 * pk.R1p * kTok * sizeof(float);
    if (smem > 48 * 1024) {
        cudaError_t e = raise_smem_limit(reinterpret_cast<const void *>(fn), smem);
        if (e != cudaSuccess)
            return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(tiles * p.S));
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, fn, p);
}

}  // namespace

cudaError_t launch_prepass(const Packed &pk, const void *x, int64_t M, float *v, bool tf32, float *g,
                           const PrepassWork &w, cudaStream_t st, int num_sms, unsigned *ready, bool slim)
{
    return launch_any(pk, x, M, v, tf32, g, w, st, num_sms, ready, slim, nullptr);
}

cudaError_t launch_prepass_partial(const Packed &pk, const void *x, int64_t M, const PrepassWork &w,
                                   const TpPush &push, cudaStream_t st, int num_sms)
{
    if (push.world < 1 || push.world > kTpMaxWorld || !push.epoch || !push.done || !push.status)
        return cudaErrorInvalidValue;
    return launch_any(pk, x, M, nullptr, false, nullptr, w, st, num_sms, nullptr, false, &push);
}

}  // namespace spear
