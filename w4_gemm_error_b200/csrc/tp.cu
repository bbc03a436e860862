// Row-parallel tensor parallelism of the C ABI (include/spear_w4ec.h): a
// layer split along K over ranks, one GPU and one process per rank.
//
// SPEAR, "A System for Post-Quantization Error-Adaptive Recovery Enabling
// Efficient Low-Bit LLM Serving", Abstract: with the EC in a tensor-parallel
// layer, the input-dependent gate forces the ranks to synchronise (the gate
// needs the complete x.w_g before its sigmoid, and the EC the complete x.A
// before its up-projection); the pages meet it with a peer-reduction kernel
// and a P2P dual write.  This library's form, per call and rank p:
//
//   push     (with the EC) the prepass's PUSH form: x_p.[w_g,p, A_p] in fp32
//            to slot p of every rank's buffer (peer stores), its stores held
//            back (bounded wait) until every rank's done word in rank p's
//            buffer has reached rank p's count of completed calls: nobody
//            still reads rank p's buffers of the previous call;
//   enter    (without the EC; one CTA) the same wait alone;
//   forward  of the shard with the EC off into rank p's partial output; its
//            weight copies start while the push runs (programmatic
//            dependent launch), its writes after the push has ended;
//   signal   raises rank p's ready word in every rank's buffer to the
//            call's count (one fence at the group's scope, then the stores);
//   reduce   waits for every rank's ready word, sums the u slots in rank
//            order and the ranks' partial outputs in rank order (peer loads),
//            adds g . (u . B) once, writes y; its last CTA advances the count
//            of completed calls and raises rank p's done word in every
//            rank's buffer.
//
// Every wait is for words that earlier launches on the other ranks' streams
// raise, bounded by kWaitBudgetCycles.  The counts live on the device, so the
// sequence can be captured in a CUDA graph.  All ranks sum the same slots in
// the same order, so they compute the same gate and the same y.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstddef>
#include <cstring>
#include <new>

#include "async_utils.cuh"
#include "device_utils.cuh"
#include "handle.h"
#include "tp.h"
#include "spear_w4ec.h"

using namespace spear;

static_assert(SPEAR_TP_MAX_WORLD == kTpMaxWorld, "the C header and the library agree on the largest group");

namespace {

constexpr uint32_t kTpMagic = 0x50545053u;  // "SPTP"

// The first 256 bytes of an exchange buffer.  ready and done are written by
// the ranks (entry q by rank q); the rest only by the owner.
struct TpCtrl {
    unsigned ready[kTpMaxWorld];   // rank q has published its partials of call c: c
    unsigned pad0[8];
    unsigned done[kTpMaxWorld];    // rank q has finished reading this buffer for call c: c
    unsigned pad1[8];
    unsigned epoch;                // calls completed by the owner
    unsigned ctas;                 // reduce: CTAs finished in this call
    unsigned pad2[14];
    // checked by the other ranks when they connect
    uint32_t magic, world, rank, R1p;
    int64_t max_M, N;
    int32_t r, pad3;
    uint32_t pad4[6];
};
static_assert(sizeof(TpCtrl) == 256, "control block size");
static_assert(offsetof(TpCtrl, done) == 64 && offsetof(TpCtrl, epoch) == 128 && offsetof(TpCtrl, magic) == 192,
              "control block layout");

constexpr size_t kCtrlBytes = sizeof(TpCtrl);

// Raises this rank's word in every rank's buffer to `e`: one fence at the
// group's scope (everything this thread has written or observed goes first),
// then the stores.
__device__ __forceinline__ void raise_words(unsigned *const *words, int world, unsigned e, int sys)
{
    tp_fence(sys);
    for (int q = 0; q < world; ++q)
        tp_store_relaxed(words[q], e, sys);
}

__global__ void __launch_bounds__(32) tp_enter_kernel(const TpCtrl *ctrl, int world, int sys, int *status)
{
    // the shard's forward may start its weight prefetch now; it waits for
    // this kernel's end before it writes anything
    pdl_launch_dependents();
    pdl_wait();
    const int q = threadIdx.x;
    if (q < world) {
        const unsigned e = *reinterpret_cast<const volatile unsigned *>(&ctrl->epoch);
        if (!tp_wait_count(&ctrl->done[q], e, sys))
            atomicOr(status, kStatusTimeout);
    }
}

// Raises this rank's ready words once the shard's forward (and the push or
// enter kernel before it) has ended.
__global__ void __launch_bounds__(32) tp_signal_kernel(TpPush push)
{
    pdl_wait();   // the shard's forward has written the partial output
    if (threadIdx.x == 0)
        raise_words(push.ready, push.world, *reinterpret_cast<const volatile unsigned *>(push.epoch) + 1u, push.sys);
}

constexpr int kRThreads = 256;   // output channels per CTA (one per thread)
constexpr int kRTok = 16;        // tokens per CTA

struct TpReduceParams {
    const uint16_t *ypart[kTpMaxWorld];   // every rank's partial output [M][N]
    unsigned *done[kTpMaxWorld];          // this rank's done word in every rank's buffer
    TpCtrl *ctrl;                         // this rank's control block
    const float *uslots;                  // this rank's u slots [world][slot_floats]
    int64_t slot_floats;
    const uint16_t *Bt;                   // [N][rp] bf16
    uint16_t *y;                          // [M][N] bf16
    int *status;
    int64_t M, N;
    int world, R1p, rp, ec, sys;
    float b_g;
};

__global__ void __launch_bounds__(kRThreads) tp_reduce_kernel(TpReduceParams p)
{
    extern __shared__ float us[];   // [kRTok][R1p + 16]: the summed u rows (zero beyond R1p)
    __shared__ float s_gate[kRTok];
    __shared__ unsigned s_e;
    const int tid = threadIdx.x;
    const int64_t n = (int64_t)blockIdx.x * kRThreads + tid;
    // the first 32 entries of row n of B^T (weights: no wait needed)
    uint4 b0[4];
#pragma unroll
    for (int c = 0; c < 4; ++c)
        b0[c] = (p.ec && n < p.N && 8 * c < p.rp) ? ld_nc(p.Bt + n * p.rp + 8 * c) : make_uint4(0, 0, 0, 0);
    pdl_launch_dependents();
    pdl_wait();   // this rank's signal kernel and the kernels before it are complete
    if (tid == 0)
        s_e = *reinterpret_cast<const volatile unsigned *>(&p.ctrl->epoch) + 1u;
    __syncthreads();
    const unsigned e = s_e;
    if (tid < p.world && !tp_wait_count(&p.ctrl->ready[tid], e, p.sys))
        atomicOr(p.status, kStatusTimeout);
    __syncthreads();

    const int64_t t0 = (int64_t)blockIdx.y * kRTok;
    const int ntok = (int)min((int64_t)kRTok, p.M - t0);
    const int SV = p.R1p + 16;
    if (p.ec) {
        // the rows of the tokens present (the loops below read no others)
        for (int i = tid; i < ntok * SV; i += kRThreads) {
            const int tt = i / SV, j = i - tt * SV;
            float u = 0.f;
            if (j < p.R1p)
                for (int q = 0; q < p.world; ++q)
                    u += __ldcg(p.uslots + q * p.slot_floats + (t0 + tt) * p.R1p + j);
            us[i] = u;
        }
        __syncthreads();
        if (tid < ntok)
            s_gate[tid] = 1.0f / (1.0f + expf(-(us[tid * SV] + p.b_g)));
        __syncthreads();
    }
    if (n < p.N) {
        // rank 0's partial output first, so that its loads are in flight
        // during the EC; the other ranks' follow in rank order
        float sum[kRTok];
        {
            const unsigned short *src = reinterpret_cast<const unsigned short *>(p.ypart[0]) + t0 * p.N + n;
#pragma unroll
            for (int i = 0; i < kRTok; ++i)
                sum[i] = i < ntok ? __uint_as_float((uint32_t)__ldcg(src + (int64_t)i * p.N) << 16) : 0.f;
        }
        float corr[kRTok];
#pragma unroll
        for (int i = 0; i < kRTok; ++i)
            corr[i] = 0.f;
        if (p.ec) {
            // 32 entries of the row per round, their four loads in flight together
            for (int j0 = 0; j0 < p.rp; j0 += 32) {
                uint4 bv[4];
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    bv[c] = j0 == 0 ? b0[c]
                                    : (j0 + 8 * c < p.rp ? ld_nc(p.Bt + n * p.rp + j0 + 8 * c) : make_uint4(0, 0, 0, 0));
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    if (j0 + 8 * c >= p.rp)
                        break;
                    const float bj[8] = {bf16_lo(bv[c].x), bf16_hi(bv[c].x), bf16_lo(bv[c].y), bf16_hi(bv[c].y),
                                         bf16_lo(bv[c].z), bf16_hi(bv[c].z), bf16_lo(bv[c].w), bf16_hi(bv[c].w)};
#pragma unroll
                    for (int i = 0; i < kRTok; ++i) {
                        if (i < ntok) {
                            const float *ur = us + i * SV + 1 + j0 + 8 * c;   // u_1 .. u_r follow the logit
#pragma unroll
                            for (int q = 0; q < 8; ++q)
                                corr[i] += ur[q] * bj[q];
                        }
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < kRTok; ++i)
                if (i < ntok)
                    corr[i] *= s_gate[i];
        }
        for (int q = 1; q < p.world; ++q) {
            const unsigned short *src = reinterpret_cast<const unsigned short *>(p.ypart[q]) + t0 * p.N + n;
#pragma unroll
            for (int i = 0; i < kRTok; ++i)
                if (i < ntok)
                    sum[i] += __uint_as_float((uint32_t)__ldcg(src + (int64_t)i * p.N) << 16);
        }
#pragma unroll
        for (int i = 0; i < kRTok; ++i)
            if (i < ntok)
                p.y[(t0 + i) * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(sum[i] + corr[i]));
    }
    // this CTA has finished reading the ranks' buffers; the last one to finish
    // advances the count of calls and tells every rank
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const unsigned total = gridDim.x * gridDim.y;
        if (atomicAdd(&p.ctrl->ctas, 1u) == total - 1) {
            __threadfence();
            p.ctrl->ctas = 0u;
            *reinterpret_cast<volatile unsigned *>(&p.ctrl->epoch) = e;
            raise_words(p.done, p.world, e, p.sys);
        }
    }
}

cudaError_t launch_pdl(const void *fn, dim3 grid, dim3 block, size_t smem, cudaStream_t st, void **args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelExC(&cfg, fn, args);
}

}  // namespace

struct spear_w4ec_tp {
    int device = 0;
    spear_w4ec *shard = nullptr;
    int rank = 0, world = 1;
    int64_t max_M = 0, N = 0;
    int R1p = 0, r = 0;
    void *buf = nullptr;
    size_t bytes = 0, u_off = 0, y_off = 0;
    int64_t slot_floats = 0;
    void *peer[kTpMaxWorld] = {};
    bool opened[kTpMaxWorld] = {};
    bool connected = false;
    int sys = 1;    // ordering scope of the group's words: 0 when every buffer is on this device in this process
};

namespace {

TpCtrl *ctrl_of(void *base) { return static_cast<TpCtrl *>(base); }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Reads every rank's control block and checks it against this rank's view.
int check_peers(spear_w4ec_tp *t)
{
    for (int q = 0; q < t->world; ++q) {
        TpCtrl c;
        cudaError_t e = cudaMemcpy(&c, t->peer[q], sizeof(c), cudaMemcpyDefault);
        if (e != cudaSuccess)
            return status_of(e);
        if (c.magic != kTpMagic || c.world != (uint32_t)t->world || c.rank != (uint32_t)q || c.max_M != t->max_M ||
            c.N != t->N || c.r != t->r || c.R1p != (uint32_t)t->R1p)
            return SPEAR_ERR_INVALID;
    }
    return SPEAR_OK;
}

void close_peers(spear_w4ec_tp *t)
{
    for (int q = 0; q < kTpMaxWorld; ++q) {
        if (t->opened[q])
            cudaIpcCloseMemHandle(t->peer[q]);
        t->opened[q] = false;
        t->peer[q] = nullptr;
    }
    t->connected = false;
}

int run_partial(spear_w4ec_tp *t, const void *x, int64_t M, uint32_t flags, cudaStream_t st)
{
    spear_w4ec *h = t->shard;
    const bool ec = !(flags & SPEAR_EC_OFF) && t->r > 0;
    TpCtrl *mine = ctrl_of(t->buf);
    TpPush push = {};
    push.world = t->world;
    push.sys = t->sys;
    push.epoch = &mine->epoch;
    push.done = mine->done;
    push.status = h->status;
    for (int q = 0; q < t->world; ++q) {
        push.dst[q] = reinterpret_cast<float *>(static_cast<char *>(t->peer[q]) + t->u_off) +
                      (size_t)t->rank * t->slot_floats;
        push.ready[q] = &ctrl_of(t->peer[q])->ready[t->rank];
    }
    cudaError_t e;
    if (ec) {
        e = launch_prepass_partial(h->pk, x, M, h->pre, push, st, h->num_sms);
    } else {
        int world = t->world, sys = t->sys;
        int *status = h->status;
        const TpCtrl *cm = mine;
        void *enter_args[] = {&cm, &world, &sys, &status};
        e = launch_pdl(reinterpret_cast<const void *>(tp_enter_kernel), dim3(1), dim3(32), 0, st, enter_args);
    }
    if (e != cudaSuccess)
        return status_of(e);
    void *ypart = static_cast<char *>(t->buf) + t->y_off;
    const uint32_t path = flags & (SPEAR_FORCE_DECODE | SPEAR_FORCE_TC);
    const int rc = forward_checked(h, x, ypart, M, path | SPEAR_EC_OFF, st);
    if (rc != SPEAR_OK)
        return rc;
    void *sig_args[] = {&push};
    e = launch_pdl(reinterpret_cast<const void *>(tp_signal_kernel), dim3(1), dim3(32), 0, st, sig_args);
    return e == cudaSuccess ? SPEAR_OK : status_of(e);
}

int run_reduce(spear_w4ec_tp *t, void *y, int64_t M, uint32_t flags, cudaStream_t st)
{
    spear_w4ec *h = t->shard;
    TpReduceParams p = {};
    for (int q = 0; q < t->world; ++q) {
        p.ypart[q] = reinterpret_cast<const uint16_t *>(static_cast<const char *>(t->peer[q]) + t->y_off);
        p.done[q] = &ctrl_of(t->peer[q])->done[t->rank];
    }
    p.ctrl = ctrl_of(t->buf);
    p.uslots = reinterpret_cast<const float *>(static_cast<const char *>(t->buf) + t->u_off);
    p.slot_floats = t->slot_floats;
    p.Bt = h->pk.Bt;
    p.y = static_cast<uint16_t *>(y);
    p.status = h->status;
    p.M = M;
    p.N = t->N;
    p.world = t->world;
    p.R1p = t->R1p;
    p.rp = h->pk.rp;
    p.ec = (!(flags & SPEAR_EC_OFF) && t->r > 0) ? 1 : 0;
    p.sys = t->sys;
    p.b_g = h->pk.b_g;
    const dim3 grid((unsigned)((t->N + kRThreads - 1) / kRThreads), (unsigned)((M + kRTok - 1) / kRTok));
    const size_t smem = (size_t)kRTok * (t->R1p + 16) * sizeof(float);
    void *args[] = {&p};
    const cudaError_t e = launch_pdl(reinterpret_cast<const void *>(tp_reduce_kernel), grid, dim3(kRThreads), smem,
                                     st, args);
    return e == cudaSuccess ? SPEAR_OK : status_of(e);
}

int check_call(spear_w4ec_tp *t, int64_t M)
{
    if (!t || M < 0)
        return SPEAR_ERR_INVALID;
    if (M > t->max_M)
        return SPEAR_ERR_INVALID;
    if (!t->connected)
        return SPEAR_ERR_STATE;
    return SPEAR_OK;
}

}  // namespace

extern "C" {

int spear_w4ec_tp_create(spear_w4ec_tp **out, spear_w4ec *shard, int32_t rank, int32_t world, int64_t max_M)
{
    if (!out)
        return SPEAR_ERR_INVALID;
    *out = nullptr;
    if (!shard || world < 1 || world > kTpMaxWorld || rank < 0 || rank >= world || max_M < 1 ||
        max_M > shard->max_M)
        return SPEAR_ERR_INVALID;
    if (!shard->packed)
        return SPEAR_ERR_STATE;
    DeviceGuard guard(shard->device);
    if (!guard.ok())
        return SPEAR_ERR_CUDA;
    spear_w4ec_tp *t = new (std::nothrow) spear_w4ec_tp();
    if (!t)
        return SPEAR_ERR_NOMEM;
    t->device = shard->device;
    t->shard = shard;
    t->rank = rank;
    t->world = world;
    t->max_M = max_M;
    t->N = shard->pk.N;
    t->r = shard->pk.r;
    t->R1p = shard->pk.r > 0 ? shard->pk.R1p : 16;
    t->slot_floats = max_M * t->R1p;
    t->u_off = kCtrlBytes;
    t->y_off = (t->u_off + (size_t)world * t->slot_floats * sizeof(float) + 255) / 256 * 256;
    t->bytes = t->y_off + (size_t)max_M * (size_t)t->N * 2;
    cudaError_t e = cudaMalloc(&t->buf, t->bytes);
    if (e == cudaSuccess)
        e = cudaMemset(t->buf, 0, t->bytes);
    if (e == cudaSuccess) {
        TpCtrl c;
        std::memset(&c, 0, sizeof(c));
        c.magic = kTpMagic;
        c.world = (uint32_t)world;
        c.rank = (uint32_t)rank;
        c.R1p = (uint32_t)t->R1p;
        c.max_M = max_M;
        c.N = t->N;
        c.r = t->r;
        e = cudaMemcpy(t->buf, &c, sizeof(c), cudaMemcpyHostToDevice);
    }
    if (e != cudaSuccess) {
        cudaFree(t->buf);
        delete t;
        return status_of(e);
    }
    *out = t;
    return SPEAR_OK;
}

int spear_w4ec_tp_buffer(const spear_w4ec_tp *t, void **base, size_t *bytes, size_t *u_offset, size_t *y_offset)
{
    if (!t)
        return SPEAR_ERR_INVALID;
    if (base)
        *base = t->buf;
    if (bytes)
        *bytes = t->bytes;
    if (u_offset)
        *u_offset = t->u_off;
    if (y_offset)
        *y_offset = t->y_off;
    return SPEAR_OK;
}

int spear_w4ec_tp_ipc_handle(const spear_w4ec_tp *t, void *handle)
{
    if (!t || !handle)
        return SPEAR_ERR_INVALID;
    static_assert(sizeof(cudaIpcMemHandle_t) == SPEAR_TP_IPC_HANDLE_BYTES, "IPC handle size");
    DeviceGuard guard(t->device);
    if (!guard.ok())
        return SPEAR_ERR_CUDA;
    cudaIpcMemHandle_t hd;
    const cudaError_t e = cudaIpcGetMemHandle(&hd, t->buf);
    if (e != cudaSuccess)
        return status_of(e);
    std::memcpy(handle, &hd, sizeof(hd));
    return SPEAR_OK;
}

int spear_w4ec_tp_connect_ipc(spear_w4ec_tp *t, const void *handles)
{
    if (!t || !handles)
        return SPEAR_ERR_INVALID;
    DeviceGuard guard(t->device);
    if (!guard.ok())
        return SPEAR_ERR_CUDA;
    close_peers(t);
    const unsigned char *hb = static_cast<const unsigned char *>(handles);
    // this rank's own entry must be its own handle, and no other entry may be
    // (a process cannot open its own handle)
    cudaIpcMemHandle_t own;
    cudaError_t e = cudaIpcGetMemHandle(&own, t->buf);
    if (e != cudaSuccess)
        return status_of(e);
    for (int q = 0; q < t->world; ++q) {
        const bool same = std::memcmp(hb + (size_t)q * SPEAR_TP_IPC_HANDLE_BYTES, &own, sizeof(own)) == 0;
        if (same != (q == t->rank))
            return SPEAR_ERR_INVALID;
    }
    for (int q = 0; q < t->world; ++q) {
        if (q == t->rank) {
            t->peer[q] = t->buf;
            continue;
        }
        cudaIpcMemHandle_t hd;
        std::memcpy(&hd, hb + (size_t)q * SPEAR_TP_IPC_HANDLE_BYTES, sizeof(hd));
        void *p = nullptr;
        e = cudaIpcOpenMemHandle(&p, hd, cudaIpcMemLazyEnablePeerAccess);
        if (e != cudaSuccess) {
            cudaGetLastError();
            close_peers(t);
            if (e == cudaErrorPeerAccessUnsupported)
                return SPEAR_ERR_UNSUPPORTED;
            return (e == cudaErrorInvalidValue || e == cudaErrorInvalidResourceHandle) ? SPEAR_ERR_INVALID
                                                                                       : status_of(e);
        }
        t->peer[q] = p;
        t->opened[q] = true;
    }
    const int rc = check_peers(t);
    if (rc != SPEAR_OK) {
        close_peers(t);
        return rc;
    }
    t->sys = t->world > 1 ? 1 : 0;   // the other ranks are other processes
    t->connected = true;
    return SPEAR_OK;
}

int spear_w4ec_tp_connect(spear_w4ec_tp *t, void *const *buffers)
{
    if (!t || !buffers)
        return SPEAR_ERR_INVALID;
    if (buffers[t->rank] != t->buf)
        return SPEAR_ERR_INVALID;
    DeviceGuard guard(t->device);
    if (!guard.ok())
        return SPEAR_ERR_CUDA;
    close_peers(t);
    int sys = 0;
    for (int q = 0; q < t->world; ++q) {
        if (!buffers[q])
            return SPEAR_ERR_INVALID;
        cudaPointerAttributes a;
        if (cudaPointerGetAttributes(&a, buffers[q]) != cudaSuccess || a.type != cudaMemoryTypeDevice) {
            cudaGetLastError();
            return SPEAR_ERR_INVALID;
        }
        if (a.device != t->device) {
            sys = 1;
            int can = 0;
            if (cudaDeviceCanAccessPeer(&can, t->device, a.device) != cudaSuccess || !can)
                return SPEAR_ERR_UNSUPPORTED;
            const cudaError_t e = cudaDeviceEnablePeerAccess(a.device, 0);
            if (e == cudaErrorPeerAccessAlreadyEnabled)
                cudaGetLastError();
            else if (e != cudaSuccess)
                return status_of(e);
        }
        t->peer[q] = buffers[q];
    }
    const int rc = check_peers(t);
    if (rc != SPEAR_OK) {
        close_peers(t);
        return rc;
    }
    t->sys = sys;
    t->connected = true;
    return SPEAR_OK;
}

int spear_w4ec_tp_partial(spear_w4ec_tp *t, const void *x, int64_t M, uint32_t flags, void *stream)
{
    int rc = check_call(t, M);
    if (rc != SPEAR_OK || M == 0)
        return rc;
    if (!x || !aligned16(x))
        return SPEAR_ERR_INVALID;
    DeviceGuard guard(t->device);
    if (!guard.ok())
        return SPEAR_ERR_CUDA;
    return run_partial(t, x, M, flags, static_cast<cudaStream_t>(stream));
}

int spear_w4ec_tp_reduce(spear_w4ec_tp *t, void *y, int64_t M, uint32_t flags, void *stream)
{
    int rc = check_call(t, M);
    if (rc != SPEAR_OK || M == 0)
        return rc;
    if (!y || !aligned16(y))
        return SPEAR_ERR_INVALID;
    DeviceGuard guard(t->device);
    if (!guard.ok())
        return SPEAR_ERR_CUDA;
    return run_reduce(t, y, M, flags, static_cast<cudaStream_t>(stream));
}

int spear_w4ec_tp_forward(spear_w4ec_tp *t, const void *x, void *y, int64_t M, uint32_t flags, void *stream)
{
    int rc = check_call(t, M);
    if (rc != SPEAR_OK || M == 0)
        return rc;
    if (!x || !y || !aligned16(x) || !aligned16(y))
        return SPEAR_ERR_INVALID;
    DeviceGuard guard(t->device);
    if (!guard.ok())
        return SPEAR_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    rc = run_partial(t, x, M, flags, st);
    return rc == SPEAR_OK ? run_reduce(t, y, M, flags, st) : rc;
}

int spear_w4ec_tp_destroy(spear_w4ec_tp *t)
{
    if (!t)
        return SPEAR_OK;
    DeviceGuard guard(t->device);
    cudaDeviceSynchronize();
    close_peers(t);
    cudaFree(t->buf);
    delete t;
    return SPEAR_OK;
}

}  // extern "C"
