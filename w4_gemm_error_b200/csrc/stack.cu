// Layer stack of the C ABI (include/spear_w4ec.h): a fixed sequence of packed
// W4 + EC layers run on one stream, with the EC of each op switched on or off
// by a caller-given placement.
//
// SPEAR, "A System for Post-Quantization Error-Adaptive Recovery Enabling
// Efficient Low-Bit LLM Serving", Abstract: Error Compensators sit only at
// the most error-sensitive layers.  Which layers those are is an input here;
// an op whose placement is off runs its layer as the plain W4 GEMM.
#include <cuda_runtime.h>

#include <algorithm>
#include <new>
#include <vector>

#include "handle.h"
#include "tensor_map.h"
#include "spear_w4ec.h"

using namespace spear;

struct spear_w4ec_stack {
    int device = 0;
    int64_t max_M = 0;
    std::vector<spear_w4ec_stack_op> ops;
    std::vector<void *> bufs;   // index 2.. : intermediates; 0 and 1 are the caller's x and y
    int64_t in_width = 0;       // K of the ops reading buffer 0
    int64_t out_width = 0;      // N of the last op
    void *x_stage = nullptr;    // staging of the host-buffer call
    void *y_stage = nullptr;
    // the persistent decode kernel's plan (stack_decode.cu), when every op fits it
    bool persist = false;
    int num_sms = 0;
    bool fault_launch = false, fault_timeout = false;
    spear::StackOpDev *p_ops = nullptr;    // device [n_ops]
    CUtensorMap *p_maps = nullptr;         // device [n_ops][2]
    unsigned *p_ws = nullptr;              // device: [2 n_ops] counters, then the u accumulators
    size_t p_ws_bytes = 0;
};

namespace {

constexpr int32_t kMaxOps = 4096;

void free_stack(spear_w4ec_stack *s)
{
    for (void *b : s->bufs)
        cudaFree(b);
    cudaFree(s->x_stage);
    cudaFree(s->y_stage);
    cudaFree(s->p_ops);
    cudaFree(s->p_maps);
    cudaFree(s->p_ws);
}

// The persistent kernel's plan: per op its operands, buffers, the op it must
// wait for (the latest earlier op that writes what it reads, or reads or
// writes what it writes), where its u comes from, and where the round-robin
// deal of its items starts.  Leaves s->persist false (and allocates nothing)
// when some op does not fit the kernel.
cudaError_t plan_persistent(spear_w4ec_stack *s)
{
    const int n = (int)s->ops.size();
    s->num_sms = s->ops[0].layer->num_sms;
    for (const spear_w4ec_stack_op &op : s->ops)
        if (!stack_decode_layer_ok(op.layer->pk))
            return cudaSuccess;
    if (!tensor_maps_available() || !stack_decode_fits(s->num_sms))
        return cudaSuccess;
    std::vector<StackOpDev> dev(n);
    std::vector<CUtensorMap> maps(2 * (size_t)n);
    auto ec_of = [&](int l) { return s->ops[l].ec && s->ops[l].layer->pk.r > 0; };
    int64_t base = 0, u_floats = 0;
    for (int l = 0; l < n; ++l) {
        const spear_w4ec_stack_op &op = s->ops[l];
        const Packed &pk = op.layer->pk;
        StackOpDev &d = dev[l];
        d = StackOpDev{};
        d.s = pk.s;
        d.z = pk.z;
        d.Bt = pk.Bt;
        d.xbuf = op.in == 0 ? nullptr : static_cast<const uint16_t *>(s->bufs[op.in]);
        d.ybuf = op.out == 1 ? nullptr : static_cast<uint16_t *>(s->bufs[op.out]);
        d.status = op.layer->status;
        d.K = (int)pk.K;
        d.N = (int)pk.N;
        d.nch = (int)(pk.Kp / 256);
        d.rp = pk.rp;
        d.R1p = pk.R1p;
        d.b_g = pk.b_g;
        d.ec = ec_of(l) ? 1 : 0;
        d.wait_op = -1;
        for (int j = l - 1; j >= 0 && d.wait_op < 0; --j) {
            const spear_w4ec_stack_op &o = s->ops[j];
            if (o.out == op.in || o.in == op.out || o.out == op.out)
                d.wait_op = j;
        }
        const bool chained = l > 0 && s->ops[l - 1].out == op.in;
        d.u_mode = !d.ec ? 0 : (chained ? 2 : 1);
        if (l + 1 < n && ec_of(l + 1) && s->ops[l + 1].in == op.out) {
            const Packed &nx = s->ops[l + 1].layer->pk;
            d.fuse_next = 1;
            d.Gnext = nx.G;
            d.R1p_next = nx.R1p;
            d.Kp_next = (int)nx.Kp;
        }
        d.n_g = d.u_mode == 1 ? pk.R1p / 16 * d.nch : 0;
        d.n_tiles = (int)((pk.N + 15) / 16);
        d.base = (int)(base % s->num_sms);
        base += d.n_g + d.n_tiles;
        if (d.ec) {
            d.u_off = (int)u_floats;
            u_floats += (int64_t)pk.R1p * 16;
        }
        cudaError_t e = stack_decode_maps(pk, &maps[2 * l], &maps[2 * l + 1]);
        if (e != cudaSuccess)
            return e;
    }
    s->p_ws_bytes = (size_t)2 * n * sizeof(unsigned) + (size_t)u_floats * sizeof(float);
    s->p_ws_bytes = (s->p_ws_bytes + 15) / 16 * 16;
    cudaError_t e = cudaMalloc(&s->p_ops, sizeof(StackOpDev) * n);
    if (e == cudaSuccess)
        e = cudaMalloc(&s->p_maps, sizeof(CUtensorMap) * 2 * (size_t)n);
    if (e == cudaSuccess)
        e = cudaMalloc(&s->p_ws, s->p_ws_bytes);
    if (e == cudaSuccess)
        e = cudaMemcpy(s->p_ops, dev.data(), sizeof(StackOpDev) * n, cudaMemcpyHostToDevice);
    if (e == cudaSuccess)
        e = cudaMemcpy(s->p_maps, maps.data(), sizeof(CUtensorMap) * 2 * (size_t)n, cudaMemcpyHostToDevice);
    if (e != cudaSuccess)
        return e;
    for (const spear_w4ec_stack_op &op : s->ops) {
        s->fault_launch = s->fault_launch || op.layer->fault_launch;
        s->fault_timeout = s->fault_timeout || op.layer->fault_timeout;
    }
    s->persist = true;
    return cudaSuccess;
}

constexpr uint32_t kPathFlags = SPEAR_FORCE_FUSED | SPEAR_FORCE_SPLIT | SPEAR_FORCE_DECODE | SPEAR_FORCE_TC;

int run_persistent(spear_w4ec_stack *s, const void *x, void *y, int64_t M, uint32_t flags, cudaStream_t st)
{
    if (!s->persist || M > kStackMaxTokens || (flags & kPathFlags))
        return SPEAR_ERR_UNSUPPORTED;
    if (s->fault_launch)
        return SPEAR_ERR_CUDA;
    unsigned *done = s->p_ws;
    float *uacc = reinterpret_cast<float *>(s->p_ws + 2 * s->ops.size());
    const cudaError_t e = launch_stack_decode(s->p_ops, s->p_maps, (int)s->ops.size(), x, y, M,
                                              !(flags & SPEAR_EC_OFF), done, uacc, s->p_ws_bytes, s->fault_timeout,
                                              st, s->num_sms);
    return e == cudaSuccess ? SPEAR_OK : status_of(e);
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int run_ops(spear_w4ec_stack *s, const void *x, void *y, int64_t M, uint32_t flags, cudaStream_t st)
{
    if (flags & SPEAR_STACK_PERSISTENT)
        return run_persistent(s, x, y, M, flags & ~(uint32_t)SPEAR_STACK_PERSISTENT, st);
    for (const spear_w4ec_stack_op &op : s->ops) {
        const void *in = op.in == 0 ? x : s->bufs[op.in];
        void *out = op.out == 1 ? y : s->bufs[op.out];
        const uint32_t f = flags | (op.ec ? 0u : (uint32_t)SPEAR_EC_OFF);
        const int rc = forward_checked(op.layer, in, out, M, f, st);
        if (rc != SPEAR_OK)
            return rc;
    }
    return SPEAR_OK;
}

}  // namespace

extern "C" {

int spear_w4ec_stack_create(spear_w4ec_stack **out, const spear_w4ec_stack_op *ops, int32_t n_ops,
                            int64_t max_M)
{
    if (!out)
        return SPEAR_ERR_INVALID;
    *out = nullptr;
    if (!ops || n_ops < 1 || n_ops > kMaxOps || max_M < 1)
        return SPEAR_ERR_INVALID;
    const int32_t n_bufs = n_ops + 2;
    std::vector<int64_t> width(n_bufs, 0), cap(n_bufs, 0);
    int64_t in_width = 0;
    const int device = ops[0].layer ? ops[0].layer->device : -1;
    for (int32_t i = 0; i < n_ops; ++i) {
        const spear_w4ec_stack_op &op = ops[i];
        if (!op.layer || op.layer->device != device || op.layer->max_M < max_M)
            return SPEAR_ERR_INVALID;
        if (op.ec != 0 && op.ec != 1)
            return SPEAR_ERR_INVALID;
        if (op.in < 0 || op.in == 1 || op.in >= n_bufs || op.out < 1 || op.out >= n_bufs || op.in == op.out)
            return SPEAR_ERR_INVALID;
        if ((op.out == 1) != (i == n_ops - 1))
            return SPEAR_ERR_INVALID;   // only the last op writes the output
        const int64_t K = op.layer->pk.K, N = op.layer->pk.N;
        if (op.in == 0) {
            if (in_width && in_width != K)
                return SPEAR_ERR_INVALID;
            in_width = K;
        } else if (width[op.in] != K) {
            return SPEAR_ERR_INVALID;   // not written yet (0), or written with another width
        }
        width[op.out] = N;
        cap[op.out] = std::max(cap[op.out], N);
    }
    if (!in_width)
        return SPEAR_ERR_INVALID;       // no op reads the input
    for (int32_t i = 0; i < n_ops; ++i)
        if (!ops[i].layer->packed)
            return SPEAR_ERR_STATE;

    DeviceGuard guard(device);
    if (!guard.ok())
        return SPEAR_ERR_CUDA;
    spear_w4ec_stack *s = new (std::nothrow) spear_w4ec_stack();
    if (!s)
        return SPEAR_ERR_NOMEM;
    s->device = device;
    s->max_M = max_M;
    s->ops.assign(ops, ops + n_ops);
    s->in_width = in_width;
    s->out_width = ops[n_ops - 1].layer->pk.N;
    s->bufs.assign(n_bufs, nullptr);
    cudaError_t e = cudaSuccess;
    for (int32_t b = 2; b < n_bufs && e == cudaSuccess; ++b)
        if (cap[b])
            e = cudaMalloc(&s->bufs[b], (size_t)max_M * (size_t)cap[b] * 2);
    if (e == cudaSuccess)
        e = cudaMalloc(&s->x_stage, (size_t)max_M * (size_t)in_width * 2);
    if (e == cudaSuccess)
        e = cudaMalloc(&s->y_stage, (size_t)max_M * (size_t)s->out_width * 2);
    if (e == cudaSuccess)
        e = plan_persistent(s);
    if (e != cudaSuccess) {
        free_stack(s);
        delete s;
        return status_of(e);
    }
    // each layer names the one that runs after it (the last names the first)
    for (int32_t i = 0; i < n_ops; ++i) {
        const int rc = spear_w4ec_set_next(ops[i].layer, ops[(i + 1) % n_ops].layer);
        if (rc != SPEAR_OK) {
            free_stack(s);
            delete s;
            return rc;
        }
    }
    *out = s;
    return SPEAR_OK;
}

int spear_w4ec_stack_forward(spear_w4ec_stack *s, const void *x, void *y, int64_t M, uint32_t flags,
                             void *stream)
{
    if (!s || M < 0)
        return SPEAR_ERR_INVALID;
    if (M == 0)
        return SPEAR_OK;
    if (M > s->max_M || !x || !y || !aligned16(x) || !aligned16(y))
        return SPEAR_ERR_INVALID;
    DeviceGuard guard(s->device);
    if (!guard.ok())
        return SPEAR_ERR_CUDA;
    return run_ops(s, x, y, M, flags, static_cast<cudaStream_t>(stream));
}

int spear_w4ec_stack_forward_host(spear_w4ec_stack *s, const void *x_host, void *y_host, int64_t M,
                                  uint32_t flags, void *stream)
{
    if (!s || M < 0)
        return SPEAR_ERR_INVALID;
    if (M == 0)
        return SPEAR_OK;
    if (M > s->max_M || !x_host || !y_host)
        return SPEAR_ERR_INVALID;
    DeviceGuard guard(s->device);
    if (!guard.ok())
        return SPEAR_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(s->x_stage, x_host, (size_t)M * (size_t)s->in_width * 2,
                                    cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess)
        return status_of(e);
    const int rc = run_ops(s, s->x_stage, s->y_stage, M, flags, st);
    if (rc != SPEAR_OK)
        return rc;
    e = cudaMemcpyAsync(y_host, s->y_stage, (size_t)M * (size_t)s->out_width * 2, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(st);
    return status_of(e);
}

int spear_w4ec_stack_buffer(const spear_w4ec_stack *s, int32_t index, void **ptr)
{
    if (!s || !ptr || index < 2 || index >= (int32_t)s->bufs.size() || !s->bufs[index])
        return SPEAR_ERR_INVALID;
    *ptr = s->bufs[index];
    return SPEAR_OK;
}

int spear_w4ec_stack_destroy(spear_w4ec_stack *s)
{
    if (!s)
        return SPEAR_OK;
    DeviceGuard guard(s->device);
    cudaDeviceSynchronize();
    free_stack(s);
    delete s;
    return SPEAR_OK;
}

}  // extern "C"
