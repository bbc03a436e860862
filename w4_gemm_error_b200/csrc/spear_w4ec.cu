// C ABI of the W4 + per-token-gated low-rank Error Compensator linear layer
// (declared in include/spear_w4ec.h): handle life cycle, argument checks,
// workspace, the adaptive fused/split dispatch and the kernel sequence of a
// forward pass.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "spear_w4ec.h"
#include "device_utils.cuh"
#include "handle.h"
#include "kernels.h"
#include "tc_gemm.h"

using namespace spear;

namespace {


const char *env_fault()
{
    const char *f = std::getenv("SPEAR_FAULT");
    return f ? f : "";
}

int64_t round_up(int64_t a, int64_t b) { return (a + b - 1) / b * b; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <class T>
cudaError_t alloc_zero(T **p, size_t count)
{
    *p = nullptr;
    if (count == 0)
        return cudaSuccess;
    cudaError_t e = cudaMalloc(reinterpret_cast<void **>(p), count * sizeof(T));
    if (e != cudaSuccess)
        return e;
    return cudaMemset(*p, 0, count * sizeof(T));
}

void free_all(spear_w4ec *h)
{
    cudaFree(h->pk.codes);
    cudaFree(h->pk.s);
    cudaFree(h->pk.z);
    cudaFree(h->pk.G);
    cudaFree(h->pk.Bt);
    cudaFree(h->pk.Bts);
    cudaFree(h->v);
    cudaFree(h->gbuf);
    cudaFree(h->pre.part);
    cudaFree(h->pre.counters);
    cudaFree(h->dec.ws_u);
    cudaFree(h->dec.flags);
    cudaFree(h->dec.ws_stream);
    cudaFree(h->dec.cnt_stream);
    decode_free(h->dec);
    tc_free(h->tc);
    cudaFree(h->status);
    cudaFree(h->vready);
    cudaFree(h->x_stage);
    cudaFree(h->y_stage);
}

int from_cuda(cudaError_t e)
{
    if (e == cudaSuccess)
        return SPEAR_OK;
    if (e == cudaErrorMemoryAllocation)
        return SPEAR_ERR_NOMEM;
    return SPEAR_ERR_CUDA;
}

bool tc_supported(const spear_w4ec *h) { return tc_available(h->pk); }

// Kernel family and EC placement for M tokens: an explicit request, the tuned
// table entry, or the default (the split-K decode kernel for a few tokens,
// the tcgen05 tile kernel above, the EC fused in both).
// Untuned path: the decode kernel up to 32 tokens; beyond, the tcgen05
// kernel (which splits K on layers whose 128-row tiles fill at most half of
// the SMs).
uint32_t default_path(const spear_w4ec *h, int64_t M)
{
    const bool dec = decode_supported(h->pk, h->num_sms);
    if (!tc_supported(h) || (dec && M <= kDecodeMaxTokens))
        return SPEAR_FORCE_DECODE;
    return SPEAR_FORCE_TC;
}

uint32_t resolve(const spear_w4ec *h, int64_t M, uint32_t flags)
{
    uint32_t path = flags & (SPEAR_FORCE_DECODE | SPEAR_FORCE_TC);
    uint32_t mode = flags & (SPEAR_FORCE_FUSED | SPEAR_FORCE_SPLIT);
    const uint32_t tuned = h->table[bucket_of(M)];
    if (!path)
        path = tuned ? (tuned & (SPEAR_FORCE_DECODE | SPEAR_FORCE_TC)) : default_path(h, M);
    if (!mode)
        mode = tuned ? (tuned & (SPEAR_FORCE_FUSED | SPEAR_FORCE_SPLIT)) : SPEAR_FORCE_FUSED;
    if (!mode)
        mode = SPEAR_FORCE_FUSED;
    return path | mode;
}

// Gate and v for M tokens: the tcgen05 kernel from 256 tokens on, the
// split-K mma.sync kernel below that.
// With `ready`, each CTA (tcgen05) or token tile (mma.sync) counts its v into
// ready[0]; *expected receives the number of counts.
cudaError_t run_prepass(const spear_w4ec *h, const void *x, int64_t M, bool tf32, cudaStream_t st,
                        unsigned *ready = nullptr, unsigned *expected = nullptr)
{
    if (M >= 256 && tc_prepass_supported(h->pk)) {
        if (expected)
            *expected = (unsigned)((M + 127) / 128);
        return launch_tc_prepass(h->pk, x, M, h->v, tf32, h->gbuf, h->tc, h->status, st, ready);
    }
    if (expected)
        *expected = (unsigned)((M + 15) / 16);
    // beside a tcgen05 kernel with tiles of at most 64 tokens (M <= 64), the
    // register-capped prepass shares the SMs with it instead of holding them
    return launch_prepass(h->pk, x, M, h->v, tf32, h->gbuf, h->pre, st, h->num_sms, ready, ready && M <= 64);
}

int run_forward(const spear_w4ec *h, const void *x, void *y, int64_t M, uint32_t flags, cudaStream_t st)
{
    const Packed &pk = h->pk;
    const bool ec = pk.r > 0 && !(flags & SPEAR_EC_OFF);
    const uint32_t choice = resolve(h, M, flags);
    if ((choice & SPEAR_FORCE_DECODE) && (choice & SPEAR_FORCE_TC))
        return SPEAR_ERR_INVALID;
    if ((choice & SPEAR_FORCE_FUSED) && (choice & SPEAR_FORCE_SPLIT))
        return SPEAR_ERR_INVALID;
    const bool fused = (choice & SPEAR_FORCE_FUSED) != 0;
    if (h->fault_launch)
        return SPEAR_ERR_CUDA;
    cudaError_t e = cudaSuccess;
    const bool decode = (choice & SPEAR_FORCE_DECODE) != 0;
    if (decode && !decode_supported(pk, h->num_sms))
        return SPEAR_ERR_UNSUPPORTED;
    // the decode kernel computes its own gate and EC down-projection when fused;
    // before the fused tcgen05 kernel, the prepass counts its v into vready so
    // that the tcgen05 kernel can start its main stages alongside it
    const bool early = ec && fused && (choice & SPEAR_FORCE_TC) && tc_supported(h);
    unsigned expected = 0;
    if (ec && !(decode && fused)) {
        e = run_prepass(h, x, M, (choice & SPEAR_FORCE_TC) != 0 && fused, st, early ? h->vready : nullptr,
                        &expected);
        if (e != cudaSuccess)
            return from_cuda(e);
    }
    if (choice & SPEAR_FORCE_TC) {
        if (!tc_supported(h))
            return SPEAR_ERR_UNSUPPORTED;
        e = launch_tc(pk, x, y, M, h->v, ec && fused, h->tc, h->status, h->fault_timeout, st, h->num_sms,
                      early ? h->vready : nullptr, expected);
        if (e != cudaSuccess || (early && h->fault_timeout)) {
            // nothing will reset the prepass's counts: clear them for the next forward
            cudaMemsetAsync(h->vready, 0, 2 * sizeof(unsigned), st);
        }
        if (e != cudaSuccess)
            return from_cuda(e);
    } else {
        for (int64_t t0 = 0; t0 < M; t0 += kDecodeMaxTokens) {
            const int64_t m = std::min<int64_t>(kDecodeMaxTokens, M - t0);
            e = launch_decode(pk, static_cast<const uint16_t *>(x) + t0 * pk.K,
                              static_cast<uint16_t *>(y) + t0 * pk.N, m, ec && fused, h->dec, h->status, st,
                              h->num_sms);
            if (e != cudaSuccess)
                return from_cuda(e);
        }
    }
    if (ec && !fused) {
        e = launch_ec_apply(pk, h->v, y, M, st);
        if (e != cudaSuccess)
            return from_cuda(e);
    }
    return SPEAR_OK;
}

// Pack (W given: symmetric or asymmetric RTN) or import (codes, s, z given)
// the layer, then the EC operands and the kernels' tensor maps.
int pack_layer(spear_w4ec *h, const void *W, const void *codes, const float *s, const uint8_t *z, const void *A,
               const void *B, const void *w_g, float b_g, void *stream, bool asym)
{
    if (!h || (W && !aligned16(W)) || (!W && !codes))
        return SPEAR_ERR_INVALID;
    if (h->pk.r > 0 && (!A || !B || !w_g))
        return SPEAR_ERR_INVALID;
    DeviceGuard guard(h->device);
    if (!guard.ok())
        return SPEAR_ERR_CUDA;
    h->pk.b_g = b_g;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = W ? launch_pack(h->pk, W, A, B, w_g, h->status, st, asym)
                      : launch_import(h->pk, codes, s, z, A, B, w_g, h->status, st);
    if (e != cudaSuccess)
        return from_cuda(e);
    e = tc_prepare(h->pk, h->tc);
    if (e == cudaSuccess)
        e = decode_prepare(h->pk, h->dec);
    if (e != cudaSuccess)
        return from_cuda(e);
    h->packed = true;
    return SPEAR_OK;
}

}  // namespace

namespace spear {

int status_of(cudaError_t e) { return from_cuda(e); }

int bucket_of(int64_t M)
{
    int b = 0;
    int64_t cap = 1;
    while (b < 8 && M > cap) {
        cap *= 2;
        ++b;
    }
    return b;  // 1,2,4,...,128 -> 0..7, >128 -> 8
}

bool path_supported(const spear_w4ec *h, uint32_t path)
{
    if (path == SPEAR_FORCE_TC)
        return tc_supported(h);
    if (path == SPEAR_FORCE_DECODE)
        return decode_supported(h->pk, h->num_sms);
    return false;
}

int forward_checked(const spear_w4ec *h, const void *x, void *y, int64_t M, uint32_t flags, cudaStream_t st)
{
    return run_forward(h, x, y, M, flags, st);
}

}  // namespace spear

extern "C" {

const char *spear_w4ec_strerror(int status)
{
    switch (status) {
    case SPEAR_OK: return "ok";
    case SPEAR_ERR_INVALID: return "invalid argument";
    case SPEAR_ERR_UNSUPPORTED: return "unsupported shape or path";
    case SPEAR_ERR_NOMEM: return "out of memory";
    case SPEAR_ERR_CUDA: return "CUDA error";
    case SPEAR_ERR_TIMEOUT: return "device-side wait timed out";
    case SPEAR_ERR_DEVICE: return "kernel reported bad data (non-finite weights or scaled EC operand)";
    case SPEAR_ERR_STATE: return "call out of order (layer not packed)";
    default: return "unknown status";
    }
}

int spear_w4ec_create(spear_w4ec **out, int64_t K, int64_t N, int32_t r, const spear_w4ec_opts *opts)
{
    if (!out)
        return SPEAR_ERR_INVALID;
    *out = nullptr;
    if (K <= 0 || N <= 0 || K % 8 || N % 8 || r < 0 || r > 128)
        return SPEAR_ERR_INVALID;
    int dev = (opts && opts->device >= 0) ? opts->device : -1;
    if (dev < 0 && cudaGetDevice(&dev) != cudaSuccess)
        return SPEAR_ERR_CUDA;
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || dev >= ndev)
        return SPEAR_ERR_INVALID;
    if (std::strcmp(env_fault(), "alloc") == 0)
        return SPEAR_ERR_NOMEM;
    DeviceGuard guard(dev);
    if (!guard.ok())
        return SPEAR_ERR_CUDA;

    spear_w4ec *h = new (std::nothrow) spear_w4ec();
    if (!h)
        return SPEAR_ERR_NOMEM;
    h->device = dev;
    h->max_M = (opts && opts->max_M > 0) ? opts->max_M : 4096;
    cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, dev);
    for (auto &row : h->cost_us)
        for (float &c : row)
            c = -1.0f;
    h->fault_launch = std::strcmp(env_fault(), "launch") == 0;
    h->fault_timeout = std::strcmp(env_fault(), "timeout") == 0;

    Packed &pk = h->pk;
    pk.K = K;
    pk.N = N;
    pk.Kp = round_up(K, 256);
    pk.Np = round_up(N, 128);
    pk.r = r;
    pk.rp = r > 0 ? (int)round_up(r, 16) : 0;
    pk.R1p = r > 0 ? (int)round_up(r + 1, 16) : 0;
    pk.b_g = 0.f;

    cudaError_t e = cudaSuccess;
    auto chk = [&](cudaError_t x) {
        if (e == cudaSuccess)
            e = x;
    };
    chk(alloc_zero(&pk.codes, (size_t)pk.Np * pk.Kp / 8));
    chk(alloc_zero(&pk.s, (size_t)pk.Np));
    chk(alloc_zero(&pk.z, (size_t)pk.Np));
    if (r > 0) {
        chk(alloc_zero(&pk.G, (size_t)pk.R1p * pk.Kp));
        chk(alloc_zero(&pk.Bt, (size_t)pk.Np * pk.rp));
        chk(alloc_zero(&pk.Bts, (size_t)pk.Np * pk.rp));
        chk(alloc_zero(&h->v, (size_t)h->max_M * pk.rp));
        chk(alloc_zero(&h->gbuf, (size_t)h->max_M));
        h->pre.part_floats = prepass_part_floats(pk, h->max_M, h->num_sms);
        h->pre.n_counters = prepass_counters(h->max_M);
        chk(alloc_zero(&h->pre.part, h->pre.part_floats));
        chk(alloc_zero(&h->pre.counters, (size_t)h->pre.n_counters));
    }
    chk(alloc_zero(&h->dec.ws_u, decode_u_floats(pk)));
    chk(alloc_zero(&h->dec.flags, (size_t)kDecodeFlags));
    chk(alloc_zero(&h->dec.ws_stream, decode_stream_ws_floats(pk)));
    chk(alloc_zero(&h->dec.cnt_stream, (size_t)kDecodeStreamCounters));
    chk(tc_alloc(pk, h->max_M, h->num_sms, h->tc));
    chk(alloc_zero(&h->status, 1));
    chk(alloc_zero(&h->vready, 2));
    if (e == cudaSuccess)
        e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
        free_all(h);
        delete h;
        return from_cuda(e);
    }
    *out = h;
    return SPEAR_OK;
}

int spear_w4ec_pack(spear_w4ec *h, const void *W, const void *A, const void *B, const void *w_g, float b_g,
                    void *stream)
{
    return pack_layer(h, W, nullptr, nullptr, nullptr, A, B, w_g, b_g, stream, false);
}

int spear_w4ec_pack_asym(spear_w4ec *h, const void *W, const void *A, const void *B, const void *w_g, float b_g,
                         void *stream)
{
    return pack_layer(h, W, nullptr, nullptr, nullptr, A, B, w_g, b_g, stream, true);
}

int spear_w4ec_import(spear_w4ec *h, const void *codes, const float *s, const uint8_t *z, const void *A,
                      const void *B, const void *w_g, float b_g, void *stream)
{
    if (!codes || !s || !z)
        return SPEAR_ERR_INVALID;
    return pack_layer(h, nullptr, codes, s, z, A, B, w_g, b_g, stream, false);
}

int spear_w4ec_forward(const spear_w4ec *h, const void *x, void *y, int64_t M, uint32_t flags, void *stream)
{
    if (!h || M < 0)
        return SPEAR_ERR_INVALID;
    if (M == 0)
        return SPEAR_OK;
    if (!h->packed)
        return SPEAR_ERR_STATE;
    if (M > h->max_M || !x || !y || !aligned16(x) || !aligned16(y))
        return SPEAR_ERR_INVALID;
    DeviceGuard guard(h->device);
    if (!guard.ok())
        return SPEAR_ERR_CUDA;
    return run_forward(h, x, y, M, flags, static_cast<cudaStream_t>(stream));
}

int spear_w4ec_forward_host(spear_w4ec *h, const void *x_host, void *y_host, int64_t M, uint32_t flags,
                            void *stream)
{
    if (!h || M < 0)
        return SPEAR_ERR_INVALID;
    if (M == 0)
        return SPEAR_OK;
    if (!h->packed)
        return SPEAR_ERR_STATE;
    if (M > h->max_M || !x_host || !y_host)
        return SPEAR_ERR_INVALID;
    DeviceGuard guard(h->device);
    if (!guard.ok())
        return SPEAR_ERR_CUDA;
    cudaError_t e = cudaSuccess;
    if (!h->x_stage) {
        e = cudaMalloc(&h->x_stage, (size_t)h->max_M * h->pk.K * 2);
        if (e == cudaSuccess)
            e = cudaMalloc(&h->y_stage, (size_t)h->max_M * h->pk.N * 2);
        if (e != cudaSuccess) {
            cudaFree(h->x_stage);
            h->x_stage = nullptr;
            h->y_stage = nullptr;
            return from_cuda(e);
        }
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    e = cudaMemcpyAsync(h->x_stage, x_host, (size_t)M * h->pk.K * 2, cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess)
        return from_cuda(e);
    int rc = run_forward(h, h->x_stage, h->y_stage, M, flags, st);
    if (rc != SPEAR_OK)
        return rc;
    e = cudaMemcpyAsync(y_host, h->y_stage, (size_t)M * h->pk.N * 2, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(st);
    return from_cuda(e);
}

int spear_w4ec_destroy(spear_w4ec *h)
{
    if (!h)
        return SPEAR_OK;
    DeviceGuard guard(h->device);
    cudaDeviceSynchronize();
    // no handle may go on prefetching this one's memory
    for (spear_w4ec *p : h->prev)
        if (p != h) {
            p->next = nullptr;
            p->dec.pf = nullptr;
            p->dec.pf_bytes = 0;
        }
    if (h->next && h->next != h) {
        auto &v = h->next->prev;
        v.erase(std::remove(v.begin(), v.end(), h), v.end());
    }
    free_all(h);
    delete h;
    return SPEAR_OK;
}

int spear_w4ec_set_next(spear_w4ec *h, spear_w4ec *next)
{
    if (!h || (next && next->device != h->device))
        return SPEAR_ERR_INVALID;
    if (h->next) {
        auto &v = h->next->prev;
        v.erase(std::remove(v.begin(), v.end(), h), v.end());
    }
    h->next = next;
    h->dec.pf = nullptr;
    h->dec.pf_bytes = 0;
    if (next) {
        next->prev.push_back(h);
        h->dec.pf = next->pk.codes;
        h->dec.pf_bytes = (size_t)next->pk.Np * (size_t)next->pk.Kp / 2;
    }
    return SPEAR_OK;
}

int spear_w4ec_get_packed(const spear_w4ec *h, void *codes, float *s, uint8_t *z, void *stream)
{
    if (!h)
        return SPEAR_ERR_INVALID;
    if (!h->packed)
        return SPEAR_ERR_STATE;
    DeviceGuard guard(h->device);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const Packed &pk = h->pk;
    cudaError_t e = cudaSuccess;
    if (codes)
        e = launch_untile_codes(pk, static_cast<uint32_t *>(codes), st);
    if (e == cudaSuccess && s)
        e = cudaMemcpyAsync(s, pk.s, (size_t)pk.N * sizeof(float), cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess && z)
        e = cudaMemcpyAsync(z, pk.z, (size_t)pk.N, cudaMemcpyDeviceToDevice, st);
    return from_cuda(e);
}

int spear_w4ec_get_gate(const spear_w4ec *h, const void *x, float *g, int64_t M, void *stream)
{
    if (!h || M < 0 || !x || !g || !aligned16(x))
        return SPEAR_ERR_INVALID;
    if (h->pk.r == 0)
        return SPEAR_ERR_UNSUPPORTED;
    if (!h->packed)
        return SPEAR_ERR_STATE;
    if (M > h->max_M)
        return SPEAR_ERR_INVALID;
    if (M == 0)
        return SPEAR_OK;
    DeviceGuard guard(h->device);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = run_prepass(h, x, M, false, st);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(g, h->gbuf, (size_t)M * sizeof(float), cudaMemcpyDeviceToDevice, st);
    return from_cuda(e);
}

int spear_w4ec_sync_status(spear_w4ec *h, void *stream)
{
    if (!h)
        return SPEAR_ERR_INVALID;
    DeviceGuard guard(h->device);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int bits = 0;
    cudaError_t e = cudaStreamSynchronize(st);
    if (e == cudaSuccess)
        e = cudaMemcpy(&bits, h->status, sizeof(int), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && bits)
        e = cudaMemset(h->status, 0, sizeof(int));
    if (e != cudaSuccess)
        return from_cuda(e);
    if (bits & kStatusTimeout)
        return SPEAR_ERR_TIMEOUT;
    if (bits & kStatusNonFinite)
        return SPEAR_ERR_DEVICE;
    return SPEAR_OK;
}

int spear_w4ec_dispatch(const spear_w4ec *h, int64_t M, uint32_t *choice)
{
    if (!h || M < 0 || !choice)
        return SPEAR_ERR_INVALID;
    *choice = resolve(h, M, 0);
    return SPEAR_OK;
}

int spear_w4ec_tune(spear_w4ec *h, const void *x, void *y, int64_t M, void *stream, uint32_t *choice)
{
    if (!h || M <= 0 || !x || !y || !aligned16(x) || !aligned16(y))
        return SPEAR_ERR_INVALID;
    if (!h->packed)
        return SPEAR_ERR_STATE;
    if (M > h->max_M)
        return SPEAR_ERR_INVALID;
    DeviceGuard guard(h->device);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // every legal choice with the EC (fused and split), and each path with the EC off
    std::vector<uint32_t> cands;
    const uint32_t paths[2] = {SPEAR_FORCE_DECODE, SPEAR_FORCE_TC};
    for (uint32_t path : paths) {
        if (!path_supported(h, path))
            continue;
        cands.push_back(path | SPEAR_FORCE_FUSED);
        if (h->pk.r > 0) {
            cands.push_back(path | SPEAR_FORCE_SPLIT);
            cands.push_back(path | SPEAR_FORCE_FUSED | SPEAR_EC_OFF);
        }
    }
    cudaEvent_t e0, e1;
    if (cudaEventCreate(&e0) != cudaSuccess)
        return SPEAR_ERR_CUDA;
    if (cudaEventCreate(&e1) != cudaSuccess) {
        cudaEventDestroy(e0);
        return SPEAR_ERR_CUDA;
    }
    const int b = bucket_of(M);
    float best_ms = 1e30f;
    uint32_t best = 0;
    int rc = SPEAR_OK;
    for (uint32_t cand : cands) {
        for (int i = 0; i < 3 && rc == SPEAR_OK; ++i)
            rc = run_forward(h, x, y, M, cand, st);
        if (rc != SPEAR_OK)
            break;
        std::vector<float> times;
        for (int i = 0; i < 9 && rc == SPEAR_OK; ++i) {
            cudaEventRecord(e0, st);
            rc = run_forward(h, x, y, M, cand, st);
            cudaEventRecord(e1, st);
            cudaEventSynchronize(e1);
            float ms = 0.f;
            cudaEventElapsedTime(&ms, e0, e1);
            times.push_back(ms);
        }
        if (rc != SPEAR_OK)
            break;
        std::sort(times.begin(), times.end());
        const float med = times[times.size() / 2];
        h->cost_us[b][cost_index(cand)] = med * 1000.0f;
        if (cand & SPEAR_EC_OFF) {
            h->cost_us[b][cost_index(cand | SPEAR_FORCE_SPLIT)] = med * 1000.0f;
            continue;   // a time without the EC, for the cost model only
        }
        if (med < best_ms) {
            best_ms = med;
            best = cand;
        }
    }
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
    if (rc != SPEAR_OK)
        return rc;
    h->table[bucket_of(M)] = best;
    if (choice)
        *choice = best;
    return from_cuda(cudaStreamSynchronize(st));
}

}  // extern "C"

namespace spear {

cudaError_t raise_smem_limit(const void *func, size_t bytes)
{
    struct Entry {
        const void *func;
        int device;
        size_t bytes;
    };
    static std::vector<Entry> done;
    static std::mutex mu;
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lock(mu);
    for (const Entry &e : done)
        if (e.func == func && e.device == dev && e.bytes >= bytes)
            return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess)
        done.push_back({func, dev, bytes});
    return e;
}

}  // namespace spear
