// Per-token gate with no allocation: a variant of the prepass kernel whose
// split-K scratch lives in a file-scope __device__ array instead of a
// handle's workspace.
//
// For callers that may not allocate device memory at all -- code running
// inside a CUDA graph capture, a real-time serving loop with a fixed memory
// budget, or a host framework that owns every allocation through its own
// pool -- this entry point needs neither a handle nor cudaMalloc:
//     g[t] = 1 / (1 + exp(-(x[t,:] . w_g + b_g)))
// It computes the same gate as spear_w4ec_get_gate, from the caller's own
// x and w_g.
//
// The scratch is one static array (kScratchBytes, held by every GPU that
// loads the library until the process exits) shared by all calls: split-K
// partial sums and one counter per 16-token tile.  Every call clears the
// counters before its kernel runs; calls that overlap on the GPU (different
// streams without ordering) race on the array.
#include <cuda_runtime.h>

#include <mutex>

#include "device_utils.cuh"
#include "kernels.h"
#include "spear_w4ec.h"

namespace spear {
namespace {

constexpr int64_t kMaxTokens = 4096;           // largest M accepted
constexpr int kTok = 16;                       // tokens per CTA
constexpr int kMaxTiles = (int)(kMaxTokens / kTok);
constexpr int kMaxSplits = 64;
constexpr size_t kPartialFloats = 16384;       // split-K partial sums (64 KB)
constexpr size_t kScratchBytes = kPartialFloats * sizeof(float) + kMaxTiles * sizeof(unsigned);

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

// Eight threads per token, each summing 16-byte pieces of x[t,:] * w_g over
// the CTA's k range; the last CTA of a tile sums the split partials in order.
__global__ void __launch_bounds__(128)
gate_noalloc_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ wg, int64_t M, int64_t K,
                    float b_g, int S, int64_t kps, float *__restrict__ g, unsigned char *scratch)
{
    float *part = reinterpret_cast<float *>(scratch);
    unsigned *counters = reinterpret_cast<unsigned *>(scratch + kPartialFloats * sizeof(float));
    __shared__ int s_last;
    const int tile = blockIdx.x / S, ks = blockIdx.x - tile * S;
    const int tt = threadIdx.x >> 3, lane8 = threadIdx.x & 7;
    const int64_t t = (int64_t)tile * kTok + tt;
    const int64_t k0 = ks * kps, k1 = min(K, k0 + kps);
    float acc = 0.f;
    if (t < M) {
        for (int64_t k = k0 + 8 * lane8; k < k1; k += 64) {
            const uint4 xv = ld_nc(x + t * K + k), wv = ld_nc(wg + k);
            acc += bf16_lo(xv.x) * bf16_lo(wv.x) + bf16_hi(xv.x) * bf16_hi(wv.x) + bf16_lo(xv.y) * bf16_lo(wv.y) +
                   bf16_hi(xv.y) * bf16_hi(wv.y) + bf16_lo(xv.z) * bf16_lo(wv.z) + bf16_hi(xv.z) * bf16_hi(wv.z) +
                   bf16_lo(xv.w) * bf16_lo(wv.w) + bf16_hi(xv.w) * bf16_hi(wv.w);
        }
    }
#pragma unroll
    for (int o = 4; o > 0; o >>= 1)
        acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
    if (S == 1) {
        if (lane8 == 0 && t < M)
            g[t] = 1.0f / (1.0f + expf(-(acc + b_g)));
        return;
    }
    if (lane8 == 0)
        part[((size_t)tile * S + ks) * kTok + tt] = acc;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0)
        s_last = (atomicAdd(&counters[tile], 1u) == (unsigned)(S - 1));
    __syncthreads();
    if (!s_last)
        return;
    __threadfence();
    if (threadIdx.x < kTok) {
        const int64_t tk = (int64_t)tile * kTok + threadIdx.x;
        float sum = 0.f;
        for (int q = 0; q < S; ++q)
            sum += __ldcg(part + ((size_t)tile * S + q) * kTok + threadIdx.x);
        if (tk < M)
            g[tk] = 1.0f / (1.0f + expf(-(sum + b_g)));
    }
    if (threadIdx.x == 0)
        counters[tile] = 0u;
}

// Device address of the static scratch, looked up once per device.
std::mutex g_mu;
unsigned char *g_addr[64] = {};

cudaError_t scratch_address(int dev, unsigned char **out)
{
    if (dev < 0 || dev >= 64)
        return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_addr[dev]) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
        if (e != cudaSuccess)
            return e;
        g_addr[dev] = static_cast<unsigned char *>(p);
    }
    *out = g_addr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace spear

using namespace spear;

extern "C" int spear_w4ec_gate_noalloc(const void *x, int64_t M, int64_t K, const void *w_g, float b_g, float *g,
                                       void *stream)
{
    if (M < 0 || K <= 0 || K % 8)
        return SPEAR_ERR_INVALID;
    if (M > kMaxTokens)
        return SPEAR_ERR_INVALID;  // beyond the static scratch: at most 4096 tokens per call
    if (M == 0)
        return SPEAR_OK;
    if (!x || !w_g || !g || (reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(w_g) & 15))
        return SPEAR_ERR_INVALID;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return SPEAR_ERR_CUDA;
    unsigned char *scratch = nullptr;
    if (scratch_address(dev, &scratch) != cudaSuccess)
        return SPEAR_ERR_CUDA;
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int tiles = (int)((M + kTok - 1) / kTok);
    const int64_t k_pieces = (K + 63) / 64;
    int S = (2 * sms + tiles - 1) / tiles;
    if (S > kMaxSplits)
        S = kMaxSplits;
    if (S > k_pieces)
        S = (int)k_pieces;
    if (S < 1)
        S = 1;
    while (S > 1 && (size_t)tiles * S * kTok > kPartialFloats)
        --S;
    const int64_t kps = ((K + 64LL * S - 1) / (64LL * S)) * 64;   // k per split, a multiple of 64
    S = (int)((K + kps - 1) / kps);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the counters must start at zero whatever an earlier call left behind
    if (cudaMemsetAsync(scratch + kPartialFloats * sizeof(float), 0, kMaxTiles * sizeof(unsigned), st) !=
        cudaSuccess)
        return SPEAR_ERR_CUDA;
    gate_noalloc_kernel<<<tiles * S, 128, 0, st>>>(static_cast<const uint16_t *>(x), static_cast<const uint16_t *>(w_g),
                                                   M, K, b_g, S, kps, g, scratch);
    return cudaGetLastError() == cudaSuccess ? SPEAR_OK : SPEAR_ERR_CUDA;
}
