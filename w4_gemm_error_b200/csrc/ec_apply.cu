// Unfused Error Compensator: y += v . B applied by its own kernel after a
// plain W4 GEMM wrote y.  This is the "split" alternative that the adaptive
// kernel-fusion dispatch (SPEAR, "A System for Post-Quantization
// Error-Adaptive Recovery Enabling Efficient Low-Bit LLM Serving", Abstract)
// weighs against the fused kernels; y is rounded to bf16 twice on this path
// (after the GEMM and after the correction); v is read in fp32.
//
// One thread per output channel n (consecutive n -> coalesced y rows), a CTA
// handles 256 channels and 32 tokens; v for those tokens is staged in shared
// memory as fp32 and Bt[n, :] is streamed in 16-byte pieces.
#include "device_utils.cuh"
#include "kernels.h"

namespace spear {
namespace {

constexpr int kThreads = 256;
constexpr int kTokChunk = 32;

__global__ void __launch_bounds__(kThreads)
ec_apply_kernel(const float *__restrict__ vf, const uint16_t *__restrict__ Bt, uint16_t *__restrict__ y,
                int64_t M, int64_t N, int rp)
{
    extern __shared__ float vs[];  // [kTokChunk][rp]
    pdl_launch_dependents();
    pdl_wait();  // y and v are written by the kernels before this one
    const int64_t t0 = (int64_t)blockIdx.y * kTokChunk;
    const int ntok = (int)min((int64_t)kTokChunk, M - t0);
    for (int e = threadIdx.x; e < kTokChunk * rp; e += kThreads) {
        const int tt = e / rp, j = e - tt * rp;
        vs[e] = tt < ntok ? vf[(t0 + tt) * rp + j] : 0.f;
    }
    __syncthreads();
    const int64_t n = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (n >= N)
        return;
    float acc[kTokChunk];
#pragma unroll
    for (int i = 0; i < kTokChunk; ++i)
        acc[i] = 0.f;
    for (int j = 0; j < rp; j += 8) {
        const uint4 bv = ld_nc(Bt + n * rp + j);
        const float bj[8] = {bf16_lo(bv.x), bf16_hi(bv.x), bf16_lo(bv.y), bf16_hi(bv.y),
                             bf16_lo(bv.z), bf16_hi(bv.z), bf16_lo(bv.w), bf16_hi(bv.w)};
#pragma unroll
        for (int i = 0; i < kTokChunk; ++i) {
            const float *vr = vs + i * rp + j;
#pragma unroll
            for (int q = 0; q < 8; ++q)
                acc[i] += vr[q] * bj[q];
        }
    }
#pragma unroll
    for (int i = 0; i < kTokChunk; ++i) {
        if (i < ntok) {
            uint16_t *yp = y + (t0 + i) * N + n;
            const float cur = __uint_as_float((uint32_t)*yp << 16);
            *yp = __bfloat16_as_ushort(__float2bfloat16_rn(cur + acc[i]));
        }
    }
}

}  // namespace

cudaError_t launch_ec_apply(const Packed &pk, const float *vf, void *y, int64_t M, cudaStream_t st)
{
    if (M <= 0 || pk.r == 0)
        return cudaSuccess;
    dim3 grid((unsigned)((pk.N + kThreads - 1) / kThreads), (unsigned)((M + kTokChunk - 1) / kTokChunk));
    const size_t smem = (size_t)kTokChunk * pk.rp * sizeof(float);
    if (smem > 48 * 1024) {
        cudaError_t e = raise_smem_limit(reinterpret_cast<const void *>(ec_apply_kernel), smem);
        if (e != cudaSuccess)
            return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, ec_apply_kernel, vf, (const uint16_t *)pk.Bt, static_cast<uint16_t *>(y), M,
                              pk.N, pk.rp);
}

}  // namespace spear
