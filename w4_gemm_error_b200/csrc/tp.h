// Row-parallel tensor parallelism (a layer split along K over ranks): the
// library-internal pieces that tp.cu shares with prepass.cu.
#pragma once
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.h"

namespace spear {

constexpr int kTpMaxWorld = 8;

// Where the raw partials of one rank's EC down-projection go, and the words
// that order the ranks:
//   dst[q]    slot of this rank in rank q's exchange buffer, [max_M][R1p] fp32
//   ready[q]  this rank's ready word in rank q's buffer
//   epoch     this rank's count of completed calls (read only here)
//   tiles     count of 16-token tiles written in this call (zero between calls)
//   sys       1 when some rank's buffer is on another GPU (system-scope
//             ordering), 0 when all are on this device (GPU scope suffices)
struct TpPush {
    float *dst[kTpMaxWorld];
    unsigned *ready[kTpMaxWorld];
    int world;
    int sys;
    const unsigned *epoch;
    unsigned *tiles;
};

#ifdef __CUDACC__
// The ordering operations of the group at its scope: the system when some
// rank is on another GPU, else the GPU (a system-scope fence costs several
// microseconds on B200).
__device__ __forceinline__ void tp_fence(int sys)
{
    if (sys)
        asm volatile("fence.acq_rel.sys;" ::: "memory");
    else
        asm volatile("fence.acq_rel.gpu;" ::: "memory");
}
__device__ __forceinline__ void tp_store_relaxed(unsigned *p, unsigned v, int sys)
{
    if (sys)
        asm volatile("st.relaxed.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
    else
        asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned tp_load_acquire(const unsigned *p, int sys)
{
    unsigned v;
    if (sys)
        asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    else
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
#endif

// Raw partials u[t][j] = x[t,:] . G[j,:] of the shard (row 0 of G is w_g, rows
// 1..r the columns of A; no bias, no sigmoid), fp32 with the same split-K and
// fixed-order sums as launch_prepass, written to every rank's slot; the last
// tile to be written raises the ready words to epoch + 1 (a fence at the
// group's scope, then the stores).  Waits (griddepcontrol.wait) for the
// kernel before it in the stream, so everything that kernel and its
// predecessors wrote is visible to the other ranks once they see the ready
// word.
cudaError_t launch_prepass_partial(const Packed &pk, const void *x, int64_t M, const PrepassWork &w,
                                   const TpPush &push, cudaStream_t st, int num_sms);

}  // namespace spear
