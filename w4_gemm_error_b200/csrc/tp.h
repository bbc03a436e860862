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
//   done      the done words in this rank's buffer, [world] (entry q written by rank q)
//   epoch     this rank's count of completed calls (read only here)
//   status    the shard's status word (a wait that runs out sets its timeout bit)
//   sys       1 when some rank's buffer is on another GPU (system-scope
//             ordering), 0 when all are on this device (GPU scope suffices)
struct TpPush {
    float *dst[kTpMaxWorld];
    unsigned *ready[kTpMaxWorld];
    int world;
    int sys;
    const unsigned *done;
    const unsigned *epoch;
    int *status;
};

#ifdef __CUDACC__
#include "async_utils.cuh"

// The ordering operations of the group at its scope: the system when some
// rank is on another GPU, else the GPU (on B200 a system-scope fence takes
// about 1.5 us longer than a GPU-scope one).
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
// Waits (bounded by kWaitBudgetCycles) until the word reaches `target`
// (counts compared modulo 2^32); false if the wait ran out.
__device__ __forceinline__ bool tp_wait_count(const unsigned *w, unsigned target, int sys)
{
    const long long t0 = clock64();
    while ((int)(tp_load_acquire(w, sys) - target) < 0) {
        if (clock64() - t0 > kWaitBudgetCycles)
            return false;
        __nanosleep(64);
    }
    return true;
}
#endif

// Raw partials u[t][j] = x[t,:] . G[j,:] of the shard (row 0 of G is w_g, rows
// 1..r the columns of A; no bias, no sigmoid), fp32 with the same split-K and
// fixed-order sums as launch_prepass, written to this rank's slot of every
// rank's buffer once every rank's done word here has reached this rank's
// count of completed calls (bounded wait: nobody still reads the slots);
// each writing CTA ends with a fence at the group's scope.  The ready words
// are raised later, by the kernel after the shard's forward.
cudaError_t launch_prepass_partial(const Packed &pk, const void *x, int64_t M, const PrepassWork &w,
                                   const TpPush &push, cudaStream_t st, int num_sms);

}  // namespace spear
