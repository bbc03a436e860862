// tcgen05 / TMEM tile kernel for larger token counts (library-internal).
#pragma once
#include <cuda_runtime.h>
#include <cstdint>

#include "kernels.h"

namespace spear {

struct TcWork {
    void *maps = nullptr;        // host-side tensor maps of the packed operands
    float *part = nullptr;       // split-K partials
    size_t part_floats = 0;
    unsigned *counters = nullptr;
    int n_counters = 0;
};

bool tc_available(const Packed &pk);
cudaError_t tc_alloc(const Packed &pk, int64_t max_M, int num_sms, TcWork &w);
void tc_free(TcWork &w);
cudaError_t tc_prepare(const Packed &pk, TcWork &w);
// Gate and v = g * (x . A) for many tokens on the tensor cores (128 tokens per CTA).
// `ready` (may be null): counted once per CTA (release) when its v is written;
// ceil(M / 128) counts in all.
bool tc_prepass_supported(const Packed &pk);
cudaError_t launch_tc_prepass(const Packed &pk, const void *x, int64_t M, float *v, bool tf32, float *g,
                              const TcWork &w, int *status, cudaStream_t st, unsigned *ready);
// v: the prepass output in fp32 rounded to tf32 ([M][rp]), read when `ec` is set.
// v_ready (may be null; used only with `ec`): the kernel starts its main stages
// without waiting for its predecessor, which must be a prepass that counts
// v_expected completions into v_ready[0] and starts its dependents only once x is
// complete; v_ready[0..1] are zero between calls.
cudaError_t launch_tc(const Packed &pk, const void *x, void *y, int64_t M, const float *v, bool ec,
                      const TcWork &w, int *status, bool zero_wait_budget, cudaStream_t st, int num_sms,
                      unsigned *v_ready, unsigned v_expected);

}  // namespace spear
