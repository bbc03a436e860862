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
bool tc_prepass_supported(const Packed &pk);
cudaError_t launch_tc_prepass(const Packed &pk, const void *x, int64_t M, float *v, bool tf32, float *g,
                              const TcWork &w, int *status, cudaStream_t st);
// v: the prepass output in fp32 rounded to tf32 ([M][rp]), read when `ec` is set.
cudaError_t launch_tc(const Packed &pk, const void *x, void *y, int64_t M, const float *v, bool ec,
                      const TcWork &w, int *status, bool zero_wait_budget, cudaStream_t st, int num_sms);

}  // namespace spear
