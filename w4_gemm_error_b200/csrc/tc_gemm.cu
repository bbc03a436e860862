// Placeholder until the tcgen05 tile kernel lands: reports the path as unavailable.
#include "tc_gemm.h"

namespace spear {

bool tc_available(const Packed &) { return false; }
cudaError_t tc_alloc(const Packed &, int64_t, int, TcWork &) { return cudaSuccess; }
void tc_free(TcWork &) {}
cudaError_t tc_prepare(const Packed &, TcWork &) { return cudaSuccess; }
cudaError_t launch_tc(const Packed &, const void *, void *, int64_t, const uint16_t *, bool, const TcWork &, int *,
                      bool, cudaStream_t, int)
{
    return cudaErrorNotSupported;
}

}  // namespace spear
