// Library-internal view of a layer handle (the struct behind the opaque
// spear_w4ec of include/spear_w4ec.h) and the calls that other translation
// units of the library share with spear_w4ec.cu.
#pragma once
#include <cuda_runtime.h>

#include <cstdint>
#include <vector>

#include "spear_w4ec.h"
#include "kernels.h"
#include "tc_gemm.h"

using spear::DecodeWork;
using spear::Packed;
using spear::PrepassWork;
using spear::TcWork;

struct spear_w4ec {
    int device = 0;
    int num_sms = 148;
    int64_t max_M = 0;
    Packed pk{};
    bool packed = false;
    // workspace
    float *v = nullptr;         // [max_M][rp] fp32: g_t * (x . A) (tf32-rounded for the tcgen05 path)
    float *gbuf = nullptr;      // [max_M] gate values
    PrepassWork pre{};
    DecodeWork dec{};
    TcWork tc{};
    int *status = nullptr;      // sticky device status bits
    unsigned *vready = nullptr; // prepass -> tcgen05 kernel: [0] counts of v written, [1] CTAs done
    // staging for forward_host
    void *x_stage = nullptr;
    void *y_stage = nullptr;
    // dispatch table: flags per M bucket, 0 = not tuned
    uint32_t table[9] = {0, 0, 0, 0, 0, 0, 0, 0, 0};
    // measured microseconds per forward, per M bucket and choice (see
    // spear::cost_index), negative where not measured
    float cost_us[9][8];
    // host-side fault injection (SPEAR_FAULT=alloc|launch|timeout)
    bool fault_launch = false;
    bool fault_timeout = false;
    // cross-layer prefetch hint: the layer that follows this one, and the
    // handles that name this one as theirs
    spear_w4ec *next = nullptr;
    std::vector<spear_w4ec *> prev;
};

namespace spear {

// Makes a device current for the lifetime of the guard, then restores the
// caller's device.
class DeviceGuard {
  public:
    explicit DeviceGuard(int dev)
    {
        if (cudaGetDevice(&prev_) != cudaSuccess)
            prev_ = -1;
        if (prev_ != dev)
            ok_ = cudaSetDevice(dev) == cudaSuccess;
    }
    ~DeviceGuard()
    {
        int cur = -1;
        if (prev_ >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev_)
            cudaSetDevice(prev_);
    }
    bool ok() const { return ok_; }

  private:
    int prev_ = -1;
    bool ok_ = true;
};

// Status of a CUDA runtime result (SPEAR_ERR_NOMEM for an allocation failure).
int status_of(cudaError_t e);

// Slot of a (path, EC placement, EC on/off) choice in cost_us: tcgen05 path
// + 4, split EC + 2, EC off + 1 (EC off ignores the placement; its time is
// kept in both placement slots).
inline int cost_index(uint32_t flags)
{
    return ((flags & SPEAR_FORCE_TC) ? 4 : 0) + ((flags & SPEAR_FORCE_SPLIT) ? 2 : 0) + ((flags & SPEAR_EC_OFF) ? 1 : 0);
}

// M bucket of the dispatch table: 1, 2, 4, ..., 128 -> 0..7, more -> 8.
int bucket_of(int64_t M);

// Whether the handle's device can run a kernel family (SPEAR_FORCE_DECODE or
// SPEAR_FORCE_TC) on this layer.
bool path_supported(const spear_w4ec *h, uint32_t path);

// The kernel sequence of one forward pass of a packed layer.  The caller has
// checked the arguments (1 <= M <= max_M, 16-byte aligned device x and y) and
// made the handle's device current.
int forward_checked(const spear_w4ec *h, const void *x, void *y, int64_t M, uint32_t flags, cudaStream_t st);

}  // namespace spear
