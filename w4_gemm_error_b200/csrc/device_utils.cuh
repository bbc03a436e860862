// Small device helpers shared by the kernels of libspear_w4ec (sm_100a).
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

namespace spear {

// Sticky status bits written by kernels into the handle's device status word.
enum : int { kStatusNonFinite = 1, kStatusTimeout = 2 };

__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t b, uint32_t c)
{
    // (a & b) | c
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// d = a * b + c on bf16x2 (round to nearest); exact when the result is a small integer.
__device__ __forceinline__ uint32_t fma_bf16x2(uint32_t a, uint32_t b, uint32_t c)
{
    uint32_t d;
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// Stored nibble order of a code word (the tiled layout on the device): the
// codes of k = 8j + {0, 2, 4, 6} sit in nibbles 0..3 and those of k = 8j +
// {1, 3, 5, 7} in nibbles 4..7, so that the nibble pair (m, m + 4), 16 bits
// apart, is the consecutive pair k = 8j + 2m, 8j + 2m + 1.  Bit offset of the
// code of k = 8j + i:
__host__ __device__ constexpr int nibble_shift(int i) { return 4 * ((i & 1) * 4 + (i >> 1)); }

// Two int4 codes, the nibbles at bit positions `sh` and `sh + 16` of w, as a
// bf16x2 pair of exact integers (q_lo - zp, q_hi - zp).  The nibble is placed
// in the low mantissa bits of 128.0 (0x4300), giving 128 + q exactly; the fma
// then subtracts 128 + zp, which is exact because the result is an integer
// of magnitude <= 15.  neg_bias = bf16x2(-(128 + zp), -(128 + zp)).
__device__ __forceinline__ uint32_t dequant_pair(uint32_t w_shifted, uint32_t neg_bias)
{
    const uint32_t t = lop3_and_or(w_shifted, 0x000F000Fu, 0x43004300u);
    return fma_bf16x2(t, 0x3F803F80u /* (1.0, 1.0) */, neg_bias);
}

// As dequant_pair with a per-row multiplier: mul = bf16x2(1, 1) with neg_bias
// as above, or mul = neg_bias = 0 for a row whose scale is 0 (its weights are
// 0 whatever its codes say), for a kernel that applies a stand-in scale of 1
// to such rows after accumulating.
__device__ __forceinline__ uint32_t dequant_pair_mul(uint32_t w_shifted, uint32_t mul, uint32_t neg_bias)
{
    const uint32_t t = lop3_and_or(w_shifted, 0x000F000Fu, 0x43004300u);
    return fma_bf16x2(t, mul, neg_bias);
}

// D (16x8 fp32) += A (16x16 bf16, row) * B (16x8 bf16, col).  Not volatile: its
// only effect is on d, so the compiler may interleave independent MMAs.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Streaming 16-byte load that is read once (no L1 allocation).
__device__ __forceinline__ uint4 ld_stream(const void *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint4 ld_nc(const void *p)
{
    return __ldg(reinterpret_cast<const uint4 *>(p));
}

// Programmatic dependent launch: let the next kernel in the stream start, and
// wait for the previous kernel's results (no-ops without the launch attribute).
__device__ __forceinline__ void pdl_launch_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// fp32 rounded to the tf32 grid (10 explicit mantissa bits, round to nearest, ties away).
__device__ __forceinline__ float to_tf32(float x)
{
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return __uint_as_float(r);
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

}  // namespace spear
