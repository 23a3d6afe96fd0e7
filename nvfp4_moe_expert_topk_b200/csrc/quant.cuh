// quant.cuh -- the NVFP4 16-element block quantiser, shared by the
// activation quantiser and the fused epilogue of the L1 GEMM.
//
// For one block of 16 fp32 values and global scale gs (NVFP4: E2M1 values,
// one E4M3 scale per 16 elements, one fp32 global multiplier --
// "nvfp4-megamoe-kernel / CURRENT_BUG.md", page 2 "What the quant method
// does"):  a = max|x_i|;  v = (a / 6) * gs;  s = E4M3(v);
// r = (s == 0) ? 0 : gs / value(s);  q_i = E2M1(x_i * r).
// Every fp32 step rounds to nearest (explicit _rn intrinsics, so no FMA
// contraction or fast-math substitution can change a code), and both format
// conversions round to nearest even with saturation.
#pragma once

#include "ptx.cuh"

namespace nvfp4 {

// Returns the scale byte; lo / hi receive the 16 codes (element 0 in the low
// nibble of lo).
__device__ __forceinline__ uint32_t quantize16(const float (&x)[16], float gs, uint32_t &lo, uint32_t &hi)
{
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i)
        a = fmaxf(a, fabsf(x[i]));
    const float v = __fmul_rn(__fdiv_rn(a, 6.0f), gs);
    const uint32_t s = cvt_e4m3(v);
    const float r = (s == 0u) ? 0.0f : __fdiv_rn(gs, e4m3_value(s));
    float p[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
        p[i] = __fmul_rn(x[i], r);
    lo = cvt_e2m1x8(p);
    hi = cvt_e2m1x8(p + 8);
    return s;
}

// Byte offset, inside an NVFP4_SCALES_MMA buffer, of the 4 scale bytes of
// row `row`, 64-element block `kb` (kb_per_block = cols / 64).
__device__ __forceinline__ int64_t mma_scale_offset(int64_t row, int64_t kb, int64_t kb_per_block)
{
    return ((row >> 7) * kb_per_block + kb) * 512 + (row & 31) * 16 + ((row >> 5) & 3) * 4;
}

} // namespace nvfp4
