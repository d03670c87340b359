// Exact binary16 helpers shared by the library's kernels.
//
// Scales are positive finite binary16 values, addressed by their bit pattern
// j = 0x0001 .. 0x7BFF (bit order is value order).  Codes follow CliffQuant's
// quantiser (project page, "What CliffQuant changes"): q = clip(round-half-even(w/s), -8, 7).
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

namespace cq {

constexpr int kGroup = 128;
constexpr uint32_t kLast = 0x7BFFu;    // largest finite binary16 pattern (65504)
constexpr uint32_t kBeyond = 0x7C00u;  // one past the grid
constexpr unsigned kFull = 0xFFFFFFFFu;

__device__ __forceinline__ float half_value(uint32_t bits)
{
    return __half2float(__ushort_as_half(static_cast<unsigned short>(bits)));
}

// Value of a positive binary16 pattern j in [1, 0x7C00] (0x7C00 gives 65536),
// built from bits without a conversion instruction: for j >= 0x400 the fp32
// pattern is (j << 13) + 0x38000000; for subnormal halves the same construction
// with the exponent one higher gives 2^-14 + j 2^-24, and 2^-14 is subtracted
// exactly.
__device__ __forceinline__ float grid_value(uint32_t j)
{
    const bool sub = j < 0x400u;
    const float v = __uint_as_float((j << 13) + (sub ? 0x38800000u : 0x38000000u));
    return sub ? v - 0x1p-14f : v;
}

// |q| >= m for |w| = aw at scale s, before clipping: round-half-even(aw/s) >= m.
// s * (m - 1/2) is exact in fp32 (11-bit s times a 5-bit odd/2 factor).
__device__ __forceinline__ bool code_at_least(float aw, float s, int m)
{
    const float t = s * (static_cast<float>(m) - 0.5f);
    return aw > t || (aw == t && (m & 1) == 0);
}

// min(round-half-even(aw / s), K), exact: an fp32 estimate corrected by the
// exact threshold tests above (the estimate is within one of the answer).
__device__ __forceinline__ int abs_code(float aw, float s, int K)
{
    const float x = fminf(__fdividef(aw, s), 15.0f);
    int n = __float2int_rn(x);
    if (n > 0 && !code_at_least(aw, s, n))
        n -= 1;
    else if (code_at_least(aw, s, n + 1))
        n += 1;
    return min(n, K);
}

template <typename T>
__device__ __forceinline__ T warp_sum(T v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v += __shfl_xor_sync(kFull, v, o);
    return v;
}

}  // namespace cq
