// Comparison scale policies and the reconstruction proxy.
//
// The project page's "Held-out reconstruction proxy" table compares three
// scale policies on the module-macro worst-environment weighted MSE:
// CliffQuant minimax (cq_select.cu), Pooled-WMSE (the environments' diagonals
// averaged first, then the same search with one environment) and AbsMax (the
// matched baseline checkpoint's scale, |w|max / 7).  This file holds the
// AbsMax policy, the pooling of diagonals, the objective of given scales and
// the proxy's fixed-order reductions over modules and environments.

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cfloat>
#include <cstdint>

#include "cq.h"
#include "cq_device.cuh"

namespace cq {
namespace {

constexpr int kStageWarps = 4;   // warps per CTA of the staged kernels
constexpr int kStageCtas = 6;    // AbsMax: CTAs per SM its shared-memory staging allows (registers capped to fit)
constexpr int kRowPitch = 272;   // bytes per staged 256-byte row: the 16-byte pad puts the 16-byte reads
                                 // of 8 consecutive rows (one shared-memory phase) on disjoint banks
constexpr int kStageBytes = 32 * kRowPitch;

// Stage 32 rows of 128 binary16 weights (row r at W + row_of(r) * 128, rows
// r >= n skipped) into shared memory: 16 coalesced 16-byte loads per lane in
// two batches of 8 (4 KB in flight per warp), streaming past L1.
template <typename RowOf>
__device__ __forceinline__ void stage_rows(uint8_t *sm, const uint16_t *__restrict__ W, int n, int lane,
                                           RowOf row_of)
{
#pragma unroll
    for (int half = 0; half < 2; half++) {
        uint4 v[8];
#pragma unroll
        for (int k = 0; k < 8; k++) {
            const int c = (8 * half + k) * 32 + lane, r = c >> 4;
            v[k] = (r < n) ? __ldcs(reinterpret_cast<const uint4 *>(W + row_of(r) * kGroup) + (c & 15))
                           : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int k = 0; k < 8; k++) {
            const int c = (8 * half + k) * 32 + lane;
            *reinterpret_cast<uint4 *>(sm + (c >> 4) * kRowPitch + (c & 15) * 16) = v[k];
        }
    }
}

// stage_rows with asynchronous copies (global -> shared, bypassing L1): all 16
// of a lane's 16-byte copies in flight at once and no registers held; rows
// r >= n are zero-filled (source size 0).
template <typename RowOf>
__device__ __forceinline__ void stage_rows_async(uint8_t *sm, const uint16_t *__restrict__ W, int n, int lane,
                                                 RowOf row_of)
{
#pragma unroll
    for (int k = 0; k < 16; k++) {
        const int c = k * 32 + lane, r = c >> 4;
        const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(sm + r * kRowPitch + (c & 15) * 16));
        const uint16_t *src = (r < n) ? W + row_of(r) * kGroup + (c & 15) * 8 : W;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(r < n ? 16 : 0)
                     : "memory");
    }
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// min(round-half-even(aw / s), cap) for aw >= 0, exact.  The estimate
// aw * (1/s) is within one of the answer; adding 1.5 * 2^23 rounds it to the
// nearest integer (ties even) in the low mantissa bits.  Near a half-integer
// the exact threshold tests s (n -+ 1/2) (11-bit s times a 5-bit factor)
// decide instead.
__device__ __forceinline__ int code_of(float aw, float s, float inv, int cap)
{
    constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
    const float x = fminf(aw * inv, 15.0f);
    const float y = x + kRound;
    const float n = y - kRound;
    const int ni = __float_as_int(y) - 0x4B400000;
    // x is within 15 * 2^-23 of aw / s, so away from a half-integer its own
    // rounding is the exact one (x - n is exact)
    if (fabsf(fabsf(x - n) - 0.5f) > 0x1p-12f)
        return min(ni, cap);
    const float lo = s * (n - 0.5f), hi = s * (n + 0.5f);
    const bool odd = ni & 1;
    const int below = (aw < lo || (aw == lo && odd)) ? 1 : 0;  // rne < n
    const int above = (aw > hi || (aw == hi && odd)) ? 1 : 0;  // rne > n
    return min(ni - below + above, cap);
}

// Codes of the 8 weights in one 16-byte chunk (binary16 bits, two per word)
// at scale s, packed as (q + 8) nibbles low first.  Fast path: the signed
// estimate x = w * (1/s) is within 9 * 2^-23 of w / s, and adding 1.5 * 2^23
// rounds it to the nearest integer n (ties even) in the low mantissa bits; away
// from a half-integer that n is the exact round-half-even of w / s, and the
// clip to [-8, 7] follows.  When any of the 8 lies within 2^-12 of a
// half-integer, the chunk is redone with the exact threshold tests of code_of.
__device__ __forceinline__ uint32_t code_word(uint4 v, float s, float inv)
{
    constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
    const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
    uint32_t word = 0;
    bool near = false;
#pragma unroll
    for (int h = 0; h < 8; h++) {
        const uint32_t b = (wd[h >> 1] >> (16 * (h & 1))) & 0xFFFFu;
        const float x = __half2float(__ushort_as_half(static_cast<unsigned short>(b))) * inv;
        const float y = x + kRound;
        const int n = __float_as_int(y) - 0x4B400000;
        near |= fabsf(fabsf(x - (y - kRound)) - 0.5f) <= 0x1p-12f;
        const int q = min(max(n, -8), 7);
        word |= static_cast<uint32_t>((q & 0xF) ^ 8) << (4 * h);
    }
    if (near) {
        word = 0;
#pragma unroll
        for (int h = 0; h < 8; h++) {
            const uint32_t b = (wd[h >> 1] >> (16 * (h & 1))) & 0xFFFFu;
            const bool neg = b & 0x8000u;
            const int c = code_of(half_value(b & 0x7FFFu), s, inv, neg ? 8 : 7);
            word |= static_cast<uint32_t>(((neg ? -c : c) + 8) & 0xF) << (4 * h);
        }
    }
    return word;
}

// The signed codes q of the 8 weights of one 16-byte chunk at scale s, by the
// fast path of code_word (estimate, magic-constant rounding, clip to [-8, 7]),
// redone with the exact threshold tests when any lies within 2^-12 of a
// half-integer.
__device__ __forceinline__ void codes8(uint4 v, float s, float inv, int (&q)[8])
{
    constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
    const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
    bool near = false;
#pragma unroll
    for (int h = 0; h < 8; h++) {
        const uint32_t b = (wd[h >> 1] >> (16 * (h & 1))) & 0xFFFFu;
        const float x = __half2float(__ushort_as_half(static_cast<unsigned short>(b))) * inv;
        const float y = x + kRound;
        near |= fabsf(fabsf(x - (y - kRound)) - 0.5f) <= 0x1p-12f;
        q[h] = min(max(__float_as_int(y) - 0x4B400000, -8), 7);
    }
    if (near) {
#pragma unroll
        for (int h = 0; h < 8; h++) {
            const uint32_t b = (wd[h >> 1] >> (16 * (h & 1))) & 0xFFFFu;
            const bool neg = b & 0x8000u;
            const int c = code_of(half_value(b & 0x7FFFu), s, inv, neg ? 8 : 7);
            q[h] = neg ? -c : c;
        }
    }
}

// code_word for an AbsMax scale in the normal binary16 range: then
// |w| / s <= 7 / (1 - 2^-11) < 7.5 for every weight of the group, so every code
// is already in [-7, 7] and needs no clip.  Two weights go through each step:
// their estimates' rounded integers sit in the low halves of y, which one byte
// permute packs; (n & 15) ^ 8 forms both nibbles at once.  near is set when a
// weight lies within 2^-12 of a half-integer (the caller then takes code_word).
__device__ __forceinline__ uint32_t code_word_unclipped(uint4 v, float inv, bool &near)
{
    constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
    const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
    float dmax = 0.0f;
    uint32_t b[4];
#pragma unroll
    for (int p = 0; p < 4; p++) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&wd[p]));
        const float x0 = f.x * inv, x1 = f.y * inv;
        const float y0 = x0 + kRound, y1 = x1 + kRound;
        dmax = fmaxf(dmax, fmaxf(fabsf(x0 - (y0 - kRound)), fabsf(x1 - (y1 - kRound))));
        const uint32_t nb = (__byte_perm(__float_as_uint(y0), __float_as_uint(y1), 0x5410) & 0x000F000Fu) ^ 0x00080008u;
        b[p] = nb | (nb >> 12);  // byte 0: the pair's two nibbles, low weight first
    }
    near = dmax >= 0.5f - 0x1p-12f;
    return __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
}

// AbsMax: s = binary16 nearest (ties even) to max_i |w_i| / 7 computed in
// fp64, raised to the smallest positive pattern when it rounds to 0; codes are
// the quantiser's at s.  Non-finite weights give scale 0x0001 and zero codes,
// as in the minimax kernel.  One thread per group; each warp stages 32
// consecutive groups and writes their codes back as contiguous 16-byte stores.
__global__ void __launch_bounds__(kStageWarps * 32, kStageCtas) absmax_kernel(const uint16_t *__restrict__ W, int64_t G,
                                                                  uint16_t *__restrict__ out_scales,
                                                                  uint32_t *__restrict__ out_codes)
{
    __shared__ __align__(16) uint8_t stage[kStageWarps][kStageBytes];
    const int lane = threadIdx.x & 31;
    uint8_t *sm = stage[threadIdx.x >> 5];
    uint8_t *row = sm + lane * kRowPitch;
    const int64_t chunks = (G + 31) / 32;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * kStageWarps + (threadIdx.x >> 5); t < chunks;
         t += static_cast<int64_t>(gridDim.x) * kStageWarps) {
        const int64_t g0 = t * 32;
        const int n = static_cast<int>(min(static_cast<int64_t>(32), G - g0));
        __syncwarp();
        stage_rows_async(sm, W, n, lane, [g0](int r) { return g0 + r; });
        if (lane == 0) {
            // the warp's chunk two strides ahead into L2 (on the first pass the next one too),
            // one 8 KB bulk prefetch each, while this one is computed
            const int64_t step = static_cast<int64_t>(gridDim.x) * kStageWarps * 32;
            if (g0 + 2 * step + 32 <= G)
                asm volatile("cp.async.bulk.prefetch.L2.global [%0], 8192;" ::"l"(W + (g0 + 2 * step) * kGroup)
                             : "memory");
            if (g0 < step && g0 + step + 32 <= G)
                asm volatile("cp.async.bulk.prefetch.L2.global [%0], 8192;" ::"l"(W + (g0 + step) * kGroup)
                             : "memory");
        }
        __syncwarp();
        if (lane < n) {
            uint32_t m2 = 0;
#pragma unroll
            for (int j = 0; j < 16; j++) {
                const uint4 v = *reinterpret_cast<const uint4 *>(row + j * 16);
                m2 = __vmaxu2(m2, __vmaxu2(__vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu),
                                           __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu)));
            }
            const uint32_t mag = max(m2 & 0xFFFFu, m2 >> 16);
            uint32_t sbits = 1u;
            if (mag < kBeyond) {
                const double amax = static_cast<double>(half_value(mag));
                sbits = min(max(static_cast<uint32_t>(__half_as_ushort(__double2half(amax / 7.0))), 1u), kLast);
            }
            const float s = grid_value(sbits);
            const float inv = 1.0f / s;
            // code word j (8 nibbles) overwrites bytes 4j..4j+3 of the row, which chunk j has already passed
            if (sbits >= 0x400u && mag < kBeyond) {
#pragma unroll 4
                for (int j = 0; j < 16; j++) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(row + j * 16);
                    bool near;
                    uint32_t word = code_word_unclipped(v, inv, near);
                    if (near)
                        word = code_word(v, s, inv);
                    *reinterpret_cast<uint32_t *>(row + 4 * j) = word;
                }
            } else {
#pragma unroll 4
                for (int j = 0; j < 16; j++) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(row + j * 16);
                    *reinterpret_cast<uint32_t *>(row + 4 * j) = mag < kBeyond ? code_word(v, s, inv) : 0x88888888u;
                }
            }
            out_scales[g0 + lane] = static_cast<uint16_t>(sbits);
        }
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 4; k++) {
            const int c = k * 32 + lane, r = c >> 2;
            if (r < n)
                reinterpret_cast<uint4 *>(out_codes + (g0 + r) * 16)[c & 3] =
                    *reinterpret_cast<const uint4 *>(sm + r * kRowPitch + (c & 3) * 16);
        }
    }
}

// Pooled diagonals: out[i] = fp32 of (sum over e ascending of d_{e,i}, in
// fp64) / E, rounded to nearest even.
__global__ void pool_kernel(const float *__restrict__ D, int E, int64_t n, float *__restrict__ out)
{
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
        double acc = 0.0;
        for (int e = 0; e < E; e++)
            acc = __dadd_rn(acc, static_cast<double>(D[e * n + i]));
        out[i] = __double2float_rn(__ddiv_rn(acc, static_cast<double>(E)));
    }
}

// Objective of given scales: per_env[g][e] = sum_i d_{e,i} (w_i - s q_i)^2 in
// fp64, the products and sums rounded in the definition's own order (i
// ascending, r = w - s q exact, then r*r, then d*rr, then the running sum; no
// contraction), and out[g] = max_e of those.  One thread per group.
//
// Per-column diagonals (K > 0): a CTA takes 128 rows of one column block, so
// all its threads share that block's diagonals, which it stages once in fp64
// and reads back as broadcasts.  Per-group diagonals (K == 0): a warp takes 32
// consecutive groups and each thread streams its own.
template <int E, bool kPerColumn>
__global__ void __launch_bounds__(kStageWarps * 32) objective_kernel(const uint16_t *__restrict__ W, int64_t G,
                                                                     const float *__restrict__ D, int64_t K,
                                                                     const uint16_t *__restrict__ scales,
                                                                     double *__restrict__ per_env,
                                                                     double *__restrict__ out)
{
    __shared__ __align__(16) uint8_t stage[kStageWarps][kStageBytes];
    __shared__ double dstage[kPerColumn ? E : 1][kGroup];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    uint8_t *sm = stage[wid];
    const uint8_t *row = sm + lane * kRowPitch;
    const int64_t gpr = kPerColumn ? K / kGroup : 1;
    const int64_t rows = G / gpr;
    constexpr int kRowsPerItem = kPerColumn ? 32 * kStageWarps : 32;
    const int64_t items = kPerColumn ? ((rows + kRowsPerItem - 1) / kRowsPerItem) * gpr : (G + 31) / 32;
    const int64_t first = kPerColumn ? blockIdx.x : static_cast<int64_t>(blockIdx.x) * kStageWarps + wid;
    const int64_t step = kPerColumn ? gridDim.x : static_cast<int64_t>(gridDim.x) * kStageWarps;
    for (int64_t t = first; t < items; t += step) {
        const int64_t cb = kPerColumn ? t % gpr : 0;
        const int64_t r0 = kPerColumn ? (t / gpr) * kRowsPerItem + 32 * wid : t * 32;
        const int n = static_cast<int>(max(min(static_cast<int64_t>(32), (kPerColumn ? rows : G) - r0),
                                           static_cast<int64_t>(0)));
        if (kPerColumn) {
            __syncthreads();  // the previous item's diagonals are no longer read
            for (int e = wid; e < E; e += kStageWarps) {
                const float4 d4 = __ldg(reinterpret_cast<const float4 *>(D + e * K + cb * kGroup) + lane);
                dstage[e][4 * lane] = d4.x;
                dstage[e][4 * lane + 1] = d4.y;
                dstage[e][4 * lane + 2] = d4.z;
                dstage[e][4 * lane + 3] = d4.w;
            }
        }
        __syncwarp();
        stage_rows(sm, W, n, lane, [=](int r) { return (r0 + r) * gpr + cb; });
        if (kPerColumn)
            __syncthreads();
        else
            __syncwarp();
        if (lane >= n)
            continue;
        const int64_t g = (r0 + lane) * gpr + cb;
        const float s = grid_value(scales[g]);
        const float inv = 1.0f / s;
        const double nsd = -static_cast<double>(s);
        double acc[E];
#pragma unroll
        for (int e = 0; e < E; e++)
            acc[e] = 0.0;
        const float *dg = kPerColumn ? nullptr : D + g * kGroup;
#pragma unroll 1
        for (int j = 0; j < 16; j++) {
            const uint4 v = *reinterpret_cast<const uint4 *>(row + j * 16);
            const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
            int qc[8];
            codes8(v, s, inv, qc);
#pragma unroll
            for (int h = 0; h < 8; h++) {
                const uint32_t bits = (wd[h >> 1] >> (16 * (h & 1))) & 0xFFFFu;
                const double r = fma(nsd, static_cast<double>(qc[h]), static_cast<double>(half_value(bits)));
                const double rr = __dmul_rn(r, r);
#pragma unroll
                for (int e = 0; e < E; e++) {
                    const double d = kPerColumn ? dstage[e][8 * j + h]
                                                : static_cast<double>(__ldcs(dg + e * G * kGroup + 8 * j + h));
                    acc[e] = __dadd_rn(acc[e], __dmul_rn(d, rr));
                }
            }
        }
        double f = acc[0];
#pragma unroll
        for (int e = 0; e < E; e++) {
            per_env[g * E + e] = acc[e];
            if (acc[e] > f)
                f = acc[e];
        }
        out[g] = f;
    }
}

// Reconstruction proxy, first step: one CTA per module m (groups
// offsets[m] .. offsets[m+1]-1).  Each thread sums a strided subset of the
// module's groups for every environment, then a fixed-order tree combines the
// threads, so the result depends only on the input.  module_env[m][e] =
// scale * sum / count; module_worst[m] = max_e of those.  Offsets are clamped to
// [0, G], so no read leaves per_env; an empty module gives 0/0 = NaN.
constexpr int kProxyThreads = 128;
__global__ void __launch_bounds__(kProxyThreads) module_env_kernel(const double *__restrict__ per_env, int64_t G,
                                                                   int E, const int64_t *__restrict__ offsets,
                                                                   double scale,
                                                                   double *__restrict__ module_env,
                                                                   double *__restrict__ module_worst)
{
    __shared__ double red[CQ_MAX_E][kProxyThreads];
    const int m = blockIdx.x;
    const int64_t g1 = min(max(offsets[m + 1], static_cast<int64_t>(0)), G);
    const int64_t g0 = min(max(offsets[m], static_cast<int64_t>(0)), g1);
    double acc[CQ_MAX_E];
#pragma unroll
    for (int e = 0; e < CQ_MAX_E; e++)
        acc[e] = 0.0;
    for (int64_t g = g0 + threadIdx.x; g < g1; g += kProxyThreads) {
#pragma unroll
        for (int e = 0; e < CQ_MAX_E; e++)
            if (e < E)
                acc[e] += per_env[g * E + e];
    }
#pragma unroll
    for (int e = 0; e < CQ_MAX_E; e++)
        red[e][threadIdx.x] = acc[e];
    __syncthreads();
    for (int w = kProxyThreads / 2; w > 0; w >>= 1) {
        if (threadIdx.x < w)
            for (int e = 0; e < E; e++)
                red[e][threadIdx.x] += red[e][threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        const double count = static_cast<double>(g1 - g0);
        double worst = 0.0;
        for (int e = 0; e < E; e++) {
            const double v = red[e][0] / count * scale;
            module_env[static_cast<int64_t>(m) * E + e] = v;
            worst = (e == 0 || v > worst || v != v) ? v : worst;
        }
        module_worst[m] = worst;
    }
}

// Second step: macro[0] = mean over modules of module_worst, one CTA, the same
// fixed-order reduction.
__global__ void __launch_bounds__(kProxyThreads) macro_mean_kernel(const double *__restrict__ module_worst,
                                                                   int64_t nmod, double *__restrict__ macro)
{
    __shared__ double red[kProxyThreads];
    double acc = 0.0;
    for (int64_t m = threadIdx.x; m < nmod; m += kProxyThreads)
        acc += module_worst[m];
    red[threadIdx.x] = acc;
    __syncthreads();
    for (int w = kProxyThreads / 2; w > 0; w >>= 1) {
        if (threadIdx.x < w)
            red[threadIdx.x] += red[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0)
        macro[0] = red[0] / static_cast<double>(nmod);
}

int sms_of_current()
{
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

bool is_aligned(const void *p, size_t a)
{
    return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

// Grid of a grid-stride kernel over `chunks` warp-sized work items: as many
// CTAs as fit on the device at once, fewer when there is less work.
template <typename Kernel>
unsigned resident_grid(Kernel kernel, int64_t chunks, int chunks_per_cta = kStageWarps)
{
    int per_sm = 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kStageWarps * 32, 0) != cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    const int64_t cap = static_cast<int64_t>(sms_of_current()) * per_sm;
    const int64_t need = (chunks + chunks_per_cta - 1) / chunks_per_cta;
    return static_cast<unsigned>(need < cap ? need : cap);
}

template <int E>
cudaError_t launch_objective(const uint16_t *W, int64_t G, const float *D, int64_t K, const uint16_t *scales,
                             double *per_env, double *out, cudaStream_t st)
{
    if (K > 0) {
        const int64_t rows_per_item = 32 * kStageWarps;
        const int64_t items = ((G / (K / kGroup) + rows_per_item - 1) / rows_per_item) * (K / kGroup);
        auto k = objective_kernel<E, true>;
        k<<<resident_grid(k, items, 1), kStageWarps * 32, 0, st>>>(W, G, D, K, scales, per_env, out);
    } else {
        auto k = objective_kernel<E, false>;
        k<<<resident_grid(k, (G + 31) / 32), kStageWarps * 32, 0, st>>>(W, G, D, K, scales, per_env, out);
    }
    return cudaGetLastError();
}

}  // namespace
}  // namespace cq

using namespace cq;

extern "C" {

cq_status cq_absmax_scales(const uint16_t *W, int64_t G, uint16_t *out_scales, uint32_t *out_codes, void *stream)
{
    if (G < 0)
        return CQ_ERR_INVALID_ARG;
    if (G >= (static_cast<int64_t>(1) << 32))
        return CQ_ERR_UNSUPPORTED;
    if (G == 0)
        return CQ_OK;
    if (!W || !out_scales || !out_codes || !is_aligned(W, 16) || !is_aligned(out_codes, 16) ||
        !is_aligned(out_scales, 2))
        return CQ_ERR_INVALID_ARG;
    absmax_kernel<<<resident_grid(absmax_kernel, (G + 31) / 32), kStageWarps * 32, 0,
                    static_cast<cudaStream_t>(stream)>>>(W, G, out_scales, out_codes);
    return cudaGetLastError() == cudaSuccess ? CQ_OK : CQ_ERR_CUDA;
}

cq_status cq_pool_diagonals(const float *D, int E, int64_t n, float *out, void *stream)
{
    if (E < 1 || n < 0)
        return CQ_ERR_INVALID_ARG;
    if (E > CQ_MAX_E)
        return CQ_ERR_UNSUPPORTED;
    if (n == 0)
        return CQ_OK;
    if (!D || !out)
        return CQ_ERR_INVALID_ARG;
    int64_t blocks = (n + 255) / 256;
    const int64_t cap = static_cast<int64_t>(sms_of_current()) * 8;
    if (blocks > cap)
        blocks = cap;
    pool_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(D, E, n, out);
    return cudaGetLastError() == cudaSuccess ? CQ_OK : CQ_ERR_CUDA;
}

cq_status cq_group_objective(const uint16_t *W, int64_t G, const float *D, int E, int64_t K, const uint16_t *scales,
                             double *per_env, double *out_objective, void *stream)
{
    if (G < 0 || K < 0 || E < 1)
        return CQ_ERR_INVALID_ARG;
    if (E > CQ_MAX_E || G >= (static_cast<int64_t>(1) << 32))
        return CQ_ERR_UNSUPPORTED;
    if (K > 0 && (K % kGroup != 0 || G % (K / kGroup) != 0))
        return CQ_ERR_INVALID_ARG;
    if (G == 0)
        return CQ_OK;
    if (!W || !D || !scales || !per_env || !out_objective || !is_aligned(W, 16) || !is_aligned(D, 16) ||
        !is_aligned(scales, 2) || !is_aligned(per_env, 8) || !is_aligned(out_objective, 8))
        return CQ_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t err = cudaErrorInvalidValue;
    switch (E) {
    case 1: err = launch_objective<1>(W, G, D, K, scales, per_env, out_objective, st); break;
    case 2: err = launch_objective<2>(W, G, D, K, scales, per_env, out_objective, st); break;
    case 3: err = launch_objective<3>(W, G, D, K, scales, per_env, out_objective, st); break;
    case 4: err = launch_objective<4>(W, G, D, K, scales, per_env, out_objective, st); break;
    case 5: err = launch_objective<5>(W, G, D, K, scales, per_env, out_objective, st); break;
    case 6: err = launch_objective<6>(W, G, D, K, scales, per_env, out_objective, st); break;
    case 7: err = launch_objective<7>(W, G, D, K, scales, per_env, out_objective, st); break;
    case 8: err = launch_objective<8>(W, G, D, K, scales, per_env, out_objective, st); break;
    default: break;
    }
    return err == cudaSuccess ? CQ_OK : CQ_ERR_CUDA;
}

cq_status cq_reconstruction_proxy(const double *per_env, int64_t G, int E, int64_t nmod, const int64_t *offsets,
                                  double scale, double *module_env, double *module_worst, double *macro, void *stream)
{
    if (G < 0 || E < 1 || nmod < 0 || !(scale == scale))
        return CQ_ERR_INVALID_ARG;
    if (E > CQ_MAX_E || nmod >= (static_cast<int64_t>(1) << 31))
        return CQ_ERR_UNSUPPORTED;
    if (nmod == 0)
        return CQ_OK;
    if ((G > 0 && !per_env) || !offsets || !module_env || !module_worst || !macro || !is_aligned(per_env, 8) ||
        !is_aligned(offsets, 8) || !is_aligned(module_env, 8) || !is_aligned(module_worst, 8) ||
        !is_aligned(macro, 8))
        return CQ_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    module_env_kernel<<<static_cast<unsigned>(nmod), kProxyThreads, 0, st>>>(per_env, G, E, offsets, scale,
                                                                             module_env, module_worst);
    if (cudaGetLastError() != cudaSuccess)
        return CQ_ERR_CUDA;
    macro_mean_kernel<<<1, kProxyThreads, 0, st>>>(module_worst, nmod, macro);
    return cudaGetLastError() == cudaSuccess ? CQ_OK : CQ_ERR_CUDA;
}

}  // extern "C"
