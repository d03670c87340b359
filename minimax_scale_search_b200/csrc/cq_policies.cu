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

constexpr int kPolicyWarps = 8;
constexpr int kGroupsPerWarp = 4;  // loads in flight per warp

// AbsMax: s = binary16 nearest (ties even) to max_i |w_i| / 7 computed in
// fp64, raised to the smallest positive pattern when it rounds to 0; codes are
// the quantiser's at s.  Non-finite weights give scale 0x0001 and zero codes,
// as in the minimax kernel.  One warp per group, four groups per iteration.
__global__ void __launch_bounds__(kPolicyWarps * 32) absmax_kernel(const uint16_t *__restrict__ W, int64_t G,
                                                                   uint16_t *__restrict__ out_scales,
                                                                   uint32_t *__restrict__ out_codes)
{
    const int lane = threadIdx.x & 31;
    const int64_t warp = static_cast<int64_t>(blockIdx.x) * kPolicyWarps + (threadIdx.x >> 5);
    const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kPolicyWarps;
    for (int64_t g0 = warp * kGroupsPerWarp; g0 < G; g0 += nwarps * kGroupsPerWarp) {
        uint2 wv[kGroupsPerWarp];
#pragma unroll
        for (int u = 0; u < kGroupsPerWarp; u++)
            wv[u] = (g0 + u < G) ? reinterpret_cast<const uint2 *>(W + (g0 + u) * kGroup)[lane] : make_uint2(0, 0);
#pragma unroll
        for (int u = 0; u < kGroupsPerWarp; u++) {
            const int64_t g = g0 + u;
            if (g >= G)
                break;
            const uint32_t wb[4] = {wv[u].x & 0xFFFFu, wv[u].x >> 16, wv[u].y & 0xFFFFu, wv[u].y >> 16};
            uint32_t mag = 0;
#pragma unroll
            for (int m = 0; m < 4; m++)
                mag = max(mag, wb[m] & 0x7FFFu);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                mag = max(mag, __shfl_xor_sync(kFull, mag, o));
            uint32_t sbits = 1u;
            if (mag < 0x7C00u) {
                const double amax = static_cast<double>(half_value(mag));
                sbits = __half_as_ushort(__double2half(amax / 7.0));
                sbits = min(max(sbits, 1u), kLast);
            }
            const float s = grid_value(sbits);
            uint32_t h = 0;
#pragma unroll
            for (int m = 0; m < 4; m++) {
                int q = 0;
                if (mag < 0x7C00u) {
                    const int aq = abs_code(half_value(wb[m] & 0x7FFFu), s, (wb[m] & 0x8000u) ? 8 : 7);
                    q = (wb[m] & 0x8000u) ? -aq : aq;
                }
                h |= static_cast<uint32_t>((q + 8) & 0xF) << (4 * m);
            }
            const uint32_t up = __shfl_down_sync(kFull, h, 1);
            if ((lane & 1) == 0)
                out_codes[g * 16 + (lane >> 1)] = h | (up << 16);
            if (lane == 0)
                out_scales[g] = static_cast<uint16_t>(sbits);
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

// Objective of given scales: out[g] = max_e sum_i d_{e,i} (w_i - s q_i)^2 in
// fp64, summed over i ascending without contraction (the definition's own
// order).  One thread per (group, environment) pair.
__global__ void objective_kernel(const uint16_t *__restrict__ W, int64_t G, const float *__restrict__ D, int E,
                                 int64_t K, const uint16_t *__restrict__ scales, double *__restrict__ out)
{
    const int64_t pairs = G * E;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t gpr = K > 0 ? K / kGroup : 1;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < pairs; t += stride) {
        const int64_t g = t / E;
        const int e = static_cast<int>(t - g * E);
        const uint16_t *w = W + g * kGroup;
        const float *d = (K > 0) ? D + e * K + (g % gpr) * kGroup : D + (static_cast<int64_t>(e) * G + g) * kGroup;
        const uint32_t sb = scales[g];
        const float s = grid_value(sb);
        const double sd = s;
        double acc = 0.0;
        for (int i = 0; i < kGroup; i++) {
            const uint32_t b = w[i];
            const int aq = abs_code(half_value(b & 0x7FFFu), s, (b & 0x8000u) ? 8 : 7);
            const double q = (b & 0x8000u) ? -static_cast<double>(aq) : static_cast<double>(aq);
            const double r = static_cast<double>(half_value(b)) - sd * q;  // exact
            acc = __dadd_rn(acc, __dmul_rn(static_cast<double>(d[i]), __dmul_rn(r, r)));
        }
        out[t] = acc;
    }
}

__global__ void env_max_kernel(const double *__restrict__ per_env, int64_t G, int E, double *__restrict__ out)
{
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; g < G; g += stride) {
        double f = per_env[g * E];
        for (int e = 1; e < E; e++) {
            const double v = per_env[g * E + e];
            if (v > f)
                f = v;
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
    if (!W || !out_scales || !out_codes || !is_aligned(W, 16) || !is_aligned(out_codes, 4) ||
        !is_aligned(out_scales, 2))
        return CQ_ERR_INVALID_ARG;
    const int64_t warps = (G + kGroupsPerWarp - 1) / kGroupsPerWarp;
    int64_t blocks = (warps + kPolicyWarps - 1) / kPolicyWarps;
    const int64_t cap = static_cast<int64_t>(sms_of_current()) * 8;
    if (blocks > cap)
        blocks = cap;
    absmax_kernel<<<static_cast<unsigned>(blocks), kPolicyWarps * 32, 0, static_cast<cudaStream_t>(stream)>>>(
        W, G, out_scales, out_codes);
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
    if (!W || !D || !scales || !per_env || !out_objective || !is_aligned(per_env, 8) ||
        !is_aligned(out_objective, 8))
        return CQ_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t cap = static_cast<int64_t>(sms_of_current()) * 16;
    int64_t blocks = (G * E + 255) / 256;
    objective_kernel<<<static_cast<unsigned>(blocks < cap ? blocks : cap), 256, 0, st>>>(W, G, D, E, K, scales,
                                                                                          per_env);
    if (cudaGetLastError() != cudaSuccess)
        return CQ_ERR_CUDA;
    blocks = (G + 255) / 256;
    env_max_kernel<<<static_cast<unsigned>(blocks < cap ? blocks : cap), 256, 0, st>>>(per_env, G, E, out_objective);
    return cudaGetLastError() == cudaSuccess ? CQ_OK : CQ_ERR_CUDA;
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
