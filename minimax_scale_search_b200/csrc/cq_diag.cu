// Per-environment sensitivity diagonals from calibration activations.
//
// CliffQuant project page, "What CliffQuant changes" and "The negative result
// that changed the method": the solver's diagonals d_{e,i} are empirical
// activation-weighted sensitivities, one set per calibration environment,
// normalised separately.  For the inputs X_e (N_e tokens x K) of environment e:
//   m_{e,k} = (1 / N_e) sum_t x_{t,k}^2,   d_{e,k} = m_{e,k} / mean_j m_{e,j}.
//
// The column sums stream X once (HBM-bound).  A cluster of 8 CTAs owns one
// (environment, 256-column slab); its 64 warps take interleaved rows, each lane
// 8 adjacent columns (one 16-byte load per row for 16-bit inputs), and
// accumulate x^2 in fp64 with an exact product (x^2 of a bf16, fp16 or fp32
// value fits in 53 bits, so fma(x, x, acc) rounds once, like a plain add).
// Warps combine in shared memory and the 8 CTAs through distributed shared
// memory, both in a fixed order: the result is deterministic and needs no
// scratch in HBM.  A second kernel normalises each environment.

#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "cq.h"

namespace cg = cooperative_groups;

namespace cq {
namespace {

constexpr int kDiagWarps = 8;
constexpr int kDiagThreads = kDiagWarps * 32;
constexpr int kDiagCluster = 8;
constexpr int kSlab = 256;          // columns per cluster: 8 per lane
constexpr int kRowSlots = kDiagCluster * kDiagWarps;
constexpr int kRowUnroll = 4;       // rows in flight per warp

struct EnvRows {
    int64_t off[CQ_MAX_E + 1];
};

// Eight consecutive elements of one row as exact doubles.
template <int DT>
__device__ __forceinline__ void load8(const void *__restrict__ X, int64_t idx, double (&v)[8])
{
    if (DT == CQ_DTYPE_FP32) {
        const float4 a = __ldcs(reinterpret_cast<const float4 *>(static_cast<const float *>(X) + idx));
        const float4 b = __ldcs(reinterpret_cast<const float4 *>(static_cast<const float *>(X) + idx) + 1);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
        const uint4 u = __ldcs(reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(X) + idx));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 8; j++) {
            const uint32_t b = (w[j >> 1] >> (16 * (j & 1))) & 0xFFFFu;
            const float f = (DT == CQ_DTYPE_BF16) ? __uint_as_float(b << 16)
                                                  : __half2float(__ushort_as_half(static_cast<unsigned short>(b)));
            v[j] = static_cast<double>(f);
        }
    }
}

template <int DT>
__global__ void __cluster_dims__(kDiagCluster, 1, 1) __launch_bounds__(kDiagThreads)
    column_squares_kernel(const void *__restrict__ X, int64_t K, int nslabs, EnvRows rows, double *__restrict__ means)
{
    __shared__ double part[kDiagWarps][kSlab];
    __shared__ double cta_sum[kSlab];
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = static_cast<int>(cluster.block_rank());
    const int cid = blockIdx.x / kDiagCluster;
    const int e = cid / nslabs;
    const int64_t col0 = static_cast<int64_t>(cid % nslabs) * kSlab;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int64_t col = col0 + 8 * lane;
    const int64_t a = rows.off[e], b = rows.off[e + 1];
    double acc[8];
#pragma unroll
    for (int j = 0; j < 8; j++)
        acc[j] = 0.0;
    if (col < K) {
        int64_t t = a + rank * kDiagWarps + wid;
        for (; t + (kRowUnroll - 1) * kRowSlots < b; t += kRowUnroll * kRowSlots) {
            double v[kRowUnroll][8];
#pragma unroll
            for (int u = 0; u < kRowUnroll; u++)
                load8<DT>(X, (t + u * kRowSlots) * K + col, v[u]);
#pragma unroll
            for (int u = 0; u < kRowUnroll; u++)
#pragma unroll
                for (int j = 0; j < 8; j++)
                    acc[j] = fma(v[u][j], v[u][j], acc[j]);
        }
        for (; t < b; t += kRowSlots) {
            double v[8];
            load8<DT>(X, t * K + col, v);
#pragma unroll
            for (int j = 0; j < 8; j++)
                acc[j] = fma(v[j], v[j], acc[j]);
        }
    }
#pragma unroll
    for (int j = 0; j < 8; j++)
        part[wid][8 * lane + j] = acc[j];
    __syncthreads();
    double s = 0.0;
#pragma unroll
    for (int w = 0; w < kDiagWarps; w++)
        s += part[w][threadIdx.x];
    cta_sum[threadIdx.x] = s;
    cluster.sync();
    if (rank == 0) {
        double total = 0.0;
#pragma unroll
        for (int r = 0; r < kDiagCluster; r++)
            total += cluster.map_shared_rank(cta_sum, r)[threadIdx.x];
        if (col0 + threadIdx.x < K)
            means[static_cast<int64_t>(e) * K + col0 + threadIdx.x] = total / static_cast<double>(b - a);
    }
    cluster.sync();  // peers keep their shared memory until rank 0 has read it
}

// d[e][k] = fp32(m[e][k] / mean_j m[e][j]), one CTA per environment; the mean
// is a fixed-order sum (strided per thread, then a tree).
__global__ void __launch_bounds__(kDiagThreads) normalise_kernel(const double *__restrict__ means, int64_t K,
                                                                 float *__restrict__ D)
{
    __shared__ double red[kDiagThreads];
    const double *m = means + static_cast<int64_t>(blockIdx.x) * K;
    double s = 0.0;
    for (int64_t k = threadIdx.x; k < K; k += kDiagThreads)
        s += m[k];
    red[threadIdx.x] = s;
    __syncthreads();
    for (int w = kDiagThreads / 2; w > 0; w >>= 1) {
        if (threadIdx.x < w)
            red[threadIdx.x] += red[threadIdx.x + w];
        __syncthreads();
    }
    const double mean = red[0] / static_cast<double>(K);
    float *d = D + static_cast<int64_t>(blockIdx.x) * K;
    for (int64_t k = threadIdx.x; k < K; k += kDiagThreads)
        d[k] = __double2float_rn(m[k] / mean);
}

bool aligned_to(const void *p, size_t a)
{
    return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

}  // namespace
}  // namespace cq

using namespace cq;

extern "C" {

cq_status cq_estimate_diagonals(const void *X, int dtype, int64_t K, const int64_t *row_offsets, int E,
                                double *means, float *D, void *stream)
{
    if (E < 1 || K < 0 || !row_offsets || (dtype != CQ_DTYPE_BF16 && dtype != CQ_DTYPE_FP16 && dtype != CQ_DTYPE_FP32))
        return CQ_ERR_INVALID_ARG;
    if (E > CQ_MAX_E)
        return CQ_ERR_UNSUPPORTED;
    if (K % 8 != 0 || row_offsets[0] < 0)
        return CQ_ERR_INVALID_ARG;
    EnvRows rows;
    for (int e = 0; e <= E; e++) {
        if (e > 0 && row_offsets[e] < row_offsets[e - 1])
            return CQ_ERR_INVALID_ARG;
        rows.off[e] = row_offsets[e];
    }
    if (K == 0)
        return CQ_OK;
    const int64_t nslabs = (K + kSlab - 1) / kSlab;
    if (nslabs * E * kDiagCluster >= (static_cast<int64_t>(1) << 31))
        return CQ_ERR_UNSUPPORTED;
    if ((row_offsets[E] > 0 && (!X || !aligned_to(X, 16))) || !means || !D || !aligned_to(means, 8) ||
        !aligned_to(D, 4))
        return CQ_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const unsigned grid = static_cast<unsigned>(nslabs * E * kDiagCluster);
    const int ns = static_cast<int>(nslabs);
    if (dtype == CQ_DTYPE_BF16)
        column_squares_kernel<CQ_DTYPE_BF16><<<grid, kDiagThreads, 0, st>>>(X, K, ns, rows, means);
    else if (dtype == CQ_DTYPE_FP16)
        column_squares_kernel<CQ_DTYPE_FP16><<<grid, kDiagThreads, 0, st>>>(X, K, ns, rows, means);
    else
        column_squares_kernel<CQ_DTYPE_FP32><<<grid, kDiagThreads, 0, st>>>(X, K, ns, rows, means);
    if (cudaGetLastError() != cudaSuccess)
        return CQ_ERR_CUDA;
    normalise_kernel<<<E, kDiagThreads, 0, st>>>(means, K, D);
    return cudaGetLastError() == cudaSuccess ? CQ_OK : CQ_ERR_CUDA;
}

}  // extern "C"
