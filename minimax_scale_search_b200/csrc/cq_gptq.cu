// GPTQ v1 tensors from the selection's output, and their dequantisation.
//
// CliffQuant project page and the model card, "Quantization configuration":
// the release is a GPTQ v1 checkpoint, 4-bit, group size 128, symmetric,
// act-order off.  Layout (public GPTQ v1 format) for a linear layer with
// weight [R, K], R output features and K input features:
//   qweight int32 [K/8][R]     word (k, r): inputs 8k..8k+7 of output r, input 8k+j in bits 4j..4j+3
//   qzeros  int32 [K/128][R/8] word (g, c): zero points of outputs 8c..8c+7, stored minus one
//   scales  fp16  [K/128][R]
//   g_idx   int32 [K]          i / 128
// and w[r][i] = scales[g][r] * (u - (z + 1)) with g = g_idx[i].
//
// The selection's codes of group (r, c) are 16 words of 8 input-adjacent
// nibbles (q + 8), low nibble first: word j of group (r, c) is exactly
// qweight[16c + j][r].  So the export is a transpose of the [R][K/8] word
// matrix, a transpose of the [R][K/128] scale matrix and two constant fills,
// all HBM-bound and done by one launch: the transposes run as 64 x 64 tiles
// through shared memory (reads and writes both coalesced, 256-byte runs; the
// words with 16-byte accesses), the dequantiser as 32 x 32.

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "cq.h"

namespace cq {
namespace {

constexpr int kTile = 32;
constexpr int kDequantRows = 4;      // dequantisation: CTA of 32 x 4 threads, 8 words per thread; registers
                                     // capped so 8 CTAs fit per SM

constexpr int kBigTile = 64;         // transpose tile edge
constexpr int kBigRows = 4;          // CTA of 64 x 4 threads, 16 elements per thread

// dst[c][r] = src[r][c] for an [rows][cols] matrix, one 64 x 64 tile per CTA
// iteration (grid-stride over tiles): every row segment read and written is
// 64 elements long, and a thread has 16 loads in flight.  The export takes
// this path (three launches) only when the code words or qweight are not
// 16-byte aligned.
template <typename T>
__global__ void __launch_bounds__(kBigTile * kBigRows) transpose_kernel(const T *__restrict__ src, int64_t rows,
                                                                       int64_t cols, T *__restrict__ dst)
{
    __shared__ T tile[kBigTile][kBigTile + 1];
    const int64_t tiles_c = (cols + kBigTile - 1) / kBigTile;
    const int64_t tiles = ((rows + kBigTile - 1) / kBigTile) * tiles_c;
    const int tx = threadIdx.x, ty = threadIdx.y;
    for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x) {
        const int64_t r0 = (t / tiles_c) * kBigTile, c0 = (t % tiles_c) * kBigTile;
        __syncthreads();
#pragma unroll
        for (int k = 0; k < kBigTile; k += kBigRows) {
            const int64_t r = r0 + ty + k, c = c0 + tx;
            if (r < rows && c < cols)
                tile[ty + k][tx] = src[r * cols + c];
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < kBigTile; k += kBigRows) {
            const int64_t c = c0 + ty + k, r = r0 + tx;
            if (r < rows && c < cols)
                dst[c * rows + r] = tile[tx][ty + k];
        }
    }
}

// The whole export in one launch.  CTA iterations [0, tw) transpose 64 x 64
// tiles of code words with 16-byte loads and stores (4 per thread per tile);
// [tw, tw + ts) transpose 64 x 64 tiles of scales; then every thread joins a
// grid-stride fill of qzeros and g_idx.  R % 8 == 0 and K8 % 16 == 0 keep every
// 16-byte access inside its row.
constexpr int kExportThreads = 256;

__global__ void __launch_bounds__(kExportThreads) export_kernel(const uint32_t *__restrict__ codes,
                                                                const uint16_t *__restrict__ scales, int64_t R,
                                                                int64_t K, uint32_t *__restrict__ qweight,
                                                                uint16_t *__restrict__ gscales,
                                                                int32_t *__restrict__ qzeros, int32_t *__restrict__ g_idx)
{
    __shared__ uint32_t tile[kBigTile][kBigTile + 1];
    const int64_t K8 = K / 8, ng = K / 128;
    const int64_t tr = (R + kBigTile - 1) / kBigTile;
    const int64_t twc = (K8 + kBigTile - 1) / kBigTile, tsc = (ng + kBigTile - 1) / kBigTile;
    const int64_t tw = tr * twc, ts = tr * tsc;
    const int tid = threadIdx.x;
    for (int64_t t = blockIdx.x; t < tw + ts; t += gridDim.x) {
        __syncthreads();
        if (t < tw) {
            const int64_t r0 = (t / twc) * kBigTile, c0 = (t % twc) * kBigTile;
            uint4 v[4];
#pragma unroll
            for (int k = 0; k < 4; k++) {
                const int i = tid + kExportThreads * k, r = i >> 4, c4 = i & 15;
                const int64_t gr = r0 + r, gc = c0 + 4 * c4;
                v[k] = (gr < R && gc < K8) ? __ldcs(reinterpret_cast<const uint4 *>(codes + gr * K8 + gc))
                                           : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int k = 0; k < 4; k++) {
                const int i = tid + kExportThreads * k, r = i >> 4, c4 = i & 15;
                tile[r][4 * c4] = v[k].x;
                tile[r][4 * c4 + 1] = v[k].y;
                tile[r][4 * c4 + 2] = v[k].z;
                tile[r][4 * c4 + 3] = v[k].w;
            }
            __syncthreads();
#pragma unroll
            for (int k = 0; k < 4; k++) {
                const int i = tid + kExportThreads * k, c = i >> 4, r4 = i & 15;
                const int64_t gc = c0 + c, gr = r0 + 4 * r4;
                if (gc < K8 && gr < R)
                    *reinterpret_cast<uint4 *>(qweight + gc * R + gr) =
                        make_uint4(tile[4 * r4][c], tile[4 * r4 + 1][c], tile[4 * r4 + 2][c], tile[4 * r4 + 3][c]);
            }
        } else {
            const int64_t u = t - tw;
            const int64_t r0 = (u / tsc) * kBigTile, c0 = (u % tsc) * kBigTile;
            const int tx = tid & 63, ty = tid >> 6;
#pragma unroll
            for (int k = 0; k < kBigTile; k += 4) {
                const int64_t r = r0 + ty + k, c = c0 + tx;
                if (r < R && c < ng)
                    tile[ty + k][tx] = scales[r * ng + c];
            }
            __syncthreads();
#pragma unroll
            for (int k = 0; k < kBigTile; k += 4) {
                const int64_t c = c0 + ty + k, r = r0 + tx;
                if (r < R && c < ng)
                    gscales[c * R + r] = static_cast<uint16_t>(tile[tx][ty + k]);
            }
        }
    }
    const int64_t nz = ng * (R / 8);
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kExportThreads;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * kExportThreads + tid; i < nz + K; i += stride) {
        if (i < nz)
            qzeros[i] = 0x77777777;
        else
            g_idx[i - nz] = static_cast<int32_t>((i - nz) / 128);
    }
}

// qzeros = 0x77777777 (zero point 8, stored minus one) and g_idx[i] = i / 128.
__global__ void fill_kernel(int32_t *__restrict__ qzeros, int64_t nz, int32_t *__restrict__ g_idx, int64_t K)
{
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nz + K; i += stride) {
        if (i < nz)
            qzeros[i] = 0x77777777;
        else
            g_idx[i - nz] = static_cast<int32_t>((i - nz) / 128);
    }
}

__device__ __forceinline__ int64_t clamp_group(int g, int64_t ngroups)
{
    return g < 0 ? 0 : (g >= ngroups ? ngroups - 1 : g);
}

// Dequantisation, one 32 (words along k) x 32 (outputs) tile per CTA
// iteration: the tile's qweight words are read coalesced along r, then each
// lane writes the 8 values of one word, so a warp stores 256 consecutive
// values of one output row.  Group indices outside [0, K/128) are clamped.
template <bool kHalf>
__global__ void __launch_bounds__(kTile * kDequantRows, 8) dequant_kernel(const uint32_t *__restrict__ qweight,
                                                                          const uint32_t *__restrict__ qzeros,
                                                                          const uint16_t *__restrict__ scales,
                                                                          const int32_t *__restrict__ g_idx,
                                                                          int64_t R, int64_t K, void *__restrict__ out)
{
    __shared__ uint32_t tile[kTile][kTile + 1];
    const int64_t K8 = K / 8, ngroups = K / 128;
    const int64_t tiles_r = (R + kTile - 1) / kTile;
    const int64_t tiles = ((K8 + kTile - 1) / kTile) * tiles_r;
    const int tx = threadIdx.x, ty = threadIdx.y;
    // fp16 output: each thread's words of the next tile are loaded into
    // registers while the current tile is dequantised and stored (the fp32
    // output, twice the bytes per word, was faster without it)
    constexpr int kPer = kTile / kDequantRows;
    uint32_t nxt[kPer];
    auto load = [&](int64_t t) {
        const int64_t k0 = (t / tiles_r) * kTile, r0 = (t % tiles_r) * kTile;
#pragma unroll
        for (int k = 0; k < kPer; k++) {
            const int64_t kk = k0 + ty + k * kDequantRows, r = r0 + tx;
            nxt[k] = (kk < K8 && r < R) ? qweight[kk * R + r] : 0u;
        }
    };
    if (kHalf && static_cast<int64_t>(blockIdx.x) < tiles)
        load(blockIdx.x);
    for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x) {
        const int64_t k0 = (t / tiles_r) * kTile, r0 = (t % tiles_r) * kTile;
        __syncthreads();
        if (kHalf) {
#pragma unroll
            for (int k = 0; k < kPer; k++)
                tile[ty + k * kDequantRows][tx] = nxt[k];
        } else {
#pragma unroll
            for (int k = 0; k < kTile; k += kDequantRows) {
                const int64_t kk = k0 + ty + k, r = r0 + tx;
                if (kk < K8 && r < R)
                    tile[ty + k][tx] = qweight[kk * R + r];
            }
        }
        __syncthreads();
        if (kHalf && t + gridDim.x < tiles)
            load(t + gridDim.x);
        const int64_t kk = k0 + tx;
        if (kk >= K8)
            continue;
        const int4 ga = reinterpret_cast<const int4 *>(g_idx)[2 * kk];
        const int4 gb = reinterpret_cast<const int4 *>(g_idx)[2 * kk + 1];
        const int gi[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
        bool uniform = true;
#pragma unroll
        for (int j = 1; j < 8; j++)
            uniform = uniform && gi[j] == gi[0];
        const int64_t g0 = clamp_group(gi[0], ngroups);
        // fp32 output: the word's scale and zero word for each of this thread's rows,
        // loaded together before the rows (the fp16 output was faster loading them per row)
        uint16_t sbq[kPer];
        uint32_t zwq[kPer];
        if (!kHalf && uniform) {
#pragma unroll
            for (int q = 0; q < kPer; q++) {
                const int64_t r = r0 + ty + q * kDequantRows;
                sbq[q] = r < R ? scales[g0 * R + r] : static_cast<uint16_t>(0);
                zwq[q] = r < R ? qzeros[g0 * (R / 8) + r / 8] : 0u;
            }
        }
#pragma unroll
        for (int k = 0; k < kTile; k += kDequantRows) {
            const int64_t r = r0 + ty + k;
            if (r >= R)
                continue;
            const uint32_t word = tile[tx][ty + k];
            if (kHalf && uniform) {
                const uint16_t sb = scales[g0 * R + r];
                if ((sb & 0x7C00u) != 0x7C00u) {
                    // binary16 arithmetic, two values per step: 0x6400 | u is 1024 + u, so
                    // (1024 + u) - (1024 + z + 1) = u - (z + 1) exactly, and one rounding of
                    // its product with the scale is the fp32 product (exact) rounded to binary16
                    const int z1 = static_cast<int>((qzeros[g0 * (R / 8) + r / 8] >> (4 * (r % 8))) & 0xFu) + 1;
                    const __half2 s2 = __half2half2(__ushort_as_half(sb));
                    const __half2 zz = __half2half2(__ushort_as_half(static_cast<unsigned short>(0x6400 + z1)));
                    uint32_t pr[4];
#pragma unroll
                    for (int j = 0; j < 4; j++) {
                        const uint32_t x = ((word >> (4 * j)) & 0x000F000Fu) | 0x64006400u;  // values j and j + 4
                        const __half2 p = __hmul2(__hsub2(*reinterpret_cast<const __half2 *>(&x), zz), s2);
                        pr[j] = *reinterpret_cast<const uint32_t *>(&p);
                    }
                    *reinterpret_cast<uint4 *>(static_cast<__half *>(out) + r * K + 8 * kk) =
                        make_uint4(__byte_perm(pr[0], pr[1], 0x5410), __byte_perm(pr[2], pr[3], 0x5410),
                                   __byte_perm(pr[0], pr[1], 0x7632), __byte_perm(pr[2], pr[3], 0x7632));
                    continue;
                }
            }
            float v[8];
            if (uniform) {  // one group for the word's 8 inputs (always so with act-order off)
                const float s = __half2float(__ushort_as_half(kHalf ? scales[g0 * R + r] : sbq[k / kDequantRows]));
                const int z1 = static_cast<int>(((kHalf ? qzeros[g0 * (R / 8) + r / 8] : zwq[k / kDequantRows]) >>
                                                 (4 * (r % 8))) & 0xFu) + 1;
#pragma unroll
                for (int j = 0; j < 8; j++)
                    v[j] = s * static_cast<float>(static_cast<int>((word >> (4 * j)) & 0xFu) - z1);
            } else {
#pragma unroll
                for (int j = 0; j < 8; j++) {
                    const int64_t g = clamp_group(gi[j], ngroups);
                    const float s = __half2float(__ushort_as_half(scales[g * R + r]));
                    const int z = static_cast<int>((qzeros[g * (R / 8) + r / 8] >> (4 * (r % 8))) & 0xFu);
                    const int u = static_cast<int>((word >> (4 * j)) & 0xFu);
                    v[j] = s * static_cast<float>(u - (z + 1));  // exact: 11-bit scale times |n| <= 16
                }
            }
            if (kHalf) {
                uint32_t h[4];
#pragma unroll
                for (int j = 0; j < 4; j++)
                    h[j] = static_cast<uint32_t>(__half_as_ushort(__float2half_rn(v[2 * j]))) |
                           (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(v[2 * j + 1]))) << 16);
                *reinterpret_cast<uint4 *>(static_cast<__half *>(out) + r * K + 8 * kk) =
                    make_uint4(h[0], h[1], h[2], h[3]);
            } else {
                float4 *o = reinterpret_cast<float4 *>(static_cast<float *>(out) + r * K + 8 * kk);
                o[0] = make_float4(v[0], v[1], v[2], v[3]);
                o[1] = make_float4(v[4], v[5], v[6], v[7]);
            }
        }
    }
}

unsigned tile_grid(int64_t tiles)
{
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t cap = static_cast<int64_t>(sms > 0 ? sms : 148) * 16;
    return static_cast<unsigned>(tiles < cap ? tiles : cap);
}

bool aligned(const void *p, size_t a)
{
    return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

cq_status check_shape(int64_t R, int64_t K)
{
    if (R < 0 || K < 0 || K % 128 != 0 || R % 8 != 0)
        return CQ_ERR_INVALID_ARG;
    if (R >= (static_cast<int64_t>(1) << 31) || K >= (static_cast<int64_t>(1) << 31))
        return CQ_ERR_UNSUPPORTED;
    return CQ_OK;
}

}  // namespace
}  // namespace cq

using namespace cq;

extern "C" {

cq_status cq_gptq_export(const uint16_t *scales, const uint32_t *codes, int64_t R, int64_t K, int32_t *qweight,
                         int32_t *qzeros, uint16_t *gptq_scales, int32_t *g_idx, void *stream)
{
    const cq_status st = check_shape(R, K);
    if (st != CQ_OK)
        return st;
    if (R == 0 || K == 0)
        return CQ_OK;
    if (!scales || !codes || !qweight || !qzeros || !gptq_scales || !g_idx || !aligned(scales, 2) ||
        !aligned(codes, 4) || !aligned(qweight, 4) || !aligned(qzeros, 4) || !aligned(gptq_scales, 2) ||
        !aligned(g_idx, 4))
        return CQ_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t K8 = K / 8, ng = K / 128;
    if (aligned(codes, 16) && aligned(qweight, 16)) {
        const int64_t tiles = ((R + 63) / 64) * ((K8 + 63) / 64 + (ng + 63) / 64);
        export_kernel<<<tile_grid(tiles), kExportThreads, 0, s>>>(codes, scales, R, K,
                                                                  reinterpret_cast<uint32_t *>(qweight),
                                                                  gptq_scales, qzeros, g_idx);
        return cudaGetLastError() == cudaSuccess ? CQ_OK : CQ_ERR_CUDA;
    }
    const dim3 block(kBigTile, kBigRows);
    transpose_kernel<uint32_t><<<tile_grid(((R + 63) / 64) * ((K8 + 63) / 64)), block, 0, s>>>(
        codes, R, K8, reinterpret_cast<uint32_t *>(qweight));
    if (cudaGetLastError() != cudaSuccess)
        return CQ_ERR_CUDA;
    transpose_kernel<uint16_t><<<tile_grid(((R + 63) / 64) * ((ng + 63) / 64)), block, 0, s>>>(scales, R, ng,
                                                                                               gptq_scales);
    if (cudaGetLastError() != cudaSuccess)
        return CQ_ERR_CUDA;
    const int64_t nz = ng * (R / 8);
    fill_kernel<<<tile_grid((nz + K + 255) / 256), 256, 0, s>>>(qzeros, nz, g_idx, K);
    return cudaGetLastError() == cudaSuccess ? CQ_OK : CQ_ERR_CUDA;
}

cq_status cq_gptq_dequantize(const int32_t *qweight, const int32_t *qzeros, const uint16_t *gptq_scales,
                             const int32_t *g_idx, int64_t R, int64_t K, int out_fp16, void *out, void *stream)
{
    const cq_status st = check_shape(R, K);
    if (st != CQ_OK)
        return st;
    if (out_fp16 != 0 && out_fp16 != 1)
        return CQ_ERR_INVALID_ARG;
    if (R == 0 || K == 0)
        return CQ_OK;
    if (!qweight || !qzeros || !gptq_scales || !g_idx || !out || !aligned(qweight, 4) || !aligned(qzeros, 4) ||
        !aligned(gptq_scales, 2) || !aligned(g_idx, 16) || !aligned(out, 16))
        return CQ_ERR_INVALID_ARG;
    const dim3 block(kTile, kDequantRows);
    const unsigned grid = tile_grid(((R + 31) / 32) * ((K / 8 + 31) / 32));
    const uint32_t *qw = reinterpret_cast<const uint32_t *>(qweight);
    const uint32_t *qz = reinterpret_cast<const uint32_t *>(qzeros);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (out_fp16)
        dequant_kernel<true><<<grid, block, 0, s>>>(qw, qz, gptq_scales, g_idx, R, K, out);
    else
        dequant_kernel<false><<<grid, block, 0, s>>>(qw, qz, gptq_scales, g_idx, R, K, out);
    return cudaGetLastError() == cudaSuccess ? CQ_OK : CQ_ERR_CUDA;
}

}  // extern "C"
