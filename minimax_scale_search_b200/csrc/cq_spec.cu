// Exact minimax scale selection for a general quantiser spec: codes in
// [qmin, qmax] (qmin <= -1 <= 1 <= qmax) and groups of n <= 1024 weights.
//
// CliffQuant project page, "What CliffQuant changes" (the objective, the
// quantiser and the binary16 scale domain with the lower pattern winning a tie)
// and "Use the solver" (QuantizerSpec(qmin, qmax)).  The warp-per-group kernel
// in cq_select.cu is specialised to (-8, 7) and 128 weights; this path serves
// every other spec with the same result definition.
//
// One warp per group (a grid of one-warp CTAs, grid-stride over groups; many
// groups in flight per SM hide the latency of each group's serial steps):
//  1. stage w (exact fp32 and fp64, and |w| with its code cap) and the group's
//     diagonals per weight (fp64 for the exact sums, fp32 for the chunk bounds);
//  2. U: an upper bound of the smallest objective, from warp-parallel sums at
//     the AbsMax-type scales fp16(max|w|/qmax), fp16(max|w|/|qmin|), their
//     grid neighbours and the first scale at which every code is 0, two
//     scales per pass over the weights;
//  3. a certified window [J0, J1], by two bisections that share one pass over
//     the weights per step: below a scale, the clipped weights' error
//     sum_e-max of sum d (|w| - c s)^2 only grows as s falls; above one, the
//     error of the weights that round to 0, sum d w^2, only grows as s rises.
//     Both are fp64 lower bounds of the exact objective, taken with a 2^-40
//     margin that covers the rounding of either side (n <= 4096), so a scale
//     they exclude has an objective above U and cannot be the minimum or tie it;
//  4. the window in at most 256 chunks of C >= 8 scales (C a power of two),
//     each with an fp32 interval lower bound of the objective, one lane per
//     chunk; chunks whose bound exceeds U are dropped;
//  5. best first: the chunks with the smallest bounds, 32 scales at a time,
//     have every scale evaluated in the definition's own order (i ascending,
//     r = w - s q exact, r*r, d*rr and the running sum rounded separately,
//     environments maxed in order), so each value equals the oracle's bit for
//     bit; a chunk is dropped once its bound exceeds the best value found so
//     far, which leaves every scale in it strictly worse.  Above the first
//     all-zero scale j_z every scale has the same value, so only j_z is
//     evaluated there;
//  6. the (objective, pattern) minimum over the evaluated scales and its codes.
//
// The fp32 bounds assume no fp32 overflow or subnormal result: every term is
// d dist^2 with dist 0 or in [2^-24, 65504], so they are used only when every
// nonzero d lies in [2^-64, 2^80] (terms 0 or in [2^-112, 2^112], sums below
// 2^122); otherwise every chunk's bound is 0 and the scan covers the window.

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cfloat>
#include <cstdint>

#include "cq.h"
#include "cq_device.cuh"

namespace cq {
namespace {

constexpr int kCandidates = 7;
constexpr int kLaneChunks = 8;                 // chunk bounds held per lane: at most 256 chunks
constexpr uint32_t kMinChunk = 8;              // smallest chunk, in scales
constexpr float kKeepChunk = 1.0f - 0x1p-12f;  // covers the fp32 rounding of a bound
constexpr float kTrustLo = 0x1p-64f, kTrustHi = 0x1p80f;  // d range for the fp32 bounds

struct SpecParams {
    const uint16_t *W;
    int64_t G;
    const float *D;
    int E;
    int64_t K;
    int qmin, qmax, n;
    uint16_t *out_scales;
    int8_t *out_codes;
    double *out_obj;
    uint8_t *out_flags;
};

// min(round-half-even(aw / s), cap) for aw >= 0, exact (cap <= 128): an
// estimate from 1/s, rounded by adding 1.5 * 2^23; near a half-integer the
// exact thresholds s (m -+ 1/2) (an 11-bit scale times a factor of at most 9
// bits) decide instead.
__device__ __forceinline__ int spec_code(float aw, float s, float inv, int cap)
{
    constexpr float kRound = 12582912.0f;
    const float x = fminf(aw * inv, static_cast<float>(cap + 1));
    const float y = x + kRound;
    const float m = y - kRound;
    const int mi = __float_as_int(y) - 0x4B400000;
    // x is within 129 * 2^-23 < 2^-15 of aw / s, so away from a half-integer
    // its own rounding is the exact one (x - m is exact)
    if (fabsf(fabsf(x - m) - 0.5f) > 0x1p-12f)
        return min(mi, cap);
    const float lo = s * (m - 0.5f), hi = s * (m + 0.5f);
    const bool odd = mi & 1;
    const int below = (aw < lo || (aw == lo && odd)) ? 1 : 0;
    const int above = (aw > hi || (aw == hi && odd)) ? 1 : 0;
    return min(mi - below + above, cap);
}

// fp32 diagonals per weight, padded to whole float4 loads; fp64 ones padded
// to whole double2 loads
template <int E>
constexpr int kPadE = E <= 4 ? 4 : 8;
template <int E>
constexpr int kPadD = (E + 1) & ~1;

// The E fp64 diagonals of weight i, from kPadD<E> / 2 16-byte loads.
template <int E>
__device__ __forceinline__ void load_dd(const double *dd, int i, double (&d)[kPadD<E>])
{
    const double2 *dp = reinterpret_cast<const double2 *>(dd + i * kPadD<E>);
#pragma unroll
    for (int h = 0; h < kPadD<E> / 2; h++) {
        const double2 v = dp[h];
        d[2 * h] = v.x;
        d[2 * h + 1] = v.y;
    }
}

struct Smem {
    float *wf;   // [n] exact weights
    double *wd;  // [n]
    double *dd;  // [n][kPadD]
    float *df;   // [n][kPadE] the same diagonals in fp32 (exact), for the chunk bounds
    float2 *ac;  // [n] (|w|, the code cap of w's sign)
    float *cbs;  // [kLaneChunks * 32] chunk bounds
};

// Objective at grid index j, in the definition's order; one thread.
template <int E>
__device__ double objective_at(const Smem &sm, int n, int qmin, int qmax, uint32_t j)
{
    const float s = grid_value(j);
    const float inv = 1.0f / s;
    const double nsd = -static_cast<double>(s);
    double acc[CQ_MAX_E];
#pragma unroll
    for (int e = 0; e < CQ_MAX_E; e++)
        acc[e] = 0.0;
    // the codes of 8 consecutive weights are computed independently; each
    // environment's running sum still takes the weights in ascending order
    auto term = [&](int i) {
        const float w = sm.wf[i];
        const bool neg = w < 0.0f;
        const int c = spec_code(fabsf(w), s, inv, neg ? -qmin : qmax);
        const double r = fma(nsd, static_cast<double>(neg ? -c : c), sm.wd[i]);
        const double rr = __dmul_rn(r, r);
        double d[kPadD<E>];
        load_dd<E>(sm.dd, i, d);
#pragma unroll
        for (int e = 0; e < E; e++)
            acc[e] = __dadd_rn(acc[e], __dmul_rn(d[e], rr));
    };
    int i = 0;
    for (; i + 8 <= n; i += 8) {
#pragma unroll
        for (int u = 0; u < 8; u++)
            term(i + u);
    }
    for (; i < n; i++)
        term(i);
    double f = acc[0];
#pragma unroll
    for (int e = 1; e < CQ_MAX_E; e++)
        if (e < E && acc[e] > f)
            f = acc[e];
    return f;
}

// Warp-wide (min objective, lowest pattern); every lane gets the result.
__device__ __forceinline__ void warp_best(double &f, uint32_t &j)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const double of = __shfl_xor_sync(kFull, f, o);
        const uint32_t oj = __shfl_xor_sync(kFull, j, o);
        if (of < f || (of == f && oj < j)) {
            f = of;
            j = oj;
        }
    }
}

// m0 = max over e of the warp-wide sums of a0[e], m1 = the same for a1[e], on
// every lane.  A reduce-scatter halves the values a lane carries at each of
// the first log2(2N) butterfly steps (N = E rounded up to a power of two), so
// after the five steps the block of 32 / (2N) consecutive lanes starting at
// lane j 32 / (2N) holds sum j: lanes 0-15 the sums of a0, lanes 16-31 those
// of a1.  The max over the blocks of each half follows.  The summation order
// differs from a plain butterfly; the callers' margins cover any order.
template <int E>
__device__ __forceinline__ void warp_max_of_sums2(const double (&a0)[E], const double (&a1)[E], int lane, double &m0,
                                                  double &m1)
{
    constexpr int N = E <= 1 ? 1 : E <= 2 ? 2 : E <= 4 ? 4 : 8;
    constexpr int N2 = 2 * N;
    double x[N2];
#pragma unroll
    for (int i = 0; i < N; i++) {
        x[i] = i < E ? a0[i] : 0.0;
        x[N + i] = i < E ? a1[i] : 0.0;
    }
    int o = 16;
#pragma unroll
    for (int h = N2 / 2; h >= 1; h /= 2, o >>= 1) {
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < h; i++) {
            const double send = up ? x[i] : x[i + h];
            const double keep = up ? x[i + h] : x[i];
            x[i] = keep + __shfl_xor_sync(kFull, send, o);
        }
    }
#pragma unroll
    for (; o > 0; o >>= 1)
        x[0] += __shfl_xor_sync(kFull, x[0], o);
#pragma unroll
    for (int b = 32 / N2; b < 16; b <<= 1)
        x[0] = fmax(x[0], __shfl_xor_sync(kFull, x[0], b));
    m0 = __shfl_sync(kFull, x[0], 0);
    m1 = __shfl_sync(kFull, x[0], 16);
}

// Two window bounds in one pass over the weights, each the max over
// environments of a per-environment sum of per-weight terms (the lanes take
// weights lane, lane + 32, ...; any order: a bound, used with a margin):
// b0 = the clipped weights' error at grid index j0, b1 = the error of the
// weights that quantise to 0 at j1.  Every lane gets both.
template <int E>
__device__ void bound_pair(const Smem &sm, int n, int qmin, int qmax, uint32_t j0, uint32_t j1, double &b0,
                           double &b1)
{
    const float s0 = grid_value(j0), s1 = grid_value(j1);
    const double sd0 = s0;
    double a0[E], a1[E];
#pragma unroll
    for (int e = 0; e < E; e++) {
        a0[e] = 0.0;
        a1[e] = 0.0;
    }
    for (int i = threadIdx.x & 31; i < n; i += 32) {
        const float w = sm.wf[i];
        const float aw = fabsf(w);
        const int cap = w < 0.0f ? -qmin : qmax;
        double t0 = 0.0, t1 = 0.0;
        if (code_at_least(aw, s0, cap + 1)) {
            const double x = static_cast<double>(aw) - cap * sd0;
            t0 = x * x;
        }
        if (!code_at_least(aw, s1, 1))
            t1 = sm.wd[i] * sm.wd[i];
        double d[kPadD<E>];
        load_dd<E>(sm.dd, i, d);
#pragma unroll
        for (int e = 0; e < E; e++) {
            a0[e] += d[e] * t0;
            a1[e] += d[e] * t1;
        }
    }
    warp_max_of_sums2<E>(a0, a1, threadIdx.x & 31, b0, b1);
}

// Upper bounds of the objective at grid indices ja and jb, from one pass over
// the weights, which the warp sums in any order: the exact value's fp64 sums
// err by at most n 2^-53 relative either way, so the warp sum times
// (1 + 2^-40) is at least the definition's own value for n <= 4096.  Every
// lane gets both.
template <int E>
__device__ void upper_pair(const Smem &sm, int n, int qmin, int qmax, uint32_t ja, uint32_t jb, double &ua,
                           double &ub)
{
    const float sa = grid_value(ja), sb = grid_value(jb);
    const float inva = 1.0f / sa, invb = 1.0f / sb;
    const double nsa = -static_cast<double>(sa), nsb = -static_cast<double>(sb);
    double a0[E], a1[E];
#pragma unroll
    for (int e = 0; e < E; e++) {
        a0[e] = 0.0;
        a1[e] = 0.0;
    }
    for (int i = threadIdx.x & 31; i < n; i += 32) {
        const float w = sm.wf[i];
        const bool neg = w < 0.0f;
        const int cap = neg ? -qmin : qmax;
        const int c0 = spec_code(fabsf(w), sa, inva, cap), c1 = spec_code(fabsf(w), sb, invb, cap);
        const double r0 = fma(nsa, static_cast<double>(neg ? -c0 : c0), sm.wd[i]);
        const double r1 = fma(nsb, static_cast<double>(neg ? -c1 : c1), sm.wd[i]);
        const double rr0 = r0 * r0, rr1 = r1 * r1;
        double d[kPadD<E>];
        load_dd<E>(sm.dd, i, d);
#pragma unroll
        for (int e = 0; e < E; e++) {
            a0[e] = fma(d[e], rr0, a0[e]);
            a1[e] = fma(d[e], rr1, a1[e]);
        }
    }
    warp_max_of_sums2<E>(a0, a1, threadIdx.x & 31, ua, ub);
    ua *= 1.0 + 0x1p-40;
    ub *= 1.0 + 0x1p-40;
}

// A lower bound of the objective at every scale in [s_lo, s_hi]: at any such s
// the residual of weight i is at least its distance to the union of the
// intervals [k s_lo, k s_hi], k = 0..cap, which is zero if |w| lies in one of
// them and otherwise min(|w| - k1 s_hi, k2 s_lo - |w|) with k1 the largest k
// whose interval ends at or below |w| (at most cap) and k2 = k1 + 1 (at most
// cap).  An fp32 floor off by one only lowers the computed distance.  Each
// term passes through 3 fp32 roundings and the running sum through n - 1, so
// for n <= 1024 the computed bound errs by less than 2^-14 relative; a chunk is
// skipped only when the bound times 1 - 2^-12 exceeds U, which leaves the exact
// bound, and so the definition's fp64 objective at every scale of the chunk,
// above U.
template <int E>
__device__ float chunk_bound(const Smem &sm, int n, int qmin, int qmax, float s_lo, float s_hi)
{
    const float inv_hi = 1.0f / s_hi;
    float acc[CQ_MAX_E];
#pragma unroll
    for (int e = 0; e < CQ_MAX_E; e++)
        acc[e] = 0.0f;
    for (int i = 0; i < n; i++) {
        const float2 a = sm.ac[i];
        const float aw = a.x, cap = a.y;
        const float k1 = fminf(floorf(aw * inv_hi), cap);
        const float e1 = fmaxf(fmaf(-k1, s_hi, aw), 0.0f);
        const float e2 = k1 < cap ? fmaxf(fmaf(k1 + 1.0f, s_lo, -aw), 0.0f) : INFINITY;
        const float dist = fminf(e1, e2);
        const float d2 = dist * dist;
        const float4 *dv = reinterpret_cast<const float4 *>(sm.df + i * kPadE<E>);
        float dq[kPadE<E>];
#pragma unroll
        for (int h = 0; h < kPadE<E> / 4; h++) {
            const float4 v = dv[h];
            dq[4 * h] = v.x;
            dq[4 * h + 1] = v.y;
            dq[4 * h + 2] = v.z;
            dq[4 * h + 3] = v.w;
        }
#pragma unroll
        for (int e = 0; e < E; e++)
            acc[e] = fmaf(dq[e], d2, acc[e]);
    }
    float best = 0.0f;
#pragma unroll
    for (int e = 0; e < CQ_MAX_E; e++)
        if (e < E)
            best = fmaxf(best, acc[e]);
    return best;
}

template <int E>
__global__ void __launch_bounds__(32) spec_kernel(SpecParams p)
{
    extern __shared__ __align__(16) unsigned char dyn[];
    const int n = p.n;
    const int lane = threadIdx.x & 31;
    Smem sm;
    // 16-byte aligned first: df; then 8-byte items; then 4-byte items
    sm.df = reinterpret_cast<float *>(dyn);
    sm.dd = reinterpret_cast<double *>(sm.df + static_cast<size_t>(kPadE<E>) * n);
    sm.wd = sm.dd + static_cast<size_t>(kPadD<E>) * n;
    sm.ac = reinterpret_cast<float2 *>(sm.wd + n);
    sm.wf = reinterpret_cast<float *>(sm.ac + n);
    sm.cbs = sm.wf + n;
    const int64_t gpr = p.K > 0 ? p.K / n : 1;
    constexpr double kKeep = 1.0 - 0x1p-40;
    for (int64_t g = blockIdx.x; g < p.G; g += gridDim.x) {
        __syncwarp();
        // 1. stage
        float am = 0.0f;
        bool bad = false, odd = false;
        for (int i = lane; i < n; i += 32) {
            const uint32_t b = p.W[g * n + i];
            bad |= (b & 0x7FFFu) >= kBeyond;
            const float w = half_value(b);
            sm.wf[i] = w;
            sm.wd[i] = w;
            sm.ac[i] = make_float2(fabsf(w), static_cast<float>(w < 0.0f ? -p.qmin : p.qmax));
            am = fmaxf(am, fabsf(w));
#pragma unroll
            for (int e = 0; e < E; e++) {
                const float d = p.K > 0 ? p.D[e * p.K + (g % gpr) * n + i] : p.D[(e * p.G + g) * n + i];
                bad |= !(d >= 0.0f && d <= FLT_MAX);
                odd |= d != 0.0f && !(d >= kTrustLo && d <= kTrustHi);
                sm.dd[i * kPadD<E> + e] = d;
                sm.df[i * kPadE<E> + e] = d;
            }
            if (kPadD<E> > E)
                sm.dd[i * kPadD<E> + E] = 0.0;
#pragma unroll
            for (int e = E; e < kPadE<E>; e++)
                sm.df[i * kPadE<E> + e] = 0.0f;
        }
        bad = __any_sync(kFull, bad);
        const bool trust = !__any_sync(kFull, odd);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            am = fmaxf(am, __shfl_xor_sync(kFull, am, o));
        const float amax = am;
        __syncwarp();
        if (bad || amax == 0.0f) {
            for (int i = lane; i < n; i += 32)
                p.out_codes[g * n + i] = 0;
            if (lane == 0) {
                p.out_scales[g] = 0x0001;
                if (p.out_obj)
                    p.out_obj[g] = 0.0;
                if (p.out_flags)
                    p.out_flags[g] = bad ? CQ_FLAG_NONFINITE : CQ_FLAG_TRIVIAL;
            }
            continue;
        }
        // 2. upper bound U.  Every lane evaluates the same candidates, so U and
        // jb are uniform; jb lies in the window found below (its bounds are
        // below U there) and not above j_z, so the scan evaluates it exactly.
        uint32_t jz = kLast + 1;  // first scale where every code is 0 (s >= 2 max|w|)
        {
            const float two = 2.0f * amax;  // exact
            if (two <= 65504.0f)
                jz = max(static_cast<uint32_t>(__half_as_ushort(__float2half_ru(two))), 1u);
        }
        double U = INFINITY;
        uint32_t jb = 1;
        // candidates in pairs (the last paired with itself; j_z dropped when
        // above the grid); the first of equal bounds is kept
        for (int t = 0; t < kCandidates; t += 2) {
            uint32_t jp[2];
#pragma unroll
            for (int k = 0; k < 2; k++) {
                const int tt = min(t + k, kCandidates - 1);
                if (tt == kCandidates - 1) {
                    jp[k] = jz;
                } else {
                    const double base = static_cast<double>(amax) / (tt < 3 ? p.qmax : -p.qmin);
                    const int off = (tt % 3) - 1;
                    const int jc = static_cast<int>(__half_as_ushort(__double2half(base))) + off;
                    jp[k] = static_cast<uint32_t>(min(max(jc, 1), static_cast<int>(kLast)));
                }
            }
            double u[2];
            upper_pair<E>(sm, n, p.qmin, p.qmax, min(jp[0], kLast), min(jp[1], kLast), u[0], u[1]);
#pragma unroll
            for (int k = 0; k < 2; k++) {
                if (jp[k] <= kLast && u[k] < U) {
                    U = u[k];
                    jb = jp[k];
                }
            }
        }
        // 3. certified window [J0, J1]: one bisection over [1, jb] for the
        // smallest index the clipping bound keeps (it falls as s rises), one over
        // [jb, kLast] for the largest the dead-zone bound keeps (it rises with
        // s), advancing together with one pass over the weights per step.  jb
        // is kept by both; the indices 0 and kLast + 1 stand for excluded ends.
        uint32_t ex0 = 0u, ok0 = jb, ex1 = kLast + 1u, ok1 = jb;
        for (;;) {
            const bool go0 = ex0 + 1u != ok0, go1 = ok1 + 1u != ex1;
            if (!go0 && !go1)
                break;
            const uint32_t m0 = go0 ? (ex0 + ok0) / 2u : ok0;
            const uint32_t m1 = go1 ? (ex1 + ok1) / 2u : ok1;
            double b0, b1;
            bound_pair<E>(sm, n, p.qmin, p.qmax, m0, m1, b0, b1);
            if (go0) {
                if (b0 * kKeep > U)
                    ex0 = m0;
                else
                    ok0 = m0;
            }
            if (go1) {
                if (b1 * kKeep > U)
                    ex1 = m1;
                else
                    ok1 = m1;
            }
        }
        const uint32_t J0 = ok0, J1 = min(ok1, jz);
        // 4. chunk bounds; lane L holds chunks L + 32 m in cb[m] (INFINITY when
        // dropped; bit m of `gone` once taken).  C doubles from 8 until 256
        // chunks cover the window.
        const uint32_t len = J1 - J0 + 1;
        uint32_t C = kMinChunk;
        while (C * 32u * kLaneChunks < len)
            C *= 2;
        const int nch = static_cast<int>((len + C - 1) / C);
        for (int ch = lane; ch < nch; ch += 32) {
            float v = 0.0f;
            if (trust) {
                const uint32_t a = J0 + static_cast<uint32_t>(ch) * C;
                const uint32_t b = min(a + C - 1, J1);
                v = chunk_bound<E>(sm, n, p.qmin, p.qmax, grid_value(a), grid_value(b));
                if (v * kKeepChunk > U)
                    v = INFINITY;
            }
            sm.cbs[ch] = v;
        }
        __syncwarp();
        float cb[kLaneChunks];
#pragma unroll
        for (int m = 0; m < kLaneChunks; m++) {
            const int ch = lane + 32 * m;
            cb[m] = ch < nch ? sm.cbs[ch] : INFINITY;
        }
        // 5. best first.  A batch takes up to 32 / C chunks (one for C >= 32, its
        // scales in C / 32 passes), smallest bound first (lowest chunk on ties),
        // while that bound times 1 - 2^-12 does not exceed thr: U, then the best
        // objective evaluated.  A chunk left over has every objective above
        // thr, so strictly above the minimum.  Per lane, the (objective,
        // pattern) minimum in that order.
        double bf = INFINITY;
        uint32_t bj = 0xFFFFFFFFu;
        double thr = U;
        const int per = C >= 32u ? 1 : static_cast<int>(32u / C);
        const int passes = C >= 32u ? static_cast<int>(C / 32u) : 1;
        uint32_t gone = 0;
        for (;;) {
            int mine = -1;
            int taken = 0;
            for (int t = 0; t < per; t++) {
                float v = INFINITY;
                int mi = 0;
#pragma unroll
                for (int m = 0; m < kLaneChunks; m++) {
                    if (!((gone >> m) & 1u) && cb[m] < v) {
                        v = cb[m];
                        mi = m;
                    }
                }
                int c = v < INFINITY ? lane + 32 * mi : 0x7FFFFFFF;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    const float ov = __shfl_xor_sync(kFull, v, o);
                    const int oc = __shfl_xor_sync(kFull, c, o);
                    if (ov < v || (ov == v && oc < c)) {
                        v = ov;
                        c = oc;
                    }
                }
                if (c == 0x7FFFFFFF || v * kKeepChunk > thr)
                    break;  // uniform: every lane holds the same (v, c)
                if (lane == (c & 31))
                    gone |= 1u << (c >> 5);
                if (C >= 32u || lane / static_cast<int>(C) == t)
                    mine = c;
                taken++;
            }
            if (taken == 0)
                break;
            for (int ps = 0; ps < passes; ps++) {
                const uint32_t off = C >= 32u ? static_cast<uint32_t>(ps * 32 + lane) : static_cast<uint32_t>(lane) % C;
                const uint32_t j = J0 + static_cast<uint32_t>(mine) * C + off;
                if (mine >= 0 && j <= J1) {
                    const double v = objective_at<E>(sm, n, p.qmin, p.qmax, j);
                    if (v < bf || (v == bf && j < bj)) {
                        bf = v;
                        bj = j;
                    }
                }
            }
            double mf = bf;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                mf = fmin(mf, __shfl_xor_sync(kFull, mf, o));
            thr = fmin(thr, mf);
        }
        warp_best(bf, bj);
        // 6. outputs
        const float s = grid_value(bj);
        const float inv = 1.0f / s;
        for (int i = lane; i < n; i += 32) {
            const float w = sm.wf[i];
            const bool neg = w < 0.0f;
            const int c = spec_code(fabsf(w), s, inv, neg ? -p.qmin : p.qmax);
            p.out_codes[g * n + i] = static_cast<int8_t>(neg ? -c : c);
        }
        if (lane == 0) {
            p.out_scales[g] = static_cast<uint16_t>(bj);
            if (p.out_obj)
                p.out_obj[g] = bf;
            if (p.out_flags)
                p.out_flags[g] = 0;
        }
    }
}

template <int E>
cudaError_t launch_spec(const SpecParams &p, cudaStream_t st)
{
    const int n = p.n;
    const size_t smem = static_cast<size_t>(n) * (kPadE<E> * sizeof(float) + kPadD<E> * sizeof(double) + sizeof(double) +
                                                  sizeof(float2) + sizeof(float)) +
                        kLaneChunks * 32 * sizeof(float);
    cudaError_t err = cudaSuccess;
    if (smem > 48 * 1024 &&
        (err = cudaFuncSetAttribute(spec_kernel<E>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(smem))) != cudaSuccess)
        return err;
    int per_sm = 1, dev = 0, sms = 148;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, spec_kernel<E>, 32, smem) != cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t cap = static_cast<int64_t>(sms) * per_sm;
    const unsigned grid = static_cast<unsigned>(p.G < cap ? p.G : cap);
    spec_kernel<E><<<grid, 32, smem, st>>>(p);
    return cudaGetLastError();
}

}  // namespace

// The W4 kernel's search for eligible specs (cq_select.cu).
cq_status select_spec_fast(const uint16_t *W, int64_t G, const float *D, int E, int64_t K, int qmin, int qmax,
                           int n, uint16_t *out_scales, int8_t *out_q, double *out_obj, uint8_t *out_flags,
                           cudaStream_t st);
}  // namespace cq

using namespace cq;

extern "C" {

cq_status cq_select_scales_spec(const uint16_t *W, int64_t G, const float *D, int E, int64_t K,
                                const cq_quantizer_spec *spec, uint16_t *out_scales, int8_t *out_codes,
                                double *out_objective, uint8_t *out_flags, void *stream)
{
    if (!spec || G < 0 || K < 0 || E < 1)
        return CQ_ERR_INVALID_ARG;
    const int n = spec->group_size;
    if (spec->qmin > -1 || spec->qmax < 1 || n < 1)
        return CQ_ERR_INVALID_ARG;
    if (spec->qmin < -128 || spec->qmax > 127 || n > CQ_SPEC_MAX_GROUP || E > CQ_MAX_E ||
        G >= (static_cast<int64_t>(1) << 31))
        return CQ_ERR_UNSUPPORTED;
    if (K > 0 && (K % n != 0 || G % (K / n) != 0))
        return CQ_ERR_INVALID_ARG;
    if (G == 0)
        return CQ_OK;
    if (!W || !D || !out_scales || !out_codes)
        return CQ_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(W) & 1) || (reinterpret_cast<uintptr_t>(D) & 3) ||
        (reinterpret_cast<uintptr_t>(out_scales) & 1) || (reinterpret_cast<uintptr_t>(out_objective) & 7))
        return CQ_ERR_INVALID_ARG;
    if (spec->kernel != CQ_SPEC_KERNEL_AUTO && spec->kernel != CQ_SPEC_KERNEL_GENERAL)
        return CQ_ERR_INVALID_ARG;
    if ((n == kGroup || n == 64) && spec->kernel == CQ_SPEC_KERNEL_AUTO) {
        const cq_status fs = select_spec_fast(W, G, D, E, K, spec->qmin, spec->qmax, n, out_scales, out_codes,
                                              out_objective, out_flags, static_cast<cudaStream_t>(stream));
        if (fs != CQ_ERR_UNSUPPORTED)
            return fs;
    }
    SpecParams p{W, G, D, E, K, spec->qmin, spec->qmax, n, out_scales, out_codes, out_objective, out_flags};
    cudaError_t err = cudaErrorInvalidValue;
    switch (E) {
    case 1: err = launch_spec<1>(p, static_cast<cudaStream_t>(stream)); break;
    case 2: err = launch_spec<2>(p, static_cast<cudaStream_t>(stream)); break;
    case 3: err = launch_spec<3>(p, static_cast<cudaStream_t>(stream)); break;
    case 4: err = launch_spec<4>(p, static_cast<cudaStream_t>(stream)); break;
    case 5: err = launch_spec<5>(p, static_cast<cudaStream_t>(stream)); break;
    case 6: err = launch_spec<6>(p, static_cast<cudaStream_t>(stream)); break;
    case 7: err = launch_spec<7>(p, static_cast<cudaStream_t>(stream)); break;
    case 8: err = launch_spec<8>(p, static_cast<cudaStream_t>(stream)); break;
    default: break;
    }
    return err == cudaSuccess ? CQ_OK : CQ_ERR_CUDA;
}

}  // extern "C"
