/*
 * cq.h — C ABI of libcq.so: exact minimax FP16 group-scale selection for
 * symmetric W4 quantisation with group size 128, on NVIDIA B200 (sm_100a).
 *
 * The operation (CliffQuant project page, "What CliffQuant changes"): for each
 * group of 128 weights w_i and E environment diagonals d_{e,i} >= 0, choose the
 * positive finite IEEE binary16 scale s minimising
 *
 *     f(s) = max_e  sum_i d_{e,i} * (w_i - s * q_i(s))^2,
 *     q_i(s) = clip(round-half-even(w_i / s), -8, 7),
 *
 * over all 31,743 such scales, an exact objective tie going to the lower FP16
 * bit pattern, and emit the 4-bit codes.  The codes are packed as (q + 8)
 * nibbles, 8 per uint32, low nibble first: word j of a group holds codes
 * 8j .. 8j+7.  The quantiser is QuantizerSpec(qmin=-8, qmax=7) of the page's
 * "Use the solver" example.  The candidate scales the page's solver outline
 * names (code transitions, quadratic vertices, environment intersections) are
 * realised here as a search over the runs of constant codes between code
 * transitions; the exhaustive enumeration of all 31,743 values is the
 * fallback when a group's screen cannot certify its answer.
 *
 * Conventions for every entry point:
 *  - All pointers named W, D, out_* and workspace are DEVICE pointers on the
 *    current CUDA device, except where a name ends in _host.  The caller owns
 *    every buffer; the library keeps no pointer after a call returns.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Device work is enqueued on it asynchronously; nothing here
 *    synchronises the host unless its comment says so.
 *  - Argument errors are returned synchronously, before anything is enqueued.
 *    CQ_ERR_CUDA means a CUDA runtime call failed (the CUDA error is left
 *    for cudaGetLastError()).
 *  - Results are deterministic: the same inputs give the same output bytes.
 *  - Non-finite or negative inputs never trap: the affected group gets scale
 *    0x0001 and all codes 0 (nibble 8), and the NONFINITE counter and flag are
 *    set; cq_get_status() and cq_read_counters() report it as CQ_ERR_NONFINITE.
 */
#ifndef CQ_H
#define CQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define CQ_GROUP 128          /* weights per group */
#define CQ_WORDS 16           /* packed uint32 words per group */
#define CQ_MAX_E 8            /* environments supported */
#define CQ_NUM_COUNTERS 8

typedef enum {
    CQ_OK = 0,
    CQ_ERR_INVALID_ARG = 1,      /* null pointer, bad size, layout or alignment */
    CQ_ERR_UNSUPPORTED = 2,      /* E > CQ_MAX_E, or G >= 2^32 */
    CQ_ERR_CUDA = 3,             /* a CUDA runtime call failed */
    CQ_ERR_NONFINITE = 4,        /* (cq_read_counters) some group had non-finite/negative input */
    CQ_ERR_WORKSPACE = 5,        /* workspace missing, too small or misaligned */
    CQ_ERR_TOO_LARGE = 6         /* (cq_select_scales_noalloc) G above CQ_NOALLOC_MAX_GROUPS */
} cq_status;

/* Indices into the device counters kept in the workspace. */
enum {
    CQ_CNT_FALLBACK = 0,     /* groups decided by the exhaustive 31,743-scale pass */
    CQ_CNT_NEAR_TIE = 1,     /* groups whose best two candidates are within flag_rel_gap */
    CQ_CNT_NONFINITE = 2,    /* groups with non-finite weights or non-finite/negative d */
    CQ_CNT_TRIVIAL = 3,      /* all-zero groups (scale 0x0001, codes 0) */
    CQ_CNT_FINALISTS = 4,    /* total fp64-rescored candidate scales */
    CQ_CNT_UNCERTAIN = 5,    /* runs whose screen could not be certified */
    CQ_CNT_QUEUE = 6,        /* internal: fallback queue length */
    CQ_CNT_SURVIVORS = 7     /* runs that passed the fp32 screen (summed over groups) */
};

/* Per-group flag bits written to out_flags. */
#define CQ_FLAG_TRIVIAL   0x01
#define CQ_FLAG_FALLBACK  0x02
#define CQ_FLAG_NEAR_TIE  0x04
#define CQ_FLAG_NONFINITE 0x08

typedef struct {
    int32_t finalist_cap;     /* max fp64-rescored scales per group before the exhaustive
                                 fallback; 1..64, 0 = default (32) */
    int32_t force_exhaustive; /* nonzero: decide every non-trivial group by the exhaustive pass */
    double flag_rel_gap;      /* CQ_FLAG_NEAR_TIE when the best two finalists are within this
                                 relative gap; 0 = default (1e-12) */
    void *ev_main_begin;      /* nullable cudaEvent_t recorded on `stream` just before the main
                                 selection kernel (profiling hook) */
    void *ev_main_end;        /* nullable cudaEvent_t recorded just after it, before the fallback */
    int32_t intersections;    /* nonzero: search each run that survives the screen with the
                                 pairwise environment-intersection solver (the page's
                                 "environment intersections" candidates) instead of a vertex
                                 test and binary search; identical results, slower on the
                                 0.8B-scale sweep, so off by default */
} cq_opts;

/* Bytes of device workspace cq_select_scales_ex needs for G groups.  The
 * workspace holds the counters and the fallback queue (8 bytes per group). */
size_t cq_workspace_bytes(int64_t G, int E);

/* Select scales and codes for G groups.
 *  W          [G][128] binary16 bit patterns, 16-byte aligned.
 *  D          fp32 diagonals, 16-byte aligned, in one of two layouts:
 *               K > 0:  per column [E][K]; K % 128 == 0 and G % (K/128) == 0;
 *                       group g uses columns (g % (K/128))*128 .. +127, i.e. W
 *                       is a row-major [G/(K/128)][K] matrix grouped along rows.
 *               K == 0: per group [E][G][128].
 *  E          number of environments, 1..CQ_MAX_E.
 *  out_scales [G] binary16 bit patterns of the chosen scales (0x0001..0x7BFF).
 *  out_codes  [G][16] packed codes, 4-byte aligned.
 * Unlike the other selection entry points this one allocates: it takes its
 * workspace (cq_workspace_bytes(G, E), about 8 bytes per group) from a
 * stream-ordered memory pool that the library creates for each device on
 * first use, and frees it on `stream` after the kernels.  The pool's release
 * threshold is unlimited, so freed blocks stay reserved for the next call and
 * the pool keeps its high-water mark until the process exits or the caller
 * calls cq_trim_memory().  For no allocation at all, pass a workspace to
 * cq_select_scales_ex (or use cq_select_scales_noalloc). */
cq_status cq_select_scales(const uint16_t *W, int64_t G, const float *D, int E, int64_t K,
                           uint16_t *out_scales, uint32_t *out_codes, void *stream);

/* As cq_select_scales, with caller-provided workspace (device, 256-byte
 * aligned, at least cq_workspace_bytes(G, E)), options (nullable = defaults)
 * and optional outputs:
 *  out_objective  nullable, fp64 [G]: the objective at the chosen scale.
 *  out_flags      nullable, uint8 [G]: CQ_FLAG_* bits.
 * The workspace counters are reset at the start of every call.  Calls that
 * share a workspace must be ordered on one stream.  The call only enqueues
 * work on `stream` (no allocation, no host synchronisation), so it can be
 * captured in a CUDA graph and replayed on new contents of the same buffers. */
cq_status cq_select_scales_ex(const uint16_t *W, int64_t G, const float *D, int E, int64_t K,
                              uint16_t *out_scales, uint32_t *out_codes, void *stream,
                              const cq_opts *opts, void *workspace, size_t workspace_bytes,
                              double *out_objective, uint8_t *out_flags);

/* Host-buffer variant: W_host, D_host, out_scales_host and out_codes_host are
 * HOST pointers (page-locked memory gives overlapped copies).  The call
 * allocates device buffers (from the same library pool as cq_select_scales),
 * streams the groups through them in chunks with host<->device copies
 * overlapped with compute on `stream`, and returns after the results are in
 * the host buffers (it synchronises `stream`). */
cq_status cq_select_scales_host(const uint16_t *W_host, int64_t G, const float *D_host, int E,
                                int64_t K, uint16_t *out_scales_host, uint32_t *out_codes_host,
                                void *stream);

/* ---- comparison policies and the reconstruction proxy ----------------------
 * The project page's "Held-out reconstruction proxy" table (and the model
 * card's section of the same name) compares CliffQuant's minimax scales with
 * two policies, Pooled-WMSE and AbsMax, on the "module-macro worst-environment
 * weighted MSE".  These entry points compute those policies and that proxy
 * on the GPU.  All pointers are device pointers; all are asynchronous on
 * `stream`; argument errors return before anything is enqueued. */

/* AbsMax policy (the matched baseline checkpoint's scales): per group
 * s = binary16 nearest (ties to even) to max_i |w_i| / 7 computed in fp64,
 * raised to 0x0001 when that rounds to 0 (all-zero groups); codes are the
 * quantiser's at s, packed like cq_select_scales.  A group with a non-finite
 * weight gets scale 0x0001 and zero codes.
 *  W [G][128] binary16 bits and out_codes [G][16] 16-byte aligned; out_scales [G]. */
cq_status cq_absmax_scales(const uint16_t *W, int64_t G, uint16_t *out_scales, uint32_t *out_codes, void *stream);

/* Pooled diagonals for the Pooled-WMSE policy: out[i] = fp32, rounded to
 * nearest even, of (sum over e = 0..E-1 of D[e*n + i], summed in fp64 in that
 * order) / E.  D is [E][n] fp32 (n = K for per-column, G*128 for per-group
 * diagonals); out is [n].  The policy is cq_select_scales with E = 1 on out. */
cq_status cq_pool_diagonals(const float *D, int E, int64_t n, float *out, void *stream);

/* Objective of given scales (the proxy's per-group term): per_env[g*E + e] =
 * sum_i d_{e,i} (w_i - s q_i(s))^2 in fp64, summed over i ascending without
 * fused multiply-adds, and out_objective[g] = max_e of those; s = scales[g]
 * (binary16 bits, a positive finite pattern 0x0001..0x7BFF).  W and D as for
 * cq_select_scales (both 16-byte aligned); per_env [G][E] and out_objective
 * [G] are fp64 and 8-byte aligned.  The values are unspecified for non-finite
 * input or other scale patterns; the kernel reads and writes only the
 * buffers above either way. */
cq_status cq_group_objective(const uint16_t *W, int64_t G, const float *D, int E, int64_t K,
                             const uint16_t *scales, double *per_env, double *out_objective,
                             void *stream);

/* Module-macro worst-environment weighted MSE, from cq_group_objective's
 * per_env output [G][E].  Module m holds groups offsets[m] .. offsets[m+1]-1
 * (offsets: nmod+1 ascending int64 on the device, clamped to [0, G] so that no
 * read leaves per_env); then
 *   module_env[m*E + e] = scale * (sum of per_env[g*E + e] over its groups) / count,
 *   module_worst[m]     = max_e module_env[m*E + e],
 *   macro[0]            = mean over m of module_worst[m].
 * With scale = 1/128 these are per-weight means.  Sums use a fixed order, so
 * the results are deterministic; a module with no groups gives NaN.  All
 * pointers are 8-byte-aligned device pointers. */
cq_status cq_reconstruction_proxy(const double *per_env, int64_t G, int E, int64_t nmod,
                                  const int64_t *offsets, double scale, double *module_env,
                                  double *module_worst, double *macro, void *stream);

/* ---- GPTQ v1 tensors --------------------------------------------------------
 * The project page and the model card ("Quantization configuration") release
 * a GPTQ v1 checkpoint: 4-bit, group size 128, symmetric, act-order off.  The
 * pages do not print the layout; these follow the public GPTQ v1 format for a
 * linear layer with weight [R][K] (R outputs, K inputs, groups along K as in
 * cq_select_scales with per-column diagonals):
 *   qweight int32 [K/8][R]     inputs 8k..8k+7 of output r, input 8k+j in bits 4j..4j+3
 *   qzeros  int32 [K/128][R/8] zero points of outputs 8c..8c+7, stored minus one (0x77777777)
 *   scales  fp16  [K/128][R]   binary16 bits
 *   g_idx   int32 [K]          i / 128
 * Requires K % 128 == 0 and R % 8 == 0 (else CQ_ERR_INVALID_ARG).  All
 * pointers are device pointers with their element's alignment. */

/* Export: from the selection's scales [R*K/128] and packed codes [R*K/128][16]
 * (group r*(K/128) + c is row r, columns 128c..128c+127) to the four tensors.
 * One launch when codes and qweight are 16-byte aligned; three (the same
 * bytes) when either is only 4-byte aligned. */
cq_status cq_gptq_export(const uint16_t *scales, const uint32_t *codes, int64_t R, int64_t K,
                         int32_t *qweight, int32_t *qzeros, uint16_t *gptq_scales, int32_t *g_idx,
                         void *stream);

/* Dequantisation by the v1 rule w[r][i] = scales[g][r] * (u - (z + 1)), g = g_idx[i]
 * (clamped to [0, K/128)), into out [R][K] (out and g_idx 16-byte aligned): fp32 when
 * out_fp16 == 0 (exact), binary16 rounded to nearest even when out_fp16 == 1.
 * Reads only the four tensors: an unpacker independent of the export. */
cq_status cq_gptq_dequantize(const int32_t *qweight, const int32_t *qzeros, const uint16_t *gptq_scales,
                             const int32_t *g_idx, int64_t R, int64_t K, int out_fp16, void *out,
                             void *stream);

/* ---- sensitivity diagonals ----------------------------------------------------
 * The project page ("What CliffQuant changes"; "The negative result that
 * changed the method") takes separately normalised per-environment diagonals
 * estimated as empirical activation-weighted sensitivity.  From calibration
 * inputs X [rows][K] (row-major, 16-byte aligned, K % 8 == 0), environment e
 * owning rows row_offsets[e] .. row_offsets[e+1]-1 (a HOST array of E+1
 * ascending offsets, 1 <= E <= CQ_MAX_E):
 *   means[e][k] = (sum over its rows of x^2) / N_e   fp64 [E][K], 8-byte aligned
 *   D[e][k]     = fp32(means[e][k] / mean_j means[e][j])   fp32 [E][K]
 * Squares are exact and summed in fp64 in a fixed order (deterministic).  An
 * environment with no rows, or only zero activations, gives NaN.  D is the
 * per-column diagonal layout cq_select_scales takes. */
#define CQ_DTYPE_BF16 0
#define CQ_DTYPE_FP16 1
#define CQ_DTYPE_FP32 2
cq_status cq_estimate_diagonals(const void *X, int dtype, int64_t K, const int64_t *row_offsets, int E,
                                double *means, float *D, void *stream);

/* ---- general quantiser spec ---------------------------------------------------
 * "Use the solver" on the project page passes QuantizerSpec(qmin, qmax); this
 * entry point takes any qmin in [-128, -1], qmax in [1, 127] and group size n
 * in [1, CQ_SPEC_MAX_GROUP], with the same objective, binary16 scale domain
 * and tie rule as cq_select_scales.  W [G][n] binary16 bits; D per column
 * [E][K] (K % n == 0, group g uses columns (g mod K/n)*n ..; G a whole number
 * of rows) or per group [E][G][n] (K == 0).  Outputs: out_scales [G],
 * out_codes int8 [G][n] (the codes q themselves), optional out_objective fp64
 * [G] (8-byte aligned) and out_flags [G] (CQ_FLAG_TRIVIAL / CQ_FLAG_NONFINITE;
 * such groups get scale 0x0001, zero codes and objective 0).  Scales, codes
 * and objectives are the definition's own fp64 values, bit for bit.
 *
 * Two kernels serve it.  A code range [-m, m] or [-m, m - 1] with m <= 16 at
 * group size 128, or m <= 8 at group size 64 (the 2- to 5-bit ranges and the
 * symmetric ones),
 * and W, D 16-byte aligned, out_codes 4-byte aligned: the W4 kernel's search
 * with that range's caps, its finalists rescored in the definition's order;
 * this takes a workspace from the library pool, like cq_select_scales.  Any
 * other spec: a certified window plus an exact best-first scan of the grid
 * (no allocation).  spec->kernel = CQ_SPEC_KERNEL_GENERAL forces the second. */
#define CQ_SPEC_KERNEL_AUTO 0
#define CQ_SPEC_KERNEL_GENERAL 1
typedef struct cq_quantizer_spec {
    int32_t qmin;
    int32_t qmax;
    int32_t group_size;
    int32_t kernel;  /* CQ_SPEC_KERNEL_AUTO (0) or CQ_SPEC_KERNEL_GENERAL */
} cq_quantizer_spec;
#define CQ_SPEC_MAX_GROUP 1024
cq_status cq_select_scales_spec(const uint16_t *W, int64_t G, const float *D, int E, int64_t K,
                                const cq_quantizer_spec *spec, uint16_t *out_scales, int8_t *out_codes,
                                double *out_objective, uint8_t *out_flags, void *stream);

/* Largest G that cq_select_scales_noalloc accepts. */
#define CQ_NOALLOC_MAX_GROUPS (1 << 20)

/* Allocation-free variant of cq_select_scales, for callers that cannot
 * allocate device memory at call time: code running inside an allocator
 * callback or under an external memory budget, an embedded runtime whose
 * device memory is planned up front, or a host thread that must not touch
 * the CUDA allocator.  It has no counterpart on the method's pages; it is a
 * property of this library.
 *
 * Same arguments, layouts and results as cq_select_scales.  The selection
 * kernel's scratch (its counters and the exhaustive-fallback queue) lives in
 * one fixed array of 256 + 8 * CQ_NOALLOC_MAX_GROUPS bytes (about 8 MiB)
 * compiled into the library, which every GPU that loads the library keeps
 * until the process exits.  Nothing is allocated or freed: no cudaMalloc, no
 * cudaFree, no pool or library allocation.
 *  - G > CQ_NOALLOC_MAX_GROUPS returns CQ_ERR_TOO_LARGE before anything is
 *    enqueued.
 *  - The first call on a device looks up that device's address of the array
 *    (cudaGetSymbolAddress) and keeps it; make that first call before any
 *    stream capture on the device.
 *  - Every call uses the same array; the counters in it are cleared on
 *    `stream` at the start of each call.  Calls whose work overlaps on the
 *    GPU (on different streams, or from different host threads without
 *    ordering) race on the array: order them on one stream or otherwise.
 *  - The return value is the only status this entry point reports: its
 *    counters are not readable by the caller.  A group with non-finite or
 *    negative input still gets scale 0x0001 and all codes 0, which looks
 *    like an all-zero group; a caller that must detect such input checks it
 *    first, or uses cq_select_scales_ex with its own workspace and out_flags. */
cq_status cq_select_scales_noalloc(const uint16_t *W, int64_t G, const float *D, int E, int64_t K,
                                   uint16_t *out_scales, uint32_t *out_codes, void *stream);

/* Release the memory that cq_select_scales and cq_select_scales_host keep
 * cached in the current device's library pool (cudaMemPoolTrimTo to zero).
 * Blocks still in use by enqueued work are kept.  A no-op when the pool was
 * never created.  Returns CQ_ERR_CUDA when a CUDA call fails. */
cq_status cq_trim_memory(void);

/* Copy the workspace counters to host_counters[CQ_NUM_COUNTERS] (host
 * memory).  Synchronises `stream`.  Returns CQ_ERR_NONFINITE when the last
 * call saw non-finite input, else CQ_OK (or CQ_ERR_CUDA / CQ_ERR_INVALID_ARG). */
cq_status cq_read_counters(const void *workspace, uint32_t *host_counters, void *stream);

/* Status of the last call that used `workspace`: synchronises `stream`, then
 * returns CQ_ERR_NONFINITE when that call saw non-finite or negative input,
 * CQ_ERR_CUDA when the stream reports an error, CQ_ERR_INVALID_ARG for a null
 * workspace, else CQ_OK.  The same as cq_read_counters without the counts. */
cq_status cq_get_status(const void *workspace, void *stream);

/* Static, human-readable name of a status code. */
const char *cq_status_string(cq_status status);

/* Library version, major*10000 + minor*100 + patch. */
int cq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* CQ_H */
