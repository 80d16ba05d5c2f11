/*
 * ln.h -- C ABI of libln.so: LayerNorm forward and analytical backward on an
 * NVIDIA B200 (sm_100a).
 *
 * The operation.  "llm.c's Origin and the Future of LLM Compilers" (CUDA MODE
 * talk page), chapter "Deconstructing PyTorch Abstractions and Setting
 * Reference Baselines", describes LayerNorm forward and backward written over
 * bare float arrays with no tensor abstraction; "llm.c: Large Language Model
 * Training in Pure C/CUDA Without Dependencies", features "Tensor Memory
 * Layout" (flat 1-D row-major arrays, explicit stride arithmetic) and "Exact
 * Analytical Backward Pass" (hand-derived LayerNorm gradients).  The pages do
 * not print the equations; this library computes the textbook definition:
 *
 *   mean[r] = (1/C) sum_c x[r,c]
 *   rstd[r] = 1 / sqrt((1/C) sum_c (x[r,c] - mean[r])^2 + eps)
 *   out     = (x - mean[r]) * rstd[r] * weight[c] + bias[c]
 *
 *   xhat    = (x - mean[r]) * rstd[r],   g = dout * weight[c]
 *   dinp    = rstd[r] * (g - (1/C) sum_c g - xhat * (1/C) sum_c g * xhat)
 *   dweight = sum over all N rows of dout * xhat
 *   dbias   = sum over all N rows of dout
 *
 * Layout.  Activations (inp, out, dout, dinp) are flat row-major [N * C]
 * arrays: row r starts at element r * C.  weight, bias, dweight and dbias hold
 * C elements, mean and rstd hold N.  All pointers are DEVICE pointers of the
 * current CUDA device, owned by the caller; the library never frees them.
 *
 * Types.  `dtype` (LN_F32, LN_BF16 or LN_F16) is the element type of inp,
 * out, dout, dinp, weight and bias.  mean, rstd, dweight and dbias are always
 * fp32.  Arithmetic is fp32 in registers; bf16 and fp16 results are rounded
 * to nearest-even (fp16 results beyond 65504 become infinite, as rounding
 * requires).  The pages this library follows name fp32 and bf16 kernels;
 * fp16 is the other 16-bit training format and takes the same paths.
 *
 * Semantics shared by every call.
 *   - Asynchronous on `stream` (NULL: the legacy default stream); no host
 *     synchronisation; the library creates no streams of its own.
 *   - Any number of host threads may call at once, each on its own stream:
 *     the library's per-device state and caches are guarded, and results do
 *     not depend on which thread called first (ln_backward_noalloc's shared
 *     array is the one exception; see there).
 *   - Outputs are overwritten, never accumulated into, except where
 *     ln_backward_ex is asked to accumulate.
 *   - Results are deterministic: the same inputs give bitwise-identical
 *     outputs on every call (no floating-point atomics).
 *   - No call works in place: an output must not share a byte with another
 *     output or with an array the call reads (LN_ERR_ALIAS, checked on the
 *     host before anything is launched).  Inputs may overlap one another.
 *     The accumulating backward reads the outputs it adds to; that is the
 *     same array, not an overlap.
 *   - Any alignment is accepted.  Fully 16-byte-aligned arrays with C * size
 *     a multiple of 16 bytes take the vectorised path; others a scalar path.
 *   - Errors are returned as an ln_status value; nothing is launched when
 *     validation fails, and no kernel asserts or traps.
 *   - ln_forward, ln_forward_residual, ln_backward and ln_backward_ex calls
 *     can be captured into a CUDA graph (the backward's workspace then
 *     becomes graph allocation nodes); make one uncaptured call of the same
 *     shape on the device first, so that one-time set-up (the device's memory
 *     pool, kernel attributes) happens outside the capture.
 *   - 1 <= C <= LN_MAX_C; 0 <= N <= LN_MAX_N; N * C <= LN_MAX_ELEMS.
 *     N == 0 launches nothing in the forward; in the backward it only
 *     zero-fills dweight and dbias (pointers other than dweight and dbias
 *     may then be NULL).
 */
#ifndef LN_H
#define LN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, declared here so that C callers need no CUDA
 * header. */
struct CUstream_st;
typedef struct CUstream_st *ln_stream_t;

#define LN_MAX_C ((int64_t)1 << 24)
#define LN_MAX_N ((int64_t)1 << 40)
#define LN_MAX_ELEMS ((int64_t)1 << 50)   /* bound on N * C */

typedef enum {
    LN_F32 = 0,   /* IEEE binary32 */
    LN_BF16 = 1,  /* bfloat16 (8 significant bits, binary32 exponent range) */
    LN_F16 = 2    /* IEEE binary16 (11 significant bits, largest finite 65504) */
} ln_dtype;

typedef enum {
    LN_OK = 0,
    LN_ERR_NULL = 1,       /* a required pointer is NULL */
    LN_ERR_SHAPE = 2,      /* N < 0, N > LN_MAX_N, C < 1, C > LN_MAX_C or
                              N * C > LN_MAX_ELEMS */
    LN_ERR_DTYPE = 3,      /* dtype is not LN_F32, LN_BF16 or LN_F16 */
    LN_ERR_EPS = 4,        /* eps is not finite, or not > 0 */
    LN_ERR_WORKSPACE = 5,  /* the backward's workspace could not be allocated */
    LN_ERR_CUDA = 6,       /* a CUDA runtime call or launch failed */
    LN_ERR_SCRATCH = 7,    /* ln_backward_noalloc: C > LN_NOALLOC_MAX_C */
    LN_ERR_FLAGS = 8,      /* ln_backward_ex: unknown bits in flags */
    LN_ERR_ALIAS = 9       /* an output overlaps another output or an array
                              the call reads */
} ln_status;

/*
 * LayerNorm forward over N rows of C channels.
 *   out   [N*C] dtype, written      normalised, scaled and shifted rows
 *   mean  [N]   fp32,  written      per-row mean
 *   rstd  [N]   fp32,  written      per-row 1/sqrt(var + eps), var biased (1/C)
 *   inp   [N*C] dtype, read
 *   weight, bias [C] dtype, read
 *   eps   finite, > 0 (1e-5 in GPT-2)
 * out, mean and rstd must not overlap one another or inp, weight or bias
 * (LN_ERR_ALIAS).  Returns LN_OK or an ln_status error.
 */
int ln_forward(void *out, float *mean, float *rstd, const void *inp,
               const void *weight, const void *bias, int64_t N, int64_t C,
               float eps, int dtype, ln_stream_t stream);

/*
 * LayerNorm backward for the loss gradient dout, given the statistics that
 * ln_forward saved for the same inp.
 *   dinp    [N*C] dtype, written    gradient w.r.t. inp
 *   dweight [C]   fp32,  written    sum over rows of dout * xhat
 *   dbias   [C]   fp32,  written    sum over rows of dout
 *   dout    [N*C] dtype, read
 *   inp     [N*C] dtype, read
 *   weight  [C]   dtype, read
 *   mean, rstd [N] fp32, read
 * The column sums are formed in two stages with a fixed summation order:
 * per-block partial sums into a library-owned workspace drawn, stream-ordered,
 * from a per-device memory pool (returned to the pool on `stream` after use),
 * then one fixed-order sum of the partials.  dinp, dweight and dbias must
 * not overlap one another or dout, inp, weight, mean or rstd (LN_ERR_ALIAS).
 * Returns LN_OK or an ln_status error (LN_ERR_WORKSPACE when the pool cannot
 * supply the workspace).
 */
int ln_backward(void *dinp, float *dweight, float *dbias, const void *dout,
                const void *inp, const void *weight, const float *mean,
                const float *rstd, int64_t N, int64_t C, int dtype,
                ln_stream_t stream);

/*
 * LayerNorm forward of a residual sum, the step that precedes LayerNorm in a
 * GPT-2 block: "llm.c: Large Language Model Training in Pure C/CUDA Without
 * Dependencies" credits its speed to custom fused kernels (feature list, and
 * the question "Can llm.c achieve competitive training speeds with
 * PyTorch?").  Here the residual add is fused into the forward, so the sum is
 * read from registers instead of being written and read back:
 *   x         = resid + branch, rounded to dtype (each element rounded once,
 *               to nearest-even)
 *   resid_out = x
 *   out, mean, rstd = ln_forward(x)      (the rounded x, so that the saved
 *                                         residual and the statistics agree)
 *   resid_out [N*C] dtype, written       the residual stream after the add
 *   out, mean, rstd                      as in ln_forward
 *   resid, branch [N*C] dtype, read      the two summands
 *   weight, bias [C] dtype, read; eps as in ln_forward
 * resid_out, out, mean and rstd must not overlap one another or any input
 * (no in-place update; LN_ERR_ALIAS).  Bytes moved: 4*N*C*size (two reads, two writes) against 5*N*C*size
 * for a separate add and ln_forward.  Returns LN_OK or an ln_status error.
 */
int ln_forward_residual(void *resid_out, void *out, float *mean, float *rstd,
                        const void *resid, const void *branch, const void *weight,
                        const void *bias, int64_t N, int64_t C, float eps, int dtype,
                        ln_stream_t stream);

/* Flags of ln_backward_ex (bitwise or). */
/* dinp += the gradient: the previous dinp is read and each sum is rounded to
 * dtype once.  For a residual stream, whose gradient is the sum of the
 * branches' gradients ("llm.c: Large Language Model Training in Pure C/CUDA
 * Without Dependencies", question "How does llm.c handle distributed
 * multi-GPU training?": gradients are accumulated locally before they are
 * synchronised). */
#define LN_BWD_ACCUMULATE_DINP 1u
/* dweight += and dbias += the column sums (fp32), e.g. over micro-batches of
 * one optimiser step. */
#define LN_BWD_ACCUMULATE_DPARAMS 2u
/* mean and rstd are recomputed from inp (with eps, exactly as ln_forward
 * computes them) instead of being read; the mean and rstd arguments may then
 * be NULL.  Saves the 8*N bytes of the saved statistics, and lets a caller
 * drop them (activation recomputation). */
#define LN_BWD_RECOMPUTE_STATS 4u

/*
 * ln_backward with variants: flags == 0 is exactly ln_backward (eps is then
 * unused).  Arguments as in ln_backward, plus
 *   eps    finite, > 0; read only with LN_BWD_RECOMPUTE_STATS
 *   flags  a combination of LN_BWD_ACCUMULATE_DINP, LN_BWD_ACCUMULATE_DPARAMS
 *          and LN_BWD_RECOMPUTE_STATS; other bits give LN_ERR_FLAGS
 * With LN_BWD_ACCUMULATE_DINP, dinp is read as well as written (it must hold
 * the previous gradient); with LN_BWD_ACCUMULATE_DPARAMS, dweight and dbias
 * are read and N == 0 leaves them unchanged.  With LN_BWD_RECOMPUTE_STATS
 * mean and rstd are not read, so their overlaps are not checked.  The column
 * sums keep their fixed order, so results stay deterministic.
 */
int ln_backward_ex(void *dinp, float *dweight, float *dbias, const void *dout,
                   const void *inp, const void *weight, const float *mean,
                   const float *rstd, int64_t N, int64_t C, float eps, int dtype,
                   unsigned int flags, ln_stream_t stream);

/*
 * ln_backward_noalloc: the same computation and arguments as ln_backward, for
 * callers that cannot allocate device memory.  (No counterpart on the pages
 * this library follows: it exists for callers, not for the method.)  Who
 * needs it: programs that reserve all device memory in one arena at start-up
 * and forbid allocation afterwards, code running inside another allocator
 * (where an allocation would re-enter it), and hosts whose memory accounting
 * must not see a second pool.  ln_backward takes its partial sums from a
 * stream-ordered pool; this variant keeps them in a static device array of
 * LN_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads the
 * library holds until the process exits.  It calls no cudaMalloc, cudaFree or
 * other allocating routine, and does not create the memory pool that
 * ln_backward uses (a process that only calls this entry point has none).
 *   - The first call on a device (made with that device current) looks up the
 *     array's device address once; make that call before any stream capture.
 *   - All calls share the one array.  Each call overwrites what it reads, so
 *     nothing needs clearing, but calls whose kernels overlap on the GPU
 *     (other streams, other host threads) race on it: serialise them.
 *   - C > LN_NOALLOC_MAX_C (one partial row of 2*C fp32 must fit) returns
 *     LN_ERR_SCRATCH without launching; wide rows run on fewer blocks than
 *     ln_backward would use, so they may be slower.
 * Results match ln_backward within the library's stated tolerances (the
 * column sums may be grouped differently when the array caps the grid).
 */
#define LN_NOALLOC_SCRATCH_BYTES ((int64_t)4 << 20)
#define LN_NOALLOC_MAX_C (LN_NOALLOC_SCRATCH_BYTES / 8)
int ln_backward_noalloc(void *dinp, float *dweight, float *dbias, const void *dout,
                        const void *inp, const void *weight, const float *mean,
                        const float *rstd, int64_t N, int64_t C, int dtype,
                        ln_stream_t stream);

/* Static description of an ln_status value (never NULL). */
const char *ln_status_string(int status);

/* Number of kernels this library has launched in this process (all devices,
 * all streams).  For accounting in benchmarks and tests. */
uint64_t ln_launch_count(void);

/* Diagnostics: the bits that kernels of this library set on the current
 * device when one of their bounded waits ran out (1: a consumer gave up on a
 * stage's data, 2: the producer gave up on a stage's release, 4: a bulk copy
 * in flight did not land in time).  0 means healthy; any other value means
 * the results of the calls since the last clear are not to be trusted.
 * Writes the bits to *bits and, when clear != 0, resets them.  Synchronises
 * the current device.  Returns LN_OK, LN_ERR_NULL or LN_ERR_CUDA. */
int ln_device_status(unsigned int *bits, int clear);

/*
 * Caps the workspace that one ln_backward or ln_backward_ex call on the
 * current device may draw from the pool, in bytes (0, the default: no cap).
 * A call that needs more (G * 2 * C * 4 bytes, G the backward's grid, about
 * the SM count) returns LN_ERR_WORKSPACE before launching anything, exactly
 * as when the pool cannot supply it; the setting stays until changed, and
 * later calls that fit run normally.  For callers that budget device memory
 * per library, and for exercising the workspace-failure path without
 * exhausting a shared GPU.  ln_backward_noalloc is not affected.  Returns
 * LN_OK, LN_ERR_SHAPE for bytes < 0, or LN_ERR_CUDA.
 */
int ln_set_workspace_limit(int64_t bytes);

/*
 * The CUDA error behind the most recent LN_ERR_CUDA returned on the calling
 * host thread: its name, number and description, and the runtime call that
 * raised it (for example "cudaErrorInvalidValue (1: invalid argument) in
 * cudaLaunchKernelEx").  Never NULL; the text is owned by the library and
 * stays valid until the thread's next failing call.  Calls that succeed do
 * not reset it.
 */
const char *ln_last_cuda_error(void);

/* Library ABI version: 3 (2 plus ln_set_workspace_limit and
 * ln_last_cuda_error; 2 was 1 plus ln_forward_residual, ln_backward_ex and
 * LN_F16). */
int ln_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LN_H */
