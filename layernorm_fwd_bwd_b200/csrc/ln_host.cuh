// ln_host.cuh -- host-side plumbing shared by the translation units of
// libln.so: argument bundles, launch helpers and the occupancy cache (whose
// storage, with the launch counter, lives in ln_api.cu), and the dispatch
// entry points that ln_inst.cu instantiates once per element type and
// variant.
#pragma once

#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "../../include/ln.h"

namespace lnh {

// ---- defined in ln_api.cu
bool occ_find(const void *fn, int dev, int threads, size_t smem, int *occ);
void occ_store(const void *fn, int dev, int threads, size_t smem, int occ);
// Makes the kernel's dynamic shared-memory limit on `dev` (the current
// device) at least `smem`.  The limit is one value per kernel and device, so
// it only ever grows: a call with a smaller size leaves the larger limit of
// an earlier call in place.
cudaError_t raise_smem_limit(const void *fn, int dev, size_t smem);
void count_launches(uint64_t n);
// Records, for the calling host thread, the CUDA error behind the
// LN_ERR_CUDA the library is about to return and the call that raised it
// (read back with ln_last_cuda_error); returns LN_ERR_CUDA.
int note_cuda_error(cudaError_t e, const char *call);
// The stream-ordered pool that the pooled backward draws its partial sums
// from on `dev` (created on the first call for that device, with it
// current), and the per-call workspace cap set by ln_set_workspace_limit
// (0: none).
cudaError_t workspace_pool(int dev, cudaMemPool_t *pool, uint64_t *limit);
// Validation and dispatch of every backward entry point; scratch != nullptr
// keeps the partial sums in that device array (scratch_floats floats)
// instead of drawing them from the pool.
int backward_entry(void *dinp, float *dweight, float *dbias, const void *dout,
                   const void *inp, const void *weight, const float *mean, const float *rstd,
                   int64_t N, int64_t C, float eps, int dtype, unsigned flags,
                   ln_stream_t stream, float *scratch, int64_t scratch_floats);

constexpr size_t kMaxWorkspaceBytes = size_t(256) << 20;

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
// Status of a CUDA result whose failure the failing step has already noted
// (launch, blocks_per_sm and raise_smem_limit note their own errors).
inline int status_of(cudaError_t e) { return e == cudaSuccess ? LN_OK : LN_ERR_CUDA; }

// Resident blocks per SM of `kernel` at this block size and dynamic shared
// memory (computed once per kernel, device and size).  Every call, cached or
// not, first makes sure the kernel's dynamic shared-memory limit on that
// device admits `smem`, since a launch is checked against the limit in force
// when it is made, not against the one of the call that filled the cache.
template <typename K>
cudaError_t blocks_per_sm(K kernel, int dev, int threads, size_t smem, int *occ) {
    const void *fn = reinterpret_cast<const void *>(kernel);
    cudaError_t e = raise_smem_limit(fn, dev, smem);
    if (e != cudaSuccess) return e;
    if (occ_find(fn, dev, threads, smem, occ)) return cudaSuccess;
    int n = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem);
    if (e != cudaSuccess) {
        note_cuda_error(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
        return e;
    }
    if (n < 1) {
        note_cuda_error(cudaErrorInvalidConfiguration,
                        "cudaOccupancyMaxActiveBlocksPerMultiprocessor (no block fits an SM)");
        return cudaErrorInvalidConfiguration;
    }
    occ_store(fn, dev, threads, smem, n);
    *occ = n;
    return cudaSuccess;
}

// Every kernel of the library starts with griddepcontrol.wait before any
// global memory access, so every launch may use programmatic stream
// serialization: the next kernel's blocks are scheduled while the current
// one drains, and its first global access still waits for it.
template <typename K, typename... Args>
cudaError_t launch(K kernel, int grid, int threads, size_t smem, cudaStream_t stream,
                   Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
    if (e == cudaSuccess)
        count_launches(1);
    else
        note_cuda_error(e, "cudaLaunchKernelEx");
    return e;
}

// Forward call.  Residual variant: the normalised row is x = inp + branch
// (rounded to the element type), also written to resid_out.
struct FwdArgs {
    void *out;
    float *mean;
    float *rstd;
    const void *inp;
    const void *weight;
    const void *bias;
    void *resid_out;          // residual variant only
    const void *branch;       // residual variant only
    int64_t N;
    int C;
    float inv_C;
    float eps;
    cudaStream_t stream;
    int dev;
    int sms;
    unsigned int *status;     // device status word
};

// Backward call.  The per-block partial sums come from `scratch` (capacity
// scratch_floats, no allocation) when it is set, else from the device's
// workspace pool (workspace_pool).
struct BwdArgs {
    void *dinp;
    float *dweight;
    float *dbias;
    const void *dout;
    const void *inp;
    const void *weight;
    const float *mean;        // unused when recomputing the statistics
    const float *rstd;
    int64_t N;
    int C;
    float inv_C;
    float eps;                // used when recomputing the statistics
    bool accumulate_params;   // dweight/dbias += instead of =
    cudaStream_t stream;
    int dev;
    int sms;
    float *scratch;
    int64_t scratch_floats;
    unsigned int *status;
};

// Instantiated in ln_inst.cu for T in {float, bf16, f16} and every MODE (see
// lnk::kFwdResidual, lnk::kBwdAccumulate, lnk::kBwdRecompute).
template <typename T, int MODE>
int fwd_dispatch(const FwdArgs &a);
template <typename T, int MODE>
int bwd_dispatch(const BwdArgs &a);

}  // namespace lnh
