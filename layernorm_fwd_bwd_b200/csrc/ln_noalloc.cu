// ln_noalloc.cu -- ln_backward_noalloc: the LayerNorm backward for callers
// that cannot allocate device memory.
//
// ln_backward draws its per-block partial sums from a stream-ordered memory
// pool.  Some callers cannot let a library allocate: programs that reserve
// all device memory in one arena at start-up and forbid allocation afterwards,
// code that runs inside another allocator (where calling an allocator would
// re-enter it), and hosts whose memory accounting must not see a second pool.
// This entry point computes the same result with its partial sums in a
// file-scope static device array of LN_NOALLOC_SCRATCH_BYTES, which every GPU
// that loads the library holds until the process exits.  It calls no
// cudaMalloc, cudaFree or other allocating routine.
//
// Set-up: the first call on a device (with that device current) looks up the
// array's device address with cudaGetSymbolAddress and caches it; make that
// first call before any stream capture.  In host code the array's name is only
// a host-side stand-in, never a device address, so kernels are always given
// the looked-up pointer.
//
// Sharing: every call uses the same array and the array keeps the previous
// call's contents.  Each block overwrites its whole partial row before the
// finalise reads it, so nothing needs clearing; but calls whose kernels
// overlap on the GPU (different streams, or several host threads) race on the
// array and must be serialised by the caller.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/ln.h"
#include "ln_host.cuh"

static __device__ __align__(256) float ln_noalloc_scratch[LN_NOALLOC_SCRATCH_BYTES / sizeof(float)];

namespace {

constexpr int kMaxDevices = 64;
constexpr int64_t kScratchFloats = LN_NOALLOC_SCRATCH_BYTES / sizeof(float);

struct ScratchDevice {
    std::once_flag once;
    float *scratch = nullptr;   // device address of ln_noalloc_scratch
    cudaError_t err = cudaSuccess;
};
ScratchDevice g_sd[kMaxDevices];

// Runs once per device, with that device current.
cudaError_t scratch_device(int dev, ScratchDevice **out) {
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    ScratchDevice &d = g_sd[dev];
    std::call_once(d.once, [&]() {
        d.err = cudaGetSymbolAddress(reinterpret_cast<void **>(&d.scratch), ln_noalloc_scratch);
    });
    *out = &d;
    return d.err;
}

}  // namespace

extern "C" int ln_backward_noalloc(void *dinp, float *dweight, float *dbias,
                                   const void *dout, const void *inp, const void *weight,
                                   const float *mean, const float *rstd, int64_t N,
                                   int64_t C, int dtype, ln_stream_t stream) {
    if (N < 0 || N > LN_MAX_N || C < 1 || C > LN_MAX_C || N > LN_MAX_ELEMS / C)
        return LN_ERR_SHAPE;
    if (dtype != LN_F32 && dtype != LN_BF16 && dtype != LN_F16) return LN_ERR_DTYPE;
    if (C > LN_NOALLOC_MAX_C) return LN_ERR_SCRATCH;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return lnh::note_cuda_error(e, "cudaGetDevice");
    ScratchDevice *sd = nullptr;
    e = scratch_device(dev, &sd);
    if (e != cudaSuccess)
        return lnh::note_cuda_error(e, "cudaGetSymbolAddress (no-alloc scratch array)");
    return lnh::backward_entry(dinp, dweight, dbias, dout, inp, weight, mean, rstd, N, C, 0.f,
                               dtype, 0u, stream, sd->scratch, kScratchFloats);
}
