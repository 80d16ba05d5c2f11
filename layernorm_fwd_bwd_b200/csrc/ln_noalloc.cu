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

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/ln.h"
#include "ln_kernels.cuh"
#include "ln_select.cuh"

// Defined in ln_api.cu: adds to the count ln_launch_count() reports, and the
// device status word of the current device.
void ln_internal_count_launches(uint64_t n);
unsigned int *ln_internal_status_word();

static __device__ __align__(256) float ln_noalloc_scratch[LN_NOALLOC_SCRATCH_BYTES / sizeof(float)];

namespace {

constexpr int kMaxDevices = 64;
constexpr int64_t kScratchFloats = LN_NOALLOC_SCRATCH_BYTES / sizeof(float);

struct ScratchDevice {
    std::once_flag once;
    float *scratch = nullptr;   // device address of ln_noalloc_scratch
    int sms = 0;
    cudaError_t err = cudaSuccess;
};
ScratchDevice g_sd[kMaxDevices];

// Runs once per device, with that device current.
cudaError_t scratch_device(int dev, ScratchDevice **out) {
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    ScratchDevice &d = g_sd[dev];
    std::call_once(d.once, [&]() {
        cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void **>(&d.scratch),
                                             ln_noalloc_scratch);
        if (e == cudaSuccess)
            e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
        d.err = e;
    });
    *out = &d;
    return d.err;
}

struct Args {
    void *dinp;
    float *dweight;
    float *dbias;
    const void *dout;
    const void *inp;
    const void *weight;
    const float *mean;
    const float *rstd;
    int64_t N;
    int C;
    float inv_C;
    cudaStream_t stream;
    int sms;
    float *scratch;
    unsigned int *status;
};

template <typename K, typename... Ts>
cudaError_t launch(K kernel, int grid, int threads, size_t smem, cudaStream_t stream,
                   bool pdl, Ts... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    // Every kernel here starts with pdl_enter() (griddepcontrol.wait before
    // any global memory access), so programmatic serialization is always
    // safe; `pdl` is kept for call-site readability.
    (void)pdl;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
    if (e == cudaSuccess) ln_internal_count_launches(1);
    return e;
}

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Row kernel on G blocks (block b owns `per_block` consecutive units of
// `unit_rows` rows), then the fixed-order column finalise.
template <typename T, bool TMA, typename K>
int run_kernel(const Args &a, K kern, int threads, size_t smem, int rows_granule,
               int unit_rows) {
    cudaError_t e = cudaSuccess;
    if (smem > 48 * 1024)
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    int occ = 0;
    if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, threads, smem);
    if (e != cudaSuccess || occ < 1) return LN_ERR_CUDA;
    // one partial row of 2C floats per block, all within the static array
    const int64_t units = ceil_div(a.N, unit_rows);
    int64_t G = std::min<int64_t>(int64_t(a.sms) * occ, ceil_div(a.N, rows_granule));
    G = std::min<int64_t>(G, kScratchFloats / (2 * int64_t(a.C)));
    G = std::max<int64_t>(G, 1);
    const int64_t per_block = ceil_div(units, G);
    G = ceil_div(units, per_block);
    if constexpr (TMA) {
        e = launch(kern, (int)G, threads, smem, a.stream, false, static_cast<T *>(a.dinp),
                   a.scratch, static_cast<const T *>(a.dout), static_cast<const T *>(a.inp),
                   static_cast<const T *>(a.weight), a.mean, a.rstd, a.N, a.C, a.inv_C,
                   per_block, a.status);
    } else {
        e = launch(kern, (int)G, threads, smem, a.stream, false, static_cast<T *>(a.dinp),
                   a.scratch, static_cast<const T *>(a.dout), static_cast<const T *>(a.inp),
                   static_cast<const T *>(a.weight), a.mean, a.rstd, a.N, a.C, a.inv_C,
                   per_block * unit_rows);
    }
    if (e == cudaSuccess)
        e = launch(lnk::ln_colsum_kernel, (int)ceil_div(2 * int64_t(a.C), 32),
                   lnk::kColsumThreads, 0, a.stream, true, a.dweight, a.dbias,
                   static_cast<const float *>(a.scratch), (int)G, a.C);
    return e == cudaSuccess ? LN_OK : LN_ERR_CUDA;
}

// One-shot tile backward with cluster partials in the static array; -1 when
// the partial rows do not fit there or the cluster shape cannot be resident.
template <typename T, int V>
int run_tile(const Args &a) {
    constexpr int NW = lnk::kTileWarps;
    constexpr int TL = lnk::kTileBwdTiles;
    constexpr int CL = lnk::kTileCluster;
    auto kern = lnk::ln_bwd_tile_kernel<T, V, NW, TL, CL>;
    const int threads = 32 * NW;
    const size_t smem = lnk::bwd_tile_smem<T, NW, TL>(a.C);
    const int64_t blocks = ceil_div(ceil_div(a.N, NW * TL), CL) * CL;
    const int64_t clusters = blocks / CL;
    if (blocks > INT32_MAX || clusters * 2 * int64_t(a.C) > kScratchFloats) return -1;
    cudaError_t e = cudaSuccess;
    if (smem > 48 * 1024)
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = a.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int nclusters = 0;
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg);
    if (e != cudaSuccess || nclusters < 1) {
        cudaGetLastError();
        return -1;
    }
    e = cudaLaunchKernelEx(&cfg, kern, static_cast<T *>(a.dinp), a.scratch,
                           static_cast<const T *>(a.dout), static_cast<const T *>(a.inp),
                           static_cast<const T *>(a.weight), a.mean, a.rstd, a.N, a.C, a.inv_C,
                           a.status);
    if (e == cudaSuccess) {
        ln_internal_count_launches(1);
        e = launch(lnk::ln_colsum_kernel, (int)ceil_div(2 * int64_t(a.C), 32),
                   lnk::kColsumThreads, 0, a.stream, true, a.dweight, a.dbias,
                   static_cast<const float *>(a.scratch), (int)clusters, a.C);
    }
    return e == cudaSuccess ? LN_OK : LN_ERR_CUDA;
}

template <typename T>
struct Vec {
    const Args &a;
    int status = LN_OK;
    template <int V, int W, int GROUPS>
    void run() {
        if constexpr (W == 1 && LN_BWD_STYLE == 2) {
            const int st = run_tile<T, V>(a);
            if (st >= 0) {
                status = st;
                return;
            }
        }
        status = run_kernel<T, false>(a, lnk::ln_bwd_vec_kernel<T, V, W, GROUPS>,
                                      32 * W * GROUPS, lnk::bwd_vec_smem<W, GROUPS>(a.C),
                                      GROUPS, 1);
    }
    template <int V, int W>
    void ring() {
        constexpr int NC = lnk::BwdRingConsumers<W>::value;
        constexpr int S = lnk::BwdStages<V, NC>::value;
        constexpr int RT = NC / W;                        // rows per tile
        status = run_kernel<T, true>(
            a, lnk::ln_bwd_tma_kernel<T, V, NC, S, LN_BWD_RING_RR != 0, W>, 32 * (NC + 1),
            lnk::bwd_tma_smem<T, NC, S, W>(a.C), RT, RT);
    }
};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <typename T>
int dispatch(const Args &a) {
    constexpr int E = lnk::Vec<T>::E;
    const bool vec_ok = (int64_t(a.C) * sizeof(T)) % 16 == 0 && aligned16(a.dinp) &&
                        aligned16(a.dout) && aligned16(a.inp) && aligned16(a.weight);
    if (vec_ok) {
        Vec<T> v{a};
        if (LN_BWD_STYLE == 1 && lnk::visit_bwd_ring<T>(a.C / E, v)) return v.status;
        if (lnk::visit_bwd_vec<T>(a.C / E, v)) return v.status;
    }
    const int threads = (int)std::min<int64_t>(512, ceil_div(a.C, 32) * 32);
    return run_kernel<T, false>(a, lnk::ln_bwd_scalar_kernel<T>, threads, 0, 1, 1);
}

}  // namespace

extern "C" int ln_backward_noalloc(void *dinp, float *dweight, float *dbias,
                                   const void *dout, const void *inp, const void *weight,
                                   const float *mean, const float *rstd, int64_t N,
                                   int64_t C, int dtype, ln_stream_t stream) {
    if (N < 0 || N > LN_MAX_N || C < 1 || C > LN_MAX_C || N > LN_MAX_ELEMS / C)
        return LN_ERR_SHAPE;
    if (dtype != LN_F32 && dtype != LN_BF16) return LN_ERR_DTYPE;
    if (C > LN_NOALLOC_MAX_C) return LN_ERR_SCRATCH;
    if (!dweight || !dbias) return LN_ERR_NULL;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (N == 0) {
        cudaError_t e = cudaMemsetAsync(dweight, 0, size_t(C) * sizeof(float), s);
        if (e == cudaSuccess) e = cudaMemsetAsync(dbias, 0, size_t(C) * sizeof(float), s);
        return e == cudaSuccess ? LN_OK : LN_ERR_CUDA;
    }
    if (!dinp || !dout || !inp || !weight || !mean || !rstd) return LN_ERR_NULL;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LN_ERR_CUDA;
    ScratchDevice *sd = nullptr;
    if (scratch_device(dev, &sd) != cudaSuccess) return LN_ERR_CUDA;
    unsigned int *status = ln_internal_status_word();
    if (!status) return LN_ERR_CUDA;
    Args a{dinp, dweight, dbias, dout, inp, weight, mean, rstd, N, (int)C,
           1.0f / float(C), s, sd->sms, sd->scratch, status};
    return dtype == LN_F32 ? dispatch<float>(a) : dispatch<lnk::bf16>(a);
}
