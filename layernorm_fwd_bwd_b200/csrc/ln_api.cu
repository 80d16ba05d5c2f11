// ln_api.cu -- C ABI of libln.so (declared in include/ln.h): argument
// validation, kernel selection, launch geometry and the backward's workspace.
//
// Geometry.  Every kernel runs on a persistent grid of (SM count) x (resident
// blocks per SM, from the occupancy calculator for the exact block size and
// shared memory), capped by the number of rows.  Arrays that are all 16-byte
// aligned, with C * sizeof(T) a multiple of 16, take the vectorised kernels
// (variant chosen in ln_select.cuh); any other call takes the scalar kernels.
//
// Workspace.  The backward needs G * 2C fp32 partial sums (G = its grid).
// They are drawn stream-ordered from a memory pool that the library creates
// once per device (release threshold: never), and handed back on the same
// stream right after the finalise kernel, so calls on different streams never
// share a buffer and steady-state calls reuse pool memory without a
// cudaMalloc.
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>
#include <unordered_map>

#include "../../include/ln.h"
#include "ln_kernels.cuh"
#include "ln_select.cuh"

namespace {

constexpr int kMaxDevices = 64;
constexpr size_t kMaxWorkspaceBytes = size_t(256) << 20;

std::atomic<uint64_t> g_launches{0};

// Bits set by kernels that gave up a bounded wait (see ln_tma.cuh); read with
// ln_device_status().
static __device__ unsigned int ln_status_word;

struct DeviceState {
    std::once_flag once;
    int sms = 0;
    int max_smem_optin = 0;
    cudaMemPool_t pool = nullptr;
    unsigned int *status = nullptr;   // device address of ln_status_word
    cudaError_t init_error = cudaSuccess;
};
DeviceState g_dev[kMaxDevices];

cudaError_t device_state(int dev, DeviceState **out) {
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    DeviceState &d = g_dev[dev];
    std::call_once(d.once, [&]() {
        cudaError_t e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
        if (e == cudaSuccess)
            e = cudaDeviceGetAttribute(&d.max_smem_optin,
                                       cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e == cudaSuccess) {
            cudaMemPoolProps props = {};
            props.allocType = cudaMemAllocationTypePinned;
            props.location.type = cudaMemLocationTypeDevice;
            props.location.id = dev;
            e = cudaMemPoolCreate(&d.pool, &props);
        }
        if (e == cudaSuccess) {
            uint64_t keep = UINT64_MAX;
            e = cudaMemPoolSetAttribute(d.pool, cudaMemPoolAttrReleaseThreshold, &keep);
        }
        if (e == cudaSuccess)
            e = cudaGetSymbolAddress(reinterpret_cast<void **>(&d.status), ln_status_word);
        d.init_error = e;
    });
    *out = &d;
    return d.init_error;
}

// Occupancy (resident blocks per SM) per kernel, device and dynamic shared
// memory size, computed once.
struct OccKey {
    const void *fn;
    int dev;
    int threads;
    size_t smem;
    bool operator==(const OccKey &o) const {
        return fn == o.fn && dev == o.dev && threads == o.threads && smem == o.smem;
    }
};
struct OccHash {
    size_t operator()(const OccKey &k) const {
        return std::hash<const void *>()(k.fn) ^ (size_t(k.dev) << 1) ^
               (size_t(k.threads) << 8) ^ (k.smem << 20);
    }
};
std::mutex g_occ_mu;
std::unordered_map<OccKey, int, OccHash> g_occ;

template <typename K>
cudaError_t blocks_per_sm(K kernel, int dev, int threads, size_t smem, int *occ) {
    const OccKey key{reinterpret_cast<const void *>(kernel), dev, threads, smem};
    {
        std::lock_guard<std::mutex> lk(g_occ_mu);
        auto it = g_occ.find(key);
        if (it != g_occ.end()) {
            *occ = it->second;
            return cudaSuccess;
        }
    }
    cudaError_t e = cudaSuccess;
    if (smem > 48 * 1024)
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
    int n = 0;
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem);
    if (e != cudaSuccess) return e;
    if (n < 1) return cudaErrorInvalidConfiguration;
    std::lock_guard<std::mutex> lk(g_occ_mu);
    g_occ[key] = n;
    *occ = n;
    return cudaSuccess;
}

template <typename K, typename... Args>
cudaError_t launch(K kernel, int grid, int threads, size_t smem, cudaStream_t stream,
                   bool pdl, Args... args) {
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
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
    if (e == cudaSuccess) g_launches.fetch_add(1, std::memory_order_relaxed);
    return e;
}

// Launch with a 1-D thread-block cluster of `cluster` blocks.
template <typename K, typename... Args>
cudaError_t launch_cluster(K kernel, int grid, int threads, size_t smem, cudaStream_t stream,
                           int cluster, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
    if (e == cudaSuccess) g_launches.fetch_add(1, std::memory_order_relaxed);
    return e;
}

// Whether a cluster launch of `kernel` can be resident at all (cached).
template <typename K>
cudaError_t cluster_fits(K kernel, int dev, int threads, size_t smem, int cluster, bool *fits) {
    const OccKey key{reinterpret_cast<const void *>(kernel), dev, -cluster, smem + threads};
    {
        std::lock_guard<std::mutex> lk(g_occ_mu);
        auto it = g_occ.find(key);
        if (it != g_occ.end()) {
            *fits = it->second > 0;
            return cudaSuccess;
        }
    }
    cudaError_t e = cudaSuccess;
    if (smem > 48 * 1024)
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)cluster);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveClusters(&n, kernel, &cfg);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lk(g_occ_mu);
    g_occ[key] = n;
    *fits = n > 0;
    return cudaSuccess;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

int status_of(cudaError_t e) { return e == cudaSuccess ? LN_OK : LN_ERR_CUDA; }

// ------------------------------------------------------------------ forward

struct FwdArgs {
    void *out;
    float *mean;
    float *rstd;
    const void *inp;
    const void *weight;
    const void *bias;
    int64_t N;
    int C;
    float inv_C;
    float eps;
    cudaStream_t stream;
    int dev;
    int sms;
    unsigned int *status;
};

template <typename T>
struct FwdVec {
    const FwdArgs &a;
    cudaError_t err = cudaSuccess;
    template <int V, int W, int GROUPS>
    void run() {
        if constexpr (W == 1 && LN_FWD_STYLE == 2) {
            if (ceil_div(a.N, lnk::kTileWarps * lnk::kTileFwdTiles) <= INT32_MAX) {
                if constexpr (V >= LN_TILE_FWD_W2_FROM_V)
                    run_tile<(V + 1) / 2, 2>();
                else
                    run_tile<V, 1>();
                return;
            }
        }
        if constexpr (W == 1 && LN_FWD_STYLE >= 1) {
            run_tma<V>();
            return;
        }
        auto kern = lnk::ln_fwd_vec_kernel<T, V, W, GROUPS>;
        const int threads = 32 * W * GROUPS;
        const size_t smem = lnk::fwd_vec_smem<W, GROUPS>(a.C);
        int occ = 0;
        err = blocks_per_sm(kern, a.dev, threads, smem, &occ);
        if (err != cudaSuccess) return;
        const int64_t grid = std::min<int64_t>(ceil_div(a.N, GROUPS), int64_t(a.sms) * occ);
        err = launch(kern, (int)grid, threads, smem, a.stream, false,
                     static_cast<T *>(a.out), a.mean, a.rstd,
                     static_cast<const T *>(a.inp), static_cast<const T *>(a.weight),
                     static_cast<const T *>(a.bias), a.N, a.C, a.inv_C, a.eps);
    }
    template <int V, int RW>
    void run_tile() {
        constexpr int E = lnk::Vec<T>::E;
        if (a.C / E == 32 * RW * V)
            run_tile_k<V, RW, true>();
        else
            run_tile_k<V, RW, false>();
    }
    template <int V, int RW, bool FULL>
    void run_tile_k() {
        constexpr int NW = lnk::kTileWarps * RW;          // 8 rows per tile either way
        constexpr int TL = lnk::kTileFwdTiles;
        auto kern = lnk::ln_fwd_tile_kernel<T, V, NW, TL, RW, FULL>;
        const int threads = 32 * NW;
        const size_t smem = lnk::fwd_tile_smem<T, NW, TL, RW>(a.C);
        int occ = 0;
        err = blocks_per_sm(kern, a.dev, threads, smem, &occ);   // also sets the smem limit
        if (err != cudaSuccess) return;
        const int64_t grid = ceil_div(a.N, (NW / RW) * TL);
        err = launch(kern, (int)grid, threads, smem, a.stream, false,
                     static_cast<T *>(a.out), a.mean, a.rstd,
                     static_cast<const T *>(a.inp), static_cast<const T *>(a.weight),
                     static_cast<const T *>(a.bias), a.N, a.C, a.inv_C, a.eps, a.status);
    }
    template <int V>
    void run_tma() {
        constexpr int NC = lnk::kTmaFwdConsumers;
        constexpr int S = lnk::FwdStages<V>::value;
        auto kern = lnk::ln_fwd_tma_kernel<T, V, NC, S>;
        const int threads = 32 * (NC + 1);
        const size_t smem = lnk::fwd_tma_smem<T, NC, S>(a.C);
        int occ = 0;
        err = blocks_per_sm(kern, a.dev, threads, smem, &occ);
        if (err != cudaSuccess) return;
        const int64_t grid = std::min<int64_t>(ceil_div(a.N, NC), int64_t(a.sms) * occ);
        err = launch(kern, (int)grid, threads, smem, a.stream, false,
                     static_cast<T *>(a.out), a.mean, a.rstd,
                     static_cast<const T *>(a.inp), static_cast<const T *>(a.weight),
                     static_cast<const T *>(a.bias), a.N, a.C, a.inv_C, a.eps, a.status);
    }
};

template <typename T, bool BLOCK_ROW>
cudaError_t fwd_scalar(const FwdArgs &a) {
    auto kern = lnk::ln_fwd_scalar_kernel<T, BLOCK_ROW>;
    const int threads = BLOCK_ROW ? (a.C > 4096 ? 512 : 256) : 256;
    const int groups = BLOCK_ROW ? 1 : threads / 32;
    int occ = 0;
    cudaError_t e = blocks_per_sm(kern, a.dev, threads, 0, &occ);
    if (e != cudaSuccess) return e;
    const int64_t grid = std::min<int64_t>(ceil_div(a.N, groups), int64_t(a.sms) * occ);
    return launch(kern, (int)grid, threads, 0, a.stream, false, static_cast<T *>(a.out),
                  a.mean, a.rstd, static_cast<const T *>(a.inp),
                  static_cast<const T *>(a.weight), static_cast<const T *>(a.bias), a.N,
                  a.C, a.inv_C, a.eps);
}

template <typename T>
cudaError_t fwd_dispatch(const FwdArgs &a) {
    constexpr int E = lnk::Vec<T>::E;
    const bool vec_ok = (int64_t(a.C) * sizeof(T)) % 16 == 0 && aligned16(a.out) &&
                        aligned16(a.inp) && aligned16(a.weight) && aligned16(a.bias);
    if (vec_ok) {
        FwdVec<T> v{a};
        if (lnk::visit_fwd_vec<T>(a.C / E, v)) return v.err;
    }
    if (a.C <= 1024) return fwd_scalar<T, false>(a);
    return fwd_scalar<T, true>(a);
}

// ----------------------------------------------------------------- backward

struct BwdArgs {
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
    int dev;
    int sms;
    cudaMemPool_t pool;
    unsigned int *status;
};

// Runs the row kernel on G blocks, then the fixed-order column finalise
// (programmatic dependent launch).  Block b of the row kernel owns
// `per_block` consecutive units of `unit_rows` rows; TMA kernels also take the
// device status word.
template <typename T, bool TMA, typename K>
int bwd_run(const BwdArgs &a, K kern, int threads, size_t smem, int rows_granule,
            int unit_rows) {
    int occ = 0;
    if (blocks_per_sm(kern, a.dev, threads, smem, &occ) != cudaSuccess) return LN_ERR_CUDA;
    const int64_t units = ceil_div(a.N, unit_rows);
    int64_t G = std::min<int64_t>(int64_t(a.sms) * occ, ceil_div(a.N, rows_granule));
    // keep the partial sums within kMaxWorkspaceBytes (matters only for very
    // wide rows, where fewer, longer-running blocks are the price)
    G = std::min<int64_t>(G, int64_t(kMaxWorkspaceBytes / (size_t(a.C) * 2 * sizeof(float))));
    G = std::max<int64_t>(G, 1);
    const int64_t per_block = ceil_div(units, G);
    G = ceil_div(units, per_block);

    float *partial = nullptr;
    const size_t ws_bytes = size_t(G) * 2 * size_t(a.C) * sizeof(float);
    if (cudaMallocFromPoolAsync(reinterpret_cast<void **>(&partial), ws_bytes, a.pool,
                                a.stream) != cudaSuccess) {
        cudaGetLastError();   // clear the non-sticky allocation error
        return LN_ERR_WORKSPACE;
    }
    cudaError_t e;
    if constexpr (TMA) {
        e = launch(kern, (int)G, threads, smem, a.stream, false, static_cast<T *>(a.dinp),
                   partial, static_cast<const T *>(a.dout), static_cast<const T *>(a.inp),
                   static_cast<const T *>(a.weight), a.mean, a.rstd, a.N, a.C, a.inv_C,
                   per_block, a.status);
    } else {
        e = launch(kern, (int)G, threads, smem, a.stream, false, static_cast<T *>(a.dinp),
                   partial, static_cast<const T *>(a.dout), static_cast<const T *>(a.inp),
                   static_cast<const T *>(a.weight), a.mean, a.rstd, a.N, a.C, a.inv_C,
                   per_block * unit_rows);
    }
    if (e == cudaSuccess) {
        const int cblocks = (int)ceil_div(2 * int64_t(a.C), 32);
        e = launch(lnk::ln_colsum_kernel, cblocks, lnk::kColsumThreads, 0, a.stream, true,
                   a.dweight, a.dbias, static_cast<const float *>(partial), (int)G, a.C);
    }
    const cudaError_t ef = cudaFreeAsync(partial, a.stream);
    if (e == cudaSuccess) e = ef;
    return status_of(e);
}

// One-shot tile backward: clusters of kTileCluster blocks, one partial row per
// cluster, then the fixed-order finalise.  Returns -1 when the cluster shape
// cannot be resident (the caller then takes the persistent kernels).
template <typename T, int V>
int bwd_tile_run(const BwdArgs &a) {
    constexpr int NW = lnk::kTileWarps;
    constexpr int TL = lnk::kTileBwdTiles;
    constexpr int CL = lnk::kTileCluster;
    auto kern = lnk::ln_bwd_tile_kernel<T, V, NW, TL, CL>;
    const int threads = 32 * NW;
    const size_t smem = lnk::bwd_tile_smem<T, NW, TL>(a.C);
    const int64_t blocks = ceil_div(ceil_div(a.N, NW * TL), CL) * CL;
    if (blocks > INT32_MAX) return -1;
    bool fits = false;
    if (cluster_fits(kern, a.dev, threads, smem, CL, &fits) != cudaSuccess) {
        cudaGetLastError();
        return -1;
    }
    if (!fits) return -1;
    const int64_t clusters = blocks / CL;
    float *partial = nullptr;
    const size_t ws_bytes = size_t(clusters) * 2 * size_t(a.C) * sizeof(float);
    if (cudaMallocFromPoolAsync(reinterpret_cast<void **>(&partial), ws_bytes, a.pool,
                                a.stream) != cudaSuccess) {
        cudaGetLastError();
        return LN_ERR_WORKSPACE;
    }
    cudaError_t e = launch_cluster(kern, (int)blocks, threads, smem, a.stream, CL,
                                   static_cast<T *>(a.dinp), partial,
                                   static_cast<const T *>(a.dout), static_cast<const T *>(a.inp),
                                   static_cast<const T *>(a.weight), a.mean, a.rstd, a.N, a.C,
                                   a.inv_C, a.status);
    if (e == cudaSuccess) {
        const int cblocks = (int)ceil_div(2 * int64_t(a.C), 32);
        e = launch(lnk::ln_colsum_kernel, cblocks, lnk::kColsumThreads, 0, a.stream, true,
                   a.dweight, a.dbias, static_cast<const float *>(partial), (int)clusters, a.C);
    }
    const cudaError_t ef = cudaFreeAsync(partial, a.stream);
    if (e == cudaSuccess) e = ef;
    return status_of(e);
}

template <typename T>
struct BwdVec {
    const BwdArgs &a;
    int status = LN_OK;
    template <int V, int W, int GROUPS>
    void run() {
        if constexpr (W == 1 && LN_BWD_STYLE == 2) {
            const int st = bwd_tile_run<T, V>(a);
            if (st >= 0) {
                status = st;
                return;
            }
        }
        status = bwd_run<T, false>(a, lnk::ln_bwd_vec_kernel<T, V, W, GROUPS>,
                                   32 * W * GROUPS, lnk::bwd_vec_smem<W, GROUPS>(a.C),
                                   GROUPS, 1);
    }
    template <int V, int W>
    void ring() {
        constexpr int NC = lnk::BwdRingConsumers<W>::value;
        constexpr int S = lnk::BwdStages<V, NC>::value;
        constexpr int RT = NC / W;                        // rows per tile
        status = bwd_run<T, true>(
            a, lnk::ln_bwd_tma_kernel<T, V, NC, S, LN_BWD_RING_RR != 0, W>, 32 * (NC + 1),
            lnk::bwd_tma_smem<T, NC, S, W>(a.C), RT, RT);
    }
};

template <typename T>
int bwd_scalar(const BwdArgs &a) {
    int threads = (int)std::min<int64_t>(512, ceil_div(a.C, 32) * 32);
    return bwd_run<T, false>(a, lnk::ln_bwd_scalar_kernel<T>, threads, 0, 1, 1);
}

template <typename T>
int bwd_dispatch(const BwdArgs &a) {
    constexpr int E = lnk::Vec<T>::E;
    const bool vec_ok = (int64_t(a.C) * sizeof(T)) % 16 == 0 && aligned16(a.dinp) &&
                        aligned16(a.dout) && aligned16(a.inp) && aligned16(a.weight);
    if (vec_ok) {
        BwdVec<T> v{a};
        if (LN_BWD_STYLE == 1 && lnk::visit_bwd_ring<T>(a.C / E, v)) return v.status;
        if (lnk::visit_bwd_vec<T>(a.C / E, v)) return v.status;
    }
    return bwd_scalar<T>(a);
}

int current_device(int *dev, DeviceState **ds) {
    if (cudaGetDevice(dev) != cudaSuccess) return LN_ERR_CUDA;
    if (device_state(*dev, ds) != cudaSuccess) return LN_ERR_CUDA;
    return LN_OK;
}

int check_shape(int64_t N, int64_t C) {
    if (N < 0 || N > LN_MAX_N || C < 1 || C > LN_MAX_C) return LN_ERR_SHAPE;
    if (N > LN_MAX_ELEMS / C) return LN_ERR_SHAPE;
    return LN_OK;
}

}  // namespace

// Launches made by ln_noalloc.cu count in ln_launch_count() too.
void ln_internal_count_launches(uint64_t n) {
    g_launches.fetch_add(n, std::memory_order_relaxed);
}

// Device address of the status word on the current device (nullptr on error).
unsigned int *ln_internal_status_word() {
    int dev = 0;
    DeviceState *ds = nullptr;
    if (current_device(&dev, &ds) != LN_OK) return nullptr;
    return ds->status;
}

extern "C" {

int ln_forward(void *out, float *mean, float *rstd, const void *inp, const void *weight,
               const void *bias, int64_t N, int64_t C, float eps, int dtype,
               ln_stream_t stream) {
    if (int st = check_shape(N, C)) return st;
    if (dtype != LN_F32 && dtype != LN_BF16) return LN_ERR_DTYPE;
    if (!std::isfinite(eps) || !(eps > 0.f)) return LN_ERR_EPS;
    if (N == 0) return LN_OK;
    if (!out || !mean || !rstd || !inp || !weight || !bias) return LN_ERR_NULL;
    int dev = 0;
    DeviceState *ds = nullptr;
    if (int st = current_device(&dev, &ds)) return st;
    FwdArgs a{out, mean, rstd, inp, weight, bias, N, (int)C, 1.0f / float(C), eps,
              reinterpret_cast<cudaStream_t>(stream), dev, ds->sms, ds->status};
    const cudaError_t e = dtype == LN_F32 ? fwd_dispatch<float>(a)
                                          : fwd_dispatch<lnk::bf16>(a);
    return status_of(e);
}

int ln_backward(void *dinp, float *dweight, float *dbias, const void *dout,
                const void *inp, const void *weight, const float *mean, const float *rstd,
                int64_t N, int64_t C, int dtype, ln_stream_t stream) {
    if (int st = check_shape(N, C)) return st;
    if (dtype != LN_F32 && dtype != LN_BF16) return LN_ERR_DTYPE;
    if (!dweight || !dbias) return LN_ERR_NULL;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (N == 0) {
        cudaError_t e = cudaMemsetAsync(dweight, 0, size_t(C) * sizeof(float), s);
        if (e == cudaSuccess) e = cudaMemsetAsync(dbias, 0, size_t(C) * sizeof(float), s);
        return status_of(e);
    }
    if (!dinp || !dout || !inp || !weight || !mean || !rstd) return LN_ERR_NULL;
    int dev = 0;
    DeviceState *ds = nullptr;
    if (int st = current_device(&dev, &ds)) return st;
    BwdArgs a{dinp, dweight, dbias, dout, inp, weight, mean, rstd, N, (int)C,
              1.0f / float(C), s, dev, ds->sms, ds->pool, ds->status};
    return dtype == LN_F32 ? bwd_dispatch<float>(a) : bwd_dispatch<lnk::bf16>(a);
}

const char *ln_status_string(int status) {
    switch (status) {
        case LN_OK: return "LN_OK: success";
        case LN_ERR_NULL: return "LN_ERR_NULL: a required pointer is NULL";
        case LN_ERR_SHAPE: return "LN_ERR_SHAPE: N or C out of range (0 <= N <= 2^40, 1 <= C <= 2^24, N*C <= 2^50)";
        case LN_ERR_DTYPE: return "LN_ERR_DTYPE: dtype must be LN_F32 (0) or LN_BF16 (1)";
        case LN_ERR_EPS: return "LN_ERR_EPS: eps must be finite and > 0";
        case LN_ERR_WORKSPACE: return "LN_ERR_WORKSPACE: backward workspace allocation failed";
        case LN_ERR_CUDA: return "LN_ERR_CUDA: a CUDA runtime call or kernel launch failed";
        case LN_ERR_SCRATCH: return "LN_ERR_SCRATCH: C exceeds the static scratch of ln_backward_noalloc";
        default: return "unknown ln_status";
    }
}

uint64_t ln_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int ln_device_status(unsigned int *bits, int clear) {
    if (!bits) return LN_ERR_NULL;
    int dev = 0;
    DeviceState *ds = nullptr;
    if (int st = current_device(&dev, &ds)) return st;
    if (cudaMemcpy(bits, ds->status, sizeof(unsigned int), cudaMemcpyDeviceToHost) !=
        cudaSuccess)
        return LN_ERR_CUDA;
    if (clear && cudaMemset(ds->status, 0, sizeof(unsigned int)) != cudaSuccess)
        return LN_ERR_CUDA;
    return LN_OK;
}

int ln_version(void) { return 1; }

}  // extern "C"
