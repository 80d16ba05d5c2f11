// ln_api.cu -- C ABI of libln.so (declared in include/ln.h): argument
// validation, per-device state, the occupancy cache and launch counter, and
// the choice of the dispatch instantiation (element type and variant); the
// kernels are selected and launched in ln_dispatch.cuh.
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <mutex>
#include <unordered_map>

#include "../../include/ln.h"
#include "ln_host.cuh"
#include "ln_kernels.cuh"

namespace {

constexpr int kMaxDevices = 64;

std::atomic<uint64_t> g_launches{0};

// Bits set by kernels that gave up a bounded wait (see ln_tma.cuh); read with
// ln_device_status().
static __device__ unsigned int ln_status_word;

struct DeviceState {
    std::once_flag once;
    int sms = 0;
    unsigned int *status = nullptr;   // device address of ln_status_word
    cudaError_t init_error = cudaSuccess;
    // The workspace pool of ln_backward / ln_backward_ex, created on the
    // first pooled call only, so that a process that only ever calls
    // ln_backward_noalloc never creates one.
    std::once_flag pool_once;
    cudaMemPool_t pool = nullptr;
    cudaError_t pool_error = cudaSuccess;
    std::atomic<uint64_t> workspace_limit{0};   // bytes per call; 0: no cap
};
DeviceState g_dev[kMaxDevices];

cudaError_t device_state(int dev, DeviceState **out) {
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    DeviceState &d = g_dev[dev];
    std::call_once(d.once, [&]() {
        cudaError_t e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
        if (e == cudaSuccess)
            e = cudaGetSymbolAddress(reinterpret_cast<void **>(&d.status), ln_status_word);
        d.init_error = e;
    });
    *out = &d;
    return d.init_error;
}

// The last CUDA error behind an LN_ERR_CUDA on this host thread, and the
// call that raised it.
struct LastCudaError {
    cudaError_t code = cudaSuccess;
    const char *call = "";
};
thread_local LastCudaError t_last_error;
thread_local char t_last_error_text[256];

// Occupancy (resident blocks per SM) per kernel, device, block size and
// dynamic shared memory size.
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

int current_device(int *dev, DeviceState **ds) {
    cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess) return lnh::note_cuda_error(e, "cudaGetDevice");
    e = device_state(*dev, ds);
    if (e != cudaSuccess)
        return lnh::note_cuda_error(e, "device set-up (SM count, status word address)");
    return LN_OK;
}

// Smallest dynamic shared-memory limit known to be in force per kernel and
// device (raised by raise_smem_limit, never lowered).
struct FnDev {
    const void *fn;
    int dev;
    bool operator==(const FnDev &o) const { return fn == o.fn && dev == o.dev; }
};
struct FnDevHash {
    size_t operator()(const FnDev &k) const {
        return std::hash<const void *>()(k.fn) ^ (size_t(k.dev) << 1);
    }
};
std::mutex g_smem_mu;
std::unordered_map<FnDev, size_t, FnDevHash> g_smem_limit;

int check_shape(int64_t N, int64_t C) {
    if (N < 0 || N > LN_MAX_N || C < 1 || C > LN_MAX_C) return LN_ERR_SHAPE;
    if (N > LN_MAX_ELEMS / C) return LN_ERR_SHAPE;
    return LN_OK;
}

bool valid_dtype(int dtype) { return dtype == LN_F32 || dtype == LN_BF16 || dtype == LN_F16; }
size_t elem_size(int dtype) { return dtype == LN_F32 ? 4 : 2; }

// Whether the byte ranges [a, a + na) and [b, b + nb) share a byte.
bool overlap(const void *a, size_t na, const void *b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return na && nb && x < y + nb && y < x + na;
}

// One array of a call: its address and size in bytes (0 for an array the
// call does not touch).
struct Span {
    const void *p;
    size_t n;
};

// Whether one of the first n_out spans (the call's outputs) shares a byte
// with any other span of the call.
bool aliased(const Span *s, int n_out, int n) {
    for (int i = 0; i < n_out; ++i)
        for (int j = 0; j < n; ++j)
            if (j != i && overlap(s[i].p, s[i].n, s[j].p, s[j].n)) return true;
    return false;
}
bool valid_eps(float eps) { return std::isfinite(eps) && eps > 0.f; }

template <typename T>
int fwd_call(const lnh::FwdArgs &a, bool residual) {
    return residual ? lnh::fwd_dispatch<T, lnk::kFwdResidual>(a) : lnh::fwd_dispatch<T, 0>(a);
}

template <typename T>
int bwd_call(const lnh::BwdArgs &a, int mode) {
    switch (mode) {
        case 0: return lnh::bwd_dispatch<T, 0>(a);
        case lnk::kBwdAccumulate: return lnh::bwd_dispatch<T, lnk::kBwdAccumulate>(a);
        case lnk::kBwdRecompute: return lnh::bwd_dispatch<T, lnk::kBwdRecompute>(a);
        default:
            return lnh::bwd_dispatch<T, lnk::kBwdAccumulate | lnk::kBwdRecompute>(a);
    }
}

int forward_entry(void *out, float *mean, float *rstd, const void *inp, const void *weight,
                  const void *bias, void *resid_out, const void *branch, bool residual,
                  int64_t N, int64_t C, float eps, int dtype, ln_stream_t stream) {
    if (int st = check_shape(N, C)) return st;
    if (!valid_dtype(dtype)) return LN_ERR_DTYPE;
    if (!valid_eps(eps)) return LN_ERR_EPS;
    if (N == 0) return LN_OK;
    if (!out || !mean || !rstd || !inp || !weight || !bias) return LN_ERR_NULL;
    if (residual && (!resid_out || !branch)) return LN_ERR_NULL;
    const size_t act = size_t(N) * size_t(C) * elem_size(dtype);
    const size_t par = size_t(C) * elem_size(dtype), stat = size_t(N) * sizeof(float);
    const size_t racts = residual ? act : 0;
    const Span spans[] = {{out, act},  {mean, stat},   {rstd, stat}, {resid_out, racts},
                          {inp, act},  {weight, par},  {bias, par},  {branch, racts}};
    if (aliased(spans, 4, 8)) return LN_ERR_ALIAS;
    int dev = 0;
    DeviceState *ds = nullptr;
    if (int st = current_device(&dev, &ds)) return st;
    const lnh::FwdArgs a{out,       mean,       rstd,           inp,
                         weight,    bias,       resid_out,      branch,
                         N,         (int)C,     1.0f / float(C), eps,
                         reinterpret_cast<cudaStream_t>(stream), dev, ds->sms, ds->status};
    switch (dtype) {
        case LN_F32: return fwd_call<float>(a, residual);
        case LN_BF16: return fwd_call<lnk::bf16>(a, residual);
        default: return fwd_call<lnk::f16>(a, residual);
    }
}

}  // namespace

namespace lnh {

bool occ_find(const void *fn, int dev, int threads, size_t smem, int *occ) {
    std::lock_guard<std::mutex> lk(g_occ_mu);
    auto it = g_occ.find(OccKey{fn, dev, threads, smem});
    if (it == g_occ.end()) return false;
    *occ = it->second;
    return true;
}

void occ_store(const void *fn, int dev, int threads, size_t smem, int occ) {
    std::lock_guard<std::mutex> lk(g_occ_mu);
    g_occ[OccKey{fn, dev, threads, smem}] = occ;
}

cudaError_t raise_smem_limit(const void *fn, int dev, size_t smem) {
    if (smem <= 48 * 1024) return cudaSuccess;   // within every kernel's default limit
    std::lock_guard<std::mutex> lk(g_smem_mu);
    size_t &limit = g_smem_limit[FnDev{fn, dev}];
    if (limit >= smem) return cudaSuccess;
    const cudaError_t e =
        cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) {
        note_cuda_error(e, "cudaFuncSetAttribute(MaxDynamicSharedMemorySize)");
        return e;
    }
    limit = smem;
    return cudaSuccess;
}

void count_launches(uint64_t n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

int note_cuda_error(cudaError_t e, const char *call) {
    t_last_error.code = e;
    t_last_error.call = call;
    return LN_ERR_CUDA;
}

cudaError_t workspace_pool(int dev, cudaMemPool_t *pool, uint64_t *limit) {
    DeviceState &d = g_dev[dev];   // dev was validated by device_state
    std::call_once(d.pool_once, [&]() {
        cudaMemPoolProps props = {};
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaError_t e = cudaMemPoolCreate(&d.pool, &props);
        if (e == cudaSuccess) {
            uint64_t keep = UINT64_MAX;
            e = cudaMemPoolSetAttribute(d.pool, cudaMemPoolAttrReleaseThreshold, &keep);
        }
        d.pool_error = e;
    });
    *pool = d.pool;
    *limit = d.workspace_limit.load(std::memory_order_relaxed);
    return d.pool_error;
}

// The backward behind ln_backward, ln_backward_ex and ln_backward_noalloc
// (scratch != nullptr: partial sums in that array instead of the pool).
int backward_entry(void *dinp, float *dweight, float *dbias, const void *dout,
                   const void *inp, const void *weight, const float *mean, const float *rstd,
                   int64_t N, int64_t C, float eps, int dtype, unsigned flags,
                   ln_stream_t stream, float *scratch, int64_t scratch_floats) {
    if (int st = check_shape(N, C)) return st;
    if (!valid_dtype(dtype)) return LN_ERR_DTYPE;
    if (flags & ~unsigned(LN_BWD_ACCUMULATE_DINP | LN_BWD_ACCUMULATE_DPARAMS |
                          LN_BWD_RECOMPUTE_STATS))
        return LN_ERR_FLAGS;
    const bool recompute = (flags & LN_BWD_RECOMPUTE_STATS) != 0;
    const bool acc_params = (flags & LN_BWD_ACCUMULATE_DPARAMS) != 0;
    if (recompute && !valid_eps(eps)) return LN_ERR_EPS;
    if (!dweight || !dbias) return LN_ERR_NULL;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (N == 0) {
        if (acc_params) return LN_OK;   // nothing to add
        cudaError_t e = cudaMemsetAsync(dweight, 0, size_t(C) * sizeof(float), s);
        if (e == cudaSuccess) e = cudaMemsetAsync(dbias, 0, size_t(C) * sizeof(float), s);
        return e == cudaSuccess ? LN_OK : note_cuda_error(e, "cudaMemsetAsync");
    }
    if (!dinp || !dout || !inp || !weight) return LN_ERR_NULL;
    if (!recompute && (!mean || !rstd)) return LN_ERR_NULL;
    const size_t act = size_t(N) * size_t(C) * elem_size(dtype);
    const size_t par = size_t(C) * elem_size(dtype), grad = size_t(C) * sizeof(float);
    const size_t stat = recompute ? 0 : size_t(N) * sizeof(float);   // unread when recomputed
    const Span spans[] = {{dinp, act}, {dweight, grad}, {dbias, grad}, {dout, act},
                          {inp, act},  {weight, par},   {mean, stat},  {rstd, stat}};
    if (aliased(spans, 3, 8)) return LN_ERR_ALIAS;
    int dev = 0;
    DeviceState *ds = nullptr;
    if (int st = current_device(&dev, &ds)) return st;
    const BwdArgs a{dinp,          dweight,   dbias,    dout,     inp,
                    weight,        mean,      rstd,     N,        (int)C,
                    1.0f / float(C), eps,     acc_params, s,      dev,
                    ds->sms,       scratch,   scratch_floats, ds->status};
    const int mode = ((flags & LN_BWD_ACCUMULATE_DINP) ? lnk::kBwdAccumulate : 0) |
                     (recompute ? lnk::kBwdRecompute : 0);
    switch (dtype) {
        case LN_F32: return bwd_call<float>(a, mode);
        case LN_BF16: return bwd_call<lnk::bf16>(a, mode);
        default: return bwd_call<lnk::f16>(a, mode);
    }
}

}  // namespace lnh

extern "C" {

int ln_forward(void *out, float *mean, float *rstd, const void *inp, const void *weight,
               const void *bias, int64_t N, int64_t C, float eps, int dtype,
               ln_stream_t stream) {
    return forward_entry(out, mean, rstd, inp, weight, bias, nullptr, nullptr, false, N, C, eps,
                         dtype, stream);
}

int ln_forward_residual(void *resid_out, void *out, float *mean, float *rstd,
                        const void *resid, const void *branch, const void *weight,
                        const void *bias, int64_t N, int64_t C, float eps, int dtype,
                        ln_stream_t stream) {
    return forward_entry(out, mean, rstd, resid, weight, bias, resid_out, branch, true, N, C,
                         eps, dtype, stream);
}

int ln_backward(void *dinp, float *dweight, float *dbias, const void *dout,
                const void *inp, const void *weight, const float *mean, const float *rstd,
                int64_t N, int64_t C, int dtype, ln_stream_t stream) {
    return lnh::backward_entry(dinp, dweight, dbias, dout, inp, weight, mean, rstd, N, C, 0.f,
                               dtype, 0u, stream, nullptr, 0);
}

int ln_backward_ex(void *dinp, float *dweight, float *dbias, const void *dout,
                   const void *inp, const void *weight, const float *mean, const float *rstd,
                   int64_t N, int64_t C, float eps, int dtype, unsigned int flags,
                   ln_stream_t stream) {
    return lnh::backward_entry(dinp, dweight, dbias, dout, inp, weight, mean, rstd, N, C, eps,
                               dtype, flags, stream, nullptr, 0);
}

const char *ln_status_string(int status) {
    switch (status) {
        case LN_OK: return "LN_OK: success";
        case LN_ERR_NULL: return "LN_ERR_NULL: a required pointer is NULL";
        case LN_ERR_SHAPE: return "LN_ERR_SHAPE: N or C out of range (0 <= N <= 2^40, 1 <= C <= 2^24, N*C <= 2^50)";
        case LN_ERR_DTYPE: return "LN_ERR_DTYPE: dtype must be LN_F32 (0), LN_BF16 (1) or LN_F16 (2)";
        case LN_ERR_EPS: return "LN_ERR_EPS: eps must be finite and > 0";
        case LN_ERR_WORKSPACE: return "LN_ERR_WORKSPACE: backward workspace allocation failed";
        case LN_ERR_CUDA: return "LN_ERR_CUDA: a CUDA runtime call or kernel launch failed";
        case LN_ERR_SCRATCH: return "LN_ERR_SCRATCH: C exceeds the static scratch of ln_backward_noalloc";
        case LN_ERR_FLAGS: return "LN_ERR_FLAGS: unknown bits in the flags of ln_backward_ex";
        case LN_ERR_ALIAS: return "LN_ERR_ALIAS: an output overlaps an input or another output";
        default: return "unknown ln_status";
    }
}

uint64_t ln_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int ln_device_status(unsigned int *bits, int clear) {
    if (!bits) return LN_ERR_NULL;
    int dev = 0;
    DeviceState *ds = nullptr;
    if (int st = current_device(&dev, &ds)) return st;
    cudaError_t e = cudaMemcpy(bits, ds->status, sizeof(unsigned int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return lnh::note_cuda_error(e, "cudaMemcpy (device status word)");
    if (clear && (e = cudaMemset(ds->status, 0, sizeof(unsigned int))) != cudaSuccess)
        return lnh::note_cuda_error(e, "cudaMemset (device status word)");
    return LN_OK;
}

int ln_set_workspace_limit(int64_t bytes) {
    if (bytes < 0) return LN_ERR_SHAPE;
    int dev = 0;
    DeviceState *ds = nullptr;
    if (int st = current_device(&dev, &ds)) return st;
    ds->workspace_limit.store(uint64_t(bytes), std::memory_order_relaxed);
    return LN_OK;
}

const char *ln_last_cuda_error(void) {
    const LastCudaError &l = t_last_error;
    if (l.code == cudaSuccess) return "no CUDA error recorded on this thread";
    snprintf(t_last_error_text, sizeof t_last_error_text, "%s (%d: %s) in %s",
             cudaGetErrorName(l.code), int(l.code), cudaGetErrorString(l.code), l.call);
    return t_last_error_text;
}

int ln_version(void) { return 3; }

}  // extern "C"
