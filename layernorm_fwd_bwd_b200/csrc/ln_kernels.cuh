// ln_kernels.cuh -- sm_100a kernels for LayerNorm forward and analytical
// backward over flat row-major activations.
//
// Operation: "llm.c's Origin and the Future of LLM Compilers" (CUDA MODE talk
// page), chapter "Deconstructing PyTorch Abstractions and Setting Reference
// Baselines" (forward and backward over bare float arrays), and "llm.c: Large
// Language Model Training in Pure C/CUDA Without Dependencies", feature "Exact
// Analytical Backward Pass".  Techniques: "Building GPT-2 from scratch",
// exercise table, row A3 ("vectorised loads, warp reductions, chasing peak
// bandwidth").
//
// Every kernel here is HBM-bound (about 1-3 flop per byte, no contraction), so
// the design is about bytes in flight and touching each byte once:
//   * a row lives in registers between its reduction passes, loaded once with
//     16-byte streaming loads (ld.global.cs) and written once with 16-byte
//     streaming stores;
//   * statistics are reduced with warp shuffles (one warp per row) or warp
//     shuffles plus one shared-memory exchange (several warps per row);
//   * the mean is taken as pivot + mean(x - pivot) with the pivot x[r, 0], and
//     the variance from the deviations held in registers: a plain fp32 sum of
//     x, or E[x^2] - E[x]^2, loses the variance of rows such as 100 + 0.01 z;
//   * weight and bias are staged once per block in shared memory;
//   * the column sums of the backward are deterministic: each block of the
//     row kernel owns a fixed set of rows (register-resident and scalar
//     kernels: a contiguous range; TMA ring: tiles dealt round-robin over
//     the blocks), accumulates its columns in registers, combines its warps
//     in a fixed order and writes one partial row; a second kernel sums the
//     G partial rows in a fixed order.  Which rows a block owns depends only
//     on N, C and the grid G, and G = SMs x resident blocks per SM (capped
//     by the rows, and by the static array for ln_backward_noalloc), so the
//     bits of dweight/dbias are fixed for a given device model and call, but
//     may differ between devices with different SM counts.  No float atomics
//     anywhere.
// No kernel waits on another block or on a flag: the only cross-kernel
// dependency is programmatic dependent launch (griddepcontrol), resolved by
// the hardware when the producing grid completes.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lnk {

using bf16 = __nv_bfloat16;
using f16 = __half;

// The dynamic shared memory of every kernel in this library, declared once
// with one alignment (128 bytes: TMA bulk-copy destinations and mbarriers are
// carved from it at 128-byte offsets).
extern __shared__ __align__(128) unsigned char ln_dyn_smem[];

// Elements per 16-byte vector.
template <typename T> struct Vec;
template <> struct Vec<float> { static constexpr int E = 4; };
template <> struct Vec<bf16> { static constexpr int E = 8; };
template <> struct Vec<f16> { static constexpr int E = 8; };

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(bf16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float to_f32(f16 v) { return __half2float(v); }

// fp32 -> T, rounded to nearest-even.
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float v) {
    return __float2bfloat16_rn(v);
}
template <> __device__ __forceinline__ f16 from_f32<f16>(float v) { return __float2half_rn(v); }

// Butterfly all-reduce: every lane ends with the same bits (each level adds
// the same two values, in either order).
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ void warp_sum2(float &a, float &b) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        a += __shfl_xor_sync(0xffffffffu, a, o);
        b += __shfl_xor_sync(0xffffffffu, b, o);
    }
}

__device__ __forceinline__ void warp_sum3(float &a, float &b, float &c) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        a += __shfl_xor_sync(0xffffffffu, a, o);
        b += __shfl_xor_sync(0xffffffffu, b, o);
        c += __shfl_xor_sync(0xffffffffu, c, o);
    }
}

// Block-wide sums for the scalar kernels (blockDim.x a multiple of 32).
__device__ __forceinline__ float block_sum(float v, float *slot, int nwarps) {
    v = warp_sum(v);
    if (nwarps == 1) return v;
    if ((threadIdx.x & 31) == 0) slot[threadIdx.x >> 5] = v;
    __syncthreads();
    float tot = 0.f;
    for (int k = 0; k < nwarps; ++k) tot += slot[k];
    return tot;
}

__device__ __forceinline__ void block_sum2(float &a, float &b, float *slot, int nwarps) {
    warp_sum2(a, b);
    if (nwarps == 1) return;
    if ((threadIdx.x & 31) == 0) {
        slot[threadIdx.x >> 5] = a;
        slot[32 + (threadIdx.x >> 5)] = b;
    }
    __syncthreads();
    a = 0.f;
    b = 0.f;
    for (int k = 0; k < nwarps; ++k) {
        a += slot[k];
        b += slot[32 + k];
    }
}

// Programmatic dependent launch (sm_90+).  Every kernel of this library is
// launched with programmatic stream serialization and starts with
// pdl_enter(): it first waits until the previous grid on the stream has
// completed and its writes are visible (so stream order holds for every
// global memory access that follows), then allows the next grid to be
// scheduled.  What overlaps is only the launch and block scheduling of the
// next kernel with the tail of the current one.
__device__ __forceinline__ void pdl_enter() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Packed fp32 pairs.  Blackwell executes add/sub/mul/fma on two fp32 values
// held in one 64-bit register as a single instruction (PTX .f32x2, sm_100+),
// each lane rounded exactly as the scalar instruction would round it.  The
// element math below runs on such pairs, which halves its instruction count.
// ---------------------------------------------------------------------------
typedef unsigned long long f32x2;   // {lo, hi}

__device__ __forceinline__ f32x2 pair(float lo, float hi) {
    f32x2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void split(f32x2 v, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ f32x2 add2(f32x2 a, f32x2 b) {
    f32x2 d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ f32x2 sub2(f32x2 a, f32x2 b) {
    f32x2 d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ f32x2 mul2(f32x2 a, f32x2 b) {
    f32x2 d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ f32x2 fma2(f32x2 a, f32x2 b, f32x2 c) {
    f32x2 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ float hsum(f32x2 v) {
    float lo, hi;
    split(v, lo, hi);
    return lo + hi;
}

// A 16-byte vector of T as P = E/2 fp32 pairs, and back (bf16 and fp16
// rounded to nearest-even).  Element 2k of a 16-bit vector sits in the low
// half of word k (little endian).  Widening a bf16 is placing its 16 bits in
// the high half of a word; fp16 takes the hardware conversion.
template <typename T>
__device__ __forceinline__ void to_pairs(const uint4 &v, f32x2 (&p)[Vec<T>::E / 2]);
template <>
__device__ __forceinline__ void to_pairs<float>(const uint4 &v, f32x2 (&p)[2]) {
    p[0] = pair(__uint_as_float(v.x), __uint_as_float(v.y));
    p[1] = pair(__uint_as_float(v.z), __uint_as_float(v.w));
}
__device__ __forceinline__ f32x2 bf16x2_pair(uint32_t w) {
    return pair(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
__device__ __forceinline__ f32x2 f16x2_pair(uint32_t w) {
    __half2 h;
    memcpy(&h, &w, 4);
    const float2 f = __half22float2(h);
    return pair(f.x, f.y);
}
template <>
__device__ __forceinline__ void to_pairs<bf16>(const uint4 &v, f32x2 (&p)[4]) {
    p[0] = bf16x2_pair(v.x);
    p[1] = bf16x2_pair(v.y);
    p[2] = bf16x2_pair(v.z);
    p[3] = bf16x2_pair(v.w);
}
template <>
__device__ __forceinline__ void to_pairs<f16>(const uint4 &v, f32x2 (&p)[4]) {
    p[0] = f16x2_pair(v.x);
    p[1] = f16x2_pair(v.y);
    p[2] = f16x2_pair(v.z);
    p[3] = f16x2_pair(v.w);
}
// Pair q of a 16-byte vector (q < E/2), unpacked on its own.
template <typename T>
__device__ __forceinline__ f32x2 pair_at(const uint4 &v, int q);
template <>
__device__ __forceinline__ f32x2 pair_at<float>(const uint4 &v, int q) {
    return q == 0 ? pair(__uint_as_float(v.x), __uint_as_float(v.y))
                  : pair(__uint_as_float(v.z), __uint_as_float(v.w));
}
__device__ __forceinline__ uint32_t word_at(const uint4 &v, int q) {
    return q == 0 ? v.x : (q == 1 ? v.y : (q == 2 ? v.z : v.w));
}
template <>
__device__ __forceinline__ f32x2 pair_at<bf16>(const uint4 &v, int q) {
    return bf16x2_pair(word_at(v, q));
}
template <>
__device__ __forceinline__ f32x2 pair_at<f16>(const uint4 &v, int q) {
    return f16x2_pair(word_at(v, q));
}
template <typename T>
__device__ __forceinline__ uint4 from_pairs(const f32x2 (&p)[Vec<T>::E / 2]);
template <>
__device__ __forceinline__ uint4 from_pairs<float>(const f32x2 (&p)[2]) {
    float a, b, c, d;
    split(p[0], a, b);
    split(p[1], c, d);
    return make_uint4(__float_as_uint(a), __float_as_uint(b), __float_as_uint(c),
                      __float_as_uint(d));
}
__device__ __forceinline__ uint32_t pack_bf16x2(f32x2 v) {
    float lo, hi;
    split(v, lo, hi);
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);   // round to nearest-even
    uint32_t w;
    memcpy(&w, &h, 4);
    return w;
}
__device__ __forceinline__ uint32_t pack_f16x2(f32x2 v) {
    float lo, hi;
    split(v, lo, hi);
    __half2 h = __floats2half2_rn(lo, hi);              // round to nearest-even
    uint32_t w;
    memcpy(&w, &h, 4);
    return w;
}
template <>
__device__ __forceinline__ uint4 from_pairs<bf16>(const f32x2 (&p)[4]) {
    return make_uint4(pack_bf16x2(p[0]), pack_bf16x2(p[1]), pack_bf16x2(p[2]),
                      pack_bf16x2(p[3]));
}
template <>
__device__ __forceinline__ uint4 from_pairs<f16>(const f32x2 (&p)[4]) {
    return make_uint4(pack_f16x2(p[0]), pack_f16x2(p[1]), pack_f16x2(p[2]), pack_f16x2(p[3]));
}
// P pairs of fp32 values from shared memory (16-byte aligned address).
template <int P>
__device__ __forceinline__ void smem_pairs(const float *src, f32x2 (&p)[P]) {
    const ulonglong2 *q = reinterpret_cast<const ulonglong2 *>(src);
#pragma unroll
    for (int k = 0; k < P / 2; ++k) {
        const ulonglong2 u = q[k];
        p[2 * k] = u.x;
        p[2 * k + 1] = u.y;
    }
}

// ---------------------------------------------------------------------------
// Kernel variants, chosen at compile time by a MODE template parameter.
// ---------------------------------------------------------------------------
// Forward: the row is x = inp + branch, rounded to T; x is written to
// resid_out and normalised (the rounded x, so that the saved residual stream
// and the statistics describe the same values).
constexpr int kFwdResidual = 1;
// Backward: dinp += the gradient (the previous dinp is read and the sum is
// rounded to T once).
constexpr int kBwdAccumulate = 1;
// Backward: mean and rstd are recomputed from inp with the forward's
// pivot-shifted two-pass statistics instead of being read from the arrays.
constexpr int kBwdRecompute = 2;

// a + b elementwise for two 16-byte vectors of T, each sum rounded to T.
// fp32: the sum itself.  bf16 / fp16: the fp32 sum of two such values is
// exact, or (operands far apart in magnitude) within half an fp32 ulp of a
// value that is far from any bf16 / fp16 rounding boundary, so rounding it to
// nearest-even gives the correctly rounded sum.
template <typename T>
__device__ __forceinline__ uint4 add_round(const uint4 &a, const uint4 &b) {
    constexpr int P = Vec<T>::E / 2;
    f32x2 pa[P], pb[P];
    to_pairs<T>(a, pa);
    to_pairs<T>(b, pb);
#pragma unroll
    for (int q = 0; q < P; ++q) pa[q] = add2(pa[q], pb[q]);
    return from_pairs<T>(pa);
}
// One element of the rounded sum (same value as the vector form).
template <typename T>
__device__ __forceinline__ float add_round1(T a, T b) {
    return to_f32(from_f32<T>(to_f32(a) + to_f32(b)));
}

// Barrier over the TPR threads of one row group (barrier 0 is the block's;
// groups use 1 .. GROUPS).
template <int TPR, int GROUPS>
__device__ __forceinline__ void group_sync(int group) {
    if constexpr (GROUPS == 1) {
        __syncthreads();
    } else {
        asm volatile("bar.sync %0, %1;" ::"r"(group + 1), "r"(TPR) : "memory");
    }
}

// Sum over the W warps of one row group.  `slot` holds 2W floats private to
// the group; callers alternate slots so that a slot is never rewritten before
// every thread of the group has read it.
template <int W, int GROUPS>
__device__ __forceinline__ float group_sum(float v, float *slot, int group, int warp,
                                           int lane) {
    v = warp_sum(v);
    if constexpr (W == 1) {
        return v;
    } else {
        if (lane == 0) slot[warp] = v;
        group_sync<32 * W, GROUPS>(group);
        float tot = 0.f;
#pragma unroll
        for (int k = 0; k < W; ++k) tot += slot[k];
        return tot;
    }
}

template <int W, int GROUPS>
__device__ __forceinline__ void group_sum2(float &a, float &b, float *slot, int group,
                                           int warp, int lane) {
    warp_sum2(a, b);
    if constexpr (W > 1) {
        if (lane == 0) {
            slot[warp] = a;
            slot[W + warp] = b;
        }
        group_sync<32 * W, GROUPS>(group);
        a = 0.f;
        b = 0.f;
#pragma unroll
        for (int k = 0; k < W; ++k) {
            a += slot[k];
            b += slot[W + k];
        }
    }
}

// Shared memory of the vectorised kernels (bytes), shared by every launcher.
template <int W, int GROUPS>
__host__ __device__ constexpr size_t fwd_vec_smem(int C) {
    // weight and bias as fp32, then [GROUPS][2 slots][W] reduction floats
    return size_t(2) * C * 4 + (W > 1 ? size_t(GROUPS) * 2 * W * 4 : 0);
}
template <int W, int GROUPS>
__host__ __device__ constexpr size_t bwd_vec_smem(int C) {
    // weight as fp32, the combine buffer [GROUPS/2][2C], then
    // [GROUPS][2 slots][2W] reduction floats
    return size_t(C) * 4 + (GROUPS > 1 ? size_t(GROUPS / 2) * 2 * C * 4 : 0) +
           (W > 1 ? size_t(GROUPS) * 4 * W * 4 : 0);
}

// ---------------------------------------------------------------------------
// Forward, vectorised path.
//
// A row is owned by TPR = 32*W threads (a row group); thread t of the group
// holds 16-byte vectors j = t + i*TPR (i < V) of the row; a block holds
// GROUPS groups.  Rows go round-robin over a persistent grid.  The row is
// loaded once, turned into deviations from the pivot x[r, 0] and kept in
// registers as fp32 pairs through both reductions.
// With MODE & kFwdResidual the row is inp + branch (rounded to T), which is
// also written to resid_out.
// Requirements (checked by the host): inp, out, weight, bias (and branch,
// resid_out) 16-byte aligned, C * sizeof(T) a multiple of 16, C / E <= V * TPR.
// ---------------------------------------------------------------------------
template <typename T, int V, int W, int GROUPS, int MODE = 0>
__global__ void __launch_bounds__(32 * W * GROUPS)
ln_fwd_vec_kernel(T *__restrict__ out, float *__restrict__ mean, float *__restrict__ rstd,
                  const T *__restrict__ inp, const T *__restrict__ weight,
                  const T *__restrict__ bias, T *__restrict__ resid_out,
                  const T *__restrict__ branch, int64_t N, int C, float inv_C, float eps) {
    pdl_enter();
    constexpr bool RES = (MODE & kFwdResidual) != 0;
    constexpr int E = Vec<T>::E;
    constexpr int P = E / 2;
    constexpr int TPR = 32 * W;
    unsigned char *smem = ln_dyn_smem;
    const int nvec = C / E;
    float *s_w = reinterpret_cast<float *>(smem);
    float *s_b = s_w + C;
    for (int c = threadIdx.x; c < C; c += blockDim.x) {
        s_w[c] = to_f32(weight[c]);
        s_b[c] = to_f32(bias[c]);
    }
    __syncthreads();

    const int group = threadIdx.x / TPR;
    const int t = threadIdx.x - group * TPR;
    const int warp = t >> 5;
    const int lane = threadIdx.x & 31;
    float *s_red = s_b + C + group * 2 * W;      // [2][W] of this group (W > 1)

    for (int64_t r = (int64_t)blockIdx.x * GROUPS + group; r < N;
         r += (int64_t)gridDim.x * GROUPS) {
        const uint4 *xr = reinterpret_cast<const uint4 *>(inp) + r * nvec;
        uint4 xv[V];
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int j = t + i * TPR;
            xv[i] = (j < nvec) ? __ldcs(xr + j) : make_uint4(0u, 0u, 0u, 0u);
        }
        if constexpr (RES) {
            const uint4 *br = reinterpret_cast<const uint4 *>(branch) + r * nvec;
            uint4 *xo = reinterpret_cast<uint4 *>(resid_out) + r * nvec;
            uint4 bv[V];
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const int j = t + i * TPR;
                bv[i] = (j < nvec) ? __ldcs(br + j) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const int j = t + i * TPR;
                xv[i] = add_round<T>(xv[i], bv[i]);
                if (j < nvec) __stcs(xo + j, xv[i]);
            }
        }
        float pivot;
        if constexpr (W == 1) {
            float lo, hi;
            f32x2 p0[P];
            to_pairs<T>(xv[0], p0);            // lane 0 holds columns 0 .. E-1
            split(p0[0], lo, hi);
            pivot = __shfl_sync(0xffffffffu, lo, 0);
        } else if constexpr (RES) {
            pivot = add_round1<T>(inp[r * C], branch[r * C]);
        } else {
            pivot = to_f32(inp[r * C]);
        }
        const f32x2 K = pair(pivot, pivot);

        f32x2 d[V][P];
        f32x2 acc = pair(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const bool ok = t + i * TPR < nvec;
            to_pairs<T>(xv[i], d[i]);
#pragma unroll
            for (int k = 0; k < P; ++k) {
                d[i][k] = sub2(d[i][k], K);
                if (ok) acc = add2(acc, d[i][k]);
            }
        }
        const float mean_d = group_sum<W, GROUPS>(hsum(acc), s_red, group, warp, lane) * inv_C;
        const f32x2 M = pair(mean_d, mean_d);

        f32x2 q = pair(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const bool ok = t + i * TPR < nvec;
#pragma unroll
            for (int k = 0; k < P; ++k) {
                d[i][k] = sub2(d[i][k], M);          // x - mean, from the pivot
                if (ok) q = fma2(d[i][k], d[i][k], q);
            }
        }
        const float var = group_sum<W, GROUPS>(hsum(q), s_red + W, group, warp, lane) * inv_C;
        const float rs = rsqrtf(var + eps);
        const f32x2 R = pair(rs, rs);

        uint4 *yr = reinterpret_cast<uint4 *>(out) + r * nvec;
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int j = t + i * TPR;
            if (j < nvec) {
                f32x2 wp[P], bp[P], o[P];
                smem_pairs<P>(s_w + j * E, wp);
                smem_pairs<P>(s_b + j * E, bp);
#pragma unroll
                for (int k = 0; k < P; ++k) o[k] = fma2(mul2(d[i][k], R), wp[k], bp[k]);
                __stcs(yr + j, from_pairs<T>(o));
            }
        }
        if (t == 0) {
            mean[r] = pivot + mean_d;
            rstd[r] = rs;
        }
    }
}

// ---------------------------------------------------------------------------
// Backward, vectorised path.  Same row ownership as the forward.  Block b
// owns rows [b*rows_per_block, (b+1)*rows_per_block); its row groups take
// rows row0+g, row0+g+GROUPS, ...  Each thread accumulates dout*xhat and dout
// for its own columns over all its rows, as fp32 pairs in registers.  At the
// end the groups are added pairwise in a fixed tree (g += g + GROUPS/2, then
// g += g + GROUPS/4, ...) and group 0 writes partial[b][0:C] (dweight part)
// and partial[b][C:2C] (dbias part).
//   dinp = rstd * (g - mean(g) - xhat * mean(g xhat)) is evaluated as
//   fma(g, rstd, fma(xhat, -rstd*mean(g xhat), -rstd*mean(g))).
// MODE & kBwdAccumulate: the previous dinp vector is loaded where the new one
// is formed and added before rounding.  MODE & kBwdRecompute: mean and rstd come from the
// row itself (pivot x[r, 0], deviations d = (x - pivot) - mean(x - pivot),
// rstd = 1/sqrt(mean(d^2) + eps)), and xhat = d * rstd.
// ---------------------------------------------------------------------------
template <typename T, int V, int W, int GROUPS, int MODE = 0>
__global__ void __launch_bounds__(32 * W * GROUPS, 32 * W * GROUPS <= 256 ? 2 : 1)
ln_bwd_vec_kernel(T *__restrict__ dinp, float *__restrict__ partial,
                  const T *__restrict__ dout, const T *__restrict__ inp,
                  const T *__restrict__ weight, const float *__restrict__ mean,
                  const float *__restrict__ rstd, int64_t N, int C, float inv_C,
                  int64_t rows_per_block, float eps) {
    pdl_enter();
    constexpr bool ACC = (MODE & kBwdAccumulate) != 0;
    constexpr bool RECOMP = (MODE & kBwdRecompute) != 0;
    constexpr int E = Vec<T>::E;
    constexpr int P = E / 2;
    constexpr int TPR = 32 * W;
    unsigned char *smem = ln_dyn_smem;
    const int nvec = C / E;
    float *s_w = reinterpret_cast<float *>(smem);
    float *s_acc = s_w + C;                                   // [GROUPS/2][2C]
    float *s_red0 = s_acc + (GROUPS > 1 ? (GROUPS / 2) * 2 * C : 0);


    for (int c = threadIdx.x; c < C; c += blockDim.x) s_w[c] = to_f32(weight[c]);
    __syncthreads();

    const int group = threadIdx.x / TPR;
    const int t = threadIdx.x - group * TPR;
    const int warp = t >> 5;
    const int lane = threadIdx.x & 31;
    float *s_red = s_red0 + group * 4 * W;                    // [2][2W] of this group

    f32x2 acc_w[V][P], acc_b[V][P];
#pragma unroll
    for (int i = 0; i < V; ++i)
#pragma unroll
        for (int k = 0; k < P; ++k) {
            acc_w[i][k] = pair(0.f, 0.f);
            acc_b[i][k] = pair(0.f, 0.f);
        }

    const int64_t row0 = (int64_t)blockIdx.x * rows_per_block;
    const int64_t row1 = min(N, row0 + rows_per_block);
    int parity = 0;
    for (int64_t r = row0 + group; r < row1; r += GROUPS) {
        const uint4 *xr = reinterpret_cast<const uint4 *>(inp) + r * nvec;
        const uint4 *dr = reinterpret_cast<const uint4 *>(dout) + r * nvec;
        uint4 *gr = reinterpret_cast<uint4 *>(dinp) + r * nvec;
        uint4 xv[V], dv[V];
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int j = t + i * TPR;
            if (j < nvec) {
                xv[i] = __ldcs(xr + j);
                dv[i] = __ldcs(dr + j);
            } else {
                xv[i] = make_uint4(0u, 0u, 0u, 0u);
                dv[i] = xv[i];
            }
        }
        // xhat = (x - K) * S, or ((x - K) - MD) * S when recomputing
        float s;
        f32x2 K, MD = pair(0.f, 0.f);
        if constexpr (RECOMP) {
            float pivot;
            if constexpr (W == 1) {
                float lo, hi;
                f32x2 p0[P];
                to_pairs<T>(xv[0], p0);        // lane 0 holds columns 0 .. E-1
                split(p0[0], lo, hi);
                pivot = __shfl_sync(0xffffffffu, lo, 0);
            } else {
                pivot = to_f32(inp[r * C]);
            }
            K = pair(pivot, pivot);
            f32x2 sd = pair(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < V; ++i) {
                if (t + i * TPR < nvec) {
                    f32x2 x[P];
                    to_pairs<T>(xv[i], x);
#pragma unroll
                    for (int k = 0; k < P; ++k) sd = add2(sd, sub2(x[k], K));
                }
            }
            const float md =
                group_sum<W, GROUPS>(hsum(sd), s_red + parity * 2 * W, group, warp, lane) * inv_C;
            parity ^= 1;
            MD = pair(md, md);
            f32x2 sq = pair(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < V; ++i) {
                if (t + i * TPR < nvec) {
                    f32x2 x[P];
                    to_pairs<T>(xv[i], x);
#pragma unroll
                    for (int k = 0; k < P; ++k) {
                        const f32x2 d = sub2(sub2(x[k], K), MD);
                        sq = fma2(d, d, sq);
                    }
                }
            }
            const float var =
                group_sum<W, GROUPS>(hsum(sq), s_red + parity * 2 * W, group, warp, lane) * inv_C;
            parity ^= 1;
            s = rsqrtf(var + eps);
        } else {
            const float m = __ldg(mean + r);
            s = __ldg(rstd + r);
            K = pair(m, m);
        }
        const f32x2 S = pair(s, s);
        auto xhat = [&](f32x2 x) {
            f32x2 d = sub2(x, K);
            if constexpr (RECOMP) d = sub2(d, MD);
            return mul2(d, S);
        };

        f32x2 s1 = pair(0.f, 0.f), s2 = pair(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int j = t + i * TPR;
            if (j < nvec) {
                f32x2 x[P], dy[P], wp[P];
                to_pairs<T>(xv[i], x);
                to_pairs<T>(dv[i], dy);
                smem_pairs<P>(s_w + j * E, wp);
#pragma unroll
                for (int k = 0; k < P; ++k) {
                    const f32x2 xh = xhat(x[k]);
                    const f32x2 g = mul2(dy[k], wp[k]);
                    s1 = add2(s1, g);
                    s2 = fma2(g, xh, s2);
                }
            }
        }
        float a = hsum(s1), b = hsum(s2);
        group_sum2<W, GROUPS>(a, b, s_red + parity * 2 * W, group, warp, lane);
        parity ^= 1;
        const float na = -s * (a * inv_C);      // -rstd * mean(g)
        const float nc = -s * (b * inv_C);      // -rstd * mean(g xhat)
        const f32x2 NA = pair(na, na);
        const f32x2 NC = pair(nc, nc);

#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int j = t + i * TPR;
            if (j < nvec) {
                f32x2 x[P], dy[P], wp[P], o[P];
                to_pairs<T>(xv[i], x);
                to_pairs<T>(dv[i], dy);
                smem_pairs<P>(s_w + j * E, wp);
#pragma unroll
                for (int k = 0; k < P; ++k) {
                    const f32x2 xh = xhat(x[k]);
                    const f32x2 g = mul2(dy[k], wp[k]);
                    o[k] = fma2(g, S, fma2(xh, NC, NA));
                    acc_w[i][k] = fma2(dy[k], xh, acc_w[i][k]);
                    acc_b[i][k] = add2(acc_b[i][k], dy[k]);
                }
                if constexpr (ACC) {
                    f32x2 pp[P];
                    to_pairs<T>(__ldcs(gr + j), pp);
#pragma unroll
                    for (int k = 0; k < P; ++k) o[k] = add2(o[k], pp[k]);
                }
                __stcs(gr + j, from_pairs<T>(o));
            }
        }
    }

    // Fixed-order tree over the row groups: at each level, groups
    // [h, 2h) park their sums in s_acc and groups [0, h) add them.
    if constexpr (GROUPS > 1) {
#pragma unroll
        for (int h = GROUPS / 2; h >= 1; h /= 2) {
            if (group >= h && group < 2 * h) {
                float *dst = s_acc + (group - h) * 2 * C;
#pragma unroll
                for (int i = 0; i < V; ++i) {
                    const int j = t + i * TPR;
                    if (j < nvec) {
                        ulonglong2 *pw = reinterpret_cast<ulonglong2 *>(dst + j * E);
                        ulonglong2 *pb = reinterpret_cast<ulonglong2 *>(dst + C + j * E);
#pragma unroll
                        for (int k = 0; k < P / 2; ++k) {
                            pw[k] = make_ulonglong2(acc_w[i][2 * k], acc_w[i][2 * k + 1]);
                            pb[k] = make_ulonglong2(acc_b[i][2 * k], acc_b[i][2 * k + 1]);
                        }
                    }
                }
            }
            __syncthreads();
            if (group < h) {
                const float *src = s_acc + group * 2 * C;
#pragma unroll
                for (int i = 0; i < V; ++i) {
                    const int j = t + i * TPR;
                    if (j < nvec) {
                        f32x2 pw[P], pb[P];
                        smem_pairs<P>(src + j * E, pw);
                        smem_pairs<P>(src + C + j * E, pb);
#pragma unroll
                        for (int k = 0; k < P; ++k) {
                            acc_w[i][k] = add2(acc_w[i][k], pw[k]);
                            acc_b[i][k] = add2(acc_b[i][k], pb[k]);
                        }
                    }
                }
            }
            __syncthreads();
        }
    }
    if (group == 0) {
        float *pblk = partial + (int64_t)blockIdx.x * 2 * C;
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int j = t + i * TPR;
            if (j < nvec) {
                ulonglong2 *pw = reinterpret_cast<ulonglong2 *>(pblk + j * E);
                ulonglong2 *pb = reinterpret_cast<ulonglong2 *>(pblk + C + j * E);
#pragma unroll
                for (int k = 0; k < P / 2; ++k) {
                    pw[k] = make_ulonglong2(acc_w[i][2 * k], acc_w[i][2 * k + 1]);
                    pb[k] = make_ulonglong2(acc_b[i][2 * k], acc_b[i][2 * k + 1]);
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Column finalise: dweight[c] = sum_b partial[b][c], dbias[c] =
// sum_b partial[b][C + c], b = 0 .. G-1.  A block of kColsumThreads covers 32
// of the 2C flattened columns with S = kColsumThreads/32 slices: slice y sums
// the partial rows b = y, y + S, ... in increasing order (16 loads issued
// before their adds), then slice 0 adds the S slice sums in order.  The order
// depends on G only, so the result is deterministic.  With accumulate != 0
// the previous dweight[c] / dbias[c] is added to the finished sum.
// ---------------------------------------------------------------------------
constexpr int kColsumThreads = 1024;

static __global__ void __launch_bounds__(kColsumThreads)
ln_colsum_kernel(float *__restrict__ dweight, float *__restrict__ dbias,
                 const float *__restrict__ partial, int G, int C, int accumulate) {
    pdl_enter();
    constexpr int S = kColsumThreads / 32;
    __shared__ float s[S][33];
    const int tx = threadIdx.x & 31;
    const int ty = threadIdx.x >> 5;
    const int64_t twoC = 2 * (int64_t)C;
    const int64_t j = (int64_t)blockIdx.x * 32 + tx;
    float acc = 0.f;
    if (j < twoC) {
        for (int b0 = ty; b0 < G; b0 += S * 16) {
            float v[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const int b = b0 + S * q;
                v[q] = b < G ? partial[(int64_t)b * twoC + j] : 0.f;
            }
#pragma unroll
            for (int q = 0; q < 16; ++q) acc += v[q];
        }
    }
    s[ty][tx] = acc;
    __syncthreads();
    if (ty == 0 && j < twoC) {
        float tot = s[0][tx];
#pragma unroll
        for (int k = 1; k < S; ++k) tot += s[k][tx];
        float *dst = j < C ? dweight + j : dbias + (j - C);
        if (accumulate) tot = *dst + tot;
        *dst = tot;
    }
}

// ---------------------------------------------------------------------------
// Scalar paths: any alignment, any C.  Each element is read with a plain
// scalar load (coalesced across the threads of a row); the row is re-read
// from L1/L2 for each pass instead of being held in registers.
// ---------------------------------------------------------------------------
template <typename T, bool BLOCK_ROW, int MODE = 0>
__global__ void __launch_bounds__(512)
ln_fwd_scalar_kernel(T *__restrict__ out, float *__restrict__ mean,
                     float *__restrict__ rstd, const T *__restrict__ inp,
                     const T *__restrict__ weight, const T *__restrict__ bias,
                     T *__restrict__ resid_out, const T *__restrict__ branch, int64_t N,
                     int C, float inv_C, float eps) {
    pdl_enter();
    constexpr bool RES = (MODE & kFwdResidual) != 0;
    __shared__ float s_red[2][32];
    const int tpr = BLOCK_ROW ? (int)blockDim.x : 32;
    const int groups = blockDim.x / tpr;
    const int group = threadIdx.x / tpr;
    const int t = threadIdx.x - group * tpr;
    const int nwarps = BLOCK_ROW ? (tpr >> 5) : 1;

    for (int64_t r = (int64_t)blockIdx.x * groups + group; r < N;
         r += (int64_t)gridDim.x * groups) {
        const T *x = inp + r * C;
        const T *br = branch + (RES ? r * C : 0);
        // element c of the row (the rounded sum in the residual variant)
        auto xc = [&](int c) {
            if constexpr (RES)
                return add_round1<T>(x[c], br[c]);
            else
                return to_f32(x[c]);
        };
        const float pivot = xc(0);
        float s = 0.f;
        for (int c = t; c < C; c += tpr) s += xc(c) - pivot;
        s = block_sum(s, s_red[0], nwarps);
        const float mean_d = s * inv_C;
        float q = 0.f;
        for (int c = t; c < C; c += tpr) {
            const float d = (xc(c) - pivot) - mean_d;
            q += d * d;
        }
        q = block_sum(q, s_red[1], nwarps);
        const float rs = rsqrtf(q * inv_C + eps);
        T *y = out + r * C;
        for (int c = t; c < C; c += tpr) {
            const float v = xc(c);
            if constexpr (RES) resid_out[r * C + c] = from_f32<T>(v);
            y[c] = from_f32<T>(((v - pivot) - mean_d) * rs * to_f32(weight[c]) +
                               to_f32(bias[c]));
        }
        if (t == 0) {
            mean[r] = pivot + mean_d;
            rstd[r] = rs;
        }
    }
}

// One row at a time per block; thread t owns columns t, t + blockDim, ...
// and accumulates its column sums directly in the block's partial row
// (written on the block's first row, added to afterwards; zero-filled when
// the block has no rows).
template <typename T, int MODE = 0>
__global__ void __launch_bounds__(512)
ln_bwd_scalar_kernel(T *__restrict__ dinp, float *__restrict__ partial,
                     const T *__restrict__ dout, const T *__restrict__ inp,
                     const T *__restrict__ weight, const float *__restrict__ mean,
                     const float *__restrict__ rstd, int64_t N, int C, float inv_C,
                     int64_t rows_per_block, float eps) {
    pdl_enter();
    constexpr bool ACC = (MODE & kBwdAccumulate) != 0;
    constexpr bool RECOMP = (MODE & kBwdRecompute) != 0;
    __shared__ float s_red[2][64];
    const int tpr = blockDim.x;
    const int nwarps = tpr >> 5;
    float *pw = partial + (int64_t)blockIdx.x * 2 * C;
    float *pb = pw + C;
    const int64_t row0 = (int64_t)blockIdx.x * rows_per_block;
    const int64_t row1 = min(N, row0 + rows_per_block);
    int parity = 0;
    bool first = true;
    for (int64_t r = row0; r < row1; ++r) {
        const T *x = inp + r * C;
        const T *dy = dout + r * C;
        // xhat = ((x - K) - md) * s: K = mean[r], md = 0 from the saved
        // statistics, or the pivot x[r, 0] and the mean deviation from it
        float K, md = 0.f, s;
        if constexpr (RECOMP) {
            K = to_f32(x[0]);
            float sd = 0.f;
            for (int c = threadIdx.x; c < C; c += tpr) sd += to_f32(x[c]) - K;
            sd = block_sum(sd, s_red[parity], nwarps);
            parity ^= 1;
            md = sd * inv_C;
            float q = 0.f;
            for (int c = threadIdx.x; c < C; c += tpr) {
                const float d = (to_f32(x[c]) - K) - md;
                q += d * d;
            }
            q = block_sum(q, s_red[parity], nwarps);
            parity ^= 1;
            s = rsqrtf(q * inv_C + eps);
        } else {
            K = mean[r];
            s = rstd[r];
        }
        float s1 = 0.f, s2 = 0.f;
        for (int c = threadIdx.x; c < C; c += tpr) {
            const float xh = ((to_f32(x[c]) - K) - md) * s;
            const float g = to_f32(dy[c]) * to_f32(weight[c]);
            s1 += g;
            s2 += g * xh;
        }
        block_sum2(s1, s2, s_red[parity], nwarps);
        parity ^= 1;
        const float a = s1 * inv_C;
        const float cc = s2 * inv_C;
        T *gx = dinp + r * C;
        for (int c = threadIdx.x; c < C; c += tpr) {
            const float dyc = to_f32(dy[c]);
            const float xh = ((to_f32(x[c]) - K) - md) * s;
            const float g = dyc * to_f32(weight[c]);
            float v = s * (g - a - xh * cc);
            if constexpr (ACC) v += to_f32(gx[c]);
            gx[c] = from_f32<T>(v);
            if (first) {
                pw[c] = dyc * xh;
                pb[c] = dyc;
            } else {
                pw[c] += dyc * xh;
                pb[c] += dyc;
            }
        }
        first = false;
    }
    if (first) {
        for (int c = threadIdx.x; c < C; c += tpr) {
            pw[c] = 0.f;
            pb[c] = 0.f;
        }
    }
}

}  // namespace lnk
