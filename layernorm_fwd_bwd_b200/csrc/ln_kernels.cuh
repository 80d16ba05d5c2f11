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
//   * the column sums of the backward are deterministic: each block owns a
//     fixed, contiguous range of rows, accumulates its columns in registers,
//     combines its row groups in a fixed order and writes one partial row;
//     a second kernel sums the partial rows in a fixed order.  No float
//     atomics anywhere.
// No kernel waits on another block or on a flag: the only cross-kernel
// dependency is programmatic dependent launch (griddepcontrol), resolved by
// the hardware when the producing grid completes.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lnk {

using bf16 = __nv_bfloat16;

// Elements per 16-byte vector.
template <typename T> struct Vec;
template <> struct Vec<float> { static constexpr int E = 4; };
template <> struct Vec<bf16> { static constexpr int E = 8; };

__device__ __forceinline__ void unpack(const uint4 &v, float (&f)[4]) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
}

// bf16 element 2k sits in the low half of word k (little endian); widening a
// bf16 to fp32 is placing its 16 bits in the high half of a word.
__device__ __forceinline__ void unpack(const uint4 &v, float (&f)[8]) {
    f[0] = __uint_as_float(v.x << 16);
    f[1] = __uint_as_float(v.x & 0xffff0000u);
    f[2] = __uint_as_float(v.y << 16);
    f[3] = __uint_as_float(v.y & 0xffff0000u);
    f[4] = __uint_as_float(v.z << 16);
    f[5] = __uint_as_float(v.z & 0xffff0000u);
    f[6] = __uint_as_float(v.w << 16);
    f[7] = __uint_as_float(v.w & 0xffff0000u);
}

__device__ __forceinline__ uint4 pack(const float (&f)[4]) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]),
                      __float_as_uint(f[2]), __float_as_uint(f[3]));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);   // round to nearest-even
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ uint4 pack(const float (&f)[8]) {
    return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                      pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
}

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(bf16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float v) {
    return __float2bfloat16_rn(v);
}

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

// Sum over the W warps of one row (W > 1: all threads of the block work on
// the same row).  `slot` holds W floats; callers alternate slots so that a
// slot is never rewritten before every thread has read it.
template <int W>
__device__ __forceinline__ float row_sum(float v, float *slot, int warp, int lane) {
    v = warp_sum(v);
    if constexpr (W == 1) {
        return v;
    } else {
        if (lane == 0) slot[warp] = v;
        __syncthreads();
        float tot = 0.f;
#pragma unroll
        for (int k = 0; k < W; ++k) tot += slot[k];
        return tot;
    }
}

template <int W>
__device__ __forceinline__ void row_sum2(float &a, float &b, float *slot, int warp,
                                         int lane) {
    warp_sum2(a, b);
    if constexpr (W > 1) {
        if (lane == 0) {
            slot[warp] = a;
            slot[W + warp] = b;
        }
        __syncthreads();
        a = 0.f;
        b = 0.f;
#pragma unroll
        for (int k = 0; k < W; ++k) {
            a += slot[k];
            b += slot[W + k];
        }
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

// Programmatic dependent launch (sm_90+): let the next grid on the stream be
// scheduled now / wait until the previous grid has completed and its writes
// are visible.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait_primary() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Forward, vectorised path.
//
// A row is owned by TPR = 32*W threads; thread t holds 16-byte vectors
// j = t + i*TPR (i < V) of the row.  W == 1: GROUPS rows per block, one warp
// per row, shuffle-only reductions.  W > 1: one row per block iteration.
// Rows are distributed round-robin over a persistent grid.
// Requirements (checked by the host): inp, out, weight, bias 16-byte aligned,
// C * sizeof(T) a multiple of 16, C / E <= V * TPR.
// ---------------------------------------------------------------------------
template <typename T, int V, int W, int GROUPS>
__global__ void __launch_bounds__(32 * W * GROUPS)
ln_fwd_vec_kernel(T *__restrict__ out, float *__restrict__ mean, float *__restrict__ rstd,
                  const T *__restrict__ inp, const T *__restrict__ weight,
                  const T *__restrict__ bias, int64_t N, int C, float inv_C, float eps) {
    static_assert(W == 1 || GROUPS == 1, "multi-warp rows run one row per block");
    constexpr int E = Vec<T>::E;
    constexpr int TPR = 32 * W;
    extern __shared__ __align__(16) unsigned char smem[];
    const int nvec = C / E;
    uint4 *s_w = reinterpret_cast<uint4 *>(smem);
    uint4 *s_b = s_w + nvec;
    float *s_red = reinterpret_cast<float *>(s_b + nvec);   // [2][W] when W > 1

    const uint4 *w4 = reinterpret_cast<const uint4 *>(weight);
    const uint4 *b4 = reinterpret_cast<const uint4 *>(bias);
    for (int i = threadIdx.x; i < nvec; i += blockDim.x) {
        s_w[i] = __ldg(w4 + i);
        s_b[i] = __ldg(b4 + i);
    }
    __syncthreads();

    const int group = threadIdx.x / TPR;
    const int t = threadIdx.x - group * TPR;
    const int warp = t >> 5;
    const int lane = threadIdx.x & 31;

    for (int64_t r = (int64_t)blockIdx.x * GROUPS + group; r < N;
         r += (int64_t)gridDim.x * GROUPS) {
        const uint4 *xr = reinterpret_cast<const uint4 *>(inp) + r * nvec;
        uint4 xv[V];
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int j = t + i * TPR;
            xv[i] = (j < nvec) ? __ldcs(xr + j) : make_uint4(0u, 0u, 0u, 0u);
        }
        float pivot;
        if constexpr (W == 1) {
            float f[E];
            unpack(xv[0], f);            // lane 0 holds columns 0 .. E-1
            pivot = __shfl_sync(0xffffffffu, f[0], 0);
        } else {
            pivot = to_f32(inp[r * C]);
        }

        float s = 0.f;
#pragma unroll
        for (int i = 0; i < V; ++i) {
            if (t + i * TPR < nvec) {
                float f[E];
                unpack(xv[i], f);
#pragma unroll
                for (int e = 0; e < E; ++e) s += f[e] - pivot;
            }
        }
        s = row_sum<W>(s, s_red, warp, lane);
        const float mean_d = s * inv_C;         // mean - pivot

        float q = 0.f;
#pragma unroll
        for (int i = 0; i < V; ++i) {
            if (t + i * TPR < nvec) {
                float f[E];
                unpack(xv[i], f);
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const float d = (f[e] - pivot) - mean_d;
                    q += d * d;
                }
            }
        }
        q = row_sum<W>(q, s_red + W, warp, lane);
        const float rs = rsqrtf(q * inv_C + eps);

        uint4 *yr = reinterpret_cast<uint4 *>(out) + r * nvec;
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int j = t + i * TPR;
            if (j < nvec) {
                float f[E], wf[E], bf[E], o[E];
                unpack(xv[i], f);
                unpack(s_w[j], wf);
                unpack(s_b[j], bf);
#pragma unroll
                for (int e = 0; e < E; ++e)
                    o[e] = ((f[e] - pivot) - mean_d) * rs * wf[e] + bf[e];
                __stcs(yr + j, pack(o));
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
// for its own columns over all its rows in registers.  At the end the row
// groups are added in order 0, 1, ..., GROUPS-1 and the block writes
// partial[b][0:C] (dweight part) and partial[b][C:2C] (dbias part).
// ---------------------------------------------------------------------------
template <typename T, int V, int W, int GROUPS>
__global__ void __launch_bounds__(32 * W * GROUPS)
ln_bwd_vec_kernel(T *__restrict__ dinp, float *__restrict__ partial,
                  const T *__restrict__ dout, const T *__restrict__ inp,
                  const T *__restrict__ weight, const float *__restrict__ mean,
                  const float *__restrict__ rstd, int64_t N, int C, float inv_C,
                  int64_t rows_per_block) {
    static_assert(W == 1 || GROUPS == 1, "multi-warp rows run one row per block");
    constexpr int E = Vec<T>::E;
    constexpr int TPR = 32 * W;
    extern __shared__ __align__(16) unsigned char smem[];
    const int nvec = C / E;
    uint4 *s_w = reinterpret_cast<uint4 *>(smem);
    float *s_acc = reinterpret_cast<float *>(s_w + nvec);            // [2C] if GROUPS > 1
    float *s_red = s_acc + (GROUPS > 1 ? 2 * C : 0);                 // [2][2W] if W > 1

    pdl_launch_dependents();

    const uint4 *w4 = reinterpret_cast<const uint4 *>(weight);
    for (int i = threadIdx.x; i < nvec; i += blockDim.x) s_w[i] = __ldg(w4 + i);
    __syncthreads();

    const int group = threadIdx.x / TPR;
    const int t = threadIdx.x - group * TPR;
    const int warp = t >> 5;
    const int lane = threadIdx.x & 31;

    float acc_w[V][E], acc_b[V][E];
#pragma unroll
    for (int i = 0; i < V; ++i)
#pragma unroll
        for (int e = 0; e < E; ++e) {
            acc_w[i][e] = 0.f;
            acc_b[i][e] = 0.f;
        }

    const int64_t row0 = (int64_t)blockIdx.x * rows_per_block;
    const int64_t row1 = min(N, row0 + rows_per_block);
    int parity = 0;
    for (int64_t r = row0 + group; r < row1; r += GROUPS) {
        const uint4 *xr = reinterpret_cast<const uint4 *>(inp) + r * nvec;
        const uint4 *dr = reinterpret_cast<const uint4 *>(dout) + r * nvec;
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
        const float m = __ldg(mean + r);
        const float s = __ldg(rstd + r);

        float s1 = 0.f, s2 = 0.f;
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int j = t + i * TPR;
            if (j < nvec) {
                float x[E], dy[E], wf[E];
                unpack(xv[i], x);
                unpack(dv[i], dy);
                unpack(s_w[j], wf);
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const float xh = (x[e] - m) * s;
                    const float g = dy[e] * wf[e];
                    s1 += g;
                    s2 += g * xh;
                }
            }
        }
        row_sum2<W>(s1, s2, s_red + parity * 2 * W, warp, lane);
        parity ^= 1;
        const float a = s1 * inv_C;     // mean of g
        const float c = s2 * inv_C;     // mean of g * xhat

        uint4 *gr = reinterpret_cast<uint4 *>(dinp) + r * nvec;
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int j = t + i * TPR;
            if (j < nvec) {
                float x[E], dy[E], wf[E], o[E];
                unpack(xv[i], x);
                unpack(dv[i], dy);
                unpack(s_w[j], wf);
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const float xh = (x[e] - m) * s;
                    const float g = dy[e] * wf[e];
                    o[e] = s * (g - a - xh * c);
                    acc_w[i][e] += dy[e] * xh;
                    acc_b[i][e] += dy[e];
                }
                __stcs(gr + j, pack(o));
            }
        }
    }

    float *pblk = partial + (int64_t)blockIdx.x * 2 * C;
    if constexpr (GROUPS == 1) {
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int j = t + i * TPR;
            if (j < nvec) {
                float4 *pw = reinterpret_cast<float4 *>(pblk + j * E);
                float4 *pb = reinterpret_cast<float4 *>(pblk + C + j * E);
#pragma unroll
                for (int k = 0; k < E / 4; ++k) {
                    pw[k] = make_float4(acc_w[i][4 * k], acc_w[i][4 * k + 1],
                                        acc_w[i][4 * k + 2], acc_w[i][4 * k + 3]);
                    pb[k] = make_float4(acc_b[i][4 * k], acc_b[i][4 * k + 1],
                                        acc_b[i][4 * k + 2], acc_b[i][4 * k + 3]);
                }
            }
        }
    } else {
        for (int gi = 0; gi < GROUPS; ++gi) {
            if (group == gi) {
#pragma unroll
                for (int i = 0; i < V; ++i) {
                    const int j = t + i * TPR;
                    if (j < nvec) {
#pragma unroll
                        for (int e = 0; e < E; ++e) {
                            const int col = j * E + e;
                            if (gi == 0) {
                                s_acc[col] = acc_w[i][e];
                                s_acc[C + col] = acc_b[i][e];
                            } else {
                                s_acc[col] += acc_w[i][e];
                                s_acc[C + col] += acc_b[i][e];
                            }
                        }
                    }
                }
            }
            __syncthreads();
        }
        const float4 *src = reinterpret_cast<const float4 *>(s_acc);
        float4 *dst = reinterpret_cast<float4 *>(pblk);
        for (int k = threadIdx.x; k < (2 * C) / 4; k += blockDim.x) dst[k] = src[k];
    }
}

// ---------------------------------------------------------------------------
// Column finalise: dweight[c] = sum_b partial[b][c], dbias[c] =
// sum_b partial[b][C + c], b = 0 .. G-1.  A block covers 32 of the 2C
// flattened columns; its 8 warps each sum the partial rows b = warp,
// warp + 8, ... in increasing order, and warp 0 then adds the 8 results in
// order 0..7.  The order depends on G only, so the result is deterministic.
// ---------------------------------------------------------------------------
static __global__ void __launch_bounds__(256)
ln_colsum_kernel(float *__restrict__ dweight, float *__restrict__ dbias,
                 const float *__restrict__ partial, int G, int C) {
    pdl_wait_primary();
    __shared__ float s[8][33];
    const int tx = threadIdx.x & 31;
    const int ty = threadIdx.x >> 5;
    const int64_t twoC = 2 * (int64_t)C;
    const int64_t j = (int64_t)blockIdx.x * 32 + tx;
    float acc = 0.f;
    if (j < twoC) {
        for (int b = ty; b < G; b += 8) acc += partial[(int64_t)b * twoC + j];
    }
    s[ty][tx] = acc;
    __syncthreads();
    if (ty == 0 && j < twoC) {
        float tot = s[0][tx];
#pragma unroll
        for (int k = 1; k < 8; ++k) tot += s[k][tx];
        if (j < C)
            dweight[j] = tot;
        else
            dbias[j - C] = tot;
    }
}

// ---------------------------------------------------------------------------
// Scalar paths: any alignment, any C.  Each element is read with a plain
// scalar load (coalesced across the threads of a row); the row is re-read
// from L1/L2 for each pass instead of being held in registers.
// ---------------------------------------------------------------------------
template <typename T, bool BLOCK_ROW>
__global__ void __launch_bounds__(512)
ln_fwd_scalar_kernel(T *__restrict__ out, float *__restrict__ mean,
                     float *__restrict__ rstd, const T *__restrict__ inp,
                     const T *__restrict__ weight, const T *__restrict__ bias, int64_t N,
                     int C, float inv_C, float eps) {
    __shared__ float s_red[2][32];
    const int tpr = BLOCK_ROW ? (int)blockDim.x : 32;
    const int groups = blockDim.x / tpr;
    const int group = threadIdx.x / tpr;
    const int t = threadIdx.x - group * tpr;
    const int nwarps = BLOCK_ROW ? (tpr >> 5) : 1;

    for (int64_t r = (int64_t)blockIdx.x * groups + group; r < N;
         r += (int64_t)gridDim.x * groups) {
        const T *x = inp + r * C;
        const float pivot = to_f32(x[0]);
        float s = 0.f;
        for (int c = t; c < C; c += tpr) s += to_f32(x[c]) - pivot;
        s = block_sum(s, s_red[0], nwarps);
        const float mean_d = s * inv_C;
        float q = 0.f;
        for (int c = t; c < C; c += tpr) {
            const float d = (to_f32(x[c]) - pivot) - mean_d;
            q += d * d;
        }
        q = block_sum(q, s_red[1], nwarps);
        const float rs = rsqrtf(q * inv_C + eps);
        T *y = out + r * C;
        for (int c = t; c < C; c += tpr)
            y[c] = from_f32<T>(((to_f32(x[c]) - pivot) - mean_d) * rs * to_f32(weight[c]) +
                               to_f32(bias[c]));
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
template <typename T>
__global__ void __launch_bounds__(512)
ln_bwd_scalar_kernel(T *__restrict__ dinp, float *__restrict__ partial,
                     const T *__restrict__ dout, const T *__restrict__ inp,
                     const T *__restrict__ weight, const float *__restrict__ mean,
                     const float *__restrict__ rstd, int64_t N, int C, float inv_C,
                     int64_t rows_per_block) {
    __shared__ float s_red[2][64];
    pdl_launch_dependents();
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
        const float m = mean[r];
        const float s = rstd[r];
        float s1 = 0.f, s2 = 0.f;
        for (int c = threadIdx.x; c < C; c += tpr) {
            const float xh = (to_f32(x[c]) - m) * s;
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
            const float xh = (to_f32(x[c]) - m) * s;
            const float g = dyc * to_f32(weight[c]);
            gx[c] = from_f32<T>(s * (g - a - xh * cc));
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
