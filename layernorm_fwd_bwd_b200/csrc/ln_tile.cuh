// ln_tile.cuh -- one-shot tile kernels: each block streams a fixed set of row
// tiles into shared memory with TMA bulk copies, uses every stage exactly
// once, and exits.
//
// Why one-shot.  Measured on B200 with copy kernels of the LayerNorm access
// pattern (no arithmetic): short-lived blocks that each move 16 rows reach
// 5.6 TB/s (forward-shaped, 100 MB in + 100 MB out) and 6.1 TB/s
// (backward-shaped, 2 x 100 MB in + 100 MB out), while persistent grids that
// loop over rows stay near 5.2 and 5.7 TB/s.  Issuing all of a block's copies
// at once also keeps the bytes in flight in shared memory rather than in
// registers, and since no stage is ever refilled there is no stage-release
// protocol and no write-after-read hazard between warps and the copy engine.
//
// Layout of a block: NW warps; the block covers TILES tiles of NW
// consecutive rows (row r of tile t is handled by warp r % NW).  Thread 0
// initialises one mbarrier per tile (plus one for the parameters), issues
// every bulk copy, and the warps wait (bounded) on their tile's barrier.
//
// Backward column sums.  One-shot blocks would each need a partial row of
// dweight/dbias; instead blocks form clusters of CL blocks.  Each block adds
// its warps' column sums in a fixed tree into shared memory, the cluster
// synchronises, block rank k adds slice k of the CL block sums (ranks in
// order 0..CL-1) through distributed shared memory and writes it to the
// cluster's partial row; a second cluster barrier keeps every block's shared
// memory alive until those reads are done.  One partial row per cluster, fixed
// summation order: deterministic.
#pragma once

#include <cooperative_groups.h>

#include "ln_tma.cuh"

namespace lnk {

// Shared memory: [128 B barriers][params: n * C * sizeof(T), 128-aligned]
//                [tiles: TILES * NW * row_bytes * arrays][backward: 2C fp32]
template <typename T, int NW, int TILES, int W = 1>
__host__ __device__ constexpr size_t fwd_tile_smem(int C) {
    // barriers, raw weight + bias, TILES tiles of NW / W rows, and the
    // row-group exchange slots when rows are shared by W > 1 warps
    return 128 + align128(size_t(2) * C * sizeof(T)) +
           align128(size_t(TILES) * (NW / W) * C * sizeof(T)) +
           (W > 1 ? size_t(NW / W) * 2 * 3 * W * 4 : 0);
}
template <typename T, int NW, int TILES>
__host__ __device__ constexpr size_t bwd_tile_tiles_bytes(int C) {
    const size_t tiles = size_t(TILES) * NW * 2 * C * sizeof(T);
    const size_t tree = size_t(NW / 2) * 2 * C * 4;           // reuses the tile area
    return align128(tiles > tree ? tiles : tree);
}
template <typename T, int NW, int TILES>
__host__ __device__ constexpr size_t bwd_tile_smem(int C) {
    return 128 + align128(size_t(C) * sizeof(T)) + bwd_tile_tiles_bytes<T, NW, TILES>(C) +
           size_t(2) * C * 4;
}

// Waits on `bar` (phase 0); on timeout records the error and returns false.
__device__ __forceinline__ bool tile_wait(uint64_t *bar, unsigned *status, unsigned bit) {
    if (mbar_wait(bar, 0)) return true;
    atomicOr(status, bit);
    return false;
}

// ---------------------------------------------------------------------------
// Forward.  NW warps; W warps share a row, so a tile holds RT = NW / W rows
// and the block covers TILES tiles.  Warp w serves row w / W of each tile and
// vectors j = (w % W) * 32 + lane + i * 32 * W of it.  The pivot is the row's
// first element, read from shared memory by every warp of the row; with
// W > 1 the row sums meet through group_exchange (ln_tma.cuh).
// Requirements (checked by the host): inp/out/weight/bias 16-byte aligned,
// C * sizeof(T) a multiple of 16, C / E <= 32 * W * V (== when FULL).
// ---------------------------------------------------------------------------
template <typename T, int V, int NW, int TILES, int W = 1, bool FULL = false>
__global__ void __launch_bounds__(32 * NW)
ln_fwd_tile_kernel(T *__restrict__ out, float *__restrict__ mean, float *__restrict__ rstd,
                   const T *__restrict__ inp, const T *__restrict__ weight,
                   const T *__restrict__ bias, int64_t N, int C, float inv_C, float eps,
                   unsigned *__restrict__ status) {
    pdl_enter();
    static_assert(TILES + 1 <= 16, "barriers fit in 128 bytes");
    static_assert(NW % W == 0 && NW / W <= 15, "row groups");
    constexpr int E = Vec<T>::E;
    constexpr int P = E / 2;
    constexpr int RT = NW / W;                                // rows per tile
    constexpr int TPR = 32 * W;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem);      // [0]: params, [1+t]: tile t
    const uint32_t row_bytes = uint32_t(C) * sizeof(T);
    unsigned char *s_par = smem + 128;                         // weight then bias, raw
    unsigned char *s_tiles = s_par + align128(size_t(2) * row_bytes);
    float *s_red = reinterpret_cast<float *>(
        s_tiles + align128(size_t(TILES) * RT * row_bytes));   // [RT][2][3W] (W > 1)
    // FULL: the row is exactly 32 * W * V vectors, so no lane is ever past
    // its end and every bound check below folds away at compile time
    const int nvec = FULL ? 32 * W * V : C / E;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int group = warp / W;
    const int sub = warp - group * W;
    const int t = sub * 32 + lane;
    const int64_t row0 = int64_t(blockIdx.x) * (RT * TILES);

    if (threadIdx.x == 0) {
        for (int k = 0; k <= TILES; ++k) mbar_init(&bars[k], 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(&bars[0], 2 * row_bytes);
        bulk_load(s_par, weight, row_bytes, &bars[0]);
        bulk_load(s_par + row_bytes, bias, row_bytes, &bars[0]);
        for (int k = 0; k < TILES; ++k) {
            const int64_t r = row0 + int64_t(k) * RT;
            if (r < N) {
                const uint32_t bytes = uint32_t(min64(RT, N - r)) * row_bytes;
                mbar_arrive_expect_tx(&bars[1 + k], bytes);
                bulk_load(s_tiles + size_t(k) * RT * row_bytes,
                          reinterpret_cast<const unsigned char *>(inp) + r * row_bytes, bytes,
                          &bars[1 + k]);
            }
        }
    }
    __syncthreads();

    // weight and bias stay in shared memory (raw dtype) and are read where
    // they are used, so nothing row-invariant occupies registers
    const uint4 *ws = reinterpret_cast<const uint4 *>(s_par);
    const uint4 *bs = reinterpret_cast<const uint4 *>(s_par + row_bytes);
    // A warp whose wait runs out records it; with W > 1 it still follows its
    // row's exchanges (on meaningless data) so that the row's warps leave
    // together.
    bool abort = !tile_wait(&bars[0], status, kStatusWaitFull);
    int parity = 0;
#pragma unroll 1
    for (int k = 0; k < TILES; ++k) {
        if (abort && W == 1) break;
        const int64_t r = row0 + int64_t(k) * RT + group;
        if (r >= N) break;                                    // uniform over the row group
        if (!tile_wait(&bars[1 + k], status, kStatusWaitFull)) abort = true;
        if (abort && W == 1) break;
        const unsigned char *row = s_tiles + (size_t(k) * RT + group) * row_bytes;
        const uint4 *src = reinterpret_cast<const uint4 *>(row);
        uint4 xv[V];
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int j = t + TPR * i;
            xv[i] = j < nvec ? src[j] : make_uint4(0u, 0u, 0u, 0u);
        }
        const float pivot = to_f32(reinterpret_cast<const T *>(row)[0]);
        const f32x2 K = pair(pivot, pivot);
        f32x2 d[V][P];
        f32x2 acc = pair(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const bool in = t + TPR * i < nvec;
            to_pairs(xv[i], d[i]);
#pragma unroll
            for (int q = 0; q < P; ++q) {
                d[i][q] = sub2(d[i][q], K);
                if (in) acc = add2(acc, d[i][q]);
            }
        }
        float sum = warp_sum(hsum(acc)), unused = 0.f;
        abort = group_exchange<W>(sum, unused, abort, s_red + (group * 2 + parity) * 3 * W,
                                  group, sub, lane);
        parity ^= 1;
        const float mean_d = sum * inv_C;
        const f32x2 M = pair(mean_d, mean_d);
        f32x2 sq = pair(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const bool in = t + TPR * i < nvec;
#pragma unroll
            for (int q = 0; q < P; ++q) {
                d[i][q] = sub2(d[i][q], M);
                if (in) sq = fma2(d[i][q], d[i][q], sq);
            }
        }
        float var = warp_sum(hsum(sq));
        abort = group_exchange<W>(var, unused, abort, s_red + (group * 2 + parity) * 3 * W,
                                  group, sub, lane);
        parity ^= 1;
        const float rs = rsqrtf(var * inv_C + eps);
        const f32x2 R = pair(rs, rs);
        uint4 *yr = reinterpret_cast<uint4 *>(out) + r * nvec;
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int j = t + TPR * i;
            if (j < nvec) {
                f32x2 wp[P], bp[P], o[P];
                to_pairs(ws[j], wp);
                to_pairs(bs[j], bp);
#pragma unroll
                for (int q = 0; q < P; ++q) o[q] = fma2(mul2(d[i][q], R), wp[q], bp[q]);
                __stcs(yr + j, from_pairs(o));
            }
        }
        if (t == 0) {
            mean[r] = pivot + mean_d;
            rstd[r] = rs;
        }
        if (abort) break;                                     // the row group leaves together
    }
    // No block may exit while one of its copies still writes shared memory:
    // after a timeout, thread 0 waits (bounded) for every copy it issued.
    if (!__syncthreads_and(!abort) && threadIdx.x == 0) {
        for (int k = 0; k <= TILES; ++k) {
            if (k > 0 && row0 + int64_t(k - 1) * RT >= N) break;
            if (!mbar_wait(&bars[k], 0)) atomicOr(status, kStatusDrain);
        }
    }
}

// ---------------------------------------------------------------------------
// Backward.  Block: NW warps x TILES tiles of NW rows; clusters of CL blocks
// (grid padded to a multiple of CL; blocks past the last row contribute
// zeros).  partial[cluster][0:C] / [C:2C] receive the cluster's dweight /
// dbias sums.
// ---------------------------------------------------------------------------
template <typename T, int V, int NW, int TILES, int CL>
__global__ void __launch_bounds__(32 * NW)
ln_bwd_tile_kernel(T *__restrict__ dinp, float *__restrict__ partial,
                   const T *__restrict__ dout, const T *__restrict__ inp,
                   const T *__restrict__ weight, const float *__restrict__ mean,
                   const float *__restrict__ rstd, int64_t N, int C, float inv_C,
                   unsigned *__restrict__ status) {
    pdl_enter();
    static_assert(TILES + 1 <= 16, "barriers fit in 128 bytes");
    static_assert(NW >= 2 && NW <= 16, "warps per block");
    namespace cg = cooperative_groups;
    constexpr int E = Vec<T>::E;
    constexpr int P = E / 2;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem);
    const uint32_t row_bytes = uint32_t(C) * sizeof(T);
    unsigned char *s_w = smem + 128;
    unsigned char *s_tiles = s_w + align128(row_bytes);
    float *s_part = reinterpret_cast<float *>(s_tiles + bwd_tile_tiles_bytes<T, NW, TILES>(C));
    const int nvec = C / E;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t row0 = int64_t(blockIdx.x) * (NW * TILES);
    const size_t tile_bytes = size_t(NW) * row_bytes;         // one array of one tile
    const bool has_rows = row0 < N;                           // false: cluster padding


    if (threadIdx.x == 0) {
        for (int t = 0; t <= TILES; ++t) mbar_init(&bars[t], 1);
        fence_mbar_init();
    }
    if (threadIdx.x == 0 && has_rows) {
        mbar_arrive_expect_tx(&bars[0], row_bytes);
        bulk_load(s_w, weight, row_bytes, &bars[0]);
        for (int t = 0; t < TILES; ++t) {
            const int64_t r = row0 + int64_t(t) * NW;
            if (r < N) {
                const uint32_t bytes = uint32_t(min64(NW, N - r)) * row_bytes;
                unsigned char *dst = s_tiles + size_t(t) * 2 * tile_bytes;
                mbar_arrive_expect_tx(&bars[1 + t], 2 * bytes);
                bulk_load(dst, reinterpret_cast<const unsigned char *>(inp) + r * row_bytes, bytes,
                          &bars[1 + t]);
                bulk_load(dst + tile_bytes,
                          reinterpret_cast<const unsigned char *>(dout) + r * row_bytes, bytes,
                          &bars[1 + t]);
            }
        }
    }
    // statistics of this warp's rows, fetched while the copies are in flight
    float m_t[TILES], s_t[TILES];
#pragma unroll
    for (int t = 0; t < TILES; ++t) {
        const int64_t r = row0 + int64_t(t) * NW + warp;
        m_t[t] = r < N ? __ldg(mean + r) : 0.f;
        s_t[t] = r < N ? __ldg(rstd + r) : 0.f;
    }
    __syncthreads();

    f32x2 acc_w[V][P], acc_b[V][P];
#pragma unroll
    for (int i = 0; i < V; ++i)
#pragma unroll
        for (int q = 0; q < P; ++q) {
            acc_w[i][q] = pair(0.f, 0.f);
            acc_b[i][q] = pair(0.f, 0.f);
        }

    const uint4 *ws = reinterpret_cast<const uint4 *>(s_w);     // read where used
    bool ok = !has_rows || tile_wait(&bars[0], status, kStatusWaitFull);
#pragma unroll
    for (int t = 0; t < TILES; ++t) {
        const int64_t r = row0 + int64_t(t) * NW + warp;
        if (!ok || r >= N) break;                             // warp-uniform
        if (!tile_wait(&bars[1 + t], status, kStatusWaitFull)) {
            ok = false;
            break;
        }
        const unsigned char *base = s_tiles + size_t(t) * 2 * tile_bytes + size_t(warp) * row_bytes;
        const uint4 *xs = reinterpret_cast<const uint4 *>(base);
        const uint4 *ds = reinterpret_cast<const uint4 *>(base + tile_bytes);
        uint4 xv[V], dv[V];
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int j = lane + 32 * i;
            xv[i] = j < nvec ? xs[j] : make_uint4(0u, 0u, 0u, 0u);
            dv[i] = j < nvec ? ds[j] : make_uint4(0u, 0u, 0u, 0u);
        }
        const float m = m_t[t], s = s_t[t];
        const f32x2 M = pair(m, m);
        const f32x2 Sx = pair(s, s);
        f32x2 s1 = pair(0.f, 0.f), s2 = pair(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < V; ++i) {
            if (lane + 32 * i < nvec) {
                f32x2 x[P], dy[P], wp[P];
                to_pairs(xv[i], x);
                to_pairs(dv[i], dy);
                to_pairs(ws[lane + 32 * i], wp);
#pragma unroll
                for (int q = 0; q < P; ++q) {
                    const f32x2 xh = mul2(sub2(x[q], M), Sx);
                    const f32x2 g = mul2(dy[q], wp[q]);
                    s1 = add2(s1, g);
                    s2 = fma2(g, xh, s2);
                }
            }
        }
        float a = hsum(s1), b = hsum(s2);
        warp_sum2(a, b);
        const float na = -s * (a * inv_C);
        const float nc = -s * (b * inv_C);
        const f32x2 NA = pair(na, na);
        const f32x2 NCc = pair(nc, nc);
        uint4 *gr = reinterpret_cast<uint4 *>(dinp) + r * nvec;
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int j = lane + 32 * i;
            if (j < nvec) {
                f32x2 x[P], dy[P], wp[P], o[P];
                to_pairs(xv[i], x);
                to_pairs(dv[i], dy);
                to_pairs(ws[lane + 32 * i], wp);
#pragma unroll
                for (int q = 0; q < P; ++q) {
                    const f32x2 xh = mul2(sub2(x[q], M), Sx);
                    const f32x2 g = mul2(dy[q], wp[q]);
                    o[q] = fma2(g, Sx, fma2(xh, NCc, NA));
                    acc_w[i][q] = fma2(dy[q], xh, acc_w[i][q]);
                    acc_b[i][q] = add2(acc_b[i][q], dy[q]);
                }
                __stcs(gr + j, from_pairs(o));
            }
        }
    }

    // Every copy landed or (after a timeout) is waited for before the tile
    // area is reused for the tree below.
    if (!__syncthreads_and(ok) && threadIdx.x == 0) {
        for (int t = 0; t <= TILES && has_rows; ++t) {
            if (t > 0 && row0 + int64_t(t - 1) * NW >= N) break;
            if (!mbar_wait(&bars[t], 0)) atomicOr(status, kStatusDrain);
        }
    }
    __syncthreads();

    // Block: fixed-order tree over the NW warps (as in the persistent kernels).
    float *s_tree = reinterpret_cast<float *>(s_tiles);
    constexpr int kTop = (NW > 8) ? 8 : (NW > 4) ? 4 : (NW > 2) ? 2 : 1;
    int n = NW;
#pragma unroll
    for (int h = kTop; h >= 1; h /= 2) {
        if (warp >= h && warp < n) {
            float *dst = s_tree + (warp - h) * 2 * C;
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const int j = lane + 32 * i;
                if (j < nvec) {
                    ulonglong2 *pw = reinterpret_cast<ulonglong2 *>(dst + j * E);
                    ulonglong2 *pb = reinterpret_cast<ulonglong2 *>(dst + C + j * E);
#pragma unroll
                    for (int q = 0; q < P / 2; ++q) {
                        pw[q] = make_ulonglong2(acc_w[i][2 * q], acc_w[i][2 * q + 1]);
                        pb[q] = make_ulonglong2(acc_b[i][2 * q], acc_b[i][2 * q + 1]);
                    }
                }
            }
        }
        __syncthreads();
        if (warp < n - h) {
            const float *src = s_tree + warp * 2 * C;
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const int j = lane + 32 * i;
                if (j < nvec) {
                    f32x2 pw[P], pb[P];
                    smem_pairs<P>(src + j * E, pw);
                    smem_pairs<P>(src + C + j * E, pb);
#pragma unroll
                    for (int q = 0; q < P; ++q) {
                        acc_w[i][q] = add2(acc_w[i][q], pw[q]);
                        acc_b[i][q] = add2(acc_b[i][q], pb[q]);
                    }
                }
            }
        }
        __syncthreads();
        n = h;
    }
    if (warp == 0) {
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int j = lane + 32 * i;
            if (j < nvec) {
                ulonglong2 *pw = reinterpret_cast<ulonglong2 *>(s_part + j * E);
                ulonglong2 *pb = reinterpret_cast<ulonglong2 *>(s_part + C + j * E);
#pragma unroll
                for (int q = 0; q < P / 2; ++q) {
                    pw[q] = make_ulonglong2(acc_w[i][2 * q], acc_w[i][2 * q + 1]);
                    pb[q] = make_ulonglong2(acc_b[i][2 * q], acc_b[i][2 * q + 1]);
                }
            }
        }
    }

    // Cluster: rank k adds float4 slice k of the CL block sums in rank order.
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    const int rank = int(cluster.block_rank());
    const int quads = (2 * C) / 4;                            // 2C is a multiple of 8
    const int per = (quads + CL - 1) / CL;
    const int q0 = rank * per;
    const int q1 = min(quads, q0 + per);
    float4 *dst = reinterpret_cast<float4 *>(partial + int64_t(blockIdx.x / CL) * 2 * C);
    for (int q = q0 + int(threadIdx.x); q < q1; q += blockDim.x) {
        float4 tot = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int k = 0; k < CL; ++k) {
            const float4 v = reinterpret_cast<const float4 *>(cluster.map_shared_rank(s_part, k))[q];
            tot.x += v.x;
            tot.y += v.y;
            tot.z += v.z;
            tot.w += v.w;
        }
        dst[q] = tot;
    }
    cluster.sync();
}

}  // namespace lnk
