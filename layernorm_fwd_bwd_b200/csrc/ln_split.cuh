// ln_split.cuh -- the LayerNorm backward for wide rows with row warps and
// column warps fed by one TMA bulk-copy ring.
//
// Operation: the hand-derived LayerNorm gradient of "llm.c: Large Language
// Model Training in Pure C/CUDA Without Dependencies", feature "Exact
// Analytical Backward Pass" (dinp, and dweight/dbias summed over all rows);
// arithmetic as in ln_kernels.cuh.  Technique: "Building GPT-2 from scratch",
// exercise table, row A3 (vectorised loads, warp reductions, chasing peak
// bandwidth).
//
// Why a second ring kernel.  In ln_bwd_tma_kernel every consumer warp owns
// a row AND the column sums of the columns it touches, so a lane holds its
// row (x - mean, dout * weight) and two accumulators per element it covers.
// At 7 vectors per lane (bf16 C = 1600) the accumulators alone are 112
// registers, so such rows are spread over three warps per row, with empty
// lanes and a row exchange through shared memory per row.  Here the two jobs
// are separated, and both read the same shared-memory stages:
//   * NR row warps, one row each per tile (tile = NR consecutive rows): the
//     row sums S1 = sum g, S2 = sum g * (x - mean) (g = dout * weight) and
//     dinp.  They keep g unpacked in registers between the two passes, read
//     x again from the stage in pass 2, and hold no accumulator at all.
//   * NCOL column warps, each owning a fixed slice of about nvec / NCOL
//     16-byte column vectors for the whole launch: for every row of every
//     tile, in row order, they add dout * xhat and dout into their slice's
//     fp32 accumulators (VC vectors per lane).  The sums keep a fixed order
//     (rows in tile order, tiles in the block's fixed sequence), so results
//     are deterministic, and at the end each column warp writes its slice of
//     the block's partial row directly: no combine tree.
//   * one producer warp streams the tiles (inp and dout rows, and the
//     previous dinp when accumulating) with 1-D bulk copies (cp.async.bulk,
//     no multicast) into S stages; S is as many as fit in the block's shared
//     memory (read back from %dynamic_smem_size, 2..8).
// A stage is free once every row warp has finished its row (pass 2 reads x,
// and the previous dinp when accumulating, from the stage) and every column
// warp has passed over all its rows: its "empty" mbarrier counts NR + NCOL
// arrivals, each after a fence.proxy.async that orders the warp's reads
// before the next bulk copy into the stage.  Waits are bounded exactly as in
// ln_tma.cuh.
#pragma once

#include "ln_tma.cuh"

namespace lnk {

constexpr int kSplitMaxStages = 8;   // the 128-byte barrier area holds 16 mbarriers

// Shared memory layout (bytes):
//   [0, 128)              full[8], empty[8] mbarriers
//   [128, 128 + A)        weight as fp32, A = C*4 rounded up to 128
//   [.., + S * stage)     the ring; stage = NS arrays of NR rows
__host__ __device__ constexpr size_t split_ring_offset(int C) {
    return 128 + align128(size_t(C) * 4);
}
template <typename T, int NR, int NS>
__host__ __device__ constexpr size_t split_stage_bytes(int C) {
    return size_t(NS) * NR * size_t(C) * sizeof(T);
}
// Stages that fit in `budget` bytes of shared memory at row width C, capped
// at kSplitMaxStages; below 2 the variant does not fit.
template <typename T, int NR, int NS>
__host__ __device__ constexpr int split_stages(int C, size_t budget) {
    const size_t off = split_ring_offset(C);
    const size_t st = split_stage_bytes<T, NR, NS>(C);
    const size_t n = budget > off ? (budget - off) / st : 0;
    return n > size_t(kSplitMaxStages) ? kSplitMaxStages : int(n);
}
template <typename T, int NR, int NS>
__host__ __device__ constexpr size_t split_smem(int C, int S) {
    return split_ring_offset(C) + size_t(S) * split_stage_bytes<T, NR, NS>(C);
}

__device__ __forceinline__ uint32_t dynamic_smem_bytes() {
    uint32_t n;
    asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(n));
    return n;
}

// Backward.  VR vectors per lane on a row warp (rows of up to 32 * VR
// vectors), VC vectors per lane on a column warp (slices of up to 32 * VC
// vectors), NR row warps, NCOL column warps, then the producer warp.  Tiles
// of NR rows go round-robin over the persistent grid.  MODE: 0, or
// kBwdAccumulate (dinp += the gradient; the previous dinp is the third array
// of a stage).  The arguments are those of ln_bwd_tma_kernel
// (tiles_per_block is unused: the assignment is always round-robin).
template <typename T, int VR, int VC, int NR, int NCOL, int MODE = 0>
__global__ void __launch_bounds__(32 * (NR + NCOL + 1), 1)
ln_bwd_split_kernel(T *__restrict__ dinp, float *__restrict__ partial,
                    const T *__restrict__ dout, const T *__restrict__ inp,
                    const T *__restrict__ weight, const float *__restrict__ mean,
                    const float *__restrict__ rstd, int64_t N, int C, float inv_C,
                    int64_t tiles_per_block, float eps, unsigned *__restrict__ status) {
    pdl_enter();
    static_assert((MODE & kBwdRecompute) == 0, "statistics are read, not recomputed");
    static_assert(NR >= 2 && NR <= 32 && NCOL >= 1, "warp roles");
    constexpr bool ACC = (MODE & kBwdAccumulate) != 0;
    constexpr int NS = ACC ? 3 : 2;                          // arrays per stage
    constexpr int E = Vec<T>::E;
    constexpr int P = E / 2;
    constexpr int RT = NR;                                   // rows per tile
    (void)tiles_per_block;
    (void)eps;
    unsigned char *smem = ln_dyn_smem;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem);
    uint64_t *empty = full + kSplitMaxStages;
    float *s_w = reinterpret_cast<float *>(smem + 128);      // weight as fp32
    unsigned char *ring = smem + split_ring_offset(C);
    const int nvec = C / E;
    const uint32_t row_bytes = uint32_t(C) * sizeof(T);
    const uint32_t half_bytes = RT * row_bytes;              // one array of a stage
    const uint32_t stage_bytes = NS * half_bytes;
    int S = int((dynamic_smem_bytes() - uint32_t(split_ring_offset(C))) / stage_bytes);
    S = S < kSplitMaxStages ? S : kSplitMaxStages;           // the host gives 2..8
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], NR + NCOL);
        }
        fence_mbar_init();
    }
    for (int c = threadIdx.x; c < C; c += blockDim.x) s_w[c] = to_f32(weight[c]);
    __syncthreads();

    const int64_t ntiles = (N + RT - 1) / RT;
    const int64_t tile0 = blockIdx.x;
    const int64_t tstep = gridDim.x;
    const int64_t ntiles_here = tile0 < ntiles ? (ntiles - 1 - tile0) / tstep + 1 : 0;

    if (warp == NR + NCOL) {
        // ------------------------------------------------------- producer
        if (lane == 0) {
            int64_t k = 0;
            int st = 0;
            uint32_t fill = 0;   // parity of tile k's use of its stage: (k / S) & 1
            for (; k < ntiles_here; ++k) {
                // the stage's previous use (tile k - S) has parity fill ^ 1
                if (k >= S && !mbar_wait(&empty[st], fill ^ 1u)) {
                    atomicOr(status, kStatusWaitEmpty);
                    break;
                }
                const int64_t row0 = (tile0 + k * tstep) * RT;
                const uint32_t bytes = uint32_t(min64(RT, N - row0)) * row_bytes;
                mbar_arrive_expect_tx(&full[st], NS * bytes);
                unsigned char *dst = ring + size_t(st) * stage_bytes;
                bulk_load(dst, reinterpret_cast<const unsigned char *>(inp) + row0 * row_bytes,
                          bytes, &full[st]);
                bulk_load(dst + half_bytes,
                          reinterpret_cast<const unsigned char *>(dout) + row0 * row_bytes, bytes,
                          &full[st]);
                if constexpr (ACC)
                    bulk_load(dst + 2 * half_bytes,
                              reinterpret_cast<const unsigned char *>(dinp) + row0 * row_bytes,
                              bytes, &full[st]);
                if (++st == S) {
                    st = 0;
                    fill ^= 1u;
                }
            }
            // wait (bounded) for the copies still in flight before exiting
            for (int64_t q = (k > S ? k - S : 0); q < k; ++q)
                if (!mbar_wait(&full[q % S], uint32_t((q / S) & 1)))
                    atomicOr(status, kStatusDrain);
        }
        return;
    }

    if (warp < NR) {
        // ------------------------------------------------------- row warps
        // Pass 1 reads the row from the stage and keeps g = dout * weight
        // unpacked in registers (VR * E of them); pass 2 reads x again from
        // the stage.  Measured on B200 this beats holding the packed row (no
        // second unpack of dout, no second weight read) and holding x - mean
        // as well (which needs more registers than 16 warps leave).  The
        // stage is released after pass 2.
        const int64_t rstep = tstep * RT;
        int64_t r = tile0 * RT + warp;
        float m_next = 0.f, s_next = 0.f;
        if (ntiles_here > 0 && r < N) {
            m_next = __ldg(mean + r);
            s_next = __ldg(rstd + r);
        }
        int st = 0;
        uint32_t parity = 0;
        for (int64_t k = 0; k < ntiles_here; ++k, r += rstep) {
            if (!mbar_wait(&full[st], parity)) {
                if (lane == 0) atomicOr(status, kStatusWaitFull);
                break;
            }
            const bool valid = r < N;
            const float m = m_next, s = s_next;
            if (k + 1 < ntiles_here && r + rstep < N) {
                m_next = __ldg(mean + r + rstep);
                s_next = __ldg(rstd + r + rstep);
            }
            const unsigned char *stage = ring + size_t(st) * stage_bytes + warp * row_bytes;
            const uint4 *xs = reinterpret_cast<const uint4 *>(stage);
            const uint4 *ds = reinterpret_cast<const uint4 *>(stage + half_bytes);
            const uint4 *ps = reinterpret_cast<const uint4 *>(stage + 2 * half_bytes);
            const int st_now = st;
            if (++st == S) {
                st = 0;
                parity ^= 1u;
            }
            if (valid) {
                // pass 1: S1 = sum g, S2 = sum g * d with d = x - mean, one
                // running sum per pair slot q, added in a fixed order
                const f32x2 K = pair(m, m), Sx = pair(s, s);
                f32x2 s1[P], s2[P], gk[VR][P];
#pragma unroll
                for (int q = 0; q < P; ++q) {
                    s1[q] = pair(0.f, 0.f);
                    s2[q] = pair(0.f, 0.f);
                }
#pragma unroll
                for (int i = 0; i < VR; ++i) {
                    const int j = lane + 32 * i;
                    if (j < nvec) {
                        f32x2 x[P], dy[P], wp[P];
                        to_pairs<T>(xs[j], x);
                        to_pairs<T>(ds[j], dy);
                        smem_pairs<P>(s_w + j * E, wp);
#pragma unroll
                        for (int q = 0; q < P; ++q) {
                            gk[i][q] = mul2(dy[q], wp[q]);
                            s1[q] = add2(s1[q], gk[i][q]);
                            s2[q] = fma2(gk[i][q], sub2(x[q], K), s2[q]);
                        }
                    }
                }
#pragma unroll
                for (int q = 1; q < P; ++q) {
                    s1[0] = add2(s1[0], s1[q]);
                    s2[0] = add2(s2[0], s2[q]);
                }
                float a = hsum(s1[0]), b = hsum(s2[0]);
                warp_sum2(a, b);
                // pass 2: dinp = g * rstd + NA + d * NC, NA = -rstd * mean(g),
                // NC = -rstd^3 * mean(g * d)
                const float na = -s * (a * inv_C);
                const float nc = -(s * s) * (s * (b * inv_C));
                const f32x2 NA = pair(na, na), NCc = pair(nc, nc);
                uint4 *gr = reinterpret_cast<uint4 *>(dinp) + r * nvec;
#pragma unroll
                for (int i = 0; i < VR; ++i) {
                    const int j = lane + 32 * i;
                    if (j < nvec) {
                        f32x2 x[P], o[P];
                        to_pairs<T>(xs[j], x);
#pragma unroll
                        for (int q = 0; q < P; ++q)
                            o[q] = fma2(gk[i][q], Sx, fma2(sub2(x[q], K), NCc, NA));
                        if constexpr (ACC) {
                            f32x2 pp[P];
                            to_pairs<T>(ps[j], pp);
#pragma unroll
                            for (int q = 0; q < P; ++q) o[q] = add2(o[q], pp[q]);
                        }
                        __stcs(gr + j, from_pairs<T>(o));
                    }
                }
            }
            fence_proxy_async_smem();                 // reads done before the refill
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st_now]);
        }
        return;
    }

    // ----------------------------------------------------------- column warps
    // Warp cw owns the vectors [cw * SL, cw * SL + SL) of every row (SL =
    // ceil(nvec / NCOL)); lane l holds vectors cw * SL + l + 32 * i, i < VC.
    const int cw = warp - NR;
    const int SL = (nvec + NCOL - 1) / NCOL;
    const int j0 = cw * SL;
    f32x2 acc_w[VC][P], acc_b[VC][P];
#pragma unroll
    for (int i = 0; i < VC; ++i)
#pragma unroll
        for (int q = 0; q < P; ++q) {
            acc_w[i][q] = pair(0.f, 0.f);
            acc_b[i][q] = pair(0.f, 0.f);
        }
    bool mine[VC];
#pragma unroll
    for (int i = 0; i < VC; ++i) {
        const int o = lane + 32 * i;
        mine[i] = o < SL && j0 + o < nvec;
    }
    // statistics of a tile's rows: lane l < RT holds row l's, one tile ahead
    float m_next = 0.f, s_next = 0.f;
    if (ntiles_here > 0 && lane < RT && tile0 * RT + lane < N) {
        m_next = __ldg(mean + tile0 * RT + lane);
        s_next = __ldg(rstd + tile0 * RT + lane);
    }
    int st = 0;
    uint32_t parity = 0;
    for (int64_t k = 0; k < ntiles_here; ++k) {
        if (!mbar_wait(&full[st], parity)) {
            if (lane == 0) atomicOr(status, kStatusWaitFull);
            break;
        }
        const int64_t row0 = (tile0 + k * tstep) * RT;
        const int rows = int(min64(RT, N - row0));
        const float mt = m_next, rt = s_next;
        if (k + 1 < ntiles_here) {
            const int64_t rn = row0 + tstep * RT + lane;
            m_next = (lane < RT && rn < N) ? __ldg(mean + rn) : 0.f;
            s_next = (lane < RT && rn < N) ? __ldg(rstd + rn) : 0.f;
        }
        const unsigned char *stage = ring + size_t(st) * stage_bytes;
#pragma unroll 2
        for (int rr = 0; rr < rows; ++rr) {
            const float m = __shfl_sync(0xffffffffu, mt, rr);
            const float s = __shfl_sync(0xffffffffu, rt, rr);
            const f32x2 K = pair(m, m), Sx = pair(s, s);
            const uint4 *xs = reinterpret_cast<const uint4 *>(stage + rr * row_bytes) + j0;
            const uint4 *ds =
                reinterpret_cast<const uint4 *>(stage + half_bytes + rr * row_bytes) + j0;
#pragma unroll
            for (int i = 0; i < VC; ++i) {
                if (mine[i]) {
                    f32x2 x[P], dy[P];
                    to_pairs<T>(xs[lane + 32 * i], x);
                    to_pairs<T>(ds[lane + 32 * i], dy);
#pragma unroll
                    for (int q = 0; q < P; ++q) {
                        const f32x2 xh = mul2(sub2(x[q], K), Sx);
                        acc_w[i][q] = fma2(dy[q], xh, acc_w[i][q]);
                        acc_b[i][q] = add2(acc_b[i][q], dy[q]);
                    }
                }
            }
        }
        fence_proxy_async_smem();                     // reads done before the refill
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
        if (++st == S) {
            st = 0;
            parity ^= 1u;
        }
    }
    float *pblk = partial + (int64_t)blockIdx.x * 2 * C;
#pragma unroll
    for (int i = 0; i < VC; ++i) {
        if (mine[i]) {
            const int j = j0 + lane + 32 * i;
            ulonglong2 *pw = reinterpret_cast<ulonglong2 *>(pblk + j * E);
            ulonglong2 *pb = reinterpret_cast<ulonglong2 *>(pblk + C + j * E);
#pragma unroll
            for (int q = 0; q < P / 2; ++q) {
                pw[q] = make_ulonglong2(acc_w[i][2 * q], acc_w[i][2 * q + 1]);
                pb[q] = make_ulonglong2(acc_b[i][2 * q], acc_b[i][2 * q + 1]);
            }
        }
    }
}

}  // namespace lnk
