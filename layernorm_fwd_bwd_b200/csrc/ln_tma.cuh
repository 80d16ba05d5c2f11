// ln_tma.cuh -- the TMA and mbarrier helpers (bounded waits, 1-D bulk copies,
// also used by the one-shot forward in ln_tile.cuh) and the LayerNorm
// backward fed by a TMA bulk-copy ring.
//
// Operation: the hand-derived LayerNorm gradient of "llm.c: Large Language
// Model Training in Pure C/CUDA Without Dependencies", feature "Exact
// Analytical Backward Pass" (dinp, and dweight/dbias summed over all rows);
// the accumulating variant adds into the previous gradients, as that page's
// multi-GPU question says gradients are accumulated locally.  Arithmetic as
// in ln_kernels.cuh.
//
// Why a ring: the register-resident kernels keep at most one row per warp in flight
// (1.5 KB for a bf16 row of 768), and a warp spends most of each row on
// arithmetic, so a bf16 launch cannot keep enough bytes in flight to reach
// the HBM roofline.  Here one producer warp per block streams whole tiles of
// consecutive rows (one contiguous range of global memory) into a ring of S
// shared-memory stages with 1-D bulk copies (cp.async.bulk, no multicast),
// so the bytes in flight live in shared memory (S * tile bytes per block)
// instead of registers.  Consumer warps take one row each from the stage,
// compute exactly as the register-resident kernels do, and release the stage.
//
// Synchronisation: per stage one "full" mbarrier (producer's expect_tx + the
// copy's completion) and one "empty" mbarrier (one arrival per consumer warp,
// after a fence.proxy.async that orders the warp's shared-memory reads before
// the next bulk copy into the stage).
// Every wait is bounded (kWaitLimitNs of %globaltimer, and an iteration cap):
// on expiry the thread records an error bit in *status, stops, and the
// producer waits (again bounded) for its copies in flight before the block
// exits.  Nothing here waits on another block.
#pragma once

#include "ln_kernels.cuh"

namespace lnk {

constexpr uint64_t kWaitLimitNs = 1000000000ull;   // 1 s
constexpr uint32_t kMaxWaitIters = 1u << 30;

// status bits
constexpr unsigned kStatusWaitFull = 1u;    // a consumer gave up on a stage's data
constexpr unsigned kStatusWaitEmpty = 2u;   // the producer gave up on a stage's release
constexpr unsigned kStatusDrain = 4u;       // a copy in flight did not land in time

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// Order this thread's generic-proxy shared-memory reads before later
// async-proxy writes (the next bulk copy into the same stage).  Without it a
// stage can be refilled before the reads that preceded its release were
// performed -- a write-after-read race that measurably corrupts rows.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Wait until the phase of `bar` with the given parity has completed; false
// if that did not happen within kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t it = 1; it < kMaxWaitIters; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 63u) == 0 && global_ns() - t0 > kWaitLimitNs) return false;
    }
    return false;
}
// 1-D bulk copy global -> this block's shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes,
                                          uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__host__ __device__ constexpr size_t align128(size_t x) { return (x + 127) & ~size_t(127); }
__device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

// Shared memory layout (bytes):
//   [0, 128)            full[S], empty[S] mbarriers (S <= 8)
//   [128, 128 + A)      weight as fp32, A = C*4 rounded up to 128
//   [.., + S * stage)   the ring; stage = NS arrays (inp, dout and, when
//                       accumulating, the previous dinp) of the tile's rows
//   [.., ..)            row-group exchange slots (W > 1)
template <typename T>
__host__ __device__ constexpr size_t tma_ring_offset(int C) {
    return 128 + align128(size_t(C) * 4);
}
template <typename T, int NC, int S, int W, int NS>
__host__ __device__ constexpr size_t bwd_tma_ring_bytes(int C) {
    // the ring (NC/W rows of each array per stage), also reused for the
    // end-of-block combine: every row group parks 2C floats
    const size_t ring = size_t(S) * (NC / W) * NS * C * sizeof(T);
    const size_t comb = size_t(NC / W) * 2 * C * 4;
    return ring > comb ? ring : comb;
}
template <typename T, int NC, int S, int W, int NS>
__host__ __device__ constexpr size_t bwd_tma_smem(int C) {
    // weight as fp32 (read twice per row: unpacking bf16 there costs more
    // issue slots than the wider shared-memory reads), the ring, and the
    // row-group exchange slots when rows are shared by W > 1 warps
    return tma_ring_offset<T>(C) + align128(bwd_tma_ring_bytes<T, NC, S, W, NS>(C)) +
           (W > 1 ? size_t(NC / W) * 2 * 4 * W * 4 : 0);
}

// Producer side: stream tiles k = 0, 1, ... of this
// block (tile index tile_of(k)) into the ring.  Before returning -- after the
// last tile, or after recording an error -- it waits (bounded) until its
// last copies have landed, so the block never exits with a copy still
// writing into its shared memory.
template <int S, typename TileOf, typename Issue>
__device__ __forceinline__ void tma_produce(uint64_t *full, uint64_t *empty,
                                            int64_t ntiles_here, unsigned *status,
                                            TileOf tile_of, Issue issue) {
    int64_t k = 0;
    for (; k < ntiles_here; ++k) {
        const int st = int(k % S);
        const int64_t use = k / S;
        if (use > 0 && !mbar_wait(&empty[st], uint32_t((use - 1) & 1))) {
            atomicOr(status, kStatusWaitEmpty);
            break;
        }
        issue(tile_of(k), st, &full[st]);
    }
    for (int64_t q = (k > S ? k - S : 0); q < k; ++q)
        if (!mbar_wait(&full[q % S], uint32_t((q / S) & 1))) atomicOr(status, kStatusDrain);
}

// ---------------------------------------------------------------------------
// Row-group exchange for rows shared by W warps: each warp posts its partial
// sums (a, b) and an abort flag into a slot of its group, the group meets at a
// named barrier, and every warp reads all W entries in the same order.  Slots
// alternate by parity, so a slot is rewritten only after every warp of the
// group has passed the next barrier (and so has read it).  A slot holds 3W
// floats here and 4W in group_exchange3 (three sums and the flag).
template <int W>
__device__ __forceinline__ bool group_exchange(float &a, float &b, bool abort, float *slot,
                                               int group, int sub, int lane) {
    if constexpr (W == 1) {
        return abort;
    } else {
        if (lane == 0) {
            slot[3 * sub + 0] = a;
            slot[3 * sub + 1] = b;
            slot[3 * sub + 2] = abort ? 1.f : 0.f;
        }
        asm volatile("bar.sync %0, %1;" ::"r"(group + 1), "r"(32 * W) : "memory");
        a = 0.f;
        b = 0.f;
        float any = 0.f;
#pragma unroll
        for (int k = 0; k < W; ++k) {
            a += slot[3 * k + 0];
            b += slot[3 * k + 1];
            any += slot[3 * k + 2];
        }
        return any != 0.f;
    }
}

template <int W>
__device__ __forceinline__ bool group_exchange3(float &a, float &b, float &c, bool abort,
                                                float *slot, int group, int sub, int lane) {
    if constexpr (W == 1) {
        return abort;
    } else {
        if (lane == 0) {
            slot[4 * sub + 0] = a;
            slot[4 * sub + 1] = b;
            slot[4 * sub + 2] = c;
            slot[4 * sub + 3] = abort ? 1.f : 0.f;
        }
        asm volatile("bar.sync %0, %1;" ::"r"(group + 1), "r"(32 * W) : "memory");
        a = 0.f;
        b = 0.f;
        c = 0.f;
        float any = 0.f;
#pragma unroll
        for (int k = 0; k < W; ++k) {
            a += slot[4 * k + 0];
            b += slot[4 * k + 1];
            c += slot[4 * k + 2];
            any += slot[4 * k + 3];
        }
        return any != 0.f;
    }
}

// ---------------------------------------------------------------------------
// Backward.  NC consumer warps (15 by default: with the producer warp a
// 512-thread block, one per SM, 128 registers per thread), W warps per row,
// so a tile holds RT = NC / W consecutive rows; tiles go round-robin over
// the persistent grid (RR) or in contiguous ranges.  A stage holds the tile's
// inp rows, then its dout rows and, when accumulating (MODE &
// kBwdAccumulate), the previous dinp rows.  Warp w serves row w / W of each
// tile and, within it, vectors j = (w % W) * 32 + lane + i * 32 * W; it keeps
// dout*xhat and dout for those columns in registers.  Row sums of the W warps
// of a row meet in shared memory (group_exchange).  At the end the RT row
// groups park their column sums in shared memory and the whole block adds
// them in group order and writes the block's partial row.  mean/rstd of the next
// row are prefetched one tile ahead; with MODE & kBwdRecompute they are not
// read at all but recomputed from the staged row (pivot x[r, 0], two-pass
// deviations, as in the forward).
// ---------------------------------------------------------------------------
// Whether rows shared by W > 1 warps (plain backward) also keep g from pass 1.
#ifndef LN_RING_KEEP_G_SHARED_PLAIN
#define LN_RING_KEEP_G_SHARED_PLAIN 1
#endif
// Whether the recomputing backward, where it does not keep g, reduces the
// row's variance together with its two backward sums (one butterfly and one
// row exchange of three values instead of two in a row).  The variance's
// per-lane sums and reduction order are the same, so mean and rstd are
// bit-identical either way; dinp and dweight then take the form that scales
// x - mean by rstd once per element (rounding differs in the last bits).
// Where g is kept, the column sums would have to wait for pass 2 and the
// packed dout would hold its registers until then: slower on B200.
#ifndef LN_RING_FUSE_RECOMP_VAR
#define LN_RING_FUSE_RECOMP_VAR 1
#endif

template <typename T, int V, int NC, int S, bool RR, int W = 1, int MODE = 0>
__global__ void __launch_bounds__(32 * (NC + 1), (NC + 1) * 32 <= 256 ? 2 : 1)
ln_bwd_tma_kernel(T *__restrict__ dinp, float *__restrict__ partial,
                  const T *__restrict__ dout, const T *__restrict__ inp,
                  const T *__restrict__ weight, const float *__restrict__ mean,
                  const float *__restrict__ rstd, int64_t N, int C, float inv_C,
                  int64_t tiles_per_block, float eps, unsigned *__restrict__ status) {
    pdl_enter();
    static_assert(S >= 2 && S <= 8, "ring depth");
    static_assert(NC % W == 0 && NC / W >= 2 && NC / W <= 15, "row groups");
    constexpr bool ACC = (MODE & kBwdAccumulate) != 0;
    constexpr bool RECOMP = (MODE & kBwdRecompute) != 0;
    // floats per warp in a row-exchange slot: 4 for group_exchange3
    constexpr int XW = RECOMP ? 4 : 3;
    constexpr int NS = ACC ? 3 : 2;                          // arrays per stage
    constexpr int E = Vec<T>::E;
    constexpr int P = E / 2;
    constexpr int RT = NC / W;                               // rows per tile
    constexpr int TPR = 32 * W;                              // threads per row
    unsigned char *smem = ln_dyn_smem;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem);
    uint64_t *empty = full + S;
    float *s_w = reinterpret_cast<float *>(smem + 128);      // weight as fp32
    unsigned char *ring = smem + tma_ring_offset<T>(C);
    const int nvec = C / E;
    const uint32_t row_bytes = uint32_t(C) * sizeof(T);
    const uint32_t half_bytes = RT * row_bytes;              // one array of a stage
    const uint32_t stage_bytes = NS * half_bytes;
    float *s_red = reinterpret_cast<float *>(
        ring + align128(bwd_tma_ring_bytes<T, NC, S, W, NS>(C)));   // [RT][2][4W] (W > 1)
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int group = warp / W;                              // row in the tile
    const int sub = warp - group * W;
    const int t = sub * 32 + lane;                           // thread within its row


    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], NC);
        }
        fence_mbar_init();
    }
    for (int c = threadIdx.x; c < C; c += blockDim.x) s_w[c] = to_f32(weight[c]);
    __syncthreads();

    // Tiles of this block: RR (round-robin) takes tiles b, b + G, b + 2G, ...
    // so that the blocks in flight cover one compact window of memory;
    // otherwise a contiguous range of tiles_per_block tiles.  Either is a
    // fixed assignment, so the column sums stay deterministic.
    const int64_t ntiles = (N + RT - 1) / RT;
    const int64_t tile0 = RR ? int64_t(blockIdx.x) : int64_t(blockIdx.x) * tiles_per_block;
    const int64_t tstep = RR ? int64_t(gridDim.x) : 1;
    const int64_t ntiles_here =
        RR ? (tile0 < ntiles ? (ntiles - 1 - tile0) / tstep + 1 : 0)
           : (tile0 < ntiles ? min64(tiles_per_block, ntiles - tile0) : 0);

    f32x2 acc_w[V][P], acc_b[V][P];
#pragma unroll
    for (int i = 0; i < V; ++i)
#pragma unroll
        for (int q = 0; q < P; ++q) {
            acc_w[i][q] = pair(0.f, 0.f);
            acc_b[i][q] = pair(0.f, 0.f);
        }

    if (warp == NC) {
        if (lane == 0) {
            tma_produce<S>(
                full, empty, ntiles_here, status, [&](int64_t k) { return tile0 + k * tstep; },
                [&](int64_t tile, int st, uint64_t *bar) {
                    const int64_t row0 = tile * RT;
                    const uint32_t bytes = uint32_t(min64(RT, N - row0)) * row_bytes;
                    mbar_arrive_expect_tx(bar, NS * bytes);
                    unsigned char *dst = ring + size_t(st) * stage_bytes;
                    bulk_load(dst, reinterpret_cast<const unsigned char *>(inp) + row0 * row_bytes,
                              bytes, bar);
                    bulk_load(dst + half_bytes,
                              reinterpret_cast<const unsigned char *>(dout) + row0 * row_bytes,
                              bytes, bar);
                    if constexpr (ACC)
                        bulk_load(dst + 2 * half_bytes,
                                  reinterpret_cast<const unsigned char *>(dinp) +
                                      row0 * row_bytes,
                                  bytes, bar);
                });
        }
    } else {
        const int64_t rstep = tstep * RT;
        int64_t r = tile0 * RT + group;
        float m_next = 0.f, s_next = 0.f;
        if (!RECOMP && ntiles_here > 0 && r < N) {
            m_next = __ldg(mean + r);
            s_next = __ldg(rstd + r);
        }
        int parity = 0;
        for (int64_t k = 0; k < ntiles_here; ++k, r += rstep) {
            const int st = int(k % S);
            // A warp whose wait runs out records it and, when it shares its
            // row with other warps, still follows the row's exchange (with
            // meaningless data) so that the group leaves together.
            bool abort = !mbar_wait(&full[st], uint32_t((k / S) & 1));
            if (abort) {
                if (lane == 0) atomicOr(status, kStatusWaitFull);
                if constexpr (W == 1) break;
            }
            const bool valid = r < N;                 // uniform over the row group
            float m = m_next, s = s_next;
            if (!RECOMP && k + 1 < ntiles_here && r + rstep < N) {   // next row's statistics
                m_next = __ldg(mean + r + rstep);
                s_next = __ldg(rstd + r + rstep);
            }
            const unsigned char *stage = ring + size_t(st) * stage_bytes + group * row_bytes;
            const uint4 *xs = reinterpret_cast<const uint4 *>(stage);
            const uint4 *ds = reinterpret_cast<const uint4 *>(stage + half_bytes);
            const uint4 *ps = reinterpret_cast<const uint4 *>(stage + 2 * half_bytes);
            uint4 xv[V], dv[V];
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const int j = t + TPR * i;
                const bool ok = valid && j < nvec;
                xv[i] = ok ? xs[j] : make_uint4(0u, 0u, 0u, 0u);
                dv[i] = ok ? ds[j] : make_uint4(0u, 0u, 0u, 0u);
            }
            const float pivot = (RECOMP && valid) ? to_f32(reinterpret_cast<const T *>(stage)[0])
                                                  : 0.f;
            // Release the stage once this warp's reads of it are done: right
            // away, or after pass 2 when it also holds the previous dinp.
            auto release = [&]() {
                fence_proxy_async_smem();             // reads done before the refill
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[st]);
            };
            if constexpr (!ACC) release();
            if (!valid) {
                if constexpr (ACC) release();
                continue;
            }

            // Pass 1 / pass 2.  Pass 1 sums g = dout * weight and g * d over the
            // row (d = x - mean) and pass 2 evaluates
            //   dinp = g*rstd + NA + d*NC,  NA = -rstd*mean(g),
            //   NC = -rstd^3*mean(g*d)   (xhat = d*rstd).
            // Where the register budget allows (KEEP_D), pass 1 keeps d as fp32
            // pairs, so pass 2 never unpacks x again; otherwise both passes
            // rebuild d from the packed row (summing g * d rather than g * xhat
            // saves pass 1 a multiply per element: 41.0 -> 40.7 us at bf16
            // C = 1024 on B200).  Where it also allows (KEEP_G: one warp
            // per row, or a shared row of the plain backward; narrow enough
            // rows), pass 1 keeps g = dout * weight too
            // and adds the row's dout * xhat and dout to the column sums, so
            // pass 2 touches neither the packed dout nor the weight (the same
            // operations in the same order: identical results, about a fifth
            // fewer instructions per row).  Recomputing the statistics, d is
            // (x - pivot) - mean(x - pivot) and K, MD below are the pivot and
            // that mean; from the saved statistics K = mean[r] and MD = 0.
            constexpr bool KEEP_D = sizeof(T) == 4 || V <= 3;
            constexpr bool KEEP_G =
                KEEP_D && (W == 1 || LN_RING_KEEP_G_SHARED_PLAIN) &&
                (W == 1 || MODE == 0) && V <= (sizeof(T) == 4 ? (ACC ? 4 : 5) : (ACC ? 2 : 3));
            constexpr bool FUSE_VAR = RECOMP && !KEEP_G && LN_RING_FUSE_RECOMP_VAR;
            uint4 *gr = reinterpret_cast<uint4 *>(dinp) + r * nvec;
            f32x2 d[KEEP_D ? V : 1][P];
            f32x2 gk[KEEP_G ? V : 1][P];
            f32x2 K = pair(m, m), MD = pair(0.f, 0.f);
            if constexpr (RECOMP) {
                K = pair(pivot, pivot);
                f32x2 sd = pair(0.f, 0.f);
#pragma unroll
                for (int i = 0; i < V; ++i) {
                    const bool in = t + TPR * i < nvec;
                    f32x2 x[P];
                    to_pairs<T>(xv[i], x);
#pragma unroll
                    for (int q = 0; q < P; ++q) {
                        const f32x2 dq = sub2(x[q], K);
                        if constexpr (KEEP_D) d[i][q] = dq;
                        if (in) sd = add2(sd, dq);
                    }
                }
                float a = warp_sum(hsum(sd)), unused = 0.f;
                abort = group_exchange<W>(a, unused, abort, s_red + (group * 2 + parity) * XW * W,
                                          group, sub, lane);
                parity ^= 1;
                const float md = a * inv_C;
                MD = pair(md, md);
            }
            if constexpr (RECOMP && !FUSE_VAR) {
                float unused = 0.f;
                f32x2 sq = pair(0.f, 0.f);
#pragma unroll
                for (int i = 0; i < V; ++i) {
                    const bool in = t + TPR * i < nvec;
                    f32x2 x[P];
                    if constexpr (!KEEP_D) to_pairs<T>(xv[i], x);
#pragma unroll
                    for (int q = 0; q < P; ++q) {
                        f32x2 dq;
                        if constexpr (KEEP_D) {
                            d[i][q] = sub2(d[i][q], MD);
                            dq = d[i][q];
                        } else {
                            dq = sub2(sub2(x[q], K), MD);
                        }
                        if (in) sq = fma2(dq, dq, sq);
                    }
                }
                float v = warp_sum(hsum(sq));
                abort = group_exchange<W>(v, unused, abort, s_red + (group * 2 + parity) * XW * W,
                                          group, sub, lane);
                parity ^= 1;
                s = rsqrtf(v * inv_C + eps);
            }
            float *slot = s_red + (group * 2 + parity) * XW * W;
            parity ^= 1;
            f32x2 Sx = pair(s, s);
            f32x2 s1 = pair(0.f, 0.f), s2 = pair(0.f, 0.f), sq = pair(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const int j = t + TPR * i;
                if constexpr (FUSE_VAR && KEEP_D) {
#pragma unroll
                    for (int q = 0; q < P; ++q) {
                        d[i][q] = sub2(d[i][q], MD);
                        if (j < nvec) sq = fma2(d[i][q], d[i][q], sq);
                    }
                }
                if constexpr (KEEP_D && !RECOMP) {
                    // d for every slot (dead lanes' values are never used)
                    f32x2 dq[P];
                    to_pairs<T>(xv[i], dq);
#pragma unroll
                    for (int q = 0; q < P; ++q) d[i][q] = sub2(dq[q], K);
                }
                if (j < nvec) {
                    f32x2 dy[P], wp[P];
                    to_pairs<T>(dv[i], dy);
                    smem_pairs<P>(s_w + j * E, wp);
                    if constexpr (KEEP_G) {
#pragma unroll
                        for (int q = 0; q < P; ++q) {
                            gk[i][q] = mul2(dy[q], wp[q]);
                            s1 = add2(s1, gk[i][q]);
                            s2 = fma2(gk[i][q], d[i][q], s2);     // sum g * d
                            const f32x2 xh = mul2(d[i][q], Sx);
                            acc_w[i][q] = fma2(dy[q], xh, acc_w[i][q]);
                            acc_b[i][q] = add2(acc_b[i][q], dy[q]);
                        }
                    } else if constexpr (KEEP_D) {
#pragma unroll
                        for (int q = 0; q < P; ++q) {
                            const f32x2 g = mul2(dy[q], wp[q]);
                            s1 = add2(s1, g);
                            s2 = fma2(g, d[i][q], s2);            // sum g * d
                        }
                    } else {
                        f32x2 x[P];
                        to_pairs<T>(xv[i], x);
#pragma unroll
                        for (int q = 0; q < P; ++q) {
                            f32x2 dq = sub2(x[q], K);
                            if constexpr (RECOMP) dq = sub2(dq, MD);
                            const f32x2 g = mul2(dy[q], wp[q]);
                            s1 = add2(s1, g);
                            if constexpr (FUSE_VAR) sq = fma2(dq, dq, sq);
                            s2 = fma2(g, dq, s2);                 // sum g * d
                        }
                    }
                }
            }
            float a = hsum(s1), b = hsum(s2);
            if constexpr (FUSE_VAR) {
                float v = hsum(sq);
                warp_sum3(a, b, v);
                abort = group_exchange3<W>(a, b, v, abort, slot, group, sub, lane);
                s = rsqrtf(v * inv_C + eps);
                Sx = pair(s, s);
            } else {
                warp_sum2(a, b);
                abort = group_exchange<W>(a, b, abort, slot, group, sub, lane);
            }
            const float na = -s * (a * inv_C);
            const float nc = -(s * s) * (s * (b * inv_C));   // b: sum of g * d
            const f32x2 NA = pair(na, na);
            const f32x2 NCc = pair(nc, nc);
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const int j = t + TPR * i;
                if (j < nvec) {
                    f32x2 o[P];
                    if constexpr (KEEP_G) {
#pragma unroll
                        for (int q = 0; q < P; ++q)
                            o[q] = fma2(gk[i][q], Sx, fma2(d[i][q], NCc, NA));
                    } else {
                        f32x2 wp[P];
                        smem_pairs<P>(s_w + j * E, wp);
#pragma unroll
                        for (int q = 0; q < P; ++q) {
                            const f32x2 dy = pair_at<T>(dv[i], q);
                            const f32x2 g = mul2(dy, wp[q]);
                            f32x2 xh;
                            if constexpr (KEEP_D) {
                                o[q] = fma2(g, Sx, fma2(d[i][q], NCc, NA));
                                xh = mul2(d[i][q], Sx);
                            } else {
                                f32x2 dq = sub2(pair_at<T>(xv[i], q), K);
                                if constexpr (RECOMP) dq = sub2(dq, MD);
                                xh = mul2(dq, Sx);
                                o[q] = fma2(g, Sx, fma2(dq, NCc, NA));
                            }
                            acc_w[i][q] = fma2(dy, xh, acc_w[i][q]);
                            acc_b[i][q] = add2(acc_b[i][q], dy);
                        }
                    }
                    if constexpr (ACC) {
                        f32x2 pp[P];
                        to_pairs<T>(ps[j], pp);
#pragma unroll
                        for (int q = 0; q < P; ++q) o[q] = add2(o[q], pp[q]);
                    }
                    __stcs(gr + j, from_pairs<T>(o));
                }
            }
            if constexpr (ACC) release();
            if (abort) break;                         // the whole row group leaves here
        }
    }

    // Combine the RT row groups' column sums in a fixed order: every group
    // parks its 2C sums in the ring (free again once every warp has passed the
    // barrier: all copies were consumed, or drained by the producer), then all
    // threads of the block each add up a few columns over groups 0 .. RT-1 in
    // that order and write the block's partial row.  One barrier and one round
    // of shared-memory reads, where a pairwise tree takes two barriers per
    // level.  Measured on B200 (bf16, back-to-back calls): backward 54.2 ->
    // 53.5 us at C = 768, 42.8 -> 42.0 at C = 1024; 58.5 -> 59.1 at C = 3072,
    // where four-warp rows leave only three groups to combine.
    __syncthreads();
    float *s_acc = reinterpret_cast<float *>(ring);
    if (warp < NC) {
        float *dst = s_acc + group * 2 * C;
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int j = t + TPR * i;
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
    float4 *pblk = reinterpret_cast<float4 *>(partial + (int64_t)blockIdx.x * 2 * C);
    for (int f = threadIdx.x; f < C / 2; f += blockDim.x) {     // 2C floats as float4
        float4 sum = reinterpret_cast<const float4 *>(s_acc)[f];
        for (int g = 1; g < RT; ++g) {
            const float4 v = reinterpret_cast<const float4 *>(s_acc + g * 2 * C)[f];
            sum.x += v.x;
            sum.y += v.y;
            sum.z += v.z;
            sum.w += v.w;
        }
        pblk[f] = sum;
    }
}

}  // namespace lnk
