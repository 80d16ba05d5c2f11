// ln_tile.cuh -- the one-shot tile forward: each block streams a fixed set of
// row tiles into shared memory with TMA bulk copies, uses every stage exactly
// once, and exits.
//
// Operation: the LayerNorm forward of "llm.c's Origin and the Future of LLM
// Compilers" (CUDA MODE talk page), chapter "Deconstructing PyTorch
// Abstractions and Setting Reference Baselines", over the flat row-major
// arrays of "llm.c: Large Language Model Training in Pure C/CUDA Without
// Dependencies", feature "Tensor Memory Layout"; the residual variant fuses
// the add before it, as that page's feature list credits custom fused
// kernels.  Arithmetic as in ln_kernels.cuh.
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
// The residual variant (MODE & kFwdResidual) copies the tiles of both inputs
// under the same barrier and forms x = inp + branch in registers.
#pragma once

#include "ln_tma.cuh"

namespace lnk {

// Shared memory: [128 B barriers][raw weight + bias, 128-aligned]
//                [NS input arrays x TILES tiles x RT rows][exchange slots]
template <typename T, int NW, int TILES, int W = 1, int NS = 1>
__host__ __device__ constexpr size_t fwd_tile_smem(int C) {
    // barriers, raw weight + bias, TILES tiles of NW / W rows of each of the
    // NS input arrays, and the row-group exchange slots when rows are shared
    // by W > 1 warps
    return 128 + align128(size_t(2) * C * sizeof(T)) +
           align128(size_t(NS) * TILES * (NW / W) * C * sizeof(T)) +
           (W > 1 ? size_t(NW / W) * 2 * 3 * W * 4 : 0);
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
// Resident blocks per SM the register allocation must allow.  Wide 16-bit
// rows on one warp (6+ vectors per lane, 2.4+ KB) fit three 2-tile blocks of
// 8 warps in shared memory; unconstrained they take 82+ registers and only
// two blocks would fit.  fp32 rows of 5-8 vectors per lane: unconstrained,
// ptxas settles at 48 registers and spills; a bound of three blocks gives it
// 74-80 registers without spills, at 5-6 vectors one resident block fewer
// than shared memory would allow (measured on B200: fp32 C = 768 62.1 ->
// 61.4 us, C = 896 42.6 -> 42.2, C = 640 and 1024 unchanged).  (0: no
// constraint.)
#ifndef LN_TILE_FWD_MINB
#define LN_TILE_FWD_MINB(T, V, NW)                                                 \
    (((NW) == 8 && ((sizeof(T) == 2 && (V) >= 6) || (sizeof(T) == 4 && (V) >= 5))) \
         ? 3                                                                       \
         : 0)
#endif
// Requirements (checked by the host): inp/out/weight/bias (and branch,
// resid_out) 16-byte aligned, C * sizeof(T) a multiple of 16,
// C / E <= 32 * W * V (== when FULL).
// ---------------------------------------------------------------------------
template <typename T, int V, int NW, int TILES, int W = 1, bool FULL = false, int MODE = 0>
__global__ void __launch_bounds__(32 * NW, LN_TILE_FWD_MINB(T, V, NW))
ln_fwd_tile_kernel(T *__restrict__ out, float *__restrict__ mean, float *__restrict__ rstd,
                   const T *__restrict__ inp, const T *__restrict__ weight,
                   const T *__restrict__ bias, T *__restrict__ resid_out,
                   const T *__restrict__ branch, int64_t N, int C, float inv_C, float eps,
                   int rows_pb, unsigned *__restrict__ status) {
    pdl_enter();
    constexpr bool RES = (MODE & kFwdResidual) != 0;
    constexpr int NS = RES ? 2 : 1;                           // input arrays
    static_assert(TILES + 1 <= 16, "barriers fit in 128 bytes");
    static_assert(NW % W == 0 && NW / W <= 15, "row groups");
    constexpr int E = Vec<T>::E;
    constexpr int P = E / 2;
    constexpr int RT = NW / W;                                // rows per tile
    constexpr int TPR = 32 * W;
    unsigned char *smem = ln_dyn_smem;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem);      // [0]: params, [1+t]: tile t
    const uint32_t row_bytes = uint32_t(C) * sizeof(T);
    unsigned char *s_par = smem + 128;                         // weight then bias, raw
    unsigned char *s_tiles = s_par + align128(size_t(2) * row_bytes);
    // branch tiles follow the inp tiles (residual variant)
    unsigned char *s_tiles2 = s_tiles + size_t(TILES) * RT * row_bytes;
    float *s_red = reinterpret_cast<float *>(
        s_tiles + align128(size_t(NS) * TILES * RT * row_bytes));   // [RT][2][3W] (W > 1)
    // FULL: the row is exactly 32 * W * V vectors, so no lane is ever past
    // its end and every bound check below folds away at compile time
    const int nvec = FULL ? 32 * W * V : C / E;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int group = warp / W;
    const int sub = warp - group * W;
    const int t = sub * 32 + lane;
    // this block's rows: [row0, row_end), rows_pb <= RT * TILES of them (the
    // host picks rows_pb so that the grid fills the resident blocks evenly)
    const int64_t row0 = int64_t(blockIdx.x) * rows_pb;
    const int64_t row_end = min64(N, row0 + rows_pb);

    if (threadIdx.x == 0) {
        for (int k = 0; k <= TILES; ++k) mbar_init(&bars[k], 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(&bars[0], 2 * row_bytes);
        bulk_load(s_par, weight, row_bytes, &bars[0]);
        bulk_load(s_par + row_bytes, bias, row_bytes, &bars[0]);
        for (int k = 0; k < TILES; ++k) {
            const int64_t r = row0 + int64_t(k) * RT;
            if (r < row_end) {
                const uint32_t bytes = uint32_t(min64(RT, row_end - r)) * row_bytes;
                mbar_arrive_expect_tx(&bars[1 + k], NS * bytes);
                bulk_load(s_tiles + size_t(k) * RT * row_bytes,
                          reinterpret_cast<const unsigned char *>(inp) + r * row_bytes, bytes,
                          &bars[1 + k]);
                if constexpr (RES)
                    bulk_load(s_tiles2 + size_t(k) * RT * row_bytes,
                              reinterpret_cast<const unsigned char *>(branch) + r * row_bytes,
                              bytes, &bars[1 + k]);
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
        if (r >= row_end) break;                              // uniform over the row group
        if (!tile_wait(&bars[1 + k], status, kStatusWaitFull)) abort = true;
        if (abort && W == 1) break;
        const unsigned char *row = s_tiles + (size_t(k) * RT + group) * row_bytes;
        const uint4 *src = reinterpret_cast<const uint4 *>(row);
        // in(i, j): vector j of round i lies in the row.  With one warp per row
        // the host picks V = ceil(nvec / 32), so rounds 0 .. V-2 are complete
        // for every lane and only the last round needs the bound check.
        auto in = [&](int i, int j) { return FULL || (W == 1 && i < V - 1) || j < nvec; };
        uint4 xv[V];
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int j = t + TPR * i;
            xv[i] = in(i, j) ? src[j] : make_uint4(0u, 0u, 0u, 0u);
        }
        float pivot;
        if constexpr (RES) {
            const unsigned char *row2 = s_tiles2 + (size_t(k) * RT + group) * row_bytes;
            const uint4 *src2 = reinterpret_cast<const uint4 *>(row2);
            uint4 *xo = reinterpret_cast<uint4 *>(resid_out) + r * nvec;
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const int j = t + TPR * i;
                const uint4 bv = in(i, j) ? src2[j] : make_uint4(0u, 0u, 0u, 0u);
                xv[i] = add_round<T>(xv[i], bv);
                if (in(i, j)) __stcs(xo + j, xv[i]);
            }
            pivot = add_round1<T>(reinterpret_cast<const T *>(row)[0],
                                  reinterpret_cast<const T *>(row2)[0]);
        } else {
            pivot = to_f32(reinterpret_cast<const T *>(row)[0]);
        }
        const f32x2 K = pair(pivot, pivot);
        f32x2 d[V][P];
        f32x2 acc = pair(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const bool live = in(i, t + TPR * i);
            to_pairs<T>(xv[i], d[i]);
#pragma unroll
            for (int q = 0; q < P; ++q) {
                d[i][q] = sub2(d[i][q], K);
                if (live) acc = add2(acc, d[i][q]);
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
            const bool live = in(i, t + TPR * i);
#pragma unroll
            for (int q = 0; q < P; ++q) {
                d[i][q] = sub2(d[i][q], M);
                if (live) sq = fma2(d[i][q], d[i][q], sq);
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
            if (in(i, j)) {
                f32x2 wp[P], bp[P], o[P];
                to_pairs<T>(ws[j], wp);
                to_pairs<T>(bs[j], bp);
#pragma unroll
                for (int q = 0; q < P; ++q) o[q] = fma2(mul2(d[i][q], R), wp[q], bp[q]);
                __stcs(yr + j, from_pairs<T>(o));
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
            if (k > 0 && row0 + int64_t(k - 1) * RT >= row_end) break;
            if (!mbar_wait(&bars[k], 0)) atomicOr(status, kStatusDrain);
        }
    }
}

}  // namespace lnk
