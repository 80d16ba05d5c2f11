// ln_dispatch.cuh -- kernel selection and launch geometry of the forward and
// the backward, for one element type T and one variant MODE.  ln_inst.cu
// instantiates these once per combination (each in its own object, so the
// kernels of the combinations compile in parallel).
//
// Geometry.  The forward's tile kernel runs one block per 8 to 16 rows
// (one-shot; tile_rows_per_block picks the count); every other kernel runs on
// a persistent grid of (SM count) x (resident
// blocks per SM, from the occupancy calculator for the exact block size and
// shared memory), capped by the number of rows.  Arrays that are all 16-byte
// aligned, with C * sizeof(T) a multiple of 16, take the vectorised kernels
// (variant chosen in ln_select.cuh); any other call takes the scalar kernels.
//
// Workspace.  The backward needs G * 2C fp32 partial sums (G = its grid).
// They are drawn stream-ordered from a memory pool that the library creates
// on the first pooled call on a device (release threshold: never), and handed
// back on the same stream right after the finalise kernel, so calls on
// different streams never share a buffer and steady-state calls reuse pool
// memory without a cudaMalloc; or, for ln_backward_noalloc, they live in a
// static array whose size caps G (that path never creates the pool).
#pragma once

#include "ln_host.cuh"
#include "ln_kernels.cuh"
#include "ln_select.cuh"

namespace lnh {

// ------------------------------------------------------------------ forward

// Rows per one-shot block, at most `max_rows` and at least half of it: the
// block count ceil(N / rows) is cut into ceil(blocks / resident) waves of
// `resident` blocks, and a wave takes about as long as a block's rows, so
// the value with the fewest rows in total (waves * rows) wins; ties go to
// more rows per block.  GPT-2 1.5B (N = 16384, 444 resident): 13 rows, 3
// full waves, instead of 16 rows and 2.3 waves.  Measured on B200: forward
// 32.76 -> 32.29 us (124M), 22.94 -> 22.65 (350M), 21.02 -> 20.85 (1.5B);
// less than the model says, since blocks of one wave do not end together.
inline int tile_rows_per_block(int64_t N, int max_rows, int64_t resident) {
    int best = max_rows;
    int64_t best_cost = INT64_MAX;
    for (int rows = max_rows; rows >= (max_rows + 1) / 2; --rows) {
        const int64_t waves = ceil_div(ceil_div(N, rows), resident);
        const int64_t cost = waves * rows;
        if (cost < best_cost) {
            best_cost = cost;
            best = rows;
        }
    }
    return best;
}

// Whether every block count that tile_rows_per_block can pick for `max_rows`
// (at least half of it per block) fits the grid's x dimension.
inline bool tile_grid_fits(int64_t N, int max_rows) {
    return ceil_div(N, (max_rows + 1) / 2) <= INT32_MAX;
}

template <typename T, int MODE>
struct FwdVec {
    const FwdArgs &a;
    cudaError_t err = cudaSuccess;
    static constexpr int kArrays = (MODE & lnk::kFwdResidual) ? 2 : 1;   // input arrays

    template <int V, int W, int GROUPS>
    void run() {
        if constexpr (W == 1) {
            if constexpr (V >= LN_TILE_FWD_W2_FROM_V) {
                run_tile_two<(V + 1) / 2>();
                return;
            } else if (tile_grid_fits(a.N, lnk::kTileWarps * lnk::kTileFwdTiles)) {
                run_tile<V, 1>();
                return;
            }
        }
        auto kern = lnk::ln_fwd_vec_kernel<T, V, W, GROUPS, MODE>;
        const int threads = 32 * W * GROUPS;
        const size_t smem = lnk::fwd_vec_smem<W, GROUPS>(a.C);
        int occ = 0;
        err = blocks_per_sm(kern, a.dev, threads, smem, &occ);
        if (err != cudaSuccess) return;
        const int64_t grid = std::min<int64_t>(ceil_div(a.N, GROUPS), int64_t(a.sms) * occ);
        err = launch(kern, (int)grid, threads, smem, a.stream, static_cast<T *>(a.out), a.mean,
                     a.rstd, static_cast<const T *>(a.inp), static_cast<const T *>(a.weight),
                     static_cast<const T *>(a.bias), static_cast<T *>(a.resid_out),
                     static_cast<const T *>(a.branch), a.N, a.C, a.inv_C, a.eps);
    }
    // Rows of 9..16 vectors per lane on two warps per row (V per warp).  When
    // two tiles per block do not fit in shared memory (the residual
    // variant's two arrays at bf16 C > 3.4K), one tile per block: a row's
    // arithmetic does not depend on the tile count, so the residual forward
    // still normalises exactly as ln_forward of its stored sum would.
    template <int V>
    void run_tile_two() {
        constexpr int NW = lnk::kTileWarps * 2;
        constexpr int TL = lnk::kTileFwdTiles;
        constexpr int RT = NW / 2;   // rows per tile
        if (lnk::fwd_tile_smem<T, NW, TL, 2, kArrays>(a.C) <= lnk::kMaxSmemPerBlock &&
            tile_grid_fits(a.N, RT * TL)) {
            run_tile<V, 2>();
        } else if (lnk::fwd_tile_smem<T, NW, 1, 2, kArrays>(a.C) <= lnk::kMaxSmemPerBlock &&
                   tile_grid_fits(a.N, RT)) {
            run_tile<V, 2, 1>();
        } else {
            run<4, 4, 2>();
        }
    }
    // Rows of 17..32 vectors per lane on four warps per row (V per warp):
    // blocks of 16 warps (4 rows per tile, 128 registers per thread) with as
    // many tiles (1..3) as fit in shared memory.  Measured on B200 (bf16,
    // 500 back-to-back calls) against the register-resident kernel with 8
    // warps per row: C = 8192 30.0 us against 38.3 (N = 4096), 98.2 against
    // 123.0 (N = 16384); C = 6144 32.4 against 37.7; C = 5120 35.1 against
    // 37.3; C = 4608 39.6 against 38.4.  Preferring fewer tiles so that two
    // blocks share an SM was slower at every width (34-51 us).
    template <int V>
    void run_tile_four() {
        constexpr int RW = 4, NW = 16, RT = NW / RW;   // RT rows per tile
        if (lnk::fwd_tile_smem<T, NW, 3, RW, kArrays>(a.C) <= lnk::kMaxSmemPerBlock &&
            tile_grid_fits(a.N, RT * 3)) {
            run_tile<V, RW, 3, NW>();
        } else if (lnk::fwd_tile_smem<T, NW, 2, RW, kArrays>(a.C) <= lnk::kMaxSmemPerBlock &&
                   tile_grid_fits(a.N, RT * 2)) {
            run_tile<V, RW, 2, NW>();
        } else if (lnk::fwd_tile_smem<T, NW, 1, RW, kArrays>(a.C) <= lnk::kMaxSmemPerBlock &&
                   tile_grid_fits(a.N, RT)) {
            run_tile<V, RW, 1, NW>();
        } else {
            run<4, 8, 1>();
        }
    }
    // Rows that fill every lane's V vectors exactly take a variant without
    // per-vector bound checks.
    template <int V, int RW, int TL = lnk::kTileFwdTiles, int NWB = lnk::kTileWarps * RW>
    void run_tile() {
        constexpr int E = lnk::Vec<T>::E;
        if (a.C / E == 32 * RW * V)
            run_tile_k<V, RW, TL, true, NWB>();
        else
            run_tile_k<V, RW, TL, false, NWB>();
    }
    template <int V, int RW, int TL, bool FULL, int NW = lnk::kTileWarps * RW>
    void run_tile_k() {   // NW warps: NW / RW rows per tile (8 for one or two warps per row)
        auto kern = lnk::ln_fwd_tile_kernel<T, V, NW, TL, RW, FULL, MODE>;
        const int threads = 32 * NW;
        const size_t smem = lnk::fwd_tile_smem<T, NW, TL, RW, kArrays>(a.C);
        int occ = 0;
        err = blocks_per_sm(kern, a.dev, threads, smem, &occ);   // also sets the smem limit
        if (err != cudaSuccess) return;
        const int rows = tile_rows_per_block(a.N, (NW / RW) * TL, int64_t(a.sms) * occ);
        const int64_t grid = ceil_div(a.N, rows);
        err = launch(kern, (int)grid, threads, smem, a.stream, static_cast<T *>(a.out), a.mean,
                     a.rstd, static_cast<const T *>(a.inp), static_cast<const T *>(a.weight),
                     static_cast<const T *>(a.bias), static_cast<T *>(a.resid_out),
                     static_cast<const T *>(a.branch), a.N, a.C, a.inv_C, a.eps, rows,
                     a.status);
    }
};

template <typename T, int MODE, bool BLOCK_ROW>
cudaError_t fwd_scalar(const FwdArgs &a) {
    auto kern = lnk::ln_fwd_scalar_kernel<T, BLOCK_ROW, MODE>;
    const int threads = BLOCK_ROW ? (a.C > 4096 ? 512 : 256) : 256;
    const int groups = BLOCK_ROW ? 1 : threads / 32;
    int occ = 0;
    cudaError_t e = blocks_per_sm(kern, a.dev, threads, 0, &occ);
    if (e != cudaSuccess) return e;
    const int64_t grid = std::min<int64_t>(ceil_div(a.N, groups), int64_t(a.sms) * occ);
    return launch(kern, (int)grid, threads, 0, a.stream, static_cast<T *>(a.out), a.mean,
                  a.rstd, static_cast<const T *>(a.inp), static_cast<const T *>(a.weight),
                  static_cast<const T *>(a.bias), static_cast<T *>(a.resid_out),
                  static_cast<const T *>(a.branch), a.N, a.C, a.inv_C, a.eps);
}

template <typename T, int MODE>
int fwd_dispatch(const FwdArgs &a) {
    constexpr int E = lnk::Vec<T>::E;
    constexpr bool RES = (MODE & lnk::kFwdResidual) != 0;
    const bool vec_ok = (int64_t(a.C) * sizeof(T)) % 16 == 0 && aligned16(a.out) &&
                        aligned16(a.inp) && aligned16(a.weight) && aligned16(a.bias) &&
                        (!RES || (aligned16(a.resid_out) && aligned16(a.branch)));
    if (vec_ok) {
        FwdVec<T, MODE> v{a};
        if (lnk::visit_fwd_vec<T>(a.C / E, v)) return status_of(v.err);
    }
    if (a.C <= 1024) return status_of(fwd_scalar<T, MODE, false>(a));
    return status_of(fwd_scalar<T, MODE, true>(a));
}

// ----------------------------------------------------------------- backward

// Runs the row kernel on G blocks, then the fixed-order column finalise.
// Block b of the row kernel owns `per_block` consecutive units of `unit_rows`
// rows (TMA ring kernels: tiles, assigned round-robin; they also take the
// device status word).
template <typename T, bool TMA, typename K>
int bwd_run(const BwdArgs &a, K kern, int threads, size_t smem, int rows_granule,
            int unit_rows) {
    int occ = 0;
    if (blocks_per_sm(kern, a.dev, threads, smem, &occ) != cudaSuccess) return LN_ERR_CUDA;
    const int64_t units = ceil_div(a.N, unit_rows);
    int64_t G = std::min<int64_t>(int64_t(a.sms) * occ, ceil_div(a.N, rows_granule));
    // keep the partial sums within the workspace bound (matters only for very
    // wide rows, where fewer, longer-running blocks are the price)
    G = std::min<int64_t>(G, int64_t(kMaxWorkspaceBytes / (size_t(a.C) * 2 * sizeof(float))));
    if (a.scratch) G = std::min<int64_t>(G, a.scratch_floats / (2 * int64_t(a.C)));
    G = std::max<int64_t>(G, 1);
    const int64_t per_block = ceil_div(units, G);
    G = ceil_div(units, per_block);

    float *partial = a.scratch;
    if (!partial) {
        const size_t ws_bytes = size_t(G) * 2 * size_t(a.C) * sizeof(float);
        cudaMemPool_t pool = nullptr;
        uint64_t limit = 0;
        const cudaError_t ep = workspace_pool(a.dev, &pool, &limit);
        if (ep != cudaSuccess) return note_cuda_error(ep, "cudaMemPoolCreate (workspace pool)");
        if (limit != 0 && ws_bytes > limit) return LN_ERR_WORKSPACE;
        if (cudaMallocFromPoolAsync(reinterpret_cast<void **>(&partial), ws_bytes, pool,
                                    a.stream) != cudaSuccess) {
            cudaGetLastError();   // clear the non-sticky allocation error
            return LN_ERR_WORKSPACE;
        }
    }
    cudaError_t e;
    if constexpr (TMA) {
        e = launch(kern, (int)G, threads, smem, a.stream, static_cast<T *>(a.dinp), partial,
                   static_cast<const T *>(a.dout), static_cast<const T *>(a.inp),
                   static_cast<const T *>(a.weight), a.mean, a.rstd, a.N, a.C, a.inv_C,
                   per_block, a.eps, a.status);
    } else {
        e = launch(kern, (int)G, threads, smem, a.stream, static_cast<T *>(a.dinp), partial,
                   static_cast<const T *>(a.dout), static_cast<const T *>(a.inp),
                   static_cast<const T *>(a.weight), a.mean, a.rstd, a.N, a.C, a.inv_C,
                   per_block * unit_rows, a.eps);
    }
    if (e == cudaSuccess) {
        const int cblocks = (int)ceil_div(2 * int64_t(a.C), 32);
        e = launch(lnk::ln_colsum_kernel, cblocks, lnk::kColsumThreads, 0, a.stream, a.dweight,
                   a.dbias, static_cast<const float *>(partial), (int)G, a.C,
                   a.accumulate_params ? 1 : 0);
    }
    if (!a.scratch) {
        const cudaError_t ef = cudaFreeAsync(partial, a.stream);
        if (e == cudaSuccess && ef != cudaSuccess) {
            note_cuda_error(ef, "cudaFreeAsync");
            e = ef;
        }
    }
    return status_of(e);
}

template <typename T, int MODE>
struct BwdVec {
    const BwdArgs &a;
    int status = LN_OK;
    template <int V, int W, int GROUPS>
    void run() {
        status = bwd_run<T, false>(a, lnk::ln_bwd_vec_kernel<T, V, W, GROUPS, MODE>,
                                   32 * W * GROUPS, lnk::bwd_vec_smem<W, GROUPS>(a.C),
                                   GROUPS, 1);
    }
    template <int VR, int VC>
    void split() {
        constexpr int NS = lnk::BwdRingArrays<MODE>::value;
        constexpr int NR = lnk::kSplitRowWarps;
        constexpr int S_MAX = lnk::kSplitMaxStages;
        const int S =
            std::min(lnk::split_stages<T, NR, NS>(a.C, lnk::kMaxSmemPerBlock), S_MAX);
        constexpr int NCOL = lnk::SplitCols<VR>::value;
        status = bwd_run<T, true>(a, lnk::ln_bwd_split_kernel<T, VR, VC, NR, NCOL, MODE>,
                                  32 * (NR + NCOL + 1), lnk::split_smem<T, NR, NS>(a.C, S),
                                  NR, NR);
    }
    template <int V, int W>
    void ring() {
        constexpr int NS = lnk::BwdRingArrays<MODE>::value;
        constexpr int NC = lnk::BwdRingConsumers<W>::value;
        constexpr int S = lnk::BwdStages<V, NC, NS>::value;
        constexpr int RT = NC / W;                        // rows per tile
        status = bwd_run<T, true>(
            a, lnk::ln_bwd_tma_kernel<T, V, NC, S, LN_BWD_RING_RR != 0, W, MODE>,
            32 * (NC + 1), lnk::bwd_tma_smem<T, NC, S, W, NS>(a.C), RT, RT);
    }
};

template <typename T, int MODE>
int bwd_dispatch(const BwdArgs &a) {
    constexpr int E = lnk::Vec<T>::E;
    const bool vec_ok = (int64_t(a.C) * sizeof(T)) % 16 == 0 && aligned16(a.dinp) &&
                        aligned16(a.dout) && aligned16(a.inp) && aligned16(a.weight);
    if (vec_ok) {
        BwdVec<T, MODE> v{a};
        if (lnk::visit_bwd_ring<T, MODE>(a.C / E, v)) return v.status;
        if (lnk::visit_bwd_vec<T>(a.C / E, v)) return v.status;
    }
    const int threads = (int)std::min<int64_t>(512, ceil_div(a.C, 32) * 32);
    return bwd_run<T, false>(a, lnk::ln_bwd_scalar_kernel<T, MODE>, threads, 0, 1, 1);
}

}  // namespace lnh
