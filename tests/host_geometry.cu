// host_geometry.cu -- host-side check of the library's kernel selection and
// launch geometry.  It runs on a machine without a GPU: nothing here calls
// the CUDA runtime, launches a kernel or instantiates one.
//
// For every row width the vectorised paths serve (1..2100 16-byte vectors),
// every element type and every variant, it visits the selection exactly as
// the launchers do (lnk::visit_fwd_vec, lnk::visit_bwd_ring,
// lnk::visit_bwd_vec) and checks:
//   - the chosen variant covers the row, with the fewest vectors per lane
//     (one-warp rows) or the fewest warps per row (shared rows);
//   - each family serves exactly its range: one-warp tiles up to 8 vectors
//     per lane, two-warp tiles up to 16, the backward ring up to its limits,
//     the register-resident kernels beyond, nothing past 2048 vectors;
//   - the variant's shared memory fits in one block, for the tile kernels
//     also with the one-tile and register-resident fallbacks the launcher
//     may take;
//   - the ring has 2..8 stages (its 128-byte barrier area holds 16) and
//     whole row groups of consumer warps; the split ring (row and column
//     warps) serves exactly the 16-bit rows of its range, its column warps
//     cover their slices and its 2..8 stages fit;
//   - every bulk copy is a whole number of 16-byte units, and the bytes one
//     mbarrier phase expects (all the copies that complete on it) stay below
//     the 2^20 limit of an mbarrier's transaction count.
// It also compares lnh::tile_rows_per_block with a brute-force search.
//
// Output: "sel <fwd|bwd> <dtype> <mode> <first nvec> <last nvec> <variant>"
// for each run of widths with the same choice, one "FAIL ..." line per
// failed check, and "checks <n> failures <m>".  Exit status 1 on failure.
#include <cstdint>
#include <cstdio>
#include <string>
#include <vector>

#include "../layernorm_fwd_bwd_b200/csrc/ln_dispatch.cuh"

namespace {

std::vector<std::string> g_fail;
long g_checks = 0;

void check(bool ok, const std::string &what) {
    ++g_checks;
    if (!ok) g_fail.push_back(what);
}

template <typename T> const char *tname();
template <> const char *tname<float>() { return "f32"; }
template <> const char *tname<lnk::bf16>() { return "bf16"; }
template <> const char *tname<lnk::f16>() { return "f16"; }

int cdiv(int a, int b) { return (a + b - 1) / b; }
std::string num(long v) { return std::to_string(v); }

constexpr size_t kMax = lnk::kMaxSmemPerBlock;
constexpr size_t kMaxTx = (size_t(1) << 20) - 1;   // mbarrier transaction count limit

// The bulk copies of a tile or stage: `arrays` copies of `rows` rows of
// `row_bytes` each, all completing on one mbarrier phase.
void check_copies(const std::string &ctx, size_t row_bytes, int rows, int arrays) {
    check(row_bytes % 16 == 0, ctx + "bulk copies are whole 16-byte units");
    check(size_t(arrays) * rows * row_bytes <= kMaxTx,
          ctx + "one phase expects fewer than 2^20 bytes");
}
constexpr int kMaxVec = 16 * 32 * 4;     // widest row of the register-resident kernels
constexpr int kWidest = 2100;            // widths visited: past kMaxVec

template <typename T, int MODE>
struct FwdChoice {
    int nvec;
    std::string label;
    static constexpr int E = lnk::Vec<T>::E;
    static constexpr int kArrays = (MODE & lnk::kFwdResidual) ? 2 : 1;

    std::string ctx() const {
        return std::string("fwd ") + tname<T>() + " mode " + num(MODE) + " nvec " + num(nvec) +
               ": ";
    }
    // W == 1: the one-warp tile kernel (the launcher takes the
    // register-resident kernel instead only past 2^34 rows); W > 1: the
    // register-resident kernel.
    template <int V, int W, int G>
    void run() {
        const int C = nvec * E;
        if (W == 1) {
            label = "tile V=" + num(V) + " W=1";
            check(V == cdiv(nvec, 32), ctx() + "one-warp rows take the fewest vectors per lane");
            check(V < LN_TILE_FWD_W2_FROM_V, ctx() + "one-warp tiles stay below the two-warp split");
            check(lnk::fwd_tile_smem<T, lnk::kTileWarps, lnk::kTileFwdTiles, 1, kArrays>(C) <= kMax,
                  ctx() + "tile shared memory fits");
            check_copies(ctx(), size_t(C) * sizeof(T), lnk::kTileWarps, kArrays);
            check_copies(ctx() + "weight and bias: ", size_t(C) * sizeof(T), 1, 2);
            check(lnk::fwd_vec_smem<1, G>(C) <= kMax, ctx() + "register-resident fallback fits");
        } else {
            label = "vec V=" + num(V) + " W=" + num(W);
            check(32 * W * V >= nvec, ctx() + "register-resident rows are covered");
            check(W == 4 || 32 * (W / 2) * V < nvec,
                  ctx() + "register-resident rows take the fewest warps");
            check(!LN_TILE_FWD_TWO_WARPS || nvec > 2 * 32 * 8,
                  ctx() + "rows of up to 16 vectors per lane take the two-warp tile");
            check(!LN_TILE_FWD_FOUR_WARPS || nvec > 4 * 32 * 8,
                  ctx() + "rows of up to 32 vectors per lane take the four-warp tile");
            check(lnk::fwd_vec_smem<W, G>(C) <= kMax, ctx() + "register-resident smem fits");
        }
    }
    template <int V>
    void run_tile_two() {
        const int C = nvec * E;
        constexpr int NW = 2 * lnk::kTileWarps;
        label = "tile2 V=" + num(V) + " W=2";
        if (lnk::fwd_tile_smem<T, NW, lnk::kTileFwdTiles, 2, kArrays>(C) > kMax)
            label += " tiles=1";
        check(64 * V >= nvec && 64 * (V - 1) < nvec,
              ctx() + "two-warp rows take the fewest vectors per lane");
        check(nvec > 32 * 8, ctx() + "two-warp rows are wider than one warp serves");
        check(lnk::fwd_tile_smem<T, NW, 1, 2, kArrays>(C) <= kMax,
              ctx() + "a one-tile two-warp block fits");
        check_copies(ctx(), size_t(C) * sizeof(T), NW / 2, kArrays);
        check_copies(ctx() + "weight and bias: ", size_t(C) * sizeof(T), 1, 2);
        check(nvec <= 4 * 32 * 4 && lnk::fwd_vec_smem<4, 2>(C) <= kMax,
              ctx() + "the four-warp register-resident fallback covers the row");
    }
    template <int V>
    void run_tile_four() {
        const int C = nvec * E;
        constexpr int NW = 16, RW = 4;
        int tl = 0;
        if (lnk::fwd_tile_smem<T, NW, 3, RW, kArrays>(C) <= kMax) tl = 3;
        else if (lnk::fwd_tile_smem<T, NW, 2, RW, kArrays>(C) <= kMax) tl = 2;
        else if (lnk::fwd_tile_smem<T, NW, 1, RW, kArrays>(C) <= kMax) tl = 1;
        label = "tile4 V=" + num(V) + " W=4 tiles=" + num(tl);
        check(128 * V >= nvec && 128 * (V - 1) < nvec,
              ctx() + "four-warp rows take the fewest vectors per lane");
        check(nvec > 2 * 32 * 8, ctx() + "four-warp rows are wider than two warps serve");
        check(tl >= 1, ctx() + "a one-tile four-warp block fits");
        check_copies(ctx(), size_t(C) * sizeof(T), NW / RW, kArrays);
        check_copies(ctx() + "weight and bias: ", size_t(C) * sizeof(T), 1, 2);
        check(nvec <= 8 * 32 * 4 && lnk::fwd_vec_smem<8, 1>(C) <= kMax,
              ctx() + "the eight-warp register-resident fallback covers the row");
    }
};

template <typename T, int MODE>
struct BwdChoice {
    int nvec;
    std::string label;
    static constexpr int E = lnk::Vec<T>::E;
    static constexpr int NS = lnk::BwdRingArrays<MODE>::value;
    static constexpr int ONE = lnk::RingVmax<T, MODE>::one;
    static constexpr int VS = lnk::RingVmax<T, MODE>::shared;

    std::string ctx() const {
        return std::string("bwd ") + tname<T>() + " mode " + num(MODE) + " nvec " + num(nvec) +
               ": ";
    }
    template <int V, int W>
    void ring() {
        const int C = nvec * E;
        constexpr int NC = lnk::BwdRingConsumers<W>::value;
        constexpr int S = lnk::BwdStages<V, NC, NS>::value;
        label = "ring V=" + num(V) + " W=" + num(W) + " S=" + num(S);
        check(32 * W * V >= nvec, ctx() + "ring rows are covered");
        if (W == 1)
            check(V == cdiv(nvec, 32) && V <= ONE,
                  ctx() + "one-warp ring rows take the fewest vectors per lane");
        else
            check(V == VS && W == cdiv(nvec, 32 * VS) && nvec > 32 * ONE &&
                      (!lnk::SplitServes<T, MODE>::value || cdiv(nvec, 32) < LN_SPLIT_FROM_V ||
                       nvec > 32 * lnk::kSplitMaxV),
                  ctx() + "shared ring rows: the fixed vectors per lane, the fewest warps, "
                          "only past one warp's and the split kernel's reach");
        if (lnk::SplitServes<T, MODE>::value)
            check(cdiv(nvec, 32) < LN_SPLIT_FROM_V || cdiv(nvec, 32) > lnk::kSplitMaxV,
                  ctx() + "rows the split kernel serves do not take the ring");
        check(S >= 2 && S <= 8, ctx() + "ring depth 2..8");
        check(NC % W == 0 && NC >= W, ctx() + "whole row groups of consumer warps");
        check(lnk::bwd_tma_smem<T, NC, S, W, NS>(C) <= kMax, ctx() + "ring shared memory fits");
        check_copies(ctx(), size_t(C) * sizeof(T), NC / W, NS);
    }
    template <int VR, int VC>
    void split() {
        const int C = nvec * E;
        constexpr int NR = lnk::kSplitRowWarps, NCOL = lnk::SplitCols<VR>::value;
        const int S = lnk::split_stages<T, NR, NS>(C, kMax);
        label = "split VR=" + num(VR) + " VC=" + num(VC) + " S=" + num(S);
        check(lnk::SplitServes<T, MODE>::value, ctx() + "split rows: 16-bit, statistics read");
        check(VR == cdiv(nvec, 32) && VR >= LN_SPLIT_FROM_V && VR <= lnk::kSplitMaxV,
              ctx() + "split rows take the fewest vectors per row-warp lane, in its range");
        check(32 * VC >= cdiv(nvec, NCOL) && 32 * (VC - 1) < cdiv(nvec, NCOL),
              ctx() + "column warps cover their slices with the fewest vectors per lane");
        check(S >= 2 && S <= lnk::kSplitMaxStages, ctx() + "split ring depth 2..8");
        check(2 * lnk::kSplitMaxStages * 8 <= 128, ctx() + "split barriers fit in 128 bytes");
        check(lnk::split_smem<T, NR, NS>(C, S) <= kMax, ctx() + "split shared memory fits");
        check(lnk::split_ring_offset(C) % 128 == 0, ctx() + "split ring starts 128-aligned");
        check(NR + NCOL + 1 <= 16, ctx() + "split block of at most 16 warps (128 registers)");
        check_copies(ctx(), size_t(C) * sizeof(T), NR, NS);
    }
    template <int V, int W, int G>
    void run() {
        const int C = nvec * E;
        label = "vec V=" + num(V) + " W=" + num(W);
        check(nvec > lnk::kRingMaxW * 32 * VS && nvec > 32 * ONE,
              ctx() + "the register-resident backward serves only rows past the ring");
        check(32 * W * V >= nvec, ctx() + "register-resident rows are covered");
        check(W == 4 || 32 * (W / 2) * V < nvec,
              ctx() + "register-resident rows take the fewest warps");
        check(lnk::bwd_vec_smem<W, G>(C) <= kMax, ctx() + "register-resident smem fits");
    }
};

// Prints each run of widths that share a choice.
struct Runs {
    std::string head, label;
    int first = 0, last = 0;
    void add(int nvec, const std::string &l) {
        if (!label.empty() && l == label && nvec == last + 1) {
            last = nvec;
            return;
        }
        flush();
        label = l;
        first = last = nvec;
    }
    void flush() {
        if (!label.empty())
            std::printf("sel %s %d %d %s\n", head.c_str(), first, last, label.c_str());
        label.clear();
    }
};

template <typename T, int MODE>
void forward_all() {
    Runs runs{std::string("fwd ") + tname<T>() + " " + num(MODE)};
    for (int nvec = 1; nvec <= kWidest; ++nvec) {
        FwdChoice<T, MODE> c{nvec, ""};
        const bool found = lnk::visit_fwd_vec<T>(nvec, c);
        check(found == (nvec <= kMaxVec),
              c.ctx() + "a vectorised forward exists exactly up to 2048 vectors");
        runs.add(nvec, found ? c.label : std::string("scalar"));
    }
    runs.flush();
}

template <typename T, int MODE>
void backward_all() {
    Runs runs{std::string("bwd ") + tname<T>() + " " + num(MODE)};
    for (int nvec = 1; nvec <= kWidest; ++nvec) {
        BwdChoice<T, MODE> c{nvec, ""};
        bool found = lnk::visit_bwd_ring<T, MODE>(nvec, c);
        if (!found) found = lnk::visit_bwd_vec<T>(nvec, c);
        check(found == (nvec <= kMaxVec),
              c.ctx() + "a vectorised backward exists exactly up to 2048 vectors");
        runs.add(nvec, found ? c.label : std::string("scalar"));
    }
    runs.flush();
}

void rows_per_block_all() {
    const int64_t Ns[] = {1, 7, 8, 9, 100, 4097, 16384, 32768, 65536, 1000003,
                          int64_t(1) << 34};
    const int64_t residents[] = {1, 148, 296, 444, 592, 1184};
    for (int64_t N : Ns)
        for (int max_rows : {8, 16})
            for (int64_t res : residents) {
                const int got = lnh::tile_rows_per_block(N, max_rows, res);
                // fewest rows in total (whole waves of `res` blocks times rows
                // per block); among equals, more rows per block
                int want = 0;
                int64_t want_cost = 0;
                for (int rows = (max_rows + 1) / 2; rows <= max_rows; ++rows) {
                    const int64_t blocks = (N + rows - 1) / rows;
                    const int64_t cost = (blocks + res - 1) / res * rows;
                    if (want == 0 || cost <= want_cost) {
                        want = rows;
                        want_cost = cost;
                    }
                }
                check(got == want, "tile_rows_per_block(" + num(N) + ", " + num(max_rows) + ", " +
                                       num(res) + ") = " + num(got) + ", brute force " +
                                       num(want));
            }
    check(lnh::tile_rows_per_block(16384, 16, 444) == 13,
          "GPT-2 1.5B forward: 13 rows per block on 444 resident blocks");

    // tile_grid_fits accepts a row count exactly when every rows-per-block
    // choice gives a block count that fits the grid's x dimension.
    const int64_t I = INT32_MAX;
    for (int max_rows : {4, 8, 12, 16})
        for (int64_t k = 1; k <= 16; ++k)
            for (int64_t d = -3; d <= 3; ++d) {
                const int64_t N = k * I + d;
                if (N < 1) continue;
                bool all_fit = true;
                for (int rows = (max_rows + 1) / 2; rows <= max_rows; ++rows)
                    all_fit = all_fit && (N + rows - 1) / rows <= I;
                check(lnh::tile_grid_fits(N, max_rows) == all_fit,
                      "tile_grid_fits(" + num(N) + ", " + num(max_rows) + ")");
                if (lnh::tile_grid_fits(N, max_rows))
                    for (int64_t res : residents) {
                        const int rows = lnh::tile_rows_per_block(N, max_rows, res);
                        check((N + rows - 1) / rows <= I, "tile grid of " + num(N) +
                                                              " rows fits the x dimension");
                    }
            }
}

}  // namespace

int main() {
    forward_all<float, 0>();
    forward_all<float, lnk::kFwdResidual>();
    forward_all<lnk::bf16, 0>();
    forward_all<lnk::bf16, lnk::kFwdResidual>();
    forward_all<lnk::f16, 0>();
    forward_all<lnk::f16, lnk::kFwdResidual>();
    backward_all<float, 0>();
    backward_all<float, lnk::kBwdAccumulate>();
    backward_all<float, lnk::kBwdRecompute>();
    backward_all<float, lnk::kBwdAccumulate | lnk::kBwdRecompute>();
    backward_all<lnk::bf16, 0>();
    backward_all<lnk::bf16, lnk::kBwdAccumulate>();
    backward_all<lnk::bf16, lnk::kBwdRecompute>();
    backward_all<lnk::bf16, lnk::kBwdAccumulate | lnk::kBwdRecompute>();
    backward_all<lnk::f16, 0>();
    backward_all<lnk::f16, lnk::kBwdAccumulate>();
    backward_all<lnk::f16, lnk::kBwdRecompute>();
    backward_all<lnk::f16, lnk::kBwdAccumulate | lnk::kBwdRecompute>();
    rows_per_block_all();
    for (const std::string &f : g_fail) std::printf("FAIL %s\n", f.c_str());
    std::printf("checks %ld failures %zu\n", g_checks, g_fail.size());
    return g_fail.empty() ? 0 : 1;
}
