// ln_select.cuh -- which kernel variant serves a row of nvec 16-byte vectors.
// Shared by every launcher so that the variant and its shared-memory size are
// chosen in exactly one place.
//
// Forward: rows of up to 8 vectors per lane take the one-shot tile kernel
// (ln_tile.cuh) with one warp per row, rows of 9..16 the same kernel with two
// warps per row, rows of 17..32 with four; wider rows take the persistent
// register-resident kernel with 16 warps per row and 4 vectors per thread.
// Backward: rows of up to 4 (bf16, fp16) / 6 (fp32) vectors per lane take the
// persistent TMA-ring kernel (ln_tma.cuh) on one warp per row; 16-bit rows of
// 7..8 vectors per lane (plain and accumulating) the split ring of row and
// column warps (ln_split.cuh); other wider rows the ring with W = 2..7 warps
// per row; rows wider than that take the register-resident kernel (W =
// 4..16 warps per row, 4 vectors per thread).
// Rows wider than the widest variant, and any misaligned call, take the
// scalar kernels.
#pragma once

#include "ln_kernels.cuh"
#include "ln_split.cuh"
#include "ln_tile.cuh"
#include "ln_tma.cuh"

#ifndef LN_FWD_GROUPS_W1
#define LN_FWD_GROUPS_W1 8
#endif
#ifndef LN_BWD_GROUPS_W1
#define LN_BWD_GROUPS_W1 8
#endif
#ifndef LN_BWD_RING_RR
#define LN_BWD_RING_RR 1          // ring backward: tiles round-robin over blocks
#endif
#ifndef LN_TILE_FWD_TILES
#define LN_TILE_FWD_TILES 2       // tiles of 8 rows per forward block
#endif

namespace lnk {

// Largest dynamic shared memory of one block on sm_100 (227 KB).
constexpr size_t kMaxSmemPerBlock = 232448;

// consumer warps (= rows per tile) per block; the producer warp comes on top
#ifndef LN_TMA_BWD_CONSUMERS
#define LN_TMA_BWD_CONSUMERS 15   // + 1 producer warp: 512 threads, one block per SM
#endif
constexpr int kTmaBwdConsumers = LN_TMA_BWD_CONSUMERS;
// consumer warps of the backward ring when W warps share a row
template <int W> struct BwdRingConsumers {
    static constexpr int value = (kTmaBwdConsumers / W) * W;
};
// forward tile kernel: one-warp rows of at least this many vectors per lane
// are split over two warps.  Measured on B200 (bf16 C = 1600, 7 vectors per
// lane): one warp 24.6-25.0 us, two warps of 4 vectors 25.6-27.0 us (a fifth
// of their slots empty, plus two row exchanges); equal for fp32 C = 768.  So
// rows up to 8 vectors stay on one warp (9: never split).
#ifndef LN_TILE_FWD_W2_FROM_V
#define LN_TILE_FWD_W2_FROM_V 9
#endif
// Rows of 9..16 vectors per lane (bf16 C = 2049..4096): the tile kernel with
// two warps per row (at most 8 vectors per lane each) instead of the
// register-resident kernel with four.
#ifndef LN_TILE_FWD_TWO_WARPS
#define LN_TILE_FWD_TWO_WARPS 1
#endif
// Rows of 17..32 vectors per lane (bf16 C = 4097..8192): the tile kernel with
// four warps per row instead of the register-resident kernel with eight.
#ifndef LN_TILE_FWD_FOUR_WARPS
#define LN_TILE_FWD_FOUR_WARPS 1
#endif
constexpr int kTileWarps = 8;   // rows per forward tile (warps per tile, doubled at two per row)
constexpr int kTileFwdTiles = LN_TILE_FWD_TILES;

// Arrays streamed through the backward ring: inp and dout, plus the previous
// dinp when accumulating.
template <int MODE> struct BwdRingArrays {
    static constexpr int value = (MODE & kBwdAccumulate) ? 3 : 2;
};

#ifndef LN_TMA_BWD_STAGES
#define LN_TMA_BWD_STAGES 0       // 0: from the shared-memory budget (below)
#endif
// Backward ring depth: as many stages (2..6) of NC rows of NS arrays, at up to
// 32*V*16 bytes a row, as fit in about 200 KB (208 KB with three arrays) for
// one block per SM (100 KB at two).  Measured: a deeper ring lifts fp32 rows
// from 5.6 to 6.2 TB/s.
template <int V, int NC, int NS = 2> struct BwdStages {
    static constexpr size_t kBudget = (NC + 1) * 32 <= 256 ? (100u << 10)
                                      : NS > 2             ? (208u << 10)
                                                           : (200u << 10);
    static constexpr size_t kStage = size_t(NC) * NS * 32 * V * 16;
    static constexpr int kFit = int(kBudget / kStage);
    static constexpr int value =
        LN_TMA_BWD_STAGES ? LN_TMA_BWD_STAGES : (kFit < 2 ? 2 : (kFit > 6 ? 6 : kFit));
};

// Shared memory of a ring variant at the widest row it serves.
template <typename T, int V, int W, int NS>
constexpr size_t bwd_ring_smem_max() {
    constexpr int NC = BwdRingConsumers<W>::value;
    constexpr int S = BwdStages<V, NC, NS>::value;
    return bwd_tma_smem<T, NC, S, W, NS>(32 * W * V * Vec<T>::E);
}

// Calls visitor.template run<V, W, GROUPS>() for the forward variant; returns
// false when no vectorised variant covers nvec.
template <typename T, typename Visitor>
bool visit_fwd_vec(int nvec, Visitor &v) {
    switch ((nvec + 31) / 32) {
        case 1: v.template run<1, 1, LN_FWD_GROUPS_W1>(); return true;
        case 2: v.template run<2, 1, LN_FWD_GROUPS_W1>(); return true;
        case 3: v.template run<3, 1, LN_FWD_GROUPS_W1>(); return true;
        case 4: v.template run<4, 1, LN_FWD_GROUPS_W1>(); return true;
        case 5: v.template run<5, 1, LN_FWD_GROUPS_W1>(); return true;
        case 6: v.template run<6, 1, LN_FWD_GROUPS_W1>(); return true;
        case 7: v.template run<7, 1, LN_FWD_GROUPS_W1>(); return true;
        case 8: v.template run<8, 1, LN_FWD_GROUPS_W1>(); return true;
        default: break;
    }
    if constexpr (LN_TILE_FWD_TWO_WARPS) {
        switch ((nvec + 63) / 64) {          // vectors per lane on two warps per row
            case 5: v.template run_tile_two<5>(); return true;
            case 6: v.template run_tile_two<6>(); return true;
            case 7: v.template run_tile_two<7>(); return true;
            case 8: v.template run_tile_two<8>(); return true;
            default: break;
        }
    }
    if constexpr (LN_TILE_FWD_FOUR_WARPS) {
        switch ((nvec + 127) / 128) {        // vectors per lane on four warps per row
            case 5: v.template run_tile_four<5>(); return true;
            case 6: v.template run_tile_four<6>(); return true;
            case 7: v.template run_tile_four<7>(); return true;
            case 8: v.template run_tile_four<8>(); return true;
            default: break;
        }
    }
    if (nvec <= 4 * 32 * 4) { v.template run<4, 4, 2>(); return true; }
    if (nvec <= 8 * 32 * 4) { v.template run<4, 8, 1>(); return true; }
    if (nvec <= 16 * 32 * 4) { v.template run<4, 16, 1>(); return true; }
    return false;
}

// Backward ring (ln_tma.cuh).  One warp per row while a lane holds at most
// `one` vectors; wider rows are split over W = 2..7 warps with `shared`
// vectors per lane, which keeps x - mean in registers between the two
// passes.  Measured on B200: bf16 C = 1024 is faster on one warp (4 vectors,
// recomputing x - mean) than on two (the row-group exchange costs more than
// it saves); C = 1600 is faster on three warps (43 us) than on two with 4
// vectors (46 us).  With three arrays per stage (accumulating) a stage is
// half as large again, so fp32 rows stop at 4 vectors per lane, where two
// stages of the widest rows still fit in shared memory; recomputing the
// statistics, bf16 rows of 4 vectors per lane would spill, so they go to two
// warps.
// 16-bit rows: the widest one-warp row and the vectors per lane when W > 1
// warps share a row.  Measured on B200 (backward us, bf16): one = 4 / shared
// = 3 gives C = 1024 41.7-43.0 and C = 1600 40.9-41.1; shared = 2 (C = 1600
// on 4 warps, 78 % of the slots used against 69 %) 46.0-47.5 at C = 1600;
// one = 3 with shared = 2 (C = 1024 on two warps, an exact fit) 46.5-49.1 at
// C = 1024 -- the row exchanges cost more than the empty slots.
#ifndef LN_RING_ONE_16
#define LN_RING_ONE_16 4
#endif
#ifndef LN_RING_SHARED_16
#define LN_RING_SHARED_16 3
#endif
template <typename T, int MODE> struct RingVmax {   // 16-bit elements (bf16, fp16)
    static constexpr int one =
        (MODE & kBwdRecompute) && LN_RING_ONE_16 > 3 ? 3 : LN_RING_ONE_16;
    static constexpr int shared = LN_RING_SHARED_16;
};
template <int MODE> struct RingVmax<float, MODE> {
    static constexpr bool kAcc = (MODE & kBwdAccumulate) != 0;
    static constexpr int one = kAcc ? 4 : 6, shared = kAcc ? 4 : 5;
};

// The split backward (ln_split.cuh): 8 row warps (rows per tile), column
// warps and the producer.  It takes 16-bit rows of LN_SPLIT_FROM_V ..
// kSplitMaxV vectors per row-warp lane in the plain and dinp-accumulating
// backward; with recomputed statistics (the column warps would need the row
// warps' results first) those rows stay on the shared-row ring.  At most 16
// warps, so that ptxas can give every thread 128 registers (one scheduler's
// 16384 registers over 4 warps); the row warps keep g = dout * weight
// unpacked (up to 64 of them).
// Measured on B200 (bf16, back-to-back calls, median of 7 interleaved rounds,
// against the ring kernel): C = 2048 25.5 us against 28.4, C = 1600 36.9
// against 39.6; C = 1536 34.9 against 35.0, C = 1280 27.9 against 27.6,
// C = 1152 31.8 against 30.9, C = 1024 44.9 against 41.9.  So rows from 7
// vectors per lane.
#ifndef LN_SPLIT_FROM_V
#define LN_SPLIT_FROM_V 7
#endif
constexpr int kSplitRowWarps = 8;
constexpr int kSplitMaxV = 8;
template <typename T, int MODE> struct SplitServes {
    static constexpr bool value = sizeof(T) == 2 && (MODE & kBwdRecompute) == 0;
};
// Column warps for rows of up to 32 * VR vectors: one column vector per lane
// (VR warps) while the block stays within 16 warps, else 4 warps of two.
template <int VR> struct SplitCols {
    static constexpr int value = kSplitRowWarps + VR + 1 <= 16 ? VR : 4;
};
// Column-warp vectors per lane for rows of 32 * VR vectors.
template <int VR> struct SplitVc {
    static constexpr int value =
        ((32 * VR + SplitCols<VR>::value - 1) / SplitCols<VR>::value + 31) / 32;
};

// Shared rows of the ring: up to kRingMaxW warps per row (15, 12 or 14
// consumer warps at W = 5, 6, 7: whole row groups within the 16-warp block).
// Past that the register-resident kernels take over.
#ifndef LN_RING_MAX_W
#define LN_RING_MAX_W 7
#endif
constexpr int kRingMaxW = LN_RING_MAX_W;
static_assert(kRingMaxW == 4 || kRingMaxW == 7, "ring widths: up to 4 or 7 warps per row");

// Calls visitor.template ring<V, W>() or visitor.template split<VR, VC>();
// false when rows are wider than kRingMaxW warps of the ring cover.
template <typename T, int MODE, typename Visitor>
bool visit_bwd_ring(int nvec, Visitor &v) {
    constexpr int NS = BwdRingArrays<MODE>::value;
    constexpr int V1 = RingVmax<T, MODE>::one;
    constexpr int VS = RingVmax<T, MODE>::shared;
    static_assert(bwd_ring_smem_max<T, V1, 1, NS>() <= kMaxSmemPerBlock, "ring fits");
    static_assert(bwd_ring_smem_max<T, VS, 2, NS>() <= kMaxSmemPerBlock, "ring fits");
    static_assert(bwd_ring_smem_max<T, VS, 3, NS>() <= kMaxSmemPerBlock, "ring fits");
    static_assert(bwd_ring_smem_max<T, VS, 4, NS>() <= kMaxSmemPerBlock, "ring fits");
    static_assert(kRingMaxW < 5 || bwd_ring_smem_max<T, VS, 5, NS>() <= kMaxSmemPerBlock,
                  "ring fits");
    static_assert(kRingMaxW < 6 || bwd_ring_smem_max<T, VS, 6, NS>() <= kMaxSmemPerBlock,
                  "ring fits");
    static_assert(kRingMaxW < 7 || bwd_ring_smem_max<T, VS, 7, NS>() <= kMaxSmemPerBlock,
                  "ring fits");
    const int v1 = (nvec + 31) / 32;
    if constexpr (SplitServes<T, MODE>::value) {
        if (v1 >= LN_SPLIT_FROM_V && v1 <= kSplitMaxV) {
            switch (v1) {
                case 4: v.template split<4, SplitVc<4>::value>(); return true;
                case 5: v.template split<5, SplitVc<5>::value>(); return true;
                case 6: v.template split<6, SplitVc<6>::value>(); return true;
                case 7: v.template split<7, SplitVc<7>::value>(); return true;
                case 8: v.template split<8, SplitVc<8>::value>(); return true;
                default: break;
            }
        }
    }
    switch (v1) {
        case 1: v.template ring<1, 1>(); return true;
        case 2: v.template ring<2, 1>(); return true;
        case 3: v.template ring<3, 1>(); return true;
        default: break;
    }
    if constexpr (V1 >= 4) {
        if (v1 == 4) { v.template ring<4, 1>(); return true; }
    }
    if constexpr (V1 > 4) {
        if (v1 == 5) { v.template ring<5, 1>(); return true; }
        if (v1 == 6) { v.template ring<6, 1>(); return true; }
    }
    const int w = (nvec + 32 * VS - 1) / (32 * VS);          // warps per row at VS
    switch (w) {
        case 2: v.template ring<VS, 2>(); return true;
        case 3: v.template ring<VS, 3>(); return true;
        case 4: v.template ring<VS, 4>(); return true;
        default: break;
    }
    if constexpr (kRingMaxW >= 7) {
        switch (w) {
            case 5: v.template ring<VS, 5>(); return true;
            case 6: v.template ring<VS, 6>(); return true;
            case 7: v.template ring<VS, 7>(); return true;
            default: break;
        }
    }
    return false;
}

// Backward rows wider than the ring covers (more than kRingMaxW * 32 * shared
// vectors): the register-resident kernel with W = 4, 8 or 16 warps per row
// and 4 vectors per thread.  Calls visitor.template run<V, W, GROUPS>();
// false when rows are wider still.
template <typename T, typename Visitor>
bool visit_bwd_vec(int nvec, Visitor &v) {
    if (nvec <= 4 * 32 * 4) { v.template run<4, 4, 2>(); return true; }
    if (nvec <= 8 * 32 * 4) { v.template run<4, 8, 1>(); return true; }
    if (nvec <= 16 * 32 * 4) { v.template run<4, 16, 1>(); return true; }
    return false;
}

}  // namespace lnk
