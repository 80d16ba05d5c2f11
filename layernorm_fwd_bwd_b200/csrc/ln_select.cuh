// ln_select.cuh -- which vectorised kernel variant serves a row of nvec
// 16-byte vectors.  Shared by every launcher so that the variant and its
// shared-memory size are chosen in exactly one place.
//
// Forward: one warp per row (8 rows per 256-thread block) while the row fits
// in V <= 8 vectors per lane; wider rows use W = 4, 8 or 16 warps per row with
// 4 vectors per thread.  Backward: the per-thread column accumulators
// (2 * V * E floats) stay at or below 64 registers, so one warp per row serves
// up to V = 6 (fp32) / 4 (bf16) vectors per lane and wider rows use W = 2, 4,
// 8 or 16 warps per row with 4 vectors per thread.  Blocks hold 256 threads
// (512 for W = 16).  Rows wider than the widest variant take the scalar path.
#pragma once

#include "ln_kernels.cuh"
#include "ln_tile.cuh"
#include "ln_tma.cuh"

#ifndef LN_FWD_GROUPS_W1
#define LN_FWD_GROUPS_W1 8
#endif
#ifndef LN_BWD_GROUPS_W1
#define LN_BWD_GROUPS_W1 8
#endif

// Rows served by one warp each: the forward runs, by default, the one-shot
// tile kernel (ln_tile.cuh; style 2) and the backward the persistent TMA-ring
// kernel (ln_tma.cuh; style 1).  Style 0 selects the persistent
// register-resident kernels (ln_kernels.cuh).  Measured on B200 at GPT-2 124M
// shapes: forward tile 35 us vs ring 45 us vs register 41 us; backward ring
// 59 us vs register 65 us vs cluster tile 120 us.
#ifndef LN_FWD_STYLE
#define LN_FWD_STYLE 2
#endif
#ifndef LN_BWD_STYLE
#define LN_BWD_STYLE 1
#endif
#ifndef LN_BWD_RING_RR
#define LN_BWD_RING_RR 1          // ring backward: tiles round-robin over blocks
#endif
#ifndef LN_TILE_FWD_TILES
#define LN_TILE_FWD_TILES 2       // tiles of 8 rows per forward block
#endif
#ifndef LN_TILE_BWD_TILES
#define LN_TILE_BWD_TILES 2       // tiles of 8 rows per backward block
#endif
#ifndef LN_TILE_CLUSTER
#define LN_TILE_CLUSTER 8         // backward blocks per cluster
#endif

namespace lnk {

// consumer warps (= rows per tile) per block; the producer warp comes on top
#ifndef LN_TMA_FWD_CONSUMERS
#define LN_TMA_FWD_CONSUMERS 8
#endif
#ifndef LN_TMA_BWD_CONSUMERS
#define LN_TMA_BWD_CONSUMERS 15   // + 1 producer warp: 512 threads, one block per SM
#endif
constexpr int kTmaFwdConsumers = LN_TMA_FWD_CONSUMERS;
constexpr int kTmaBwdConsumers = LN_TMA_BWD_CONSUMERS;
// consumer warps of the backward ring when W warps share a row
template <int W> struct BwdRingConsumers {
    static constexpr int value = (kTmaBwdConsumers / W) * W;
};
// forward tile kernel: rows of up to 4 vectors per lane take one warp, wider
// one-warp rows (5..8 vectors) are split over two warps (fewer registers,
// more warps per SM)
#ifndef LN_TILE_FWD_W2_FROM_V
#define LN_TILE_FWD_W2_FROM_V 5
#endif
constexpr int kTileWarps = 8;                 // warps (= rows per tile) per tile block
constexpr int kTileFwdTiles = LN_TILE_FWD_TILES;
constexpr int kTileBwdTiles = LN_TILE_BWD_TILES;
constexpr int kTileCluster = LN_TILE_CLUSTER;

// Ring depth: a stage holds 7-8 rows of up to 32*V 16-byte vectors (twice
// that in the backward, inp and dout); keep the ring near 48-96 KB per block.
template <int V> struct FwdStages { static constexpr int value = V <= 4 ? 4 : 2; };
#ifndef LN_TMA_BWD_STAGES
#define LN_TMA_BWD_STAGES 0       // 0: from the shared-memory budget (below)
#endif
// Backward ring depth: as many stages (2..6) of NC rows of inp and dout, at
// up to 32*V*16 bytes a row, as fit in about 200 KB for one block per SM
// (100 KB at two).  Measured: a deeper ring lifts fp32 rows from 5.6 to
// 6.2 TB/s.
template <int V, int NC> struct BwdStages {
    static constexpr size_t kBudget = (NC + 1) * 32 <= 256 ? (100u << 10) : (200u << 10);
    static constexpr size_t kStage = size_t(NC) * 2 * 32 * V * 16;
    static constexpr int kFit = int(kBudget / kStage);
    static constexpr int value =
        LN_TMA_BWD_STAGES ? LN_TMA_BWD_STAGES : (kFit < 2 ? 2 : (kFit > 6 ? 6 : kFit));
};

// Backward, one warp per row: at most 6 (fp32) / 4 (bf16) vectors per lane,
// i.e. at most 48 / 64 column accumulators per thread.
template <typename T> struct BwdVmaxW1 { static constexpr int value = 6; };
template <> struct BwdVmaxW1<bf16> { static constexpr int value = 4; };

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
    if (nvec <= 4 * 32 * 4) { v.template run<4, 4, 2>(); return true; }
    if (nvec <= 8 * 32 * 4) { v.template run<4, 8, 1>(); return true; }
    if (nvec <= 16 * 32 * 4) { v.template run<4, 16, 1>(); return true; }
    return false;
}

// Backward ring (ln_tma.cuh).  One warp per row while a lane holds at most
// 4 (bf16) / 6 (fp32) vectors; wider rows are split over W = 2..4 warps with
// 3 (bf16) / 5 (fp32) vectors per lane, which keeps x - mean in registers
// between the two passes.  Measured on B200: bf16 C = 1024 is faster on one
// warp (4 vectors, recomputing x - mean) than on two (the row-group exchange
// costs more than it saves); C = 1600 is faster on three warps (43 us) than
// on two with 4 vectors (46 us).  Calls visitor.template ring<V, W>();
// false when rows are wider than 4 warps cover.
template <typename T> struct RingVmax { static constexpr int one = 6, shared = 5; };
template <> struct RingVmax<bf16> { static constexpr int one = 4, shared = 3; };

template <typename T, typename Visitor>
bool visit_bwd_ring(int nvec, Visitor &v) {
    constexpr int V1 = RingVmax<T>::one;
    constexpr int VS = RingVmax<T>::shared;
    const int v1 = (nvec + 31) / 32;
    switch (v1) {
        case 1: v.template ring<1, 1>(); return true;
        case 2: v.template ring<2, 1>(); return true;
        case 3: v.template ring<3, 1>(); return true;
        case 4: v.template ring<4, 1>(); return true;
        default: break;
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
        default: return false;
    }
}

template <typename T, typename Visitor>
bool visit_bwd_vec(int nvec, Visitor &v) {
    constexpr int VM = BwdVmaxW1<T>::value;
    const int v1 = (nvec + 31) / 32;
    if (v1 <= VM) {
        switch (v1) {
            case 1: v.template run<1, 1, LN_BWD_GROUPS_W1>(); return true;
            case 2: v.template run<2, 1, LN_BWD_GROUPS_W1>(); return true;
            case 3: v.template run<3, 1, LN_BWD_GROUPS_W1>(); return true;
            case 4: v.template run<4, 1, LN_BWD_GROUPS_W1>(); return true;
            default: break;
        }
        if constexpr (VM > 4) {
            switch (v1) {
                case 5: v.template run<5, 1, LN_BWD_GROUPS_W1>(); return true;
                case 6: v.template run<6, 1, LN_BWD_GROUPS_W1>(); return true;
                default: break;
            }
        }
    }
    if (nvec <= 2 * 32 * 4) { v.template run<4, 2, 4>(); return true; }
    if (nvec <= 4 * 32 * 4) { v.template run<4, 4, 2>(); return true; }
    if (nvec <= 8 * 32 * 4) { v.template run<4, 8, 1>(); return true; }
    if (nvec <= 16 * 32 * 4) { v.template run<4, 16, 1>(); return true; }
    return false;
}

}  // namespace lnk
