// ftk_prune.cuh -- score-bound key pruning (FlashTopK README, "Highlights":
// adaptive key pruning decides per call whether to skip keys by a score
// bound).
//
// The pages name the bound but give no formula.  This one is the
// per-dimension box bound.  For a block B of 128 consecutive keys let
//     hi[d] = max_{s in B} sigma_s k[s,d],   lo[d] = min_{s in B} sigma_s k[s,d].
// Every key of B lies in that box, so with c = (hi + lo) / 2, r = (hi - lo) / 2
//     U_h = q_h . c + |q_h| . r  >=  q_h . sigma_s k_s  >=  q_h . c - |q_h| . r = L_h
// and, for sigma_s > 0 (sigma_s ReLU(x) = ReLU(sigma_s x)),
//     I[t,s] <= UB[t,B] = sum_{w_h >= 0} w_h ReLU(U_h) + sum_{w_h < 0} w_h ReLU(L_h).
// A (row tile, block) pair is skipped when every row t of the tile whose
// window meets B has
//     UB[t,B] + eps * A_t * M_B < tau_t,
//     A_t = sum_h |w_h| sum_d |q_hd|,   M_B = max_d max(|hi_d|, |lo_d|).
// A_t * M_B bounds the size of every term of both UB and I[t,s], so the
// margin (eps = 2^-10) covers the float32 rounding of the bound and of the
// scan's own scores (each within 1e-4 of that size): a skipped key could
// never have been collected (I >= tau), and the result is unchanged.
// Blocks holding a NaN key, a sigma that is not finite and > 0, or a
// non-finite product are never skipped (M_B = +inf).
//
// Cost: the box reads kv once.  The bound is SIMT float32 work of about
// 8K FMAs per (row, block) pair, 1/128 of the scan's pairs but off the
// tensor cores, so the call first estimates the skippable fraction on a
// sample of (tile, block) pairs and builds the skip bitmap only when the
// estimate reaches kPruneCutoff.
#pragma once

#include <stdint.h>

#include "ftk_device.cuh"

namespace ftk {

constexpr int kBlockKeys = 128;        // keys per bound block (= the scan's key tile)
constexpr int kBoundWordBlocks = 32;   // blocks per bitmap word / per bound work item
constexpr float kPruneEps = 0.0009765625f;  // 2^-10
constexpr float kPruneCutoff = 0.25f;  // auto mode: prune when >= 25% of pairs are skippable
constexpr int kEstTiles = 8;           // sampled row tiles of the estimate
constexpr int kEstBlocks = 32;         // sampled blocks per sampled tile
constexpr int kEstChunk = 2;           // sampled blocks per estimate work item

enum { BOUND_EST = 0, BOUND_FULL = 1, BOUND_OUT = 2 };

// Box of every key block: c and r of 128 dims, and M_B (+inf: never skip).
struct BoxArgs {
    const void *kv;
    const float *kv_scales;  // NULL: all ones
    int64_t S;
    int32_t nblocks;
    float *box;              // [nblocks][2][128]: c then r
    float *mb;               // [nblocks]
};

struct BoundArgs {
    const void *q;
    const float *weights;
    const int32_t *ks, *ke;  // NULL for BOUND_OUT (no windows)
    int64_t T, S;
    int32_t rt;              // rows per row tile
    int32_t ntiles;
    int32_t nblocks;
    int32_t nwords;          // bitmap words per row tile
    const float *box;
    const float *mb;
    const float *tau;        // [T]
    const int32_t *c_lo, *c_hi;  // scan key range of each row tile
    int32_t est_tiles;       // BOUND_EST: sampled tiles
    uint32_t *bits;          // BOUND_FULL: [ntiles][nwords]
    // Device counters (all in the call's info block): estimate counts, the
    // prune mode (0 auto: decide from the estimate, 1 forced), and the
    // outputs prune_enabled and blocks_pruned.
    uint32_t *est_total, *est_pruned;
    int32_t mode;
    int32_t *prune_enabled;
    unsigned long long *blocks_pruned;
    // BOUND_OUT
    float *out;
    int64_t ld;
};

}  // namespace ftk
