// ftk_rows.cuh -- exact row top-k over bf16 / fp32 rows (DeepSelect README,
// "Supported Cases" and "Usage"; also the selection step of dense recovery).
//
// One thread-block cluster per row; CTA c of the cluster owns a contiguous
// chunk of the row.  The row is read from HBM exactly once:
//   1. load: 16-byte vector loads; each element becomes a 16-bit
//      order-preserving key prefix, kept in shared memory, and feeds a
//      2048-bin histogram of its top 11 bits;
//   2. the cluster sums its histograms through distributed shared memory
//      and finds the bin holding the k-th largest key; a 32-bin pass over
//      the low 5 bits pins the exact 16-bit prefix.  bf16 keys are 16 bits,
//      so the threshold is exact; fp32 rows take two more 8-bit passes over
//      just the elements whose prefix ties, re-reading their full value
//      (an L2 hit);
//   3. with the exact k-th key u* known, every CTA counts its keys above
//      and equal to u*; ties at u* go to the smallest column indices (CTA
//      order, then index order), and an ordered compaction writes the
//      selected columns in ascending order.
// Nothing is sorted and no global scratch memory is used.
#pragma once

#include <cooperative_groups.h>

#include "ftk_device.cuh"

namespace ftk {

namespace cg = cooperative_groups;

constexpr int kRowsThreads = 512;
constexpr int kRowsWarps = kRowsThreads / 32;
constexpr int kRowsMaxCluster = 8;
constexpr int kRowsMaxChunk = 49152;  // 16-bit keys per CTA (96 KB)
constexpr int kHist1 = 2048;          // top 11 bits of the 16-bit prefix
constexpr int kHist2 = 256;

struct RowsArgs {
    const void *x;              // row r starts at x + r * ld elements
    int64_t ld;                 // row stride in elements
    int64_t cols;               // row length when no windows are given
    int64_t rows;               // rows covered by the grid
    const int32_t *nrows_dev;   // optional device count: rows >= *nrows_dev - nrows_off are skipped
    int32_t nrows_off;
    const int32_t *row_map;     // optional: output row of grid row r (also indexes win_*)
    const int32_t *win_ks;      // optional windows: row length ke - ks,
    const int32_t *win_ke;      //   reported index = ks + column
    int32_t *out_idx;           // [*, k]
    void *out_val;              // [*, k] of the input dtype (or NULL)
    int k;
    int chunk;                  // columns per CTA, multiple of 8
    uint32_t *status;
};

struct RowsSmem {
    uint32_t hist[kHist1];
    uint32_t tot[kHist1];
    uint32_t hist2[kHist2];
    uint32_t tot2[kHist2];
    uint32_t warp_gt[kRowsWarps];
    uint32_t warp_eq[kRowsWarps];
    uint32_t cta_gt;            // published to the cluster
    uint32_t cta_eq;
    uint32_t scan[kRowsThreads / 4 + 32];
    uint32_t sel_bin;
    uint32_t sel_above;
    uint32_t nan_seen;
};

template <int DT>
struct RowsTraits;

template <>
struct RowsTraits<FTK_BF16> {
    using elem = uint16_t;
    static constexpr int kVec = 8;  // elements per 16-byte load
    __device__ static uint32_t key16(uint32_t bits) { return bf16_key(bits); }
    __device__ static bool isnan_bits(uint32_t bits) { return bf16_bits_isnan(bits); }
};

template <>
struct RowsTraits<FTK_F32> {
    using elem = uint32_t;
    static constexpr int kVec = 4;
    __device__ static uint32_t key16(uint32_t bits) { return f32_key(bits) >> 16; }
    __device__ static bool isnan_bits(uint32_t bits) { return f32_bits_isnan(bits); }
};

// Sum of `count` bins of the histogram `local` over every CTA of the
// cluster, written to `tot` (each CTA computes the same totals).
__device__ __forceinline__ void cluster_sum_hist(cg::cluster_group &cluster, uint32_t *local,
                                                 uint32_t *tot, int count)
{
    const unsigned cs = cluster.num_blocks();
    for (int b = threadIdx.x; b < count; b += blockDim.x) {
        uint32_t s = 0;
        for (unsigned r = 0; r < cs; ++r) s += cluster.map_shared_rank(local, r)[b];
        tot[b] = s;
    }
}

// Finds the bin b holding the k-th largest element of the histogram
// tot[0..count): sum(tot[b+1..]) < k <= sum(tot[b..]).  Writes the bin and
// the count above it to sm.sel_bin / sm.sel_above.  Block-wide.
__device__ __forceinline__ void find_kth_bin(RowsSmem &sm, const uint32_t *tot, int count,
                                             uint32_t k)
{
    // Each thread owns `per` consecutive bins counted from the top.
    const int per = (count + blockDim.x - 1) / blockDim.x;
    const int t = threadIdx.x;
    uint32_t mine = 0;
    for (int i = 0; i < per; ++i) {
        int b = count - 1 - (t * per + i);
        if (b >= 0) mine += tot[b];
    }
    // Exclusive scan of `mine` over threads (warp shuffles + warp totals).
    const int lane = t & 31, warp = t >> 5;
    uint32_t incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) sm.scan[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int nw = blockDim.x / 32;
        uint32_t v = lane < nw ? sm.scan[lane] : 0;
        uint32_t inc = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t u = __shfl_up_sync(0xFFFFFFFFu, inc, o);
            if (lane >= o) inc += u;
        }
        if (lane < nw) sm.scan[32 + lane] = inc - v;  // exclusive warp offsets
    }
    __syncthreads();
    uint32_t above = sm.scan[32 + warp] + incl - mine;  // elements in bins above my group
    if (above < k && above + mine >= k) {
        for (int i = 0; i < per; ++i) {
            int b = count - 1 - (t * per + i);
            if (b < 0) break;
            if (above + tot[b] >= k) {
                sm.sel_bin = static_cast<uint32_t>(b);
                sm.sel_above = above;
                break;
            }
            above += tot[b];
        }
    }
    __syncthreads();
}

template <int DT>
__device__ __forceinline__ uint32_t load_bits(const typename RowsTraits<DT>::elem *row, int64_t c)
{
    return static_cast<uint32_t>(row[c]);
}

// Full 32-bit key of column c (fp32 rows only; re-reads the value).
__device__ __forceinline__ uint32_t full_key32(const uint32_t *row, int64_t c)
{
    return f32_key(__ldg(row + c));
}

template <int DT>
__global__ void __launch_bounds__(kRowsThreads, 1) rows_topk_kernel(const RowsArgs a)
{
    using Tr = RowsTraits<DT>;
    using elem = typename Tr::elem;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    RowsSmem &sm = *reinterpret_cast<RowsSmem *>(smem_raw);
    uint16_t *keys = reinterpret_cast<uint16_t *>(smem_raw + sizeof(RowsSmem));

    cg::cluster_group cluster = cg::this_cluster();
    const unsigned cs = cluster.num_blocks();
    const unsigned rank = cluster.block_rank();
    const int64_t r = blockIdx.x / cs;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // Row selection is uniform over the cluster, so whole clusters exit together.
    if (r >= a.rows) return;
    if (a.nrows_dev && r >= static_cast<int64_t>(*a.nrows_dev) - a.nrows_off) return;
    const int64_t orow = a.row_map ? a.row_map[r] : r;
    int64_t len = a.cols, base_index = 0;
    if (a.win_ks) {
        base_index = a.win_ks[orow];
        len = static_cast<int64_t>(a.win_ke[orow]) - base_index;
        if (len < 0) len = 0;
    }
    const int k = a.k;
    const elem *row = reinterpret_cast<const elem *>(a.x) + r * a.ld;
    int32_t *oidx = a.out_idx + orow * k;
    elem *oval = a.out_val ? reinterpret_cast<elem *>(a.out_val) + orow * k : nullptr;
    const int64_t c0 = static_cast<int64_t>(rank) * a.chunk;
    const int64_t c1 = min(len, c0 + a.chunk);
    const int n = c1 > c0 ? static_cast<int>(c1 - c0) : 0;  // my columns

    // Short row: everything is selected, in column order, then padding.
    if (len <= k) {
        for (int i = tid; i < n; i += blockDim.x) {
            uint32_t bits = load_bits<DT>(row, c0 + i);
            if (Tr::isnan_bits(bits)) set_status(a.status, FTK_STATUS_NAN);
            oidx[c0 + i] = static_cast<int32_t>(base_index + c0 + i);
            if (oval) oval[c0 + i] = static_cast<elem>(bits);
        }
        if (rank == 0) {
            for (int64_t j = len + tid; j < k; j += blockDim.x) {
                oidx[j] = -1;
                if (oval) oval[j] = DT == FTK_BF16 ? static_cast<elem>(0xFF80u)
                                                   : static_cast<elem>(0xFF800000u);
            }
        }
        return;
    }

    // ---- 1. load the chunk once: 16-bit key prefixes + 2048-bin histogram ----
    for (int b = tid; b < kHist1; b += blockDim.x) sm.hist[b] = 0;
    for (int b = tid; b < kHist2; b += blockDim.x) sm.hist2[b] = 0;
    if (tid == 0) sm.nan_seen = 0;
    __syncthreads();
    {
        bool nan = false;
        const int nvec = n / Tr::kVec;
        const uint4 *src = reinterpret_cast<const uint4 *>(row + c0);
        constexpr int U = 4;
        int v = tid;
        for (; v + (U - 1) * kRowsThreads < nvec; v += U * kRowsThreads) {
            uint4 w[U];
#pragma unroll
            for (int u = 0; u < U; ++u) w[u] = __ldg(src + v + u * kRowsThreads);
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const uint32_t *p = reinterpret_cast<const uint32_t *>(&w[u]);
                const int e0 = (v + u * kRowsThreads) * Tr::kVec;
#pragma unroll
                for (int j = 0; j < Tr::kVec; ++j) {
                    uint32_t bits = DT == FTK_BF16 ? ((p[j / 2] >> (16 * (j & 1))) & 0xFFFFu) : p[j];
                    nan |= Tr::isnan_bits(bits);
                    uint32_t k16 = Tr::key16(bits);
                    keys[e0 + j] = static_cast<uint16_t>(k16);
                    atomicAdd(&sm.hist[k16 >> 5], 1u);
                }
            }
        }
        for (; v < nvec; v += kRowsThreads) {
            uint4 w = __ldg(src + v);
            const uint32_t *p = reinterpret_cast<const uint32_t *>(&w);
            const int e0 = v * Tr::kVec;
#pragma unroll
            for (int j = 0; j < Tr::kVec; ++j) {
                uint32_t bits = DT == FTK_BF16 ? ((p[j / 2] >> (16 * (j & 1))) & 0xFFFFu) : p[j];
                nan |= Tr::isnan_bits(bits);
                uint32_t k16 = Tr::key16(bits);
                keys[e0 + j] = static_cast<uint16_t>(k16);
                atomicAdd(&sm.hist[k16 >> 5], 1u);
            }
        }
        for (int e = nvec * Tr::kVec + tid; e < n; e += kRowsThreads) {
            uint32_t bits = load_bits<DT>(row, c0 + e);
            nan |= Tr::isnan_bits(bits);
            uint32_t k16 = Tr::key16(bits);
            keys[e] = static_cast<uint16_t>(k16);
            atomicAdd(&sm.hist[k16 >> 5], 1u);
        }
        if (nan) sm.nan_seen = 1;
    }
    cluster.sync();

    // ---- 2. exact threshold key u* ----
    cluster_sum_hist(cluster, sm.hist, sm.tot, kHist1);
    __syncthreads();
    find_kth_bin(sm, sm.tot, kHist1, static_cast<uint32_t>(k));
    const uint32_t b1 = sm.sel_bin;
    uint32_t above = sm.sel_above;

    for (int e = tid; e < n; e += kRowsThreads) {
        uint32_t k16 = keys[e];
        if ((k16 >> 5) == b1) atomicAdd(&sm.hist2[k16 & 31u], 1u);
    }
    cluster.sync();
    cluster_sum_hist(cluster, sm.hist2, sm.tot2, 32);
    __syncthreads();
    find_kth_bin(sm, sm.tot2, 32, static_cast<uint32_t>(k) - above);
    const uint32_t pref16 = (b1 << 5) | sm.sel_bin;
    above += sm.sel_above;
    uint32_t ustar;  // full key of the k-th largest element
    if (DT == FTK_BF16) {
        ustar = pref16;
    } else {
        // Two 8-bit passes over the low half of the key, restricted to the
        // elements whose 16-bit prefix equals pref16 (full values re-read).
        const uint32_t *row32 = reinterpret_cast<const uint32_t *>(row);
        uint32_t prefix = pref16;
        for (int pass = 0; pass < 2; ++pass) {
            cluster.sync();  // everyone is done reading the previous hist2
            for (int b = tid; b < kHist2; b += blockDim.x) sm.hist2[b] = 0;
            __syncthreads();
            const int shift = pass == 0 ? 8 : 0;
            for (int e = tid; e < n; e += kRowsThreads) {
                if (keys[e] != pref16) continue;
                uint32_t key = full_key32(row32, c0 + e);
                if ((key >> (shift + 8)) == prefix) atomicAdd(&sm.hist2[(key >> shift) & 255u], 1u);
            }
            cluster.sync();
            cluster_sum_hist(cluster, sm.hist2, sm.tot2, kHist2);
            __syncthreads();
            find_kth_bin(sm, sm.tot2, kHist2, static_cast<uint32_t>(k) - above);
            prefix = (prefix << 8) | sm.sel_bin;
            above += sm.sel_above;
        }
        ustar = prefix;
    }
    const uint32_t need = static_cast<uint32_t>(k) - above;  // ties at u* to take, >= 1

    // ---- 3. ordered selection ----
    // Warp w scans the contiguous segment [seg0, seg1) of my chunk.
    const int seg = ((n + kRowsWarps - 1) / kRowsWarps + 31) & ~31;
    const int seg0 = min(n, warp * seg), seg1 = min(n, seg0 + seg);
    const uint32_t *row32 = reinterpret_cast<const uint32_t *>(row);
    auto classify = [&](int e, bool &gt, bool &eq) {
        uint32_t k16 = keys[e];
        if (DT == FTK_BF16) {
            gt = k16 > ustar;
            eq = k16 == ustar;
        } else {
            const uint32_t up = ustar >> 16;
            if (k16 != up) {
                gt = k16 > up;
                eq = false;
            } else {
                uint32_t key = full_key32(row32, c0 + e);
                gt = key > ustar;
                eq = key == ustar;
            }
        }
    };
    uint32_t my_gt = 0, my_eq = 0;
    for (int e0 = seg0; e0 < seg1; e0 += 32) {
        const int e = e0 + lane;
        bool gt = false, eq = false;
        if (e < seg1) classify(e, gt, eq);
        my_gt += __popc(__ballot_sync(0xFFFFFFFFu, gt));
        my_eq += __popc(__ballot_sync(0xFFFFFFFFu, eq));
    }
    if (lane == 0) {
        sm.warp_gt[warp] = my_gt;
        sm.warp_eq[warp] = my_eq;
    }
    __syncthreads();
    if (tid == 0) {
        uint32_t g = 0, q = 0;
        for (int w = 0; w < kRowsWarps; ++w) {
            uint32_t tg = sm.warp_gt[w], tq = sm.warp_eq[w];
            sm.warp_gt[w] = g;  // exclusive prefixes
            sm.warp_eq[w] = q;
            g += tg;
            q += tq;
        }
        sm.cta_gt = g;
        sm.cta_eq = q;
    }
    cluster.sync();
    // Ties are taken in CTA order; output positions follow CTA order too.
    uint32_t eq_before = 0, sel_before = 0;
    for (unsigned rr = 0; rr < rank; ++rr) {
        RowsSmem *o = cluster.map_shared_rank(&sm, rr);
        uint32_t g = o->cta_gt, q = o->cta_eq;
        uint32_t take = eq_before >= need ? 0u : min(q, need - eq_before);
        sel_before += g + take;
        eq_before += q;
    }
    const uint32_t my_take = eq_before >= need ? 0u : min(sm.cta_eq, need - eq_before);
    const uint32_t w_gt = sm.warp_gt[warp], w_eq = sm.warp_eq[warp];
    uint32_t pos = sel_before + w_gt + min(w_eq, my_take);  // next output slot of this warp
    uint32_t eq_rank = w_eq;                                // CTA-local tie rank
    for (int e0 = seg0; e0 < seg1; e0 += 32) {
        const int e = e0 + lane;
        bool gt = false, eq = false;
        if (e < seg1) classify(e, gt, eq);
        const uint32_t lt_mask = (1u << lane) - 1u;
        const uint32_t eq_bal = __ballot_sync(0xFFFFFFFFu, eq);
        const uint32_t my_rank = eq_rank + __popc(eq_bal & lt_mask);
        const bool sel = gt || (eq && my_rank < my_take);
        const uint32_t sel_bal = __ballot_sync(0xFFFFFFFFu, sel);
        if (sel) {
            const uint32_t p = pos + __popc(sel_bal & lt_mask);
            if (p < static_cast<uint32_t>(k)) {
                oidx[p] = static_cast<int32_t>(base_index + c0 + e);
                if (oval) oval[p] = row[c0 + e];  // original bits (keeps -0.0)
            } else {
                set_status(a.status, FTK_STATUS_INTERNAL);
            }
        }
        pos += __popc(sel_bal);
        eq_rank += __popc(eq_bal);
    }
    if (tid == 0 && sm.nan_seen) set_status(a.status, FTK_STATUS_NAN);
    cluster.sync();  // keep my shared memory alive until every CTA is done with it
}

}  // namespace ftk
