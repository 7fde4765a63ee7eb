// ftk_rows.cuh -- exact row top-k over bf16 / fp32 rows (DeepSelect README,
// "Supported Cases" and "Usage"; also the selection step of dense recovery).
//
// One thread-block cluster per row; CTA c of the cluster owns a contiguous
// chunk of the row, and each of its warps a contiguous segment of the chunk.
// The row is streamed from HBM once:
//   1. a spread sample of the chunk (1024 values) gives a threshold F with no
//      atomics: the minimum over groups of the group maxima, the group size
//      chosen so that about >= 2 * topk * chunk / row elements lie above F;
//   2. the stream (cp.async into a 4-stage shared-memory ring) checks each
//      16-byte vector with a packed max against F and, only for the rare
//      vectors that reach it, writes the elements >= F, in column order,
//      into the warp's candidate list in shared memory;
//   3. the cluster finds the exact k-th largest candidate key u*: every CTA
//      gathers all candidate keys of the cluster through distributed shared
//      memory and radix-selects them locally (or, with very many
//      candidates, sums per-CTA histograms across the cluster).  If every
//      CTA kept all its elements >= u* (u* >= each F) and no candidate list
//      overflowed, u* is the row's k-th largest value; otherwise an exact
//      multi-pass radix select re-reads the row (L2);
//   4. ties at u* go to the smallest columns (CTA order, then segment order)
//      and an ordered compaction writes the selected columns in ascending
//      order.
// No sort, no global scratch.
#pragma once

#include <cooperative_groups.h>

#include "ftk_device.cuh"

namespace ftk {

namespace cg = cooperative_groups;

constexpr int kRowsThreads = 512;
constexpr int kRowsWarps = kRowsThreads / 32;
constexpr int kRowsMaxCluster = 8;
constexpr int kRowsCapWarp = 512;    // candidates per warp
constexpr int kRowsStages = 4;       // cp.async ring stages (one 16-byte vector per thread each)
constexpr int kRowsGather = kRowsStages * kRowsThreads * 4;  // keys gathered into the (free) ring
constexpr int64_t kRowsMaxCols = int64_t(1) << 30;

struct RowsArgs {
    const void *x;              // row r starts at x + r * ld elements
    int64_t ld;                 // row stride in elements
    int64_t cols;               // row length when no windows are given
    int64_t rows;               // rows covered by the grid
    const int32_t *nrows_dev;   // optional device count: rows >= *nrows_dev - nrows_off are skipped
    int32_t nrows_off;
    uint32_t val_fill;          // value bits of the padding slots (x's dtype)
    const int32_t *row_map;     // optional: output row of grid row r (also indexes win_*)
    const int32_t *win_ks;      // optional windows: row length ke - ks,
    const int32_t *win_ke;      //   reported index = ks + column
    const int32_t *row_end;     // optional: row r holds columns [0, row_end[r]) (clamped to [0, cols])
    void *out_idx;              // [*, ldo] int32 or int64 (the kernel's index type)
    void *out_val;              // [*, ldo] of the input dtype (or NULL)
    int k;
    int chunk;                  // columns per CTA, multiple of 8
    uint32_t *status;
    int64_t ldo;                // output row stride in elements (>= k)
    int64_t idx_fill;           // index of the padding slots of rows shorter than k
};
// Kept at 128 bytes: a larger kernel parameter block made the striding
// (LOOP) kernels spill registers.
static_assert(sizeof(RowsArgs) <= 128, "RowsArgs grew past 128 bytes");

struct RowsSmem {
    uint32_t cand_bits[kRowsWarps * kRowsCapWarp];  // raw value bits
    int32_t cand_col[kRowsWarps * kRowsCapWarp];    // column within the chunk
    uint4 ring[kRowsStages][kRowsThreads];           // stream staging; later the gathered keys
    uint32_t wmin[kRowsWarps];
    uint32_t hist[256];
    uint32_t tot[256];
    uint32_t warp_cnt[kRowsWarps];
    uint32_t warp_gt[kRowsWarps];
    uint32_t warp_eq[kRowsWarps];
    uint32_t sel_bin, sel_above;
    uint32_t r_gt[kRowsMaxCluster], r_eq[kRowsMaxCluster];  // per-CTA counts, this CTA's view
    // published to the cluster
    uint32_t cta_cnt, cta_fkey, cta_over, cta_gt, cta_eq;
    uint32_t nan_seen, overflow;
};

template <int DT>
struct RowsTraits;


template <>
struct RowsTraits<FTK_BF16> {
    using elem = uint16_t;
    static constexpr int kVec = 8;  // elements per 16-byte vector
    // 32-bit order-preserving key (the bf16 key in the top half).
    __device__ static uint32_t key(uint32_t bits) { return bf16_key(bits) << 16; }
    __device__ static bool isnan_bits(uint32_t bits) { return bf16_bits_isnan(bits); }
    __device__ static uint32_t element(const uint4 &v, int j)
    {
        const int q = j >> 1;  // register selects, no dynamic indexing
        const uint32_t w = q == 0 ? v.x : q == 1 ? v.y : q == 2 ? v.z : v.w;
        return (j & 1) ? (w >> 16) : (w & 0xFFFFu);
    }
    // True if some element of the vector may be >= F, for a strictly
    // positive F whose raw bits are in both halves of f2 (positive bf16
    // values order like signed 16-bit integers, negative ones are negative).
    __device__ static bool any_ge_pos(const uint4 &v, uint32_t f2)
    {
        const uint32_t m = __vmaxs2(__vmaxs2(v.x, v.y), __vmaxs2(v.z, v.w));
        return __vcmpges2(m, f2) != 0u;
    }
    // Bit j set for each element j >= F (strictly positive F, raw bits in
    // both halves of f2).
    __device__ static uint32_t ge_mask_pos(const uint4 &v, uint32_t f2)
    {
        uint32_t m = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t w = i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
            const uint32_t c = __vcmpges2(w, f2);  // 0xFFFF per matching half
            m |= ((c & 1u) | ((c >> 15) & 2u)) << (2 * i);
        }
        return m;
    }
    // Running max of the magnitudes (NaN detection).
    __device__ static uint32_t mag_max(uint32_t acc, const uint4 &v)
    {
        const uint32_t m = 0x7FFF7FFFu;
        return __vmaxu2(__vmaxu2(acc, __vmaxu2(v.x & m, v.y & m)), __vmaxu2(v.z & m, v.w & m));
    }
    __device__ static bool mag_has_nan(uint32_t acc)
    {
        return (acc & 0xFFFFu) > 0x7F80u || (acc >> 16) > 0x7F80u;
    }
};

template <>
struct RowsTraits<FTK_F32> {
    using elem = uint32_t;
    static constexpr int kVec = 4;
    __device__ static uint32_t key(uint32_t bits) { return f32_key(bits); }
    __device__ static bool isnan_bits(uint32_t bits) { return f32_bits_isnan(bits); }
    __device__ static uint32_t element(const uint4 &v, int j)
    {
        return j == 0 ? v.x : j == 1 ? v.y : j == 2 ? v.z : v.w;
    }
    // Positive floats order like signed 32-bit integers.
    __device__ static bool any_ge_pos(const uint4 &v, uint32_t f)
    {
        const int32_t m = max(max(static_cast<int32_t>(v.x), static_cast<int32_t>(v.y)),
                              max(static_cast<int32_t>(v.z), static_cast<int32_t>(v.w)));
        return m >= static_cast<int32_t>(f);
    }
    __device__ static uint32_t ge_mask_pos(const uint4 &v, uint32_t f)
    {
        const int32_t fi = static_cast<int32_t>(f);
        return (static_cast<int32_t>(v.x) >= fi ? 1u : 0u) | (static_cast<int32_t>(v.y) >= fi ? 2u : 0u) |
               (static_cast<int32_t>(v.z) >= fi ? 4u : 0u) | (static_cast<int32_t>(v.w) >= fi ? 8u : 0u);
    }
    __device__ static uint32_t mag_max(uint32_t acc, const uint4 &v)
    {
        const uint32_t m = 0x7FFFFFFFu;
        return max(max(acc, max(v.x & m, v.y & m)), max(v.z & m, v.w & m));
    }
    __device__ static bool mag_has_nan(uint32_t acc) { return acc > 0x7F800000u; }
};

// Adds 1 to hist[bin] for every active lane.  When all active lanes of the
// warp share one bin (as the top digits of a narrow candidate range and
// heavy ties do), one atomic adds their count.  Every lane of the warp must
// call it.
__device__ __forceinline__ void hist_add(uint32_t *hist, uint32_t bin, bool active)
{
    const uint32_t act = __ballot_sync(0xFFFFFFFFu, active);
    if (!act) return;
    const int lane = threadIdx.x & 31;
    const int leader = __ffs(act) - 1;
    const uint32_t b0 = __shfl_sync(0xFFFFFFFFu, bin, leader);
    if (__all_sync(0xFFFFFFFFu, !active || bin == b0)) {
        if (lane == leader) atomicAdd(&hist[b0], static_cast<uint32_t>(__popc(act)));
    } else if (active) {
        atomicAdd(&hist[bin], 1u);
    }
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src, bool pred)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
                 "r"(pred ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Finds the bin b holding the k-th largest element of tot[0..256):
// sum(tot[b+1..]) < k <= sum(tot[b..]); writes sm.sel_bin / sm.sel_above.
// Block-wide.
__device__ __forceinline__ void find_kth_bin256(RowsSmem &sm, uint32_t k)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp == 0) {
        uint32_t c[8], sum = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            c[i] = sm.tot[255 - 8 * lane - i];
            sum += c[i];
        }
        uint32_t inc = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t u = __shfl_up_sync(0xFFFFFFFFu, inc, o);
            if (lane >= o) inc += u;
        }
        uint32_t above = inc - sum;
        if (above < k && inc >= k) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (above + c[i] >= k) {
                    sm.sel_bin = 255 - 8 * lane - i;
                    sm.sel_above = above;
                    break;
                }
                above += c[i];
            }
        }
    }
    __syncthreads();
}

// Sums hist over the cluster into tot (every CTA computes the same totals).
__device__ __forceinline__ void cluster_sum256(cg::cluster_group &cluster, RowsSmem &sm)
{
    const unsigned cs = cluster.num_blocks();
    for (int b = threadIdx.x; b < 256; b += blockDim.x) {
        uint32_t s = 0;
        for (unsigned r = 0; r < cs; ++r) s += cluster.map_shared_rank(sm.hist, r)[b];
        sm.tot[b] = s;
    }
}

__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

// Top-k of grid row r by the whole cluster.  Returns with every cp.async
// of this CTA complete and, for rows that used distributed shared memory,
// with every CTA of the cluster done reading this CTA's shared memory.
template <int DT, typename IT>
__device__ __forceinline__ void rows_topk_row(const RowsArgs &a, RowsSmem &sm, cg::cluster_group &cluster,
                                              unsigned cs, unsigned rank, int64_t r)
{
    using Tr = RowsTraits<DT>;
    using elem = typename Tr::elem;
    constexpr int VEC = Tr::kVec;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t lt_mask = (1u << lane) - 1u;
    const int64_t orow = a.row_map ? a.row_map[r] : r;
    int64_t len = a.cols, base_index = 0;
    if (a.win_ks) {
        base_index = a.win_ks[orow];
        len = static_cast<int64_t>(a.win_ke[orow]) - base_index;
        if (len < 0) len = 0;
    }
    if (a.row_end) {
        const int64_t e = a.row_end[orow];
        len = e < 0 ? 0 : (e < len ? e : len);
    }
    const int k = a.k;
    const elem *row = reinterpret_cast<const elem *>(a.x) + r * a.ld;
    // Every output index is below 2^31 (cols <= 2^30; windows are int32), so
    // it is formed in 32 bits and only widened by the store when IT is int64.
    IT *oidx = static_cast<IT *>(a.out_idx) + orow * a.ldo;
    elem *oval = a.out_val ? static_cast<elem *>(a.out_val) + orow * a.ldo : nullptr;
    const int64_t c0 = static_cast<int64_t>(rank) * a.chunk;
    const int64_t c1 = min(len, c0 + static_cast<int64_t>(a.chunk));
    const int n = c1 > c0 ? static_cast<int>(c1 - c0) : 0;  // my columns

    // Short row: everything is selected, in column order, then padding.
    if (len <= k) {
        for (int i = tid; i < n; i += blockDim.x) {
            const uint32_t bits = row[c0 + i];
            if (Tr::isnan_bits(bits)) set_status(a.status, FTK_STATUS_NAN);
            oidx[c0 + i] = static_cast<IT>(static_cast<int32_t>(base_index + c0 + i));
            if (oval) oval[c0 + i] = static_cast<elem>(bits);
        }
        if (rank == 0) {
            for (int64_t j = len + tid; j < k; j += blockDim.x) {
                oidx[j] = static_cast<IT>(a.idx_fill);
                if (oval) oval[j] = static_cast<elem>(a.val_fill);
            }
        }
        return;
    }

    if (tid == 0) {
        sm.nan_seen = 0;
        sm.overflow = 0;
    }

    // ---- 1. threshold F from a spread sample (no atomics) ----
    const int nvec = n / VEC;
    const int per = (nvec + kRowsWarps - 1) / kRowsWarps;
    const int v0 = min(nvec, warp * per), v1 = min(nvec, v0 + per);
    const uint4 *src = reinterpret_cast<const uint4 *>(row + c0);
    constexpr int kSampleThreads = 128;                 // warps 0..3, 8 samples per lane
    constexpr int kSampleVecs = 8 / VEC;                // vectors per sampling lane
    const bool sampled = nvec >= kSampleThreads * kSampleVecs;
    uint32_t lmax = 0;
    if (sampled && tid < kSampleThreads) {
#pragma unroll
        for (int q = 0; q < kSampleVecs; ++q) {
            const int64_t sv = static_cast<int64_t>(tid * kSampleVecs + q) * nvec / (kSampleThreads * kSampleVecs);
            const uint4 x = __ldg(src + sv);
#pragma unroll
            for (int j = 0; j < VEC; ++j) lmax = max(lmax, Tr::key(Tr::element(x, j)));
        }
    }
    // Stream prologue: the first ring stages are in flight while F is found.
    const int nb = (v1 - v0 + 31) / 32;  // 32-vector batches of my warp
#pragma unroll
    for (int b = 0; b < kRowsStages; ++b) {
        const int v = v0 + b * 32 + lane;
        cp_async16(&sm.ring[b][tid], v < v1 ? src + v : src, b < nb && v < v1);
        cp_async_commit();
    }
    // F = min over groups of the group maxima.  With G samples per group and
    // M groups, about ln(M / ln 2) / G of the values lie above it; take the
    // largest group that still leaves >= 2 * k / len of them.
    const double want = 2.0 * static_cast<double>(k) / static_cast<double>(len);
    int g = -1;  // log2 of lanes per group (0..7); -1: keep everything
    for (int gg = 7; gg >= 0; --gg) {
        const double G = 8.0 * (1 << gg), M = 1024.0 / G;
        if (log(M / 0.6931471805599453) / G >= want) {
            g = gg;
            break;
        }
    }
    if (warp < 4) {
        uint32_t m = lmax;
        const int gl = g < 0 ? 0 : (g > 5 ? 5 : g);  // lanes per group inside a warp: 2^gl
        for (int o = 1; o < (1 << gl); o <<= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        // min over the groups inside this warp (g < 5), or the warp max (g >= 5)
        uint32_t w = m;
        for (int o = (1 << gl); o < 32; o <<= 1) w = min(w, __shfl_xor_sync(0xFFFFFFFFu, w, o));
        if (lane == 0) sm.wmin[warp] = w;
    }
    __syncthreads();
    uint32_t fkey;
    if (n == 0) {
        fkey = 0xFFFFFFFFu;  // no elements, no candidates
    } else if (!sampled || g < 0) {
        fkey = 0u;           // keep everything
    } else if (g <= 5) {
        fkey = min(min(sm.wmin[0], sm.wmin[1]), min(sm.wmin[2], sm.wmin[3]));
    } else if (g == 6) {
        fkey = min(max(sm.wmin[0], sm.wmin[1]), max(sm.wmin[2], sm.wmin[3]));
    } else {
        fkey = max(max(sm.wmin[0], sm.wmin[1]), max(sm.wmin[2], sm.wmin[3]));
    }
    if (DT == FTK_BF16 && fkey != 0xFFFFFFFFu) fkey &= 0xFFFF0000u;
    if (tid == 0) sm.cta_fkey = fkey;
    // A strictly positive F allows the packed raw-bits test.
    const bool fpos = fkey > 0x80000000u && fkey != 0xFFFFFFFFu;
    const uint32_t fbits = f32_from_key(fkey);  // F as f32 bits
    const uint32_t fraw = DT == FTK_BF16 ? ((fbits >> 16) | (fbits & 0xFFFF0000u)) : fbits;

    // ---- 2. stream the chunk; keep the elements >= F in column order ----
    {
        uint32_t *cb = sm.cand_bits + warp * kRowsCapWarp;
        int32_t *cc = sm.cand_col + warp * kRowsCapWarp;
        uint32_t wcnt = 0, mag = 0;
        for (int b = 0; b < nb; ++b) {
            cp_async_wait<kRowsStages - 1>();  // batch b has landed (my own slot)
            const int slot = b % kRowsStages;
            const uint4 x = sm.ring[slot][tid];
            {
                const int vn = v0 + (b + kRowsStages) * 32 + lane;
                cp_async16(&sm.ring[slot][tid], vn < v1 ? src + vn : src, vn < v1);
                cp_async_commit();
            }
            const int v = v0 + b * 32 + lane;
            bool hit = false;
            if (v < v1) {
                mag = Tr::mag_max(mag, x);
                if (fpos) {
                    hit = Tr::any_ge_pos(x, fraw);
                } else {
#pragma unroll
                    for (int j = 0; j < VEC; ++j) hit |= Tr::key(Tr::element(x, j)) >= fkey;
                }
            }
            if (__ballot_sync(0xFFFFFFFFu, hit)) {
                uint32_t m = 0;
                if (hit) {
                    if (fpos) {
                        m = Tr::ge_mask_pos(x, fraw);
                    } else {
#pragma unroll
                        for (int j = 0; j < VEC; ++j)
                            if (Tr::key(Tr::element(x, j)) >= fkey) m |= 1u << j;
                    }
                }
                const uint32_t c = __popc(m);
                uint32_t incl = c;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const uint32_t t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                    if (lane >= o) incl += t;
                }
                uint32_t pos = wcnt + incl - c;
                const int col0 = v * VEC;
                while (m) {  // the set bits, in column order
                    const int j = __ffs(m) - 1;
                    m &= m - 1u;
                    if (pos < static_cast<uint32_t>(kRowsCapWarp)) {
                        cb[pos] = Tr::element(x, j);
                        cc[pos] = col0 + j;
                    }
                    ++pos;
                }
                wcnt += __shfl_sync(0xFFFFFFFFu, incl, 31);
            }
        }
        cp_async_wait<0>();
        // ragged tail (n not a multiple of VEC): the last warp, in order
        bool tail_nan = false;
        if (warp == kRowsWarps - 1) {
            for (int e0 = nvec * VEC; e0 < n; e0 += 32) {
                const int e = e0 + lane;
                uint32_t bits = 0;
                bool hit = false;
                if (e < n) {
                    bits = row[c0 + e];
                    tail_nan |= Tr::isnan_bits(bits);
                    hit = Tr::key(bits) >= fkey;
                }
                const uint32_t bal = __ballot_sync(0xFFFFFFFFu, hit);
                const uint32_t pos = wcnt + __popc(bal & lt_mask);
                if (hit && pos < static_cast<uint32_t>(kRowsCapWarp)) {
                    cb[pos] = bits;
                    cc[pos] = e;
                }
                wcnt += __popc(bal);
            }
        }
        if (Tr::mag_has_nan(mag) || tail_nan) sm.nan_seen = 1;
        if (lane == 0) {
            sm.warp_cnt[warp] = min(wcnt, static_cast<uint32_t>(kRowsCapWarp));
            if (wcnt > static_cast<uint32_t>(kRowsCapWarp)) sm.overflow = 1;
        }
    }
    __syncthreads();
    if (tid == 0) {
        uint32_t t = 0;
        for (int ww = 0; ww < kRowsWarps; ++ww) t += sm.warp_cnt[ww];
        sm.cta_cnt = t;
        sm.cta_over = sm.overflow;
    }
    if (tid < kRowsMaxCluster) {
        sm.r_gt[tid] = 0;
        sm.r_eq[tid] = 0;
    }
    cluster.sync();  // every candidate list of the cluster is final from here on

    // ---- 3. exact threshold key u* ----
    uint32_t total = 0, fmax = 0, over = 0;
    for (unsigned rr = 0; rr < cs; ++rr) {
        const RowsSmem *o = cluster.map_shared_rank(&sm, rr);
        total += o->cta_cnt;
        fmax = max(fmax, o->cta_fkey == 0xFFFFFFFFu ? 0u : o->cta_fkey);
        over |= o->cta_over;
    }
    // Uniform across the cluster: every CTA reads the same values.
    bool exact_ok = !over && total >= static_cast<uint32_t>(k);
    uint32_t ustar = 0, above = 0;
    const int passes = DT == FTK_BF16 ? 2 : 4;
    if (exact_ok && total <= static_cast<uint32_t>(kRowsGather)) {
        uint32_t *gath = reinterpret_cast<uint32_t *>(sm.ring);  // the ring is free now
        // Few candidates: every CTA gathers all candidate keys of the cluster
        // into its own shared memory once and selects locally (identical
        // result in every CTA, no cluster barrier between passes).
        uint32_t off = 0;  // start of list (rr, warp) in gath
        uint32_t kmn = 0xFFFFFFFFu, kmx = 0u;  // bounds of the gathered keys
        for (unsigned rr = 0; rr < cs; ++rr) {
            const RowsSmem *o = cluster.map_shared_rank(&sm, rr);
            uint32_t before = 0;
            for (int ww = 0; ww < warp; ++ww) before += o->warp_cnt[ww];
            const uint32_t cnt = o->warp_cnt[warp];
            const uint32_t *cb = o->cand_bits + warp * kRowsCapWarp;
            for (uint32_t i = lane; i < cnt; i += 32) {
                const uint32_t u = Tr::key(cb[i]);
                gath[off + before + i] = u;
                kmn = min(kmn, u);
                kmx = max(kmx, u);
            }
            off += o->cta_cnt;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            kmn = min(kmn, __shfl_xor_sync(0xFFFFFFFFu, kmn, o));
            kmx = max(kmx, __shfl_xor_sync(0xFFFFFFFFu, kmx, o));
        }
        if (lane == 0) {
            sm.tot[warp] = kmn;
            sm.tot[kRowsWarps + warp] = kmx;
        }
        __syncthreads();
        for (int ww = 0; ww < kRowsWarps; ++ww) {
            kmn = min(kmn, sm.tot[ww]);
            kmx = max(kmx, sm.tot[kRowsWarps + ww]);
        }
        // Bits above the highest one where the keys differ are common to
        // all of them: the 8-bit radix digits start below those.
        const int lo_bit = 32 - 8 * passes;  // bf16 keys sit in the upper half
        const uint32_t diff = kmn ^ kmx;
        const int top = diff ? 31 - __clz(diff) : -1;
        uint32_t mask = top < 0 ? 0xFFFFFFFFu : (top == 31 ? 0u : ~((2u << top) - 1u));
        uint32_t prefix = kmx & mask, krem = static_cast<uint32_t>(k);
        for (int hi = top; hi >= lo_bit; hi -= 8) {
            const int shift = hi - 7 >= lo_bit ? hi - 7 : lo_bit;
            const uint32_t dmask = (2u << (hi - shift)) - 1u;
            for (int b = tid; b < 256; b += blockDim.x) sm.hist[b] = 0;
            __syncthreads();
            for (uint32_t i0 = 0; i0 < total; i0 += blockDim.x) {
                const uint32_t i = i0 + tid;
                const uint32_t u = i < total ? gath[i] : 0u;
                hist_add(sm.hist, (u >> shift) & dmask, i < total && (u & mask) == prefix);
            }
            __syncthreads();
            for (int b = tid; b < 256; b += blockDim.x) sm.tot[b] = sm.hist[b];
            __syncthreads();
            find_kth_bin256(sm, krem);
            prefix |= sm.sel_bin << shift;
            mask |= dmask << shift;
            krem -= sm.sel_above;
            above += sm.sel_above;
            __syncthreads();
        }
        ustar = prefix;
        // The candidates are exactly each chunk's elements >= its F, so they
        // hold every element >= u* iff u* >= every F.
        exact_ok = ustar >= fmax;
    } else if (exact_ok) {
        // Many candidates (heavy ties): per-CTA histograms of my own lists,
        // summed over the cluster through distributed shared memory.
        uint32_t prefix = 0, mask = 0, krem = static_cast<uint32_t>(k);
        for (int p = 0; p < passes; ++p) {
            const int shift = 24 - 8 * p;
            for (int b = tid; b < 256; b += blockDim.x) sm.hist[b] = 0;
            __syncthreads();
            {
                const uint32_t cnt = sm.warp_cnt[warp];
                const uint32_t *cb = sm.cand_bits + warp * kRowsCapWarp;
                for (uint32_t i0 = 0; i0 < cnt; i0 += 32) {
                    const uint32_t i = i0 + lane;
                    const uint32_t u = i < cnt ? Tr::key(cb[i]) : 0u;
                    hist_add(sm.hist, (u >> shift) & 255u, i < cnt && (u & mask) == prefix);
                }
            }
            cluster.sync();
            cluster_sum256(cluster, sm);
            __syncthreads();
            find_kth_bin256(sm, krem);
            prefix |= sm.sel_bin << shift;
            mask |= 255u << shift;
            krem -= sm.sel_above;
            above += sm.sel_above;
            cluster.sync();  // every CTA is done reading my hist
        }
        ustar = prefix;
        exact_ok = ustar >= fmax;
    }
    if (!exact_ok) {
        // Exact multi-pass radix select over the whole row (re-read from L2).
        uint32_t prefix = 0, mask = 0, krem = static_cast<uint32_t>(k);
        above = 0;
        for (int p = 0; p < passes; ++p) {
            const int shift = 24 - 8 * p;
            for (int b = tid; b < 256; b += blockDim.x) sm.hist[b] = 0;
            __syncthreads();
            for (int e0 = 0; e0 < n; e0 += blockDim.x) {
                const int e = e0 + tid;
                const uint32_t u = e < n ? Tr::key(row[c0 + e]) : 0u;
                hist_add(sm.hist, (u >> shift) & 255u, e < n && (u & mask) == prefix);
            }
            cluster.sync();
            cluster_sum256(cluster, sm);
            __syncthreads();
            find_kth_bin256(sm, krem);
            prefix |= sm.sel_bin << shift;
            mask |= 255u << shift;
            krem -= sm.sel_above;
            above += sm.sel_above;
            cluster.sync();
        }
        ustar = prefix;
    }
    const uint32_t need = static_cast<uint32_t>(k) - above;  // ties at u* to take, >= 1

    // ---- 4. ordered selection ----
    // Segment order is column order: the fast path walks each warp's
    // candidate list, the fallback each warp's contiguous slice of the chunk.
    const int seg = ((n + kRowsWarps - 1) / kRowsWarps + 31) & ~31;
    const int s0 = min(n, warp * seg), s1 = min(n, s0 + seg);
    const uint32_t wlen = exact_ok ? sm.warp_cnt[warp] : static_cast<uint32_t>(s1 - s0);
    auto item = [&](uint32_t i, uint32_t &bits, int &col) {
        if (exact_ok) {
            bits = sm.cand_bits[warp * kRowsCapWarp + i];
            col = sm.cand_col[warp * kRowsCapWarp + i];
        } else {
            col = s0 + static_cast<int>(i);
            bits = row[c0 + col];
        }
    };
    uint32_t my_gt = 0, my_eq = 0;
    for (uint32_t i0 = 0; i0 < wlen; i0 += 32) {
        const uint32_t i = i0 + lane;
        bool gt = false, eq = false;
        if (i < wlen) {
            uint32_t bits;
            int col;
            item(i, bits, col);
            const uint32_t u = Tr::key(bits);
            gt = u > ustar;
            eq = u == ustar;
        }
        my_gt += __popc(__ballot_sync(0xFFFFFFFFu, gt));
        my_eq += __popc(__ballot_sync(0xFFFFFFFFu, eq));
    }
    if (lane == 0) {
        sm.warp_gt[warp] = my_gt;
        sm.warp_eq[warp] = my_eq;
    }
    if (exact_ok) {
        // Counts of the CTAs before me, from their lists in place.
        for (unsigned rr = 0; rr < rank; ++rr) {
            const RowsSmem *o = cluster.map_shared_rank(&sm, rr);
            const uint32_t cnt = o->warp_cnt[warp];
            const uint32_t *cb = o->cand_bits + warp * kRowsCapWarp;
            uint32_t g = 0, q = 0;
            for (uint32_t i0 = 0; i0 < cnt; i0 += 32) {
                const uint32_t i = i0 + lane;
                const uint32_t u = i < cnt ? Tr::key(cb[i]) : 0u;
                g += __popc(__ballot_sync(0xFFFFFFFFu, i < cnt && u > ustar));
                q += __popc(__ballot_sync(0xFFFFFFFFu, i < cnt && u == ustar));
            }
            if (lane == 0 && (g | q)) {
                atomicAdd(&sm.r_gt[rr], g);
                atomicAdd(&sm.r_eq[rr], q);
            }
        }
    }
    __syncthreads();
    if (tid == 0) {
        uint32_t g = 0, q = 0;
        for (int ww = 0; ww < kRowsWarps; ++ww) {
            const uint32_t tg = sm.warp_gt[ww], tq = sm.warp_eq[ww];
            sm.warp_gt[ww] = g;  // exclusive prefixes
            sm.warp_eq[ww] = q;
            g += tg;
            q += tq;
        }
        sm.cta_gt = g;
        sm.cta_eq = q;
    }
    if (exact_ok) {
        __syncthreads();
        cluster_arrive();  // no more reads of other CTAs' shared memory
    } else {
        cluster.sync();
        for (unsigned rr = tid; rr < rank; rr += blockDim.x) {
            const RowsSmem *o = cluster.map_shared_rank(&sm, rr);
            sm.r_gt[rr] = o->cta_gt;
            sm.r_eq[rr] = o->cta_eq;
        }
        __syncthreads();
        cluster_arrive();
    }
    uint32_t eq_before = 0, sel_before = 0;
    for (unsigned rr = 0; rr < rank; ++rr) {
        const uint32_t g = sm.r_gt[rr], q = sm.r_eq[rr];
        const uint32_t take = eq_before >= need ? 0u : min(q, need - eq_before);
        sel_before += g + take;
        eq_before += q;
    }
    const uint32_t my_take = eq_before >= need ? 0u : min(sm.cta_eq, need - eq_before);
    const uint32_t w_gt = sm.warp_gt[warp], w_eq = sm.warp_eq[warp];
    uint32_t pos = sel_before + w_gt + min(w_eq, my_take);  // next output slot of this warp
    uint32_t eq_rank = w_eq;                                // CTA-local tie rank
    for (uint32_t i0 = 0; i0 < wlen; i0 += 32) {
        const uint32_t i = i0 + lane;
        uint32_t bits = 0;
        int col = 0;
        bool gt = false, eq = false;
        if (i < wlen) {
            item(i, bits, col);
            const uint32_t u = Tr::key(bits);
            gt = u > ustar;
            eq = u == ustar;
        }
        const uint32_t eq_bal = __ballot_sync(0xFFFFFFFFu, eq);
        const uint32_t rank_eq = eq_rank + __popc(eq_bal & lt_mask);
        const bool sel = gt || (eq && rank_eq < my_take);
        const uint32_t sel_bal = __ballot_sync(0xFFFFFFFFu, sel);
        if (sel) {
            const uint32_t p = pos + __popc(sel_bal & lt_mask);
            if (p < static_cast<uint32_t>(k)) {
                oidx[p] = static_cast<IT>(static_cast<int32_t>(base_index + c0 + col));
                if (oval) oval[p] = static_cast<elem>(bits);
            } else {
                set_status(a.status, FTK_STATUS_INTERNAL);
            }
        }
        pos += __popc(sel_bal);
        eq_rank += __popc(eq_bal);
    }
    if (tid == 0 && sm.nan_seen) set_status(a.status, FTK_STATUS_NAN);
    __syncwarp();
    cluster_wait();  // keep my shared memory alive until every CTA is done with it
}

// One cluster per row.  LOOP: clusters stride over the rows (the count may
// be on the device), so a grid sized for the SMs serves any row count;
// otherwise the grid holds one cluster per row.  IT: the output index type
// (int32_t or int64_t).
template <int DT, bool LOOP, typename IT>
__global__ void __launch_bounds__(kRowsThreads, 2) rows_topk_kernel(const RowsArgs a)
{
    extern __shared__ __align__(16) uint8_t smem_raw[];
    RowsSmem &sm = *reinterpret_cast<RowsSmem *>(smem_raw);
    cg::cluster_group cluster = cg::this_cluster();
    const unsigned cs = cluster.num_blocks();
    const unsigned rank = cluster.block_rank();
    int64_t nrows = a.rows;
    if (a.nrows_dev) {
        const int64_t c = static_cast<int64_t>(*a.nrows_dev) - a.nrows_off;
        nrows = c < nrows ? c : nrows;
    }
    // Row selection is uniform over the cluster: its CTAs walk the same rows.
    if constexpr (!LOOP) {
        const int64_t r = blockIdx.x / cs;
        if (r < nrows) rows_topk_row<DT, IT>(a, sm, cluster, cs, rank, r);
    } else {
        for (int64_t r = blockIdx.x / cs; r < nrows; r += gridDim.x / cs) {
            rows_topk_row<DT, IT>(a, sm, cluster, cs, rank, r);
            cp_async_wait<0>();
            __syncthreads();  // shared memory is free for the next row
        }
    }
}

}  // namespace ftk
