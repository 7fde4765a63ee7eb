// ftk_rows.cuh -- exact row top-k over bf16 / fp32 rows (DeepSelect README,
// "Supported Cases" and "Usage"; also the selection step of dense recovery).
//
// One thread-block cluster per row; CTA c of the cluster owns a contiguous
// chunk of the row and each of its 8 warps a contiguous segment of the
// chunk.  The row is read from HBM once, in the common case:
//   1. stream: every warp streams its segment through its own ring of
//      shared-memory stages filled by bulk copies (cp.async.bulk, no
//      multicast; lane 0 issues them, an mbarrier per stage), so about 8 KB
//      per warp are in flight without any thread issuing loads;
//   2. threshold F, while the first stages are in flight: a spread sample of
//      the chunk (one 16-byte vector per thread) and F = the r-th largest
//      sample (two levels of 11-bit bins; for bf16 exact, for fp32 to within
//      the lowest 10 key bits), r chosen so that the whole row very likely
//      keeps >= topk elements >= F;
//   3. filter: each vector is tested against F with one packed compare; the
//      rare vectors holding an element >= F are noted and, once per stage,
//      their elements go in column order to the warp's candidate list in
//      shared memory.  Elements equal to F that find the list full are only
//      counted (heavy ties);
//   4. exact k-th key u*: the cluster filters with one F (the largest of
//      its CTAs' estimates, exchanged while the first stages load), so every
//      list holds all of its chunk's elements > F and its elements == F are
//      stored or counted.  If at least topk elements are >= F, the k-th
//      largest is >= F: when fewer than topk are > F it is F itself (heavy
//      ties need no selection), otherwise every CTA gathers all candidate
//      keys of the cluster through distributed shared memory and
//      radix-selects those > F locally (11-bit digits);
//   5. output: the counts of each list (> u*, == u*) give every warp its
//      output slots; ties at u* go to the smallest columns (CTA order, then
//      warp order, then list order), written in ascending column order.
// Rows where step 4's conditions fail (adversarial or structured rows, very
// many candidates) take an exact fallback: multi-pass radix select over the
// chunk (8-bit digits, histograms summed over the cluster), a counting pass
// and an ordered writing pass, each streaming the chunk through the same
// rings and skipping what lies below F once the row is known to hold topk
// elements >= F.  No sort, no global scratch.
#pragma once

#include <cooperative_groups.h>
#include <type_traits>

#include "ftk_device.cuh"

namespace ftk {

namespace cg = cooperative_groups;

constexpr int kRowsThreads = 256;
constexpr int kRowsWarps = kRowsThreads / 32;
constexpr int kRowsMaxCluster = 8;
constexpr int kRowsLists = kRowsMaxCluster * kRowsWarps;  // candidate lists of a cluster
constexpr int kRowsCapWarp = 512;      // candidates per warp list
constexpr int kRowsStages = 2;         // ring stages per warp
constexpr int kRowsStageVecs = 256;    // 16-byte vectors per stage (4 KB)
constexpr int kRowsGather = kRowsWarps * kRowsStages * kRowsStageVecs * 4;  // keys that fit the rings
constexpr int kRowsBins = 2048;        // 11-bit digits
constexpr int kRowsKeepAll = 4096;     // chunks of at most this many elements keep all of them
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
    uint4 ring[kRowsWarps][kRowsStages][kRowsStageVecs];  // stream stages; later the gathered keys
    uint32_t cand_bits[kRowsWarps][kRowsCapWarp];         // raw value bits
    int32_t cand_col[kRowsWarps][kRowsCapWarp];           // column within the chunk
    uint32_t hist[kRowsBins];
    uint4 samp[kRowsThreads];                             // the spread sample (one vector per thread)
    uint64_t full[kRowsWarps][kRowsStages];               // one mbarrier per ring stage
    // this CTA's lists, read by the other CTAs of the cluster
    uint32_t w_cnt[kRowsWarps];    // stored entries
    uint32_t w_gtf[kRowsWarps];    // stored entries > F
    uint32_t w_eqs[kRowsWarps];    // stored entries == F
    uint32_t w_eqf[kRowsWarps];    // entries == F, stored or counted past the end of a full list
    uint32_t w_all[kRowsWarps];    // entries >= F, stored or not
    uint32_t w_kmax[kRowsWarps];   // largest stored key
    uint32_t cta_fkey, cta_over, cta_gt, cta_eq;
    // every list of the cluster in column order (index rank * kRowsWarps + warp)
    uint32_t l_off[kRowsLists + 1], l_cnt[kRowsLists];
    uint32_t l_gt[kRowsLists];     // entries > u*
    uint32_t l_eq[kRowsLists];     // stored entries == u*
    uint32_t l_eqt[kRowsLists];    // entries == u*, stored or counted
    uint32_t l_take[kRowsLists], l_selb[kRowsLists];
    uint32_t wsum[kRowsWarps];
    uint32_t red[2 * kRowsWarps];
    uint32_t sel_bin, sel_above, fmin, short_eq;
    uint32_t g_gt, g_eqt, g_over, g_kmax, g_all;
    uint32_t nan_seen, overflow;
};

// The warps' stage notes tile the histogram exactly (each warp clears its
// part after its stream).
static_assert(kRowsWarps * kRowsStageVecs == kRowsBins && kRowsStageVecs % 128 == 0, "notes tile the histogram");

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
    // Packed signed / unsigned 16-bit maxima.
    __device__ static uint32_t smax(uint32_t a, uint32_t b)
    {
        uint32_t d;
        asm("max.s16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
        return d;
    }
    __device__ static uint32_t umax(uint32_t a, uint32_t b)
    {
        uint32_t d;
        asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
        return d;
    }
    // The vector's elements as signed / unsigned 16-bit integers, reduced
    // to their maxima (two halves).
    __device__ static uint32_t vsmax(const uint4 &v) { return smax(smax(v.x, v.y), smax(v.z, v.w)); }
    __device__ static uint32_t vumax(const uint4 &v) { return umax(umax(v.x, v.y), umax(v.z, v.w)); }
    static constexpr uint32_t kSmaxInit = 0x80008000u;
    // For a strictly positive F: true if some element of the vector whose
    // signed maxima are m is >= F.  Positive bf16 values order like signed
    // 16-bit integers, negative ones are negative.  fm1 holds F's raw bits
    // minus one in both halves.
    __device__ static bool ge_from_smax(uint32_t m, uint32_t fm1) { return smax(m, fm1) != fm1; }
    __device__ static uint32_t fm1_of(uint32_t fraw16) { return (fraw16 - 1u) * 0x10001u; }
    // Bit j set for each element j >= F (strictly positive F; fm1 as for
    // ge_from_smax).
    __device__ static uint32_t ge_mask_pos(const uint4 &v, uint32_t fm1)
    {
        uint32_t m = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t w = i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
            const uint32_t d = smax(w, fm1) ^ fm1;  // a half is non-zero iff it is >= F
            m |= ((d & 0xFFFFu) ? 1u : 0u) << (2 * i);
            m |= ((d >> 16) ? 2u : 0u) << (2 * i);
        }
        return m;
    }
    // NaN seen, from the running maxima of the raw elements as signed
    // (a positive NaN is above 0x7F80) and unsigned (a negative NaN is
    // above 0xFF80) 16-bit integers.
    __device__ static bool nan_from(uint32_t s, uint32_t u)
    {
        return static_cast<int16_t>(s & 0xFFFFu) > 0x7F80 || static_cast<int16_t>(s >> 16) > 0x7F80 ||
               (u & 0xFFFFu) > 0xFF80u || (u >> 16) > 0xFF80u;
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
    __device__ static uint32_t smax(uint32_t a, uint32_t b)
    {
        return static_cast<uint32_t>(max(static_cast<int32_t>(a), static_cast<int32_t>(b)));
    }
    __device__ static uint32_t umax(uint32_t a, uint32_t b) { return max(a, b); }
    __device__ static uint32_t vsmax(const uint4 &v) { return smax(smax(v.x, v.y), smax(v.z, v.w)); }
    __device__ static uint32_t vumax(const uint4 &v) { return umax(umax(v.x, v.y), umax(v.z, v.w)); }
    static constexpr uint32_t kSmaxInit = 0x80000000u;
    // Positive floats order like signed 32-bit integers.
    __device__ static bool ge_from_smax(uint32_t m, uint32_t fm1)
    {
        return static_cast<int32_t>(m) > static_cast<int32_t>(fm1);
    }
    __device__ static uint32_t fm1_of(uint32_t fraw) { return fraw - 1u; }
    __device__ static uint32_t ge_mask_pos(const uint4 &v, uint32_t fm1)
    {
        const int32_t fi = static_cast<int32_t>(fm1);
        return (static_cast<int32_t>(v.x) > fi ? 1u : 0u) | (static_cast<int32_t>(v.y) > fi ? 2u : 0u) |
               (static_cast<int32_t>(v.z) > fi ? 4u : 0u) | (static_cast<int32_t>(v.w) > fi ? 8u : 0u);
    }
    __device__ static bool nan_from(uint32_t s, uint32_t u)
    {
        return static_cast<int32_t>(s) > 0x7F800000 || u > 0xFF800000u;
    }
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

// One atomic per active lane, no warp vote first: independent calls can
// overlap (colliding lanes are serialised by the shared-memory unit).
__device__ __forceinline__ void hist_add_plain(uint32_t *hist, uint32_t bin, bool active)
{
    if (active) atomicAdd(&hist[bin], 1u);
}

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v)
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xFFFFFFFFu, v, o);
        if (lane >= o) v += t;
    }
    return v;
}

// Finds the bin b of h[0 .. NB) holding the r-th largest counted element:
// sum(h[b+1 ..]) < r <= sum(h[b ..]).  Sets sm.sel_bin (0xFFFFFFFF if the
// counts sum to less than r) and sm.sel_above = sum(h[b+1 ..]).  Block-wide
// (two barriers); h must not change during the call.
template <int NB>
__device__ __forceinline__ bool find_bin_top(RowsSmem &sm, const uint32_t *h, uint32_t r)
{
    constexpr int B = NB / kRowsThreads;
    static_assert(B >= 1 && B * kRowsThreads == NB, "bins per thread");
    // (the warp index through a shuffle: provably warp-uniform, so per-warp
    // addresses stay in uniform registers)
    const int tid = threadIdx.x, lane = tid & 31, warp = __shfl_sync(0xFFFFFFFFu, tid >> 5, 0);
    uint32_t c[B], sum = 0;
#pragma unroll
    for (int i = 0; i < B; ++i) {
        c[i] = h[NB - 1 - B * tid - i];
        sum += c[i];
    }
    uint32_t inc = warp_incl_scan(sum);
    if (lane == 31) sm.wsum[warp] = inc;
    if (tid == 0) sm.sel_bin = 0xFFFFFFFFu;
    __syncthreads();
    uint32_t wb = 0;
#pragma unroll
    for (int w = 0; w < kRowsWarps; ++w) wb += w < warp ? sm.wsum[w] : 0u;
    inc += wb;
    uint32_t ab = inc - sum;
    if (ab < r && inc >= r) {
#pragma unroll
        for (int i = 0; i < B; ++i) {
            if (ab + c[i] >= r) {
                sm.sel_bin = static_cast<uint32_t>(NB - 1 - B * tid - i);
                sm.sel_above = ab;
                break;
            }
            ab += c[i];
        }
    }
    __syncthreads();
    return sm.sel_bin != 0xFFFFFFFFu;
}

// Block-wide sum of one value per thread (two barriers).
__device__ __forceinline__ uint32_t block_sum(RowsSmem &sm, uint32_t v)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = __reduce_add_sync(0xFFFFFFFFu, v);
    if (lane == 0) sm.red[warp] = v;
    __syncthreads();
    uint32_t s = 0;
#pragma unroll
    for (int w = 0; w < kRowsWarps; ++w) s += sm.red[w];
    __syncthreads();
    return s;
}

__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Bounded wait for a ring stage (bulk copies from valid memory always
// land; a wait that outlasts kWaitNs reports FTK_STATUS_TIMEOUT and gives up).
__device__ __forceinline__ bool stage_wait(uint64_t *bar, uint32_t parity, uint32_t *status)
{
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63u) == 0 && global_ns() - t0 > kWaitNs) {
            set_status(status, FTK_STATUS_TIMEOUT);
            return false;
        }
    }
}

__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

// One warp's stream of the vectors [wv0, wv1) of src through its ring.
// prologue(): lane 0 issues the first stages.  run(visit): waits for each
// stage in order, calls visit(x, valid, v) on every lane for each of its
// vectors (v: index into src; warp-collective), and refills the stage.
// ph holds the parity each stage's barrier waits for next (warp-uniform);
// every issued copy is waited for exactly once.
struct WarpStream {
    RowsSmem &sm;
    const uint4 *src;
    int wv0, nv, nst, warp, lane;
    uint32_t &ph;
    uint32_t *status;

    __device__ __forceinline__ void issue(int j) const
    {
        const int s = j % kRowsStages;
        const int cnt = min(kRowsStageVecs, nv - j * kRowsStageVecs);
        const uint32_t bytes = static_cast<uint32_t>(cnt) * 16u;
        mbar_arrive_expect_tx(&sm.full[warp][s], bytes);
        bulk_load(&sm.ring[warp][s][0], src + wv0 + j * kRowsStageVecs, bytes, &sm.full[warp][s]);
    }

    __device__ __forceinline__ void prologue() const
    {
        if (lane == 0) {
            fence_proxy_async();  // earlier generic accesses of the ring precede the copies
            for (int j = 0; j < min(kRowsStages, nst); ++j) issue(j);
        }
    }

    // Waits for the stages prologue() issued, without using them.
    __device__ __forceinline__ void drain() const
    {
        for (int j = 0; j < min(kRowsStages, nst); ++j) {
            const int s = j % kRowsStages;
            (void)stage_wait(&sm.full[warp][s], (ph >> s) & 1u, status);
            ph ^= 1u << s;
        }
        __syncwarp();
    }

    template <typename Visit>
    __device__ __forceinline__ bool run(Visit &&visit) const
    {
        return run(visit, [](const uint4 *, int) {});
    }

    // end(buf, vb) runs on every lane after the stage's vectors were
    // visited and before the stage is refilled (buf: the stage, vb: the
    // index of its first vector).
    template <typename Visit, typename End>
    __device__ __forceinline__ bool run(Visit &&visit, End &&end) const
    {
        bool ok = true;
        int issued = min(kRowsStages, nst);
        for (int j = 0; j < issued; ++j) {
            const int s = j % kRowsStages;
            const bool got = stage_wait(&sm.full[warp][s], (ph >> s) & 1u, status);
            ph ^= 1u << s;
            ok = __all_sync(0xFFFFFFFFu, ok && got);
            if (ok) {
                const uint4 *buf = sm.ring[warp][s];
                const int cnt = min(kRowsStageVecs, nv - j * kRowsStageVecs);
                const int vb = wv0 + j * kRowsStageVecs;
                // every vector of the stage read first (the loads overlap)
                uint4 xs[kRowsStageVecs / 32];
                if (cnt == kRowsStageVecs) {  // a full stage: every vector valid
#pragma unroll
                    for (int it = 0; it < kRowsStageVecs / 32; ++it) xs[it] = buf[it * 32 + lane];
#pragma unroll
                    for (int it = 0; it < kRowsStageVecs / 32; ++it) visit(xs[it], true, vb + it * 32 + lane);
                } else {  // the chunk's last, partial stage
#pragma unroll
                    for (int it = 0; it < kRowsStageVecs / 32; ++it) {
                        const int i = it * 32 + lane;
                        xs[it] = i < cnt ? buf[i] : make_uint4(0u, 0u, 0u, 0u);
                    }
#pragma unroll
                    for (int it = 0; it < kRowsStageVecs / 32; ++it) {
                        const int i = it * 32 + lane;
                        visit(xs[it], i < cnt, vb + i);
                    }
                }
                end(buf, vb);
            }
            __syncwarp();
            if (ok && j + kRowsStages < nst) {
                // The warp's reads of the stage are complete (their values
                // are in registers): the copy may overwrite it.
                if (lane == 0) issue(j + kRowsStages);
                ++issued;
            }
        }
        return ok;
    }
};

// Per-lane masks of the elements of x that are > u (gt) and == u (eq).
template <int DT>
__device__ __forceinline__ void cmp_masks(const uint4 &x, uint32_t u, uint32_t &gt, uint32_t &eq)
{
    using Tr = RowsTraits<DT>;
    gt = 0;
    eq = 0;
#pragma unroll
    for (int j = 0; j < Tr::kVec; ++j) {
        const uint32_t k = Tr::key(Tr::element(x, j));
        gt |= (k > u ? 1u : 0u) << j;
        eq |= (k == u ? 1u : 0u) << j;
    }
}

// Exact fallback for the cluster's row: u* by radix select over the chunks
// (8-bit digits, histograms summed over the cluster), then a counting pass
// and an ordered writing pass, all streamed through the rings.  Every CTA of
// the cluster calls it (it holds cluster barriers).  Ends with
// cluster_arrive() (no more reads of other CTAs' shared memory).
template <int DT, typename IT>
__device__ __noinline__ void rows_fallback(const RowsArgs &a, RowsSmem &sm, cg::cluster_group &cluster,
                                           unsigned cs, unsigned rank, const typename RowsTraits<DT>::elem *row,
                                           int64_t c0, int n, int64_t base_index, IT *oidx,
                                           typename RowsTraits<DT>::elem *oval, uint32_t &ph, uint32_t lo)
{
    using Tr = RowsTraits<DT>;
    using elem = typename Tr::elem;
    constexpr int VEC = Tr::kVec;
    // (the warp index through a shuffle: provably warp-uniform, so per-warp
    // addresses stay in uniform registers)
    const int tid = threadIdx.x, lane = tid & 31, warp = __shfl_sync(0xFFFFFFFFu, tid >> 5, 0);
    const int k = a.k;
    const int nvec = n / VEC;
    const int per = (nvec + kRowsWarps - 1) / kRowsWarps;
    const int wv0 = min(nvec, warp * per), wv1 = min(nvec, wv0 + per);
    const uint4 *src = reinterpret_cast<const uint4 *>(row + c0);
    const WarpStream ws{sm, src, wv0, wv1 - wv0, (wv1 - wv0 + kRowsStageVecs - 1) / kRowsStageVecs,
                        warp, lane, ph, a.status};
    const bool tail_warp = warp == kRowsWarps - 1;
    uint32_t *tot = sm.hist + 256;
    // A vector certainly holds no key >= t when t is strictly positive and
    // the packed maximum of its raw elements is below t's raw bits; the
    // passes skip such vectors whole (one test for the warp).
    auto fm1_of_key = [&](uint32_t t) {
        const uint32_t tb = f32_from_key(t);
        return Tr::fm1_of(DT == FTK_BF16 ? (tb >> 16) : tb);
    };
    auto may_hold = [&](const uint4 &x, uint32_t t, uint32_t t_fm1) {
        return t <= 0x80000000u || Tr::ge_from_smax(Tr::vsmax(x), t_fm1);
    };
    // Keys below lo cannot be the k-th largest (lo is 0 or a bound the row
    // has >= topk keys at or above).
    const uint32_t lo_fm1 = lo > 0x80000000u ? fm1_of_key(lo) : 0u;

    // ---- u*: radix select over the row, 8-bit digits ----
    const int passes = DT == FTK_BF16 ? 2 : 4;
    uint32_t prefix = 0, mask = 0, krem = static_cast<uint32_t>(k), above = 0;
    for (int p = 0; p < passes; ++p) {
        const int shift = 24 - 8 * p;
        if (tid < 256) sm.hist[tid] = 0;
        __syncthreads();
        ws.prologue();
        ws.run([&](const uint4 &x, bool valid, int) {
            const bool cand = valid && may_hold(x, lo, lo_fm1);
            if (lo != 0u) {
                // Few keys reach the histogram: each lane adds its own, with
                // no warp vote.
                if (cand) {
#pragma unroll
                    for (int j = 0; j < VEC; ++j) {
                        const uint32_t u = Tr::key(Tr::element(x, j));
                        if (u >= lo && (u & mask) == prefix) atomicAdd(&sm.hist[(u >> shift) & 255u], 1u);
                    }
                }
                return;
            }
            if (!__any_sync(0xFFFFFFFFu, cand)) return;  // (warp-uniform)
#pragma unroll
            for (int j = 0; j < VEC; ++j) {
                const uint32_t u = Tr::key(Tr::element(x, j));
                hist_add(sm.hist, (u >> shift) & 255u, cand && (u & mask) == prefix);
            }
        });
        if (tail_warp) {
            for (int e0 = nvec * VEC; e0 < n; e0 += 32) {
                const int e = e0 + lane;
                const uint32_t u = e < n ? Tr::key(row[c0 + e]) : 0u;
                hist_add(sm.hist, (u >> shift) & 255u, e < n && u >= lo && (u & mask) == prefix);
            }
        }
        cluster.sync();
        if (tid < 256) {
            uint32_t s = 0;
            for (unsigned rr = 0; rr < cs; ++rr) s += cluster.map_shared_rank(sm.hist, rr)[tid];
            tot[tid] = s;
        }
        __syncthreads();
        find_bin_top<256>(sm, tot, krem);
        const uint32_t b = sm.sel_bin == 0xFFFFFFFFu ? 0u : sm.sel_bin;  // (always found: k < len)
        if (sm.sel_bin == 0xFFFFFFFFu && tid == 0) set_status(a.status, FTK_STATUS_INTERNAL);
        prefix |= b << shift;
        mask |= 255u << shift;
        krem -= sm.sel_bin == 0xFFFFFFFFu ? 0u : sm.sel_above;
        above += sm.sel_bin == 0xFFFFFFFFu ? 0u : sm.sel_above;
        cluster.sync();  // every CTA is done reading my histogram
    }
    const uint32_t ustar = prefix;
    const uint32_t need = static_cast<uint32_t>(k) - above;  // ties at u* to take, >= 1
    // (the histogram is all zero again for the next row's sample)
    for (int b = tid; b < 512; b += kRowsThreads) sm.hist[b] = 0;

    // ---- counts of > u* and == u* per warp segment ----
    const uint32_t us_fm1 = ustar > 0x80000000u ? fm1_of_key(ustar) : 0u;
    uint32_t g = 0, q = 0;
    ws.prologue();
    ws.run([&](const uint4 &x, bool valid, int) {
        if (!__any_sync(0xFFFFFFFFu, valid && may_hold(x, ustar, us_fm1))) return;  // (warp-uniform)
        uint32_t gt, eq;
        cmp_masks<DT>(x, ustar, gt, eq);
        if (valid) {
            g += __popc(gt);
            q += __popc(eq);
        }
    });
    if (tail_warp) {
        for (int e = nvec * VEC + lane; e < n; e += 32) {
            const uint32_t u = Tr::key(row[c0 + e]);
            g += u > ustar ? 1u : 0u;
            q += u == ustar ? 1u : 0u;
        }
    }
    g = __reduce_add_sync(0xFFFFFFFFu, g);
    q = __reduce_add_sync(0xFFFFFFFFu, q);
    if (lane == 0) {
        sm.l_gt[warp] = g;
        sm.l_eq[warp] = q;
    }
    __syncthreads();
    if (tid == 0) {
        uint32_t tg = 0, tq = 0;
        for (int w = 0; w < kRowsWarps; ++w) {
            const uint32_t a0 = sm.l_gt[w], b0 = sm.l_eq[w];
            sm.l_gt[w] = tg;  // exclusive prefixes within the CTA
            sm.l_eq[w] = tq;
            tg += a0;
            tq += b0;
        }
        sm.cta_gt = tg;
        sm.cta_eq = tq;
    }
    cluster.sync();
    uint32_t eq_before = 0, sel_before = 0;
    for (unsigned rr = 0; rr < rank; ++rr) {
        const RowsSmem *o = cluster.map_shared_rank(&sm, rr);
        const uint32_t og = o->cta_gt, oq = o->cta_eq;
        const uint32_t take = eq_before >= need ? 0u : min(oq, need - eq_before);
        sel_before += og + take;
        eq_before += oq;
    }
    __syncthreads();
    cluster_arrive();  // no more reads of other CTAs' shared memory

    // ---- ordered writing pass ----
    const uint32_t my_take = eq_before >= need ? 0u : min(sm.cta_eq, need - eq_before);
    const uint32_t w_gt = sm.l_gt[warp], w_eq = sm.l_eq[warp];
    uint32_t pos = sel_before + w_gt + min(w_eq, my_take);  // next output slot of this warp
    uint32_t eq_rank = w_eq;                                // CTA-local tie rank
    auto emit = [&](uint32_t gt, uint32_t eq, const uint4 &x, int col0) {
        // this lane's elements in column order, ranks from warp prefix sums
        const uint32_t ce = __popc(eq);
        const uint32_t eb = warp_incl_scan(ce) - ce;
        uint32_t sel = gt;
        uint32_t er = eq_rank + eb;
        uint32_t m = eq;
        while (m) {
            const int j = __ffs(m) - 1;
            m &= m - 1u;
            if (er < my_take) sel |= 1u << j;
            ++er;
        }
        const uint32_t cnt = __popc(sel);
        const uint32_t incl = warp_incl_scan(cnt);
        uint32_t p = pos + incl - cnt;
        while (sel) {
            const int j = __ffs(sel) - 1;
            sel &= sel - 1u;
            if (p < static_cast<uint32_t>(k)) {
                oidx[p] = static_cast<IT>(static_cast<int32_t>(base_index + c0 + col0 + j));
                if (oval) oval[p] = static_cast<elem>(Tr::element(x, j));
            } else {
                set_status(a.status, FTK_STATUS_INTERNAL);
            }
            ++p;
        }
        pos += __shfl_sync(0xFFFFFFFFu, incl, 31);
        eq_rank += __shfl_sync(0xFFFFFFFFu, eb + ce, 31);
    };
    ws.prologue();
    ws.run([&](const uint4 &x, bool valid, int v) {
        if (!__any_sync(0xFFFFFFFFu, valid && may_hold(x, ustar, us_fm1))) return;  // (warp-uniform)
        uint32_t gt = 0, eq = 0;
        if (valid) cmp_masks<DT>(x, ustar, gt, eq);
        if (__ballot_sync(0xFFFFFFFFu, (gt | eq) != 0u)) emit(gt, eq, x, v * VEC);
    });
    if (tail_warp) {
        for (int e0 = nvec * VEC; e0 < n; e0 += 32) {
            const int e = e0 + lane;
            uint32_t gt = 0, eq = 0, bits = 0;
            if (e < n) {
                bits = row[c0 + e];
                const uint32_t u = Tr::key(bits);
                gt = u > ustar ? 1u : 0u;
                eq = u == ustar ? 1u : 0u;
            }
            // one element per lane: element 0 of a vector whose .x holds it
            const uint4 x = make_uint4(bits, 0u, 0u, 0u);
            if (__ballot_sync(0xFFFFFFFFu, (gt | eq) != 0u)) emit(gt, eq, x, e - 0);
        }
    }
}

// Where row r's data and this CTA's chunk of it are, and its warp
// segment (vectors [wv0, wv1) of the chunk).
template <int DT>
struct RowGeom {
    int64_t orow, len, base_index, c0;
    int n, nvec, wv0, wv1;
    const typename RowsTraits<DT>::elem *row;

    __device__ __forceinline__ RowGeom(const RowsArgs &a, int64_t r, unsigned rank, int warp)
    {
        constexpr int VEC = RowsTraits<DT>::kVec;
        orow = a.row_map ? a.row_map[r] : r;
        len = a.cols;
        base_index = 0;
        if (a.win_ks) {
            base_index = a.win_ks[orow];
            len = static_cast<int64_t>(a.win_ke[orow]) - base_index;
            if (len < 0) len = 0;
        }
        if (a.row_end) {
            const int64_t e = a.row_end[orow];
            len = e < 0 ? 0 : (e < len ? e : len);
        }
        row = reinterpret_cast<const typename RowsTraits<DT>::elem *>(a.x) + r * a.ld;
        c0 = static_cast<int64_t>(rank) * a.chunk;
        const int64_t c1 = min(len, c0 + static_cast<int64_t>(a.chunk));
        n = c1 > c0 ? static_cast<int>(c1 - c0) : 0;
        nvec = n / VEC;
        const int per = (nvec + kRowsWarps - 1) / kRowsWarps;
        wv0 = min(nvec, warp * per);
        wv1 = min(nvec, wv0 + per);
    }
    __device__ __forceinline__ const uint4 *src() const { return reinterpret_cast<const uint4 *>(row + c0); }
    // The spread sample of the chunk is taken (else every element is kept).
    __device__ __forceinline__ bool sampled() const { return nvec >= kRowsThreads && n > kRowsKeepAll; }
    // Issues this CTA's first ring stages and its sample load (cp.async into
    // sm.samp) for the row.
    __device__ __forceinline__ void prefetch(RowsSmem &sm, int warp, int lane, uint32_t &ph, uint32_t *status) const
    {
        const WarpStream ws{sm, src(), wv0, wv1 - wv0, (wv1 - wv0 + kRowsStageVecs - 1) / kRowsStageVecs,
                            warp, lane, ph, status};
        ws.prologue();
        if (sampled()) {
            const int t = threadIdx.x;
            const uint4 *p = src() + static_cast<int64_t>(t) * nvec / kRowsThreads;
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(&sm.samp[t])), "l"(p) : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    }
};

// Top-k of grid row r by the whole cluster.  Returns with every bulk copy
// of this CTA landed and every CTA of the cluster done with this CTA's
// shared memory.
// Top-k of grid row r by the whole cluster.  Returns with every bulk copy
// of this CTA landed (but those of the next row, see below) and every CTA
// of the cluster done with this CTA's shared memory.
// pre: on entry, whether row r's first stages and sample were issued
// already (RowGeom::prefetch); on return, whether those of row rnext were.
// With one CTA per row (cs == 1) the rings are idle once the row has
// streamed, so the next row's first stages load while this row's
// candidates are selected and written (rnext < 0: no next row).
template <int DT, typename IT>
__device__ __forceinline__ void rows_topk_row(const RowsArgs &a, RowsSmem &sm, cg::cluster_group &cluster,
                                              unsigned cs, unsigned rank, int64_t r, uint32_t &ph, bool &pre,
                                              int64_t rnext)
{
    using Tr = RowsTraits<DT>;
    using elem = typename Tr::elem;
    constexpr int VEC = Tr::kVec;
    // (the warp index through a shuffle: provably warp-uniform, so per-warp
    // addresses stay in uniform registers)
    const int tid = threadIdx.x, lane = tid & 31, warp = __shfl_sync(0xFFFFFFFFu, tid >> 5, 0);
    const uint32_t lt_mask = (1u << lane) - 1u;
    const RowGeom<DT> gm(a, r, rank, warp);
    const int64_t orow = gm.orow, len = gm.len, base_index = gm.base_index, c0 = gm.c0;
    const int n = gm.n;  // my columns
    const int k = a.k;
    const elem *row = gm.row;
    // Every output index is below 2^31 (cols <= 2^30; windows are int32), so
    // it is formed in 32 bits and only widened by the store when IT is int64.
    IT *oidx = static_cast<IT *>(a.out_idx) + orow * a.ldo;
    elem *oval = a.out_val ? static_cast<elem *>(a.out_val) + orow * a.ldo : nullptr;

    // Short row: everything is selected, in column order, then padding.
    // (Rows like this are never prefetched.)
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
        pre = false;
        return;
    }

    const int nvec = gm.nvec;
    const int wv0 = gm.wv0, wv1 = gm.wv1;
    const uint4 *src = gm.src();
    const WarpStream ws{sm, src, wv0, wv1 - wv0, (wv1 - wv0 + kRowsStageVecs - 1) / kRowsStageVecs,
                        warp, lane, ph, a.status};
    if (tid == 0) {
        sm.nan_seen = 0;
        sm.overflow = 0;
        sm.fmin = 0xFFFFFFFFu;
    }
    if (!pre) gm.prefetch(sm, warp, lane, ph, a.status);  // the first stages load while F is found
    pre = false;

    // ---- threshold F from a spread sample of the chunk ----
    uint32_t fkey = 0u;  // 0: keep every element
    asm volatile("cp.async.wait_all;" ::: "memory");  // my sample vector has landed
    if (gm.sampled()) {
        const uint4 sx = sm.samp[tid];
        // Samples above the row's k-th largest value: about
        // lam = k * m / len; F is the r-th largest sample with r a few
        // standard deviations above lam.
        const float m = static_cast<float>(kRowsThreads * VEC);
        const float lam = static_cast<float>(k) * m / static_cast<float>(len);
        const float rf = ceilf(lam + 4.f * sqrtf(lam) + 4.f);
        if (rf < m) {  // (the histogram is all zero here)
            // Two levels of 11-bit bins: the top bits of the keys, then the
            // next bits of the keys in the first level's bin (bf16: the
            // whole key, so F is the r-th largest sample itself; a coarse F
            // would let in up to a quarter octave more candidates).  The
            // second level's bins use the candidate lists' space, idle until
            // the stream.
            uint32_t *h2 = sm.cand_bits[0];
            for (int b = tid; b < kRowsBins; b += kRowsThreads) h2[b] = 0;
            uint32_t keys[VEC];
#pragma unroll
            for (int j = 0; j < VEC; ++j) {
                keys[j] = Tr::key(Tr::element(sx, j));
                hist_add_plain(sm.hist, keys[j] >> 21, true);
            }
            __syncthreads();
            find_bin_top<kRowsBins>(sm, sm.hist, static_cast<uint32_t>(rf));
            const uint32_t b = sm.sel_bin;  // found: the counts sum to m > r
            const uint32_t r2 = static_cast<uint32_t>(rf) - sm.sel_above;  // rank within bin b, >= 1
#pragma unroll
            for (int j = 0; j < VEC; ++j) hist_add_plain(h2, (keys[j] >> 10) & 0x7FFu, (keys[j] >> 21) == b);
            __syncthreads();  // (also: every thread has read b before it is overwritten)
            find_bin_top<kRowsBins>(sm, h2, r2);
            const uint32_t b2 = sm.sel_bin;  // found: bin b holds >= r2 samples
            uint32_t mn = 0xFFFFFFFFu;
#pragma unroll
            for (int j = 0; j < VEC; ++j)
                if ((keys[j] >> 21) == b && ((keys[j] >> 10) & 0x7FFu) == b2) mn = min(mn, keys[j]);
            mn = __reduce_min_sync(0xFFFFFFFFu, mn);
            if (lane == 0) atomicMin(&sm.fmin, mn);
            __syncthreads();
            fkey = sm.fmin == 0xFFFFFFFFu ? 0u : sm.fmin;
        }
    }
    if (cs > 1) {
        // One threshold for the whole row: the largest F of the cluster
        // (exchanged while the first stages are still in flight).  Every
        // list then holds its chunk's elements >= F, ties at F stored or
        // counted.
        if (tid == 0) sm.cta_fkey = fkey;
        cluster.sync();
        if (lane < static_cast<int>(cs))
            fkey = cluster.map_shared_rank(&sm, static_cast<unsigned>(lane))->cta_fkey;
        else
            fkey = 0u;
        fkey = __reduce_max_sync(0xFFFFFFFFu, fkey);
    }
    // A strictly positive F allows the packed raw-bits test.
    const bool fpos = fkey > 0x80000000u;
    const uint32_t fbits = f32_from_key(fkey);  // F as f32 bits (bf16: its top half)
    const uint32_t fraw = DT == FTK_BF16 ? ((fbits >> 16) | (fbits & 0xFFFF0000u)) : fbits;

    // ---- stream the chunk; keep the elements >= F in column order ----
    {
        uint32_t *cb = sm.cand_bits[warp];
        int32_t *cc = sm.cand_col[warp];
        uint32_t wcnt = 0, lost = 0, smx = Tr::kSmaxInit, umx = 0u;
        bool over = false;
        const uint32_t fm1 = Tr::fm1_of(DT == FTK_BF16 ? (fraw & 0xFFFFu) : fraw);
        // Element `bits` (column col) at list position pos; past the list's
        // end a tie at F is only counted, anything else is an overflow.
        auto put = [&](uint32_t pos, uint32_t bits, int col) {
            if (pos < static_cast<uint32_t>(kRowsCapWarp)) {
                cb[pos] = bits;
                cc[pos] = col;
            } else if (Tr::key(bits) == fkey) {
                ++lost;
            } else {
                over = true;
            }
        };
        // The warp-exclusive prefix and the total of the lanes' counts c <=
        // VEC, from one ballot per bit of c (independent, not a shuffle
        // chain); two ballots when every count is below 4.
        auto offsets = [&](uint32_t c, uint32_t &pre, uint32_t &tot) {
            pre = 0;
            tot = 0;
            const int nb = __all_sync(0xFFFFFFFFu, c < 4u) ? 2 : (VEC == 8 ? 4 : 3);
#pragma unroll
            for (int bt = 0; bt < 4; ++bt) {
                if (bt < nb) {
                    const uint32_t bb = __ballot_sync(0xFFFFFFFFu, (c >> bt) & 1u);
                    pre += static_cast<uint32_t>(__popc(bb & lt_mask)) << bt;
                    tot += static_cast<uint32_t>(__popc(bb)) << bt;
                }
            }
        };
        // Elements >= F of a vector, as a bit mask.
        auto ge_mask = [&](const uint4 &x) {
            if (fpos) return Tr::ge_mask_pos(x, fm1);
            uint32_t m = 0;
#pragma unroll
            for (int j = 0; j < VEC; ++j)
                if (Tr::key(Tr::element(x, j)) >= fkey) m |= 1u << j;
            return m;
        };
        // A vector with an element >= F is rare, but with 32 lanes some lane
        // has one in most iterations: the stage's hit vectors are noted (their
        // index in the stage, in column order) and appended once per stage,
        // 32 at a time, before the stage is refilled; each element is read
        // from the stage where it lies.  The notes use the histogram's space,
        // idle while the row streams.
        uint32_t *note = sm.hist + warp * kRowsStageVecs;
        uint32_t nhit = 0;  // warp-uniform
        auto append_noted = [&](const uint4 *buf, int vb) {
            __syncwarp();  // the notes are visible to every lane
            for (uint32_t h0 = 0; h0 < nhit; h0 += 32) {
                const uint32_t h = h0 + lane;
                uint32_t msk = 0;
                int i = 0;
                if (h < nhit) {
                    i = static_cast<int>(note[h]);
                    msk = ge_mask(buf[i]);
                }
                const elem *ev = reinterpret_cast<const elem *>(buf + i);
                const int col0 = (vb + i) * VEC;
                const uint32_t c = __popc(msk);
                if (__all_sync(0xFFFFFFFFu, c <= 2u)) {
                    // The common case: at most two elements per lane.  When
                    // the list has room for all of them, they are stored
                    // without a loop or a capacity check.
                    const uint32_t b1 = __ballot_sync(0xFFFFFFFFu, c == 1u);
                    const uint32_t b2 = __ballot_sync(0xFFFFFFFFu, c == 2u);
                    const uint32_t tot = __popc(b1) + 2u * __popc(b2);
                    if (wcnt + tot <= static_cast<uint32_t>(kRowsCapWarp)) {
                        if (c) {
                            const uint32_t pos = wcnt + __popc(b1 & lt_mask) + 2u * __popc(b2 & lt_mask);
                            const int j1 = __ffs(msk) - 1, j2 = 31 - __clz(msk);
                            cb[pos] = static_cast<uint32_t>(ev[j1]);
                            cc[pos] = col0 + j1;
                            if (c == 2u) {
                                cb[pos + 1] = static_cast<uint32_t>(ev[j2]);
                                cc[pos + 1] = col0 + j2;
                            }
                        }
                        wcnt += tot;
                        continue;
                    }
                }
                uint32_t pre, tot;
                offsets(c, pre, tot);
                uint32_t pos = wcnt + pre;
                while (msk) {  // the set bits, in column order
                    const int j = __ffs(msk) - 1;
                    msk &= msk - 1u;
                    put(pos++, static_cast<uint32_t>(ev[j]), col0 + j);
                }
                wcnt += tot;
            }
            nhit = 0;
            __syncwarp();  // every note is read before the next stage writes them
        };
        // One vector: running maxima (for the NaN check) and the hit note.
        // FP: F is strictly positive (packed raw-bits test); VALID: the
        // vector lies in the chunk.
        auto visit = [&](auto fp, const uint4 &x, bool valid, int v) {
            constexpr bool FP = decltype(fp)::value;
            bool hit = false;
            if (valid) {
                const uint32_t vs = Tr::vsmax(x);
                smx = Tr::smax(smx, vs);
                umx = Tr::umax(umx, Tr::vumax(x));
                if constexpr (FP) {
                    hit = Tr::ge_from_smax(vs, fm1);
                } else {
#pragma unroll
                    for (int j = 0; j < VEC; ++j) hit |= Tr::key(Tr::element(x, j)) >= fkey;
                }
            }
            const uint32_t bal = __ballot_sync(0xFFFFFFFFu, hit);
            if (hit) note[nhit + __popc(bal & lt_mask)] = static_cast<uint32_t>(v - wv0) % kRowsStageVecs;
            nhit += __popc(bal);
        };
        if (fpos)
            ws.run([&](const uint4 &x, bool valid, int v) { visit(std::true_type{}, x, valid, v); }, append_noted);
        else
            ws.run([&](const uint4 &x, bool valid, int v) { visit(std::false_type{}, x, valid, v); }, append_noted);
        // The notes are done with: the warp's part of the histogram is
        // cleared for the radix select (ordered by the barrier that follows
        // the stream).
#pragma unroll
        for (int q = 0; q < kRowsStageVecs / 128; ++q)
            reinterpret_cast<uint4 *>(note)[q * 32 + lane] = make_uint4(0u, 0u, 0u, 0u);
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
                if (hit) put(wcnt + __popc(bal & lt_mask), bits, e);
                wcnt += __popc(bal);
            }
        }
        if (Tr::nan_from(smx, umx) || tail_nan) sm.nan_seen = 1;
        // The stored entries > F and == F, and the largest key, from the list.
        uint32_t ngt = 0, neq = 0, kmx = 0u;
        const uint32_t stored = min(wcnt, static_cast<uint32_t>(kRowsCapWarp));
        __syncwarp();  // the list is visible to every lane
        for (uint32_t i0 = 0; i0 < stored; i0 += 32) {
            const uint32_t i = i0 + lane;
            if (i < stored) {
                const uint32_t key = Tr::key(cb[i]);
                ngt += key > fkey ? 1u : 0u;
                neq += key == fkey ? 1u : 0u;
                kmx = max(kmx, key);
            }
        }
        lost = __reduce_add_sync(0xFFFFFFFFu, lost);
        ngt = __reduce_add_sync(0xFFFFFFFFu, ngt);
        neq = __reduce_add_sync(0xFFFFFFFFu, neq);
        kmx = __reduce_max_sync(0xFFFFFFFFu, kmx);
        over = __any_sync(0xFFFFFFFFu, over);
        if (lane == 0) {
            sm.w_cnt[warp] = min(wcnt, static_cast<uint32_t>(kRowsCapWarp));
            sm.w_all[warp] = wcnt;
            sm.w_gtf[warp] = ngt;
            sm.w_eqs[warp] = neq;
            sm.w_eqf[warp] = neq + lost;
            sm.w_kmax[warp] = kmx;
            if (over) sm.overflow = 1;
        }
    }
    // One CTA per row: the rings are idle from here on, so the next row's
    // first stages and sample load while this row's candidates are selected.
    const bool has_next = cs == 1 && rnext >= 0;
    const RowGeom<DT> gn(a, has_next ? rnext : r, rank, warp);
    bool pre_next = false;
    if (has_next && gn.len > k) {
        gn.prefetch(sm, warp, lane, ph, a.status);
        pre_next = true;
    }
    __syncthreads();
    if (tid == 0) sm.cta_over = sm.overflow;
    cluster.sync();  // every candidate list of the cluster is final from here on

    // ---- the cluster's lists in column order ----
    const int nl = static_cast<int>(cs) * kRowsWarps;
    const uint32_t fu = fkey;
    if (warp == 0) {
        uint32_t cnt[2], ov = 0, gsum = 0, esum = 0, kmax = 0, asum = 0;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int L = lane + 32 * h;
            cnt[h] = 0;
            if (L < nl) {
                const RowsSmem *o = cluster.map_shared_rank(&sm, static_cast<unsigned>(L / kRowsWarps));
                const int w = L % kRowsWarps;
                cnt[h] = o->w_cnt[w];
                const uint32_t g = o->w_gtf[w], et = o->w_eqf[w];
                sm.l_cnt[L] = cnt[h];
                sm.l_gt[L] = g;
                sm.l_eq[L] = o->w_eqs[w];
                sm.l_eqt[L] = et;
                gsum += g;
                esum += et;
                asum += o->w_all[w];
                kmax = max(kmax, o->w_kmax[w]);
                ov |= o->cta_over;
            }
        }
        const uint32_t i0 = warp_incl_scan(cnt[0]);
        const uint32_t t0 = __shfl_sync(0xFFFFFFFFu, i0, 31);
        const uint32_t i1 = warp_incl_scan(cnt[1]) + t0;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int L = lane + 32 * h;
            if (L < nl) sm.l_off[L] = (h == 0 ? i0 : i1) - cnt[h];
        }
        ov = __reduce_or_sync(0xFFFFFFFFu, ov);
        gsum = __reduce_add_sync(0xFFFFFFFFu, gsum);
        esum = __reduce_add_sync(0xFFFFFFFFu, esum);
        kmax = __reduce_max_sync(0xFFFFFFFFu, kmax);
        asum = __reduce_add_sync(0xFFFFFFFFu, asum);
        if (lane == 31) sm.l_off[nl] = i1;
        if (lane == 0) {
            sm.g_over = ov;
            sm.g_gt = gsum;
            sm.g_eqt = esum;
            sm.g_kmax = kmax;
            sm.g_all = asum;
        }
    }
    __syncthreads();
    // At least topk elements >= F makes the k-th largest >= F, so the
    // lists hold it and everything above it.  Fewer than topk elements > F
    // make it equal to F: no selection is needed.
    const uint32_t total = sm.l_off[nl];
    bool exact_ok = !sm.g_over && sm.g_gt + sm.g_eqt >= static_cast<uint32_t>(k);
    uint32_t ustar = fu, above = sm.g_gt;
    if (exact_ok && sm.g_gt >= static_cast<uint32_t>(k)) {
        // u* > Fu: every CTA gathers all candidate keys of the cluster (the
        // rings are free now) and radix-selects those > Fu locally: the same
        // result in every CTA.
        exact_ok = total <= static_cast<uint32_t>(kRowsGather);
        if (exact_ok) {
            // cs > 1: the keys gathered into the rings; cs == 1: my own lists
            // in place (the rings hold the next row's first stages).
            uint32_t *gath = reinterpret_cast<uint32_t *>(sm.ring);
            auto for_keys = [&](auto &&fn) {  // fn(key, active) on every thread, uniformly
                if (cs > 1) {
                    for (uint32_t i0 = 0; i0 < total; i0 += kRowsThreads) {
                        const uint32_t i = i0 + tid;
                        fn(i < total ? gath[i] : 0u, i < total);
                    }
                } else {  // every warp its own list, four rounds read at a time
                    const uint32_t cnt = sm.w_cnt[warp];
                    for (uint32_t i0 = 0; i0 < cnt; i0 += 4 * 32) {
                        uint32_t kv[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const uint32_t i = i0 + 32 * u + lane;
                            kv[u] = i < cnt ? Tr::key(sm.cand_bits[warp][i]) : 0u;
                        }
#pragma unroll
                        for (int u = 0; u < 4; ++u) fn(kv[u], i0 + 32 * u + lane < cnt);
                    }
                }
            };
            if (cs > 1) {
                // Warp w gathers the lists (rr, w), rr < cs: entry f of its
                // share is entry f - pf[rr] of list rr, pf[rr] <= f < pf[rr + 1];
                // eight loads in flight per lane.
                uint32_t pf[kRowsMaxCluster + 1];
                pf[0] = 0;
#pragma unroll
                for (int rr = 0; rr < kRowsMaxCluster; ++rr)
                    pf[rr + 1] = pf[rr] + (rr < static_cast<int>(cs) ? sm.l_cnt[rr * kRowsWarps + warp] : 0u);
                const uint32_t mine = pf[kRowsMaxCluster];
                for (uint32_t f0 = 0; f0 < mine; f0 += 32 * 8) {
                    uint32_t v[8], dst[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const uint32_t f = f0 + 32 * u + lane;
                        v[u] = 0u;
                        dst[u] = 0xFFFFFFFFu;
                        if (f < mine) {
                            int rr = 0;
                            uint32_t base = 0;
#pragma unroll
                            for (int q = 1; q < kRowsMaxCluster; ++q)
                                if (f >= pf[q]) {
                                    rr = q;
                                    base = pf[q];
                                }
                            const uint32_t *cb =
                                cluster.map_shared_rank(&sm.cand_bits[warp][0], static_cast<unsigned>(rr));
                            v[u] = cb[f - base];
                            dst[u] = sm.l_off[rr * kRowsWarps + warp] + (f - base);
                        }
                    }
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        if (dst[u] != 0xFFFFFFFFu) gath[dst[u]] = Tr::key(v[u]);
                }
                __syncthreads();
            }
            const uint32_t kmx = sm.g_kmax;
            // Keys > Fu lie in [Fu + one step, kmx]: bits above the highest
            // one where those bounds differ are common to all of them, and
            // the 11-bit radix digits start below those.
            const int lo_bit = DT == FTK_BF16 ? 16 : 0;  // bf16 keys sit in the upper half
            const uint32_t kmn = fu + (DT == FTK_BF16 ? 0x10000u : 1u);
            const uint32_t diff = kmn ^ kmx;
            const int top = diff ? 31 - __clz(diff) : -1;
            uint32_t mask = top < 0 ? 0xFFFFFFFFu : (top == 31 ? 0u : ~((2u << top) - 1u));
            uint32_t prefix = kmx & mask, krem = static_cast<uint32_t>(k);
            above = 0;
            bool found = true;
            // The histogram is all zero on entry to each pass (cleared after
            // the stream, then after each pass: it is all zero again for the
            // next row's sample).
            for (int hi = top; hi >= lo_bit && found; hi -= 11) {
                const int shift = hi - 10 >= lo_bit ? hi - 10 : lo_bit;
                const uint32_t dmask = (2u << (hi - shift)) - 1u;
                if (hi != top) __syncthreads();  // the previous pass cleared it
                for_keys([&](uint32_t u, bool act) {
                    hist_add_plain(sm.hist, (u >> shift) & dmask, act && u > fu && (u & mask) == prefix);
                });
                __syncthreads();
                found = find_bin_top<kRowsBins>(sm, sm.hist, krem);
                for (int b = tid; b < kRowsBins; b += kRowsThreads) sm.hist[b] = 0;
                if (found) {
                    prefix |= sm.sel_bin << shift;
                    mask |= dmask << shift;
                    krem -= sm.sel_above;
                    above += sm.sel_above;
                }
            }
            ustar = prefix;
            exact_ok = found;
            if (exact_ok && cs == 1) {
                // Per list (my own): keys > u* and keys == u* (all stored:
                // u* > Fu).  The list is compacted in place, in column order,
                // to those entries: the ordered output walks only them.
                uint32_t *cb = sm.cand_bits[warp];
                int32_t *cc = sm.cand_col[warp];
                const uint32_t cnt = sm.w_cnt[warp];
                uint32_t g = 0, q = 0;
                for (uint32_t i0 = 0; i0 < cnt; i0 += 32) {
                    const uint32_t i = i0 + lane;
                    const uint32_t bits = i < cnt ? cb[i] : 0u;
                    const int32_t col = i < cnt ? cc[i] : 0;
                    const uint32_t u = Tr::key(bits);
                    const bool gt = i < cnt && u > ustar, eq = i < cnt && u == ustar;
                    const uint32_t kb = __ballot_sync(0xFFFFFFFFu, gt || eq);
                    // (entries kept so far <= i0: the writes reach only
                    // entries this round has read)
                    __syncwarp();
                    if (gt || eq) {
                        const uint32_t p = g + q + __popc(kb & lt_mask);
                        cb[p] = bits;
                        cc[p] = col;
                    }
                    g += __popc(__ballot_sync(0xFFFFFFFFu, gt));
                    q += __popc(__ballot_sync(0xFFFFFFFFu, eq));
                }
                if (lane == 0) {
                    sm.l_gt[warp] = g;
                    sm.l_eq[warp] = q;
                    sm.l_eqt[warp] = q;
                    sm.w_cnt[warp] = g + q;
                }
            } else if (exact_ok) {
                // Per list: keys > u* and keys == u* (all stored: u* > Fu).
                for (int l = warp; l < nl; l += kRowsWarps) {
                    const uint32_t cnt = sm.l_cnt[l], off = sm.l_off[l];
                    uint32_t g = 0, q = 0;
                    for (uint32_t i0 = 0; i0 < cnt; i0 += 32) {
                        const uint32_t i = i0 + lane;
                        const uint32_t u = i >= cnt ? 0u : cs > 1 ? gath[off + i] : Tr::key(sm.cand_bits[l][i]);
                        g += __popc(__ballot_sync(0xFFFFFFFFu, i < cnt && u > ustar));
                        q += __popc(__ballot_sync(0xFFFFFFFFu, i < cnt && u == ustar));
                    }
                    if (lane == 0) {
                        sm.l_gt[l] = g;
                        sm.l_eq[l] = q;
                        sm.l_eqt[l] = q;
                    }
                }
            }
        }
        __syncthreads();
    }
    if (exact_ok) {
        // In column order, each list's share of the ties at u* and its first
        // output slot.
        if (warp == 0) {
            const uint32_t need = static_cast<uint32_t>(k) - above;  // ties at u* to take, >= 1
            uint32_t eqt[2], sel[2], take[2];
            bool shrt = false;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int L = lane + 32 * h;
                eqt[h] = L < nl ? sm.l_eqt[L] : 0u;
            }
            const uint32_t e0 = warp_incl_scan(eqt[0]);
            const uint32_t et = __shfl_sync(0xFFFFFFFFu, e0, 31);
            const uint32_t e1 = warp_incl_scan(eqt[1]) + et;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int L = lane + 32 * h;
                const uint32_t eb = (h == 0 ? e0 : e1) - eqt[h];  // ties before list L
                take[h] = eb >= need ? 0u : min(eqt[h], need - eb);
                sel[h] = 0;
                if (L < nl) {
                    shrt |= take[h] > sm.l_eq[L];  // needs ties it did not store
                    sel[h] = sm.l_gt[L] + take[h];
                }
            }
            const uint32_t s0 = warp_incl_scan(sel[0]);
            const uint32_t st = __shfl_sync(0xFFFFFFFFu, s0, 31);
            const uint32_t s1 = warp_incl_scan(sel[1]) + st;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int L = lane + 32 * h;
                if (L < nl) {
                    sm.l_take[L] = take[h];
                    sm.l_selb[L] = (h == 0 ? s0 : s1) - sel[h];
                }
            }
            shrt = __any_sync(0xFFFFFFFFu, shrt);
            if (lane == 0) sm.short_eq = shrt ? 1u : 0u;
        }
        __syncthreads();
        exact_ok = sm.short_eq == 0;
    }
    // exact_ok is uniform over the cluster: every CTA decided it from the
    // same published lists.
    if (!exact_ok) {
        if (pre_next) {  // the fallback streams through the rings again
            const WarpStream wn{sm, gn.src(), gn.wv0, gn.wv1 - gn.wv0,
                                (gn.wv1 - gn.wv0 + kRowsStageVecs - 1) / kRowsStageVecs, warp, lane, ph, a.status};
            wn.drain();
            asm volatile("cp.async.wait_all;" ::: "memory");
            pre_next = false;
        }
        __syncthreads();
        // At least topk elements >= F: the k-th largest is >= F, and the
        // fallback's passes look at nothing below it.
        const uint32_t lo = sm.g_all >= static_cast<uint32_t>(k) ? fkey : 0u;
        rows_fallback<DT, IT>(a, sm, cluster, cs, rank, row, c0, n, base_index, oidx, oval, ph, lo);
    } else {
        __syncthreads();
        cluster_arrive();  // no more reads of other CTAs' shared memory
        // ---- ordered output of my lists ----
        const int L = static_cast<int>(rank) * kRowsWarps + warp;
        const uint32_t cnt = sm.w_cnt[warp], take = sm.l_take[L];
        uint32_t pos = sm.l_selb[L], eq_rank = 0;
        for (uint32_t i0 = 0; i0 < cnt; i0 += 4 * 32) {
            // four rounds of the list's entries read first (loads overlap)
            uint32_t bits[4];
            int col[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const uint32_t i = i0 + 32 * u + lane;
                bits[u] = i < cnt ? sm.cand_bits[warp][i] : 0u;
                col[u] = i < cnt ? sm.cand_col[warp][i] : 0;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const uint32_t i = i0 + 32 * u + lane;
                const uint32_t key = Tr::key(bits[u]);
                const bool gt = i < cnt && key > ustar;
                const bool eq = i < cnt && key == ustar;
                const uint32_t eq_bal = __ballot_sync(0xFFFFFFFFu, eq);
                const bool sel = gt || (eq && eq_rank + __popc(eq_bal & lt_mask) < take);
                const uint32_t sel_bal = __ballot_sync(0xFFFFFFFFu, sel);
                if (sel) {
                    const uint32_t p = pos + __popc(sel_bal & lt_mask);
                    if (p < static_cast<uint32_t>(k)) {
                        oidx[p] = static_cast<IT>(static_cast<int32_t>(base_index + c0 + col[u]));
                        if (oval) oval[p] = static_cast<elem>(bits[u]);
                    } else {
                        set_status(a.status, FTK_STATUS_INTERNAL);
                    }
                }
                pos += __popc(sel_bal);
                eq_rank += __popc(eq_bal);
            }
        }
    }
    if (tid == 0 && sm.nan_seen) set_status(a.status, FTK_STATUS_NAN);
    fence_proxy_async();  // generic writes of the rings precede later bulk copies into them
    __syncwarp();
    cluster_wait();  // keep my shared memory alive until every CTA is done with it
    pre = pre_next;
}

// One cluster per row.  LOOP: clusters stride over the rows (the count may
// be on the device), so a grid sized for the SMs serves any row count;
// otherwise the grid holds one cluster per row.  IT: the output index type
// (int32_t or int64_t).
template <int DT, bool LOOP, typename IT>
__global__ void __launch_bounds__(kRowsThreads, 2) rows_topk_kernel(const RowsArgs a)
{
    griddep_wait();  // the previous kernel on the stream is complete
    griddep_launch_next();
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
    if (static_cast<int64_t>(blockIdx.x / cs) >= nrows) return;  // whole clusters exit together
    if (threadIdx.x == 0) {
        for (int w = 0; w < kRowsWarps; ++w)
            for (int s = 0; s < kRowsStages; ++s) mbar_init(&sm.full[w][s], 1);
        fence_barrier_init();
    }
    // The histogram is all zero on entry to each row (each row leaves it so).
    for (int b = threadIdx.x; b < kRowsBins; b += kRowsThreads) sm.hist[b] = 0;
    __syncthreads();
    uint32_t ph = 0;   // parity each stage barrier of my warp waits for next
    bool pre = false;  // the row's first stages and sample were issued already
    // Row selection is uniform over the cluster: its CTAs walk the same rows.
    if constexpr (!LOOP) {
        rows_topk_row<DT, IT>(a, sm, cluster, cs, rank, blockIdx.x / cs, ph, pre, -1);
    } else {
        const int64_t step = gridDim.x / cs;
        for (int64_t r = blockIdx.x / cs; r < nrows; r += step) {
            rows_topk_row<DT, IT>(a, sm, cluster, cs, rank, r, ph, pre, r + step < nrows ? r + step : -1);
            __syncthreads();  // shared memory is free for the next row
        }
    }
}

}  // namespace ftk
