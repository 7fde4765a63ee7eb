// ftk_select.cu -- exact fused indexer top-k (ftk_select) and the dense
// score dump (ftk_score_dense).
//
// Per call, all stream-ordered, no host synchronisation:
//   plan       one CTA: zeroes the per-call state, checks every window and
//              lays out the work items of the sample and scan passes;
//   sample     score_kernel<SAMPLE>: each query tile scores a strided sample
//              of its windows (stride a power of two, so the sample of each
//              row is a strided sample of the row's own window -- FlashTopK
//              README, "Highlights": CP-compatible per-row thresholds);
//   threshold  per row: tau = the r-th largest sampled score, r chosen so
//              that about oversample * topk keys pass; tau = -inf when the
//              whole window fits in the candidate buffer;
//   prune      (unless switched off) the score bound of every 128-key block:
//              box of the keys, a sampled estimate of the skippable
//              fraction, and, when it pays, the skip bitmap of (row tile,
//              block) pairs that cannot hold a candidate (ftk_prune.cuh);
//   scan       score_kernel<COLLECT>: fused scoring of every key tile not
//              skipped, keeping I >= tau;
//   refine     per row: exact radix select of the topk candidates with the
//              (score desc, index asc) order, written in ascending index
//              order; rows whose candidates overflowed or fell short of
//              min(topk, L) are listed for recovery instead (triage);
//   recovery   score_kernel<DUMP> rescores the listed rows' whole windows
//              into scratch rows with the same arithmetic, and the row top-k
//              kernel selects from them (FlashTopK README, "Highlights":
//              rows the sampled threshold misses are rescored on the GPU).
#include <cudaTypedefs.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>

#include "ftk_host.h"
#include "ftk_prune.cuh"
#include "ftk_rows.cuh"
#include "ftk_score.cuh"

namespace ftk {

constexpr int kPlanThreads = 1024;
constexpr int kSelThreads = 256;
constexpr int kBitmapWords = 2048;   // 65536-key segments for the ordered output
constexpr int kMaxRowTile = 16;      // largest row_tile_of(dtype)

// Device copy of ftk_info plus counters (same layout for the leading part).
struct DevInfo {
    ftk_info info;
    uint32_t est_total, est_pruned;  // sampled (tile, block) pairs of the prune estimate
    int32_t work_next;               // the scan's shared work-item counter
};

// ---------------------------------------------------------------------------
// plan
// ---------------------------------------------------------------------------

struct PlanArgs {
    int64_t T, S;
    const int32_t *ks, *ke;
    int32_t ntiles;
    int32_t rt;               // rows per tile
    int32_t sample_keys;
    int32_t chunk_keys;       // keys per scan work item
    int32_t sample_chunk;     // samples per sample-pass work item
    // sample pass
    int32_t *s_lo, *s_hi, *s_lg, *s_start;
    // scan pass
    int32_t *c_lo, *c_hi, *c_start;
    int32_t *cnt;
    int32_t *bad_count;
    DevInfo *info;
    int64_t launches;
    // dense calls: every row with a valid window goes to rows_out (the
    // dense pass's row list, count in *bad_count); the others are padded
    int32_t dense;
    int32_t topk;
    int32_t *rows_out;
    int32_t *out_idx;
    float *out_val;
};

__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t *sh, uint32_t &total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    uint32_t inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t u = __shfl_up_sync(0xFFFFFFFFu, inc, o);
        if (lane >= o) inc += u;
    }
    if (lane == 31) sh[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        const uint32_t x = lane < nw ? sh[lane] : 0;
        uint32_t y = x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t u = __shfl_up_sync(0xFFFFFFFFu, y, o);
            if (lane >= o) y += u;
        }
        if (lane < nw) sh[32 + lane] = y - x;
        if (lane == 31) sh[64] = y;
    }
    __syncthreads();
    const uint32_t r = sh[32 + warp] + inc - v;
    total = sh[64];
    __syncthreads();
    return r;
}

__global__ void __launch_bounds__(kPlanThreads) plan_kernel(const PlanArgs p)
{
    griddep_wait();  // the previous kernel on the stream is complete
    griddep_launch_next();
    __shared__ uint32_t sh[96];
    const int tid = threadIdx.x;
    bool bad = false;
#pragma unroll 4
    for (int64_t t = tid; t < p.T; t += blockDim.x) {
        p.cnt[t] = 0;
        bad |= !window_ok(p.ks[t], p.ke[t], p.S);
    }
    if (tid == 0) {
        *p.bad_count = 0;
        memset(&p.info->info, 0, sizeof(ftk_info));
        p.info->info.rows = p.T;
        p.info->info.kernel_launches = p.launches;
        p.info->est_total = 0;
        p.info->est_pruned = 0;
        p.info->work_next = 0;
    }
    __syncthreads();
    if (bad) atomicOr(&p.info->info.status, FTK_STATUS_BAD_WINDOW);
    if (p.dense) {
        // The row list of the dense pass (valid windows, in row order); every
        // key of a window counts as a candidate.
        uint32_t carry = 0;
        unsigned long long ltot = 0, lmax = 0;
        for (int64_t base = 0; base < p.T; base += blockDim.x) {
            const int64_t t = base + tid;
            bool ok = false;
            if (t < p.T) {
                const int64_t a = p.ks[t], b = p.ke[t];
                ok = window_ok(a, b, p.S);
                if (ok) {
                    ltot += static_cast<unsigned long long>(b - a);
                    lmax = max(lmax, static_cast<unsigned long long>(b - a));
                }
            }
            uint32_t tot;
            const uint32_t e = block_excl_scan(ok ? 1u : 0u, sh, tot);
            if (ok) p.rows_out[carry + e] = static_cast<int32_t>(t);
            carry += tot;
        }
        if (ltot) atomicAdd(reinterpret_cast<unsigned long long *>(&p.info->info.candidates_total), ltot);
        if (lmax) atomicMax(reinterpret_cast<unsigned long long *>(&p.info->info.candidates_max), lmax);
        if (tid == 0) *p.bad_count = static_cast<int32_t>(carry);
        // rows with an invalid window: all (-1, -inf)
        if (__syncthreads_or(bad ? 1 : 0)) {
            for (int64_t t = 0; t < p.T; ++t) {
                if (window_ok(p.ks[t], p.ke[t], p.S)) continue;
                for (int j = tid; j < p.topk; j += blockDim.x) {
                    p.out_idx[t * p.topk + j] = -1;
                    if (p.out_val) p.out_val[t * p.topk + j] = -INFINITY;
                }
            }
        }
        return;
    }
    unsigned long long nblocks = 0;  // (row tile, key block) pairs of the scan
    uint32_t carry_s = 0, carry_c = 0;
    for (int32_t base = 0; base < p.ntiles; base += blockDim.x) {
        const int32_t tile = base + tid;
        uint32_t ns = 0, nc = 0;
        if (tile < p.ntiles) {
            // The tile's windows: every load issued before any is used.
            int32_t wa[kMaxRowTile], wb[kMaxRowTile];
#pragma unroll
            for (int j = 0; j < kMaxRowTile; ++j) {
                const int64_t t = static_cast<int64_t>(tile) * p.rt + j;
                const bool in = j < p.rt && t < p.T;
                wa[j] = in ? p.ks[t] : 0;
                wb[j] = in ? p.ke[t] : 0;
            }
            int64_t lo = INT64_MAX, hi = -1;
#pragma unroll
            for (int j = 0; j < kMaxRowTile; ++j) {
                const int64_t a = wa[j], b = wb[j];
                if (!window_ok(a, b, p.S) || a == b) continue;  // (absent rows: 0 == 0)
                lo = min(lo, a);
                hi = max(hi, b);
            }
            int32_t slo = 0, shi = 0, slg = 0, clo = 0, chi = 0;
            if (hi >= 0) {
                const int64_t L = hi - lo;
                const int64_t want = (L + p.sample_keys - 1) / p.sample_keys;  // >= 1
                int lg = 0;
                while ((int64_t(1) << lg) < want) ++lg;
                const int64_t j0 = (lo + (int64_t(1) << lg) - 1) >> lg;
                const int64_t j1 = (hi + (int64_t(1) << lg) - 1) >> lg;
                slo = static_cast<int32_t>(j0);
                shi = static_cast<int32_t>(j1);
                slg = lg;
                ns = j1 > j0 ? static_cast<uint32_t>((j1 - j0 + p.sample_chunk - 1) / p.sample_chunk) : 0u;
                const int64_t lo_al = lo & ~static_cast<int64_t>(kKeyTile - 1);
                clo = static_cast<int32_t>(lo_al);
                chi = static_cast<int32_t>(hi);
                nc = static_cast<uint32_t>((hi - lo_al + p.chunk_keys - 1) / p.chunk_keys);
                nblocks += static_cast<unsigned long long>((hi - lo_al + kKeyTile - 1) / kKeyTile);
            }
            p.s_lo[tile] = slo;
            p.s_hi[tile] = shi;
            p.s_lg[tile] = slg;
            p.c_lo[tile] = clo;
            p.c_hi[tile] = chi;
        }
        uint32_t tot_s, tot_c;
        const uint32_t es = block_excl_scan(ns, sh, tot_s);
        const uint32_t ec = block_excl_scan(nc, sh, tot_c);
        if (tile < p.ntiles) {
            p.s_start[tile] = static_cast<int32_t>(carry_s + es);
            p.c_start[tile] = static_cast<int32_t>(carry_c + ec);
        }
        carry_s += tot_s;
        carry_c += tot_c;
    }
    if (tid == 0) {
        p.s_start[p.ntiles] = static_cast<int32_t>(carry_s);
        p.c_start[p.ntiles] = static_cast<int32_t>(carry_c);
    }
    if (nblocks) atomicAdd(reinterpret_cast<unsigned long long *>(&p.info->info.blocks_total), nblocks);
}

// ---------------------------------------------------------------------------
// block-level radix select on 32-bit keys
// ---------------------------------------------------------------------------

struct SelShared {
    uint32_t hist[256];
    uint32_t bin, above, bin_count;
    uint32_t red[96];
};

// The k-th largest (1 <= k <= count of keys) of key(i), i < n, where key
// is any functor.  *gt receives how many keys are strictly larger and, if
// given, *eq how many are equal to it (the last digit's bin count).
// kmin / kmax, if given, bound every key: the bits above the highest bit
// where they differ are common to all keys, and the radix passes (8-bit
// digits) start below them.  Block-wide; every thread of the block calls it.
template <class KeyFn>
__device__ uint32_t block_kth_largest(int n, uint32_t k, KeyFn key, SelShared &ss, uint32_t *gt,
                                      uint32_t kmin = 0u, uint32_t kmax = 0xFFFFFFFFu,
                                      uint32_t *eq = nullptr)
{
    const uint32_t diff = kmin ^ kmax;
    const int top = diff ? 31 - __clz(diff) : -1;  // highest bit where keys may differ
    uint32_t mask = top < 0 ? 0xFFFFFFFFu : (top == 31 ? 0u : ~((2u << top) - 1u));
    uint32_t prefix = kmax & mask, above_total = 0;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int hi = top; hi >= 0; hi -= 8) {
        const int shift = hi >= 7 ? hi - 7 : 0;
        const uint32_t dmask = (2u << (hi - shift)) - 1u;  // digit of hi - shift + 1 <= 8 bits
        for (int b = tid; b < 256; b += blockDim.x) ss.hist[b] = 0;
        __syncthreads();
        for (int i = tid; i < n; i += blockDim.x) {
            const uint32_t u = key(i);
            if ((u & mask) == prefix) atomicAdd(&ss.hist[(u >> shift) & dmask], 1u);
        }
        __syncthreads();
        if (warp == 0) {
            // lane l owns bins 255-8l .. 248-8l (highest first)
            uint32_t c[8], sum = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                c[i] = ss.hist[255 - 8 * lane - i];
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
                        ss.bin = 255 - 8 * lane - i;
                        ss.above = above;
                        ss.bin_count = c[i];
                        break;
                    }
                    above += c[i];
                }
            }
        }
        __syncthreads();
        const uint32_t bin = ss.bin;
        prefix |= bin << shift;
        mask |= dmask << shift;
        k -= ss.above;
        above_total += ss.above;
        // The last pass has digit shift 0: its bin holds exactly the keys
        // equal to the result.
        if (eq) *eq = ss.bin_count;
        __syncthreads();
    }
    *gt = above_total;
    if (eq && top < 0) *eq = static_cast<uint32_t>(n);  // every key is kmax
    return prefix;
}

// ---------------------------------------------------------------------------
// threshold
// ---------------------------------------------------------------------------

struct ThreshArgs {
    int64_t T, S;
    const int32_t *ks, *ke;
    const int32_t *s_lo, *s_hi, *s_lg;
    const float *samp;
    int64_t sld;
    float *tau;
    int32_t cap;
    int32_t topk;
    int32_t rt;
    float oversample;
};

__global__ void __launch_bounds__(kSelThreads) threshold_kernel(const ThreshArgs p)
{
    griddep_wait();  // the previous kernel on the stream is complete
    griddep_launch_next();
    extern __shared__ uint32_t tkeys[];
    __shared__ SelShared ss;
    const int64_t t = blockIdx.x;
    const int64_t a = p.ks[t], b = p.ke[t];
    const int64_t L = b - a;
    if (!window_ok(a, b, p.S) || L <= p.cap) {
        if (threadIdx.x == 0) p.tau[t] = -INFINITY;
        return;
    }
    const int tile = static_cast<int>(t / p.rt);
    const int lg = p.s_lg[tile];
    const int64_t st = int64_t(1) << lg;
    const int J = p.s_hi[tile] - p.s_lo[tile];
    const int64_t mt = ((b + st - 1) >> lg) - ((a + st - 1) >> lg);  // samples in my window
    int64_t r = static_cast<int64_t>(ceil(static_cast<double>(p.oversample) * p.topk *
                                          static_cast<double>(mt) / static_cast<double>(L)));
    if (r < 1) r = 1;
    if (mt <= 0 || r > mt) {
        if (threadIdx.x == 0) p.tau[t] = -INFINITY;
        return;
    }
    const float *row = p.samp + t * p.sld;
    // Eight loads in flight per thread, then the conversions.
    for (int i0 = 0; i0 < J; i0 += 8 * kSelThreads) {
        uint32_t v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int i = i0 + j * kSelThreads + threadIdx.x;
            v[j] = i < J ? __float_as_uint(__ldg(row + i)) : 0u;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int i = i0 + j * kSelThreads + threadIdx.x;
            if (i < J) tkeys[i] = f32_key(v[j]);
        }
    }
    __syncthreads();
    uint32_t gt;
    const uint32_t u = block_kth_largest(J, static_cast<uint32_t>(r), [&](int i) { return tkeys[i]; }, ss, &gt);
    if (threadIdx.x == 0) p.tau[t] = __uint_as_float(f32_from_key(u));
}

// ---------------------------------------------------------------------------
// refine + triage
// ---------------------------------------------------------------------------

struct RefineArgs {
    int64_t T, S;
    const int32_t *ks, *ke;
    const int32_t *cnt;
    const float *cand_val;
    const int32_t *cand_idx;
    int32_t cap;
    int32_t topk;
    int32_t *out_idx;
    float *out_val;
    int32_t *bad_rows;
    int32_t *bad_count;
    DevInfo *info;
};

__device__ __forceinline__ void pad_row(int32_t *oi, float *ov, int from, int k)
{
    for (int j = from + threadIdx.x; j < k; j += blockDim.x) {
        oi[j] = -1;
        if (ov) ov[j] = -INFINITY;
    }
}

// Shared memory is kept small (keys only; the candidates' key indices are
// re-read from global memory, eight loads in flight per thread, where the
// bitmap passes need them) so that several rows' CTAs share an SM: the
// kernel is latency-bound per row.
__global__ void __launch_bounds__(kSelThreads, 6) refine_kernel(const RefineArgs p)
{
    griddep_wait();  // the previous kernel on the stream is complete
    griddep_launch_next();
    extern __shared__ __align__(16) uint32_t rsm[];
    __shared__ SelShared ss;
    __shared__ uint32_t bitmap[kBitmapWords];
    __shared__ uint16_t wpre[kBitmapWords];  // selected keys before each word (<= capacity)
    __shared__ int nan_seen;
    const int64_t t = blockIdx.x;
    const int k = p.topk;
    int32_t *oi = p.out_idx + t * k;
    float *ov = p.out_val ? p.out_val + t * k : nullptr;
    const int64_t a = p.ks[t], b = p.ke[t];
    if (!window_ok(a, b, p.S)) {
        pad_row(oi, ov, 0, k);
        return;
    }
    const int64_t L = b - a;
    const int32_t c = p.cnt[t];
    const int64_t need_min = L < k ? L : k;
    if (c > p.cap || c < need_min) {
        if (threadIdx.x == 0) {
            const int pos = atomicAdd(p.bad_count, 1);
            p.bad_rows[pos] = static_cast<int32_t>(t);
            atomicAdd(reinterpret_cast<unsigned long long *>(
                          c > p.cap ? &p.info->info.rows_overflow : &p.info->info.rows_underflow),
                      1ull);
        }
        return;
    }
    const int n = c;
    uint32_t *keys = rsm;
    if (threadIdx.x == 0) nan_seen = 0;
    __syncthreads();
    const float *cv = p.cand_val + t * p.cap;
    const int32_t *ci = p.cand_idx + t * p.cap;
    bool nan = false;
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;  // bounds of the keys, for the radix select
    // Eight value loads in flight per thread, then the stores.
    for (int i0 = 0; i0 < n; i0 += 8 * kSelThreads) {
        uint32_t v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int i = i0 + j * kSelThreads + threadIdx.x;
            v[j] = i < n ? __float_as_uint(__ldg(cv + i)) : 0u;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int i = i0 + j * kSelThreads + threadIdx.x;
            if (i < n) {
                nan |= f32_bits_isnan(v[j]);
                const uint32_t u = f32_key(v[j]);
                keys[i] = u;
                kmin = min(kmin, u);
                kmax = max(kmax, u);
            }
        }
    }
    if (nan) nan_seen = 1;
    if (threadIdx.x == 0) {
        atomicAdd(reinterpret_cast<unsigned long long *>(&p.info->info.candidates_total),
                  static_cast<unsigned long long>(n));
        atomicMax(reinterpret_cast<unsigned long long *>(&p.info->info.candidates_max),
                  static_cast<unsigned long long>(n));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        kmin = min(kmin, __shfl_xor_sync(0xFFFFFFFFu, kmin, o));
        kmax = max(kmax, __shfl_xor_sync(0xFFFFFFFFu, kmax, o));
    }
    if ((threadIdx.x & 31) == 0) {
        ss.red[threadIdx.x >> 5] = kmin;
        ss.red[32 + (threadIdx.x >> 5)] = kmax;
    }
    __syncthreads();
    if (nan_seen && threadIdx.x == 0) atomicOr(&p.info->info.status, FTK_STATUS_NAN);
    for (int w = 0; w < kSelThreads / 32; ++w) {
        kmin = min(kmin, ss.red[w]);
        kmax = max(kmax, ss.red[32 + w]);
    }
    __syncthreads();  // ss.red is free again

    // Threshold key u* and the tie cut idx*: selected = key > u*, or
    // key == u* and index <= idx* (the smallest indices among the ties).
    uint32_t ustar = 0, idxcut = 0xFFFFFFFFu;
    if (n > k) {
        uint32_t gt, eq;
        ustar = block_kth_largest(n, static_cast<uint32_t>(k), [&](int i) { return keys[i]; }, ss, &gt,
                                  kmin, kmax, &eq);
        const uint32_t need = static_cast<uint32_t>(k) - gt;
        if (eq > need) {
            // need-th smallest index among the ties = need-th largest of ~index.
            uint32_t g2;
            const uint32_t inv = block_kth_largest(
                n, need,
                [&](int i) { return keys[i] == ustar ? ~static_cast<uint32_t>(__ldg(ci + i)) : 0u; }, ss, &g2);
            idxcut = ~inv;
        }
    }
    auto selected = [&](int i, int32_t s) {
        const uint32_t u = keys[i];
        return u > ustar || (u == ustar && static_cast<uint32_t>(s) <= idxcut);
    };

    // Ordered output: rank of a selected key = number of selected keys with
    // a smaller index, from a bitmap over the window (65536-key segments).
    uint32_t out_base = 0;
    for (int64_t seg0 = a; seg0 < b; seg0 += 32 * kBitmapWords) {
        const int64_t seg1 = min(b, seg0 + 32 * kBitmapWords);
        const int words = static_cast<int>((seg1 - seg0 + 31) >> 5);
        for (int w = threadIdx.x; w < words; w += blockDim.x) bitmap[w] = 0;
        __syncthreads();
        for (int i0 = 0; i0 < n; i0 += 8 * kSelThreads) {
            int32_t x[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int i = i0 + j * kSelThreads + threadIdx.x;
                x[j] = i < n ? __ldg(ci + i) : -1;
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int i = i0 + j * kSelThreads + threadIdx.x;
                const int64_t s = x[j];
                if (i < n && s >= seg0 && s < seg1 && selected(i, x[j])) {
                    const uint32_t off = static_cast<uint32_t>(s - seg0);
                    atomicOr(&bitmap[off >> 5], 1u << (off & 31u));
                }
            }
        }
        __syncthreads();
        constexpr int per = kBitmapWords / kSelThreads;
        uint32_t cnt = 0;
        const int w0 = threadIdx.x * per;
#pragma unroll
        for (int i = 0; i < per; ++i) cnt += w0 + i < words ? __popc(bitmap[w0 + i]) : 0u;
        uint32_t total;
        uint32_t run = block_excl_scan(cnt, ss.red, total);
#pragma unroll
        for (int i = 0; i < per; ++i) {
            if (w0 + i < words) {
                wpre[w0 + i] = static_cast<uint16_t>(run);
                run += __popc(bitmap[w0 + i]);
            }
        }
        __syncthreads();
        for (int i0 = 0; i0 < n; i0 += 8 * kSelThreads) {
            int32_t x[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int i = i0 + j * kSelThreads + threadIdx.x;
                x[j] = i < n ? __ldg(ci + i) : -1;
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int i = i0 + j * kSelThreads + threadIdx.x;
                const int64_t s = x[j];
                if (i < n && s >= seg0 && s < seg1 && selected(i, x[j])) {
                    const uint32_t off = static_cast<uint32_t>(s - seg0);
                    const uint32_t w = off >> 5;
                    const uint32_t rank =
                        out_base + wpre[w] + __popc(bitmap[w] & ((1u << (off & 31u)) - 1u));
                    if (rank < static_cast<uint32_t>(k)) {
                        oi[rank] = static_cast<int32_t>(s);
                        if (ov) ov[rank] = __uint_as_float(f32_from_key(keys[i]));
                    } else {
                        atomicOr(&p.info->info.status, FTK_STATUS_INTERNAL);
                    }
                }
            }
        }
        out_base += total;
        __syncthreads();
    }
    pad_row(oi, ov, static_cast<int>(out_base), k);
}

// ---------------------------------------------------------------------------
// host helpers
// ---------------------------------------------------------------------------

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    // Looked up once; a failed lookup is retried on the next call.
    static std::atomic<PFN_cuTensorMapEncodeTiled_v12000> cached{nullptr};
    PFN_cuTensorMapEncodeTiled_v12000 fn = cached.load(std::memory_order_acquire);
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess) {
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
            cached.store(fn, std::memory_order_release);
        }
    }
    return fn;
}

// 2-D map over rows of 128 elements (row stride `stride_bytes`), box of
// (128 bytes, box_rows) with the 128-byte swizzle; out-of-range rows read 0.
static bool make_map(CUtensorMap *m, int dtype, const void *base, uint64_t rows,
                     uint64_t stride_bytes, uint32_t box_rows)
{
    auto fn = encode_fn();
    if (!fn) return false;
    const bool f8 = dtype == FTK_F8E4M3;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(kDim), rows};
    cuuint64_t strides[1] = {stride_bytes};
    cuuint32_t box[2] = {f8 ? 128u : 64u, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, f8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                    const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

static int num_sms()
{
    int dev = 0, n = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

enum PruneMode { PRUNE_AUTO = 0, PRUNE_ON = 1, PRUNE_OFF = 2 };
constexpr int64_t kAutoPruneRows = 128;
// Calls of at most this many query rows (and at most 2^25 (row, key) pairs,
// one recovery pass) take the dense path: the threshold machinery's fixed
// stages cost more than scoring and selecting every key of a few rows.
constexpr int64_t kDenseRows = 128;
constexpr int64_t kDensePairs = int64_t(1) << 25;

struct SelectCfg {
    int heads;      // 32 or 64
    int m;          // sample keys
    float beta;
    int cap;
    PruneMode prune;
    int rec_rows;
    int64_t scratch_floats;  // recovery scratch reserved, >= rec_rows * scratch row stride
    bool dense;              // score every key and select with the row top-k
};

// Row stride of the recovery scratch (floats): S rounded up to 8.
static int64_t scratch_ld_of(int64_t S) { return (S + 7) / 8 * 8; }

static SelectCfg resolve_cfg(int64_t T, int64_t S, int topk, const ftk_config *c)
{
    SelectCfg r;
    r.heads = c && c->heads == 64 ? 64 : 32;
    r.m = c && c->sample_keys > 0 ? c->sample_keys : 4096;
    r.beta = c && c->oversample > 0.f ? c->oversample : 1.5f;
    // Default capacity 2.5 * topk: the candidate count of a row is about
    // 1.5 * topk with a spread of a few percent, and a row past the
    // capacity costs a dense recovery pass.
    r.cap = c && c->capacity > 0 ? c->capacity : topk * 5 / 2;
    if (r.cap > 2 * FTK_MAX_TOPK) r.cap = 2 * FTK_MAX_TOPK;
    const int pr = c ? c->prune : 0;
    r.prune = pr == 0 ? PRUNE_AUTO : pr > 0 ? PRUNE_ON : PRUNE_OFF;
    // The automatic decision needs its sampled estimate, and the bound's
    // fixed cost (the box of every key block) pays only over enough query
    // rows: calls of fewer than kAutoPruneRows rows scan densely unless
    // pruning is asked for.
    if (r.prune == PRUNE_AUTO && T < kAutoPruneRows) r.prune = PRUNE_OFF;
    // Strides are powers of two up to 2^(kNumStrideMaps - 1).
    const int64_t min_m = (S + (int64_t(1) << (kNumStrideMaps - 1)) - 1) >> (kNumStrideMaps - 1);
    if (r.m < min_m) r.m = static_cast<int>(min_m);
    if (r.m < 32) r.m = 32;
    if (r.m > 32768) r.m = 32768;
    // Recovery scratch: rec_rows rows of ld floats.  The reservation is a
    // non-decreasing function of T and S (so a workspace planned for (T, S)
    // serves every call with smaller T and S), and rec_rows is what fits.
    const int64_t ld = scratch_ld_of(S);
    const int64_t tcap = (T + kMaxRowTile - 1) / kMaxRowTile * kMaxRowTile;
    int64_t budget;
    if (c && c->recovery_rows > 0) {
        budget = (static_cast<int64_t>(c->recovery_rows) + kMaxRowTile - 1) / kMaxRowTile * kMaxRowTile * ld;
    } else {
        // 2^27 floats (512 MB), or 64 rows when rows are longer than 2^21 keys
        budget = int64_t(1) << 27;
        if (budget < 64 * ld) budget = 64 * ld;
    }
    if (budget > tcap * ld) budget = tcap * ld;
    r.scratch_floats = budget;
    r.rec_rows = static_cast<int>(budget / ld / kMaxRowTile * kMaxRowTile);
    const int64_t dense_rows = !c || c->dense_rows == 0 ? kDenseRows : c->dense_rows < 0 ? 0 : c->dense_rows;
    r.dense = T <= dense_rows && T * S <= kDensePairs && T <= r.rec_rows;
    return r;
}

struct SelectWs {
    DevInfo *info;
    int32_t *s_lo, *s_hi, *s_lg, *s_start, *c_lo, *c_hi, *c_start;
    float *samp;
    int64_t sld;
    float *tau;
    int32_t *cnt;
    float *cand_val;
    int32_t *cand_idx;
    int32_t *bad_rows;
    int32_t *bad_count;
    float *scratch;
    int64_t scratch_ld;
    float *box;       // [nblocks][2][128] score-bound box of each key block
    float *mb;        // [nblocks]
    uint32_t *prune_bits;  // [ntiles][nwords]
    int32_t nblocks, nwords;
};

static bool carve_select(Carver &cv, int64_t T, int64_t S, const SelectCfg &c, SelectWs &w)
{
    // Row tiles of the smallest row tile of either dtype (the size query
    // does not know the dtype).
    const int64_t min_rt = row_tile_of(FTK_BF16, c.heads) < row_tile_of(FTK_F8E4M3, c.heads)
                               ? row_tile_of(FTK_BF16, c.heads)
                               : row_tile_of(FTK_F8E4M3, c.heads);
    const int64_t ntiles = (T + min_rt - 1) / min_rt;
    w.info = cv.take<DevInfo>(1);
    w.s_lo = cv.take<int32_t>(ntiles);
    w.s_hi = cv.take<int32_t>(ntiles);
    w.s_lg = cv.take<int32_t>(ntiles);
    w.s_start = cv.take<int32_t>(ntiles + 1);
    w.c_lo = cv.take<int32_t>(ntiles);
    w.c_hi = cv.take<int32_t>(ntiles);
    w.c_start = cv.take<int32_t>(ntiles + 1);
    w.sld = (c.m + 3) / 4 * 4;
    w.samp = cv.take<float>(T * w.sld);
    w.tau = cv.take<float>(T);
    w.cnt = cv.take<int32_t>(T);
    w.cand_val = cv.take<float>(T * static_cast<int64_t>(c.cap));
    w.cand_idx = cv.take<int32_t>(T * static_cast<int64_t>(c.cap));
    w.bad_rows = cv.take<int32_t>(T);
    w.bad_count = cv.take<int32_t>(1);
    w.scratch_ld = scratch_ld_of(S);
    w.scratch = cv.take<float>(c.scratch_floats);
    w.nblocks = static_cast<int32_t>((S + kBlockKeys - 1) / kBlockKeys);
    w.nwords = (w.nblocks + kBoundWordBlocks - 1) / kBoundWordBlocks;
    if (c.prune != PRUNE_OFF) {
        w.box = cv.take<float>(static_cast<int64_t>(w.nblocks) * 2 * kDim);
        w.mb = cv.take<float>(w.nblocks);
        w.prune_bits = cv.take<uint32_t>(ntiles * w.nwords);
    } else {
        w.box = nullptr;
        w.mb = nullptr;
        w.prune_bits = nullptr;
    }
    return cv.ok;
}

template <int DT, int MODE, bool PR, bool H64>
static ftk_status launch_score(const ScoreArgs &a, const CUtensorMap &tq, const KvMaps &kvm,
                               int grid, cudaStream_t st)
{
    const int smem = ScoreSmemLayout<DT>::kBytes;
    auto kern = score_kernel<DT, MODE, PR, H64>;
    const ftk_status e = ensure_smem_limit(reinterpret_cast<const void *>(kern), smem);
    if (e != FTK_OK) return e;
    return launch_kernel(kern, dim3(grid), dim3(kScoreThreads), smem, st, 1, a, tq, kvm);
}

template <int MODE, bool PR = false>
static ftk_status launch_score_dt(int dtype, int heads, const ScoreArgs &a, const CUtensorMap &tq,
                                  const KvMaps &kvm, int grid, cudaStream_t st)
{
    if (heads == 64) {
        if (dtype == FTK_F8E4M3) return launch_score<FTK_F8E4M3, MODE, PR, true>(a, tq, kvm, grid, st);
        return launch_score<FTK_BF16, MODE, PR, true>(a, tq, kvm, grid, st);
    }
    if (dtype == FTK_F8E4M3) return launch_score<FTK_F8E4M3, MODE, PR, false>(a, tq, kvm, grid, st);
    return launch_score<FTK_BF16, MODE, PR, false>(a, tq, kvm, grid, st);
}

// q as rows of 128 elements (T * heads of them, boxes of 32 = one MMA row
// each), and kv at every sample stride.
static bool build_maps(int dtype, int heads, const void *q, const void *kv, int64_t T, int64_t S, int max_lg,
                       CUtensorMap *tq, KvMaps *kvm)
{
    const uint64_t esz = dtype == FTK_F8E4M3 ? 1 : 2;
    if (!make_map(tq, dtype, q, static_cast<uint64_t>(T) * heads, kDim * esz, kHeads)) return false;
    for (int i = 0; i < kNumStrideMaps; ++i) {
        if (i > max_lg) {
            kvm->m[i] = kvm->m[0];
            continue;
        }
        const uint64_t st = uint64_t(1) << i;
        const uint64_t rows = (static_cast<uint64_t>(S) + st - 1) / st;
        if (!make_map(&kvm->m[i], dtype, kv, rows, kDim * esz * st, kKeyTile)) return false;
    }
    return true;
}

static ftk_status check_select_args(int dtype, int heads, const void *q, const void *kv, const float *w,
                                    const int32_t *ks, const int32_t *ke, int64_t T, int64_t S,
                                    int topk, const int32_t *out_idx)
{
    if (dtype != FTK_F8E4M3 && dtype != FTK_BF16) return FTK_ERR_UNSUPPORTED;
    if (heads != 32 && heads != 64) return FTK_ERR_INVALID_ARG;
    if (!q || !kv || !w || !ks || !ke || !out_idx) return FTK_ERR_INVALID_ARG;
    if (T < 1 || S < 1 || T >= (int64_t(1) << 31) / heads || S >= (int64_t(1) << 31) - kChunkKeys)
        return FTK_ERR_INVALID_ARG;
    if (topk < 1 || topk > FTK_MAX_TOPK) return FTK_ERR_TOPK_RANGE;
    if (!aligned16(q) || !aligned16(kv) || !aligned16(w)) return FTK_ERR_ALIGNMENT;
    return FTK_OK;
}

ftk_status check_select_call(int dtype, const void *q, const void *kv, const float *w, const int32_t *ks,
                             const int32_t *ke, int64_t T, int64_t S, int topk, const int32_t *out_idx,
                             const ftk_config *config)
{
    if (config && (config->reserved ||
                   (config->heads != 0 && config->heads != 32 && config->heads != 64)))
        return FTK_ERR_INVALID_ARG;
    const int heads = config && config->heads == 64 ? 64 : 32;
    return check_select_args(dtype, heads, q, kv, w, ks, ke, T, S, topk, out_idx);
}

// The caller's event handles, copied (the caller's array need not outlive
// ftk_set_stage_events); g_stage_count == 0 means the hook is off.
thread_local void *g_stage_events[8];
thread_local int g_stage_count = 0;

static void stage_mark(int i, cudaStream_t s)
{
    if (i < g_stage_count && cudaEventRecord(static_cast<cudaEvent_t>(g_stage_events[i]), s) != cudaSuccess) {
        (void)cudaGetLastError();  // a bad event must not poison the launch checks
        g_stage_count = 0;
    }
}

}  // namespace ftk

using namespace ftk;

extern "C" ftk_status ftk_set_stage_events(void *const *events, int n)
{
    if (events == nullptr || n == 0) {
        g_stage_count = 0;
        return FTK_OK;
    }
    if (n < 7) return FTK_ERR_INVALID_ARG;
    const int used = n < 8 ? n : 8;
    for (int i = 0; i < used; ++i)
        if (events[i] == nullptr) return FTK_ERR_INVALID_ARG;
    for (int i = 0; i < used; ++i) g_stage_events[i] = events[i];
    g_stage_count = used;
    return FTK_OK;
}

extern "C" size_t ftk_select_workspace_size(int64_t T, int64_t S, int topk, const ftk_config *config)
{
    if (T < 1 || S < 1 || topk < 1 || topk > FTK_MAX_TOPK) return 0;
    if (config && config->heads != 0 && config->heads != 32 && config->heads != 64) return 0;
    const SelectCfg c = resolve_cfg(T, S, topk, config);
    Carver cv{nullptr, 0};
    SelectWs w;
    carve_select(cv, T, S, c, w);
    return cv.used;
}

extern "C" ftk_status ftk_read_info(const void *workspace, ftk_info *out, void *stream)
{
    if (!workspace || !out) return FTK_ERR_INVALID_ARG;
    cudaStream_t st = as_stream(stream);
    cudaError_t e = cudaMemcpyAsync(out, workspace, sizeof(ftk_info), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    return cuda_status(e);
}

extern "C" ftk_status ftk_select(ftk_dtype dtype, const void *q, const void *kv,
                                 const float *kv_scales, const float *weights, const int32_t *ks,
                                 const int32_t *ke, int64_t T, int64_t S, int topk,
                                 int32_t *out_idx, float *out_val, void *workspace,
                                 size_t workspace_bytes, const ftk_config *config, void *stream)
{
    ftk_status st = check_select_call(dtype, q, kv, weights, ks, ke, T, S, topk, out_idx, config);
    if (st != FTK_OK) return st;
    const int heads = config && config->heads == 64 ? 64 : 32;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return FTK_ERR_WORKSPACE;
    const SelectCfg c = resolve_cfg(T, S, topk, config);
    if (c.cap < topk) return FTK_ERR_INVALID_ARG;
    Carver cv{static_cast<uint8_t *>(workspace), workspace_bytes};
    SelectWs w;
    if (!carve_select(cv, T, S, c, w)) return FTK_ERR_WORKSPACE;
    st = check_device();
    if (st != FTK_OK) return st;
    cudaStream_t s = as_stream(stream);

    const int64_t want = (S + c.m - 1) / c.m;
    int max_lg = 0;
    while ((int64_t(1) << max_lg) < want) ++max_lg;
    if (max_lg >= kNumStrideMaps) return FTK_ERR_UNSUPPORTED;
    CUtensorMap tq;
    KvMaps kvm;
    if (!build_maps(dtype, heads, q, kv, T, S, max_lg, &tq, &kvm)) return FTK_ERR_CUDA;

    const int rt = row_tile_of(dtype, heads);
    const int32_t ntiles = static_cast<int32_t>((T + rt - 1) / rt);
    const int sms = num_sms();
    uint32_t *status = &w.info->info.status;

    // The dense pass over the listed rows [b0, b0 + nrows) of w.bad_rows
    // (count on the device): dense_scores writes every key's score of their
    // windows into the scratch, dense_select takes each row's top-k from
    // them (the row top-k kernel).
    auto dense_scores = [&](int64_t b0, int nrows) -> ftk_status {
        ScoreArgs da = {};
        da.T = T;
        da.S = S;
        da.kv_scales = kv_scales;
        da.weights = weights;
        da.ks = ks;
        da.ke = ke;
        da.rows = w.bad_rows + b0;
        da.nrows = nrows;
        da.count_dev = w.bad_count;
        da.count_off = static_cast<int32_t>(b0);
        da.out = w.scratch;
        da.ld = w.scratch_ld;
        da.status = status;
        return launch_score_dt<MODE_DUMP>(dtype, heads, da, tq, kvm, sms, s);
    };
    auto dense_select = [&](int64_t b0, int nrows, int rcluster, int rchunk) -> ftk_status {
        RowsArgs ra2 = {};
        ra2.x = w.scratch;
        ra2.ld = w.scratch_ld;
        ra2.cols = S;
        ra2.rows = nrows;
        ra2.nrows_dev = w.bad_count;
        ra2.nrows_off = static_cast<int32_t>(b0);
        ra2.row_map = w.bad_rows + b0;
        ra2.win_ks = ks;
        ra2.win_ke = ke;
        ra2.out_idx = out_idx;
        ra2.out_val = out_val;
        ra2.ldo = topk;
        ra2.idx_fill = -1;
        ra2.val_fill = 0xFF800000u;  // -inf
        ra2.k = topk;
        ra2.chunk = rchunk;
        ra2.status = status;
        return launch_rows_topk(FTK_F32, ra2, rcluster, s);
    };

    stage_mark(0, s);
    PlanArgs pa;
    pa.T = T;
    pa.S = S;
    pa.ks = ks;
    pa.ke = ke;
    pa.ntiles = ntiles;
    pa.rt = rt;
    pa.sample_keys = c.m;
    // Scan work items: up to kChunkTiles key tiles each, fewer when the call is
    // small (few query rows, decode-like) so that the items still cover
    // every SM about twice.
    {
        const int64_t pairs = static_cast<int64_t>(ntiles) * ((S + kKeyTile - 1) / kKeyTile);
        int64_t ct = (pairs + 2 * static_cast<int64_t>(sms) - 1) / (2 * static_cast<int64_t>(sms));
        ct = ct < kMinChunkTiles ? kMinChunkTiles : (ct > kChunkTiles ? kChunkTiles : ct);
        pa.chunk_keys = static_cast<int32_t>(ct * kKeyTile);
        // The sample pass has one item per row tile; with fewer row tiles
        // than SMs, its samples are split so the items cover the SMs twice.
        int64_t sc = int64_t(1) << 30;
        if (ntiles < sms) {
            const int64_t pieces = (2 * static_cast<int64_t>(sms) + ntiles - 1) / ntiles;
            sc = (c.m + pieces - 1) / pieces;
            sc = (sc + kKeyTile - 1) / kKeyTile * kKeyTile;
            if (sc < 4 * kKeyTile) sc = 4 * kKeyTile;
        }
        pa.sample_chunk = static_cast<int32_t>(sc);
    }
    pa.s_lo = w.s_lo;
    pa.s_hi = w.s_hi;
    pa.s_lg = w.s_lg;
    pa.s_start = w.s_start;
    pa.c_lo = w.c_lo;
    pa.c_hi = w.c_hi;
    pa.c_start = w.c_start;
    pa.cnt = w.cnt;
    pa.bad_count = w.bad_count;
    pa.info = w.info;
    pa.launches = 5 + 2 * ((T + c.rec_rows - 1) / c.rec_rows) + (c.prune == PRUNE_OFF ? 0 : c.prune == PRUNE_AUTO ? 4 : 2);
    pa.dense = c.dense ? 1 : 0;
    pa.topk = topk;
    pa.rows_out = w.bad_rows;
    pa.out_idx = out_idx;
    pa.out_val = out_val;
    if (c.dense) {
        // Few query rows: one dense pass over every row (plan, dump, row
        // top-k); the sample, threshold, scan and refine stages are skipped.
        pa.launches = 3;
        // (Stage marks: the dense scores stand in the scan's place, the row
        // top-k in the refine's; the skipped stages take no time.)
        if ((st = launch_kernel(plan_kernel, dim3(1), dim3(kPlanThreads), 0, s, 1, pa)) != FTK_OK) return st;
        for (int i : {1, 2, 3, 7}) stage_mark(i, s);
        int rcluster = 1, rchunk = 8;
        rows_plan(T, S, topk, &rcluster, &rchunk);
        if ((st = dense_scores(0, static_cast<int>(T))) != FTK_OK) return st;
        stage_mark(4, s);
        if ((st = dense_select(0, static_cast<int>(T), rcluster, rchunk)) != FTK_OK) return st;
        stage_mark(5, s);
        stage_mark(6, s);
        return FTK_OK;
    }
    if ((st = launch_kernel(plan_kernel, dim3(1), dim3(kPlanThreads), 0, s, 1, pa)) != FTK_OK) return st;
    stage_mark(1, s);

    ScoreArgs sa = {};
    sa.T = T;
    sa.S = S;
    sa.kv_scales = kv_scales;
    sa.weights = weights;
    sa.ks = ks;
    sa.ke = ke;
    sa.rows = nullptr;
    sa.nrows = T;
    sa.planned = 1;
    sa.chunk_keys = pa.sample_chunk;
    sa.ntiles = ntiles;
    sa.status = status;
    // sample pass
    sa.tile_lo = w.s_lo;
    sa.tile_hi = w.s_hi;
    sa.tile_lg = w.s_lg;
    sa.item_start = w.s_start;
    sa.out = w.samp;
    sa.ld = w.sld;
    st = launch_score_dt<MODE_SAMPLE>(dtype, heads, sa, tq, kvm, sms, s);  // CTAs without an item exit
    if (st != FTK_OK) return st;
    stage_mark(2, s);

    ThreshArgs ta;
    ta.T = T;
    ta.S = S;
    ta.ks = ks;
    ta.ke = ke;
    ta.s_lo = w.s_lo;
    ta.s_hi = w.s_hi;
    ta.s_lg = w.s_lg;
    ta.samp = w.samp;
    ta.sld = w.sld;
    ta.tau = w.tau;
    ta.cap = c.cap;
    ta.topk = topk;
    ta.rt = rt;
    ta.oversample = c.beta;
    {
        const size_t smem = static_cast<size_t>(w.sld) * 4;
        st = ensure_smem_limit(reinterpret_cast<const void *>(threshold_kernel), static_cast<int>(smem));
        if (st != FTK_OK) return st;
        st = launch_kernel(threshold_kernel, dim3(static_cast<unsigned>(T)), dim3(kSelThreads), smem, s, 1, ta);
        if (st != FTK_OK) return st;
    }
    stage_mark(3, s);

    if (c.prune != PRUNE_OFF) {
        BoxArgs xa;
        xa.kv = kv;
        xa.kv_scales = kv_scales;
        xa.S = S;
        xa.nblocks = w.nblocks;
        xa.box = w.box;
        xa.mb = w.mb;
        if ((st = launch_box(dtype, xa, s)) != FTK_OK) return st;
        BoundArgs ba = {};
        ba.q = q;
        ba.weights = weights;
        ba.ks = ks;
        ba.ke = ke;
        ba.T = T;
        ba.S = S;
        ba.rt = rt;
        ba.ntiles = ntiles;
        ba.nblocks = w.nblocks;
        ba.nwords = w.nwords;
        ba.box = w.box;
        ba.mb = w.mb;
        ba.tau = w.tau;
        ba.c_lo = w.c_lo;
        ba.c_hi = w.c_hi;
        ba.est_tiles = ntiles < kEstTiles ? ntiles : kEstTiles;
        ba.bits = w.prune_bits;
        ba.est_total = &w.info->est_total;
        ba.est_pruned = &w.info->est_pruned;
        ba.mode = c.prune == PRUNE_AUTO ? 0 : 1;
        ba.prune_enabled = &w.info->info.prune_enabled;
        ba.blocks_pruned = reinterpret_cast<unsigned long long *>(&w.info->info.blocks_pruned);
        if (c.prune == PRUNE_AUTO) {
            st = launch_bound(dtype, BOUND_EST, ba, ba.est_tiles * (kEstBlocks / kEstChunk), s, heads);
            if (st != FTK_OK) return st;
        }
        const int64_t items = static_cast<int64_t>(ntiles) * w.nwords;
        const int64_t cap = static_cast<int64_t>(sms) * 2;
        st = launch_bound(dtype, BOUND_FULL, ba, static_cast<int>(items < cap ? items : cap), s, heads);
        if (st != FTK_OK) return st;
    }
    stage_mark(7, s);

    // scan (dynamic schedule over the planned items)
    sa.chunk_keys = pa.chunk_keys;
    sa.work_next = &w.info->work_next;
    sa.tile_lo = w.c_lo;
    sa.tile_hi = w.c_hi;
    sa.tile_lg = nullptr;
    sa.item_start = w.c_start;
    sa.tau = w.tau;
    sa.cnt = w.cnt;
    sa.cand_val = w.cand_val;
    sa.cand_idx = w.cand_idx;
    sa.cap = c.cap;
    sa.out = nullptr;
    sa.prune_bits = w.prune_bits;
    sa.prune_words = w.nwords;
    sa.prune_on = &w.info->info.prune_enabled;
    // auto: both variants, the device-side decision picks one (the other
    // returns at once); always: the pruned one; off: the plain one
    if (c.prune != PRUNE_ON) {
        st = launch_score_dt<MODE_COLLECT, false>(dtype, heads, sa, tq, kvm, sms, s);
        if (st != FTK_OK) return st;
    }
    if (c.prune != PRUNE_OFF) {
        st = launch_score_dt<MODE_COLLECT, true>(dtype, heads, sa, tq, kvm, sms, s);
        if (st != FTK_OK) return st;
    }
    stage_mark(4, s);

    RefineArgs ra;
    ra.T = T;
    ra.S = S;
    ra.ks = ks;
    ra.ke = ke;
    ra.cnt = w.cnt;
    ra.cand_val = w.cand_val;
    ra.cand_idx = w.cand_idx;
    ra.cap = c.cap;
    ra.topk = topk;
    ra.out_idx = out_idx;
    ra.out_val = out_val;
    ra.bad_rows = w.bad_rows;
    ra.bad_count = w.bad_count;
    ra.info = w.info;
    {
        const size_t smem = static_cast<size_t>(c.cap) * 4;
        st = ensure_smem_limit(reinterpret_cast<const void *>(refine_kernel), static_cast<int>(smem));
        if (st != FTK_OK) return st;
        st = launch_kernel(refine_kernel, dim3(static_cast<unsigned>(T)), dim3(kSelThreads), smem, s, 1, ra);
        if (st != FTK_OK) return st;
    }
    stage_mark(5, s);

    // dense recovery of the listed rows, rec_rows at a time; the row count
    // is on the device and usually small, so plan the row top-k for few
    // rows (widest clusters) and let its clusters stride over the rest
    int rcluster = 1, rchunk = 8;
    rows_plan(c.rec_rows < 16 ? c.rec_rows : 16, S, topk, &rcluster, &rchunk);
    for (int64_t b0 = 0; b0 < T; b0 += c.rec_rows) {
        if ((st = dense_scores(b0, c.rec_rows)) != FTK_OK) return st;
        if ((st = dense_select(b0, c.rec_rows, rcluster, rchunk)) != FTK_OK) return st;
    }
    stage_mark(6, s);
    return FTK_OK;
}

extern "C" size_t ftk_score_dense_workspace_size(int64_t nrows)
{
    (void)nrows;
    return 256;
}

extern "C" ftk_status ftk_score_dense_heads(ftk_dtype dtype, int heads, const void *q, const void *kv,
                                            const float *kv_scales, const float *weights,
                                            const int32_t *ks, const int32_t *ke, int64_t T, int64_t S,
                                            const int32_t *rows, int64_t nrows, float *out, int64_t ld,
                                            void *workspace, size_t workspace_bytes, void *stream)
{
    ftk_status st = check_select_args(dtype, heads, q, kv, weights, ks, ke, T, S, 1, rows ? rows : ks);
    if (st != FTK_OK) return st;
    // ld >= S: every valid window (ke <= S) fits its row, whatever the
    // windows hold on the device
    if (!out || nrows < 1 || nrows > T * 64 || ld < S || (ld & 3)) return FTK_ERR_INVALID_ARG;
    if (!rows && nrows > T) return FTK_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < 256 || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return FTK_ERR_WORKSPACE;
    st = check_device();
    if (st != FTK_OK) return st;
    CUtensorMap tq;
    KvMaps kvm;
    if (!build_maps(dtype, heads, q, kv, T, S, 0, &tq, &kvm)) return FTK_ERR_CUDA;
    ScoreArgs da = {};
    da.T = T;
    da.S = S;
    da.kv_scales = kv_scales;
    da.weights = weights;
    da.ks = ks;
    da.ke = ke;
    da.rows = rows;
    da.nrows = nrows;
    da.out = out;
    da.ld = ld;
    da.status = static_cast<uint32_t *>(workspace);
    cudaStream_t s = as_stream(stream);
    cudaError_t e = cudaMemsetAsync(workspace, 0, 4, s);
    if (e != cudaSuccess) return cuda_status(e);
    return launch_score_dt<MODE_DUMP>(dtype, heads, da, tq, kvm, num_sms(), s);
}

extern "C" ftk_status ftk_score_dense(ftk_dtype dtype, const void *q, const void *kv,
                                      const float *kv_scales, const float *weights,
                                      const int32_t *ks, const int32_t *ke, int64_t T, int64_t S,
                                      const int32_t *rows, int64_t nrows, float *out, int64_t ld,
                                      void *workspace, size_t workspace_bytes, void *stream)
{
    return ftk_score_dense_heads(dtype, 32, q, kv, kv_scales, weights, ks, ke, T, S, rows, nrows, out, ld,
                                 workspace, workspace_bytes, stream);
}
