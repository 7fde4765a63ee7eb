// ftk_rows.cu -- host side of the row top-k (ftk_topk_rows) and the launch
// helper the dense-recovery step reuses.
#include <math.h>
#include <stdint.h>

#include <atomic>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "ftk_host.h"
#include "ftk_rows.cuh"

namespace ftk {

ftk_status check_device()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cuda_status(cudaErrorInvalidDevice);
    static std::atomic<int> cached[64];  // 0 unknown, 1 ok, 2 wrong arch (threads may race here)
    const int c = dev >= 0 && dev < 64 ? cached[dev].load(std::memory_order_relaxed) : 0;
    if (c) return c == 1 ? FTK_OK : FTK_ERR_DEVICE;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return cuda_status(cudaErrorInvalidDevice);
    const bool ok = major == 10 && minor == 0;
    if (dev >= 0 && dev < 64) cached[dev].store(ok ? 1 : 2, std::memory_order_relaxed);
    return ok ? FTK_OK : FTK_ERR_DEVICE;
}

static int env_int(const char *name, int dflt)
{
    const char *v = getenv(name);
    return v && *v ? atoi(v) : dflt;
}

void rows_plan(int64_t rows, int64_t cols, int k, int *cluster, int *chunk)
{
    // At least one CTA per SM (148), and few enough expected candidates per
    // warp (~4 * k over the row) to stay well inside a warp's candidate list.
    int cs = 1;
    while (cs < kRowsMaxCluster &&
           (rows * cs < 148 || 4 * static_cast<int64_t>(k) > static_cast<int64_t>(cs) * kRowsWarps * (kRowsCapWarp / 2)))
        cs *= 2;
    const int forced = env_int("FTK_ROWS_CLUSTER", 0);
    if (forced == 1 || forced == 2 || forced == 4 || forced == 8) cs = forced;
    int64_t ch = (cols + cs - 1) / cs;
    ch = (ch + 7) / 8 * 8;
    *cluster = cs;
    *chunk = static_cast<int>(ch);
}

template <int DT>
static ftk_status launch_rows_dt(const RowsArgs &a, int cluster, bool idx64, cudaStream_t stream)
{
    // One cluster per row if they all fit at once (two CTAs per SM) and the
    // row count is known here; else as many clusters as fit, striding.
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t fit = 2 * static_cast<int64_t>(sms) / cluster;
    if (fit < 1) fit = 1;
    const bool loop = a.nrows_dev != nullptr || a.rows > fit;
    const int64_t nclusters = loop ? (a.rows < fit ? a.rows : fit) : a.rows;
    const size_t smem = sizeof(RowsSmem);
    auto kern = idx64 ? (loop ? rows_topk_kernel<DT, true, int64_t> : rows_topk_kernel<DT, false, int64_t>)
                      : (loop ? rows_topk_kernel<DT, true, int32_t> : rows_topk_kernel<DT, false, int32_t>);
    const ftk_status e = ensure_smem_limit(reinterpret_cast<const void *>(kern), static_cast<int>(smem));
    if (e != FTK_OK) return e;
    return launch_kernel(kern, dim3(static_cast<unsigned>(nclusters * cluster)), dim3(kRowsThreads), smem, stream,
                         static_cast<unsigned>(cluster), a);
}

ftk_status launch_rows_topk(int dtype, const RowsArgs &a, int cluster, cudaStream_t stream, bool idx64)
{
    if (a.chunk <= 0 || a.chunk % 8) return FTK_ERR_UNSUPPORTED;
    if (a.ldo < a.k) return FTK_ERR_INVALID_ARG;
    if (dtype == FTK_BF16) return launch_rows_dt<FTK_BF16>(a, cluster, idx64, stream);
    if (dtype == FTK_F32) return launch_rows_dt<FTK_F32>(a, cluster, idx64, stream);
    return FTK_ERR_UNSUPPORTED;
}

// ---------------------------------------------------------------------------
// sorted output: each row's k (value, column) pairs by value descending,
// column ascending (DeepSelect README, "Usage": sorted=True)
// ---------------------------------------------------------------------------

constexpr int kSortThreads = 512;

// One CTA per row: a bitonic sort of 64-bit keys (~value key, position) in
// shared memory, padded to kp = the power of two >= k with keys that sort
// last.  The unsorted output is in ascending column order, so ordering
// equal values by position orders them by column; the values and columns
// are then moved by position, bit for bit (-0.0 stays -0.0).  The padding
// slots of a row shorter than k (positions >= its length) keep their place
// at the end whatever their fill value.  Without a value output the key
// is read from x at the selected column.
template <int DT, typename IT>
__global__ void __launch_bounds__(kSortThreads) sort_rows_kernel(const void *x, int64_t ld,
                                                                 const int32_t *row_end, int64_t cols,
                                                                 void *vals, IT *idx, int64_t ldo, int k,
                                                                 int kp)
{
    griddep_wait();  // the previous kernel on the stream is complete
    griddep_launch_next();
    using Tr = RowsTraits<DT>;
    using elem = typename Tr::elem;
    extern __shared__ unsigned long long skey[];
    const int64_t r = blockIdx.x;
    int64_t len = cols;
    if (row_end) {
        const int64_t e = row_end[r];
        len = e < 0 ? 0 : (e < len ? e : len);
    }
    const int nreal = len < k ? static_cast<int>(len) : k;
    elem *v = vals ? static_cast<elem *>(vals) + r * ldo : nullptr;
    const elem *xr = static_cast<const elem *>(x) + r * ld;
    IT *ix = idx + r * ldo;
    for (int i = threadIdx.x; i < kp; i += blockDim.x) {
        unsigned long long c = ~0ull;
        if (i < nreal) {
            const uint32_t bits = static_cast<uint32_t>(v ? v[i] : xr[ix[i]]);
            c = (static_cast<unsigned long long>(~Tr::key(bits)) << 32) | static_cast<uint32_t>(i);
        } else if (i < k) {
            c = (0xFFFFFFFFull << 32) | static_cast<uint32_t>(i);
        }
        skey[i] = c;
    }
    __syncthreads();
    for (int size = 2; size <= kp; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = threadIdx.x; i < kp / 2; i += blockDim.x) {
                const int lo = 2 * i - (i & (stride - 1));
                const int hi = lo + stride;
                const bool up = (lo & size) == 0;
                const unsigned long long a = skey[lo], b = skey[hi];
                if ((a > b) == up) {
                    skey[lo] = b;
                    skey[hi] = a;
                }
            }
            __syncthreads();
        }
    }
    constexpr int kPer = FTK_MAX_TOPK / kSortThreads;  // outputs per thread (k <= FTK_MAX_TOPK)
    elem mv[kPer];
    IT mi[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
        const int i = threadIdx.x + j * kSortThreads;
        if (i < k) {
            const int pos = static_cast<int>(static_cast<uint32_t>(skey[i]));
            if (v) mv[j] = v[pos];
            mi[j] = ix[pos];
        }
    }
    __syncthreads();  // every read of the unsorted row precedes the writes (in place)
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
        const int i = threadIdx.x + j * kSortThreads;
        if (i < k) {
            if (v) v[i] = mv[j];
            ix[i] = mi[j];
        }
    }
}

template <int DT>
static void launch_sort_dt(const RowsArgs &a, bool idx64, unsigned rows, int kp, size_t smem,
                           cudaStream_t stream)
{
    if (idx64)
        sort_rows_kernel<DT, int64_t><<<rows, kSortThreads, smem, stream>>>(
            a.x, a.ld, a.row_end, a.cols, a.out_val, static_cast<int64_t *>(a.out_idx), a.ldo, a.k, kp);
    else
        sort_rows_kernel<DT, int32_t><<<rows, kSortThreads, smem, stream>>>(
            a.x, a.ld, a.row_end, a.cols, a.out_val, static_cast<int32_t *>(a.out_idx), a.ldo, a.k, kp);
}

// Sorts the output of a finished row top-k call described by `a`.
static ftk_status launch_sort_rows(int dtype, const RowsArgs &a, bool idx64, cudaStream_t stream)
{
    int kp = 1;
    while (kp < a.k) kp <<= 1;
    const size_t smem = static_cast<size_t>(kp) * sizeof(unsigned long long);
    const unsigned rows = static_cast<unsigned>(a.rows);
    if (dtype == FTK_BF16)
        launch_sort_dt<FTK_BF16>(a, idx64, rows, kp, smem, stream);
    else
        launch_sort_dt<FTK_F32>(a, idx64, rows, kp, smem, stream);
    return cuda_status(cudaGetLastError());
}

// float -> bf16 bits, round to nearest even (a NaN stays a quiet NaN).
static uint32_t bf16_bits(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u) return ((u >> 16) | 0x40u) & 0xFFFFu;
    return (u + 0x7FFFu + ((u >> 16) & 1u)) >> 16;
}

static ftk_status topk_rows_impl(ftk_dtype dtype, const void *x, int64_t rows, int64_t cols,
                                 int64_t row_stride, const int32_t *row_end, int topk,
                                 const ftk_rows_options &o, void *out_idx, void *out_val,
                                 uint32_t *status, void *stream)
{
    if (dtype != FTK_BF16 && dtype != FTK_F32) return FTK_ERR_UNSUPPORTED;
    if (!x || !out_idx) return FTK_ERR_INVALID_ARG;
    if (rows < 1 || cols < 1 || row_stride < cols || rows > (int64_t(1) << 31) / kRowsMaxCluster)
        return FTK_ERR_INVALID_ARG;
    if (topk < 1 || topk > FTK_MAX_TOPK) return FTK_ERR_TOPK_RANGE;
    if (cols > kRowsMaxCols) return FTK_ERR_UNSUPPORTED;
    if ((o.sorted != 0 && o.sorted != 1) || (o.index_bits != 32 && o.index_bits != 64))
        return FTK_ERR_INVALID_ARG;
    const int64_t ldo = o.out_stride ? o.out_stride : topk;
    if (ldo < topk || ldo > INT32_MAX) return FTK_ERR_INVALID_ARG;  // offsets stay within int64
    if (o.index_bits == 32 && (o.idx_fill < INT32_MIN || o.idx_fill > INT32_MAX)) return FTK_ERR_INVALID_ARG;
    const int esz = dtype == FTK_BF16 ? 2 : 4;
    if (!aligned16(x) || (row_stride * esz) % 16) return FTK_ERR_ALIGNMENT;
    if (reinterpret_cast<uintptr_t>(out_idx) % (o.index_bits / 8) ||
        reinterpret_cast<uintptr_t>(out_val) % esz)
        return FTK_ERR_ALIGNMENT;
    ftk_status st = check_device();
    if (st != FTK_OK) return st;
    RowsArgs a = {};
    a.x = x;
    a.ld = row_stride;
    a.cols = cols;
    a.rows = rows;
    a.row_end = row_end;
    a.out_idx = out_idx;
    a.out_val = out_val;
    a.ldo = ldo;
    a.idx_fill = o.idx_fill;
    if (dtype == FTK_BF16) {
        a.val_fill = bf16_bits(o.val_fill);
    } else {
        memcpy(&a.val_fill, &o.val_fill, sizeof a.val_fill);
    }
    a.k = topk;
    a.status = status;
    int cluster = 1, chunk = 8;
    rows_plan(rows, cols, topk, &cluster, &chunk);
    a.chunk = chunk;
    const bool idx64 = o.index_bits == 64;
    st = launch_rows_topk(dtype, a, cluster, as_stream(stream), idx64);
    if (st != FTK_OK || !o.sorted) return st;
    return launch_sort_rows(dtype, a, idx64, as_stream(stream));
}

}  // namespace ftk

using namespace ftk;

extern "C" void ftk_rows_options_init(ftk_rows_options *o)
{
    if (!o) return;
    memset(o, 0, sizeof *o);
    o->sorted = 0;
    o->index_bits = 32;
    o->out_stride = 0;
    o->idx_fill = -1;
    o->val_fill = -INFINITY;
}

extern "C" ftk_status ftk_topk_rows(ftk_dtype dtype, const void *x, int64_t rows, int64_t cols,
                                    int64_t row_stride, int topk, int32_t *out_idx,
                                    void *out_val, uint32_t *status, void *stream)
{
    ftk_rows_options o;
    ftk_rows_options_init(&o);
    return topk_rows_impl(dtype, x, rows, cols, row_stride, nullptr, topk, o, out_idx, out_val, status,
                          stream);
}

extern "C" ftk_status ftk_topk_rows_end(ftk_dtype dtype, const void *x, int64_t rows, int64_t cols,
                                        int64_t row_stride, const int32_t *row_end, int topk,
                                        int32_t *out_idx, void *out_val, uint32_t *status,
                                        void *stream)
{
    if (!row_end) return FTK_ERR_INVALID_ARG;
    ftk_rows_options o;
    ftk_rows_options_init(&o);
    return topk_rows_impl(dtype, x, rows, cols, row_stride, row_end, topk, o, out_idx, out_val, status,
                          stream);
}

extern "C" ftk_status ftk_topk_rows_sorted(ftk_dtype dtype, const void *x, int64_t rows, int64_t cols,
                                           int64_t row_stride, const int32_t *row_end, int topk,
                                           int32_t *out_idx, void *out_val, uint32_t *status,
                                           void *stream)
{
    if (!out_val) return FTK_ERR_INVALID_ARG;
    ftk_rows_options o;
    ftk_rows_options_init(&o);
    o.sorted = 1;
    return topk_rows_impl(dtype, x, rows, cols, row_stride, row_end, topk, o, out_idx, out_val, status,
                          stream);
}

extern "C" ftk_status ftk_topk_rows_ex(ftk_dtype dtype, const void *x, int64_t rows, int64_t cols,
                                       int64_t row_stride, const int32_t *row_end, int topk,
                                       const ftk_rows_options *options, void *out_idx, void *out_val,
                                       uint32_t *status, void *stream)
{
    ftk_rows_options o;
    ftk_rows_options_init(&o);
    if (options) o = *options;
    return topk_rows_impl(dtype, x, rows, cols, row_stride, row_end, topk, o, out_idx, out_val, status,
                          stream);
}
