/*
 * ftk.h -- C ABI of libftk: fused lightning-indexer scoring with exact,
 * deterministic per-query top-k, and a standalone row top-k, for NVIDIA
 * B200 (sm_100a).
 *
 * Plain C: pointers, sizes, enums.  No CUDA or torch types appear here; a
 * CUDA stream is passed as `void *` (a cudaStream_t, NULL = legacy default
 * stream).  "device" pointers are CUDA device memory of the current device;
 * "host" pointers are ordinary CPU memory.
 *
 * Conventions shared by every call
 *  - Calls are asynchronous and stream-ordered unless stated otherwise; they
 *    never synchronise the host with the device (except ftk_read_info).
 *  - Argument errors that the host can see (NULL pointers, sizes, dtypes,
 *    topk range, alignment, workspace size) return a negative ftk_status and
 *    launch nothing.
 *  - Errors that only the device can see (a window outside [0, S], a NaN
 *    score, a bounded wait that gave up) never abort a kernel: they set bits
 *    of a device status word (FTK_STATUS_*), readable after the stream
 *    completes.
 *  - The caller owns every buffer.  The library allocates no device memory.
 *  - Output order: the selected keys of a row are written in ascending key
 *    index, which makes the output bits a pure function of the inputs
 *    (FlashTopK README, "Highlights": the same bits on every run).
 */
#ifndef FTK_H
#define FTK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Indexer shape (FlashTopK README, "Support": indexers of 32 heads x 128). */
#define FTK_HEADS 32
#define FTK_DIM 128
/* topk range (FlashTopK README, "Support"; DeepSelect README, "Supported
 * Cases": topk must be <= 4096). */
#define FTK_MAX_TOPK 4096

typedef enum {
    FTK_F8E4M3 = 1, /* float8 e4m3fn, 1 byte */
    FTK_BF16 = 2,   /* bfloat16, 2 bytes */
    FTK_F32 = 3     /* float32, 4 bytes */
} ftk_dtype;

typedef enum {
    FTK_OK = 0,
    FTK_ERR_INVALID_ARG = -1, /* NULL pointer, negative/oversized size, bad dtype */
    FTK_ERR_UNSUPPORTED = -2, /* a valid request this build does not handle */
    FTK_ERR_TOPK_RANGE = -3,  /* topk outside [1, FTK_MAX_TOPK] */
    FTK_ERR_ALIGNMENT = -4,   /* pointer or row stride not 16-byte aligned */
    FTK_ERR_WORKSPACE = -5,   /* workspace NULL, misaligned or too small */
    FTK_ERR_CUDA = -6,        /* a CUDA runtime call failed */
    FTK_ERR_DEVICE = -7       /* current device is not compute capability 10.0 */
} ftk_status;

/* Device status bits (ftk_info.status, and the status word of
 * ftk_topk_rows).  A row hit by BAD_WINDOW is written as all (-1, -inf);
 * a row hit by NAN has unspecified contents. */
#define FTK_STATUS_BAD_WINDOW 0x1u /* ks < 0, ks > ke or ke > S in some row */
#define FTK_STATUS_NAN 0x2u        /* a NaN score or input value was seen */
#define FTK_STATUS_TIMEOUT 0x4u    /* a bounded device wait gave up */
#define FTK_STATUS_BAD_SCALE 0x8u  /* a kv_scales entry was <= 0 or not finite */
#define FTK_STATUS_INTERNAL 0x10u  /* an internal bounds check failed */

/* Tuning knobs of ftk_select.  None of them changes the result (the
 * selection is exact); they trade speed against the rate of rows that need
 * dense recovery.  Pass NULL for the defaults. */
typedef struct {
    int32_t sample_keys; /* target strided-sample size per row, m (default 4096) */
    float oversample;    /* beta: the threshold keeps ~beta*topk keys (default 1.5) */
    int32_t capacity;    /* C: candidate slots per row (0: 5*topk/2, at most 2*FTK_MAX_TOPK) */
    int32_t prune;       /* score-bound key pruning (FlashTopK README, "Highlights":
                          * adaptive key pruning by a score bound): 0 auto, the
                          * default (for calls of at least 128 query rows,
                          * estimate the skippable share of key blocks on a
                          * sample and prune if it is >= 25%; smaller calls scan
                          * densely), 1 always, -1 off */
    int32_t recovery_rows; /* rows rescored densely per recovery pass (0: auto) */
    int32_t heads;         /* indexer heads H: 32 (or 0, the default) or 64 (FlashTopK
                            * README, "Roadmap": other head counts such as 64); q is then
                            * [T, H, 128] and weights [T, H]. */
    int32_t dense_rows;    /* calls of at most this many query rows (and at most 2^25
                            * (row, key) pairs, and rows that fit one recovery pass)
                            * score every key of every window and select with the
                            * row top-k instead of the sampled threshold (0: 128, the
                            * default; -1: never).  Such calls skip the sample,
                            * threshold, pruning and refine stages (prune has no
                            * effect); info counts every window key as a candidate. */
    int32_t reserved;      /* must be 0 */
} ftk_config;

/* Per-call information (FlashTopK README, "Usage": last_info), filled on
 * the device by ftk_select and read back with ftk_read_info. */
typedef struct {
    uint32_t status;          /* FTK_STATUS_* bits */
    int32_t prune_enabled;    /* 1 if the call scanned with key pruning */
    int64_t rows;             /* T */
    int64_t rows_underflow;   /* rows whose threshold kept fewer than min(topk, L) keys */
    int64_t rows_overflow;    /* rows whose candidates exceeded the capacity */
    int64_t blocks_total;     /* (query tile, 128-key block) pairs in the windows */
    int64_t blocks_pruned;    /* of which skipped by the score bound */
    int64_t candidates_total; /* sum over rows of candidates kept */
    int64_t candidates_max;   /* largest per-row candidate count */
    int64_t kernel_launches;  /* kernels the call launched */
} ftk_info;

/*
 * ftk_select -- for every query row t, the topk keys s of its window
 * [ks[t], ke[t]) with the largest indexer score
 *     I[t,s] = sigma_s * sum_{h<32} w[t,h] * ReLU(q[t,h] . kv[s])
 * (FlashTopK README, "Quick start"), exact, with ties at the k-th score
 * resolved to the smallest key indices (FlashTopK README, "Highlights").
 *
 *   dtype      FTK_F8E4M3 or FTK_BF16 (q and kv share it)
 *   q          device [T, 32, 128] of dtype, contiguous, 16-byte aligned
 *   kv         device [S, 128] of dtype, contiguous, 16-byte aligned
 *   kv_scales  device [S] float32 sigma_s, or NULL for all ones (BF16 keys);
 *              values must be > 0 (checked, FTK_STATUS_BAD_SCALE)
 *   weights    device [T, 32] float32, 16-byte aligned
 *   ks, ke     device [T] int32 windows, 0 <= ks <= ke <= S
 *   T, S       1 <= T < 2^26 (the T * 32 head rows stay below 2^31) and
 *              1 <= S < 2^31 - 8192
 *   topk       1 .. FTK_MAX_TOPK
 *   out_idx    device [T, topk] int32: selected key indices in ascending
 *              order; rows whose window holds L < topk keys get the L keys
 *              then index -1
 *   out_val    device [T, topk] float32 scores of out_idx (-inf for padding),
 *              or NULL to skip them
 *   workspace  device scratch of at least ftk_select_workspace_size() bytes,
 *              256-byte aligned; owned by the caller; one call at a time per
 *              workspace (calls on different streams need different ones)
 *   config     host pointer to tuning knobs, or NULL
 *   stream     cudaStream_t
 * Scores are computed with FP8/BF16 products and float32 accumulation; each
 * returned score is within 1e-4 * sigma_s * sum_h |w[t,h]| *
 * sum_d |q[t,h,d] * kv[s,d]| of the exact value.
 */
ftk_status ftk_select(ftk_dtype dtype, const void *q, const void *kv,
                      const float *kv_scales, const float *weights,
                      const int32_t *ks, const int32_t *ke, int64_t T,
                      int64_t S, int topk, int32_t *out_idx, float *out_val,
                      void *workspace, size_t workspace_bytes,
                      const ftk_config *config, void *stream);

/* Bytes of workspace ftk_select needs for these sizes (FlashTopK README,
 * "Usage": Selector.plan(max_rows, max_kv) owns the workspace).  A
 * workspace sized for (T, S) serves any call with smaller T and S and the
 * same topk and config.  Returns 0 for invalid sizes. */
size_t ftk_select_workspace_size(int64_t T, int64_t S, int topk,
                                 const ftk_config *config);

/* Copies the ftk_info of the last ftk_select run on this workspace to the
 * host struct *out.  Synchronises `stream` first.  workspace: device. */
ftk_status ftk_read_info(const void *workspace, ftk_info *out, void *stream);

/*
 * ftk_topk_rows -- row top-k (DeepSelect README, "Supported Cases" and
 * "Usage"): for each row r of x, the topk columns with the largest values,
 * ties to the smaller column index, output in ascending column order.
 *
 *   dtype       FTK_BF16 or FTK_F32
 *   x           device [rows, cols] of dtype; row r starts at
 *               x + r * row_stride elements; x and row_stride * elem_size
 *               must be 16-byte aligned (DeepSelect README, "Usage": the row
 *               stride alignment requirement)
 *   rows        >= 1;  cols: 1 .. 2^30
 *   topk        1 .. FTK_MAX_TOPK; rows with cols < topk are padded with
 *               index -1 and value -inf
 *   out_idx     device [rows, topk] int32
 *   out_val     device [rows, topk] of dtype (x's), or NULL to skip values
 *               (DeepSelect README, "Usage": return_value=False)
 *   status      device uint32 word that receives FTK_STATUS_NAN bits
 *               (OR-ed in; DeepSelect README, "NaN handling" aborts instead),
 *               or NULL
 *   stream      cudaStream_t
 * Diagnostics: the environment variable FTK_ROWS_CLUSTER = 1, 2, 4 or 8
 * forces the number of CTAs (one thread-block cluster) per row instead of
 * the planned one; the result is the same, only the speed changes.
 */
ftk_status ftk_topk_rows(ftk_dtype dtype, const void *x, int64_t rows,
                         int64_t cols, int64_t row_stride, int topk,
                         int32_t *out_idx, void *out_val, uint32_t *status,
                         void *stream);

/*
 * ftk_topk_rows_end -- ftk_topk_rows over variable-length rows (DeepSelect
 * README, "Variable-length rows": a per-row exclusive end): row r holds
 * only its columns [0, row_end[r]), row_end[r] clamped to [0, cols]; rows
 * that end up shorter than topk are padded with index -1 and value -inf.
 *   row_end   device [rows] int32 (must not be NULL)
 * Other arguments, layout and errors as for ftk_topk_rows.
 */
ftk_status ftk_topk_rows_end(ftk_dtype dtype, const void *x, int64_t rows,
                             int64_t cols, int64_t row_stride,
                             const int32_t *row_end, int topk,
                             int32_t *out_idx, void *out_val,
                             uint32_t *status, void *stream);

/*
 * ftk_topk_rows_sorted -- ftk_topk_rows (or ftk_topk_rows_end when row_end
 * is not NULL) with each row's output ordered by value descending, ties by
 * column ascending, padding last (DeepSelect README, "Usage": sorted=True;
 * the unsorted calls return ascending columns, i.e. sorted_index=True).
 *   row_end   device [rows] int32 per-row exclusive end, or NULL
 *   out_val   required (not NULL): the sort needs the values
 * Other arguments, layout and errors as for ftk_topk_rows.
 */
ftk_status ftk_topk_rows_sorted(ftk_dtype dtype, const void *x, int64_t rows,
                                int64_t cols, int64_t row_stride,
                                const int32_t *row_end, int topk,
                                int32_t *out_idx, void *out_val,
                                uint32_t *status, void *stream);

/*
 * Options of ftk_topk_rows_ex (DeepSelect README, "Usage" and
 * "Variable-length rows": sorted, sorted_index, indices_type, the output
 * buffers' row stride and the out-of-bound fill values).  Fill a struct
 * with ftk_rows_options_init, then change what differs.
 *   sorted       0: each row's output in ascending column order (what
 *                DeepSelect calls sorted_index=True, which also serves
 *                sorted_index=False); 1: by value descending, ties by
 *                column ascending, padding last
 *   index_bits   32: out_idx is int32_t; 64: int64_t (indices_type)
 *   out_stride   elements between consecutive output rows of out_idx and
 *                out_val; 0 means topk; otherwise topk .. 2^31 - 1
 *   idx_fill     index of the padding slots of rows shorter than topk
 *                (idx_oob_fill_value); within int32 when index_bits = 32
 *   val_fill     value of those slots (value_oob_fill_value), stored in
 *                x's dtype (rounded to nearest even for bf16)
 * Defaults: sorted 0, index_bits 32, out_stride 0, idx_fill -1,
 * val_fill -inf.
 */
typedef struct {
    int32_t sorted;
    int32_t index_bits;
    int64_t out_stride;
    int64_t idx_fill;
    float val_fill;
} ftk_rows_options;

/* Writes the defaults above into *options (no-op on NULL). */
void ftk_rows_options_init(ftk_rows_options *options);

/*
 * ftk_topk_rows_ex -- the row top-k with every option: ftk_topk_rows,
 * ftk_topk_rows_end and ftk_topk_rows_sorted are this call with default
 * options (and sorted = 1 for the last).
 *   row_end   device [rows] int32 per-row exclusive end, clamped to
 *             [0, cols], or NULL (every row has cols columns)
 *   options   as above, or NULL for the defaults
 *   out_idx   device [rows, out_stride] int32 or int64 (index_bits),
 *             aligned to its element size; slots [0, topk) of each row are
 *             written
 *   out_val   device [rows, out_stride] of x's dtype, aligned to its
 *             element size, or NULL; with sorted = 1 and no value output
 *             the sort reads each selected value from x
 * Errors: FTK_ERR_INVALID_ARG for an option outside the ranges above,
 * FTK_ERR_ALIGNMENT for misaligned outputs; the rest as for ftk_topk_rows.
 */
ftk_status ftk_topk_rows_ex(ftk_dtype dtype, const void *x, int64_t rows,
                            int64_t cols, int64_t row_stride,
                            const int32_t *row_end, int topk,
                            const ftk_rows_options *options, void *out_idx,
                            void *out_val, uint32_t *status, void *stream);

/*
 * ftk_score_dense -- the fused scores themselves, for checking: for each
 * listed row r (query t = rows ? rows[r] : r) writes
 *     out[r * ld + (s - ks[t])] = I[t, s]   for s in [ks[t], ke[t])
 * with exactly the arithmetic ftk_select uses (same kernel, same bits).
 * Entries past a row's window are left untouched.
 *   rows   device [nrows] int32 query indices, or NULL for 0 .. nrows-1
 *   out    device float32 [nrows, ld], ld >= S (so that every valid window
 *          fits its row), ld % 4 == 0
 *   workspace  as for ftk_select, sized by ftk_score_dense_workspace_size
 * Other arguments as for ftk_select.
 */
ftk_status ftk_score_dense(ftk_dtype dtype, const void *q, const void *kv,
                           const float *kv_scales, const float *weights,
                           const int32_t *ks, const int32_t *ke, int64_t T,
                           int64_t S, const int32_t *rows, int64_t nrows,
                           float *out, int64_t ld, void *workspace,
                           size_t workspace_bytes, void *stream);

size_t ftk_score_dense_workspace_size(int64_t nrows);

/* ftk_score_dense for an indexer of `heads` heads (32 or 64): q
 * [T, heads, 128], weights [T, heads]; otherwise as ftk_score_dense (which
 * is this call with heads = 32). */
ftk_status ftk_score_dense_heads(ftk_dtype dtype, int heads, const void *q,
                                 const void *kv, const float *kv_scales,
                                 const float *weights, const int32_t *ks,
                                 const int32_t *ke, int64_t T, int64_t S,
                                 const int32_t *rows, int64_t nrows, float *out,
                                 int64_t ld, void *workspace,
                                 size_t workspace_bytes, void *stream);

/*
 * ftk_block_bound -- the score bound that ftk_select's key pruning uses
 * (FlashTopK README, "Highlights": keys are skipped by a score bound; the
 * pages give no formula, this is the per-dimension box bound).  For every
 * query row t < T and key block b (keys [128 b, min(128 b + 128, S)))
 * writes out[t * ld + b] = UB[t, b] >= I[t, s] for every key s of block b:
 *     hi[d] = max_s sigma_s kv[s,d],  lo[d] = min_s sigma_s kv[s,d]
 *     U_h = sum_d max(q[t,h,d] hi[d], q[t,h,d] lo[d]),  L_h = same with min
 *     UB  = sum_{w[t,h] >= 0} w[t,h] ReLU(U_h) + sum_{w[t,h] < 0} w[t,h] ReLU(L_h)
 * computed in float32 (within about 1e-5 * sum_h |w| sum_d |q| max(|hi|,
 * |lo|) of the exact value).  A block holding a NaN key, a kv_scales entry
 * that is not finite and > 0, or a product that overflows gets +inf.
 *   out        device float32 [T, ld], ld >= ceil(S / 128)
 *   workspace  device, >= ftk_block_bound_workspace_size(S) bytes,
 *              256-byte aligned
 * Other arguments as for ftk_select (no windows: every block of every row).
 */
ftk_status ftk_block_bound(ftk_dtype dtype, const void *q, const void *kv,
                           const float *kv_scales, const float *weights,
                           int64_t T, int64_t S, float *out, int64_t ld,
                           void *workspace, size_t workspace_bytes,
                           void *stream);

size_t ftk_block_bound_workspace_size(int64_t S);

/* ftk_block_bound for an indexer of `heads` heads (32 or 64): q
 * [T, heads, 128], weights [T, heads], the sums over h run over every head;
 * otherwise as ftk_block_bound (which is this call with heads = 32). */
ftk_status ftk_block_bound_heads(ftk_dtype dtype, int heads, const void *q,
                                 const void *kv, const float *kv_scales,
                                 const float *weights, int64_t T, int64_t S,
                                 float *out, int64_t ld, void *workspace,
                                 size_t workspace_bytes, void *stream);

/*
 * ftk_windows_from_cu_seqlens -- causal windows of packed sequences
 * (FlashTopK README, "Usage": windows_from_cu_seqlens).  Sequence j owns
 * query rows [cu_q[j], cu_q[j+1]) and keys [cu_k[j], cu_k[j+1]); its
 * queries are its last tokens, so its i-th query sees keys
 *     [cu_k[j], cu_k[j] + (Lk_j - Lq_j) + i + 1)
 * (FlashTopK README, "Quick start": query i sees keys [0, S - T + i + 1)),
 * clamped to an empty window when Lk_j < Lq_j - i.
 *   cu_q, cu_k  device [nseq + 1] int32 prefix offsets, cu_q[nseq] == T
 *   ks, ke      device [T] int32 outputs
 */
ftk_status ftk_windows_from_cu_seqlens(const int32_t *cu_q,
                                       const int32_t *cu_k, int64_t nseq,
                                       int64_t T, int32_t *ks, int32_t *ke,
                                       void *stream);

/*
 * ftk_select_noalloc -- ftk_select without a caller-supplied workspace, for
 * callers that cannot allocate device memory (code inside another
 * allocator's arena or under a memory cap, code that must not fail with an
 * out-of-memory error at call time, plain C hosts with no allocator).  It
 * allocates nothing: its scratch is a fixed __device__ array of
 * FTK_NOALLOC_SCRATCH_BYTES inside the library, held by every GPU that
 * loads the library until the process exits.  The pages describe no such
 * call; it has no counterpart there.
 *
 * Arguments and results are those of ftk_select (same kernels, same bits),
 * minus the workspace.  If config->recovery_rows is 0 (or config is NULL),
 * the recovery batch is the largest that fits the array.
 * Returns FTK_ERR_WORKSPACE when the problem needs more scratch than
 * FTK_NOALLOC_SCRATCH_BYTES (smaller T, S or topk fit).
 * The array's device address is looked up (cudaGetSymbolAddress) on the
 * first call in each CUDA context of a device and again whenever the
 * context changes (say after cudaDeviceReset); make the first call on a
 * device before any stream capture.  Argument errors are those of
 * ftk_select and are reported first.
 * All calls share the one array and leave their state in it (each call
 * clears what it needs): calls that overlap on the same GPU, for example
 * on two streams, race on it, so serialise them.  The per-call information
 * (status bits such as FTK_STATUS_BAD_WINDOW or FTK_STATUS_NAN included)
 * is read with ftk_noalloc_read_info.
 */
#define FTK_NOALLOC_SCRATCH_BYTES (64u << 20)
ftk_status ftk_select_noalloc(ftk_dtype dtype, const void *q, const void *kv,
                              const float *kv_scales, const float *weights,
                              const int32_t *ks, const int32_t *ke, int64_t T,
                              int64_t S, int topk, int32_t *out_idx,
                              float *out_val, const ftk_config *config,
                              void *stream);

/* The ftk_info of the last ftk_select_noalloc call on the current device,
 * copied from the start of the fixed array after the stream completes
 * (synchronises the stream, like ftk_read_info); it allocates nothing.
 * Valid only when no other ftk_select_noalloc call on this device ran in
 * between. */
ftk_status ftk_noalloc_read_info(ftk_info *out, void *stream);

/* Diagnostic timing hook.  While set, every ftk_select call made from the
 * calling host thread records events[i] (cudaEvent_t values created by the
 * caller, passed as void *) on the call's stream at its stage boundaries:
 * 0 start, 1 plan done, 2 sample pass done, 3 thresholds done, 4 scan done,
 * 5 refine done, 6 recovery done, and, when n >= 8, 7 pruning done (after
 * the score-bound kernels, before the scan; right after 3 when pruning is
 * off).  n must be 0 (or events NULL) to stop, else >= 7 with non-NULL
 * events (the first min(n, 8) are used; FTK_ERR_INVALID_ARG otherwise).
 * If recording fails the hook switches itself off.  The handles are copied
 * (the array itself need not outlive this call); the events must stay valid
 * while the hook is set.  The library does not own the events. */
ftk_status ftk_set_stage_events(void *const *events, int n);

/* Human-readable name of an ftk_status value (static string). */
const char *ftk_status_string(int status);

/* Library version as MAJOR * 10000 + MINOR * 100 + PATCH. */
int ftk_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FTK_H */
