// ftk_score.cuh -- fused lightning-indexer scoring on the 5th-generation
// tensor cores (tcgen05 + TMEM, operands staged by TMA).
//
// Score (FlashTopK README, "Quick start"):
//     I[t,s] = sigma_s * sum_{h<32} w[t,h] * ReLU(q[t,h] . k[s])
//
// GEMM orientation: A = a tile of 128 keys (M = 128, K = 128 head dims),
// B = a tile of 8 queries x 32 heads (N = 256), both K-major with the
// 128-byte swizzle.  A work item holds a group of QG such query tiles
// resident in shared memory (QG = 2 for FP8) and streams key tiles through
// a TMA ring; each key tile feeds QG MMAs, one per query tile, which halves
// the key traffic from L2 per FLOP.  The fp32 accumulator (128 lanes x 256
// columns) alternates between two tensor-memory buffers (2 x 256 of the 512
// columns); with QG = 2 one key tile fills both, and an accumulator goes
// back to the MMA warp as soon as every epilogue warp has loaded it.  TMEM lane = key, so each epilogue thread
// owns one key and reduces the 32 heads of a query in registers: ReLU, the
// head weights and sigma are applied and the T x S x 32 intermediate never
// leaves the SM.
//
// Warp roles (18 warps):
//   warp 0      TMA producer: the query group per work item, key tiles
//               through a multi-stage mbarrier ring;
//   warp 1      TMEM allocator and MMA issuer (one elected thread);
//   warps 2-17  epilogue: warp w reads TMEM lane quarter (w % 4) and the
//               queries 2*((w-2)/4), 2*((w-2)/4)+1 of every query tile, four
//               warps per scheduler so that their dependency chains
//               interleave.
//
// Head reduction: for each (query, key), two partial sums over the even and
// the odd heads (the two lanes of one packed fma chain, correctly rounded,
// in head order), added, times sigma, plus +0.0 (which turns -0.0 into
// +0.0).  ReLU propagates NaN, so a NaN dot product makes the score NaN,
// which the candidate test keeps and the refine step reports.
//
// 64 heads (H64 = true; FlashTopK README, "Roadmap": other head counts
// such as 64): q [T, 64, 128] is the same bytes as [2T, 32, 128], so query
// t occupies MMA rows 2t and 2t + 1 (heads 0..31 and 32..63) and the
// tiles, TMA loads and TMEM layout stay as they are (4 queries per MMA
// tile).  The epilogue warp that holds those two rows finishes one score
//     I = sigma * ((even_a + odd_a) + (even_b + odd_b)) + 0.0
// from the two halves' partial sums and makes one threshold decision per
// query.
//
// Pruning (PR = true): key tiles that the score bound marks for the item's
// row tile are skipped by all three roles (see ftk_prune.cuh).
//
// Modes (one kernel body, so every mode produces bit-identical scores):
//   SAMPLE   keys are a strided sample k[j*stride] (a strided TMA view of kv);
//            scores go to a dense [row, sample] buffer (the threshold input);
//   COLLECT  keeps the keys with I >= tau[t] (NaN kept too, so that it is
//            seen): warp ballot + shared-memory staging, flushed to per-row
//            candidate buffers with one global atomic per query per flush;
//   DUMP     writes every in-window score to out[row, s - ks[t]] (dense
//            recovery of rows the threshold missed, and score checks).
#pragma once

#include "ftk_device.cuh"

namespace ftk {

enum ScoreMode { MODE_SAMPLE = 0, MODE_COLLECT = 1, MODE_DUMP = 2 };

constexpr int kQTile = 8;            // queries per MMA tile -> N = 256
constexpr int kKeyTile = 128;        // keys per tile -> M = 128
constexpr int kChunkTiles = 64;      // key tiles per work item (8192 keys)
constexpr int kChunkKeys = kChunkTiles * kKeyTile;
constexpr int kEpiWarps = 16;        // warps 2..17
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kScoreThreads = 64 + kEpiThreads;  // + producer and MMA warps
constexpr int kEpiQueries = kQTile * 4 / kEpiWarps;  // queries per epilogue warp per query tile (2)
constexpr int kNumStrideMaps = 20;   // sample strides 2^0 .. 2^19

template <int DT>
struct ScoreCfg;

template <>
struct ScoreCfg<FTK_F8E4M3> {
    static constexpr int kAtoms = 1;       // 128-byte swizzle atoms along K (128 dims x 1 B)
    static constexpr int kQG = 2;          // query tiles per work item (rows per item: 16)
    static constexpr int kKStages = 4;
    static constexpr int kWarpStage = 128; // staged candidates per (epilogue warp, query)
    static constexpr int kMmaK = 4;        // MMAs per tile (K = 32 each)
    static constexpr uint32_t kIdesc = instr_desc(0, 0, 128, 256);  // e4m3 x e4m3 -> f32
};

template <>
struct ScoreCfg<FTK_BF16> {
    static constexpr int kAtoms = 2;       // 128 dims x 2 B = two 128-byte atoms
    static constexpr int kQG = 1;          // rows per item: 8
    static constexpr int kKStages = 3;
    static constexpr int kWarpStage = 128;
    static constexpr int kMmaK = 8;        // K = 16 each
    static constexpr uint32_t kIdesc = instr_desc(1, 1, 128, 256);  // bf16 x bf16 -> f32
};

// Rows of the row list per work item (the planning granularity): the
// queries of the item's MMA tiles (a 64-head query takes two MMA rows).
__host__ __device__ constexpr int row_tile_of(int dtype, int heads = 32)
{
    return (dtype == FTK_F8E4M3 ? ScoreCfg<FTK_F8E4M3>::kQG : ScoreCfg<FTK_BF16>::kQG) * kQTile /
           (heads == 64 ? 2 : 1);
}

struct ScoreArgs {
    int64_t T, S;
    const float *kv_scales;   // [S] or NULL (all ones)
    const float *weights;     // [T, heads]
    const int32_t *ks, *ke;   // [T]
    // Row list: position p of the list is query rows[p] (identity if NULL).
    // The list holds min(nrows, *count_dev - count_off) rows when count_dev
    // is given (device-side counts, e.g. the rows that need recovery).
    const int32_t *rows;
    int64_t nrows;
    const int32_t *count_dev;
    int32_t count_off;
    // Schedule over row tiles of row_tile_of(dtype) rows.  Planned: per-tile
    // ranges and an item prefix written by the plan kernel.  Static: item =
    // (tile, chunk of keys), ranges found on the fly, chunk size chosen at
    // kernel start from the rows in the list (make_sched).  SAMPLE and
    // COLLECT run planned, DUMP static.
    int32_t planned;
    int32_t *work_next;       // planned: shared item counter (dynamic schedule), or NULL
    int32_t chunk_keys;       // planned: keys (SAMPLE: samples) per work item, a multiple of 128
    const int32_t *tile_lo, *tile_hi, *tile_lg, *item_start;
    int32_t ntiles;
    // COLLECT
    const float *tau;         // [T]
    int32_t *cnt;             // [T] running candidate counts
    float *cand_val;          // [T, cap]
    int32_t *cand_idx;        // [T, cap]
    int32_t cap;
    // COLLECT with key pruning: bit b of word prune_bits[tile * prune_words
    // + b / 32] set means key block b (keys 128 b .. 128 b + 127) holds no
    // candidate of any row of the tile.  Read only if prune_bits is set
    // and *prune_on != 0 (both decided on the device before the scan).
    const uint32_t *prune_bits;
    int32_t prune_words;
    const int32_t *prune_on;
    // SAMPLE / DUMP output rows of stride ld
    float *out;
    int64_t ld;
    uint32_t *status;
};

struct KvMaps {
    CUtensorMap m[kNumStrideMaps];  // m[i]: kv rows 0, 2^i, 2*2^i, ... (m[0] = kv itself)
};

struct Item {
    int32_t tile;
    int32_t key0;   // first key (SAMPLE: first sample index j)
    int32_t kend;   // end key (SAMPLE: end sample index)
    int32_t nkt;    // key tiles in this item
    int32_t lg;     // SAMPLE: log2 of the stride
    int32_t base;   // SAMPLE: first sample index of the tile (output column 0)
};

__device__ __forceinline__ int64_t list_rows(const ScoreArgs &a)
{
    int64_t n = a.nrows;
    if (a.count_dev) {
        int64_t c = static_cast<int64_t>(*a.count_dev) - a.count_off;
        n = c < 0 ? 0 : (c < n ? c : n);
    }
    return n;
}

__device__ __forceinline__ bool window_ok(int64_t ks, int64_t ke, int64_t S)
{
    return ks >= 0 && ks <= ke && ke <= S;
}

// Query row of list position p, or -1 if the position is empty or the
// row's window is invalid (such rows are masked out of every tile).
__device__ __forceinline__ int32_t list_query(const ScoreArgs &a, int64_t p, int64_t nlist)
{
    if (p >= nlist) return -1;
    const int64_t t = a.rows ? a.rows[p] : p;
    if (t < 0 || t >= a.T) return -1;
    if (!window_ok(a.ks[t], a.ke[t], a.S)) return -1;
    return static_cast<int32_t>(t);
}

// True if the scan skips key tile kt of item m (its key block was pruned
// for the item's row tile).  Collect items start on a key-tile boundary.
__device__ __forceinline__ bool tile_pruned(const ScoreArgs &a, const Item &m, int kt)
{
    const int32_t blk = (m.key0 / kKeyTile) + kt;
    const uint32_t w = __ldg(a.prune_bits + static_cast<int64_t>(m.tile) * a.prune_words + (blk >> 5));
    return (w >> (blk & 31)) & 1u;
}

// Static schedules: a few rows (dense recovery of the rows a threshold
// missed, the dense path) must still spread over every SM, so the key chunk
// of an item shrinks until the row tiles in use give about one item per CTA
// (one query-tile load and one pipeline fill per CTA).
constexpr int kMinChunkTiles = 8;

struct Sched {
    int32_t chunk_keys;  // keys per item (static)
    int32_t chunks;      // items per row tile (static)
    int64_t tiles;       // row tiles in use (static)
};

template <int MODE, int RT>
__device__ __forceinline__ Sched make_sched(const ScoreArgs &a, int64_t nlist)
{
    Sched sc;
    sc.tiles = (nlist + RT - 1) / RT;
    sc.chunk_keys = kChunkKeys;
    sc.chunks = 0;
    if (MODE == MODE_DUMP) {  // the one static-schedule mode
        const int64_t kt = (a.S + kKeyTile - 1) / kKeyTile + 1;  // + 1: the aligned start
        // Row tiles split into as many chunks as give every CTA one item.
        const int64_t per = sc.tiles < gridDim.x ? gridDim.x / sc.tiles : 1;
        int64_t ct = (kt + per - 1) / per;
        ct = ct < kMinChunkTiles ? kMinChunkTiles : (ct > kChunkTiles ? kChunkTiles : ct);
        sc.chunk_keys = static_cast<int32_t>(ct * kKeyTile);
        sc.chunks = static_cast<int32_t>((kt + ct - 1) / ct);
    }
    return sc;
}

template <int MODE, int RT>
__device__ __forceinline__ bool get_item(const ScoreArgs &a, const Sched &sc, int it, int64_t nlist,
                                         Item &m)
{
    if (a.planned) {
        const int32_t nt = a.ntiles;
        if (it >= a.item_start[nt]) return false;
        int lo = 0, hi = nt;  // largest tile with item_start[tile] <= it
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (a.item_start[mid] <= it) lo = mid; else hi = mid;
        }
        m.tile = lo;
        const int chunk = it - a.item_start[lo];
        if (MODE == MODE_SAMPLE) {
            m.lg = a.tile_lg[lo];
            m.base = a.tile_lo[lo];
            m.key0 = m.base + chunk * a.chunk_keys;
            m.kend = min(a.tile_hi[lo], m.key0 + a.chunk_keys);
        } else {
            m.lg = 0;
            m.key0 = a.tile_lo[lo] + chunk * a.chunk_keys;
            m.kend = min(a.tile_hi[lo], m.key0 + a.chunk_keys);
        }
    } else {
        m.tile = it / sc.chunks;
        const int chunk = it - m.tile * sc.chunks;
        m.lg = 0;
        // The tile's rows and windows, every load issued before any is used.
        const int64_t p0 = static_cast<int64_t>(m.tile) * RT;
        int32_t tq[RT], wa[RT], wb[RT];
#pragma unroll
        for (int j = 0; j < RT; ++j)
            tq[j] = p0 + j < nlist ? (a.rows ? a.rows[p0 + j] : static_cast<int32_t>(p0 + j)) : -1;
#pragma unroll
        for (int j = 0; j < RT; ++j) {
            const bool in = tq[j] >= 0 && tq[j] < a.T;
            wa[j] = in ? a.ks[tq[j]] : 0;
            wb[j] = in ? a.ke[tq[j]] : -1;
        }
        int64_t lo = INT64_MAX, hi = -1;
#pragma unroll
        for (int j = 0; j < RT; ++j) {
            if (!window_ok(wa[j], wb[j], a.S) || wa[j] == wb[j]) continue;
            lo = min(lo, static_cast<int64_t>(wa[j]));
            hi = max(hi, static_cast<int64_t>(wb[j]));
        }
        if (hi < 0) return false;
        lo &= ~static_cast<int64_t>(kKeyTile - 1);
        const int64_t k0 = lo + static_cast<int64_t>(chunk) * sc.chunk_keys;
        if (k0 >= hi) return false;
        m.key0 = static_cast<int32_t>(k0);
        m.kend = static_cast<int32_t>(min(hi, k0 + sc.chunk_keys));
    }
    m.nkt = (m.kend - m.key0 + kKeyTile - 1) / kKeyTile;
    return m.nkt > 0;
}

// Next work item of this CTA (static round-robin over the item space), or
// false when there are no more.  Every role walks the same sequence.
template <int MODE, int RT>
__device__ __forceinline__ bool next_item(const ScoreArgs &a, const Sched &sc, int &it, int64_t nlist,
                                          Item &m)
{
    for (;; it += gridDim.x) {
        if (a.planned) {
            if (it >= a.item_start[a.ntiles]) return false;
        } else {
            if (it >= static_cast<int64_t>(sc.chunks) * sc.tiles) return false;
        }
        if (get_item<MODE, RT>(a, sc, it, nlist, m)) return true;
    }
}

__device__ __forceinline__ uint64_t pack2(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ void ffma2(uint64_t &acc, uint64_t a, uint64_t b)
{
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}

// ReLU on the ALU pipe: max(x, 0), NaN propagating.
__device__ __forceinline__ float relu_alu(float x)
{
    float r;
    asm("max.NaN.f32 %0, %1, 0f00000000;" : "=f"(r) : "f"(x));
    return r;
}

// Twice the ReLU on the FMA pipe: x + |x| (= 2x or +0; NaN propagates).  Its
// weight is pre-halved, so (w/2) * (x + |x|) is bit for bit w * ReLU(x).
__device__ __forceinline__ float relu2_fma(float x) { return __fadd_rn(x, fabsf(x)); }

// The head reduction of a (query, key) pair, sum_h w_h * max(x_h, 0): one
// packed fma chain per query whose two lanes hold the even and the odd
// heads, each advancing in head order with correctly rounded fmas, so that
//   I = sigma * (sum_{h even} w_h ReLU(x_h) + sum_{h odd} w_h ReLU(x_h)) + 0.0
// (the +0.0 turns a -0.0 into +0.0).  Every mode (sample, scan, dump) runs
// exactly this arithmetic, so the three see the same bits.
//
// One step covers two queries and heads h0 .. h0+15: xa / xb hold those 16
// columns of query 0 / 1, w0 / w1 point at the queries' 32 weights as
// stored (heads = 2, 3 mod 4 pre-halved).  Half of the ReLUs run on the ALU
// pipe and half on the FMA pipe.
__device__ __forceinline__ void head_step2(const float (&xa)[16], const float (&xb)[16],
                                           const float *w0, const float *w1, int h0,
                                           uint64_t &p, uint64_t &q)
{
#pragma unroll
    for (int h = 0; h < 16; h += 4) {
        const ulonglong2 wv = *reinterpret_cast<const ulonglong2 *>(w0 + h0 + h);
        const ulonglong2 wu = *reinterpret_cast<const ulonglong2 *>(w1 + h0 + h);
        ffma2(p, wv.x, pack2(relu_alu(xa[h + 0]), relu_alu(xa[h + 1])));
        ffma2(q, wu.x, pack2(relu_alu(xb[h + 0]), relu_alu(xb[h + 1])));
        ffma2(p, wv.y, pack2(relu2_fma(xa[h + 2]), relu2_fma(xa[h + 3])));
        ffma2(q, wu.y, pack2(relu2_fma(xb[h + 2]), relu2_fma(xb[h + 3])));
    }
}

// Stored weight of head h: heads = 2, 3 (mod 4) are halved (see head_step2).
__device__ __forceinline__ float stored_weight(float w, int h) { return (h & 2) ? 0.5f * w : w; }

__device__ __forceinline__ float head_finish(uint64_t p, float sigma)
{
    float even, odd;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(even), "=f"(odd) : "l"(p));
    return __fmaf_rn(sigma, __fadd_rn(even, odd), 0.0f);
}

// The score of a 64-head query held as two 32-head halves (p: heads 0..31,
// q: heads 32..63, each an even/odd pair of partial sums):
//   I = sigma * ((p.even + p.odd) + (q.even + q.odd)) + 0.0.
__device__ __forceinline__ float head_finish_pair(uint64_t p, uint64_t q, float sigma)
{
    float pe, po, qe, qo;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(pe), "=f"(po) : "l"(p));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(qe), "=f"(qo) : "l"(q));
    return __fmaf_rn(sigma, __fadd_rn(__fadd_rn(pe, po), __fadd_rn(qe, qo)), 0.0f);
}

template <int DT>
struct ScoreSmemLayout {
    using C = ScoreCfg<DT>;
    static constexpr int kQTileBytes = C::kAtoms * kQTile * kHeads * 128;  // 32 KB per atom
    static constexpr int kQBytes = C::kQG * kQTileBytes;
    static constexpr int kKBytes = C::kAtoms * kKeyTile * 128;             // 16 KB per atom
    static constexpr int kWarpQueries = C::kQG * kEpiQueries;              // queries per epilogue warp
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kQBytes;
    static constexpr int kStageEntries = kEpiWarps * kWarpQueries * C::kWarpStage;
    static constexpr int kOffStageVal = kOffK + C::kKStages * kKBytes;
    static constexpr int kOffStageIdx = kOffStageVal + kStageEntries * 4;
    static constexpr int kOffW = kOffStageIdx + kStageEntries * 4;
    static constexpr int kOffMisc = kOffW + kEpiWarps * kWarpQueries * kHeads * 4;
    static constexpr int kMiscBytes = 512;  // >= sizeof(ScoreMisc), checked below
    static constexpr int kBytes = kOffMisc + kMiscBytes + 1024;  // + alignment slack
};

struct ScoreMisc {
    uint64_t kv_full[4], kv_empty[4];
    uint64_t q_full, q_empty;
    uint64_t acc_full[2], acc_empty[2];
    uint64_t item_full[2], item_empty[2];  // the work-item queue (producer -> all roles)
    uint64_t final_bar;
    uint32_t tmem_base;
    int32_t abort;
    int32_t item_q[2];                     // item index, -1: no more items
    Item item_m[2];                        // the item itself (valid when item_q >= 0)
};

static_assert(sizeof(ScoreMisc) <= ScoreSmemLayout<FTK_F8E4M3>::kMiscBytes, "misc area");
static_assert(ScoreSmemLayout<FTK_F8E4M3>::kBytes <= 227 * 1024, "fp8 smem budget");
static_assert(ScoreSmemLayout<FTK_BF16>::kBytes <= 227 * 1024, "bf16 smem budget");
static_assert(ScoreCfg<FTK_F8E4M3>::kKStages <= 4 && ScoreCfg<FTK_BF16>::kKStages <= 4, "barriers");

// PR: the scan skips pruned key tiles.  With pruning possible, both
// COLLECT variants are launched and the one that does not match the
// device-side decision (*prune_on) returns at once, so an unpruned scan runs
// exactly the plain tile loop.
template <int DT, int MODE, bool PR, bool H64>
__global__ void __launch_bounds__(kScoreThreads, 1)
    score_kernel(const __grid_constant__ ScoreArgs a, const __grid_constant__ CUtensorMap tm_q,
                 const __grid_constant__ KvMaps kvm)
{
    griddep_wait();  // the previous kernel on the stream is complete
    griddep_launch_next();
    if (MODE == MODE_COLLECT && a.prune_bits != nullptr && ((*a.prune_on != 0) != PR)) return;
    using C = ScoreCfg<DT>;
    using Lay = ScoreSmemLayout<DT>;
    constexpr int QG = C::kQG;
    // H64: a 64-head query is two consecutive 32-head rows of the MMA tile
    // (the same bytes: q [T, 64, 128] == [2T, 32, 128]).
    constexpr int VPQ = H64 ? 2 : 1;     // MMA rows (32 heads each) per query
    constexpr int QPT = kQTile / VPQ;    // queries per MMA tile
    constexpr int RT = QG * QPT;         // queries per work item
    extern __shared__ uint8_t smem_dyn[];
    // 1024-byte alignment: the 128-byte swizzle pattern repeats every 8 rows.
    // (Offsetting the __shared__ array itself keeps every derived pointer
    // visibly in shared memory, so its loads and stores stay shared-space.)
    uint8_t *smem = smem_dyn + ((1024u - (smem_u32(smem_dyn) & 1023u)) & 1023u);
    uint8_t *sq = smem + Lay::kOffQ;
    uint8_t *sk = smem + Lay::kOffK;
    float *stage_val = reinterpret_cast<float *>(smem + Lay::kOffStageVal);
    int32_t *stage_idx = reinterpret_cast<int32_t *>(smem + Lay::kOffStageIdx);
    float *sw = reinterpret_cast<float *>(smem + Lay::kOffW);
    ScoreMisc &ms = *reinterpret_cast<ScoreMisc *>(smem + Lay::kOffMisc);
    volatile int *abort = &ms.abort;

    // The warp index through a shuffle from lane 0 is provably uniform over
    // the warp, so the values derived from it (role branches, TMEM
    // addresses) stay in uniform registers.
    const int warp = __shfl_sync(0xFFFFFFFFu, static_cast<int>(threadIdx.x >> 5), 0), lane = threadIdx.x & 31;
    const int64_t nlist = list_rows(a);
    if (nlist <= 0) return;  // e.g. a recovery pass with no rows left: no TMEM, no barriers
    const Sched sc = make_sched<MODE, RT>(a, nlist);
    constexpr bool pruned = MODE == MODE_COLLECT && PR;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::kKStages; ++i) {
            mbar_init(&ms.kv_full[i], 1);
            mbar_init(&ms.kv_empty[i], 1);
        }
        mbar_init(&ms.q_full, 1);
        mbar_init(&ms.q_empty, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&ms.acc_full[i], 1);
            mbar_init(&ms.acc_empty[i], kEpiWarps);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&ms.item_full[i], 1);
            mbar_init(&ms.item_empty[i], 1 + kEpiWarps);
        }
        mbar_init(&ms.final_bar, 1);
        ms.abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(&ms.tmem_base, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ms.tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (MODE == MODE_SAMPLE && lane != 0 && a.kv_scales) {
            // The idle lanes of the producer warp check a share of the
            // scales, which must be > 0 and finite (FTK_STATUS_BAD_SCALE:
            // the pruning's score bound assumes sigma > 0).
            bool bad = false;
            const int64_t stride = static_cast<int64_t>(gridDim.x) * 31;
            for (int64_t i = static_cast<int64_t>(blockIdx.x) * 31 + (lane - 1); i < a.S; i += stride) {
                const float sg = __ldg(a.kv_scales + i);
                bad |= !(sg > 0.f) || isinf(sg);
            }
            if (bad) set_status(a.status, FTK_STATUS_BAD_SCALE);
        }
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            int ks_ = 0;
            uint32_t kph = 0, qph = 0;
            int k_armed[4] = {0, 0, 0, 0};  // loads issued per stage, for the abort drain
            uint32_t k_armed_ph[4] = {0, 0, 0, 0};
            int q_armed = 0;
            uint32_t q_armed_ph = 0;
            Item m;
            // Work items: taken from the shared counter (dynamic: a CTA that
            // finishes early takes more) or in the static round-robin order,
            // and handed to the MMA and epilogue roles through the queue.
            const bool dynamic = a.planned && a.work_next != nullptr;
            const int32_t total = a.planned ? a.item_start[a.ntiles] : 0;
            int islot = 0, it_s = blockIdx.x;
            uint32_t iph = 0;
            for (;;) {
                int it = -1;
                if (!*abort) {
                    if (dynamic) {
                        it = atomicAdd(a.work_next, 1);
                        if (it >= total) it = -1;
                        else get_item<MODE, RT>(a, sc, it, nlist, m);
                    } else if (next_item<MODE, RT>(a, sc, it_s, nlist, m)) {
                        it = it_s;
                        it_s += gridDim.x;
                    }
                }
                // The item's query rows, every load issued before any is
                // used (list position -> row -> window).
                int32_t tq[RT];
                if (it >= 0) {
                    const int64_t p0 = static_cast<int64_t>(m.tile) * RT;
#pragma unroll
                    for (int j = 0; j < RT; ++j)
                        tq[j] = p0 + j < nlist ? (a.rows ? a.rows[p0 + j] : static_cast<int32_t>(p0 + j)) : -1;
#pragma unroll
                    for (int j = 0; j < RT; ++j) {  // placeholder rows are masked in the epilogue
                        const bool in = tq[j] >= 0 && tq[j] < a.T;
                        if (!in || !window_ok(a.ks[tq[j]], a.ke[tq[j]], a.S)) tq[j] = 0;
                    }
                }
                if (!mbar_wait(&ms.item_empty[islot], iph ^ 1u, abort, a.status)) break;
                ms.item_q[islot] = it;
                if (it >= 0) ms.item_m[islot] = m;  // the other roles read it, not recompute it
                mbar_arrive(&ms.item_full[islot]);
                if (++islot == 2) { islot = 0; iph ^= 1u; }
                if (it < 0) break;
                // The query group: the 32 head rows of each of RT queries.
                if (!mbar_wait(&ms.q_empty, qph ^ 1u, abort, a.status)) break;
                mbar_arrive_expect_tx(&ms.q_full, Lay::kQBytes);
                q_armed = 1;
                q_armed_ph = qph;
                for (int vt = 0; vt < QG; ++vt) {
                    for (int j = 0; j < kQTile; ++j) {  // MMA row j: half j % VPQ of query j / VPQ
                        const int32_t t = tq[vt * QPT + j / VPQ];
                        for (int at = 0; at < C::kAtoms; ++at)
                            tma_load_2d(sq + vt * Lay::kQTileBytes + at * (Lay::kQTileBytes / C::kAtoms) +
                                            j * kHeads * 128,
                                        &tm_q, &ms.q_full, at * 64, (t * VPQ + j % VPQ) * kHeads);
                    }
                }
                qph ^= 1u;
                const CUtensorMap *map = &kvm.m[MODE == MODE_SAMPLE ? m.lg : 0];
                for (int kt = 0; kt < m.nkt; ++kt) {
                    if (pruned && tile_pruned(a, m, kt)) continue;
                    if (!mbar_wait(&ms.kv_empty[ks_], kph ^ 1u, abort, a.status)) break;
                    mbar_arrive_expect_tx(&ms.kv_full[ks_], Lay::kKBytes);
                    k_armed[ks_] = 1;
                    k_armed_ph[ks_] = kph;
                    const int32_t y = m.key0 + kt * kKeyTile;
                    for (int at = 0; at < C::kAtoms; ++at)
                        tma_load_2d(sk + ks_ * Lay::kKBytes + at * (Lay::kKBytes / C::kAtoms), map,
                                    &ms.kv_full[ks_], at * 64, y);
                    if (++ks_ == C::kKStages) { ks_ = 0; kph ^= 1u; }
                }
            }
            if (*abort) {
                // Drain: every issued TMA load lands before the CTA exits.
                for (int i = 0; i < C::kKStages; ++i)
                    if (k_armed[i]) mbar_wait_drain(&ms.kv_full[i], k_armed_ph[i]);
                if (q_armed) mbar_wait_drain(&ms.q_full, q_armed_ph);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int ks_ = 0, ab = 0;
            uint32_t kph = 0, qph = 0, aph = 0;
            bool issued = false, ok = true;
            Item m;
            int islot = 0;
            uint32_t iph = 0;
            while (ok && !*abort) {
                if (!mbar_wait(&ms.item_full[islot], iph, abort, a.status)) break;
                const int it = *reinterpret_cast<volatile int32_t *>(&ms.item_q[islot]);
                if (it >= 0) m = ms.item_m[islot];
                mbar_arrive(&ms.item_empty[islot]);
                if (++islot == 2) { islot = 0; iph ^= 1u; }
                if (it < 0) break;
                if (!mbar_wait(&ms.q_full, qph, abort, a.status)) break;
                qph ^= 1u;
                tc_fence_after();
                const uint32_t qaddr = smem_u32(sq);
                for (int kt = 0; kt < m.nkt && ok; ++kt) {
                    if (pruned && tile_pruned(a, m, kt)) continue;
                    if (!mbar_wait(&ms.kv_full[ks_], kph, abort, a.status)) {
                        ok = false;
                        break;
                    }
                    const uint32_t kaddr = smem_u32(sk + ks_ * Lay::kKBytes);
#pragma unroll
                    for (int vt = 0; vt < QG; ++vt) {
                        if (!mbar_wait(&ms.acc_empty[ab], aph ^ 1u, abort, a.status)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t d = tmem + static_cast<uint32_t>(ab * 256);
                        const uint32_t baddr = qaddr + vt * Lay::kQTileBytes;
#pragma unroll
                        for (int kk = 0; kk < C::kMmaK; ++kk) {
                            const int at = kk / 4, off = (kk % 4) * 32;
                            const uint64_t ad = smem_desc_sw128(kaddr + at * (Lay::kKBytes / C::kAtoms) + off);
                            const uint64_t bd = smem_desc_sw128(baddr + at * (Lay::kQTileBytes / C::kAtoms) + off);
                            if (DT == FTK_F8E4M3)
                                mma_f8f6f4(d, ad, bd, C::kIdesc, kk > 0 ? 1u : 0u);
                            else
                                mma_f16(d, ad, bd, C::kIdesc, kk > 0 ? 1u : 0u);
                        }
                        issued = true;
                        mma_commit(&ms.acc_full[ab]);
                        if (++ab == 2) { ab = 0; aph ^= 1u; }
                    }
                    mma_commit(&ms.kv_empty[ks_]);  // key tile free once its MMAs are done
                    if (++ks_ == C::kKStages) { ks_ = 0; kph ^= 1u; }
                }
                mma_commit(&ms.q_empty);
            }
            // Every issued MMA completes before TMEM is released.
            if (issued) {
                mma_commit(&ms.final_bar);
                mbar_wait_drain(&ms.final_bar, 0);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // Each epilogue warp works on its own: its queries' parameters and
        // weights, and its own candidate staging, so the tile loop has no
        // cross-warp synchronisation besides releasing the accumulator.
        constexpr int NQ = kEpiQueries;          // MMA rows per warp per query tile (2)
        constexpr int NR = NQ / VPQ;             // queries per warp per query tile
        constexpr int WQ = QG * NR;              // queries per warp
        const int ew = warp - 2;                 // 0..15
        const int quad = warp & 3;               // TMEM lane quarter
        const int qg = ew >> 2;                  // query pair within each query tile
        const int key_lane = quad * 32 + lane;   // row of the 128-key tile
        const uint32_t tlane = tmem + (static_cast<uint32_t>(quad * 32) << 16);
        const uint32_t lt_mask = (1u << lane) - 1u;
        float *my_w = sw + ew * QG * NQ * kHeads;  // by MMA row: (vt * NQ + r) * 32 + head
        float *my_sv = stage_val + ew * WQ * C::kWarpStage;
        int32_t *my_si = stage_idx + ew * WQ * C::kWarpStage;
        int ab = 0;
        uint32_t aph = 0;
        bool bad_scale = false;
        Item m;
        int islot = 0;
        uint32_t iph = 0;
        while (!*abort) {
            const bool got_item = mbar_wait(&ms.item_full[islot], iph, abort, a.status);
            if (!__all_sync(0xFFFFFFFFu, got_item)) break;
            const int it = *reinterpret_cast<volatile int32_t *>(&ms.item_q[islot]);
            if (it >= 0) m = ms.item_m[islot];
            __syncwarp();  // every lane has the item before the slot is released
            if (lane == 0) mbar_arrive(&ms.item_empty[islot]);
            if (++islot == 2) { islot = 0; iph ^= 1u; }
            if (it < 0) break;
            // Per-item parameters of this warp's queries (warp-uniform).  Slot
            // qq = vt * NR + qi is query qg * NR + qi of query tile vt, whose
            // MMA rows are qg * NQ + qi * VPQ + (0 .. VPQ - 1).
            int32_t qt[WQ], qpos[WQ], wlo[WQ], wlen[WQ];
            float qtau[WQ];
            {
                const int sl = lane % WQ;
                const int64_t p = static_cast<int64_t>(m.tile) * RT + (sl / NR) * QPT + qg * NR + (sl % NR);
                int32_t t_l = -1, ks_l = 0, ke_l = 0;
                float tau_l = 0.f;
                if (lane < WQ) {
                    t_l = list_query(a, p, nlist);
                    if (t_l >= 0) {
                        ks_l = a.ks[t_l];
                        ke_l = a.ke[t_l];
                        if (MODE == MODE_COLLECT) tau_l = a.tau[t_l];
                    }
                }
#pragma unroll
                for (int qq = 0; qq < WQ; ++qq) {
                    qt[qq] = __shfl_sync(0xFFFFFFFFu, t_l, qq);
                    wlo[qq] = __shfl_sync(0xFFFFFFFFu, ks_l, qq);
                    wlen[qq] = __shfl_sync(0xFFFFFFFFu, ke_l, qq) - wlo[qq];
                    qtau[qq] = __shfl_sync(0xFFFFFFFFu, tau_l, qq);
                    qpos[qq] = m.tile * RT + (qq / NR) * QPT + qg * NR + (qq % NR);
#pragma unroll
                    for (int v = 0; v < VPQ; ++v)
                        my_w[((qq / NR) * NQ + (qq % NR) * VPQ + v) * kHeads + lane] =
                            qt[qq] >= 0 ? stored_weight(a.weights[(static_cast<int64_t>(qt[qq]) * VPQ + v) * kHeads +
                                                                  lane],
                                                        lane)
                                        : 0.f;
                }
                __syncwarp();
            }
            int cnt[WQ];  // staged candidates per query (warp-uniform)
#pragma unroll
            for (int qq = 0; qq < WQ; ++qq) cnt[qq] = 0;
            bool flush_due = false;  // some staging could overflow within one more key tile
            // Keys are int32 (S < 2^31).  A query outside the list has the
            // empty window [0, 0).  In SAMPLE mode key j of the tile is
            // sample j, at kv row j << lg.
            const float *scales = a.kv_scales;
            int32_t kidx_next = m.key0 + key_lane;
            float sig_next = 1.f;
            if (scales) {
                const int64_t s0 = static_cast<int64_t>(kidx_next) << m.lg;
                if (kidx_next < m.kend && s0 < a.S) sig_next = __ldg(scales + s0);
            }
            bool ok = true;
            for (int kt = 0; kt < m.nkt && ok; ++kt) {
                const int32_t kidx = kidx_next;
                const float sigma = sig_next;
                kidx_next += kKeyTile;
                if (scales && kt + 1 < m.nkt) {  // sigma one tile ahead
                    if (MODE == MODE_SAMPLE) {
                        const int64_t s1 = static_cast<int64_t>(kidx_next) << m.lg;
                        sig_next = (kidx_next < m.kend && s1 < a.S) ? __ldg(scales + s1) : 1.f;
                    } else {  // unit stride, kend <= S
                        sig_next = kidx_next < m.kend ? __ldg(scales + kidx_next) : 1.f;
                    }
                }
                const bool skip = pruned && tile_pruned(a, m, kt);  // warp-uniform
                // (The sample pass validates every scale; the dense dump
                // checks the ones it reads.)
                if (MODE == MODE_DUMP)
                    bad_scale |= !skip && scales && kidx < m.kend && (!(sigma > 0.f) || isinf(sigma));
                const int32_t s = MODE == MODE_SAMPLE ? (kidx << m.lg) : kidx;
                if (!skip) {
#pragma unroll
                for (int vt = 0; vt < QG; ++vt) {
                    // With two query tiles per key tile, tile vt always uses
                    // accumulator vt (every key tile consumes both).
                    const int abx = QG == 2 ? vt : ab;
                    const bool got = mbar_wait(&ms.acc_full[abx], aph, abort, a.status);
                    if (!__all_sync(0xFFFFFFFFu, got)) {  // also reconverges the warp
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t c0 = tlane + static_cast<uint32_t>(abx * 256 + qg * NQ * 32);
                    const float *w0 = my_w + (vt * NQ) * kHeads;
                    uint64_t p = 0, q = 0;  // (+0.0, +0.0)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        float xa[16], xb[16];
                        tmem_ld16x2(c0 + hh * 16, c0 + 32 + hh * 16, xa, xb);
                        if (hh == 1) {
                            // Every column of this tile is in registers: hand the
                            // accumulator back to the MMA warp.
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&ms.acc_empty[abx]);
                        }
                        head_step2(xa, xb, w0, w0 + kHeads, hh * 16, p, q);
                    }
                    if (QG == 2) {
                        if (vt == 1) aph ^= 1u;
                    } else if (++ab == 2) {
                        ab = 0;
                        aph ^= 1u;
                    }
                    float I[NR];
                    if constexpr (H64) {
                        I[0] = head_finish_pair(p, q, sigma);
                    } else {
                        I[0] = head_finish(p, sigma);
                        I[1] = head_finish(q, sigma);
                    }
                    if (MODE == MODE_COLLECT) {
                        // Candidates are rare: one vote for both queries, the
                        // staging only when some lane has one.
                        bool take[NR];
                        bool anyt = false;
#pragma unroll
                        for (int qi = 0; qi < NR; ++qi) {
                            const int qq = vt * NR + qi;
                            // s in [wlo, wlo + wlen) as one unsigned compare
                            const bool valid = static_cast<uint32_t>(s - wlo[qq]) < static_cast<uint32_t>(wlen[qq]);
                            take[qi] = valid && !(I[qi] < qtau[qq]);  // NaN is kept, to be seen
                            anyt |= take[qi];
                        }
                        if (__any_sync(0xFFFFFFFFu, anyt)) {
#pragma unroll
                            for (int qi = 0; qi < NR; ++qi) {
                                const int qq = vt * NR + qi;
                                const uint32_t bal = __ballot_sync(0xFFFFFFFFu, take[qi]);
                                const int pos = cnt[qq] + __popc(bal & lt_mask);
                                if (take[qi]) {
                                    my_sv[qq * C::kWarpStage + pos] = I[qi];
                                    my_si[qq * C::kWarpStage + pos] = s;
                                }
                                cnt[qq] += __popc(bal);
                                flush_due |= cnt[qq] > C::kWarpStage - 32;
                            }
                        }
                    }
#pragma unroll
                    for (int qi = 0; qi < (MODE == MODE_COLLECT ? 0 : NR); ++qi) {
                        const int qq = vt * NR + qi;
                        const bool valid = static_cast<uint32_t>(s - wlo[qq]) < static_cast<uint32_t>(wlen[qq]);
                        if (MODE == MODE_SAMPLE) {
                            if (qt[qq] >= 0 && kidx < m.kend)
                                a.out[static_cast<int64_t>(qt[qq]) * a.ld + (kidx - m.base)] =
                                    valid ? I[qi] : -INFINITY;
                        } else {
                            if (valid) a.out[static_cast<int64_t>(qpos[qq]) * a.ld + (s - wlo[qq])] = I[qi];
                        }
                    }
                }
                }
                if (MODE == MODE_COLLECT && ok) {
                    // A key tile adds <= 32 entries per warp and query: flush
                    // the queries whose staging could overflow in the next
                    // tile, and everything at the item's end.
                    const bool last = kt == m.nkt - 1;
                    if (last || flush_due) {
                        flush_due = false;
                        bool need[WQ], any = false;
#pragma unroll
                        for (int qq = 0; qq < WQ; ++qq) {
                            need[qq] = cnt[qq] > 0 && (last || cnt[qq] > C::kWarpStage - 32);
                            any |= need[qq];
                        }
                        if (any) {
                            __syncwarp();  // staged entries visible to every lane
                            int base[WQ];
#pragma unroll
                            for (int qq = 0; qq < WQ; ++qq) base[qq] = 0;
                            if (lane == 0) {
#pragma unroll
                                for (int qq = 0; qq < WQ; ++qq)  // independent atomics, latencies overlap
                                    if (need[qq] && qt[qq] >= 0) base[qq] = atomicAdd(a.cnt + qt[qq], cnt[qq]);
                            }
#pragma unroll
                            for (int qq = 0; qq < WQ; ++qq) {
                                if (!need[qq]) continue;
                                const int b = __shfl_sync(0xFFFFFFFFu, base[qq], 0);
                                if (qt[qq] >= 0) {
                                    float *cv = a.cand_val + static_cast<int64_t>(qt[qq]) * a.cap;
                                    int32_t *ci = a.cand_idx + static_cast<int64_t>(qt[qq]) * a.cap;
                                    for (int i = lane; i < cnt[qq]; i += 32) {
                                        const int slot = b + i;
                                        if (slot < a.cap) {
                                            cv[slot] = my_sv[qq * C::kWarpStage + i];
                                            ci[slot] = my_si[qq * C::kWarpStage + i];
                                        }
                                    }
                                }
                                cnt[qq] = 0;
                            }
                            __syncwarp();
                        }
                    }
                }
            }
            if (!ok) break;
        }
        if (bad_scale) set_status(a.status, FTK_STATUS_BAD_SCALE);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace ftk
