// ftk_prune.cu -- the kernels of score-bound key pruning (the bound, its
// margin and the per-call decision are described in ftk_prune.cuh), and the
// ftk_block_bound entry point that exposes the bound itself.
#include <cuda_fp8.h>

#include "ftk_host.h"
#include "ftk_prune.cuh"

namespace ftk {

constexpr int kBoxThreads = 256;

// ---------------------------------------------------------------------------
// box: c, r and M_B of every 128-key block
// ---------------------------------------------------------------------------

// The raw bits of four consecutive elements of kv row s from dim 4*g
// (FP8: one word; BF16: two words, the second unused for FP8).
template <int DT>
__device__ __forceinline__ uint2 load4_raw(const void *kv, int64_t s, int g)
{
    if (DT == FTK_F8E4M3)
        return make_uint2(__ldg(reinterpret_cast<const uint32_t *>(static_cast<const uint8_t *>(kv) + s * kDim) + g), 0u);
    return __ldg(reinterpret_cast<const uint2 *>(static_cast<const uint16_t *>(kv) + s * kDim) + g);
}

template <int DT>
__device__ __forceinline__ void unpack4(uint2 x, float (&v)[4])
{
    if (DT == FTK_F8E4M3) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(
                static_cast<__nv_fp8x2_storage_t>((x.x >> (16 * i)) & 0xFFFFu), __NV_E4M3);
            v[2 * i] = __half2float(__half(__half_raw{h.x}));
            v[2 * i + 1] = __half2float(__half(__half_raw{h.y}));
        }
    } else {
        v[0] = __uint_as_float(x.x << 16);
        v[1] = __uint_as_float(x.x & 0xFFFF0000u);
        v[2] = __uint_as_float(x.y << 16);
        v[3] = __uint_as_float(x.y & 0xFFFF0000u);
    }
}

// One CTA per block: warp w takes keys w, w+8, ...; lane g dims 4g..4g+3.
template <int DT>
__global__ void __launch_bounds__(kBoxThreads) box_kernel(const BoxArgs a)
{
    griddep_wait();  // the previous kernel on the stream is complete
    griddep_launch_next();
    __shared__ float sh_hi[8][kDim], sh_lo[8][kDim];
    __shared__ float sh_m[8];
    __shared__ int sh_bad;
    const int b = blockIdx.x;
    const int warp = threadIdx.x >> 5, g = threadIdx.x & 31;
    if (threadIdx.x == 0) sh_bad = 0;
    float hi[4], lo[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        hi[i] = -INFINITY;
        lo[i] = INFINITY;
    }
    bool bad = false;
    const int64_t s0 = static_cast<int64_t>(b) * kBlockKeys;
    // All 16 loads of the warp in flight at once, then the reduction.
    constexpr int kPer = kBlockKeys / 8;
    uint2 raw[kPer];
    float sig[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
        const int64_t s = s0 + warp + 8 * j;
        const bool in = s < a.S;
        raw[j] = in ? load4_raw<DT>(a.kv, s, g) : make_uint2(0u, 0u);
        sig[j] = in && a.kv_scales ? __ldg(a.kv_scales + s) : 1.f;
    }
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
        if (s0 + warp + 8 * j >= a.S) break;
        bad |= !(sig[j] > 0.f) || isinf(sig[j]);
        float v[4];
        unpack4<DT>(raw[j], v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float x = sig[j] * v[i];
            bad |= !isfinite(x);
            hi[i] = fmaxf(hi[i], x);
            lo[i] = fminf(lo[i], x);
        }
    }
    __syncthreads();
    if (bad) sh_bad = 1;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        sh_hi[warp][4 * g + i] = hi[i];
        sh_lo[warp][4 * g + i] = lo[i];
    }
    __syncthreads();
    float m = 0.f;
    if (threadIdx.x < kDim) {
        const int d = threadIdx.x;
        float h = sh_hi[0][d], l = sh_lo[0][d];
#pragma unroll
        for (int w = 1; w < 8; ++w) {
            h = fmaxf(h, sh_hi[w][d]);
            l = fminf(l, sh_lo[w][d]);
        }
        float *box = a.box + static_cast<int64_t>(b) * 2 * kDim;
        box[d] = 0.5f * (h + l);
        box[kDim + d] = 0.5f * (h - l);
        m = fmaxf(fabsf(h), fabsf(l));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if (g == 0) sh_m[warp] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float mm = sh_m[0];
        for (int w = 1; w < kDim / 32; ++w) mm = fmaxf(mm, sh_m[w]);
        a.mb[b] = sh_bad ? INFINITY : mm;
    }
}

// ---------------------------------------------------------------------------
// bound: UB of (row, block) pairs, one warp per row, lane = head
// ---------------------------------------------------------------------------

// The 128 elements of q[t, h] as floats (exact: e4m3 and bf16 are subsets
// of float32).
template <int DT>
__device__ __forceinline__ void load_q(const void *q, int64_t row, float (&qf)[kDim])
{
    if (DT == FTK_F8E4M3) {
        const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(q) + row * kDim);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint4 x = __ldg(src + i);
            const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(
                        static_cast<__nv_fp8x2_storage_t>((w[j] >> (16 * k)) & 0xFFFFu), __NV_E4M3);
                    qf[16 * i + 4 * j + 2 * k] = __half2float(__half(__half_raw{h.x}));
                    qf[16 * i + 4 * j + 2 * k + 1] = __half2float(__half(__half_raw{h.y}));
                }
            }
        }
    } else {
        const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(q) + row * kDim);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint4 x = __ldg(src + i);
            const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                qf[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
                qf[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
            }
        }
    }
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

constexpr int kBoundWarps = 8;  // a warp takes rows warp, warp + 8 of the row tile

struct BoundSmem {
    float box[kBoundWordBlocks][2 * kDim];
    float mb[kBoundWordBlocks];
    int32_t blk[kBoundWordBlocks];
    uint32_t pass[kBoundWarps];
    float ub[kBoundWarps][kBoundWordBlocks];  // 64 heads: a row's bound, summed over its two halves
    int32_t nblk;
};

// Work items.  EST: (sampled tile, chunk of kEstChunk sampled blocks).
// FULL: (row tile, bitmap word) over every word meeting the tile's scan
// range.  OUT: (row tile, word) over all blocks.
// H: the indexer's heads.  32: lane = head.  64: lane = heads lane and
// lane + 32, taken in two passes (q of one head is 128 floats in registers).
template <int DT, int MODE, int H>
__global__ void __launch_bounds__(kBoundWarps * 32, 1) bound_kernel(const BoundArgs a)
{
    griddep_wait();  // the previous kernel on the stream is complete
    griddep_launch_next();
    __shared__ BoundSmem sm;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (MODE == BOUND_FULL) {
        bool on;
        if (a.mode != 0) {
            on = true;
        } else {
            const uint32_t tot = *a.est_total, pr = *a.est_pruned;
            on = tot > 0 && static_cast<float>(pr) >= kPruneCutoff * static_cast<float>(tot);
        }
        if (blockIdx.x == 0 && threadIdx.x == 0) *a.prune_enabled = on ? 1 : 0;
        if (!on) return;
    }
    const int64_t nitems = MODE == BOUND_EST ? static_cast<int64_t>(a.est_tiles) * (kEstBlocks / kEstChunk)
                                             : static_cast<int64_t>(a.ntiles) * a.nwords;
    for (int64_t it = blockIdx.x; it < nitems; it += gridDim.x) {
        int32_t tile, word = 0, b0 = 0, b1 = a.nblocks;
        if (MODE == BOUND_EST) {
            const int i = static_cast<int>(it / (kEstBlocks / kEstChunk));
            tile = static_cast<int32_t>(static_cast<int64_t>(i) * a.ntiles / a.est_tiles);
        } else {
            tile = static_cast<int32_t>(it / a.nwords);
            word = static_cast<int32_t>(it % a.nwords);
        }
        if (MODE != BOUND_OUT) {
            const int32_t lo = a.c_lo[tile], hi = a.c_hi[tile];
            if (hi <= lo) continue;  // tile with no key to scan
            b0 = lo / kBlockKeys;
            b1 = (hi + kBlockKeys - 1) / kBlockKeys;
        }
        // blocks of this item
        if (threadIdx.x == 0) {
            int n = 0;
            if (MODE == BOUND_EST) {
                const int nbr = b1 - b0;
                const int nsb = nbr < kEstBlocks ? nbr : kEstBlocks;
                const int u0 = static_cast<int>(it % (kEstBlocks / kEstChunk)) * kEstChunk;
                for (int u = u0; u < u0 + kEstChunk && u < nsb; ++u)
                    sm.blk[n++] = b0 + static_cast<int32_t>(static_cast<int64_t>(u) * nbr / nsb);
            } else {
                const int32_t w0 = word * kBoundWordBlocks;
                for (int j = 0; j < kBoundWordBlocks; ++j)
                    if (w0 + j >= b0 && w0 + j < b1) sm.blk[n++] = w0 + j;
            }
            sm.nblk = n;
        }
        __syncthreads();
        const int nblk = sm.nblk;
        if (nblk == 0) {
            __syncthreads();
            continue;
        }
        for (int i = threadIdx.x; i < nblk * (2 * kDim / 4); i += blockDim.x) {
            const int j = i / (2 * kDim / 4), e = i % (2 * kDim / 4);
            reinterpret_cast<float4 *>(sm.box[j])[e] =
                __ldg(reinterpret_cast<const float4 *>(a.box + static_cast<int64_t>(sm.blk[j]) * 2 * kDim) + e);
        }
        if (threadIdx.x < nblk) sm.mb[threadIdx.x] = __ldg(a.mb + sm.blk[threadIdx.x]);

        __syncthreads();
        uint32_t pass = 0xFFFFFFFFu;  // AND over this warp's rows
        for (int rr = warp; rr < a.rt; rr += kBoundWarps) {
            const int64_t t = static_cast<int64_t>(tile) * a.rt + rr;
            bool row_ok = t < a.T;
            int32_t wks = 0, wke = 0;
            float tau = 0.f;
            if (row_ok && MODE != BOUND_OUT) {
                wks = a.ks[t];
                wke = a.ke[t];
                row_ok = wks >= 0 && wks < wke && wke <= a.S;
                tau = a.tau[t];
            }
            if (!row_ok) continue;  // masked row: no constraint
            uint32_t row_pass = 0;
            if constexpr (H == 32) {
                float qf[kDim];
                load_q<DT>(a.q, t * kHeads + lane, qf);
                const float w = a.weights[t * kHeads + lane];
                float l1 = 0.f;
#pragma unroll
                for (int i = 0; i < kDim; ++i) l1 += fabsf(qf[i]);
                const float A = warp_sum(fabsf(w) * l1);            // sum_h |w_h| |q_h|_1
                const float P = warp_sum(w >= 0.f ? w * l1 : 0.f);  // sum_{w_h >= 0} w_h |q_h|_1
                for (int j = 0; j < nblk; ++j) {
                    const int32_t B = sm.blk[j];
                    const float M = sm.mb[j];
                    if (MODE != BOUND_OUT) {
                        const int32_t k0 = B * kBlockKeys;
                        if (!(wks < k0 + kBlockKeys && wke > k0)) {  // window misses the block
                            row_pass |= 1u << j;
                            continue;
                        }
                        if (!(M < INFINITY)) continue;  // never skipped
                        if (P * M + kPruneEps * A * M < tau) {
                            row_pass |= 1u << j;  // |U_h| <= |q_h|_1 M_B: the coarse bound decides
                            continue;
                        }
                    }
                    const float4 *c4 = reinterpret_cast<const float4 *>(sm.box[j]);
                    const float4 *r4 = c4 + kDim / 4;
                    float a0 = 0.f, a1 = 0.f, e0 = 0.f, e1 = 0.f;
#pragma unroll
                    for (int i = 0; i < kDim / 4; ++i) {
                        const float4 c = c4[i], r = r4[i];
                        const float *x = qf + 4 * i;
                        a0 = fmaf(x[0], c.x, a0);
                        e0 = fmaf(fabsf(x[0]), r.x, e0);
                        a1 = fmaf(x[1], c.y, a1);
                        e1 = fmaf(fabsf(x[1]), r.y, e1);
                        a0 = fmaf(x[2], c.z, a0);
                        e0 = fmaf(fabsf(x[2]), r.z, e0);
                        a1 = fmaf(x[3], c.w, a1);
                        e1 = fmaf(fabsf(x[3]), r.w, e1);
                    }
                    const float mid = a0 + a1, rad = e0 + e1;
                    const float term = w >= 0.f ? w * fmaxf(mid + rad, 0.f) : w * fmaxf(mid - rad, 0.f);
                    const float ub = warp_sum(term);
                    if (MODE == BOUND_OUT) {
                        if (lane == 0) a.out[t * a.ld + B] = M < INFINITY ? ub : INFINITY;
                    } else if (ub + kPruneEps * A * M < tau) {
                        row_pass |= 1u << j;
                    }
                }
            } else {
                constexpr int NH = H / kHeads;  // head halves per lane
                float A = 0.f, P = 0.f;          // sum_h |w_h| |q_h|_1 and sum_{w_h >= 0} w_h |q_h|_1
#pragma unroll 1
                for (int hh = 0; hh < NH; ++hh) {
                    float qf[kDim];
                    load_q<DT>(a.q, (t * NH + hh) * kHeads + lane, qf);
                    const float w = a.weights[t * H + hh * kHeads + lane];
                    float l1 = 0.f;
#pragma unroll
                    for (int i = 0; i < kDim; ++i) l1 += fabsf(qf[i]);
                    A += warp_sum(fabsf(w) * l1);
                    P += warp_sum(w >= 0.f ? w * l1 : 0.f);
                }
                uint32_t fine = 0;  // blocks the coarse bound does not decide
                for (int j = 0; j < nblk; ++j) {
                    if (MODE != BOUND_OUT) {
                        const float M = sm.mb[j];
                        const int32_t k0 = sm.blk[j] * kBlockKeys;
                        if (!(wks < k0 + kBlockKeys && wke > k0)) {  // window misses the block
                            row_pass |= 1u << j;
                            continue;
                        }
                        if (!(M < INFINITY)) continue;  // never skipped
                        if (P * M + kPruneEps * A * M < tau) {
                            row_pass |= 1u << j;
                            continue;
                        }
                    }
                    fine |= 1u << j;
                }
#pragma unroll 1
                for (int hh = 0; hh < NH; ++hh) {
                    float qf[kDim];
                    load_q<DT>(a.q, (t * NH + hh) * kHeads + lane, qf);
                    const float w = a.weights[t * H + hh * kHeads + lane];
                    for (int j = 0; j < nblk; ++j) {
                        if (!((fine >> j) & 1u)) continue;
                        const float4 *c4 = reinterpret_cast<const float4 *>(sm.box[j]);
                        const float4 *r4 = c4 + kDim / 4;
                        float a0 = 0.f, a1 = 0.f, e0 = 0.f, e1 = 0.f;
#pragma unroll
                        for (int i = 0; i < kDim / 4; ++i) {
                            const float4 c = c4[i], r = r4[i];
                            const float *x = qf + 4 * i;
                            a0 = fmaf(x[0], c.x, a0);
                            e0 = fmaf(fabsf(x[0]), r.x, e0);
                            a1 = fmaf(x[1], c.y, a1);
                            e1 = fmaf(fabsf(x[1]), r.y, e1);
                            a0 = fmaf(x[2], c.z, a0);
                            e0 = fmaf(fabsf(x[2]), r.z, e0);
                            a1 = fmaf(x[3], c.w, a1);
                            e1 = fmaf(fabsf(x[3]), r.w, e1);
                        }
                        const float mid = a0 + a1, rad = e0 + e1;
                        const float term = w >= 0.f ? w * fmaxf(mid + rad, 0.f) : w * fmaxf(mid - rad, 0.f);
                        const float part = warp_sum(term);
                        if (lane == 0) sm.ub[warp][j] = hh == 0 ? part : sm.ub[warp][j] + part;
                    }
                }
                __syncwarp();
                for (int j = 0; j < nblk; ++j) {
                    if (!((fine >> j) & 1u)) continue;
                    const float ub = sm.ub[warp][j], M = sm.mb[j];
                    if (MODE == BOUND_OUT) {
                        if (lane == 0) a.out[t * a.ld + sm.blk[j]] = M < INFINITY ? ub : INFINITY;
                    } else if (ub + kPruneEps * A * M < tau) {
                        row_pass |= 1u << j;
                    }
                }
                __syncwarp();  // sm.ub is read before the next row writes it
            }
            pass &= row_pass;
        }
        if (MODE != BOUND_OUT) {
            if (lane == 0) sm.pass[warp] = pass;
            __syncthreads();
            if (threadIdx.x == 0) {
                uint32_t all = (nblk == 32) ? 0xFFFFFFFFu : ((1u << nblk) - 1u);
                for (int r = 0; r < kBoundWarps; ++r) all &= sm.pass[r];
                if (MODE == BOUND_EST) {
                    atomicAdd(a.est_total, static_cast<uint32_t>(nblk));
                    atomicAdd(a.est_pruned, static_cast<uint32_t>(__popc(all)));
                } else {
                    // bit j of the word is block word*32 + j; blocks outside
                    // the range are never queried by the scan
                    uint32_t bitsw = 0;
                    for (int j = 0; j < nblk; ++j)
                        if ((all >> j) & 1u) bitsw |= 1u << (sm.blk[j] - word * kBoundWordBlocks);
                    a.bits[static_cast<int64_t>(tile) * a.nwords + word] = bitsw;
                    if (bitsw) atomicAdd(a.blocks_pruned, static_cast<unsigned long long>(__popc(bitsw)));
                }
            }
        }
        __syncthreads();
    }
}

template <int DT>
static ftk_status launch_box_dt(const BoxArgs &a, cudaStream_t s)
{
    return launch_kernel(box_kernel<DT>, dim3(a.nblocks), dim3(kBoxThreads), 0, s, 1, a);
}

ftk_status launch_box(int dtype, const BoxArgs &a, cudaStream_t s)
{
    return dtype == FTK_F8E4M3 ? launch_box_dt<FTK_F8E4M3>(a, s) : launch_box_dt<FTK_BF16>(a, s);
}

template <int DT, int H>
static ftk_status launch_bound_dt(int mode, const BoundArgs &a, int grid, cudaStream_t s)
{
    const int threads = kBoundWarps * 32;
    if (mode == BOUND_EST) return launch_kernel(bound_kernel<DT, BOUND_EST, H>, dim3(grid), dim3(threads), 0, s, 1, a);
    if (mode == BOUND_FULL) return launch_kernel(bound_kernel<DT, BOUND_FULL, H>, dim3(grid), dim3(threads), 0, s, 1, a);
    return launch_kernel(bound_kernel<DT, BOUND_OUT, H>, dim3(grid), dim3(threads), 0, s, 1, a);
}

ftk_status launch_bound(int dtype, int mode, const BoundArgs &a, int grid, cudaStream_t s, int heads)
{
    if (heads == 64)
        return dtype == FTK_F8E4M3 ? launch_bound_dt<FTK_F8E4M3, 64>(mode, a, grid, s)
                                   : launch_bound_dt<FTK_BF16, 64>(mode, a, grid, s);
    return dtype == FTK_F8E4M3 ? launch_bound_dt<FTK_F8E4M3, 32>(mode, a, grid, s)
                               : launch_bound_dt<FTK_BF16, 32>(mode, a, grid, s);
}

static int sm_count()
{
    int dev = 0, n = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

}  // namespace ftk

using namespace ftk;

extern "C" size_t ftk_block_bound_workspace_size(int64_t S)
{
    if (S < 1) return 0;
    const int64_t nb = (S + kBlockKeys - 1) / kBlockKeys;
    return align_up(static_cast<size_t>(nb) * 2 * kDim * sizeof(float), 256) +
           align_up(static_cast<size_t>(nb) * sizeof(float), 256);
}

extern "C" ftk_status ftk_block_bound_heads(ftk_dtype dtype, int heads, const void *q, const void *kv,
                                            const float *kv_scales, const float *weights, int64_t T,
                                            int64_t S, float *out, int64_t ld, void *workspace,
                                            size_t workspace_bytes, void *stream)
{
    if (dtype != FTK_F8E4M3 && dtype != FTK_BF16) return FTK_ERR_UNSUPPORTED;
    if (heads != 32 && heads != 64) return FTK_ERR_INVALID_ARG;
    if (!q || !kv || !weights || !out) return FTK_ERR_INVALID_ARG;
    if (T < 1 || S < 1 || T >= (int64_t(1) << 31) / heads || S >= (int64_t(1) << 31) - kBlockKeys)
        return FTK_ERR_INVALID_ARG;
    const int64_t nb = (S + kBlockKeys - 1) / kBlockKeys;
    if (ld < nb) return FTK_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(kv)) return FTK_ERR_ALIGNMENT;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
        workspace_bytes < ftk_block_bound_workspace_size(S))
        return FTK_ERR_WORKSPACE;
    ftk_status st = check_device();
    if (st != FTK_OK) return st;
    cudaStream_t s = as_stream(stream);
    Carver cv{static_cast<uint8_t *>(workspace), workspace_bytes};
    BoxArgs ba;
    ba.kv = kv;
    ba.kv_scales = kv_scales;
    ba.S = S;
    ba.nblocks = static_cast<int32_t>(nb);
    ba.box = cv.take<float>(nb * 2 * kDim);
    ba.mb = cv.take<float>(nb);
    if ((st = launch_box(dtype, ba, s)) != FTK_OK) return st;
    BoundArgs a = {};
    a.q = q;
    a.weights = weights;
    a.T = T;
    a.S = S;
    a.rt = 16;
    a.ntiles = static_cast<int32_t>((T + a.rt - 1) / a.rt);
    a.nblocks = ba.nblocks;
    a.nwords = static_cast<int32_t>((nb + kBoundWordBlocks - 1) / kBoundWordBlocks);
    a.box = ba.box;
    a.mb = ba.mb;
    a.out = out;
    a.ld = ld;
    const int64_t items = static_cast<int64_t>(a.ntiles) * a.nwords;
    const int64_t cap = static_cast<int64_t>(sm_count()) * 4;
    return launch_bound(dtype, BOUND_OUT, a, static_cast<int>(items < cap ? items : cap), s, heads);
}

extern "C" ftk_status ftk_block_bound(ftk_dtype dtype, const void *q, const void *kv,
                                      const float *kv_scales, const float *weights, int64_t T,
                                      int64_t S, float *out, int64_t ld, void *workspace,
                                      size_t workspace_bytes, void *stream)
{
    return ftk_block_bound_heads(dtype, 32, q, kv, kv_scales, weights, T, S, out, ld, workspace,
                                 workspace_bytes, stream);
}
