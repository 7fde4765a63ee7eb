// ftk_noalloc.cu -- ftk_select for callers that cannot allocate device
// memory: the scratch lives in a fixed array compiled into the library.
//
// Some callers cannot call cudaMalloc: code running inside another
// allocator's arena or under a memory cap that forbids new allocations,
// code that must never fail on an out-of-memory at call time, and hosts
// with no allocator of their own (plain C callers without torch or a pool).
// This entry point gives them fused score + top-k with no allocation at
// all: it runs exactly the ftk_select kernels, with their scratch placed in
// g_noalloc_scratch, a file-scope __device__ array of
// FTK_NOALLOC_SCRATCH_BYTES that every GPU loading the library holds until
// the process exits.
#include <atomic>

#include "ftk_host.h"

namespace ftk {

static __device__ __align__(256) uint8_t g_noalloc_scratch[FTK_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch per device.  In host code the array's
// name is only a host-side stand-in, so the address comes from
// cudaGetSymbolAddress, once per device, with that device current.
static void *scratch_on_device(int dev)
{
    static std::atomic<void *> addr[64];  // host threads may race here
    if (dev < 0 || dev >= 64) return nullptr;
    void *p = addr[dev].load(std::memory_order_acquire);
    if (!p) {
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {
            (void)cudaGetLastError();
            return nullptr;
        }
        addr[dev].store(p, std::memory_order_release);
    }
    return p;
}

}  // namespace ftk

using namespace ftk;

extern "C" ftk_status ftk_select_noalloc(ftk_dtype dtype, const void *q, const void *kv,
                                         const float *kv_scales, const float *weights,
                                         const int32_t *ks, const int32_t *ke, int64_t T,
                                         int64_t S, int topk, int32_t *out_idx, float *out_val,
                                         const ftk_config *config, void *stream)
{
    if (T < 1 || S < 1 || topk < 1 || topk > FTK_MAX_TOPK) {
        // Same argument errors as ftk_select (it reports them first).
        return ftk_select(dtype, q, kv, kv_scales, weights, ks, ke, T, S, topk, out_idx, out_val,
                          nullptr, 0, config, stream);
    }
    // With the default recovery batch the scratch would be sized for up to
    // 512 MB of recovery rows; within the fixed array, use the largest batch
    // that fits (at least one 16-row tile), unless the caller chose one.
    ftk_config cfg = {};
    if (config) cfg = *config;
    if (cfg.recovery_rows <= 0) {
        int32_t rows = 16;
        for (int32_t r = 16; r <= 1 << 20; r *= 2) {
            cfg.recovery_rows = r;
            const size_t need = ftk_select_workspace_size(T, S, topk, &cfg);
            if (need == 0 || need > FTK_NOALLOC_SCRATCH_BYTES) break;
            rows = r;
            if (r >= T) break;
        }
        cfg.recovery_rows = rows;
    }
    const size_t need = ftk_select_workspace_size(T, S, topk, &cfg);
    if (need == 0 || need > FTK_NOALLOC_SCRATCH_BYTES) return FTK_ERR_WORKSPACE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cuda_status(cudaErrorInvalidDevice);
    void *scratch = scratch_on_device(dev);
    if (!scratch) return FTK_ERR_CUDA;
    return ftk_select(dtype, q, kv, kv_scales, weights, ks, ke, T, S, topk, out_idx, out_val,
                      scratch, FTK_NOALLOC_SCRATCH_BYTES, &cfg, stream);
}
