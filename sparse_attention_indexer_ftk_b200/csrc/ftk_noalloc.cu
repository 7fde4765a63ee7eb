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
#include <mutex>

#include "ftk_host.h"

namespace ftk {

static __device__ __align__(256) uint8_t g_noalloc_scratch[FTK_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch in the current context.  In host code
// the array's name is only a host-side stand-in, so the address comes from
// cudaGetSymbolAddress, with the device current.  It is cached per device
// together with the context it was taken in: a context that was destroyed
// and created again (cudaDeviceReset, a released and re-retained primary
// context) reloads the module at another address, and the next call looks
// the address up again instead of using a stale one.
static void *scratch_on_device(int dev)
{
    struct Entry {
        void *ctx;
        void *addr;
    };
    static Entry cache[64] = {};
    static std::mutex mu;  // host threads may race here
    if (dev < 0 || dev >= 64) return nullptr;
    void *ctx = current_context();
    std::lock_guard<std::mutex> lock(mu);
    if (ctx && cache[dev].ctx == ctx && cache[dev].addr) return cache[dev].addr;
    // (Also makes the device's primary context current on this thread if no
    // context was.)
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {
        (void)cudaGetLastError();
        return nullptr;
    }
    ctx = current_context();
    if (!ctx) return nullptr;
    cache[dev].ctx = ctx;
    cache[dev].addr = p;
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
    // ftk_select's argument errors come first, as ftk_select reports them.
    ftk_status st = check_select_call(dtype, q, kv, weights, ks, ke, T, S, topk, out_idx, config);
    if (st != FTK_OK) return st;
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

// The ftk_info of the last ftk_select_noalloc call on the current device:
// ftk_select keeps it at the start of its scratch.
extern "C" ftk_status ftk_noalloc_read_info(ftk_info *out, void *stream)
{
    if (!out) return FTK_ERR_INVALID_ARG;
    cudaStream_t st = as_stream(stream);
    cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_noalloc_scratch, sizeof(ftk_info), 0,
                                              cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    return cuda_status(e);
}
