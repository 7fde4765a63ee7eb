// ftk_api.cu -- small C-ABI entry points: status strings, version, packed
// causal windows.
#include <cudaTypedefs.h>

#include <stdlib.h>

#include <atomic>
#include <mutex>

#include "ftk_device.cuh"
#include "ftk_host.h"

namespace ftk {

bool pdl_enabled()
{
    static const bool on = [] {
        const char *e = getenv("FTK_NO_PDL");
        return !(e && e[0] == '1');
    }();
    return on;
}

void *current_context()
{
    // cuCtxGetCurrent through the runtime's driver entry point (the library
    // does not link the driver library itself).
    static std::atomic<PFN_cuCtxGetCurrent_v4000> cached{nullptr};
    PFN_cuCtxGetCurrent_v4000 fn = cached.load(std::memory_order_acquire);
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
        cached.store(fn, std::memory_order_release);
    }
    CUcontext ctx = nullptr;
    return fn(&ctx) == CUDA_SUCCESS ? static_cast<void *>(ctx) : nullptr;
}

ftk_status ensure_smem_limit(const void *func, int bytes)
{
    struct Entry {
        const void *func;
        void *ctx;
        int bytes;
    };
    static Entry table[256];
    static int used = 0;
    static std::mutex mu;
    void *ctx = current_context();
    if (ctx) {
        std::lock_guard<std::mutex> lock(mu);
        for (int i = 0; i < used; ++i)
            if (table[i].func == func && table[i].ctx == ctx && table[i].bytes >= bytes) return FTK_OK;
    }
    const cudaError_t e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return cuda_status(e);
    ctx = current_context();  // (the call above may have made the context current)
    if (ctx) {
        std::lock_guard<std::mutex> lock(mu);
        for (int i = 0; i < used; ++i) {
            if (table[i].func == func && table[i].ctx == ctx) {
                if (table[i].bytes < bytes) table[i].bytes = bytes;
                return FTK_OK;
            }
        }
        if (used < 256) table[used++] = Entry{func, ctx, bytes};
    }
    return FTK_OK;
}

// One thread per query row: finds its sequence by binary search over cu_q
// and writes the causal window of a query that is among its sequence's last
// tokens (FlashTopK README, "Usage": windows_from_cu_seqlens; "Quick start":
// query i of the chunk sees keys [0, S - T + i + 1)).
__global__ void windows_kernel(const int32_t *cu_q, const int32_t *cu_k, int64_t nseq, int64_t T,
                               int32_t *ks, int32_t *ke)
{
    const int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
    if (t >= T) return;
    int64_t lo = 0, hi = nseq;  // find j with cu_q[j] <= t < cu_q[j+1]
    while (hi - lo > 1) {
        const int64_t mid = (lo + hi) / 2;
        if (cu_q[mid] <= t) lo = mid; else hi = mid;
    }
    const int64_t j = lo;
    const int64_t i = t - cu_q[j];
    const int64_t lq = static_cast<int64_t>(cu_q[j + 1]) - cu_q[j];
    const int64_t lk = static_cast<int64_t>(cu_k[j + 1]) - cu_k[j];
    int64_t end = lk - lq + i + 1;
    if (end < 0) end = 0;
    if (end > lk) end = lk;
    ks[t] = cu_k[j];
    ke[t] = static_cast<int32_t>(cu_k[j] + end);
}

}  // namespace ftk

using namespace ftk;

extern "C" const char *ftk_status_string(int status)
{
    switch (status) {
    case FTK_OK: return "ok";
    case FTK_ERR_INVALID_ARG: return "invalid argument";
    case FTK_ERR_UNSUPPORTED: return "unsupported";
    case FTK_ERR_TOPK_RANGE: return "topk out of range [1, 4096]";
    case FTK_ERR_ALIGNMENT: return "pointer or row stride not 16-byte aligned";
    case FTK_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case FTK_ERR_CUDA: return "CUDA runtime error";
    case FTK_ERR_DEVICE: return "device is not compute capability 10.0 (sm_100a)";
    default: return "unknown status";
    }
}

extern "C" int ftk_version(void) { return 100; }

extern "C" ftk_status ftk_windows_from_cu_seqlens(const int32_t *cu_q, const int32_t *cu_k,
                                                  int64_t nseq, int64_t T, int32_t *ks,
                                                  int32_t *ke, void *stream)
{
    if (!cu_q || !cu_k || !ks || !ke || nseq < 1 || T < 0 || T >= (int64_t(1) << 31))
        return FTK_ERR_INVALID_ARG;
    if (T == 0) return FTK_OK;
    ftk_status st = check_device();
    if (st != FTK_OK) return st;
    const int threads = 256;
    const unsigned blocks = static_cast<unsigned>((T + threads - 1) / threads);
    windows_kernel<<<blocks, threads, 0, as_stream(stream)>>>(cu_q, cu_k, nseq, T, ks, ke);
    return cuda_status(cudaGetLastError());
}
