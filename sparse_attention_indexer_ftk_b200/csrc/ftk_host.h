// ftk_host.h -- host-side helpers shared by the libftk entry points.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ftk.h"

namespace ftk {

inline cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// FTK_OK when the current device is compute capability 10.0 (B200, sm_100a).
ftk_status check_device();

// Maps a CUDA error to FTK_ERR_CUDA (and clears the sticky launch error
// only for launch-configuration errors, which do not poison the context).
inline ftk_status cuda_status(cudaError_t e)
{
    if (e == cudaSuccess) return FTK_OK;
    (void)cudaGetLastError();
    return FTK_ERR_CUDA;
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Bump allocator over a caller-owned workspace (256-byte aligned pieces).
struct Carver {
    uint8_t *base;
    size_t size;
    size_t used = 0;
    bool ok = true;
    template <class T>
    T *take(size_t count)
    {
        size_t off = align_up(used, 256);
        size_t bytes = align_up(count * sizeof(T), 256);
        if (base == nullptr || off + bytes > size) {
            ok = false;
            used = off + bytes;
            return nullptr;
        }
        used = off + bytes;
        return reinterpret_cast<T *>(base + off);
    }
};

// The calling thread's current CUDA context (a driver handle), or NULL.
void *current_context();

// False when the environment variable FTK_NO_PDL is set to 1 (read once).
bool pdl_enabled();

// Launches kern with programmatic stream serialization (unless disabled):
// the kernel may be scheduled while the kernel before it on the stream
// finishes, which hides launch latency between the many short kernels of a
// call; every kernel of the library starts with griddep_wait(), so it reads
// nothing before its predecessor is complete.  cluster > 1 adds
// thread-block clusters of that many CTAs.
template <typename... KArgs, typename... Args>
inline ftk_status launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                unsigned cluster, Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    unsigned n = 0;
    if (cluster > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = cluster;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    if (pdl_enabled()) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, static_cast<Args &&>(args)...));
}

// Raises the dynamic shared-memory limit of kernel `func` to at least
// `bytes`, once per (kernel, context): later calls find it in a small table
// instead of calling cudaFuncSetAttribute again.  A context that is
// destroyed and created again is a new context, so the limit is set anew.
ftk_status ensure_smem_limit(const void *func, int bytes);

// The host-visible argument checks of ftk_select (dtype, head count and
// reserved config fields, pointers, sizes, topk range, alignment), in the
// order ftk_select reports them; FTK_OK if the call may proceed.
ftk_status check_select_call(int dtype, const void *q, const void *kv, const float *w, const int32_t *ks,
                             const int32_t *ke, int64_t T, int64_t S, int topk, const int32_t *out_idx,
                             const ftk_config *config);

struct RowsArgs;
struct BoxArgs;
struct BoundArgs;
// Score-bound pruning kernels (ftk_prune.cu): the box of every key block,
// and the bound in mode BOUND_EST / BOUND_FULL / BOUND_OUT.
ftk_status launch_box(int dtype, const BoxArgs &a, cudaStream_t stream);
ftk_status launch_bound(int dtype, int mode, const BoundArgs &a, int grid, cudaStream_t stream, int heads = 32);
// Launches the row top-k kernel for the given dtype (FTK_BF16 / FTK_F32)
// with one cluster of `cluster` CTAs per grid row.
ftk_status launch_rows_topk(int dtype, const RowsArgs &a, int cluster, cudaStream_t stream, bool idx64 = false);
// Cluster size and per-CTA chunk for rows of `cols` columns.
void rows_plan(int64_t rows, int64_t cols, int k, int *cluster, int *chunk);

}  // namespace ftk
