// kvq_common.h -- host-side helpers shared by the library's translation units: error
// reporting, argument checks and the programmatic-dependent-launch wrapper.
#pragma once

#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdint>
#include <cstdio>

#include <nvtx3/nvToolsExt.h>

#include "kvq.h"

namespace kvq {

// An NVTX range around each entry point, so profilers show the library's calls by name
// (free when no tool is attached).
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

constexpr int kBlock = 16;  // elements per quantization block
constexpr int kThreads = 256;
constexpr int kMaxBatch = KVQ_MAX_BATCH;
constexpr uint64_t kMaxElems = 1ull << 36;

// Message of the last failure of the calling thread (kvq_last_error).
extern thread_local char g_last_error[512];

inline kvq_status fail(kvq_status st, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
inline kvq_status fail(kvq_status st, const char* fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return st;
}

inline kvq_status ok()
{
    g_last_error[0] = '\0';
    return KVQ_OK;
}

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Launch with programmatic stream serialization (see pdl_begin): the kernel may be
// scheduled while the previous grid on the stream drains, and waits for it on entry.
template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, unsigned threads, cudaStream_t s, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

inline kvq_status launched(cudaError_t e, const char* what)
{
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(KVQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    }
    return KVQ_OK;
}

// CTAs along x for `units` units of one tensor, kThreads (times `per_thread`) per CTA.
inline unsigned tiles(uint64_t units, uint64_t per_thread = 1)
{
    const uint64_t per_cta = static_cast<uint64_t>(kThreads) * per_thread;
    return static_cast<unsigned>((units + per_cta - 1) / per_cta);
}

inline kvq_status check_shape(int64_t n_elems, int32_t head_dim)
{
    if (head_dim <= 0 || head_dim % kBlock != 0)
        return fail(KVQ_ERR_INVALID_ARG, "head_dim %d is not a positive multiple of 16", head_dim);
    if (n_elems < 0 || n_elems % head_dim != 0)
        return fail(KVQ_ERR_INVALID_ARG, "n_elems %lld is not a non-negative multiple of head_dim %d",
                    static_cast<long long>(n_elems), head_dim);
    if (static_cast<uint64_t>(n_elems) > kMaxElems)
        return fail(KVQ_ERR_UNSUPPORTED, "n_elems %lld above 2^36", static_cast<long long>(n_elems));
    return KVQ_OK;
}

}  // namespace kvq
