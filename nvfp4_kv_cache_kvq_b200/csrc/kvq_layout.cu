// kvq_layout.cu -- the "blocked" layout of a scale matrix: the 128 x 4 tiles that
// block-scaled MMA operands read, which "How NVFP4 Quantization Works in LongLive 2.0",
// section "Stage 3: KV-Cache De-quantization at Inference", step 1, converts back to a
// plain 2D view ("from_blocked").
//
// A [rows, cols] matrix of one-byte scales (cols = head_dim / 16 for a K or V tensor of
// rows x head_dim) is padded to rows' = ceil(rows / 128) * 128 and cols' = ceil(cols / 4) * 4
// (zeros), cut into 128 x 4 tiles stored in row-tile-major order, 512 bytes each, and
// inside a tile scale (r, c) sits at byte (r % 32) * 16 + ((r % 128) / 32) * 4 + c % 4.
//
// Kernels: one thread per 4-byte word of the blocked buffer (the 4 scales of one row in
// one tile), so the blocked side is read or written fully coalesced.
#include <cuda_runtime.h>

#include <cstdint>

#include "kvq.h"
#include "kvq_common.h"
#include "kvq_device.cuh"

namespace kvq {
namespace {

struct LayoutArgs {
    const uint8_t* src;
    uint8_t* dst;
    int64_t rows;
    int32_t cols;
    int64_t col_tiles;  // ceil(cols / 4)
    uint64_t words;     // 4-byte words of the blocked buffer
};

// Word w of tile t holds row r = row_tile * 128 + (w % 4) * 32 + w / 4, columns
// [col_tile * 4, col_tile * 4 + 4).
__device__ __forceinline__ void word_position(const LayoutArgs& a, uint64_t i, int64_t& r, int64_t& c0)
{
    const uint64_t tile = i / 128, w = i % 128;
    r = static_cast<int64_t>(tile / a.col_tiles) * 128 + static_cast<int64_t>((w % 4) * 32 + w / 4);
    c0 = static_cast<int64_t>(tile % a.col_tiles) * 4;
}

__global__ void __launch_bounds__(kThreads) to_blocked_kernel(const LayoutArgs a)
{
    pdl_begin();
    const uint64_t i = static_cast<uint64_t>(blockIdx.x) * kThreads + threadIdx.x;
    if (i >= a.words)
        return;
    int64_t r, c0;
    word_position(a, i, r, c0);
    uint32_t word = 0;
    if (r < a.rows) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (c0 + k < a.cols)
                word |= static_cast<uint32_t>(__ldg(a.src + r * a.cols + c0 + k)) << (8 * k);
    }
    reinterpret_cast<uint32_t*>(a.dst)[i] = word;
}

__global__ void __launch_bounds__(kThreads) from_blocked_kernel(const LayoutArgs a)
{
    pdl_begin();
    const uint64_t i = static_cast<uint64_t>(blockIdx.x) * kThreads + threadIdx.x;
    if (i >= a.words)
        return;
    int64_t r, c0;
    word_position(a, i, r, c0);
    if (r >= a.rows)
        return;
    const uint32_t word = __ldg(reinterpret_cast<const uint32_t*>(a.src) + i);
#pragma unroll
    for (int k = 0; k < 4; ++k)
        if (c0 + k < a.cols)
            a.dst[r * a.cols + c0 + k] = static_cast<uint8_t>(word >> (8 * k));
}

kvq_status layout_impl(bool to_blocked, const uint8_t* src, int64_t rows, int32_t cols, uint8_t* dst,
                       cudaStream_t s)
{
    const char* what = to_blocked ? "kvq_scales_to_blocked" : "kvq_scales_from_blocked";
    if (rows < 0 || cols <= 0)
        return fail(KVQ_ERR_INVALID_ARG, "%s: rows %lld, cols %d", what, static_cast<long long>(rows), cols);
    if (rows == 0)
        return ok();
    if (src == nullptr || dst == nullptr)
        return fail(KVQ_ERR_INVALID_ARG, "%s: null pointer", what);
    const uint8_t* blocked = to_blocked ? dst : src;
    if (!aligned(blocked, 4))
        return fail(KVQ_ERR_MISALIGNED, "%s: the blocked buffer must be 4-byte aligned", what);
    LayoutArgs a;
    a.src = src;
    a.dst = dst;
    a.rows = rows;
    a.cols = cols;
    a.col_tiles = (cols + 3) / 4;
    a.words = static_cast<uint64_t>((rows + 127) / 128) * static_cast<uint64_t>(a.col_tiles) * 128;
    if (a.words * 4 > kMaxElems)
        return fail(KVQ_ERR_UNSUPPORTED, "%s: above 2^36 bytes", what);
    const dim3 grid(tiles(a.words));
    return launched(to_blocked ? launch(to_blocked_kernel, grid, kThreads, s, a)
                               : launch(from_blocked_kernel, grid, kThreads, s, a),
                    what);
}

}  // namespace
}  // namespace kvq

using namespace kvq;

extern "C" {

kvq_status kvq_scales_to_blocked(const uint8_t* scales, int64_t rows, int32_t cols, uint8_t* blocked,
                                 kvq_stream_t stream)
{
    NvtxRange nvtx_range("kvq_scales_to_blocked");
    kvq_status st = layout_impl(true, scales, rows, cols, blocked, reinterpret_cast<cudaStream_t>(stream));
    return st == KVQ_OK ? ok() : st;
}

kvq_status kvq_scales_from_blocked(const uint8_t* blocked, int64_t rows, int32_t cols, uint8_t* scales,
                                   kvq_stream_t stream)
{
    NvtxRange nvtx_range("kvq_scales_from_blocked");
    kvq_status st = layout_impl(false, blocked, rows, cols, scales, reinterpret_cast<cudaStream_t>(stream));
    return st == KVQ_OK ? ok() : st;
}

kvq_status kvq_blocked_scale_bytes(int64_t rows, int32_t cols, uint64_t* bytes)
{
    if (rows < 0 || cols <= 0 || bytes == nullptr)
        return fail(KVQ_ERR_INVALID_ARG, "kvq_blocked_scale_bytes: rows %lld, cols %d", static_cast<long long>(rows),
                    cols);
    *bytes = static_cast<uint64_t>((rows + 127) / 128) * 128u * static_cast<uint64_t>((cols + 3) / 4) * 4u;
    return ok();
}

}  // extern "C"
