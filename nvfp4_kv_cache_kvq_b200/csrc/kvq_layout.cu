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
// Kernels: one thread per 16-byte group of a tile -- group k of a tile holds rows k,
// k + 32, k + 64, k + 96 of its 128-row slice, 4 scales each. Consecutive threads take
// the column tiles of one k, then the next k, so each plain-side access of a warp covers
// whole consecutive rows, and on the blocked side every 16-byte group is written or read
// once, in runs of whole groups. When cols is a multiple of 4 and the plain buffer
// 4-byte aligned (WORD), the plain side moves a 4-byte word per row; otherwise byte by
// byte.
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
    uint32_t col_tiles;  // ceil(cols / 4)
    uint64_t groups;     // 16-byte groups of the blocked buffer (32 per tile)
};

// Thread g: column tile ct = g % col_tiles, then k = (g / col_tiles) % 32 and row tile
// (g / col_tiles) / 32; its group is number k of tile (row tile * col_tiles + ct), at byte
// 16 * group of the blocked buffer. Groups number at most 2^36 / 16 = 2^32, so 32-bit
// arithmetic suffices.
__device__ __forceinline__ uint64_t group_position(const LayoutArgs& a, uint64_t g, int64_t& r0, int64_t& c0)
{
    const uint32_t gi = static_cast<uint32_t>(g);
    const uint32_t rk = gi / a.col_tiles, ct = gi - rk * a.col_tiles;
    const uint32_t k = rk & 31, row_tile = rk >> 5;
    r0 = static_cast<int64_t>(row_tile) * 128 + k;
    c0 = static_cast<int64_t>(ct) * 4;
    return (static_cast<uint64_t>(row_tile) * a.col_tiles + ct) * 32 + k;
}

// The 4 scales of row r at columns c0 .. c0 + 3 (zeros past rows and cols).
template <bool WORD>
__device__ __forceinline__ uint32_t plain_word(const LayoutArgs& a, int64_t r, int64_t c0)
{
    uint32_t word = 0;
    if (r >= a.rows) {
    } else if (WORD) {
        word = __ldg(reinterpret_cast<const uint32_t*>(a.src + r * a.cols + c0));
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (c0 + k < a.cols)
                word |= static_cast<uint32_t>(__ldg(a.src + r * a.cols + c0 + k)) << (8 * k);
    }
    return word;
}

template <bool WORD>
__device__ __forceinline__ void store_plain_word(const LayoutArgs& a, int64_t r, int64_t c0, uint32_t word)
{
    if (r >= a.rows) {
    } else if (WORD) {
        *reinterpret_cast<uint32_t*>(a.dst + r * a.cols + c0) = word;
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (c0 + k < a.cols)
                a.dst[r * a.cols + c0 + k] = static_cast<uint8_t>(word >> (8 * k));
    }
}

constexpr int kGroupsPerThread = 2;  // threads g and g + gridDim.x * kThreads of a wave, both loads issued first

template <bool WORD>
__global__ void __launch_bounds__(kThreads) to_blocked_kernel(const LayoutArgs a)
{
    pdl_begin();
    const uint64_t stride = static_cast<uint64_t>(gridDim.x) * kThreads;
    const uint64_t g0 = static_cast<uint64_t>(blockIdx.x) * kThreads + threadIdx.x;
    uint32_t w[kGroupsPerThread][4];
    uint64_t grp[kGroupsPerThread];
#pragma unroll
    for (int i = 0; i < kGroupsPerThread; ++i) {
        const uint64_t g = g0 + i * stride;
        if (g >= a.groups)
            continue;
        int64_t r0, c0;
        grp[i] = group_position(a, g, r0, c0);
#pragma unroll
        for (int q = 0; q < 4; ++q)
            w[i][q] = plain_word<WORD>(a, r0 + 32 * q, c0);
    }
#pragma unroll
    for (int i = 0; i < kGroupsPerThread; ++i)
        if (g0 + i * stride < a.groups)
            st_v4(a.dst + grp[i] * 16, w[i][0], w[i][1], w[i][2], w[i][3]);
}

template <bool WORD>
__global__ void __launch_bounds__(kThreads) from_blocked_kernel(const LayoutArgs a)
{
    pdl_begin();
    const uint64_t stride = static_cast<uint64_t>(gridDim.x) * kThreads;
    const uint64_t g0 = static_cast<uint64_t>(blockIdx.x) * kThreads + threadIdx.x;
    uint4 w[kGroupsPerThread];
    int64_t r0[kGroupsPerThread], c0[kGroupsPerThread];
#pragma unroll
    for (int i = 0; i < kGroupsPerThread; ++i) {
        const uint64_t g = g0 + i * stride;
        r0[i] = a.rows;  // nothing to store
        if (g >= a.groups)
            continue;
        const uint64_t grp = group_position(a, g, r0[i], c0[i]);
        if (r0[i] < a.rows)
            w[i] = ld_nc_v4(a.src + grp * 16);
    }
#pragma unroll
    for (int i = 0; i < kGroupsPerThread; ++i) {
        if (r0[i] >= a.rows)
            continue;
        store_plain_word<WORD>(a, r0[i], c0[i], w[i].x);
        store_plain_word<WORD>(a, r0[i] + 32, c0[i], w[i].y);
        store_plain_word<WORD>(a, r0[i] + 64, c0[i], w[i].z);
        store_plain_word<WORD>(a, r0[i] + 96, c0[i], w[i].w);
    }
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
    if (!aligned(blocked, 16))
        return fail(KVQ_ERR_MISALIGNED, "%s: the blocked buffer must be 16-byte aligned", what);
    LayoutArgs a;
    a.src = src;
    a.dst = dst;
    a.rows = rows;
    a.cols = cols;
    a.col_tiles = static_cast<uint32_t>((cols + 3) / 4);
    a.groups = static_cast<uint64_t>((rows + 127) / 128) * a.col_tiles * 32;
    if (a.groups * 16 > kMaxElems || a.groups > 0xFFFFFFFFull)
        return fail(KVQ_ERR_UNSUPPORTED, "%s: above 2^36 bytes", what);
    const dim3 grid(tiles((a.groups + kGroupsPerThread - 1) / kGroupsPerThread));
    const uint8_t* plain = to_blocked ? src : dst;
    const bool word = cols % 4 == 0 && aligned(plain, 4);
    cudaError_t e;
    if (to_blocked)
        e = word ? launch(to_blocked_kernel<true>, grid, kThreads, s, a) : launch(to_blocked_kernel<false>, grid, kThreads, s, a);
    else
        e = word ? launch(from_blocked_kernel<true>, grid, kThreads, s, a)
                 : launch(from_blocked_kernel<false>, grid, kThreads, s, a);
    return launched(e, what);
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
