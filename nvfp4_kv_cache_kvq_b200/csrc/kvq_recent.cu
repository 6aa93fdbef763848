// kvq_recent.cu -- the RECENT cache policy: the RTN_INT4 RECENT2 method of "KV Cache
// Quantization for Self-Forcing Video Generation" (appendix Table 3). The newest
// recent_blocks frame-blocks of a K or V cache stay in a bf16 ring; a block leaving the
// ring is RTN-quantized into the cache prefix (quantize-on-write); a read dequantizes the
// prefix and copies the bf16 tail back in. The codec is the library's RTN kernels
// (kvq_rtn.cu); the bf16 moves are one batched 256-bit copy kernel.
#include <cuda_runtime.h>

#include <cstdint>
#include <vector>

#include "kvq.h"
#include "kvq_common.h"
#include "kvq_device.cuh"

namespace kvq {
namespace {

constexpr uint64_t kCopyWord = 32;  // bytes per thread of copy_kernel

struct CopyBatch {
    const uint8_t* src[kMaxBatch];
    uint8_t* dst[kMaxBatch];
    uint64_t words;  // 32-byte words per copy
};

// Copy blockIdx.y of the batch, one 32-byte word per thread.
__global__ void __launch_bounds__(kThreads) copy_kernel(const CopyBatch cb)
{
    pdl_begin();
    const uint64_t w = static_cast<uint64_t>(blockIdx.x) * kThreads + threadIdx.x;
    if (w >= cb.words)
        return;
    uint32_t v[8];
    ld_nc_v8(cb.src[blockIdx.y] + w * kCopyWord, v);
    st_v8(cb.dst[blockIdx.y] + w * kCopyWord, v);
}

// n copies of `bytes` each (a multiple of 32, both ends 32-byte aligned), batched.
kvq_status copy_batch(const std::vector<const uint8_t*>& src, const std::vector<uint8_t*>& dst, uint64_t bytes,
                      cudaStream_t s, const char* what)
{
    const uint64_t words = bytes / kCopyWord;
    if (words == 0)
        return KVQ_OK;
    for (size_t base = 0; base < src.size(); base += kMaxBatch) {
        const size_t m = src.size() - base < static_cast<size_t>(kMaxBatch) ? src.size() - base : kMaxBatch;
        CopyBatch cb{};
        cb.words = words;
        for (size_t i = 0; i < m; ++i) {
            cb.src[i] = src[base + i];
            cb.dst[i] = dst[base + i];
        }
        const dim3 grid(tiles(words), static_cast<unsigned>(m));
        const kvq_status st = launched(launch(copy_kernel, grid, kThreads, s, cb), what);
        if (st != KVQ_OK)
            return st;
    }
    return KVQ_OK;
}

kvq_status check_caches(const kvq_recent_cache* c, int32_t n, const char* what)
{
    if (n < 0)
        return fail(KVQ_ERR_INVALID_ARG, "%s: negative cache count", what);
    if (n > 0 && c == nullptr)
        return fail(KVQ_ERR_INVALID_ARG, "%s: null cache array", what);
    for (int32_t i = 0; i < n; ++i) {
        const kvq_recent_cache& k = c[i];
        if (k.packed == nullptr || k.scales == nullptr || k.recent == nullptr)
            return fail(KVQ_ERR_INVALID_ARG, "%s: null cache buffer", what);
        if (k.capacity_blocks <= 0 || k.rows_per_block <= 0 || k.recent_blocks <= 0)
            return fail(KVQ_ERR_INVALID_ARG, "%s: bad cache sizes", what);
        if (k.bits != 2 && k.bits != 4)
            return fail(KVQ_ERR_INVALID_ARG, "%s: bits %d is not 2 or 4", what, k.bits);
        const kvq_status st = check_shape(k.rows_per_block * static_cast<int64_t>(k.head_dim), k.head_dim);
        if (st != KVQ_OK)
            return st;
        if (k.capacity_blocks > (int64_t{1} << 40) / k.rows_per_block)
            return fail(KVQ_ERR_UNSUPPORTED, "%s: cache too large", what);
        if (!aligned(k.recent, 32) || !aligned(k.packed, 2 * k.bits) || !aligned(k.scales, 2))
            return fail(KVQ_ERR_MISALIGNED, "%s: recent 32-byte, codes %d-byte, scales 2-byte aligned", what,
                        2 * k.bits);
        if (k.rows_per_block != c[0].rows_per_block || k.head_dim != c[0].head_dim || k.bits != c[0].bits ||
            k.recent_blocks != c[0].recent_blocks)
            return fail(KVQ_ERR_INVALID_ARG, "%s: caches differ in shape, bits or recent_blocks", what);
    }
    return KVQ_OK;
}

}  // namespace
}  // namespace kvq

using namespace kvq;

extern "C" {

kvq_status kvq_recent_append_batch(const kvq_recent_cache* caches, int32_t n_caches, int64_t block,
                                   const void* const* xs, kvq_stream_t stream)
{
    NvtxRange nvtx_range("kvq_recent_append_batch");
    const char* what = "kvq_recent_append_batch";
    kvq_status st = check_caches(caches, n_caches, what);
    if (st != KVQ_OK)
        return st;
    if (n_caches == 0)
        return ok();
    if (xs == nullptr)
        return fail(KVQ_ERR_INVALID_ARG, "%s: null input array", what);
    for (int32_t i = 0; i < n_caches; ++i) {
        if (xs[i] == nullptr)
            return fail(KVQ_ERR_INVALID_ARG, "%s: null input", what);
        if (!aligned(xs[i], 32))
            return fail(KVQ_ERR_MISALIGNED, "%s: inputs must be 32-byte aligned", what);
        if (block < 0 || block >= caches[i].capacity_blocks)
            return fail(KVQ_ERR_CAPACITY, "%s: block %lld outside [0, %lld)", what, static_cast<long long>(block),
                        static_cast<long long>(caches[i].capacity_blocks));
    }
    const kvq_recent_cache& c0 = caches[0];
    const int64_t elems = c0.rows_per_block * c0.head_dim;
    const uint64_t bf16_bytes = static_cast<uint64_t>(elems) * 2;
    const int64_t slot = block % c0.recent_blocks;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    std::vector<const uint8_t*> src(n_caches);
    std::vector<uint8_t*> dst(n_caches);
    if (block >= c0.recent_blocks) {
        // the block leaving the bf16 window sits in the slot the new block takes
        const int64_t evicted = block - c0.recent_blocks;
        std::vector<const void*> qx(n_caches);
        std::vector<uint8_t*> qp(n_caches);
        std::vector<uint16_t*> qs(n_caches);
        for (int32_t i = 0; i < n_caches; ++i) {
            qx[i] = static_cast<const uint8_t*>(caches[i].recent) + slot * bf16_bytes;
            qp[i] = caches[i].packed + evicted * elems * c0.bits / 8;
            qs[i] = caches[i].scales + evicted * elems / kBlock;
        }
        st = kvq_rtn_quantize_batch(qx.data(), n_caches, elems, c0.head_dim, c0.bits, qp.data(), qs.data(), stream);
        if (st != KVQ_OK)
            return st;
    }
    for (int32_t i = 0; i < n_caches; ++i) {
        src[i] = static_cast<const uint8_t*>(xs[i]);
        dst[i] = static_cast<uint8_t*>(caches[i].recent) + slot * bf16_bytes;
    }
    st = copy_batch(src, dst, bf16_bytes, s, what);
    return st == KVQ_OK ? ok() : st;
}

kvq_status kvq_recent_read_batch(const kvq_recent_cache* caches, int32_t n_caches, int64_t n_blocks,
                                 void* const* ys, kvq_stream_t stream)
{
    NvtxRange nvtx_range("kvq_recent_read_batch");
    const char* what = "kvq_recent_read_batch";
    kvq_status st = check_caches(caches, n_caches, what);
    if (st != KVQ_OK)
        return st;
    if (n_caches == 0 || n_blocks == 0)
        return ok();
    if (n_blocks < 0)
        return fail(KVQ_ERR_INVALID_ARG, "%s: negative block count", what);
    if (ys == nullptr)
        return fail(KVQ_ERR_INVALID_ARG, "%s: null output array", what);
    for (int32_t i = 0; i < n_caches; ++i) {
        if (ys[i] == nullptr)
            return fail(KVQ_ERR_INVALID_ARG, "%s: null output", what);
        if (!aligned(ys[i], 32))
            return fail(KVQ_ERR_MISALIGNED, "%s: outputs must be 32-byte aligned", what);
        if (n_blocks > caches[i].capacity_blocks)
            return fail(KVQ_ERR_CAPACITY, "%s: %lld blocks past the capacity", what, static_cast<long long>(n_blocks));
    }
    const kvq_recent_cache& c0 = caches[0];
    const int64_t elems = c0.rows_per_block * c0.head_dim;
    const uint64_t bf16_bytes = static_cast<uint64_t>(elems) * 2;
    const int64_t r = n_blocks < c0.recent_blocks ? n_blocks : c0.recent_blocks;
    const int64_t prefix = n_blocks - r;
    if (prefix > 0) {
        std::vector<const uint8_t*> dp(n_caches);
        std::vector<const uint16_t*> ds(n_caches);
        for (int32_t i = 0; i < n_caches; ++i) {
            dp[i] = caches[i].packed;
            ds[i] = caches[i].scales;
        }
        st = kvq_rtn_dequantize_batch(dp.data(), ds.data(), n_caches, prefix * elems, c0.head_dim, c0.bits, ys,
                                      stream);
        if (st != KVQ_OK)
            return st;
    }
    std::vector<const uint8_t*> src;
    std::vector<uint8_t*> dst;
    for (int32_t i = 0; i < n_caches; ++i)
        for (int64_t b = prefix; b < n_blocks; ++b) {
            src.push_back(static_cast<const uint8_t*>(caches[i].recent) + (b % c0.recent_blocks) * bf16_bytes);
            dst.push_back(static_cast<uint8_t*>(ys[i]) + b * bf16_bytes);
        }
    st = copy_batch(src, dst, bf16_bytes, reinterpret_cast<cudaStream_t>(stream), what);
    return st == KVQ_OK ? ok() : st;
}

}  // extern "C"
