// kvq_attention.cu -- attention reading the packed NVFP4 K/V cache directly: each K/V
// tile is dequantized into shared memory (the same arithmetic, hence the same bf16
// values, as kvq_dequantize_cache) and consumed there by tcgen05 tensor-core MMAs, so
// the dense bf16 cache is never written to HBM. The pages dequantize the active cache to
// BF16 before attention ("KV Cache Quantization for Self-Forcing Video Generation",
// appendix Table 3) and find that those transient BF16 buffers dominate peak memory
// (abstract; Figure 6); "How to Use KV Cache Quantization with LongLive's
// LongLiveQuantizationConfig" ("CUDA De-quantization Pipeline") dequantizes "during the
// attention operation".
//
// One CTA = 128 queries of one head, 4 warps; thread t owns query row t (TMEM lane t).
// For every tile of 128 keys:
//   1. dequantize K (row per key) and V (transposed: row per dim) into 128B-swizzled,
//      K-major shared memory;
//   2. S = Q K^T: 8 tcgen05.mma (M=128, N=128, K=16 each) into TMEM columns [0, 128);
//   3. online softmax on the TMEM rows (tcgen05.ld), P = bf16(exp2(s - m)) to shared
//      memory, O (TMEM columns [128, 256)) rescaled by exp2(m_old - m_new);
//   4. O += P V: 8 more tcgen05.mma.
// The MMAs are issued by thread 0 and signalled by tcgen05.commit on an mbarrier; every
// wait is bounded (on timeout the kernel records an error, frees its TMEM and returns).
#include <cuda_runtime.h>

#include <cstdint>

#include "kvq.h"
#include "kvq_common.h"
#include "kvq_device.cuh"

namespace kvq {
namespace {

constexpr int kBM = 128;         // queries per CTA
constexpr int kBN = 128;         // keys per tile
constexpr int kD = 128;          // head_dim (the only one supported)
constexpr int kAttnThreads = 128;
constexpr int kTileBytes = 32768;  // one 128 x 128 bf16 operand
constexpr int kSmemBytes = 4 * kTileBytes + 1024;  // Q, K, V^T, P + alignment slack
constexpr uint32_t kTmemCols = 256;                 // S: [0, 128), O: [128, 256)
constexpr uint64_t kWaitNs = 1000000000ull;        // give up on an mbarrier after 1 s

struct AttnArgs {
    const uint16_t* q;  // bf16 [n_q, heads, 128]
    uint16_t* o;        // bf16 [n_q, heads, 128]
    const uint8_t* kp;  // K cache: codes, scales, chunk amax (block 0 / chunk 0)
    const uint8_t* ks;
    const float* ka;
    const uint8_t* vp;  // V cache
    const uint8_t* vs;
    const float* va;
    int32_t n_q, heads;
    int64_t n_kv;              // keys (tokens)
    int64_t tokens_per_chunk;  // keys per amax chunk
    float scale_log2;          // softmax scale * log2(e)
    int* status;               // set to 1 on a wait timeout
};

// Byte offset of 16-byte chunk `chunk` (0..7) of row `row` in K-block `kb` of a 128-row,
// K-major operand with the 128-byte swizzle: K-blocks of 64 bf16 (16 KB each), 8-row
// groups of 1024 B, the chunk index XOR-ed with row % 8.
__device__ __forceinline__ uint32_t sw128(int row, int kb, int chunk)
{
    return kb * 16384 + (row >> 3) * 1024 + (row & 7) * 128 + ((chunk ^ (row & 7)) << 4);
}

// Shared-memory matrix descriptor of a 128B-swizzled K-major operand starting at
// shared-window address `saddr` (1024-aligned K-block plus the K offset): 8-row groups
// 1024 B apart, descriptor version 1, swizzle mode 128B.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr)
{
    return static_cast<uint64_t>((saddr >> 4) & 0x3FFF) | (1ull << 16) | (64ull << 32) | (1ull << 46) |
           (2ull << 61);
}

// Instruction descriptor of tcgen05.mma kind::f16: fp32 accumulate, bf16 A and B, both
// K-major, M = 128, N = 128.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((kBN >> 3) << 17) | ((kBM >> 4) << 24);

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t a, uint64_t b, bool accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                 ::"r"(tmem_d), "l"(a), "l"(b), "r"(kIdesc), "r"(accumulate ? 1u : 0u)
                 : "memory");
}

// D (TMEM) = A[128 x 128] B[128 x 128]^T, both K-major in shared memory, as 8 MMAs of K = 16.
__device__ __forceinline__ void mma_tile(uint32_t tmem_d, uint32_t a_base, uint32_t b_base, bool accumulate)
{
#pragma unroll
    for (int kb = 0; kb < 2; ++kb)
#pragma unroll
        for (int s = 0; s < 4; ++s)
            mma_bf16(tmem_d, sw128_desc(a_base + kb * 16384 + s * 32), sw128_desc(b_base + kb * 16384 + s * 32),
                     accumulate || kb > 0 || s > 0);
}

__device__ __forceinline__ void commit(uint32_t mbar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
                 : "memory");
}

__device__ __forceinline__ uint64_t globaltimer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Wait, for at most kWaitNs, for phase `parity` of an mbarrier; true when it completed.
__device__ __forceinline__ bool wait_phase(uint32_t mbar, uint32_t parity)
{
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        uint32_t done;
        asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                     "selp.u32 %0, 1, 0, p;\n\t}"
                     : "=r"(done)
                     : "r"(mbar), "r"(parity)
                     : "memory");
        if (done)
            return true;
        if (globaltimer_ns() - t0 > kWaitNs)
            return false;
    }
}

__device__ __forceinline__ void tmem_ld32(uint32_t addr, float (&v)[32])
{
    uint32_t r[32];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                 "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
                   "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
                   "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
                   "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(addr)
                 : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i)
        v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32(uint32_t addr, const float (&v)[32])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
                 "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
                 ::"r"(addr), "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]),
                 "f"(v[7]), "f"(v[8]), "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]),
                 "f"(v[15]), "f"(v[16]), "f"(v[17]), "f"(v[18]), "f"(v[19]), "f"(v[20]), "f"(v[21]), "f"(v[22]),
                 "f"(v[23]), "f"(v[24]), "f"(v[25]), "f"(v[26]), "f"(v[27]), "f"(v[28]), "f"(v[29]), "f"(v[30]),
                 "f"(v[31])
                 : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Dequantized bf16 words of one 16-element block: y = bf16_rne(value * S),
// S = e4m3_value(c) * gs -- the arithmetic of dequant_kernel, so the same bits.
__device__ __forceinline__ void dequant16(const uint8_t* packed, const uint8_t* scales, int64_t block, float gs,
                                          uint32_t (&y)[8])
{
    const uint2 q = ld_nc_v2(packed + block * 8);
    float S, unused;
    e4m3x2_to_f32(__ldg(scales + block), S, unused);
    S = __fmul_rn(S, gs);
    const uint64_t S2 = f32x2_pack(S, S);
    float v[8];
    e2m1x8_to_f32(q.x, v);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float lo, hi;
        f32x2_unpack(f32x2_mul(f32x2_pack(v[2 * j], v[2 * j + 1]), S2), lo, hi);
        y[j] = bf16x2_from_f32(hi, lo);
    }
    e2m1x8_to_f32(q.y, v);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float lo, hi;
        f32x2_unpack(f32x2_mul(f32x2_pack(v[2 * j], v[2 * j + 1]), S2), lo, hi);
        y[4 + j] = bf16x2_from_f32(hi, lo);
    }
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ void st_shared_b32(uint32_t addr, uint32_t v)
{
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__global__ void __launch_bounds__(kAttnThreads, 1) attention_kernel(const AttnArgs a)
{
    pdl_begin();
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t mbar_s, mbar_o;
    __shared__ uint32_t tmem_base_s;
    __shared__ float gs_k[kBN], gs_v[kBN];

    const int tid = threadIdx.x, warp = tid >> 5;
    const int qt = blockIdx.x, h = blockIdx.y;
    const uint32_t base = (static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw)) + 1023u) & ~1023u;
    const uint32_t sQ = base, sK = base + kTileBytes, sV = base + 2 * kTileBytes, sP = base + 3 * kTileBytes;
    const uint32_t bar_s = static_cast<uint32_t>(__cvta_generic_to_shared(&mbar_s));
    const uint32_t bar_o = static_cast<uint32_t>(__cvta_generic_to_shared(&mbar_o));
    const int64_t H = a.heads;

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         static_cast<uint32_t>(__cvta_generic_to_shared(&tmem_base_s))),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_s) : "memory");
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_o) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // Q tile -> shared memory (rows past n_q are zero)
    for (int i = tid; i < kBM * 16; i += kAttnThreads) {
        const int row = i >> 4, kb = (i >> 3) & 1, ch = i & 7;
        const int64_t qrow = static_cast<int64_t>(qt) * kBM + row;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (qrow < a.n_q)
            v = ld_nc_v4(a.q + (qrow * H + h) * kD + kb * 64 + ch * 8);
        st_shared_v4(sQ + sw128(row, kb, ch), v.x, v.y, v.z, v.w);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = tmem_base_s;
    const uint32_t tmem_s = tmem, tmem_o = tmem + kBN;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;

    float m_run = -INFINITY, l_run = 0.0f;
    bool ok = true;
    // the mbarrier phase whose MMAs are in flight (waited for again before TMEM is freed
    // when a wait times out)
    uint32_t pending_bar = 0, pending_parity = 0;
    const int64_t n_tiles = (a.n_kv + kBN - 1) / kBN;
    for (int64_t j = 0; j < n_tiles && ok; ++j) {
        const int64_t key0 = j * kBN;
        // the previous tile's MMAs must be done before K, V^T, P and O are touched again
        if (j > 0) {
            ok = __syncthreads_and(wait_phase(bar_o, static_cast<uint32_t>((j - 1) & 1)));
            if (!ok)
                break;
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        }
        // per-key global scales of the tile (one amax chunk per key)
        {
            const int64_t key = key0 + tid;
            float gk = 0.0f, gv = 0.0f;
            if (key < a.n_kv) {
                const int64_t chunk = key / a.tokens_per_chunk;
                gk = __fdiv_rn(__ldg(a.ka + chunk), 2688.0f);
                gv = __fdiv_rn(__ldg(a.va + chunk), 2688.0f);
            }
            gs_k[tid] = gk;
            gs_v[tid] = gv;
        }
        __syncthreads();
        // K tile: key rows, 8 blocks of 16 dims each -> two 16-byte chunks per block
        for (int i = tid; i < kBN * 8; i += kAttnThreads) {
            const int key = i >> 3, blk = i & 7;
            uint32_t y[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
            if (key0 + key < a.n_kv)
                dequant16(a.kp, a.ks, ((key0 + key) * H + h) * 8 + blk, gs_k[key], y);
            const int kb = blk >> 2, ch = (blk & 3) * 2;
            st_shared_v4(sK + sw128(key, kb, ch), y[0], y[1], y[2], y[3]);
            st_shared_v4(sK + sw128(key, kb, ch + 1), y[4], y[5], y[6], y[7]);
        }
        // V^T tile: dim rows; a thread takes a pair of keys and one block of 16 dims and
        // writes, per dim, the two keys' values as one 32-bit word
        for (int i = tid; i < (kBN / 2) * 8; i += kAttnThreads) {
            const int pair = i & 63, blk = i >> 6;
            const int k0 = 2 * pair;
            uint32_t y0[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u}, y1[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
            if (key0 + k0 < a.n_kv)
                dequant16(a.vp, a.vs, ((key0 + k0) * H + h) * 8 + blk, gs_v[k0], y0);
            if (key0 + k0 + 1 < a.n_kv)
                dequant16(a.vp, a.vs, ((key0 + k0 + 1) * H + h) * 8 + blk, gs_v[k0 + 1], y1);
            const int kb = k0 >> 6, ch = (k0 & 63) >> 3, in_chunk = (k0 & 7) * 2;
#pragma unroll
            for (int d = 0; d < 16; ++d) {
                const uint32_t lo = (d & 1) ? (y0[d >> 1] >> 16) : (y0[d >> 1] & 0xFFFFu);
                const uint32_t hi = (d & 1) ? (y1[d >> 1] >> 16) : (y1[d >> 1] & 0xFFFFu);
                st_shared_b32(sV + sw128(blk * 16 + d, kb, ch) + in_chunk, lo | (hi << 16));
            }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncthreads();
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        // S = Q K^T
        if (tid == 0) {
            mma_tile(tmem_s, sQ, sK, false);
            commit(bar_s);
        }
        pending_bar = bar_s;
        pending_parity = static_cast<uint32_t>(j & 1);
        ok = __syncthreads_and(wait_phase(bar_s, static_cast<uint32_t>(j & 1)));
        if (!ok)
            break;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        // online softmax on row tid: pass 1, the row max of this tile
        const int valid = static_cast<int>(a.n_kv - key0 < kBN ? a.n_kv - key0 : kBN);
        float m_tile = -INFINITY;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
            float s[32];
            tmem_ld32(tmem_s + lane_off + c * 32, s);
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (c * 32 + i < valid)
                    m_tile = fmaxf(m_tile, s[i] * a.scale_log2);
        }
        const float m_new = fmaxf(m_run, m_tile);
        const float alpha = exp2f(m_run - m_new);
        // pass 2: P = exp2(s * scale_log2 - m_new), bf16, into row tid of P (K-major)
        float l_tile = 0.0f;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
            float s[32];
            tmem_ld32(tmem_s + lane_off + c * 32, s);
            uint32_t pw[16];
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
                const float p0 = c * 32 + i < valid ? exp2f(s[i] * a.scale_log2 - m_new) : 0.0f;
                const float p1 = c * 32 + i + 1 < valid ? exp2f(s[i + 1] * a.scale_log2 - m_new) : 0.0f;
                l_tile += p0;
                l_tile += p1;
                pw[i >> 1] = bf16x2_from_f32(p1, p0);
            }
            const int kb = c >> 1, ch0 = (c & 1) * 4;
#pragma unroll
            for (int u = 0; u < 4; ++u)
                st_shared_v4(sP + sw128(tid, kb, ch0 + u), pw[4 * u], pw[4 * u + 1], pw[4 * u + 2], pw[4 * u + 3]);
        }
        l_run = l_run * alpha + l_tile;
        m_run = m_new;
        // rescale O by alpha before this tile's P V accumulates into it
        if (j > 0) {
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                float o[32];
                tmem_ld32(tmem_o + lane_off + c * 32, o);
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    o[i] *= alpha;
                tmem_st32(tmem_o + lane_off + c * 32, o);
            }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        __syncthreads();
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        // O += P V
        if (tid == 0) {
            mma_tile(tmem_o, sP, sV, j > 0);
            commit(bar_o);
        }
        pending_bar = bar_o;
        pending_parity = static_cast<uint32_t>(j & 1);
    }
    if (ok && n_tiles > 0) {
        ok = __syncthreads_and(wait_phase(bar_o, static_cast<uint32_t>((n_tiles - 1) & 1)));
        if (ok) {
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const int64_t qrow = static_cast<int64_t>(qt) * kBM + tid;
            const float inv_l = 1.0f / l_run;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                float o[32];
                tmem_ld32(tmem_o + lane_off + c * 32, o);
                if (qrow < a.n_q) {
                    uint32_t w[16];
#pragma unroll
                    for (int i = 0; i < 32; i += 2)
                        w[i >> 1] = bf16x2_from_f32(o[i + 1] * inv_l, o[i] * inv_l);
                    uint16_t* dst = a.o + (qrow * H + h) * kD + c * 32;
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        st_v4(dst + 8 * u, w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
                }
            }
        }
    }
    if (!ok) {
        if (tid == 0)
            atomicExch(a.status, 1);
        if (pending_bar != 0)
            wait_phase(pending_bar, pending_parity);
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
}

}  // namespace
}  // namespace kvq

using namespace kvq;

extern "C" {

kvq_status kvq_attention(const void* q, int32_t n_queries, int32_t heads, const kvq_cache* k_cache,
                         const kvq_cache* v_cache, int64_t n_keys, float softmax_scale, void* out, int* status,
                         kvq_stream_t stream)
{
    NvtxRange nvtx_range("kvq_attention");
    if (k_cache == nullptr || v_cache == nullptr)
        return fail(KVQ_ERR_INVALID_ARG, "kvq_attention: null cache");
    if (k_cache->head_dim != kD || v_cache->head_dim != kD)
        return fail(KVQ_ERR_UNSUPPORTED, "kvq_attention: head_dim must be 128");
    if (n_queries < 0 || heads <= 0 || n_keys < 0)
        return fail(KVQ_ERR_INVALID_ARG, "kvq_attention: bad sizes");
    if (n_queries == 0)
        return ok();
    if (n_keys == 0)
        return fail(KVQ_ERR_INVALID_ARG, "kvq_attention: no keys");
    if (q == nullptr || out == nullptr || status == nullptr)
        return fail(KVQ_ERR_INVALID_ARG, "kvq_attention: null pointer");
    for (const kvq_cache* c : {k_cache, v_cache}) {
        if (c->packed == nullptr || c->scales == nullptr || c->amax == nullptr)
            return fail(KVQ_ERR_INVALID_ARG, "kvq_attention: null cache buffer");
        if (c->rows_per_chunk <= 0 || c->rows_per_chunk % heads != 0)
            return fail(KVQ_ERR_INVALID_ARG, "kvq_attention: rows_per_chunk must be a multiple of heads");
        if (n_keys * heads > c->capacity_rows)
            return fail(KVQ_ERR_CAPACITY, "kvq_attention: %lld keys past the cache capacity",
                        static_cast<long long>(n_keys));
        if (!aligned(c->packed, 8) || !aligned(c->amax, 4))
            return fail(KVQ_ERR_MISALIGNED, "kvq_attention: cache packed 8-byte, amax 4-byte aligned");
    }
    if (k_cache->rows_per_chunk != v_cache->rows_per_chunk)
        return fail(KVQ_ERR_INVALID_ARG, "kvq_attention: K and V caches differ in rows_per_chunk");
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(status, 4))
        return fail(KVQ_ERR_MISALIGNED, "kvq_attention: q and out must be 16-byte aligned");
    AttnArgs a;
    a.q = static_cast<const uint16_t*>(q);
    a.o = static_cast<uint16_t*>(out);
    a.kp = k_cache->packed;
    a.ks = k_cache->scales;
    a.ka = k_cache->amax;
    a.vp = v_cache->packed;
    a.vs = v_cache->scales;
    a.va = v_cache->amax;
    a.n_q = n_queries;
    a.heads = heads;
    a.n_kv = n_keys;
    a.tokens_per_chunk = k_cache->rows_per_chunk / heads;
    a.scale_log2 = softmax_scale * 1.4426950408889634f;
    a.status = status;
    cudaError_t e = cudaFuncSetAttribute(attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess)
        return launched(e, "kvq_attention");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((n_queries + kBM - 1) / kBM, heads);
    cfg.blockDim = dim3(kAttnThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = reinterpret_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    kvq_status st = launched(cudaLaunchKernelEx(&cfg, attention_kernel, a), "kvq_attention");
    return st == KVQ_OK ? ok() : st;
}

}  // extern "C"
