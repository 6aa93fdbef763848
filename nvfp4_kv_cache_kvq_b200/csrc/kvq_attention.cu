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
// Work unit (one CTA): two query tiles of 128 rows of one head against one range of key
// tiles (128 keys each). When the keys are split over several units, each leaves a
// partial result (unnormalized O, reference max m and sum l per row) in the caller's
// workspace and combine_kernel merges them; the split count is chosen so the units fill
// the SMs in whole waves.
//
// Roles inside the CTA (416 threads):
//   warps 0-3, 4-7  softmax of query tile 0 / 1: thread t owns row t (TMEM lane t);
//   warps 8-11      producers: load the packed K and V of a key tile (one tile ahead, in
//                   registers) and dequantize it into 128B-swizzled shared memory, K as
//                   key rows and V transposed (dim rows), both K-major MMA operands;
//   warp 12         allocates TMEM; its lane 0 issues every tcgen05.mma and commit.
// TMEM (512 columns, fp32): S0, S1 at columns 0 and 128; O0, O1 at 256 and 384.
// The MMA thread issues, per key tile j: PV0(j), S0(j+1), PV1(j), S1(j+1), so each query
// tile's softmax overlaps the other tile's MMAs (the ping-pong of FlashAttention-4 on
// Blackwell). The softmax keeps a reference row max and rescales O only when the max
// grows by more than 2^8 (exact in real arithmetic: O and l share the reference). Every
// wait is bounded (1 s); on a timeout the kernel records an error, lets its MMAs drain,
// frees its TMEM and returns.
#include <cuda_runtime.h>

#include <cstdint>

#include "kvq.h"
#include "kvq_common.h"
#include "kvq_device.cuh"

namespace kvq {
namespace {

constexpr int kBM = 128;  // rows per query tile
constexpr int kQT = 2;    // query tiles per CTA
constexpr int kBN = 128;  // keys per tile
constexpr int kD = 128;   // head_dim (the only one supported)
constexpr int kSoftmaxThreads = kQT * 128;
constexpr int kProducerThreads = 128;
constexpr int kMmaWarp = (kSoftmaxThreads + kProducerThreads) / 32;  // 12
constexpr int kAttnThreads = (kMmaWarp + 1) * 32;                   // 416
// (13 warps: the SM sub-partition that holds 4 of them caps registers at 128 per thread)
constexpr int kTileBytes = 32768;  // one 128 x 128 bf16 operand
// dynamic shared memory: Q0, Q1, K, V^T, P0, P1 (each 1024-aligned)
constexpr int kOffQ = 0, kOffK = 2 * kTileBytes, kOffV = 3 * kTileBytes, kOffP = 4 * kTileBytes;
constexpr int kSmemBytes = 6 * kTileBytes + 1024;  // + alignment slack
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitNs = 1000000000ull;  // give up on an mbarrier after 1 s
constexpr float kRescaleLog2 = 8.0f;          // rescale O when the row max grows by > 2^8
constexpr int kMaxSplits = 64;
constexpr int kCombineThreads = 256;  // 8 rows (warps) per CTA
constexpr uint64_t kPartialBytesPerRow = kD * 4 + 8;

// mbarriers
enum {
    kKFull, kKEmpty, kVFull, kVEmpty,
    kSFull0, kSFull1, kPFull0, kPFull1, kODone0, kODone1,
    kDone, kNumBars
};

struct AttnArgs {
    const uint16_t* q;  // bf16 [n_q, heads, 128]
    uint16_t* o;        // bf16 [n_q, heads, 128]
    float* part_o;      // fp32 [splits][n_q][heads][128] (splits > 1)
    float2* part_ml;    // (m, l) [splits][n_q][heads] (splits > 1)
    const uint8_t* kp;  // K cache: codes, scales, chunk amax
    const uint8_t* ks;
    const float* ka;
    const uint8_t* vp;  // V cache
    const uint8_t* vs;
    const float* va;
    int32_t n_q, heads, splits, key_tiles;
    int64_t n_kv;              // keys (tokens)
    int64_t tokens_per_chunk;  // keys per amax chunk
    float scale_log2;          // softmax scale * log2(e)
    int* status;               // set to 1 on a wait timeout
};

// ------------------------------------------------------------------ PTX wrappers

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

// D (TMEM) (+)= A[128 x 128] B[128 x 128]^T, both K-major in shared memory, as 8 MMAs of K = 16.
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

__device__ __forceinline__ void mbar_init(uint32_t mbar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(mbar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t mbar)
{
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(mbar) : "memory");
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

// The same wait, decided for the whole warp (tcgen05.ld/st need a converged warp).
__device__ __forceinline__ bool warp_wait(uint32_t mbar, uint32_t parity)
{
    return __all_sync(0xFFFFFFFFu, wait_phase(mbar, parity));
}

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

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

// 2^x by the hardware approximation (relative error about 2^-22; 0 for x = -inf).
__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ void st_shared_v2(uint32_t addr, uint32_t a, uint32_t b)
{
    asm volatile("st.shared.v2.b32 [%0], {%1,%2};" ::"r"(addr), "r"(a), "r"(b) : "memory");
}

// ------------------------------------------------------------------ dequantization

// Eight codes (one word) of a block with scale S -> four bf16x2 words: y = bf16_rne(value
// * S), the fp32 product rounded once -- the dequantizer's arithmetic, so the same bits.
__device__ __forceinline__ void dequant8(uint32_t codes, float S, uint32_t (&y)[4])
{
    float v[8];
    e2m1x8_to_f32(codes, v);
    const uint64_t S2 = f32x2_pack(S, S);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float lo, hi;
        f32x2_unpack(f32x2_mul(f32x2_pack(v[2 * j], v[2 * j + 1]), S2), lo, hi);
        y[j] = bf16x2_from_f32(hi, lo);
    }
}

// S = e4m3_value(code) * gs for the scale code in byte `byte` of `codes`.
__device__ __forceinline__ float block_scale(uint32_t codes, int byte, float gs)
{
    float lo, hi;
    e4m3x2_to_f32((codes >> (8 * byte)) & 0xFFu, lo, hi);
    return __fmul_rn(lo, gs);
}

// The packed bytes of one key tile a producer thread dequantizes: one key's whole K row
// (8 blocks), and 4 consecutive keys x 2 blocks (32 dims) of V.
struct RawTile {
    uint4 kc[4];      // K codes, 64 bytes
    uint2 ksc;        // K scale codes, blocks 0..7
    float kgs;        // K global scale of the key
    uint4 vc[4];      // V codes of keys 0..3 (2 blocks = 16 bytes each)
    uint32_t vsc[2];  // V scale codes: key k's two bytes at bits 16*(k&1) of vsc[k>>1]
    float vgs[4];
};

__device__ __forceinline__ float global_scale(const float* amax, int64_t key, int64_t tokens_per_chunk)
{
    return __fdiv_rn(__ldg(amax + key / tokens_per_chunk), 2688.0f);
}

// Producer p's share of key tile [key0, key0 + 128): K row of key key0 + p; V keys
// key0 + 4*(p%32) .. +3, dims 32*(p/32) .. +31. Keys past n_kv read as zero codes.
__device__ __forceinline__ void load_tile(const AttnArgs& a, int h, int64_t key0, int p, RawTile& r)
{
    const int64_t H = a.heads;
    const int64_t kkey = key0 + p;
    if (kkey < a.n_kv) {
        const int64_t row = kkey * H + h;
        const uint8_t* src = a.kp + row * 64;
#pragma unroll
        for (int i = 0; i < 4; ++i)
            r.kc[i] = ld_nc_v4(src + 16 * i);
        r.ksc = ld_nc_v2(a.ks + row * 8);
        r.kgs = global_scale(a.ka, kkey, a.tokens_per_chunk);
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            r.kc[i] = make_uint4(0u, 0u, 0u, 0u);
        r.ksc = make_uint2(0u, 0u);
        r.kgs = 0.0f;
    }
    const int quad = p & 31, quarter = p >> 5;
    r.vsc[0] = r.vsc[1] = 0u;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int64_t key = key0 + 4 * quad + k;
        if (key < a.n_kv) {
            const int64_t row = key * H + h;
            r.vc[k] = ld_nc_v4(a.vp + row * 64 + quarter * 16);
            const uint32_t sc = __ldg(reinterpret_cast<const uint16_t*>(a.vs + row * 8 + quarter * 2));
            r.vsc[k >> 1] |= sc << (16 * (k & 1));
            r.vgs[k] = global_scale(a.va, key, a.tokens_per_chunk);
        } else {
            r.vc[k] = make_uint4(0u, 0u, 0u, 0u);
            r.vgs[k] = 0.0f;
        }
    }
}

// K row p of the tile into sK (key rows, dims contiguous, K-major).
__device__ __forceinline__ void store_k(const RawTile& r, int p, uint32_t sK)
{
#pragma unroll
    for (int b = 0; b < 8; ++b) {
        const float S = block_scale(b < 4 ? r.ksc.x : r.ksc.y, b & 3, r.kgs);
        const uint4 c = r.kc[b >> 1];
        uint32_t y0[4], y1[4];
        dequant8((b & 1) ? c.z : c.x, S, y0);
        dequant8((b & 1) ? c.w : c.y, S, y1);
        const int kb = b >> 2, ch = 2 * (b & 3);
        st_shared_v4(sK + sw128(p, kb, ch), y0[0], y0[1], y0[2], y0[3]);
        st_shared_v4(sK + sw128(p, kb, ch + 1), y1[0], y1[1], y1[2], y1[3]);
    }
}

// V of 4 keys x 32 dims into sVt (dim rows, keys contiguous, K-major): per dim, the four
// keys' values as one 8-byte store.
__device__ __forceinline__ void store_v(const RawTile& r, int p, uint32_t sV)
{
    const int quad = p & 31, quarter = p >> 5;
    const int kb = quad >> 4, chunk = (quad & 15) >> 1, byte = (quad & 1) * 8;
#pragma unroll
    for (int bb = 0; bb < 2; ++bb) {
        uint32_t y[4][8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float S = block_scale(r.vsc[k >> 1] >> (16 * (k & 1)), bb, r.vgs[k]);
            uint32_t lo[4], hi[4];
            dequant8(bb ? r.vc[k].z : r.vc[k].x, S, lo);
            dequant8(bb ? r.vc[k].w : r.vc[k].y, S, hi);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                y[k][i] = lo[i];
                y[k][4 + i] = hi[i];
            }
        }
#pragma unroll
        for (int dp = 0; dp < 8; ++dp) {
            const int d = quarter * 32 + bb * 16 + 2 * dp;
            st_shared_v2(sV + sw128(d, kb, chunk) + byte, __byte_perm(y[0][dp], y[1][dp], 0x5410),
                         __byte_perm(y[2][dp], y[3][dp], 0x5410));
            st_shared_v2(sV + sw128(d + 1, kb, chunk) + byte, __byte_perm(y[0][dp], y[1][dp], 0x7632),
                         __byte_perm(y[2][dp], y[3][dp], 0x7632));
        }
    }
}

// ------------------------------------------------------------------ kernels

__global__ void __launch_bounds__(kAttnThreads, 1) attention_kernel(const AttnArgs a)
{
    pdl_begin();
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t bars[kNumBars];
    __shared__ uint32_t tmem_base_s;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qp = blockIdx.x, split = blockIdx.y, h = blockIdx.z;
    const int t_begin = static_cast<int>(static_cast<int64_t>(split) * a.key_tiles / a.splits);
    const int t_end = static_cast<int>(static_cast<int64_t>(split + 1) * a.key_tiles / a.splits);
    const int n_tiles = t_end - t_begin;
    const int64_t q0 = static_cast<int64_t>(qp) * (kQT * kBM);
    const int n_qt = a.n_q - q0 > kBM ? 2 : 1;  // query tiles holding rows
    const int64_t H = a.heads;

    const uint32_t base = (static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw)) + 1023u) & ~1023u;
    const uint32_t bar0 = static_cast<uint32_t>(__cvta_generic_to_shared(&bars[0]));
    auto bar = [bar0](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };

    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         static_cast<uint32_t>(__cvta_generic_to_shared(&tmem_base_s))),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        mbar_init(bar(kKFull), kProducerThreads);
        mbar_init(bar(kVFull), kProducerThreads);
        mbar_init(bar(kKEmpty), 1);
        mbar_init(bar(kVEmpty), 1);
        mbar_init(bar(kSFull0), 1);
        mbar_init(bar(kSFull1), 1);
        mbar_init(bar(kPFull0), 128);
        mbar_init(bar(kPFull1), 128);
        mbar_init(bar(kODone0), 1);
        mbar_init(bar(kODone1), 1);
        mbar_init(bar(kDone), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // both query tiles -> shared memory (rows past n_q are zero)
    for (int i = tid; i < kQT * kBM * 16; i += kAttnThreads) {
        const int g = i >> 11, row = (i >> 4) & 127, kb = (i >> 3) & 1, ch = i & 7;
        const int64_t qrow = q0 + g * kBM + row;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (qrow < a.n_q)
            v = ld_nc_v4(a.q + (qrow * H + h) * kD + kb * 64 + ch * 8);
        st_shared_v4(base + kOffQ + g * kTileBytes + sw128(row, kb, ch), v.x, v.y, v.z, v.w);
    }
    fence_async_smem();
    tc_before_sync();
    __syncthreads();
    tc_after_sync();
    const uint32_t tmem = tmem_base_s;

    if (tid < kSoftmaxThreads) {
        // ---------------------------------------------------------------- softmax
        const int g = tid >> 7, r = tid & 127;
        if (g < n_qt) {
            const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
            const uint32_t tS = tmem + g * 128 + lane_off, tO = tmem + 256 + g * 128 + lane_off;
            const uint32_t sP = base + kOffP + g * kTileBytes;
            const uint32_t bS = bar(kSFull0 + g), bP = bar(kPFull0 + g), bO = bar(kODone0 + g);
            float m_run = -INFINITY, l_run = 0.0f;
            bool ok = true;
            for (int j = 0; j < n_tiles; ++j) {
                ok = warp_wait(bS, j & 1);
                if (!ok)
                    break;
                tc_after_sync();
                const int64_t key0 = static_cast<int64_t>(t_begin + j) * kBN;
                const int valid = static_cast<int>(a.n_kv - key0 < kBN ? a.n_kv - key0 : kBN);
                // pass 1: the row max of this tile
                float mt = -INFINITY;
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    float s[32];
                    tmem_ld32(tS + c * 32, s);
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (c * 32 + i < valid)
                            mt = fmaxf(mt, s[i]);
                }
                mt = __fmul_rn(mt, a.scale_log2);
                const float m_cand = fmaxf(m_run, mt);
                const bool need = m_cand > m_run + kRescaleLog2;
                const float m_use = need ? m_cand : m_run;
                const float alpha = need ? ex2(m_run - m_use) : 1.0f;
                // P and O of this query tile are free once the previous P V is done
                if (j > 0) {
                    ok = warp_wait(bO, (j - 1) & 1);
                    if (!ok)
                        break;
                    tc_after_sync();
                }
                // pass 2: P = bf16(2^(s * scale_log2 - m)) into row r of P (K-major)
                float lt = 0.0f;
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    float s[32];
                    tmem_ld32(tS + c * 32, s);
                    uint32_t pw[16];
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        const float p0 = c * 32 + i < valid ? ex2(__fmaf_rn(s[i], a.scale_log2, -m_use)) : 0.0f;
                        const float p1 =
                            c * 32 + i + 1 < valid ? ex2(__fmaf_rn(s[i + 1], a.scale_log2, -m_use)) : 0.0f;
                        lt = __fadd_rn(lt, p0);
                        lt = __fadd_rn(lt, p1);
                        pw[i >> 1] = bf16x2_from_f32(p1, p0);
                    }
                    const int kb = c >> 1, ch0 = (c & 1) * 4;
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        st_shared_v4(sP + sw128(r, kb, ch0 + u), pw[4 * u], pw[4 * u + 1], pw[4 * u + 2],
                                     pw[4 * u + 3]);
                }
                l_run = __fmaf_rn(l_run, alpha, lt);
                m_run = m_use;
                // rescale O (the warp does it if any of its rows needs it)
                if (j > 0 && __any_sync(0xFFFFFFFFu, need)) {
#pragma unroll 1
                    for (int c = 0; c < 4; ++c) {
                        float o[32];
                        tmem_ld32(tO + c * 32, o);
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            o[i] = __fmul_rn(o[i], alpha);
                        tmem_st32(tO + c * 32, o);
                    }
                }
                fence_async_smem();
                tc_before_sync();
                mbar_arrive(bP);
            }
            if (ok && n_tiles > 0) {
                ok = warp_wait(bO, (n_tiles - 1) & 1);
                if (ok) {
                    tc_after_sync();
                    const int64_t qrow = q0 + g * kBM + r;
                    const bool has_row = qrow < a.n_q;
                    const int64_t prow = (static_cast<int64_t>(split) * a.n_q + qrow) * H + h;
                    const float inv_l = 1.0f / l_run;
#pragma unroll 1
                    for (int c = 0; c < 4; ++c) {
                        float o[32];
                        tmem_ld32(tO + c * 32, o);
                        if (!has_row)
                            continue;
                        if (a.splits == 1) {
                            uint32_t w[16];
#pragma unroll
                            for (int i = 0; i < 32; i += 2)
                                w[i >> 1] = bf16x2_from_f32(__fmul_rn(o[i + 1], inv_l), __fmul_rn(o[i], inv_l));
                            uint16_t* dst = a.o + (qrow * H + h) * kD + c * 32;
#pragma unroll
                            for (int u = 0; u < 4; ++u)
                                st_v4(dst + 8 * u, w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
                        } else {
                            float* dst = a.part_o + prow * kD + c * 32;
#pragma unroll
                            for (int u = 0; u < 8; ++u)
                                st_v4(dst + 4 * u, __float_as_uint(o[4 * u]), __float_as_uint(o[4 * u + 1]),
                                      __float_as_uint(o[4 * u + 2]), __float_as_uint(o[4 * u + 3]));
                        }
                    }
                    if (has_row && a.splits > 1)
                        a.part_ml[prow] = make_float2(m_run, l_run);
                }
            }
            if (!ok && lane == 0)
                atomicExch(a.status, 1);
        }
    } else if (warp < kMmaWarp) {
        // ---------------------------------------------------------------- producers
        const int p = tid - kSoftmaxThreads;
        const uint32_t sK = base + kOffK, sV = base + kOffV;
        RawTile cur, nxt;
        bool ok = true;
        if (n_tiles > 0)
            load_tile(a, h, static_cast<int64_t>(t_begin) * kBN, p, cur);
        for (int j = 0; j < n_tiles; ++j) {
            if (j + 1 < n_tiles)
                load_tile(a, h, static_cast<int64_t>(t_begin + j + 1) * kBN, p, nxt);
            if (j > 0 && !(ok = wait_phase(bar(kKEmpty), (j - 1) & 1)))
                break;
            store_k(cur, p, sK);
            fence_async_smem();
            mbar_arrive(bar(kKFull));
            if (j > 0 && !(ok = wait_phase(bar(kVEmpty), (j - 1) & 1)))
                break;
            store_v(cur, p, sV);
            fence_async_smem();
            mbar_arrive(bar(kVFull));
            cur = nxt;
        }
        if (!ok && lane == 0)
            atomicExch(a.status, 1);
    } else if (lane == 0) {
        // ---------------------------------------------------------------- MMA issue
        bool ok = true;
        if (n_tiles > 0) {
            ok = wait_phase(bar(kKFull), 0);
            if (ok) {
                tc_after_sync();
                for (int g = 0; g < n_qt; ++g) {
                    mma_tile(tmem + g * 128, base + kOffQ + g * kTileBytes, base + kOffK, false);
                    commit(bar(kSFull0 + g));
                }
                commit(bar(kKEmpty));
            }
            for (int j = 0; ok && j < n_tiles; ++j) {
                if (!(ok = wait_phase(bar(kVFull), j & 1)))
                    break;
                tc_after_sync();
                for (int g = 0; g < n_qt; ++g) {
                    if (!(ok = wait_phase(bar(kPFull0 + g), j & 1)))
                        break;
                    tc_after_sync();
                    mma_tile(tmem + 256 + g * 128, base + kOffP + g * kTileBytes, base + kOffV, j > 0);
                    commit(bar(kODone0 + g));
                    if (g == n_qt - 1)
                        commit(bar(kVEmpty));
                    if (j + 1 < n_tiles) {
                        if (g == 0) {
                            if (!(ok = wait_phase(bar(kKFull), (j + 1) & 1)))
                                break;
                            tc_after_sync();
                        }
                        mma_tile(tmem + g * 128, base + kOffQ + g * kTileBytes, base + kOffK, false);
                        commit(bar(kSFull0 + g));
                        if (g == n_qt - 1)
                            commit(bar(kKEmpty));
                    }
                }
            }
        }
        commit(bar(kDone));  // completes once every MMA issued above has
        if (!wait_phase(bar(kDone), 0))
            ok = false;
        if (!ok)
            atomicExch(a.status, 1);
    }
    tc_before_sync();
    __syncthreads();
    if (warp == kMmaWarp)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
}

// Merge the per-split partial results of one (query, head) row per warp:
// out = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s, M = max_s m_s.
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const AttnArgs a)
{
    pdl_begin();
    const int64_t rows = static_cast<int64_t>(a.n_q) * a.heads;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * (kCombineThreads / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows)
        return;
    float M = -INFINITY;
    for (int s = 0; s < a.splits; ++s)
        M = fmaxf(M, a.part_ml[s * rows + row].x);
    float L = 0.0f, acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    for (int s = 0; s < a.splits; ++s) {
        const float2 ml = a.part_ml[s * rows + row];
        const float w = ex2(ml.x - M);
        L = __fmaf_rn(w, ml.y, L);
        const float4 o = *reinterpret_cast<const float4*>(a.part_o + (s * rows + row) * kD + 4 * lane);
        acc[0] = __fmaf_rn(w, o.x, acc[0]);
        acc[1] = __fmaf_rn(w, o.y, acc[1]);
        acc[2] = __fmaf_rn(w, o.z, acc[2]);
        acc[3] = __fmaf_rn(w, o.w, acc[3]);
    }
    const float inv = 1.0f / L;
    st_v2(a.o + row * kD + 4 * lane, bf16x2_from_f32(__fmul_rn(acc[1], inv), __fmul_rn(acc[0], inv)),
          bf16x2_from_f32(__fmul_rn(acc[3], inv), __fmul_rn(acc[2], inv)));
}

int sm_count()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) !=
                                                  cudaSuccess)
        return 0;
    return n;
}

// Key splits: minimize waves x (key tiles per unit + 2), the 2 standing for the unit's
// fixed costs (query load, pipeline fill, epilogue); ties go to fewer splits.
int choose_splits(int64_t units, int key_tiles, int sms)
{
    if (sms <= 0)
        return 1;
    int best = 1;
    int64_t best_cost = INT64_MAX;
    for (int s = 1; s <= kMaxSplits && s <= key_tiles; ++s) {
        const int64_t waves = (units * s + sms - 1) / sms;
        const int64_t cost = waves * ((key_tiles + s - 1) / s + 2);
        if (cost < best_cost) {
            best_cost = cost;
            best = s;
        }
    }
    return best;
}

uint64_t partial_bytes(int splits, int32_t n_q, int32_t heads)
{
    return splits > 1 ? static_cast<uint64_t>(splits) * n_q * heads * kPartialBytesPerRow : 0;
}

}  // namespace
}  // namespace kvq

using namespace kvq;

extern "C" {

kvq_status kvq_attention_workspace_bytes(int32_t n_queries, int32_t heads, int64_t n_keys, uint64_t* bytes)
{
    if (bytes == nullptr || n_queries < 0 || heads <= 0 || n_keys < 0)
        return fail(KVQ_ERR_INVALID_ARG, "kvq_attention_workspace_bytes: bad arguments");
    *bytes = 0;
    if (n_queries == 0 || n_keys == 0)
        return ok();
    const int key_tiles = static_cast<int>((n_keys + kBN - 1) / kBN);
    const int64_t units = static_cast<int64_t>((n_queries + kQT * kBM - 1) / (kQT * kBM)) * heads;
    *bytes = partial_bytes(choose_splits(units, key_tiles, sm_count()), n_queries, heads);
    return ok();
}

kvq_status kvq_attention(const void* q, int32_t n_queries, int32_t heads, const kvq_cache* k_cache,
                         const kvq_cache* v_cache, int64_t n_keys, float softmax_scale, void* out, void* workspace,
                         uint64_t workspace_bytes, int* status, kvq_stream_t stream)
{
    NvtxRange nvtx_range("kvq_attention");
    if (k_cache == nullptr || v_cache == nullptr)
        return fail(KVQ_ERR_INVALID_ARG, "kvq_attention: null cache");
    if (k_cache->head_dim != kD || v_cache->head_dim != kD)
        return fail(KVQ_ERR_UNSUPPORTED, "kvq_attention: head_dim must be 128");
    if (n_queries < 0 || heads <= 0 || heads > 65535 || n_keys < 0)
        return fail(KVQ_ERR_INVALID_ARG, "kvq_attention: bad sizes");
    if (!(softmax_scale > 0.0f) || !(softmax_scale < INFINITY))
        return fail(KVQ_ERR_INVALID_ARG, "kvq_attention: softmax_scale must be positive and finite");
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
        if (!aligned(c->packed, 16) || !aligned(c->scales, 8) || !aligned(c->amax, 4))
            return fail(KVQ_ERR_MISALIGNED,
                        "kvq_attention: cache packed 16-byte, scales 8-byte, amax 4-byte aligned");
    }
    if (k_cache->rows_per_chunk != v_cache->rows_per_chunk)
        return fail(KVQ_ERR_INVALID_ARG, "kvq_attention: K and V caches differ in rows_per_chunk");
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(status, 4))
        return fail(KVQ_ERR_MISALIGNED, "kvq_attention: q and out must be 16-byte aligned");
    const int64_t key_tiles = (n_keys + kBN - 1) / kBN;
    if (key_tiles > INT32_MAX)
        return fail(KVQ_ERR_INVALID_ARG, "kvq_attention: too many keys");
    const int64_t qpairs = (n_queries + kQT * kBM - 1) / (kQT * kBM);
    int splits = choose_splits(qpairs * heads, static_cast<int>(key_tiles), sm_count());
    while (splits > 1 && partial_bytes(splits, n_queries, heads) > workspace_bytes)
        --splits;
    if (splits > 1 && (workspace == nullptr || !aligned(workspace, 16)))
        return fail(KVQ_ERR_MISALIGNED, "kvq_attention: workspace must be 16-byte aligned");

    AttnArgs a;
    a.q = static_cast<const uint16_t*>(q);
    a.o = static_cast<uint16_t*>(out);
    a.part_o = static_cast<float*>(workspace);
    a.part_ml = splits > 1 ? reinterpret_cast<float2*>(static_cast<uint8_t*>(workspace) +
                                                       static_cast<uint64_t>(splits) * n_queries * heads * kD * 4)
                           : nullptr;
    a.kp = k_cache->packed;
    a.ks = k_cache->scales;
    a.ka = k_cache->amax;
    a.vp = v_cache->packed;
    a.vs = v_cache->scales;
    a.va = v_cache->amax;
    a.n_q = n_queries;
    a.heads = heads;
    a.splits = splits;
    a.key_tiles = static_cast<int32_t>(key_tiles);
    a.n_kv = n_keys;
    a.tokens_per_chunk = k_cache->rows_per_chunk / heads;
    a.scale_log2 = softmax_scale * 1.4426950408889634f;
    a.status = status;

    cudaError_t e = cudaFuncSetAttribute(attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess)
        return launched(e, "kvq_attention");
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(qpairs), static_cast<unsigned>(splits), static_cast<unsigned>(heads));
    cfg.blockDim = dim3(kAttnThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = reinterpret_cast<cudaStream_t>(stream);
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    kvq_status st = launched(cudaLaunchKernelEx(&cfg, attention_kernel, a), "kvq_attention");
    if (st != KVQ_OK || splits == 1)
        return st == KVQ_OK ? ok() : st;
    const int64_t rows = static_cast<int64_t>(n_queries) * heads;
    const int64_t rows_per_cta = kCombineThreads / 32;
    cfg.gridDim = dim3(static_cast<unsigned>((rows + rows_per_cta - 1) / rows_per_cta));
    cfg.blockDim = dim3(kCombineThreads);
    cfg.dynamicSmemBytes = 0;
    st = launched(cudaLaunchKernelEx(&cfg, combine_kernel, a), "kvq_attention (combine)");
    return st == KVQ_OK ? ok() : st;
}

}  // extern "C"
