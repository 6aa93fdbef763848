// kvq_attention.cu -- attention reading the packed NVFP4 K/V cache directly: each K/V
// tile is dequantized into shared memory (the same arithmetic, hence the same bf16
// values, as kvq_dequantize_cache) and consumed there by tcgen05 tensor-core MMAs, so
// the dense bf16 cache is never written to HBM. The pages dequantize the active cache to
// BF16 before attention ("KV Cache Quantization for Self-Forcing Video Generation",
// appendix Table 3) and find that those transient BF16 buffers dominate peak memory
// (abstract; Figure 6); "How to Use KV Cache Quantization with LongLive's
// LongLiveQuantizationConfig" ("CUDA De-quantization Pipeline") dequantizes the cache while
// attention runs.
//
// Work unit (one CTA): two query tiles of 128 rows of one head against one range of key
// tiles (128 keys each). When the keys are split over several units, each leaves a
// partial result (unnormalized O, reference max m and sum l per row) in the caller's
// workspace and combine_kernel merges them; the split count is chosen so the units fill
// the SMs in whole waves. Three instantiations: single CTAs; CTA pairs (PAIR: a cluster
// of two issuing cta_group::2 MMAs with M = 256, each CTA holding its own 2 x 128 rows
// and dequantizing half of every K and V tile); and single CTAs whose two slots share
// one query tile and split the key range (DUAL, for units of at most 128 rows). The
// host splits the query rows into at most two launches (pairs over whole 512-row
// blocks, single or dual CTAs for the rest) by a cost model measured on this part.
//
// Roles inside the CTA (544 threads, 17 warps):
//   warps 0-3, 4-7  softmax of query tile 0 / 1 (with DUAL both take tile 0, each over
//                   its half of the key range): thread t owns row t (TMEM lane t). Per
//                   key tile: the row max of S first, then p = 2^(s - m) written as bf16
//                   into TMEM over the S columns already read. Warp 0 allocates and frees
//                   the TMEM.
//   warps 8-15      producers: load the packed K and V of a key tile (the next one while
//                   the current is consumed, in registers) and dequantize it into
//                   128B-swizzled shared memory as key rows: K is the K-major B operand of
//                   Q K^T, V the MN-major B operand of P V. K and V have two stages each.
//   warp 16         issues every tcgen05.mma (one elected lane) in the order S_0(0), S_1(0),
//                   then per key tile j: P_0 V(j), S_0(j+1), P_1 V(j), S_1(j+1). Tile 1's S
//                   thus lands half a period after tile 0's, and each tile's softmax runs
//                   while the other tile's MMAs execute (the ping-pong of FlashAttention-4
//                   on Blackwell); a tcgen05.mma blocks its issuer while the tensor pipe's
//                   queue is full, which is why no softmax thread issues them.
// TMEM (512 columns, fp32): S0, S1 at columns 0 and 128; O0, O1 at 256 and 384. P_g, the
// bf16 probabilities, is written over the first 64 columns of S_g (two keys per column)
// and is the A operand of P V straight from TMEM, so P never passes through shared
// memory and P V reads only V there. S_g(j+1) overwrites P_g(j) only after P V(j) has
// read it: a thread's tcgen05.mma operations run in the order it issues them.
// The softmax keeps a reference row max and rescales O only when the max grows by more
// than 2^8 (exact in real arithmetic: O and l share the reference). Every wait is bounded
// (1 s); on a timeout the kernel records an error, lets its MMAs drain, frees its TMEM
// and returns.
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

#include "kvq.h"
#include "kvq_common.h"
#include "kvq_device.cuh"
#include "kvq_testing.h"

namespace kvq {
namespace {

constexpr int kBM = 128;  // rows per query tile
constexpr int kQT = 2;    // query tiles per CTA
constexpr int kBN = 128;  // keys per tile
constexpr int kD = 128;   // head_dim (the only one supported)
constexpr int kSoftmaxThreads = kQT * 128;
constexpr int kProducerThreads = 256;
constexpr int kMmaWarp = (kSoftmaxThreads + kProducerThreads) / 32;  // warp 16 issues every MMA
constexpr int kAttnThreads = kSoftmaxThreads + kProducerThreads + 32;  // 544: 17 warps
constexpr int kTileBytes = 32768;  // one 128 x 128 bf16 operand
constexpr uint32_t kTmemCols = 512;

// Shared-memory geometry of one CTA. Alone (PAIR false) a CTA holds whole K and V tiles;
// in a CTA pair each holds half of every tile -- keys 64 rank .. + 63 of K, dims 64 rank
// .. + 63 of V -- the halves a cta_group::2 MMA takes from each CTA as its B operand.
// Layout: Q0, Q1, K stages 0 and 1, V stages 0 and 1, each 1024-aligned.
template <bool PAIR>
struct Geo {
    static constexpr int kKRows = PAIR ? kBN / 2 : kBN;  // key rows of K
    static constexpr int kVDims = PAIR ? kD / 2 : kD;    // dims of V
    static constexpr int kKBlock = kKRows * 128;         // one 64-dim K-block of K: kKRows x 128 B
    static constexpr int kKBytes = 2 * kKBlock;
    static constexpr int kVBytes = kBN * kVDims * 2;
    static constexpr int kOffQ = 0, kOffK = 2 * kTileBytes, kOffV = kOffK + 2 * kKBytes;
    static constexpr int kSmemBytes = kOffV + 2 * kVBytes + 1024;  // + alignment slack
    static constexpr int kKPieces = kKRows * 4 / kProducerThreads;   // 16-byte K pieces per producer thread
    static constexpr int kVQuarters = kVDims / 32;                   // 32-dim quarters of V per key row
    static constexpr int kVPieces = kBN * kVQuarters / kProducerThreads;
    static constexpr int kRowsPerUnit = (PAIR ? 2 : 1) * kQT * kBM;  // query rows per CTA (pair)
    static constexpr int kCtas = PAIR ? 2 : 1;
};
// Registers per thread. A sub-partition holds at most 16 K registers and five of the 17
// warps share one, so the CTA is launched with kLaunchRegs = 96 each (16 K / (5 * 32),
// rounded down to the allocation step of 8). The softmax warpgroups then hand
// kLaunchRegs - kSoftmaxRegs each back and the producer warpgroups take the same amount
// (setmaxnreg), so the two sums match exactly; the MMA warp keeps kLaunchRegs.
constexpr int kLaunchRegs = 96;
constexpr int kSoftmaxRegs = 80, kProducerRegs = 2 * kLaunchRegs - kSoftmaxRegs;
static_assert(kSoftmaxThreads == kProducerThreads && kProducerRegs <= 256 && kSoftmaxRegs % 8 == 0 &&
                  kProducerRegs % 8 == 0 && kSoftmaxRegs >= 24 && 5 * 32 * kLaunchRegs <= 16384,
              "register split must balance");
constexpr uint64_t kWaitNs = 1000000000ull;  // give up on an mbarrier after 1 s
// The bound of the data-path waits: kWaitNs, shortened only by the test hook
// kvq_testing_set_attention_wait. The final wait for the MMAs to drain before TMEM is
// freed always keeps kWaitNs.
__constant__ uint64_t c_wait_ns = kWaitNs;
// Test hook: nonzero makes the MMA warp first wait on an mbarrier that nothing arrives on,
// so the call's waits give up (after c_wait_ns) without any fault.
__constant__ uint32_t c_stall_mma = 0;
constexpr float kRescaleLog2 = 8.0f;          // rescale O when the row max grows by > 2^8
constexpr int kMaxSplits = 64;
constexpr int kCombineThreads = 256;  // 8 rows (warps) per CTA
constexpr uint64_t kPartialBytesPerRow = kD * 4 + 8;

// mbarriers
enum {
    kKFull0, kKFull1, kKEmpty0, kKEmpty1, kVFull0, kVFull1, kVEmpty0, kVEmpty1,
    kSFull0, kSFull1, kPFull0, kPFull1, kODone0, kODone1, kMmaDone,
    kNever,  // never arrived on: the test hook's stalled wait
    kNumBars
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
    int32_t n_q, heads, key_tiles;
    int32_t splits;            // partial results per row: gridDim.y, times 2 with DUAL
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

// Descriptor of a 128B-swizzled MN-major operand: rows of 64 contiguous MN elements, one
// row per K index; 8-row (K) groups 1024 B apart (stride byte offset) and the second
// 64-element MN half 16 KB away (leading byte offset).
__device__ __forceinline__ uint64_t sw128_mn_desc(uint32_t saddr)
{
    return static_cast<uint64_t>((saddr >> 4) & 0x3FFF) | (1024ull << 16) | (64ull << 32) | (1ull << 46) |
           (2ull << 61);
}

// Instruction descriptor of tcgen05.mma kind::f16: fp32 accumulate, bf16 A and B, A
// K-major, N = 128, M = 128 (one CTA) or 256 (a CTA pair); B K-major (kIdesc) or
// MN-major (kIdescBmn, bit 16).
template <bool PAIR>
constexpr uint32_t kIdesc =
    (1u << 4) | (1u << 7) | (1u << 10) | ((kBN >> 3) << 17) | ((static_cast<uint32_t>(PAIR ? 2 : 1) * kBM >> 4) << 24);
template <bool PAIR>
constexpr uint32_t kIdescBmn = kIdesc<PAIR> | (1u << 16);

// The MMA warp's instructions, in elected-lane form: the whole warp runs them, converged,
// and elect.sync picks the one lane that issues -- always the same lane, so its commits
// track all of its MMAs. With PAIR they are the cta_group::2 forms, issued by CTA 0 of
// the pair for both CTAs (no output lane masked), and commits arrive on both CTAs'
// copies of the barrier.

// S (TMEM) = Q[128 x 128] K[128 x 128]^T, both K-major in shared memory, as 8 MMAs of K = 16.
template <bool PAIR>
__device__ __forceinline__ void mma_qk(uint32_t tmem_d, uint32_t q_base, uint32_t k_base)
{
#pragma unroll
    for (int kb = 0; kb < 2; ++kb)
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const uint64_t ad = sw128_desc(q_base + kb * 16384 + s * 32);
            const uint64_t bd = sw128_desc(k_base + kb * Geo<PAIR>::kKBlock + s * 32);
            const uint32_t acc = kb > 0 || s > 0 ? 1u : 0u;
            if (PAIR)
                asm volatile("{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
                             "@e tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5, %5, %5, %5, %5}, p;"
                             "\n\t}" ::"r"(tmem_d), "l"(ad), "l"(bd), "r"(kIdesc<PAIR>), "r"(acc), "r"(0u)
                             : "memory");
            else
                asm volatile("{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
                             "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                             ::"r"(tmem_d), "l"(ad), "l"(bd), "r"(kIdesc<PAIR>), "r"(acc)
                             : "memory");
        }
}

// O (TMEM) (+)= P[128 x 128 keys] V[128 keys x 128]: P in TMEM (row i in lane i, keys 2c
// and 2c + 1 in the low and high halves of column c), V row-major in shared memory (key
// rows, the MN-major B operand). Key step t of 16 keys: P columns 8t on, V 2048 B (two
// 8-row groups) further.
template <bool PAIR>
__device__ __forceinline__ void mma_pv(uint32_t tmem_d, uint32_t tmem_p, uint32_t v_base, bool accumulate)
{
#pragma unroll
    for (int t = 0; t < 8; ++t) {
        const uint64_t bd = sw128_mn_desc(v_base + t * 2048);
        const uint32_t acc = accumulate || t > 0 ? 1u : 0u;
        if (PAIR)
            asm volatile("{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
                         "@e tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, {%5, %5, %5, %5, %5, %5, %5, %5}, p;"
                         "\n\t}" ::"r"(tmem_d), "r"(tmem_p + 8 * t), "l"(bd), "r"(kIdescBmn<PAIR>), "r"(acc), "r"(0u)
                         : "memory");
        else
            asm volatile("{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
                         "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
                         ::"r"(tmem_d), "r"(tmem_p + 8 * t), "l"(bd), "r"(kIdescBmn<PAIR>), "r"(acc)
                         : "memory");
    }
}

// Arrive on mbar once every MMA the elected lane has issued so far is complete (on both
// CTAs' copies with PAIR).
template <bool PAIR>
__device__ __forceinline__ void commit(uint32_t mbar)
{
    if (PAIR)
        asm volatile("{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
                     "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
                     "\n\t}" ::"r"(mbar), "h"(static_cast<uint16_t>(3))
                     : "memory");
    else
        asm volatile("{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
                     "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(mbar)
                     : "memory");
}

// `count` arrivals on the barrier at this offset of CTA 0 of the pair (with PAIR; a
// peer-CTA arrive from CTA 1) or of this CTA. What the arrival publishes is ordered by
// the callers' tcgen05 and async-proxy fences, as for any arrive.
template <bool PAIR>
__device__ __forceinline__ void arrive_count(uint32_t mbar, uint32_t count)
{
    if (PAIR)
        asm volatile("{\n\t.reg .b32 ra;\n\tmapa.shared::cluster.u32 ra, %0, 0;\n\t"
                     "mbarrier.arrive.shared::cluster.b64 _, [ra], %1;\n\t}" ::"r"(mbar), "r"(count)
                     : "memory");
    else
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(mbar), "r"(count) : "memory");
}

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void mbar_init(uint32_t mbar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(mbar), "r"(count) : "memory");
}

__device__ __forceinline__ uint64_t globaltimer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Wait, for at most `limit` ns (the data-path bound by default), for phase `parity` of an
// mbarrier; true when it completed.
__device__ __forceinline__ bool wait_phase(uint32_t mbar, uint32_t parity, uint64_t limit = c_wait_ns)
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
        if (globaltimer_ns() - t0 > limit)
            return false;
    }
}

// The same wait, decided for the whole warp (tcgen05.ld/st need a converged warp).
__device__ __forceinline__ bool warp_wait(uint32_t mbar, uint32_t parity, uint64_t limit = c_wait_ns)
{
    return __all_sync(0xFFFFFFFFu, wait_phase(mbar, parity, limit));
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

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

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
// Loads of the next tile, issued where they stand: volatile, so the compiler cannot sink
// them past the waits that follow (they are the prefetch).
__device__ __forceinline__ uint4 prefetch_v4(const void* p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t prefetch_u16(const void* p)
{
    uint16_t v;
    asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ float prefetch_f32(const float* p)
{
    float v;
    asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(v) : "l"(p));
    return v;
}

// One 16-byte piece of a key row: two blocks (32 dims, quarter q of the row). Nothing is
// computed from the loaded values here (they are the prefetch of the next tile and must
// not stall the thread): a key past n_kv loads row 0 instead and is zeroed at
// dequantization, where gs = amax / 2688 is taken too.
struct RawPiece {
    uint4 c;      // codes
    uint32_t sc;  // the two blocks' scale codes in the low 16 bits
    float amax;   // chunk amax of the key
};

// gs = RN(amax / 2688). With MARK, without a division: Markstein's correction step (P.
// Markstein, "Computation of elementary functions on the IBM RISC System/6000 processor",
// IBM J. Res. Dev. 34(1), 1990) with y = RN(1/2688): q = RN(amax y), r = amax - 2688 q
// (exact as one fma), RN(q + r y). It equals the IEEE quotient for every fp32 amax from
// 2^-119 up (checked exhaustively over the five binades from 2^-119 to 2^-114, which hold
// every amax whose quotient is subnormal from there on, amax below about 2^-114.6, and
// on a sample of the rest); below 2^-119 it does not. A
// single CTA takes MARK when every chunk amax its keys use is in [2^-119, FLT_MAX] (the
// IEEE division, with its rare slow path, in the producer loop cost 13 % of a single
// CTA's time per key tile).
constexpr float kMarkMinAmax = 0x1p-119f;
constexpr int64_t kMarkScanMax = 4096;

__device__ __forceinline__ bool markstein_amax(float amax)
{
    return amax >= kMarkMinAmax && amax <= 0x1.fffffep127f;
}

template <bool MARK>
__device__ __forceinline__ float global_scale(float amax)
{
    if (MARK) {
        constexpr float kInvDen = 0x1.861862p-12f;  // RN(1 / 2688)
        const float q = __fmul_rn(amax, kInvDen);
        const float r = __fmaf_rn(-q, 2688.0f, amax);
        return __fmaf_rn(r, kInvDen, q);
    }
    return __fdiv_rn(amax, 2688.0f);
}

// Keys and chunk indices fit in 32 bits (a cache holds at most 2^36 elements, i.e. 2^29
// rows of 128).
__device__ __forceinline__ void load_piece(const uint8_t* packed, const uint8_t* scales, const float* amax,
                                           const AttnArgs& a, int h, int64_t key, int q, RawPiece& r)
{
    key = key < a.n_kv ? key : 0;
    const int64_t off = (key * a.heads + h) * 64 + 16 * q;
    const uint32_t chunk = static_cast<uint32_t>(key) / static_cast<uint32_t>(a.tokens_per_chunk);
    r.c = prefetch_v4(packed + off);
    r.sc = prefetch_u16(scales + off / 8);
    r.amax = prefetch_f32(amax + chunk);
}

// Byte offset of 16-byte chunk `chunk` (0..7) of row `row` in 64-wide block `kb` of a
// 128B-swizzled operand whose blocks hold `rows` rows (8-row groups of 1024 B, the chunk
// index XOR-ed with row % 8).
__device__ __forceinline__ uint32_t sw128r(int row, int kb, int chunk, int rows)
{
    return kb * rows * 128 + (row >> 3) * 1024 + (row & 7) * 128 + ((chunk ^ (row & 7)) << 4);
}

// The piece dequantized (the dequant kernel's arithmetic) into row `row`, chunks ch0 ..
// ch0 + 3 of block kb of a swizzled operand of `rows` rows per block (K as the K-major B
// operand of Q K^T, V as the MN-major B operand of P V: the same bytes); a key past n_kv
// gives zeros. With swap the two blocks are stored in the other order, so that threads
// of neighbouring quarters hit different 16-byte bank groups of a shared-memory wavefront.
template <bool MARK>
__device__ __forceinline__ void store_piece(const RawPiece& r, bool valid, int row, int kb, int ch0, int rows,
                                            bool swap, uint32_t sT)
{
    const float gs = valid ? global_scale<MARK>(r.amax) : 0.0f;
    const float SA = block_scale(r.sc, swap ? 1 : 0, gs), SB = block_scale(r.sc, swap ? 0 : 1, gs);
    const int s2 = swap ? 2 : 0;
    uint32_t y[4];
    dequant8(swap ? r.c.z : r.c.x, SA, y);
    st_shared_v4(sT + sw128r(row, kb, ch0 + (0 ^ s2), rows), y[0], y[1], y[2], y[3]);
    dequant8(swap ? r.c.w : r.c.y, SA, y);
    st_shared_v4(sT + sw128r(row, kb, ch0 + (1 ^ s2), rows), y[0], y[1], y[2], y[3]);
    dequant8(swap ? r.c.x : r.c.z, SB, y);
    st_shared_v4(sT + sw128r(row, kb, ch0 + (2 ^ s2), rows), y[0], y[1], y[2], y[3]);
    dequant8(swap ? r.c.y : r.c.w, SB, y);
    st_shared_v4(sT + sw128r(row, kb, ch0 + (3 ^ s2), rows), y[0], y[1], y[2], y[3]);
}

// ------------------------------------------------------------------ softmax pieces

// max(a, b, c) in one instruction (sm_100).
__device__ __forceinline__ float max3(float a, float b, float c)
{
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

constexpr int kW = 16;  // columns of S per TMEM load

// kW columns of this warp's 32 TMEM lanes, without the wait: the registers are valid
// only after tmem_wait_ld() and must not be read before it.
__device__ __forceinline__ void tmem_ldw_async(uint32_t addr, uint32_t (&r)[kW])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
                 : "r"(addr)
                 : "memory");
}

// Max of row S over the tile's valid keys (MASK: only the first `valid`): four loads of 32
// columns, each reduced in four independent chains of three-input max.
template <bool MASK>
__device__ __forceinline__ float tile_row_max(uint32_t tS, int valid)
{
    float m[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
        float v[32];
        tmem_ld32(tS + c * 32, v);
        if (MASK) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
                v[i] = c * 32 + i < valid ? v[i] : -INFINITY;
        }
#pragma unroll
        for (int i = 0; i < 32; i += 8) {
            m[0] = max3(m[0], v[i], v[i + 1]);
            m[1] = max3(m[1], v[i + 2], v[i + 3]);
            m[2] = max3(m[2], v[i + 4], v[i + 5]);
            m[3] = max3(m[3], v[i + 6], v[i + 7]);
        }
    }
    return fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
}

// 2^x for a pair of fp32 on the FMA pipe, for part of the softmax's exponentials (the ex2
// unit takes the rest; FlashAttention-4 on Blackwell splits them the same way, since one
// ex2 unit per sub-partition sets the softmax's pace). Range reduction after W. J. Cody
// and W. Waite, "Software Manual for the Elementary Functions" (1980): x = n + f with n =
// round(x) (adding 1.5 * 2^23 rounds to an integer and leaves n in the low mantissa bits)
// and f in [-1/2, 1/2]; 2^f by a cubic fitted here to the relative error of 2^f on
// [-1/2, 1/2] (iterated weighted least squares; max relative error 1.43e-4, far under
// the 2^-9 of P's bf16 rounding); 2^n by adding n to the exponent field. x is clamped at
// -125, so the result stays a normal number.
__device__ __forceinline__ uint64_t exp2_poly(uint64_t x2)
{
    float x0, x1;
    f32x2_unpack(x2, x0, x1);
    const uint64_t x = f32x2_pack(fmaxf(x0, -125.0f), fmaxf(x1, -125.0f));
    const uint64_t one2 = f32x2_pack(1.0f, 1.0f);
    const uint64_t t = f32x2_fma(x, one2, f32x2_pack(12582912.0f, 12582912.0f));
    const uint64_t n = f32x2_fma(t, one2, f32x2_pack(-12582912.0f, -12582912.0f));
    const uint64_t f = f32x2_fma(n, f32x2_pack(-1.0f, -1.0f), x);
    uint64_t p = f32x2_fma(f32x2_pack(0.055453190757429514f, 0.055453190757429514f), f,
                           f32x2_pack(0.24236350527675452f, 0.24236350527675452f));
    p = f32x2_fma(p, f, f32x2_pack(0.6931914699126007f, 0.6931914699126007f));
    p = f32x2_fma(p, f, f32x2_pack(0.9999423493565059f, 0.9999423493565059f));
    float p0, p1, t0, t1;
    f32x2_unpack(p, p0, p1);
    f32x2_unpack(t, t0, t1);
    return f32x2_pack(__uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23)),
                      __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23)));
}

// Pairs of each kW-column chunk whose exponentials go to exp2_poly (bit i: pair i).
constexpr uint32_t kPolyPairs = 0x88;

// kW columns (chunk c) of the row: p = 2^(s * scale_log2 - m) (0 past `valid` when MASK),
// summed into the packed accumulators and written as bf16 pairs to TMEM columns
// tS + c kW / 2 on, which hold S columns this thread has already read.
template <bool MASK>
__device__ __forceinline__ void exp_chunk(const uint32_t (&sr)[kW], int c, uint32_t tS, int valid, uint64_t sc2,
                                          uint64_t nm2, uint64_t& la, uint64_t& lb)
{
    const uint64_t one2 = f32x2_pack(1.0f, 1.0f);
    uint32_t pw[kW / 2];
#pragma unroll
    for (int i = 0; i < kW; i += 2) {
        const int col = c * kW + i;
        const uint64_t x2 = f32x2_fma(f32x2_pack(__uint_as_float(sr[i]), __uint_as_float(sr[i + 1])), sc2, nm2);
        float p0, p1;
        if ((kPolyPairs >> (i >> 1)) & 1) {
            f32x2_unpack(exp2_poly(x2), p0, p1);
        } else {
            float x0, x1;
            f32x2_unpack(x2, x0, x1);
            p0 = ex2(x0);
            p1 = ex2(x1);
        }
        if (MASK) {
            if (col >= valid)
                p0 = 0.0f;
            if (col + 1 >= valid)
                p1 = 0.0f;
        }
        if ((i >> 1) & 1)
            lb = f32x2_fma(f32x2_pack(p0, p1), one2, lb);
        else
            la = f32x2_fma(f32x2_pack(p0, p1), one2, la);
        pw[i >> 1] = bf16x2_from_f32(p1, p0);
    }
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
                 ::"r"(tS + c * (kW / 2)), "r"(pw[0]), "r"(pw[1]), "r"(pw[2]), "r"(pw[3]), "r"(pw[4]), "r"(pw[5]),
                 "r"(pw[6]), "r"(pw[7])
                 : "memory");
}

// p = 2^(s * scale_log2 - m) for row S of the tile (0 past `valid` when MASK), written as
// bf16 into the first 64 columns of S (word c holds keys 2c, 2c + 1); returns the fp32
// sum of p. The TMEM load of the next kW columns is in flight while the current ones are
// computed; a chunk's P lands on columns loaded before it.
template <bool MASK>
__device__ __forceinline__ float tile_row_exp(uint32_t tS, int valid, float scale_log2, float m)
{
    constexpr int kChunks = kBN / kW;
    const uint64_t sc2 = f32x2_pack(scale_log2, scale_log2), nm2 = f32x2_pack(-m, -m);
    uint64_t la = 0, lb = 0;  // two packed partial sums (+0.0 bit patterns)
    uint32_t r0[kW], r1[kW];
    tmem_ldw_async(tS, r0);
    tmem_wait_ld();
#pragma unroll 1
    for (int k = 0; k < kChunks / 2; ++k) {
        const int c = 2 * k;
        tmem_ldw_async(tS + (c + 1) * kW, r1);
        exp_chunk<MASK>(r0, c, tS, valid, sc2, nm2, la, lb);
        tmem_wait_ld();
        if (k < kChunks / 2 - 1)
            tmem_ldw_async(tS + (c + 2) * kW, r0);
        exp_chunk<MASK>(r1, c + 1, tS, valid, sc2, nm2, la, lb);
        if (k < kChunks / 2 - 1)
            tmem_wait_ld();
    }
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    float a0, a1, b0, b1;
    f32x2_unpack(la, a0, a1);
    f32x2_unpack(lb, b0, b1);
    return __fadd_rn(__fadd_rn(a0, a1), __fadd_rn(b0, b1));
}

// ------------------------------------------------------------------ kernels

// PAIR: the kernel runs as clusters of two CTAs (x even, x odd) that share every K/V
// tile and issue cta_group::2 MMAs (M = 256: query tile slot g is rows 512 u + 256 g ..
// + 255 of the pair, CTA `rank` holding the 128 from 512 u + 256 g + 128 rank); else one
// CTA per unit of 256 query rows (slot g: rows 256 u + 128 g .. + 127). DUAL: both slots
// hold one query tile and split the CTA's key range (units of at most 128 rows).
template <bool PAIR, bool DUAL>
__global__ void __maxnreg__(kLaunchRegs) attention_kernel(const AttnArgs a)
{
    using G = Geo<PAIR>;
    pdl_begin();
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t bars[kNumBars];
    __shared__ uint32_t tmem_base_s;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = PAIR ? cluster_rank() : 0u;  // CTA 0 of a pair issues the MMAs
    const int unit = PAIR ? blockIdx.x >> 1 : blockIdx.x, split = blockIdx.y, h = blockIdx.z;
    const int t_begin = static_cast<int>(static_cast<int64_t>(split) * a.key_tiles / gridDim.y);
    const int t_end = static_cast<int>(static_cast<int64_t>(split + 1) * a.key_tiles / gridDim.y);
    const int64_t u0 = static_cast<int64_t>(unit) * G::kRowsPerUnit;   // first row of the unit
    const int64_t q0 = u0 + rank * kBM;                                // this CTA's first row
    constexpr int kSlotRows = G::kCtas * kBM;                          // rows between slots
    const int n_tiles = t_end - t_begin;
    // dual: both slots hold query tile 0; slot 0 takes the first n_lead key tiles of the
    // range, slot 1 the rest, and each writes its own partial result (2 split + slot)
    constexpr bool dual = DUAL;
    const int n_qt = dual || a.n_q - u0 > kSlotRows ? 2 : 1;         // slots in use
    const int n_lead = dual ? (n_tiles + 1) >> 1 : n_tiles;          // slot 0's key tiles
    auto slot_tiles = [&](int g) { return dual && g ? n_tiles - n_lead : n_lead; };
    // the pipeline runs over stream tiles s: key tile t_begin + s, or with dual slot
    // s % 2's tile s / 2; stream tile s lives in stage s % 2 with barrier phase (s / 2) % 2
    auto key_tile = [&](int s) { return dual ? t_begin + ((s & 1) ? n_lead : 0) + (s >> 1) : t_begin + s; };
    auto stream = [&](int g, int j) { return dual ? 2 * j + g : j; };
    const int64_t H = a.heads;

    const uint32_t base = (static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw)) + 1023u) & ~1023u;
    const uint32_t bar0 = static_cast<uint32_t>(__cvta_generic_to_shared(&bars[0]));
    auto bar = [bar0](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
    // stream tile s lives in K stage s % 2; its barriers' phase is s / 2
    auto sK = [base](int j) { return base + G::kOffK + static_cast<uint32_t>(j & 1) * G::kKBytes; };
    auto kfull = [&bar](int j) { return bar(kKFull0 + (j & 1)); };
    auto kempty = [&bar](int j) { return bar(kKEmpty0 + (j & 1)); };
    // and in V stage s % 2
    auto sV = [base](int j) { return base + G::kOffV + static_cast<uint32_t>(j & 1) * G::kVBytes; };
    auto vfull = [&bar](int j) { return bar(kVFull0 + (j & 1)); };
    auto vempty = [&bar](int j) { return bar(kVEmpty0 + (j & 1)); };

    if (warp == 0) {
        // a pair allocates together: warp 0 of both CTAs, the same destination offset
        const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(&tmem_base_s));
        if (PAIR) {
            asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst), "r"(kTmemCols)
                         : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
        } else {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst), "r"(kTmemCols)
                         : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        }
    }
    if (tid == 0) {
        // the "full" barriers count arrivals from every producer / softmax thread of the
        // pair (only CTA 0's copy is waited on); the others take one commit each
        for (int st = 0; st < 2; ++st) {
            mbar_init(bar(kKFull0 + st), G::kCtas * kProducerThreads);
            mbar_init(bar(kKEmpty0 + st), 1);  // one commit after the last MMA reading the stage
            mbar_init(bar(kVFull0 + st), G::kCtas * kProducerThreads);
            mbar_init(bar(kVEmpty0 + st), 1);
        }
        for (int g = 0; g < kQT; ++g) {
            mbar_init(bar(kSFull0 + g), 1);
            mbar_init(bar(kPFull0 + g), G::kCtas * kBM);
            mbar_init(bar(kODone0 + g), 1);
        }
        mbar_init(bar(kMmaDone), 1);
        mbar_init(bar(kNever), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // the query tiles -> shared memory (rows past n_q are zero; one tile with dual)
    for (int i = tid; i < (dual ? 1 : kQT) * kBM * 16; i += kAttnThreads) {
        const int g = i >> 11, row = (i >> 4) & 127, kb = (i >> 3) & 1, ch = i & 7;
        const int64_t qrow = q0 + g * kSlotRows + row;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (qrow < a.n_q)
            v = ld_nc_v4(a.q + (qrow * H + h) * kD + kb * 64 + ch * 8);
        st_shared_v4(base + G::kOffQ + g * kTileBytes + sw128(row, kb, ch), v.x, v.y, v.z, v.w);
    }
    // the correction step for the global scales if every chunk amax of the CTA's keys is
    // in its exact range (a range over more than kMarkScanMax chunks takes the division).
    // Only with DUAL, where the producers set the pace (each slot's chain has half the
    // key tiles). A pair's producers, and those of a single CTA with two query tiles,
    // wait for the softmax; there a second producer loop in the kernel measured 4-6 %
    // slower overall.
    constexpr bool producer_bound = !PAIR && DUAL;
    int off_range = producer_bound ? 0 : 1;
    if (producer_bound) {
        const int64_t k_lo = static_cast<int64_t>(t_begin) * kBN;
        const int64_t k_hi = min(static_cast<int64_t>(t_end) * kBN, a.n_kv);
        if (k_hi > k_lo) {
            const int64_t c0 = k_lo / a.tokens_per_chunk, c1 = (k_hi - 1) / a.tokens_per_chunk;
            if (c1 - c0 >= kMarkScanMax)
                off_range = 1;
            else
                for (int64_t c = c0 + tid; c <= c1; c += kAttnThreads)
                    off_range |= static_cast<int>(!markstein_amax(__ldg(a.ka + c))) |
                                 static_cast<int>(!markstein_amax(__ldg(a.va + c)));
        }
    }
    fence_async_smem();
    tc_before_sync();
    const bool mark = __syncthreads_or(off_range) == 0;
    if (PAIR)
        cluster_sync();  // both CTAs' barriers initialized and TMEM allocated before any peer access
    tc_after_sync();
    const uint32_t tmem = __shfl_sync(0xFFFFFFFFu, tmem_base_s, 0);

    if (tid < kSoftmaxThreads) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
        // ---------------------------------------------------------------- softmax
        const int g = __shfl_sync(0xFFFFFFFFu, tid >> 7, 0), r = tid & 127;
        if (g < n_qt) {
            const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
            const uint32_t tS = tmem + g * 128 + lane_off, tO = tmem + 256 + g * 128 + lane_off;
            const uint32_t bS = bar(kSFull0 + g), bP = bar(kPFull0 + g), bO = bar(kODone0 + g);
            const int my_tiles = slot_tiles(g);
            float m_run = -INFINITY, l_run = 0.0f;
            bool ok = true;
            for (int j = 0; ok && j < my_tiles; ++j) {
                ok = warp_wait(bS, j & 1);
                if (!ok)
                    break;
                tc_after_sync();
                const int64_t key0 = static_cast<int64_t>(key_tile(stream(g, j))) * kBN;
                const int valid = static_cast<int>(a.n_kv - key0 < kBN ? a.n_kv - key0 : kBN);
                // the row max first; the reference moves (and O is rescaled) only when the
                // max exceeds it by more than 2^8, which is rare after the first tiles
                const float mt = __fmul_rn(
                    valid == kBN ? tile_row_max<false>(tS, valid) : tile_row_max<true>(tS, valid), a.scale_log2);
                const float m_cand = j == 0 ? mt : fmaxf(m_run, mt);
                const bool need = j == 0 || m_cand > m_run + kRescaleLog2;
                const float m_use = need ? m_cand : m_run;
                const float alpha = j == 0 ? 0.0f : (need ? ex2(m_run - m_use) : 1.0f);
                // P over the S columns already read (S_g(j) was written after P V(j-1) had
                // read P_g(j-1): both come from the MMA warp, in that order)
                const float lt = valid == kBN ? tile_row_exp<false>(tS, valid, a.scale_log2, m_use)
                                              : tile_row_exp<true>(tS, valid, a.scale_log2, m_use);
                l_run = __fmaf_rn(l_run, alpha, lt);
                m_run = m_use;
                // rescale O (the warp does it if any of its rows needs it) once P V(j-1) is done
                if (j > 0 && __any_sync(0xFFFFFFFFu, need)) {
                    ok = warp_wait(bO, (j - 1) & 1);
                    if (!ok)
                        break;
                    tc_after_sync();
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
                tc_before_sync();
                __syncwarp();
                if (lane == 0)
                    arrive_count<PAIR>(bP, 32);
            }
            if (ok && my_tiles == 0 && dual) {
                // an empty key range (a one-tile range's slot 1): a partial of weight 0
                const int64_t qrow = q0 + r;
                const int64_t prow = (static_cast<int64_t>(2 * split + 1) * a.n_q + qrow) * H + h;
                if (qrow < a.n_q) {
                    for (int c = 0; c < kD; c += 4)
                        st_v4(a.part_o + prow * kD + c, 0u, 0u, 0u, 0u);
                    a.part_ml[prow] = make_float2(-INFINITY, 0.0f);
                }
            }
            if (ok && my_tiles > 0) {
                ok = warp_wait(bO, (my_tiles - 1) & 1);
                if (ok) {
                    tc_after_sync();
                    const int64_t qrow = q0 + (dual ? 0 : g * kSlotRows) + r;
                    const bool has_row = qrow < a.n_q;
                    const int64_t prow = (static_cast<int64_t>(dual ? 2 * split + g : split) * a.n_q + qrow) * H + h;
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
    } else if (warp == kMmaWarp) {
        // ---------------------------------------------------------------- MMA issue
        // (CTA 0 of a pair issues for both CTAs; CTA 1's MMA warp has nothing to do)
        // Without dual both slots read each stream tile (one stage release per tile, after
        // the last slot); with dual each stream tile belongs to one slot.
        const uint32_t sQ0 = base + G::kOffQ, sQ1 = dual ? sQ0 : base + G::kOffQ + kTileBytes;
        bool ok = true;
        const int steps = rank == 0 ? n_lead : 0;
        if (c_stall_mma && steps > 0)
            ok = warp_wait(bar(kNever), 0);  // gives up after c_wait_ns: nothing is issued
        if (steps > 0) {
            // S_g(0) for each slot: stream tile 0 for both, or with dual tiles 0 and 1
            for (int g = 0; ok && g < n_qt; ++g) {
                if (slot_tiles(g) == 0)
                    break;
                const int s = stream(g, 0);
                if (g == 0 || dual) {
                    ok = warp_wait(kfull(s), 0);
                    if (!ok)
                        break;
                    tc_after_sync();
                }
                mma_qk<PAIR>(tmem + g * 128, g == 0 ? sQ0 : sQ1, sK(s));
                commit<PAIR>(bar(kSFull0 + g));
                if (dual || g == n_qt - 1)
                    commit<PAIR>(kempty(s));
            }
        }
        for (int j = 0; ok && j < steps; ++j) {
            for (int g = 0; g < n_qt; ++g) {
                // O_g += P_g V(s), then S_g(j+1) = Q_g K(s')^T for the slot's next tile s'
                const int gt = slot_tiles(g), s = stream(g, j);
                if (j >= gt)
                    break;
                ok = warp_wait(bar(kPFull0 + g), j & 1) &&
                     ((g > 0 && !dual) || warp_wait(vfull(s), (s >> 1) & 1));
                if (!ok)
                    break;
                tc_after_sync();
                mma_pv<PAIR>(tmem + 256 + g * 128, tmem + g * 128, sV(s), j > 0);
                commit<PAIR>(bar(kODone0 + g));
                if (dual || g == n_qt - 1)
                    commit<PAIR>(vempty(s));
                if (j + 1 < gt) {
                    const int s2 = stream(g, j + 1);
                    if (g == 0 || dual) {
                        ok = warp_wait(kfull(s2), (s2 >> 1) & 1);
                        if (!ok)
                            break;
                        tc_after_sync();
                    }
                    mma_qk<PAIR>(tmem + g * 128, g == 0 ? sQ0 : sQ1, sK(s2));
                    commit<PAIR>(bar(kSFull0 + g));
                    if (dual || g == n_qt - 1)
                        commit<PAIR>(kempty(s2));
                }
            }
        }
        if (rank == 0) {
            commit<PAIR>(bar(kMmaDone));  // completes once every MMA issued has
            if (!warp_wait(bar(kMmaDone), 0, kWaitNs))  // the drain keeps the full bound
                ok = false;
        }
        if (!ok && lane == 0)
            atomicExch(a.status, 1);
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kProducerRegs));
        // ---------------------------------------------------------------- producers
        // K runs one key tile ahead of V: K(j+1) is stored before V(j), the order in which
        // the MMA warp consumes them (P_0 V(j) comes before S_0(j+1) but the V stage it
        // needs was freed a tile earlier). Each tensor's raw pieces are refilled right
        // after its tile is stored, so the loads land while the other tensor is
        // dequantized and the barriers are awaited. Piece i of thread p: K row
        // (p + 256 i) / 4 of this CTA's key rows, quarter p % 4; V key row (p + 256 i) /
        // kVQuarters, quarter p % kVQuarters of this CTA's dims. A warp's arrivals are one
        // arrive of 32 (on CTA 0's barrier with PAIR).
        // the producer loop, with the global scale by the correction step (MARK) or by
        // IEEE division; the choice is uniform over the CTA
        auto produce = [&](auto mark_tag) {
            constexpr bool MARK = decltype(mark_tag)::value;
            const int p = tid - kSoftmaxThreads;
            const int k_q = p & 3, v_q = p % G::kVQuarters;
            auto k_row = [&](int i) { return (p + kProducerThreads * i) >> 2; };
            auto v_row = [&](int i) { return (p + kProducerThreads * i) / G::kVQuarters; };
            // the first key of the K and V tile loaded last: each load_x(j) is followed by
            // put_x(j) before the next load_x
            int64_t k_key0 = 0, v_key0 = 0;
            auto k_key = [&](int i) { return k_key0 + rank * (kBN - G::kKRows) + k_row(i); };
            auto v_key = [&](int i) { return v_key0 + v_row(i); };
            RawPiece rk[G::kKPieces], rv[G::kVPieces];
            auto load_k = [&](int j) {
                k_key0 = static_cast<int64_t>(key_tile(j)) * kBN;
    #pragma unroll
                for (int i = 0; i < G::kKPieces; ++i)
                    load_piece(a.kp, a.ks, a.ka, a, h, k_key(i), k_q, rk[i]);
            };
            auto load_v = [&](int j) {
                v_key0 = static_cast<int64_t>(key_tile(j)) * kBN;
    #pragma unroll
                for (int i = 0; i < G::kVPieces; ++i)
                    load_piece(a.vp, a.vs, a.va, a, h, v_key(i), v_q + static_cast<int>(rank) * G::kVQuarters, rv[i]);
            };
            auto put_k = [&](int j) {
    #pragma unroll
                for (int i = 0; i < G::kKPieces; ++i)
                    store_piece<MARK>(rk[i], k_key(i) < a.n_kv, k_row(i), k_q >> 1, (k_q & 1) * 4, G::kKRows, (k_q & 2) != 0,
                                sK(j));
                fence_async_smem();
                __syncwarp();
                if (lane == 0)
                    arrive_count<PAIR>(kfull(j), 32);
            };
            auto put_v = [&](int j) {
    #pragma unroll
                for (int i = 0; i < G::kVPieces; ++i)
                    store_piece<MARK>(rv[i], v_key(i) < a.n_kv, v_row(i), v_q >> 1, (v_q & 1) * 4, kBN, (v_q & 2) != 0,
                                sV(j));
                fence_async_smem();
                __syncwarp();
                if (lane == 0)
                    arrive_count<PAIR>(vfull(j), 32);
            };
            bool ok = true;
            if (dual) {
                // the MMA warp takes S(0), S(1), then P V(s) and S(s + 2) for each stream tile
                // s; stage s % 2 of K is freed by S(s), of V by P V(s)
                load_k(0);
                load_v(0);
                put_k(0);
                if (n_tiles > 1) {
                    load_k(1);
                    put_k(1);
                    if (n_tiles > 2)
                        load_k(2);
                }
                for (int s = 0; s < n_tiles; ++s) {
                    if (s > 1 && !(ok = wait_phase(vempty(s), ((s >> 1) - 1) & 1)))
                        break;
                    put_v(s);
                    if (s + 1 < n_tiles)
                        load_v(s + 1);
                    if (s + 2 < n_tiles) {
                        if (!(ok = wait_phase(kempty(s + 2), (s >> 1) & 1)))
                            break;
                        put_k(s + 2);
                        if (s + 3 < n_tiles)
                            load_k(s + 3);
                    }
                }
                if (!ok && lane == 0)
                    atomicExch(a.status, 1);
            } else {
            if (n_tiles > 0) {
                load_k(0);
                load_v(0);
                put_k(0);
                if (n_tiles > 1)
                    load_k(1);
            }
            for (int j = 0; j < n_tiles; ++j) {
                if (j + 1 < n_tiles) {
                    // stage (j+1) % 2 was last read by the S MMAs of key tile j - 1
                    if (j > 0 && !(ok = wait_phase(kempty(j + 1), (((j + 1) >> 1) - 1) & 1)))
                        break;
                    put_k(j + 1);
                    if (j + 2 < n_tiles)
                        load_k(j + 2);
                }
                // stage j % 2 was last read by the P V MMAs of value tile j - 2
                if (j > 1 && !(ok = wait_phase(vempty(j), ((j >> 1) - 1) & 1)))
                    break;
                put_v(j);
                if (j + 1 < n_tiles)
                    load_v(j + 1);
            }
            if (!ok && lane == 0)
                atomicExch(a.status, 1);
            }
        };
        if (producer_bound && mark)
            produce(std::integral_constant<bool, producer_bound>{});
        else
            produce(std::false_type{});
    }
    tc_before_sync();
    __syncthreads();
    if (PAIR)
        cluster_sync();  // CTA 0's MMAs, which write both CTAs' TMEM, are all complete
    if (warp == 0) {
        if (PAIR)
            asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                         : "memory");
        else
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                         : "memory");
    }
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

bool cluster_launch_supported()
{
    int dev = 0, v = 0;
    return cudaGetDevice(&dev) == cudaSuccess &&
           cudaDeviceGetAttribute(&v, cudaDevAttrClusterLaunch, dev) == cudaSuccess && v != 0;
}

// The launch plan: the query rows split into at most two parts, each launched on its own
// (CTA pairs or single CTAs) with its key splits, workspace region and combine. A pair's
// steady state takes about 15/16 of the time per query row of a single CTA (its M = 256
// MMAs occupy each SM 76 cycles against 95 for M = 128; measured 7 % faster at 1024 and
// 2048 queries), but its unit is 512 rows against 256. A single CTA whose rows fit one
// query tile (at most 128) runs dual: its two slots split the CTA's key range, and its
// producers, which then set the pace, skip the division (measured 0.74 of a two-tile
// unit's time). In units of a single CTA's time per key tile, a single unit costs 16 (12
// when dual), a pair unit 30; the plan takes the cheapest of all single CTAs, all pairs,
// and pairs over the whole 512-row blocks with single CTAs for the rest (ties to fewer
// launches). 1560 queries take three pairs for 1536 rows and one dual CTA for the last 24.
struct AttnPart {
    bool pair, dual;
    int32_t row0, rows;  // query rows [row0, row0 + rows)
    int64_t units;
    int splits;          // key ranges (gridDim.y); partial results per row: splits << dual
    uint64_t ws_offset;  // of its partials in the workspace
    int partials() const { return splits << (dual ? 1 : 0); }
};

struct AttnPlan {
    int n_parts;
    AttnPart part[2];
    uint64_t ws_bytes;
};

constexpr uint64_t kWsAlign = 256;

void finish_plan(AttnPlan& pl, int32_t heads)
{
    uint64_t off = 0;
    for (int i = 0; i < pl.n_parts; ++i) {
        pl.part[i].ws_offset = off;
        off += (partial_bytes(pl.part[i].partials(), pl.part[i].rows, heads) + kWsAlign - 1) / kWsAlign * kWsAlign;
    }
    pl.ws_bytes = off;
}

int64_t single_cost(int64_t rows)
{
    return rows <= kBM ? 12 : 16 * ((rows + Geo<false>::kRowsPerUnit - 1) / Geo<false>::kRowsPerUnit);
}

AttnPlan plan_attention(int32_t n_q, int32_t heads, int64_t key_tiles)
{
    constexpr int64_t kPairRows = Geo<true>::kRowsPerUnit;
    const int64_t cost_single = single_cost(n_q);
    const int64_t cost_pair = 30 * ((n_q + kPairRows - 1) / kPairRows);  // 64-bit: n_q may be near 2^31
    const int32_t full_rows = static_cast<int32_t>(n_q / kPairRows * kPairRows), rest = n_q - full_rows;
    const int64_t cost_mixed = 30 * (full_rows / kPairRows) + (rest > 0 ? single_cost(rest) : 0);
    const bool pairs_ok = cluster_launch_supported();
    const int sms = sm_count();
    AttnPlan pl{};
    auto part = [&](bool pair, int32_t row0, int32_t rows) {
        const int64_t unit_rows = pair ? kPairRows : Geo<false>::kRowsPerUnit;
        AttnPart pt{};
        pt.pair = pair;
        pt.row0 = row0;
        pt.rows = rows;
        pt.units = (rows + unit_rows - 1) / unit_rows;
        // dual needs at least two key tiles per CTA: the split is chosen over half the tiles
        pt.dual = !pair && rows <= kBM && key_tiles >= 2;
        const int kt = static_cast<int>(pt.dual ? key_tiles / 2 : key_tiles);
        pt.splits = choose_splits(pt.units * heads, kt, pair ? sms / 2 : sms);
        return pt;
    };
    if (!pairs_ok || (cost_single <= cost_pair && cost_single <= cost_mixed)) {
        pl.n_parts = 1;
        pl.part[0] = part(false, 0, n_q);
    } else if (rest == 0 || cost_pair <= cost_mixed || full_rows == 0) {
        pl.n_parts = 1;
        pl.part[0] = part(true, 0, n_q);
    } else {
        pl.n_parts = 2;
        pl.part[0] = part(true, 0, full_rows);
        pl.part[1] = part(false, full_rows, rest);
    }
    finish_plan(pl, heads);
    return pl;
}

// Check the register count (setmaxnreg moves registers between warpgroups inside the
// CTA's launch allocation, so the split balances only if the kernel is launched with
// exactly kLaunchRegs registers per thread: refuse to launch otherwise, since an
// unbalanced split would wait for registers forever), set the shared-memory size, launch.
template <bool PAIR, bool DUAL>
kvq_status launch_attention(const AttnArgs& a, int64_t units, int splits, int heads, cudaStream_t stream)
{
    cudaFuncAttributes fa{};
    cudaError_t e = cudaFuncGetAttributes(&fa, attention_kernel<PAIR, DUAL>);
    if (e != cudaSuccess)
        return launched(e, "kvq_attention");
    if (fa.numRegs != kLaunchRegs)
        return fail(KVQ_ERR_UNSUPPORTED, "kvq_attention: kernel built with %d registers per thread, its register split needs %d",
                    fa.numRegs, kLaunchRegs);
    e = cudaFuncSetAttribute(attention_kernel<PAIR, DUAL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Geo<PAIR>::kSmemBytes);
    if (e != cudaSuccess)
        return launched(e, "kvq_attention");
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = PAIR ? 2 : 1;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(Geo<PAIR>::kCtas * units), static_cast<unsigned>(splits),
                       static_cast<unsigned>(heads));
    cfg.blockDim = dim3(kAttnThreads);
    cfg.dynamicSmemBytes = Geo<PAIR>::kSmemBytes;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = PAIR ? 2 : 1;
    return launched(cudaLaunchKernelEx(&cfg, attention_kernel<PAIR, DUAL>, a), "kvq_attention");
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
    const int64_t key_tiles = (n_keys + kBN - 1) / kBN;
    if (key_tiles > INT32_MAX)
        return fail(KVQ_ERR_INVALID_ARG, "kvq_attention_workspace_bytes: too many keys");
    *bytes = plan_attention(n_queries, heads, key_tiles).ws_bytes;
    return ok();
}

kvq_status kvq_attention_launches(int32_t n_queries, int32_t heads, int64_t n_keys, int32_t* launches)
{
    if (launches == nullptr || n_queries < 0 || heads <= 0 || n_keys < 0)
        return fail(KVQ_ERR_INVALID_ARG, "kvq_attention_launches: bad arguments");
    *launches = 0;
    if (n_queries == 0)
        return ok();
    const int64_t key_tiles = (n_keys + kBN - 1) / kBN;
    if (key_tiles > INT32_MAX)
        return fail(KVQ_ERR_INVALID_ARG, "kvq_attention_launches: too many keys");
    const AttnPlan plan = plan_attention(n_queries, heads, key_tiles);
    for (int i = 0; i < plan.n_parts; ++i)
        *launches += plan.part[i].partials() > 1 ? 2 : 1;
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
    if (static_cast<int64_t>(n_queries) * heads / (kCombineThreads / 32) >= INT32_MAX)
        return fail(KVQ_ERR_UNSUPPORTED, "kvq_attention: n_queries * heads too large");
    // a workspace smaller than the plan's takes fewer key splits (the part with the most
    // partials first), and in the end no dual
    AttnPlan plan = plan_attention(n_queries, heads, key_tiles);
    while (plan.ws_bytes > workspace_bytes) {
        AttnPart& big =
            plan.n_parts == 2 && plan.part[1].partials() > plan.part[0].partials() ? plan.part[1] : plan.part[0];
        if (big.splits > 1)
            --big.splits;
        else if (big.dual)
            big.dual = false;
        else
            break;
        finish_plan(plan, heads);
    }
    if (plan.ws_bytes > 0 && (workspace == nullptr || !aligned(workspace, 16)))
        return fail(KVQ_ERR_MISALIGNED, "kvq_attention: workspace must be 16-byte aligned");

    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    for (int i = 0; i < plan.n_parts; ++i) {
        const AttnPart& pt = plan.part[i];
        const uint64_t row_off = static_cast<uint64_t>(pt.row0) * heads * kD;
        float* part_ws = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + pt.ws_offset);
        AttnArgs a;
        a.q = static_cast<const uint16_t*>(q) + row_off;
        a.o = static_cast<uint16_t*>(out) + row_off;
        const int partials = pt.partials();
        a.part_o = partials > 1 ? part_ws : nullptr;
        a.part_ml = partials > 1 ? reinterpret_cast<float2*>(part_ws + static_cast<uint64_t>(partials) * pt.rows * heads * kD)
                                 : nullptr;
        a.kp = k_cache->packed;
        a.ks = k_cache->scales;
        a.ka = k_cache->amax;
        a.vp = v_cache->packed;
        a.vs = v_cache->scales;
        a.va = v_cache->amax;
        a.n_q = pt.rows;
        a.heads = heads;
        a.splits = partials;
        a.key_tiles = static_cast<int32_t>(key_tiles);
        a.n_kv = n_keys;
        a.tokens_per_chunk = k_cache->rows_per_chunk / heads;
        a.scale_log2 = softmax_scale * 1.4426950408889634f;
        a.status = status;

        // (the plan takes dual only for single CTAs)
        kvq_status st = pt.pair   ? launch_attention<true, false>(a, pt.units, pt.splits, heads, s)
                        : pt.dual ? launch_attention<false, true>(a, pt.units, pt.splits, heads, s)
                                  : launch_attention<false, false>(a, pt.units, pt.splits, heads, s);
        if (st != KVQ_OK)
            return st;
        if (partials == 1)
            continue;
        const int64_t rows = static_cast<int64_t>(pt.rows) * heads;
        const int64_t rows_per_cta = kCombineThreads / 32;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>((rows + rows_per_cta - 1) / rows_per_cta));
        cfg.blockDim = dim3(kCombineThreads);
        cfg.stream = s;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        st = launched(cudaLaunchKernelEx(&cfg, combine_kernel, a), "kvq_attention (combine)");
        if (st != KVQ_OK)
            return st;
    }
    return ok();
}

}  // extern "C"

// ---------------------------------------------------------------------------------------
// kvq_attention_noalloc: kvq_attention for callers that cannot allocate device memory.
// The key-split partials live in this file-scope array instead of a caller workspace.
// The array is allocated with this file's kernels on every GPU that runs them and is
// held until the process exits; every call on a GPU shares it.

namespace kvq {
namespace {

constexpr uint64_t kNoAllocScratchBytes = uint64_t{32} << 20;  // 32 MiB

static __device__ __align__(256) uint8_t g_attention_scratch[kNoAllocScratchBytes];

// Device address of g_attention_scratch on the current device (in host code the array's
// name is only a host-side stand-in). It is looked up on every call, a host-side query
// that allocates nothing: a cached address would outlive a context reset
// (cudaDeviceReset) and point into the destroyed context. The first lookup on a device
// may load this file's device code.
kvq_status scratch_address(void** ptr)
{
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_attention_scratch);
    if (e != cudaSuccess)
        return launched(e, "kvq_attention_noalloc (scratch address)");
    *ptr = p;
    return KVQ_OK;
}

}  // namespace
}  // namespace kvq

extern "C" {

kvq_status kvq_attention_noalloc(const void* q, int32_t n_queries, int32_t heads, const kvq_cache* k_cache,
                                 const kvq_cache* v_cache, int64_t n_keys, float softmax_scale, void* out,
                                 int* status, kvq_stream_t stream)
{
    NvtxRange nvtx_range("kvq_attention_noalloc");
    uint64_t need = 0;
    kvq_status st = kvq_attention_workspace_bytes(n_queries, heads, n_keys, &need);
    if (st != KVQ_OK)
        return st;
    if (need > kNoAllocScratchBytes)
        return fail(KVQ_ERR_CAPACITY,
                    "kvq_attention_noalloc: %d queries x %d heads over %lld keys need %llu bytes of scratch; the "
                    "built-in scratch holds %llu (use kvq_attention with a workspace)",
                    n_queries, heads, static_cast<long long>(n_keys), static_cast<unsigned long long>(need),
                    static_cast<unsigned long long>(kNoAllocScratchBytes));
    void* scratch = nullptr;
    if (need > 0 && (st = scratch_address(&scratch)) != KVQ_OK)
        return st;
    // the same call as kvq_attention with the recommended workspace: the same key split,
    // hence the same result; when *status stays 0 every partial the combine reads was
    // written first by this call, so the scratch needs no clearing (after a wait that
    // gave up, *status is 1 and out may hold partials an earlier call left in the scratch)
    return kvq_attention(q, n_queries, heads, k_cache, v_cache, n_keys, softmax_scale, out, scratch, need, status,
                         stream);
}

}  // extern "C"

extern "C" void kvq_testing_set_attention_wait(uint64_t wait_ns)
{
    const uint64_t v = wait_ns ? wait_ns : kWaitNs;
    const uint32_t stall = wait_ns ? 1u : 0u;
    cudaMemcpyToSymbol(c_wait_ns, &v, sizeof(v));
    cudaMemcpyToSymbol(c_stall_mma, &stall, sizeof(stall));
}
