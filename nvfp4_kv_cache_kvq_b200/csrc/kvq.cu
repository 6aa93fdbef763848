// kvq.cu -- libkvq: blockwise NVFP4 KV-cache quantize / dequantize for B200 (sm_100a).
//
// The method ("How NVFP4 Quantization Works in LongLive 2.0 for Transformer Inference",
// sections "Understanding the NVFP4 Format", "Stage 1" and "Stage 3"; "How to Use KV
// Cache Quantization with LongLive's LongLiveQuantizationConfig", sections "FP4
// Quantization in the Causal Model", "CUDA De-quantization Pipeline", "Configuration
// Parameters Reference") is restated in include/kvq.h. This file holds the kernels and
// the C ABI around them.
//
// Kernels (streaming passes; no tensor cores, no shared-memory staging of data: every
// access is a fully coalesced 256-bit or narrower vector access):
//   fill_kernel      sets the amax slots a quantize is about to reduce into.
//   amax_kernel      max |x| over each tensor: 256-bit loads, a max.xorsign.abs.bf16x2
//                    tree per block, warp redux, one atomic max per CTA.
//   quantize_kernel  UPT units of BPT blocks per thread: one 256-bit load per block,
//                    block amax, e4m3 scale(s) by the rule, e2m1 codes via
//                    cvt.satfinite.e2m1x2, 8 bytes of codes + 1 scale byte per block
//                    stored; its round-trip modes also write the bf16 reconstruction.
//   dequant_kernel   the mirror image: 8 bytes + 1 scale byte -> one 256-bit bf16 store
//                    per block; in a cache, every CTA lies in one chunk (one amax).
// Every kernel takes a batch of tensors, so one launch covers every layer's K and V of
// an append or a read, and every launch is a programmatic dependent launch (pdl_begin).
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <atomic>
#include <cstring>

#include "kvq.h"
#include "kvq_common.h"
#include "kvq_device.cuh"
#include "kvq_testing.h"

namespace kvq {

constexpr float kGlobalDen = 2688.0f;   // e2m1 max * e4m3 max = 6 * 448

// ---------------------------------------------------------------- batch descriptors

struct AmaxBatch {
    const void* x[kMaxBatch];
    uint32_t* out[kMaxBatch];  // fp32 amax, reduced as its (non-negative) bit pattern
    uint64_t n_blocks;
};

struct ZeroBatch {
    uint32_t* out[kMaxBatch];
    int n;
    uint32_t value;  // written to every out[i]
};

struct QuantTensor {
    const void* x;
    uint8_t* packed;    // codes out (unused in MODE kYOnly)
    uint8_t* scales;    // scale codes out (unused in MODE kYOnly)
    const float* amax;  // amax used for this tensor
    float* amax_copy;   // when non-null, also receives *amax
    void* y;            // bf16 reconstruction out (MODE kCodesAndY, kYOnly)
};

// What quantize_kernel writes: the codes, the codes and the bf16 round trip, or the
// round trip alone ("fake quantization").
enum QuantMode { kCodes = 0, kCodesAndY = 1, kYOnly = 2 };

struct QuantBatch {
    QuantTensor t[kMaxBatch];
    uint64_t n_blocks;  // blocks per tensor
};

struct DequantTensor {
    const uint8_t* packed;  // block 0 of the cache (or tensor)
    const uint8_t* scales;  // block 0 of the cache (or tensor)
    const float* amax;      // chunk amax array (or the tensor amax)
    void* y;                // receives block blk_lo onwards
};

struct DequantBatch {
    DequantTensor t[kMaxBatch];
    uint64_t blk_lo, blk_hi;    // block range [blk_lo, blk_hi) to dequantize
    uint64_t blocks_per_chunk;  // blocks sharing one amax
    uint64_t chunk0;            // chunk of blk_lo; blockIdx.y counts chunks from here
};

// Work layout. Every CTA owns one contiguous tile of its tensor, and consecutive CTAs
// own consecutive tiles, so the CTAs resident at any moment stream through one compact
// window of memory. On B200 this measured 10-15% more DRAM throughput than a
// persistent grid-stride loop over the same bytes.
constexpr int kAmaxIters = 4;  // blocks per thread in amax_kernel
constexpr int kQWarps = kThreads / 32 - 1;  // quantize warps of fused_quantize_kernel (one warp reduces amax)
constexpr int kQThreads = kQWarps * 32;

// ---------------------------------------------------------------- kernels

__global__ void __launch_bounds__(64) fill_kernel(const ZeroBatch z)
{
    pdl_begin();
    int i = threadIdx.x;
    if (i < z.n)
        *z.out[i] = z.value;
}

// grid (tiles, tensors); a tile is kThreads * kAmaxIters blocks.
__global__ void __launch_bounds__(kThreads) amax_kernel(const AmaxBatch B)
{
    pdl_begin();
    const char* x = static_cast<const char*>(B.x[blockIdx.y]);
    const uint64_t base = static_cast<uint64_t>(blockIdx.x) * (kThreads * kAmaxIters) + threadIdx.x;
    uint32_t w[kAmaxIters][8];
#pragma unroll
    for (int i = 0; i < kAmaxIters; ++i) {
        const uint64_t b = base + i * kThreads;
        if (b < B.n_blocks)
            ld_nc_v8(x + b * 32, w[i]);
        else
#pragma unroll
            for (int k = 0; k < 8; ++k)
                w[i][k] = 0u;
    }
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < kAmaxIters; ++i)
        m = max(m, block_absmax_bits(w[i]));
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    __shared__ uint32_t warp_max[kThreads / 32];
    if ((threadIdx.x & 31) == 0)
        warp_max[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
        m = threadIdx.x < kThreads / 32 ? warp_max[threadIdx.x] : 0u;
        m = __reduce_max_sync(0xFFFFFFFFu, m);
        if (threadIdx.x == 0 && m != 0u)
            atomicMax(B.out[blockIdx.y], m << 16);  // bf16 bits -> fp32 bits
    }
}

// IEEE reciprocal of a decoded block scale; 0 when it is infinite (S == 0 or S tiny), so
// that every value of the block is sent to a signed zero.
__device__ __forceinline__ float safe_rcp(float S)
{
    float inv = __frcp_rn(S);
    return inv == __int_as_float(0x7F800000) ? 0.0f : inv;
}

// Per-CTA tables of the decoded block scale S(c) = e4m3_value(c) * gs and of its safe
// reciprocal, for every e4m3 code c the quantizer can produce (0..126).
struct ScaleTables {
    float S[128];
    float inv[128];
};

__device__ __forceinline__ void build_scale_tables(ScaleTables& t, float gs)
{
    for (int c = threadIdx.x; c < 128; c += kThreads) {
        float v, unused;
        e4m3x2_to_f32(static_cast<uint32_t>(c), v, unused);
        const float S = c == 127 ? 0.0f : __fmul_rn(v, gs);
        t.S[c] = S;
        t.inv[c] = safe_rcp(S);
    }
    __syncthreads();
}

// The same tables built by one warp for its own use (no CTA barrier).
__device__ __forceinline__ void build_scale_tables_warp(ScaleTables& t, float gs)
{
    for (int c = threadIdx.x & 31; c < 128; c += 32) {
        float v, unused;
        e4m3x2_to_f32(static_cast<uint32_t>(c), v, unused);
        const float S = c == 127 ? 0.0f : __fmul_rn(v, gs);
        t.S[c] = S;
        t.inv[c] = safe_rcp(S);
    }
    __syncwarp();
}

// The block's 16 bf16 values as eight fp32 pairs (element 2j low, 2j + 1 high).
__device__ __forceinline__ void block_pairs(const uint32_t (&w)[8], uint64_t (&xp)[8])
{
#pragma unroll
    for (int j = 0; j < 8; ++j)
        xp[j] = f32x2_pack(bf16lo_to_f32(w[j]), bf16hi_to_f32(w[j]));
}

// The e2m1 codes of one block under decoded-scale reciprocal inv (two words).
__device__ __forceinline__ void encode_values(const uint64_t (&xp)[8], float inv, uint32_t& q0, uint32_t& q1)
{
    const uint64_t inv2 = f32x2_pack(inv, inv);
    float v0[8], v1[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        f32x2_unpack(f32x2_mul(xp[j], inv2), v0[2 * j], v0[2 * j + 1]);
        f32x2_unpack(f32x2_mul(xp[4 + j], inv2), v1[2 * j], v1[2 * j + 1]);
    }
    q0 = e2m1x8_from_f32(v0);
    q1 = e2m1x8_from_f32(v1);
}

// One mse candidate: the codes of the block under scale S (reciprocal inv) and their
// squared reconstruction error. Residuals x - value*S are one fma each (computed as
// fma(value, -S, x)); squares accumulate by fma into the pair (even-position sum,
// odd-position sum) in index order; the two sums are then added.
__device__ __forceinline__ float encode_values_sq_error(const uint64_t (&xp)[8], float S, float inv, uint32_t& q0,
                                                        uint32_t& q1)
{
    const uint64_t inv2 = f32x2_pack(inv, inv);
    const uint64_t nS2 = f32x2_pack(-S, -S);
    float v0[8], v1[8], val0[8], val1[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        f32x2_unpack(f32x2_mul(xp[j], inv2), v0[2 * j], v0[2 * j + 1]);
        f32x2_unpack(f32x2_mul(xp[4 + j], inv2), v1[2 * j], v1[2 * j + 1]);
    }
    q0 = e2m1x8_encode_decode(v0, val0);
    q1 = e2m1x8_encode_decode(v1, val1);
    uint64_t acc = f32x2_pack(0.0f, 0.0f);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint64_t d = f32x2_fma(f32x2_pack(val0[2 * j], val0[2 * j + 1]), nS2, xp[j]);
        acc = f32x2_fma(d, d, acc);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint64_t d = f32x2_fma(f32x2_pack(val1[2 * j], val1[2 * j + 1]), nS2, xp[4 + j]);
        acc = f32x2_fma(d, d, acc);
    }
    float se, so;
    f32x2_unpack(acc, se, so);
    return __fadd_rn(se, so);
}

// Correctly rounded quotients without a division per block: Markstein's correction step
// (P. Markstein, "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990). With y = RN(1/b) (CUDA's IEEE reciprocal,
// __frcp_rn) and q = RN(a*y), the remainder r = a - b*q is exact as one fma and
// RN(q + r*y) is the IEEE quotient RN(a/b), as long as nothing under- or overflows.
// For a/6 this holds for every bf16 amax (checked exhaustively). For s/gs it holds when
// gs is in [2^-80, 2^125] and the quotient is in [2^-12, 464], the only range where the
// quotient decides an e4m3 code (below 2^-12 every code is 0, above 464 every code
// saturates to 448). Clamping at 512 keeps an overflowing quotient (a caller's amax_in
// far below the data) on the saturating side, as the IEEE quotient is.
struct Quotients {
    float gs, inv_gs;
    bool markstein;  // gs in [2^-80, 2^125]; else IEEE division
};

__device__ __forceinline__ float markstein(float a, float b, float y)
{
    const float q = __fmul_rn(a, y);
    const float r = __fmaf_rn(-q, b, a);
    return __fmaf_rn(r, y, q);
}

__device__ __forceinline__ float div6(float a)
{
    return markstein(a, 6.0f, __int_as_float(0x3E2AAAAB));  // RN(1/6)
}

// e4m3 input of a block scale s: (s / gs), exactly where it decides the code. MARK is
// the per-tensor choice between the corrected product and IEEE division; it is a
// template parameter so that each kernel path holds only one of the two.
template <bool MARK>
__device__ __forceinline__ float scale_ratio(float s, const Quotients& qt)
{
    return MARK ? fminf(markstein(s, qt.gs, qt.inv_gs), 512.0f) : __fdiv_rn(s, qt.gs);
}

// Quantize one block held in w (16 bf16). Returns the scale code; q0/q1 get the codes.
// With MARK, gs >= 2^-80 is non-zero; otherwise gs == 0 (an all-zero tensor or amax_in
// == 0) forces every scale code to 0.
template <int RULE, bool MARK>
__device__ __forceinline__ uint32_t quantize_block(const uint32_t (&w)[8], const Quotients& qt,
                                                   const ScaleTables& tab, uint32_t& q0, uint32_t& q1)
{
    const bool gs_zero = !MARK && qt.gs == 0.0f;
    const float amax_b = __uint_as_float(block_absmax_bits(w) << 16);
    uint64_t xp[8];
    block_pairs(w, xp);
    if (RULE == KVQ_RULE_STATIC_6 || RULE == KVQ_RULE_STATIC_4) {
        // amax_b / 4 is exact, so the product by 0.25 equals the IEEE quotient
        const float s = RULE == KVQ_RULE_STATIC_6 ? div6(amax_b) : __fmul_rn(amax_b, 0.25f);
        const uint32_t c = gs_zero ? 0u : (e4m3x2_from_f32(0.0f, scale_ratio<MARK>(s, qt)) & 0xFFu);
        encode_values(xp, tab.inv[c], q0, q1);
        return c;
    } else {
        const float r6 = scale_ratio<MARK>(div6(amax_b), qt);
        const float r4 = scale_ratio<MARK>(__fmul_rn(amax_b, 0.25f), qt);
        const uint32_t c2 = gs_zero ? 0u : e4m3x2_from_f32(r4, r6);  // c6 in bits 0..7, c4 in 8..15
        const uint32_t c6 = c2 & 0xFFu, c4 = c2 >> 8;
        uint32_t a0, a1, b0, b1;
        const float e6 = encode_values_sq_error(xp, tab.S[c6], tab.inv[c6], a0, a1);
        const float e4 = encode_values_sq_error(xp, tab.S[c4], tab.inv[c4], b0, b1);
        const bool use4 = e4 < e6;
        q0 = use4 ? b0 : a0;
        q1 = use4 ? b1 : a1;
        return use4 ? c4 : c6;
    }
}

// One block: 8 code bytes (two words) and its decoded scale S -> 16 bf16 (eight words),
// y = bf16_rne(value * S).
__device__ __forceinline__ void bf16_from_codes(uint32_t q0, uint32_t q1, float S, uint32_t (&y)[8])
{
    const uint64_t S2 = f32x2_pack(S, S);
    float v[8];
    e2m1x8_to_f32(q0, v);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float lo, hi;
        f32x2_unpack(f32x2_mul(f32x2_pack(v[2 * j], v[2 * j + 1]), S2), lo, hi);
        y[j] = bf16x2_from_f32(hi, lo);
    }
    e2m1x8_to_f32(q1, v);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float lo, hi;
        f32x2_unpack(f32x2_mul(f32x2_pack(v[2 * j], v[2 * j + 1]), S2), lo, hi);
        y[4 + j] = bf16x2_from_f32(hi, lo);
    }
}

// The input of unit u of a tensor: blocks [u*BPT, u*BPT + BPT) clipped to n_blocks (a
// pair unit whose second block is past the end loads one).
template <int BPT>
__device__ __forceinline__ void load_unit(const QuantTensor& T, uint64_t u, uint64_t n_blocks, uint32_t (&w)[2][8])
{
    const char* x = static_cast<const char*>(T.x);
    const uint64_t b0 = u * BPT;
    ld_nc_v8(x + b0 * 32, w[0]);
    if (BPT == 2 && b0 + 1 < n_blocks)
        ld_nc_v8(x + b0 * 32 + 32, w[1]);
}

// Quantize unit u from its loaded input w: codes, scales and (MODE) the bf16 round trip.
template <int RULE, int BPT, bool MARK, int MODE>
__device__ __forceinline__ void quantize_loaded(const QuantTensor& T, uint64_t u, uint64_t n_blocks,
                                                const Quotients& qt, const ScaleTables& tab, const uint32_t (&w)[2][8])
{
    char* y = static_cast<char*>(T.y);
    const uint64_t b0 = u * BPT;
    if (BPT == 2 && b0 + 1 < n_blocks) {
        uint32_t q0, q1, q2, q3;
        const uint32_t c0 = quantize_block<RULE, MARK>(w[0], qt, tab, q0, q1);
        const uint32_t c1 = quantize_block<RULE, MARK>(w[1], qt, tab, q2, q3);
        if (MODE != kYOnly) {
            st_v4(T.packed + b0 * 8, q0, q1, q2, q3);
            *reinterpret_cast<uint16_t*>(T.scales + b0) = static_cast<uint16_t>(c0 | (c1 << 8));
        }
        if (MODE != kCodes) {
            uint32_t yy[8];
            bf16_from_codes(q0, q1, tab.S[c0], yy);
            st_v8(y + b0 * 32, yy);
            bf16_from_codes(q2, q3, tab.S[c1], yy);
            st_v8(y + b0 * 32 + 32, yy);
        }
    } else {  // BPT == 1, or the odd last block of a pair unit
        uint32_t q0, q1;
        const uint32_t c0 = quantize_block<RULE, MARK>(w[0], qt, tab, q0, q1);
        if (MODE != kYOnly) {
            st_v2(T.packed + b0 * 8, q0, q1);
            T.scales[b0] = static_cast<uint8_t>(c0);
        }
        if (MODE != kCodes) {
            uint32_t yy[8];
            bf16_from_codes(q0, q1, tab.S[c0], yy);
            st_v8(y + b0 * 32, yy);
        }
    }
}

// Unit u of a tensor, loaded and quantized.
template <int RULE, int BPT, bool MARK, int MODE>
__device__ __forceinline__ void quantize_unit(const QuantTensor& T, uint64_t u, uint64_t n_blocks,
                                              const Quotients& qt, const ScaleTables& tab)
{
    uint32_t w[2][8];
    load_unit<BPT>(T, u, n_blocks, w);
    quantize_loaded<RULE, BPT, MARK, MODE>(T, u, n_blocks, qt, tab, w);
}

// The global scale of a tensor amax and how its block-scale quotients are computed.
__device__ __forceinline__ Quotients make_quotients(float amax)
{
    Quotients qt;
    qt.gs = __fdiv_rn(amax, kGlobalDen);
    qt.markstein = qt.gs >= 0x1p-80f && qt.gs <= 0x1p125f;
    qt.inv_gs = qt.markstein ? __frcp_rn(qt.gs) : 0.0f;
    return qt;
}

// Units u0, u0 + STRIDE, ... (n_units of them, stopping at the tensor's end) of one
// thread, BPT blocks each. MARK is uniform per tensor, so each path holds one quotient
// form only.
template <int RULE, int BPT, int MODE, bool MARK, int STRIDE = kThreads>
__device__ __forceinline__ void quantize_units(const QuantTensor& T, uint64_t u0, int n_units, uint64_t n_blocks,
                                               const Quotients& qt, const ScaleTables& tab)
{
#pragma unroll 1
    for (int i = 0; i < n_units; ++i) {
        const uint64_t u = u0 + static_cast<uint64_t>(i) * STRIDE;
        if (u * BPT >= n_blocks)
            return;
        quantize_unit<RULE, BPT, MARK, MODE>(T, u, n_blocks, qt, tab);
    }
}

// grid (tiles, tensors), UPT units of BPT blocks per thread; the amax of every tensor is
// already known (the caller's amax_in, or a separate amax pass). The tiles and tensors
// are walked in the reverse of amax_kernel's order, so the data amax_kernel read last
// (still in L2) is quantized first. With BPT = 2 the packed pointer must be 16-byte and
// the scale pointer 2-byte aligned. MODE selects the outputs (QuantMode); the round trip
// y = bf16_rne(value * S) is the same arithmetic as dequant_kernel, so it is bit-equal to
// quantizing and then dequantizing.
template <int RULE, int BPT, int MODE, int UPT = 1>
__global__ void __launch_bounds__(kThreads) quantize_kernel(const QuantBatch B)
{
    pdl_begin();
    __shared__ ScaleTables tab;
    const QuantTensor& T = B.t[gridDim.y - 1 - blockIdx.y];
    const float amax = __ldg(T.amax);
    const Quotients qt = make_quotients(amax);
    if (T.amax_copy != nullptr && blockIdx.x == 0 && threadIdx.x == 0)
        *T.amax_copy = amax;
    build_scale_tables(tab, qt.gs);
    const uint64_t u0 = static_cast<uint64_t>(gridDim.x - 1 - blockIdx.x) * (kThreads * UPT) + threadIdx.x;
    if (qt.markstein)
        quantize_units<RULE, BPT, MODE, true>(T, u0, UPT, B.n_blocks, qt, tab);
    else
        quantize_units<RULE, BPT, MODE, false>(T, u0, UPT, B.n_blocks, qt, tab);
}

// ---------------------------------------------------------------- device error word

// Sticky per-device error word: a kernel whose bounded wait gave up ORs a bit into it;
// kvq_device_status() reads and clears it. It is the only state the codec kernels keep.
__device__ unsigned int g_device_error;
constexpr unsigned kDeviceErrWaitTimeout = 1u;

// ---------------------------------------------------------------- one-launch amax + quantize
//
// fused_quantize_kernel computes every tensor's amax and quantizes the tensor in the same
// launch, so a tensor that fits in L2 is read from DRAM once: the quantize pass reads it
// back from L2. Each tensor is cut into tiles of kTileBlocks blocks, and the tiles are
// dealt to the CTAs round-robin in tensor-major order (CTA b takes tiles b, b + G, ...;
// G = gridDim.x, at most the CTAs the GPU holds at once). In every CTA
//   one warp (the amax warp) takes its tiles' amax parts: a TMA bulk copy into shared
//   memory, a max over it, folded into the tensor's amax slot;
//   the other kQWarps warps take the same tiles' quantize parts, each once its tensor's
//   amax is complete, meeting among themselves at a named barrier per tile (amax
//   broadcast, scale tables).
// The amax warp runs ahead of its own CTA's quantize warps by at most `window` tiles (one
// tensor and one and a half grids): far enough that a tensor's amax is mostly complete
// before its quantize tiles ask for it, close enough that the tiles in between are still
// in L2 when they are quantized (a global throttle, an amax warp waiting for tensor t - L
// to be quantized everywhere, measured slower and missed L2 on most re-reads). Progress,
// by induction over the tensors: let t be the first tensor whose amax is incomplete. The
// quantize warps of a CTA owning one of t's amax tiles do not wait on earlier tensors, so
// they reach a tile of tensor t or later (position >= t's first tile) or finish; the
// window, at least one tensor, then reaches every tile of t, so the CTA's amax warp folds
// its tiles of t and t completes. With every CTA resident, each wait ends. The quantize
// warps share nothing with the amax warp but the position they publish.
//
// The synchronisation lives in the caller's amax slot, so the launch needs no memory of
// its own. fill_kernel sets the slot to kSlotBase before the launch; then
//   bits 16..31  max |x| so far, as bf16 bits. Every |x| is a bf16 value, so the fp32 amax
//                has zero low bits and the high half is all of it;
//   bits  0..15  kSlotBase + the number of amax tiles folded in (below 0x7F7F, so read as a
//                bf16 it is non-negative and finite, and the max below leaves it alone).
// A tile folds its max into the high half (bf16 max; the low lane against +0) and then
// adds 1, both read-modify-writes of the same word by one thread, so each count covers
// its max; neither waits for a reply. A reader waits (bounded) until the low half is 0
// or above the number of tiles, takes the high half, and, if the low half was not 0,
// stores the plain fp32 amax (low half 0): once every tile is in nothing else writes the
// slot, so all readers store the same word, and every tensor has a reader. If a wait
// gives up, the reader stores a NaN in the slot, raises kDeviceErrWaitTimeout, and its
// tile writes nothing; readers skip a NaN slot.

constexpr uint32_t kTileBlocks = 896;             // blocks of a tile (kQThreads x 2 units x 2 blocks)
constexpr uint32_t kTileBytes = kTileBlocks * 32;
constexpr uint32_t kSlotBase = 1u;
constexpr uint32_t kQBarrier = 1;                 // named barrier of the quantize warps

struct FusedBatch {
    QuantTensor t[kMaxBatch];  // t.amax: the slot, set to kSlotBase before the launch
    uint64_t n_blocks;         // blocks per tensor
    uint64_t wait_ns;          // bound of every wait
    uint32_t n_tensors;
    uint32_t tiles;            // tiles per tensor
    uint32_t q_units;          // units per quantize thread of a tile: kTileBlocks / (kQThreads * BPT)
    uint32_t expect_a;         // amax tiles a quantize tile waits for (tiles)
    uint32_t window;           // tiles the amax warp may run ahead of its CTA's quantize position
    uint32_t n_sm;             // multiprocessors of the device
};

constexpr uint32_t kNaNBits = 0x7FC00000u;
constexpr uint32_t kQDone = 0xFFFFFFFFu;  // published quantize position: no more tiles

__device__ __forceinline__ uint32_t* slot_of(const FusedBatch& B, uint32_t t)
{
    return reinterpret_cast<uint32_t*>(const_cast<float*>(B.t[t].amax));
}

// The slot word is complete: every amax tile folded in (low half above expect_a), or
// the plain amax left by a reader (low half 0).
__device__ __forceinline__ bool slot_complete(uint32_t v, uint32_t expect_a)
{
    const uint32_t c = v & 0xFFFFu;
    return c == 0u || c > expect_a;
}

// The amax bits of tensor t, or kNaNBits if the wait gave up (or an earlier one did).
__device__ __forceinline__ uint32_t await_amax(const FusedBatch& B, uint32_t t)
{
    uint32_t* slot = slot_of(B, t);
    uint32_t v = ld_relaxed_u32(slot);
    if (!slot_complete(v, B.expect_a)) {
        // polls back off from 64 to 512 ns: the slot is one word that every CTA of the
        // tensor reads and its amax tiles fold into (measured 3 % faster than 64 ns polls)
        const uint64_t t0 = globaltimer_ns();
        uint32_t ns = 64;
        while (!slot_complete(v = ld_relaxed_u32(slot), B.expect_a)) {
            if (globaltimer_ns() - t0 > B.wait_ns) {
                st_relaxed_u32(slot, kNaNBits);
                atomicOr(&g_device_error, kDeviceErrWaitTimeout);
                return kNaNBits;
            }
            __nanosleep(ns);
            ns = ns < 512u ? 2 * ns : ns;
        }
    }
    if ((v & 0xFFFF0000u) == kNaNBits)
        return kNaNBits;
    if ((v & 0xFFFFu) != 0)  // complete but not yet plain: every reader may store the same amax
        st_relaxed_u32(slot, v & 0xFFFF0000u);
    return v & 0xFFFF0000u;
}

// The amax warp: the amax parts of tiles blockIdx.x, blockIdx.x + G, ... Each waits until
// the CTA's quantize warps have reached within `window` of it.
__device__ __forceinline__ void amax_warp(const FusedBatch& B, uint4* stage, uint64_t* bar, const uint32_t* q_pos)
{
    const uint32_t lane = threadIdx.x & 31;
    const uint64_t n_tiles = static_cast<uint64_t>(B.n_tensors) * B.tiles;
    uint32_t phase = 0;
#pragma unroll 1
    for (uint64_t a = blockIdx.x; a < n_tiles; a += gridDim.x, phase ^= 1) {
        uint32_t qp = ld_volatile_smem(q_pos);
        if (qp != kQDone && a > static_cast<uint64_t>(qp) + B.window) {
            const uint64_t t0 = globaltimer_ns();
            while ((qp = ld_volatile_smem(q_pos)) != kQDone && a > static_cast<uint64_t>(qp) + B.window) {
                if (globaltimer_ns() - t0 > B.wait_ns) {
                    if (lane == 0)
                        atomicOr(&g_device_error, kDeviceErrWaitTimeout);
                    return;  // no copy in flight
                }
                __nanosleep(256);
            }
        }
        const uint32_t t = static_cast<uint32_t>(a / B.tiles);
        const uint64_t b0 = (a % B.tiles) * kTileBlocks;
        const uint32_t nb = static_cast<uint32_t>(B.n_blocks - b0 < kTileBlocks ? B.n_blocks - b0 : kTileBlocks);
        __syncwarp();  // every lane has read the stage of the previous tile
        if (lane == 0) {
            fence_proxy_async_smem();
            bulk_load(stage, static_cast<const char*>(B.t[t].x) + b0 * 32, nb * 32, bar);
        }
        // (a hardware-suspended wait: 3 % faster on two-tensor jobs than polling with sleeps)
        bool landed = mbar_try_parity(bar, phase);
        if (!landed) {
            const uint64_t t0 = globaltimer_ns();
            while (!(landed = mbar_try_parity(bar, phase)) && globaltimer_ns() - t0 <= B.wait_ns) {
            }
        }
        if (!landed) {  // a copy that does not land in the bound: wait once more, then leave
            if (lane == 0)
                atomicOr(&g_device_error, kDeviceErrWaitTimeout);
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_parity(bar, phase) && globaltimer_ns() - t0 <= B.wait_ns) {
            }
            return;
        }
        // lane-wise |x| maxima over the tile's 16-byte vectors, then across lanes
        const uint32_t n16 = nb * 2;
        uint32_t m0 = 0, m1 = 0, m2 = 0, m3 = 0;
#pragma unroll 4
        for (uint32_t i = lane; i < n16; i += 32) {
            const uint4 w = stage[i];
            m0 = absmax_bf16x2(m0, w.x);
            m1 = absmax_bf16x2(m1, w.y);
            m2 = absmax_bf16x2(m2, w.z);
            m3 = absmax_bf16x2(m3, w.w);
        }
        uint32_t m = absmax_bf16x2(absmax_bf16x2(m0, m1), absmax_bf16x2(m2, m3)) & 0x7FFF7FFFu;
        m = __reduce_max_sync(0xFFFFFFFFu, max(m & 0xFFFFu, m >> 16));
        if (lane == 0) {  // fold: max into the high half, then count; no reply awaited
            uint32_t* slot = slot_of(B, t);
            red_max_bf16_high(slot, m);
            red_add_relaxed_u32(slot, 1u);
        }
    }
}

template <int RULE, int BPT, int MODE>
__global__ void __launch_bounds__(kThreads) fused_quantize_kernel(const FusedBatch B)
{
    __shared__ __align__(128) uint4 stage[kTileBytes / 16];
    __shared__ ScaleTables tab;
    __shared__ uint64_t bar;
    __shared__ uint32_t q_pos;  // the quantize warps' current tile
    __shared__ uint32_t amax_bcast;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        q_pos = 0;
    }
    pdl_begin();
    __syncthreads();  // the last CTA-wide barrier: from here the amax warp and the rest run apart
    // The amax warp's index rotates with the wave of CTAs (CTAs b and b + n_sm usually share
    // an SM), so the amax warps of an SM sit on different sub-partitions.
    const uint32_t warp = threadIdx.x >> 5, a_warp = (blockIdx.x / B.n_sm) & 3u;
    if (warp == a_warp) {
        amax_warp(B, stage, &bar, &q_pos);
        return;
    }
    const uint32_t qt_idx = (warp < a_warp ? warp : warp - 1) * 32 + (threadIdx.x & 31);  // 0 .. kQThreads-1
    const uint64_t n_tiles = static_cast<uint64_t>(B.n_tensors) * B.tiles;
    Quotients qt;
    uint32_t tab_tensor = 0xFFFFFFFFu;
#pragma unroll 1
    for (uint64_t q = blockIdx.x; q < n_tiles; q += gridDim.x) {
        const uint32_t t = static_cast<uint32_t>(q / B.tiles), tile = static_cast<uint32_t>(q % B.tiles);
        if (qt_idx == 0) {
            st_volatile_smem(&q_pos, static_cast<uint32_t>(q));  // publish the position, then wait
            amax_bcast = await_amax(B, t);
        }
        named_barrier(kQBarrier, kQThreads);  // the amax is known; the tables are free
        const uint32_t amax_bits = amax_bcast;
        if (amax_bits == kNaNBits) {
            named_barrier(kQBarrier, kQThreads);  // everyone has read amax_bcast
            continue;
        }
        if (t != tab_tensor) {
            qt = make_quotients(__uint_as_float(amax_bits));
            for (uint32_t c = qt_idx; c < 128; c += kQThreads) {
                float v, unused;
                e4m3x2_to_f32(c, v, unused);
                const float S = c == 127 ? 0.0f : __fmul_rn(v, qt.gs);
                tab.S[c] = S;
                tab.inv[c] = safe_rcp(S);
            }
            tab_tensor = t;
        }
        named_barrier(kQBarrier, kQThreads);  // tables ready; amax_bcast read by everyone
        const uint64_t u0 = static_cast<uint64_t>(tile) * (kQThreads * B.q_units) + qt_idx;
        if (qt.markstein)
            quantize_units<RULE, BPT, MODE, true, kQThreads>(B.t[t], u0, B.q_units, B.n_blocks, qt, tab);
        else
            quantize_units<RULE, BPT, MODE, false, kQThreads>(B.t[t], u0, B.q_units, B.n_blocks, qt, tab);
    }
    if (qt_idx == 0)
        st_volatile_smem(&q_pos, kQDone);
}

// One block: 8 code bytes and its scale code under global scale gs -> 16 bf16.
__device__ __forceinline__ void dequant_block(uint32_t q0, uint32_t q1, uint32_t c, float gs, uint32_t (&y)[8])
{
    float S, unused;
    e4m3x2_to_f32(c & 0xFFu, S, unused);
    bf16_from_codes(q0, q1, __fmul_rn(S, gs), y);
}

// grid (tiles, chunks, tensors). Each CTA lies inside one chunk, so its amax (and global
// scale) is one load per CTA. Blocks are numbered from block 0 of the cache; units of BPT
// blocks are aligned to that numbering, and blocks outside [blk_lo, blk_hi) are skipped.
template <int BPT>
__global__ void __launch_bounds__(kThreads) dequant_kernel(const DequantBatch B)
{
    pdl_begin();
    const DequantTensor& T = B.t[blockIdx.z];
    const uint64_t chunk = B.chunk0 + blockIdx.y;
    const uint64_t c_lo = chunk * B.blocks_per_chunk;
    const uint64_t lo = c_lo > B.blk_lo ? c_lo : B.blk_lo;
    const uint64_t c_hi = c_lo + B.blocks_per_chunk;
    const uint64_t hi = c_hi < B.blk_hi ? c_hi : B.blk_hi;
    if (lo >= hi)
        return;
    const uint64_t u = lo / BPT + static_cast<uint64_t>(blockIdx.x) * kThreads + threadIdx.x;
    const uint64_t b0 = u * BPT;
    if (b0 >= hi)
        return;
    const float gs = __fdiv_rn(__ldg(T.amax + chunk), kGlobalDen);
    char* y = static_cast<char*>(T.y);
    if (BPT == 2 && b0 + 1 < hi) {  // both blocks of the unit readable (block b0 may be lo - 1)
        const uint4 q = ld_nc_v4(T.packed + b0 * 8);
        const uint32_t c = __ldg(reinterpret_cast<const uint16_t*>(T.scales + b0));
        uint32_t y0[8];
        if (b0 >= lo) {
            dequant_block(q.x, q.y, c, gs, y0);
            st_v8(y + (b0 - B.blk_lo) * 32, y0);
        }
        dequant_block(q.z, q.w, c >> 8, gs, y0);
        st_v8(y + (b0 + 1 - B.blk_lo) * 32, y0);
    } else {  // BPT == 1, or a unit whose second block is past the range
        const uint64_t b = (BPT == 2 && b0 < lo) ? b0 + 1 : b0;
        const uint2 q = ld_nc_v2(T.packed + b * 8);
        uint32_t y0[8];
        dequant_block(q.x, q.y, __ldg(T.scales + b), gs, y0);
        st_v8(y + (b - B.blk_lo) * 32, y0);
    }
}

// ---------------------------------------------------------------- host side

thread_local char g_last_error[512] = "";

kvq_status check_rule(kvq_scale_rule rule)
{
    if (rule != KVQ_RULE_STATIC_6 && rule != KVQ_RULE_STATIC_4 && rule != KVQ_RULE_MSE)
        return fail(KVQ_ERR_INVALID_ARG, "unknown scale rule %d", static_cast<int>(rule));
    return KVQ_OK;
}


// Units per thread of quantize_kernel. The mse rule is instruction-bound; 8 units per
// thread amortize the per-CTA scale tables (+4% on B200) as long as the launch keeps
// enough CTAs to fill the GPU many times over (else the last partial wave costs more).
// The static rules are DRAM-bound either way and keep one unit per thread.
constexpr uint64_t kMinCtasForUpt8 = 2048;

template <int RULE, int BPT, int U>
cudaError_t launch_quantize_upt(int mode, uint64_t units, int n, const QuantBatch& qb, cudaStream_t s)
{
    const dim3 grid(tiles(units, U), n);
    if (mode == kCodes)
        return launch(quantize_kernel<RULE, BPT, kCodes, U>, grid, kThreads, s, qb);
    if (mode == kCodesAndY)
        return launch(quantize_kernel<RULE, BPT, kCodesAndY, U>, grid, kThreads, s, qb);
    return launch(quantize_kernel<RULE, BPT, kYOnly, U>, grid, kThreads, s, qb);
}

template <int RULE, int BPT>
cudaError_t launch_quantize_mode(int mode, uint64_t units, int n, const QuantBatch& qb, cudaStream_t s)
{
    if (RULE == KVQ_RULE_MSE && static_cast<uint64_t>(tiles(units, 8)) * n >= kMinCtasForUpt8)
        return launch_quantize_upt<RULE, BPT, 8>(mode, units, n, qb, s);
    return launch_quantize_upt<RULE, BPT, 1>(mode, units, n, qb, s);
}

template <int RULE>
cudaError_t launch_quantize_bpt(int bpt, int mode, uint64_t units, int n, const QuantBatch& qb, cudaStream_t s)
{
    return bpt == 2 ? launch_quantize_mode<RULE, 2>(mode, units, n, qb, s)
                    : launch_quantize_mode<RULE, 1>(mode, units, n, qb, s);
}

cudaError_t launch_quantize(kvq_scale_rule rule, int bpt, int mode, uint64_t units, int n, const QuantBatch& qb,
                            cudaStream_t s)
{
    if (rule == KVQ_RULE_STATIC_6)
        return launch_quantize_bpt<KVQ_RULE_STATIC_6>(bpt, mode, units, n, qb, s);
    if (rule == KVQ_RULE_STATIC_4)
        return launch_quantize_bpt<KVQ_RULE_STATIC_4>(bpt, mode, units, n, qb, s);
    return launch_quantize_bpt<KVQ_RULE_MSE>(bpt, mode, units, n, qb, s);
}

// Test hook (kvq_testing.h): extra A arrivals a Q-ticket waits for, and its wait bound.
thread_local uint32_t g_test_extra_a = 0;
thread_local uint64_t g_test_wait_ns = 0;

constexpr uint64_t kFusedWaitNs = 2000000000ull;  // 2 s
constexpr uint64_t kFusedMaxBlocks = 2ull << 20;  // 64 MiB of bf16: larger tensors take two passes

// CTAs of `kernel` the device holds at once (kThreads each), cached per device.
template <typename Kernel>
int resident_ctas(Kernel kernel)
{
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return 0;
    if (dev < 64) {
        const int c = cache[dev].load(std::memory_order_relaxed);
        if (c > 0)
            return c;
    }
    int sms = 0, occ = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, kThreads, 0) != cudaSuccess)
        return 0;
    const int r = (occ > 0 ? occ : 1) * (sms > 0 ? sms : 1);
    if (dev < 64)
        cache[dev].store(r, std::memory_order_relaxed);
    return r;
}

int sm_count()
{
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                  cudaSuccess)
        return 1;
    return sms > 0 ? sms : 1;
}

template <int RULE, int BPT, int MODE>
cudaError_t launch_fused(FusedBatch& fb, cudaStream_t s)
{
    auto kernel = fused_quantize_kernel<RULE, BPT, MODE>;
    const int res = resident_ctas(kernel);
    if (res <= 0)
        return cudaErrorUnknown;
    static_assert(kTileBlocks % (kQThreads * 2) == 0, "a tile is whole units of every width");
    fb.q_units = kTileBlocks / (kQThreads * BPT);
    const uint64_t n_tiles = static_cast<uint64_t>(fb.n_tensors) * fb.tiles;
    const uint64_t grid = n_tiles < static_cast<uint64_t>(res) ? n_tiles : static_cast<uint64_t>(res);
    // the amax warp may run one tensor and one and a half grids ahead of its CTA's quantize
    // warps. Measured on the rollout's appends (60 tensors of 4.8 MB): 1.75 or 2 grids ran
    // 4 % faster but the quantize re-reads then missed L2 (3.3 DRAM bytes per element
    // against 2.5); 3 grids ran slower.
    fb.window = fb.tiles + static_cast<uint32_t>(grid + grid / 2);
    fb.n_sm = static_cast<uint32_t>(sm_count());
    return launch(kernel, dim3(static_cast<unsigned>(grid)), kThreads, s, fb);
}

// (codes only: the round trip's bf16 output is a single-tensor call, which takes two passes)
template <int RULE>
cudaError_t launch_fused_bpt(int bpt, FusedBatch& fb, cudaStream_t s)
{
    return bpt == 2 ? launch_fused<RULE, 2, kCodes>(fb, s) : launch_fused<RULE, 1, kCodes>(fb, s);
}

// The one-launch plan for n tensors of n_blocks blocks, or false for tensors larger than
// kFusedMaxBlocks (their second read would not come from L2 anyway) and for a single
// tensor: with no other tensor's amax to overlap its quantize tiles, the two passes (every
// warp on the amax, then the codes, reading back from L2 what fits) measured 10-20 % faster
// from 2^15 to 2^21 blocks.
bool plan_fused(uint64_t n_blocks, int n, FusedBatch& fb)
{
    if (n < 2 || n_blocks == 0 || n_blocks > kFusedMaxBlocks)
        return false;
    fb.n_blocks = n_blocks;
    fb.n_tensors = static_cast<uint32_t>(n);
    fb.tiles = static_cast<uint32_t>((n_blocks + kTileBlocks - 1) / kTileBlocks);
    fb.expect_a = fb.tiles + g_test_extra_a;
    fb.wait_ns = g_test_wait_ns ? g_test_wait_ns : kFusedWaitNs;
    return kSlotBase + fb.expect_a < 0x7F00u;
}

// Quantize a batch of equally sized tensors whose amax slots are given. When
// compute_amax, the amax is reduced into the slots first: in the same launch
// (fused_quantize_kernel) for two or more tensors of up to kFusedMaxBlocks blocks
// (codes only), else by amax_kernel before quantize_kernel.
kvq_status run_quantize(const QuantBatch& qb, int n, bool compute_amax, kvq_scale_rule rule, cudaStream_t s,
                        int mode = kCodes)
{
    if (n == 0 || qb.n_blocks == 0)
        return KVQ_OK;
    bool pairs = true;
    if (mode != kYOnly)
        for (int i = 0; i < n; ++i)
            pairs = pairs && aligned(qb.t[i].packed, 16) && aligned(qb.t[i].scales, 2);
    const int bpt = pairs ? 2 : 1;
    kvq_status st;
    if (compute_amax) {
        for (int i = 0; i < n; ++i)
            for (int j = 0; j < i; ++j)
                if (qb.t[i].amax == qb.t[j].amax)
                    return fail(KVQ_ERR_INVALID_ARG, "tensors %d and %d share one amax output", j, i);
        FusedBatch fb;
        const bool fused = mode == kCodes && plan_fused(qb.n_blocks, n, fb);
        ZeroBatch z{};
        for (int i = 0; i < n; ++i)
            z.out[i] = reinterpret_cast<uint32_t*>(const_cast<float*>(qb.t[i].amax));
        z.n = n;
        z.value = fused ? kSlotBase : 0u;
        if ((st = launched(launch(fill_kernel, dim3(1), 64, s, z), "fill_kernel")) != KVQ_OK)
            return st;
        if (fused) {
            for (int i = 0; i < n; ++i)
                fb.t[i] = qb.t[i];
            cudaError_t e;
            if (rule == KVQ_RULE_STATIC_6)
                e = launch_fused_bpt<KVQ_RULE_STATIC_6>(bpt, fb, s);
            else if (rule == KVQ_RULE_STATIC_4)
                e = launch_fused_bpt<KVQ_RULE_STATIC_4>(bpt, fb, s);
            else
                e = launch_fused_bpt<KVQ_RULE_MSE>(bpt, fb, s);
            return launched(e, "fused_quantize_kernel");
        }
        AmaxBatch ab{};
        for (int i = 0; i < n; ++i) {
            ab.x[i] = qb.t[i].x;
            ab.out[i] = z.out[i];
        }
        ab.n_blocks = qb.n_blocks;
        if ((st = launched(launch(amax_kernel, dim3(tiles(qb.n_blocks, kAmaxIters), n), kThreads, s, ab),
                           "amax_kernel")) != KVQ_OK)
            return st;
    }
    const uint64_t units = pairs ? (qb.n_blocks + 1) / 2 : qb.n_blocks;
    return launched(launch_quantize(rule, bpt, mode, units, n, qb, s), "quantize_kernel");
}

// Dequantize blocks [blk_lo, blk_hi) of n equally laid-out tensors; packed/scales point at
// block 0 of each. One launch per group of at most 65535 chunks (the grid's y limit).
kvq_status run_dequantize(DequantBatch db, int n, cudaStream_t s)
{
    if (n == 0 || db.blk_hi <= db.blk_lo)
        return KVQ_OK;
    bool pairs = true;
    for (int i = 0; i < n; ++i)
        pairs = pairs && aligned(db.t[i].packed, 16) && aligned(db.t[i].scales, 2);
    const int bpt = pairs ? 2 : 1;
    const uint64_t bpc = db.blocks_per_chunk;
    const uint64_t first = db.blk_lo / bpc, last = (db.blk_hi - 1) / bpc;
    // units of one chunk, plus one for a chunk that starts inside a unit
    const unsigned gx = tiles((bpc + bpt - 1) / bpt + 1);
    for (uint64_t c0 = first; c0 <= last; c0 += 65535) {
        const uint64_t nc = (last - c0 + 1) < 65535 ? (last - c0 + 1) : 65535;
        db.chunk0 = c0;
        const dim3 grid(gx, static_cast<unsigned>(nc), n);
        kvq_status st = launched(pairs ? launch(dequant_kernel<2>, grid, kThreads, s, db)
                                       : launch(dequant_kernel<1>, grid, kThreads, s, db),
                                 "dequant_kernel");
        if (st != KVQ_OK)
            return st;
    }
    return KVQ_OK;
}

kvq_status check_cache(const kvq_cache* c, const char* what)
{
    if (c == nullptr)
        return fail(KVQ_ERR_INVALID_ARG, "%s: null cache", what);
    if (c->head_dim <= 0 || c->head_dim % kBlock != 0)
        return fail(KVQ_ERR_INVALID_ARG, "%s: head_dim %d is not a positive multiple of 16", what, c->head_dim);
    if (c->rows_per_chunk <= 0 || c->capacity_rows < 0)
        return fail(KVQ_ERR_INVALID_ARG, "%s: bad rows_per_chunk / capacity_rows", what);
    if (c->packed == nullptr || c->scales == nullptr || c->amax == nullptr)
        return fail(KVQ_ERR_INVALID_ARG, "%s: null cache buffer", what);
    if (!aligned(c->packed, 8) || !aligned(c->amax, 4))
        return fail(KVQ_ERR_MISALIGNED, "%s: cache packed must be 8-byte and amax 4-byte aligned", what);
    const uint64_t elems = static_cast<uint64_t>(c->capacity_rows) * static_cast<uint64_t>(c->head_dim);
    if (elems > kMaxElems)
        return fail(KVQ_ERR_UNSUPPORTED, "%s: cache above 2^36 elements", what);
    const uint64_t bpc = static_cast<uint64_t>(c->rows_per_chunk) * static_cast<uint64_t>(c->head_dim / kBlock);
    if (bpc > 0xFFFFFFFFull)
        return fail(KVQ_ERR_UNSUPPORTED, "%s: chunk above 2^32 blocks", what);
    return KVQ_OK;
}

}  // namespace kvq

namespace kvq {

// Shared body of kvq_quantize, kvq_quantize_batch and kvq_quantize_dequantize: n
// equally sized tensors. amax_in null: each tensor's amax is computed into amax_out[i].
// amax_in given: amax_in[i] is used and copied to amax_out[i] when that is given too.
kvq_status quantize_impl(const char* what, const void* const* xs, int32_t n, int64_t n_elems, int32_t head_dim,
                         kvq_scale_rule rule, const float* const* amax_in, float* const* amax_out,
                         uint8_t* const* packed, uint8_t* const* scales, void* const* ys, int mode,
                         cudaStream_t s)
{
    kvq_status st;
    if ((st = check_shape(n_elems, head_dim)) != KVQ_OK || (st = check_rule(rule)) != KVQ_OK)
        return st;
    if (n < 0)
        return fail(KVQ_ERR_INVALID_ARG, "%s: negative tensor count", what);
    if (n == 0)
        return ok();
    if (amax_in == nullptr && amax_out == nullptr)
        return fail(KVQ_ERR_INVALID_ARG, "%s: amax_in and amax_out are both null", what);
    if (xs == nullptr)
        return fail(KVQ_ERR_INVALID_ARG, "%s: null xs array", what);
    if (mode != kYOnly && (packed == nullptr || scales == nullptr))
        return fail(KVQ_ERR_INVALID_ARG, "%s: null packed / scales array", what);
    if (mode != kCodes && ys == nullptr)
        return fail(KVQ_ERR_INVALID_ARG, "%s: null y array", what);
    for (int i = 0; i < n; ++i) {
        const float* ain = amax_in ? amax_in[i] : nullptr;
        float* aout = amax_out ? amax_out[i] : nullptr;
        if (ain == nullptr && aout == nullptr)
            return fail(KVQ_ERR_INVALID_ARG, "%s: amax_in and amax_out are both null", what);
        if (amax_in != nullptr && ain == nullptr)
            return fail(KVQ_ERR_INVALID_ARG, "%s: amax_in given for some tensors only", what);
        if (n_elems > 0 && (xs[i] == nullptr || (mode != kYOnly && (packed[i] == nullptr || scales[i] == nullptr)) ||
                            (mode != kCodes && ys[i] == nullptr)))
            return fail(KVQ_ERR_INVALID_ARG, "%s: null tensor pointer", what);
        if (!aligned(xs[i], 32) || (mode != kYOnly && !aligned(packed[i], 8)) || (mode != kCodes && !aligned(ys[i], 32)) ||
            !aligned(ain, 4) || !aligned(aout, 4))
            return fail(KVQ_ERR_MISALIGNED, "%s: x and y must be 32-byte, packed 8-byte, amax 4-byte aligned", what);
    }
    if (n_elems == 0) {
        // the amax of an empty tensor is 0; a given amax is passed through
        for (int i = 0; i < n; ++i) {
            float* aout = amax_out ? amax_out[i] : nullptr;
            const float* ain = amax_in ? amax_in[i] : nullptr;
            if (aout == nullptr)
                continue;
            cudaError_t e = ain ? cudaMemcpyAsync(aout, ain, 4, cudaMemcpyDeviceToDevice, s) : cudaMemsetAsync(aout, 0, 4, s);
            if (e != cudaSuccess)
                return fail(KVQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
        }
        return ok();
    }
    const uint64_t n_blocks = static_cast<uint64_t>(n_elems) / kBlock;
    for (int base = 0; base < n; base += kMaxBatch) {
        const int m = n - base < kMaxBatch ? n - base : kMaxBatch;
        QuantBatch qb{};
        qb.n_blocks = n_blocks;
        for (int i = 0; i < m; ++i) {
            const int j = base + i;
            const float* ain = amax_in ? amax_in[j] : nullptr;
            float* aout = amax_out ? amax_out[j] : nullptr;
            qb.t[i].x = xs[j];
            qb.t[i].packed = mode != kYOnly ? packed[j] : nullptr;
            qb.t[i].scales = mode != kYOnly ? scales[j] : nullptr;
            qb.t[i].amax = ain ? ain : aout;
            qb.t[i].amax_copy = (ain && aout && aout != ain) ? aout : nullptr;
            qb.t[i].y = mode != kCodes ? ys[j] : nullptr;
        }
        if ((st = run_quantize(qb, m, amax_in == nullptr, rule, s, mode)) != KVQ_OK)
            return st;
    }
    return ok();
}

kvq_status dequantize_impl(const uint8_t* const* packed, const uint8_t* const* scales, const float* const* amax,
                           int32_t n, int64_t n_elems, int32_t head_dim, void* const* ys, cudaStream_t s)
{
    kvq_status st;
    if ((st = check_shape(n_elems, head_dim)) != KVQ_OK)
        return st;
    if (n < 0)
        return fail(KVQ_ERR_INVALID_ARG, "kvq_dequantize: negative tensor count");
    if (n == 0 || n_elems == 0)
        return ok();
    if (packed == nullptr || scales == nullptr || amax == nullptr || ys == nullptr)
        return fail(KVQ_ERR_INVALID_ARG, "kvq_dequantize: null host array");
    for (int i = 0; i < n; ++i) {
        if (packed[i] == nullptr || scales[i] == nullptr || amax[i] == nullptr || ys[i] == nullptr)
            return fail(KVQ_ERR_INVALID_ARG, "kvq_dequantize: null pointer");
        if (!aligned(ys[i], 32) || !aligned(packed[i], 8) || !aligned(amax[i], 4))
            return fail(KVQ_ERR_MISALIGNED, "kvq_dequantize: y must be 32-byte, packed 8-byte, amax 4-byte aligned");
    }
    for (int base = 0; base < n; base += kMaxBatch) {
        const int m = n - base < kMaxBatch ? n - base : kMaxBatch;
        DequantBatch db{};
        db.blk_lo = 0;
        db.blk_hi = static_cast<uint64_t>(n_elems) / kBlock;
        db.blocks_per_chunk = db.blk_hi;  // one chunk: the tensor
        for (int i = 0; i < m; ++i) {
            db.t[i].packed = packed[base + i];
            db.t[i].scales = scales[base + i];
            db.t[i].amax = amax[base + i];
            db.t[i].y = ys[base + i];
        }
        if ((st = run_dequantize(db, m, s)) != KVQ_OK)
            return st;
    }
    return ok();
}

}  // namespace kvq

using namespace kvq;

extern "C" {

kvq_status kvq_quantize(const void* x, int64_t n_elems, int32_t head_dim, kvq_scale_rule rule,
                        const float* amax_in, float* amax_out, uint8_t* packed, uint8_t* scales,
                        kvq_stream_t stream)
{
    NvtxRange nvtx_range("kvq_quantize");
    return quantize_impl("kvq_quantize", &x, 1, n_elems, head_dim, rule, amax_in ? &amax_in : nullptr,
                         amax_out ? &amax_out : nullptr, &packed, &scales, nullptr, kCodes,
                         reinterpret_cast<cudaStream_t>(stream));
}

kvq_status kvq_quantize_batch(const void* const* xs, int32_t n_tensors, int64_t n_elems, int32_t head_dim,
                              kvq_scale_rule rule, const float* const* amax_in, float* const* amax_out,
                              uint8_t* const* packed, uint8_t* const* scales, kvq_stream_t stream)
{
    NvtxRange nvtx_range("kvq_quantize_batch");
    return quantize_impl("kvq_quantize_batch", xs, n_tensors, n_elems, head_dim, rule, amax_in, amax_out, packed,
                         scales, nullptr, kCodes, reinterpret_cast<cudaStream_t>(stream));
}

kvq_status kvq_quantize_dequantize(const void* x, int64_t n_elems, int32_t head_dim, kvq_scale_rule rule,
                                   const float* amax_in, float* amax_out, uint8_t* packed, uint8_t* scales,
                                   void* y, kvq_stream_t stream)
{
    NvtxRange nvtx_range("kvq_quantize_dequantize");
    if ((packed == nullptr) != (scales == nullptr))
        return fail(KVQ_ERR_INVALID_ARG, "kvq_quantize_dequantize: packed and scales must be both given or both null");
    const int mode = packed ? kCodesAndY : kYOnly;
    return quantize_impl("kvq_quantize_dequantize", &x, 1, n_elems, head_dim, rule, amax_in ? &amax_in : nullptr,
                         amax_out ? &amax_out : nullptr, &packed, &scales, &y, mode,
                         reinterpret_cast<cudaStream_t>(stream));
}

kvq_status kvq_dequantize_batch(const uint8_t* const* packed, const uint8_t* const* scales, const float* const* amax,
                                int32_t n_tensors, int64_t n_elems, int32_t head_dim, void* const* ys,
                                kvq_stream_t stream)
{
    NvtxRange nvtx_range("kvq_dequantize_batch");
    return dequantize_impl(packed, scales, amax, n_tensors, n_elems, head_dim, ys,
                           reinterpret_cast<cudaStream_t>(stream));
}

kvq_status kvq_dequantize(const uint8_t* packed, const uint8_t* scales, const float* amax, int64_t n_elems,
                          int32_t head_dim, void* y, kvq_stream_t stream)
{
    NvtxRange nvtx_range("kvq_dequantize");
    return dequantize_impl(&packed, &scales, &amax, 1, n_elems, head_dim, &y, reinterpret_cast<cudaStream_t>(stream));
}

kvq_status kvq_append_batch(const kvq_cache* caches, const int64_t* row_offsets, const void* const* xs,
                            int32_t n_tensors, int64_t n_rows, kvq_scale_rule rule, kvq_stream_t stream)
{
    NvtxRange nvtx_range("kvq_append_batch");
    kvq_status st;
    if ((st = check_rule(rule)) != KVQ_OK)
        return st;
    if (n_tensors < 0 || n_rows < 0)
        return fail(KVQ_ERR_INVALID_ARG, "kvq_append_batch: negative count");
    if (n_tensors == 0)
        return ok();
    if (caches == nullptr || row_offsets == nullptr || xs == nullptr)
        return fail(KVQ_ERR_INVALID_ARG, "kvq_append_batch: null host array");
    const int32_t D = caches[0].head_dim;
    for (int i = 0; i < n_tensors; ++i) {
        const kvq_cache* c = &caches[i];
        if ((st = check_cache(c, "kvq_append")) != KVQ_OK)
            return st;
        if (c->head_dim != D)
            return fail(KVQ_ERR_INVALID_ARG, "kvq_append_batch: head_dim differs between tensors");
        const int64_t off = row_offsets[i];
        if (off < 0 || off % c->rows_per_chunk != 0)
            return fail(KVQ_ERR_INVALID_ARG, "kvq_append: row_offset %lld is not a non-negative multiple of "
                        "rows_per_chunk %lld", static_cast<long long>(off), static_cast<long long>(c->rows_per_chunk));
        if (n_rows > c->rows_per_chunk)
            return fail(KVQ_ERR_INVALID_ARG, "kvq_append: n_rows %lld exceeds rows_per_chunk %lld",
                        static_cast<long long>(n_rows), static_cast<long long>(c->rows_per_chunk));
        if (off > c->capacity_rows - n_rows)
            return fail(KVQ_ERR_CAPACITY, "kvq_append: rows [%lld, %lld) past capacity %lld",
                        static_cast<long long>(off), static_cast<long long>(off + n_rows),
                        static_cast<long long>(c->capacity_rows));
        if (n_rows > 0 && xs[i] == nullptr)
            return fail(KVQ_ERR_INVALID_ARG, "kvq_append: null x");
        if (!aligned(xs[i], 32))
            return fail(KVQ_ERR_MISALIGNED, "kvq_append: x must be 32-byte aligned");
    }
    if (n_rows == 0)
        return ok();
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const uint64_t n_blocks = static_cast<uint64_t>(n_rows) * static_cast<uint64_t>(D / kBlock);
    for (int base = 0; base < n_tensors; base += kMaxBatch) {
        const int n = n_tensors - base < kMaxBatch ? n_tensors - base : kMaxBatch;
        QuantBatch qb{};
        qb.n_blocks = n_blocks;
        for (int i = 0; i < n; ++i) {
            const kvq_cache* c = &caches[base + i];
            const int64_t off = row_offsets[base + i];
            const uint64_t e0 = static_cast<uint64_t>(off) * static_cast<uint64_t>(D);
            qb.t[i].x = xs[base + i];
            qb.t[i].packed = c->packed + e0 / 2;
            qb.t[i].scales = c->scales + e0 / kBlock;
            qb.t[i].amax = c->amax + off / c->rows_per_chunk;
            qb.t[i].amax_copy = nullptr;
        }
        if ((st = run_quantize(qb, n, true, rule, s)) != KVQ_OK)
            return st;
    }
    return ok();
}

kvq_status kvq_append(const kvq_cache* cache, int64_t row_offset, const void* x, int64_t n_rows,
                      kvq_scale_rule rule, kvq_stream_t stream)
{
    NvtxRange nvtx_range("kvq_append");
    return kvq_append_batch(cache, &row_offset, &x, 1, n_rows, rule, stream);
}

kvq_status kvq_dequantize_cache_batch(const kvq_cache* caches, void* const* ys, int32_t n_tensors,
                                      int64_t row_begin, int64_t row_end, kvq_stream_t stream)
{
    NvtxRange nvtx_range("kvq_dequantize_cache_batch");
    kvq_status st;
    if (n_tensors < 0)
        return fail(KVQ_ERR_INVALID_ARG, "kvq_dequantize_cache_batch: negative count");
    if (n_tensors == 0)
        return ok();
    if (caches == nullptr || ys == nullptr)
        return fail(KVQ_ERR_INVALID_ARG, "kvq_dequantize_cache_batch: null host array");
    if (row_begin < 0 || row_end < row_begin)
        return fail(KVQ_ERR_INVALID_ARG, "kvq_dequantize_cache: bad row range [%lld, %lld)",
                    static_cast<long long>(row_begin), static_cast<long long>(row_end));
    const int32_t D = caches[0].head_dim;
    const int64_t rpc = caches[0].rows_per_chunk;
    for (int i = 0; i < n_tensors; ++i) {
        const kvq_cache* c = &caches[i];
        if ((st = check_cache(c, "kvq_dequantize_cache")) != KVQ_OK)
            return st;
        if (c->head_dim != D || c->rows_per_chunk != rpc)
            return fail(KVQ_ERR_INVALID_ARG, "kvq_dequantize_cache_batch: head_dim / rows_per_chunk differ");
        if (row_end > c->capacity_rows)
            return fail(KVQ_ERR_CAPACITY, "kvq_dequantize_cache: row_end %lld past capacity %lld",
                        static_cast<long long>(row_end), static_cast<long long>(c->capacity_rows));
        if (row_end > row_begin && ys[i] == nullptr)
            return fail(KVQ_ERR_INVALID_ARG, "kvq_dequantize_cache: null y");
        if (!aligned(ys[i], 32))
            return fail(KVQ_ERR_MISALIGNED, "kvq_dequantize_cache: y must be 32-byte aligned");
    }
    if (row_end == row_begin)
        return ok();
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const uint64_t bpr = static_cast<uint64_t>(D / kBlock);
    for (int base = 0; base < n_tensors; base += kMaxBatch) {
        const int n = n_tensors - base < kMaxBatch ? n_tensors - base : kMaxBatch;
        DequantBatch db{};
        db.blk_lo = static_cast<uint64_t>(row_begin) * bpr;
        db.blk_hi = static_cast<uint64_t>(row_end) * bpr;
        db.blocks_per_chunk = static_cast<uint64_t>(rpc) * bpr;
        for (int i = 0; i < n; ++i) {
            const kvq_cache* c = &caches[base + i];
            db.t[i].packed = c->packed;
            db.t[i].scales = c->scales;
            db.t[i].amax = c->amax;
            db.t[i].y = ys[base + i];
        }
        if ((st = run_dequantize(db, n, s)) != KVQ_OK)
            return st;
    }
    return ok();
}

kvq_status kvq_dequantize_cache(const kvq_cache* cache, int64_t row_begin, int64_t row_end, void* y,
                                kvq_stream_t stream)
{
    NvtxRange nvtx_range("kvq_dequantize_cache");
    return kvq_dequantize_cache_batch(cache, &y, 1, row_begin, row_end, stream);
}

kvq_status kvq_cache_bytes(int32_t layers, int32_t heads, int64_t capacity_tokens, int32_t head_dim,
                           int64_t tokens_per_chunk, uint64_t* packed_bytes, uint64_t* scale_bytes,
                           uint64_t* amax_bytes)
{
    NvtxRange nvtx_range("kvq_cache_bytes");
    if (layers <= 0 || heads <= 0 || capacity_tokens < 0 || head_dim <= 0 || head_dim % kBlock != 0 ||
        tokens_per_chunk <= 0)
        return fail(KVQ_ERR_INVALID_ARG, "kvq_cache_bytes: bad dimensions");
    const uint64_t tensors = 2ull * static_cast<uint64_t>(layers);
    const uint64_t elems = static_cast<uint64_t>(capacity_tokens) * static_cast<uint64_t>(heads) *
                           static_cast<uint64_t>(head_dim);
    const uint64_t chunks = (static_cast<uint64_t>(capacity_tokens) + static_cast<uint64_t>(tokens_per_chunk) - 1) /
                            static_cast<uint64_t>(tokens_per_chunk);
    if (packed_bytes)
        *packed_bytes = tensors * (elems / 2);
    if (scale_bytes)
        *scale_bytes = tensors * (elems / kBlock);
    if (amax_bytes)
        *amax_bytes = tensors * chunks * sizeof(float);
    return ok();
}

const char* kvq_status_string(kvq_status status)
{
    switch (status) {
    case KVQ_OK: return "KVQ_OK";
    case KVQ_ERR_INVALID_ARG: return "KVQ_ERR_INVALID_ARG";
    case KVQ_ERR_MISALIGNED: return "KVQ_ERR_MISALIGNED";
    case KVQ_ERR_UNSUPPORTED: return "KVQ_ERR_UNSUPPORTED";
    case KVQ_ERR_CAPACITY: return "KVQ_ERR_CAPACITY";
    case KVQ_ERR_CUDA: return "KVQ_ERR_CUDA";
    case KVQ_ERR_TIMEOUT: return "KVQ_ERR_TIMEOUT";
    }
    return "KVQ_ERR_UNKNOWN";
}

const char* kvq_last_error(void) { return g_last_error; }

kvq_status kvq_quantize_launches(int32_t n_tensors, int64_t n_elems, int32_t head_dim, int32_t amax_given,
                                 int32_t* launches)
{
    kvq_status st;
    if ((st = check_shape(n_elems, head_dim)) != KVQ_OK)
        return st;
    if (n_tensors < 0 || launches == nullptr)
        return fail(KVQ_ERR_INVALID_ARG, "kvq_quantize_launches: negative tensor count or null output");
    const uint64_t n_blocks = static_cast<uint64_t>(n_elems) / kBlock;
    // groups of kMaxBatch tensors and a last, smaller one, each planned on its own
    auto per_group = [&](int32_t k) {
        FusedBatch fb;
        return k == 0 || n_blocks == 0 ? 0 : amax_given ? 1 : plan_fused(n_blocks, k, fb) ? 2 : 3;
    };
    *launches = n_tensors / kMaxBatch * per_group(kMaxBatch) + per_group(n_tensors % kMaxBatch);
    return ok();
}

kvq_status kvq_device_status(int32_t clear)
{
    NvtxRange nvtx_range("kvq_device_status");
    unsigned int word = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&word, g_device_error, sizeof(word));
    if (e == cudaSuccess && clear && word != 0) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero));
    }
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(KVQ_ERR_CUDA, "kvq_device_status: %s", cudaGetErrorString(e));
    }
    if (word & kDeviceErrWaitTimeout)
        return fail(KVQ_ERR_TIMEOUT, "a kernel's bounded wait for the amax of its tensor gave up");
    return ok();
}

void kvq_testing_set_fused_wait(uint32_t extra_a_tiles, uint64_t wait_ns)
{
    g_test_extra_a = extra_a_tiles;
    g_test_wait_ns = wait_ns;
}

const char* kvq_version(void) { return "0.1.0"; }

}  // extern "C"
