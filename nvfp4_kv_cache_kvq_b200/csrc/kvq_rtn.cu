// kvq_rtn.cu -- symmetric blockwise round-to-nearest integer KV codecs (INT4, INT2),
// the RTN_INT4 / RTN_INT2 / RTN_K2_V4 rows of "KV Cache Quantization for Self-Forcing
// Video Generation: A 33-Method Empirical Study", appendix Table 3 (symmetric blockwise
// quantization of K and V, block size 16, packed storage plus per-block scales).
//
// Per block of 16 elements, with qmax = 2^(bits-1) - 1 (7 or 1):
//     S   = bf16_rne(amax_b / qmax)                         (the stored 16-bit scale)
//     q_i = round_half_even(x_i / S), in [-qmax, qmax]       (q = 0 when S == 0)
//     y_i = bf16_rne(q_i * S)
// Codes are two's complement: INT4 two per byte (even element in the low nibble), INT2
// four per byte (element 4j + k in bits 2k..2k+1). The declarations in include/kvq.h
// state the layout and the arguments.
//
// Kernels: two 16-element blocks per thread (one when the buffers are not aligned for
// the wider code and scale accesses), one 256-bit load or store per block, CTA-contiguous
// tiles, batches of tensors, programmatic dependent launch -- the same skeleton as the
// NVFP4 kernels.
#include <cuda_runtime.h>

#include <cstdint>

#include "kvq.h"
#include "kvq_common.h"
#include "kvq_device.cuh"

namespace kvq {
namespace {

struct RtnTensor {
    const void* x;     // bf16 in (quantize) / out (dequantize)
    uint8_t* packed;   // codes
    uint16_t* scales;  // bf16 scale per block
};

struct RtnBatch {
    RtnTensor t[kMaxBatch];
    uint64_t n_blocks;  // blocks per tensor
};

// Exact IEEE quotients without a division (Markstein's correction step, as in kvq.cu):
// q = RN(a*y), r = fma(-q, b, a), RN(q + r*y) with y = RN(1/b). For a/7 it is exact for
// every bf16 a (checked exhaustively); for x/S with a bf16 scale S >= 2^-100 the
// quotients round to the same levels as IEEE division (checked over all bf16 S and
// 4096 x per S). Smaller scales use IEEE division.
__device__ __forceinline__ float markstein(float a, float b, float y)
{
    const float q = __fmul_rn(a, y);
    return __fmaf_rn(__fmaf_rn(-q, b, a), y, q);
}

// Round to the nearest integer, ties to even, for |t| < 2^22: adding 1.5 * 2^23 leaves
// the integer in the low mantissa bits (two's complement relative to 0x4B400000), so the
// low `bits` bits are already the packed code. Checked against nearbyint for every fp32
// in [-8, 8].
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23

template <int BITS>
__device__ __forceinline__ uint32_t rtn_code(float t)
{
    return __float_as_uint(__fadd_rn(t, kRoundMagic)) & ((1u << BITS) - 1u);
}

// One block: 16 bf16 in w -> codes (BITS * 2 bytes, in cw[0..BITS/2)) and the bf16 scale.
template <int BITS>
__device__ __forceinline__ uint32_t rtn_quantize_block(const uint32_t (&w)[8], uint32_t (&cw)[2])
{
    constexpr float kQmax = static_cast<float>((1 << (BITS - 1)) - 1);
    const float amax_b = __uint_as_float(block_absmax_bits(w) << 16);
    // amax_b / 7 by the corrected product with RN(1/7); amax_b / 1 is exact
    const float s = BITS == 4 ? markstein(amax_b, 7.0f, __int_as_float(0x3E124925)) : amax_b;
    uint16_t sb;
    asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(sb) : "f"(s));
    const float S = __uint_as_float(static_cast<uint32_t>(sb) << 16);
    cw[0] = cw[1] = 0u;
    if (S == 0.0f)
        return sb;
    float t[16];
    if (S >= 0x1p-100f) {
        // |x / S| <= qmax * (1 + 2^-8) < qmax + 1/2 for a normal S, so no level is clamped
        const float y = __frcp_rn(S);
        const uint64_t y2 = f32x2_pack(y, y), nS2 = f32x2_pack(-S, -S);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint64_t xp = f32x2_pack(bf16lo_to_f32(w[j]), bf16hi_to_f32(w[j]));
            const uint64_t q = f32x2_mul(xp, y2);
            const uint64_t r = f32x2_fma(q, nS2, xp);
            f32x2_unpack(f32x2_fma(r, y2, q), t[2 * j], t[2 * j + 1]);
        }
    } else {
        // tiny (subnormal) scales: IEEE division and the clamp the definition states
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            t[2 * j] = fminf(fmaxf(__fdiv_rn(bf16lo_to_f32(w[j]), S), -kQmax), kQmax);
            t[2 * j + 1] = fminf(fmaxf(__fdiv_rn(bf16hi_to_f32(w[j]), S), -kQmax), kQmax);
        }
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        constexpr int per_word = 32 / BITS;
        cw[i / per_word] |= rtn_code<BITS>(t[i]) << (BITS * (i % per_word));
    }
    return sb;
}

// Codes (BITS * 2 bytes) and bf16 scale bits -> 16 bf16 in y.
template <int BITS>
__device__ __forceinline__ void rtn_dequantize_block(const uint32_t (&cw)[2], uint32_t sb, uint32_t (&y)[8])
{
    constexpr int per_word = 32 / BITS;
    constexpr uint32_t kMask = (1u << BITS) - 1u, kSign = 1u << (BITS - 1);
    const float S = __uint_as_float(sb << 16);
    const uint64_t S2 = f32x2_pack(S, S);
    const uint64_t magic2 = f32x2_pack(-kRoundMagic, -kRoundMagic);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        float v[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int i = 2 * j + h;
            const uint32_t c = (cw[i / per_word] >> (BITS * (i % per_word))) & kMask;
            // 0x4B400000 + q, q the sign-extended code: the float 1.5 * 2^23 + q
            v[h] = __uint_as_float((0x4B400000u - kSign) + (c ^ kSign));
        }
        // (1.5*2^23 + q) - 1.5*2^23 = q exactly; q * S is exact in fp32, rounded to bf16
        const uint64_t q2 = f32x2_fma(f32x2_pack(1.0f, 1.0f), f32x2_pack(v[0], v[1]), magic2);
        float lo, hi;
        f32x2_unpack(f32x2_mul(q2, S2), lo, hi);
        y[j] = bf16x2_from_f32(hi, lo);
    }
}

// BPT blocks per thread (1 or 2). With 2, a thread moves 2 * BITS * 2 bytes of codes and
// 4 bytes of scales in one access each, which needs codes aligned to 4 * BITS bytes and
// scales to 4 bytes (the host picks BPT = 1 otherwise); an odd last block is handled on
// its own.
template <int BITS, int BPT>
__global__ void __launch_bounds__(kThreads) rtn_quantize_kernel(const RtnBatch B)
{
    pdl_begin();
    const RtnTensor& T = B.t[blockIdx.y];
    const uint64_t b = (static_cast<uint64_t>(blockIdx.x) * kThreads + threadIdx.x) * BPT;
    if (b >= B.n_blocks)
        return;
    const char* x = static_cast<const char*>(T.x);
    uint32_t w[8], cw[2], cw1[2];
    ld_nc_v8(x + b * 32, w);
    const uint32_t sb = rtn_quantize_block<BITS>(w, cw);
    if (BPT == 2 && b + 1 < B.n_blocks) {
        ld_nc_v8(x + b * 32 + 32, w);
        const uint32_t sb1 = rtn_quantize_block<BITS>(w, cw1);
        if (BITS == 4)
            st_v4(T.packed + b * 8, cw[0], cw[1], cw1[0], cw1[1]);
        else
            st_v2(T.packed + b * 4, cw[0], cw1[0]);
        *reinterpret_cast<uint32_t*>(T.scales + b) = sb | (sb1 << 16);
        return;
    }
    if (BITS == 4)
        st_v2(T.packed + b * 8, cw[0], cw[1]);
    else
        *reinterpret_cast<uint32_t*>(T.packed + b * 4) = cw[0];
    T.scales[b] = static_cast<uint16_t>(sb);
}

template <int BITS, int BPT>
__global__ void __launch_bounds__(kThreads) rtn_dequantize_kernel(const RtnBatch B)
{
    pdl_begin();
    const RtnTensor& T = B.t[blockIdx.y];
    const uint64_t b = (static_cast<uint64_t>(blockIdx.x) * kThreads + threadIdx.x) * BPT;
    if (b >= B.n_blocks)
        return;
    char* y = static_cast<char*>(const_cast<void*>(T.x));
    uint32_t cw[2] = {0u, 0u}, out[8];
    if (BPT == 2 && b + 1 < B.n_blocks) {
        uint32_t cw1[2] = {0u, 0u};
        if (BITS == 4) {
            const uint4 q = ld_nc_v4(T.packed + b * 8);
            cw[0] = q.x;
            cw[1] = q.y;
            cw1[0] = q.z;
            cw1[1] = q.w;
        } else {
            const uint2 q = ld_nc_v2(T.packed + b * 4);
            cw[0] = q.x;
            cw1[0] = q.y;
        }
        const uint32_t s2 = __ldg(reinterpret_cast<const uint32_t*>(T.scales + b));
        rtn_dequantize_block<BITS>(cw, s2 & 0xFFFFu, out);
        st_v8(y + b * 32, out);
        rtn_dequantize_block<BITS>(cw1, s2 >> 16, out);
        st_v8(y + b * 32 + 32, out);
        return;
    }
    if (BITS == 4) {
        const uint2 q = ld_nc_v2(T.packed + b * 8);
        cw[0] = q.x;
        cw[1] = q.y;
    } else {
        cw[0] = __ldg(reinterpret_cast<const uint32_t*>(T.packed + b * 4));
    }
    rtn_dequantize_block<BITS>(cw, __ldg(T.scales + b), out);
    st_v8(y + b * 32, out);
}

template <int BITS, int BPT>
cudaError_t launch_rtn(bool quantize, uint64_t n_blocks, int m, const RtnBatch& rb, cudaStream_t s)
{
    const dim3 grid(tiles((n_blocks + BPT - 1) / BPT), m);
    return quantize ? launch(rtn_quantize_kernel<BITS, BPT>, grid, kThreads, s, rb)
                    : launch(rtn_dequantize_kernel<BITS, BPT>, grid, kThreads, s, rb);
}

kvq_status rtn_impl(bool quantize, const void* const* xs, uint8_t* const* packed, uint16_t* const* scales,
                    int32_t n, int64_t n_elems, int32_t head_dim, int32_t bits, cudaStream_t s)
{
    const char* what = quantize ? "kvq_rtn_quantize" : "kvq_rtn_dequantize";
    kvq_status st;
    if ((st = check_shape(n_elems, head_dim)) != KVQ_OK)
        return st;
    if (bits != 2 && bits != 4)
        return fail(KVQ_ERR_INVALID_ARG, "%s: bits %d is not 2 or 4", what, bits);
    if (n < 0)
        return fail(KVQ_ERR_INVALID_ARG, "%s: negative tensor count", what);
    if (n == 0 || n_elems == 0)
        return ok();
    if (xs == nullptr || packed == nullptr || scales == nullptr)
        return fail(KVQ_ERR_INVALID_ARG, "%s: null host array", what);
    for (int i = 0; i < n; ++i) {
        if (xs[i] == nullptr || packed[i] == nullptr || scales[i] == nullptr)
            return fail(KVQ_ERR_INVALID_ARG, "%s: null pointer", what);
        if (!aligned(xs[i], 32) || !aligned(packed[i], 2 * bits) || !aligned(scales[i], 2))
            return fail(KVQ_ERR_MISALIGNED, "%s: bf16 tensor 32-byte, codes %d-byte, scales 2-byte aligned", what,
                        2 * bits);
    }
    const uint64_t n_blocks = static_cast<uint64_t>(n_elems) / kBlock;
    // two blocks per thread when every buffer allows the wider accesses
    bool wide = true;
    for (int i = 0; i < n; ++i)
        wide = wide && aligned(packed[i], 4 * bits) && aligned(scales[i], 4);
    for (int base = 0; base < n; base += kMaxBatch) {
        const int m = n - base < kMaxBatch ? n - base : kMaxBatch;
        RtnBatch rb{};
        rb.n_blocks = n_blocks;
        for (int i = 0; i < m; ++i)
            rb.t[i] = RtnTensor{xs[base + i], packed[base + i], scales[base + i]};
        cudaError_t e;
        if (bits == 4)
            e = wide ? launch_rtn<4, 2>(quantize, n_blocks, m, rb, s) : launch_rtn<4, 1>(quantize, n_blocks, m, rb, s);
        else
            e = wide ? launch_rtn<2, 2>(quantize, n_blocks, m, rb, s) : launch_rtn<2, 1>(quantize, n_blocks, m, rb, s);
        if ((st = launched(e, what)) != KVQ_OK)
            return st;
    }
    return ok();
}

}  // namespace
}  // namespace kvq

using namespace kvq;

extern "C" {

kvq_status kvq_rtn_quantize(const void* x, int64_t n_elems, int32_t head_dim, int32_t bits, uint8_t* packed,
                            uint16_t* scales, kvq_stream_t stream)
{
    NvtxRange nvtx_range("kvq_rtn_quantize");
    return rtn_impl(true, &x, &packed, &scales, 1, n_elems, head_dim, bits, reinterpret_cast<cudaStream_t>(stream));
}

kvq_status kvq_rtn_dequantize(const uint8_t* packed, const uint16_t* scales, int64_t n_elems, int32_t head_dim,
                              int32_t bits, void* y, kvq_stream_t stream)
{
    NvtxRange nvtx_range("kvq_rtn_dequantize");
    const void* yy = y;
    uint8_t* p = const_cast<uint8_t*>(packed);
    uint16_t* sc = const_cast<uint16_t*>(scales);
    return rtn_impl(false, &yy, &p, &sc, 1, n_elems, head_dim, bits, reinterpret_cast<cudaStream_t>(stream));
}

kvq_status kvq_rtn_quantize_batch(const void* const* xs, int32_t n_tensors, int64_t n_elems, int32_t head_dim,
                                  int32_t bits, uint8_t* const* packed, uint16_t* const* scales,
                                  kvq_stream_t stream)
{
    NvtxRange nvtx_range("kvq_rtn_quantize_batch");
    return rtn_impl(true, xs, packed, scales, n_tensors, n_elems, head_dim, bits,
                    reinterpret_cast<cudaStream_t>(stream));
}

kvq_status kvq_rtn_dequantize_batch(const uint8_t* const* packed, const uint16_t* const* scales, int32_t n_tensors,
                                    int64_t n_elems, int32_t head_dim, int32_t bits, void* const* ys,
                                    kvq_stream_t stream)
{
    NvtxRange nvtx_range("kvq_rtn_dequantize_batch");
    return rtn_impl(false, const_cast<const void* const*>(ys), const_cast<uint8_t* const*>(packed),
                    const_cast<uint16_t* const*>(scales), n_tensors, n_elems, head_dim, bits,
                    reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
