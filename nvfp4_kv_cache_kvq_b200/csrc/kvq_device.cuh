// kvq_device.cuh -- sm_100a device helpers for the NVFP4 KV-cache kernels: 256-bit
// streaming loads/stores and the hardware FP4 (e2m1) / FP8 (e4m3) / bf16 conversions,
// issued as inline PTX.
//
// Packed conversions put their FIRST source operand in the UPPER half (nibble, byte or
// 16-bit lane) of the result, so the even element of a pair is passed second: it lands
// in the low nibble, as the format stores it.
#pragma once

#include <cstdint>

namespace kvq {

// Programmatic dependent launch (sm_90+). Every kernel of the library starts with
// pdl_begin(): it waits until the grid launched before it on the stream has completed and
// its writes are visible (a no-op when the launch carried no programmatic dependency),
// then lets the next grid be scheduled. The next grid's launch latency thus overlaps this
// grid's tail, while its own pdl_begin() still orders every memory access after ours.
__device__ __forceinline__ void pdl_begin()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// 32 bytes (one 16-element bf16 block) from read-only global memory, not kept in L1.
__device__ __forceinline__ void ld_nc_v8(const void* p, uint32_t (&w)[8])
{
    asm("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
        : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7])
        : "l"(p));
}

__device__ __forceinline__ void st_v8(void* p, const uint32_t (&w)[8])
{
    asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(w[0]), "r"(w[1]), "r"(w[2]),
                 "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
                 : "memory");
}

__device__ __forceinline__ uint2 ld_nc_v2(const void* p)
{
    uint2 v;
    asm("ld.global.nc.L1::no_allocate.v2.b32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}

__device__ __forceinline__ uint4 ld_nc_v4(const void* p)
{
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(p));
    return v;
}

__device__ __forceinline__ void st_v2(void* p, uint32_t a, uint32_t b)
{
    asm volatile("st.global.v2.b32 [%0], {%1,%2};" ::"l"(p), "r"(a), "r"(b) : "memory");
}

__device__ __forceinline__ void st_v4(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    asm volatile("st.global.v4.b32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// Lane-wise max(|a|, |b|) of two bf16x2 words (the sign bit of each lane is the xor of
// the operands' signs and is cleared by the caller).
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// |x| max of the 16 bf16 values of a block, as the bf16 bit pattern (sign cleared). For
// finite values the integer order of |bf16| bit patterns is their numeric order.
__device__ __forceinline__ uint32_t block_absmax_bits(const uint32_t (&w)[8])
{
    const uint32_t m = absmax_bf16x2(absmax_bf16x2(absmax_bf16x2(w[0], w[1]), absmax_bf16x2(w[2], w[3])),
                                     absmax_bf16x2(absmax_bf16x2(w[4], w[5]), absmax_bf16x2(w[6], w[7])))
                       & 0x7FFF7FFFu;
    return max(m & 0xFFFFu, m >> 16);
}

// |x| max of eight bf16 values (a 16-byte vector), as the bf16 bit pattern (sign cleared).
__device__ __forceinline__ uint32_t block_absmax_bits4(const uint4& v)
{
    const uint32_t m = absmax_bf16x2(absmax_bf16x2(v.x, v.y), absmax_bf16x2(v.z, v.w)) & 0x7FFF7FFFu;
    return max(m & 0xFFFFu, m >> 16);
}

// Packed fp32 pairs (sm_100 f32x2 arithmetic): the low 32 bits hold the first value.
__device__ __forceinline__ uint64_t f32x2_pack(float lo, float hi)
{
    uint64_t d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
    return d;
}

__device__ __forceinline__ void f32x2_unpack(uint64_t v, float& lo, float& hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

// Lane-wise a * b, rounded to nearest even.
__device__ __forceinline__ uint64_t f32x2_mul(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// Lane-wise fused a * b + c, one rounding to nearest even.
__device__ __forceinline__ uint64_t f32x2_fma(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ float bf16lo_to_f32(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Two fp32 -> two e4m3 codes (round to nearest even, saturating at 448):
// lo -> bits 0..7, hi -> bits 8..15.
__device__ __forceinline__ uint32_t e4m3x2_from_f32(float hi, float lo)
{
    uint16_t d;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
    return d;
}

// Two e4m3 codes (bits 0..7 and 8..15) -> their exact values.
__device__ __forceinline__ void e4m3x2_to_f32(uint32_t codes, float& lo, float& hi)
{
    uint16_t c = static_cast<uint16_t>(codes);
    asm("{\n\t.reg .b32 h;\n\t.reg .b16 l16, h16;\n\t"
        "cvt.rn.f16x2.e4m3x2 h, %2;\n\t"
        "mov.b32 {l16, h16}, h;\n\t"
        "cvt.f32.f16 %0, l16;\n\t"
        "cvt.f32.f16 %1, h16;\n\t}"
        : "=f"(lo), "=f"(hi)
        : "h"(c));
}

// Eight fp32 -> eight e2m1 codes (round to nearest even, saturating at 6, sign kept)
// packed in one word: element j in nibble j.
__device__ __forceinline__ uint32_t e2m1x8_from_f32(const float (&v)[8])
{
    uint32_t d;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(d)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return d;
}

// Eight fp32 -> eight e2m1 codes packed in one word (as e2m1x8_from_f32), and the exact
// values of those codes, decoded straight from each pair's byte register.
__device__ __forceinline__ uint32_t e2m1x8_encode_decode(const float (&v)[8], float (&val)[8])
{
    uint32_t d;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t.reg .b32 h0, h1, h2, h3;\n\t"
        ".reg .b16 l0, u0, l1, u1, l2, u2, l3, u3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %10, %9;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %12, %11;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %14, %13;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %16, %15;\n\t"
        "cvt.rn.f16x2.e2m1x2 h0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 h1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 h2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 h3, b3;\n\t"
        "mov.b32 {l0, u0}, h0;\n\t"
        "mov.b32 {l1, u1}, h1;\n\t"
        "mov.b32 {l2, u2}, h2;\n\t"
        "mov.b32 {l3, u3}, h3;\n\t"
        "cvt.f32.f16 %1, l0;\n\t"
        "cvt.f32.f16 %2, u0;\n\t"
        "cvt.f32.f16 %3, l1;\n\t"
        "cvt.f32.f16 %4, u1;\n\t"
        "cvt.f32.f16 %5, l2;\n\t"
        "cvt.f32.f16 %6, u2;\n\t"
        "cvt.f32.f16 %7, l3;\n\t"
        "cvt.f32.f16 %8, u3;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(d), "=f"(val[0]), "=f"(val[1]), "=f"(val[2]), "=f"(val[3]), "=f"(val[4]), "=f"(val[5]),
          "=f"(val[6]), "=f"(val[7])
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return d;
}

// One word of eight e2m1 codes -> their exact values (nibble j -> out[j]). Each byte is
// isolated with a shift and a truncating cvt. (Unpacking the word with a vector
// mov into four .b8 registers is NOT used: when the word had itself been packed from .b8
// registers in the same kernel, that unpack returned zeros for bytes 2 and 3 on sm_100a
// with CUDA 12.9; the shift form is exact in every case.)
__device__ __forceinline__ void e2m1x8_to_f32(uint32_t q, float (&out)[8])
{
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t.reg .b32 s1, s2, s3, h0, h1, h2, h3;\n\t"
        ".reg .b16 l0, u0, l1, u1, l2, u2, l3, u3;\n\t"
        "shr.b32 s1, %8, 8;\n\t"
        "shr.b32 s2, %8, 16;\n\t"
        "shr.b32 s3, %8, 24;\n\t"
        "cvt.u8.u32 b0, %8;\n\t"
        "cvt.u8.u32 b1, s1;\n\t"
        "cvt.u8.u32 b2, s2;\n\t"
        "cvt.u8.u32 b3, s3;\n\t"
        "cvt.rn.f16x2.e2m1x2 h0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 h1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 h2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 h3, b3;\n\t"
        "mov.b32 {l0, u0}, h0;\n\t"
        "mov.b32 {l1, u1}, h1;\n\t"
        "mov.b32 {l2, u2}, h2;\n\t"
        "mov.b32 {l3, u3}, h3;\n\t"
        "cvt.f32.f16 %0, l0;\n\t"
        "cvt.f32.f16 %1, u0;\n\t"
        "cvt.f32.f16 %2, l1;\n\t"
        "cvt.f32.f16 %3, u1;\n\t"
        "cvt.f32.f16 %4, l2;\n\t"
        "cvt.f32.f16 %5, u2;\n\t"
        "cvt.f32.f16 %6, l3;\n\t"
        "cvt.f32.f16 %7, u3;\n\t}"
        : "=f"(out[0]), "=f"(out[1]), "=f"(out[2]), "=f"(out[3]), "=f"(out[4]), "=f"(out[5]), "=f"(out[6]),
          "=f"(out[7])
        : "r"(q));
}

// Two fp32 -> bf16x2 (round to nearest even): lo -> bits 0..15, hi -> bits 16..31.
__device__ __forceinline__ uint32_t bf16x2_from_f32(float hi, float lo)
{
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

}  // namespace kvq

namespace kvq {

// ---- device-scope atomics and waits on one 32-bit word (relaxed: the word itself
// carries every value another CTA needs, so no other memory is ordered by them)

__device__ __forceinline__ uint32_t ld_relaxed_u32(const uint32_t* p)
{
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_relaxed_u32(uint32_t* p, uint32_t v)
{
    asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t atom_add_relaxed_u32(uint32_t* p, uint32_t v)
{
    uint32_t old;
    asm volatile("atom.relaxed.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

__device__ __forceinline__ void red_add_relaxed_u32(uint32_t* p, uint32_t v)
{
    asm volatile("red.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Lane-wise bf16 max on the two 16-bit halves of *p: the low half with +0, the high half
// with m (bf16 bits). No flush to zero, so a non-negative low half (any value up to
// 0x7F7F read as bf16) is left exactly as it was.
__device__ __forceinline__ void red_max_bf16_high(uint32_t* p, uint32_t m)
{
    const uint16_t lo = 0, hi = static_cast<uint16_t>(m);
    asm volatile("red.relaxed.gpu.global.v2.bf16.max.noftz [%0], {%1, %2};" ::"l"(p), "h"(lo), "h"(hi) : "memory");
}

__device__ __forceinline__ uint64_t globaltimer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

}  // namespace kvq

namespace kvq {

// ---- one-dimensional TMA bulk copy into this CTA's shared memory, completed on an mbarrier

__device__ __forceinline__ uint32_t smem_addr(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

// Order this thread's earlier generic-proxy accesses of shared memory before later
// async-proxy (TMA) accesses, and make an mbarrier init visible to the async proxy.
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// bytes (a multiple of 16, both addresses 16-byte aligned) from global src to shared dst;
// the mbarrier's current phase completes when they have landed.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar))
                 : "memory");
}

// Phase `parity` of the mbarrier is complete. try_wait lets the hardware suspend the
// thread for a while before it answers false, so a caller's wait loop issues few
// instructions.
__device__ __forceinline__ bool mbar_try_parity(uint64_t* bar, uint32_t parity)
{
    uint32_t done;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(done)
                 : "r"(smem_addr(bar)), "r"(parity)
                 : "memory");
    return done != 0;
}

}  // namespace kvq

namespace kvq {

// Named barrier `id` among `threads` threads (a multiple of 32) of the CTA.
__device__ __forceinline__ void named_barrier(uint32_t id, uint32_t threads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ uint32_t ld_volatile_smem(const uint32_t* p)
{
    uint32_t v;
    asm volatile("ld.volatile.shared.u32 %0, [%1];" : "=r"(v) : "r"(smem_addr(p)) : "memory");
    return v;
}

__device__ __forceinline__ void st_volatile_smem(uint32_t* p, uint32_t v)
{
    asm volatile("st.volatile.shared.u32 [%0], %1;" ::"r"(smem_addr(p)), "r"(v) : "memory");
}

}  // namespace kvq
