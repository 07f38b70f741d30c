// Device helpers shared by the quantizer and the fused decode kernel: fp16
// vector math of absmax row quantization and a bounded grid-wide barrier.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

#include "ptx.cuh"

namespace llmint8 {

// One bounded grid-wide barrier (all CTAs are co-resident: the kernel is
// launched cooperatively). sync[0] counts arrivals and sync[1] is the
// generation, read and written together as one 64-bit word (8-byte
// aligned), so that an arrival learns both in a single atomic round trip.
// The last arrival moves to the next generation and clears the count in
// one add; the others wait for the generation to change. *gen (if given)
// receives the generation this barrier opened. The arrival is a release
// and the wait an acquire at GPU scope, so writes that the calling thread
// made, or that its CTA made before a CTA barrier, are visible to every
// CTA after the barrier.
__device__ __forceinline__ bool grid_barrier(uint32_t *sync, uint32_t nblocks, uint32_t *gen = nullptr)
{
    unsigned long long *word = reinterpret_cast<unsigned long long *>(sync);
    unsigned long long old;
    asm volatile("atom.acq_rel.gpu.add.u64 %0, [%1], 1;" : "=l"(old) : "l"(word) : "memory");
    const uint32_t g = (uint32_t)(old >> 32);
    if (gen)
        *gen = g + 1;
    if ((uint32_t)old + 1u == nblocks) {
        const unsigned long long next = (1ull << 32) - nblocks; // generation + 1, count back to 0
        asm volatile("red.release.gpu.add.u64 [%0], %1;" ::"l"(word), "l"(next) : "memory");
        return true;
    }
    const uint64_t t0 = global_timer_ns();
    for (;;) {
        unsigned long long cur;
        asm volatile("ld.acquire.gpu.u64 %0, [%1];" : "=l"(cur) : "l"(word) : "memory");
        if ((uint32_t)(cur >> 32) != g)
            return true;
        if (global_timer_ns() - t0 > kWaitLimitNs)
            return false;
        __nanosleep(32);
    }
}

// Per 16-byte vector (8 fp16 values): |x| as half2 pairs and their maximum.
__device__ __forceinline__ __half2 vec_abs_max(const uint4 &v, __half2 (&a)[4])
{
    const __half2 *h = reinterpret_cast<const __half2 *>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i)
        a[i] = __habs2(h[i]);
    return __hmax2(__hmax2(a[0], a[1]), __hmax2(a[2], a[3]));
}

__device__ __forceinline__ uint32_t pack4(uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// Codes of 8 fp16 values with multiplier s: per value the fp32 product x * s
// rounded to nearest even, then rint() of it by adding 1.5 * 2^23 in
// round-to-nearest-even (the low byte of the sum is the code). The two
// roundings must stay separate (no fused multiply-add), as in the definition.
// (Scalar on purpose: the packed fp32x2 multiply/add was checked on B200 and
// gave different codes than the oracle for some values.)
__device__ __forceinline__ uint2 codes8(const uint4 &v, float s)
{
    const __half2 *h = reinterpret_cast<const __half2 *>(&v);
    uint32_t b[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(h[i]);
        b[2 * i] = __float_as_uint(__fadd_rn(__fmul_rn(f.x, s), 12582912.0f));
        b[2 * i + 1] = __float_as_uint(__fadd_rn(__fmul_rn(f.y, s), 12582912.0f));
    }
    return make_uint2(pack4(b[0], b[1], b[2], b[3]), pack4(b[4], b[5], b[6], b[7]));
}

// Zero the fp16 values of a 16-byte vector whose bit is set in `kbyte`
// (bit e = element e): known outlier columns drop out of the maximum and get
// code 0.
__device__ __forceinline__ void mask_known(uint4 &v, uint32_t kbyte)
{
    uint32_t *w = reinterpret_cast<uint32_t *>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t m = (kbyte >> (2 * i)) & 3u;
        w[i] &= ~(((m & 1u) * 0x0000FFFFu) | ((m >> 1) * 0xFFFF0000u));
    }
}

// Bits e of the result: element e of the 16-byte vector has |x| >= t16.
__device__ __forceinline__ uint32_t hit_mask8(const uint4 &v, __half t16)
{
    const __half2 *h = reinterpret_cast<const __half2 *>(&v);
    uint32_t hit = 0u;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __half2 a = __habs2(h[i]);
        if (__hge(__low2half(a), t16))
            hit |= 1u << (2 * i);
        if (__hge(__high2half(a), t16))
            hit |= 2u << (2 * i);
    }
    return hit;
}

// The last two steps of every epilogue: y + bias (fp32), then the
// activation (LLMINT8_ACT_GELU_TANH: BLOOM's GELU in tanh form, page
// "优化故事：Bloom 推理", section "唾手可得的优化"), before the single fp16
// rounding.
__device__ __forceinline__ float bias_act(float y, float bias, int act)
{
    y += bias;
    if (act == 1)
        y = 0.5f * y * (1.0f + tanhf(0.79788456f * y * (1.0f + 0.044715f * y * y)));
    return y;
}

} // namespace llmint8
