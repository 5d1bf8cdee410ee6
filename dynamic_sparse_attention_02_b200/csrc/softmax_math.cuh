// softmax_math.cuh -- device arithmetic shared by the attention engines:
// MUFU exp2, packed fp32 pairs (sm_100 f32x2 instructions: two IEEE
// operations per instruction), 2^x on the FMA pipe (steps and constants in
// exp2_poly.h), bf16 packing and bit masks.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "exp2_poly.h"

namespace minfer {

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ---- packed fp32 pairs (one 64-bit register pair, two lanes of work)
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.ftz.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.ftz.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// 2^x for a pair on the FMA pipe (steps and constants in exp2_poly.h).  A
// quarter of the softmax exponentials take this path: the two slots' softmax
// warps share the MUFU unit, which is otherwise the busiest pipe of the loop.
__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x2) {
    float a, b;
    f2_unpack(x2, a, b);
    const uint64_t xc = f2_pack(fmaxf(a, kExp2Clamp), fmaxf(b, kExp2Clamp));
    const uint64_t t = f2_add(xc, f2_pack(kExp2Round, kExp2Round));
    const uint64_t tn = f2_add(t, f2_pack(-kExp2Round, -kExp2Round));
    const uint64_t fr = f2_fma(tn, f2_pack(-1.f, -1.f), xc);
    uint64_t q = f2_fma(f2_pack(kExp2C3, kExp2C3), fr, f2_pack(kExp2C2, kExp2C2));
    q = f2_fma(q, fr, f2_pack(kExp2C1, kExp2C1));
    q = f2_fma(q, fr, f2_pack(kExp2C0, kExp2C0));
    uint32_t qlo, qhi, tlo, thi;
    asm("mov.b64 {%0, %1}, %2;" : "=r"(qlo), "=r"(qhi) : "l"(q));
    asm("mov.b64 {%0, %1}, %2;" : "=r"(tlo), "=r"(thi) : "l"(t));
    uint64_t r;  // 2^n by adding n (low bits of t) to the exponent field
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(qlo + (tlo << 23)), "r"(qhi + (thi << 23)));
    return r;
}

// bits 0 .. k-1 set (none for k <= 0, all for k >= 64)
__device__ __forceinline__ uint64_t low_bits(long long k) {
    return k <= 0 ? 0ull : (k >= 64 ? ~0ull : (1ull << k) - 1ull);
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

}  // namespace minfer
