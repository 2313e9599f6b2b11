// exp2_fma.cuh -- packed fp32 pair arithmetic (sm_100 f32x2 instructions) and
// 2^x evaluated on the FMA pipe, for softmax code that splits its
// exponentials between the MUFU unit and the FMA units.
#pragma once

#include <stdint.h>

namespace gqe {

__device__ __forceinline__ uint64_t pk2(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void up2(uint64_t v, float& a, float& b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// 2^x for a pair of fp32 values on the FMA pipe, x in [-126, 8]: Cody-Waite
// style range reduction x = n + f, n = round(x), f in [-1/2, 1/2], 2^f by a
// cubic fitted by least squares on Chebyshev nodes (exp2_poly_fit.py; max
// relative error 1.2e-4), 2^n added to the exponent field.  Adding 1.5 * 2^23
// leaves round(x) in the low mantissa bits of t, so t's bit pattern shifted
// left by 23 is n << 23.
__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x) {
    const uint64_t kMagic = pk2(12582912.0f, 12582912.0f);
    const uint64_t kNegMagic = pk2(-12582912.0f, -12582912.0f);
    const uint64_t kNeg1 = pk2(-1.0f, -1.0f);
    const uint64_t c0 = pk2(1.0f, 1.0f);
    const uint64_t c1 = pk2(6.933686137e-01f, 6.933686137e-01f);
    const uint64_t c2 = pk2(2.422178388e-01f, 2.422178388e-01f);
    const uint64_t c3 = pk2(5.459282547e-02f, 5.459282547e-02f);
    const uint64_t t = fadd2(x, kMagic);
    const uint64_t n = fadd2(t, kNegMagic);
    const uint64_t f = ffma2(n, kNeg1, x);
    uint64_t q = ffma2(c3, f, c2);
    q = ffma2(q, f, c1);
    q = ffma2(q, f, c0);
    float t0, t1, q0, q1;
    up2(t, t0, t1);
    up2(q, q0, q1);
    return pk2(__uint_as_float(__float_as_uint(q0) + (__float_as_uint(t0) << 23)),
               __uint_as_float(__float_as_uint(q1) + (__float_as_uint(t1) << 23)));
}

// The form the softmax uses: inputs below -126 are clamped to -126 (their
// true values are below 2^-126 and vanish next to the row sum, which is >= 1).
__device__ __forceinline__ uint64_t exp2_poly2_clamped(float x0, float x1) {
    return exp2_poly2(pk2(fmaxf(x0, -126.f), fmaxf(x1, -126.f)));
}

}  // namespace gqe
