// kpa_f32x2.cuh -- packed fp32 pair arithmetic (the sm_100 f32x2 forms: one
// instruction for two lanes' worth of FP32 work), bf16 pair widening, and a 2^x
// for pairs on the FMA pipe.
#pragma once

#include <stdint.h>

namespace kpa {
namespace f32x2 {

__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
    float2 r;
    asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rc, ra, rb;\n\t"
        "mov.b64 {%0, %1}, rc;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return r;
}

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    float2 r;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\t"
        "mov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return r;
}

__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
    float2 r;
    asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rc, ra, rb;\n\t"
        "mov.b64 {%0, %1}, rc;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return r;
}

__device__ __forceinline__ float2 fsub2(float2 a, float2 b) {
    float2 r;
    asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "sub.rn.f32x2 rc, ra, rb;\n\t"
        "mov.b64 {%0, %1}, rc;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return r;
}

// bf16x2 word -> (low element, high element) as floats
__device__ __forceinline__ float2 unpack_bf16x2(uint32_t v) {
    return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
}

// 2^x (x <= 8) for a pair, on the FMA pipe instead of the transcendental unit:
// Cody-Waite reduction x = n + f with n = round(x) and f in [-1/2, 1/2], a degree-4
// polynomial for 2^f, and 2^n added into the exponent field.  The coefficients are
// the float32 output of fit_exp2_poly.py (next to this file): a weighted least-squares
// fit on [-1/2, 1/2] reweighted toward equal relative ripple; that script also
// evaluates this exact float32 sequence over [-126, 8] (maximum relative error 2.7e-6).
// x is clamped at -126 so the scaled result stays representable (it is then ~1e-38).
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
    constexpr float kRound = 12582912.f;            // 1.5 * 2^23: x + kRound holds round(x) in its low bits
    constexpr float c0 = 0x1.ffffe8p-1f, c1 = 0x1.62e0dep-1f, c2 = 0x1.ec06dap-3f, c3 = 0x1.ca13f8p-5f,
                    c4 = 0x1.399750p-7f;
    x.x = fmaxf(x.x, -126.f);
    x.y = fmaxf(x.y, -126.f);
    const float2 j = fadd2(x, make_float2(kRound, kRound));
    const float2 f = fsub2(x, fsub2(j, make_float2(kRound, kRound)));
    float2 p = ffma2(make_float2(c4, c4), f, make_float2(c3, c3));
    p = ffma2(p, f, make_float2(c2, c2));
    p = ffma2(p, f, make_float2(c1, c1));
    p = ffma2(p, f, make_float2(c0, c0));
    return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(j.x) << 23)),
                       __int_as_float(__float_as_int(p.y) + (__float_as_int(j.y) << 23)));
}

}  // namespace f32x2
}  // namespace kpa
