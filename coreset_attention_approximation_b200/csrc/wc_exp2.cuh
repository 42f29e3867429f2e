// wc_exp2.cuh — 2^x on the FMA and ALU pipes, and packed fp32 pairs (sm_100a).
//
// The exp-GEMM's softmax warps share each SM sub-partition's exponential unit
// (MUFU: 4 results per clock, against 32 lanes of fused multiply-add per
// clock), and per 128-key tile that unit is as busy as the tensor pipe.
// exp2_fma2 computes two exponentials without the exponential unit, so part
// of every row can move to the FMA / ALU pipes:
//   x <- max(x, -127)
//   t  = x + (1.5 * 2^23 + 127)       rounded to nearest: t's low mantissa bits hold n + 127,
//                                     n = rint(x)
//   f  = x - (t - (1.5 * 2^23 + 127)) in [-1/2, 1/2], exact: the additive range reduction of
//                                     Cody and Waite ("Software Manual for the Elementary
//                                     Functions", 1980), which for base 2 needs no split constant
//   p  = c0 + f (c1 + f (c2 + f c3))  the degree-3 polynomial of least maximum relative error
//                                     to 2^f on [-1/2, 1/2], fitted by the Remez exchange
//                                     algorithm (remez_exp2.py prints these coefficients)
//   s  = the float with bits t << 23  = 2^n, its exponent field n + 127 (0, i.e. s = 0, when
//                                     n = -127)
//   2^x = p s
// Accuracy: relative error at most 2^-13.5 against 2^x for -125 <= x <= 127
// (fit 2^-13.71, plus the fp32 roundings of the Horner steps); below -125
// the absolute error is under 2^-125, and x <= -127 (-inf included) gives
// exactly 0, as the exponential unit does.  The exp-GEMM rounds its
// exponentials to fp16 (relative step 2^-11).  tests/test_exp2_poly.py checks
// the bound on the CPU (an fp32 emulation) and on the GPU (wc_selftest_exp2).
//
// The packed helpers wrap sm_100's two-lane fp32 instructions (fma / add /
// sub / mul .rn.f32x2): one issue slot for two IEEE fp32 results, each rounded
// as the scalar instruction would round it.
#pragma once

#include <stdint.h>

namespace wc {

// Coefficients of the Remez fit (degree 3, relative error 7.478e-05 on [-1/2, 1/2]).
constexpr float kExp2C0 = 0x1.fff692p-1f;
constexpr float kExp2C1 = 0x1.62f31ap-1f;
constexpr float kExp2C2 = 0x1.f0de1ap-3f;
constexpr float kExp2C3 = 0x1.c3f76p-5f;
constexpr float kExp2Shift = 0x1.8000fep+23f;   // 1.5 * 2^23 + 127
constexpr float kExp2Lo = -127.f;

__device__ __forceinline__ uint64_t pack2(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ float2 unpack2(uint64_t r) {
    float2 v;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(v.x), "=f"(v.y) : "l"(r));
    return v;
}

// a * b + c per lane, one rounding each
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(pack2(a.x, a.y)), "l"(pack2(b.x, b.y)), "l"(pack2(c.x, c.y)));
    return unpack2(d);
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(pack2(a.x, a.y)), "l"(pack2(b.x, b.y)));
    return unpack2(d);
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(pack2(a.x, a.y)), "l"(pack2(b.x, b.y)));
    return unpack2(d);
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(pack2(a.x, a.y)), "l"(pack2(b.x, b.y)));
    return unpack2(d);
}

// max(a, b, c) in one instruction (sm_100's three-input max)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// (2^x.x, 2^x.y) without the exponential unit (see the top of this file)
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
    x.x = fmaxf(x.x, kExp2Lo);
    x.y = fmaxf(x.y, kExp2Lo);
    const float2 t = add2(x, make_float2(kExp2Shift, kExp2Shift));
    const float2 f = sub2(x, sub2(t, make_float2(kExp2Shift, kExp2Shift)));
    float2 p = fma2(make_float2(kExp2C3, kExp2C3), f, make_float2(kExp2C2, kExp2C2));
    p = fma2(p, f, make_float2(kExp2C1, kExp2C1));
    p = fma2(p, f, make_float2(kExp2C0, kExp2C0));
    const float2 sc = make_float2(__int_as_float(__float_as_int(t.x) << 23), __int_as_float(__float_as_int(t.y) << 23));
    return mul2(p, sc);
}

}  // namespace wc
