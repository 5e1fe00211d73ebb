// Software 2^x on the FMA pipe, for moving a share of the attention kernels'
// exponentials off the special-function unit (build knobs CP_FWD_POLY_PAIRS and
// CP_BWD_POLY_PAIRS, off by default: on B200 that share measured slower), and
// checked against the hardware ex2 by cp_selftest_exp2.
//
// Method: Cody & Waite range reduction, x = j + f with j = round(x) and
// f in [-1/2, 1/2], then 2^x = 2^j * p(f), where p is the degree-3 polynomial
// that minimises the maximum relative error of p(f) / 2^f - 1 on [-1/2, 1/2]
// (Remez exchange algorithm; coefficients printed by gen_exp2_poly.py next to
// this file).  Maximum relative error 7.5e-5, 26x below bf16's half-ulp.
//
// The rounding of x to j uses the 1.5 * 2^23 shift: adding it leaves round(x)
// in the low mantissa bits of t, and shifting t's bits left by 23 moves j into
// the exponent field (the constant's own bits shift out).  Inputs are clamped
// at -125 so p(f) * 2^j stays a normal float: results below 2^-125 come out as
// ~2^-125 instead of smaller, which no use here can see.  Inputs must be
// finite and at most 127.
#pragma once
#include <cstdint>

namespace cpattn {

constexpr float kExp2C0 = 0.9999280571937561f;
constexpr float kExp2C1 = 0.6932609677314758f;
constexpr float kExp2C2 = 0.2426111251115799f;
constexpr float kExp2C3 = 0.0551716685295105f;

// ---- packed fp32x2 arithmetic (one instruction for two lanes of data)
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b)
{
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

__device__ __forceinline__ float fmax3(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// 2^x for two values at once.
__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x2)
{
    float a, b;
    f2_unpack(x2, a, b);
    a = fmaxf(a, -125.f);
    b = fmaxf(b, -125.f);
    const uint64_t xc = f2_pack(a, b);
    const uint64_t shift = f2_pack(12582912.f, 12582912.f);
    const uint64_t t = f2_add(xc, shift);                           // j in the low bits
    const uint64_t j = f2_add(t, f2_pack(-12582912.f, -12582912.f)); // round(x)
    const uint64_t f = f2_fma(j, f2_pack(-1.f, -1.f), xc);          // x - j in [-1/2, 1/2]
    uint64_t p = f2_fma(f2_pack(kExp2C3, kExp2C3), f, f2_pack(kExp2C2, kExp2C2));
    p = f2_fma(p, f, f2_pack(kExp2C1, kExp2C1));
    p = f2_fma(p, f, f2_pack(kExp2C0, kExp2C0));
    float p0, p1, t0, t1;
    f2_unpack(p, p0, p1);
    f2_unpack(t, t0, t1);
    const float r0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
    const float r1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
    return f2_pack(r0, r1);
}

__device__ __forceinline__ float exp2_poly(float x)
{
    float a, b;
    f2_unpack(exp2_poly2(f2_pack(x, x)), a, b);
    return a;
}

}  // namespace cpattn
