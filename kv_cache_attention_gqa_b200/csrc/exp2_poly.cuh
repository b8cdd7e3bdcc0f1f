// 2^x on the FMA/ALU pipes, to move part of the softmax exponentials off the special-function
// unit. The prefill kernel measured slower with it (its softmax is bound by latency, not by that
// unit), so GQA_PREFILL_POLY_EVERY keeps it off by default.
//
// Method: Cody-Waite range reduction. x = n + f with n = rint(x), obtained by adding 1.5 * 2^23
// (which leaves the rounded integer in the low mantissa bits), and f = x - n in [-1/2, 1/2].
// 2^f is a degree-3 polynomial, a relative-error minimax fit on [-1/2, 1/2] made for this
// library by Remez exchange (max relative error 7.5e-5 in fp32 coefficients, far below the 2^-9
// rounding of the bf16 P it feeds; tests/test_exp2_poly.py re-derives the constants). 2^n is added to the exponent field: bits(2^f) + (bits(t) << 23).
// Inputs are clamped to >= -126 so the exponent field cannot wrap; callers use this only where
// every input is finite (blocks without masked keys), so masked weights stay exactly 0.
#pragma once

#include <stdint.h>

namespace gqa {

// polynomial coefficients c0..c3 of 2^f ~ c0 + c1 f + c2 f^2 + c3 f^3 (fp32 bit patterns)
#define GQA_EXP2_POLY_C0 0x3f7ffb49u
#define GQA_EXP2_POLY_C1 0x3f31798du
#define GQA_EXP2_POLY_C2 0x3e786f0du
#define GQA_EXP2_POLY_C3 0x3d61fbb0u

// y = 2^x for two inputs, with packed fp32x2 arithmetic
__device__ __forceinline__ void exp2_poly2(float x0, float x1, float& y0, float& y1) {
  uint32_t r0, r1;
  asm("{\n\t"
      ".reg .b32 a0, a1, t0, t1, p0, p1, k;\n\t"
      ".reg .b64 x, t, n, f, p, vm, vnm, vneg, vc0, vc1, vc2, vc3;\n\t"
      "max.f32 a0, %2, 0fC2FC0000;\n\t"   // clamp to -126
      "max.f32 a1, %3, 0fC2FC0000;\n\t"
      "mov.b64 x, {a0, a1};\n\t"
      "mov.b32 k, 0f4B400000;\n\tmov.b64 vm, {k, k};\n\t"    // 1.5 * 2^23
      "mov.b32 k, 0fCB400000;\n\tmov.b64 vnm, {k, k};\n\t"
      "mov.b32 k, 0fBF800000;\n\tmov.b64 vneg, {k, k};\n\t"  // -1
      "add.rn.f32x2 t, x, vm;\n\t"        // rint(x) in the low bits of t
      "add.rn.f32x2 n, t, vnm;\n\t"       // n = rint(x) as float
      "fma.rn.f32x2 f, n, vneg, x;\n\t"   // f = x - n
      "mov.b64 vc3, {%7, %7};\n\tmov.b64 vc2, {%6, %6};\n\t"
      "mov.b64 vc1, {%5, %5};\n\tmov.b64 vc0, {%4, %4};\n\t"
      "fma.rn.f32x2 p, vc3, f, vc2;\n\t"  // Horner
      "fma.rn.f32x2 p, p, f, vc1;\n\t"
      "fma.rn.f32x2 p, p, f, vc0;\n\t"
      "mov.b64 {p0, p1}, p;\n\t"
      "mov.b64 {t0, t1}, t;\n\t"
      "shl.b32 t0, t0, 23;\n\tshl.b32 t1, t1, 23;\n\t"
      "add.s32 %0, p0, t0;\n\tadd.s32 %1, p1, t1;\n\t"
      "}"
      : "=r"(r0), "=r"(r1)
      : "f"(x0), "f"(x1), "f"(__uint_as_float(GQA_EXP2_POLY_C0)),
        "f"(__uint_as_float(GQA_EXP2_POLY_C1)), "f"(__uint_as_float(GQA_EXP2_POLY_C2)),
        "f"(__uint_as_float(GQA_EXP2_POLY_C3)));
  y0 = __uint_as_float(r0);
  y1 = __uint_as_float(r1);
}

}  // namespace gqa
