// softmax_math.cuh -- exponentials of the prefill softmax that run on the FMA
// pipe, shared by the prefill kernel and its GPU self-test.
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace osp {

// 2^x for a pair of floats on the FMA pipe, keeping the special-function
// unit free for the rest of the row.  Range reduction x = n + f with
// n = round(x) (the 1.5 * 2^23 shift puts n in the low mantissa bits) and
// f in [-1/2, 1/2]; 2^f by a cubic in Horner form; 2^n added into the
// exponent field.  The cubic's coefficients are the relative-error minimax
// fit of 2^f on [-1/2, 1/2] (Chebyshev nodes refined by Lawson's iteration,
// rounded to fp32: online_softmax_paged_b200/exp2_poly_fit.py derives them),
// with a maximum relative error of 7.5e-5 in fp32 over the kernel's range,
// far below the bf16 rounding of P.  x is clamped to >= -125 so the result
// stays a normal number (2^-125 is 0 next to a running sum l >= 1).
__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x2) {
    constexpr float kShift = 12582912.0f;  // 1.5 * 2^23
    constexpr float c0 = 0x1.fff692p-1f, c1 = 0x1.62f31ap-1f, c2 = 0x1.f0de1ap-3f, c3 = 0x1.c3f75ep-5f;
    float x0, x1;
    f2_unpack(x2, x0, x1);
    x0 = fmaxf(x0, -125.f);
    x1 = fmaxf(x1, -125.f);
    const uint64_t xc = f2_pack(x0, x1);
    const uint64_t t = f2_add(xc, f2_pack(kShift, kShift));                        // n in the low mantissa bits
    const uint64_t nr = f2_fma(t, f2_pack(-1.f, -1.f), f2_pack(kShift, kShift));  // -n
    const uint64_t fr = f2_add(xc, nr);                                            // f = x - n
    uint64_t r = f2_fma(f2_pack(c3, c3), fr, f2_pack(c2, c2));
    r = f2_fma(r, fr, f2_pack(c1, c1));
    r = f2_fma(r, fr, f2_pack(c0, c0));
    float p0, p1, t0, t1;
    f2_unpack(r, p0, p1);
    f2_unpack(t, t0, t1);
    p0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
    p1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
    return f2_pack(p0, p1);
}

}  // namespace osp
