// FP8 e4m3 quantisation of 128-channel blocks: the block scale s = amax / 448
// and the codes e4m3(x / s), both correctly rounded.  Shared by the dispatch
// kernels (dispatch.cu) and the fused route + dispatch kernel, so they write
// the same bytes.
#pragma once

#include "common.cuh"

namespace moe {

// s = amax / 448 rounded to nearest even.  For amax >= 2^-80 this is
// Markstein's correction of amax * RN(1/448) (exact there; checked against
// IEEE division for every bf16 amax and 1.6e7 fp32 ones), else IEEE division.
__device__ __forceinline__ float scale_of(float amax) {
    if (amax >= 0x1p-80f) {
        const float r = 0x1.24924ap-9f;  // RN(1/448)
        const float q0 = __fmul_rn(amax, r);
        const float e = __fmaf_rn(-q0, 448.0f, amax);
        return __fmaf_rn(e, r, q0);
    }
    return __fdiv_rn(amax, 448.0f);
}

// q = x / s rounded to nearest even, for normal x, s: Markstein's correction
// of x * r with r = 1/s correctly rounded (P. Markstein, "Computation of
// elementary functions on the IBM RISC System/6000 processor", IBM J. Res.
// Dev. 34(1), 1990): with r = RN(1/s), q0 = RN(x r) and the remainder
// e = x - q0 s exact (one fma), RN(q0 + e r) = RN(x / s).  The remainder is
// formed negated, n = q0 s - x, and the quotient as RN(q0 + (-n) r): the same
// values for x != 0, and for x = -0 the sums (-0) + (+0) -> +0 and
// (-0) + (-0) -> -0 keep the sign of the zero quotient (three operations, the
// negations being free operand modifiers).
__device__ __forceinline__ float div_markstein(float x, float s, float r) {
    const float q0 = __fmul_rn(x, r);
    const float n = __fmaf_rn(q0, s, -x);
    return __fmaf_rn(-n, r, q0);
}

// 16 values -> 16 e4m3 codes (value i in byte i), given the block scale s.
__device__ __forceinline__ U4 quant16(const float (&f)[16], float s) {
    uint32_t w[4];
    if (s == 0.f) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t r = 0;
#pragma unroll
            for (int b = 0; b < 4; ++b) r |= ((__float_as_uint(f[4 * i + b]) >> 31) << 7) << (8 * b);
            w[i] = r;
        }
    } else if (s >= 0x1p-90f) {
        // For |x| >= 2^-102 the remainder x - q0 s is exact, so the quotient is
        // correctly rounded; smaller x give |x / s| < 2^-11, which is a signed
        // e4m3 zero whatever its last fp32 bits.  (Checked against IEEE
        // division over 6e7 inputs: identical codes.)
        const float r = __frcp_rn(s);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t lo = pack_e4m3x2(div_markstein(f[4 * i], s, r), div_markstein(f[4 * i + 1], s, r));
            const uint32_t hi = pack_e4m3x2(div_markstein(f[4 * i + 2], s, r), div_markstein(f[4 * i + 3], s, r));
            w[i] = lo | (hi << 16);
        }
    } else {  // tiny scale: plain IEEE division
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t lo = pack_e4m3x2(__fdiv_rn(f[4 * i], s), __fdiv_rn(f[4 * i + 1], s));
            const uint32_t hi = pack_e4m3x2(__fdiv_rn(f[4 * i + 2], s), __fdiv_rn(f[4 * i + 3], s));
            w[i] = lo | (hi << 16);
        }
    }
    return U4{w[0], w[1], w[2], w[3]};
}

}  // namespace moe
