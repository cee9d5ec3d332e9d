// Per-element quantizer arithmetic of the ParetoQ-style fake-quantizer, as
// device functions shared by the forward, backward and pack kernels.
//
// Sources: "ParetoQ, the strongest low-bit QAT I could find", sections
// "Finding 3" (level sets), "Paper vs. code" (SEQ formula, clip 0.99,
// round-half-even, STE clipping gate); "ParetoQ: Improving Scaling Laws ..."
// rebuttal, section on SEQ vs LSQ (SEQ code domain, ternary bins).
//
// Every fp32 step uses an explicit round-to-nearest intrinsic so that the
// compiler cannot contract a multiply and an add into one FMA; x = w/alpha
// is the IEEE-correct division.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "pq.h"

namespace pq {

template <int Q>
struct Traits;

template <>
struct Traits<PQ_BINARY> {
    static constexpr float lo = -1.0f, hi = 1.0f;
    static constexpr int bits = 2;
};
template <>
struct Traits<PQ_TERNARY> {
    static constexpr float lo = -0.99f, hi = 0.99f;
    static constexpr int bits = 2;
};
template <>
struct Traits<PQ_SEQ2> {
    static constexpr float lo = -0.99f, hi = 0.99f;
    static constexpr int bits = 2;
};
template <>
struct Traits<PQ_SEQ2_B> {
    static constexpr float lo = -0.99f, hi = 0.99f;
    static constexpr int bits = 2;
};
template <>
struct Traits<PQ_LSQ2> {
    static constexpr float lo = -2.0f, hi = 1.0f;
    static constexpr int bits = 2;
};
template <>
struct Traits<PQ_LSQ3> {
    static constexpr float lo = -4.0f, hi = 3.0f;
    static constexpr int bits = 4;
};
template <>
struct Traits<PQ_LSQ4> {
    static constexpr float lo = -8.0f, hi = 7.0f;
    static constexpr int bits = 4;
};

// fl(2/3): 2/3 rounded once to fp32. For integer-valued r in {-1,-0,0,1},
// r * fl(2/3) equals fl(r / 1.5); for m in {-1.5,-0.5,0.5,1.5},
// fl(m * fl(2/3)) equals fl(m / 1.5) (checked exhaustively against the
// reference in the parity tests), so no division is needed for the levels.
constexpr float kTwoThirds = 2.0f / 3.0f;

// ------------------------------------------------------------ x = w / alpha
// Per-row scale: alpha, its correctly rounded reciprocal, and whether the
// reciprocal-based quotient may be used for this row.
struct RowScale {
    float a;
    float y;    // RN(1 / alpha)
    bool fast;  // alpha in [2^-60, 2^60]
};

__device__ __forceinline__ RowScale row_scale(float a) {
    RowScale s;
    s.a = a;
    s.y = __frcp_rn(a);
    s.fast = (a >= 0x1p-60f) && (a <= 0x1p60f);
    return s;
}

// RN(w / alpha) from y = RN(1 / alpha) with fused multiply-adds only:
// q0 = RN(w*y) is within two ulps of the quotient, one remainder step
// brings q1 within one ulp, and then, with the exact remainder
// r1 = w - alpha*q1, RN(q1 + r1*y) is the correctly rounded quotient
// (Markstein's theorem on the final correction of a quotient). The
// magnitude guards keep every intermediate a normal number, which the
// theorem needs; outside them the IEEE division runs instead.
__device__ __forceinline__ float div_fast(float w, const RowScale& s) {
    const float q0 = __fmul_rn(w, s.y);
    const float r0 = __fmaf_rn(-s.a, q0, w);
    const float q1 = __fmaf_rn(r0, s.y, q0);
    const float r1 = __fmaf_rn(-s.a, q1, w);
    return __fmaf_rn(r1, s.y, q1);
}

__device__ __forceinline__ bool div_fast_ok(float w) {
    const float m = fabsf(w);
    return m >= 0x1p-60f && m <= 0x1p60f;
}

// x[i] = RN(v[i] / alpha) for one chunk of 8 weights.
__device__ __forceinline__ void divide8(const float (&v)[8], const RowScale& s,
                                        float (&x)[8]) {
    bool all = s.fast;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        x[i] = div_fast(v[i], s);
        all = all && div_fast_ok(v[i]);
    }
    if (!all) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (!s.fast || !div_fast_ok(v[i])) x[i] = __fdiv_rn(v[i], s.a);
    }
}

// ---------------------------------------------------------- x -> level
// Round half to even for |t| < 2^22: t + 1.5*2^23 lies in [2^23, 2^24),
// where floats are spaced by 1, so the addition rounds t to an integer
// with ties to even (1.5*2^23 is even); subtracting the constant again is
// exact. The low bits of the sum's encoding hold that integer in two's
// complement, since the constant's low 22 mantissa bits are zero.
constexpr float kRoundShift = 12582912.0f;  // 1.5 * 2^23

struct Elem {
    float level;    // level in alpha units (a zero level keeps the sign of t)
    bool inside;    // lo <= x <= hi (STE gate, closed range)
    uint32_t code;  // two's-complement code in the low Traits<Q>::bits bits
};

template <int Q>
__device__ __forceinline__ Elem quantize_x(float x) {
    using T = Traits<Q>;
    Elem e;
    if constexpr (T::lo == -T::hi) {
        e.inside = fabsf(x) <= T::hi;  // same as lo <= x <= hi
    } else {
        e.inside = (x >= T::lo) && (x <= T::hi);
    }
    if constexpr (Q == PQ_BINARY) {
        const bool pos = x >= 0.0f;  // sign(+-0) = +1
        e.level = pos ? 1.0f : -1.0f;
        e.code = pos ? 1u : 3u;
    } else {
        const float xc = fminf(fmaxf(x, T::lo), T::hi);
        float t;
        if constexpr (Q == PQ_SEQ2) {
            t = __fmaf_rn(xc, 2.0f, -0.5f);  // 2*xc is exact: one rounding
        } else if constexpr (Q == PQ_SEQ2_B) {
            t = __fsub_rn(__fmul_rn(xc, 1.5f), 0.5f);  // two roundings
        } else if constexpr (Q == PQ_TERNARY) {
            t = __fmul_rn(xc, 1.5f);
        } else {  // LSQ integer grid
            t = xc;
        }
        const float tm = __fadd_rn(t, kRoundShift);
        float r = __fsub_rn(tm, kRoundShift);
        e.code = __float_as_uint(tm);
        if constexpr (Q == PQ_SEQ2) {
            e.level = __fmaf_rn(r, 0.5f, 0.25f);  // (r + 0.5)/2, exact
        } else if constexpr (Q == PQ_SEQ2_B) {
            // (r + 0.5) * fl(2/3) rounded once, as r*c + 0.5*c fused
            e.level = __fmaf_rn(r, kTwoThirds, 0.5f * kTwoThirds);
        } else if constexpr (Q == PQ_TERNARY) {
            r = copysignf(r, t);  // round(-0.3) is -0.0
            e.level = __fmul_rn(r, kTwoThirds);
        } else {
            e.level = copysignf(r, t);
        }
    }
    return e;
}

// Level (alpha units) of a stored code field f: sign-extend it to the code
// c, turn c into a float without the conversion unit (the add/subtract
// constant in reverse: the encoding of 1.5*2^23 + c, minus 1.5*2^23), and
// apply the forward's level formula. A zero level is +0.0.
template <int Q>
__device__ __forceinline__ float level_of_field(uint32_t f) {
    constexpr int B = Traits<Q>::bits;
    const int c = static_cast<int>(f << (32 - B)) >> (32 - B);
    const float cf = __fsub_rn(__int_as_float(0x4B400000 + c), kRoundShift);
    if constexpr (Q == PQ_SEQ2) {
        return __fmaf_rn(cf, 0.5f, 0.25f);
    } else if constexpr (Q == PQ_SEQ2_B) {
        return __fmaf_rn(cf, kTwoThirds, 0.5f * kTwoThirds);
    } else if constexpr (Q == PQ_TERNARY) {
        return __fmul_rn(cf, kTwoThirds);
    } else {  // LSQ grid and binary: the code is the level
        return cf;
    }
}

// Two's-complement code field of width Traits<Q>::bits.
template <int Q>
__device__ __forceinline__ uint32_t code_field(const Elem& e) {
    constexpr uint32_t mask = (1u << Traits<Q>::bits) - 1u;
    return e.code & mask;
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t h16) {
    return __uint_as_float(h16 << 16);
}

}  // namespace pq
