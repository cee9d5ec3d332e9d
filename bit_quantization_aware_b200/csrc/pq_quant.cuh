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

struct Elem {
    float x;      // fl(w / alpha)
    float r;      // integer-valued rounded code (may be -0.0)
    float level;  // level in alpha units
    bool inside;  // lo <= x <= hi (STE gate, closed range)
};

template <int Q>
__device__ __forceinline__ Elem quantize(float w, float alpha) {
    using T = Traits<Q>;
    Elem e;
    e.x = __fdiv_rn(w, alpha);
    e.inside = (e.x >= T::lo) && (e.x <= T::hi);
    if constexpr (Q == PQ_BINARY) {
        e.r = (e.x >= 0.0f) ? 1.0f : -1.0f;
        e.level = e.r;
    } else {
        const float xc = fminf(fmaxf(e.x, T::lo), T::hi);
        if constexpr (Q == PQ_SEQ2) {
            e.r = rintf(__fsub_rn(__fmul_rn(xc, 2.0f), 0.5f));
            e.level = __fmul_rn(__fadd_rn(e.r, 0.5f), 0.5f);
        } else if constexpr (Q == PQ_SEQ2_B) {
            e.r = rintf(__fsub_rn(__fmul_rn(xc, 1.5f), 0.5f));
            e.level = __fmul_rn(__fadd_rn(e.r, 0.5f), kTwoThirds);
        } else if constexpr (Q == PQ_TERNARY) {
            e.r = rintf(__fmul_rn(xc, 1.5f));
            e.level = __fmul_rn(e.r, kTwoThirds);
        } else {  // LSQ integer grid
            e.r = rintf(xc);
            e.level = e.r;
        }
    }
    return e;
}

// Two's-complement code field of width Traits<Q>::bits.
template <int Q>
__device__ __forceinline__ uint32_t code_field(float r) {
    constexpr uint32_t mask = (1u << Traits<Q>::bits) - 1u;
    return static_cast<uint32_t>(__float2int_rz(r)) & mask;
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t h16) {
    return __uint_as_float(h16 << 16);
}

}  // namespace pq
