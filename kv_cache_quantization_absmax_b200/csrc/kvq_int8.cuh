// Bit-exact per-row absmax INT8 quantization of a group of values, shared by the
// quantize kernels and the decode step's append of a new token.
//
// The code is rint_even(fl32(x / s)) with s = fl32(max|x| / 127) the stored fp32 scale
// ("Q-TensorFormer" model card, section 6, symmetric INT8 equation).  The fast path
// multiplies by a reciprocal r of s and rounds with the 1.5 * 2^23 addition (for
// |q| < 2^22 the sum's ulp is 1, so round-to-nearest-even of the addition is
// rint_even(q), and the code is the low byte of the sum's bit pattern).  r comes from
// the hardware reciprocal approximation refined by one Newton-Raphson step,
// r1 = r0 + r0 (1 - s r0) (two FMAs): its relative error is below 2^-23.  Then
// |x r - x / s| <= 2^-22 |x / s| <= 3.1e-5 and |fl32(x / s) - x / s| <= 3.9e-6 for
// |x / s| <= 127.00002, so whenever q = x r is more than 2^-14 (6.1e-5) away from a
// half-integer both quotients round to the same integer.  A group with an element
// closer than that, or with a subnormal scale (1 / s would overflow), recomputes its
// codes with the IEEE division __fdiv_rn and __float2int_rn, plus the page's clamp.
// The codes do not depend on how a row is split into groups.
#pragma once

#include <stdint.h>

namespace kvq {
namespace i8 {

constexpr float kRoundMagic = 12582912.0f;          // 1.5 * 2^23
constexpr float kTieGuard = 0.5f - 6.103515625e-05f; // 0.5 - 2^-14
constexpr float kFltMinNormal = 1.17549435e-38f;

// Low bytes of four words -> one word (byte i of the result = low byte of w_i).
__device__ __forceinline__ uint32_t pack_low_bytes(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3) {
    uint32_t lo = __byte_perm(w0, w1, 0x0040);
    uint32_t hi = __byte_perm(w2, w3, 0x0040);
    return __byte_perm(lo, hi, 0x5410);
}

// 1/s for a normal s: hardware approximation + one Newton-Raphson step.
__device__ __forceinline__ float reciprocal_nr(float s) {
    float r0;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r0) : "f"(s));
    const float e = __fmaf_rn(-s, r0, 1.0f);
    return __fmaf_rn(r0, e, r0);
}

// Reciprocal used by the fast path (0 for a zero scale, which makes every code 0).
__device__ __forceinline__ float scale_reciprocal(float s) {
    return (s >= kFltMinNormal) ? reciprocal_nr(s) : 0.0f;
}

// The stored scale of a row whose largest magnitude is a.
__device__ __forceinline__ float row_scale(float a) { return __fdiv_rn(a, 127.0f); }

// Quantize N (a multiple of 4) values sharing scale s into N/4 packed words.
template <int N>
__device__ __forceinline__ void quantize_values(const float* f, float s, float rinv, uint32_t* out) {
    const bool s_zero = (s == 0.0f);
    const bool fast_ok = s_zero || (s >= kFltMinNormal);
    uint32_t y[N];
    float tmax = 0.0f;
#pragma unroll
    for (int e = 0; e < N; ++e) {
        const float q = __fmul_rn(f[e], rinv);
        const float yf = __fadd_rn(q, kRoundMagic);
        const float t = __fsub_rn(q, __fsub_rn(yf, kRoundMagic));
        tmax = fmaxf(tmax, fabsf(t));
        y[e] = __float_as_uint(yf);
    }
    if (!(fast_ok && tmax <= kTieGuard)) {
#pragma unroll
        for (int e = 0; e < N; ++e) {
            int c = __float2int_rn(__fdiv_rn(f[e], s));
            c = min(max(c, -128), 127);
            y[e] = static_cast<uint32_t>(c);
        }
    }
#pragma unroll
    for (int w = 0; w < N / 4; ++w)
        out[w] = pack_low_bytes(y[4 * w], y[4 * w + 1], y[4 * w + 2], y[4 * w + 3]);
}

}  // namespace i8
}  // namespace kvq
