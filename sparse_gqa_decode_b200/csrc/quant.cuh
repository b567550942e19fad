// quant.cuh -- exact INT8 codes (shared by the quantize kernels and the fused score+quantize
// pass of the decode pipeline, so both produce the same bits).
//
// "优化稀疏注意力中的令牌丢弃机制" (Optimizing token dropping in sparse attention), section 6:
// q_val = round(val / scale).  Reading: the quotient is the correctly rounded float32 x/s,
// rounded half to even, clamped to [-127, 127]; a zero scale gives zero codes.
//
// Without one IEEE divide per element: q' = x * RN(1/s) differs from Q = RN(x/s) by at most
// |x/s| * 2^-23 + ulp(Q)/2 <= 2.3e-5 (|x/s| <= 127 * (1 + 2^-23) for the group's own scale),
// so round_half_even(q') == round_half_even(Q) unless q' lies within 2.3e-5 of a
// half-integer; whenever q' is within 1e-4 of one (or is not finite) the IEEE division
// __fdiv_rn(x, s) decides instead.
#pragma once

#include "common.cuh"

namespace sgd {

__device__ __forceinline__ int code_of(float x, float s, float r) {
    float q = x * r;
    float n = rintf(q);
    if (!(fabsf(q - n) < 0.4999f)) {
        q = __fdiv_rn(x, s);
        n = rintf(q);
    }
    n = fminf(fmaxf(n, -127.f), 127.f);
    return (int)n;
}

template <typename T>
struct Vec;  // 16 bytes of input -> VE elements -> VE code bytes
template <>
struct Vec<__nv_bfloat16> {
    static constexpr int VE = 8;
    __device__ static void unpack(const uint4 &w, float (&x)[8]) {
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            x[2 * i] = __uint_as_float(ww[i] << 16);
            x[2 * i + 1] = __uint_as_float(ww[i] & 0xffff0000u);
        }
    }
};
template <>
struct Vec<float> {
    static constexpr int VE = 4;
    __device__ static void unpack(const uint4 &w, float (&x)[4]) {
        x[0] = __uint_as_float(w.x);
        x[1] = __uint_as_float(w.y);
        x[2] = __uint_as_float(w.z);
        x[3] = __uint_as_float(w.w);
    }
};

// Codes of four values as the bytes of one word.  Per pair of values, with packed f32x2
// arithmetic: t = fma(x, r, M) with M = 1.5 * 2^23 rounds the exact product x*r to an integer
// held in the low mantissa bits of t (|x*r| < 2^22), so the low byte of t is that integer in
// two's complement; -n = M - t is exact and e = fma(x, r, -n) is the rounding residual.
// |e| < 0.4999 keeps the fast result; otherwise (near a half-integer, or not finite) code_of's
// IEEE division decides.  |x*r| <= 127.0001 for the group's own scale, so the fast integer
// already lies in [-127, 127].
// The rare exact path of codes4, kept out of line so that the unrolled fast path stays compact.
static __device__ __noinline__ uint32_t codes4_exact(float x0, float x1, float x2, float x3, float s, float r) {
    return (uint32_t)(code_of(x0, s, r) & 0xff) | ((uint32_t)(code_of(x1, s, r) & 0xff) << 8) |
           ((uint32_t)(code_of(x2, s, r) & 0xff) << 16) | ((uint32_t)(code_of(x3, s, r) & 0xff) << 24);
}

__device__ __forceinline__ uint64_t f32x2(float lo, float hi) {
    return (uint64_t)__float_as_uint(lo) | ((uint64_t)__float_as_uint(hi) << 32);
}

// The fast result of codes4 and whether it stands (no branch).
__device__ __forceinline__ uint32_t codes4_fast(const float *x, float r, bool &fast) {
    const uint64_t rr = f32x2(r, r), mm = f32x2(12582912.f, 12582912.f);
    uint64_t t01, t23, n01, n23, e01, e23;
    const uint64_t x01 = f32x2(x[0], x[1]), x23 = f32x2(x[2], x[3]);
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(t01) : "l"(x01), "l"(rr), "l"(mm));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(t23) : "l"(x23), "l"(rr), "l"(mm));
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(n01) : "l"(mm), "l"(t01));
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(n23) : "l"(mm), "l"(t23));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(e01) : "l"(x01), "l"(rr), "l"(n01));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(e23) : "l"(x23), "l"(rr), "l"(n23));
    const float e[4] = {__uint_as_float((uint32_t)e01), __uint_as_float((uint32_t)(e01 >> 32)),
                        __uint_as_float((uint32_t)e23), __uint_as_float((uint32_t)(e23 >> 32))};
    fast = fabsf(e[0]) < 0.4999f && fabsf(e[1]) < 0.4999f && fabsf(e[2]) < 0.4999f && fabsf(e[3]) < 0.4999f;
    return __byte_perm(__byte_perm((uint32_t)t01, (uint32_t)(t01 >> 32), 0x0040),
                       __byte_perm((uint32_t)t23, (uint32_t)(t23 >> 32), 0x0040), 0x5410);
}

// OUTLINE: take the rare exact path through an out-of-line call (keeps a large unrolled caller
// compact; a small grid-stride loop is faster with it inline).
template <bool OUTLINE = false>
__device__ __forceinline__ uint32_t codes4(const float *x, float s, float r) {
    bool fast;
    uint32_t w = codes4_fast(x, r, fast);
    if (!fast) {
        if constexpr (OUTLINE) {
            w = codes4_exact(x[0], x[1], x[2], x[3], s, r);
        } else {
            w = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) w |= (uint32_t)(code_of(x[j], s, r) & 0xff) << (8 * j);
        }
    }
    return w;
}

// Codes of four values under a calibrated scale s, which need not cover them: each value is first
// clamped to +-c, c = RN(127 * s).  A value inside is unchanged; one at or beyond c has a
// quotient of at least 127 * (1 - 2^-24), so its code is +-127 before and after the clamp; and
// |clamped * r| <= 127 * (1 + 2^-24)^2 stays in codes4's range.
template <bool OUTLINE = false>
__device__ __forceinline__ uint32_t codes4_sat(const float *x, float s, float r, float c) {
    float y[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) y[j] = fminf(fmaxf(x[j], -c), c);
    return codes4<OUTLINE>(y, s, r);
}

// A calibrated per-tensor scale as read by every thread: a negative or non-finite value counts as
// zero (zero codes) and, where `report`, sets SGD_STATUS_BAD_SCALE.
__device__ __forceinline__ float calibrated_scale(const float *p, int32_t *status, bool report) {
    const float s = __ldg(p);
    if (s >= 0.f && s <= 3.402823466e38f) return s;
    if (report) atomicOr(status, SGD_STATUS_BAD_SCALE);
    return 0.f;
}

template <int VE, bool SAT = false>
__device__ __forceinline__ void store_codes(int8_t *dst, const float (&x)[VE], float s, float r, float c = 0.f) {
    uint32_t w[VE / 4];
#pragma unroll
    for (int i = 0; i < VE / 4; ++i) {
        if constexpr (SAT)
            w[i] = (s != 0.f) ? codes4_sat(x + 4 * i, s, r, c) : 0u;
        else
            w[i] = (s != 0.f) ? codes4(x + 4 * i, s, r) : 0u;
    }
    if constexpr (VE == 8)
        *reinterpret_cast<uint2 *>(dst) = make_uint2(w[0], w[1]);
    else
        *reinterpret_cast<uint32_t *>(dst) = w[0];
}

}  // namespace sgd
