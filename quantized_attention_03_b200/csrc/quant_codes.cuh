// INT8 codes of the per-block (or per-token) quantization, shared by the quantization
// kernel and the attention kernel's in-prologue Q quantization, so that both produce the
// same bytes.
//
// 「SageAttention：低比特量化Attention，实现推理加速」, section 技术方案: a block's
// scale is amax / 127 (fp32) and an element's code is the round-half-even integer of the
// fp32 quotient x / scale.
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace sage {

__device__ __forceinline__ void unpack8(const uint4 &u, float (&f)[8])
{
    const __half2 *h = reinterpret_cast<const __half2 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const float2 t = __half22float2(h[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}

constexpr float kRound = 12582912.0f;            // 1.5 * 2^23: adding it rounds to an integer
constexpr int kRoundBits = 0x4B400000;

// round-half-even(fl(x / s)) clamped to [-127, 127], where fl(x / s) is the IEEE fp32
// quotient and r = fl(1 / s). The product x * r is within 2^-15 of fl(x / s) (|x / s| <=
// 127.5 keeps every ulp <= 2^-17), so both round to the same integer unless the product
// lies within 2^-15 of a half-integer; those rare elements take the exact division.
__device__ __forceinline__ int8_t int8_code(float x, float s, float r)
{
    if (s == 0.0f)
        return 0;
    const float q = x * r;
    const float b = q + kRound;                    // RNE integer in the low mantissa bits
    const float d = fabsf(q - (b - kRound));       // distance to that integer, <= 1/2
    int c = __float_as_int(b) - kRoundBits;
    if (d > 0.5f - 3.0517578125e-05f)              // near a tie: exact IEEE quotient
        c = __float2int_rn(__fdiv_rn(x, s));
    c = max(-127, min(127, c));
    return (int8_t)c;
}

// The eight codes int8_code(x, s, r) of x[0..3] (pairs), packed little-endian. The
// product x * r, rounded to an integer by the 1.5 * 2^23 bias, is computed on packed
// fp32 pairs; the code is the low byte of the biased float's bits (their integer part
// is 0x4B400000 + code). No clamp is needed: s = fl(amax / 127) and r = fl(1 / s) give
// |x r| <= 127 (1 + 2^-22) < 127.5. Elements within 2^-15 of a tie are redone with the
// exact quotient (rare).
__device__ __forceinline__ uint2 int8_codes8(const float2 (&x)[4], float s, float r)
{
    if (s == 0.0f)
        return make_uint2(0u, 0u);
    constexpr float kTie = 0.5f - 3.0517578125e-05f;
    uint32_t bits[8];
    bool tie = false;
#pragma unroll
    for (int j = 0; j < 4; j++) {
        const float2 t = mul2(x[j], make_float2(r, r));
        const float2 b = add2(t, make_float2(kRound, kRound));
        const float2 n = add2(b, make_float2(-kRound, -kRound));
        const float2 d = fma2(n, make_float2(-1.0f, -1.0f), t);   // t - round(t), exact
        tie |= (fabsf(d.x) > kTie) | (fabsf(d.y) > kTie);
        bits[2 * j] = __float_as_uint(b.x);
        bits[2 * j + 1] = __float_as_uint(b.y);
    }
    if (tie) {
#pragma unroll
        for (int j = 0; j < 4; j++) {
            bits[2 * j] = (uint8_t)int8_code(x[j].x, s, r);
            bits[2 * j + 1] = (uint8_t)int8_code(x[j].y, s, r);
        }
    }
    uint2 w;
    w.x = __byte_perm(__byte_perm(bits[0], bits[1], 0x0040), __byte_perm(bits[2], bits[3], 0x0040),
                      0x5410);
    w.y = __byte_perm(__byte_perm(bits[4], bits[5], 0x0040), __byte_perm(bits[6], bits[7], 0x0040),
                      0x5410);
    return w;
}

}  // namespace sage
