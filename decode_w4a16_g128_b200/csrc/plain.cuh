// plain.cuh - the layer's plain definition for one output, the kernels' path for outputs whose
// fast result is not finite.
//
// Every kernel computes a group's contribution as (s / 8) P8 + (b - 16 s) X with
// P8 = sum (128 + 8 q) x and X = sum x: exact integer codes on the tensor cores, one FP32
// scale and shifted bias per group (tiny-llm "Week 2 Day 6: SIMD-Matrix Prefill", Task 3: one
// scale and bias per 128 reduction values).  P8 and X are up to 248 x 128 times larger than
// x itself, so for |x| beyond about 2^113 they can overflow FP32 where the plain sum does
// not, and two overflowed terms of opposite sign give NaN.  An intermediate overflow
// always leaves the final FP32 value infinite or NaN, so each kernel checks the value it is
// about to round and, when it is not finite, recomputes that output here: w = s q + b, then
// acc += x w over ascending k, every product and sum rounded to FP32 on its own (no fused
// multiply-add).  This is the definition of y itself; on ordinary data it never runs.
#pragma once

#include <cstdint>

namespace w4a16 {

__device__ __forceinline__ float plain_output(const uint16_t *x_row, const uint32_t *wq_row, const uint16_t *s_row,
                                           const uint16_t *b_row, int G) {
    float acc = 0.f;
    for (int g = 0; g < G; ++g) {
        const float s = __uint_as_float(static_cast<uint32_t>(s_row[g]) << 16);
        const float b = __uint_as_float(static_cast<uint32_t>(b_row[g]) << 16);
        for (int j = 0; j < 16; ++j) {
            const uint32_t word = wq_row[g * 16 + j];
            for (int i = 0; i < 8; ++i) {
                const float q = static_cast<float>((word >> (4 * i)) & 15u);
                const float w = __fadd_rn(__fmul_rn(s, q), b);
                const float x = __uint_as_float(static_cast<uint32_t>(x_row[g * 128 + 8 * j + i]) << 16);
                acc = __fadd_rn(acc, __fmul_rn(x, w));
            }
        }
    }
    return acc;
}

}  // namespace w4a16
