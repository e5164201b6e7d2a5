// quant.cuh - on-GPU W4 group-128 quantiser: FP32 or BF16 weights -> the packed format the
// layer reads (codes [N, K/8] uint32, scales and biases [N, K/128] BF16).
//
// Role: the step before the layer, a quantised-weights writer on the GPU ("MLX Metal
// Kernels v0.20.0" release notes, "Next roadmap items": a quantized package tensor-data
// writer).  The recipe is the affine min/max quantisation the layer's inputs are defined
// with (the reference problem: scale = (max - min) / 15, bias = min, q = round and clamp
// to 0..15, eight codes per uint32 with k % 8 == 0 in bits 0-3), spelled out per group:
//   lo, hi = min, max of the group's 128 values (a zero lo or hi is taken as +0)
//   scale  = bf16_rne((hi - lo) / 15), bias = bf16_rne(lo)          (FP32 sub and div)
//   q[k]   = 0 if scale == 0, else clamp(rint((w[k] - bias) / scale), 0, 15)
//            with the BF16 scale and bias widened, FP32 sub and IEEE div, rint to even.
// Every step is correctly rounded, so the result is bit-identical to a sequential CPU
// implementation of the same recipe; min and max are order-independent once the sign
// of a zero is fixed.
//
// Shape: the work is a stream (4 or 2 bytes read per weight, 0.53 written), so the kernel
// keeps the instruction count per group low and the loads wide: eight lanes per (row, group)
// pair, lane s of the eight holding k = 16 s .. 16 s + 15 (64 contiguous bytes of FP32, 32
// of BF16; the eight lanes cover the group's 512 or 256 bytes), four pairs per warp.  Min
// and max take three butterfly steps within the eight lanes; each lane writes its own two
// code words (8 contiguous bytes), so the 16 words of a group leave as 64 contiguous bytes.
// A grid of a few CTAs per SM loops over the pairs.
#pragma once

#include "ptx.cuh"

namespace w4a16 {
namespace qz {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kLanesPerPair = 8;
constexpr int kPairsPerWarp = 32 / kLanesPerPair;

// the 16 values k = 16 s .. 16 s + 15 of a group, lane s of its eight
template <bool kBf16>
__device__ __forceinline__ void load16(const void *w, long long idx, float (&v)[16]) {
    if (kBf16) {
        const uint16_t *p = static_cast<const uint16_t *>(w) + idx;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint4 u = ldg_nc_v4(p + 8 * h);
            const uint32_t q[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                v[8 * h + 2 * j] = __uint_as_float(q[j] << 16);
                v[8 * h + 2 * j + 1] = __uint_as_float(q[j] & 0xFFFF0000u);
            }
        }
    } else {
        const float *p = static_cast<const float *>(w) + idx;
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const uint4 u = ldg_nc_v4(p + 4 * h);
            v[4 * h] = __uint_as_float(u.x);
            v[4 * h + 1] = __uint_as_float(u.y);
            v[4 * h + 2] = __uint_as_float(u.z);
            v[4 * h + 3] = __uint_as_float(u.w);
        }
    }
}

template <bool kBf16>
__global__ void __launch_bounds__(kThreads) quantize_kernel(const void *__restrict__ w, uint32_t *__restrict__ wq,
                                                            uint16_t *__restrict__ scales,
                                                            uint16_t *__restrict__ biases, long long N, int K) {
    const int G = K / 128;
    const long long pairs = N * G;
    const int lane = threadIdx.x & 31;
    const int sub = lane & (kLanesPerPair - 1);
    const long long warp = static_cast<long long>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
    const long long stride = static_cast<long long>(gridDim.x) * kWarps * kPairsPerWarp;
    for (long long first = warp * kPairsPerWarp; first < pairs; first += stride) {
        // pair `it` of this lane's eight; the shuffles stay within the eight, and a warp whose
        // last pairs lie past the end repeats its last valid pair (its results are not stored)
        const long long it_raw = first + (lane >> 3);
        const bool live = it_raw < pairs;
        const long long it = live ? it_raw : pairs - 1;
        const long long n = it / G;
        const int g = static_cast<int>(it - n * G);
        float v[16];
        load16<kBf16>(w, n * K + g * 128 + 16 * sub, v);
        float lo = v[0], hi = v[0];
#pragma unroll
        for (int j = 1; j < 16; ++j) {
            lo = fminf(lo, v[j]);
            hi = fmaxf(hi, v[j]);
        }
#pragma unroll
        for (int o = 1; o < kLanesPerPair; o <<= 1) {
            lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
            hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
        }
        if (lo == 0.f) lo = 0.f;   // +0 for either zero
        if (hi == 0.f) hi = 0.f;
        const uint16_t sb = __bfloat16_as_ushort(__float2bfloat16_rn(__fdiv_rn(__fsub_rn(hi, lo), 15.f)));
        const uint16_t bb = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
        const float sc = __uint_as_float(static_cast<uint32_t>(sb) << 16);
        const float bi = __uint_as_float(static_cast<uint32_t>(bb) << 16);
        // t = RN(d / sc) decides the code only through rint(t) and the clamps, which change
        // value only where t crosses a half-integer.  d * RN(1 / sc) lies within two ulps of
        // RN(d / sc) (|t| < 16 here: two ulps < 4e-6), so when it is farther than 1.6e-5 from
        // every half-integer it rounds to the same code; otherwise (and when the reciprocal
        // overflows, for subnormal scales) the correctly rounded division decides.
        const float rc = __frcp_rn(sc);
        uint32_t word[2] = {0u, 0u};
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            uint32_t code = 0u;
            if (sc != 0.f) {
                const float d = __fsub_rn(v[j], bi);
                float t = __fmul_rn(d, rc);
                if (!(fabsf(t) < 1e30f) || fabsf(fabsf(t - rintf(t)) - 0.5f) < 1.6e-5f) t = __fdiv_rn(d, sc);
                const float r = rintf(t);
                code = r < 0.f ? 0u : (r > 15.f ? 15u : static_cast<uint32_t>(r));
            }
            word[j >> 3] |= code << (4 * (j & 7));
        }
        if (live) {
            *reinterpret_cast<uint2 *>(wq + n * (K / 8) + g * 16 + 2 * sub) = make_uint2(word[0], word[1]);
            if (sub == 0) {
                scales[n * G + g] = sb;
                biases[n * G + g] = bb;
            }
        }
    }
}

}  // namespace qz
}  // namespace w4a16
