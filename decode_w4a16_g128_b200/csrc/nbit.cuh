// nbit.cuh - the affine group-128 layer with 2- or 8-bit codes, M <= 8 (decode).
//
// Role in the layer: the "Route affine qmv_wide by bit-width and batch size" PR routes the
// affine format by its bit width and holds a group's dequantised weights in registers across
// the M activation rows; tiny-llm "Week 2 Day 6: SIMD-Matrix Prefill", Task 3, applies one
// scale and bias per 128 reduction values.  With b-bit codes a uint32 holds 32 / b of them,
// the lowest in the lowest bits; scales and biases are the 4-bit format's.
//
// Compute: the 4-bit row-block kernel's factorisation.  m16n8k16 BF16 MMAs take the CODES as
// A (16 weight rows x 16 k) and x as B (16 k x the M <= 8 activation rows), with codes entered
// as exact BF16 values off + step q, so that one group of one row gives
//   P = sum (off + step q) x = off X + step sum q x,     X = sum x (MMAs against all-ones A)
//   contribution = s sum q x + b X = (s / step) P + (b - (off / step) s) X.
//   2 bits: off 128, step 32: BF16 128.0 (0x4300) with the code in mantissa bits 5-6.
//   8 bits: the two nibbles h, l of a code as two A operands on one accumulator, h as
//           2048 + 128 h (0x4500, mantissa bits 3-6) and l as 128 + 8 l (0x4300, bits 3-6):
//           their sum is 2176 + 8 q, so off 2176, step 8.
// Every value off + step q is an integer below 2^12 with at most 8 significant bits, so it is
// exact in BF16; its products with BF16 x are exact in FP32.
//
// Schedule: a CTA owns RB row blocks of 16 rows and all of K; its 8 warps take contiguous,
// equal runs of the groups.  Lane (g, t) = (lane / 4, lane % 4) reads k = 32 t .. 32 t + 31
// of a group for rows g and g + 8 of every row block (b words per row: one 8-byte load for 2
// bits, two 16-byte loads for 8 bits) and the same 32 k of x row g (four 16-byte loads).  A
// permutation of k shared by A and B leaves the dot products unchanged, so each lane pairs
// codes and x values in whatever order its words hold them.  The codes, scales and biases
// of D groups are in flight per warp; the warps' partial sums are added in warp order
// through shared memory, so the result does not depend on timing.  The kernel has no waits
// besides the CTA barriers and the dependency wait on the preceding kernel.
#pragma once

#include "ptx.cuh"

namespace w4a16 {

// The layer's plain definition for one output with b-bit codes (b = 2 or 8; 32 / b codes per word,
// the lowest code in the lowest bits), the path for outputs whose fast result is not finite:
// w = s q + b, then acc += x w over ascending k, every product and sum rounded on its own.
template <int BITS>
__device__ __forceinline__ float plain_output_bits(const uint16_t *x_row, const uint32_t *wq_row, const uint16_t *s_row,
                                                const uint16_t *b_row, int G) {
    constexpr int kPer = 32 / BITS;
    constexpr uint32_t kMask = (1u << BITS) - 1u;
    float acc = 0.f;
    for (int g = 0; g < G; ++g) {
        const float s = __uint_as_float(static_cast<uint32_t>(s_row[g]) << 16);
        const float b = __uint_as_float(static_cast<uint32_t>(b_row[g]) << 16);
        for (int j = 0; j < 4 * BITS; ++j) {
            const uint32_t word = wq_row[g * 4 * BITS + j];
            for (int i = 0; i < kPer; ++i) {
                const float q = static_cast<float>((word >> (BITS * i)) & kMask);
                const float w = __fadd_rn(__fmul_rn(s, q), b);
                const float x = __uint_as_float(static_cast<uint32_t>(x_row[g * 128 + kPer * j + i]) << 16);
                acc = __fadd_rn(acc, __fmul_rn(x, w));
            }
        }
    }
    return acc;
}

namespace nb {

constexpr int kMaxM = 8;
constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;

template <int BITS>
struct Cfg;
template <>
struct Cfg<2> {
    static constexpr int RB = 2;             // row blocks of 16 rows per CTA (x read once for both)
    static constexpr int D = 2;              // groups in flight per warp
    static constexpr float kStep = 32.f;
    static constexpr float kOffOverStep = 4.f;
};
template <>
struct Cfg<8> {
    static constexpr int RB = 1;
    static constexpr int D = 2;
    static constexpr float kStep = 8.f;
    static constexpr float kOffOverStep = 272.f;   // 2176 / 8
};

template <int BITS>
constexpr int rows_per_cta() { return 16 * Cfg<BITS>::RB; }

struct Params {
    const uint16_t *x;        // bf16 [M, K]
    const uint32_t *wq;       // [N, K b / 32] packed codes
    const uint16_t *scales;   // bf16 [N, G]
    const uint16_t *biases;   // bf16 [N, G]
    uint16_t *y;              // bf16 [M, N]
    int M, N, K, G;
};

// (u & mask) | base on two halves at once: codes placed in the mantissa of a BF16 constant
__device__ __forceinline__ uint32_t or_into_2x(uint32_t u, uint32_t mask, uint32_t base) {
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(u), "r"(mask), "r"(base));
    return r;
}

// codes j and j + 8 of a word of 2-bit codes -> BF16 (128 + 32 q_j, 128 + 32 q_{j+8})
template <int J>
__device__ __forceinline__ uint32_t pair2(uint32_t v) {
    constexpr int sh = 5 - 2 * J;                     // bits 2 J and 2 J + 16 to bits 5 and 21
    const uint32_t u = sh >= 0 ? (v << (sh >= 0 ? sh : 0)) : (v >> (sh < 0 ? -sh : 0));
    return or_into_2x(u, 0x00600060u, 0x43004300u);
}

__device__ __forceinline__ uint32_t lo_halves_nb(uint32_t a, uint32_t b) { return prmt(a, b, 0x5410u); }
__device__ __forceinline__ uint32_t hi_halves_nb(uint32_t a, uint32_t b) { return prmt(a, b, 0x7632u); }

__device__ __forceinline__ uint32_t comp(const uint4 &v, int i) {
    return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

// One group's operands of one lane: codes of rows g and g + 8 of each row block, their scales
// and biases, and 32 values of x row g.
template <int BITS>
struct Stage {
    uint32_t c[Cfg<BITS>::RB][2][BITS];
    uint16_t s[Cfg<BITS>::RB][2], b[Cfg<BITS>::RB][2];
    uint4 x[4];
};

template <int BITS>
__device__ __forceinline__ void load_stage(Stage<BITS> &st, const Params &p, int gg, int row0, int g, int t,
                                           bool xlive) {
    constexpr int RB = Cfg<BITS>::RB;
    const long long wpr = static_cast<long long>(p.K) * BITS / 32;   // words per row
#pragma unroll
    for (int rb = 0; rb < RB; ++rb)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int r = row0 + 16 * rb + g + 8 * h;
            const bool live = r < p.N;
            const uint32_t *src = p.wq + static_cast<long long>(live ? r : 0) * wpr + gg * 4 * BITS + BITS * t;
            if constexpr (BITS == 2) {
                const uint2 v = live ? __ldg(reinterpret_cast<const uint2 *>(src)) : make_uint2(0u, 0u);
                st.c[rb][h][0] = v.x;
                st.c[rb][h][1] = v.y;
            } else {
                const uint4 v0 = live ? __ldg(reinterpret_cast<const uint4 *>(src)) : make_uint4(0u, 0u, 0u, 0u);
                const uint4 v1 = live ? __ldg(reinterpret_cast<const uint4 *>(src) + 1) : make_uint4(0u, 0u, 0u, 0u);
                st.c[rb][h][0] = v0.x; st.c[rb][h][1] = v0.y; st.c[rb][h][2] = v0.z; st.c[rb][h][3] = v0.w;
                st.c[rb][h][4] = v1.x; st.c[rb][h][5] = v1.y; st.c[rb][h][6] = v1.z; st.c[rb][h][7] = v1.w;
            }
            const long long sidx = static_cast<long long>(live ? r : 0) * p.G + gg;
            st.s[rb][h] = live ? __ldg(p.scales + sidx) : static_cast<uint16_t>(0);
            st.b[rb][h] = live ? __ldg(p.biases + sidx) : static_cast<uint16_t>(0);
        }
    const uint16_t *xs = p.x + static_cast<long long>(xlive ? g : 0) * p.K + gg * 128 + 32 * t;
#pragma unroll
    for (int q = 0; q < 4; ++q) st.x[q] = xlive ? ldg_v4(xs + 8 * q) : make_uint4(0u, 0u, 0u, 0u);
}

template <int BITS>
__device__ __forceinline__ void compute_stage(const Stage<BITS> &st, float (&out)[Cfg<BITS>::RB][4]) {
    constexpr int RB = Cfg<BITS>::RB;
    constexpr uint32_t kOnes = 0x3F803F80u;          // BF16 (1.0, 1.0)
    const uint32_t ones[4] = {kOnes, kOnes, kOnes, kOnes};
    // B fragments: 8 MMAs of 16 k, two registers each, paired like the codes below
    uint32_t bf[8][2];
    if constexpr (BITS == 2) {
        // MMA (w, jj): x elements 16 w + 2 jj (+ 8) and 16 w + 2 jj + 1 (+ 8) of the lane's 32
#pragma unroll
        for (int w = 0; w < 2; ++w)
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const uint32_t a = comp(st.x[2 * w], jj), b = comp(st.x[2 * w + 1], jj);
                bf[4 * w + jj][0] = lo_halves_nb(a, b);
                bf[4 * w + jj][1] = hi_halves_nb(a, b);
            }
    } else {
        // MMA c: x elements 4 c, 4 c + 2 and 4 c + 1, 4 c + 3 (bytes 0, 2 and 1, 3 of word c)
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const uint32_t a = comp(st.x[c / 2], 2 * (c % 2)), b = comp(st.x[c / 2], 2 * (c % 2) + 1);
            bf[c][0] = lo_halves_nb(a, b);
            bf[c][1] = hi_halves_nb(a, b);
        }
    }
    // group sums of x rows 2t, 2t + 1 (two independent chains)
    float xa[4] = {0.f, 0.f, 0.f, 0.f}, xb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        mma_bf16_16816(xa, ones, bf[2 * c][0], bf[2 * c][1], xa);
        mma_bf16_16816(xb, ones, bf[2 * c + 1][0], bf[2 * c + 1][1], xb);
    }
    const float X0 = xa[0] + xb[0], X1 = xa[1] + xb[1];
#pragma unroll
    for (int rb = 0; rb < RB; ++rb) {
        float da[4] = {0.f, 0.f, 0.f, 0.f}, db[4] = {0.f, 0.f, 0.f, 0.f};
        if constexpr (BITS == 2) {
#pragma unroll
            for (int w = 0; w < 2; ++w) {
                const uint32_t va = st.c[rb][0][w], vb = st.c[rb][1][w];
                float (&d)[4] = w == 0 ? da : db;
                const uint32_t a0[4] = {pair2<0>(va), pair2<0>(vb), pair2<1>(va), pair2<1>(vb)};
                mma_bf16_16816(d, a0, bf[4 * w + 0][0], bf[4 * w + 0][1], d);
                const uint32_t a1[4] = {pair2<2>(va), pair2<2>(vb), pair2<3>(va), pair2<3>(vb)};
                mma_bf16_16816(d, a1, bf[4 * w + 1][0], bf[4 * w + 1][1], d);
                const uint32_t a2[4] = {pair2<4>(va), pair2<4>(vb), pair2<5>(va), pair2<5>(vb)};
                mma_bf16_16816(d, a2, bf[4 * w + 2][0], bf[4 * w + 2][1], d);
                const uint32_t a3[4] = {pair2<6>(va), pair2<6>(vb), pair2<7>(va), pair2<7>(vb)};
                mma_bf16_16816(d, a3, bf[4 * w + 3][0], bf[4 * w + 3][1], d);
            }
        } else {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint32_t va = st.c[rb][0][c], vb = st.c[rb][1][c];
                // low nibbles of bytes (0, 2) and (1, 3) as 128 + 8 l
                const uint32_t al[4] = {or_into_2x(va << 3, 0x00780078u, 0x43004300u),
                                        or_into_2x(vb << 3, 0x00780078u, 0x43004300u),
                                        or_into_2x(va >> 5, 0x00780078u, 0x43004300u),
                                        or_into_2x(vb >> 5, 0x00780078u, 0x43004300u)};
                mma_bf16_16816(da, al, bf[c][0], bf[c][1], da);
                // high nibbles as 2048 + 128 h
                const uint32_t ah[4] = {or_into_2x(va >> 1, 0x00780078u, 0x45004500u),
                                        or_into_2x(vb >> 1, 0x00780078u, 0x45004500u),
                                        or_into_2x(va >> 9, 0x00780078u, 0x45004500u),
                                        or_into_2x(vb >> 9, 0x00780078u, 0x45004500u)};
                mma_bf16_16816(db, ah, bf[c][0], bf[c][1], db);
            }
        }
        // rows g (A row g) and g + 8: (s / step) P + (b - (off / step) s) X
        const float sa = bf16_to_f32(st.s[rb][0]), sb = bf16_to_f32(st.s[rb][1]);
        const float ba = fmaf(-Cfg<BITS>::kOffOverStep, sa, bf16_to_f32(st.b[rb][0]));
        const float bb = fmaf(-Cfg<BITS>::kOffOverStep, sb, bf16_to_f32(st.b[rb][1]));
        const float ssa = sa / Cfg<BITS>::kStep, ssb = sb / Cfg<BITS>::kStep;   // a power of two: exact
        out[rb][0] = fmaf(ba, X0, fmaf(ssa, da[0] + db[0], out[rb][0]));
        out[rb][1] = fmaf(ba, X1, fmaf(ssa, da[1] + db[1], out[rb][1]));
        out[rb][2] = fmaf(bb, X0, fmaf(ssb, da[2] + db[2], out[rb][2]));
        out[rb][3] = fmaf(bb, X1, fmaf(ssb, da[3] + db[3], out[rb][3]));
    }
}

// Two CTAs per SM: 256 threads x 128 registers each.
template <int BITS>
__global__ void __launch_bounds__(kThreads, 2) nbit_kernel(const Params p) {
    constexpr int RB = Cfg<BITS>::RB, D = Cfg<BITS>::D;
    __shared__ float red[kWarps][RB][16][kMaxM];
    pdl_launch_dependents();
    pdl_wait();   // x (and possibly the weights) may come from the preceding kernel
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int row0 = static_cast<int>(blockIdx.x) * 16 * RB;
    const int ga = warp * p.G / kWarps, gb = (warp + 1) * p.G / kWarps;
    const bool xlive = g < p.M;
    float out[RB][4];
#pragma unroll
    for (int rb = 0; rb < RB; ++rb) out[rb][0] = out[rb][1] = out[rb][2] = out[rb][3] = 0.f;
    Stage<BITS> st[D];
#pragma unroll
    for (int j = 0; j < D; ++j)
        if (ga + j < gb) load_stage<BITS>(st[j], p, ga + j, row0, g, t, xlive);
    for (int gi = ga; gi < gb; gi += D) {
#pragma unroll
        for (int j = 0; j < D; ++j) {
            const int gg = gi + j;
            if (gg >= gb) break;
            compute_stage<BITS>(st[j], out);
            if (gg + D < gb) load_stage<BITS>(st[j], p, gg + D, row0, g, t, xlive);
        }
    }
    // C fragment: rows g, g + 8 of each row block, x rows 2t, 2t + 1
#pragma unroll
    for (int rb = 0; rb < RB; ++rb) {
        red[warp][rb][g][2 * t] = out[rb][0];
        red[warp][rb][g][2 * t + 1] = out[rb][1];
        red[warp][rb][g + 8][2 * t] = out[rb][2];
        red[warp][rb][g + 8][2 * t + 1] = out[rb][3];
    }
    __syncthreads();
    constexpr int RC = 16 * RB;
    for (int i = threadIdx.x; i < RC * p.M; i += kThreads) {
        const int m = i / RC, r = i - m * RC;
        const int row = row0 + r;
        if (row >= p.N) continue;
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) v += red[w][r / 16][r % 16][m];
        if (!isfinite(__bfloat162float(__float2bfloat16_rn(v))))   // the plain definition instead
            v = plain_output_bits<BITS>(p.x + static_cast<long long>(m) * p.K,
                                        p.wq + static_cast<long long>(row) * (static_cast<long long>(p.K) * BITS / 32),
                                        p.scales + static_cast<long long>(row) * p.G,
                                        p.biases + static_cast<long long>(row) * p.G, p.G);
        p.y[static_cast<long long>(m) * p.N + row] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
    }
}

}  // namespace nb
}  // namespace w4a16
