// rows.cuh - row-block W4A16 matvec for M <= 8 (decode), no split of K across CTAs.
//
// Role in the layer: tiny-llm "Week 2 Day 6: SIMD-Matrix Prefill", Task 1,
// keeps a matvec schedule for M <= 8; Task 3 applies one scale and bias per
// 128-group.  This is a B200 design, not that Metal kernel.
//
// Why a second matvec: in a stream of back-to-back decode projections a call's
// time is mostly latency (the previous call's completion, x, a cross-CTA
// fix-up), not bytes.  Here every CTA owns R = 8 n_oct whole weight rows over
// the whole of K, so no partial sum leaves the CTA, and its codes, scales and
// biases (at most ~100 KB) are all fetched by TMA / bulk copies at the start.
// With the static-weights flag that happens before the dependency wait, and
// since a CTA takes under half of an SM, the next call's CTAs become resident
// beside this call's and fetch their weights while this one computes.
//
// Layout in shared memory:
//   codes  ceil(G/2) boxes of [R rows x 128 bytes] (32 code words: two groups),
//          128-byte swizzle (16-byte chunk c of row r stored at c ^ (r & 7))
//   scales [R][G] BF16, biases [R][G] BF16 (contiguous rows of the inputs)
//   after the main loop the codes area holds the compute warps' partial sums
//
// Compute: m16n8k16 BF16 tensor-core MMAs with x as A (16 rows, the M <= 8
// activation rows then zeros) and the codes as B (16 k x 8 weight rows), one
// warp per contiguous range of groups.  Codes enter as the exact BF16 values
// 128 + q; for each group and weight row the MMA yields P' = P + 128 X, with
// X the group sum of x (from MMAs of x against ones), and the epilogue adds
// s P' + (b - 128 s) X in FP32.  Per lane (m = lane / 4, t = lane % 4) and
// group: four code words 4t .. 4t+3 of its weight row and the same 32 k of x
// row m; word q, nibble pairs (0,4),(1,5) feed MMA 2q and (2,6),(3,7) MMA
// 2q+1, with x permuted to match (any permutation of k shared by A and B
// leaves the dot product unchanged).
//
// The partial sums of the compute warps are added in warp order (deterministic).
#pragma once

#include "ptx.cuh"

namespace w4a16 {
namespace mvr {

constexpr int kMaxM = 8;
constexpr int kComputeWarps = 8;
constexpr int kThreads = (1 + kComputeWarps) * 32;   // warp 0: producer
constexpr int kMaxOct = 9;                           // weight-row octets per CTA: R <= 72
constexpr int kBudget = 110 * 1024;                  // shared memory per CTA: two CTAs per SM
constexpr uint32_t kBarReduce = 1;                   // named barrier of the compute warps

__host__ __device__ constexpr int boxes(int G) { return (G + 1) / 2; }
__host__ __device__ constexpr long long codes_bytes(int noct, int G) { return 8ll * noct * 128 * boxes(G); }
__host__ __device__ constexpr long long sb_bytes(int noct, int G) {   // scales or biases, 16-byte rounded
    return (16ll * noct * G + 15) / 16 * 16;
}
__host__ __device__ constexpr long long red_bytes(int noct) { return 4ll * kComputeWarps * 8 * noct * kMaxM; }
__host__ __device__ constexpr long long smem_bytes(int noct, int G) {
    const long long work = codes_bytes(noct, G) > red_bytes(noct) ? codes_bytes(noct, G) : red_bytes(noct);
    return work + 2 * sb_bytes(noct, G) + 8ll * (boxes(G) + 1) + 1024;   // + barriers + alignment slack
}

// Octets per CTA for an N x K matrix on `sms` SMs: as few CTAs as cover the rows in
// one pass, at most two per SM; 0 if no such split fits the budget (the stream-K
// matvec serves that size).
__host__ __device__ constexpr int plan_octets(long long N, long long K, int sms) {
    if (N <= 0 || K <= 0 || sms <= 0) return 0;
    const long long oct = (N + 7) / 8;
    const int G = static_cast<int>(K / 128);
    const long long hi = (oct + sms - 1) / sms;               // one CTA per SM
    const long long lo = (oct + 2ll * sms - 1) / (2ll * sms);  // two CTAs per SM
    for (long long n = hi < kMaxOct ? hi : kMaxOct; n >= lo && n >= 1; --n)
        if (smem_bytes(static_cast<int>(n), G) <= kBudget) return static_cast<int>(n);
    return 0;
}

struct Params {
    const uint16_t *x;        // bf16 [M, K]
    const uint16_t *scales;   // bf16 [N, G]
    const uint16_t *biases;   // bf16 [N, G]
    uint16_t *y;              // bf16 [M, N]
    int M, N, K, G;
    int noct;                 // weight-row octets per CTA (R = 8 noct)
    int static_weights;       // codes, scales and biases may be read before the dependency wait
};

// BF16 pair (lo, hi) of two words' low / high halves
__device__ __forceinline__ uint32_t lo_halves(uint32_t a, uint32_t b) { return prmt(a, b, 0x5410u); }
__device__ __forceinline__ uint32_t hi_halves(uint32_t a, uint32_t b) { return prmt(a, b, 0x7632u); }

// D += A B with A = x fragment (rows m, m+8: a1 = a3 = 0) and B = (b0, b1); d2, d3 stay 0
__device__ __forceinline__ void mma_x(float (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
    const uint32_t a[4] = {a0, 0u, a2, 0u};
    mma_bf16_16816(d, a, b0, b1, d);
}

// Two CTAs per SM: 2 x 288 threads x 112 registers <= 65536.
__global__ void __maxnreg__(112)
    rows_kernel(const __grid_constant__ CUtensorMap tm_w, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int G = p.G, noct = p.noct, R = 8 * noct;
    const int nbox = boxes(G);
    const long long cbytes = codes_bytes(noct, G) > red_bytes(noct) ? codes_bytes(noct, G) : red_bytes(noct);
    uint16_t *sc = reinterpret_cast<uint16_t *>(smem + cbytes);
    uint16_t *bi = reinterpret_cast<uint16_t *>(smem + cbytes + sb_bytes(noct, G));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + cbytes + 2 * sb_bytes(noct, G));
    uint64_t *box_full = bars, *sb_full = bars + nbox;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long r0 = static_cast<long long>(blockIdx.x) * R;   // first weight row of this CTA

    if (threadIdx.x == 0) {
        pdl_launch_dependents();   // the next call may start fetching its weights
        for (int b = 0; b <= nbox; ++b) mbar_init(&bars[b], 1);
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == 0) {
        // ------------------------------------------------------------ producer (one thread)
        if (lane != 0) return;
        prefetch_tmap(&tm_w);
        if (!p.static_weights) pdl_wait();
        // scales and biases of rows r0 .. r0+R-1: one contiguous [rows][G] block each
        const long long rows = max(0ll, min(static_cast<long long>(R), p.N - r0));
        const uint32_t bytes = static_cast<uint32_t>(rows * G * 2);
        const uint32_t bulk = bytes & ~15u;
        for (uint32_t e = bulk / 2; e < bytes / 2; ++e) {   // ragged end
            sc[e] = __ldg(p.scales + r0 * G + e);
            bi[e] = __ldg(p.biases + r0 * G + e);
        }
        mbar_arrive_expect_tx(sb_full, 2 * bulk);
        if (bulk) {
            bulk_load(sc, p.scales + r0 * G, bulk, sb_full);
            bulk_load(bi, p.biases + r0 * G, bulk, sb_full);
        }
        // codes: box b = words 32 b .. 32 b + 31 of rows r0 .. r0+R-1 (zeros past N and K)
        for (int b = 0; b < nbox; ++b) {
            mbar_arrive_expect_tx(&box_full[b], static_cast<uint32_t>(R) * 128);
            tma_load_2d(smem + static_cast<long long>(b) * R * 128, &tm_w, &box_full[b], 32 * b, static_cast<int>(r0));
        }
        // leave no copy in flight
        for (int b = 0; b <= nbox; ++b) mbar_wait(&bars[b], 0, /*give_up_on_status=*/false);
        return;
    }

    // ---------------------------------------------------------------- compute warps
    const int w = warp - 1;
    const int m = lane >> 2, t = lane & 3;   // x row (A row, D row); thread in quad
    const bool live = m < p.M;
    const int ga = w * G / kComputeWarps, gb = (w + 1) * G / kComputeWarps;   // this warp's groups
    float out[kMaxOct][2];
#pragma unroll
    for (int o = 0; o < kMaxOct; ++o) out[o][0] = out[o][1] = 0.f;
    constexpr uint32_t kOnes = 0x3F803F80u;   // BF16 (1.0, 1.0)
    pdl_wait();   // x may come from the preceding kernel
    bool ok = ga >= gb || mbar_wait(sb_full, 0);
    const uint4 *xrow = reinterpret_cast<const uint4 *>(p.x + static_cast<long long>(live ? m : 0) * p.K);
    uint4 xv[4];
    if (ok && ga < gb) {
#pragma unroll
        for (int q = 0; q < 4; ++q) xv[q] = live ? __ldg(xrow + 16 * ga + 4 * t + q) : make_uint4(0, 0, 0, 0);
    }
    const uint32_t cbase = smem_u32(smem);
    for (int g = ga; ok && g < gb; ++g) {
        // A fragments of this group (x permuted like the codes), and the next group's x
        uint32_t a[4][2][2];   // [word q][MMA 2q + h][a0, a2]
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            a[q][0][0] = lo_halves(xv[q].x, xv[q].z);   // x0, x4
            a[q][0][1] = hi_halves(xv[q].x, xv[q].z);   // x1, x5
            a[q][1][0] = lo_halves(xv[q].y, xv[q].w);   // x2, x6
            a[q][1][1] = hi_halves(xv[q].y, xv[q].w);   // x3, x7
        }
        if (g + 1 < gb) {
#pragma unroll
            for (int q = 0; q < 4; ++q) xv[q] = live ? __ldg(xrow + 16 * (g + 1) + 4 * t + q) : make_uint4(0, 0, 0, 0);
        }
        // group sum of x row m (every column of D holds it)
        float xs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int h = 0; h < 2; ++h) mma_x(xs, a[q][h][0], a[q][h][1], kOnes, kOnes);
        const float X = xs[0];
        if (((g - ga) == 0 || (g & 1) == 0) && !mbar_wait(&box_full[g >> 1], 0)) { ok = false; break; }
        // chunk 4 (g % 2) + t of row 8 o + m in box g / 2, swizzled by the row's low bits (= m)
        const uint32_t cw = cbase + static_cast<uint32_t>(g >> 1) * R * 128 + m * 128 +
                            ((static_cast<uint32_t>(4 * (g & 1) + t) ^ static_cast<uint32_t>(m)) << 4);
#pragma unroll
        for (int o = 0; o < kMaxOct; ++o) {
            if (o >= noct) break;
            const uint4 c = lds128(cw + o * 8 * 128);
            const uint32_t cw4[4] = {c.x, c.y, c.z, c.w};
            float pa[4] = {0.f, 0.f, 0.f, 0.f}, pb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t v = cw4[q];
                mma_x(pa, a[q][0][0], a[q][0][1], codes_to_bf16x2_plus128(v), codes_to_bf16x2_plus128(v >> 4));
                mma_x(pb, a[q][1][0], a[q][1][1], codes_to_bf16x2_plus128(v >> 8), codes_to_bf16x2_plus128(v >> 12));
            }
            // weight rows 8 o + 2 t, 8 o + 2 t + 1 of this CTA
            const int n0 = 8 * o + 2 * t;
            const float s0 = bf16_to_f32(sc[n0 * G + g]), s1 = bf16_to_f32(sc[(n0 + 1) * G + g]);
            const float b0 = fmaf(-128.f, s0, bf16_to_f32(bi[n0 * G + g]));
            const float b1 = fmaf(-128.f, s1, bf16_to_f32(bi[(n0 + 1) * G + g]));
            out[o][0] = fmaf(b0, X, fmaf(s0, pa[0] + pb[0], out[o][0]));
            out[o][1] = fmaf(b1, X, fmaf(s1, pa[1] + pb[1], out[o][1]));
        }
    }
    // ---------------------------------------------------------------- fixed-order sum over warps
    named_bar_sync(kBarReduce, kComputeWarps * 32);   // every warp is done with the codes
    float *red = reinterpret_cast<float *>(smem);     // [warp][row n < R][x row m < 8]
#pragma unroll
    for (int o = 0; o < kMaxOct; ++o) {
        if (o >= noct) break;
        const int n0 = 8 * o + 2 * t;
        red[(w * R + n0) * kMaxM + m] = out[o][0];
        red[(w * R + n0 + 1) * kMaxM + m] = out[o][1];
    }
    named_bar_sync(kBarReduce, kComputeWarps * 32);
    for (int i = threadIdx.x - 32; i < R * p.M; i += kComputeWarps * 32) {
        const int n = i / p.M, mm = i - n * p.M;
        float v = 0.f;
#pragma unroll
        for (int ww = 0; ww < kComputeWarps; ++ww) v += red[(ww * R + n) * kMaxM + mm];
        if (r0 + n < p.N) p.y[static_cast<long long>(mm) * p.N + r0 + n] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
    }
}

}  // namespace mvr
}  // namespace w4a16
