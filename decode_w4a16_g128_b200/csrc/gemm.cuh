// gemm.cuh - tcgen05 tensor-core W4A16 GEMM for M > 8 (prefill).
//
// Role in the layer: tiny-llm "Week 2 Day 6: SIMD-Matrix Prefill", Task 1,
// routes M > 8 to a tiled matrix kernel; Task 3 hoists one scale and bias per
// 128-group and reuses them across that group's reduction tiles.  This is a
// B200 design with 5th-generation tensor cores, not that 32x32x32 Metal tile.
//
// One CTA computes a BM x BN = 128 x 128 tile of y (128 rows of x, 128 rows
// of W) over a contiguous range of 128-groups (all of K, or one split).  Per
// group:
//   * warp 0 (one thread) TMA-loads the x tile [128 x 128] BF16 as two
//     64-column boxes with the 128-byte swizzle (the K-major operand layout
//     of the tensor cores), and the packed codes [128 rows x 16 words];
//   * warps 2-5 turn the codes into the BF16 values 128 + q (exact) and write
//     them into the swizzled K-major B tile; rows 128..143 of every B tile hold
//     BF16 1.0 once and for all;
//   * warp 1 (one thread) issues 8 tcgen05.mma (M=128, N=144, K=16) into a
//     fresh TMEM accumulator (two buffers alternate), so columns 0..127 hold
//     P' = sum_k x (128 + q) and columns 128..143 hold X = sum_k x of the group;
//   * warps 6-13 read the accumulator (tcgen05.ld) and add
//     s * P' + (b - 128 s) * X to FP32 running sums in registers: the group's
//     scale and bias are applied once per (group, output), in FP32.
// At the end every epilogue thread owns one row of y and 64 columns.
//
// Every product is exact (integer codes, BF16 x); only FP32 sums round, so the
// result matches the plain FP32 definition within the one-ulp tolerance.
#pragma once

#include "ptx.cuh"

namespace w4a16 {
namespace gm {

constexpr int BM = 128;                 // x rows per tile (MMA M)
constexpr int BN = 128;                 // W rows per tile
constexpr int NMMA = BN + 16;           // MMA N: 16 rows of ones append the group sums of x
constexpr int kXStages = 2;
constexpr int kWStages = 4;
constexpr int kBStages = 2;
constexpr int kSBSlots = 4;
constexpr int kAccBufs = 2;
constexpr int kXAtom = BM * 128;        // one 64-column swizzled atom of x: 16 KB
constexpr int kXBytes = 2 * kXAtom;     // 32 KB
constexpr int kWBytes = BN * 64;        // packed codes of one group: 8 KB
constexpr int kBAtom = NMMA * 128;      // one 64-k atom of B: 18 KB
constexpr int kBBytes = 2 * kBAtom;     // 36 KB
constexpr int kSBBytes = BN * 8;        // (s, b - 128 s) per row as FP32
constexpr int kWarpTma = 0, kWarpMma = 1, kWarpDeq = 2, kDeqWarps = 4, kWarpEpi = 6, kEpiWarps = 8;
constexpr int kThreads = (kWarpEpi + kEpiWarps) * 32;   // 448
constexpr int kTmemCols = 512;          // power of two >= kAccBufs * kAccStride
constexpr int kAccStride = 256;         // TMEM columns between the accumulator buffers

constexpr int kOffX = 0;
constexpr int kOffB = kOffX + kXStages * kXBytes;
constexpr int kOffW = kOffB + kBStages * kBBytes;
constexpr int kOffSB = kOffW + kWStages * kWBytes;
constexpr int kOffBar = kOffSB + kSBSlots * kSBBytes;
constexpr int kNumBars = 2 * kXStages + 2 * kWStages + 2 * kBStages + 2 * kSBSlots + 2 * kAccBufs;
constexpr int kSmemBytes = kOffBar + kNumBars * 8 + 16 + 1024;   // + TMEM address, + alignment slack
static_assert(kOffB % 1024 == 0 && kBAtom % 1024 == 0 && kXAtom % 1024 == 0, "swizzled tiles need 1 KB alignment");
// Split-K partial tile [BM][kPartStride] FP32, reusing the B stages once the main loop
// is over; rows padded to 132 floats so that 8 threads storing 8 rows hit 8 bank groups.
constexpr int kPartStride = BN + 4;
constexpr int kOffPart = kOffB;
static_assert(BM * kPartStride * 4 <= kBStages * kBBytes, "partial tile must fit in the B stages");
constexpr int kMaxSplits = 8;           // portable cluster size

struct Params {
    const uint16_t *scales;   // bf16 [N, G]
    const uint16_t *biases;   // bf16 [N, G]
    uint16_t *y;              // bf16 [M, N]
    int M, N, G;
    int splits;               // K splits (gridDim.x, the cluster size)
};

__device__ __forceinline__ uint32_t bf16x2_plus128(uint32_t v, uint32_t v4, uint32_t sel) {
    // bytes sel of (v, v >> 4) -> two low nibbles in bits 0-3 and 16-19 -> BF16 128 + code
    return codes_to_bf16x2_plus128(prmt(v, v4, sel));
}

__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
    uint64_t *x_full = bars, *x_empty = x_full + kXStages;
    uint64_t *w_full = x_empty + kXStages, *w_empty = w_full + kWStages;
    uint64_t *b_full = w_empty + kWStages, *b_empty = b_full + kBStages;
    uint64_t *sb_full = b_empty + kBStages, *sb_empty = sb_full + kSBSlots;
    uint64_t *acc_full = sb_empty + kSBSlots, *acc_empty = acc_full + kAccBufs;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kNumBars);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int split = blockIdx.x, tile_n = blockIdx.y, tile_m = blockIdx.z;   // splits of a tile: one cluster
    const int G = p.G;
    const int g0 = static_cast<int>(static_cast<long long>(split) * G / p.splits);
    const int g1 = static_cast<int>(static_cast<long long>(split + 1) * G / p.splits);
    const int ng = g1 - g0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kXStages; ++i) { mbar_init(&x_full[i], 1); mbar_init(&x_empty[i], 1); }
        for (int i = 0; i < kWStages; ++i) { mbar_init(&w_full[i], 1); mbar_init(&w_empty[i], kDeqWarps); }
        for (int i = 0; i < kBStages; ++i) { mbar_init(&b_full[i], kDeqWarps); mbar_init(&b_empty[i], 1); }
        for (int i = 0; i < kSBSlots; ++i) { mbar_init(&sb_full[i], kDeqWarps); mbar_init(&sb_empty[i], kEpiWarps); }
        for (int i = 0; i < kAccBufs; ++i) { mbar_init(&acc_full[i], 1); mbar_init(&acc_empty[i], kEpiWarps); }
        fence_mbar_init();
    }
    if (warp == kWarpMma) {   // the whole warp allocates the accumulators
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (warp >= kWarpDeq && warp < kWarpDeq + kDeqWarps) {
        // rows 128..143 of every B atom: BF16 1.0, so the MMA also sums x over the group
        const int t = threadIdx.x - kWarpDeq * 32;
        for (int i = t; i < kBStages * 2 * 16 * 8; i += kDeqWarps * 32) {
            const int atom = i / (16 * 8), rem = i - atom * (16 * 8);
            uint4 *dst = reinterpret_cast<uint4 *>(smem + kOffB + atom * kBAtom + (BN + rem / 8) * 128) + (rem % 8);
            *dst = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
        }
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == kWarpTma) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tmap(&tm_x);
            prefetch_tmap(&tm_w);
            pdl_wait();
            constexpr int kLead = kWStages - 1;   // codes run ahead of x: dequantisation comes first
            int wi = 0, xi = 0;
            for (int step = 0; step < ng + kLead; ++step) {
                if (wi < ng) {
                    const int s = wi % kWStages;
                    if (wi >= kWStages && !mbar_wait(&w_empty[s], ((wi / kWStages) - 1) & 1)) break;
                    mbar_arrive_expect_tx(&w_full[s], kWBytes);
                    tma_load_2d(smem + kOffW + s * kWBytes, &tm_w, &w_full[s], (g0 + wi) * 16, tile_n * BN);
                    ++wi;
                }
                if (step >= kLead && xi < ng) {
                    const int s = xi % kXStages;
                    if (xi >= kXStages && !mbar_wait(&x_empty[s], ((xi / kXStages) - 1) & 1)) break;
                    mbar_arrive_expect_tx(&x_full[s], kXBytes);
                    uint8_t *dst = smem + kOffX + s * kXBytes;
                    tma_load_2d(dst, &tm_x, &x_full[s], (g0 + xi) * 128, tile_m * BM);
                    tma_load_2d(dst + kXAtom, &tm_x, &x_full[s], (g0 + xi) * 128 + 64, tile_m * BM);
                    ++xi;
                }
            }
            // leave no copy in flight
            for (int i = max(0, wi - kWStages); i < wi; ++i)
                mbar_wait(&w_full[i % kWStages], (i / kWStages) & 1, false);
            for (int i = max(0, xi - kXStages); i < xi; ++i)
                mbar_wait(&x_full[i % kXStages], (i / kXStages) & 1, false);
        }
    } else if (warp == kWarpMma) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_bf16(BM, NMMA);
            for (int gi = 0; gi < ng; ++gi) {
                const int xs = gi % kXStages, bs = gi % kBStages, buf = gi % kAccBufs;
                if (!mbar_wait(&x_full[xs], (gi / kXStages) & 1)) break;
                if (!mbar_wait(&b_full[bs], (gi / kBStages) & 1)) break;
                if (gi >= kAccBufs && !mbar_wait(&acc_empty[buf], ((gi / kAccBufs) - 1) & 1)) break;
                tc_fence_after();
                const uint32_t a0 = smem_u32(smem + kOffX + xs * kXBytes);
                const uint32_t b0 = smem_u32(smem + kOffB + bs * kBBytes);
                const uint32_t d = tmem_base + buf * kAccStride;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t koff = (kk & 3) * 32;   // 16 BF16 of K inside a 64-column atom
                    const uint64_t ad = umma_desc_sw128(a0 + (kk >> 2) * kXAtom + koff);
                    const uint64_t bd = umma_desc_sw128(b0 + (kk >> 2) * kBAtom + koff);
                    umma_bf16(d, ad, bd, idesc, kk > 0);
                }
                umma_commit(&x_empty[xs]);
                umma_commit(&b_empty[bs]);
                umma_commit(&acc_full[buf]);
            }
        }
    } else if (warp < kWarpEpi) {
        // ------------------------------------------------------------ dequantisation
        const int t = threadIdx.x - kWarpDeq * 32;   // 0..127
        const long long row_sb = static_cast<long long>(tile_n) * BN + t;   // scale/bias row of this thread
        for (int gi = 0; gi < ng; ++gi) {
            const int g = g0 + gi;
            // this thread's scale and bias, issued early
            uint16_t sbits = 0, bbits = 0;
            if (row_sb < p.N) {
                sbits = __ldg(p.scales + row_sb * G + g);
                bbits = __ldg(p.biases + row_sb * G + g);
            }
            const int ws = gi % kWStages, bs = gi % kBStages, ss = gi % kSBSlots;
            if (!mbar_wait(&w_full[ws], (gi / kWStages) & 1)) break;
            if (gi >= kBStages && !mbar_wait(&b_empty[bs], ((gi / kBStages) - 1) & 1)) break;
            const uint8_t *wsrc = smem + kOffW + ws * kWBytes;
            uint8_t *bdst = smem + kOffB + bs * kBBytes;
#pragma unroll
            for (int pass = 0; pass < 4; ++pass) {
                // item = 16 bytes (32 codes) of one row: rows 32*pass + t/4, quarter t%4
                const int row = 32 * pass + (t >> 2), q = t & 3;
                const uint4 v = *reinterpret_cast<const uint4 *>(wsrc + row * 64 + q * 16);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t vv = w[c], v4 = vv >> 4;
                    // chunk 4q + c of the group's 16 chunks of 8 k: atom (4q+c)/8, chunk j in the atom
                    const int chunk = 4 * q + c, atom = chunk >> 3, j = chunk & 7;
                    uint4 o;
                    o.x = bf16x2_plus128(vv, v4, 0x0400u);   // k0, k1
                    o.y = bf16x2_plus128(vv, v4, 0x0501u);   // k2, k3
                    o.z = bf16x2_plus128(vv, v4, 0x0602u);   // k4, k5
                    o.w = bf16x2_plus128(vv, v4, 0x0703u);   // k6, k7
                    *reinterpret_cast<uint4 *>(bdst + atom * kBAtom + row * 128 + ((j ^ (row & 7)) << 4)) = o;
                }
            }
            fence_proxy_async_smem();   // the tensor cores read B through the async proxy
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&w_empty[ws]);
                mbar_arrive(&b_full[bs]);
            }
            // scale and bias for the epilogue
            if (gi >= kSBSlots && !mbar_wait(&sb_empty[ss], ((gi / kSBSlots) - 1) & 1)) break;
            const float sc = bf16_to_f32(sbits);
            reinterpret_cast<float2 *>(smem + kOffSB + ss * kSBBytes)[t] =
                make_float2(sc, fmaf(-128.f, sc, bf16_to_f32(bbits)));
            __syncwarp();
            if (lane == 0) mbar_arrive(&sb_full[ss]);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int e = warp - kWarpEpi;           // 0..7
        const int quarter = warp & 3;            // TMEM lanes this warp may access
        const int half = e >> 2;                 // columns [64 half, 64 half + 64)
        const int m = tile_m * BM + quarter * 32 + lane;
        float acc[64];
#pragma unroll
        for (int j = 0; j < 64; ++j) acc[j] = 0.f;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
        for (int gi = 0; gi < ng; ++gi) {
            const int buf = gi % kAccBufs, ss = gi % kSBSlots;
            if (!mbar_wait(&acc_full[buf], (gi / kAccBufs) & 1)) break;
            tc_fence_after();
            if (!mbar_wait(&sb_full[ss], (gi / kSBSlots) & 1)) break;
            const float2 *sb = reinterpret_cast<const float2 *>(smem + kOffSB + ss * kSBBytes) + 64 * half;
            const uint32_t col0 = lane_base + buf * kAccStride;
            const float X = __uint_as_float(tmem_ld1(col0 + BN));
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t r[32];
                tmem_ld32(col0 + 64 * half + 32 * h, r);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float2 c = sb[32 * h + j];
                    acc[32 * h + j] = fmaf(c.y, X, fmaf(c.x, __uint_as_float(r[j]), acc[32 * h + j]));
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&acc_empty[buf]);
                mbar_arrive(&sb_empty[ss]);
            }
        }
        if (p.splits > 1) {
            // split-K: publish this CTA's partial tile; the cluster reduces it below
            float *part = reinterpret_cast<float *>(smem + kOffPart);
            const int rl = quarter * 32 + lane;
#pragma unroll
            for (int c = 0; c < 16; ++c)
                *reinterpret_cast<float4 *>(part + rl * kPartStride + 64 * half + 4 * c) =
                    make_float4(acc[4 * c], acc[4 * c + 1], acc[4 * c + 2], acc[4 * c + 3]);
        } else if (m < p.M) {
            // store: row m, columns n0 .. n0 + 63
            const long long n0 = static_cast<long long>(tile_n) * BN + 64 * half;
            uint16_t *dst = p.y + static_cast<long long>(m) * p.N + n0;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const long long n = n0 + 8 * c;
                if (n + 8 <= p.N && ((p.N & 7) == 0)) {
                    uint4 v;
                    v.x = pack_bf16x2(acc[8 * c + 0], acc[8 * c + 1]);
                    v.y = pack_bf16x2(acc[8 * c + 2], acc[8 * c + 3]);
                    v.z = pack_bf16x2(acc[8 * c + 4], acc[8 * c + 5]);
                    v.w = pack_bf16x2(acc[8 * c + 6], acc[8 * c + 7]);
                    *reinterpret_cast<uint4 *>(dst + 8 * c) = v;
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        if (n + j < p.N) dst[8 * c + j] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[8 * c + j]));
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }

    if (p.splits > 1) {
        // Split-K reduction over the cluster (the S splits of this tile): CTA rank r sums
        // rows [r*R, (r+1)*R) of the S partial tiles, in rank order, through distributed
        // shared memory, and writes them to y.
        cluster_sync_all();
        const int S = p.splits;
        const uint32_t rank = cluster_ctarank();
        const int rows_per = (BM + S - 1) / S;
        const int r_lo = static_cast<int>(rank) * rows_per;
        const int r_hi = min(BM, r_lo + rows_per);
        const uint32_t part0 = smem_u32(smem + kOffPart);
        for (int item = threadIdx.x; item < (r_hi - r_lo) * (BN / 4); item += kThreads) {
            const int rl = r_lo + item / (BN / 4), c4 = item % (BN / 4);
            const uint32_t off = part0 + (rl * kPartStride + 4 * c4) * 4;
            float4 v = ld_dsmem_f4(dsmem_addr(off, 0));
            for (int sp = 1; sp < S; ++sp) {
                const float4 w = ld_dsmem_f4(dsmem_addr(off, sp));
                v.x += w.x; v.y += w.y; v.z += w.z; v.w += w.w;
            }
            const long long mrow = static_cast<long long>(tile_m) * BM + rl;
            const long long n = static_cast<long long>(tile_n) * BN + 4 * c4;
            if (mrow < p.M) {
                uint16_t *dst = p.y + mrow * p.N + n;
                if (n + 4 <= p.N && (p.N & 3) == 0) {
                    *reinterpret_cast<uint2 *>(dst) = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
                } else {
                    const float vv[4] = {v.x, v.y, v.z, v.w};
                    for (int j = 0; j < 4; ++j)
                        if (n + j < p.N) dst[j] = __bfloat16_as_ushort(__float2bfloat16_rn(vv[j]));
                }
            }
        }
        cluster_sync_all();   // no CTA leaves while another still reads its shared memory
    }
}

}  // namespace gm
}  // namespace w4a16
