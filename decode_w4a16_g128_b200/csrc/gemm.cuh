// gemm.cuh - tcgen05 tensor-core W4A16 GEMM for M > 8 (prefill).
//
// Role in the layer: tiny-llm "Week 2 Day 6: SIMD-Matrix Prefill", Task 1,
// routes M > 8 to a tiled matrix kernel; Task 3 hoists one scale and bias per
// 128-group and reuses them across that group's reduction tiles and all rows
// of x.  This is a B200 design with 5th-generation tensor cores, not that
// 32x32x32 Metal tile.
//
// Algebra (exact-integer factorisation, per 128-group g):
//   sum_k x[m,k] w[n,k] = sum_g s[n,g] P'[n,m,g] + sum_g (b[n,g] - 128 s[n,g]) X[m,g],
//   P'[n,m,g] = sum_{k in g} (128 + q[n,k]) x[m,k],   X[m,g] = sum_{k in g} x[m,k].
// 128 + q is an exact BF16 value and x is BF16, so every product of P' is
// exact; only FP32 sums round.
//
// Roles of the operands: the tensor cores compute D[n, m] (TMEM lane = weight
// row n, column = x row m).  The dequantised codes are the A operand and live
// in TENSOR MEMORY: dequantisation warps turn a row's 128 codes of a group into
// 64 columns of BF16 pairs and store them with tcgen05.st, so they never pass
// through shared memory.  x is the B operand, staged by TMA in shared memory
// (128 rows x 128 k per group, 128-byte swizzle).  Each epilogue thread owns one
// weight row, so the group's scale is a per-thread scalar: one FMA per output
// per group, no broadcast of per-column parameters.
//
// The bias term is a small contraction of its own, done on the tensor cores.
// A preparation kernel (prep_kernel) writes, for every row m of x and group g,
// X[m,g] as three BF16 pieces whose sum is exactly the FP32 value, twice, and for
// every weight row n the matching coefficients:
//   Xs[m, 6g + j] = Xs[m, 6g + 3 + j] = piece j of X[m,g]            (j = 0, 1, 2)
//   Bc[n, 6g + j] = b[n,g],  Bc[n, 6g + 3 + j] = -128 s[n,g]         (exact BF16)
// padded with zeros to Kx = 128 ceil(6 G / 128) columns.  The GEMM runs Kx / 128
// extra "bias steps" (A = a 128-column block of Bc, B = the same block of Xs),
// spread round-robin over the K splits and added with scale 1.
// One CTA computes a BN x BM = 128 x 128 tile of y^T over a contiguous range of
// 128-groups (all of K, or one split of a cluster).  Warp roles (20 warps):
//   warp 0 (one thread)  TMA producer of the x / Xs stages (bias steps first)
//   warp 1 (one thread)  MMA issuer (and TMEM allocation)
//   warps 4-11           dequantisation: warp w owns lanes 32 (w % 4) .. +31 and
//                        the column half (w - 4) / 4 of each A buffer
//   warps 12-19          epilogue: lanes 32 (w % 4) .. +31, x rows 64 ((w - 12) / 4) .. +63
// Registers are rebalanced per warpgroup with setmaxnreg and returned to the
// launch allocation before the common tail.  All waits are bounded.
#pragma once

#include "ptx.cuh"

namespace w4a16 {
namespace gm {

constexpr int BN = 128;                 // weight rows of a tile: MMA M, TMEM lanes
constexpr int BM = 128;                 // x rows of a tile: MMA N, accumulator columns
constexpr int kXStages = 4;
constexpr int kABufs = 3;
constexpr int kDBufs = 2;
constexpr int kXAtom = BM * 128;        // 64 k of 128 x rows, 128-byte swizzle: 16 KB
constexpr int kXBytes = 2 * kXAtom;     // one group: 32 KB
constexpr int kACols = 64;              // 128 BF16 values of a row
constexpr int kACol0 = kDBufs * BM;     // A buffers follow the accumulators
constexpr int kTmemCols = 512;
static_assert(kACol0 + kABufs * kACols <= kTmemCols, "tensor memory budget");

constexpr int kWarpTma = 0, kWarpMma = 1, kWarpDeq = 4, kDeqWarps = 8, kWarpEpi = 12, kEpiWarps = 8;
constexpr int kThreads = (kWarpEpi + kEpiWarps) * 32;   // 640
constexpr int kLaunchRegs = 96;                         // per thread at launch (65536 / 640, rounded to 8)
constexpr int kRegsCtl = 32, kRegsDeq = 72, kRegsEpi = 152;
// Registers are exchanged within each SM sub-partition, which holds one warp of every
// warpgroup: a warpgroup that grows must never race one that has not yet shrunk.  The
// epilogue grows at the start (the others shrink unconditionally first) and shrinks at
// the end before arriving on named barrier kBarRegs; the others grow back only after it.
constexpr uint32_t kBarRegs = 1;
static_assert(128 * (kRegsCtl + 2 * kRegsDeq + 2 * kRegsEpi) <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");

constexpr int kBiasCoef = 6;            // bias-step entries per group
constexpr int kOffBar = kXStages * kXBytes;
// Barriers, indexed by step i: ready[i % kXStages] (x or Xs landed + every dequantisation
// warp stored A), done[i % kXStages] (the step's MMAs completed: frees its x stage, its A
// buffer and fills its accumulator), d_empty[i % kDBufs] (the epilogue read the accumulator).
// No waiter can be a whole ring behind the phase it waits for (each role is at most
// kXStages - 1 steps ahead of the next), so the parities never alias.
constexpr int kNumBars = 2 * kXStages + kDBufs;
static_assert(kABufs < kXStages && kDBufs < kXStages, "one done ring serves every buffer");
constexpr int kSmemBytes = kOffBar + kNumBars * 8 + 16 + 1024;   // + TMEM address, + alignment slack
// Split-K partial tile, [BM x rows][BN weight rows] FP32, in the x stages once the loop is over.
static_assert(BM * BN * 4 <= kXStages * kXBytes, "partial tile must fit in the x stages");
constexpr int kMaxSplits = 8;           // portable cluster size

__host__ __device__ constexpr int bias_steps(int G) { return (kBiasCoef * G + 127) / 128; }
__host__ __device__ constexpr int xs_cols(int G) { return 128 * bias_steps(G); }

struct Params {
    const uint32_t *wq;       // [N, G*16] packed codes
    const uint16_t *scales;   // bf16 [N, G]
    const uint16_t *biases;   // bf16 [N, G]
    const uint16_t *bc;       // bf16 [N, Kx] bias-step coefficients (from prep_kernel)
    uint16_t *y;              // bf16 [M, N]
    int M, N, G, Kx;
    int splits;               // K splits (gridDim.x, the cluster size)
    int static_weights;       // codes, scales and biases may be read before the dependency wait
};

// ------------------------------------------------------------------ preparation: bias-step operands

// Items [0, M G): Xs[m, 6g + j] = Xs[m, 6g + 3 + j] = piece j of X[m,g] =
// sum_{k in g} x[m,k] (FP32, k ascending), X = p0 + p1 + p2 exactly with
// p0 = bf16(X), p1 = bf16(X - p0), p2 = X - p0 - p1 (exact in BF16).
// Items [M G, M G + N G): Bc[n, 6g + j] = b[n,g], Bc[n, 6g + 3 + j] = -128 s[n,g].
// The last group of a row also writes the zero padding 6G .. Kx-1.
__global__ void __launch_bounds__(256) prep_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ scales,
                                                   const uint16_t *__restrict__ biases, uint16_t *__restrict__ xs,
                                                   uint16_t *__restrict__ bc, int M, int N, int G, int Kx) {
    pdl_launch_dependents();   // the GEMM may start its prologue
    pdl_wait();                // x may come from the previous kernel of the stream
    const long long mg = static_cast<long long>(M) * G;
    const long long total = mg + static_cast<long long>(N) * G;
    const long long K = static_cast<long long>(G) * 128;
    for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total;
         idx += static_cast<long long>(gridDim.x) * blockDim.x) {
        const bool is_x = idx < mg;
        const long long item = is_x ? idx : idx - mg;
        const long long r = item / G;
        const int g = static_cast<int>(item - r * G);
        uint32_t w0, w1, w2;
        if (is_x) {
            const uint4 *src = reinterpret_cast<const uint4 *>(x + r * K + g * 128);
            float sum = 0.f;
#pragma unroll 4
            for (int i = 0; i < 16; ++i) {
                const uint4 v = __ldg(src + i);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    sum += bf16_lo_to_f32(w[j]);
                    sum += bf16_hi_to_f32(w[j]);
                }
            }
            const uint32_t p0 = __bfloat16_as_ushort(__float2bfloat16_rn(sum));
            const float r1 = sum - bf16_to_f32(p0);
            const uint32_t p1 = __bfloat16_as_ushort(__float2bfloat16_rn(r1));
            const uint32_t p2 = __bfloat16_as_ushort(__float2bfloat16_rn(r1 - bf16_to_f32(p1)));
            w0 = p0 | (p1 << 16);
            w1 = p2 | (p0 << 16);
            w2 = p1 | (p2 << 16);
        } else {
            const uint32_t b = __ldg(biases + r * G + g);
            const uint32_t t = __bfloat16_as_ushort(__float2bfloat16_rn(-128.f * bf16_to_f32(__ldg(scales + r * G + g))));
            w0 = b | (b << 16);
            w1 = b | (t << 16);
            w2 = t | (t << 16);
        }
        uint16_t *row = (is_x ? xs : bc) + r * Kx;
        uint32_t *dst = reinterpret_cast<uint32_t *>(row + kBiasCoef * g);   // 4-byte aligned
        dst[0] = w0;
        dst[1] = w1;
        dst[2] = w2;
        if (g == G - 1)
            for (int c = kBiasCoef * G; c < Kx; c += 2) *reinterpret_cast<uint32_t *>(row + c) = 0u;
    }
}

// ------------------------------------------------------------------ GEMM

__device__ __forceinline__ uint32_t bf16x2_plus128(uint32_t v, uint32_t v4, uint32_t sel) {
    // bytes sel of (v, v >> 4) -> two codes in bits 0-3 and 16-19 -> BF16 128 + code
    return codes_to_bf16x2_plus128(prmt(v, v4, sel));
}

__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_xs,
                const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
    uint64_t *ready = bars, *done = ready + kXStages, *d_empty = done + kXStages;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kNumBars);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int split = blockIdx.x, tile_n = blockIdx.y, tile_m = blockIdx.z;   // splits of a tile: one cluster
    const int G = p.G;
    const int g0 = static_cast<int>(static_cast<long long>(split) * G / p.splits);
    const int g1 = static_cast<int>(static_cast<long long>(split + 1) * G / p.splits);
    const int ng = g1 - g0;
    // bias steps t = split, split + S, ... < Kx / 128 come first, then the groups g0 .. g1-1
    const int nbias_all = p.Kx / 128;
    const int nbs = split < nbias_all ? (nbias_all - split + p.splits - 1) / p.splits : 0;
    const int steps = nbs + ng;

    if (threadIdx.x == 0) {
        pdl_launch_dependents();
        for (int i = 0; i < kXStages; ++i) { mbar_init(&ready[i], 1 + kDeqWarps); mbar_init(&done[i], 1); }
        for (int i = 0; i < kDBufs; ++i) mbar_init(&d_empty[i], kEpiWarps);
        fence_mbar_init();
    }
    if (warp == kWarpMma) {   // the whole warp allocates tensor memory
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp < kWarpDeq) {
        regs_shrink<kRegsCtl>();
        if (warp == kWarpTma && lane == 0) {
            // -------------------------------------------------------- TMA producer
            prefetch_tmap(&tm_x);
            prefetch_tmap(&tm_xs);
            pdl_wait();   // x (and the group sums) come from the preceding kernels
            int i = 0;
            for (; i < steps; ++i) {
                const int s = i % kXStages;
                if (i >= kXStages && !mbar_wait(&done[s], ((i / kXStages) - 1) & 1)) break;   // stage free
                mbar_arrive_expect_tx(&ready[s], kXBytes);
                uint8_t *dst = smem + s * kXBytes;
                const CUtensorMap *map = i < nbs ? &tm_xs : &tm_x;
                const int col = i < nbs ? (split + i * p.splits) * 128 : (g0 + i - nbs) * 128;
                tma_load_2d(dst, map, &ready[s], col, tile_m * BM);
                tma_load_2d(dst + kXAtom, map, &ready[s], col + 64, tile_m * BM);
            }
            // leave no copy in flight: the last stages' MMAs (which consumed them) completed
            for (int j = max(0, i - kXStages); j < i; ++j)
                mbar_wait(&done[j % kXStages], (j / kXStages) & 1, false);
        } else if (warp == kWarpMma && lane == 0) {
            // -------------------------------------------------------- MMA issuer
            constexpr uint32_t idesc = umma_idesc_bf16(BN, BM);
            for (int i = 0; i < steps; ++i) {
                const int xs = i % kXStages, ab = i % kABufs, db = i % kDBufs;
                if (!mbar_wait(&ready[xs], (i / kXStages) & 1)) break;
                if (i >= kDBufs && !mbar_wait(&d_empty[db], ((i / kDBufs) - 1) & 1)) break;
                tc_fence_after();
                const uint32_t b0 = smem_u32(smem + xs * kXBytes);
                const uint32_t d = tmem_base + db * BM;
                const uint32_t a = tmem_base + kACol0 + ab * kACols;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t bd = umma_desc_sw128(b0 + (kk >> 2) * kXAtom + (kk & 3) * 32);
                    umma_bf16_ts(d, a + 8 * kk, bd, idesc, kk > 0);
                }
                umma_commit(&done[xs]);
            }
        }
        __syncwarp();
        named_bar_sync(kBarRegs, kThreads);   // the epilogue has returned its registers
        regs_grow<kLaunchRegs>();             // back to the launch allocation for the common tail
    } else if (warp < kWarpEpi) {
        regs_shrink<kRegsDeq>();
        // ------------------------------------------------------------ dequantisation
        const int quarter = warp & 3, half = (warp - kWarpDeq) >> 2;
        const long long row = static_cast<long long>(tile_n) * BN + quarter * 32 + lane;   // weight row n
        const bool row_ok = row < p.N;
        const uint4 *codes = reinterpret_cast<const uint4 *>(p.wq + (row_ok ? row : 0) * (static_cast<long long>(G) * 16));
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + kACol0 + half * 32;
        // codes of step i (words 8 half .. 8 half + 7 of its group), fetched two steps ahead;
        // bias steps carry zeros through the ring
        auto fetch = [&](int i, uint4 &lo, uint4 &hi) {
            if (row_ok && i >= nbs && i < steps) {
                const int g = g0 + i - nbs;
                lo = ldg_nc_v4(codes + g * 4 + 2 * half);
                hi = ldg_nc_v4(codes + g * 4 + 2 * half + 1);
            } else {
                lo = hi = make_uint4(0, 0, 0, 0);
            }
        };
        if (!p.static_weights) pdl_wait();
        uint4 c0, c1, n0, n1, f0, f1;
        fetch(0, c0, c1);
        fetch(1, n0, n1);
        pdl_wait();   // the bias-step coefficients come from the preparation kernel
        const uint4 *bcrow = reinterpret_cast<const uint4 *>(p.bc + (row_ok ? row : 0) * static_cast<long long>(p.Kx));
        for (int i = 0; i < steps; ++i) {
            const int ab = i % kABufs;
            fetch(i + 2, f0, f1);
            if (i >= kABufs && !mbar_wait(&done[(i - kABufs) % kXStages], ((i - kABufs) / kXStages) & 1)) break;
            tc_fence_after();   // the tensor cores' reads of this buffer precede the stores below
            uint32_t r[32];
            if (i >= nbs) {
                const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
                for (int j = 0; j < 8; ++j) {   // word j: k = 8 j .. 8 j + 7 -> columns 4 j .. 4 j + 3
                    const uint32_t v = w[j], v4 = v >> 4;
                    r[4 * j + 0] = bf16x2_plus128(v, v4, 0x0400u);
                    r[4 * j + 1] = bf16x2_plus128(v, v4, 0x0501u);
                    r[4 * j + 2] = bf16x2_plus128(v, v4, 0x0602u);
                    r[4 * j + 3] = bf16x2_plus128(v, v4, 0x0703u);
                }
            } else {   // 64 coefficients of this column half (bias steps are few: loaded here)
                const int t = split + i * p.splits;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint4 v = row_ok ? ldg_nc_v4(bcrow + t * 16 + half * 8 + j) : make_uint4(0, 0, 0, 0);
                    r[4 * j + 0] = v.x;
                    r[4 * j + 1] = v.y;
                    r[4 * j + 2] = v.z;
                    r[4 * j + 3] = v.w;
                }
            }
            c0 = n0; c1 = n1; n0 = f0; n1 = f1;
            tmem_st32(taddr + ab * kACols, r);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ready[i % kXStages]);
        }
        named_bar_sync(kBarRegs, kThreads);
        regs_grow<kLaunchRegs>();
    } else {
        regs_grow<kRegsEpi>();
        // ------------------------------------------------------------ epilogue
        const int quarter = warp & 3, half = (warp - kWarpEpi) >> 2;
        const int nl = quarter * 32 + lane;                         // weight row within the tile
        const long long row = static_cast<long long>(tile_n) * BN + nl;
        const bool row_ok = row < p.N;
        const uint16_t *srow = p.scales + (row_ok ? row : 0) * G;
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + half * 64;
        if (!p.static_weights) pdl_wait();   // scales are weights
        float acc[64];
#pragma unroll
        for (int j = 0; j < 64; ++j) acc[j] = 0.f;
        // scale of step i (1 for bias steps), fetched four steps ahead
        auto scale_of = [&](int i) {
            return (row_ok && i >= nbs && i < steps) ? bf16_to_f32(__ldg(srow + g0 + i - nbs)) : 1.f;
        };
        float q0 = scale_of(0), q1 = scale_of(1), q2 = scale_of(2), q3 = scale_of(3);
        for (int i = 0; i < steps; ++i) {
            const int db = i % kDBufs;
            const float sc = q0;
            q0 = q1; q1 = q2; q2 = q3; q3 = scale_of(i + 4);
            if (!mbar_wait(&done[i % kXStages], (i / kXStages) & 1)) break;
            tc_fence_after();
            uint32_t r0[32], r1[32];
            tmem_ld32(taddr + db * BM, r0);
            tmem_ld32(taddr + db * BM + 32, r1);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&d_empty[db]);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                acc[j] = fmaf(sc, __uint_as_float(r0[j]), acc[j]);
                acc[32 + j] = fmaf(sc, __uint_as_float(r1[j]), acc[32 + j]);
            }
        }
        pdl_wait();   // y may still be read by the preceding kernel
        const int m0 = tile_m * BM + half * 64;
        if (p.splits > 1) {
            // split-K: this CTA's partial, [x row][weight row] FP32, into the (idle) x stages
            float *part = reinterpret_cast<float *>(smem);
#pragma unroll
            for (int j = 0; j < 64; ++j) part[(half * 64 + j) * BN + nl] = acc[j];
        } else if (row_ok) {
#pragma unroll
            for (int j = 0; j < 64; ++j)
                if (m0 + j < p.M)
                    p.y[static_cast<long long>(m0 + j) * p.N + row] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[j]));
        }
        regs_shrink<kLaunchRegs>();            // released first ...
        named_bar_arrive(kBarRegs, kThreads);  // ... then the other warpgroups grow back into it
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }

    if (p.splits > 1) {
        // Split-K reduction over the cluster (the S splits of this tile): CTA rank r sums
        // x rows [r*R, (r+1)*R) of the S partial tiles, in rank order, through distributed
        // shared memory, and writes them to y.  The epilogue warps do the work.
        cluster_sync_all();
        if (warp >= kWarpEpi) {
            const int S = p.splits;
            const uint32_t rank = cluster_ctarank();
            const int rows_per = (BM + S - 1) / S;
            const int r_lo = static_cast<int>(rank) * rows_per;
            const int r_hi = min(BM, r_lo + rows_per);
            const uint32_t part0 = smem_u32(smem);
            const int t = threadIdx.x - kWarpEpi * 32;
            for (int item = t; item < (r_hi - r_lo) * (BN / 4); item += kEpiWarps * 32) {
                const int ml = r_lo + item / (BN / 4), c4 = item % (BN / 4);
                const uint32_t off = part0 + (ml * BN + 4 * c4) * 4;
                float4 v = ld_dsmem_f4(dsmem_addr(off, 0));
                for (int sp = 1; sp < S; ++sp) {
                    const float4 w = ld_dsmem_f4(dsmem_addr(off, sp));
                    v.x += w.x; v.y += w.y; v.z += w.z; v.w += w.w;
                }
                const long long mrow = static_cast<long long>(tile_m) * BM + ml;
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
        }
        cluster_sync_all();   // no CTA leaves while another still reads its shared memory
    }
}

}  // namespace gm
}  // namespace w4a16
