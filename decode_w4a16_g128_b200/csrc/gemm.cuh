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
// Two CTAs on two SMs (a CTA pair, tcgen05 cta_group::2) compute a 256 x 128 tile of
// y^T: each CTA dequantises its own 128 weight rows into its own tensor memory and
// stages 64 of the 128 x rows; the pair leader issues M = 256 MMAs that read both
// halves of each operand, so every x byte loaded from L2 serves 256 weight rows.
// Both CTAs' TMA bytes and dequantisation arrivals land on the leader's barriers;
// the leader's commits are multicast to both CTAs.  A cluster holds the S K-splits
// of a tile as S pairs (cluster rank = 2 split + pair rank).  Warp roles (20 warps
// per CTA):
//   warp 0 (one thread)  TMA producer of the x / Xs stages (bias steps first)
//   warp 2 (one thread)  TMA producer of the packed codes (64-byte swizzle)
//   warps 1, 3 (one thread each)  MMA issuers in the pair leader, even / odd steps
//                        (warp 1 also allocates tensor memory, in both CTAs)
//   warps 4-11           dequantisation: warp w owns lanes 32 (w % 4) .. +31 and
//                        the column half (w - 4) / 4 of each A buffer
//   warps 12-19          epilogue: lanes 32 (w % 4) .. +31, x rows 64 ((w - 12) / 4) .. +63
// Registers are rebalanced per warpgroup with setmaxnreg and returned to the
// launch allocation before the common tail.  All waits are bounded.
#pragma once

#include "ptx.cuh"

namespace w4a16 {
namespace gm {

constexpr int BN = 128;                 // weight rows of a CTA: its half of the pair MMA's M = 256
constexpr int kPairRows = 2 * BN;       // weight rows of a CTA pair (one output tile)
constexpr int BM = 128;                 // x rows of a tile: MMA N, accumulator columns
constexpr int kXRows = BM / 2;          // x rows staged by each CTA of the pair (its half of B)
constexpr int kXStages = 8;
constexpr int kABufs = 4;
constexpr int kDBufs = 2;
constexpr int kXAtom = kXRows * 128;    // 64 k of 64 x rows, 128-byte swizzle: 8 KB
constexpr int kXBytes = 2 * kXAtom;     // one group of this CTA's x rows: 16 KB
constexpr int kACols = 64;              // 128 BF16 values of a row
constexpr int kACol0 = kDBufs * BM;     // A buffers follow the accumulators
constexpr int kTmemCols = 512;
static_assert(kACol0 + kABufs * kACols <= kTmemCols, "tensor memory budget");

constexpr int kWarpTma = 0, kWarpMma = 1, kWarpDeq = 4, kDeqWarps = 8, kWarpEpi = 12, kEpiWarps = 8;
constexpr int kThreads = (kWarpEpi + kEpiWarps) * 32;   // 640
constexpr int kLaunchRegs = 96;                         // per thread at launch (65536 / 640, rounded to 8)
constexpr int kRegsCtl = 56, kRegsDeq = 56, kRegsEpi = 152;
// Registers are exchanged within each SM sub-partition, which holds one warp of every
// warpgroup: a warpgroup that grows must never race one that has not yet shrunk.  The
// epilogue grows at the start (the others shrink unconditionally first) and shrinks at
// the end before arriving on named barrier kBarRegs; the others grow back only after it.
constexpr uint32_t kBarRegs = 1;
static_assert(128 * (kRegsCtl + 2 * kRegsDeq + 2 * kRegsEpi) <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");

constexpr int kBiasCoef = 6;            // bias-step entries per group
constexpr int kWStages = 4;             // packed codes ring
constexpr int kWBytes = BN * 64;        // one group's codes of this CTA's 128 rows: 8 KB
constexpr int kOffW = kXStages * kXBytes;
constexpr int kOffBar = kOffW + kWStages * kWBytes;
// Barriers, indexed by step i: ready[i % kXStages] (x or Xs landed + every dequantisation
// warp stored A), done[i % kXStages] (the step's MMAs completed: frees its x stage, its A
// buffer and fills its accumulator), d_empty[i % kDBufs] (the epilogue read the accumulator).
// No waiter can be a whole ring behind the phase it waits for (each role is at most
// kXStages - 1 steps ahead of the next), so the parities never alias.  Per group j of
// codes: w_full[j % kWStages] (TMA landed), w_empty[j % kWStages] (dequantisation read it).
constexpr int kNumBars = 2 * kXStages + kDBufs + 2 * kWStages;
static_assert(kABufs < kXStages && kDBufs < kXStages, "one done ring serves every buffer");
static_assert(kNumBars * 8 + 16 <= 512, "barrier area");
// The scales of this CTA's 128 rows, [128][G] BF16, staged once per CTA after the barriers.
constexpr int kOffScales = kOffBar + 512;
constexpr int kMaxGroups = 256;         // K <= 32768 on the GEMM path
__host__ __device__ constexpr int smem_bytes(int G) { return kOffScales + 256 * G + 1024; }   // + alignment slack
static_assert(smem_bytes(kMaxGroups) <= 232448, "shared memory budget");
constexpr uint32_t kBarScales = 2;      // named barrier: the epilogue's staged scales are complete
constexpr int kWarpCodes = 2;           // TMA producer of the packed codes
constexpr int kWarpMma2 = 3;            // second MMA issuer (odd steps)
static_assert(kDBufs == 2, "each of the two MMA issuers owns one accumulator");
// Split-K partial of a CTA, [BM x rows][BN weight rows] FP32, in the x stages once the loop is over.
static_assert(BM * BN * 4 <= kXStages * kXBytes, "partial tile must fit in the x stages");
constexpr int kMaxSplits = 4;           // a cluster holds 2 x splits CTAs: at most 8 (portable size)

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
    int tma_store;            // y rows are 16-byte multiples: tiles leave through one TMA store
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
                const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_y, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
    uint64_t *ready = bars, *done = ready + kXStages, *d_empty = done + kXStages;
    uint64_t *w_full = d_empty + kDBufs, *w_empty = w_full + kWStages;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kNumBars);
    uint16_t *sc_smem = reinterpret_cast<uint16_t *>(smem + kOffScales);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();               // 2 split + pair rank
    const int pair_rank = static_cast<int>(rank & 1u);
    const uint32_t leader = rank & ~1u;
    const bool is_leader = pair_rank == 0;
    const int split = static_cast<int>(rank >> 1);
    const int tile_n = blockIdx.y, tile_m = blockIdx.z;
    const int G = p.G;
    const int g0 = static_cast<int>(static_cast<long long>(split) * G / p.splits);
    const int g1 = static_cast<int>(static_cast<long long>(split + 1) * G / p.splits);
    const int ng = g1 - g0;
    // bias steps t = split, split + S, ... < Kx / 128 come first, then the groups g0 .. g1-1
    const int nbias_all = p.Kx / 128;
    const int nbs = split < nbias_all ? (nbias_all - split + p.splits - 1) / p.splits : 0;
    const int steps = nbs + ng;
    const long long row0 = static_cast<long long>(tile_n) * kPairRows + pair_rank * BN;   // this CTA's weight rows

    if (threadIdx.x == 0) {
        pdl_launch_dependents();
        for (int i = 0; i < kXStages; ++i) { mbar_init(&ready[i], 1 + 2 * kDeqWarps); mbar_init(&done[i], 1); }
        for (int i = 0; i < kDBufs; ++i) mbar_init(&d_empty[i], 2 * kEpiWarps);
        for (int i = 0; i < kWStages; ++i) { mbar_init(&w_full[i], 1); mbar_init(&w_empty[i], kDeqWarps); }
        fence_mbar_init();
    }
    if (warp == kWarpMma) {   // one warp of each CTA of the pair allocates the pair's tensor memory
        tmem_alloc_pair(tmem_slot, kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();   // barriers initialised and tensor memory allocated in every CTA of the cluster
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // the leader's barriers, as shared::cluster addresses
    const uint32_t ready_l = dsmem_addr(smem_u32(ready), leader);
    const uint32_t d_empty_l = dsmem_addr(smem_u32(d_empty), leader);

    if (warp < kWarpDeq) {
        regs_shrink<kRegsCtl>();
        if (warp == kWarpTma && lane == 0) {
            // -------------------------------------------------------- TMA producer (both CTAs)
            prefetch_tmap(&tm_x);
            prefetch_tmap(&tm_xs);
            if (p.tma_store) prefetch_tmap(&tm_y);
            pdl_wait();   // x (and the group sums) come from the preceding kernels
            int i = 0;
            for (; i < steps; ++i) {
                const int s = i % kXStages;
                if (i >= kXStages && !mbar_wait(&done[s], ((i / kXStages) - 1) & 1)) break;   // stage free
                if (is_leader) mbar_arrive_expect_tx(&ready[s], 2 * kXBytes);   // both halves
                uint8_t *dst = smem + s * kXBytes;
                const CUtensorMap *map = i < nbs ? &tm_xs : &tm_x;
                const int col = i < nbs ? (split + i * p.splits) * 128 : (g0 + i - nbs) * 128;
                const int xrow = tile_m * BM + pair_rank * kXRows;
                tma_load_2d_pair(dst, map, ready_l + 8 * s, col, xrow);
                tma_load_2d_pair(dst + kXAtom, map, ready_l + 8 * s, col + 64, xrow);
            }
            // leave no copy in flight: the last stages' MMAs (which consumed them) completed
            for (int j = max(0, i - kXStages); j < i; ++j)
                mbar_wait(&done[j % kXStages], (j / kXStages) & 1, false);
        } else if (warp == kWarpCodes && lane == 0) {
            // -------------------------------------------------------- TMA producer of the codes (both CTAs)
            prefetch_tmap(&tm_w);
            if (!p.static_weights) pdl_wait();
            int j = 0;
            for (; j < ng; ++j) {
                const int s = j % kWStages;
                if (j >= kWStages && !mbar_wait(&w_empty[s], ((j / kWStages) - 1) & 1)) break;
                mbar_arrive_expect_tx(&w_full[s], kWBytes);
                tma_load_2d(smem + kOffW + s * kWBytes, &tm_w, &w_full[s], (g0 + j) * 16, static_cast<int>(row0));
            }
            for (int q = max(0, j - kWStages); q < j; ++q)   // leave no copy in flight
                mbar_wait(&w_full[q % kWStages], (q / kWStages) & 1, false);
        } else if ((warp == kWarpMma || warp == kWarpMma2) && lane == 0 && is_leader) {
            // -------------------------------------------------------- MMA issuers (pair leader)
            // The tensor pipe takes about one instruction ahead, so every barrier operation of
            // an issuing thread leaves it idle for its latency.  Two issuers take alternate
            // steps (so each always fills the same accumulator): one waits for its step's
            // inputs while the other's MMAs run.
            constexpr uint32_t idesc = umma_idesc_bf16(kPairRows, BM);
            const uint16_t mask = static_cast<uint16_t>(3u << leader);
            for (int i = (warp == kWarpMma ? 0 : 1); i < steps; i += 2) {
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
                    umma_bf16_ts_pair(d, a + 8 * kk, bd, idesc, kk > 0);
                }
                umma_commit_pair(&done[xs], mask);
            }
        }
        __syncwarp();
        named_bar_sync(kBarRegs, kThreads);   // the epilogue has returned its registers
        regs_grow<kLaunchRegs>();             // back to the launch allocation for the common tail
    } else if (warp < kWarpEpi) {
        regs_shrink<kRegsDeq>();
        // ------------------------------------------------------------ dequantisation (both CTAs)
        const int quarter = warp & 3, half = (warp - kWarpDeq) >> 2;
        const long long row = row0 + quarter * 32 + lane;   // weight row n
        const bool row_ok = row < p.N;
        const int rl = quarter * 32 + lane;                  // row within the CTA's codes tile
        const uint32_t sw = static_cast<uint32_t>((rl >> 1) & 3);   // 64-byte swizzle of that row
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + kACol0 + half * 32;
        pdl_wait();   // the bias-step coefficients come from the preparation kernel
        const uint4 *bcrow = reinterpret_cast<const uint4 *>(p.bc + (row_ok ? row : 0) * static_cast<long long>(p.Kx));
        for (int i = 0; i < steps; ++i) {
            const int ab = i % kABufs;
            uint32_t r[32];
            if (i >= nbs) {
                // chunks 2 half, 2 half + 1 (words 8 half .. 8 half + 7) of this row's codes
                const int j = i - nbs, ws = j % kWStages;
                if (!mbar_wait(&w_full[ws], (j / kWStages) & 1)) break;
                const uint32_t wrow = smem_u32(smem + kOffW + ws * kWBytes) + rl * 64;
                const uint4 c0 = lds128(wrow + (((2u * half) ^ sw) << 4));
                const uint4 c1 = lds128(wrow + (((2u * half + 1u) ^ sw) << 4));
                __syncwarp();
                if (lane == 0) mbar_arrive(&w_empty[ws]);   // the codes are in registers
                if (i >= kABufs && !mbar_wait(&done[(i - kABufs) % kXStages], ((i - kABufs) / kXStages) & 1)) break;
                tc_fence_after();   // the tensor cores' reads of this buffer precede the stores below
                const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {   // word jj: k = 8 jj .. 8 jj + 7 -> columns 4 jj .. 4 jj + 3
                    const uint32_t v = w[jj], v4 = v >> 4;
                    r[4 * jj + 0] = bf16x2_plus128(v, v4, 0x0400u);
                    r[4 * jj + 1] = bf16x2_plus128(v, v4, 0x0501u);
                    r[4 * jj + 2] = bf16x2_plus128(v, v4, 0x0602u);
                    r[4 * jj + 3] = bf16x2_plus128(v, v4, 0x0703u);
                }
            } else {   // 64 coefficients of this column half (bias steps are few: loaded here)
                const int t = split + i * p.splits;
                uint4 v[8];
#pragma unroll
                for (int jj = 0; jj < 8; ++jj)
                    v[jj] = row_ok ? ldg_nc_v4(bcrow + t * 16 + half * 8 + jj) : make_uint4(0, 0, 0, 0);
                if (i >= kABufs && !mbar_wait(&done[(i - kABufs) % kXStages], ((i - kABufs) / kXStages) & 1)) break;
                tc_fence_after();
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    r[4 * jj + 0] = v[jj].x;
                    r[4 * jj + 1] = v[jj].y;
                    r[4 * jj + 2] = v[jj].z;
                    r[4 * jj + 3] = v[jj].w;
                }
            }
            tmem_st32(taddr + ab * kACols, r);
            tmem_st_wait_regs(r);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(ready_l + 8 * (i % kXStages));
        }
        named_bar_sync(kBarRegs, kThreads);
        regs_grow<kLaunchRegs>();
    } else {
        regs_grow<kRegsEpi>();
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int quarter = warp & 3, half = (warp - kWarpEpi) >> 2;
        const int nl = quarter * 32 + lane;                         // weight row within the CTA
        const long long row = row0 + nl;
        const bool row_ok = row < p.N;
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + half * 64;
        if (!p.static_weights) pdl_wait();   // scales are weights
        {
            // stage the scales of this CTA's rows ([128][G] BF16, contiguous in global memory)
            // with coalesced loads; no load of this warp stays in flight across its arrivals
            const int t = threadIdx.x - kWarpEpi * 32;
            const long long rows = min(static_cast<long long>(BN), max(0ll, p.N - row0));
            const long long elems = rows * G;
            const uint16_t *src = p.scales + row0 * G;
            const long long vec = (elems * 2) / 16;
            for (long long v = t; v < vec; v += kEpiWarps * 32)
                reinterpret_cast<uint4 *>(sc_smem)[v] = ldg_nc_v4(reinterpret_cast<const uint4 *>(src) + v);
            for (long long e = vec * 8 + t; e < elems; e += kEpiWarps * 32) sc_smem[e] = __ldg(src + e);
        }
        named_bar_sync(kBarScales, kEpiWarps * 32);
        const uint16_t *srow = sc_smem + nl * G;
        float acc[64];
#pragma unroll
        for (int j = 0; j < 64; ++j) acc[j] = 0.f;
        for (int i = 0; i < steps; ++i) {
            const int db = i % kDBufs;
            const float sc = (row_ok && i >= nbs) ? bf16_to_f32(srow[g0 + i - nbs]) : 1.f;
            if (!mbar_wait(&done[i % kXStages], (i / kXStages) & 1)) break;
            tc_fence_after();
            uint32_t r0[32], r1[32];
            tmem_ld32(taddr + db * BM, r0);
            tmem_ld32(taddr + db * BM + 32, r1);
            tmem_ld_wait_regs(r0);
            tmem_ld_wait_regs(r1);   // both loads completed at the first wait; this only pins r1
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(d_empty_l + 8 * db);
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
        } else if (p.tma_store) {
            // the tile, [x row][weight row] BF16, into the (idle) x stages, then one TMA store
            uint16_t *tile = reinterpret_cast<uint16_t *>(smem);
#pragma unroll
            for (int j = 0; j < 64; ++j)
                tile[(half * 64 + j) * BN + nl] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[j]));
            fence_proxy_async_smem();   // the async proxy reads the tile
            named_bar_sync(kBarScales, kEpiWarps * 32);
            if (warp == kWarpEpi && lane == 0) {
                tma_store_2d(&tm_y, tile, static_cast<int>(row0), tile_m * BM);
                bulk_commit_group();
                bulk_wait_all();   // shared memory is released, and y written, before the CTA ends
            }
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
        tmem_dealloc_pair(tmem_base, kTmemCols);
    }

    // Every CTA of the cluster is done with its peers' barriers and shared memory only
    // after this barrier: none leaves while another may still signal or read it.
    cluster_sync_all();
    if (p.splits > 1) {
        // Split-K reduction over the S pairs of the cluster: the CTAs with this pair rank
        // hold the S partials of the same 128 weight rows; the one of split r sums x rows
        // [r*R, (r+1)*R) of them, in split order, through distributed shared memory.
        if (warp >= kWarpEpi) {
            const int S = p.splits;
            const int rows_per = (BM + S - 1) / S;
            const int r_lo = split * rows_per;
            const int r_hi = min(BM, r_lo + rows_per);
            const uint32_t part0 = smem_u32(smem);
            const int t = threadIdx.x - kWarpEpi * 32;
            for (int item = t; item < (r_hi - r_lo) * (BN / 4); item += kEpiWarps * 32) {
                const int ml = r_lo + item / (BN / 4), c4 = item % (BN / 4);
                const uint32_t off = part0 + (ml * BN + 4 * c4) * 4;
                float4 v = ld_dsmem_f4(dsmem_addr(off, static_cast<uint32_t>(pair_rank)));
                for (int sp = 1; sp < S; ++sp) {
                    const float4 w = ld_dsmem_f4(dsmem_addr(off, static_cast<uint32_t>(2 * sp + pair_rank)));
                    v.x += w.x; v.y += w.y; v.z += w.z; v.w += w.w;
                }
                const long long mrow = static_cast<long long>(tile_m) * BM + ml;
                const long long n = row0 + 4 * c4;
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
