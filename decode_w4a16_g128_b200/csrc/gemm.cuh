// gemm.cuh - tcgen05 tensor-core W4A16 GEMM for M > 8 (prefill).
//
// Role in the layer: tiny-llm "Week 2 Day 6: SIMD-Matrix Prefill", Task 1,
// routes M > 8 to a tiled matrix kernel; Task 3 hoists one scale and bias per
// 128-group and reuses them across that group's reduction tiles and all rows
// of x.  This is a B200 design with 5th-generation tensor cores, not that
// 32x32x32 Metal tile.
//
// Algebra (exact-integer factorisation, per 128-group g):
//   sum_k x[m,k] w[n,k] = sum_g (s[n,g] / 8) P8[n,m,g] + sum_g (b[n,g] - 16 s[n,g]) X[m,g],
//   P8[n,m,g] = sum_{k in g} (128 + 8 q[n,k]) x[m,k],   X[m,g] = sum_{k in g} x[m,k].
// 128 + 8 q is an exact BF16 value (the code in mantissa bits 3-6 of 128.0) and x is BF16,
// so every product of P8 is exact; only FP32 sums round.  The offset 128 is 16 code units,
// which keeps the cancellation between the two terms small when x is mostly of one sign.
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
//   Bc[n, 6g + j] = b[n,g],  Bc[n, 6g + 3 + j] = -16 s[n,g]          (exact BF16)
// padded with zeros to Kx = 128 ceil(6 G / 128) columns.  The GEMM runs Kx / 128
// extra "bias steps" (A = a 128-column block of Bc, B = the same block of Xs),
// spread round-robin over the K splits and added with scale 1.
// Two CTAs on two SMs (a CTA pair, tcgen05 cta_group::2) compute a 256 x 128 tile of
// y^T: each CTA dequantises its own 128 weight rows into its own tensor memory and
// stages 64 of the 128 x rows; the pair leader issues M = 256 MMAs that read both
// halves of each operand, so every x byte loaded from L2 serves 256 weight rows.
// Both CTAs' TMA bytes and dequantisation arrivals land on the leader's barriers;
// the leader's commits are multicast to both CTAs.  A cluster holds the S K-splits
// of a tile as S pairs (cluster rank = 2 split + pair rank).  Without a K split the
// grid is persistent (one pair per two SMs, each looping over tiles), so the next
// tile's loads, dequantisation and MMAs overlap the previous tile's last steps and its
// store.  Warp roles (20 warps per CTA):
//   warp 0 (one thread)  TMA producer of the x / Xs stages (bias steps first)
//   warp 1 (one thread)  MMA issuer in the pair leader (also allocates tensor memory,
//                        in both CTAs)
//   warp 2 (one thread)  TMA producer of the packed codes (64-byte swizzle), and of each
//                        tile's scales (a 1-D bulk copy into one of two buffers)
//   warp 3               idle
//   warps 4-11           dequantisation: warp w owns lanes 32 (w % 4) .. +31 and
//                        the column half (w - 4) / 4 of each A buffer
//   warps 12-19          epilogue: lanes 32 (w % 4) .. +31, x rows 64 ((w - 12) / 4) .. +63;
//                        a tile leaves through a staging buffer and one TMA store
// Registers are rebalanced per warpgroup with setmaxnreg and returned to the
// launch allocation before the common tail.  All waits are bounded.
#pragma once

#include "plain.cuh"
#include "ptx.cuh"

namespace w4a16 {
namespace gm {

constexpr int BN = 128;                 // weight rows of a CTA: its half of the pair MMA's M = 256
constexpr int kPairRows = 2 * BN;       // weight rows of a CTA pair (one output tile)
constexpr int BM = 128;                 // x rows of a tile: MMA N, accumulator columns
constexpr int kXRows = BM / 2;          // x rows staged by each CTA of the pair (its half of B)
constexpr int kXStages = 6;
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
constexpr int kOffOut = kOffW + kWStages * kWBytes;   // output tile staging for the TMA store
constexpr int kOutBytes = BM * BN * 2;                // [x row][weight row] BF16: 32 KB
constexpr int kOffBar = kOffOut + kOutBytes;
// Barriers, indexed by step i: ready[i % kXStages] (x or Xs landed + every dequantisation
// warp stored A + every epilogue warp read the accumulator of step i - kDBufs, which step i
// overwrites), done[i % kXStages] (the step's MMAs completed: frees its x stage, its A buffer
// and fills its accumulator).  The MMA issuer thus waits on one barrier per step: any
// barrier operation of the issuing thread stalls the tensor pipe for about a hundred cycles
// (measured: ~110 cycles per step of eight M = 256, N = 128 MMAs for one extra test), so the
// epilogue's release of an accumulator rides on the ready barrier of the step that reuses it.
// No waiter can be a whole ring behind the phase it waits for (each role is at most
// kXStages - 1 steps ahead of the next), so the parities never alias.  Per group j of
// codes: w_full[j % kWStages] (TMA landed), w_empty[j % kWStages] (dequantisation read it).
// Per output tile k of a CTA: sc_full[k % B] (its scales are staged), sc_empty[k % B] (the
// epilogue is done with them), B = scale_bufs(G).  Step, group and tile indices run on
// across the tiles of a persistent CTA.
constexpr int kScaleBufsMax = 2;
constexpr int kNumBars = 2 * kXStages + 2 * kWStages + 2 * kScaleBufsMax;
static_assert(kABufs < kXStages && kDBufs < kXStages, "one done ring serves every buffer");
static_assert(kNumBars * 8 + 16 <= 512, "barrier area");
// The scales of a tile's 128 rows of this CTA, [128][G] BF16, after the barriers: two
// buffers (the next tile's are staged while the epilogue reads this one's) up to 128
// groups, one above.
constexpr int kOffScales = kOffBar + 512;
constexpr int kMaxGroups = 256;         // K <= 32768 on the GEMM path
__host__ __device__ constexpr int scale_bufs(int G) { return G <= 128 ? 2 : 1; }
__host__ __device__ constexpr int smem_bytes(int G) {
    return kOffScales + scale_bufs(G) * 256 * G + 1024;   // + alignment slack
}
static_assert(smem_bytes(kMaxGroups) <= 232448 && smem_bytes(128) <= 232448, "shared memory budget");
constexpr uint32_t kBarEpi = 2;         // named barrier of the epilogue warps (output staging)
constexpr int kWarpCodes = 2;           // TMA producer of the packed codes
static_assert(kDBufs == 2 && (kABufs & (kABufs - 1)) == 0, "ring arithmetic of the MMA issuer");
// Split-K partial of a CTA, [BM x rows][BN weight rows] FP32, in the x stages once the loop is over.
static_assert(BM * BN * 4 <= kXStages * kXBytes, "partial tile must fit in the x stages");
constexpr int kMaxSplits = 8;           // a cluster holds 2 x splits CTAs: up to 16 (non-portable size)

__host__ __device__ constexpr int bias_steps(int G) { return (kBiasCoef * G + 127) / 128; }
__host__ __device__ constexpr int xs_cols(int G) { return 128 * bias_steps(G); }

struct Params {
    const uint16_t *x;        // bf16 [M, K] (read by TMA; directly only by the plain path)
    const uint32_t *wq;       // [N, G*16] packed codes
    const uint16_t *scales;   // bf16 [N, G]
    const uint16_t *biases;   // bf16 [N, G]
    const uint16_t *bc;       // bf16 [N, Kx] bias-step coefficients (from prep_kernel)
    uint16_t *y;              // bf16 [M, N]
    int M, N, G, Kx;
    long long tiles;          // output tiles: tiles_n x ceil(M / 128)
    int tiles_n;              // tiles along N (256 weight rows each)
    int splits;               // K splits (gridDim.x, the cluster size)
    int static_weights;       // codes, scales and biases may be read before the dependency wait
    int tma_store;            // y rows are 16-byte multiples: tiles leave through one TMA store
};

// ------------------------------------------------------------------ preparation: bias-step operands

// Xs[m, 6g + j] = Xs[m, 6g + 3 + j] = piece j of X[m,g] = sum_{k in g} x[m,k]
// (FP32: each lane of a half-warp sums 8 consecutive values, then the 16 lanes
// in a fixed tree), X = p0 + p1 + p2 exactly with
// p0 = bf16(X), p1 = bf16(X - p0), p2 = X - p0 - p1 (exact in BF16).
// Bc[n, 6g + j] = b[n,g], Bc[n, 6g + 3 + j] = -16 s[n,g] (one thread per (n, g)).
// The last group of a row also writes the zero padding 6G .. Kx-1.
__global__ void __launch_bounds__(256) prep_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ scales,
                                                   const uint16_t *__restrict__ biases, uint16_t *__restrict__ xs,
                                                   uint16_t *__restrict__ bc, int M, int N, int G, int Kx) {
    pdl_launch_dependents();   // the GEMM may start its prologue
    pdl_wait();                // x may come from the previous kernel of the stream
    const long long K = static_cast<long long>(G) * 128;
    const long long threads = static_cast<long long>(gridDim.x) * blockDim.x;
    const long long tid = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
    const int lane = threadIdx.x & 31, half = lane >> 4, l16 = lane & 15;
    // x: each half-warp sums one (row m, group g): one 16-byte load per lane, then the
    // 16 lanes' sums; the loop bound is warp-uniform so that every lane takes each shuffle
    const long long mg = static_cast<long long>(M) * G;
    for (long long wu = (tid >> 5) * 2; wu < mg; wu += (threads >> 5) * 2) {
        const long long u = wu + half;
        const bool live = u < mg;
        const long long r = live ? u / G : 0;
        const int g = live ? static_cast<int>(u - r * G) : 0;
        float sum = 0.f;
        if (live) {
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(x + r * K + g * 128) + l16);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                sum += bf16_lo_to_f32(w[j]);
                sum += bf16_hi_to_f32(w[j]);
            }
        }
#pragma unroll
        for (int o = 1; o < 16; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (live && l16 == 0) {
            const uint32_t p0 = __bfloat16_as_ushort(__float2bfloat16_rn(sum));
            const float r1 = sum - bf16_to_f32(p0);
            const uint32_t p1 = __bfloat16_as_ushort(__float2bfloat16_rn(r1));
            const uint32_t p2 = __bfloat16_as_ushort(__float2bfloat16_rn(r1 - bf16_to_f32(p1)));
            uint16_t *row = xs + r * Kx;
            uint32_t *dst = reinterpret_cast<uint32_t *>(row + kBiasCoef * g);   // 4-byte aligned
            dst[0] = p0 | (p1 << 16);
            dst[1] = p2 | (p0 << 16);
            dst[2] = p1 | (p2 << 16);
            if (g == G - 1)
                for (int c = kBiasCoef * G; c < Kx; c += 2) *reinterpret_cast<uint32_t *>(row + c) = 0u;
        }
    }
    // coefficients: one thread per (weight row n, group g)
    const long long ng = static_cast<long long>(N) * G;
    for (long long item = tid; item < ng; item += threads) {
        const long long r = item / G;
        const int g = static_cast<int>(item - r * G);
        const uint32_t b = __ldg(biases + r * G + g);
        const uint32_t t = __bfloat16_as_ushort(__float2bfloat16_rn(-16.f * bf16_to_f32(__ldg(scales + r * G + g))));
        uint16_t *row = bc + r * Kx;
        uint32_t *dst = reinterpret_cast<uint32_t *>(row + kBiasCoef * g);
        dst[0] = b | (b << 16);
        dst[1] = b | (t << 16);
        dst[2] = t | (t << 16);
        if (g == G - 1)
            for (int c = kBiasCoef * G; c < Kx; c += 2) *reinterpret_cast<uint32_t *>(row + c) = 0u;
    }
}

// ------------------------------------------------------------------ GEMM

__device__ __forceinline__ uint32_t bf16x2_128_plus_8q(uint32_t v3, uint32_t v1, uint32_t sel) {
    // bytes sel of (v3 = v << 3, v1 = v >> 1): byte j of v3 holds code 2j in bits 3-6, byte j
    // of v1 code 2j + 1 -> two codes in bits 3-6 and 19-22 -> BF16 128 + 8 code
    return codes_to_bf16x2_128_plus_8q(prmt(v3, v1, sel));
}

// 64 consecutive 32-bit columns of this thread's lane into registers (warp-collective;
// the lane field of taddr is the warp's 32-lane quarter).  The registers are written
// asynchronously: read them only after tmem_ld_wait64, which also pins them.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait64(uint32_t (&r)[64]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;" : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31]), "+r"(r[32]), "+r"(r[33]), "+r"(r[34]), "+r"(r[35]), "+r"(r[36]), "+r"(r[37]), "+r"(r[38]), "+r"(r[39]), "+r"(r[40]), "+r"(r[41]), "+r"(r[42]), "+r"(r[43]), "+r"(r[44]), "+r"(r[45]), "+r"(r[46]), "+r"(r[47]), "+r"(r[48]), "+r"(r[49]), "+r"(r[50]), "+r"(r[51]), "+r"(r[52]), "+r"(r[53]), "+r"(r[54]), "+r"(r[55]), "+r"(r[56]), "+r"(r[57]), "+r"(r[58]), "+r"(r[59]), "+r"(r[60]), "+r"(r[61]), "+r"(r[62]), "+r"(r[63]) :: "memory");
}

// a = s * x + a on two FP32 lanes at once (x a pair of FP32 bit patterns)
__device__ __forceinline__ void ffma2(unsigned long long &a, unsigned long long s2, uint32_t x0, uint32_t x1) {
    unsigned long long x;
    asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "r"(x0), "r"(x1));
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(a) : "l"(s2), "l"(x));
}
__device__ __forceinline__ unsigned long long f32x2(float lo, float hi) {
    unsigned long long v;
    asm("mov.b64 %0, {%1, %2};" : "=l"(v) : "f"(lo), "f"(hi));
    return v;
}
__device__ __forceinline__ float f32x2_lo(unsigned long long v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float f32x2_hi(unsigned long long v) { return __uint_as_float(static_cast<uint32_t>(v >> 32)); }

__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

__device__ __forceinline__ bool bf16_not_finite(uint16_t h) { return (h & 0x7F80u) == 0x7F80u; }

// BF16 of the plain definition of y[m, n] (outputs whose fast result is not finite).
__device__ __forceinline__ uint16_t plain_output_bf16(const Params &p, long long m, long long n) {
    const long long G = p.G;
    return __bfloat16_as_ushort(__float2bfloat16_rn(
        plain_output(p.x + m * 128 * G, p.wq + n * 16 * G, p.scales + n * G, p.biases + n * G, p.G)));
}

// Tile t of the output: its x rows start at 128 m, this CTA's weight rows at row0.
struct TileCoord {
    int m;
    long long row0;
};
__device__ __forceinline__ TileCoord tile_coord(long long t, int tiles_n, int pair_rank) {
    const long long m = t / tiles_n;
    return {static_cast<int>(m), (t - m * tiles_n) * kPairRows + pair_rank * BN};
}

// Position in a ring of N slots: slot and the parity of its current use.
template <int N>
struct RingPos {
    int slot = 0;
    uint32_t phase = 0;
    __device__ __forceinline__ void advance() {
        if (++slot == N) {
            slot = 0;
            phase ^= 1u;
        }
    }
};

__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_xs,
                const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_y, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
    uint64_t *ready = bars, *done = ready + kXStages;
    uint64_t *w_full = done + kXStages, *w_empty = w_full + kWStages;
    uint64_t *sc_full = w_empty + kWStages, *sc_empty = sc_full + kScaleBufsMax;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kNumBars);
    uint16_t *sc_smem = reinterpret_cast<uint16_t *>(smem + kOffScales);
    uint16_t *out_tile = reinterpret_cast<uint16_t *>(smem + kOffOut);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();               // 2 split + pair rank
    const int pair_rank = static_cast<int>(rank & 1u);
    const uint32_t leader = rank & ~1u;
    const bool is_leader = pair_rank == 0;
    const int split = static_cast<int>(rank >> 1);
    const int G = p.G;
    const int g0 = static_cast<int>(static_cast<long long>(split) * G / p.splits);
    const int g1 = static_cast<int>(static_cast<long long>(split + 1) * G / p.splits);
    const int ng = g1 - g0;
    // bias steps t = split, split + S, ... < Kx / 128 come first, then the groups g0 .. g1-1
    const int nbias_all = p.Kx / 128;
    const int nbs = split < nbias_all ? (nbias_all - split + p.splits - 1) / p.splits : 0;
    const int steps = nbs + ng;
    const int nsb = scale_bufs(G);
    // Tile schedule.  Without a K split the grid is persistent: cluster c = blockIdx.y
    // computes tiles c, c + gridDim.y, ... (tile t: tile_n = t % tiles_n, tile_m = t / tiles_n,
    // so neighbouring clusters share x rows), and one tile's pipeline drains while the next
    // one's fills.  With a K split each cluster computes the one tile (blockIdx.z, blockIdx.y),
    // whose partials are reduced through shared memory at the end.
    const bool persistent = p.splits == 1;
    const long long tile0 = persistent ? static_cast<long long>(blockIdx.y)
                                       : static_cast<long long>(blockIdx.z) * p.tiles_n + blockIdx.y;
    const long long tstride = persistent ? static_cast<long long>(gridDim.y) : p.tiles;
    const int ntl = tile0 < p.tiles ? static_cast<int>((p.tiles - tile0 + tstride - 1) / tstride) : 0;
    const long long total = static_cast<long long>(ntl) * steps;   // steps of this CTA

    if (threadIdx.x == 0) {
        pdl_launch_dependents();
        // ready: the leader's x transaction, the dequantisation and the epilogue warps of both CTAs
        for (int i = 0; i < kXStages; ++i) { mbar_init(&ready[i], 1 + 2 * kDeqWarps + 2 * kEpiWarps); mbar_init(&done[i], 1); }
        for (int i = 0; i < kWStages; ++i) { mbar_init(&w_full[i], 1); mbar_init(&w_empty[i], kDeqWarps); }
        for (int i = 0; i < kScaleBufsMax; ++i) { mbar_init(&sc_full[i], 1); mbar_init(&sc_empty[i], kEpiWarps); }
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

    if (warp < kWarpDeq) {
        regs_shrink<kRegsCtl>();
        if (warp == kWarpTma && lane == 0) {
            // -------------------------------------------------------- TMA producer of x / Xs (both CTAs)
            prefetch_tmap(&tm_x);
            prefetch_tmap(&tm_xs);
            if (p.tma_store) prefetch_tmap(&tm_y);
            pdl_wait();   // x (and the group sums) come from the preceding kernels
            RingPos<kXStages> st;
            long long issued = 0;
            bool ok = true;
            long long t = tile0;
            for (int k = 0; k < ntl && ok; ++k, t += tstride) {
                const int xrow = tile_coord(t, p.tiles_n, pair_rank).m * BM + pair_rank * kXRows;
                for (int i = 0; i < steps; ++i) {
                    // the stage is free once the MMAs of its previous step completed
                    if (issued >= kXStages && !mbar_wait(&done[st.slot], st.phase ^ 1u)) { ok = false; break; }
                    if (is_leader) mbar_arrive_expect_tx(&ready[st.slot], 2 * kXBytes);   // both halves
                    uint8_t *dst = smem + st.slot * kXBytes;
                    const CUtensorMap *map = i < nbs ? &tm_xs : &tm_x;
                    const int col = i < nbs ? (split + i * p.splits) * 128 : (g0 + i - nbs) * 128;
                    tma_load_2d_pair(dst, map, ready_l + 8 * st.slot, col, xrow);
                    tma_load_2d_pair(dst + kXAtom, map, ready_l + 8 * st.slot, col + 64, xrow);
                    ++issued;
                    st.advance();
                }
            }
            // leave no copy in flight: the last stages' MMAs (which consumed them) completed
            for (long long j = issued > kXStages ? issued - kXStages : 0; j < issued; ++j)
                mbar_wait(&done[j % kXStages], static_cast<uint32_t>((j / kXStages) & 1), false);
        } else if (warp == kWarpCodes && lane == 0) {
            // -------------------------------------------------------- codes and scales, by TMA (both CTAs)
            // The packed codes of each group, and after a tile's second group that tile's
            // scales (one contiguous [rows][G] BF16 block: a 1-D bulk copy) into their buffer.
            prefetch_tmap(&tm_w);
            if (!p.static_weights) pdl_wait();
            RingPos<kWStages> st;
            long long issued = 0;
            int staged = 0;   // tiles whose scales were staged
            bool ok = true;
            long long t = tile0;
            for (int k = 0; k < ntl && ok; ++k, t += tstride) {
                const long long row0 = tile_coord(t, p.tiles_n, pair_rank).row0;
                const int stage_at = ng > 1 ? 1 : 0;
                for (int j = 0; j < ng; ++j) {
                    if (issued >= kWStages && !mbar_wait(&w_empty[st.slot], st.phase ^ 1u)) { ok = false; break; }
                    mbar_arrive_expect_tx(&w_full[st.slot], kWBytes);
                    tma_load_2d(smem + kOffW + st.slot * kWBytes, &tm_w, &w_full[st.slot], (g0 + j) * 16,
                                static_cast<int>(row0));
                    ++issued;
                    st.advance();
                    if (j == stage_at) {
                        const int sb = nsb == 2 ? (k & 1) : 0;
                        const uint32_t use = static_cast<uint32_t>(nsb == 2 ? (k >> 1) : k);
                        // the epilogue is done with this buffer's previous tile
                        if (k >= nsb && !mbar_wait(&sc_empty[sb], (use & 1u) ^ 1u)) { ok = false; break; }
                        uint16_t *dst = sc_smem + sb * BN * G;
                        const uint16_t *src = p.scales + row0 * G;   // 16-byte aligned: row0 is a multiple of 128
                        // rows of this CTA inside y: none when the pair's second half lies past N
                        const int rows = static_cast<int>(max(0ll, min(static_cast<long long>(BN), p.N - row0)));
                        const uint32_t bytes = static_cast<uint32_t>(rows * G * 2);
                        const uint32_t bulk = bytes & ~15u;
                        for (uint32_t e = bulk / 2; e < bytes / 2; ++e) dst[e] = __ldg(src + e);   // ragged end
                        mbar_arrive_expect_tx(&sc_full[sb], bulk);
                        if (bulk) bulk_load(dst, src, bulk, &sc_full[sb]);
                        ++staged;
                    }
                }
            }
            // leave no copy in flight
            for (long long q = issued > kWStages ? issued - kWStages : 0; q < issued; ++q)
                mbar_wait(&w_full[q % kWStages], static_cast<uint32_t>((q / kWStages) & 1), false);
            for (int k = staged > nsb ? staged - nsb : 0; k < staged; ++k) {
                const int sb = nsb == 2 ? (k & 1) : 0;
                const uint32_t use = static_cast<uint32_t>(nsb == 2 ? (k >> 1) : k);
                mbar_wait(&sc_full[sb], use & 1u, false);
            }
        } else if (warp == kWarpMma && lane == 0 && is_leader) {
            // -------------------------------------------------------- MMA issuer (pair leader)
            // One thread issues every step: with a second issuing thread on another SM
            // sub-partition, the tensor-memory lanes of both sub-partitions were measured to
            // receive wrong values now and then.  Per step it waits on one barrier (the step's
            // x, A and accumulator are all ready), issues the eight MMAs and one commit, and
            // nothing else: the tensor pipe holds about one MMA ahead of the issuing thread, and
            // every further barrier test in the loop would idle it.  The MMAs do not depend
            // on the tile.
            constexpr uint32_t idesc = umma_idesc_bf16(kPairRows, BM);
            const uint16_t mask = static_cast<uint16_t>(3u << leader);
            RingPos<kXStages> xs;      // step g: ready[g % kXStages], its x stage, done[g % kXStages]
            int ab = 0, db = 0;        // A buffer g % kABufs, accumulator g % kDBufs
            for (long long g = 0; g < total; ++g) {
                if (!mbar_wait_spin(&ready[xs.slot], xs.phase)) break;
                tc_fence_after();
                const uint32_t b0 = smem_u32(smem + xs.slot * kXBytes);
                const uint32_t d = tmem_base + db * BM;
                const uint32_t a = tmem_base + kACol0 + ab * kACols;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t bd = umma_desc_sw128(b0 + (kk >> 2) * kXAtom + (kk & 3) * 32);
                    umma_bf16_ts_pair(d, a + 8 * kk, bd, idesc, kk > 0);
                }
                umma_commit_pair(&done[xs.slot], mask);
                xs.advance();
                ab = (ab + 1) & (kABufs - 1);
                db ^= 1;
            }
        }
        __syncwarp();
        named_bar_sync(kBarRegs, kThreads);   // the epilogue has returned its registers
        regs_grow<kLaunchRegs>();             // back to the launch allocation for the common tail
    } else if (warp < kWarpEpi) {
        regs_shrink<kRegsDeq>();
        // ------------------------------------------------------------ dequantisation (both CTAs)
        const int quarter = warp & 3, half = (warp - kWarpDeq) >> 2;
        const int rl = quarter * 32 + lane;                  // row within the CTA's codes tile
        const uint32_t sw = static_cast<uint32_t>((rl >> 1) & 3);   // 64-byte swizzle of that row
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + kACol0 + half * 32;
        pdl_wait();   // the bias-step coefficients come from the preparation kernel
        RingPos<kXStages> rs;   // step g: ready[g % kXStages]
        RingPos<kXStages> fs;   // step g - kABufs: done[...], the MMAs that last read A buffer g % kABufs
        RingPos<kWStages> cs;   // codes ring
        int ab = 0;
        long long g = 0;
        bool ok = true;
        long long t = tile0;
        for (int k = 0; k < ntl && ok; ++k, t += tstride) {
            const long long row = tile_coord(t, p.tiles_n, pair_rank).row0 + rl;   // weight row n
            const bool row_ok = row < p.N;
            const uint4 *bcrow = reinterpret_cast<const uint4 *>(p.bc + (row_ok ? row : 0) * static_cast<long long>(p.Kx));
            for (int i = 0; i < steps; ++i, ++g) {
                uint32_t r[32];
                if (i >= nbs) {
                    // chunks 2 half, 2 half + 1 (words 8 half .. 8 half + 7) of this row's codes
                    if (!mbar_wait(&w_full[cs.slot], cs.phase)) { ok = false; break; }
                    const uint32_t wrow = smem_u32(smem + kOffW + cs.slot * kWBytes) + rl * 64;
                    const uint4 c0 = lds128(wrow + (((2u * half) ^ sw) << 4));
                    const uint4 c1 = lds128(wrow + (((2u * half + 1u) ^ sw) << 4));
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&w_empty[cs.slot]);   // the codes are in registers
                    cs.advance();
                    if (g >= kABufs && !mbar_wait(&done[fs.slot], fs.phase)) { ok = false; break; }
                    tc_fence_after();   // the tensor cores' reads of this buffer precede the stores below
                    const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj) {   // word jj: k = 8 jj .. 8 jj + 7 -> columns 4 jj .. 4 jj + 3
                        const uint32_t v3 = w[jj] << 3, v1 = w[jj] >> 1;
                        r[4 * jj + 0] = bf16x2_128_plus_8q(v3, v1, 0x0400u);
                        r[4 * jj + 1] = bf16x2_128_plus_8q(v3, v1, 0x0501u);
                        r[4 * jj + 2] = bf16x2_128_plus_8q(v3, v1, 0x0602u);
                        r[4 * jj + 3] = bf16x2_128_plus_8q(v3, v1, 0x0703u);
                    }
                } else {   // 64 coefficients of this column half (bias steps are few: loaded here)
                    const int t = split + i * p.splits;
                    uint4 v[8];
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj)
                        v[jj] = row_ok ? ldg_nc_v4(bcrow + t * 16 + half * 8 + jj) : make_uint4(0, 0, 0, 0);
                    if (g >= kABufs && !mbar_wait(&done[fs.slot], fs.phase)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj) {
                        r[4 * jj + 0] = v[jj].x;
                        r[4 * jj + 1] = v[jj].y;
                        r[4 * jj + 2] = v[jj].z;
                        r[4 * jj + 3] = v[jj].w;
                    }
                }
                if (g >= kABufs) fs.advance();
                tmem_st32(taddr + ab * kACols, r);
                tmem_st_wait_regs(r);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(ready_l + 8 * rs.slot);
                rs.advance();
                ab = (ab + 1) & (kABufs - 1);
            }
        }
        named_bar_sync(kBarRegs, kThreads);
        regs_grow<kLaunchRegs>();
    } else {
        regs_grow<kRegsEpi>();
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int quarter = warp & 3, half = (warp - kWarpEpi) >> 2;
        const int nl = quarter * 32 + lane;                         // weight row within the CTA
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + half * 64;
        RingPos<kXStages> ds;   // step g: done[g % kXStages]
        RingPos<kXStages> fs;   // step g + kDBufs: ready[...], which the accumulator of step g frees
        int db = 0;
        long long ge = 0;       // step index across the tiles
        bool ok = true;
        // the first kDBufs steps find their accumulators free
        for (int j = 0; j < kDBufs; ++j) {
            if (lane == 0 && j < total) mbar_arrive_cluster(ready_l + 8 * fs.slot);
            fs.advance();
        }
        // Every epilogue warp takes both named barriers of every tile, also after a failed
        // wait, so that none is left waiting on a barrier that the others skipped.
        long long t = tile0;
        for (int k = 0; k < ntl; ++k, t += tstride) {
            const TileCoord tc = tile_coord(t, p.tiles_n, pair_rank);
            const int tile_m = tc.m;
            const long long row0 = tc.row0;
            const long long row = row0 + nl;
            const bool row_ok = row < p.N;
            const int sb = nsb == 2 ? (k & 1) : 0;
            const uint32_t use = static_cast<uint32_t>(nsb == 2 ? (k >> 1) : k);
            if (ok && !mbar_wait(&sc_full[sb], use & 1u)) ok = false;   // this tile's scales are staged
            const uint16_t *srow = sc_smem + sb * BN * G + nl * G;
            unsigned long long acc2[32];   // FP32 pairs: x rows 2j, 2j + 1 of this warp's 64
#pragma unroll
            for (int j = 0; j < 32; ++j) acc2[j] = 0ull;
            for (int i = 0; i < steps && ok; ++i) {
                const float sc = (row_ok && i >= nbs) ? 0.125f * bf16_to_f32(srow[g0 + i - nbs]) : 1.f;   // s / 8
                if (!mbar_wait(&done[ds.slot], ds.phase)) { ok = false; break; }
                tc_fence_after();
                uint32_t r[64];
                tmem_ld64(taddr + db * BM, r);
                tmem_ld_wait64(r);
                tc_fence_before();
                __syncwarp();
                if (lane == 0 && ge + kDBufs < total) mbar_arrive_cluster(ready_l + 8 * fs.slot);   // accumulator free
                fs.advance();
                ++ge;
                const unsigned long long sc2 = f32x2(sc, sc);
#pragma unroll
                for (int j = 0; j < 32; ++j) ffma2(acc2[j], sc2, r[2 * j], r[2 * j + 1]);
                ds.advance();
                db ^= 1;
            }
            float acc[64];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                acc[2 * j] = f32x2_lo(acc2[j]);
                acc[2 * j + 1] = f32x2_hi(acc2[j]);
            }

            __syncwarp();
            if (lane == 0) mbar_arrive(&sc_empty[sb]);   // this tile's scales are no longer read
            if (k == 0) pdl_wait();   // y may still be read by the preceding kernel
            const int m0 = tile_m * BM + half * 64;
            if (p.splits > 1) {
                // split-K (one tile per CTA): this CTA's partial, [x row][weight row] FP32,
                // into the x stages, idle once the loop is over
                float *part = reinterpret_cast<float *>(smem);
#pragma unroll
                for (int j = 0; j < 64; ++j) part[(half * 64 + j) * BN + nl] = acc[j];
            } else if (p.tma_store) {
                // the tile, [x row][weight row] BF16, into the staging buffer, then one TMA store
                // that overlaps the next tile's main loop
                if (warp == kWarpEpi && lane == 0) bulk_wait_read_all();   // the previous store read it
                named_bar_sync(kBarEpi, kEpiWarps * 32);
                unsigned long long bad = 0ull;   // outputs whose fast result is not finite
#pragma unroll
                for (int j = 0; j < 64; ++j) {
                    const uint16_t h = __bfloat16_as_ushort(__float2bfloat16_rn(acc[j]));
                    out_tile[(half * 64 + j) * BN + nl] = h;
                    if (bf16_not_finite(h)) bad |= 1ull << j;
                }
                for (; bad && row_ok; bad &= bad - 1) {   // the plain definition for those (rare)
                    const int j = __ffsll(static_cast<long long>(bad)) - 1;
                    if (m0 + j < p.M)
                        out_tile[(half * 64 + j) * BN + nl] = plain_output_bf16(p, m0 + j, row);
                }
                fence_proxy_async_smem();   // the async proxy reads the tile
                named_bar_sync(kBarEpi, kEpiWarps * 32);
                if (ok && warp == kWarpEpi && lane == 0) {
                    tma_store_2d(&tm_y, out_tile, static_cast<int>(row0), tile_m * BM);
                    bulk_commit_group();
                }
            } else if (row_ok && ok) {
                unsigned long long bad = 0ull;   // outputs whose fast result is not finite
#pragma unroll
                for (int j = 0; j < 64; ++j)
                    if (m0 + j < p.M) {
                        const uint16_t h = __bfloat16_as_ushort(__float2bfloat16_rn(acc[j]));
                        p.y[static_cast<long long>(m0 + j) * p.N + row] = h;
                        if (bf16_not_finite(h)) bad |= 1ull << j;
                    }
                for (; bad; bad &= bad - 1) {   // the plain definition for those (rare)
                    const int j = __ffsll(static_cast<long long>(bad)) - 1;
                    p.y[static_cast<long long>(m0 + j) * p.N + row] = plain_output_bf16(p, m0 + j, row);
                }
            }
        }
        if (p.tma_store && warp == kWarpEpi && lane == 0)
            bulk_wait_all();   // y written, and shared memory released, before the CTA ends
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
    if (p.splits > 1 && ntl == 1) {
        // Split-K reduction over the S pairs of the cluster: the CTAs with this pair rank
        // hold the S partials of the same 128 weight rows; the one of split r sums x rows
        // [r*R, (r+1)*R) of them, in split order, through distributed shared memory.
        const TileCoord tc = tile_coord(tile0, p.tiles_n, pair_rank);
        const int tile_m = tc.m;
        const long long row0 = tc.row0;
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
                // every partial in flight at once (a remote load takes about a microsecond),
                // then added in split order
                float4 w[kMaxSplits];
#pragma unroll
                for (int sp = 0; sp < kMaxSplits; ++sp)
                    if (sp < S) w[sp] = ld_dsmem_f4(dsmem_addr(off, static_cast<uint32_t>(2 * sp + pair_rank)));
                float4 v = w[0];
#pragma unroll
                for (int sp = 1; sp < kMaxSplits; ++sp)
                    if (sp < S) {
                        v.x += w[sp].x; v.y += w[sp].y; v.z += w[sp].z; v.w += w[sp].w;
                    }
                const long long mrow = static_cast<long long>(tile_m) * BM + ml;
                const long long n = row0 + 4 * c4;
                if (mrow < p.M) {
                    // outputs whose fast result is not finite: the plain definition
                    if (!isfinite(v.x) && n < p.N) v.x = plain_output(p.x + mrow * 128ll * G, p.wq + n * 16ll * G, p.scales + n * G, p.biases + n * G, G);
                    if (!isfinite(v.y) && n + 1 < p.N) v.y = plain_output(p.x + mrow * 128ll * G, p.wq + (n + 1) * 16ll * G, p.scales + (n + 1) * G, p.biases + (n + 1) * G, G);
                    if (!isfinite(v.z) && n + 2 < p.N) v.z = plain_output(p.x + mrow * 128ll * G, p.wq + (n + 2) * 16ll * G, p.scales + (n + 2) * G, p.biases + (n + 2) * G, G);
                    if (!isfinite(v.w) && n + 3 < p.N) v.w = plain_output(p.x + mrow * 128ll * G, p.wq + (n + 3) * 16ll * G, p.scales + (n + 3) * G, p.biases + (n + 3) * G, G);
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
