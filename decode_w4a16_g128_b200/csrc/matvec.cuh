// matvec.cuh - weight-streaming W4A16 kernel for M <= 8 (decode).
//
// Role in the layer: tiny-llm "Week 2 Day 6: SIMD-Matrix Prefill", Task 1,
// keeps a matvec schedule for M <= 8.  This is a B200 design, not that
// Metal kernel: the whole cost is reading the packed weights once (0.5 byte
// per weight plus 4 bytes of scale and bias per 128 weights), so the kernel is
// built around keeping HBM busy with few, large asynchronous copies.
//
// Work decomposition ("stream-K"): the output rows are cut into tiles of
// kRows = 128 rows, and each (row tile, 128-group) pair is one unit of work.
// The U = tiles * G units are split into `workers` contiguous ranges, one
// persistent CTA each (CTA c owns [c*U/P, (c+1)*U/P)), so every SM streams the
// same number of bytes whatever N and K are.  A tile whose groups are spread
// over several CTAs is finished by the CTA that completes it last: every
// contributor writes its FP32 partial to the workspace, and the last one to
// arrive (a per-tile atomic ticket) adds the partials in CTA order, so the sum
// does not depend on arrival order.
//
// Data movement: one thread of the producer warp walks the CTA's units two at
// a time (a "stage" holds one or two consecutive groups of one tile) and issues
// per stage one TMA tile load of packed codes ([128 rows x 128 bytes], 128-byte
// swizzle, 16 KB) and one of x ([M rows x 264] BF16: two groups plus 8
// staggering columns).  Once per row tile it issues 1-D bulk copies of the
// tile's scale and bias rows (128 x G BF16 each, contiguous in memory) into a
// small slab ring.  With the static-weights flag it issues the code and
// scale/bias copies of the first stages before waiting on the preceding kernel
// of the stream (programmatic dependent launch), so they overlap that kernel's
// tail; x is always read after the wait.
//
// Compute: 8 consumer warps each own 16 rows and run m16n8k16 BF16
// tensor-core MMAs with the codes as the A operand (16 rows x 16 k) and x as
// the B operand (16 k x 8 columns = the M <= 8 activation rows, zero-padded).
// MMA row p of warp w reads data row 16w + row_of(p): pairing rows r and r+4
// in each quarter warp makes the 128-byte swizzle spread its 16-byte reads
// over all banks.
//
// Dequantisation (Task 3 of the same page: one scale and bias per 128
// reduction values):
//   sum_k x[m,k] w[n,k] = sum_g ( s[n,g] * P[m,n,g] + b[n,g] * X[m,g] ),
//   P[m,n,g] = sum_{k in g} x[m,k] q[n,k],  X[m,g] = sum_{k in g} x[m,k].
// Codes enter the MMA as the exact BF16 values 128 + q (one LOP3 per two
// codes), so the MMA yields P + 128 X; X itself comes from MMAs with an
// all-ones A operand, computed once per stage by one warp (the duty rotates
// over the warps) and shared through shared memory; the epilogue applies s and
// (b - 128 s) once per group in FP32.  Every product is exact; only FP32 sums
// round.
#pragma once

#include "ptx.cuh"

namespace w4a16 {
namespace mv {

constexpr int kMaxM = 8;
constexpr int kWarps = 8;                 // consumer warps, 16 rows each
constexpr int kRows = 16 * kWarps;        // rows of a tile
constexpr int kThreads = (kWarps + 1) * 32;
constexpr int kGroupsPerStage = 2;
constexpr int kWBytes = kRows * 64 * kGroupsPerStage;   // 16 KB of codes per stage
constexpr int kXCols = 128 * kGroupsPerStage + 8;      // 264: 8 staggering columns
constexpr int kXRowBytes = kXCols * 2;                 // 528 B: x rows 16 B apart in bank space
constexpr int kXBytes = ((kMaxM * kXRowBytes + 1023) / 1024) * 1024;   // keeps stages 1 KB aligned
constexpr int kStageBytes = kWBytes + kXBytes;
constexpr int kFlagStaticWeights = 2;    // codes, scales and biases may be read before the wait
constexpr int kFixupBatch = 8;           // contributors whose partials are loaded at once
static_assert(kWBytes % 1024 == 0 && kStageBytes % 1024 == 0, "swizzled stages need 1 KB alignment");

// bytes of one scale (or bias) slab: kRows x G BF16, rounded to 128 B
__host__ __device__ constexpr long long slab_array_bytes(long long G) { return ((kRows * G * 2 + 127) / 128) * 128; }
__host__ __device__ constexpr long long xs_ring(int stages) { return 2 * stages; }
__host__ __device__ constexpr long long smem_bytes(int stages, int slab_slots, long long G) {
    return stages * kStageBytes + slab_slots * 2 * slab_array_bytes(G)
           + xs_ring(stages) * kGroupsPerStage * kMaxM * 4          // shared X values
           + (2 * stages + xs_ring(stages) + 4) * 8 + 16 + 1024;    // barriers, ticket, alignment slack
}

struct Params {
    const uint16_t *scales;   // bf16 [N, G]
    const uint16_t *biases;   // bf16 [N, G]
    uint16_t *y;              // bf16 [M, N]
    float *partials;          // [workers][2][kRows * 8] FP32
    int *tickets;             // [tiles], zero between launches
    int M, N, G;
    int tiles;
    long long units;          // tiles * G
    int workers;              // gridDim.x
    int stages;               // depth of the code/x ring
    int slab_slots;           // 0 (scales/biases read from global), 1 or 2
    int slab_array_bytes;     // slab_array_bytes(G)
    int flags;                // kFlagStaticWeights
};

// CTA whose range [c*U/P, (c+1)*U/P) contains unit u.
__host__ __device__ __forceinline__ long long streamk_owner(long long U, long long P, long long u) {
    return ((u + 1) * P - 1) / U;
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float v) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }

// Walks a CTA's unit range stage by stage: a stage is one or two consecutive
// groups of the same row tile.
struct StageWalker {
    int t, g;           // tile and first group of the current stage
    int n;              // groups in the current stage (1 or 2)
    long long left;     // units not yet walked (including the current stage)
    int G;
    __device__ void start(long long u0, long long u1, int G_) {
        G = G_;
        t = static_cast<int>(u0 / G);
        g = static_cast<int>(u0 - static_cast<long long>(t) * G);
        left = u1 - u0;
        n = pick();
    }
    __device__ int pick() const { return (left >= 2 && g + 1 < G) ? 2 : (left >= 1 ? 1 : 0); }
    __device__ void next() {
        left -= n;
        g += n;
        if (g == G) { g = 0; ++t; }
        n = pick();
    }
    __device__ bool tile_ends() const { return g + n == G || left == n; }
};

// data row (within a warp's 16) of MMA row p: quarter warps pair rows r, r+4
__device__ __forceinline__ int row_of(int p) { return (p & 8) | ((p & 1) << 2) | ((p >> 1) & 3); }

// At most 112 registers per thread, so that two CTAs fit on an SM: one of this
// launch and one of the next launch in the stream.
__global__ void __maxnreg__(112)
    matvec_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                  const Params p) {
    extern __shared__ uint8_t smem_raw[];
    // 1 KB alignment for the swizzled code tiles, by offsetting within the shared
    // array (so the compiler still knows every access below is a shared-memory one).
    // x is loaded through a uint32 view of [M, K/2] pairs, so its 264-column box is a
    // legal 132-element box.
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int S = p.stages;
    const int XR = static_cast<int>(xs_ring(S));
    uint8_t *slab_base = smem + S * kStageBytes;
    float *xs_base = reinterpret_cast<float *>(slab_base + p.slab_slots * 2 * p.slab_array_bytes);
    uint64_t *full = reinterpret_cast<uint64_t *>(xs_base + XR * kGroupsPerStage * kMaxM);
    uint64_t *empty = full + S;
    uint64_t *xs_full = empty + S;
    uint64_t *slab_full = xs_full + XR;
    uint64_t *slab_empty = slab_full + 2;
    int *ticket_flag = reinterpret_cast<int *>(slab_empty + 2);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const long long U = p.units;
    const long long P = p.workers;
    const long long cta = blockIdx.x;
    const long long u0 = cta * U / P;
    const long long u1 = (cta + 1) * U / P;
    const int G = p.G;
    const int slots = p.slab_slots;

    if (threadIdx.x == 0) {
        // the next kernel of the stream may start its prologue while this one runs
        pdl_launch_dependents();
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);         // producer's arrive.expect_tx; bytes complete the phase
            mbar_init(&empty[s], kWarps);   // one arrival per consumer warp
        }
        for (int s = 0; s < XR; ++s) mbar_init(&xs_full[s], 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&slab_full[s], 1);
            mbar_init(&slab_empty[s], kWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kWarps) {
        // ------------------------------------------------------------ producer (one thread)
        if (lane != 0) return;
        prefetch_tmap(&tm_w);
        prefetch_tmap(&tm_x);
        const uint32_t tx_bytes = kWBytes + p.M * kXRowBytes;
        const bool prefetch = (p.flags & kFlagStaticWeights) != 0;
        int tile_seq = -1, prev_t = -1, slabs_issued = 0;

        // scale and bias rows of tile t into slab slot (seq % slots)
        auto issue_slab = [&](int t, int seq) -> bool {
            if (slots == 0) return true;
            const int slot = seq % slots;
            if (seq >= slots && !mbar_wait(&slab_empty[slot], ((seq / slots) - 1) & 1)) return false;
            const long long first = static_cast<long long>(t) * kRows;
            const long long rows = min(static_cast<long long>(kRows), p.N - first);
            const uint32_t bytes = static_cast<uint32_t>(rows * G * 2) & ~15u;   // tail read from global
            uint8_t *dst = slab_base + slot * 2 * p.slab_array_bytes;
            if (bytes) {
                mbar_arrive_expect_tx(&slab_full[slot], 2 * bytes);
                bulk_load(dst, p.scales + first * G, bytes, &slab_full[slot]);
                bulk_load(dst + p.slab_array_bytes, p.biases + first * G, bytes, &slab_full[slot]);
            } else {
                mbar_arrive(&slab_full[slot]);
            }
            slabs_issued = seq + 1;
            return true;
        };
        // codes (and slab) of stage i; may_recycle == false: stop rather than wait for a
        // slab slot the consumers still hold (they cannot release it before x arrives)
        auto issue_codes = [&](const StageWalker &wk, int i, bool may_recycle) -> bool {
            if (wk.t != prev_t) {
                if (!may_recycle && slots && tile_seq + 1 >= slots) return false;
                prev_t = wk.t;
                if (!issue_slab(wk.t, ++tile_seq)) return false;
            }
            const int s = i % S;
            mbar_arrive_expect_tx(&full[s], tx_bytes);
            tma_load_2d(smem + s * kStageBytes, &tm_w, &full[s], wk.g * 16, wk.t * kRows);
            return true;
        };
        auto issue_x = [&](const StageWalker &wk, int i) {
            const int s = i % S;
            tma_load_2d(smem + s * kStageBytes + kWBytes, &tm_x, &full[s], wk.g * 64, 0);
        };

        StageWalker wk;
        wk.start(u0, u1, G);
        int issued = 0;
        if (prefetch) {   // empty ring: no waits needed
            StageWalker pw = wk;
            for (int i = 0; i < S && pw.n; ++i) {
                if (!issue_codes(pw, i, /*may_recycle=*/false)) break;
                issued = i + 1;
                pw.next();
            }
        }
        pdl_wait();   // x (and, without the flag, everything) may come from the previous kernel
        for (int i = 0; i < issued; ++i, wk.next()) issue_x(wk, i);
        for (int i = issued; wk.n; ++i, wk.next()) {
            const int s = i % S;
            if (i >= S && !mbar_wait(&empty[s], ((i / S) - 1) & 1)) break;
            if (!issue_codes(wk, i, /*may_recycle=*/true)) break;
            issue_x(wk, i);
            issued = i + 1;
        }
        // Leave no copy in flight: wait (bounded) for the stages and slabs issued last.
        for (int i = max(0, issued - S); i < issued; ++i)
            mbar_wait(&full[i % S], (i / S) & 1, /*give_up_on_status=*/false);
        for (int q = max(0, slabs_issued - slots); q < slabs_issued; ++q)
            mbar_wait(&slab_full[q % slots], (q / slots) & 1, /*give_up_on_status=*/false);
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int gq = lane >> 2;       // MMA group id: A rows gq, gq+8; B column (= x row) gq
    const int tq = lane & 3;        // thread in group: k-slots 2tq, 2tq+1, 2tq+8, 2tq+9
    const bool swap_half = tq >= 2; // staggered chunk order, see the x loads below
    const int rA = 16 * warp + row_of(gq);        // data rows of MMA rows gq and gq + 8
    const int rB = 16 * warp + row_of(gq + 8);
    const uint32_t kOnes = 0x3F803F80u;   // BF16 (1.0, 1.0)
    const uint32_t ones[4] = {kOnes, kOnes, kOnes, kOnes};

    // Rows M..7 of every x slab are never written by the TMA: zero them once, so the
    // B operand of absent activation rows is 0 without any per-load predication.
    for (int i = threadIdx.x; i < S * (kMaxM - p.M) * (kXRowBytes / 16); i += kWarps * 32) {
        const int per_stage = (kMaxM - p.M) * (kXRowBytes / 16);
        const int st = i / per_stage, r = i - st * per_stage;
        reinterpret_cast<uint4 *>(smem + st * kStageBytes + kWBytes + p.M * kXRowBytes)[r] = make_uint4(0, 0, 0, 0);
    }
    named_bar_sync(1, kWarps * 32);

    // Per-lane shared-memory offsets within a stage.  A: 16-byte chunk c = 4*group + tq
    // of rows rA and rB, stored at chunk (c ^ (row & 7)) by the 128-byte swizzle.
    uint32_t offA[2], offB[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        offA[j] = rA * 128 + (((4 * j + tq) ^ (rA & 7)) << 4);
        offB[j] = rB * 128 + (((4 * j + tq) ^ (rB & 7)) << 4);
    }
    // B: x row gq, the 32 values k in [32 tq, 32 tq + 32) of each group.  Threads with
    // tq >= 2 read their four 16-byte chunks in the order 2,3,0,1, which (with the
    // 528-byte row pitch) puts the 8 threads of each quarter warp on 8 distinct 16-byte
    // bank groups.  The A words are swapped the same way, so both operands of each MMA
    // refer to the same k.
    const uint32_t offX = kWBytes + gq * kXRowBytes + 64 * tq;

    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    int tile_seq = -1, prev_t = -1;
    const uint16_t *sA = nullptr, *sB = nullptr, *bA = nullptr, *bB = nullptr;   // scale/bias rows
    const int first_tile = static_cast<int>(u0 / G);
    StageWalker wk;
    wk.start(u0, u1, G);
    int s = 0, xslot = 0;                 // ring positions of stage i
    uint32_t ph = 0, xph = 0;             // their phase parities
    for (int i = 0; wk.n; ++i, wk.next(), (++s == S ? (s = 0, ph ^= 1u) : 0u),
             (++xslot == XR ? (xslot = 0, xph ^= 1u) : 0u)) {
        const int t = wk.t;
        const long long first_row = static_cast<long long>(t) * kRows;
        if (t != prev_t) {
            prev_t = t;
            ++tile_seq;
            // scale/bias rows of this tile: from the slab when it holds them all, else global
            const long long rows = min(static_cast<long long>(kRows), p.N - first_row);
            bool from_slab = false;
            if (slots) {
                const int slot = tile_seq % slots;
                mbar_wait(&slab_full[slot], (tile_seq / slots) & 1);
                from_slab = ((rows * G * 2) & 15) == 0;   // the whole slab landed
                if (from_slab) {
                    const uint16_t *ss = reinterpret_cast<const uint16_t *>(slab_base + slot * 2 * p.slab_array_bytes);
                    const uint16_t *sb = reinterpret_cast<const uint16_t *>(slab_base + slot * 2 * p.slab_array_bytes +
                                                                            p.slab_array_bytes);
                    sA = ss + rA * G; sB = ss + rB * G; bA = sb + rA * G; bB = sb + rB * G;
                }
            }
            if (!from_slab) {   // rows past N read row N-1 (their results are never stored)
                const long long nA = min(first_row + rA, static_cast<long long>(p.N) - 1);
                const long long nB = min(first_row + rB, static_cast<long long>(p.N) - 1);
                sA = p.scales + nA * G; sB = p.scales + nB * G; bA = p.biases + nA * G; bB = p.biases + nB * G;
            }
        }
        mbar_wait(&full[s], ph);
        const uint8_t *st = smem + s * kStageBytes;
        const int ng = wk.n;
        const int g0 = wk.g;

        uint4 wa[2], wb[2], xv[2][4];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            wa[j] = *reinterpret_cast<const uint4 *>(st + offA[j]);
            wb[j] = *reinterpret_cast<const uint4 *>(st + offB[j]);
#pragma unroll
            for (int r = 0; r < 4; ++r)
                xv[j][r] = *reinterpret_cast<const uint4 *>(st + offX + 256 * j + 16 * (swap_half ? (r ^ 2) : r));
        }
        // scale and bias of rows rA, rB for the stage's groups (a one-group stage reads
        // its group twice; the copy is never used)
        float sc[2][2], bi[2][2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int gj = g0 + (j < ng ? j : 0);
            sc[j][0] = bf16_bits_to_f32(sA[gj]);
            sc[j][1] = bf16_bits_to_f32(sB[gj]);
            bi[j][0] = fmaf(-128.f, sc[j][0], bf16_bits_to_f32(bA[gj]));
            bi[j][1] = fmaf(-128.f, sc[j][1], bf16_bits_to_f32(bB[gj]));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);

        if (swap_half) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                uint32_t tmp;
                tmp = wa[j].x; wa[j].x = wa[j].z; wa[j].z = tmp;
                tmp = wa[j].y; wa[j].y = wa[j].w; wa[j].w = tmp;
                tmp = wb[j].x; wb[j].x = wb[j].z; wb[j].z = tmp;
                tmp = wb[j].y; wb[j].y = wb[j].w; wb[j].w = tmp;
            }
        }

        // B fragments: MMA (r, h=0) takes k-pairs (k0,k4),(k1,k5) of x chunk r; (r, h=1)
        // takes (k2,k6),(k3,k7).
        uint32_t bf[2][4][4];
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                bf[j][r][0] = prmt(xv[j][r].x, xv[j][r].z, 0x5410u);
                bf[j][r][1] = prmt(xv[j][r].x, xv[j][r].z, 0x7632u);
                bf[j][r][2] = prmt(xv[j][r].y, xv[j][r].w, 0x5410u);
                bf[j][r][3] = prmt(xv[j][r].y, xv[j][r].w, 0x7632u);
            }

        // X = sum of x over each group of this stage: computed by the stage's duty warp
        float *xs_slot = xs_base + xslot * (kGroupsPerStage * kMaxM);
        if ((i % kWarps) == warp) {
            float xa[2][4] = {}, xb[2][4] = {};
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    mma_bf16_16816(xa[j], ones, bf[j][r][0], bf[j][r][1], xa[j]);
                    mma_bf16_16816(xb[j], ones, bf[j][r][2], bf[j][r][3], xb[j]);
                }
            if (gq == 0) {   // row 0 of the all-ones product: columns 2tq, 2tq+1
#pragma unroll
                for (int j = 0; j < 2; ++j)
                    *reinterpret_cast<float2 *>(xs_slot + j * kMaxM + 2 * tq) =
                        make_float2(xa[j][0] + xb[j][0], xa[j][1] + xb[j][1]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&xs_full[xslot]);
        }

        float pacc[2][2][4] = {};   // [group][k-pair half][fragment]
        const uint32_t A0[2][4] = {{wa[0].x, wa[0].y, wa[0].z, wa[0].w}, {wa[1].x, wa[1].y, wa[1].z, wa[1].w}};
        const uint32_t A8[2][4] = {{wb[0].x, wb[0].y, wb[0].z, wb[0].w}, {wb[1].x, wb[1].y, wb[1].z, wb[1].w}};
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                // word r of each row holds codes for 8 consecutive k; x chunk r holds the same k
                const uint32_t w0 = A0[j][r], w8 = A8[j][r];
                const uint32_t a_h0[4] = {codes_to_bf16x2_plus128(w0), codes_to_bf16x2_plus128(w8),
                                          codes_to_bf16x2_plus128(w0 >> 4), codes_to_bf16x2_plus128(w8 >> 4)};
                const uint32_t a_h1[4] = {codes_to_bf16x2_plus128(w0 >> 8), codes_to_bf16x2_plus128(w8 >> 8),
                                          codes_to_bf16x2_plus128(w0 >> 12), codes_to_bf16x2_plus128(w8 >> 12)};
                mma_bf16_16816(pacc[j][0], a_h0, bf[j][r][0], bf[j][r][1], pacc[j][0]);
                mma_bf16_16816(pacc[j][1], a_h1, bf[j][r][2], bf[j][r][3], pacc[j][1]);
            }

        // epilogue: rows rA (d0, d1) and rB (d2, d3); x rows 2tq, 2tq+1
        mbar_wait(&xs_full[xslot], xph);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            if (j >= ng) break;
            const float2 X = *reinterpret_cast<const float2 *>(xs_slot + j * kMaxM + 2 * tq);
            acc[0] = fmaf(bi[j][0], X.x, fmaf(sc[j][0], pacc[j][0][0] + pacc[j][1][0], acc[0]));
            acc[1] = fmaf(bi[j][0], X.y, fmaf(sc[j][0], pacc[j][0][1] + pacc[j][1][1], acc[1]));
            acc[2] = fmaf(bi[j][1], X.x, fmaf(sc[j][1], pacc[j][0][2] + pacc[j][1][2], acc[2]));
            acc[3] = fmaf(bi[j][1], X.y, fmaf(sc[j][1], pacc[j][0][3] + pacc[j][1][3], acc[3]));
        }

        if (!wk.tile_ends()) continue;
        if (slots) {   // this tile's slab is no longer needed
            __syncwarp();
            if (lane == 0) mbar_arrive(&slab_empty[tile_seq % slots]);
        }

        // ------------------------------------------------------------ tile output
        const long long tile_first = static_cast<long long>(t) * G;
        const long long tile_last = tile_first + G - 1;
        const long long nA = first_row + rA;
        const long long nB = first_row + rB;
        const int mA = 2 * tq, mB = 2 * tq + 1;
        float out[4] = {acc[0], acc[1], acc[2], acc[3]};
        bool write = true;
        if (!(tile_first >= u0 && tile_last < u1)) {
            // split tile: publish this CTA's partial, take a ticket, last arriver reduces
            const int slot = (t == first_tile) ? 0 : 1;
            float *mine = p.partials + (cta * 2 + slot) * (kRows * 8);
            *reinterpret_cast<float2 *>(mine + rA * 8 + 2 * tq) = make_float2(acc[0], acc[1]);
            *reinterpret_cast<float2 *>(mine + rB * 8 + 2 * tq) = make_float2(acc[2], acc[3]);
            // The barrier orders every consumer's partial before thread 0's release; the
            // acquire side of the same atomic, followed by the second barrier, orders the
            // reads below after every earlier contributor's release.
            named_bar_sync(1, kWarps * 32);
            const long long c_first = streamk_owner(U, P, tile_first);
            const long long c_last = streamk_owner(U, P, tile_last);
            if (threadIdx.x == 0) {
                const int old = atomic_add_acq_rel_gpu(&p.tickets[t], 1);
                *ticket_flag = (old == static_cast<int>(c_last - c_first));
            }
            named_bar_sync(1, kWarps * 32);
            write = *ticket_flag != 0;
            if (write) {
                // Every contributor after the first starts inside this tile, so its partial
                // is in slot 0; the first one uses slot 1 unless its range starts exactly at
                // the tile's first unit.
                const int first_slot = (c_first * U / P == tile_first) ? 0 : 1;
                out[0] = out[1] = out[2] = out[3] = 0.f;
                for (long long cb = c_first; cb <= c_last; cb += kFixupBatch) {
                    float2 v[kFixupBatch][2];
#pragma unroll
                    for (int j = 0; j < kFixupBatch; ++j) {   // issue every load of the batch first
                        const long long cc = cb + j;
                        if (cc <= c_last) {
                            const int cslot = (cc == c_first) ? first_slot : 0;
                            const float *part = p.partials + (cc * 2 + cslot) * (kRows * 8);
                            v[j][0] = __ldcg(reinterpret_cast<const float2 *>(part + rA * 8 + 2 * tq));
                            v[j][1] = __ldcg(reinterpret_cast<const float2 *>(part + rB * 8 + 2 * tq));
                        } else {
                            v[j][0] = v[j][1] = make_float2(0.f, 0.f);
                        }
                    }
#pragma unroll
                    for (int j = 0; j < kFixupBatch; ++j) {   // then add them in CTA order
                        out[0] += v[j][0].x;
                        out[1] += v[j][0].y;
                        out[2] += v[j][1].x;
                        out[3] += v[j][1].y;
                    }
                }
                if (threadIdx.x == 0) p.tickets[t] = 0;   // ready for the next launch
            }
        }
        if (write) {
            if (nA < p.N) {
                if (mA < p.M) p.y[static_cast<long long>(mA) * p.N + nA] = f32_to_bf16_bits(out[0]);
                if (mB < p.M) p.y[static_cast<long long>(mB) * p.N + nA] = f32_to_bf16_bits(out[1]);
            }
            if (nB < p.N) {
                if (mA < p.M) p.y[static_cast<long long>(mA) * p.N + nB] = f32_to_bf16_bits(out[2]);
                if (mB < p.M) p.y[static_cast<long long>(mB) * p.N + nB] = f32_to_bf16_bits(out[3]);
            }
        }
        acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
    }
}

}  // namespace mv
}  // namespace w4a16
