// rows.cuh - row-block W4A16 matvec for M <= 8 (decode).
//
// Role in the layer: tiny-llm "Week 2 Day 6: SIMD-Matrix Prefill", Task 1,
// keeps a matvec schedule for M <= 8; Task 2 asks for contiguous device loads;
// Task 3 applies one scale and bias per 128-group; the "Route affine qmv_wide
// by bit-width and batch size" PR holds a dequantised group in registers and
// reuses it across the M activation rows.  This is a B200 design, not those
// Metal kernels.
//
// Why this shape: in a stream of back-to-back decode projections a call's time is
// latency, not bytes, unless the weights are already on chip when the call's
// input arrives.  So every CTA owns RB row blocks of 16 whole weight rows over a
// K range, holds ALL of their codes, scales and biases in shared memory (one TMA
// box of [16 RB rows x 64 B] per 128-group, two copies for scales and biases)
// and requests them at its start.  With the static-weights flag that happens
// before the dependency wait; a CTA takes under half of an SM, so the next call's
// CTAs are resident beside this call's and fetch their weights while this call
// computes.  Each CTA also prefetches its share of x into L2 before the wait.
// After the wait only x-dependent work remains: the compute warps load their
// groups' x straight into registers (all of it in flight at once, two groups of
// look-ahead), run the MMAs, and the partial sums are added.
//
// Compute: m16n8k16 BF16 tensor-core MMAs with the CODES as A (16 weight rows
// x 16 k) and x as B (16 k x 8 columns = the M <= 8 activation rows, zeros
// beyond M), so every MMA row is a real weight row.  Codes enter as the exact
// BF16 values 128 + 8 q (one shift and one LOP3 per two codes); the MMA yields
// P8 = sum (128 + 8 q) x, and the group sum X = sum x comes from MMAs against
// all-ones A.  The epilogue adds (s / 8) P8 + (b - 16 s) X in FP32 per group.
// Lane (g, t) = (lane / 4, lane % 4) reads code words 4t .. 4t+3 of rows g and
// g + 8 of a row block (k = 32t .. 32t+31 of the group, one 16-byte load per
// row, conflict-free: a quarter warp covers two 64-byte rows) and the same 32 k
// of x row g.  Word c feeds two MMAs: nibble pairs (0,4),(1,5) and (2,6),(3,7),
// with x permuted identically (a permutation of k shared by A and B leaves the
// dot product unchanged).
//
// Work split: the CTA's (row block, group) units are ordered group-major and cut
// into 8 contiguous, equal ranges, one per compute warp; the warps' partial sums
// are added in warp order through shared memory.  Optionally S CTAs of a cluster
// share the same rows, each a contiguous K range: ranks 1..S-1 store their
// partials into rank 0's shared memory and arrive on its barrier (release at
// cluster scope); rank 0 adds them in rank order.  Every sum has a fixed order:
// the result does not depend on timing.
//
// Waits: every wait is on one of this CTA's own copies (rank 0 also waits for its peers'
// partial sums), bounded by a time limit after which it records W4A16_ERR_TIMEOUT.  Unlike the
// other kernels' waits they do not give up early when another CTA has recorded a timeout, and
// a wait that expires does not end the warp's loop: every copy the CTA requested is waited for
// by the warp that uses it, so none can still be in flight when the CTA's shared memory is
// reused or released.  A copy that never lands (only the test flag drops one) ends its waits
// at the limit and leaves the results undefined.
#pragma once

#include "plain.cuh"
#include "ptx.cuh"

namespace w4a16 {
namespace mvr {

constexpr int kMaxM = 8;
constexpr int kWarps = 8;                            // every warp computes; thread 0 also issues the copies
constexpr int kThreads = kWarps * 32;
constexpr int kMaxRB = 5;                            // row blocks of 16 rows per CTA
constexpr int kMaxSplits = 4;                        // CTAs of a cluster sharing rows (K split)
constexpr int kXD = 2;                               // groups of x look-ahead per warp (registers)
// Shared memory of a CTA: two fit on an SM (233472 B less 1 KB reserved per CTA).
constexpr long long kBudget = 115712;
constexpr int kGather = 8;                           // scale / bias loads in flight per thread (K split)

// A cluster owns hb blocks of 8 rows ("half blocks"); its MMA row blocks are rb = ceil(hb / 2),
// the last one half used when hb is odd.  A group's codes take 8 hb rows of 64 B; the MMA of
// a half-used block also reads the 8 rows after the slot, so the area has 512 B of slack.
__host__ __device__ constexpr int rbs_of(int hb) { return (hb + 1) / 2; }
__host__ __device__ constexpr long long codes_bytes(int hb, int gc) { return 512ll * hb * gc + 512; }
__host__ __device__ constexpr long long red_bytes(int hb) { return 4096ll * rbs_of(hb); }   // [8][rb][16][8] FP32
__host__ __device__ constexpr long long work_bytes(int hb, int gc) {
    return codes_bytes(hb, gc) > red_bytes(hb) ? codes_bytes(hb, gc) : red_bytes(hb);
}
// scales or biases [16 rb][gc] BF16 (rows past the half blocks are read, never used)
__host__ __device__ constexpr long long sb_bytes(int hb, int gc) { return (32ll * rbs_of(hb) * gc + 15) / 16 * 16; }
__host__ __device__ constexpr long long part_bytes(int hb) { return 512ll * rbs_of(hb); }   // [16 rb][8] FP32
// work | scales | biases | own partial (S > 1) | partials of ranks 1..S-1 (rank 0) | barriers
__host__ __device__ constexpr long long off_scales(int hb, int gc) { return work_bytes(hb, gc); }
__host__ __device__ constexpr long long off_biases(int hb, int gc) { return off_scales(hb, gc) + sb_bytes(hb, gc); }
__host__ __device__ constexpr long long off_part(int hb, int gc) { return off_biases(hb, gc) + sb_bytes(hb, gc); }
__host__ __device__ constexpr long long off_slots(int hb, int gc, int s) {
    return off_part(hb, gc) + (s > 1 ? part_bytes(hb) : 0);
}
__host__ __device__ constexpr long long off_bars(int hb, int gc, int s) {
    return off_slots(hb, gc, s) + (s - 1) * part_bytes(hb);
}
__host__ __device__ constexpr long long smem_bytes(int hb, int gc, int s) {
    return off_bars(hb, gc, s) + 8ll * (gc + 2) + 128;   // + barriers, + alignment slack
}

struct Params {
    const uint16_t *x;        // bf16 [M, K]
    const uint32_t *wq;       // [N, K/8] packed codes (read by TMA; directly only by the plain path)
    const uint16_t *scales;   // bf16 [N, G]
    const uint16_t *biases;   // bf16 [N, G]
    uint16_t *y;              // bf16 [M, N]
    int M, N, K, G;
    int splits;               // S: CTAs of a cluster, each a contiguous run of groups
    int gcl;                  // ceil(G / S): groups of the shared-memory layout
    int nh;                   // 8-row half blocks of the matrix, ceil(N / 8)
    int clusters;             // clusters with rows: cluster c owns half blocks [c nh / clusters, (c+1) nh / clusters)
    int hb_lo, hb_hi;         // floor / ceil(nh / clusters): tm_lo / tm_hi boxes; 8 hb_hi rows per group slot
    int static_weights;       // codes, scales and biases may be read before the dependency wait
    long long x_chunk;        // bytes of x this CTA prefetches into L2 (0: none)
    int test_drop_copy;       // tests of the timeout path: CTA 0 never loads its first group's codes
    unsigned long long wait_ns;   // limit of every wait on a copy (kWaitTimeoutNs, shorter in that test)
    int gated;                // fused gate/up: rows 16 b .. 16 b + 7 are gate rows 8 b .. 8 b + 7, rows
                              // 16 b + 8 .. 16 b + 15 the up rows of the same outputs; y [M, N / 2] =
                              // silu(gate) * up; clusters own whole 16-row blocks
    long long ldy;            // gated: elements between rows of y (a launch may write a column slice)
};

// silu(g) * u in FP32 (expf of the CUDA math library), then BF16 round to nearest even
__device__ __forceinline__ uint16_t swiglu_bf16(float g, float u) {
    const float sg = g / (1.f + expf(-g));
    return __bfloat16_as_ushort(__float2bfloat16_rn(sg * u));
}

// BF16 pair (lo, hi) of two words' low / high halves
__device__ __forceinline__ uint32_t lo_halves(uint32_t a, uint32_t b) { return prmt(a, b, 0x5410u); }
__device__ __forceinline__ uint32_t hi_halves(uint32_t a, uint32_t b) { return prmt(a, b, 0x7632u); }

__device__ __forceinline__ void load_x(uint4 (&xr)[4], const uint16_t *src, bool live) {
#pragma unroll
    for (int q = 0; q < 4; ++q) xr[q] = live ? ldg_v4(src + 8 * q) : make_uint4(0u, 0u, 0u, 0u);
}

// Two CTAs per SM: each SM sub-partition holds 2 + 2 of their warps, 4 x 32 x 128 = 16384 registers.
template <int RB>
__global__ void __maxnreg__(128) rows_kernel(const __grid_constant__ CUtensorMap tm_hi,
                                            const __grid_constant__ CUtensorMap tm_lo, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u);
    const int S = p.splits, GCL = p.gcl, G = p.G, HB = p.hb_hi;
    const int slot = 8 * HB * 64;                                        // bytes of one group's codes
    const uint32_t rank = S > 1 ? cluster_ctarank() : 0u;
    // this cluster's row blocks; clusters past p.clusters have none (they keep one CTA of
    // every call on each SM, so that the next call's CTAs land one per SM)
    const int cl = static_cast<int>(blockIdx.x) / S;
    // gated: clusters split the nh / 2 blocks of 16 rows, so that every block pairs gate and up
    const int unit = p.gated ? 2 : 1, nu = p.nh / unit;
    const int hb0 = unit * static_cast<int>(static_cast<long long>(cl) * nu / p.clusters);
    const int nhb = cl < p.clusters ? unit * static_cast<int>(static_cast<long long>(cl + 1) * nu / p.clusters) - hb0 : 0;
    const int nrb = (nhb + 1) / 2;                                       // MMA row blocks (<= RB)
    const long long r0 = 8ll * hb0;                                      // first weight row of the CTA
    const int g0 = static_cast<int>(rank * G / S), g1 = static_cast<int>((rank + 1) * G / S);
    const int GC = g1 - g0;                                              // groups of this CTA
    uint16_t *sc = reinterpret_cast<uint16_t *>(smem + off_scales(HB, GCL));
    uint16_t *bi = reinterpret_cast<uint16_t *>(smem + off_biases(HB, GCL));
    float *part = reinterpret_cast<float *>(smem + off_part(HB, GCL));
    float *slots = reinterpret_cast<float *>(smem + off_slots(HB, GCL, S));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + off_bars(HB, GCL, S));
    uint64_t *box_full = bars, *sb_full = bars + GCL, *red_full = bars + GCL + 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        pdl_launch_dependents();   // the next call may start fetching its weights
        for (int b = 0; b < GC; ++b) mbar_init(&box_full[b], 1);
        mbar_init(sb_full, 1);
        mbar_init(red_full, 1);
        if (S > 1 && rank == 0)   // the other ranks' partials arrive as bytes on this barrier
            mbar_arrive_expect_tx(red_full, static_cast<uint32_t>((S - 1) * part_bytes(HB)));
        fence_mbar_init();
    }
    if (S > 1)
        cluster_sync_all();   // rank 0's barrier is initialised before any rank can arrive on it
    else
        __syncthreads();
    if (nhb == 0) {           // no rows: hold the slot until the preceding kernel is done
        pdl_wait();
        return;
    }

    // ---------------------------------------------------------------- weights, then the wait
    if (!p.static_weights) pdl_wait();
    const long long rows = max(0ll, min(8ll * nhb, p.N - r0));
    if (threadIdx.x == 0) {
        const CUtensorMap *tm = nhb == p.hb_lo ? &tm_lo : &tm_hi;   // boxes of 8 nhb rows
        prefetch_tmap(tm);
        // codes: box b = words 16 (g0 + b) .. + 15 of rows r0 .. r0 + 8 nhb - 1 (zeros past N)
        for (int b = 0; b < GC; ++b) {
            if (b == 0 && p.test_drop_copy && blockIdx.x == 0) continue;   // its barrier never completes
            mbar_arrive_expect_tx(&box_full[b], static_cast<uint32_t>(nhb) * 512);
            tma_load_2d(smem + static_cast<long long>(b) * slot, tm, &box_full[b], 16 * (g0 + b),
                        static_cast<int>(r0));
        }
        if (S == 1) {
            // scales and biases of the CTA's rows: one contiguous [rows][G] block each
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
        } else {
            mbar_arrive(sb_full);   // gathered below, ordered by the CTA barrier
        }
        // this CTA's share of x into L2, ahead of the dependency wait
        if (p.x_chunk > 0) {
            const long long total = static_cast<long long>(p.M) * p.K * 2;
            const long long start = static_cast<long long>(blockIdx.x) * p.x_chunk;
            if (start < total)
                prefetch_l2_bulk(reinterpret_cast<const uint8_t *>(p.x) + start,
                                 static_cast<uint32_t>(min(p.x_chunk, total - start)));
        }
    }
    if (S > 1) {
        // a K range of the rows, [rows][GC] out of [N][G] (not a contiguous block and not
        // 16-byte aligned): every thread keeps kGather loads of each array in flight
        const int n = static_cast<int>(rows) * GC;
        for (int base = 0; base < n; base += kThreads * kGather) {
            uint16_t vs[kGather], vb[kGather];
#pragma unroll
            for (int j = 0; j < kGather; ++j) {
                const int i = base + j * kThreads + static_cast<int>(threadIdx.x);
                if (i < n) {
                    const int r = i / GC, c = i - r * GC;
                    const long long src = (r0 + r) * G + g0 + c;
                    vs[j] = __ldg(p.scales + src);
                    vb[j] = __ldg(p.biases + src);
                }
            }
#pragma unroll
            for (int j = 0; j < kGather; ++j) {
                const int i = base + j * kThreads + static_cast<int>(threadIdx.x);
                if (i < n) {
                    const int r = i / GC, c = i - r * GC;
                    sc[r * GCL + c] = vs[j];
                    bi[r * GCL + c] = vb[j];
                }
            }
        }
        __syncthreads();
    }

    // ---------------------------------------------------------------- compute
    const int w = warp;
    const int g = lane >> 2, t = lane & 3;
    const int U = nrb * GC;                       // units (row block, group), group-major
    const int u0 = w * U / kWarps, u1 = (w + 1) * U / kWarps;
    float out[RB][4];
#pragma unroll
    for (int rb = 0; rb < RB; ++rb) out[rb][0] = out[rb][1] = out[rb][2] = out[rb][3] = 0.f;
    constexpr uint32_t kOnes = 0x3F803F80u;       // BF16 (1.0, 1.0)
    const uint32_t ones[4] = {kOnes, kOnes, kOnes, kOnes};
    if (p.static_weights) pdl_wait();             // x may come from the preceding kernel
    if (u0 < u1) {
        const int ga = u0 / nrb, gb = (u1 - 1) / nrb + 1;   // groups [ga, gb) of the CTA's range
        const bool live = g < p.M;
        const uint16_t *xrow = p.x + static_cast<long long>(live ? g : 0) * p.K + static_cast<long long>(g0) * 128 + 32 * t;
        uint4 xr[kXD][4];
#pragma unroll
        for (int j = 0; j < kXD; ++j)
            if (ga + j < gb) load_x(xr[j], xrow + (ga + j) * 128, live);
        mbar_wait(sb_full, 0, false, p.wait_ns);
        const uint32_t cbase = smem_u32(smem) + static_cast<uint32_t>(g * 64 + t * 16);
        for (int gi = ga; gi < gb; gi += kXD) {
#pragma unroll
            for (int j = 0; j < kXD; ++j) {
                const int gg = gi + j;
                if (gg >= gb) break;
                // B fragments of group gg (x permuted like the codes), then the next x loads
                uint32_t bf[8][2];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    bf[2 * c][0] = lo_halves(xr[j][c].x, xr[j][c].z);       // x0, x4
                    bf[2 * c][1] = hi_halves(xr[j][c].x, xr[j][c].z);       // x1, x5
                    bf[2 * c + 1][0] = lo_halves(xr[j][c].y, xr[j][c].w);   // x2, x6
                    bf[2 * c + 1][1] = hi_halves(xr[j][c].y, xr[j][c].w);   // x3, x7
                }
                if (gg + kXD < gb) load_x(xr[j], xrow + (gg + kXD) * 128, live);
                // group sums of x rows 2t, 2t + 1 (two independent MMA chains)
                float xa[4] = {0.f, 0.f, 0.f, 0.f}, xb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    mma_bf16_16816(xa, ones, bf[2 * c][0], bf[2 * c][1], xa);
                    mma_bf16_16816(xb, ones, bf[2 * c + 1][0], bf[2 * c + 1][1], xb);
                }
                const float X0 = xa[0] + xb[0], X1 = xa[1] + xb[1];
                mbar_wait(&box_full[gg], 0, false, p.wait_ns);   // after a timeout the results are undefined
                const int rlo = gg == ga ? u0 - ga * nrb : 0;
                const int rhi = gg == gb - 1 ? u1 - gg * nrb : nrb;
                const uint32_t cg = cbase + static_cast<uint32_t>(gg * slot);
#pragma unroll
                for (int rb = 0; rb < RB; ++rb) {
                    if (rb < rlo || rb >= rhi) continue;
                    // words 4t .. 4t + 3 of rows 16 rb + g and 16 rb + g + 8, group gg
                    const uint4 ca = lds128(cg + rb * 16 * 64), cb = lds128(cg + rb * 16 * 64 + 8 * 64);
                    const uint32_t wa[4] = {ca.x, ca.y, ca.z, ca.w}, wb[4] = {cb.x, cb.y, cb.z, cb.w};
                    float da[4] = {0.f, 0.f, 0.f, 0.f}, db[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        // nibbles (0,4), (1,5), (2,6), (3,7) moved to bits 3-6 and 19-22
                        const uint32_t a0[4] = {codes_to_bf16x2_128_plus_8q(wa[c] << 3), codes_to_bf16x2_128_plus_8q(wb[c] << 3),
                                                codes_to_bf16x2_128_plus_8q(wa[c] >> 1), codes_to_bf16x2_128_plus_8q(wb[c] >> 1)};
                        mma_bf16_16816(da, a0, bf[2 * c][0], bf[2 * c][1], da);
                        const uint32_t a1[4] = {codes_to_bf16x2_128_plus_8q(wa[c] >> 5), codes_to_bf16x2_128_plus_8q(wb[c] >> 5),
                                                codes_to_bf16x2_128_plus_8q(wa[c] >> 9), codes_to_bf16x2_128_plus_8q(wb[c] >> 9)};
                        mma_bf16_16816(db, a1, bf[2 * c + 1][0], bf[2 * c + 1][1], db);
                    }
                    // scale and shifted bias of rows 16 rb + g (A row g) and 16 rb + g + 8 (A row g + 8)
                    const int na = (rb * 16 + g) * GCL + gg, nb = na + 8 * GCL;
                    const float sa = bf16_to_f32(sc[na]), sb = bf16_to_f32(sc[nb]);
                    const float ba = fmaf(-16.f, sa, bf16_to_f32(bi[na]));   // b - 16 s
                    const float bb = fmaf(-16.f, sb, bf16_to_f32(bi[nb]));
                    const float s8a = 0.125f * sa, s8b = 0.125f * sb;        // s / 8, exact
                    out[rb][0] = fmaf(ba, X0, fmaf(s8a, da[0] + db[0], out[rb][0]));
                    out[rb][1] = fmaf(ba, X1, fmaf(s8a, da[1] + db[1], out[rb][1]));
                    out[rb][2] = fmaf(bb, X0, fmaf(s8b, da[2] + db[2], out[rb][2]));
                    out[rb][3] = fmaf(bb, X1, fmaf(s8b, da[3] + db[3], out[rb][3]));
                }
            }
        }
    }
    // ---------------------------------------------------------------- fixed-order sums
    __syncthreads();   // every warp is done with the codes (and every copy of the CTA landed)
    float *red = reinterpret_cast<float *>(smem);   // [warp][row block][row][x row]
#pragma unroll
    for (int rb = 0; rb < RB; ++rb) {
        float *dst = red + ((w * RB + rb) * 16 + g) * kMaxM + 2 * t;
        *reinterpret_cast<float2 *>(dst) = make_float2(out[rb][0], out[rb][1]);
        *reinterpret_cast<float2 *>(dst + 8 * kMaxM) = make_float2(out[rb][2], out[rb][3]);
    }
    __syncthreads();
    const int tid = threadIdx.x;
    const int RC = 8 * nhb;                      // rows of this CTA
    const int RM = RC * p.M;
    // the sum of row r (of the CTA) for x row m over the warps, in warp order
    auto warp_sum = [&](int m, int r) {
        const float *src = red + r * kMaxM + m;   // row block r / 16, row r % 16: offset r * 8
        float v = 0.f;
#pragma unroll
        for (int ww = 0; ww < kWarps; ++ww) v += src[ww * RB * 16 * kMaxM];
        return v;
    };
    // not finite in FP32 (gated) or BF16: the plain definition of the row's output
    auto plain_row = [&](int m, long long n) {
        return plain_output(p.x + static_cast<long long>(m) * p.K, p.wq + n * (p.K / 8), p.scales + n * G,
                            p.biases + n * G, G);
    };
    if (S == 1 && p.gated) {
        const int JC = RC / 2;                   // outputs per x row: the CTA's gate rows
        for (int i = tid; i < JC * p.M; i += kWarps * 32) {
            const int m = i / JC, jl = i - m * JC;
            const int rg = 16 * (jl >> 3) + (jl & 7), ru = rg + 8;
            if (r0 + ru >= p.N) continue;
            float vg = warp_sum(m, rg), vu = warp_sum(m, ru);
            if (!isfinite(vg)) vg = plain_row(m, r0 + rg);
            if (!isfinite(vu)) vu = plain_row(m, r0 + ru);
            p.y[static_cast<long long>(m) * p.ldy + r0 / 2 + jl] = swiglu_bf16(vg, vu);
        }
    } else {
        for (int i = tid; i < RM; i += kWarps * 32) {
            const int m = i / RC, r = i - m * RC;
            float v = warp_sum(m, r);
            if (S == 1) {
                if (r0 + r < p.N) {
                    if (!isfinite(__bfloat162float(__float2bfloat16_rn(v)))) v = plain_row(m, r0 + r);
                    p.y[static_cast<long long>(m) * p.N + r0 + r] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
                }
            } else {
                part[r * kMaxM + m] = v;
            }
        }
    }
    if (S == 1) return;
    // ---------------------------------------------------------------- K split over the cluster
    if (rank != 0) {
        // this CTA's partial into slot rank - 1 of rank 0: asynchronous remote stores whose
        // bytes complete on rank 0's barrier
        __syncthreads();
        const uint32_t dst = dsmem_addr(smem_u32(slots + (rank - 1) * 16 * RB * kMaxM), 0u);
        const uint32_t bar = dsmem_addr(smem_u32(red_full), 0u);
        for (int i = tid; i < 16 * RB * kMaxM / 4; i += kWarps * 32)
            st_async_dsmem_f4(dst + 16u * i, reinterpret_cast<const float4 *>(part)[i], bar);
        return;
    }
    const bool parts = mbar_wait_cluster(red_full, 0);   // the other ranks' partial sums landed
    // the sum of row r for x row m over the ranks, in rank order
    auto rank_sum = [&](int m, int r) {
        float v = part[r * kMaxM + m];
        for (int s = 1; s < S; ++s) v += slots[((s - 1) * 16 * RB + r) * kMaxM + m];
        return v;
    };
    if (p.gated) {
        const int JC = RC / 2;
        for (int i = tid; parts && i < JC * p.M; i += kWarps * 32) {
            const int m = i / JC, jl = i - m * JC;
            const int rg = 16 * (jl >> 3) + (jl & 7), ru = rg + 8;
            if (r0 + ru >= p.N) continue;
            float vg = rank_sum(m, rg), vu = rank_sum(m, ru);
            if (!isfinite(vg)) vg = plain_row(m, r0 + rg);
            if (!isfinite(vu)) vu = plain_row(m, r0 + ru);
            p.y[static_cast<long long>(m) * p.ldy + r0 / 2 + jl] = swiglu_bf16(vg, vu);
        }
    } else {
        for (int i = tid; parts && i < RM; i += kWarps * 32) {
            const int m = i / RC, r = i - m * RC;
            float v = rank_sum(m, r);
            if (r0 + r < p.N) {
                if (!isfinite(__bfloat162float(__float2bfloat16_rn(v)))) v = plain_row(m, r0 + r);
                p.y[static_cast<long long>(m) * p.N + r0 + r] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
            }
        }
    }
}

}  // namespace mvr
}  // namespace w4a16
