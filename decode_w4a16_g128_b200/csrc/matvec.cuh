// matvec.cuh - weight-streaming W4A16 kernel for M <= 8 (decode).
//
// Role in the layer: tiny-llm "Week 2 Day 6: SIMD-Matrix Prefill", Task 1,
// keeps a matvec schedule for M <= 8.  This is a B200 design, not that
// Metal kernel: the whole cost is reading the packed weights once (0.5 byte
// per weight plus 4 bytes of scale and bias per 128 weights), so the kernel is
// built around keeping HBM busy.
//
// Work decomposition ("stream-K"): the output rows are cut into tiles of
// kRows = 16 * CW rows, and each (row tile, 128-group) pair is one unit of
// work.  The U = tiles * G units are split into `workers` contiguous ranges,
// one persistent CTA each (CTA c owns [c*U/P, (c+1)*U/P)), so every SM
// streams the same number of bytes whatever N and K are.  A tile whose
// groups are spread over several CTAs is finished by the CTA that completes
// it last: every contributor writes its FP32 partial to the workspace, and
// the last one to arrive (a per-tile atomic ticket) adds the partials in CTA
// order, so the sum does not depend on arrival order.
//
// Per CTA: warp CW is the producer.  For each unit it issues two TMA tile
// loads into a stage of a kStages-deep ring (the [kRows x 16] uint32 slab of
// packed weights and the [M x 136] BF16 slab of x for that group; the 8 extra
// columns only stagger the rows of x across shared-memory banks) and 4-byte
// cp.async copies of the scale and bias words of its rows.  Warps 0..CW-1
// consume: each owns 16 rows and runs m16n8k16 BF16 tensor-core MMAs with
// the weights as the A operand (16 rows x 16 k) and x as the B operand
// (16 k x 8 columns = the M <= 8 activation rows, zero-padded).
//
// Dequantisation (Task 3 of the same page: one scale and bias per 128
// reduction values):
//   sum_k x[m,k] w[n,k] = sum_g ( s[n,g] * P[m,n,g] + b[n,g] * X[m,g] ),
//   P[m,n,g] = sum_{k in g} x[m,k] q[n,k],  X[m,g] = sum_{k in g} x[m,k].
// Codes enter the MMA as the exact BF16 values 128 + q (one LOP3 per two
// codes), so the MMA yields P + 128 X; a second MMA with an all-ones A
// operand yields X, and the epilogue applies s and (b - 128 s) once per group
// in FP32.  Every product is exact; only FP32 sums round.
#pragma once

#include "ptx.cuh"

namespace w4a16 {
namespace mv {

constexpr int kMaxM = 8;
constexpr int kStages = 12;
constexpr int kXCols = 136;              // x box width: 128 + 8 staggering columns
constexpr int kXRowBytes = kXCols * 2;   // 272 B: rows of x land 16 B apart in bank space

template <int CW>
struct Cfg {
    static constexpr int kRows = 16 * CW;
    static constexpr int kWBytes = kRows * 64;              // 16 packed words per row per group
    static constexpr int kXBytes = kMaxM * kXRowBytes;      // 2176 = 17 * 128
    static constexpr int kSBBytes = kRows * 2 * 4;          // one scale word, one bias word per row
    static constexpr int kStageBytes = kWBytes + kXBytes + kSBBytes;
    static constexpr int kThreads = (CW + 1) * 32;
    static constexpr int kBarOffset = kStages * kStageBytes;
    static constexpr int kSmemBytes = kBarOffset + 2 * kStages * 8 + 16;
    static_assert(kStageBytes % 128 == 0, "stages must stay 128-byte aligned");
};

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
    int pdl;                  // 1: launched with programmatic stream serialisation
};

// CTA whose range [c*U/P, (c+1)*U/P) contains unit u.
__host__ __device__ __forceinline__ long long streamk_owner(long long U, long long P, long long u) {
    return ((u + 1) * P - 1) / U;
}

__device__ __forceinline__ float scale_or_bias(uint32_t word, long long idx) {
    return (idx & 1) ? bf16_hi_to_f32(word) : bf16_lo_to_f32(word);
}

// Scale (or bias) element idx from its staged 4-byte word, except the last
// element of the array when it starts a word (not staged, read directly).
__device__ __forceinline__ float load_scale_bias(uint32_t word, long long idx, long long last_idx,
                                                 const uint16_t *src) {
    if (idx == last_idx && !(idx & 1)) return __uint_as_float(static_cast<uint32_t>(__ldg(src + idx)) << 16);
    return scale_or_bias(word, idx);
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float v) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

template <int CW>
__global__ void __launch_bounds__(Cfg<CW>::kThreads, 1)
    matvec_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                  const Params p) {
    using C = Cfg<CW>;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kBarOffset);
    uint64_t *empty = full + kStages;
    int *ticket_flag = reinterpret_cast<int *>(empty + kStages);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const long long U = p.units;
    const long long P = p.workers;
    const long long cta = blockIdx.x;
    const long long u0 = cta * U / P;
    const long long u1 = (cta + 1) * U / P;
    const int n_units = static_cast<int>(u1 - u0);
    const int G = p.G;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1 + 32);   // producer's expect_tx arrival + 32 cp.async arrivals
            mbar_init(&empty[s], CW);      // one arrival per consumer warp
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == CW) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tm_w);
            prefetch_tmap(&tm_x);
        }
        if (p.pdl) pdl_wait();   // inputs may come from the previous kernel in the stream
        const uint32_t tx_bytes = C::kWBytes + p.M * kXRowBytes;
        const long long last_idx = static_cast<long long>(p.N) * G - 1;
        int issued = 0;
        for (int i = 0; i < n_units; ++i) {
            const long long u = u0 + i;
            const int t = static_cast<int>(u / G);
            const int g = static_cast<int>(u - static_cast<long long>(t) * G);
            const int s = i % kStages;
            const uint32_t ph = (i / kStages) & 1;
            if (!mbar_wait(&empty[s], ph ^ 1)) break;
            uint8_t *st = smem + s * C::kStageBytes;
            if (lane == 0) {
                mbar_arrive_expect_tx(&full[s], tx_bytes);
                tma_load_2d(st, &tm_w, &full[s], g * 16, t * C::kRows);
                tma_load_2d(st + C::kWBytes, &tm_x, &full[s], g * 128, 0);
            }
            uint32_t *sb = reinterpret_cast<uint32_t *>(st + C::kWBytes + C::kXBytes);
#pragma unroll
            for (int j = 0; j < C::kRows / 32; ++j) {
                const int r = lane + 32 * j;
                const long long n = static_cast<long long>(t) * C::kRows + r;
                if (n < p.N) {
                    const long long idx = n * G + g;
                    const long long w_idx = idx & ~1LL;   // 4-byte word holding element idx
                    // The word holding the very last element of an array with an odd
                    // element count would reach past its end; consumers read that one
                    // element from global memory instead (see load_scale_bias).
                    if (w_idx + 1 <= last_idx) {
                        cp_async_4(&sb[r], p.scales + w_idx);
                        cp_async_4(&sb[C::kRows + r], p.biases + w_idx);
                    }
                }
            }
            cp_async_arrive_noinc(&full[s]);
            issued = i + 1;
        }
        // Every load of this CTA is issued: let the next kernel in the stream start
        // its prologue on SMs as they free up (programmatic dependent launch).
        if (lane == 0) pdl_launch_dependents();
        // Leave no copy in flight: wait (bounded) for the stages issued last.
        if (lane == 0) {
            const int first = issued > kStages ? issued - kStages : 0;
            for (int i = first; i < issued; ++i)
                mbar_wait(&full[i % kStages], (i / kStages) & 1, /*give_up_on_status=*/false);
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int gq = lane >> 2;       // MMA group id: A rows gq, gq+8; B column (= x row) gq
    const int tq = lane & 3;        // thread in group: k-slots 2tq, 2tq+1, 2tq+8, 2tq+9
    const bool swap_half = tq >= 2; // staggered chunk order, see the x loads below
    const int row0 = 16 * warp + gq;
    const uint32_t kOnes = 0x3F803F80u;   // BF16 (1.0, 1.0)
    const uint32_t ones[4] = {kOnes, kOnes, kOnes, kOnes};

    const long long last_idx = static_cast<long long>(p.N) * G - 1;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int i = 0; i < n_units; ++i) {
        const long long u = u0 + i;
        const int t = static_cast<int>(u / G);
        const int g = static_cast<int>(u - static_cast<long long>(t) * G);
        const int s = i % kStages;
        const uint32_t ph = (i / kStages) & 1;
        const bool ok = mbar_wait(&full[s], ph);

        const uint32_t st = smem_u32(smem + s * C::kStageBytes);
        // A operand: 16 bytes (32 codes) of row0 and of row0 + 8, chunk tq of the group.
        uint4 wa = lds128(st + row0 * 64 + 16 * tq);
        uint4 wb = lds128(st + (row0 + 8) * 64 + 16 * tq);
        // B operand: x row gq, the 32 values k in [32 tq, 32 tq + 32).  Threads with
        // tq >= 2 read their four 16-byte chunks in the order 2,3,0,1, which (with the
        // 272-byte row pitch) puts the 8 threads of each quarter warp on 8 distinct
        // 16-byte bank groups.  The A words are swapped the same way below, so both
        // operands of each MMA refer to the same k.
        uint4 xv[4];
        const uint32_t xrow = st + C::kWBytes + gq * kXRowBytes + 64 * tq;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int c = swap_half ? (r ^ 2) : r;
            xv[r] = (gq < p.M) ? lds128(xrow + 16 * c) : make_uint4(0u, 0u, 0u, 0u);
        }
        const uint32_t sbase = st + C::kWBytes + C::kXBytes;
        const uint32_t sw0 = lds32(sbase + 4 * row0);
        const uint32_t sw1 = lds32(sbase + 4 * (row0 + 8));
        const uint32_t bw0 = lds32(sbase + 4 * (C::kRows + row0));
        const uint32_t bw1 = lds32(sbase + 4 * (C::kRows + row0 + 8));
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);

        if (swap_half) {
            uint32_t tmp;
            tmp = wa.x; wa.x = wa.z; wa.z = tmp;
            tmp = wa.y; wa.y = wa.w; wa.w = tmp;
            tmp = wb.x; wb.x = wb.z; wb.z = tmp;
            tmp = wb.y; wb.y = wb.w; wb.w = tmp;
        }
        const uint32_t A0[4] = {wa.x, wa.y, wa.z, wa.w};
        const uint32_t A8[4] = {wb.x, wb.y, wb.z, wb.w};

        float pa[4] = {0.f, 0.f, 0.f, 0.f}, pb[4] = {0.f, 0.f, 0.f, 0.f};
        float xa[4] = {0.f, 0.f, 0.f, 0.f}, xb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            // word r of each row holds codes for 8 consecutive k; x chunk r holds the same k.
            // MMA (r, h=0) takes k-pairs (k0,k4) and (k1,k5); MMA (r, h=1) takes (k2,k6), (k3,k7).
            const uint32_t w0 = A0[r], w8 = A8[r];
            const uint32_t a_h0[4] = {codes_to_bf16x2_plus128(w0), codes_to_bf16x2_plus128(w8),
                                      codes_to_bf16x2_plus128(w0 >> 4), codes_to_bf16x2_plus128(w8 >> 4)};
            const uint32_t a_h1[4] = {codes_to_bf16x2_plus128(w0 >> 8), codes_to_bf16x2_plus128(w8 >> 8),
                                      codes_to_bf16x2_plus128(w0 >> 12), codes_to_bf16x2_plus128(w8 >> 12)};
            const uint32_t b00 = prmt(xv[r].x, xv[r].z, 0x5410u);
            const uint32_t b01 = prmt(xv[r].x, xv[r].z, 0x7632u);
            const uint32_t b10 = prmt(xv[r].y, xv[r].w, 0x5410u);
            const uint32_t b11 = prmt(xv[r].y, xv[r].w, 0x7632u);
            mma_bf16_16816(pa, a_h0, b00, b01, pa);
            mma_bf16_16816(xa, ones, b00, b01, xa);
            mma_bf16_16816(pb, a_h1, b10, b11, pb);
            mma_bf16_16816(xb, ones, b10, b11, xb);
        }
        // epilogue of this group: rows row0 (d0, d1) and row0 + 8 (d2, d3); x rows 2tq, 2tq+1
        {
            const long long n0 = static_cast<long long>(t) * C::kRows + row0;
            const long long idx0 = n0 * G + g;
            const long long idx1 = (n0 + 8) * G + g;
            const float s0 = load_scale_bias(sw0, idx0, last_idx, p.scales);
            const float s1 = load_scale_bias(sw1, idx1, last_idx, p.scales);
            const float b0 = load_scale_bias(bw0, idx0, last_idx, p.biases) - 128.f * s0;
            const float b1 = load_scale_bias(bw1, idx1, last_idx, p.biases) - 128.f * s1;
            const float X0 = xa[0] + xb[0];
            const float X1 = xa[1] + xb[1];
            acc[0] = fmaf(b0, X0, fmaf(s0, pa[0] + pb[0], acc[0]));
            acc[1] = fmaf(b0, X1, fmaf(s0, pa[1] + pb[1], acc[1]));
            acc[2] = fmaf(b1, X0, fmaf(s1, pa[2] + pb[2], acc[2]));
            acc[3] = fmaf(b1, X1, fmaf(s1, pa[3] + pb[3], acc[3]));
        }
        (void)ok;   // after a timeout the values are garbage; the loop still runs to keep barriers matched

        const bool tile_ends = (g == G - 1) || (i == n_units - 1);
        if (!tile_ends) continue;

        // ------------------------------------------------------------ tile output
        const long long tile_first = static_cast<long long>(t) * G;
        const long long tile_last = tile_first + G - 1;
        const long long nA = static_cast<long long>(t) * C::kRows + row0;
        const long long nB = nA + 8;
        const int mA = 2 * tq, mB = 2 * tq + 1;
        if (tile_first >= u0 && tile_last < u1) {
            if (nA < p.N) {
                if (mA < p.M) p.y[static_cast<long long>(mA) * p.N + nA] = f32_to_bf16_bits(acc[0]);
                if (mB < p.M) p.y[static_cast<long long>(mB) * p.N + nA] = f32_to_bf16_bits(acc[1]);
            }
            if (nB < p.N) {
                if (mA < p.M) p.y[static_cast<long long>(mA) * p.N + nB] = f32_to_bf16_bits(acc[2]);
                if (mB < p.M) p.y[static_cast<long long>(mB) * p.N + nB] = f32_to_bf16_bits(acc[3]);
            }
        } else {
            // split tile: publish this CTA's partial, take a ticket, last arriver reduces
            const int slot = (t == static_cast<int>(u0 / G)) ? 0 : 1;
            float *mine = p.partials + (cta * 2 + slot) * (C::kRows * 8);
            *reinterpret_cast<float2 *>(mine + row0 * 8 + 2 * tq) = make_float2(acc[0], acc[1]);
            *reinterpret_cast<float2 *>(mine + (row0 + 8) * 8 + 2 * tq) = make_float2(acc[2], acc[3]);
            __threadfence();
            named_bar_sync(1, CW * 32);
            const long long c_first = streamk_owner(U, P, tile_first);
            const long long c_last = streamk_owner(U, P, tile_last);
            if (threadIdx.x == 0) {
                const int old = atomicAdd(&p.tickets[t], 1);
                *ticket_flag = (old == static_cast<int>(c_last - c_first));
            }
            named_bar_sync(1, CW * 32);
            if (*ticket_flag) {
                __threadfence();
                float r[4] = {0.f, 0.f, 0.f, 0.f};
                for (long long cc = c_first; cc <= c_last; ++cc) {
                    const int cslot = (t == static_cast<int>((cc * U / P) / G)) ? 0 : 1;
                    const float *part = p.partials + (cc * 2 + cslot) * (C::kRows * 8);
                    const float2 v0 = __ldcg(reinterpret_cast<const float2 *>(part + row0 * 8 + 2 * tq));
                    const float2 v1 = __ldcg(reinterpret_cast<const float2 *>(part + (row0 + 8) * 8 + 2 * tq));
                    r[0] += v0.x; r[1] += v0.y; r[2] += v1.x; r[3] += v1.y;
                }
                if (nA < p.N) {
                    if (mA < p.M) p.y[static_cast<long long>(mA) * p.N + nA] = f32_to_bf16_bits(r[0]);
                    if (mB < p.M) p.y[static_cast<long long>(mB) * p.N + nA] = f32_to_bf16_bits(r[1]);
                }
                if (nB < p.N) {
                    if (mA < p.M) p.y[static_cast<long long>(mA) * p.N + nB] = f32_to_bf16_bits(r[2]);
                    if (mB < p.M) p.y[static_cast<long long>(mB) * p.N + nB] = f32_to_bf16_bits(r[3]);
                }
                if (threadIdx.x == 0) p.tickets[t] = 0;   // ready for the next launch
            }
        }
        acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
    }
}

}  // namespace mv
}  // namespace w4a16
