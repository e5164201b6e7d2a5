// matvec.cuh - weight-streaming W4A16 kernel for M <= 8 (decode).
//
// Role in the layer: tiny-llm "Week 2 Day 6: SIMD-Matrix Prefill", Task 1,
// keeps a matvec schedule for M <= 8.  This is a B200 design, not that
// Metal kernel: the whole cost is reading the packed weights once (0.5 byte
// per weight plus 4 bytes of scale and bias per 128 weights), so the kernel is
// built around keeping HBM busy with few, large asynchronous copies and
// around keeping the per-byte instruction count low enough that the SM keeps up.
//
// Work decomposition ("stream-K"): the output rows are cut into tiles of
// kRows = 256 rows, and each (row tile, 128-group) pair is one unit of work.
// The U = tiles * G units are split into `workers` contiguous ranges, one
// persistent CTA each (CTA c owns [c*U/P, (c+1)*U/P)), so every SM streams the
// same number of bytes whatever N and K are.  A tile whose groups are spread
// over several CTAs is finished by the CTA that holds its first group (the
// "finisher"); every other contributor ("publisher") holds the tile at the
// start of its range.  A publisher writes its FP32 partial to the workspace
// and its producer thread raises the tile's flag with a GPU-scope release.
// The finisher's producer thread, once it has issued all of its copies,
// acquires the flag and bulk-copies the partials into shared memory (a small
// area, or the copy ring once it has drained: the finished tile is the CTA's
// last).  The finisher adds them in CTA order: the sum does not depend on timing.
//
// Warp roles (21 warps, one CTA per SM):
//   warp 0, lane 0  producer: per stage one TMA tile load of packed codes
//                   ([256 rows x 128 bytes], 128-byte swizzle, 32 KB: two
//                   groups of one tile) and one of x ([M rows x 256] BF16 viewed
//                   as uint32 pairs); once per tile a 1-D bulk copy of the
//                   tile's scale rows and one of its bias rows; publication and
//                   partial gathering as above.  With the static-weights flag it
//                   issues the code and scale/bias copies of the first stages
//                   before waiting on the preceding kernel of the stream
//                   (programmatic dependent launch); x is always read after.
//   warps 1-4       x preparation: turn the stage's x into the B-operand
//                   fragments of the consumers' MMAs and sum x over each group
//                   (all-ones MMAs), a quarter of the stage each, once for all
//                   consumer warps.
//   warps 5-20      consumers: warp i owns rows 16 i .. 16 i + 15 of every tile
//                   and runs m16n8k16 BF16 tensor-core MMAs with the codes as
//                   the A operand (16 rows x 16 k) and x as the B operand (16 k
//                   x 8 columns = the M <= 8 activation rows, zero-padded).
//
// Dequantisation (Task 3 of the same page: one scale and bias per 128
// reduction values):
//   sum_k x[m,k] w[n,k] = sum_g ( s[n,g] * P[m,n,g] + b[n,g] * X[m,g] ),
//   P[m,n,g] = sum_{k in g} x[m,k] q[n,k],  X[m,g] = sum_{k in g} x[m,k].
// Codes enter the MMA as the exact BF16 values 128 + 8 q (one shift and one
// LOP3 per two codes), so the MMA yields 8 P + 128 X; the epilogue applies s / 8
// and (b - 16 s) once per group in FP32.  Every product is exact; only FP32 sums
// round.
#pragma once

#include "plain.cuh"
#include "ptx.cuh"

namespace w4a16 {
namespace mv {

constexpr int kMaxM = 8;
constexpr int kConsumerWarps = 16;                // one 16-row slice of the tile each
constexpr int kPrepWarps = 4;                     // one per SM sub-partition
constexpr int kRows = 16 * kConsumerWarps;        // rows of a tile: 256
constexpr int kProducerWarp = 0;
constexpr int kFirstPrepWarp = 1;
constexpr int kFirstConsumerWarp = kFirstPrepWarp + kPrepWarps;
constexpr int kThreads = (kFirstConsumerWarp + kConsumerWarps) * 32;
constexpr int kGroupsPerStage = 2;
constexpr int kWBytes = kRows * 64 * kGroupsPerStage;   // 32 KB of codes per stage
constexpr int kXCols = 128 * kGroupsPerStage;          // x columns of a stage
constexpr int kXRowBytes = kXCols * 2;                 // 512 B
constexpr int kXBytes = kMaxM * kXRowBytes;            // raw x of a stage: 4 KB
constexpr int kFragBytes = kGroupsPerStage * 4 * 32 * 16;   // its B fragments: 4 KB
constexpr int kStageBytes = kWBytes + kXBytes + kFragBytes;
constexpr int kXSumBytes = kPrepWarps * kMaxM * 4;     // partial sums of x of a stage, one per prep warp
constexpr int kPartialFloats = kMaxM * kRows;          // one CTA's published partial: [8][256] FP32
constexpr int kPartAreaBytes = 8192;                   // prefetched partials of a finished tile
constexpr int kFlagStaticWeights = 2;    // codes, scales and biases may be read before the wait
constexpr int kFixupBatch = 8;           // partials loaded at once
constexpr int kBarriers = 6;             // slab_full[2], slab_empty[2], pub, parts
static_assert(kWBytes % 1024 == 0 && kStageBytes % 1024 == 0, "swizzled stages need 1 KB alignment");

// bytes of one scale (or bias) slab: kRows x G BF16, rounded to 128 B
__host__ __device__ constexpr long long slab_array_bytes(long long G) { return ((kRows * G * 2 + 127) / 128) * 128; }
__host__ __device__ constexpr long long smem_bytes(int stages, int slab_slots, long long G) {
    return stages * (kStageBytes + kXSumBytes) + slab_slots * 2 * slab_array_bytes(G) + kPartAreaBytes
           + (3 * stages + kBarriers) * 8 + 1024;    // barriers, alignment slack
}

struct Params {
    const uint16_t *x;        // bf16 [M, K] (read by TMA; directly only by the plain path)
    const uint32_t *wq;       // [N, K/8] packed codes (likewise)
    const uint16_t *scales;   // bf16 [N, G]
    const uint16_t *biases;   // bf16 [N, G]
    uint16_t *y;              // bf16 [M, N]
    float *partials;          // [workers][kMaxM][kRows] FP32
    int *flags;               // [tiles], zero between launches
    int M, N, G;
    int tiles;
    long long units;          // tiles * G
    int workers;              // gridDim.x
    int stages;               // depth of the code/x ring
    int slab_slots;           // 0 (scales/biases read from global), 1 or 2
    int slab_array_bytes;     // slab_array_bytes(G)
    int opts;                 // kFlagStaticWeights
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

// The split-tile roles of a CTA with unit range [u0, u1).
struct Roles {
    int pub_tile;     // tile whose partial this CTA publishes (its first tile), or -1
    int fin_tile;     // tile this CTA finishes (its last tile), or -1
    int publishers;   // CTAs publishing into fin_tile
    __device__ void init(long long U, long long P, long long cta, long long u0, long long u1, int G) {
        const long long tf = u0 / G, tl = (u1 - 1) / G;
        pub_tile = (u0 % G != 0) ? static_cast<int>(tf) : -1;
        const bool fin = (u1 % G != 0) && tl * G >= u0;
        fin_tile = fin ? static_cast<int>(tl) : -1;
        publishers = fin ? static_cast<int>(streamk_owner(U, P, (tl + 1) * G - 1) - cta) : 0;
    }
};

// One CTA per SM (a deep copy ring needs most of the shared memory).  The
// register file is split between the SM's four sub-partitions and one of them
// holds 6 of the 21 warps: at most 16384 / (6 * 32) -> 80 registers per thread.
__global__ void __maxnreg__(80)
    matvec_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                  const Params p) {
    extern __shared__ uint8_t smem_raw[];
    // 1 KB alignment for the swizzled code tiles, by offsetting within the shared
    // array (so the compiler still knows every access below is a shared-memory one).
    // x is loaded through a uint32 view of [M, K/2] pairs (a 128-element box per stage).
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int S = p.stages;
    uint8_t *xsum_base = smem + S * kStageBytes;                        // [S][4 prep warps][8] FP32
    uint8_t *slab_base = xsum_base + S * kXSumBytes;
    uint8_t *part_area = slab_base + p.slab_slots * 2 * p.slab_array_bytes;
    uint64_t *full = reinterpret_cast<uint64_t *>(part_area + kPartAreaBytes);   // codes landed + x prepared
    uint64_t *xfull = full + S;                                                  // raw x landed
    uint64_t *empty = xfull + S;
    uint64_t *slab_full = empty + S;
    uint64_t *slab_empty = slab_full + 2;
    uint64_t *pub_bar = slab_empty + 2;    // consumers wrote the published partial
    uint64_t *parts_bar = pub_bar + 1;     // finisher: partials available

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
            mbar_init(&full[s], 1 + kPrepWarps);     // producer's expect_tx arrive + x preparation
            mbar_init(&xfull[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&slab_full[s], 1);
            mbar_init(&slab_empty[s], kConsumerWarps);
        }
        mbar_init(pub_bar, kConsumerWarps);
        mbar_init(parts_bar, 1);
        fence_mbar_init();
    }
    __syncthreads();

    Roles roles;
    roles.init(U, P, cta, u0, u1, G);
    // Where the finisher reads the publishers' partials: the small partial area (copied
    // as soon as they are ready), the copy ring (copied once the ring has drained:
    // the finished tile is this CTA's last), or global memory.
    const uint32_t part_bytes = static_cast<uint32_t>(p.M) * kRows * 4;       // one publisher's partial
    const uint32_t parts_need = roles.publishers * part_bytes;
    const bool parts_in_area = parts_need <= static_cast<uint32_t>(kPartAreaBytes);
    const bool parts_in_smem = parts_need <= static_cast<uint32_t>(S) * kStageBytes;
    uint8_t *parts_dst = parts_in_area ? part_area : smem;

    if (warp == kProducerWarp) {
        // ------------------------------------------------------------ producer (one thread)
        if (lane != 0) return;
        prefetch_tmap(&tm_w);
        prefetch_tmap(&tm_x);
        const uint32_t x_bytes = p.M * kXRowBytes;
        const bool prefetch = (p.opts & kFlagStaticWeights) != 0;
        int tile_seq = -1, prev_t = -1, slabs_issued = 0;
        bool published = roles.pub_tile < 0;

        // Raise the flag of the published tile once every consumer warp has written
        // its rows of the partial (their mbarrier arrivals release the writes to this
        // thread; the release-add carries them to GPU scope).  Blocks only with `wait`.
        auto try_publish = [&](bool wait) {
            if (published) return;
            if (wait ? mbar_wait(pub_bar, 0) : mbar_test_wait(pub_bar, 0)) {
                red_release_gpu_add(&p.flags[roles.pub_tile], 1);
                published = true;
            }
        };
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
            mbar_arrive_expect_tx(&full[s], kWBytes);
            tma_load_2d(smem + s * kStageBytes, &tm_w, &full[s], wk.g * 16, wk.t * kRows);
            return true;
        };
        auto issue_x = [&](const StageWalker &wk, int i) {
            const int s = i % S;
            mbar_arrive_expect_tx(&xfull[s], x_bytes);
            tma_load_2d(smem + s * kStageBytes + kWBytes, &tm_x, &xfull[s], wk.g * 64, 0);
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
        bool ok = true;
        for (int i = issued; wk.n; ++i, wk.next()) {
            const int s = i % S;
            if (i >= S) {
                try_publish(false);
                if (!mbar_wait(&empty[s], ((i / S) - 1) & 1)) { ok = false; break; }
            }
            if (!issue_codes(wk, i, /*may_recycle=*/true)) { ok = false; break; }
            issue_x(wk, i);
            issued = i + 1;
        }
        if (ok) try_publish(true);
        bool parts_pending = false;
        if (ok && roles.fin_tile >= 0) {
            // every publisher of the finished tile raised its flag: fetch their partials
            int *flag = &p.flags[roles.fin_tile];
            const unsigned long long t0 = globaltimer();
            bool ready = true;
            for (uint32_t spin = 0; ld_acquire_gpu(flag) < roles.publishers; ++spin) {
                if ((spin & 15u) == 15u && (status_set() || globaltimer() - t0 > kWaitTimeoutNs)) {
                    if (!status_set()) record_timeout();
                    ready = false;
                    break;
                }
            }
            if (ready) {
                *flag = 0;   // no further arrivals this launch; ready for the next one
                if (parts_in_smem && !parts_in_area) {
                    // every consumer has released every stage: the ring is free
                    for (int i = max(0, issued - S); i < issued; ++i)
                        mbar_wait(&empty[i % S], (i / S) & 1, /*give_up_on_status=*/false);
                }
                if (parts_in_smem) {
                    fence_proxy_async_global();
                    mbar_arrive_expect_tx(parts_bar, parts_need);
                    for (int j = 0; j < roles.publishers; ++j)
                        bulk_load(parts_dst + j * part_bytes, p.partials + (cta + 1 + j) * kPartialFloats,
                                  part_bytes, parts_bar);
                    parts_pending = true;
                } else {
                    mbar_arrive(parts_bar);
                }
            }
        }
        // Leave no copy in flight: wait (bounded) for the stages, slabs and partials issued last.
        for (int i = max(0, issued - S); i < issued; ++i) {
            mbar_wait(&xfull[i % S], (i / S) & 1, /*give_up_on_status=*/false);
            mbar_wait(&full[i % S], (i / S) & 1, /*give_up_on_status=*/false);
        }
        for (int q = max(0, slabs_issued - slots); q < slabs_issued; ++q)
            mbar_wait(&slab_full[q % slots], (q / slots) & 1, /*give_up_on_status=*/false);
        if (parts_pending) mbar_wait(parts_bar, 0, /*give_up_on_status=*/false);
        return;
    }

    if (warp < kFirstConsumerWarp) {
        // ------------------------------------------------------------ x preparation
        // Prep warp pw handles group j = pw / 2 and code words r = 2 (pw % 2) + {0, 1}:
        // lane (gq, tq) builds the B fragment of x row gq for the k the consumers' A
        // word r holds: k0 = 128 j + 32 tq + 8 r, pairs (k0, k0+4), (k0+1, k0+5) for the
        // MMA of codes (0,4),(1,5) and (k0+2, k0+6), (k0+3, k0+7) for codes (2,6),(3,7).
        // Fragment (j, r) of lane L lives at 16 * ((4 j + r) * 32 + L) in the stage's
        // fragment area; lanes of absent x rows (gq >= M) read nothing and write zeros.
        // It also sums x over its 64 k (all-ones MMAs).
        const int pw = warp - kFirstPrepWarp;
        const int j = pw >> 1, r0 = 2 * (pw & 1);
        const int gq = lane >> 2, tq = lane & 3;
        const uint32_t kOnes = 0x3F803F80u;        // BF16 (1.0, 1.0)
        const uint32_t ones[4] = {kOnes, kOnes, kOnes, kOnes};
        const bool live_row = gq < p.M;
        StageWalker wk;
        wk.start(u0, u1, G);
        int s = 0;
        uint32_t ph = 0;
        for (; wk.n; wk.next(), (++s == S ? (s = 0, ph ^= 1u) : 0u)) {
            if (!mbar_wait(&xfull[s], ph)) break;
            const uint32_t xs = smem_u32(smem + s * kStageBytes + kWBytes);
            const uint32_t fs = xs + kXBytes;
            float xsum[4] = {};
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int r = r0 + q;
                const uint4 v = live_row ? lds128(xs + gq * kXRowBytes + 256 * j + 64 * tq + 16 * r)
                                         : make_uint4(0, 0, 0, 0);
                uint4 f;
                f.x = prmt(v.x, v.z, 0x5410u);
                f.y = prmt(v.x, v.z, 0x7632u);
                f.z = prmt(v.y, v.w, 0x5410u);
                f.w = prmt(v.y, v.w, 0x7632u);
                sts128(fs + 16 * ((4 * j + r) * 32 + lane), f);   // zeros for absent rows
                mma_bf16_16816(xsum, ones, f.x, f.y, xsum);
                mma_bf16_16816(xsum, ones, f.z, f.w, xsum);
            }
            if (gq == 0)   // row 0 of the all-ones products: sums for x rows 2tq, 2tq+1
                *reinterpret_cast<float2 *>(xsum_base + s * kXSumBytes + pw * (kMaxM * 4) + 8 * tq) =
                    make_float2(xsum[0], xsum[1]);
            fence_proxy_async_smem();   // a later bulk copy of partials may overwrite the fragments
            __syncwarp();
            if (lane == 0) mbar_arrive(&full[s]);
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    // Consumer warp `slice` owns rows 16 slice .. 16 slice + 15 of every tile and
    // both groups of each stage, one after the other.
    const int slice = warp - kFirstConsumerWarp;
    const int gq = lane >> 2;       // MMA group id: A rows gq, gq+8; B column (= x row) gq
    const int tq = lane & 3;        // thread in group: k-slots 2tq, 2tq+1, 2tq+8, 2tq+9
    const int rA = 16 * slice + row_of(gq);       // data rows of MMA rows gq and gq + 8
    const int rB = 16 * slice + row_of(gq + 8);
    const uint32_t smem_base = smem_u32(smem);
    // 128-byte swizzle: chunk c of row r is stored at chunk c ^ (r & 7)
    const uint32_t swzA = (rA & 7) << 4, swzB = (rB & 7) << 4;
    const uint32_t frag_off = kWBytes + kXBytes + 16 * lane;
    const uint32_t xsum_off = smem_u32(xsum_base) + 8 * tq;

    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    int tile_seq = -1, prev_t = -1;
    // scale/bias rows of the current tile: shared-memory slab rows, or global rows
    uint32_t sl_s = 0, sl_b = 0;            // slab addresses of row 0 of this tile
    bool slab_rows = false;
    long long gA = 0, gB = 0;               // global element offsets of rows rA, rB of this tile
    StageWalker wk;
    wk.start(u0, u1, G);
    int s = 0;                            // ring position of stage i
    uint32_t ph = 0;                      // its phase parity
    for (; wk.n; wk.next(), (++s == S ? (s = 0, ph ^= 1u) : 0u)) {
        const int t = wk.t;
        const long long first_row = static_cast<long long>(t) * kRows;
        if (t != prev_t) {
            prev_t = t;
            ++tile_seq;
            const long long rows = min(static_cast<long long>(kRows), p.N - first_row);
            slab_rows = false;
            if (slots) {
                const int slot = tile_seq % slots;
                mbar_wait(&slab_full[slot], (tile_seq / slots) & 1);
                slab_rows = ((rows * G * 2) & 15) == 0;   // the whole slab landed
                sl_s = smem_u32(slab_base + slot * 2 * p.slab_array_bytes);
                sl_b = sl_s + p.slab_array_bytes;
            }
            // rows past N read row N-1 (their results are never stored)
            gA = min(first_row + rA, static_cast<long long>(p.N) - 1) * G;
            gB = min(first_row + rB, static_cast<long long>(p.N) - 1) * G;
        }
        mbar_wait(&full[s], ph);
        const uint32_t st = smem_base + s * kStageBytes;
        const uint32_t xst = xsum_off + s * kXSumBytes;
        const int ng = wk.n;
#pragma unroll
        for (int j = 0; j < kGroupsPerStage; ++j) {
            if (j >= ng) break;
            const int g = wk.g + j;
            // chunk 4 j + tq of each row: the swizzle XORs the chunk index with row & 7
            const uint4 wa = lds128(st + rA * 128 + (((4 * j + tq) << 4) ^ swzA));
            const uint4 wb = lds128(st + rB * 128 + (((4 * j + tq) << 4) ^ swzB));
            uint4 fr[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) fr[r] = lds128(st + frag_off + 512 * (4 * j + r));
            // x sums of group j: prep warps 2 j and 2 j + 1 each summed half of it
            const float2 X0 = lds_f2(xst + 2 * j * (kMaxM * 4));
            const float2 X1 = lds_f2(xst + (2 * j + 1) * (kMaxM * 4));
            // scale and bias of rows rA, rB for group g; b' = b - 16 s
            uint32_t s0, s1, b0, b1;
            if (slab_rows) {
                s0 = lds16(sl_s + 2 * (rA * G + g));
                s1 = lds16(sl_s + 2 * (rB * G + g));
                b0 = lds16(sl_b + 2 * (rA * G + g));
                b1 = lds16(sl_b + 2 * (rB * G + g));
            } else {
                s0 = __ldg(p.scales + gA + g);
                s1 = __ldg(p.scales + gB + g);
                b0 = __ldg(p.biases + gA + g);
                b1 = __ldg(p.biases + gB + g);
            }
            float pacc[2][4] = {};   // [code pair][fragment]
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                // word r of each row holds codes for 8 consecutive k; fragment r holds the same k
                const uint32_t w0 = (r == 0) ? wa.x : (r == 1) ? wa.y : (r == 2) ? wa.z : wa.w;
                const uint32_t w8 = (r == 0) ? wb.x : (r == 1) ? wb.y : (r == 2) ? wb.z : wb.w;
                const uint32_t a_h0[4] = {codes_to_bf16x2_128_plus_8q(w0 << 3), codes_to_bf16x2_128_plus_8q(w8 << 3),
                                          codes_to_bf16x2_128_plus_8q(w0 >> 1), codes_to_bf16x2_128_plus_8q(w8 >> 1)};
                const uint32_t a_h1[4] = {codes_to_bf16x2_128_plus_8q(w0 >> 5), codes_to_bf16x2_128_plus_8q(w8 >> 5),
                                          codes_to_bf16x2_128_plus_8q(w0 >> 9), codes_to_bf16x2_128_plus_8q(w8 >> 9)};
                mma_bf16_16816(pacc[0], a_h0, fr[r].x, fr[r].y, pacc[0]);
                mma_bf16_16816(pacc[1], a_h1, fr[r].z, fr[r].w, pacc[1]);
            }
            // epilogue: rows rA (d0, d1) and rB (d2, d3); x rows 2tq, 2tq+1
            const float Xa = X0.x + X1.x, Xb = X0.y + X1.y;
            const float sA = 0.125f * bf16_bits_to_f32(s0), sB = 0.125f * bf16_bits_to_f32(s1);   // s / 8
            const float bA = fmaf(-128.f, sA, bf16_bits_to_f32(b0)), bB = fmaf(-128.f, sB, bf16_bits_to_f32(b1));   // b - 16 s
            acc[0] = fmaf(bA, Xa, fmaf(sA, pacc[0][0] + pacc[1][0], acc[0]));
            acc[1] = fmaf(bA, Xb, fmaf(sA, pacc[0][1] + pacc[1][1], acc[1]));
            acc[2] = fmaf(bB, Xa, fmaf(sB, pacc[0][2] + pacc[1][2], acc[2]));
            acc[3] = fmaf(bB, Xb, fmaf(sB, pacc[0][3] + pacc[1][3], acc[3]));
        }
        // every operand of this stage has been read: release the slot
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);

        if (!wk.tile_ends()) continue;
        if (slots) {   // this tile's slab is no longer needed
            __syncwarp();
            if (lane == 0) mbar_arrive(&slab_empty[tile_seq % slots]);
        }

        // ------------------------------------------------------------ tile output
        const long long nA = first_row + rA;
        const long long nB = first_row + rB;
        const int mA = 2 * tq, mB = 2 * tq + 1;
        float out[4] = {acc[0], acc[1], acc[2], acc[3]};
        acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
        if (t == roles.pub_tile) {
            // publish: [m][row] partial of this CTA; the producer raises the flag
            float *mine = p.partials + cta * kPartialFloats;
            if (mA < p.M) { mine[mA * kRows + rA] = out[0]; mine[mA * kRows + rB] = out[2]; }
            if (mB < p.M) { mine[mB * kRows + rA] = out[1]; mine[mB * kRows + rB] = out[3]; }
            __syncwarp();
            if (lane == 0) mbar_arrive(pub_bar);
            continue;
        }
        if (t == roles.fin_tile) {
            // add the publishers' partials, in CTA order, to this CTA's own
            if (!mbar_wait(parts_bar, 0)) continue;
            const bool hasA = mA < p.M, hasB = mB < p.M;
            if (parts_in_smem) {
                const uint32_t base = smem_u32(parts_dst);
#pragma unroll 4
                for (int j = 0; j < roles.publishers; ++j) {
                    const uint32_t part = base + j * part_bytes;
                    if (hasA) {
                        out[0] += __uint_as_float(lds32(part + 4 * (mA * kRows + rA)));
                        out[2] += __uint_as_float(lds32(part + 4 * (mA * kRows + rB)));
                    }
                    if (hasB) {
                        out[1] += __uint_as_float(lds32(part + 4 * (mB * kRows + rA)));
                        out[3] += __uint_as_float(lds32(part + 4 * (mB * kRows + rB)));
                    }
                }
            } else {
                for (int cb = 0; cb < roles.publishers; cb += kFixupBatch) {
                    float v[kFixupBatch][4];
#pragma unroll
                    for (int j = 0; j < kFixupBatch; ++j) {   // issue every load of the batch first
                        v[j][0] = v[j][1] = v[j][2] = v[j][3] = 0.f;
                        if (cb + j >= roles.publishers) continue;
                        const float *part = p.partials + (cta + 1 + cb + j) * kPartialFloats;
                        if (hasA) { v[j][0] = __ldcg(part + mA * kRows + rA); v[j][2] = __ldcg(part + mA * kRows + rB); }
                        if (hasB) { v[j][1] = __ldcg(part + mB * kRows + rA); v[j][3] = __ldcg(part + mB * kRows + rB); }
                    }
#pragma unroll
                    for (int j = 0; j < kFixupBatch; ++j)   // then add them in CTA order
#pragma unroll
                        for (int e = 0; e < 4; ++e) out[e] += v[j][e];
                }
            }
        }
        // outputs whose BF16 result is not finite: the plain definition
        const long long nn[4] = {nA, nA, nB, nB}, mm[4] = {mA, mB, mA, mB};
#pragma unroll
        for (int e = 0; e < 4; ++e)
            if (!isfinite(__bfloat162float(__float2bfloat16_rn(out[e]))) && nn[e] < p.N && mm[e] < p.M) {
                const long long K = static_cast<long long>(p.G) * 128;
                out[e] = plain_output(p.x + mm[e] * K, p.wq + nn[e] * (K / 8), p.scales + nn[e] * p.G,
                                      p.biases + nn[e] * p.G, p.G);
            }
        if (nA < p.N) {
            if (mA < p.M) p.y[static_cast<long long>(mA) * p.N + nA] = f32_to_bf16_bits(out[0]);
            if (mB < p.M) p.y[static_cast<long long>(mB) * p.N + nA] = f32_to_bf16_bits(out[1]);
        }
        if (nB < p.N) {
            if (mA < p.M) p.y[static_cast<long long>(mA) * p.N + nB] = f32_to_bf16_bits(out[2]);
            if (mB < p.M) p.y[static_cast<long long>(mB) * p.N + nB] = f32_to_bf16_bits(out[3]);
        }
    }
}

}  // namespace mv
}  // namespace w4a16
