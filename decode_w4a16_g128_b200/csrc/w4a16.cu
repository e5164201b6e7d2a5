// w4a16.cu - the C ABI declared in include/w4a16.h, built as ONE translation
// unit with every kernel of the library (so the device status word has a
// single definition).  Host code here validates arguments, plans the launch,
// owns the split bookkeeping workspace and encodes the TMA tensor maps.
// There is no host fallback: every output element is computed by a kernel.
#include "w4a16.h"

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include "gemm.cuh"
#include "matvec.cuh"
#include "nbit.cuh"
#include "quant.cuh"
#include "rows.cuh"

namespace w4a16 {
namespace {

constexpr int kVersion = 100;          // 0.1.0
constexpr int kMinTickets = 1 << 16;   // ticket slots allocated up front (grows on demand)
constexpr int kSkinnyMaxM = 32;        // the row-block matvec over slices of 8 x rows, up to this M
// Shared memory of a matvec CTA: one CTA per SM, most of the SM's shared
// memory, so that the copy ring is deep enough to cover HBM latency.
constexpr long long kMatvecBudget = 220 * 1024;
constexpr int kMatvecMaxStages = 10;
constexpr int kMatvecMinStages = 4;

std::atomic<int> g_last_cuda_error{0};

int cuda_fail(cudaError_t e) {
    g_last_cuda_error.store(static_cast<int>(e));
    return W4A16_ERR_CUDA;
}

struct DeviceInfo {
    bool ready = false;
    int status = W4A16_OK;
    int sms = 0;
    bool gemm_ok = false;     // the GEMM's register split fits its launch allocation
    int gemm_clusters = 0;    // CTA pairs of the GEMM resident at once (its persistent grid)
    int gemm_max_splits = 4;  // K splits of the GEMM: 8 where clusters of 16 CTAs can be resident
    PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
};

struct Workspace {
    float *partials = nullptr;
    size_t partial_floats = 0;
    int *tickets = nullptr;     // per-tile flags of the matvec fix-up, zero between launches
    int64_t ticket_count = 0;
    uint16_t *xs = nullptr;     // GEMM bias-step operands: x group sums [M, Kx], then coefficients [N, Kx]
    size_t xs_elems = 0;
};

std::mutex g_mu;
std::map<int, DeviceInfo> g_devices;
std::map<std::pair<int, void *>, Workspace> g_workspaces;

template <int RB>
cudaError_t rows_set_attributes_one() {
    cudaError_t e = cudaFuncSetAttribute(mvr::rows_kernel<RB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(mvr::kBudget));
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(mvr::rows_kernel<RB>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    return e;
}

cudaError_t rows_set_attributes() {
    static_assert(mvr::kMaxRB == 5, "one instantiation per row-block count");
    cudaError_t e = rows_set_attributes_one<1>();
    if (e == cudaSuccess) e = rows_set_attributes_one<2>();
    if (e == cudaSuccess) e = rows_set_attributes_one<3>();
    if (e == cudaSuccess) e = rows_set_attributes_one<4>();
    if (e == cudaSuccess) e = rows_set_attributes_one<5>();
    return e;
}

// Per-device one-time set-up: capability check, SM count, driver entry point,
// kernel attributes.  Caller holds g_mu.
int device_setup(int dev, DeviceInfo **out) {
    DeviceInfo &d = g_devices[dev];
    if (!d.ready) {
        int major = 0, minor = 0;
        cudaError_t e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail(e);
        if (major != 10 || minor != 0) {
            d.status = W4A16_ERR_DEVICE;
        } else {
            void *fn = nullptr;
            cudaDriverEntryPointQueryResult q{};
            e = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q);
            if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) return cuda_fail(e);
            d.encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
            // The GEMM's warpgroups rebalance registers with setmaxnreg; a split larger than
            // the allocation the kernel is launched with would never be granted, so the GEMM
            // path is refused (W4A16_ERR_UNSUPPORTED) unless it fits.
            cudaFuncAttributes fa{};
            e = cudaFuncGetAttributes(&fa, gm::gemm_kernel);
            if (e != cudaSuccess) return cuda_fail(e);
            d.gemm_ok = fa.numRegs * gm::kThreads >=
                        128 * (gm::kRegsCtl + 2 * gm::kRegsDeq + 2 * gm::kRegsEpi);
            // the largest shared-memory carveout: two row-block CTAs per SM (without it the
            // driver picks a split that holds one), and the same split as the other kernels
            e = rows_set_attributes();
            if (e != cudaSuccess) return cuda_fail(e);
            e = cudaFuncSetAttribute(mv::matvec_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     int(kMatvecBudget));
            if (e == cudaSuccess)   // one carveout for every launch: no reconfiguration between them
                e = cudaFuncSetAttribute(mv::matvec_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(gm::gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         gm::smem_bytes(gm::kMaxGroups));
            if (e == cudaSuccess)   // clusters of 2 x 8 K splits exceed the portable size of 8
                e = cudaFuncSetAttribute(gm::gemm_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
            if (e != cudaSuccess) return cuda_fail(e);
            // how many CTA pairs of the GEMM the device holds at once: the persistent grid
            // never exceeds it, so that no pair waits for another to finish
            cudaLaunchConfig_t occ = {};
            occ.gridDim = dim3(2, 1, 1);
            occ.blockDim = dim3(gm::kThreads, 1, 1);
            occ.dynamicSmemBytes = gm::smem_bytes(gm::kMaxGroups);
            cudaLaunchAttribute cl;
            cl.id = cudaLaunchAttributeClusterDimension;
            cl.val.clusterDim.x = 2;
            cl.val.clusterDim.y = 1;
            cl.val.clusterDim.z = 1;
            occ.attrs = &cl;
            occ.numAttrs = 1;
            int clusters = 0;
            e = cudaOccupancyMaxActiveClusters(&clusters, gm::gemm_kernel, &occ);
            if (e != cudaSuccess) return cuda_fail(e);
            d.gemm_clusters = clusters > 0 ? clusters : d.sms / 2;
            // K splits above 4 take clusters of more than 8 CTAs: only where one fits
            occ.gridDim = dim3(2 * gm::kMaxSplits, 1, 1);
            cl.val.clusterDim.x = 2 * gm::kMaxSplits;
            int big = 0;
            e = cudaOccupancyMaxActiveClusters(&big, gm::gemm_kernel, &occ);
            if (e != cudaSuccess) {
                cudaGetLastError();
                big = 0;
            }
            d.gemm_max_splits = big > 0 ? gm::kMaxSplits : 4;
        }
        d.ready = true;
    }
    *out = &d;
    return d.status;
}

int current_device(int *dev) {
    cudaError_t e = cudaGetDevice(dev);
    return e == cudaSuccess ? W4A16_OK : cuda_fail(e);
}

// Workspace of (device, stream), grown to at least the requested sizes.  A
// stream that is being captured cannot allocate, so growth there is refused.
int workspace_get(int dev, void *stream, size_t partial_floats, int64_t tickets, Workspace **out) {
    Workspace &w = g_workspaces[{dev, stream}];
    const bool grow_p = w.partial_floats < partial_floats;
    const bool grow_t = w.ticket_count < tickets;
    if (grow_p || grow_t) {
        cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
        cudaError_t e = cudaStreamIsCapturing(static_cast<cudaStream_t>(stream), &cap);
        if (e != cudaSuccess) return cuda_fail(e);
        if (cap != cudaStreamCaptureStatusNone) return W4A16_ERR_UNSUPPORTED;
        e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));   // old buffers may be in use
        if (e != cudaSuccess) return cuda_fail(e);
        if (grow_p) {
            cudaFree(w.partials);
            w.partials = nullptr;
            w.partial_floats = 0;
            if (cudaMalloc(&w.partials, partial_floats * sizeof(float)) != cudaSuccess) {
                cudaGetLastError();
                return W4A16_ERR_NO_MEMORY;
            }
            w.partial_floats = partial_floats;
        }
        if (grow_t) {
            const int64_t count = std::max<int64_t>(tickets, kMinTickets);
            cudaFree(w.tickets);
            w.tickets = nullptr;
            w.ticket_count = 0;
            if (cudaMalloc(&w.tickets, count * sizeof(int)) != cudaSuccess) {
                cudaGetLastError();
                return W4A16_ERR_NO_MEMORY;
            }
            e = cudaMemset(w.tickets, 0, count * sizeof(int));
            if (e != cudaSuccess) return cuda_fail(e);
            w.ticket_count = count;
        }
    }
    *out = &w;
    return W4A16_OK;
}

// The GEMM's bias-step operand buffer of (device, stream), grown to at least `elems` BF16 values.
int workspace_xs(int dev, void *stream, size_t elems, Workspace **out) {
    Workspace &w = g_workspaces[{dev, stream}];
    if (w.xs_elems < elems) {
        cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
        cudaError_t e = cudaStreamIsCapturing(static_cast<cudaStream_t>(stream), &cap);
        if (e != cudaSuccess) return cuda_fail(e);
        if (cap != cudaStreamCaptureStatusNone) return W4A16_ERR_UNSUPPORTED;
        e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));   // the old buffer may be in use
        if (e != cudaSuccess) return cuda_fail(e);
        cudaFree(w.xs);
        w.xs = nullptr;
        w.xs_elems = 0;
        if (cudaMalloc(&w.xs, elems * sizeof(uint16_t)) != cudaSuccess) {
            cudaGetLastError();
            return W4A16_ERR_NO_MEMORY;
        }
        w.xs_elems = elems;
    }
    *out = &w;
    return W4A16_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + nb && b0 < a0 + na;
}

struct Problem {
    const void *x;
    const uint32_t *wq;
    const void *scales;
    const void *biases;
    void *y;
    int64_t M, N, K;
};

int validate(const Problem &p) {
    if (p.M < 0 || p.N < 0 || p.K < 0) return W4A16_ERR_INVALID_ARG;
    if (p.K % 128 != 0) return W4A16_ERR_UNSUPPORTED;
    if (p.M >= (int64_t(1) << 31) || p.N >= (int64_t(1) << 31) || p.K >= (int64_t(1) << 31))
        return W4A16_ERR_UNSUPPORTED;
    if (p.M == 0 || p.N == 0) return W4A16_OK;
    if (!p.y) return W4A16_ERR_INVALID_ARG;
    if (!aligned16(p.y)) return W4A16_ERR_MISALIGNED;
    if (p.K == 0) return W4A16_OK;
    if (!p.x || !p.wq || !p.scales || !p.biases) return W4A16_ERR_INVALID_ARG;
    if (!aligned16(p.x) || !aligned16(p.wq) || !aligned16(p.scales) || !aligned16(p.biases))
        return W4A16_ERR_MISALIGNED;
    const size_t ny = size_t(p.M) * p.N * 2;
    if (overlaps(p.y, ny, p.x, size_t(p.M) * p.K * 2) || overlaps(p.y, ny, p.wq, size_t(p.N) * p.K / 2) ||
        overlaps(p.y, ny, p.scales, size_t(p.N) * (p.K / 128) * 2) ||
        overlaps(p.y, ny, p.biases, size_t(p.N) * (p.K / 128) * 2))
        return W4A16_ERR_INVALID_ARG;
    return W4A16_OK;
}

int choose_path(int64_t M, const w4a16_options *opt, int *path) {
    const int req = opt ? opt->path : W4A16_PATH_AUTO;
    if (req == W4A16_PATH_AUTO) {
        *path = M <= mv::kMaxM ? W4A16_PATH_MATVEC : W4A16_PATH_GEMM;
    } else if (req == W4A16_PATH_MATVEC) {
        if (M > mv::kMaxM) return W4A16_ERR_UNSUPPORTED;
        *path = W4A16_PATH_MATVEC;
    } else if (req == W4A16_PATH_GEMM) {
        *path = W4A16_PATH_GEMM;
    } else if (req == W4A16_PATH_MATVEC_ROWS) {
        if (M > kSkinnyMaxM) return W4A16_ERR_UNSUPPORTED;
        *path = W4A16_PATH_MATVEC_ROWS;
    } else {
        return W4A16_ERR_INVALID_ARG;
    }
    return W4A16_OK;
}

int validate_options(const w4a16_options *opt) {
    if (!opt) return W4A16_OK;
    if (opt->splits < 0 || opt->splits > gm::kMaxSplits || opt->workers < 0 || opt->sm_count < 0 ||
        opt->row_blocks < 0 || opt->row_blocks > mvr::kMaxRB)
        return W4A16_ERR_INVALID_ARG;
    if (opt->flags & ~(W4A16_FLAG_NO_PDL | W4A16_FLAG_STATIC_WEIGHTS | W4A16_FLAG_TEST_DROP_COPY))
        return W4A16_ERR_INVALID_ARG;
    return W4A16_OK;
}

// ------------------------------------------------------------------ planning

// Ring depth and scale/bias slab slots of the matvec for G groups: two slab
// slots (the next tile's scales load while this one's are in use) and as many
// stages as fit; one slot, then none (scales read from global memory), when
// two slots would leave fewer than kMatvecMinStages stages.
void matvec_smem_plan(int64_t G, int *stages, int *slots, long long *bytes) {
    auto fit = [&](int nslots) {
        for (int st = kMatvecMaxStages; st >= kMatvecMinStages; --st)
            if (mv::smem_bytes(st, nslots, G) <= kMatvecBudget) return st;
        return 0;
    };
    int st = 0, sl = 0;
    for (sl = 2; sl >= 0; --sl)
        if ((st = fit(sl))) break;
    if (sl < 0) sl = 0;
    *stages = st;
    *slots = sl;
    *bytes = mv::smem_bytes(st, sl, G);
}

// Persistent CTAs of the matvec.  A CTA holds most of an SM's shared memory, so the next
// kernel of the stream (programmatic dependent launch) can only start streaming its
// weights on SMs this one leaves free; and every tile split over several CTAs costs a
// fix-up.  Measured on B200 with back-to-back calls: k/v 2560->1024 (80 units) is
// fastest with 40 CTAs, q/o (320 units) with about 120, gate/up/down (760 units) with
// about 128, and the 151936-row vocabulary projection with every SM.
int64_t default_matvec_workers(int64_t units, int sms) {
    const int64_t most = (int64_t(sms) * 82) / 100, more = (int64_t(sms) * 87) / 100;
    if (units < 2 * most) return std::max<int64_t>(1, (units + 1) / 2);
    if (units < 4 * int64_t(sms)) return most;
    if (units < 16 * int64_t(sms)) return more;
    return sms;
}

void plan_matvec(int64_t M, int64_t N, int64_t K, int sms, const w4a16_options *opt, w4a16_plan_info *pl) {
    (void)M;
    const int64_t G = K / 128;
    int stages = 0, slots = 0;
    long long smem = 0;
    matvec_smem_plan(G, &stages, &slots, &smem);
    const int64_t tiles = (N + mv::kRows - 1) / mv::kRows;
    const int64_t units = tiles * G;
    int64_t workers = (opt && opt->workers > 0) ? opt->workers : default_matvec_workers(units, sms);
    workers = std::max<int64_t>(1, std::min<int64_t>(workers, units));
    std::memset(pl, 0, sizeof(*pl));
    pl->path = W4A16_PATH_MATVEC;
    pl->splits = 1;
    pl->grid_x = static_cast<int32_t>(workers);
    pl->grid_y = pl->grid_z = 1;
    pl->block = mv::kThreads;
    pl->smem_bytes = static_cast<int32_t>(smem);
    pl->cluster = 1;
    pl->tiles = tiles;
    pl->units = units;
    pl->workspace_bytes = int64_t(workers) * mv::kPartialFloats * 4 + std::max<int64_t>(tiles, kMinTickets) * 4;
}

// Tensor-core GEMM: output tiles of 256 weight rows x 128 x rows, each computed by a
// CTA pair; K split into `splits` contiguous runs of 128-groups (forced by the
// options, else chosen to fill the SMs, at most max_splits); the splits of a tile form
// one cluster of 2 x splits CTAs.
void plan_gemm(int64_t M, int64_t N, int64_t K, int sms, int max_splits, const w4a16_options *opt,
               w4a16_plan_info *pl) {
    const int64_t G = K / 128;
    const int64_t tm = (M + gm::BM - 1) / gm::BM, tn = (N + gm::kPairRows - 1) / gm::kPairRows;
    int64_t splits = 1;
    if (opt && opt->splits > 0) {
        splits = opt->splits;
    } else {
        // split K only when the tile pairs leave SMs idle
        const int64_t ctas = 2 * tm * tn;
        if (ctas < sms) splits = std::min<int64_t>(sms / ctas, max_splits);
        // clusters of more than 8 CTAs: only a few fit on the device at once (measured: 10
        // clusters of 14 and 8 of 16 ran in two waves, slower than the same tiles split in 4),
        // so more than 4 splits only while the whole grid stays within half of the SMs
        if (splits > 4 && ctas * splits > sms / 2) splits = 4;
        splits = std::min<int64_t>(splits, G / 2 > 0 ? G / 2 : 1);   // at least two groups per split
    }
    splits = std::max<int64_t>(1, std::min<int64_t>(splits, G));
    std::memset(pl, 0, sizeof(*pl));
    pl->path = W4A16_PATH_GEMM;
    pl->splits = static_cast<int32_t>(splits);
    pl->grid_x = static_cast<int32_t>(2 * splits);   // pairs of the splits of a tile: one cluster
    if (splits == 1) {
        // persistent: one CTA pair per two SMs, each looping over tiles
        pl->grid_y = static_cast<int32_t>(std::max<int64_t>(1, std::min<int64_t>(tm * tn, sms / 2)));
        pl->grid_z = 1;
    } else {
        pl->grid_y = static_cast<int32_t>(tn);
        pl->grid_z = static_cast<int32_t>(tm);
    }
    pl->block = gm::kThreads;
    pl->smem_bytes = gm::smem_bytes(static_cast<int>(G));
    pl->cluster = static_cast<int32_t>(2 * splits);
    pl->tiles = tm * tn;
    pl->units = tm * tn * G;
    pl->workspace_bytes = (M + N) * gm::xs_cols(static_cast<int>(G)) * 2;   // bias-step operands
}

// Row-block matvec: clusters of S CTAs share blocks of 8 whole weight rows ("half blocks",
// MMA row blocks of 16 rows, the last one half used for an odd count), each CTA of a cluster
// a contiguous run of ceil(G / S) or floor(G / S) groups.  The half blocks are spread evenly
// over at most SMs / S clusters, and the grid is padded with empty clusters to one CTA per
// SM: every call then holds exactly one CTA on each SM, so the next call's CTAs (resident
// beside it, fetching their weights) land one per SM too and no SM computes two CTAs of the
// same call.  The K split is the smallest S (1, 2, 4) whose layout fits and leaves every
// compute warp at least kRowsMinUnits units (16 rows x one group), else 2 if it fits, else the
// smallest that fits: measured on B200 in a back-to-back stream of the seven Qwen3-4B decode
// projections, a split pays for its exchange of partial sums (distributed shared memory) only
// when the warps have little work (k/v: 2.5 units per warp without a split) or when nothing
// smaller fits (the 9728-deep projection); clusters of four pack badly beside the next call's
// CTAs.  A CTA's shared memory leaves room for the next call's.
constexpr int kRowsMinUnits = 4;

struct RowsChoice {
    int hb = 0, splits = 0;    // half blocks of the fullest cluster, K splits
    int64_t clusters = 0;      // clusters with rows
    int64_t grid = 0;          // CTAs launched (clusters with rows, padded)
};

bool rows_choose(int64_t M, int64_t N, int64_t K, int sms, const w4a16_options *opt, RowsChoice *out,
                 bool gated = false) {
    (void)M;
    // gated: the unit of the split is a block of 16 rows (a gate half and its up half)
    const int64_t unit = gated ? 2 : 1;
    const int64_t NH = (N + 7) / 8, NU = NH / unit, G = K / 128;
    const int req_rb = opt ? opt->row_blocks : 0, req_s = opt ? opt->splits : 0;
    const int order[3] = {1, 2, 4};
    RowsChoice fits[3];
    int64_t units[3] = {0, 0, 0};
    int nfit = 0;
    for (int i = 0; i < 3; ++i) {
        const int s = req_s ? (i == 0 ? req_s : 0) : order[i];
        if (s == 0 || s > G) continue;
        const int64_t gcl = (G + s - 1) / s;
        const int64_t slots = std::max<int64_t>(1, sms / s);      // clusters that fit one CTA per SM
        const int64_t clusters = req_rb ? (NH + 2 * req_rb - 1) / (2 * req_rb) : std::min<int64_t>(slots, NU);
        const int64_t hb = unit * ((NU + clusters - 1) / clusters);
        if (mvr::rbs_of(static_cast<int>(std::min<int64_t>(hb, 1 << 20))) > mvr::kMaxRB) continue;
        if (mvr::smem_bytes(static_cast<int>(hb), static_cast<int>(std::min<int64_t>(gcl, 1 << 20)), s) > mvr::kBudget)
            continue;
        const int64_t grid = std::max(clusters, slots) * s;
        if (grid > (int64_t(1) << 31) - 1) continue;
        fits[nfit].hb = static_cast<int>(hb);
        fits[nfit].splits = s;
        fits[nfit].clusters = clusters;
        fits[nfit].grid = grid;
        units[nfit] = mvr::rbs_of(static_cast<int>(hb)) * gcl / mvr::kWarps;   // units per warp
        ++nfit;
    }
    if (nfit == 0) return false;
    // the smallest split that leaves the warps enough work; if none does, two (when it fits)
    int pick = -1;
    for (int i = 0; i < nfit && pick < 0; ++i)
        if (units[i] >= kRowsMinUnits) pick = i;
    for (int i = 0; i < nfit && pick < 0; ++i)
        if (fits[i].splits == 2) pick = i;
    if (pick < 0) pick = 0;
    *out = fits[pick];
    return true;
}

void plan_rows(int64_t N, int64_t K, const RowsChoice &c, w4a16_plan_info *pl, int64_t M = 1) {
    const int64_t G = K / 128;
    std::memset(pl, 0, sizeof(*pl));
    pl->slices = static_cast<int32_t>(std::max<int64_t>(1, (M + mvr::kMaxM - 1) / mvr::kMaxM));
    pl->path = W4A16_PATH_MATVEC_ROWS;
    pl->splits = c.splits;
    pl->grid_x = static_cast<int32_t>(c.grid);
    pl->grid_y = pl->grid_z = 1;
    pl->block = mvr::kThreads;
    pl->smem_bytes = static_cast<int32_t>(mvr::smem_bytes(c.hb, static_cast<int>((G + c.splits - 1) / c.splits), c.splits));
    pl->cluster = c.splits;
    pl->tiles = c.clusters;          // clusters with rows
    pl->units = (N + 7) / 8;         // 8-row half blocks
    pl->row_blocks = mvr::rbs_of(c.hb);   // MMA row blocks of 16 rows of the fullest cluster
    pl->workspace_bytes = 0;
}

// The automatic choice for 8 < M <= 32 (measured on B200, back-to-back calls of the Qwen3-4B
// projections): two slices of the row-block matvec beat the GEMM on every projection.
bool skinny_prefers_rows(int64_t M, int64_t N, int64_t K) {
    (void)N;
    (void)K;
    return (M + mvr::kMaxM - 1) / mvr::kMaxM <= 2;
}

// max_splits: the GEMM's largest K split on this device (forced splits above it are refused)
int plan(int64_t M, int64_t N, int64_t K, const w4a16_options *opt, int sms, int max_splits, w4a16_plan_info *pl) {
    int path = 0;
    int rc = choose_path(M, opt, &path);
    if (rc) return rc;
    const int req = opt ? opt->path : W4A16_PATH_AUTO;
    // 8 < M <= 32 on the automatic path: slices of the row-block matvec where the measured
    // crossover against the GEMM (whose tiles pad M to 128) says so
    const bool skinny = req == W4A16_PATH_AUTO && M > mvr::kMaxM && M <= kSkinnyMaxM &&
                        !(opt && (opt->splits > 0 || opt->workers > 0)) && skinny_prefers_rows(M, N, K);
    RowsChoice rc_rows;
    const bool rows_fit = path == W4A16_PATH_MATVEC_ROWS || path == W4A16_PATH_MATVEC || skinny
                              ? rows_choose(M, N, K, sms, opt, &rc_rows) : false;
    if (path == W4A16_PATH_MATVEC_ROWS && !rows_fit) return W4A16_ERR_UNSUPPORTED;
    if (path == W4A16_PATH_MATVEC && req == W4A16_PATH_AUTO && !(opt && opt->workers > 0) && rows_fit)
        path = W4A16_PATH_MATVEC_ROWS;
    if (skinny && rows_fit) path = W4A16_PATH_MATVEC_ROWS;
    if (path == W4A16_PATH_MATVEC_ROWS) {
        plan_rows(N, K, rc_rows, pl, M);
        return W4A16_OK;
    }
    if (path == W4A16_PATH_MATVEC) {
        plan_matvec(M, N, K, sms, opt, pl);
        return W4A16_OK;
    }
    if ((N + gm::kPairRows - 1) / gm::kPairRows > 65535 || (M + gm::BM - 1) / gm::BM > 65535 ||
        K / 128 > gm::kMaxGroups)
        return W4A16_ERR_UNSUPPORTED;
    if (opt && opt->splits > max_splits) return W4A16_ERR_UNSUPPORTED;
    plan_gemm(M, N, K, sms, max_splits, opt, pl);
    return W4A16_OK;
}

// ------------------------------------------------------------------ launches

int encode_2d(DeviceInfo *d, CUtensorMap *map, CUtensorMapDataType type, const void *base, uint64_t inner,
              uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
              CUtensorMapSwizzle swizzle) {
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = d->encode(map, type, 2, const_cast<void *>(base), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        g_last_cuda_error.store(static_cast<int>(r));
        return W4A16_ERR_CUDA;
    }
    return W4A16_OK;
}

template <int RB>
cudaError_t rows_launch_rb(const cudaLaunchConfig_t &cfg, const CUtensorMap &tm_hi, const CUtensorMap &tm_lo,
                           const mvr::Params &kp) {
    return cudaLaunchKernelEx(&cfg, mvr::rows_kernel<RB>, tm_hi, tm_lo, kp);
}

int launch_rows(DeviceInfo *d, const Problem &p, const w4a16_plan_info &pl, void *stream, bool pdl,
                bool static_weights, bool test_drop_copy, bool gated = false, int64_t ldy = 0) {
    const int G = static_cast<int>(p.K / 128);
    const int rb = pl.row_blocks, S = pl.splits;
    if (rb < 1 || rb > mvr::kMaxRB || S < 1 || S > mvr::kMaxSplits) return W4A16_ERR_INVALID_ARG;
    const int64_t NH = (p.N + 7) / 8;
    const int64_t unit = gated ? 2 : 1, NU = NH / unit;
    const int clusters = static_cast<int>(pl.tiles);
    const int hb_lo = static_cast<int>(unit * (NU / clusters)), hb_hi = static_cast<int>(unit * ((NU + clusters - 1) / clusters));
    if (mvr::rbs_of(hb_hi) != rb) return W4A16_ERR_INVALID_ARG;
    CUtensorMap tm_hi, tm_lo;
    // codes: [N, K/8] uint32, boxes of one group (16 words = 64 B) x the cluster's rows (8 hb_hi,
    // or 8 hb_lo for the clusters with one half block less), no swizzle (a quarter warp reads
    // two 64-byte rows: 8 distinct 16-byte bank groups)
    int rc = encode_2d(d, &tm_hi, CU_TENSOR_MAP_DATA_TYPE_UINT32, p.wq, p.K / 8, p.N, p.K / 2, 16,
                       static_cast<uint32_t>(8 * hb_hi), CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc) return rc;
    rc = encode_2d(d, &tm_lo, CU_TENSOR_MAP_DATA_TYPE_UINT32, p.wq, p.K / 8, p.N, p.K / 2, 16,
                   static_cast<uint32_t>(8 * hb_lo), CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc) return rc;
    mvr::Params kp;
    kp.x = static_cast<const uint16_t *>(p.x);
    kp.wq = p.wq;
    kp.scales = static_cast<const uint16_t *>(p.scales);
    kp.biases = static_cast<const uint16_t *>(p.biases);
    kp.y = static_cast<uint16_t *>(p.y);
    kp.M = static_cast<int>(p.M);
    kp.N = static_cast<int>(p.N);
    kp.K = static_cast<int>(p.K);
    kp.G = G;
    kp.splits = S;
    kp.gcl = (G + S - 1) / S;
    kp.nh = static_cast<int>(NH);
    kp.clusters = clusters;
    kp.hb_lo = hb_lo;
    kp.hb_hi = hb_hi;
    kp.static_weights = static_weights ? 1 : 0;
    kp.test_drop_copy = test_drop_copy ? 1 : 0;
    kp.gated = gated ? 1 : 0;
    kp.ldy = ldy > 0 ? ldy : p.N / 2;
    kp.wait_ns = test_drop_copy ? 200000ull : kWaitTimeoutNs;
    // every CTA prefetches an equal 16-byte-aligned share of x into L2 before the wait
    const long long xbytes = p.M * p.K * 2;
    kp.x_chunk = std::min<long long>(((xbytes + pl.grid_x - 1) / pl.grid_x + 15) / 16 * 16, 65536);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.grid_x, 1, 1);
    cfg.blockDim = dim3(pl.block, 1, 1);
    cfg.dynamicSmemBytes = pl.smem_bytes;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (S > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = S;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    cudaError_t e = cudaErrorInvalidValue;
    switch (rb) {
        case 1: e = rows_launch_rb<1>(cfg, tm_hi, tm_lo, kp); break;
        case 2: e = rows_launch_rb<2>(cfg, tm_hi, tm_lo, kp); break;
        case 3: e = rows_launch_rb<3>(cfg, tm_hi, tm_lo, kp); break;
        case 4: e = rows_launch_rb<4>(cfg, tm_hi, tm_lo, kp); break;
        case 5: e = rows_launch_rb<5>(cfg, tm_hi, tm_lo, kp); break;
    }
    return e == cudaSuccess ? W4A16_OK : cuda_fail(e);
}

int launch_matvec(DeviceInfo *d, Workspace *ws, const Problem &p, const w4a16_plan_info &pl, void *stream,
                  bool pdl, bool static_weights) {
    CUtensorMap tm_w, tm_x;
    // codes: [N, K/8] uint32, box of 2 groups (32 words = 128 B) x 128 rows, 128-byte swizzle
    int rc = encode_2d(d, &tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT32, p.wq, p.K / 8, p.N, p.K / 2,
                       16 * mv::kGroupsPerStage, mv::kRows, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
    // x viewed as [M, K/2] pairs of BF16: box of 256 BF16 (128 pairs) x M rows
    rc = encode_2d(d, &tm_x, CU_TENSOR_MAP_DATA_TYPE_UINT32, p.x, p.K / 2, p.M, p.K * 2, mv::kXCols / 2,
                   static_cast<uint32_t>(p.M), CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc) return rc;
    mv::Params kp;
    kp.x = static_cast<const uint16_t *>(p.x);
    kp.wq = p.wq;
    kp.scales = static_cast<const uint16_t *>(p.scales);
    kp.biases = static_cast<const uint16_t *>(p.biases);
    kp.y = static_cast<uint16_t *>(p.y);
    kp.partials = ws->partials;
    kp.flags = ws->tickets;
    kp.M = static_cast<int>(p.M);
    kp.N = static_cast<int>(p.N);
    kp.G = static_cast<int>(p.K / 128);
    kp.tiles = static_cast<int>(pl.tiles);
    kp.units = pl.units;
    kp.workers = pl.grid_x;
    long long smem = 0;
    matvec_smem_plan(kp.G, &kp.stages, &kp.slab_slots, &smem);
    kp.slab_array_bytes = static_cast<int>(mv::slab_array_bytes(kp.G));
    kp.opts = static_weights ? mv::kFlagStaticWeights : 0;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.grid_x, 1, 1);
    cfg.blockDim = dim3(pl.block, 1, 1);
    cfg.dynamicSmemBytes = pl.smem_bytes;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    cudaError_t e = cudaLaunchKernelEx(&cfg, mv::matvec_kernel, tm_w, tm_x, kp);
    return e == cudaSuccess ? W4A16_OK : cuda_fail(e);
}

int launch_gemm(DeviceInfo *d, Workspace *ws, const Problem &p, const w4a16_plan_info &pl, void *stream,
                bool pdl, bool static_weights) {
    const int G = static_cast<int>(p.K / 128);
    const int Kx = gm::xs_cols(G);
    CUtensorMap tm_x, tm_xs, tm_w, tm_y;
    // x: [M, K] BF16, boxes of 64 columns x 64 rows (one CTA's half of the x rows of a
    // tile), 128-byte swizzle (K-major B operand)
    int rc = encode_2d(d, &tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.x, p.K, p.M, p.K * 2, 64, gm::kXRows,
                       CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
    // group sums of x: [M, Kx] BF16, same boxes
    rc = encode_2d(d, &tm_xs, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, ws->xs, Kx, p.M, uint64_t(Kx) * 2, 64, gm::kXRows,
                   CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
    // codes: [N, K/8] uint32, boxes of one group (16 words = 64 B) x 128 rows, 64-byte swizzle
    rc = encode_2d(d, &tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT32, p.wq, p.K / 8, p.N, p.K / 2, 16, gm::BN,
                   CU_TENSOR_MAP_SWIZZLE_64B);
    if (rc) return rc;
    // y: [M, N] BF16, one box per CTA tile (128 weight rows = columns of y, 128 x rows); only
    // when its rows are 16-byte multiples (TMA strides), else the kernel stores element-wise
    const bool tma_store = (p.N * 2) % 16 == 0;
    if (tma_store) {
        rc = encode_2d(d, &tm_y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.y, p.N, p.M, p.N * 2, gm::BN, gm::BM,
                       CU_TENSOR_MAP_SWIZZLE_NONE);
        if (rc) return rc;
    } else {
        std::memset(&tm_y, 0, sizeof(tm_y));
    }
    cudaLaunchAttribute pdl_attr;
    pdl_attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl_attr.val.programmaticStreamSerializationAllowed = 1;

    // 1. bias-step operands: group sums of x and the matching weight coefficients
    uint16_t *bc = ws->xs + size_t(p.M) * Kx;
    {
        // threads: 16 per (x row, group), one per (weight row, group); the kernel loops
        const long long items = std::max<long long>(p.M * G * 16, p.N * G);
        const long long blocks = std::min<long long>((items + 255) / 256, static_cast<long long>(d->sms) * 8);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(std::max<long long>(blocks, 1)), 1, 1);
        cfg.blockDim = dim3(256, 1, 1);
        cfg.stream = static_cast<cudaStream_t>(stream);
        cfg.attrs = &pdl_attr;
        cfg.numAttrs = pdl ? 1 : 0;
        cudaError_t e = cudaLaunchKernelEx(&cfg, gm::prep_kernel, static_cast<const uint16_t *>(p.x),
                                           static_cast<const uint16_t *>(p.scales),
                                           static_cast<const uint16_t *>(p.biases), ws->xs, bc,
                                           static_cast<int>(p.M), static_cast<int>(p.N), G, Kx);
        if (e != cudaSuccess) return cuda_fail(e);
    }
    // 2. the GEMM (programmatic dependent launch on the group sums)
    gm::Params kp;
    kp.x = static_cast<const uint16_t *>(p.x);
    kp.wq = p.wq;
    kp.scales = static_cast<const uint16_t *>(p.scales);
    kp.biases = static_cast<const uint16_t *>(p.biases);
    kp.bc = bc;
    kp.y = static_cast<uint16_t *>(p.y);
    kp.M = static_cast<int>(p.M);
    kp.N = static_cast<int>(p.N);
    kp.G = G;
    kp.Kx = Kx;
    kp.splits = pl.splits;
    kp.tiles = pl.tiles;
    kp.tiles_n = static_cast<int>((p.N + gm::kPairRows - 1) / gm::kPairRows);
    kp.static_weights = static_weights ? 1 : 0;
    kp.tma_store = tma_store ? 1 : 0;
    cudaLaunchConfig_t cfg = {};
    // a persistent grid is capped at the pairs the device holds at once
    const int grid_y = pl.splits == 1 ? std::max(1, std::min(pl.grid_y, d->gemm_clusters)) : pl.grid_y;
    cfg.gridDim = dim3(pl.grid_x, grid_y, pl.grid_z);
    cfg.blockDim = dim3(pl.block, 1, 1);
    cfg.dynamicSmemBytes = pl.smem_bytes;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = pl.cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1] = pdl_attr;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, gm::gemm_kernel, tm_x, tm_xs, tm_w, tm_y, kp);
    return e == cudaSuccess ? W4A16_OK : cuda_fail(e);
}

int matmul_impl(const Problem &p, void *stream, const w4a16_options *opt) {
    int rc = validate(p);
    if (rc) return rc;
    rc = validate_options(opt);
    if (rc) return rc;
    int path = 0;
    rc = choose_path(p.M, opt, &path);
    if (rc) return rc;
    if (p.M == 0 || p.N == 0) return W4A16_OK;

    int dev = 0;
    rc = current_device(&dev);
    if (rc) return rc;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceInfo *d = nullptr;
    rc = device_setup(dev, &d);
    if (rc) return rc;
    if (p.K == 0) {   // an empty sum: every output is +0
        cudaError_t e = cudaMemsetAsync(p.y, 0, size_t(p.M) * p.N * 2, static_cast<cudaStream_t>(stream));
        return e == cudaSuccess ? W4A16_OK : cuda_fail(e);
    }
    w4a16_plan_info pl;
    rc = plan(p.M, p.N, p.K, opt, d->sms, d->gemm_max_splits, &pl);
    if (rc) return rc;
    const bool pdl = !(opt && (opt->flags & W4A16_FLAG_NO_PDL));
    const bool static_weights = opt && (opt->flags & W4A16_FLAG_STATIC_WEIGHTS);
    const bool drop = opt && (opt->flags & W4A16_FLAG_TEST_DROP_COPY);
    if (drop && (pl.path != W4A16_PATH_MATVEC_ROWS || p.M > mvr::kMaxM)) return W4A16_ERR_INVALID_ARG;
    if (pl.path == W4A16_PATH_MATVEC_ROWS) {
        // one launch per slice of 8 x rows; each slice after the first reads the weights the one
        // before has just brought into L2, and fetches them before its dependency wait
        for (int64_t m0 = 0; m0 < p.M; m0 += mvr::kMaxM) {
            const int64_t mi = std::min<int64_t>(mvr::kMaxM, p.M - m0);
            const Problem sub{static_cast<const uint16_t *>(p.x) + m0 * p.K, p.wq, p.scales, p.biases,
                              static_cast<uint16_t *>(p.y) + m0 * p.N, mi, p.N, p.K};
            rc = launch_rows(d, sub, pl, stream, pdl, pdl && (static_weights || m0 > 0), drop);
            if (rc) return rc;
        }
        return W4A16_OK;
    }
    if (pl.path == W4A16_PATH_MATVEC) {
        Workspace *ws = nullptr;
        rc = workspace_get(dev, stream, size_t(pl.grid_x) * mv::kPartialFloats, pl.tiles, &ws);
        if (rc) return rc;
        return launch_matvec(d, ws, p, pl, stream, pdl, pdl && static_weights);
    }
    if (!d->gemm_ok) return W4A16_ERR_UNSUPPORTED;
    Workspace *ws = nullptr;
    rc = workspace_xs(dev, stream, size_t(p.M + p.N) * gm::xs_cols(static_cast<int>(p.K / 128)), &ws);
    if (rc) return rc;
    return launch_gemm(d, ws, p, pl, stream, pdl, pdl && static_weights);
}

// ------------------------------------------------------------------ 2- and 8-bit codes

constexpr int64_t kBitsMaxM = 32;   // slices of 8 x rows, as the 4-bit row-block path

template <int BITS>
int launch_nbit(const Problem &p, void *stream) {
    nb::Params kp;
    kp.x = static_cast<const uint16_t *>(p.x);
    kp.wq = p.wq;
    kp.scales = static_cast<const uint16_t *>(p.scales);
    kp.biases = static_cast<const uint16_t *>(p.biases);
    kp.y = static_cast<uint16_t *>(p.y);
    kp.M = static_cast<int>(p.M);
    kp.N = static_cast<int>(p.N);
    kp.K = static_cast<int>(p.K);
    kp.G = static_cast<int>(p.K / 128);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>((p.N + nb::rows_per_cta<BITS>() - 1) / nb::rows_per_cta<BITS>()), 1, 1);
    cfg.blockDim = dim3(nb::kThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, nb::nbit_kernel<BITS>, kp);
    return e == cudaSuccess ? W4A16_OK : cuda_fail(e);
}

int matmul_bits_impl(const Problem &p, int bits, void *stream) {
    if (bits == 4) return matmul_impl(p, stream, nullptr);
    if (p.M < 0 || p.N < 0 || p.K < 0) return W4A16_ERR_INVALID_ARG;
    if (bits != 2 && bits != 8) return W4A16_ERR_UNSUPPORTED;
    if (p.K % 128 != 0 || p.M > kBitsMaxM || p.N >= (int64_t(1) << 31) || p.K >= (int64_t(1) << 31))
        return W4A16_ERR_UNSUPPORTED;
    if (p.M == 0 || p.N == 0) return W4A16_OK;
    if (!p.y) return W4A16_ERR_INVALID_ARG;
    if (!aligned16(p.y)) return W4A16_ERR_MISALIGNED;
    if (p.K > 0) {
        if (!p.x || !p.wq || !p.scales || !p.biases) return W4A16_ERR_INVALID_ARG;
        if (!aligned16(p.x) || !aligned16(p.wq) || !aligned16(p.scales) || !aligned16(p.biases))
            return W4A16_ERR_MISALIGNED;
        const size_t ny = size_t(p.M) * p.N * 2;
        if (overlaps(p.y, ny, p.x, size_t(p.M) * p.K * 2) || overlaps(p.y, ny, p.wq, size_t(p.N) * p.K * bits / 8) ||
            overlaps(p.y, ny, p.scales, size_t(p.N) * (p.K / 128) * 2) ||
            overlaps(p.y, ny, p.biases, size_t(p.N) * (p.K / 128) * 2))
            return W4A16_ERR_INVALID_ARG;
    }
    int dev = 0;
    int rc = current_device(&dev);
    if (rc) return rc;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceInfo *d = nullptr;
    rc = device_setup(dev, &d);
    if (rc) return rc;
    if (p.K == 0) {   // an empty sum: every output is +0
        cudaError_t e = cudaMemsetAsync(p.y, 0, size_t(p.M) * p.N * 2, static_cast<cudaStream_t>(stream));
        return e == cudaSuccess ? W4A16_OK : cuda_fail(e);
    }
    for (int64_t m0 = 0; m0 < p.M; m0 += nb::kMaxM) {
        const Problem sub{static_cast<const uint16_t *>(p.x) + m0 * p.K, p.wq, p.scales, p.biases,
                          static_cast<uint16_t *>(p.y) + m0 * p.N, std::min<int64_t>(nb::kMaxM, p.M - m0), p.N, p.K};
        rc = bits == 2 ? launch_nbit<2>(sub, stream) : launch_nbit<8>(sub, stream);
        if (rc) return rc;
    }
    return W4A16_OK;
}

// ------------------------------------------------------------------ allocation-free matvec

// Scratch of w4a16_matvec_noalloc: a region for the FP32 partials of up to
// kNoAllocWorkers CTAs (8 KB each, of which the kernel uses the first
// kPartialFloats), then one flag per 128 rows for up to W4A16_NOALLOC_MAX_N rows.
constexpr int kNoAllocWorkers = 160;
constexpr size_t kNoAllocPartialBytes = size_t(kNoAllocWorkers) * 8192;
static_assert(mv::kPartialFloats * sizeof(float) <= 8192, "partial slot exceeds its scratch share");
constexpr int64_t kNoAllocTiles = W4A16_NOALLOC_MAX_N / 128;   // flag slots: at least one per tile
static_assert(mv::kRows >= 128, "flag region sized for tiles of 128 rows or more");
static_assert(kNoAllocPartialBytes + kNoAllocTiles * sizeof(int) == W4A16_NOALLOC_SCRATCH_BYTES,
              "header and scratch layout disagree");
static __device__ __align__(256) unsigned char g_noalloc_scratch[W4A16_NOALLOC_SCRATCH_BYTES];

std::map<int, unsigned char *> g_noalloc_ptr;   // device address of the array, per device

int noalloc_matvec(const Problem &p, void *stream) {
    if (p.M < 0 || p.N < 0 || p.K < 0) return W4A16_ERR_INVALID_ARG;
    if (p.M > mv::kMaxM || p.N > W4A16_NOALLOC_MAX_N) return W4A16_ERR_UNSUPPORTED;   // beyond the scratch
    int rc = validate(p);
    if (rc) return rc;
    if (p.M == 0 || p.N == 0) return W4A16_OK;
    int dev = 0;
    rc = current_device(&dev);
    if (rc) return rc;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceInfo *d = nullptr;
    rc = device_setup(dev, &d);
    if (rc) return rc;
    if (p.K == 0) {
        cudaError_t e = cudaMemsetAsync(p.y, 0, size_t(p.M) * p.N * 2, static_cast<cudaStream_t>(stream));
        return e == cudaSuccess ? W4A16_OK : cuda_fail(e);
    }
    auto it = g_noalloc_ptr.find(dev);
    if (it == g_noalloc_ptr.end()) {
        // In host code the array's name is only a stand-in: look up its address on
        // this device (the current one) before handing it to a kernel.
        void *ptr = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess || !ptr) return cuda_fail(e);
        it = g_noalloc_ptr.emplace(dev, static_cast<unsigned char *>(ptr)).first;
    }
    w4a16_plan_info pl;
    w4a16_options opt = {};
    opt.path = W4A16_PATH_MATVEC;   // the stream-K kernel at its measured default CTA count
    plan_matvec(p.M, p.N, p.K, d->sms, &opt, &pl);
    if (pl.tiles > kNoAllocTiles || pl.grid_x > kNoAllocWorkers) return W4A16_ERR_UNSUPPORTED;
    Workspace ws;
    ws.partials = reinterpret_cast<float *>(it->second);
    ws.partial_floats = kNoAllocPartialBytes / sizeof(float);
    ws.tickets = reinterpret_cast<int *>(it->second + kNoAllocPartialBytes);
    ws.ticket_count = kNoAllocTiles;
    // The flags of this call must start at zero whatever an earlier call left behind (a call
    // that finishes leaves them at zero, one that gave up on a wait may not).  The clearing is
    // stream-ordered work of its own, so this entry point's kernel never overlaps the end of
    // the preceding kernel of the stream.
    cudaError_t e = cudaMemsetAsync(ws.tickets, 0, size_t(pl.tiles) * sizeof(int), static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e);
    return launch_matvec(d, &ws, p, pl, stream, /*pdl=*/true, /*static_weights=*/false);
}

}  // namespace
}  // namespace w4a16

using namespace w4a16;

extern "C" {

int w4a16_matmul(const void *x, const uint32_t *wq, const void *scales, const void *biases, void *y, int64_t M,
                 int64_t N, int64_t K, void *stream) {
    return matmul_impl(Problem{x, wq, scales, biases, y, M, N, K}, stream, nullptr);
}

int w4a16_matmul_ex(const void *x, const uint32_t *wq, const void *scales, const void *biases, void *y, int64_t M,
                    int64_t N, int64_t K, void *stream, const w4a16_options *opt) {
    return matmul_impl(Problem{x, wq, scales, biases, y, M, N, K}, stream, opt);
}

int w4a16_matmul_last_rows(const void *x, const uint32_t *wq, const void *scales, const void *biases, void *y,
                           int64_t M, int64_t keep, int64_t N, int64_t K, void *stream) {
    if (M < 0 || keep < 0 || keep > M || K < 0) return W4A16_ERR_INVALID_ARG;
    if (keep == 0) keep = M;
    const char *xs = static_cast<const char *>(x);
    if (xs) xs += (M - keep) * K * 2;   // the last `keep` rows of x
    return matmul_impl(Problem{xs, wq, scales, biases, y, keep, N, K}, stream, nullptr);
}

int w4a16_plan(int64_t M, int64_t N, int64_t K, const w4a16_options *opt, w4a16_plan_info *out) {
    if (!out) return W4A16_ERR_INVALID_ARG;
    if (M < 0 || N < 0 || K < 0) return W4A16_ERR_INVALID_ARG;
    if (K % 128 != 0) return W4A16_ERR_UNSUPPORTED;
    int rc = validate_options(opt);
    if (rc) return rc;
    int sms = opt ? opt->sm_count : 0;
    if (sms <= 0) {
        int dev = 0;
        rc = current_device(&dev);
        if (rc) return rc;
        std::lock_guard<std::mutex> lock(g_mu);
        DeviceInfo *d = nullptr;
        rc = device_setup(dev, &d);
        if (rc) return rc;
        sms = d->sms;
    }
    if (M == 0 || N == 0 || K == 0) {
        std::memset(out, 0, sizeof(*out));
        int path = 0;
        rc = choose_path(M, opt, &path);
        out->path = path;
        return rc;
    }
    return plan(M, N, K, opt, sms, gm::kMaxSplits, out);
}

int w4a16_device_status(void *stream) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e);
    int status = 0;
    e = cudaMemcpyFromSymbol(&status, g_status, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e);
    if (status == 0) return W4A16_OK;
    // A kernel gave up: clear the word and the split bookkeeping of this device.
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_status, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e);
    int dev = 0;
    if (current_device(&dev)) return W4A16_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    for (auto &kv : g_workspaces) {
        if (kv.first.first != dev || !kv.second.tickets) continue;
        e = cudaMemset(kv.second.tickets, 0, kv.second.ticket_count * sizeof(int));
        if (e != cudaSuccess) return cuda_fail(e);
    }
    return W4A16_ERR_TIMEOUT;
}

void w4a16_release(void) {
    std::lock_guard<std::mutex> lock(g_mu);
    g_noalloc_ptr.clear();   // looked up again on the next call (a device reset may move the array)
    int cur = 0;
    cudaGetDevice(&cur);
    for (auto &kv : g_workspaces) {
        cudaSetDevice(kv.first.first);
        cudaDeviceSynchronize();
        cudaFree(kv.second.partials);
        cudaFree(kv.second.tickets);
        cudaFree(kv.second.xs);
    }
    g_workspaces.clear();
    cudaSetDevice(cur);
}

const char *w4a16_status_string(int status) {
    switch (status) {
        case W4A16_OK: return "ok";
        case W4A16_ERR_INVALID_ARG: return "invalid argument";
        case W4A16_ERR_UNSUPPORTED: return "unsupported size or option";
        case W4A16_ERR_MISALIGNED: return "pointer not 16-byte aligned";
        case W4A16_ERR_CUDA: return "CUDA call failed";
        case W4A16_ERR_NO_MEMORY: return "workspace allocation failed";
        case W4A16_ERR_DEVICE: return "device is not compute capability 10.0";
        case W4A16_ERR_TIMEOUT: return "a kernel abandoned a bounded wait";
        default: return "unknown status";
    }
}

int w4a16_last_cuda_error(void) { return g_last_cuda_error.load(); }

int w4a16_version(void) { return kVersion; }

int64_t w4a16_streamk_owner(int64_t units, int64_t workers, int64_t u) {
    if (units <= 0 || workers <= 0 || workers > units || u < 0 || u >= units) return -1;
    return mv::streamk_owner(units, workers, u);
}

int w4a16_matvec_noalloc(const void *x, const uint32_t *wq, const void *scales, const void *biases, void *y,
                         int64_t M, int64_t N, int64_t K, void *stream) {
    return noalloc_matvec(Problem{x, wq, scales, biases, y, M, N, K}, stream);
}

int w4a16_gate_up(const void *x, const uint32_t *wq, const void *scales, const void *biases, void *h, int64_t M,
                  int64_t N2, int64_t K, void *stream) {
    if (M < 0 || N2 < 0 || K < 0) return W4A16_ERR_INVALID_ARG;
    if (K % 128 != 0 || N2 % 8 != 0 || M > mvr::kMaxM || N2 >= (int64_t(1) << 30) || K >= (int64_t(1) << 31))
        return W4A16_ERR_UNSUPPORTED;
    if (M == 0 || N2 == 0) return W4A16_OK;
    if (!h) return W4A16_ERR_INVALID_ARG;
    if (!aligned16(h)) return W4A16_ERR_MISALIGNED;
    const int64_t N = 2 * N2;
    if (K == 0) {   // an empty sum: silu(0) * 0 = +0 everywhere
        cudaError_t e = cudaMemsetAsync(h, 0, size_t(M) * N2 * 2, static_cast<cudaStream_t>(stream));
        return e == cudaSuccess ? W4A16_OK : cuda_fail(e);
    }
    if (!x || !wq || !scales || !biases) return W4A16_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(wq) || !aligned16(scales) || !aligned16(biases)) return W4A16_ERR_MISALIGNED;
    const size_t nh = size_t(M) * N2 * 2;
    if (overlaps(h, nh, x, size_t(M) * K * 2) || overlaps(h, nh, wq, size_t(N) * K / 2) ||
        overlaps(h, nh, scales, size_t(N) * (K / 128) * 2) || overlaps(h, nh, biases, size_t(N) * (K / 128) * 2))
        return W4A16_ERR_INVALID_ARG;
    int dev = 0;
    int rc = current_device(&dev);
    if (rc) return rc;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceInfo *d = nullptr;
    rc = device_setup(dev, &d);
    if (rc) return rc;
    // A CTA holds all of its rows' codes: where the 2 N2 rows exceed what the SMs hold at once,
    // the outputs are cut into column slices of whole 16-row blocks, one launch each (the later
    // ones fetch their weights while the one before finishes).
    const int64_t nb = N2 / 8, G = K / 128;
    int64_t chunks = 0;
    RowsChoice c;
    for (int64_t t = 1; t <= 64 && t <= nb && !chunks; ++t)
        if (rows_choose(M, 16 * ((nb + t - 1) / t), K, d->sms, nullptr, &c, true)) chunks = t;
    if (!chunks) return W4A16_ERR_UNSUPPORTED;
    for (int64_t i = 0; i < chunks; ++i) {
        const int64_t b0 = i * nb / chunks, b1 = (i + 1) * nb / chunks, rows = 16 * (b1 - b0);
        if (rows == 0) continue;
        if (!rows_choose(M, rows, K, d->sms, nullptr, &c, true)) return W4A16_ERR_UNSUPPORTED;
        w4a16_plan_info pl;
        plan_rows(rows, K, c, &pl);
        const Problem sub{x, wq + 16 * b0 * (K / 8), static_cast<const uint16_t *>(scales) + 16 * b0 * G,
                          static_cast<const uint16_t *>(biases) + 16 * b0 * G, static_cast<uint16_t *>(h) + 8 * b0,
                          M, rows, K};
        rc = launch_rows(d, sub, pl, stream, true, i > 0, false, true, N2);
        if (rc) return rc;
    }
    return W4A16_OK;
}

int w4a16_matmul_bits(const void *x, const uint32_t *wq, const void *scales, const void *biases, void *y,
                      int64_t M, int64_t N, int64_t K, int32_t bits, void *stream) {
    return matmul_bits_impl(Problem{x, wq, scales, biases, y, M, N, K}, bits, stream);
}

int w4a16_quantize(const void *w, int32_t w_dtype, uint32_t *wq, void *scales, void *biases, int64_t N, int64_t K,
                   void *stream) {
    if (N < 0 || K < 0 || (w_dtype != W4A16_DTYPE_F32 && w_dtype != W4A16_DTYPE_BF16)) return W4A16_ERR_INVALID_ARG;
    if (K % 128 != 0 || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31)) return W4A16_ERR_UNSUPPORTED;
    if (N == 0 || K == 0) return W4A16_OK;
    if (!w || !wq || !scales || !biases) return W4A16_ERR_INVALID_ARG;
    if (!aligned16(w) || !aligned16(wq) || !aligned16(scales) || !aligned16(biases)) return W4A16_ERR_MISALIGNED;
    const size_t nw = size_t(N) * K * (w_dtype == W4A16_DTYPE_F32 ? 4 : 2);
    const size_t nq = size_t(N) * K / 2, ns = size_t(N) * (K / 128) * 2;
    if (overlaps(w, nw, wq, nq) || overlaps(w, nw, scales, ns) || overlaps(w, nw, biases, ns) ||
        overlaps(wq, nq, scales, ns) || overlaps(wq, nq, biases, ns) || overlaps(scales, ns, biases, ns))
        return W4A16_ERR_INVALID_ARG;
    int dev = 0;
    int rc = current_device(&dev);
    if (rc) return rc;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceInfo *d = nullptr;
    rc = device_setup(dev, &d);
    if (rc) return rc;
    // (row, group) pairs, four per warp, eight warps per CTA, at most eight CTAs per SM
    const int64_t pairs = N * (K / 128);
    const int64_t per_cta = int64_t(qz::kWarps) * qz::kPairsPerWarp;
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>((pairs + per_cta - 1) / per_cta, int64_t(d->sms) * 8));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (w_dtype == W4A16_DTYPE_BF16)
        qz::quantize_kernel<true><<<static_cast<unsigned>(grid), qz::kThreads, 0, st>>>(
            w, wq, static_cast<uint16_t *>(scales), static_cast<uint16_t *>(biases), N, static_cast<int>(K));
    else
        qz::quantize_kernel<false><<<static_cast<unsigned>(grid), qz::kThreads, 0, st>>>(
            w, wq, static_cast<uint16_t *>(scales), static_cast<uint16_t *>(biases), N, static_cast<int>(K));
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? W4A16_OK : cuda_fail(e);
}

}  // extern "C"
