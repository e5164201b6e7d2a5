/*
 * w4a16.h - C ABI of the B200 (sm_100a) W4A16 group-128 linear layer.
 *
 *     y[M,N] = x[M,K] . dequant(wq)^T,   dequant: w[n,k] = s[n,k/128] * q[n,k] + b[n,k/128]
 *
 * The operation is the quantised linear layer of tiny-llm "Week 2 Day 6:
 * SIMD-Matrix Prefill": 4-bit weights with group size 128, BF16 activations,
 * BF16 quantisation parameters and BF16 output, FP32 matrix accumulators
 * (introduction), one scale and one bias per 128 reduction values (Task 3), a
 * matvec schedule for M <= 8 and a tiled matrix schedule for M > 8 behind one
 * unchanged interface (Task 1), a split-K successor for under-filled grids
 * (Task 5), and last-row logits (Task 4).
 *
 * Data layout (all row-major, contiguous, DEVICE memory owned by the caller):
 *   x       bf16   [M, K]
 *   wq      uint32 [N, K/8]   code q[n,k] = (wq[n*(K/8) + k/8] >> (4*(k%8))) & 15
 *                             (eight 4-bit codes per word, k % 8 == 0 in bits 0-3)
 *   scales  bf16   [N, K/128]
 *   biases  bf16   [N, K/128]
 *   y       bf16   [M, N]     written; must not overlap any input
 * Every pointer must be 16-byte aligned.  K must be a multiple of 128.
 *
 * Numerics: products and sums in FP32, each 128-wide group's scale and bias
 * applied in FP32, one BF16 round-to-nearest-even per output.  The result
 * matches the plain FP32 definition to within one BF16 ulp (+1e-3 absolute);
 * the summation order differs from it.  Identical inputs and sizes give
 * bit-identical outputs on the same device model (no atomics decide the order
 * of any floating-point sum).
 *
 * Execution: work is enqueued on `stream` (a cudaStream_t; NULL = legacy
 * default stream) on the CURRENT device; calls return without synchronising.
 * No call allocates in steady state; the first call on a (device, stream)
 * pair allocates a small library-owned workspace (see w4a16_release), so
 * that first call must not happen during stream capture.  Calls on different
 * streams use different workspaces and may overlap.
 *
 * Errors: every entry point validates its arguments on the host and returns a
 * status code without launching anything when they are invalid.  Kernels
 * never trap: a kernel that gives up on a bounded wait records
 * W4A16_ERR_TIMEOUT in a device-side status word, which w4a16_device_status
 * reports.
 */
#ifndef W4A16_H
#define W4A16_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum w4a16_status_code {
    W4A16_OK = 0,
    W4A16_ERR_INVALID_ARG = 1,  /* null pointer with non-empty sizes, negative size, bad option  */
    W4A16_ERR_UNSUPPORTED = 2,  /* K % 128 != 0, or a size beyond the supported range            */
    W4A16_ERR_MISALIGNED = 3,   /* a pointer that is not 16-byte aligned                          */
    W4A16_ERR_CUDA = 4,         /* a CUDA runtime call failed (see w4a16_last_cuda_error)         */
    W4A16_ERR_NO_MEMORY = 5,    /* the library-owned workspace could not be allocated             */
    W4A16_ERR_DEVICE = 6,       /* the current device is not compute capability 10.0             */
    W4A16_ERR_TIMEOUT = 7       /* a kernel abandoned a bounded wait (from w4a16_device_status)   */
};

/* Kernel paths (w4a16_options.path, w4a16_plan_info.path). */
enum w4a16_path {
    W4A16_PATH_AUTO = 0,        /* M <= 8: matvec; M > 8: tensor-core GEMM (Task 1 dispatch rule) */
    W4A16_PATH_MATVEC = 1,      /* weight-streaming matvec, M <= 8 only                           */
    W4A16_PATH_GEMM = 2,        /* tcgen05 tensor-core GEMM, any M >= 1                            */
    W4A16_PATH_MATVEC_ROWS = 3  /* row-block matvec, M <= 32: a CTA holds all codes, scales and biases
                                   of 16 x row_blocks weight rows over a K range in shared memory
                                   (the whole of K, or 1/splits of it with the splits of a row range
                                   added in a thread-block cluster); two CTAs fit on an SM.  Only
                                   where such a split fits (else W4A16_ERR_UNSUPPORTED).  For
                                   8 < M <= 32 it runs once per slice of 8 x rows (ceil(M / 8)
                                   launches; the later ones find the weights in L2 and fetch them
                                   while the one before finishes).
                                   W4A16_PATH_AUTO takes it for M <= 8 when it fits and no worker
                                   count is given, the stream-K matvec (W4A16_PATH_MATVEC) otherwise;
                                   for 8 < M <= 32 it takes it where the measured crossover against
                                   the GEMM says so (w4a16_plan reports the choice)             */
};

/*
 * y = x . dequant(wq)^T.  Arguments as in the layout block above.
 * M == 0 or N == 0: returns W4A16_OK and launches nothing.
 * Sizes: 0 <= M, N < 2^31, 0 <= K < 2^31 with K % 128 == 0; on the tensor-core
 * GEMM path (M > 8, or forced) also K <= 32768, else W4A16_ERR_UNSUPPORTED.
 * Ownership: all buffers belong to the caller and must stay valid until the
 * enqueued work completes.
 */
int w4a16_matmul(const void *x, const uint32_t *wq, const void *scales,
                 const void *biases, void *y, int64_t M, int64_t N, int64_t K,
                 void *stream);

/*
 * Last-rows projection ("logits_to_keep", tiny-llm "Week 2 Day 6: SIMD-Matrix
 * Prefill", Task 4): y[keep, N] = x[M-keep : M, :] . dequant(wq)^T.
 * keep == 0 keeps every row (y is [M, N]); 0 < keep <= M keeps the last keep
 * rows.  No kernel of its own: the rows are selected by offsetting x, then
 * w4a16_matmul runs with M' = keep.  keep > M or keep < 0: W4A16_ERR_INVALID_ARG.
 */
int w4a16_matmul_last_rows(const void *x, const uint32_t *wq, const void *scales,
                           const void *biases, void *y, int64_t M, int64_t keep,
                           int64_t N, int64_t K, void *stream);

/* Options for the explicit entry points; zero-initialised means "automatic". */
typedef struct w4a16_options {
    int32_t path;       /* enum w4a16_path                                                  */
    int32_t splits;     /* K splits, each a contiguous run of 128-groups; 0 = auto.  GEMM:
                           1..8 (a cluster of 2 x splits CTAs; above 4 only where the device
                           holds clusters of 16 CTAs, else W4A16_ERR_UNSUPPORTED); row-block
                           matvec: 1..4                                                      */
    int32_t workers;    /* stream-K matvec: persistent CTAs sharing the (row-tile x group) units;
                           0 = auto                                                          */
    int32_t sm_count;   /* w4a16_plan only: SM count to plan for; 0 = query the current device */
    int32_t flags;      /* W4A16_FLAG_* bits                                                 */
    int32_t row_blocks; /* row-block matvec: blocks of 16 weight rows per CTA (1..5); 0 = auto.
                           With both row_blocks and splits given, that exact launch is used. */
    int32_t reserved[2];
} w4a16_options;

/*
 * w4a16_options.flags.
 * W4A16_FLAG_NO_PDL: launch without programmatic dependent launch (the kernel
 *   then starts only after the previous work in the stream has finished).
 * W4A16_FLAG_STATIC_WEIGHTS: the caller promises that wq, scales and biases are
 *   not written by work still pending in the stream, so the kernel may start
 *   streaming them before the preceding kernel completes (x is always read
 *   after it).  This is the usual situation for model weights in a decode loop.
 * W4A16_FLAG_TEST_DROP_COPY: for tests of the timeout path only.  Valid with the
 *   row-block matvec alone (else W4A16_ERR_INVALID_ARG): CTA 0 never requests the
 *   codes of its first group, so the waits for them cannot complete, and every
 *   wait of the launch gives up after 200 us instead of 2 s.  The kernel records
 *   W4A16_ERR_TIMEOUT (read and cleared by w4a16_device_status), leaves its loops
 *   and ends normally; the output is undefined.  Nothing traps and the context
 *   stays usable.
 */
enum w4a16_flags {
    W4A16_FLAG_NO_PDL = 1,
    W4A16_FLAG_STATIC_WEIGHTS = 2,
    W4A16_FLAG_TEST_DROP_COPY = 4
};

/*
 * w4a16_matmul with explicit options (tests and benchmarks force a path or a
 * split count through it).  opt == NULL behaves like w4a16_matmul.  Forcing
 * the matvec path with M > 8 returns W4A16_ERR_UNSUPPORTED.
 */
int w4a16_matmul_ex(const void *x, const uint32_t *wq, const void *scales,
                    const void *biases, void *y, int64_t M, int64_t N, int64_t K,
                    void *stream, const w4a16_options *opt);

/* What a call of the given size would launch (host-side planning only). */
typedef struct w4a16_plan_info {
    int32_t path;            /* enum w4a16_path chosen                                  */
    int32_t splits;          /* K splits: GEMM (a cluster holds 2 x splits CTAs) or row-block
                                matvec (a cluster holds splits CTAs); 1 for the stream-K matvec */
    int32_t grid_x, grid_y, grid_z;   /* GEMM without a K split: a persistent grid of at most
                                         one CTA pair per two SMs, each pair looping over tiles */
    int32_t block;           /* threads per CTA                                         */
    int32_t smem_bytes;      /* dynamic shared memory per CTA                           */
    int32_t cluster;         /* CTAs per cluster (1 = no cluster)                       */
    int64_t tiles;           /* output tiles (row-block matvec: clusters of row_blocks x 16 rows) */
    int64_t units;           /* stream-K matvec: (row tile x 128-group) work units;
                                row-block matvec: 16-row blocks                         */
    int64_t workspace_bytes; /* library workspace the call needs                        */
    int32_t row_blocks;      /* row-block matvec: blocks of 16 weight rows per cluster   */
    int32_t slices;          /* row-block matvec: launches over slices of 8 x rows (1 for
                                M <= 8, ceil(M / 8) for 8 < M <= 32); 0 on other paths   */
} w4a16_plan_info;

/*
 * Fill *out with the launch plan for an M x N x K call.  Performs no CUDA call
 * when opt->sm_count > 0, so it also runs on machines without a GPU.
 */
int w4a16_plan(int64_t M, int64_t N, int64_t K, const w4a16_options *opt,
               w4a16_plan_info *out);

/*
 * Synchronise `stream`, then read and clear the device-side status word of the
 * current device.  Returns W4A16_OK, W4A16_ERR_TIMEOUT (a kernel abandoned a
 * bounded wait; its outputs are undefined and the library's split bookkeeping
 * has been reset) or W4A16_ERR_CUDA.
 */
int w4a16_device_status(void *stream);

/* Free every library-owned workspace on every device (synchronises them). */
void w4a16_release(void);

/* Human-readable name of a status code (static storage; never NULL). */
const char *w4a16_status_string(int status);

/* cudaError_t value of the most recent failed CUDA call made by the library. */
int w4a16_last_cuda_error(void);

/* ABI version: major * 10000 + minor * 100 + patch. */
int w4a16_version(void);

/*
 * Stream-K bookkeeping of the matvec, exported for host-side tests: the CTA
 * (0 <= c < workers) whose contiguous unit range contains unit u when `units`
 * units are split over `workers` CTAs (CTA c owns [c*units/workers,
 * (c+1)*units/workers)).  Returns -1 for arguments out of range.
 */
int64_t w4a16_streamk_owner(int64_t units, int64_t workers, int64_t u);

/*
 * Allocation-free matvec (M <= 8).  The pages have no counterpart: this entry
 * point exists for callers that cannot allocate device memory -- code running
 * under a memory pool or allocator that owns all device memory, inside a
 * capture or real-time loop where cudaMalloc is forbidden, or in processes
 * without the right to create allocations.  It runs the same kernel as
 * w4a16_matmul on the matvec path, but the scratch it needs for rows split
 * across CTAs (FP32 partial sums and per-tile tickets) lives in one
 * file-scope device array of W4A16_NOALLOC_SCRATCH_BYTES that every GPU
 * loading the library holds until the process exits.  The call itself
 * allocates nothing (no cudaMalloc, no allocating library routine).
 *
 * Limits: 1 <= M <= 8 and N <= W4A16_NOALLOC_MAX_N; larger sizes return
 * W4A16_ERR_UNSUPPORTED without launching.  Other arguments, layouts and
 * errors are those of w4a16_matmul.
 * Set-up: the first call on a device looks up the array's device address
 * (cudaGetSymbolAddress).  w4a16_release forgets the address; call it before
 * resetting a device.
 * Sharing: every call uses the same array and clears its tickets on `stream`
 * before launching, so calls whose kernels can overlap on the GPU (different
 * streams without ordering) race and give undefined results; serialise them.
 * That clearing is stream-ordered work of its own: unlike w4a16_matmul, this
 * entry point's kernel does not overlap the end of the preceding kernel.
 */
#define W4A16_NOALLOC_MAX_N 1048576
#define W4A16_NOALLOC_SCRATCH_BYTES 1343488
int w4a16_matvec_noalloc(const void *x, const uint32_t *wq, const void *scales,
                         const void *biases, void *y, int64_t M, int64_t N,
                         int64_t K, void *stream);

/*
 * Fused gate/up projection with the SwiGLU product (decode, M <= 8):
 *   h[m, j] = bf16_rne(silu(g[m, j]) * u[m, j]),  silu(g) = g / (1 + exp(-g)),
 * where g and u are the FP32 sums of two W4A16 layers over the same x (the gate
 * and up projections of a gated MLP), never rounded to BF16 in between.  Both
 * share x, so one pass of the row-block matvec reads x once and writes h
 * (llama.cpp issue "Metal prefill speedup (~68%) on M5 Max": SwiGLU fused into
 * the matrix product; its related work fuses gate/up with interleaved rows).
 *
 * Weights: the two layers' rows interleaved in blocks of 8: rows 16 b .. 16 b + 7
 * of wq, scales and biases are gate rows 8 b .. 8 b + 7 and rows 16 b + 8 .. 16 b
 * + 15 the up rows 8 b .. 8 b + 7 (2 N2 rows in all, each in the packed format
 * above).  x bf16 [M, K]; h bf16 [M, N2], written.  Sizes: 0 <= M <= 8, N2 % 8
 * == 0, K % 128 == 0, else W4A16_ERR_UNSUPPORTED; M == 0 or N2 == 0 launches
 * nothing.  Alignment, aliasing, ownership and stream semantics as w4a16_matmul.
 * A gate or up sum that is not finite in FP32 is recomputed by the plain
 * definition, as in w4a16_matmul.
 */
int w4a16_gate_up(const void *x, const uint32_t *wq, const void *scales,
                  const void *biases, void *h, int64_t M, int64_t N2, int64_t K,
                  void *stream);

/*
 * Quantiser: weights W [N, K] -> the packed format above (wq [N, K/8] codes,
 * scales and biases [N, K/128] BF16), on the GPU.
 *
 * The recipe is the affine min/max quantisation per 128-group that the
 * layer's weights are defined with (tiny-llm "Week 2 Day 6", Task 3: one
 * scale and bias per group; the reference problem's inputs: scale = (max -
 * min) / 15, bias = min, q rounded and clamped to 0..15, eight codes per
 * uint32 low nibble first).  Per row n and group g, all in FP32:
 *   lo, hi = min, max of the group's 128 values (a zero is taken as +0)
 *   scale  = bf16_rne((hi - lo) / 15)       bias = bf16_rne(lo)
 *   q[k]   = 0 when scale == 0 (a constant group), else
 *            clamp(rint((w[k] - bias) / scale), 0, 15), with the BF16
 *            scale and bias, IEEE division and rint rounding half to even.
 * Each step is correctly rounded: the output is bit-identical to the same
 * recipe computed sequentially on a CPU.  Inputs must be finite.
 *
 * Arguments: w device pointer to W, row-major FP32 (w_dtype = W4A16_DTYPE_F32)
 * or BF16 (W4A16_DTYPE_BF16); wq, scales, biases device pointers to the
 * outputs, written; N, K sizes with K % 128 == 0 (else W4A16_ERR_UNSUPPORTED);
 * N == 0 or K == 0 returns W4A16_OK and launches nothing.  Every pointer must
 * be 16-byte aligned (W4A16_ERR_MISALIGNED) and the outputs must not overlap
 * w (W4A16_ERR_INVALID_ARG).  Ownership and stream semantics as w4a16_matmul:
 * the work is enqueued on `stream` and the call returns without waiting.
 */
enum w4a16_dtype {
    W4A16_DTYPE_F32 = 0,
    W4A16_DTYPE_BF16 = 1
};
int w4a16_quantize(const void *w, int32_t w_dtype, uint32_t *wq, void *scales,
                   void *biases, int64_t N, int64_t K, void *stream);

/*
 * The same layer with 2- or 8-bit codes (the "Route affine qmv_wide by
 * bit-width and batch size" PR routes the affine format by its bit width b):
 *   y[m,n] = bf16_rne( sum_k x[m,k] * (scale[n,k/128] * q[n,k] + bias[n,k/128]) )
 * with q[n,k] = (wq[n*(K*b/32) + k/(32/b)] >> (b*(k%(32/b)))) & (2^b - 1):
 * 32 / b codes per uint32, the lowest code in the lowest bits.  x, scales,
 * biases and y are as in w4a16_matmul; wq is [N, K*b/32] uint32.  FP32
 * accumulation; the result is within one BF16 ulp (+ 1e-3 absolute) of the
 * plain sequential FP32 definition, and does not depend on timing.
 *
 * bits = 4 is w4a16_matmul itself (every path, any M).  bits = 2 and 8 run a
 * tensor-core matvec for decode: M <= 32 (in launches of 8 x rows; larger M
 * gives W4A16_ERR_UNSUPPORTED), any N, K % 128 == 0.  Other bit widths give
 * W4A16_ERR_UNSUPPORTED.  Size, alignment, overlap, K == 0 and stream rules
 * are those of w4a16_matmul (wq spans N*K*b/8 bytes); every launch uses the
 * programmatic-dependent-launch attribute and waits for the preceding kernel
 * before its first read.
 */
int w4a16_matmul_bits(const void *x, const uint32_t *wq, const void *scales,
                      const void *biases, void *y, int64_t M, int64_t N, int64_t K,
                      int32_t bits, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* W4A16_H */
