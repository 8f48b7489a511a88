/*
 * hyena.h -- C ABI of the B200-native Hyena gated FFT long convolution.
 *
 * The operation ([P4] "HyenaDNA operator walk-through" (adg.csdn.net),
 * section 二.1, HyenaOperator.forward, and section 二.2, fftconv; [P5]
 * "Native Multi-Dimensional Subquadratic Operators via Input Dependent Long
 * Convolutions", 方法论 -- 原生 ND 卷积 and 边界处理 -- for the 2-D form):
 *
 *   uc      = short_conv(u)            width-3 causal depthwise conv (optional)
 *   x0..x(order-1), v = uc split along channels in blocks of C
 *   for s = 1 .. order-1:
 *       v = x_{order-s} * v                         (elementwise gate)
 *       v = (k_s conv v)[0:L] + D_s * v              (causal long conv + skip)
 *   y  = x0 * v
 *
 * The long convolution is evaluated as the 2L-point (2-D: 2H x 2W) zero-padded
 * FFT product with a cached filter spectrum, which makes it non-circular.
 *
 * Conventions for every entry point
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never allocates, frees or retains them.  They must be 16-byte aligned.
 *  - Tensors are row-major, last dimension contiguous: 1-D [.., L], 2-D
 *    [.., H, W].  sizes = {L} for ndim 1, {H, W} for ndim 2.
 *  - dtype selects the storage of u, y (and of k in hyena_filter_spectrum):
 *    HYENA_F32 or HYENA_BF16 (round-to-nearest-even on store).  Arithmetic is
 *    fp32 throughout; spectra are stored as complex64.
 *  - All work is enqueued on `stream` (a cudaStream_t, NULL = legacy default
 *    stream) and is asynchronous: no call synchronises the host.
 *  - Arguments are validated before anything is enqueued; on any error
 *    nothing is launched and a status other than HYENA_OK is returned, with a
 *    thread-local message available from hyena_last_error_detail().
 *  - Supported shapes: 1-D L a power of two in [16, 2^20]; 2-D H, W powers of
 *    two in [16, 512]; order in [2, 8]; C >= 1, B >= 1.
 *  - Apart from the fixed scratch of hyena_gated_fftconv_noalloc (see there),
 *    the library keeps no state between calls; all entry points are
 *    thread-safe.  Calls on one stream are ordered; calls that write the
 *    same buffers from different streams race.
 */
#ifndef HYENA_B200_H
#define HYENA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { HYENA_F32 = 0, HYENA_BF16 = 1 } hyena_dtype_t;

typedef enum {
    HYENA_OK = 0,
    HYENA_ERR_INVALID_ARG = 1,        /* NULL pointer, bad dtype, B or C < 1, ...     */
    HYENA_ERR_UNSUPPORTED_SHAPE = 2,  /* L / H / W / order outside the supported set  */
    HYENA_ERR_MISALIGNED = 3,         /* a tensor pointer is not 16-byte aligned      */
    HYENA_ERR_SPECTRUM_MISMATCH = 4,  /* spectrum_bytes does not match the shape      */
    HYENA_ERR_WORKSPACE_TOO_SMALL = 5,/* workspace smaller than one row's share       */
    HYENA_ERR_CUDA = 6,               /* a CUDA launch reported an error              */
    HYENA_ERR_INTERNAL = 7,
    HYENA_ERR_TIMEOUT = 8             /* a bounded device wait ran out (reported by
                                         hyena_spectrum_check)                       */
} hyena_status_t;

/*
 * ndim: 1 (L), 2 (H x W, non-circular: zero padded, output cropped),
 * 3 (N1 x H x W volumes, each a power of two in [16, 128], non-circular:
 * every axis zero padded to twice its length, kernel anchored at the origin,
 * output cropped; [P5] 原生 ND 卷积 and 3-D medical volumes), or
 * 2 | HYENA_CIRCULAR (H x W, circular: periodic boundary, the filter on the
 * same H x W grid, v[p][q] = sum_{i,j} K[i][j] w[(p-i) mod H][(q-j) mod W] +
 * D w[p][q]).  Source: [P5] 方法论 (边界处理: circular convolution for
 * periodic physical systems, non-circular by zero padding for images and
 * volumes).  Every call that takes ndim accepts the flag; a spectrum built
 * for one form is rejected by the other (its size differs).
 */
#define HYENA_CIRCULAR 0x100

/* Version of this ABI (major * 100 + minor). */
int hyena_version(void);

/* Static name of a status code. */
const char* hyena_status_string(hyena_status_t status);

/* Thread-local description of the last error returned on this thread ("" if
 * none).  Valid until the next call on the same thread. */
const char* hyena_last_error_detail(void);

/*
 * Bytes of the spectrum buffer for C channels, shape sizes[ndim], order.
 * Returns 0 for unsupported arguments.
 */
size_t hyena_spectrum_bytes(int64_t C, int ndim, const int64_t* sizes, int order);

/*
 * hyena_filter_spectrum -- S0, the filter-spectrum cache.
 *
 * Source: [P4] section 二.1 (k = filter(l) rearranged 'l (o d) -> o d l',
 * bias 'o d'), section 二.2 (fftconv(v, k[o], bias[o])); the zero-padded FFT
 * evaluation of the long convolution.
 *
 *   k        [order-1, C, sizes...] long filters in step order (k_dtype)
 *   D        [order-1, C] fp32 skip ("bias") per step and channel, or NULL (= 0)
 *   spectrum caller-allocated device buffer of spectrum_bytes =
 *            hyena_spectrum_bytes(C, ndim, sizes, order) bytes; receives a
 *            header, the twiddle tables of this shape (double-precision values
 *            rounded to fp32) and, for every (step, channel), the zero-padded
 *            spectrum of k with D folded in (D * v = (D delta) conv v) and the
 *            inverse-FFT normalisation folded in.
 *
 * The buffer is the cache: keep it while k and D are unchanged and pass it to
 * every hyena_gated_fftconv call with the same (C, sizes, order).
 */
hyena_status_t hyena_filter_spectrum(const void* k, hyena_dtype_t k_dtype, const float* D, int64_t C,
                                     int ndim, const int64_t* sizes, int order, void* spectrum,
                                     size_t spectrum_bytes, void* stream);

/*
 * hyena_shortconv -- S1 on its own (1-D only).
 *
 * Source: [P4] section 二.1, short_filter = Conv1d(inner, inner, 3, padding=2,
 * groups=inner) truncated to the first L samples:
 *   out[b, j, t] = w[j,0] u[b,j,t-2] + w[j,1] u[b,j,t-1] + w[j,2] u[b,j,t] + bias[j],
 *   with u[.., t<0] = 0.
 *
 *   u, out [B, Ctot, L] (dtype); may not overlap.
 *   w      [Ctot, 3] fp32;  bias [Ctot] fp32 or NULL (= 0).
 */
hyena_status_t hyena_shortconv(const void* u, void* out, const float* w, const float* bias, int64_t B,
                               int64_t Ctot, int64_t L, hyena_dtype_t dtype, void* stream);

/*
 * Workspace bytes hyena_gated_fftconv uses for this shape by default (0 for
 * the on-chip path, 1-D L <= 16384).  Any workspace at least as large as one
 * row's share (hyena_gated_fftconv_workspace_min_bytes) is accepted; larger
 * workspaces let more rows share each pass.
 */
size_t hyena_gated_fftconv_workspace_bytes(int64_t B, int64_t C, int ndim, const int64_t* sizes, int order);
size_t hyena_gated_fftconv_workspace_min_bytes(int64_t C, int ndim, const int64_t* sizes, int order);

/*
 * hyena_gated_fftconv -- S1..S9, the hot path.
 *
 * Source: [P4] section 二.1 (split *x, v = uc.split(d_model); for o, x_i in
 * enumerate(reversed(x[1:])): v = v * x_i; v = fftconv(v, k[o], bias[o]);
 * y = v * x[0]); [P5] 方法论 for ndim = 2 and 3 (non-circular global
 * convolution by zero padding each axis to twice its length; output cropped
 * to the input grid, kernel anchored at the origin) and for
 * ndim = 2 | HYENA_CIRCULAR (circular, periodic boundary).
 *
 *   u        [B, (order+1)*C, sizes...] projected stream, channel blocks in the
 *            order x0, x1, ..., x(order-1), v (dtype)
 *   y        [B, C, sizes...] output (dtype); may not overlap u
 *   spectrum buffer filled by hyena_filter_spectrum for the same C, sizes,
 *            order; spectrum_bytes must equal hyena_spectrum_bytes(...)
 *   sc_w     [(order+1)*C, 3] fp32 short-conv taps applied to every chunk while
 *            loading, or NULL when u is already short-convolved (1-D only;
 *            must be NULL for ndim 2)
 *   sc_bias  [(order+1)*C] fp32 or NULL (= 0); ignored when sc_w is NULL
 *   workspace, workspace_bytes  device scratch for the multi-pass (L >= 32768)
 *            and 2-D paths; may be NULL/0 for the on-chip path.  Its contents
 *            are undefined after the call.
 */
hyena_status_t hyena_gated_fftconv(const void* u, void* y, const void* spectrum, size_t spectrum_bytes,
                                   const float* sc_w, const float* sc_bias, int64_t B, int64_t C, int ndim,
                                   const int64_t* sizes, int order, hyena_dtype_t dtype, void* workspace,
                                   size_t workspace_bytes, void* stream);

/*
 * hyena_gated_fftconv_per_sample -- S1..S9 with one long filter per (b, c)
 * row: input-dependent kernels.
 *
 * Source: [P5] 方法论 (通过寄存器与 FiLM 实现输入依赖型核: the kernel
 * K(x) = w(c) * f_theta(c; z(x)) depends on the whole input sample, so every
 * sample brings its own filters) and 实现 (nSubQ: the spectrum modulation
 * applies the input-dependent kernel inside the fused FFT -> modulate -> IFFT).
 * How the per-sample filters are generated is outside this call: they arrive
 * as k, like the shared filters of hyena_gated_fftconv.
 *
 *   spectrum buffer filled by hyena_filter_spectrum(k, k_dtype, D, B*C, ...)
 *            from k [order-1, B, C, sizes...] and D [order-1, B, C] (the
 *            per-sample filters as B*C channels); spectrum_bytes must equal
 *            hyena_spectrum_bytes(B*C, ndim, sizes, order).  Row (b, c) of
 *            order step s uses filter (s, b*C + c).
 *   everything else as hyena_gated_fftconv (same shapes, errors, workspace).
 *
 * The spectrum is read once per row instead of once per channel.  At L = 8192
 * with bf16 storage this runs the fp32 register kernel (the tensor-core kernel
 * pairs two batch rows of one channel, which needs a shared filter).
 */
hyena_status_t hyena_gated_fftconv_per_sample(const void* u, void* y, const void* spectrum, size_t spectrum_bytes,
                                              const float* sc_w, const float* sc_bias, int64_t B, int64_t C,
                                              int ndim, const int64_t* sizes, int order, hyena_dtype_t dtype,
                                              void* workspace, size_t workspace_bytes, void* stream);

/*
 * hyena_gated_fftconv_host -- hyena_gated_fftconv on inputs and outputs that
 * live in host memory, with the host<->device copies pipelined against the
 * kernels.
 *
 * The paper has no counterpart: this entry point is for callers whose stream
 * of inputs sits in host memory (serving, or data larger than the device).
 * The batch is cut into chunks of chunk_rows batch rows (0: ceil(B/4)); each
 * chunk is copied to u_dev, convolved and copied back to y_host, alternately
 * on `stream` and on a second stream the library keeps per device, so one
 * chunk's host-to-device copy overlaps the previous chunk's kernel and
 * device-to-host copy.  Chunks share the workspace, so on the workspace paths
 * their kernels run one after another.
 *
 *   u_host   [B, (order+1)*C, sizes...] host memory (page-locked for overlap;
 *            pageable memory works but its copies do not overlap)
 *   y_host   [B, C, sizes...] host memory, written when `stream` completes
 *   u_dev, y_dev  device buffers of the full u and y sizes (caller-owned)
 *   everything else as hyena_gated_fftconv (shared filters).
 * Returns after queueing; the results are in y_host once `stream` completes.
 * Argument errors are reported before anything is queued.
 */
hyena_status_t hyena_gated_fftconv_host(const void* u_host, void* y_host, void* u_dev, void* y_dev,
                                        const void* spectrum, size_t spectrum_bytes, const float* sc_w,
                                        const float* sc_bias, int64_t B, int64_t C, int ndim, const int64_t* sizes,
                                        int order, hyena_dtype_t dtype, void* workspace, size_t workspace_bytes,
                                        int64_t chunk_rows, void* stream);

/*
 * Size of the fixed scratch array used by hyena_gated_fftconv_noalloc (32 MiB).
 */
#define HYENA_NOALLOC_SCRATCH_BYTES (32u << 20)

/*
 * hyena_gated_fftconv_noalloc -- the same operation as hyena_gated_fftconv,
 * for callers that cannot allocate device memory.
 *
 * The paper has no counterpart: this entry point exists for callers that have
 * no way to provide a workspace, such as a plugin whose host framework owns
 * every device allocation, or a serving loop that must never call cudaMalloc
 * (an allocation can block, synchronise the device or fail under memory
 * pressure at a point where the work cannot be dropped).  Instead of a
 * caller workspace it uses a fixed device array of
 * HYENA_NOALLOC_SCRATCH_BYTES that is part of the library image; every GPU
 * that loads the library keeps that array until the process exits.  The
 * caller still passes u, y and the spectrum; arguments and errors are those
 * of hyena_gated_fftconv.  Nothing is allocated or freed.
 *
 *  - Limit: shapes whose workspace row (hyena_gated_fftconv_workspace_min_bytes)
 *    exceeds HYENA_NOALLOC_SCRATCH_BYTES are rejected with
 *    HYENA_ERR_WORKSPACE_TOO_SMALL; rows are processed in groups that fit.
 *  - Set-up: the first call on each device looks up the array's device
 *    address (cudaGetSymbolAddress, with that device current), which may load
 *    the library's device code; make that first call before any stream
 *    capture.
 *  - Sharing: every call on a device uses the same array, which keeps the
 *    last call's contents.  No zeroing is needed: each call writes every
 *    scratch element before reading it.  Calls that overlap on the GPU (for
 *    example on two streams) race on the array and give wrong results.
 */
hyena_status_t hyena_gated_fftconv_noalloc(const void* u, void* y, const void* spectrum, size_t spectrum_bytes,
                                           const float* sc_w, const float* sc_bias, int64_t B, int64_t C, int ndim,
                                           const int64_t* sizes, int order, hyena_dtype_t dtype, void* stream);

/*
 * Debug helper (synchronous): copies the spectrum header to the host and
 * checks it against (C, sizes, order).  Returns HYENA_OK when it matches,
 * HYENA_ERR_SPECTRUM_MISMATCH when not (e.g. never filled, or filled for
 * another shape), HYENA_ERR_TIMEOUT when an earlier convolution with this
 * spectrum ran out of the budget of a bounded tensor-core wait (the L = 8192
 * bf16 path; the outputs of that row pair were written as NaN and nothing was
 * left in flight).  Synchronises `stream`.  Rebuilding the spectrum clears the
 * record.
 */
hyena_status_t hyena_spectrum_check(const void* spectrum, int64_t C, int ndim, const int64_t* sizes, int order,
                                    void* stream);

/*
 * Test hook for the bounded waits of the tensor-core kernel (the L = 8192, bf16,
 * order <= 3 path of hyena_gated_fftconv; same arguments with ndim = 1,
 * sizes = {8192}, dtype = HYENA_BF16).  Each wait of that kernel on its
 * tensor-core work gives up after `wait_budget_ns` nanoseconds (the normal entry
 * point uses 2 s).  With issue_mma = 0 no tensor-core work is issued, so the
 * first wait runs out on a barrier that nothing completes: the kernel records
 * the timeout in the spectrum header (hyena_spectrum_check then returns
 * HYENA_ERR_TIMEOUT), writes NaN to the outputs of the row pair it was on, and
 * returns with nothing in flight.  Other shapes return
 * HYENA_ERR_UNSUPPORTED_SHAPE.  Asynchronous on `stream`.
 */
hyena_status_t hyena_debug_conv_tc(const void* u, void* y, const void* spectrum, size_t spectrum_bytes,
                                   const float* sc_w, const float* sc_bias, int64_t B, int64_t C, int order,
                                   uint64_t wait_budget_ns, int issue_mma, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* HYENA_B200_H */
