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
 *    HYENA_F32 or HYENA_BF16 (round-to-nearest-even on store).  Arithmetic:
 *    the short conv, the gates, the twiddles and the spectrum products are
 *    fp32 on every path.  With fp32 storage, and on the bf16 paths not named
 *    below, the transforms are fp32 too and the spectrum is read as
 *    complex64.  At L = 8192 with bf16 storage (order
 *    <= 3, shared filters) the DFT stages run on the tensor cores: their
 *    operands and the DFT matrices are rounded to bf16 and accumulated in
 *    fp32, and the spectrum is read as bf16 (re, im) pairs (row error a few
 *    1e-3); HYENA_FLAG_FP32_TRANSFORM (hyena_gated_fftconv_ex) selects the
 *    fp32 transform there instead.  At L = 65536 with bf16 storage (order
 *    <= 3, shared filters) the 2L-point transform of a row pair is split over
 *    a cluster of 8 CTAs: the 8-point DFTs, gates and twiddles in fp32, the
 *    16384-point part on the tensor cores as at L = 8192, the exchanges
 *    between the CTAs and the spectrum as bf16 pairs (row error ~1e-2 at
 *    order 3); HYENA_FLAG_FP32_TRANSFORM selects the fp32 multi-pass
 *    transform there.  2-D with bf16 storage and H = 256 (W a multiple of
 *    32): the column transforms (512 points) run on the tensor cores the same
 *    way, with the spectrum read as bf16 pairs (order <= 3); for 256 x 256
 *    images with an even batch and shared filters the two images of a channel
 *    travel as one complex image and the row transforms run there too (image
 *    error a few 1e-3); the circular form at 256 x 256 (bf16, even batch,
 *    shared filters, order <= 3) runs its 256-point row and column
 *    transforms the same way, the images paired; HYENA_FLAG_FP32_TRANSFORM
 *    selects the fp32 passes.
 *    With bf16 storage the intermediate of the multi-pass (L >= 32768) and
 *    N-D paths is kept as bf16 pairs in the workspace.
 *  - All work is enqueued on `stream` (a cudaStream_t, NULL = legacy default
 *    stream) and is asynchronous: no call synchronises the host.  The
 *    convolution kernels are launched with programmatic stream serialisation:
 *    one may begin (build its tables in shared memory) while the kernel before
 *    it on the stream finishes, but reads and writes no global memory before
 *    that kernel has completed, so plain stream order holds for the data.
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
                                         hyena_kernel_status)                        */
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
 *            inverse-FFT normalisation folded in.  At L = 65536 it holds that
 *            spectrum twice: in the multi-pass layout (complex64) and as the
 *            bf16 plane the cluster path reads.
 *
 * The buffer is the cache: keep it while k and D are unchanged and pass it to
 * every hyena_gated_fftconv call with the same (C, sizes, order).
 */
hyena_status_t hyena_filter_spectrum(const void* k, hyena_dtype_t k_dtype, const float* D, int64_t C,
                                     int ndim, const int64_t* sizes, int order, void* spectrum,
                                     size_t spectrum_bytes, void* stream);

/*
 * Parameters of the implicit long filter (device pointers, fp32, row-major).
 * Source: [P4] section 二.2, HyenaFilter: filter(L) = modulation(t,
 * implicit_filter(pos_emb(L))) with
 *   pos_emb(l)   = [t_l, cos(2 pi b l / L), sin(2 pi b l / L)], b = 1 .. (emb_dim-1)/2,
 *                  t_l = l / (L-1)
 *   implicit_filter = Linear(emb_dim, width) -> Sin, num_inner x
 *                  (Linear(width, width) -> Sin), Linear(width, d_model)
 *                  without bias; Sin(x) = sin(w * x), w per feature
 *   modulation   = h[l][c] exp(-alpha[c] t_l)
 * with d_model = (order-1) C outputs taken as 'l (o d) -> o d l' (output
 * channel s*C + c is the filter of order step s, channel c).
 */
typedef struct {
    int emb_dim;            /* odd, 3 .. 33 */
    int width;              /* 1 .. 128 (the HyenaOperator passes filter_order = 64) */
    int num_inner;          /* 0 .. 8 */
    const float* W_in;      /* [width, emb_dim] */
    const float* b_in;      /* [width] */
    const float* W_inner;   /* [num_inner, width, width], or NULL when num_inner = 0 */
    const float* b_inner;   /* [num_inner, width], or NULL when num_inner = 0 */
    const float* W_out;     /* [(order-1) C, width] */
    const float* w;         /* [width] Sin frequencies */
    const float* alpha;     /* [(order-1) C] decay rates */
} hyena_implicit_filter_t;

/* Workspace bytes of hyena_filter_spectrum_implicit: width x L fp32 (0 for bad arguments). */
size_t hyena_implicit_filter_workspace_bytes(int64_t L, int width);

/*
 * hyena_filter_spectrum_implicit -- S0 from the implicit filter: the filters
 * are generated on the device and go straight into the spectrum build.
 *
 * Fills `spectrum` exactly as hyena_filter_spectrum(k, HYENA_F32, D, C,
 * ndim 1, {L}, order, ...) would for the filters k [order-1, C, L] the
 * parameters generate; use it with hyena_gated_fftconv like any spectrum.
 * The MLP's hidden layers are evaluated once for all t into `workspace`
 * (hyena_implicit_filter_workspace_bytes), and each filter row is computed
 * inside the spectrum kernel, so the filters are not written to memory
 * unless k_out is given: k_out [order-1, C, L] fp32 (8-byte aligned)
 * receives a copy of them (for checking), or NULL.
 * L: the on-chip lengths, powers of two in [16, 16384]; D as in
 * hyena_filter_spectrum.  Asynchronous on `stream`.
 */
hyena_status_t hyena_filter_spectrum_implicit(const hyena_implicit_filter_t* f, const float* D, int64_t C, int64_t L,
                                              int order, void* spectrum, size_t spectrum_bytes, void* workspace,
                                              size_t workspace_bytes, float* k_out, void* stream);

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
 *            are undefined after the call.  The cluster path (L = 65536, bf16)
 *            takes 512 KB per cluster in flight from it (as many clusters
 *            as are resident at two CTAs per SM: 33 on the B200s measured);
 *            the minimum workspace runs one cluster.
 *
 * The spectrum is only read.  Conditions the kernels detect on the device (a
 * spectrum whose header does not match the shape: that kernel writes no
 * output; a bounded tensor-core wait that ran out: NaN outputs) are recorded
 * in the device's status word, see hyena_kernel_status.
 */
hyena_status_t hyena_gated_fftconv(const void* u, void* y, const void* spectrum, size_t spectrum_bytes,
                                   const float* sc_w, const float* sc_bias, int64_t B, int64_t C, int ndim,
                                   const int64_t* sizes, int order, hyena_dtype_t dtype, void* workspace,
                                   size_t workspace_bytes, void* stream);

/* Flags of hyena_gated_fftconv_ex. */
#define HYENA_FLAG_FP32_TRANSFORM 0x1u  /* every transform multiply in fp32 on the CUDA cores (no bf16 tensor-core
                                           operands); changes only 1-D L = 8192 and 65536, 2-D H = 256 and the
                                           circular 2-D 256 x 256 form with bf16 storage */

/*
 * hyena_gated_fftconv_ex -- hyena_gated_fftconv with flags (shared filters).
 * flags: 0 (same as hyena_gated_fftconv) or HYENA_FLAG_FP32_TRANSFORM; other
 * bits are rejected with HYENA_ERR_INVALID_ARG.  The pages fix no precision
 * for the transform; this lets a caller pick fp32 arithmetic throughout
 * (bf16 storage, fp32 math) at the cost of speed at L = 8192.
 */
hyena_status_t hyena_gated_fftconv_ex(const void* u, void* y, const void* spectrum, size_t spectrum_bytes,
                                      const float* sc_w, const float* sc_bias, int64_t B, int64_t C, int ndim,
                                      const int64_t* sizes, int order, hyena_dtype_t dtype, void* workspace,
                                      size_t workspace_bytes, unsigned flags, void* stream);

/*
 * hyena_kernel_status -- what the convolution kernels detected on this device
 * since the last call (the current device's status word, which every
 * convolution kernel on the device may set; reading clears it).
 *
 * The paper has no counterpart: a kernel cannot return an error, so this is
 * how conditions seen on the device reach the caller.  Synchronises `stream`
 * (make it the stream of the calls in question, or NULL), then returns
 * HYENA_OK, HYENA_ERR_TIMEOUT (a bounded wait for tensor-core work ran out:
 * the L = 8192 bf16 path wrote NaN to that row pair's outputs and left
 * nothing in flight) or HYENA_ERR_SPECTRUM_MISMATCH (a kernel found a
 * spectrum header that does not match the shape it was given -- never
 * filled, or filled for another C, size or order of the same byte size --
 * and wrote no output), or HYENA_ERR_CUDA.  The word is per device, not per
 * stream or per call: kernels running on other streams meanwhile may set
 * bits between the read and the clear, and those bits are lost.  Its address
 * is looked up once per device (calls after a device reset are not
 * supported).
 */
hyena_status_t hyena_kernel_status(void* stream);

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
 * The batch is cut into chunks of chunk_rows batch rows (0: ceil(B/4), rounded
 * up to an even count when B allows, because the L = 8192 bf16 kernel
 * transforms two batch rows of a channel together); each
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
 * hyena_in_proj -- the input projection of the Hyena operator on the tensor
 * cores.
 *
 * Source: [P4] section 二.1, HyenaOperator: in_proj = nn.Linear(d_model,
 * (order+1) d_model) on u [b, l, d], then rearrange 'b l d -> b d l':
 *   u[b][j][l] = sum_i x[b][l][i] W[j][i] + bias[j],   j < (order+1) D.
 *
 *   x     [B, L, D] bf16 (features contiguous)
 *   W     [(order+1) D, D] bf16, the nn.Linear weight (out x in)
 *   bias  [(order+1) D] fp32, or NULL (= 0)
 *   u     [B, (order+1) D, L] bf16 out: the layout hyena_gated_fftconv reads
 * bf16 operands, fp32 accumulation, bf16 result (round to nearest even).
 * D and L multiples of 8; pointers 16-byte aligned (bias 4-byte); u may not
 * overlap x or W.  Asynchronous on `stream`; errors as for the other calls; a
 * bounded device wait that runs out is reported by hyena_kernel_status.
 */
hyena_status_t hyena_in_proj(const void* x, const void* W, const float* bias, void* u, int64_t B, int64_t L,
                             int64_t D, int order, void* stream);

/*
 * hyena_out_proj -- the output projection on the tensor cores.
 *
 * Source: [P4] section 二.1: y = rearrange(v * x[0], 'b d l -> b l d'), then
 * out_proj = nn.Linear(d_model, d_model):
 *   out[b][l][j] = sum_i y[b][i][l] W[j][i] + bias[j],   j < D.
 *
 *   y     [B, D, L] bf16, the output of hyena_gated_fftconv (read in place,
 *         no transposed copy)
 *   W     [D, D] bf16 (out x in);  bias [D] fp32 or NULL
 *   out   [B, L, D] bf16
 * Same precision, shape, alignment and error rules as hyena_in_proj.
 */
hyena_status_t hyena_out_proj(const void* y, const void* W, const float* bias, void* out, int64_t B, int64_t L,
                              int64_t D, void* stream);

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
 *    HYENA_ERR_WORKSPACE_TOO_SMALL before anything is enqueued (a 128^3
 *    volume, for example); rows are processed in groups that fit (at
 *    L = 2^20: 4 rows per group with fp32 storage, 8 with bf16 storage).
 *  - Set-up: the first call on each device looks up the array's device
 *    address (cudaGetSymbolAddress, with that device current), which may load
 *    the library's device code; make that first call before any stream
 *    capture.  The address is kept for the life of the process: after
 *    cudaDeviceReset (or anything else that tears down and recreates the
 *    device's primary context) the array may live elsewhere, so calls after
 *    such a reset are not supported.
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
 * another shape).  Synchronises `stream`.
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
 * the timeout in the device's status word (hyena_kernel_status then returns
 * HYENA_ERR_TIMEOUT), writes NaN to the outputs of the row pair it was on, and
 * returns with nothing in flight.  Other shapes return
 * HYENA_ERR_UNSUPPORTED_SHAPE.  Asynchronous on `stream`.
 */
hyena_status_t hyena_debug_conv_tc(const void* u, void* y, const void* spectrum, size_t spectrum_bytes,
                                   const float* sc_w, const float* sc_bias, int64_t B, int64_t C, int order,
                                   uint64_t wait_budget_ns, int issue_mma, void* stream);

/*
 * The same test hook for the cluster kernel (1-D L = 65536, bf16, order <= 3,
 * shared filters; workspace as in hyena_gated_fftconv).  A CTA whose wait ran
 * out issues no more tensor-core work but still takes every cluster barrier,
 * so the cluster finishes; its outputs are NaN and the timeout is recorded in
 * the device's status word.  Other shapes return HYENA_ERR_UNSUPPORTED_SHAPE.
 */
hyena_status_t hyena_debug_conv_cluster(const void* u, void* y, const void* spectrum, size_t spectrum_bytes,
                                        const float* sc_w, const float* sc_bias, int64_t B, int64_t C, int order,
                                        void* workspace, size_t workspace_bytes, uint64_t wait_budget_ns,
                                        int issue_mma, void* stream);

/*
 * The same test hook for the 2-D tensor-core passes (ndim = 2, H = 256, W a
 * multiple of 32, bf16 storage, shared filters; sizes = {256, W}; no short
 * conv; workspace as in hyena_gated_fftconv): the whole 2-D convolution runs,
 * with the tensor-core kernels' waits bounded by wait_budget_ns and, for
 * issue_mma = 0, no tensor-core work issued.  A CTA whose wait ran out writes
 * NaN (workspace columns or rows, or outputs) and stops; the later passes
 * carry the NaN into y.  Other shapes return HYENA_ERR_UNSUPPORTED_SHAPE.
 */
hyena_status_t hyena_debug_conv_2d_tc(const void* u, void* y, const void* spectrum, size_t spectrum_bytes, int64_t B,
                                      int64_t C, int64_t W, int order, void* workspace, size_t workspace_bytes,
                                      uint64_t wait_budget_ns, int issue_mma, void* stream);

/*
 * The same test hook for the circular form's paired tensor-core passes
 * (ndim = 2 | HYENA_CIRCULAR, sizes = {256, 256}, bf16 storage, even B, shared
 * filters, order <= 3; spectrum and workspace as in hyena_gated_fftconv):
 * the whole circular convolution runs with the waits of its three kernels
 * bounded by wait_budget_ns and, for issue_mma = 0, no tensor-core work
 * issued; a CTA whose wait ran out writes NaN and stops.  Other arguments
 * return HYENA_ERR_UNSUPPORTED_SHAPE.
 */
hyena_status_t hyena_debug_conv_2dc_tc(const void* u, void* y, const void* spectrum, size_t spectrum_bytes, int64_t B,
                                       int64_t C, int order, void* workspace, size_t workspace_bytes,
                                       uint64_t wait_budget_ns, int issue_mma, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* HYENA_B200_H */
