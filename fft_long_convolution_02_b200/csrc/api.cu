// api.cu -- the extern "C" boundary declared in include/hyena.h: argument
// validation, planning, and dispatch to the kernel launchers.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <string>

#include "grid2dc_tc.h"
#include "hyena.h"
#include "kernels.h"
#include "plan.h"

using namespace hyena;

namespace {

thread_local std::string g_detail;

hyena_status_t fail(hyena_status_t st, const std::string& why) {
    g_detail = why;
    return st;
}

hyena_status_t ok() {
    g_detail.clear();
    return HYENA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

size_t elem_size(hyena_dtype_t d) { return d == HYENA_BF16 ? 2 : 4; }

bool valid_dtype(int d) { return d == HYENA_F32 || d == HYENA_BF16; }

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

hyena_status_t cuda_status(cudaError_t e, const char* what) {
    if (e == cudaSuccess) return ok();
    return fail(HYENA_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}


// 1, 2, 3, or 2 | HYENA_CIRCULAR (the circular 2-D form)
bool valid_ndim(int ndim) { return ndim == 1 || ndim == 2 || ndim == 3 || ndim == (2 | kCircularFlag); }

hyena_status_t plan_or_fail(int64_t C, int ndim, const int64_t* sizes, int order, Plan* p) {
    std::string why;
    if (C < 1) return fail(HYENA_ERR_INVALID_ARG, "C must be >= 1");
    if (!sizes) return fail(HYENA_ERR_INVALID_ARG, "sizes is NULL");
    if (!valid_ndim(ndim)) return fail(HYENA_ERR_INVALID_ARG, "ndim must be 1, 2, 3 or 2 | HYENA_CIRCULAR");
    if (!make_plan(C, ndim, sizes, order, p, &why)) return fail(HYENA_ERR_UNSUPPORTED_SHAPE, why);
    return HYENA_OK;
}

}  // namespace

namespace hyena {
// Records the thread-local detail message reported by hyena_last_error_detail()
// and returns st (used by entry points defined in other translation units).
hyena_status_t set_last_error_detail(hyena_status_t st, const std::string& detail) { return fail(st, detail); }
}  // namespace hyena

extern "C" {

int hyena_version(void) { return 101; }

const char* hyena_status_string(hyena_status_t s) {
    switch (s) {
        case HYENA_OK: return "HYENA_OK";
        case HYENA_ERR_INVALID_ARG: return "HYENA_ERR_INVALID_ARG";
        case HYENA_ERR_UNSUPPORTED_SHAPE: return "HYENA_ERR_UNSUPPORTED_SHAPE";
        case HYENA_ERR_MISALIGNED: return "HYENA_ERR_MISALIGNED";
        case HYENA_ERR_SPECTRUM_MISMATCH: return "HYENA_ERR_SPECTRUM_MISMATCH";
        case HYENA_ERR_WORKSPACE_TOO_SMALL: return "HYENA_ERR_WORKSPACE_TOO_SMALL";
        case HYENA_ERR_CUDA: return "HYENA_ERR_CUDA";
        case HYENA_ERR_INTERNAL: return "HYENA_ERR_INTERNAL";
        case HYENA_ERR_TIMEOUT: return "HYENA_ERR_TIMEOUT";
    }
    return "HYENA_UNKNOWN_STATUS";
}

const char* hyena_last_error_detail(void) { return g_detail.c_str(); }

size_t hyena_spectrum_bytes(int64_t C, int ndim, const int64_t* sizes, int order) {
    Plan p;
    std::string why;
    if (!sizes || !valid_ndim(ndim) || !make_plan(C, ndim, sizes, order, &p, &why)) return 0;
    return p.total_bytes;
}

hyena_status_t hyena_filter_spectrum(const void* k, hyena_dtype_t k_dtype, const float* D, int64_t C, int ndim,
                                     const int64_t* sizes, int order, void* spectrum, size_t spectrum_bytes,
                                     void* stream) {
    Plan p;
    hyena_status_t st = plan_or_fail(C, ndim, sizes, order, &p);
    if (st != HYENA_OK) return st;
    if (!k || !spectrum) return fail(HYENA_ERR_INVALID_ARG, "k and spectrum must not be NULL");
    if (!valid_dtype(k_dtype)) return fail(HYENA_ERR_INVALID_ARG, "k_dtype must be HYENA_F32 or HYENA_BF16");
    if (!aligned16(k) || !aligned16(spectrum)) return fail(HYENA_ERR_MISALIGNED, "k and spectrum must be 16-byte aligned");
    if (D && !aligned4(D)) return fail(HYENA_ERR_MISALIGNED, "D must be 4-byte aligned");
    if (spectrum_bytes != p.total_bytes)
        return fail(HYENA_ERR_SPECTRUM_MISMATCH, "spectrum_bytes must equal hyena_spectrum_bytes() = " +
                                                      std::to_string(p.total_bytes));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* sp = static_cast<uint8_t*>(spectrum);
    cudaError_t e = launch_header_and_tables(p, sp, s);
    if (e != cudaSuccess) return cuda_status(e, "table fill");
    SpectrumArgs a{k, int(k_dtype), D, sp};
    switch (p.path) {
        case PATH_ONCHIP_1D: e = launch_spectrum_onchip(p, a, s); break;
        case PATH_MULTIPASS_1D: e = launch_spectrum_multipass(p, a, s); break;
        case PATH_GRID_2D:
        case PATH_GRID_2D_CIRC: e = launch_spectrum_2d(p, a, s); break;
        case PATH_GRID_3D: e = launch_spectrum_3d(p, a, s); break;
        default: return fail(HYENA_ERR_INTERNAL, "no path");
    }
    return cuda_status(e, "spectrum kernel");
}

hyena_status_t hyena_shortconv(const void* u, void* out, const float* w, const float* bias, int64_t B, int64_t Ctot,
                               int64_t L, hyena_dtype_t dtype, void* stream) {
    if (!u || !out || !w) return fail(HYENA_ERR_INVALID_ARG, "u, out and w must not be NULL");
    if (!valid_dtype(dtype)) return fail(HYENA_ERR_INVALID_ARG, "dtype must be HYENA_F32 or HYENA_BF16");
    if (B < 1 || Ctot < 1) return fail(HYENA_ERR_INVALID_ARG, "B and Ctot must be >= 1");
    if (L < kMin1D || L > kMaxL || (L & (L - 1)) != 0)
        return fail(HYENA_ERR_UNSUPPORTED_SHAPE, "L must be a power of two in [16, 2^20]");
    if (!aligned16(u) || !aligned16(out)) return fail(HYENA_ERR_MISALIGNED, "u and out must be 16-byte aligned");
    if (!aligned4(w) || (bias && !aligned4(bias))) return fail(HYENA_ERR_MISALIGNED, "w and bias must be 4-byte aligned");
    const size_t nbytes = size_t(B) * size_t(Ctot) * size_t(L) * elem_size(dtype);
    if (overlap(u, nbytes, out, nbytes)) return fail(HYENA_ERR_INVALID_ARG, "u and out overlap");
    return cuda_status(launch_shortconv(u, out, w, bias, B, Ctot, L, int(dtype), static_cast<cudaStream_t>(stream)),
                       "shortconv kernel");
}

size_t hyena_gated_fftconv_workspace_min_bytes(int64_t C, int ndim, const int64_t* sizes, int order) {
    Plan p;
    std::string why;
    if (!sizes || !valid_ndim(ndim) || !make_plan(C, ndim, sizes, order, &p, &why)) return 0;
    return p.ws_row_bytes;
}

size_t hyena_gated_fftconv_workspace_bytes(int64_t B, int64_t C, int ndim, const int64_t* sizes, int order) {
    Plan p;
    std::string why;
    if (B < 1 || !sizes || !valid_ndim(ndim) || !make_plan(C, ndim, sizes, order, &p, &why)) return 0;
    return size_t(default_group_rows(p, B * C)) * p.ws_row_bytes;
}

}  // extern "C"

namespace {

// Validation shared by the convolution entry points; fills the plan and the
// kernel arguments.
hyena_status_t prepare_conv(const void* u, void* y, const void* spectrum, size_t spectrum_bytes, const float* sc_w,
                            const float* sc_bias, int64_t B, int64_t C, int ndim, const int64_t* sizes, int order,
                            hyena_dtype_t dtype, void* workspace, size_t workspace_bytes, Plan* pp, ConvArgs* pa,
                            bool per_sample = false) {
    Plan& p = *pp;
    hyena_status_t st = plan_or_fail(C, ndim, sizes, order, &p);
    if (st != HYENA_OK) return st;
    // the spectrum holds C filters per order step, or B*C (one per (b, c) row)
    size_t spec_total = p.total_bytes;
    size_t g2_plane = p.g2_plane_off;
    if (per_sample) {
        Plan ps;
        if (B < 1) return fail(HYENA_ERR_INVALID_ARG, "B must be >= 1");
        st = plan_or_fail(B * C, ndim, sizes, order, &ps);
        if (st != HYENA_OK) return st;
        spec_total = ps.total_bytes;
        g2_plane = ps.g2_plane_off;
    }
    if (!u || !y || !spectrum) return fail(HYENA_ERR_INVALID_ARG, "u, y and spectrum must not be NULL");
    if (B < 1) return fail(HYENA_ERR_INVALID_ARG, "B must be >= 1");
    if (!valid_dtype(dtype)) return fail(HYENA_ERR_INVALID_ARG, "dtype must be HYENA_F32 or HYENA_BF16");
    if (ndim != 1 && sc_w) return fail(HYENA_ERR_INVALID_ARG, "the 2-D and 3-D forms have no short conv: sc_w must be NULL");
    if (!aligned16(u) || !aligned16(y) || !aligned16(spectrum))
        return fail(HYENA_ERR_MISALIGNED, "u, y and spectrum must be 16-byte aligned");
    if ((sc_w && !aligned4(sc_w)) || (sc_bias && !aligned4(sc_bias)))
        return fail(HYENA_ERR_MISALIGNED, "sc_w and sc_bias must be 4-byte aligned");
    if (spectrum_bytes != spec_total)
        return fail(HYENA_ERR_SPECTRUM_MISMATCH, std::string("spectrum_bytes must equal hyena_spectrum_bytes(") +
                                                      (per_sample ? "B*C" : "C") + ", ...) = " +
                                                      std::to_string(spec_total));
    const size_t es = elem_size(dtype);
    const size_t ubytes = size_t(B) * size_t(order + 1) * size_t(C) * size_t(p.n) * es;
    const size_t ybytes = size_t(B) * size_t(C) * size_t(p.n) * es;
    if (overlap(u, ubytes, y, ybytes)) return fail(HYENA_ERR_INVALID_ARG, "u and y overlap");
    int64_t group = 0;
    if (p.ws_row_bytes > 0) {
        if (!workspace || workspace_bytes < p.ws_row_bytes)
            return fail(HYENA_ERR_WORKSPACE_TOO_SMALL,
                        "workspace must hold at least " + std::to_string(p.ws_row_bytes) + " bytes");
        if (!aligned16(workspace)) return fail(HYENA_ERR_MISALIGNED, "workspace must be 16-byte aligned");
        if (overlap(workspace, workspace_bytes, y, ybytes) || overlap(workspace, workspace_bytes, u, ubytes) ||
            overlap(workspace, workspace_bytes, spectrum, spectrum_bytes))
            return fail(HYENA_ERR_INVALID_ARG, "workspace overlaps an operand");
        group = int64_t(workspace_bytes / p.ws_row_bytes);
        if (group > B * C) group = B * C;
    }
    *pa = ConvArgs{u, y, static_cast<const uint8_t*>(spectrum), sc_w, sc_w ? sc_bias : nullptr, B, int(dtype),
                   static_cast<float2*>(workspace), group};
    pa->spec_C = per_sample ? B * C : C;
    pa->spec_per_b = per_sample ? C : 0;
    pa->g2_plane_off = g2_plane;
    return HYENA_OK;
}

hyena_status_t gated_fftconv(const void* u, void* y, const void* spectrum, size_t spectrum_bytes, const float* sc_w,
                             const float* sc_bias, int64_t B, int64_t C, int ndim, const int64_t* sizes, int order,
                             hyena_dtype_t dtype, void* workspace, size_t workspace_bytes, void* stream,
                             bool per_sample, unsigned flags = 0) {
    if (flags & ~unsigned(HYENA_FLAG_FP32_TRANSFORM)) return fail(HYENA_ERR_INVALID_ARG, "unknown flag bits");
    Plan p;
    ConvArgs a;
    hyena_status_t st = prepare_conv(u, y, spectrum, spectrum_bytes, sc_w, sc_bias, B, C, ndim, sizes, order, dtype,
                                     workspace, workspace_bytes, &p, &a, per_sample);
    if (st != HYENA_OK) return st;
    a.fp32_transform = (flags & HYENA_FLAG_FP32_TRANSFORM) != 0;
    cudaError_t e = kernel_status_word(&a.status);
    if (e != cudaSuccess) return cuda_status(e, "kernel status word");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    switch (p.path) {
        case PATH_ONCHIP_1D: e = launch_conv_onchip(p, a, s); break;
        case PATH_MULTIPASS_1D: e = launch_conv_multipass(p, a, s); break;
        case PATH_GRID_2D:
        case PATH_GRID_2D_CIRC: e = launch_conv_2d(p, a, s); break;
        case PATH_GRID_3D: e = launch_conv_3d(p, a, s); break;
        default: return fail(HYENA_ERR_INTERNAL, "no path");
    }
    return cuda_status(e, "gated fftconv kernel");
}

}  // namespace

extern "C" {

hyena_status_t hyena_gated_fftconv(const void* u, void* y, const void* spectrum, size_t spectrum_bytes,
                                   const float* sc_w, const float* sc_bias, int64_t B, int64_t C, int ndim,
                                   const int64_t* sizes, int order, hyena_dtype_t dtype, void* workspace,
                                   size_t workspace_bytes, void* stream) {
    return gated_fftconv(u, y, spectrum, spectrum_bytes, sc_w, sc_bias, B, C, ndim, sizes, order, dtype, workspace,
                         workspace_bytes, stream, false);
}

hyena_status_t hyena_gated_fftconv_ex(const void* u, void* y, const void* spectrum, size_t spectrum_bytes,
                                      const float* sc_w, const float* sc_bias, int64_t B, int64_t C, int ndim,
                                      const int64_t* sizes, int order, hyena_dtype_t dtype, void* workspace,
                                      size_t workspace_bytes, unsigned flags, void* stream) {
    return gated_fftconv(u, y, spectrum, spectrum_bytes, sc_w, sc_bias, B, C, ndim, sizes, order, dtype, workspace,
                         workspace_bytes, stream, false, flags);
}

hyena_status_t hyena_gated_fftconv_per_sample(const void* u, void* y, const void* spectrum, size_t spectrum_bytes,
                                              const float* sc_w, const float* sc_bias, int64_t B, int64_t C,
                                              int ndim, const int64_t* sizes, int order, hyena_dtype_t dtype,
                                              void* workspace, size_t workspace_bytes, void* stream) {
    return gated_fftconv(u, y, spectrum, spectrum_bytes, sc_w, sc_bias, B, C, ndim, sizes, order, dtype, workspace,
                         workspace_bytes, stream, true);
}

hyena_status_t hyena_debug_conv_tc(const void* u, void* y, const void* spectrum, size_t spectrum_bytes,
                                   const float* sc_w, const float* sc_bias, int64_t B, int64_t C, int order,
                                   uint64_t wait_budget_ns, int issue_mma, void* stream) {
    Plan p;
    ConvArgs a;
    const int64_t L = 8192;
    hyena_status_t st = prepare_conv(u, y, spectrum, spectrum_bytes, sc_w, sc_bias, B, C, 1, &L, order, HYENA_BF16,
                                     nullptr, 0, &p, &a);
    if (st != HYENA_OK) return st;
    if (order > kMaxOrderTc)
        return fail(HYENA_ERR_UNSUPPORTED_SHAPE, "the tensor-core kernel serves order <= " + std::to_string(kMaxOrderTc));
    if (wait_budget_ns == 0) return fail(HYENA_ERR_INVALID_ARG, "wait_budget_ns must be > 0");
    a.wait_budget_ns = wait_budget_ns;
    a.issue_mma = issue_mma ? 1 : 0;
    cudaError_t e = kernel_status_word(&a.status);
    if (e != cudaSuccess) return cuda_status(e, "kernel status word");
    return cuda_status(launch_conv_8192_tc(p, a, static_cast<cudaStream_t>(stream)), "tensor-core kernel");
}

hyena_status_t hyena_debug_conv_cluster(const void* u, void* y, const void* spectrum, size_t spectrum_bytes,
                                        const float* sc_w, const float* sc_bias, int64_t B, int64_t C, int order,
                                        void* workspace, size_t workspace_bytes, uint64_t wait_budget_ns,
                                        int issue_mma, void* stream) {
    Plan p;
    ConvArgs a;
    const int64_t L = kClusterL;
    hyena_status_t st = prepare_conv(u, y, spectrum, spectrum_bytes, sc_w, sc_bias, B, C, 1, &L, order, HYENA_BF16,
                                     workspace, workspace_bytes, &p, &a);
    if (st != HYENA_OK) return st;
    if (!cluster_path(p, a))
        return fail(HYENA_ERR_UNSUPPORTED_SHAPE, "the cluster kernel serves order <= " + std::to_string(kMaxOrderTc));
    if (wait_budget_ns == 0) return fail(HYENA_ERR_INVALID_ARG, "wait_budget_ns must be > 0");
    a.wait_budget_ns = wait_budget_ns;
    a.issue_mma = issue_mma ? 1 : 0;
    cudaError_t e = kernel_status_word(&a.status);
    if (e != cudaSuccess) return cuda_status(e, "kernel status word");
    return cuda_status(launch_conv_cluster(p, a, size_t(a.group_rows) * p.ws_row_bytes, static_cast<cudaStream_t>(stream)),
                       "cluster kernel");
}

hyena_status_t hyena_debug_conv_2d_tc(const void* u, void* y, const void* spectrum, size_t spectrum_bytes, int64_t B,
                                      int64_t C, int64_t W, int order, void* workspace, size_t workspace_bytes,
                                      uint64_t wait_budget_ns, int issue_mma, void* stream) {
    Plan p;
    ConvArgs a;
    const int64_t sizes[2] = {kTc2dH, W};
    hyena_status_t st = prepare_conv(u, y, spectrum, spectrum_bytes, nullptr, nullptr, B, C, 2, sizes, order, HYENA_BF16,
                                     workspace, workspace_bytes, &p, &a);
    if (st != HYENA_OK) return st;
    if (!cols_2d_tc_path(p, a))
        return fail(HYENA_ERR_UNSUPPORTED_SHAPE, "the 2-D tensor-core column pass serves H = 256, W a multiple of 32");
    if (wait_budget_ns == 0) return fail(HYENA_ERR_INVALID_ARG, "wait_budget_ns must be > 0");
    a.wait_budget_ns = wait_budget_ns;
    a.issue_mma = issue_mma ? 1 : 0;
    cudaError_t e = kernel_status_word(&a.status);
    if (e != cudaSuccess) return cuda_status(e, "kernel status word");
    return cuda_status(launch_conv_2d(p, a, static_cast<cudaStream_t>(stream)), "2-D convolution");
}

hyena_status_t hyena_debug_conv_2dc_tc(const void* u, void* y, const void* spectrum, size_t spectrum_bytes, int64_t B,
                                       int64_t C, int order, void* workspace, size_t workspace_bytes,
                                       uint64_t wait_budget_ns, int issue_mma, void* stream) {
    Plan p;
    ConvArgs a;
    const int64_t sizes[2] = {kTc2dH, kTc2dH};
    hyena_status_t st = prepare_conv(u, y, spectrum, spectrum_bytes, nullptr, nullptr, B, C, 2 | kCircularFlag, sizes,
                                     order, HYENA_BF16, workspace, workspace_bytes, &p, &a);
    if (st != HYENA_OK) return st;
    if (!pairs_2dc_tc_path(p, a))
        return fail(HYENA_ERR_UNSUPPORTED_SHAPE,
                    "the circular tensor-core passes serve 256 x 256, an even batch and order <= 3");
    if (wait_budget_ns == 0) return fail(HYENA_ERR_INVALID_ARG, "wait_budget_ns must be > 0");
    a.wait_budget_ns = wait_budget_ns;
    a.issue_mma = issue_mma ? 1 : 0;
    cudaError_t e = kernel_status_word(&a.status);
    if (e != cudaSuccess) return cuda_status(e, "kernel status word");
    return cuda_status(launch_conv_2d(p, a, static_cast<cudaStream_t>(stream)), "2-D convolution");
}

}  // extern "C"

namespace {

// Per-device second stream and events of the host-buffer pipeline, created
// on first use and kept for the life of the process.
struct HostPipe {
    cudaStream_t aux = nullptr;
    cudaEvent_t entry = nullptr, aux_done = nullptr, conv_done[2] = {nullptr, nullptr};
};
constexpr int kMaxPipeDevices = 64;
std::mutex g_pipe_mutex;
HostPipe g_pipe[kMaxPipeDevices];

cudaError_t host_pipe(int dev, HostPipe** out) {
    HostPipe& hp = g_pipe[dev];
    if (!hp.aux) {
        cudaError_t e = cudaStreamCreateWithFlags(&hp.aux, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hp.entry, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hp.aux_done, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hp.conv_done[0], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hp.conv_done[1], cudaEventDisableTiming);
        if (e != cudaSuccess) return e;
    }
    *out = &hp;
    return cudaSuccess;
}

}  // namespace

extern "C" {

hyena_status_t hyena_gated_fftconv_host(const void* u_host, void* y_host, void* u_dev, void* y_dev,
                                        const void* spectrum, size_t spectrum_bytes, const float* sc_w,
                                        const float* sc_bias, int64_t B, int64_t C, int ndim, const int64_t* sizes,
                                        int order, hyena_dtype_t dtype, void* workspace, size_t workspace_bytes,
                                        int64_t chunk_rows, void* stream) {
    Plan p;
    ConvArgs a;
    hyena_status_t st = prepare_conv(u_dev, y_dev, spectrum, spectrum_bytes, sc_w, sc_bias, B, C, ndim, sizes, order,
                                     dtype, workspace, workspace_bytes, &p, &a);
    if (st != HYENA_OK) return st;
    if (!u_host || !y_host) return fail(HYENA_ERR_INVALID_ARG, "u_host and y_host must not be NULL");
    if (chunk_rows < 0) return fail(HYENA_ERR_INVALID_ARG, "chunk_rows must be >= 0 (0: default)");
    int64_t chunk = chunk_rows > 0 ? (chunk_rows < B ? chunk_rows : B) : (B + 3) / 4;
    // default: an even number of batch rows, so that the L = 8192 bf16 kernel,
    // which transforms two batch rows of a channel together, never pairs a
    // row with zeros
    if (chunk_rows == 0 && (chunk & 1) && chunk < B) ++chunk;
    const size_t es = elem_size(dtype);
    const size_t ub = size_t(order + 1) * size_t(C) * size_t(p.n) * es;    // u bytes per batch row
    const size_t yb = size_t(C) * size_t(p.n) * es;                        // y bytes per batch row
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_status(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxPipeDevices) return fail(HYENA_ERR_INVALID_ARG, "device index beyond 64");
    std::lock_guard<std::mutex> lock(g_pipe_mutex);
    HostPipe* hp = nullptr;
    e = host_pipe(dev, &hp);
    if (e != cudaSuccess) return cuda_status(e, "host pipeline set-up");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaStream_t streams[2] = {s, hp->aux};
    // the second stream starts after the work already queued on the caller's stream
    e = cudaEventRecord(hp->entry, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(hp->aux, hp->entry, 0);
    const uint8_t* uh = static_cast<const uint8_t*>(u_host);
    uint8_t* yh = static_cast<uint8_t*>(y_host);
    uint8_t* ud = static_cast<uint8_t*>(u_dev);
    uint8_t* yd = static_cast<uint8_t*>(y_dev);
    int i = 0;
    for (int64_t b0 = 0; b0 < B && e == cudaSuccess; b0 += chunk, ++i) {
        const int64_t nb = B - b0 < chunk ? B - b0 : chunk;
        cudaStream_t cs = streams[i & 1];
        e = cudaMemcpyAsync(ud + b0 * ub, uh + b0 * ub, nb * ub, cudaMemcpyHostToDevice, cs);
        // chunks share the workspace: their convolutions run one after another
        if (e == cudaSuccess && i > 0 && p.ws_row_bytes > 0) e = cudaStreamWaitEvent(cs, hp->conv_done[(i - 1) & 1], 0);
        if (e != cudaSuccess) break;
        st = gated_fftconv(ud + b0 * ub, yd + b0 * yb, spectrum, spectrum_bytes, sc_w, sc_bias, nb, C, ndim, sizes,
                           order, dtype, workspace, workspace_bytes, cs, false);
        if (st != HYENA_OK) break;
        e = cudaEventRecord(hp->conv_done[i & 1], cs);
        if (e == cudaSuccess) e = cudaMemcpyAsync(yh + b0 * yb, yd + b0 * yb, nb * yb, cudaMemcpyDeviceToHost, cs);
    }
    // the caller's stream completes after every chunk queued on the second
    // stream, also when queueing stopped early on an error
    cudaError_t ej = cudaEventRecord(hp->aux_done, hp->aux);
    if (ej == cudaSuccess) ej = cudaStreamWaitEvent(s, hp->aux_done, 0);
    if (st != HYENA_OK) return st;
    if (e == cudaSuccess) e = ej;
    return cuda_status(e, "host pipeline");
}

hyena_status_t hyena_spectrum_check(const void* spectrum, int64_t C, int ndim, const int64_t* sizes, int order,
                                    void* stream) {
    Plan p;
    hyena_status_t st = plan_or_fail(C, ndim, sizes, order, &p);
    if (st != HYENA_OK) return st;
    if (!spectrum) return fail(HYENA_ERR_INVALID_ARG, "spectrum must not be NULL");
    SpecHeader h{};
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(&h, spectrum, sizeof(h), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_status(e, "header read");
    if (h.magic != kSpecMagic || h.version != kSpecVersion || h.path != p.path || h.C != p.C || h.L != p.L ||
        h.H != p.H || h.W != p.W || h.order != p.order || size_t(h.total_bytes) != p.total_bytes)
        return fail(HYENA_ERR_SPECTRUM_MISMATCH, "spectrum header does not match (C, sizes, order)");
    return ok();
}

}  // extern "C"
