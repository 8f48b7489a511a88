// noalloc.cu -- hyena_gated_fftconv_noalloc: the gated FFT convolution for
// callers that cannot allocate device memory.
//
// Some callers have no way to obtain a workspace: a plugin whose host
// framework owns every device allocation, or a serving loop that must never
// call cudaMalloc (it can block, synchronise the device, or fail under memory
// pressure at a point where the request cannot be dropped).  For them this
// entry point uses a fixed scratch array that is part of the library image
// instead of a caller workspace.  The caller still passes u, y and the
// spectrum.
//
// The array is a file-scope __device__ object of HYENA_NOALLOC_SCRATCH_BYTES
// (32 MiB); every GPU that loads the library keeps it until the process
// exits.  Its device address is looked up once per device with
// cudaGetSymbolAddress (host code may not use the array's name as a device
// pointer) and cached for the life of the process, so calls after a reset of
// the device (which may move the array) are not supported.  Nothing here
// allocates or frees memory.
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "hyena.h"
#include "plan.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[HYENA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

}  // namespace

namespace hyena {
hyena_status_t set_last_error_detail(hyena_status_t st, const std::string& detail);  // api.cu
}

extern "C" hyena_status_t hyena_gated_fftconv_noalloc(const void* u, void* y, const void* spectrum,
                                                      size_t spectrum_bytes, const float* sc_w,
                                                      const float* sc_bias, int64_t B, int64_t C, int ndim,
                                                      const int64_t* sizes, int order, hyena_dtype_t dtype,
                                                      void* stream) {
    // Shapes whose workspace row does not fit the fixed scratch are rejected
    // before anything else happens.
    const size_t row = hyena_gated_fftconv_workspace_min_bytes(C, ndim, sizes, order);
    if (row > size_t(HYENA_NOALLOC_SCRATCH_BYTES)) {
        return hyena::set_last_error_detail(
            HYENA_ERR_WORKSPACE_TOO_SMALL,
            "this shape needs " + std::to_string(row) + " bytes of scratch per row; the fixed scratch of "
            "hyena_gated_fftconv_noalloc holds " + std::to_string(size_t(HYENA_NOALLOC_SCRATCH_BYTES)) +
            " bytes (use hyena_gated_fftconv with a workspace)");
    }
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        return hyena::set_last_error_detail(HYENA_ERR_CUDA,
                                            std::string("cudaGetDevice failed: ") + cudaGetErrorString(e));
    }
    if (dev < 0 || dev >= kMaxDevices) {
        return hyena::set_last_error_detail(HYENA_ERR_INVALID_ARG, "device index beyond the supported 64 devices");
    }
    void* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (!g_scratch_ptr[dev]) {
            // first call on this device: look up the array's device address
            // with this device current (may load the library's device code)
            void* p = nullptr;
            e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
            if (e != cudaSuccess || !p) {
                return hyena::set_last_error_detail(
                    HYENA_ERR_CUDA, std::string("cudaGetSymbolAddress failed: ") + cudaGetErrorString(e));
            }
            g_scratch_ptr[dev] = p;
        }
        scratch = g_scratch_ptr[dev];
    }
    return hyena_gated_fftconv(u, y, spectrum, spectrum_bytes, sc_w, sc_bias, B, C, ndim, sizes, order, dtype,
                               scratch, size_t(HYENA_NOALLOC_SCRATCH_BYTES), stream);
}
