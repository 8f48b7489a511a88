// status.cu -- the per-device status word that convolution kernels use to
// report what they detect on the device, and hyena_kernel_status, which
// reads and clears it.
//
// A kernel cannot return an error code, and the entry points return before
// their kernels run.  So the kernels OR a bit into one word in device memory
// (a file-scope __device__ variable: no allocation), and the caller reads it
// when convenient:
//   bit 0  a bounded wait for tensor-core work ran out (the outputs of the
//          row pair it was on are NaN; nothing was left in flight)
//   bit 1  a convolution kernel found a spectrum whose header does not match
//          the shape it was launched for (that kernel wrote no output)
// The bits are sticky until hyena_kernel_status clears them.  Kernels in the
// other translation units get the word's device address as an argument; it
// is looked up once per device (cudaGetSymbolAddress with that device
// current) and kept for the life of the process.
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "hyena.h"
#include "kernels.h"

namespace {

static __device__ uint32_t g_kernel_status;

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
uint32_t* g_word[kMaxDevices] = {};

}  // namespace

namespace hyena {

hyena_status_t set_last_error_detail(hyena_status_t st, const std::string& detail);  // api.cu

cudaError_t kernel_status_word(uint32_t** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_word[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_kernel_status);
        if (e != cudaSuccess) return e;
        g_word[dev] = static_cast<uint32_t*>(p);
    }
    *out = g_word[dev];
    return cudaSuccess;
}

}  // namespace hyena

extern "C" hyena_status_t hyena_kernel_status(void* stream) {
    uint32_t* word = nullptr;
    cudaError_t e = hyena::kernel_status_word(&word);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t bits = 0;
    const uint32_t zero = 0;
    if (e == cudaSuccess) e = cudaMemcpyAsync(&bits, word, sizeof(bits), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(word, &zero, sizeof(zero), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess)
        return hyena::set_last_error_detail(HYENA_ERR_CUDA, std::string("status read: ") + cudaGetErrorString(e));
    if (bits & hyena::kStatusTimeout)
        return hyena::set_last_error_detail(HYENA_ERR_TIMEOUT,
                                            "a bounded wait for tensor-core work ran out; the outputs of that row "
                                            "pair were written as NaN");
    if (bits & hyena::kStatusSpectrumMismatch)
        return hyena::set_last_error_detail(HYENA_ERR_SPECTRUM_MISMATCH,
                                            "a convolution kernel found a spectrum header that does not match its "
                                            "shape (never filled, or filled for another C, size or order); its "
                                            "output was not written");
    return hyena::set_last_error_detail(HYENA_OK, "");
}
