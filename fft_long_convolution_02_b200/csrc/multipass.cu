// multipass.cu -- placeholder launchers (implemented below in this file).
#include "kernels.h"
namespace hyena {
cudaError_t launch_spectrum_multipass(const Plan&, const SpectrumArgs&, cudaStream_t) { return cudaErrorNotSupported; }
cudaError_t launch_conv_multipass(const Plan&, const ConvArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}
