// grid2d.cu -- placeholder launchers.
#include "kernels.h"
namespace hyena {
cudaError_t launch_spectrum_2d(const Plan&, const SpectrumArgs&, cudaStream_t) { return cudaErrorNotSupported; }
cudaError_t launch_conv_2d(const Plan&, const ConvArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}
