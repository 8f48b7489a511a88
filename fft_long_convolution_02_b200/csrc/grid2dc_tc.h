// grid2dc_tc.h -- launchers of the circular 2-D form's tensor-core passes
// (grid2d_tc.cu): 256 x 256 images, bf16 storage, an even batch (the two
// images of a channel paired into one complex image), orders up to
// kMaxOrderTc.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"
#include "plan.h"

namespace hyena {

// Whether a circular 2-D call takes the paired tensor-core passes.
bool pairs_2dc_tc_path(const Plan& p, const ConvArgs& a);
// The full H x W spectrum plane (bf16 pairs, column-pass thread order) from
// the complex64 spectrum rows of the circular form.
cudaError_t launch_spectrum_2dc_tc_plane(const Plan& p, const uint8_t* spectrum_rows, uint8_t* plane, int64_t nrows,
                                         cudaStream_t s);
// All order steps of images img0 .. img0+nimg-1 (both even), workspace image
// stride ws_img_stride bf16 pairs (a pair's 256 x 256 bins fit two strides).
cudaError_t launch_conv_2dc_pairs_tc(const Plan& p, const ConvArgs& a, void* ws, int64_t img0, int64_t nimg,
                                     int64_t ws_img_stride, cudaStream_t s);

}  // namespace hyena
