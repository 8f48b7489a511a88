// plan_common.h -- compile-time and run-time description of the FFT
// factorisations, shared by host planning code and device kernels.
#pragma once
#include <stdint.h>

#if defined(__CUDACC__)
#define HYENA_HD __host__ __device__
#else
#define HYENA_HD
#endif

namespace hyena {

HYENA_HD constexpr int ilog2c(int64_t x) { return x <= 1 ? 0 : 1 + ilog2c(x >> 1); }

// M = 16^a * r0, r0 in {1, 2, 4, 8}; DIF stage order: a radix-16 stages, then r0.
HYENA_HD constexpr int fft_n16(int M) { return ilog2c(M) / 4; }
HYENA_HD constexpr int fft_r0(int M) { return 1 << (ilog2c(M) % 4); }
HYENA_HD constexpr int fft_nstages(int M) { return fft_n16(M) + (fft_r0(M) > 1 ? 1 : 0); }
HYENA_HD constexpr int fft_stage_radix(int M, int i) { return i < fft_n16(M) ? 16 : fft_r0(M); }
HYENA_HD constexpr int fft_stage_len(int M, int i) { return M >> (4 * i); }
HYENA_HD constexpr int fft_stage_stride(int M, int i) { return fft_stage_len(M, i) / fft_stage_radix(M, i); }
HYENA_HD constexpr int fft_stage_tw_count(int M, int i) {
    return fft_stage_stride(M, i) > 1 ? (fft_stage_radix(M, i) - 1) * fft_stage_stride(M, i) : 0;
}
HYENA_HD constexpr int fft_stage_tw_offset(int M, int i) {
    return i <= 0 ? 0 : fft_stage_tw_offset(M, i - 1) + fft_stage_tw_count(M, i - 1);
}
HYENA_HD constexpr int fft_tw_size(int M) { return fft_stage_tw_offset(M, fft_nstages(M)); }

}  // namespace hyena
