// kernels.h -- internal launcher declarations (host side).  Every launcher
// enqueues on the given stream and returns cudaGetLastError().
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "plan.h"

namespace hyena {

enum DType { DT_F32 = 0, DT_BF16 = 1 };

// Default budget of a bounded device wait: far above a normal wait (us), and
// long enough to ride out time-slicing with other contexts on a shared GPU.
constexpr uint64_t kDefaultWaitBudgetNs = 2000000000ull;

// Bits of the per-device kernel status word (status.cu, hyena_kernel_status).
constexpr uint32_t kStatusTimeout = 1u;            // a bounded tensor-core wait ran out
constexpr uint32_t kStatusSpectrumMismatch = 2u;   // spectrum header does not match the launch

// Device address of this device's kernel status word (looked up once per device).
cudaError_t kernel_status_word(uint32_t** out);

// Records a kernel-detected condition in the status word (one thread per CTA).
__device__ __forceinline__ void report_status(uint32_t* status, uint32_t bit) {
    if (status) atomicOr(status, bit);
}

// The implicit long filter (HyenaFilter): row r = s*C + c of the filters is
// k[t] = exp(-alpha[r] t / (L-1)) * sum_j hT[j][t] W_out[r][j], where hT is
// the last hidden layer of the filter MLP, transposed ([width][L]).
struct ImplicitFilter {
    const float* hT = nullptr;
    const float* W_out = nullptr;   // [(order-1) C][width]
    const float* alpha = nullptr;   // [(order-1) C]
    float* k_out = nullptr;         // [(order-1) C][L] copy of the generated filters, or nullptr
    int width = 0;
};

struct SpectrumArgs {
    const void* k;        // [order-1, C, n]
    int k_dtype;
    const float* D;       // [order-1, C] or nullptr
    uint8_t* spectrum;    // buffer start (header at offset 0)
    // set: the filters are generated (k unused); 1-D on-chip lengths only
    bool implicit = false;
    ImplicitFilter imp{};
};

struct ConvArgs {
    const void* u;        // [B, (order+1)*C, n]
    void* y;              // [B, C, n]
    const uint8_t* spectrum;
    const float* sc_w;    // [(order+1)*C, 3] or nullptr
    const float* sc_b;    // [(order+1)*C] or nullptr
    int64_t B;
    int dtype;
    float2* workspace;    // multi-pass / 2-D only
    int64_t group_rows;   // rows per workspace group
    // L = 8192 tensor-core kernel only: budget of each bounded wait, and whether
    // the tensor-core work is issued (0 only from the timeout test hook)
    uint64_t wait_budget_ns = kDefaultWaitBudgetNs;
    int issue_mma = 1;
    // spectrum row of (order step s, b, c) = s * spec_C + b * spec_per_b + c:
    // (C, 0) for filters shared over the batch, (B*C, C) for per-sample filters
    int64_t spec_C = 0;
    int64_t spec_per_b = 0;
    // kernel status word of this device (kStatus* bits)
    uint32_t* status = nullptr;
    // bf16 storage: run the fp32 CUDA-core transforms instead of the
    // tensor-core ones (HYENA_FLAG_FP32_TRANSFORM)
    bool fp32_transform = false;
    // 2-D, H = 256: offset of the tensor-core column pass's spectrum plane in
    // this spectrum (from the plan of its own filter count: C, or B*C per sample)
    size_t g2_plane_off = 0;
};

cudaError_t launch_header_and_tables(const Plan& p, uint8_t* spectrum, cudaStream_t s);
cudaError_t launch_spectrum_onchip(const Plan& p, const SpectrumArgs& a, cudaStream_t s);
cudaError_t launch_conv_onchip(const Plan& p, const ConvArgs& a, cudaStream_t s);
cudaError_t launch_conv_8192_tc(const Plan& p, const ConvArgs& a, cudaStream_t s);
constexpr int kMaxOrderTc = 3;   // highest order the L = 8192 tensor-core kernel serves
cudaError_t launch_spectrum_multipass(const Plan& p, const SpectrumArgs& a, cudaStream_t s);
cudaError_t launch_conv_multipass(const Plan& p, const ConvArgs& a, cudaStream_t s);
// L = 65536, bf16 storage (cluster.cu): the cluster plane of the spectrum, and
// the convolution on 8-CTA clusters with workspace_bytes of scratch (512 KB
// per cluster in flight).
cudaError_t launch_spectrum_cluster(const Plan& p, const SpectrumArgs& a, cudaStream_t s);
bool cluster_path(const Plan& p, const ConvArgs& a);
cudaError_t launch_conv_cluster(const Plan& p, const ConvArgs& a, size_t workspace_bytes, cudaStream_t s);
cudaError_t launch_spectrum_2d(const Plan& p, const SpectrumArgs& a, cudaStream_t s);
// 2-D with bf16 storage and H = 256 (grid2d_tc.cu): the column pass of columns
// 0 .. W-1 on the tensor cores, and its spectrum plane from the complex64 rows.
bool cols_2d_tc_path(const Plan& p, const ConvArgs& a);
cudaError_t launch_cols_2d_tc(const Plan& p, const ConvArgs& a, void* ws, int64_t img0, int64_t nimg, int step,
                              int64_t ws_img_stride, cudaStream_t s);
cudaError_t launch_spectrum_2d_tc_plane(const Plan& p, const uint8_t* spectrum_rows, uint8_t* plane, int64_t nrows,
                                        cudaStream_t s);
// 256 x 256 images, even B, shared filters: the two images of a
// channel as one complex image, all three passes on the tensor cores
bool pairs_2d_tc_path(const Plan& p, const ConvArgs& a);
cudaError_t launch_conv_2d_pairs_tc(const Plan& p, const ConvArgs& a, void* ws, int64_t img0, int64_t nimg,
                                    int64_t ws_img_stride, cudaStream_t s);
cudaError_t launch_conv_2d(const Plan& p, const ConvArgs& a, cudaStream_t s);
cudaError_t launch_spectrum_3d(const Plan& p, const SpectrumArgs& a, cudaStream_t s);
cudaError_t launch_conv_3d(const Plan& p, const ConvArgs& a, cudaStream_t s);
// Hidden layers of the implicit filter MLP for t < L -> hT [width][L] (filtergen.cu).
struct ImplicitMlp {
    int emb_dim, width, num_inner;
    const float *W_in, *b_in, *W_inner, *b_inner, *w;
};
cudaError_t launch_filter_hidden(const ImplicitMlp& m, int64_t L, float* hT, cudaStream_t s);
cudaError_t launch_shortconv(const void* u, void* out, const float* w, const float* bias, int64_t B,
                             int64_t Ctot, int64_t L, int dtype, cudaStream_t s);

}  // namespace hyena
