// filtergen.cu -- the implicit long filter generated on the GPU and fed
// straight into the filter-spectrum build (hyena_filter_spectrum_implicit).
//
// HyenaDNA operator walk-through (adg.csdn.net), section 二.2, HyenaFilter:
//   filter(L) = modulation(t, implicit_filter(pos_emb(L)))
//   pos_emb          z[l] = [t_l, cos(2 pi b l / L), sin(2 pi b l / L)],
//                    b = 1 .. (emb_dim-1)/2, t_l = l / (L-1)
//   implicit_filter  Linear(emb_dim, width) -> Sin, then num_inner x
//                    (Linear(width, width) -> Sin), then Linear(width,
//                    d_model) without bias; Sin(x) = sin(w * x) with a
//                    per-feature frequency vector w
//   modulation       h[l][c] * exp(-alpha[c] t_l)
// and section 二.1 takes the d_model = (order-1) C outputs as
// 'l (o d) -> o d l': filter row s*C + c is output channel s*C + c.
//
// Two launches: k_filter_hidden evaluates the embedding and the hidden layers
// once for every t (shared by all channels) into hT [width][L] in the
// caller's workspace; the spectrum kernel of the on-chip path then computes
// each row's samples k[t] = exp(-alpha t_l) sum_j hT[j][t] W_out[row][j]
// directly into its FFT buffer, so the filters themselves never go to global
// memory (unless the caller asks for a copy).
#include <cuda_runtime.h>

#include <string>

#include "hyena.h"
#include "kernels.h"
#include "plan.h"

namespace hyena {

hyena_status_t set_last_error_detail(hyena_status_t st, const std::string& detail);  // api.cu

namespace {

constexpr int kMaxWidth = 128;
constexpr int kMaxEmb = 33;
constexpr int kMaxInner = 8;
constexpr int kTT = 32;            // time steps per block
constexpr int kThreadsH = 128;     // thread j computes feature j (j < width)

// Dynamic shared memory: WT [max(emb, width)][width + 1] (a layer's weight,
// transposed), h [2][kTT][width + 1], z [kTT][emb_dim].
__global__ void __launch_bounds__(kThreadsH)
k_filter_hidden(ImplicitMlp m, int64_t L, float* __restrict__ hT) {
    extern __shared__ float sm[];
    const int W = m.width, E = m.emb_dim, WP = W + 1;
    const int rows = E > W ? E : W;
    float* WT = sm;
    float* h0 = WT + rows * WP;
    float* h1 = h0 + kTT * WP;
    float* z = h1 + kTT * WP;
    const int64_t t0 = int64_t(blockIdx.x) * kTT;
    const int j = int(threadIdx.x);
    // positional embedding of the tile's time steps
    const int nb = (E - 1) / 2;
    for (int idx = j; idx < kTT * E; idx += kThreadsH) {
        const int tt = idx / E, f = idx % E;
        const int64_t l = t0 + tt;
        float v = 0.0f;
        if (l < L) {
            if (f == 0) {
                v = float(l) / float(L - 1);
            } else {
                const int b = f <= nb ? f : f - nb;
                // angle 2 pi b l / L, reduced exactly: sincospi of (2 b l mod 2L) / L
                const int64_t r = (2 * int64_t(b) * l) % (2 * L);
                float sv, cv;
                sincospif(float(r) / float(L), &sv, &cv);
                v = f <= nb ? cv : sv;
            }
        }
        z[tt * E + f] = v;
    }
    // first layer: h = Sin(W_in z + b_in)
    for (int idx = j; idx < W * E; idx += kThreadsH) {
        const int o = idx / E, i = idx % E;
        WT[i * WP + o] = __ldg(m.W_in + idx);
    }
    __syncthreads();
    const float wj = j < W ? __ldg(m.w + j) : 0.0f;
    if (j < W) {
        const float bj = __ldg(m.b_in + j);
        float acc[kTT];
#pragma unroll
        for (int tt = 0; tt < kTT; ++tt) acc[tt] = bj;
        for (int i = 0; i < E; ++i) {
            const float wv = WT[i * WP + j];
#pragma unroll
            for (int tt = 0; tt < kTT; ++tt) acc[tt] = fmaf(wv, z[tt * E + i], acc[tt]);
        }
#pragma unroll
        for (int tt = 0; tt < kTT; ++tt) h0[tt * WP + j] = sinf(wj * acc[tt]);
    }
    float* cur = h0;
    float* nxt = h1;
    // inner layers: h = Sin(W h + b)
    for (int layer = 0; layer < m.num_inner; ++layer) {
        __syncthreads();                               // previous layer done with WT and cur complete
        const float* Wl = m.W_inner + int64_t(layer) * W * W;
        for (int idx = j; idx < W * W; idx += kThreadsH) {
            const int o = idx / W, i = idx % W;
            WT[i * WP + o] = __ldg(Wl + idx);
        }
        __syncthreads();
        if (j < W) {
            const float bj = __ldg(m.b_inner + int64_t(layer) * W + j);
            float acc[kTT];
#pragma unroll
            for (int tt = 0; tt < kTT; ++tt) acc[tt] = bj;
            for (int i = 0; i < W; ++i) {
                const float wv = WT[i * WP + j];
#pragma unroll
                for (int tt = 0; tt < kTT; ++tt) acc[tt] = fmaf(wv, cur[tt * WP + i], acc[tt]);
            }
#pragma unroll
            for (int tt = 0; tt < kTT; ++tt) nxt[tt * WP + j] = sinf(wj * acc[tt]);
        }
        float* sw = cur;
        cur = nxt;
        nxt = sw;
    }
    __syncthreads();
    // hT[f][t] for the tile (consecutive t per feature row)
    for (int idx = j; idx < W * kTT; idx += kThreadsH) {
        const int f = idx / kTT, tt = idx % kTT;
        if (t0 + tt < L) hT[int64_t(f) * L + t0 + tt] = cur[tt * WP + f];
    }
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

cudaError_t launch_filter_hidden(const ImplicitMlp& m, int64_t L, float* hT, cudaStream_t s) {
    const int rows = m.emb_dim > m.width ? m.emb_dim : m.width;
    const size_t smem = (size_t(rows) * (m.width + 1) + size_t(2) * kTT * (m.width + 1) + size_t(kTT) * m.emb_dim) * 4;
    cudaError_t e = cudaFuncSetAttribute(k_filter_hidden, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    const unsigned grid = unsigned((L + kTT - 1) / kTT);
    k_filter_hidden<<<grid, kThreadsH, smem, s>>>(m, L, hT);
    return cudaGetLastError();
}

}  // namespace hyena

using namespace hyena;

extern "C" size_t hyena_implicit_filter_workspace_bytes(int64_t L, int width) {
    if (L < 2 || width < 1 || width > kMaxWidth) return 0;
    return size_t(L) * size_t(width) * 4;
}

extern "C" hyena_status_t hyena_filter_spectrum_implicit(const hyena_implicit_filter_t* f, const float* D, int64_t C,
                                                         int64_t L, int order, void* spectrum, size_t spectrum_bytes,
                                                         void* workspace, size_t workspace_bytes, float* k_out,
                                                         void* stream) {
    if (!f) return set_last_error_detail(HYENA_ERR_INVALID_ARG, "the filter parameters must not be NULL");
    if (f->emb_dim < 3 || f->emb_dim % 2 == 0 || f->emb_dim > kMaxEmb)
        return set_last_error_detail(HYENA_ERR_INVALID_ARG, "emb_dim must be odd, in [3, 33]");
    if (f->width < 1 || f->width > kMaxWidth)
        return set_last_error_detail(HYENA_ERR_INVALID_ARG, "width must be in [1, 128]");
    if (f->num_inner < 0 || f->num_inner > kMaxInner)
        return set_last_error_detail(HYENA_ERR_INVALID_ARG, "num_inner must be in [0, 8]");
    if (!f->W_in || !f->b_in || !f->W_out || !f->w || !f->alpha || (f->num_inner > 0 && (!f->W_inner || !f->b_inner)))
        return set_last_error_detail(HYENA_ERR_INVALID_ARG, "a filter parameter pointer is NULL");
    if (!spectrum || !workspace) return set_last_error_detail(HYENA_ERR_INVALID_ARG, "spectrum and workspace must not be NULL");
    const void* ptrs[] = {f->W_in, f->b_in, f->W_out, f->w, f->alpha, f->W_inner, f->b_inner, D, k_out};
    for (const void* q : ptrs)
        if (q && !aligned(q, 4)) return set_last_error_detail(HYENA_ERR_MISALIGNED, "parameters must be 4-byte aligned");
    if (k_out && !aligned(k_out, 8)) return set_last_error_detail(HYENA_ERR_MISALIGNED, "k_out must be 8-byte aligned");
    if (!aligned(spectrum, 16) || !aligned(workspace, 16))
        return set_last_error_detail(HYENA_ERR_MISALIGNED, "spectrum and workspace must be 16-byte aligned");
    Plan p;
    std::string why;
    const int64_t sizes[1] = {L};
    if (C < 1) return set_last_error_detail(HYENA_ERR_INVALID_ARG, "C must be >= 1");
    if (!make_plan(C, 1, sizes, order, &p, &why)) return set_last_error_detail(HYENA_ERR_UNSUPPORTED_SHAPE, why);
    if (p.path != PATH_ONCHIP_1D)
        return set_last_error_detail(HYENA_ERR_UNSUPPORTED_SHAPE, "implicit filters: L must be in [16, 16384]");
    if (spectrum_bytes != p.total_bytes)
        return set_last_error_detail(HYENA_ERR_SPECTRUM_MISMATCH, "spectrum_bytes must equal hyena_spectrum_bytes() = " +
                                                                      std::to_string(p.total_bytes));
    const size_t need = hyena_implicit_filter_workspace_bytes(L, f->width);
    if (workspace_bytes < need)
        return set_last_error_detail(HYENA_ERR_WORKSPACE_TOO_SMALL,
                                     "workspace must hold " + std::to_string(need) + " bytes (width x L fp32)");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* sp = static_cast<uint8_t*>(spectrum);
    float* hT = static_cast<float*>(workspace);
    cudaError_t e = launch_header_and_tables(p, sp, s);
    const ImplicitMlp m{f->emb_dim, f->width, f->num_inner, f->W_in, f->b_in, f->W_inner, f->b_inner, f->w};
    if (e == cudaSuccess) e = launch_filter_hidden(m, L, hT, s);
    if (e == cudaSuccess) {
        SpectrumArgs a{nullptr, 0, D, sp};
        a.implicit = true;
        a.imp.hT = hT;
        a.imp.W_out = f->W_out;
        a.imp.alpha = f->alpha;
        a.imp.k_out = k_out;
        a.imp.width = f->width;
        e = launch_spectrum_onchip(p, a, s);
    }
    if (e != cudaSuccess)
        return set_last_error_detail(HYENA_ERR_CUDA, std::string("implicit filter spectrum: ") + cudaGetErrorString(e));
    return set_last_error_detail(HYENA_OK, "");
}
