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
constexpr int kTT = 64;            // time steps per block
constexpr int kThreadsH = 128;     // 16 feature groups of 4 x 8 time groups of 8

// One layer of the MLP on a tile of kTT time steps: out[j][t] = sin(w[j] *
// (bias[j] + sum_i WT[i][j] in[i][t])) for j < W, with WT [K][WP4] (the
// weight transposed, rows padded to a multiple of 4) and in/out [.][kTT]
// (feature-major).  Thread (jg, tg) computes features 4 jg + 64 r (r <
// ceil(W / 64)) at time steps 8 tg .. 8 tg + 7 as a 4 x 8 register tile.
__device__ __forceinline__ void mlp_layer(const float* WT, int WP4, const float* in, int K, const float* bias,
                                          const float* w, int W, float* out) {
    const int jg = int(threadIdx.x) & 15, tg = int(threadIdx.x) >> 4;
    for (int j0 = 4 * jg; j0 < W; j0 += 64) {
        float acc[4][8];
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            const float b = j0 + a < W ? __ldg(bias + j0 + a) : 0.0f;
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[a][e] = b;
        }
        for (int i = 0; i < K; ++i) {
            const float4 wv = *reinterpret_cast<const float4*>(WT + i * WP4 + j0);
            const float4 h0 = *reinterpret_cast<const float4*>(in + i * kTT + 8 * tg);
            const float4 h1 = *reinterpret_cast<const float4*>(in + i * kTT + 8 * tg + 4);
            const float ww[4] = {wv.x, wv.y, wv.z, wv.w};
            const float hh[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[a][e] = fmaf(ww[a], hh[e], acc[a][e]);
        }
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            if (j0 + a >= W) continue;
            const float wj = __ldg(w + j0 + a);
            float4* o = reinterpret_cast<float4*>(out + (j0 + a) * kTT + 8 * tg);
            o[0] = make_float4(sinf(wj * acc[a][0]), sinf(wj * acc[a][1]), sinf(wj * acc[a][2]), sinf(wj * acc[a][3]));
            o[1] = make_float4(sinf(wj * acc[a][4]), sinf(wj * acc[a][5]), sinf(wj * acc[a][6]), sinf(wj * acc[a][7]));
        }
    }
}

// Dynamic shared memory: WT [max(emb, width)][WP4] (a layer's weight,
// transposed), h [2][width][kTT] (feature-major), z [emb_dim][kTT].
__global__ void __launch_bounds__(kThreadsH)
k_filter_hidden(ImplicitMlp m, int64_t L, float* __restrict__ hT) {
    extern __shared__ __align__(16) float sm[];
    const int W = m.width, E = m.emb_dim;
    const int WP4 = (W + 3) & ~3;
    const int rows = E > W ? E : W;
    float* WT = sm;
    float* h0 = WT + rows * WP4;
    float* h1 = h0 + WP4 * kTT;
    float* z = h1 + WP4 * kTT;
    const int64_t t0 = int64_t(blockIdx.x) * kTT;
    const int tid = int(threadIdx.x);
    // positional embedding of the tile's time steps (feature-major)
    const int nb = (E - 1) / 2;
    for (int idx = tid; idx < kTT * E; idx += kThreadsH) {
        const int f = idx / kTT, tt = idx % kTT;
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
        z[f * kTT + tt] = v;
    }
    // first layer: h = Sin(W_in z + b_in)
    for (int idx = tid; idx < W * E; idx += kThreadsH) {
        const int o = idx / E, i = idx % E;
        WT[i * WP4 + o] = __ldg(m.W_in + idx);
    }
    __syncthreads();
    mlp_layer(WT, WP4, z, E, m.b_in, m.w, W, h0);
    float* cur = h0;
    float* nxt = h1;
    // inner layers: h = Sin(W h + b)
    for (int layer = 0; layer < m.num_inner; ++layer) {
        __syncthreads();                               // previous layer done with WT, cur complete
        const float* Wl = m.W_inner + int64_t(layer) * W * W;
        for (int idx = tid; idx < W * W; idx += kThreadsH) {
            const int o = idx / W, i = idx % W;
            WT[i * WP4 + o] = __ldg(Wl + idx);
        }
        __syncthreads();
        mlp_layer(WT, WP4, cur, W, m.b_inner + int64_t(layer) * W, m.w, W, nxt);
        float* sw = cur;
        cur = nxt;
        nxt = sw;
    }
    __syncthreads();
    // hT[f][t] for the tile (consecutive t per feature row)
    for (int idx = tid; idx < W * kTT; idx += kThreadsH) {
        const int f = idx / kTT, tt = idx % kTT;
        if (t0 + tt < L) hT[int64_t(f) * L + t0 + tt] = cur[f * kTT + tt];
    }
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

cudaError_t launch_filter_hidden(const ImplicitMlp& m, int64_t L, float* hT, cudaStream_t s) {
    const int rows = m.emb_dim > m.width ? m.emb_dim : m.width;
    const int wp4 = (m.width + 3) & ~3;
    const size_t smem = (size_t(rows) * wp4 + size_t(2) * wp4 * kTT + size_t(kTT) * m.emb_dim) * 4;
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
