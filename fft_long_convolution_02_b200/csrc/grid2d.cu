// grid2d.cu -- the N-D forms: 2-D non-circular (zero padded, H x W grids of
// 16..512 each), further down the 2-D circular form and the 3-D non-circular
// form (N1 x H x W volumes of 16..128 per axis, reusing the row and column
// engines).
//
// [P5] "Native Multi-Dimensional Subquadratic Operators via Input Dependent
// Long Convolutions", 方法论 (原生 ND 卷积, 边界处理): the global convolution
// runs on the native grid through an N-D FFT, made non-circular by zero
// padding every axis to twice its length; with the gating of [P4] section
// 二.1 (v <- x_{order-s} * v, conv, y = x0 * v).  Kernel anchored at (0,0),
// output cropped to [0:H, 0:W].
//
// The 2H x 2W transform of a real, zero-padded image is evaluated as:
//   row pass (A2)    each image row: packed real FFT of length 2W via two
//                    W/2-point chains + untangle -> bins fq = 0..W (W+1 of them)
//                    -> workspace [fq][p]
//   column pass (B2) each bin column fq: 2H-point FFT of the zero-padded column
//                    (two H-point chains), times K~, inverse, keep p < H
//   row pass (C2)    re-tangle, inverse row chains, output gate -> y
// K~[fp][fq] = (DFT_2Hx2W(k padded)[fp][fq] + D) / (8 H W) is stored per
// channel as [fq][chain][position] so the column pass multiplies in the
// digit-reversed order its forward DIF leaves behind.
#include "common.cuh"
#include "cta_fft.cuh"
#include "grid2dc_tc.h"
#include "kernels.h"
#include "reg_fft.cuh"

namespace hyena {

namespace {

constexpr int kRB = 16;        // image rows per CTA in the row passes
constexpr int kCB = 4;         // bin columns per CTA in the column pass
constexpr int kRowThreads = 256;
constexpr int kColThreads2 = 128;

struct T2d {
    const float2* fftW;     // CTA FFT of size W/2
    const float2* fftH;     // CTA FFT of size H
    const float2* twist_w;  // w_W^n, n < W/2
    const float2* untw;     // pair twiddles w_2W^f, chain e then chain o
    const float2* twist_h;  // w_2H^p, p < H
};

T2d t2d(const Plan& p, const uint8_t* spectrum) {
    const float2* t = reinterpret_cast<const float2*>(spectrum + p.tables_off);
    return T2d{t + p.t_fft_a, t + p.t_fft_b, t + p.t_twist, t + p.t_untangle, t + p.t_twist_h};
}

template <int MW>
__device__ __forceinline__ float2* rowbuf(float2* smem, int ch, int r) {
    return smem + (ch * kRB + r) * fft_padded_size(MW);
}

// Row forward: rows of z (already in smem at natural positions) -> DIF ->
// untangle -> ws[fq][p0 + r] for fq in [0, W].
template <int MW, typename WT>
__device__ __forceinline__ void rows_forward_store(float2* smem, const T2d& tb, WT* __restrict__ ws_img,
                                                   int H, int p0, float dscale, float d) {
    constexpr int W = 2 * MW;
    __syncthreads();
    cta_fft_forward<MW>(smem, 2 * kRB, fft_padded_size(MW), tb.fftW);
    // pairs q: chain e q = 0..MW/2, chain o q = MW/2+1..MW; rows r fastest
    for (int idx = threadIdx.x; idx < (MW + 1) * kRB; idx += blockDim.x) {
        const int q = idx / kRB;
        const int r = idx - q * kRB;
        const bool odd = q > MW / 2;
        const int j = odd ? q - (MW / 2 + 1) : q;
        const float2* buf = rowbuf<MW>(smem, odd ? 1 : 0, r);
        const int mb = odd ? (MW - 1 - j) : ((MW - j) & (MW - 1));
        const float2 A = buf[fft_pad(fft_bin_pos<MW>(j))];
        const float2 B = buf[fft_pad(fft_bin_pos<MW>(mb))];
        const int f = odd ? 2 * j + 1 : 2 * j;
        const int g = W - f;
        float2 Xf, Xg;
        if (q == 0) {
            Xf = make_float2(2.0f * (A.x + A.y), 0.0f);
            Xg = make_float2(2.0f * (A.x - A.y), 0.0f);
        } else {
            const float2 w = __ldg(tb.untw + q);
            const float2 S = cadd(A, cconj(B));
            const float2 T = cmul_i(cmul(w, csub(A, cconj(B))));
            Xf = csub(S, T);
            Xg = cconj(cadd(S, T));
        }
        // dscale/d turn X2 into the stored quantity (spectrum build) or leave it
        Xf = make_float2(Xf.x * dscale + d, Xf.y * dscale);
        Xg = make_float2(Xg.x * dscale + d, Xg.y * dscale);
        ws_st(ws_img + int64_t(f) * H + p0 + r, Xf);
        if (g != f) ws_st(ws_img + int64_t(g) * H + p0 + r, Xg);
    }
}

// MODE 0: gated input x_{order-1} * v from u; MODE 1: the filter k.
template <int MW, typename T, int MODE>
__global__ void __launch_bounds__(kRowThreads)
k_2d_rows_fwd(const T* __restrict__ src, typename WsSel<T, MODE>::type* __restrict__ ws, T2d tb, int64_t B, int64_t C, int order, int H,
              int64_t img0, int64_t ws_img_stride, int64_t ws_img_offset) {
    extern __shared__ float2 smem[];
    constexpr int W = 2 * MW;
    const int64_t img = img0 + blockIdx.y;
    const int p0 = blockIdx.x * kRB;
    const int64_t n = int64_t(H) * W;
    const T* xg;
    const T* vr = nullptr;
    if (MODE == 0) {
        const int64_t c = img / B, b = img - (img / B) * B;
        const int64_t Ctot = int64_t(order + 1) * C;
        const T* ub = src + b * Ctot * n;
        xg = ub + (int64_t(order - 1) * C + c) * n;
        vr = ub + (int64_t(order) * C + c) * n;
    } else {
        xg = src + img * n;
    }
    for (int idx = threadIdx.x; idx < kRB * MW; idx += blockDim.x) {
        const int r = idx / MW;
        const int nn = idx - r * MW;
        const int64_t off = int64_t(p0 + r) * W + 2 * nn;
        float2 z = load2(xg + off);
        if (MODE == 0) {
            const float2 v = load2(vr + off);
            z = make_float2(z.x * v.x, z.y * v.y);
        }
        rowbuf<MW>(smem, 0, r)[fft_pad(nn)] = z;
        rowbuf<MW>(smem, 1, r)[fft_pad(nn)] = cmul(z, __ldg(tb.twist_w + nn));
    }
    auto* ws_img = ws + int64_t(blockIdx.y) * ws_img_stride + ws_img_offset;
    rows_forward_store<MW>(smem, tb, ws_img, H, p0, 1.0f, 0.0f);
}

// Column pass.  MODE 0: convolution in place.  MODE 1: spectrum build, one
// CTA per (step, channel) walking the bin columns in increasing order (the
// row-pass output sits in the upper half of the channel's region).
template <int MH, int MODE, typename WT>
__global__ void __launch_bounds__(kColThreads2)
k_2d_cols(WT* __restrict__ ws, const float2* __restrict__ spec, T2d tb, int W, int64_t B, int64_t C, int step,
          int64_t img0, int64_t ws_img_stride, int64_t spec_row_stride, const float* __restrict__ D, float s8,
          int64_t SC, int64_t SB, int line0, int line1, int lines_per_block) {
    extern __shared__ float2 smem[];
    constexpr int PS = fft_padded_size(MH);
    const int64_t img = img0 + blockIdx.y;
    static_assert(MODE == 0 || sizeof(WT) == sizeof(float2), "the spectrum build writes complex64 rows");
    WT* ws_img = ws + int64_t(blockIdx.y) * ws_img_stride;
    const int ncol = W + 1;
    const float2* sp = nullptr;
    float d = 0.0f;
    if (MODE == 0) {
        const int64_t c = img / B, b = img - c * B;
        sp = spec + (int64_t(step) * SC + b * SB + c) * spec_row_stride;
    } else {
        d = D ? __ldg(D + img) : 0.0f;
    }
    // spectrum build: this block's lines of the wave [line0, line1) (see spectrum_cols_waves)
    const int f_begin = MODE == 0 ? int(blockIdx.x) * kCB : line0 + int(blockIdx.x) * lines_per_block;
    const int f_end = MODE == 0 ? min(f_begin + kCB, ncol) : min(f_begin + lines_per_block, line1);
    const int per = MODE == 0 ? kCB : 1;
    for (int f0 = f_begin; f0 < f_end; f0 += per) {
        const int nc = min(per, f_end - f0);
        const WT* src = MODE == 0 ? ws_img : ws_img + int64_t(ncol) * MH;   // spectrum build: upper half
        for (int idx = threadIdx.x; idx < nc * MH; idx += blockDim.x) {
            const int cc = idx / MH;
            const int p = idx - cc * MH;
            const float2 v = ws_ld(src + int64_t(f0 + cc) * MH + p);
            smem[(2 * cc) * PS + fft_pad(p)] = v;
            smem[(2 * cc + 1) * PS + fft_pad(p)] = cmul(v, __ldg(tb.twist_h + p));
        }
        __syncthreads();
        cta_fft_forward<MH>(smem, 2 * nc, PS, tb.fftH);
        if (MODE == 0) {
            for (int idx = threadIdx.x; idx < 2 * nc * MH; idx += blockDim.x) {
                const int tcol = idx / MH;            // 2*cc + chain
                const int pos = idx - tcol * MH;
                const int cc = tcol >> 1, ch = tcol & 1;
                // spectrum entries in the fast column pass's order (see MODE 1)
                const float2 k = __ldg(sp + int64_t(f0 + cc) * (2 * MH) + ch * MH + (pos & 15) * (MH / 16) + (pos >> 4));
                float2* e = smem + tcol * PS + fft_pad(pos);
                *e = cmul(*e, k);
            }
            __syncthreads();
            cta_fft_inverse<MH>(smem, 2 * nc, PS, tb.fftH);
            for (int idx = threadIdx.x; idx < nc * MH; idx += blockDim.x) {
                const int cc = idx / MH;
                const int p = idx - cc * MH;
                const float2 e = smem[(2 * cc) * PS + fft_pad(p)];
                const float2 o = smem[(2 * cc + 1) * PS + fft_pad(p)];
                ws_st(ws_img + int64_t(f0 + cc) * MH + p, cadd(e, cmulc(o, __ldg(tb.twist_h + p))));
            }
        } else {
            // K~ = (X2D / 2 + D) * s8, positions in order, chain e then chain o
            // stored in the fast column pass's thread order: position 16 g + k
            // of chain ch goes to entry ch * MH + k * (MH / 16) + g
            for (int idx = threadIdx.x; idx < 2 * MH; idx += blockDim.x) {
                const int ch = idx / MH;
                const int pos = idx - ch * MH;
                const float2 v = smem[ch * PS + fft_pad(pos)];
                const int e = ch * MH + (pos & 15) * (MH / 16) + (pos >> 4);
                ws_st(ws_img + int64_t(f0) * (2 * MH) + e, make_float2((0.5f * v.x + d) * s8, 0.5f * v.y * s8));
            }
        }
        __syncthreads();
    }
}

// Row inverse pass: re-tangle, inverse row chains, output gate (FINAL) or
// next gate + next step's row forward pass.
template <int MW, typename T, bool FINAL>
__global__ void __launch_bounds__(kRowThreads)
k_2d_rows_inv(const T* __restrict__ u, T* __restrict__ y, typename WsOf<T>::type* __restrict__ ws, T2d tb, int64_t B,
              int64_t C, int order, int gnext, int H, int64_t img0, int64_t ws_img_stride) {
    extern __shared__ float2 smem[];
    constexpr int W = 2 * MW;
    const int64_t img = img0 + blockIdx.y;
    const int p0 = blockIdx.x * kRB;
    const int64_t n = int64_t(H) * W;
    auto* ws_img = ws + int64_t(blockIdx.y) * ws_img_stride;
    for (int idx = threadIdx.x; idx < (MW + 1) * kRB; idx += blockDim.x) {
        const int q = idx / kRB;
        const int r = idx - q * kRB;
        const bool odd = q > MW / 2;
        const int j = odd ? q - (MW / 2 + 1) : q;
        float2* buf = rowbuf<MW>(smem, odd ? 1 : 0, r);
        const int mb = odd ? (MW - 1 - j) : ((MW - j) & (MW - 1));
        const int f = odd ? 2 * j + 1 : 2 * j;
        const int g = W - f;
        const float2 Yf = ws_ld(ws_img + int64_t(f) * H + p0 + r);
        const float2 Yg = ws_ld(ws_img + int64_t(g) * H + p0 + r);
        const float2 w = (q == 0) ? make_float2(1.0f, 0.0f) : __ldg(tb.untw + q);
        const float2 P = cadd(Yf, cconj(Yg));
        const float2 U = cmul_i(cmulc(csub(Yf, cconj(Yg)), w));
        buf[fft_pad(fft_bin_pos<MW>(j))] = cadd(P, U);
        if (q != 0) buf[fft_pad(fft_bin_pos<MW>(mb))] = cconj(csub(P, U));
    }
    __syncthreads();
    cta_fft_inverse<MW>(smem, 2 * kRB, fft_padded_size(MW), tb.fftW);
    const int64_t c = img / B, b = img - (img / B) * B;
    const int64_t Ctot = int64_t(order + 1) * C;
    const T* ub = u + b * Ctot * n;
    const int gate = FINAL ? 0 : gnext;
    const T* xg = ub + (int64_t(gate) * C + c) * n;
    T* yr = y + (b * C + c) * n;
    for (int idx = threadIdx.x; idx < kRB * MW; idx += blockDim.x) {
        const int r = idx / MW;
        const int nn = idx - r * MW;
        const int64_t off = int64_t(p0 + r) * W + 2 * nn;
        float2* e = rowbuf<MW>(smem, 0, r) + fft_pad(nn);
        float2* o = rowbuf<MW>(smem, 1, r) + fft_pad(nn);
        const float2 tw = __ldg(tb.twist_w + nn);
        const float2 zp = cadd(*e, cmulc(*o, tw));
        const float2 x = load2(xg + off);
        const float2 z = make_float2(x.x * zp.x, x.y * zp.y);
        if (FINAL) {
            store2(yr + off, z);
        } else {
            *e = z;
            *o = cmul(z, tw);
        }
    }
    if (!FINAL) rows_forward_store<MW>(smem, tb, ws_img, H, p0, 1.0f, 0.0f);
}

// ===========================================================================
// Register-resident 2-D passes (reg_fft.cuh).
//   rows   : a CTA of 32 image rows x (W/32) threads; thread (r, g) holds 16
//            points of both row chains; the untangle / re-tangle pairs go
//            through padded shared buffers (odd stride, conflict-free).
//   columns: a CTA of 16 bin columns x (H/16) threads, both column chains per
//            thread; K~ is read in the same thread order ([chain][k][g]).
// ===========================================================================
constexpr int kFC = 16;   // bin columns per CTA in the fast column pass

template <int MW>
__host__ __device__ constexpr int row_stride_f() {
    return fft_padded_size(MW) | 1;   // odd stride: rows of a warp hit different banks
}

template <int MW, int FR, typename WT>
__device__ __forceinline__ void frows_store(float2 (&x)[2][16], float2* smem, const T2d& tb,
                                            WT* __restrict__ ws_img, int H, int p0, int r, int g) {
    constexpr int W = 2 * MW;
    constexpr int RS = row_stride_f<MW>();
    // positions 16 g + k of both chains to shared memory
    float2* be = smem + (0 * FR + r) * RS;
    float2* bo = smem + (1 * FR + r) * RS;
    const int base = fft_pad(16 * g);
#pragma unroll
    for (int k = 0; k < 16; ++k) { be[base + k] = x[0][k]; bo[base + k] = x[1][k]; }
    __syncthreads();
    // untangle: pairs q (chain e 0..MW/2, chain o MW/2+1..MW), rows fastest
    for (int idx = threadIdx.x; idx < (MW + 1) * FR; idx += blockDim.x) {
        const int q = idx / FR;
        const int rr = idx - q * FR;
        const bool odd = q > MW / 2;
        const int j = odd ? q - (MW / 2 + 1) : q;
        const float2* buf = smem + ((odd ? 1 : 0) * FR + rr) * RS;
        const int mb = odd ? (MW - 1 - j) : ((MW - j) & (MW - 1));
        const float2 A = buf[fft_pad(fft_bin_pos<MW>(j))];
        const float2 B = buf[fft_pad(fft_bin_pos<MW>(mb))];
        const int f = odd ? 2 * j + 1 : 2 * j;
        const int gg = W - f;
        float2 Xf, Xg;
        if (q == 0) {
            Xf = make_float2(2.0f * (A.x + A.y), 0.0f);
            Xg = make_float2(2.0f * (A.x - A.y), 0.0f);
        } else {
            const float2 w = __ldg(tb.untw + q);
            const float2 S = cadd(A, cconj(B));
            const float2 T = cmul_i(cmul(w, csub(A, cconj(B))));
            Xf = csub(S, T);
            Xg = cconj(cadd(S, T));
        }
        ws_st(ws_img + int64_t(f) * H + p0 + rr, Xf);
        if (gg != f) ws_st(ws_img + int64_t(gg) * H + p0 + rr, Xg);
    }
}

// Forward rows: MODE 0 gated x_{order-1} * v from u, MODE 1 the filter k.
template <int MW, int FR, typename T, int MODE>
__global__ void __launch_bounds__(FR * (MW / 16), (512 / (FR * (MW / 16))) > 0 ? 512 / (FR * (MW / 16)) : 1)
k_2df_rows_fwd(const T* __restrict__ src, typename WsSel<T, MODE>::type* __restrict__ ws, T2d tb, int64_t B, int64_t C, int order, int H,
               int64_t img0, int64_t ws_img_stride, int64_t ws_img_offset) {
    extern __shared__ float2 smem[];
    constexpr int W = 2 * MW;
    constexpr int TPT = MW / 16;
    constexpr int RS = row_stride_f<MW>();
    const int t = threadIdx.x, r = t / TPT, g = t - (t / TPT) * TPT;
    const int64_t img = img0 + blockIdx.y;
    const int p0 = blockIdx.x * FR;
    const int64_t n = int64_t(H) * W;
    const T* xg;
    const T* vr = nullptr;
    if (MODE == 0) {
        const int64_t c = img / B, b = img - (img / B) * B;
        const int64_t Ctot = int64_t(order + 1) * C;
        const T* ub = src + b * Ctot * n;
        xg = ub + (int64_t(order - 1) * C + c) * n;
        vr = ub + (int64_t(order) * C + c) * n;
    } else {
        xg = src + img * n;
    }
    float2 x[2][16];
#pragma unroll
    for (int s = 0; s < 16; ++s) {
        const int nn = g + TPT * s;
        const int64_t off = int64_t(p0 + r) * W + 2 * nn;
        float2 z = load2(xg + off);
        if (MODE == 0) {
            const float2 v = load2(vr + off);
            z = make_float2(z.x * v.x, z.y * v.y);
        }
        x[0][s] = z;
        x[1][s] = cmul(z, __ldg(tb.twist_w + nn));
    }
    float2* const buf[2] = {smem + (0 * FR + r) * RS, smem + (1 * FR + r) * RS};
    reg_fft_forward<MW, 2>(x, buf, g, tb.fftW);
    auto* ws_img = ws + int64_t(blockIdx.y) * ws_img_stride + ws_img_offset;
    frows_store<MW, FR>(x, smem, tb, ws_img, H, p0, r, g);
}

// Inverse rows: re-tangle, inverse chains, output gate (FINAL) or next gate +
// next step's forward rows.
template <int MW, int FR, typename T, bool FINAL>
__global__ void __launch_bounds__(FR * (MW / 16), (512 / (FR * (MW / 16))) > 0 ? 512 / (FR * (MW / 16)) : 1)
k_2df_rows_inv(const T* __restrict__ u, T* __restrict__ y, typename WsOf<T>::type* __restrict__ ws, T2d tb, int64_t B,
               int64_t C, int order, int gnext, int H, int64_t img0, int64_t ws_img_stride) {
    extern __shared__ float2 smem[];
    constexpr int W = 2 * MW;
    constexpr int TPT = MW / 16;
    constexpr int RS = row_stride_f<MW>();
    const int t = threadIdx.x, r = t / TPT, g = t - (t / TPT) * TPT;
    const int64_t img = img0 + blockIdx.y;
    const int p0 = blockIdx.x * FR;
    const int64_t n = int64_t(H) * W;
    auto* ws_img = ws + int64_t(blockIdx.y) * ws_img_stride;
    for (int idx = threadIdx.x; idx < (MW + 1) * FR; idx += blockDim.x) {
        const int q = idx / FR;
        const int rr = idx - q * FR;
        const bool odd = q > MW / 2;
        const int j = odd ? q - (MW / 2 + 1) : q;
        float2* buf = smem + ((odd ? 1 : 0) * FR + rr) * RS;
        const int mb = odd ? (MW - 1 - j) : ((MW - j) & (MW - 1));
        const int f = odd ? 2 * j + 1 : 2 * j;
        const int gg = W - f;
        const float2 Yf = ws_ld(ws_img + int64_t(f) * H + p0 + rr);
        const float2 Yg = ws_ld(ws_img + int64_t(gg) * H + p0 + rr);
        const float2 w = (q == 0) ? make_float2(1.0f, 0.0f) : __ldg(tb.untw + q);
        const float2 P = cadd(Yf, cconj(Yg));
        const float2 U = cmul_i(cmulc(csub(Yf, cconj(Yg)), w));
        buf[fft_pad(fft_bin_pos<MW>(j))] = cadd(P, U);
        if (q != 0) buf[fft_pad(fft_bin_pos<MW>(mb))] = cconj(csub(P, U));
    }
    __syncthreads();
    float2* const buf[2] = {smem + (0 * FR + r) * RS, smem + (1 * FR + r) * RS};
    float2 x[2][16];
    const int base = fft_pad(16 * g);
#pragma unroll
    for (int k = 0; k < 16; ++k) { x[0][k] = buf[0][base + k]; x[1][k] = buf[1][base + k]; }
    __syncthreads();
    reg_fft_inverse<MW, 2>(x, buf, g, tb.fftW);
    const int64_t c = img / B, b = img - (img / B) * B;
    const int64_t Ctot = int64_t(order + 1) * C;
    const T* ub = u + b * Ctot * n;
    const int gate = FINAL ? 0 : gnext;
    const T* xg = ub + (int64_t(gate) * C + c) * n;
    T* yr = y + (b * C + c) * n;
#pragma unroll
    for (int s = 0; s < 16; ++s) {
        const int nn = g + TPT * s;
        const int64_t off = int64_t(p0 + r) * W + 2 * nn;
        const float2 tw = __ldg(tb.twist_w + nn);
        const float2 zp = cadd(x[0][s], cmulc(x[1][s], tw));
        const float2 xv = load2(xg + off);
        const float2 z = make_float2(xv.x * zp.x, xv.y * zp.y);
        if (FINAL) {
            store2(yr + off, z);
        } else {
            x[0][s] = z;
            x[1][s] = cmul(z, tw);
        }
    }
    if (!FINAL) {
        reg_fft_forward<MW, 2>(x, buf, g, tb.fftW);
        frows_store<MW, FR>(x, smem, tb, ws_img, H, p0, r, g);
    }
}

// Column pass (convolution): 2H-point FFT of each zero-padded bin column as two
// H-point chains, times K~ (thread order), inverse, keep p < H.
// LAST: only the last bin column (f = W) of every image, thread group cc of
// block x taking image 16 x + cc (nimg images in the launch).
template <int MH, typename WT, bool LAST = false>
__global__ void __launch_bounds__(kFC * (MH / 16), (512 / (kFC * (MH / 16))) > 0 ? 512 / (kFC * (MH / 16)) : 1)
k_2df_cols(WT* __restrict__ ws, const float2* __restrict__ spec, T2d tb, int W, int64_t B, int64_t C, int step,
           int64_t img0, int64_t ws_img_stride, int64_t spec_row_stride, int64_t SC, int64_t SB, int nimg) {
    extern __shared__ float2 smem[];
    constexpr int TPT = MH / 16;
    constexpr int PS = fft_padded_size(MH);
    const int t = threadIdx.x, cc = t / TPT, g = t - (t / TPT) * TPT;
    const int li = LAST ? min(int(blockIdx.x) * kFC + cc, nimg - 1) : int(blockIdx.y);
    const int64_t img = img0 + li;
    const int f = LAST ? W : int(blockIdx.x) * kFC + cc;
    const bool active = LAST ? int(blockIdx.x) * kFC + cc < nimg : f <= W;
    const int fc = LAST ? W : (active ? f : W);
    WT* ws_img = ws + int64_t(li) * ws_img_stride;
    const int64_t c = img / B, b = img - c * B;
    const float2* sp = spec + (int64_t(step) * SC + b * SB + c) * spec_row_stride + int64_t(fc) * (2 * MH);
    if (!LAST && t < kFC) {
        // this CTA's spectrum columns into L2 while the forward transform runs
        const int f2 = int(blockIdx.x) * kFC + t;
        if (f2 <= W)
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(sp + int64_t(f2 - fc) * (2 * MH)),
                         "r"(uint32_t(2 * MH * sizeof(float2)))
                         : "memory");
    }
    float2 x[2][16];
#pragma unroll
    for (int s = 0; s < 16; ++s) {
        const int p = g + TPT * s;
        const float2 v = ws_ld(ws_img + int64_t(fc) * MH + p);
        x[0][s] = v;
        x[1][s] = cmul(v, __ldg(tb.twist_h + p));
    }
    float2* const buf[2] = {smem + (2 * cc) * PS, smem + (2 * cc + 1) * PS};
    reg_fft_forward<MH, 2>(x, buf, g, tb.fftH);
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        x[0][k] = cmul(x[0][k], __ldg(sp + k * TPT + g));
        x[1][k] = cmul(x[1][k], __ldg(sp + MH + k * TPT + g));
    }
    reg_fft_inverse<MH, 2>(x, buf, g, tb.fftH);
    if (active) {
#pragma unroll
        for (int s = 0; s < 16; ++s) {
            const int p = g + TPT * s;
            ws_st(ws_img + int64_t(fc) * MH + p, cadd(x[0][s], cmulc(x[1][s], __ldg(tb.twist_h + p))));
        }
    }
}

// ===========================================================================
// Circular form ([P5] 边界处理: circular convolution for periodic systems):
// no padding, so each axis is its own DFT length.  The W-point real FFT of a
// row is the packed W/2-point complex FFT untangled: exactly the chain e of
// the padded row pass (its even bins), giving bins k = 0..W/2 (W/2+1 columns
// of H values).  Each column then takes one H-point chain: forward, times K~,
// inverse.  K~[kh][kw] = (DFT_HxW(k)[kh][kw] + D) / (2 H W), per channel
// [kw][position] with the H positions in the register column pass's thread
// order.
// ===========================================================================

// Row forward, circular: rows of z (chain e slots of the CTA's row buffers)
// -> packed FFT -> untangle -> ws[k][p0 + r], k = 0..W/2.
template <int MW, typename WT>
__device__ __forceinline__ void rowsc_forward_store(float2* smem, const T2d& tb, WT* __restrict__ ws_img, int H,
                                                    int p0) {
    __syncthreads();
    cta_fft_forward<MW>(smem, kRB, fft_padded_size(MW), tb.fftW);
    for (int idx = threadIdx.x; idx < (MW / 2 + 1) * kRB; idx += blockDim.x) {
        const int j = idx / kRB;
        const int r = idx - j * kRB;
        const float2* buf = rowbuf<MW>(smem, 0, r);
        const float2 A = buf[fft_pad(fft_bin_pos<MW>(j))];
        const float2 B = buf[fft_pad(fft_bin_pos<MW>((MW - j) & (MW - 1)))];
        float2 Xf, Xg;
        if (j == 0) {
            Xf = make_float2(2.0f * (A.x + A.y), 0.0f);
            Xg = make_float2(2.0f * (A.x - A.y), 0.0f);
        } else {
            const float2 w = __ldg(tb.untw + j);   // w_W^j
            const float2 S = cadd(A, cconj(B));
            const float2 T = cmul_i(cmul(w, csub(A, cconj(B))));
            Xf = csub(S, T);
            Xg = cconj(cadd(S, T));
        }
        ws_st(ws_img + int64_t(j) * H + p0 + r, Xf);
        if (MW - j != j) ws_st(ws_img + int64_t(MW - j) * H + p0 + r, Xg);
    }
}

// MODE 0: gated input x_{order-1} * v from u; MODE 1: the filter k.
template <int MW, typename T, int MODE>
__global__ void __launch_bounds__(kRowThreads)
k_2dc_rows_fwd(const T* __restrict__ src, typename WsSel<T, MODE>::type* __restrict__ ws, T2d tb, int64_t B,
               int64_t C, int order, int H, int64_t img0, int64_t ws_img_stride) {
    extern __shared__ float2 smem[];
    constexpr int W = 2 * MW;
    const int64_t img = img0 + blockIdx.y;
    const int p0 = blockIdx.x * kRB;
    const int64_t n = int64_t(H) * W;
    const T* xg;
    const T* vr = nullptr;
    if (MODE == 0) {
        const int64_t c = img / B, b = img - (img / B) * B;
        const int64_t Ctot = int64_t(order + 1) * C;
        const T* ub = src + b * Ctot * n;
        xg = ub + (int64_t(order - 1) * C + c) * n;
        vr = ub + (int64_t(order) * C + c) * n;
    } else {
        xg = src + img * n;
    }
    for (int idx = threadIdx.x; idx < kRB * MW; idx += blockDim.x) {
        const int r = idx / MW;
        const int nn = idx - r * MW;
        const int64_t off = int64_t(p0 + r) * W + 2 * nn;
        float2 z = load2(xg + off);
        if (MODE == 0) {
            const float2 v = load2(vr + off);
            z = make_float2(z.x * v.x, z.y * v.y);
        }
        rowbuf<MW>(smem, 0, r)[fft_pad(nn)] = z;
    }
    rowsc_forward_store<MW>(smem, tb, ws + int64_t(blockIdx.y) * ws_img_stride, H, p0);
}

// Row inverse, circular: re-tangle, inverse packed FFT, output gate (FINAL)
// or next gate + next step's row forward pass.
template <int MW, typename T, bool FINAL>
__global__ void __launch_bounds__(kRowThreads)
k_2dc_rows_inv(const T* __restrict__ u, T* __restrict__ y, typename WsOf<T>::type* __restrict__ ws, T2d tb,
               int64_t B, int64_t C, int order, int gnext, int H, int64_t img0, int64_t ws_img_stride) {
    extern __shared__ float2 smem[];
    constexpr int W = 2 * MW;
    const int64_t img = img0 + blockIdx.y;
    const int p0 = blockIdx.x * kRB;
    const int64_t n = int64_t(H) * W;
    auto* ws_img = ws + int64_t(blockIdx.y) * ws_img_stride;
    for (int idx = threadIdx.x; idx < (MW / 2 + 1) * kRB; idx += blockDim.x) {
        const int j = idx / kRB;
        const int r = idx - j * kRB;
        float2* buf = rowbuf<MW>(smem, 0, r);
        const int mb = (MW - j) & (MW - 1);
        const float2 Yf = ws_ld(ws_img + int64_t(j) * H + p0 + r);
        const float2 Yg = ws_ld(ws_img + int64_t(MW - j) * H + p0 + r);
        const float2 w = (j == 0) ? make_float2(1.0f, 0.0f) : __ldg(tb.untw + j);
        const float2 P = cadd(Yf, cconj(Yg));
        const float2 U = cmul_i(cmulc(csub(Yf, cconj(Yg)), w));
        buf[fft_pad(fft_bin_pos<MW>(j))] = cadd(P, U);
        if (j != 0) buf[fft_pad(fft_bin_pos<MW>(mb))] = cconj(csub(P, U));
    }
    __syncthreads();
    cta_fft_inverse<MW>(smem, kRB, fft_padded_size(MW), tb.fftW);
    const int64_t c = img / B, b = img - (img / B) * B;
    const int64_t Ctot = int64_t(order + 1) * C;
    const T* ub = u + b * Ctot * n;
    const int gate = FINAL ? 0 : gnext;
    const T* xg = ub + (int64_t(gate) * C + c) * n;
    T* yr = y + (b * C + c) * n;
    for (int idx = threadIdx.x; idx < kRB * MW; idx += blockDim.x) {
        const int r = idx / MW;
        const int nn = idx - r * MW;
        const int64_t off = int64_t(p0 + r) * W + 2 * nn;
        float2* e = rowbuf<MW>(smem, 0, r) + fft_pad(nn);
        const float2 x = load2(xg + off);
        const float2 z = make_float2(x.x * e->x, x.y * e->y);
        if (FINAL) store2(yr + off, z);
        else *e = z;
    }
    if (!FINAL) rowsc_forward_store<MW>(smem, tb, ws_img, H, p0);
}

// Column pass, circular (convolution): thread group cc of the CTA takes the
// two bin columns fa = 2 (blockIdx.x kFC + cc) and fa + 1 as its two register
// transforms: H-point forward, times K~ (thread order), inverse.
template <int MH, typename WT>
__global__ void __launch_bounds__(kFC * (MH / 16), (512 / (kFC * (MH / 16))) > 0 ? 512 / (kFC * (MH / 16)) : 1)
k_2dc_cols(WT* __restrict__ ws, const float2* __restrict__ spec, T2d tb, int ncol, int64_t B, int step,
           int64_t img0, int64_t ws_img_stride, int64_t spec_row_stride, int64_t SC, int64_t SB) {
    extern __shared__ float2 smem[];
    constexpr int TPT = MH / 16;
    constexpr int PS = fft_padded_size(MH);
    const int t = threadIdx.x, cc = t / TPT, g = t - (t / TPT) * TPT;
    const int64_t img = img0 + blockIdx.y;
    const int fa = 2 * (int(blockIdx.x) * kFC + cc);
    const int f[2] = {fa < ncol ? fa : ncol - 1, fa + 1 < ncol ? fa + 1 : ncol - 1};
    WT* ws_img = ws + int64_t(blockIdx.y) * ws_img_stride;
    const int64_t c = img / B, b = img - c * B;
    const float2* sp = spec + (int64_t(step) * SC + b * SB + c) * spec_row_stride;
    float2 x[2][16];
#pragma unroll
    for (int v = 0; v < 2; ++v) {
#pragma unroll
        for (int s = 0; s < 16; ++s) x[v][s] = ws_ld(ws_img + int64_t(f[v]) * MH + g + TPT * s);
    }
    float2* const buf[2] = {smem + (2 * cc) * PS, smem + (2 * cc + 1) * PS};
    reg_fft_forward<MH, 2>(x, buf, g, tb.fftH);
#pragma unroll
    for (int v = 0; v < 2; ++v) {
#pragma unroll
        for (int k = 0; k < 16; ++k) x[v][k] = cmul(x[v][k], __ldg(sp + int64_t(f[v]) * MH + k * TPT + g));
    }
    reg_fft_inverse<MH, 2>(x, buf, g, tb.fftH);
#pragma unroll
    for (int v = 0; v < 2; ++v) {
        if (fa + v < ncol) {
#pragma unroll
            for (int s = 0; s < 16; ++s) ws_st(ws_img + int64_t(f[v]) * MH + g + TPT * s, x[v][s]);
        }
    }
}

// Spectrum build, circular: one CTA per (step, channel) walks the W/2+1 bin
// columns of the row-pass output in place: H-point forward FFT, then
// K~ = (X / 2 + D) / (2 H W) in the column pass's thread order.
template <int MH>
__global__ void __launch_bounds__(kColThreads2)
k_2dc_cols_spec(float2* __restrict__ rows, T2d tb, int ncol, int64_t row0, int64_t row_stride,
                const float* __restrict__ D, float s2) {
    extern __shared__ float2 smem[];
    const int64_t r = row0 + blockIdx.y;
    float2* img = rows + int64_t(blockIdx.y) * row_stride;
    const float d = D ? __ldg(D + r) : 0.0f;
    // each column is transformed in place (no expansion): the columns of an
    // image are independent and spread over the blocks of the grid's x
    for (int f = blockIdx.x; f < ncol; f += gridDim.x) {
        for (int p = threadIdx.x; p < MH; p += blockDim.x) smem[fft_pad(p)] = img[int64_t(f) * MH + p];
        __syncthreads();
        cta_fft_forward<MH>(smem, 1, fft_padded_size(MH), tb.fftH);
        for (int pos = threadIdx.x; pos < MH; pos += blockDim.x) {
            const float2 v = smem[fft_pad(pos)];
            const int e = (pos & 15) * (MH / 16) + (pos >> 4);
            img[int64_t(f) * MH + e] = make_float2((0.5f * v.x + d) * s2, 0.5f * v.y * s2);
        }
        __syncthreads();
    }
}

// ===========================================================================
// 3-D non-circular form ([P5] 原生 ND 卷积 on N1 x H x W grids, e.g. 3-D
// medical volumes; every axis zero padded to twice its length).  The volume
// is N1 H rows of W samples for the row passes (the 2-D row kernels with
// N1 H image rows), so the first workspace region ws1 is [fw][d][h] (fw =
// 0..W).  The column passes run one padded 2H-point transform per (fw, d)
// and store both chains' H positions as depth lines: ws2 [fw][chain][pos][d].
// The depth pass is the 2-D register column pass over those lines (2N1-point,
// times K~, inverse); the inverse column pass brings the lines back to ws1.
// K~ = (DFT_2N1x2Hx2W(k) + D) / (16 N1 H W), per channel [line][chain][pos]
// with line = (fw, chain, pos) of the column pass.
// ===========================================================================

// Forward column pass of the 3-D form: columns (fw, d) of ws1 -> ws2 lines.
// Thread group cc of the CTA takes column d = d0 + cc of bin fw.
template <int MH, typename WT>
__global__ void __launch_bounds__(kFC * (MH / 16), (512 / (kFC * (MH / 16))) > 0 ? 512 / (kFC * (MH / 16)) : 1)
k_3d_cols_fwd(WT* __restrict__ ws, T2d tb, int N1, int64_t ws1_off, int64_t ws2_off, int64_t ws_img_stride) {
    extern __shared__ float2 smem[];
    constexpr int TPT = MH / 16;
    constexpr int PS = fft_padded_size(MH);
    const int t = threadIdx.x, cc = t / TPT, g = t - (t / TPT) * TPT;
    const int dblocks = N1 / kFC;
    const int fw = int(blockIdx.x) / dblocks;
    const int d = (int(blockIdx.x) - fw * dblocks) * kFC + cc;
    WT* ws1 = ws + int64_t(blockIdx.y) * ws_img_stride + ws1_off;
    WT* ws2 = ws + int64_t(blockIdx.y) * ws_img_stride + ws2_off;
    const WT* col = ws1 + (int64_t(fw) * N1 + d) * MH;
    float2 x[2][16];
#pragma unroll
    for (int s = 0; s < 16; ++s) {
        const int h = g + TPT * s;
        const float2 v = ws_ld(col + h);
        x[0][s] = v;
        x[1][s] = cmul(v, __ldg(tb.twist_h + h));
    }
    float2* const buf[2] = {smem + (2 * cc) * PS, smem + (2 * cc + 1) * PS};
    reg_fft_forward<MH, 2>(x, buf, g, tb.fftH);
#pragma unroll
    for (int ch = 0; ch < 2; ++ch) {
#pragma unroll
        for (int k = 0; k < 16; ++k)
            ws_st(ws2 + ((int64_t(fw) * 2 + ch) * MH + 16 * g + k) * N1 + d, x[ch][k]);
    }
}

// Inverse column pass of the 3-D form: ws2 lines -> columns (fw, d) of ws1.
template <int MH, typename WT>
__global__ void __launch_bounds__(kFC * (MH / 16), (512 / (kFC * (MH / 16))) > 0 ? 512 / (kFC * (MH / 16)) : 1)
k_3d_cols_inv(WT* __restrict__ ws, T2d tb, int N1, int64_t ws1_off, int64_t ws2_off, int64_t ws_img_stride) {
    extern __shared__ float2 smem[];
    constexpr int TPT = MH / 16;
    constexpr int PS = fft_padded_size(MH);
    const int t = threadIdx.x, cc = t / TPT, g = t - (t / TPT) * TPT;
    const int dblocks = N1 / kFC;
    const int fw = int(blockIdx.x) / dblocks;
    const int d = (int(blockIdx.x) - fw * dblocks) * kFC + cc;
    WT* ws1 = ws + int64_t(blockIdx.y) * ws_img_stride + ws1_off;
    WT* ws2 = ws + int64_t(blockIdx.y) * ws_img_stride + ws2_off;
    float2 x[2][16];
#pragma unroll
    for (int ch = 0; ch < 2; ++ch) {
#pragma unroll
        for (int k = 0; k < 16; ++k) x[ch][k] = ws_ld(ws2 + ((int64_t(fw) * 2 + ch) * MH + 16 * g + k) * N1 + d);
    }
    float2* const buf[2] = {smem + (2 * cc) * PS, smem + (2 * cc + 1) * PS};
    reg_fft_inverse<MH, 2>(x, buf, g, tb.fftH);
    WT* col = ws1 + (int64_t(fw) * N1 + d) * MH;
#pragma unroll
    for (int s = 0; s < 16; ++s) {
        const int h = g + TPT * s;
        ws_st(col + h, cadd(x[0][s], cmulc(x[1][s], __ldg(tb.twist_h + h))));
    }
}

template <int MW>
size_t row_smem() {
    return size_t(2) * kRB * fft_padded_size(MW) * sizeof(float2);
}

template <int MH>
size_t col_smem2(int per) {
    return size_t(2) * per * fft_padded_size(MH) * sizeof(float2);
}

// The spectrum mode of k_2d_cols works in place: the input of line j sits at
// entries (n + j) MH .. (n + j + 1) MH of the channel's region (n lines), and
// line f writes its 2 MH outputs over entries 2 MH f .. 2 MH (f + 1), which
// hold the inputs of lines 2f - n and 2f + 1 - n.  A wave of lines [a, b)
// with b <= (a + n) / 2 therefore overwrites only inputs of lines below a,
// transformed by earlier waves, and the last line only its own input (read
// into shared memory before it is written), so the n lines run in about
// log2(n) waves of parallel blocks instead of one block per channel.
constexpr int kSpecLinesPerBlock = 4;
template <typename K>
void spectrum_cols_waves(K kb, int n, unsigned nimg, size_t smem, cudaStream_t s, float2* rows, const T2d& tb,
                         int W, int C, int64_t img0, int64_t stride, const float* D, float scale) {
    for (int a0 = 0; a0 < n;) {
        int b = (a0 + n) / 2;
        if (b <= a0) b = a0 + 1;             // a0 = n - 1: the last line
        const unsigned blocks = unsigned((b - a0 + kSpecLinesPerBlock - 1) / kSpecLinesPerBlock);
        kb<<<dim3(blocks, nimg), kColThreads2, smem, s>>>(rows, nullptr, tb, W, 1, C, 0, img0, stride, 0, D, scale, 0,
                                                           0, a0, b, kSpecLinesPerBlock);
        a0 = b;
    }
}

template <int MW, int MH>
cudaError_t spectrum_2d_t(const Plan& p, const SpectrumArgs& a, cudaStream_t s) {
    const T2d tb = t2d(p, a.spectrum);
    float2* rows = reinterpret_cast<float2*>(a.spectrum + p.spec_off);
    const int64_t nimg = (p.order - 1) * p.C;
    const int64_t stride = int64_t(p.spec_row_bytes / sizeof(float2));    // (W+1) * 2H
    const int H = int(p.H), W = int(p.W);
    const size_t smA = row_smem<MW>();
    const size_t smB = col_smem2<MH>(1);
    auto kf = k_2d_rows_fwd<MW, float, 1>;
    auto kh = k_2d_rows_fwd<MW, __nv_bfloat16, 1>;
    auto kb = k_2d_cols<MH, 1, float2>;
    cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smA));
    cudaFuncSetAttribute(kh, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smA));
    cudaFuncSetAttribute(kb, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smB));
    const float s8 = 1.0f / (8.0f * float(H) * float(W));
    for (int64_t i0 = 0; i0 < nimg; i0 += 32768) {
        const int64_t g = nimg - i0 < 32768 ? nimg - i0 : 32768;
        const dim3 gridA(H / kRB, unsigned(g));
        // row pass output goes to the upper half of each channel's region
        const int64_t upper = int64_t(W + 1) * H;
        if (a.k_dtype == DT_F32)
            kf<<<gridA, kRowThreads, smA, s>>>(static_cast<const float*>(a.k), rows + i0 * stride, tb, 1, 1, 2, H, i0,
                                               stride, upper);
        else
            kh<<<gridA, kRowThreads, smA, s>>>(static_cast<const __nv_bfloat16*>(a.k), rows + i0 * stride, tb, 1, 1,
                                               2, H, i0, stride, upper);
        spectrum_cols_waves(kb, W + 1, unsigned(g), smB, s, rows + i0 * stride, tb, W, int(p.C), i0, stride, a.D, s8);
    }
    if (p.g2_plane_off != 0) {
        const cudaError_t e = launch_spectrum_2d_tc_plane(p, reinterpret_cast<const uint8_t*>(rows), a.spectrum + p.g2_plane_off,
                                                          nimg, s);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

// Row passes: register-resident engine (ROWS_REG, W/2 >= 16) or the CTA
// engine; column pass: register-resident (COLS_REG) or the CTA engine.  Both
// write and read the same workspace layout ([bin column][H] per image).
template <int MW, int MH, typename T, bool ROWS_REG, bool COLS_REG>
cudaError_t conv_2d_t(const Plan& p, const ConvArgs& a, cudaStream_t s) {
    const T2d tb = t2d(p, a.spectrum);
    const float2* spec = reinterpret_cast<const float2*>(a.spectrum + p.spec_off);
    const T* u = static_cast<const T*>(a.u);
    T* y = static_cast<T*>(a.y);
    const int64_t nimg = a.B * p.C;
    // bf16 storage keeps the workspace in bf16 (re, im): images of the same
    // element count at half the bytes, so the caller's workspace holds twice
    // the images
    using WT = typename WsOf<T>::type;
    WT* ws = reinterpret_cast<WT*>(a.workspace);
    const int64_t cap = int64_t(a.group_rows) * int64_t(sizeof(float2) / sizeof(WT));
    const int64_t G = cap < 65535 ? cap : 65535;
    const int64_t stride = int64_t(p.ws_row_bytes / sizeof(float2));   // elements per image
    const int64_t spec_stride = int64_t(p.spec_row_bytes / sizeof(float2));
    const int H = int(p.H), W = int(p.W);
    constexpr int FR = MH < 32 ? MH : 32;   // image rows per CTA
    constexpr int NTR = FR * (MW / 16);
    constexpr int NTC = kFC * (MH / 16);
    const size_t smR = size_t(2 * FR) * row_stride_f<MW>() * sizeof(float2);
    const size_t smC = size_t(2 * kFC) * fft_padded_size(MH) * sizeof(float2);
    const size_t smB = col_smem2<MH>(kCB);
    const bool cols_tc = cols_2d_tc_path(p, a);
    cudaError_t tc_err = cudaSuccess;
    auto launch_cols = [&](int64_t i0, int64_t g, int st) {
        if constexpr (COLS_REG) {
            auto kb = k_2df_cols<MH, WT>;
            cudaFuncSetAttribute(kb, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smC));
            if (cols_tc) {
                // columns 0 .. W-1 on the tensor cores, the last bin column here
                const cudaError_t e = launch_cols_2d_tc(p, a, ws, i0, g, st - 1, stride, s);
                if (tc_err == cudaSuccess) tc_err = e;
                auto kl = k_2df_cols<MH, WT, true>;
                cudaFuncSetAttribute(kl, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smC));
                kl<<<dim3(unsigned((g + kFC - 1) / kFC), 1), NTC, smC, s>>>(ws, spec, tb, W, a.B, p.C, st - 1, i0,
                                                                             stride, spec_stride, a.spec_C,
                                                                             a.spec_per_b, int(g));
            } else {
                kb<<<dim3(unsigned((W + 1 + kFC - 1) / kFC), unsigned(g)), NTC, smC, s>>>(
                    ws, spec, tb, W, a.B, p.C, st - 1, i0, stride, spec_stride, a.spec_C, a.spec_per_b, int(g));
            }
        } else {
            auto kb = k_2d_cols<MH, 0, WT>;
            cudaFuncSetAttribute(kb, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smB));
            kb<<<dim3(unsigned((W + 1 + kCB - 1) / kCB), unsigned(g)), kColThreads2, smB, s>>>(
                ws, spec, tb, W, a.B, p.C, st - 1, i0, stride, spec_stride, nullptr, 0.0f, a.spec_C,
                a.spec_per_b, 0, 0, 0);
        }
    };
    auto launch_rows_fwd = [&](int64_t i0, int64_t g) {
        if constexpr (ROWS_REG && MW >= 16) {
            auto ka = k_2df_rows_fwd<MW, FR, T, 0>;
            cudaFuncSetAttribute(ka, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smR));
            ka<<<dim3(H / FR, unsigned(g)), NTR, smR, s>>>(u, ws, tb, a.B, p.C, p.order, H, i0, stride, 0);
        } else {
            auto ka = k_2d_rows_fwd<MW, T, 0>;
            cudaFuncSetAttribute(ka, cudaFuncAttributeMaxDynamicSharedMemorySize, int(row_smem<MW>()));
            ka<<<dim3(H / kRB, unsigned(g)), kRowThreads, row_smem<MW>(), s>>>(u, ws, tb, a.B, p.C, p.order,
                                                                              H, i0, stride, 0);
        }
    };
    auto launch_rows_inv = [&](int64_t i0, int64_t g, bool final_step, int gnext) {
        if constexpr (ROWS_REG && MW >= 16) {
            auto kc = final_step ? k_2df_rows_inv<MW, FR, T, true> : k_2df_rows_inv<MW, FR, T, false>;
            cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smR));
            kc<<<dim3(H / FR, unsigned(g)), NTR, smR, s>>>(u, y, ws, tb, a.B, p.C, p.order, gnext, H, i0,
                                                            stride);
        } else {
            auto kc = final_step ? k_2d_rows_inv<MW, T, true> : k_2d_rows_inv<MW, T, false>;
            cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, int(row_smem<MW>()));
            kc<<<dim3(H / kRB, unsigned(g)), kRowThreads, row_smem<MW>(), s>>>(u, y, ws, tb, a.B, p.C,
                                                                              p.order, gnext, H, i0, stride);
        }
    };
    if constexpr (sizeof(T) == 2) {
        // the two images of a channel as one complex image (groups of whole pairs)
        const int64_t Gp = G & ~int64_t(1);
        if (Gp >= 2 && pairs_2d_tc_path(p, a)) {
            for (int64_t i0 = 0; i0 < nimg; i0 += Gp) {
                const int64_t g = nimg - i0 < Gp ? nimg - i0 : Gp;
                const cudaError_t e = launch_conv_2d_pairs_tc(p, a, ws, i0, g, stride, s);
                if (e != cudaSuccess) return e;
            }
            return cudaGetLastError();
        }
    }
    for (int64_t i0 = 0; i0 < nimg; i0 += G) {
        const int64_t g = nimg - i0 < G ? nimg - i0 : G;
        launch_rows_fwd(i0, g);
        for (int st = 1; st < p.order; ++st) {
            launch_cols(i0, g, st);
            launch_rows_inv(i0, g, st == p.order - 1, st < p.order - 1 ? p.order - st - 1 : 0);
        }
    }
    if (tc_err != cudaSuccess) return tc_err;
    return cudaGetLastError();
}

template <int MW, int MH>
cudaError_t spectrum_2dc_t(const Plan& p, const SpectrumArgs& a, cudaStream_t s) {
    const T2d tb = t2d(p, a.spectrum);
    float2* rows = reinterpret_cast<float2*>(a.spectrum + p.spec_off);
    const int64_t nimg = (p.order - 1) * p.C;
    const int64_t stride = int64_t(p.spec_row_bytes / sizeof(float2));    // (W/2+1) * H
    const int H = int(p.H), W = int(p.W);
    const size_t smA = row_smem<MW>();
    const size_t smB = size_t(fft_padded_size(MH)) * sizeof(float2);
    auto kf = k_2dc_rows_fwd<MW, float, 1>;
    auto kh = k_2dc_rows_fwd<MW, __nv_bfloat16, 1>;
    auto kb = k_2dc_cols_spec<MH>;
    cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smA));
    cudaFuncSetAttribute(kh, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smA));
    cudaFuncSetAttribute(kb, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smB));
    const float s2 = 1.0f / (2.0f * float(H) * float(W));
    for (int64_t i0 = 0; i0 < nimg; i0 += 32768) {
        const int64_t g = nimg - i0 < 32768 ? nimg - i0 : 32768;
        const dim3 gridA(H / kRB, unsigned(g));
        if (a.k_dtype == DT_F32)
            kf<<<gridA, kRowThreads, smA, s>>>(static_cast<const float*>(a.k), rows + i0 * stride, tb, 1, 1, 2, H, i0,
                                               stride);
        else
            kh<<<gridA, kRowThreads, smA, s>>>(static_cast<const __nv_bfloat16*>(a.k), rows + i0 * stride, tb, 1, 1,
                                               2, H, i0, stride);
        kb<<<dim3(unsigned(W / 2 + 1), unsigned(g)), kColThreads2, smB, s>>>(rows + i0 * stride, tb, W / 2 + 1, i0,
                                                                             stride, a.D, s2);
    }
    if (p.g2_plane_off != 0) {
        const cudaError_t e = launch_spectrum_2dc_tc_plane(p, reinterpret_cast<const uint8_t*>(rows),
                                                           a.spectrum + p.g2_plane_off, nimg, s);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

template <int MW, int MH, typename T>
cudaError_t conv_2dc_t(const Plan& p, const ConvArgs& a, cudaStream_t s) {
    const T2d tb = t2d(p, a.spectrum);
    const float2* spec = reinterpret_cast<const float2*>(a.spectrum + p.spec_off);
    const T* u = static_cast<const T*>(a.u);
    T* y = static_cast<T*>(a.y);
    const int64_t nimg = a.B * p.C;
    using WT = typename WsOf<T>::type;
    WT* ws = reinterpret_cast<WT*>(a.workspace);
    const int64_t cap = int64_t(a.group_rows) * int64_t(sizeof(float2) / sizeof(WT));
    const int64_t G = cap < 65535 ? cap : 65535;
    const int64_t stride = int64_t(p.ws_row_bytes / sizeof(float2));     // (W/2+1) * H elements
    const int64_t spec_stride = int64_t(p.spec_row_bytes / sizeof(float2));
    const int H = int(p.H), W = int(p.W);
    const int ncol = W / 2 + 1;
    constexpr int NTC = kFC * (MH / 16);
    const size_t smC = size_t(2 * kFC) * fft_padded_size(MH) * sizeof(float2);
    auto ka = k_2dc_rows_fwd<MW, T, 0>;
    auto kb = k_2dc_cols<MH, WT>;
    auto kc = k_2dc_rows_inv<MW, T, true>;
    auto kca = k_2dc_rows_inv<MW, T, false>;
    cudaFuncSetAttribute(ka, cudaFuncAttributeMaxDynamicSharedMemorySize, int(row_smem<MW>()));
    cudaFuncSetAttribute(kb, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smC));
    cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, int(row_smem<MW>()));
    cudaFuncSetAttribute(kca, cudaFuncAttributeMaxDynamicSharedMemorySize, int(row_smem<MW>()));
    const unsigned cblocks = unsigned((ncol + 2 * kFC - 1) / (2 * kFC));
    if constexpr (sizeof(T) == 2) {
        // 256 x 256: the two images of a channel as one complex image on the tensor
        // cores (groups of whole pairs)
        const int64_t Gp = G & ~int64_t(1);
        if (Gp >= 2 && pairs_2dc_tc_path(p, a)) {
            for (int64_t i0 = 0; i0 < nimg; i0 += Gp) {
                const int64_t g = nimg - i0 < Gp ? nimg - i0 : Gp;
                const cudaError_t e = launch_conv_2dc_pairs_tc(p, a, ws, i0, g, stride, s);
                if (e != cudaSuccess) return e;
            }
            return cudaGetLastError();
        }
    }
    for (int64_t i0 = 0; i0 < nimg; i0 += G) {
        const int64_t g = nimg - i0 < G ? nimg - i0 : G;
        const dim3 gridR(H / kRB, unsigned(g));
        ka<<<gridR, kRowThreads, row_smem<MW>(), s>>>(u, ws, tb, a.B, p.C, p.order, H, i0, stride);
        for (int st = 1; st < p.order; ++st) {
            kb<<<dim3(cblocks, unsigned(g)), NTC, smC, s>>>(ws, spec, tb, ncol, a.B, st - 1, i0, stride, spec_stride,
                                                            a.spec_C, a.spec_per_b);
            if (st < p.order - 1)
                kca<<<gridR, kRowThreads, row_smem<MW>(), s>>>(u, y, ws, tb, a.B, p.C, p.order, p.order - st - 1, H,
                                                               i0, stride);
            else
                kc<<<gridR, kRowThreads, row_smem<MW>(), s>>>(u, y, ws, tb, a.B, p.C, p.order, 0, H, i0, stride);
        }
    }
    return cudaGetLastError();
}

// Depth tables of the 3-D form: the depth pass is the 2-D register column
// pass with the H tables swapped for the N1 ones.
T2d t2d_depth(const Plan& p, const uint8_t* spectrum) {
    const float2* t = reinterpret_cast<const float2*>(spectrum + p.tables_off);
    T2d tb = t2d(p, spectrum);
    tb.fftH = t + p.t_fft_d;
    tb.twist_h = t + p.t_twist_d;
    return tb;
}

// 3-D spectrum build: row pass of k into the lower quarter of each channel's
// region, forward column pass into the upper half, then the depth lines in
// spectrum mode (one CTA per channel walking the lines in increasing order,
// so each line's output only overwrites consumed input).
template <int MW, int MH, int MD>
cudaError_t spectrum_3d_t(const Plan& p, const SpectrumArgs& a, cudaStream_t s) {
    const T2d tb = t2d(p, a.spectrum);
    const T2d tbd = t2d_depth(p, a.spectrum);
    float2* rows = reinterpret_cast<float2*>(a.spectrum + p.spec_off);
    const int64_t nimg = (p.order - 1) * p.C;
    const int64_t stride = int64_t(p.spec_row_bytes / sizeof(float2));    // lines * 2 N1
    const int N1 = int(p.L), H = int(p.H), W = int(p.W);
    const int64_t nlines = int64_t(W + 1) * 2 * H;
    const int64_t ws2_off = nlines * N1;                                  // upper half
    const size_t smA = row_smem<MW>();
    const size_t smC = size_t(2 * kFC) * fft_padded_size(MH) * sizeof(float2);
    const size_t smB = col_smem2<MD>(1);
    auto kf = k_2d_rows_fwd<MW, float, 1>;
    auto kh = k_2d_rows_fwd<MW, __nv_bfloat16, 1>;
    auto kcf = k_3d_cols_fwd<MH, float2>;
    auto kb = k_2d_cols<MD, 1, float2>;
    cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smA));
    cudaFuncSetAttribute(kh, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smA));
    cudaFuncSetAttribute(kcf, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smC));
    cudaFuncSetAttribute(kb, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smB));
    const float s16 = 1.0f / (16.0f * float(N1) * float(H) * float(W));
    for (int64_t i0 = 0; i0 < nimg; i0 += 32768) {
        const int64_t g = nimg - i0 < 32768 ? nimg - i0 : 32768;
        const dim3 gridA(N1 * H / kRB, unsigned(g));
        if (a.k_dtype == DT_F32)
            kf<<<gridA, kRowThreads, smA, s>>>(static_cast<const float*>(a.k), rows + i0 * stride, tb, 1, 1, 2,
                                               N1 * H, i0, stride, 0);
        else
            kh<<<gridA, kRowThreads, smA, s>>>(static_cast<const __nv_bfloat16*>(a.k), rows + i0 * stride, tb, 1, 1,
                                               2, N1 * H, i0, stride, 0);
        kcf<<<dim3(unsigned((W + 1) * (N1 / kFC)), unsigned(g)), kFC * (MH / 16), smC, s>>>(rows + i0 * stride, tb,
                                                                                          N1, 0, ws2_off, stride);
        // k_2d_cols in spectrum mode reads its columns from the upper half
        // (offset ncol * MD = nlines * N1) and writes 2 N1 entries per line
        spectrum_cols_waves(kb, int(nlines), unsigned(g), smB, s, rows + i0 * stride, tbd, int(nlines - 1), int(p.C),
                            i0, stride, a.D, s16);
    }
    return cudaGetLastError();
}

template <int MW, int MH, int MD, typename T>
cudaError_t conv_3d_t(const Plan& p, const ConvArgs& a, cudaStream_t s) {
    const T2d tb = t2d(p, a.spectrum);
    const T2d tbd = t2d_depth(p, a.spectrum);
    const float2* spec = reinterpret_cast<const float2*>(a.spectrum + p.spec_off);
    const T* u = static_cast<const T*>(a.u);
    T* y = static_cast<T*>(a.y);
    const int64_t nimg = a.B * p.C;
    using WT = typename WsOf<T>::type;
    WT* ws = reinterpret_cast<WT*>(a.workspace);
    const int64_t cap = int64_t(a.group_rows) * int64_t(sizeof(float2) / sizeof(WT));
    const int64_t G = cap < 65535 ? cap : 65535;
    const int64_t stride = int64_t(p.ws_row_bytes / sizeof(float2));      // ws1 + ws2 elements
    const int64_t spec_stride = int64_t(p.spec_row_bytes / sizeof(float2));
    const int N1 = int(p.L), H = int(p.H), W = int(p.W);
    const int64_t nlines = int64_t(W + 1) * 2 * H;
    const int64_t ws2_off = int64_t(W + 1) * N1 * H;
    const size_t smC = size_t(2 * kFC) * fft_padded_size(MH) * sizeof(float2);
    const size_t smD = size_t(2 * kFC) * fft_padded_size(MD) * sizeof(float2);
    auto ka = k_2d_rows_fwd<MW, T, 0>;
    auto kcf = k_3d_cols_fwd<MH, WT>;
    auto kd = k_2df_cols<MD, WT>;
    auto kci = k_3d_cols_inv<MH, WT>;
    auto kc = k_2d_rows_inv<MW, T, true>;
    auto kca = k_2d_rows_inv<MW, T, false>;
    cudaFuncSetAttribute(ka, cudaFuncAttributeMaxDynamicSharedMemorySize, int(row_smem<MW>()));
    cudaFuncSetAttribute(kcf, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smC));
    cudaFuncSetAttribute(kd, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smD));
    cudaFuncSetAttribute(kci, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smC));
    cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, int(row_smem<MW>()));
    cudaFuncSetAttribute(kca, cudaFuncAttributeMaxDynamicSharedMemorySize, int(row_smem<MW>()));
    const unsigned cblocks = unsigned((W + 1) * (N1 / kFC));
    const unsigned dblocks = unsigned((nlines + kFC - 1) / kFC);
    for (int64_t i0 = 0; i0 < nimg; i0 += G) {
        const int64_t g = nimg - i0 < G ? nimg - i0 : G;
        const dim3 gridR(N1 * H / kRB, unsigned(g));
        ka<<<gridR, kRowThreads, row_smem<MW>(), s>>>(u, ws, tb, a.B, p.C, p.order, N1 * H, i0, stride, 0);
        for (int st = 1; st < p.order; ++st) {
            kcf<<<dim3(cblocks, unsigned(g)), kFC * (MH / 16), smC, s>>>(ws, tb, N1, 0, ws2_off, stride);
            kd<<<dim3(dblocks, unsigned(g)), kFC * (MD / 16), smD, s>>>(ws + ws2_off, spec, tbd, int(nlines - 1),
                                                                        a.B, p.C, st - 1, i0, stride, spec_stride,
                                                                        a.spec_C, a.spec_per_b, int(g));
            kci<<<dim3(cblocks, unsigned(g)), kFC * (MH / 16), smC, s>>>(ws, tb, N1, 0, ws2_off, stride);
            if (st < p.order - 1)
                kca<<<gridR, kRowThreads, row_smem<MW>(), s>>>(u, y, ws, tb, a.B, p.C, p.order, p.order - st - 1,
                                                               N1 * H, i0, stride);
            else
                kc<<<gridR, kRowThreads, row_smem<MW>(), s>>>(u, y, ws, tb, a.B, p.C, p.order, 0, N1 * H, i0, stride);
        }
    }
    return cudaGetLastError();
}

// Engine choice per pass, measured on B=2, C=256, 256 x 256, bf16 (us per
// call): CTA rows + register columns 843, register rows + register columns
// 921, CTA rows + CTA columns 939, register rows + CTA columns 1020.
constexpr bool kRowsReg2D = false;
constexpr bool kColsReg2D = true;

template <int MW, int MH>
cudaError_t conv_2d(const Plan& p, const ConvArgs& a, cudaStream_t s) {
    if (p.path == PATH_GRID_2D_CIRC)
        return a.dtype == DT_F32 ? conv_2dc_t<MW, MH, float>(p, a, s) : conv_2dc_t<MW, MH, __nv_bfloat16>(p, a, s);
    return a.dtype == DT_F32 ? conv_2d_t<MW, MH, float, kRowsReg2D, kColsReg2D>(p, a, s)
                             : conv_2d_t<MW, MH, __nv_bfloat16, kRowsReg2D, kColsReg2D>(p, a, s);
}

template <int MW, int MH>
cudaError_t spectrum_2d(const Plan& p, const SpectrumArgs& a, cudaStream_t s) {
    if (p.path == PATH_GRID_2D_CIRC) return spectrum_2dc_t<MW, MH>(p, a, s);
    return spectrum_2d_t<MW, MH>(p, a, s);
}

template <int MW>
cudaError_t dispatch_h_spec(const Plan& p, const SpectrumArgs& a, cudaStream_t s) {
    switch (p.H) {
        case 16: return spectrum_2d<MW, 16>(p, a, s);
        case 32: return spectrum_2d<MW, 32>(p, a, s);
        case 64: return spectrum_2d<MW, 64>(p, a, s);
        case 128: return spectrum_2d<MW, 128>(p, a, s);
        case 256: return spectrum_2d<MW, 256>(p, a, s);
        case 512: return spectrum_2d<MW, 512>(p, a, s);
        default: return cudaErrorInvalidValue;
    }
}

template <int MW>
cudaError_t dispatch_h_conv(const Plan& p, const ConvArgs& a, cudaStream_t s) {
    switch (p.H) {
        case 16: return conv_2d<MW, 16>(p, a, s);
        case 32: return conv_2d<MW, 32>(p, a, s);
        case 64: return conv_2d<MW, 64>(p, a, s);
        case 128: return conv_2d<MW, 128>(p, a, s);
        case 256: return conv_2d<MW, 256>(p, a, s);
        case 512: return conv_2d<MW, 512>(p, a, s);
        default: return cudaErrorInvalidValue;
    }
}

template <int MW, int MH>
cudaError_t dispatch_d(const Plan& p, const void* args, cudaStream_t s, bool spectrum) {
    switch (p.L) {
#define HYENA_3D_CASE(N)                                                                          \
    case N:                                                                                       \
        if (spectrum) return spectrum_3d_t<MW, MH, N>(p, *static_cast<const SpectrumArgs*>(args), s); \
        {                                                                                         \
            const ConvArgs& a = *static_cast<const ConvArgs*>(args);                              \
            return a.dtype == DT_F32 ? conv_3d_t<MW, MH, N, float>(p, a, s)                      \
                                     : conv_3d_t<MW, MH, N, __nv_bfloat16>(p, a, s);              \
        }
        HYENA_3D_CASE(16)
        HYENA_3D_CASE(32)
        HYENA_3D_CASE(64)
        HYENA_3D_CASE(128)
#undef HYENA_3D_CASE
        default: return cudaErrorInvalidValue;
    }
}

template <int MW>
cudaError_t dispatch_3d_h(const Plan& p, const void* args, cudaStream_t s, bool spectrum) {
    switch (p.H) {
        case 16: return dispatch_d<MW, 16>(p, args, s, spectrum);
        case 32: return dispatch_d<MW, 32>(p, args, s, spectrum);
        case 64: return dispatch_d<MW, 64>(p, args, s, spectrum);
        case 128: return dispatch_d<MW, 128>(p, args, s, spectrum);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t dispatch_3d(const Plan& p, const void* args, cudaStream_t s, bool spectrum) {
    switch (p.W) {
        case 16: return dispatch_3d_h<8>(p, args, s, spectrum);
        case 32: return dispatch_3d_h<16>(p, args, s, spectrum);
        case 64: return dispatch_3d_h<32>(p, args, s, spectrum);
        case 128: return dispatch_3d_h<64>(p, args, s, spectrum);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_spectrum_3d(const Plan& p, const SpectrumArgs& a, cudaStream_t s) {
    return dispatch_3d(p, &a, s, true);
}

cudaError_t launch_conv_3d(const Plan& p, const ConvArgs& a, cudaStream_t s) {
    return dispatch_3d(p, &a, s, false);
}

cudaError_t launch_spectrum_2d(const Plan& p, const SpectrumArgs& a, cudaStream_t s) {
    switch (p.W) {
        case 16: return dispatch_h_spec<8>(p, a, s);
        case 32: return dispatch_h_spec<16>(p, a, s);
        case 64: return dispatch_h_spec<32>(p, a, s);
        case 128: return dispatch_h_spec<64>(p, a, s);
        case 256: return dispatch_h_spec<128>(p, a, s);
        case 512: return dispatch_h_spec<256>(p, a, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_conv_2d(const Plan& p, const ConvArgs& a, cudaStream_t s) {
    switch (p.W) {
        case 16: return dispatch_h_conv<8>(p, a, s);
        case 32: return dispatch_h_conv<16>(p, a, s);
        case 64: return dispatch_h_conv<32>(p, a, s);
        case 128: return dispatch_h_conv<64>(p, a, s);
        case 256: return dispatch_h_conv<128>(p, a, s);
        case 512: return dispatch_h_conv<256>(p, a, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace hyena
