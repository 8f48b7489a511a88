// multipass.cu -- the four-step path for 32768 <= L <= 2^20.
//
// Same method as the on-chip path ([P4] "HyenaDNA operator walk-through"
// (adg.csdn.net), section 二.1 gating loop, section 二.2 fftconv; zero-padded
// 2L FFT as two M = L/2-point chains with a pairwise untangle / spectrum
// multiply / re-tangle), but an M-point chain no longer fits in one SM, so
// each chain DFT is split four-step style with M = M1 * M2,
// n = M2 n1 + n2, m = m1 + M1 m2:
//
//   DFT_M(x)[m1 + M1 m2] = sum_n2 w_M2^(n2 m2) w_M^(n2 m1) sum_n1 x[M2 n1 + n2] w_M1^(n1 m1)
//
//   pass A  (per block of 16 columns n2): gated input -> column DFT_M1 for
//           both chains -> times w_M^(m1 n2) -> workspace
//   pass B  (per unit = two rows m1 that hold every partner bin): row DFT_M2,
//           pair step with the spectrum, row IDFT_M2 -> workspace (in place)
//   pass C  (per block of columns): times w_M^(-m1 n2) -> column IDFT_M1 ->
//           combine the chains -> output gate -> y; for order > 2 the next
//           gate and the next step's pass A run in the same kernel (pass CA)
//
// Workspace row layout (complex64): [chain e | chain o], each M1 rows of M2
// stored as M1/2 "units" of two rows.  Chain e unit 0 holds rows (0, M1/2),
// unit u > 0 rows (u, M1-u); chain o unit u holds rows (u, M1-1-u).  Bin
// m = m1 + M1 m2 pairs with M-m (chain e) or M-1-m (chain o), which always
// lies in the same unit, so pass B needs nothing outside its unit.
// The spectrum row has the same shape: one float4 pair entry per workspace
// complex pair, written in place by the spectrum build.
//
// Rows are processed in groups sized to the caller's workspace (by default
// the whole batch up to 4 GiB: fewer launches and fewer partly filled last
// waves measured faster than groups small enough to stay in the 126 MB L2).
// With bf16 storage the workspace holds bf16 (re, im) pairs.
#include "common.cuh"
#include "cta_fft.cuh"
#include "kernels.h"
#include "reg_fft.cuh"

namespace hyena {

namespace {


struct MpTables {
    const float2* fftA;     // CTA FFT of size M1
    const float2* fftB;     // CTA FFT of size M2
    const float2* four;     // w_M^(m1 n2), [M1][M2]
    const float2* twist_hi; // w_L^(M2 n1)
    const float2* twist_lo; // w_L^(n2)
    const float2* unt1;     // w_L^(m1)
    const float2* unt2;     // w_(2 M2)^(m2)
    const float2* unt_c;    // w_2L^1
};

MpTables mp_tables(const Plan& p, const uint8_t* spectrum) {
    const float2* t = reinterpret_cast<const float2*>(spectrum + p.tables_off);
    return MpTables{t + p.t_fft_a, t + p.t_fft_b, t + p.t_four, t + p.t_twist_hi,
                    t + p.t_twist_lo, t + p.t_unt1, t + p.t_unt2, t + p.t_unt_c};
}

// (unit, which) slot of row m1 in a chain's workspace block.
template <int M1>
__device__ __forceinline__ int mp_slot(bool odd, int m1) {
    if (!odd) {
        if (m1 == 0) return 0;
        if (m1 == M1 / 2) return 1;
        return m1 < M1 / 2 ? 2 * m1 : 2 * (M1 - m1) + 1;
    }
    return m1 < M1 / 2 ? 2 * m1 : 2 * (M1 - 1 - m1) + 1;
}

// ------------------------------------------------------------------ pass B
// The pair step for one pair entry: A at bin m (row a), B at its partner.
__device__ __forceinline__ void pair_conv(float2& A, float2& Bv, float2 w, float4 kk) {
    const float2 S = cadd(A, cconj(Bv));
    const float2 T = cmul_i(cmul(w, csub(A, cconj(Bv))));
    const float2 Yf = cmul(csub(S, T), make_float2(kk.x, kk.y));
    const float2 Yg = cmul(cconj(cadd(S, T)), make_float2(kk.z, kk.w));
    const float2 P = cadd(Yf, cconj(Yg));
    const float2 U = cmul_i(cmulc(csub(Yf, cconj(Yg)), w));
    A = cadd(P, U);
    Bv = cconj(csub(P, U));
}

__device__ __forceinline__ float4 pair_spec(float2 A, float2 Bv, float2 w, float d, float s4) {
    const float2 S = cadd(A, cconj(Bv));
    const float2 T = cmul_i(cmul(w, csub(A, cconj(Bv))));
    const float2 Xf = cscale(csub(S, T), 0.5f);
    const float2 Xg = cscale(cconj(cadd(S, T)), 0.5f);
    return make_float4((Xf.x + d) * s4, Xf.y * s4, (Xg.x + d) * s4, Xg.y * s4);
}

// MODE 0: convolution (multiply by the spectrum, inverse row DFT, store back);
//         workspace row i of the launch is (b, c) row r = row0 + i, r = c*B + b,
//         and uses spectrum row (step, c).
// MODE 1: spectrum build: workspace row i is spectrum row r = row0 + i
//         (= step*C + c); the pair entries of K~ replace the unit in place.
template <int M2, int MODE, typename W>
__device__ __forceinline__ void mp_unit_generic(W* __restrict__ ws, const float4* __restrict__ spec,
                                                const MpTables& tb, int M1, int64_t row0, int64_t ws_row_stride,
                                                int64_t spec_row_stride4, int step, int64_t B, int64_t C,
                                                const float* __restrict__ D, int unit_index, float2* smem,
                                                int64_t SC, int64_t SB) {
    constexpr int PS = fft_padded_size(M2);
    const int M = M1 * M2;
    const int64_t L = int64_t(2) * M;
    const bool odd = unit_index >= M1 / 2;
    const int u = odd ? unit_index - M1 / 2 : unit_index;
    const int ra = u;                       // first row of the unit (0 for chain e unit 0)
    const int64_t r = row0 + blockIdx.y;
    static_assert(MODE == 0 || sizeof(W) == sizeof(float2), "the spectrum build writes complex64 rows");
    W* unit = ws + int64_t(blockIdx.y) * ws_row_stride + (odd ? M : 0) + int64_t(2 * u) * M2;
    float2* b0 = smem;
    float2* b1 = smem + PS;
    for (int i = threadIdx.x; i < M2; i += blockDim.x) {
        b0[fft_pad(i)] = ws_ld(unit + i);
        b1[fft_pad(i)] = ws_ld(unit + M2 + i);
    }
    __syncthreads();
    cta_fft_forward<M2>(smem, 2, PS, tb.fftB);
    const float2 wodd = odd ? __ldg(tb.unt_c) : make_float2(1.0f, 0.0f);
    const float2 wa = __ldg(tb.unt1 + ra);
    const float2 wb0 = __ldg(tb.unt1 + M1 / 2);
    const float4* sp = nullptr;
    float4* sp_out = nullptr;
    float d = 0.0f;
    const float s4 = 1.0f / float(4 * L);
    if (MODE == 0) {
        const int64_t c = r / B, b = r - c * B;
        sp = spec + (int64_t(step) * SC + b * SB + c) * spec_row_stride4 + (odd ? M / 2 : 0) + int64_t(u) * M2;
    } else {
        sp_out = reinterpret_cast<float4*>(unit);   // the unit's 2*M2 complex = M2 float4 entries
        d = D ? __ldg(D + r) : 0.0f;
    }
    for (int e = threadIdx.x; e < M2; e += blockDim.x) {
        float2* bufA;
        float2* bufB;
        int pa, pb;
        float2 w;
        bool special = false;
        if (!odd && u == 0) {
            if (e == 0) {
                special = true;
                bufA = b0; bufB = b0;
                pa = fft_pad(fft_bin_pos<M2>(0));
                pb = fft_pad(fft_bin_pos<M2>(M2 / 2));
                w = make_float2(0.0f, -1.0f);   // w_2L^(L/2)
            } else if (e < M2 / 2) {
                bufA = b0; bufB = b0;
                pa = fft_pad(fft_bin_pos<M2>(e));
                pb = fft_pad(fft_bin_pos<M2>(M2 - e));
                w = __ldg(tb.unt2 + e);
            } else {
                const int jj = e - M2 / 2;
                bufA = b1; bufB = b1;
                pa = fft_pad(fft_bin_pos<M2>(jj));
                pb = fft_pad(fft_bin_pos<M2>(M2 - 1 - jj));
                w = cmul(wb0, __ldg(tb.unt2 + jj));
            }
        } else {
            bufA = b0; bufB = b1;
            pa = fft_pad(fft_bin_pos<M2>(e));
            pb = fft_pad(fft_bin_pos<M2>(M2 - 1 - e));
            w = cmul(cmul(wa, __ldg(tb.unt2 + e)), wodd);
        }
        if (special) {
            // f = 0 and f = L from Z[0]; the self pair f = L/2 (bin m = M/2)
            const float2 A = bufA[pa];
            const float2 Cc = bufB[pb];
            if (MODE == 0) {
                const float4 kk = __ldg(sp + e);
                const float y0 = 2.0f * (A.x + A.y) * kk.x;
                const float yL = 2.0f * (A.x - A.y) * kk.y;
                float2 c1 = Cc, c2 = Cc;
                pair_conv(c1, c2, w, make_float4(kk.z, kk.w, kk.z, kk.w));
                bufA[pa] = make_float2(y0 + yL, y0 - yL);
                bufB[pb] = c1;
            } else {
                const float4 h = pair_spec(Cc, Cc, w, d, s4);
                sp_out[e] = make_float4((A.x + A.y + d) * s4, (A.x - A.y + d) * s4, h.x, h.y);
            }
        } else {
            float2 A = bufA[pa];
            float2 Bv = bufB[pb];
            if (MODE == 0) {
                pair_conv(A, Bv, w, __ldg(sp + e));
                bufA[pa] = A;
                bufB[pb] = Bv;
            } else {
                sp_out[e] = pair_spec(A, Bv, w, d, s4);
            }
        }
    }
    if (MODE == 1) return;
    __syncthreads();
    cta_fft_inverse<M2>(smem, 2, PS, tb.fftB);
    for (int i = threadIdx.x; i < M2; i += blockDim.x) {
        ws_st(unit + i, b0[fft_pad(i)]);
        ws_st(unit + M2 + i, b1[fft_pad(i)]);
    }
}

// ===========================================================================
// Register-resident passes (reg_fft.cuh).  Column passes: a CTA of M1 threads
// handles 16 columns n2; thread t = 16 g + j holds 16 points of column j for
// both chains.  Row pass: a CTA handles NU units of two rows; thread g of a
// unit holds 16 points of both rows.  After the forward row FFT, row a's
// position q pairs with row b's position M2-1-q (every digit of the bin is
// complemented), so thread g finds its partners at thread M2/16-1-g, slot
// 15-k; the spectrum entries of these units are stored in that thread order,
// entry [k][g].  Chain e unit 0 (rows 0 and M1/2, partners inside each row)
// keeps the natural entry order and the generic kernel above.
// ===========================================================================

// Four-step twiddles w_M^(m1 n2) of a thread's 16 column positions 16 g + k,
// m1 = fft_pos_bin(16 g + k).  For M1 = 128 and 256 the bins of k = 0..7 and of
// k = 8..15 are two runs with step 16, so three table entries and 14 complex
// multiplies replace 16 scattered table reads (relative error < 1e-6).
template <int M1>
struct ColTw {
    float2 a, b, step;
    __device__ __forceinline__ ColTw(const MpTables& tb, int M2, int n2, int g) {
        static_assert(M1 == 128 || M1 == 256, "run structure holds for M1 = 128, 256");
        a = __ldg(tb.four + int64_t(fft_pos_bin<M1>(16 * g)) * M2 + n2);
        b = __ldg(tb.four + int64_t(fft_pos_bin<M1>(16 * g + 8)) * M2 + n2);
        step = __ldg(tb.four + int64_t(16) * M2 + n2);          // w_M^(16 n2)
    }
    // twiddle of position k (call with k = 0, 1, ..., 15 in order)
    __device__ __forceinline__ float2 next(int k) {
        float2 r;
        if (k < 8) { r = a; a = cmul(a, step); }
        else { r = b; b = cmul(b, step); }
        return r;
    }
};

template <int M1, typename W>
__device__ __forceinline__ void cols_store_ws(float2 (&x)[2][16], const MpTables& tb, W* __restrict__ ws_row,
                                              int M2, int n2, int g) {
    const int M = M1 * M2;
    ColTw<M1> tw(tb, M2, n2, g);
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const int m1 = fft_pos_bin<M1>(16 * g + k);
        const float2 w = tw.next(k);
        ws_st(ws_row + int64_t(mp_slot<M1>(false, m1)) * M2 + n2, cmul(x[0][k], w));
        ws_st(ws_row + M + int64_t(mp_slot<M1>(true, m1)) * M2 + n2, cmul(x[1][k], w));
    }
}

// Input staging of the column passes: the CTA's columns n2_0 .. n2_0+15 of
// every row n1 of one channel row are 32 consecutive samples from
// 2 (M2 n1 + n2_0); they and the two samples before them (the short conv's
// halo) are copied to shared memory with 16-byte loads.  Segment n1 sits at
// seg + n1 kSegStride: the samples start at element 8, the halo at 6.
constexpr int kSegStride = 40;

template <int M1, typename T>
constexpr size_t seg_bytes() {
    return size_t(M1) * kSegStride * sizeof(T);
}

// Issue (cp.async, not waited) the copies of one channel row's segments.
template <int M1, typename T>
__device__ __forceinline__ void stage_segments(const T* __restrict__ src, int M2, int n2_0, T* __restrict__ seg) {
    constexpr int PER = 16 / int(sizeof(T));      // elements per 16-byte chunk
    constexpr int NCH = 32 / PER;                  // chunks per segment
    for (int idx = threadIdx.x; idx < M1 * (NCH + 1); idx += blockDim.x) {
        const int n1 = idx / (NCH + 1), ch = idx - n1 * (NCH + 1);
        const int64_t t0 = 2 * (int64_t(M2) * n1 + n2_0);
        T* dst = seg + n1 * kSegStride;
        if (ch < NCH) {
            cp_async_bytes16(dst + 8 + ch * PER, src + t0 + ch * PER);
        } else if (t0 >= 2) {
            cp_async_small<2 * int(sizeof(T))>(dst + 6, src + t0 - 2);
        } else {
            dst[6] = T(0.0f);
            dst[7] = T(0.0f);
        }
    }
}

// Short conv (or the raw samples, taps off) at the two samples of column j of
// a staged segment.
template <typename T>
__device__ __forceinline__ float2 seg_pair(const T* row, int j, const Taps& tp) {
    const float2 cur = load2_shared(row + 8 + 2 * j);
    if (!tp.on) return cur;
    const float2 prev = load2_shared(row + 6 + 2 * j);
    float2 r;
    r.x = fmaf(tp.w0, prev.x, fmaf(tp.w1, prev.y, fmaf(tp.w2, cur.x, tp.b)));
    r.y = fmaf(tp.w0, prev.y, fmaf(tp.w1, cur.x, fmaf(tp.w2, cur.y, tp.b)));
    return r;
}

// MODE 0: gated input x_{order-1} * v from u (first order step); MODE 1: filter k.
template <int M1, typename T, int MODE>
__global__ void __launch_bounds__(M1, 512 / M1)
k_mpf_cols_fwd(const T* __restrict__ src, typename WsSel<T, MODE>::type* __restrict__ ws, MpTables tb,
               const float* __restrict__ sc_w,
               const float* __restrict__ sc_b, int64_t B, int64_t C, int order, int M2, int64_t row0,
               int64_t ws_row_stride) {
    extern __shared__ float2 smem[];
    constexpr int TPT = M1 / 16;
    constexpr int PS = fft_padded_size(M1);
    const int t = threadIdx.x, j = t & 15, g = t >> 4;
    const int n2 = blockIdx.x * 16 + j;
    const int64_t r = row0 + blockIdx.y;
    const int64_t L = int64_t(2) * M1 * M2;
    auto* ws_row = ws + int64_t(blockIdx.y) * ws_row_stride;
    const T* xg;
    const T* vr = nullptr;
    Taps tg{}, tv{};
    if (MODE == 0) {
        const int64_t c = r / B, b = r - (r / B) * B;
        const int64_t Ctot = int64_t(order + 1) * C;
        const T* ub = src + b * Ctot * L;
        xg = ub + (int64_t(order - 1) * C + c) * L;
        vr = ub + (int64_t(order) * C + c) * L;
        tg = load_taps(sc_w, sc_b, int64_t(order - 1) * C + c);
        tv = load_taps(sc_w, sc_b, int64_t(order) * C + c);
    } else {
        xg = src + r * L;
    }
    float2 x[2][16];
    T* seg = reinterpret_cast<T*>(smem);                  // x segments, then v segments
    T* segv = seg + M1 * kSegStride;
    const int n2_0 = blockIdx.x * 16;
    stage_segments<M1, T>(xg, M2, n2_0, seg);
    if (MODE == 0) stage_segments<M1, T>(vr, M2, n2_0, segv);
    cp_async_commit();
    cp_async_wait_all();
    __syncthreads();
    const Taps raw{0.0f, 0.0f, 1.0f, 0.0f, false};
#pragma unroll
    for (int s = 0; s < 16; ++s) {
        const int n1 = g + TPT * s;
        x[0][s] = seg_pair(seg + n1 * kSegStride, j, MODE == 0 ? tg : raw);
        if (MODE == 0) {
            const float2 v = seg_pair(segv + n1 * kSegStride, j, tv);
            x[0][s] = make_float2(x[0][s].x * v.x, x[0][s].y * v.y);
        }
    }
    __syncthreads();                                   // staging read: the FFT reuses the buffer
    const float2 tlo = __ldg(tb.twist_lo + n2);
#pragma unroll
    for (int s = 0; s < 16; ++s) x[1][s] = cmul(x[0][s], cmul(__ldg(tb.twist_hi + g + TPT * s), tlo));
    float2* const buf[2] = {smem + j * PS, smem + (16 + j) * PS};
    reg_fft_forward<M1, 2>(x, buf, g, tb.fftA);
    cols_store_ws<M1>(x, tb, ws_row, M2, n2, g);
}

// Inverse columns.  FINAL: output gate x0, store y.  Otherwise gate with
// x_{gnext} and run the next step's forward column pass in place.
template <int M1, typename T, bool FINAL>
__global__ void __launch_bounds__(M1, 512 / M1)
k_mpf_cols_inv(const T* __restrict__ u, T* __restrict__ y, typename WsOf<T>::type* __restrict__ ws, MpTables tb,
               const float* __restrict__ sc_w, const float* __restrict__ sc_b, int64_t B, int64_t C, int order,
               int gnext, int M2, int64_t row0, int64_t ws_row_stride) {
    extern __shared__ float2 smem[];
    constexpr int TPT = M1 / 16;
    constexpr int PS = fft_padded_size(M1);
    const int t = threadIdx.x, j = t & 15, g = t >> 4;
    const int n2 = blockIdx.x * 16 + j;
    const int M = M1 * M2;
    const int64_t r = row0 + blockIdx.y;
    const int64_t L = int64_t(2) * M;
    auto* ws_row = ws + int64_t(blockIdx.y) * ws_row_stride;
    // the gate's channel row is copied (cp.async) while the inverse FFT runs;
    // its region follows the FFT buffer
    const int gate = FINAL ? 0 : gnext;
    T* const seg = reinterpret_cast<T*>(smem + 32 * PS);
    float2 x[2][16];
    {
        ColTw<M1> tw(tb, M2, n2, g);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const int m1 = fft_pos_bin<M1>(16 * g + k);
            const float2 w = tw.next(k);
            x[0][k] = cmulc(ws_ld(ws_row + int64_t(mp_slot<M1>(false, m1)) * M2 + n2), w);
            x[1][k] = cmulc(ws_ld(ws_row + M + int64_t(mp_slot<M1>(true, m1)) * M2 + n2), w);
        }
    }
    {
        const int64_t c = r / B, b = r - c * B;
        const T* xg = u + (b * int64_t(order + 1) * C + int64_t(gate) * C + c) * L;
        stage_segments<M1, T>(xg, M2, blockIdx.x * 16, seg);
        cp_async_commit();
    }
    float2* const buf[2] = {smem + j * PS, smem + (16 + j) * PS};
    reg_fft_inverse<M1, 2>(x, buf, g, tb.fftA);
    const int64_t c = r / B, b = r - c * B;
    const Taps tg = load_taps(sc_w, sc_b, int64_t(gate) * C + c);
    cp_async_wait_all();
    __syncthreads();
    T* yr = y + (b * C + c) * L;
    const float2 tlo = __ldg(tb.twist_lo + n2);
#pragma unroll
    for (int s = 0; s < 16; ++s) {
        const int n1 = g + TPT * s;
        const int64_t n = int64_t(M2) * n1 + n2;
        const float2 tw = cmul(__ldg(tb.twist_hi + n1), tlo);
        const float2 zp = cadd(x[0][s], cmulc(x[1][s], tw));
        const float2 a = seg_pair(seg + n1 * kSegStride, j, tg);
        const float2 z = make_float2(a.x * zp.x, a.y * zp.y);
        if (FINAL) {
            store2(yr + 2 * n, z);
        } else {
            x[0][s] = z;
            x[1][s] = cmul(z, tw);
        }
    }
    if (!FINAL) {
        __syncthreads();
        reg_fft_forward<M1, 2>(x, buf, g, tb.fftA);
        cols_store_ws<M1>(x, tb, ws_row, M2, n2, g);
    }
}

// Row pass over the units other than chain e unit 0.  Units are numbered
// 0 .. M1-2: chain e units 1 .. M1/2-1, then chain o units 0 .. M1/2-1.
// MODE 0: convolution; MODE 1: spectrum build (pair entries in [k][g] order).
template <int M2, int NU, int MODE, typename W>
__global__ void __launch_bounds__(NU * (M2 / 16), 512 / (NU * (M2 / 16)) > 0 ? 512 / (NU * (M2 / 16)) : 1)
k_mpf_rows(W* __restrict__ ws, const float4* __restrict__ spec, MpTables tb, int M1, int64_t row0,
           int64_t ws_row_stride, int64_t spec_row_stride4, int step, int64_t B, int64_t C,
           const float* __restrict__ D, int64_t SC, int64_t SB) {
    extern __shared__ float2 smem[];
    if (blockIdx.x == gridDim.x - 1) {
        // chain e unit 0 (rows 0 and M1/2; partners inside each row, natural entry order)
        mp_unit_generic<M2, MODE, W>(ws, spec, tb, M1, row0, ws_row_stride, spec_row_stride4, step, B, C, D, 0, smem,
                                     SC, SB);
        return;
    }
    constexpr int TPT = M2 / 16;
    constexpr int PS = fft_padded_size(M2);
    const int t = threadIdx.x, w = t / TPT, g = t - (t / TPT) * TPT;
    const int M = M1 * M2;
    const int64_t L = int64_t(2) * M;
    const int units = M1 - 1;
    const int ug = int(blockIdx.x) * NU + w;
    const bool active = ug < units;
    const int ugc = active ? ug : units - 1;
    const bool odd = ugc >= M1 / 2 - 1;
    const int u = odd ? ugc - (M1 / 2 - 1) : ugc + 1;
    const int ra = u;
    W* unit = ws + int64_t(blockIdx.y) * ws_row_stride + (odd ? M : 0) + int64_t(2 * u) * M2;
    float2* const buf[2] = {smem + (2 * w) * PS, smem + (2 * w + 1) * PS};
    float2 x[2][16];
#pragma unroll
    for (int s = 0; s < 16; ++s) {
        x[0][s] = ws_ld(unit + g + TPT * s);
        x[1][s] = ws_ld(unit + M2 + g + TPT * s);
    }
    reg_fft_forward<M2, 2>(x, buf, g, tb.fftB);
    // pair step: row b goes through shared memory to its partner thread
    const int base = fft_pad(16 * g);
    const int pbase = fft_pad(16 * (TPT - 1 - g));
#pragma unroll
    for (int k = 0; k < 16; ++k) buf[1][base + k] = x[1][k];
    __syncthreads();
    const int64_t r = row0 + blockIdx.y;
    float2 wa = __ldg(tb.unt1 + ra);
    if (odd) wa = cmul(wa, __ldg(tb.unt_c));
    if (MODE == 0) {
        const int64_t c = r / B, b = r - c * B;
        const float4* sp = spec + (int64_t(step) * SC + b * SB + c) * spec_row_stride4 + (odd ? M / 2 : 0) +
                           int64_t(u) * M2;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const int m2 = fft_pos_bin<M2>(16 * g + k);
            const float2 wk = cmul(wa, __ldg(tb.unt2 + m2));
            float2 A = x[0][k];
            float2 Bv = buf[1][pbase + 15 - k];
            pair_conv(A, Bv, wk, __ldg(sp + k * TPT + g));
            x[0][k] = A;
            buf[1][pbase + 15 - k] = Bv;
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < 16; ++k) x[1][k] = buf[1][base + k];
        __syncthreads();
        reg_fft_inverse<M2, 2>(x, buf, g, tb.fftB);
        if (active) {
#pragma unroll
            for (int s = 0; s < 16; ++s) {
                ws_st(unit + g + TPT * s, x[0][s]);
                ws_st(unit + M2 + g + TPT * s, x[1][s]);
            }
        }
    } else {
        const float d = D ? __ldg(D + r) : 0.0f;
        const float s4 = 1.0f / float(4 * L);
        float4 out[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const int m2 = fft_pos_bin<M2>(16 * g + k);
            const float2 wk = cmul(wa, __ldg(tb.unt2 + m2));
            out[k] = pair_spec(x[0][k], buf[1][pbase + 15 - k], wk, d, s4);
        }
        __syncthreads();   // every thread of the block has loaded its unit
        if (active) {
            float4* sp_out = reinterpret_cast<float4*>(unit);
#pragma unroll
            for (int k = 0; k < 16; ++k) sp_out[k * TPT + g] = out[k];
        }
    }
}

template <int M2>
constexpr int rows_nu() {
    return (M2 / 16) >= 256 ? 1 : 256 / (M2 / 16);
}

template <int M1, int M2>
cudaError_t spectrum_mp(const Plan& p, const SpectrumArgs& a, cudaStream_t s) {
    const MpTables tb = mp_tables(p, a.spectrum);
    float2* rows = reinterpret_cast<float2*>(a.spectrum + p.spec_off);
    const int64_t nrows = (p.order - 1) * p.C;
    const int64_t stride = int64_t(p.spec_row_bytes / sizeof(float2));
    constexpr int NU = rows_nu<M2>();
    const size_t smA = size_t(32) * fft_padded_size(M1) * sizeof(float2);
    const size_t smB = size_t(2) * fft_padded_size(M2) * sizeof(float2);
    const size_t smR = size_t(2 * NU) * fft_padded_size(M2) * sizeof(float2);
    auto kaf = k_mpf_cols_fwd<M1, float, 1>;
    auto kah = k_mpf_cols_fwd<M1, __nv_bfloat16, 1>;
    auto kr = k_mpf_rows<M2, NU, 1, float2>;
    cudaFuncSetAttribute(kaf, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smA));
    cudaFuncSetAttribute(kah, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smA));
    cudaFuncSetAttribute(kr, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smR));
    const unsigned rblocks = unsigned((M1 - 1 + NU - 1) / NU);
    for (int64_t r0 = 0; r0 < nrows; r0 += 32768) {
        const int64_t g = nrows - r0 < 32768 ? nrows - r0 : 32768;
        if (a.k_dtype == DT_F32)
            kaf<<<dim3(M2 / 16, unsigned(g)), M1, smA, s>>>(static_cast<const float*>(a.k), rows + r0 * stride, tb,
                                                             nullptr, nullptr, 1, 1, 2, M2, r0, stride);
        else
            kah<<<dim3(M2 / 16, unsigned(g)), M1, smA, s>>>(static_cast<const __nv_bfloat16*>(a.k), rows + r0 * stride,
                                                             tb, nullptr, nullptr, 1, 1, 2, M2, r0, stride);
        // every unit; the last block of each row takes chain e unit 0
        kr<<<dim3(rblocks + 1, unsigned(g)), NU * (M2 / 16), smR, s>>>(rows + r0 * stride, nullptr, tb, M1, r0,
                                                                       stride, 0, 0, 1, p.C, a.D, 0, 0);
    }
    return cudaGetLastError();
}

template <int M1, int M2, typename T>
cudaError_t conv_mp_t(const Plan& p, const ConvArgs& a, cudaStream_t s) {
    const MpTables tb = mp_tables(p, a.spectrum);
    const float4* spec = reinterpret_cast<const float4*>(a.spectrum + p.spec_off);
    const T* u = static_cast<const T*>(a.u);
    T* y = static_cast<T*>(a.y);
    const int64_t rows = a.B * p.C;
    // bf16 storage keeps the workspace in bf16 (re, im): rows of 2M elements
    // of half the size, so the caller's workspace holds twice the rows
    using W = typename WsOf<T>::type;
    W* ws = reinterpret_cast<W*>(a.workspace);
    const int64_t cap = int64_t(a.group_rows) * int64_t(sizeof(float2) / sizeof(W));
    int64_t G = cap < 65535 ? cap : 65535;
    const int64_t stride = int64_t(p.ws_row_bytes / sizeof(float2));   // 2M elements
    const int64_t spec_stride4 = int64_t(p.spec_row_bytes / 16);
    constexpr int NU = rows_nu<M2>();
    const size_t smA = size_t(32) * fft_padded_size(M1) * sizeof(float2);
    const size_t smAf = smA > 2 * seg_bytes<M1, T>() ? smA : 2 * seg_bytes<M1, T>();   // x and v segments
    const size_t smAi = smA + seg_bytes<M1, T>();                                       // FFT buffer + gate
    const size_t smR = size_t(2 * NU) * fft_padded_size(M2) * sizeof(float2);
    auto ka = k_mpf_cols_fwd<M1, T, 0>;
    auto kr = k_mpf_rows<M2, NU, 0, W>;
    auto kc = k_mpf_cols_inv<M1, T, true>;
    auto kca = k_mpf_cols_inv<M1, T, false>;
    cudaFuncSetAttribute(ka, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smAf));
    cudaFuncSetAttribute(kr, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smR));
    cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smAi));
    cudaFuncSetAttribute(kca, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smAi));
    const unsigned rblocks = unsigned((M1 - 1 + NU - 1) / NU);
    for (int64_t r0 = 0; r0 < rows; r0 += G) {
        const int64_t g = rows - r0 < G ? rows - r0 : G;
        const dim3 gridA(M2 / 16, unsigned(g));
        ka<<<gridA, M1, smAf, s>>>(u, ws, tb, a.sc_w, a.sc_b, a.B, p.C, p.order, M2, r0, stride);
        for (int st = 1; st < p.order; ++st) {
            kr<<<dim3(rblocks + 1, unsigned(g)), NU * (M2 / 16), smR, s>>>(ws, spec, tb, M1, r0, stride,
                                                                           spec_stride4, st - 1, a.B, p.C, nullptr,
                                                                           a.spec_C, a.spec_per_b);
            if (st < p.order - 1) {
                kca<<<gridA, M1, smAi, s>>>(u, y, ws, tb, a.sc_w, a.sc_b, a.B, p.C, p.order,
                                            p.order - st - 1, M2, r0, stride);
            } else {
                kc<<<gridA, M1, smAi, s>>>(u, y, ws, tb, a.sc_w, a.sc_b, a.B, p.C, p.order, 0, M2, r0,
                                           stride);
            }
        }
    }
    return cudaGetLastError();
}

template <int M1, int M2>
cudaError_t conv_mp(const Plan& p, const ConvArgs& a, cudaStream_t s) {
    return a.dtype == DT_F32 ? conv_mp_t<M1, M2, float>(p, a, s) : conv_mp_t<M1, M2, __nv_bfloat16>(p, a, s);
}

}  // namespace

#define HYENA_MP_SWITCH(FN)                                   \
    switch (p.M) {                                            \
        case 1 << 14: return FN<128, 128>(p, a, s);           \
        case 1 << 15: return FN<128, 256>(p, a, s);           \
        case 1 << 16: return FN<256, 256>(p, a, s);           \
        case 1 << 17: return FN<256, 512>(p, a, s);           \
        case 1 << 18: return FN<256, 1024>(p, a, s);          \
        case 1 << 19: return FN<256, 2048>(p, a, s);          \
        default: return cudaErrorInvalidValue;                \
    }

cudaError_t spectrum_mp_any(const Plan& p, const SpectrumArgs& a, cudaStream_t s) {
    HYENA_MP_SWITCH(spectrum_mp)
}

cudaError_t conv_mp_any(const Plan& p, const ConvArgs& a, cudaStream_t s) {
    HYENA_MP_SWITCH(conv_mp)
}

// The multi-pass rows, and at L = 65536 the cluster plane (cluster.cu) too.
cudaError_t launch_spectrum_multipass(const Plan& p, const SpectrumArgs& a, cudaStream_t s) {
    const cudaError_t e = spectrum_mp_any(p, a, s);
    if (e != cudaSuccess) return e;
    return launch_spectrum_cluster(p, a, s);
}

// bf16 storage at L = 65536 with shared filters runs on the cluster kernel,
// its scratch taken from the workspace; the rest on the multi-pass kernels.
cudaError_t launch_conv_multipass(const Plan& p, const ConvArgs& a, cudaStream_t s) {
    if (cluster_path(p, a)) return launch_conv_cluster(p, a, size_t(a.group_rows) * p.ws_row_bytes, s);
    return conv_mp_any(p, a, s);
}

}  // namespace hyena
