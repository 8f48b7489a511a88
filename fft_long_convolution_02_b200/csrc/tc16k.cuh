// tc16k.cuh -- the complex FFT of N = 16384 points on the sm_100a tensor
// cores (tcgen05), shared by the L = 8192 kernel (onchip_tc.cu) and the
// cluster kernel for L = 65536 (cluster.cu).
//
// FFT_N factors as 16 x 32 x 32 (decimation in frequency):
//   n = a + 1024 s, a = b + 32 q,   f = k1 + 16 k2 + 512 k3
//   stage 1: Y1[a][k1]    = sum_s z[a + 1024 s] w16^(s k1)     x w_N^(a k1)
//   stage 2: Y2[k1,b][k2] = sum_q Y1[b + 32 q][k1] w32^(q k2)  x w1024^(b k2)
//   stage 3: X[k1,k2][k3] = sum_b Y2[k1,b][k2] w32^(b k3)
// and the inverse runs the same stages backwards.  Every stage is one batched
// product of the stage's vectors (rows) with the real form of a DFT matrix:
// operands bf16 in shared memory, fp32 accumulators in tensor memory.  The
// inverse uses the forward matrices through IDFT(x) = conj(DFT(conj x)): the
// spectrum pass stores conj(X K~), so the last inverse stage leaves the
// conjugate of the result.  The first stage (its inputs s) and the last
// inverse stage (its outputs s) belong to the caller, which may use only part
// of s (zero padding, a partial output).
//
// Between stages every thread reads accumulator rows from tensor memory,
// applies the twiddles in fp32 and scatters the values into the next stage's
// operand.  The row orders below are chosen so that each thread's values for
// one destination row are four consecutive slots: one 16-byte store.
//   stage-1 rows   rho1(a)     = 128 T + 32 Q + 8 (b & 3) + (b >> 2), q = a >> 5,
//                                b = a & 31, T = (q & 3) + 4 (q >> 4), Q = (q >> 2) & 3
//   stage-2 rows   rho2(k1, b) = 128 (b & 3) + 32 (k1 >> 2) + 8 (k1 & 3) + (b >> 2)
//   stage-3 rows   rho2(k1, k2)
//   stage-2' rows  128 (k1 & 3) + 32 (k1 >> 2) + b
//   stage-1' rows  a
// A CTA has 256 threads; thread (warp w, lane): lane quarter Q = w & 3, half
// h = w >> 2.  Stage-1 accumulators: 8 tiles x 32 columns; stages 2, 3, 3',
// 2': 4 tiles x 64 columns (256 tensor-memory columns).
//
// Precision: the stage operands and the DFT matrices are rounded to bf16 (8
// significant bits) six times per transform pair; the resulting row error is
// a few 1e-3 relative to the output.
#pragma once
#include <cuda_bf16.h>

#include "common.cuh"
#include "tc_util.cuh"

namespace hyena {
namespace tc16k {

using bf16 = __nv_bfloat16;

constexpr int N = 16384;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kSBO16 = 2 * tc::kLBO;   // operand with K = 16
constexpr uint32_t kSBO32 = 4 * tc::kLBO;   // K = 32
constexpr uint32_t kSBO64 = 8 * tc::kLBO;   // K = 64
constexpr uint32_t kAbytes = 64 * kSBO64;   // 512 rows x K 64 = 1024 rows x K 32
constexpr uint32_t kB32bytes = 8 * kSBO64;  // N 64 x K 64
constexpr uint32_t kTW2bytes = 4 * 16 * 8 * 16;

__device__ __forceinline__ uint32_t pack_bf16(float re, float im) {
    __nv_bfloat162 h = __floats2bfloat162_rn(re, im);
    return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

__device__ __forceinline__ void sts128(uint8_t* base, uint32_t off, uint32_t x, uint32_t y, uint32_t z,
                                       uint32_t w) {
    *reinterpret_cast<uint4*>(base + off) = make_uint4(x, y, z, w);
}

__device__ __forceinline__ int rho1(int a) {
    const int q = a >> 5, b = a & 31;
    return 128 * ((q & 3) + 4 * (q >> 4)) + 32 * ((q >> 2) & 3) + 8 * (b & 3) + (b >> 2);
}

// w_N^e for any integer e: quarter-turn reduction onto the tables
// (twist[j] = w_N^(2j), odd[j] = w_N^(2j+1), j < 2048).
__device__ __forceinline__ float2 wN(int e, const float2* __restrict__ twist, const float2* __restrict__ odd) {
    e &= N - 1;
    const int q = e >> 12, r = e & 4095;
    float2 v = (r & 1) ? __ldg(odd + (r >> 1)) : __ldg(twist + (r >> 1));
    if (q & 1) v = make_float2(v.y, -v.x);   // times -i
    if (q & 2) v = make_float2(-v.x, -v.y);  // times -1
    return v;
}

__device__ __forceinline__ float sc1(const bf16* __restrict__ x, int n, const Taps& tp) {
    const float c = __bfloat162float(x[n]);
    const float p1 = n >= 1 ? __bfloat162float(x[n - 1]) : 0.0f;
    const float p2 = n >= 2 ? __bfloat162float(x[n - 2]) : 0.0f;
    return fmaf(tp.w0, p2, fmaf(tp.w1, p1, fmaf(tp.w2, c, tp.b)));
}

// Two complex values in split form: re = (re_a, re_b), im = (im_a, im_b), so
// that a complex multiply is two packed fp32x2 multiply-adds per value.
struct C2 {
    float2 re, im;
};
__device__ __forceinline__ C2 cmul2(const C2& a, const C2& w) {
    C2 r;
    r.re = __ffma2_rn(make_float2(-a.im.x, -a.im.y), w.im, __fmul2_rn(a.re, w.re));
    r.im = __ffma2_rn(a.im, w.re, __fmul2_rn(a.re, w.im));
    return r;
}
__device__ __forceinline__ C2 c2_splat(float2 w) { return C2{make_float2(w.x, w.x), make_float2(w.y, w.y)}; }
__device__ __forceinline__ C2 c2_of(float2 a, float2 b) { return C2{make_float2(a.x, b.x), make_float2(a.y, b.y)}; }
// Accumulator columns 4p .. 4p+3 hold outputs 2p, 2p+1 as (re, re, im, im).
template <int NCOL>
__device__ __forceinline__ C2 c2_at(const float (&d)[NCOL], int p) {
    return C2{make_float2(d[4 * p], d[4 * p + 1]), make_float2(d[4 * p + 2], d[4 * p + 3])};
}

// Real form of a DFT matrix as a K-major B operand, entry of w_R^(s k): column
// j = 2 s + (0: re, 1: im) of input s; row n holds output k = 2 (n >> 2) + (n & 1),
// real part for (n >> 1) & 1 == 0, else imaginary part, so that the accumulator
// columns of outputs 2p, 2p+1 read (re, re, im, im).  w32 holds (cos, sin) of
// 2 pi i / 32, i < 32 (R divides 32).  The sizes are compile-time constants,
// so that the index arithmetic is shifts and masks.
template <int R, int NOUT, int NIN, uint32_t SBO>
__device__ inline void fill_dft(uint8_t* Bm, const float2* w32) {
    static_assert(32 % R == 0 && (NIN & (NIN - 1)) == 0, "DFT matrix sizes");
    for (int idx = threadIdx.x; idx < 4 * NOUT * NIN; idx += blockDim.x) {
        const int n = idx / (2 * NIN), j = idx % (2 * NIN);
        const int k = 2 * (n >> 2) + (n & 1);
        const bool im_row = (n >> 1) & 1;
        const int e = (k * (j >> 1)) % R;
        const float2 cs = w32[e * (32 / R)];                // w = cv - i sv
        const float cv = cs.x, sv = cs.y;
        float v;
        if (!im_row) v = (j & 1) == 0 ? cv : sv;            // re: Re w xr - Im w xi
        else v = (j & 1) == 0 ? -sv : cv;                   // im: Im w xr + Re w xi
        *reinterpret_cast<bf16*>(Bm + tc::kmaj_off(n, j, SBO)) = __float2bfloat16_rn(v);
    }
}

// Publish this thread's operand writes and issue the stage's MMAs from one
// thread (tiles x ksteps MMAs of M = 128), committed to `mbar`.  Nothing is
// issued once a wait has run out (go == false), so nothing is left in flight.
__device__ __forceinline__ void stage_issue(uint32_t a, uint32_t sbo_a, uint32_t b, uint32_t sbo_b, int tiles,
                                            int ksteps, uint32_t idesc, uint32_t tmem, uint32_t dcols,
                                            uint64_t* mbar, bool go) {
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    if (threadIdx.x == 0 && go) {
        tc::fence_after_sync();
        for (int T = 0; T < tiles; ++T)
            for (int ks = 0; ks < ksteps; ++ks)
                tc::mma_bf16(tmem + uint32_t(T) * dcols,
                             tc::smem_desc(a + uint32_t(T) * 16u * sbo_a + uint32_t(ks) * 2u * tc::kLBO, sbo_a),
                             tc::smem_desc(b + uint32_t(ks) * 2u * tc::kLBO, sbo_b), idesc, uint32_t(ks));
        tc::commit(mbar);
    }
}
// Wait (bounded by budget_ns) for the last issued stage; after a wait has run
// out (ok == false) no further waits are made.
__device__ __forceinline__ bool stage_wait(uint64_t* mbar, uint32_t& phase, bool ok, uint64_t budget_ns) {
    if (!ok) return false;
    const bool done = tc::mbar_wait(mbar, phase, budget_ns);
    phase ^= 1u;
    tc::fence_after_sync();
    return done;
}

// Raw samples n0 .. n0+7 and the two before them (n0 % 8 == 0) of one row.
struct Raw8 {
    uint4 cur;
    uint32_t halo;
};
__device__ __forceinline__ Raw8 load8(const bf16* __restrict__ x, int n0) {
    Raw8 r;
    r.cur = __ldg(reinterpret_cast<const uint4*>(x + n0));
    r.halo = n0 >= 2 ? __ldg(reinterpret_cast<const uint32_t*>(x + n0 - 2)) : 0u;
    return r;
}
// Short conv of the same 8 samples of the two rows of a pair at once: o[i] =
// (sc of row b0, sc of row b1) at sample i, with packed fp32x2 FMAs; tap pairs
// (w for row b0, w for row b1).
struct Taps2 {
    float2 w0, w1, w2, b;
};
__device__ __forceinline__ Taps2 taps2(const Taps& t, float m1) {
    return Taps2{make_float2(t.w0, m1 * t.w0), make_float2(t.w1, m1 * t.w1), make_float2(t.w2, m1 * t.w2),
                 make_float2(t.b, m1 * t.b)};
}
__device__ __forceinline__ void sc8x2(const Raw8& r0, const Raw8& r1, const Taps2& tp, float2 (&o)[8]) {
    const float2 v[10] = {make_float2(bf_lo(r0.halo), bf_lo(r1.halo)),   make_float2(bf_hi(r0.halo), bf_hi(r1.halo)),
                          make_float2(bf_lo(r0.cur.x), bf_lo(r1.cur.x)), make_float2(bf_hi(r0.cur.x), bf_hi(r1.cur.x)),
                          make_float2(bf_lo(r0.cur.y), bf_lo(r1.cur.y)), make_float2(bf_hi(r0.cur.y), bf_hi(r1.cur.y)),
                          make_float2(bf_lo(r0.cur.z), bf_lo(r1.cur.z)), make_float2(bf_hi(r0.cur.z), bf_hi(r1.cur.z)),
                          make_float2(bf_lo(r0.cur.w), bf_lo(r1.cur.w)), make_float2(bf_hi(r0.cur.w), bf_hi(r1.cur.w))};
#pragma unroll
    for (int i = 0; i < 8; ++i)
        o[i] = __ffma2_rn(tp.w0, v[i], __ffma2_rn(tp.w1, v[i + 1], __ffma2_rn(tp.w2, v[i + 2], tp.b)));
}

// Row pairs: pair P of a [B, C] problem is channel c = P / ceil(B/2) with
// batch rows b0 = 2 (P mod ceil(B/2)) and b0 + 1 (has1: that row exists).
struct PairRef {
    int c, b0;
    bool has1;
};
__device__ __forceinline__ PairRef pair_ref(int P, int B) {
    const int nbp = (B + 1) / 2;
    PairRef r;
    r.c = P / nbp;
    r.b0 = 2 * (P - r.c * nbp);
    r.has1 = r.b0 + 1 < B;
    return r;
}

// w1024^e = exp(-2 pi i e / 1024), e < 1024, from sincospif (within an ulp
// or two of the correctly rounded value).
__device__ __forceinline__ float2 w1024(int e) {
    float sv, cv;
    sincospif(float(e) * (1.0f / 512.0f), &sv, &cv);
    return make_float2(cv, -sv);
}

// TW2[(T * 16 + kp) * 8 + l] = (Re w0, Re w1, Im w0, Im w1), w0 = w1024^(b k),
// w1 = w1024^(b (k+1)), b = 4 l + T, k = 2 kp: the stage-2 / stage-3' twiddles.
// Computed in place (no global reads), so that the setup does not wait on memory.
__device__ __forceinline__ void fill_tw2(float4* TW2) {
    for (int idx = threadIdx.x; idx < 4 * 16 * 8; idx += blockDim.x) {
        const int l = idx & 7, kp = (idx >> 3) & 15, T = idx >> 7;
        const int bb = 4 * l + T, k = 2 * kp;
        const float2 w0 = w1024((bb * k) & 1023);
        const float2 w1 = w1024((bb * (k + 1)) & 1023);
        TW2[idx] = make_float4(w0.x, w1.x, w0.y, w1.y);
    }
}

// (cos, sin) of 2 pi i / 32, i < 32, for fill_dft (one thread per entry;
// the caller synchronises before use).
__device__ __forceinline__ void fill_w32(float2* w32) {
    if (threadIdx.x < 32) {
        float sv, cv;
        sincospif(2.0f * float(threadIdx.x) / 32.0f, &sv, &cv);
        w32[threadIdx.x] = make_float2(cv, sv);
    }
}

// What the middle stages of one transform pair need.
struct Ctx {
    uint8_t* A;              // stage operand (kAbytes)
    const float4* TW2;       // fill_tw2 table in shared memory
    const float2* twist;     // w_N^(2j), j < 2048
    const float2* odd;       // w_N^(2j+1), j < 2048
    uint32_t tmem, tl;       // tensor-memory base, this warp's lane quarter
    uint32_t a_addr, b32_addr;
    uint64_t* mbar;
    uint64_t budget;         // bounded-wait budget (ns)
    int issue_mma;
    int lane, Q, hh;
};

// From the issued stage 1 to the stage-1' operand: waits for stage 1, runs
// pass 1, stage 2, pass 2, stage 3 with the spectrum pass (plane = this
// transform's K~ in the order spec8192_pos gives, bf16 (re, im)), stage 3',
// pass 3', stage 2' and pass 2'.  On return the stage-1' operand is in A
// (rows a, K 32 = 16 complex k1), not yet published; the caller issues stage
// 1' with its own B matrix.  `ok` turns false once a wait has run out, after
// which nothing more is issued or waited for.
__device__ __forceinline__ void middle(const Ctx& x, const uint32_t* __restrict__ plane, uint32_t& phase, bool& ok) {
    uint8_t* A = x.A;
    const float4* TW2 = x.TW2;
    const float2* twist = x.twist;
    const float2* odd = x.odd;
    const uint32_t tmem = x.tmem, tl = x.tl, a_addr = x.a_addr, b32_addr = x.b32_addr;
    const int lane = x.lane, Q = x.Q, hh = x.hh;
    // ---------------- stage 1: 8 tiles x (K 16 -> N 32)
    {
        // twiddle w_N^(a k1); vector a = b + 32 q, b = 4 (lane & 7) + (lane >> 3),
        // q = j + 4 Q + 16 h -> stage-2 row (k1, b), chunk Q + 4 h (slots q, j = 0..3).
        // Twiddles run in pairs (k1, k1 + 1), stepped by beta^2.
        const int b1 = 4 * (lane & 7) + (lane >> 3);
        C2 pw[4], st2[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 beta = wN(b1 + 32 * (j + 4 * Q + 16 * hh), twist, odd);
            pw[j] = c2_of(make_float2(1.0f, 0.0f), beta);
            st2[j] = c2_splat(cmul(beta, beta));
        }
        ok = stage_wait(x.mbar, phase, ok, x.budget);
        // row rho2(k1, b): row / 8 = 16 (lane >> 3) + 4 (k1 >> 2) + (k1 & 3), row % 8 = lane & 7
        const uint32_t base = uint32_t(16 * (lane >> 3)) * kSBO64 + uint32_t(Q + 4 * hh) * tc::kLBO +
                              uint32_t(lane & 7) * 16u;
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
            float d[4][16];
#pragma unroll
            for (int j = 0; j < 4; ++j) tc::tmem_ld16(tl + uint32_t(32 * (4 * hh + j) + 16 * half), d[j]);
            tc::tmem_ld_wait();
#pragma unroll
            for (int pp = 0; pp < 4; ++pp) {
                const int k1 = 8 * half + 2 * pp;
                C2 v[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    v[j] = cmul2(c2_at(d[j], pp), pw[j]);
                    pw[j] = cmul2(pw[j], st2[j]);
                }
                sts128(A, base + uint32_t(4 * (k1 >> 2) + (k1 & 3)) * kSBO64,
                       pack_bf16(v[0].re.x, v[0].im.x), pack_bf16(v[1].re.x, v[1].im.x),
                       pack_bf16(v[2].re.x, v[2].im.x), pack_bf16(v[3].re.x, v[3].im.x));
                sts128(A, base + uint32_t(4 * ((k1 + 1) >> 2) + ((k1 + 1) & 3)) * kSBO64,
                       pack_bf16(v[0].re.y, v[0].im.y), pack_bf16(v[1].re.y, v[1].im.y),
                       pack_bf16(v[2].re.y, v[2].im.y), pack_bf16(v[3].re.y, v[3].im.y));
            }
        }
    }
    // ---------------- stage 2: 4 tiles x (K 64 -> N 64)
    stage_issue(a_addr, kSBO64, b32_addr, kSBO64, 4, 4, tc::idesc_bf16(128, 64), tmem, 64, x.mbar, ok && x.issue_mma);
    ok = stage_wait(x.mbar, phase, ok, x.budget);
    {
        // rows (k1 = 4 Q + lane / 8, b = 4 (lane & 7) + T), outputs k2 = 16 h + ..
        // twiddle w1024^(b k2) -> stage-3 row (k1, k2), chunk lane & 7
        // row rho2(k1, k2), k2 = 16 h + 4 gq + i: row / 8 = 16 i + 4 Q + (lane >> 3), row % 8 = 4 h + gq
        const uint32_t base = uint32_t(4 * Q + (lane >> 3)) * kSBO64 + uint32_t(lane & 7) * tc::kLBO +
                              uint32_t(4 * hh) * 16u;
        const float4* tw = TW2 + 64 * hh + (lane & 7);
#pragma unroll 1
        for (int gq = 0; gq < 4; ++gq) {
            float d[4][8];
#pragma unroll
            for (int T = 0; T < 4; ++T) tc::tmem_ld8(tl + uint32_t(64 * T + 32 * hh + 8 * gq), d[T]);
            tc::tmem_ld_wait();
#pragma unroll
            for (int ip = 0; ip < 2; ++ip) {
                C2 v[4];
#pragma unroll
                for (int T = 0; T < 4; ++T) {
                    const float4 w = tw[(T * 16 + 2 * gq + ip) * 8];
                    v[T] = cmul2(c2_at(d[T], ip), C2{make_float2(w.x, w.y), make_float2(w.z, w.w)});
                }
                const int i = 2 * ip;
                sts128(A, base + uint32_t(16 * i) * kSBO64 + uint32_t(gq) * 16u,
                       pack_bf16(v[0].re.x, v[0].im.x), pack_bf16(v[1].re.x, v[1].im.x),
                       pack_bf16(v[2].re.x, v[2].im.x), pack_bf16(v[3].re.x, v[3].im.x));
                sts128(A, base + uint32_t(16 * (i + 1)) * kSBO64 + uint32_t(gq) * 16u,
                       pack_bf16(v[0].re.y, v[0].im.y), pack_bf16(v[1].re.y, v[1].im.y),
                       pack_bf16(v[2].re.y, v[2].im.y), pack_bf16(v[3].re.y, v[3].im.y));
            }
        }
    }
    // ---------------- stage 3; meanwhile this thread loads its spectrum values
    stage_issue(a_addr, kSBO64, b32_addr, kSBO64, 4, 4, tc::idesc_bf16(128, 64), tmem, 64, x.mbar, ok && x.issue_mma);
    {
        // row (k1 = 4 Q + lane / 8, k2 = 4 (lane & 7) + T) keeps its place, slots
        // k3 = 16 h + 4 i + e; spectrum entry uint4 (T * 4 + i) of this thread
        // holds K~ at e = 0..3 (bf16 hi plane).  Stores conj(X K~).
        const uint4* kq = reinterpret_cast<const uint4*>(plane) +
                          (Q * 2 + hh) * 16 * 32 + lane;
        uint4 kv[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) kv[i] = __ldg(kq + 32 * i);
        ok = stage_wait(x.mbar, phase, ok, x.budget);
#pragma unroll
        for (int TH = 0; TH < 8; ++TH) {
            // half TH & 1 of tile T's 32 accumulator columns
            const int T = TH >> 1;
            float d[16];
            tc::tmem_ld16(tl + uint32_t(64 * T + 32 * hh + 16 * (TH & 1)), d);
            tc::tmem_ld_wait();
            const uint32_t rowoff = uint32_t(16 * T + 4 * Q + (lane >> 3)) * kSBO64 + uint32_t(4 * hh) * tc::kLBO +
                                    uint32_t(lane & 7) * 16u;
#pragma unroll
            for (int q4 = 2 * (TH & 1); q4 < 2 * (TH & 1) + 2; ++q4) {
                const uint4 kk = kv[4 * T + q4];
                // bins i = 4 q4 .. 4 q4 + 3 as two split pairs
                const C2 K0{make_float2(bf_lo(kk.x), bf_lo(kk.y)), make_float2(bf_hi(kk.x), bf_hi(kk.y))};
                const C2 K1{make_float2(bf_lo(kk.z), bf_lo(kk.w)), make_float2(bf_hi(kk.z), bf_hi(kk.w))};
                const C2 v0 = cmul2(c2_at(d, 2 * (q4 & 1)), K0);
                const C2 v1 = cmul2(c2_at(d, 2 * (q4 & 1) + 1), K1);
                sts128(A, rowoff + q4 * tc::kLBO, pack_bf16(v0.re.x, -v0.im.x), pack_bf16(v0.re.y, -v0.im.y),
                       pack_bf16(v1.re.x, -v1.im.x), pack_bf16(v1.re.y, -v1.im.y));
            }
        }
    }
    // ---------------- stage 3' (inverse, on conj)
    stage_issue(a_addr, kSBO64, b32_addr, kSBO64, 4, 4, tc::idesc_bf16(128, 64), tmem, 64, x.mbar, ok && x.issue_mma);
    ok = stage_wait(x.mbar, phase, ok, x.budget);
    {
        // rows (k1 = 4 Q + lane / 8, k2 = 4 (lane & 7) + T), outputs b = 16 h + ..
        // twiddle w1024^(b k2) -> stage-2' row (k1, b), chunk lane & 7
        // row 128 (lane >> 3) + 32 Q + b, b = 16 h + 4 gq + i:
        // row / 8 = 16 (lane >> 3) + 4 Q + 2 h + (gq >> 1), row % 8 = 4 (gq & 1) + i
        const uint32_t base = uint32_t(16 * (lane >> 3) + 4 * Q + 2 * hh) * kSBO64 + uint32_t(lane & 7) * tc::kLBO;
        const float4* tw = TW2 + 64 * hh + (lane & 7);
#pragma unroll 1
        for (int gq = 0; gq < 4; ++gq) {
            float d[4][8];
#pragma unroll
            for (int T = 0; T < 4; ++T) tc::tmem_ld8(tl + uint32_t(64 * T + 32 * hh + 8 * gq), d[T]);
            tc::tmem_ld_wait();
#pragma unroll
            for (int ip = 0; ip < 2; ++ip) {
                C2 v[4];
#pragma unroll
                for (int T = 0; T < 4; ++T) {
                    const float4 w = tw[(T * 16 + 2 * gq + ip) * 8];
                    v[T] = cmul2(c2_at(d[T], ip), C2{make_float2(w.x, w.y), make_float2(w.z, w.w)});
                }
                const int i = 2 * ip;
                sts128(A, base + uint32_t(gq >> 1) * kSBO64 + uint32_t(4 * (gq & 1) + i) * 16u,
                       pack_bf16(v[0].re.x, v[0].im.x), pack_bf16(v[1].re.x, v[1].im.x),
                       pack_bf16(v[2].re.x, v[2].im.x), pack_bf16(v[3].re.x, v[3].im.x));
                sts128(A, base + uint32_t(gq >> 1) * kSBO64 + uint32_t(4 * (gq & 1) + i + 1) * 16u,
                       pack_bf16(v[0].re.y, v[0].im.y), pack_bf16(v[1].re.y, v[1].im.y),
                       pack_bf16(v[2].re.y, v[2].im.y), pack_bf16(v[3].re.y, v[3].im.y));
            }
        }
    }
    // ---------------- stage 2'
    stage_issue(a_addr, kSBO64, b32_addr, kSBO64, 4, 4, tc::idesc_bf16(128, 64), tmem, 64, x.mbar, ok && x.issue_mma);
    {
        // rows (k1 = 4 Q + T, b = lane), outputs q = 16 h + ..; twiddle w_N^((b + 32 q) k1)
        // -> stage-1' row a = b + 32 q, chunk Q (slots k1 = 4 Q .. 4 Q + 3)
        // row a = lane + 32 (16 h + 4 gq + i): a / 8 = (lane >> 3) + 64 h + 16 gq + 4 i, a % 8 = lane & 7
        const uint32_t base = uint32_t((lane >> 3) + 64 * hh) * kSBO32 + uint32_t(Q) * tc::kLBO +
                              uint32_t(lane & 7) * 16u;
        // twiddles in pairs (q, q + 1), stepped by w_N^(64 k1)
        C2 pw[4], st2[4];
#pragma unroll
        for (int T = 0; T < 4; ++T) {
            const int k1 = 4 * Q + T;
            const float2 p0 = wN((lane + 512 * hh) * k1, twist, odd);
            pw[T] = c2_of(p0, cmul(p0, wN(32 * k1, twist, odd)));
            st2[T] = c2_splat(wN(64 * k1, twist, odd));
        }
        ok = stage_wait(x.mbar, phase, ok, x.budget);
#pragma unroll 1
        for (int gq = 0; gq < 4; ++gq) {
            float d[4][8];
#pragma unroll
            for (int T = 0; T < 4; ++T) tc::tmem_ld8(tl + uint32_t(64 * T + 32 * hh + 8 * gq), d[T]);
            tc::tmem_ld_wait();
#pragma unroll
            for (int ip = 0; ip < 2; ++ip) {
                C2 v[4];
#pragma unroll
                for (int T = 0; T < 4; ++T) {
                    v[T] = cmul2(c2_at(d[T], ip), pw[T]);
                    pw[T] = cmul2(pw[T], st2[T]);
                }
                const int i = 2 * ip;
                sts128(A, base + uint32_t(16 * gq + 4 * i) * kSBO32, pack_bf16(v[0].re.x, v[0].im.x),
                       pack_bf16(v[1].re.x, v[1].im.x), pack_bf16(v[2].re.x, v[2].im.x),
                       pack_bf16(v[3].re.x, v[3].im.x));
                sts128(A, base + uint32_t(16 * gq + 4 * (i + 1)) * kSBO32, pack_bf16(v[0].re.y, v[0].im.y),
                       pack_bf16(v[1].re.y, v[1].im.y), pack_bf16(v[2].re.y, v[2].im.y),
                       pack_bf16(v[3].re.y, v[3].im.y));
            }
        }
    }
}

}  // namespace tc16k
}  // namespace hyena
