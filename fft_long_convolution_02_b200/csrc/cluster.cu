// cluster.cu -- L = 65536, bf16 storage: the gated FFT convolution of a row
// pair kept on chip across a cluster of 8 CTAs, its DFT stages on the tensor
// cores.
//
// Same method as the other paths ([P4] "HyenaDNA operator walk-through"
// (adg.csdn.net), section 二.1 gating loop, section 二.2 fftconv: the causal
// long convolution as a zero-padded 2L-point FFT, spectrum product, inverse
// FFT), and, as in the L = 8192 kernel, two batch rows b0, b1 of a channel
// travel as one complex signal z = g[b0] + i g[b1].  The zero-padded
// transform has NO = 2L = 131072 points, too many for one SM, so it is split
// over the R = 8 CTAs of a cluster (thread-block cluster, distributed shared
// memory) in four-step form with NO = R x NI, NI = 16384:
//
//   n = a + NI s (a < NI; s < 4 non-zero),   f = k1 + R f' (k1 < R, f' < NI)
//   F1 (CTA j, its a-range):  Y1[k1][a] = w_NO^(a k1) sum_s z[a + NI s] w_8^(s k1)
//   F2 (CTA k1):              X[k1 + R f'] = DFT_NI(Y1[k1][.])[f']
//
// CTA j computes F1 for a = a' + 1024 s', s' in {2j, 2j+1} (all a' < 1024)
// and stores Y1[k1][a] straight into CTA k1's stage-1 operand (row a', slot
// s') through distributed shared memory; CTA k1 then runs the tensor-core FFT
// of tc16k.cuh on its 16384 points (all 16 stage-1 inputs non-zero), the
// spectrum product with K~[k1 + R f'] = (FFT_NO(k) + D)[k1 + R f'] / NO, and
// the inverse stages, which leave conj(V[k1][a]) with
//   V[k1][a] = sum_f' X K~ [k1 + R f'] w_NI^(-a f'),
//   y[a + NI s] = sum_k1 w_8^(-s k1) w_NO^(-a k1) V[k1][a]     (s < 4).
// The inverse exchange goes through a per-cluster scratch in global memory
// (the caller's workspace, 512 KB per cluster, L2-resident): CTA k1 writes
// conj V[k1][.] as bf16 pairs, and CTA j reads back the 8 values of each of
// its a and finishes the 8-point inverse DFT (I1).  I1 of one order step
// feeds the next step's gate and F1 directly, and the last one the output
// gate, so between the input loads and the output stores nothing of a row
// pair touches HBM except the scratch round trip.
//
// Synchronisation per order step: one cluster barrier after F1 (all stage-1
// operands complete; it also orders the previous step's scratch reads
// before this step's scratch writes) and one after the scratch writes (all
// CTAs' last MMAs done, so every operand buffer is free for the next F1).
// Tensor-core waits are bounded; after a wait has run out a CTA issues no
// more MMAs but still takes every barrier, so the cluster never stalls.
//
// Spectrum: the L = 65536 spectrum buffer carries, after the multi-pass
// rows, the cluster plane: per (step, c) the 8 sub-planes K~[k1 + R f'] as
// bf16 (re, im) at position spec8192_pos(f') (the order in which the
// tensor-core spectrum pass reads them), built here in fp32 (F1 directly
// from the filter, then a 16384-point CTA FFT per sub-plane).
#include <cuda_bf16.h>

#include <atomic>

#include "common.cuh"
#include "cta_fft.cuh"
#include "kernels.h"
#include "pairs4096.cuh"
#include "plan_common.h"
#include "tc16k.cuh"
#include "tc_util.cuh"

namespace hyena {

namespace {

using namespace tc16k;

constexpr int LC = int(kClusterL);   // 65536
constexpr int NI = 16384;            // points per CTA
constexpr int NO = 2 * LC;           // 131072 = kClusterR * NI
constexpr int RC = kClusterR;        // 8
constexpr int NT = 256;
static_assert(NO == RC * NI, "cluster split");

// ---------------------------------------------------------------- helpers

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_id() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_count() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}
// All threads of all CTAs of the cluster; release / acquire order the shared
// and global writes before the barrier with the reads after it.
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}
// Shared-memory address `saddr` of this CTA, as seen in CTA `rank`'s window.
__device__ __forceinline__ uint32_t map_rank(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
__device__ __forceinline__ void st_cluster(uint32_t addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
// Make this thread's generic-proxy writes to (remote) shared memory visible
// to the tensor cores' async proxy before the barrier that publishes them.
__device__ __forceinline__ void fence_proxy_async_cluster() {
    asm volatile("fence.proxy.async.shared::cluster;" ::: "memory");
}

// w_8^m = exp(-2 pi i m / 8)
__device__ __forceinline__ float2 w8(int m) {
    constexpr float c = 0.70710678118654752f;
    float2 v = (m & 1) ? make_float2(c, -c) : make_float2(1.0f, 0.0f);
    if (m & 2) v = make_float2(v.y, -v.x);      // times -i
    if (m & 4) v = make_float2(-v.x, -v.y);     // times -1
    return v;
}

// Table pointers of the cluster path inside the spectrum buffer.
struct ClTables {
    const float2* fft;     // CTA FFT of 16384 points
    const float2* wa;      // w_NO^a, a < 16384
    const float2* even;    // w_NI^(2j), j < 2048
    const float2* odd;     // w_NI^(2j+1), j < 2048
};
ClTables cl_tables(const Plan& p, const uint8_t* spectrum) {
    const float2* t = reinterpret_cast<const float2*>(spectrum + p.tables_off);
    return ClTables{t + p.t_cl_fft, t + p.t_cl_wa, t + p.t_cl_even, t + p.t_cl_odd};
}

// ------------------------------------------------------- spectrum plane
// CTA (k1, row r = step * C + c): Y1[a] = w_NO^(a k1) sum_s k[a + NI s] w_8^(s k1)
// for a < NI, the 16384-point FFT, K~ = (X + D) / NO as bf16 pairs.
template <typename TK>
__global__ void __launch_bounds__(512)
k_spectrum_cluster(const TK* __restrict__ k, const float* __restrict__ D, uint32_t* __restrict__ plane,
                   ClTables tb) {
    extern __shared__ float2 smem[];
    const int k1 = blockIdx.x;
    const int64_t row = blockIdx.y;
    const TK* kr = k + row * LC;
    const float d = D ? __ldg(D + row) : 0.0f;
    for (int a = threadIdx.x; a < NI; a += blockDim.x) {
        float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const float x = load1(kr + a + NI * s);
            const float2 w = w8((s * k1) & 7);
            acc.x = fmaf(x, w.x, acc.x);
            acc.y = fmaf(x, w.y, acc.y);
        }
        // w_NO^(a k1): a k1 = e_hi NI + e_lo, w_NO^(NI e_hi) = w_8^(e_hi)
        const int e = a * k1;
        const float2 w = cmul(__ldg(tb.wa + (e & (NI - 1))), w8(e >> 14));
        smem[fft_pad(a)] = cmul(acc, w);
    }
    __syncthreads();
    cta_fft_forward<NI>(smem, 1, fft_padded_size(NI), tb.fft);
    uint32_t* out = plane + (row * RC + k1) * int64_t(NI);
    const float sN = 1.0f / float(NO);
    for (int f = threadIdx.x; f < NI; f += blockDim.x) {
        const float2 X = smem[fft_pad(fft_bin_pos<NI>(f))];
        const __nv_bfloat162 hb = __floats2bfloat162_rn((X.x + d) * sN, X.y * sN);
        out[spec8192_pos(f)] = *reinterpret_cast<const uint32_t*>(&hb);
    }
}

// ------------------------------------------------------------ convolution

constexpr uint32_t kB1fBytes = 4 * kSBO32;      // 16-point DFT, N 32 x K 32
constexpr uint32_t kOffB1f = kAbytes;
constexpr uint32_t kOffB32c = kOffB1f + kB1fBytes;
constexpr uint32_t kOffTW2c = kOffB32c + kB32bytes;
// F1 staging: per warp two buffers of up to 16 runs of 40 samples (bf16)
constexpr uint32_t kStageRun = 80;
constexpr uint32_t kStageBuf = 16 * kStageRun;
constexpr uint32_t kOffStage = kOffTW2c + kTW2bytes;
constexpr size_t kSmemC = size_t(kOffStage) + (NT / 32) * 2 * kStageBuf;
static_assert(kOffTW2c % 16 == 0 && kOffStage % 16 == 0, "table / staging alignment");
// two CTAs per SM: 2 x (dynamic + 1 KB static + 1 KB reserved) <= 228 KB
static_assert(2 * (kSmemC + 2048) <= 233472, "two CTAs per SM");

struct ClArgs {
    const bf16* u;            // [B, (order+1) C, L]
    bf16* y;                  // [B, C, L]
    const uint8_t* spectrum;  // header at offset 0
    const uint32_t* plane;    // cluster plane (spectrum + plane_off)
    const float* sc_w;
    const float* sc_b;
    const float2* wa;         // w_NO^a, a < NI
    const float2* even;       // w_NI^(2j)
    const float2* odd;        // w_NI^(2j+1)
    uint32_t* scratch;        // [clusters][RC][NI] bf16 (re, im): conj V
    int64_t tables_off, plane_off;
    int B, C, order, npairs;
    uint64_t budget;
    int issue_mma;
    uint32_t* status;
};

// 8-point DFT of (z0, z1, z2, z3, 0, 0, 0, 0): even outputs DFT_4(z), odd
// outputs DFT_4(z_s w_8^s).
__device__ __forceinline__ void dft4(float2 x0, float2 x1, float2 x2, float2 x3, float2& o0, float2& o1,
                                     float2& o2, float2& o3) {
    const float2 e0 = cadd(x0, x2), e1 = csub(x0, x2), f0 = cadd(x1, x3), f1 = csub(x1, x3);
    o0 = cadd(e0, f0);
    o2 = csub(e0, f0);
    o1 = make_float2(e1.x + f1.y, e1.y - f1.x);   // e1 - i f1
    o3 = make_float2(e1.x - f1.y, e1.y + f1.x);   // e1 + i f1
}
__device__ __forceinline__ void dft8_of4(const float2 (&z)[4], float2 (&Y)[8]) {
    constexpr float c = 0.70710678118654752f;
    dft4(z[0], z[1], z[2], z[3], Y[0], Y[2], Y[4], Y[6]);
    const float2 z1 = make_float2(c * (z[1].x + z[1].y), c * (z[1].y - z[1].x));    // z1 w_8
    const float2 z2 = make_float2(z[2].y, -z[2].x);                                  // z2 w_8^2
    const float2 z3 = make_float2(c * (z[3].y - z[3].x), -c * (z[3].x + z[3].y));   // z3 w_8^3
    dft4(z[0], z1, z2, z3, Y[1], Y[3], Y[5], Y[7]);
}
// Outputs s < 4 of the 8-point DFT of x.
__device__ __forceinline__ void dft8_first4(const float2 (&x)[8], float2 (&o)[4]) {
    constexpr float c = 0.70710678118654752f;
    float2 e[4], d[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        e[m] = cadd(x[m], x[m + 4]);
        d[m] = csub(x[m], x[m + 4]);
    }
    d[1] = make_float2(c * (d[1].x + d[1].y), c * (d[1].y - d[1].x));
    d[2] = make_float2(d[2].y, -d[2].x);
    d[3] = make_float2(c * (d[3].y - d[3].x), -c * (d[3].x + d[3].y));
    o[0] = cadd(cadd(e[0], e[1]), cadd(e[2], e[3]));
    o[1] = cadd(cadd(d[0], d[1]), cadd(d[2], d[3]));
    const float2 ee = csub(e[0], e[2]), ef = csub(e[1], e[3]);
    const float2 de = csub(d[0], d[2]), df = csub(d[1], d[3]);
    o[2] = make_float2(ee.x + ef.y, ee.y - ef.x);
    o[3] = make_float2(de.x + df.y, de.y - df.x);
}


// Samples n-2, n-1, n of one row (zero before its start).
struct S3 {
    float m2, m1, c;
};
// Short conv at one sample of both rows: (row b0, row b1).
__device__ __forceinline__ float2 sc_pair(const S3& r0, const S3& r1, const Taps2& tp) {
    return __ffma2_rn(tp.w0, make_float2(r0.m2, r1.m2),
                      __ffma2_rn(tp.w1, make_float2(r0.m1, r1.m1), __ffma2_rn(tp.w2, make_float2(r0.c, r1.c), tp.b)));
}


// Row pair operands of one order step.
struct PairRows {
    const bf16* u0;   // row b0 of u
    const bf16* u1;   // row b1 (row b0 again when the pair has one row)
    float m1;         // 1, or 0 for a pair with one row
};

// F1 of one order step.  Thread (warp w, lane l) takes, in round r < 2, the
// row a' = 32 q + l, q = 16 half + 2 w + r, and its four s' = 4 quad + m
// (m < 4): a = a' + 1024 s'.  For each (r, m) the warp stages the 34 samples
// n - 2 .. n (n = a + NI s) of every input row it needs (the gate rows, and
// at the first step the value rows, at s < 4) in shared memory with cp.async,
// one item ahead of the arithmetic: z[s] = sc(x_g)[n] v[n] (STEP1: v = sc(v),
// else v = the previous step's I1 at a), Y1[k1][a] = w_NO^(a k1) DFT_8(z)[k1].
// The four s' of a row are one 16-byte chunk (chunk `quad` of row rho1(a'))
// of CTA k1's stage-1 operand, written after each round.
// MODE 2 runs the same loop for the output gate: I1 of the last step, times
// sc(x0) (cg = x0's rows), stored to y (y0, y1: rows b0, b1 of y; ok = false
// writes NaN).
template <int MODE>
__device__ __forceinline__ void f1_step(const ClArgs& p, const PairRows& rw, int64_t cg, int64_t cv,
                                        const Taps2& tg, const Taps2& tv, int half, int quad, int warp, int lane,
                                        const uint32_t* __restrict__ scr, uint32_t a_addr, uint8_t* stage,
                                        bf16* y0 = nullptr, bf16* y1 = nullptr, bool ok = true) {
    constexpr bool STEP1 = MODE == 0;
    constexpr int NR = STEP1 ? 4 : 2;           // input rows per s
    constexpr int NC = 4 * NR;                  // staged runs per item
    auto issue = [&](int it) {
        const int base = 32 * (16 * half + 2 * warp + (it >> 2)) + 1024 * (4 * quad + (it & 3));
        uint8_t* dst = stage + (it & 1) * kStageBuf;
        for (int k = lane; k < NC * 5; k += 32) {
            const int c = k / 5, ch = k - 5 * (k / 5);
            const int s = c / NR, rr = c - NR * (c / NR);
            const bf16* row = (rr & 1 ? rw.u1 : rw.u0) + (rr < 2 ? cg : cv);
            const int e = base + NI * s - 8 + 8 * ch;          // first sample of this 16-byte piece
            const bool in = e >= 0;
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(tc::smem_u32(dst + c * kStageRun + 16 * ch)),
                         "l"(row + (in ? e : 0)), "r"(in ? 16 : 0)
                         : "memory");
        }
        cp_async_commit();
    };
    auto s3_at = [&](const uint8_t* buf, int c) {
        const bf16* r = reinterpret_cast<const bf16*>(buf + c * kStageRun) + 6 + lane;
        S3 o;
        o.m2 = __bfloat162float(r[0]);
        o.m1 = __bfloat162float(r[1]);
        o.c = __bfloat162float(r[2]);
        return o;
    };
    // a of item it: a' = 32 (16 half + 2 warp + it / 4) + lane, s' = 4 quad + it % 4
    auto item_a = [&](int it) { return 32 * (16 * half + 2 * warp + (it >> 2)) + lane + 1024 * (4 * quad + (it & 3)); };
    // the twiddle base and (after the first step) the scratch values of the
    // next item are loaded one item ahead, like its staged samples
    float2 w1n = __ldg(p.wa + item_a(0));
    uint32_t svn[STEP1 ? 1 : RC];
    if constexpr (!STEP1) {
#pragma unroll
        for (int k1 = 0; k1 < RC; ++k1) svn[k1] = __ldcg(scr + int64_t(k1) * NI + item_a(0));
    }
    issue(0);
#pragma unroll 1
    for (int r = 0; r < 2; ++r) {
        const int ap = 32 * (16 * half + 2 * warp + r) + lane;
        uint32_t v[RC][4];                      // [k1][m]: bf16 pairs
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const int it = 4 * r + m;
            if (it < 7) issue(it + 1);
            else cp_async_commit();
            const int a = ap + 1024 * (4 * quad + m);
            const float2 w1 = w1n;
            uint32_t sv[STEP1 ? 1 : RC];
#pragma unroll
            for (int k1 = 0; k1 < (STEP1 ? 1 : RC); ++k1) sv[k1] = svn[k1];
            if (it < 7) {
                const int an = item_a(it + 1);
                w1n = __ldg(p.wa + an);
                if constexpr (!STEP1) {
#pragma unroll
                    for (int k1 = 0; k1 < RC; ++k1) svn[k1] = __ldcg(scr + int64_t(k1) * NI + an);
                }
            }
            asm volatile("cp.async.wait_group 1;\n" ::: "memory");
            __syncwarp();
            const uint8_t* buf = stage + (it & 1) * kStageBuf;
            float2 z[4];
            if constexpr (STEP1) {
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    z[s] = __fmul2_rn(sc_pair(s3_at(buf, 4 * s), s3_at(buf, 4 * s + 1), tg),
                                      sc_pair(s3_at(buf, 4 * s + 2), s3_at(buf, 4 * s + 3), tv));
            } else {
                // I1 of the previous step at a: conj U[k1] = w_NO^(a k1) conj V[k1][a]
                float2 x[8];
                float2 w = w1;
#pragma unroll
                for (int k1 = 0; k1 < RC; ++k1) {
                    const float2 vc = make_float2(bf_lo(sv[k1]), bf_hi(sv[k1]));
                    if (k1 == 0) {
                        x[0] = vc;
                    } else {
                        x[k1] = cmul(vc, w);
                        if (k1 + 1 < RC) w = cmul(w, w1);
                    }
                }
                float2 o[4];
                dft8_first4(x, o);
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    const float2 ys = make_float2(o[s].x, -rw.m1 * o[s].y);   // y = conj (row b1 masked)
                    z[s] = __fmul2_rn(sc_pair(s3_at(buf, 2 * s), s3_at(buf, 2 * s + 1), tg), ys);
                }
            }
            __syncwarp();                       // buffer read before the next issue refills it
            if constexpr (MODE == 2) {
                const bf16 nanv = __float2bfloat16_rn(__int_as_float(0x7fc00000));
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    // a timed-out wait poisons the output
                    y0[a + NI * s] = ok ? __float2bfloat16_rn(z[s].x) : nanv;
                    if (rw.m1 != 0.0f) y1[a + NI * s] = ok ? __float2bfloat16_rn(z[s].y) : nanv;
                }
                continue;
            }
            float2 o[8];
            dft8_of4(z, o);
            float2 w = w1;
            v[0][m] = pack_bf16(o[0].x, o[0].y);
#pragma unroll
            for (int k1 = 1; k1 < RC; ++k1) {
                const float2 tw = cmul(o[k1], w);
                v[k1][m] = pack_bf16(tw.x, tw.y);
                if (k1 + 1 < RC) w = cmul(w, w1);
            }
        }
        if constexpr (MODE == 2) continue;
        const uint32_t off = a_addr + tc::chunk_off(rho1(ap), quad, kSBO32);
#pragma unroll
        for (int k1 = 0; k1 < RC; ++k1) {
            const uint32_t dst = map_rank(off, uint32_t(k1));
            asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(v[k1][0]),
                         "r"(v[k1][1]), "r"(v[k1][2]), "r"(v[k1][3])
                         : "memory");
        }
    }
    cp_async_wait_all();
}

__global__ void __launch_bounds__(NT, 2)
k_conv_cluster(const __grid_constant__ ClArgs p) {
    extern __shared__ __align__(1024) uint8_t smem_cl[];
    __shared__ __align__(8) uint64_t mbar;
    __shared__ uint32_t tmem_base;
    // the header is requested first and checked after the table setup (which
    // reads no global memory); every CTA of a cluster reads the same header, so
    // they all leave together, before the first cluster barrier
    const SpecHeader* h = reinterpret_cast<const SpecHeader*>(p.spectrum);
    const SpecHeader hv = *h;
    const bool hdr_ok = (hv.magic == kSpecMagic) & (hv.path == PATH_MULTIPASS_1D) & (hv.C == p.C) & (hv.L == LC) &
                        (hv.order == p.order) & (hv.tables_off == p.tables_off) & (hv.reserved[0] == p.plane_off);
    uint8_t* A = smem_cl;
    float4* TW2 = reinterpret_cast<float4*>(smem_cl + kOffTW2c);
    const int t = threadIdx.x;
    const int warp = t >> 5, lane = t & 31;
    const int Q = warp & 3, hh = warp >> 2;
    const int rank = int(cluster_rank());
    const int quad = rank >> 1, half = rank & 1;

    float2* w32 = reinterpret_cast<float2*>(smem_cl);   // operand area, free until the first F1
    fill_w32(w32);
    __syncthreads();
    fill_dft<16, 16, 16, kSBO32>(smem_cl + kOffB1f, w32);
    fill_dft<32, 32, 32, kSBO64>(smem_cl + kOffB32c, w32);
    fill_tw2(TW2);
    if (!hdr_ok) {
        if (t == 0) report_status(p.status, kStatusSpectrumMismatch);
        return;
    }
    if (t == 0) tc::mbar_init(&mbar, 1);
    if (warp == 0) tc::tmem_alloc(&tmem_base, kTmemCols);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = tmem_base;
    const uint32_t tl = tmem + (uint32_t(32 * Q) << 16);
    const uint32_t a_addr = tc::smem_u32(A);
    const uint32_t b1f_addr = tc::smem_u32(smem_cl + kOffB1f);
    const uint32_t b32_addr = tc::smem_u32(smem_cl + kOffB32c);
    uint32_t phase = 0;
    bool ok = true, reported = false;
    const Ctx tx{A, TW2, p.even, p.odd, tmem, tl, a_addr, b32_addr, &mbar, p.budget, p.issue_mma, lane, Q, hh};
    // every CTA of the cluster is running and set up before the first remote store
    cluster_sync();

    const int qc = int(cluster_id()), nq = int(cluster_count());
    const uint32_t* scr = p.scratch + int64_t(qc) * RC * NI;
    for (int P = qc; P < p.npairs; P += nq) {
        const PairRef pr = pair_ref(P, p.B);
        for (int st = 1; st < p.order; ++st) {
            const int g = p.order - st;
            // ---- (I1 of the previous step,) gate, F1 scatter to the cluster
            {
                const int64_t Ctot = int64_t(p.order + 1) * p.C;
                PairRows rw;
                rw.u0 = p.u + int64_t(pr.b0) * Ctot * LC;
                rw.u1 = pr.has1 ? rw.u0 + Ctot * LC : rw.u0;
                rw.m1 = pr.has1 ? 1.0f : 0.0f;
                const int64_t cg = (int64_t(g) * p.C + pr.c) * LC, cv = (int64_t(p.order) * p.C + pr.c) * LC;
                const Taps2 tg = taps2(load_taps(p.sc_w, p.sc_b, int64_t(g) * p.C + pr.c), 1.0f);
                const Taps2 tv = taps2(load_taps(p.sc_w, p.sc_b, int64_t(p.order) * p.C + pr.c), rw.m1);
                uint8_t* stage = smem_cl + kOffStage + warp * 2 * kStageBuf;
                if (st == 1) f1_step<0>(p, rw, cg, cv, tg, tv, half, quad, warp, lane, scr, a_addr, stage);
                else f1_step<1>(p, rw, cg, cv, tg, tv, half, quad, warp, lane, scr, a_addr, stage);
            }
            fence_proxy_async_cluster();
            cluster_sync();
            // ---- this CTA's spectrum sub-plane into L2 while the stages before its pass run
            if (t < 4)
                asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(
                                 p.plane + ((int64_t(st - 1) * p.C + pr.c) * RC + rank) * NI + t * (NI / 4)),
                             "r"(uint32_t(NI)) : "memory");
            // ---- F2 and its inverse on this CTA's 16384 points
            stage_issue(a_addr, kSBO32, b1f_addr, kSBO32, 8, 2, tc::idesc_bf16(128, 32), tmem, 32, &mbar,
                        ok && p.issue_mma);
            middle(tx, p.plane + ((int64_t(st - 1) * p.C + pr.c) * RC + rank) * NI, phase, ok);
            stage_issue(a_addr, kSBO32, b1f_addr, kSBO32, 8, 2, tc::idesc_bf16(128, 32), tmem, 32, &mbar,
                        ok && p.issue_mma);
            ok = stage_wait(&mbar, phase, ok, p.budget);
            // ---- conj V[rank][a'] (stage-1' rows a', outputs s') to the scratch
            {
                uint32_t* out = p.scratch + (int64_t(qc) * RC + rank) * NI;
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const int T = 4 * hh + jj;
                    const int ar = 128 * T + 32 * Q + lane;
                    float d[32];
                    tc::tmem_ld32(tl + uint32_t(32 * T), d);
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int s2 = 0; s2 < 16; ++s2) {
                        const int col = 4 * (s2 >> 1) + (s2 & 1);          // re at col, im at col + 2
                        __stcg(out + ar + 1024 * s2, pack_bf16(d[col], d[col + 2]));
                    }
                }
            }
            if (!ok && !reported) {
                if (t == 0) report_status(p.status, kStatusTimeout);
                reported = true;
            }
            tc::fence_before_sync();
            cluster_sync();
            tc::fence_after_sync();
        }
        // ---- I1 of the last step and the output gate y = sc(x0) v
        {
            const int64_t Ctot = int64_t(p.order + 1) * p.C;
            PairRows rw;
            rw.u0 = p.u + int64_t(pr.b0) * Ctot * LC;
            rw.u1 = pr.has1 ? rw.u0 + Ctot * LC : rw.u0;
            rw.m1 = pr.has1 ? 1.0f : 0.0f;
            const Taps2 t0 = taps2(load_taps(p.sc_w, p.sc_b, pr.c), 1.0f);
            bf16* y0 = p.y + (int64_t(pr.b0) * p.C + pr.c) * LC;
            uint8_t* stage = smem_cl + kOffStage + warp * 2 * kStageBuf;
            f1_step<2>(p, rw, int64_t(pr.c) * LC, 0, t0, t0, half, quad, warp, lane, scr, a_addr, stage, y0,
                       y0 + int64_t(p.C) * LC, ok);
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

cudaError_t launch_spectrum_cluster(const Plan& p, const SpectrumArgs& a, cudaStream_t s) {
    if (p.cl_plane_off == 0) return cudaSuccess;
    const ClTables tb = cl_tables(p, a.spectrum);
    uint32_t* plane = reinterpret_cast<uint32_t*>(a.spectrum + p.cl_plane_off);
    const size_t smem = size_t(fft_padded_size(NI)) * sizeof(float2);
    const dim3 grid(RC, unsigned((p.order - 1) * p.C));
    if (a.k_dtype == DT_F32) {
        auto kern = k_spectrum_cluster<float>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess) return e;
        kern<<<grid, 512, smem, s>>>(static_cast<const float*>(a.k), a.D, plane, tb);
    } else {
        auto kern = k_spectrum_cluster<__nv_bfloat16>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess) return e;
        kern<<<grid, 512, smem, s>>>(static_cast<const __nv_bfloat16*>(a.k), a.D, plane, tb);
    }
    return cudaGetLastError();
}

bool cluster_path(const Plan& p, const ConvArgs& a) {
    return p.cl_plane_off != 0 && p.L == kClusterL && a.dtype == DT_BF16 && p.order <= kMaxOrderTc &&
           a.spec_per_b == 0 && !a.fp32_transform;
}

size_t cluster_scratch_bytes() { return size_t(RC) * NI * 4; }
constexpr int kMaxClusterDevices = 64;

// Never launched: the cluster kernel's block size and shared memory without
// its tensor-memory allocation, for the occupancy calculator (which counts one
// CTA per SM for any kernel that allocates tensor memory, although two of
// k_conv_cluster fit: 2 x 256 columns, 2 x 256 threads x 128 registers).
__global__ void __launch_bounds__(NT, 2) k_cluster_occupancy_probe() {}

cudaError_t launch_conv_cluster(const Plan& p, const ConvArgs& a, size_t workspace_bytes, cudaStream_t s) {
    const int64_t npairs = p.C * ((a.B + 1) / 2);
    if (npairs > INT32_MAX || a.B > INT32_MAX || p.C > INT32_MAX) return cudaErrorInvalidValue;
    if (npairs == 0) return cudaSuccess;
    auto kern = k_conv_cluster;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmemC));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = RC;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = kSmemC;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(RC);
    // Clusters resident at once with two CTAs per SM, queried once per device
    // on the probe kernel (same block size and shared memory): the grid is
    // persistent with a static share of pairs per cluster, so a cluster that
    // could not be resident would start only when another ends.  How many
    // 8-CTA clusters fit depends on how the SMs are spread over the GPCs (33
    // on the B200s measured; 34 did not fit).
    static std::atomic<int> g_max_clusters[kMaxClusterDevices];
    int dev = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxClusterDevices) return cudaErrorInvalidDevice;
    int max_clusters = g_max_clusters[dev].load(std::memory_order_relaxed);
    if (max_clusters == 0) {
        // the probe's dynamic shared memory stands for the kernel's dynamic and static parts
        cudaFuncAttributes fa{};
        e = cudaFuncGetAttributes(&fa, kern);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t pcfg = cfg;
        pcfg.dynamicSmemBytes = kSmemC + fa.sharedSizeBytes;
        e = cudaFuncSetAttribute(k_cluster_occupancy_probe, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(pcfg.dynamicSmemBytes));
        if (e != cudaSuccess) return e;
        e = cudaOccupancyMaxActiveClusters(&max_clusters, k_cluster_occupancy_probe, &pcfg);
        if (e != cudaSuccess) return e;
        if (max_clusters < 1) return cudaErrorInvalidConfiguration;
        g_max_clusters[dev].store(max_clusters, std::memory_order_relaxed);
    }
    // one scratch slice per cluster, from the caller's workspace
    int64_t nclusters = int64_t(workspace_bytes / cluster_scratch_bytes());
    if (nclusters > int64_t(max_clusters)) nclusters = int64_t(max_clusters);
    if (nclusters > npairs) nclusters = npairs;
    if (nclusters < 1) return cudaErrorInvalidValue;
    cfg.gridDim = dim3(unsigned(nclusters * RC));
    ClArgs args{};
    const ClTables tb = cl_tables(p, a.spectrum);
    args.u = static_cast<const bf16*>(a.u);
    args.y = static_cast<bf16*>(a.y);
    args.spectrum = a.spectrum;
    args.plane = reinterpret_cast<const uint32_t*>(a.spectrum + p.cl_plane_off);
    args.sc_w = a.sc_w;
    args.sc_b = a.sc_b;
    args.wa = tb.wa;
    args.even = tb.even;
    args.odd = tb.odd;
    args.scratch = reinterpret_cast<uint32_t*>(a.workspace);
    args.tables_off = int64_t(p.tables_off);
    args.plane_off = int64_t(p.cl_plane_off);
    args.B = int(a.B);
    args.C = int(p.C);
    args.order = p.order;
    args.npairs = int(npairs);
    args.budget = a.wait_budget_ns;
    args.issue_mma = a.issue_mma;
    args.status = a.status;
    e = cudaLaunchKernelEx(&cfg, kern, args);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace hyena
