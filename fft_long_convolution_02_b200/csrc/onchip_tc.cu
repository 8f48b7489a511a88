// onchip_tc.cu -- L = 8192, bf16 storage: the gated FFT convolution with its
// DFT stages on the tensor cores (tcgen05).
//
// Two batch rows b0, b1 of one channel share the filter, and the filter is
// real, so they travel as one complex signal z = g[b0] + i g[b1] (g = the
// gated input of the order step): the circular convolution of z with the
// zero-padded filter k has real part y[b0] and imaginary part y[b1].  Each
// CTA therefore runs one complex FFT of N = 2L = 16384 points (upper half of
// the input zero), a point-wise product with K~ = (FFT_N(k) + D) / N, and the
// inverse FFT, keeping the first L outputs -- no real-to-complex untangling.
//
// The transform is the tensor-core FFT of tc16k.cuh (16 x 32 x 32 stages).
// Here the input is zero for s >= 8 (stage 1 has K = 16) and only the outputs
// s < 8 of the last inverse stage are needed (stage 1' has N = 16); the
// spectrum pass's conjugation folds into the output gate.
//
// Precision: the stage operands and the DFT matrices are rounded to bf16 (8
// significant bits) six times per order step; the resulting row error is a
// few 1e-3 relative to the output, inside the bf16-storage tolerance.  fp32
// storage keeps the fp32 kernel.
#include "common.cuh"
#include "kernels.h"
#include "plan_common.h"
#include "tc16k.cuh"
#include "tc_util.cuh"

namespace hyena {

namespace {

using namespace tc16k;

constexpr int L = 8192;
constexpr int NT = 256;
constexpr uint32_t kB1bytes = 4 * kSBO16;   // N 32 x K 16
constexpr uint32_t kB1ibytes = 2 * kSBO32;  // N 16 x K 32
constexpr uint32_t kOffA1 = kAbytes - 128 * kSBO16;   // stage-1 operand (1024 rows x K 16)
constexpr uint32_t kOffB1 = kAbytes;
constexpr uint32_t kOffB32 = kOffB1 + kB1bytes;
constexpr uint32_t kOffB1i = kOffB32 + kB32bytes;
constexpr uint32_t kOffTW2 = kOffB1i + kB1ibytes;
constexpr size_t kSmem = size_t(kOffTW2) + kTW2bytes;
static_assert(L * 4 <= kOffA1, "output staging must not overlap the stage-1 operand");
static_assert(kOffTW2 % 16 == 0, "twiddle table alignment");

// Step-1 input of a pair: thread t covers a = a0 .. a0+7 (a0 = 8 (t & 127)) at
// s = 4 (t >> 7) + j, j < 4, i.e. samples n0 = a0 + 1024 s of x_g and v of
// both rows.
struct PairInput {
    Raw8 x[2][4], v[2][4];
};

__device__ __forceinline__ void load_pair_input(PairInput& in, const bf16* __restrict__ u, const PairRef& pr,
                                                int C, int order, int j0) {
    const int64_t Ctot = int64_t(order + 1) * C;
    const int t = threadIdx.x;
    const int chalf = t >> 7, a0 = 8 * (t & 127);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const bf16* ub = u + int64_t(pr.b0 + (r && pr.has1 ? 1 : 0)) * Ctot * L;
        const bf16* xg = ub + (int64_t(order - 1) * C + pr.c) * L;
        const bf16* vv = ub + (int64_t(order) * C + pr.c) * L;
#pragma unroll
        for (int j = j0; j < j0 + 2; ++j) {
            const int n0 = a0 + 1024 * (4 * chalf + j);
            in.x[r][j] = load8(xg, n0);
            in.v[r][j] = load8(vv, n0);
        }
    }
}

__global__ void __launch_bounds__(NT, 2)
k_conv_8192_tc(const bf16* __restrict__ u, bf16* __restrict__ y, const uint8_t* __restrict__ spectrum,
               const float* __restrict__ sc_w, const float* __restrict__ sc_b, int B, int C, int order,
               int npairs, int64_t tables_off, int64_t spec_off, int64_t Ctot, uint64_t wait_budget_ns,
               int issue_mma, uint32_t* status) {
    extern __shared__ __align__(1024) uint8_t smem_tc[];
    __shared__ __align__(8) uint64_t mbar;
    __shared__ uint32_t tmem_base;
    // the layout offsets are kernel parameters (checked against the header above),
    // so that the table pointers need no registers of their own
    const float2* tables = reinterpret_cast<const float2*>(spectrum + tables_off);
    const float2* twist = tables + fft_tw_size(L / 2);        // w_L^j = w_N^(2j)
    const float2* odd = twist + L / 2 + (L / 4 + 1);          // w_N^(2j+1)
    const uint32_t* spec = reinterpret_cast<const uint32_t*>(spectrum + spec_off);   // plane 0 of each row

    // A: stage operands.  The stage-1 operand sits in the upper part so that
    // the previous pair's output staging (bf16 pairs, lower 32 KB) survives
    // until its output gate has run.
    uint8_t* A = smem_tc;
    uint8_t* A1 = smem_tc + kOffA1;
    uint32_t* Vs = reinterpret_cast<uint32_t*>(smem_tc);      // output staging: (re, -im) as bf16 pairs
    float4* TW2 = reinterpret_cast<float4*>(smem_tc + kOffTW2);
    const int t = threadIdx.x;
    const int warp = t >> 5, lane = t & 31;
    const int Q = warp & 3, hh = warp >> 2;

    // the 32 distinct entries of the DFT matrices once (in the operand area, free
    // until the first pair), then the matrices by lookup
    float2* w32 = reinterpret_cast<float2*>(smem_tc);
    fill_w32(w32);
    __syncthreads();
    fill_dft<16, 16, 8, kSBO16>(smem_tc + kOffB1, w32);
    fill_dft<32, 32, 32, kSBO64>(smem_tc + kOffB32, w32);
    fill_dft<16, 8, 16, kSBO32>(smem_tc + kOffB1i, w32);
    fill_tw2(TW2);
    // launched with programmatic stream serialisation: the tables above (no global
    // memory) are built while the previous kernel on the stream finishes; nothing
    // global is read or written before this wait
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const SpecHeader hv = *reinterpret_cast<const SpecHeader*>(spectrum);   // all fields at once
    const bool hdr_ok = (hv.magic == kSpecMagic) & (hv.path == PATH_ONCHIP_1D) & (hv.C == C) & (hv.L == L) &
                        (hv.order == order) & (hv.spec_row_bytes == int64_t(N) * 8) & (hv.tables_off == tables_off) &
                        (hv.spec_off == spec_off);
    if (!hdr_ok) {                                  // uniform: every thread read the same header
        if (t == 0) report_status(status, kStatusSpectrumMismatch);
        return;
    }
    if (t == 0) tc::mbar_init(&mbar, 1);
    if (warp == 0) tc::tmem_alloc(&tmem_base, kTmemCols);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = tmem_base;
    const uint32_t tl = tmem + (uint32_t(32 * Q) << 16);     // this warp's lane quarter
    const uint32_t a_addr = tc::smem_u32(A);
    const uint32_t a1_addr = tc::smem_u32(A1);
    const uint32_t b1_addr = tc::smem_u32(smem_tc + kOffB1);
    const uint32_t b32_addr = tc::smem_u32(smem_tc + kOffB32);
    const uint32_t b1i_addr = tc::smem_u32(smem_tc + kOffB1i);
    uint32_t phase = 0;
    bool ok = true;
    const Ctx tx{A, TW2, twist, odd, tmem, tl, a_addr, b32_addr, &mbar, wait_budget_ns, issue_mma, lane, Q, hh};

    // Output gate of a finished pair: y = sc(x0) * v from the staging buffer.
    // Thread t covers samples n0 = 8 (t + 256 jj) of both rows.
    auto output_gate = [&](const PairRef& pr) {
        const Taps2 t0 = taps2(load_taps(sc_w, sc_b, pr.c), 1.0f);
        const bf16* x00 = u + (int64_t(pr.b0) * Ctot + pr.c) * L;
        const bf16* x01 = pr.has1 ? x00 + Ctot * L : x00;
        bf16* y0 = y + (int64_t(pr.b0) * C + pr.c) * L;
        bf16* y1 = y0 + int64_t(C) * L;
#pragma unroll
        for (int jh = 0; jh < 4; jh += 2) {
            Raw8 xr[2][2];
#pragma unroll
            for (int jo = 0; jo < 2; ++jo) {
                xr[0][jo] = load8(x00, 8 * (t + 256 * (jh + jo)));
                xr[1][jo] = load8(x01, 8 * (t + 256 * (jh + jo)));
            }
#pragma unroll
            for (int jo = 0; jo < 2; ++jo) {
                const int n0 = 8 * (t + 256 * (jh + jo));
                const uint4 va = *reinterpret_cast<const uint4*>(Vs + n0);
                const uint4 vb = *reinterpret_cast<const uint4*>(Vs + n0 + 4);
                const uint32_t vw[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
                float2 xs[8];
                sc8x2(xr[0][jo], xr[1][jo], t0, xs);
                uint32_t o0[4], o1[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    // v staging holds (row b0, row b1) per sample
                    const float2 ya = __fmul2_rn(xs[2 * i], make_float2(bf_lo(vw[2 * i]), bf_hi(vw[2 * i])));
                    const float2 yb = __fmul2_rn(xs[2 * i + 1], make_float2(bf_lo(vw[2 * i + 1]), bf_hi(vw[2 * i + 1])));
                    o0[i] = pack_bf16(ya.x, yb.x);
                    o1[i] = pack_bf16(ya.y, yb.y);
                }
                const uint4 nan4 = make_uint4(0x7fc07fc0u, 0x7fc07fc0u, 0x7fc07fc0u, 0x7fc07fc0u);
                // a timed-out wait poisons the output
                *reinterpret_cast<uint4*>(y0 + n0) = ok ? make_uint4(o0[0], o0[1], o0[2], o0[3]) : nan4;
                if (pr.has1) *reinterpret_cast<uint4*>(y1 + n0) = ok ? make_uint4(o1[0], o1[1], o1[2], o1[3]) : nan4;
            }
        }
    };

    PairInput in;
    PairRef prev{0, 0, false};
    bool have_prev = false;

    for (int P = blockIdx.x; P < npairs; P += gridDim.x) {
        // this CTA's last pair: the next kernel may start its setup on the slots that
        // the CTAs already done leave free
        if (P + int(gridDim.x) >= npairs) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
        const PairRef pr = pair_ref(P, B);
        const int c = pr.c;
        const bf16* u0 = u + int64_t(pr.b0) * Ctot * L;
        const bf16* u1 = pr.has1 ? u0 + Ctot * L : u0;
        // this pair's step-1 input (the other CTA of the SM covers the load
        // latency; holding the next pair's samples in registers instead costs
        // spills that are slower than the wait)
        load_pair_input(in, u, pr, C, order, 0);
        load_pair_input(in, u, pr, C, order, 2);
        // ---------------- step-1 operand: z = sc(x_{order-1}) sc(v), g[b0] + i g[b1]
        {
            // an odd batch's last pair has no row b1: its v taps are zero, so z = g[b0]
            const Taps2 tg = taps2(load_taps(sc_w, sc_b, int64_t(order - 1) * C + c), 1.0f);
            const Taps2 tv = taps2(load_taps(sc_w, sc_b, int64_t(order) * C + c), pr.has1 ? 1.0f : 0.0f);
            const int chalf = t >> 7, a0 = 8 * (t & 127);
            // rows rho1(a0 + i) = rho1(a0) + 8 (i & 3) + (i >> 2) (a0 % 8 == 0); slots 4 chalf + j
            const int r0 = rho1(a0);
            const uint32_t base = uint32_t(r0 >> 3) * kSBO16 + uint32_t(chalf) * tc::kLBO + uint32_t(r0 & 7) * 16u;
#pragma unroll
            for (int jp = 0; jp < 4; jp += 2) {
                uint32_t pk[8][2];
#pragma unroll
                for (int jo = 0; jo < 2; ++jo) {
                    const int j = jp + jo;
                    float2 xs[8], vs[8];
                    sc8x2(in.x[0][j], in.x[1][j], tg, xs);
                    sc8x2(in.v[0][j], in.v[1][j], tv, vs);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float2 z = __fmul2_rn(xs[i], vs[i]);         // (g[b0], g[b1]) = (re, im)
                        pk[i][jo] = pack_bf16(z.x, z.y);
                    }
                }
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    *reinterpret_cast<uint2*>(A1 + base + uint32_t(i & 3) * kSBO16 + uint32_t(i >> 2) * 16u + 4u * jp) =
                        make_uint2(pk[i][0], pk[i][1]);
            }
            stage_issue(a1_addr, kSBO16, b1_addr, kSBO16, 8, 1, tc::idesc_bf16(128, 32), tmem, 32, &mbar, ok && issue_mma);
            if (t < 4)   // this pair's spectrum plane into L2 before its spectrum pass
                asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(spec + int64_t(c) * (2 * N) + t * (N / 4)),
                             "r"(uint32_t(N)) : "memory");
            if (have_prev) {
                output_gate(prev);                  // overlaps the stage-1 MMAs
                have_prev = false;
            }
            __syncthreads();                        // staging read by every thread before pass 1 overwrites it
        }
        for (int st = 1; st < order; ++st) {
            if (st > 1) {
                // previous step's output v = conj(stage-1' accumulators), row a, output s;
                // z = sc(x_g) v with g = order - st
                const int g = order - st;
                const Taps tg = load_taps(sc_w, sc_b, int64_t(g) * C + c);
                const bf16* xg0 = u0 + (int64_t(g) * C + c) * L;
                const bf16* xg1 = u1 + (int64_t(g) * C + c) * L;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int a = 128 * (4 * hh + j) + 32 * Q + lane;
                    float d[16];
                    tc::tmem_ld16(tl + uint32_t(16 * (4 * hh + j)), d);
                    tc::tmem_ld_wait();
                    uint32_t pk[8];
#pragma unroll
                    for (int s = 0; s < 8; ++s) {
                        const int n = a + 1024 * s;
                        const int col = 4 * (s >> 1) + (s & 1);            // re at col, im at col + 2
                        const float za = sc1(xg0, n, tg) * d[col];
                        const float zb = pr.has1 ? sc1(xg1, n, tg) * -d[col + 2] : 0.0f;
                        pk[s] = pack_bf16(za, zb);
                    }
                    sts128(A1, tc::chunk_off(rho1(a), 0, kSBO16), pk[0], pk[1], pk[2], pk[3]);
                    sts128(A1, tc::chunk_off(rho1(a), 1, kSBO16), pk[4], pk[5], pk[6], pk[7]);
                }
                stage_issue(a1_addr, kSBO16, b1_addr, kSBO16, 8, 1, tc::idesc_bf16(128, 32), tmem, 32, &mbar, ok && issue_mma);
            }
            tc16k::middle(tx, spec + (int64_t(st - 1) * C + c) * (2 * N), phase, ok);
            // ---------------- stage 1': 8 tiles x (K 32 -> N 16), outputs s < 8 only
            stage_issue(a_addr, kSBO32, b1i_addr, kSBO32, 8, 2, tc::idesc_bf16(128, 16), tmem, 16, &mbar, ok && issue_mma);
            if (st < order - 1) ok = stage_wait(&mbar, phase, ok, wait_budget_ns);
        }
        ok = stage_wait(&mbar, phase, ok, wait_budget_ns);
        // output staging v = conj(D1') as (re, -im) bf16 pairs in natural order;
        // the output gate runs during the next pair's stage 1
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int a = 128 * (4 * hh + j) + 32 * Q + lane;
            float d[16];
            tc::tmem_ld16(tl + uint32_t(16 * (4 * hh + j)), d);
            tc::tmem_ld_wait();
#pragma unroll
            for (int s8 = 0; s8 < 8; ++s8) {
                const int col = 4 * (s8 >> 1) + (s8 & 1);                 // re at col, im at col + 2
                Vs[a + 1024 * s8] = pack_bf16(d[col], -d[col + 2]);
            }
        }
        prev = pr;
        have_prev = true;
        if (__syncthreads_or(!ok)) {                    // a tensor-core wait ran out (uniform decision)
            ok = false;
            if (t == 0) report_status(status, kStatusTimeout);
            break;
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (have_prev) output_gate(prev);
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

cudaError_t launch_conv_8192_tc(const Plan& p, const ConvArgs& a, cudaStream_t s) {
    auto kern = k_conv_8192_tc;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmem));
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t npairs = p.C * ((a.B + 1) / 2);
    if (npairs > INT32_MAX || a.B > INT32_MAX) return cudaErrorInvalidValue;   // 32-bit pair indices
    int64_t grid = int64_t(2) * sms;
    if (grid > npairs) grid = npairs;
    // programmatic stream serialisation (see the kernel's prologue)
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(grid));
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = kSmem;
    cfg.stream = s;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<const bf16*>(a.u), static_cast<bf16*>(a.y), a.spectrum, a.sc_w,
                              a.sc_b, int(a.B), int(p.C), p.order, int(npairs), int64_t(p.tables_off),
                              int64_t(p.spec_off), int64_t(p.order + 1) * p.C, a.wait_budget_ns, a.issue_mma,
                              a.status);
}

}  // namespace hyena
