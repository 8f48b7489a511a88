// grid2d_tc.cu -- the 2-D forms on the tensor cores (tcgen05) with bf16
// storage ([P5] "Native Multi-Dimensional Subquadratic Operators"
// (gist.science), 方法论: N-D FFT convolution, non-circular by 2x zero
// padding): the column pass of the non-circular form at H = 256 (first part),
// the paired-image row, column and row passes at 256 x 256 (second part), and
// the circular form's paired passes at 256 x 256 (third part).
//
// The row pass leaves, per image, W + 1 bin columns of H = 256 complex values
// (bf16 (re, im) in the workspace).  Each column needs its 2H = 512-point DFT
// (rows H .. 2H-1 are zero), the product with its spectrum column and the
// inverse, keeping rows p < H.  With n = a + 32 s (a < 32, s < 8 non-zero)
// and bin k = k1 + 16 k2 (k1 < 16, k2 < 32):
//   X[k1 + 16 k2] = sum_a w32^(a k2) w512^(a k1) sum_s x[a + 32 s] w16^(s k1)
// so a task of 32 columns (16384 points) runs the first two stages of the
// 16384-point tensor-core FFT (tc16k.cuh: stage 1 over s, K = 16; stage 2
// over a, K = 64) with the twiddle w512^(a k1) between them, the spectrum
// product on the stage-2 accumulators, and the inverse through the same
// matrices (IDFT(x) = conj(DFT(conj x))): stage 2', the same twiddle, and
// stage 1' with only the outputs s < 8.  Rows of the stage-1 operand are
// a_tc = c + 32 a for column c of the task, i.e. b = c and q = a in the row
// orders of tc16k.cuh.
//
// Columns 0 .. W-1 run here (W / 32 tasks per image); the last column (bin W)
// stays on the register-engine column kernel.  The spectrum comes from a bf16
// plane in this kernel's thread order, gathered from the complex64 spectrum
// rows when the spectrum is built.
//
// Precision: column values, DFT matrices and the stage operands are bf16
// (fp32 accumulation), four roundings per transform pair; the 2-D row error
// stays a few 1e-3.
#include "common.cuh"
#include "cta_fft.cuh"
#include "kernels.h"
#include "plan_common.h"
#include "tc16k.cuh"
#include "tc_util.cuh"

namespace hyena {

namespace {

using namespace tc16k;

constexpr int MH = int(kTc2dH);   // column length H
constexpr int NCOL = 32;          // columns per task
constexpr int NT = 256;
static_assert(NCOL * MH * 2 == N, "a task is one 16384-point transform");
constexpr uint32_t kB1bytes = 4 * kSBO16;   // N 32 x K 16
constexpr uint32_t kB1ibytes = 2 * kSBO32;  // N 16 x K 32
constexpr uint32_t kOffA1 = kAbytes - 128 * kSBO16;   // stage-1 operand (1024 rows x K 16)
// the stage-2' operand's 8-row groups 1168 bytes apart instead of 1152: the
// spectrum pass writes rows 128 (k1 & 3) + 32 (k1 >> 2) + b, whose 16-byte
// stores then spread over all eight bank groups
constexpr uint32_t kSBO64s = kSBO64 + 16;
constexpr uint32_t kAbytesC = 64 * kSBO64s > kAbytes ? 64 * kSBO64s : kAbytes;
constexpr uint32_t kOffB1 = kAbytesC;
constexpr uint32_t kOffB32 = kOffB1 + kB1bytes;
constexpr uint32_t kOffB1i = kOffB32 + kB32bytes;
constexpr uint32_t kOffW512 = kOffB1i + kB1ibytes;
constexpr size_t kSmem = size_t(kOffW512) + 512 * sizeof(float2);
static_assert(NCOL * MH * 4 <= kOffA1, "output staging must not overlap the stage-1 operand");
static_assert(kOffA1 + 128 * kSBO16 <= kAbytesC, "stage-1 operand inside the operand area");
static_assert(kOffW512 % 16 == 0, "twiddle table alignment");
constexpr int kPlaneTask = N;     // bf16 (re, im) entries of the spectrum plane per task

// Spectrum plane entry e (uint32 bf16 pair) of task-plane index idx4 (uint4):
// idx4 = ((Q * 2 + h) * 16 + i) * 32 + lane, i = 4 T + q4 holds, for lane
// quarter Q, half h and tile T, row (k1 = 4 Q + lane / 8, column c = 4 (lane & 7) + T)
// and bins k2 = 16 h + 4 q4 + e (e < 4): the order the spectrum pass reads.
__device__ __forceinline__ void plane_entry(int idx4, int e, int& c, int& k) {
    const int lane = idx4 & 31, i = (idx4 >> 5) & 15, qh = idx4 >> 9;
    const int Q = qh >> 1, h = qh & 1, T = i >> 2, q4 = i & 3;
    const int k1 = 4 * Q + (lane >> 3);
    c = 4 * (lane & 7) + T;
    k = k1 + 16 * (16 * h + 4 * q4 + e);
}

// The plane from the complex64 spectrum rows: per row 2W/32 column blocks x
// 4096 uint4, columns f = 0 .. 2W-1 of the 2H x 2W transform.  Bin k of a
// stored column f <= W sits in the row at f * 2H + (k & 1) * H + the register
// engine's slot of position fft_bin_pos(k >> 1) (see the 2-D spectrum build);
// the columns f > W follow from the symmetry of the transform of a real
// filter, K~[k][f] = conj K~[-k mod 2H][2W - f].
__global__ void k_2d_plane_tc(const float2* __restrict__ rows, uint4* __restrict__ plane, int64_t nrows, int W,
                              int64_t row_stride) {
    const int64_t per_row = int64_t(2 * W / NCOL) * (kPlaneTask / 4);
    for (int64_t g = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; g < nrows * per_row;
         g += int64_t(gridDim.x) * blockDim.x) {
        const int64_t r = g / per_row;
        const int rem = int(g - r * per_row);
        const int task = rem / (kPlaneTask / 4), idx4 = rem - task * (kPlaneTask / 4);
        uint32_t v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            int c, k;
            plane_entry(idx4, e, c, k);
            const int f = NCOL * task + c;
            const bool mirror = f > W;
            const int fs = mirror ? 2 * W - f : f, ks = mirror ? (2 * MH - k) & (2 * MH - 1) : k;
            const int pos = fft_bin_pos<MH>(ks >> 1);
            const float2 K = rows[r * row_stride + int64_t(fs) * (2 * MH) + (ks & 1) * MH + (pos & 15) * (MH / 16) +
                                  (pos >> 4)];
            v[e] = pack_bf16(K.x, mirror ? -K.y : K.y);
        }
        plane[g] = make_uint4(v[0], v[1], v[2], v[3]);
    }
}


// Tables of a 2-D tensor-core kernel: the 32 entries of the DFT matrices (in
// the operand area, free until the first task), w512^e (e < 512), and the
// DFT matrices the kernel uses (S1: stage 1, K 16 -> N 32; S2: the 32-point
// stages; S1I: stage 1', K 32 -> N 16).
template <bool S1, bool S2, bool S1I>
__device__ __forceinline__ void setup_tables(uint8_t* smem, float2* w512) {
    float2* w32 = reinterpret_cast<float2*>(smem);
    fill_w32(w32);
    for (int e = threadIdx.x; e < 512; e += NT) {
        float sv, cv;
        sincospif(float(e) * (1.0f / 256.0f), &sv, &cv);   // w512^e = exp(-2 pi i e / 512)
        w512[e] = make_float2(cv, -sv);
    }
    __syncthreads();
    if (S1) fill_dft<16, 16, 8, kSBO16>(smem + kOffB1, w32);
    if (S2) fill_dft<32, 32, 32, kSBO64>(smem + kOffB32, w32);
    if (S1I) fill_dft<16, 8, 16, kSBO32>(smem + kOffB1i, w32);
}

// Stage-1 operand of a task: rows a_tc = c + 32 a (c < 32 the task's column or
// row, a < 32), slots s < 8 holding x[c][a + 32 s] = get(c, a, s) (a bf16
// pair); thread t takes rows a0 .. a0+7 (a0 = 8 (t & 127)) at slots
// 4 (t >> 7) .. +3 (the store pattern of the L = 8192 kernel's stage 1).
template <typename Get>
__device__ __forceinline__ void build_stage1(uint8_t* A1, Get get) {
    const int t = threadIdx.x;
    const int chalf = t >> 7, a0 = 8 * (t & 127);
    const int r0 = rho1(a0);
    const uint32_t base = uint32_t(r0 >> 3) * kSBO16 + uint32_t(chalf) * tc::kLBO + uint32_t(r0 & 7) * 16u;
    uint32_t x[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int atc = a0 + i;
#pragma unroll
        for (int j = 0; j < 4; ++j) x[i][j] = get(atc & 31, atc >> 5, 4 * chalf + j);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int jp = 0; jp < 4; jp += 2)
            *reinterpret_cast<uint2*>(A1 + base + uint32_t(i & 3) * kSBO16 + uint32_t(i >> 2) * 16u + 4u * jp) =
                make_uint2(x[i][jp], x[i][jp + 1]);
}

// Wait for stage 1, then pass 1: twiddle w512^(q k1) (q = j + 4 Q + 16 h, the a
// of the stage-1 row) into the stage-2 rows (k1, b) of tc16k.cuh's order.
__device__ __forceinline__ void pass1_512(uint8_t* A, const float2* w512, uint32_t tl, int Q, int hh, int lane,
                                          uint64_t* mbar, uint32_t& phase, bool& ok, uint64_t budget) {
    C2 pw[4], st2[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2 beta = w512[j + 4 * Q + 16 * hh];
        pw[j] = c2_of(make_float2(1.0f, 0.0f), beta);
        st2[j] = c2_splat(cmul(beta, beta));
    }
    ok = stage_wait(mbar, phase, ok, budget);
    const uint32_t base = uint32_t(16 * (lane >> 3)) * kSBO64 + uint32_t(Q + 4 * hh) * tc::kLBO + uint32_t(lane & 7) * 16u;
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
            sts128(A, base + uint32_t(4 * (k1 >> 2) + (k1 & 3)) * kSBO64, pack_bf16(v[0].re.x, v[0].im.x),
                   pack_bf16(v[1].re.x, v[1].im.x), pack_bf16(v[2].re.x, v[2].im.x), pack_bf16(v[3].re.x, v[3].im.x));
            sts128(A, base + uint32_t(4 * ((k1 + 1) >> 2) + ((k1 + 1) & 3)) * kSBO64, pack_bf16(v[0].re.y, v[0].im.y),
                   pack_bf16(v[1].re.y, v[1].im.y), pack_bf16(v[2].re.y, v[2].im.y), pack_bf16(v[3].re.y, v[3].im.y));
        }
    }
}

// Wait for stage 2', then pass 2': rows (k1 = 4 Q + T, b = lane), outputs q =
// 16 h + ..; twiddle w512^(q k1) -> stage-1' row b + 32 q, chunk Q (slots k1 =
// 4 Q .. 4 Q + 3).
__device__ __forceinline__ void pass2i_512(uint8_t* A, const float2* w512, uint32_t tl, int Q, int hh, int lane,
                                           uint64_t* mbar, uint32_t& phase, bool& ok, uint64_t budget) {
    const uint32_t base = uint32_t((lane >> 3) + 64 * hh) * kSBO32 + uint32_t(Q) * tc::kLBO + uint32_t(lane & 7) * 16u;
    C2 pw[4], st2[4];
#pragma unroll
    for (int T = 0; T < 4; ++T) {
        const int k1 = 4 * Q + T;
        const float2 p0 = w512[(16 * hh * k1) & 511];
        pw[T] = c2_of(p0, cmul(p0, w512[k1]));
        st2[T] = c2_splat(w512[(2 * k1) & 511]);
    }
    ok = stage_wait(mbar, phase, ok, budget);
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
                   pack_bf16(v[1].re.x, v[1].im.x), pack_bf16(v[2].re.x, v[2].im.x), pack_bf16(v[3].re.x, v[3].im.x));
            sts128(A, base + uint32_t(16 * gq + 4 * (i + 1)) * kSBO32, pack_bf16(v[0].re.y, v[0].im.y),
                   pack_bf16(v[1].re.y, v[1].im.y), pack_bf16(v[2].re.y, v[2].im.y), pack_bf16(v[3].re.y, v[3].im.y));
        }
    }
}

__global__ void __launch_bounds__(NT, 2)
k_2d_cols_tc(__nv_bfloat162* __restrict__ ws, const uint8_t* __restrict__ spectrum, int C, int W, int64_t B,
             int step, int64_t img0, int nimg, int64_t ws_img_stride, int64_t plane_off, int64_t SC, int64_t SB,
             int hdr_W, uint64_t wait_budget_ns, int issue_mma, uint32_t* status) {
    extern __shared__ __align__(1024) uint8_t smem_2t[];
    __shared__ __align__(8) uint64_t mbar;
    __shared__ uint32_t tmem_base;
    uint8_t* A = smem_2t;
    uint8_t* A1 = smem_2t + kOffA1;
    uint32_t* Vs = reinterpret_cast<uint32_t*>(smem_2t);     // output staging [column][p]
    float2* w512 = reinterpret_cast<float2*>(smem_2t + kOffW512);
    const int t = threadIdx.x;
    const int warp = t >> 5, lane = t & 31;
    const int Q = warp & 3, hh = warp >> 2;

    setup_tables<true, true, true>(smem_2t, w512);
    // launched with programmatic stream serialisation in the paired passes: the
    // tables are built while the previous kernel finishes; nothing global is read
    // or written before this wait
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const SpecHeader hv = *reinterpret_cast<const SpecHeader*>(spectrum);
    const bool hdr_ok = (hv.magic == kSpecMagic) & (hv.path == PATH_GRID_2D) & (hv.H == MH) & (hv.W == hdr_W) &
                        (hv.reserved[1] == plane_off);
    if (!hdr_ok) {
        if (t == 0) report_status(status, kStatusSpectrumMismatch);
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
    const uint32_t a1_addr = tc::smem_u32(A1);
    const uint32_t b1_addr = tc::smem_u32(smem_2t + kOffB1);
    const uint32_t b32_addr = tc::smem_u32(smem_2t + kOffB32);
    const uint32_t b1i_addr = tc::smem_u32(smem_2t + kOffB1i);
    const uint4* plane = reinterpret_cast<const uint4*>(spectrum + plane_off);
    uint32_t phase = 0;
    bool ok = true;
    const int groups = W / NCOL;                  // column blocks of an image (its first W columns)
    const int pgroups = 2 * hdr_W / NCOL;         // column blocks of a plane row
    const int ntasks = nimg * groups;

    for (int task = blockIdx.x; task < ntasks; task += gridDim.x) {
        const int li = task / groups, cg = task - li * groups;
        const int64_t img = img0 + li;
        uint32_t* col0 = reinterpret_cast<uint32_t*>(ws + int64_t(li) * ws_img_stride) + int64_t(NCOL * cg) * MH;
        const int64_t c = img / B, b = img - c * B;
        const uint4* kq = plane + ((int64_t(step) * SC + b * SB + c) * pgroups + cg) * (kPlaneTask / 4) +
                          (Q * 2 + hh) * 16 * 32 + lane;
        // ---------------- stage-1 operand: rows a_tc = c + 32 a, slots s < 8 (x[c][a + 32 s])
        build_stage1(A1, [&](int cc, int aa, int sl) { return col0[cc * MH + aa + 32 * sl]; });
        stage_issue(a1_addr, kSBO16, b1_addr, kSBO16, 8, 1, tc::idesc_bf16(128, 32), tmem, 32, &mbar, ok && issue_mma);
        if (t < 12 && task + int(gridDim.x) < ntasks) {
            // the next task's 32 columns (32 KB) and spectrum block (64 KB) into L2
            const int nt = task + int(gridDim.x), nli = nt / groups, ncg = nt - nli * groups;
            const int64_t nimg_i = img0 + nli, nc = nimg_i / B, nb = nimg_i - nc * B;
            const uint8_t* src = t < 4 ? reinterpret_cast<const uint8_t*>(reinterpret_cast<const uint32_t*>(
                                             ws + int64_t(nli) * ws_img_stride) + int64_t(NCOL * ncg) * MH) + 8192 * t
                                       : reinterpret_cast<const uint8_t*>(
                                             plane + ((int64_t(step) * SC + nb * SB + nc) * pgroups + ncg) *
                                                         (kPlaneTask / 4)) + 8192 * (t - 4);
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(8192u) : "memory");
        }
        // ---------------- pass 1: twiddle w512^(q k1), q = j + 4 Q + 16 h (= a), rows of stage 2 (k1, b = c)
        pass1_512(A, w512, tl, Q, hh, lane, &mbar, phase, ok, wait_budget_ns);
        // ---------------- stage 2 (over a); meanwhile this thread loads its spectrum values
        stage_issue(a_addr, kSBO64, b32_addr, kSBO64, 4, 4, tc::idesc_bf16(128, 64), tmem, 64, &mbar, ok && issue_mma);
        {
            // rows (k1 = 4 Q + lane / 8, b = 4 (lane & 7) + T), bins k2 = 16 h + 4 q4 + e; the
            // product conj(X K~) goes to the stage-2' row 128 (k1 & 3) + 32 (k1 >> 2) + b,
            // chunk k2 / 4 (the row order of tc16k's pass 2')
            uint4 kv[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) kv[i] = __ldg(kq + 32 * i);
            ok = stage_wait(&mbar, phase, ok, wait_budget_ns);
#pragma unroll
            for (int TH = 0; TH < 8; ++TH) {
                const int T = TH >> 1;
                float d[16];
                tc::tmem_ld16(tl + uint32_t(64 * T + 32 * hh + 16 * (TH & 1)), d);
                tc::tmem_ld_wait();
                const int row = 128 * (lane >> 3) + 32 * Q + 4 * (lane & 7) + T;
#pragma unroll
                for (int q4 = 2 * (TH & 1); q4 < 2 * (TH & 1) + 2; ++q4) {
                    const uint4 kk = kv[4 * T + q4];
                    const C2 K0{make_float2(bf_lo(kk.x), bf_lo(kk.y)), make_float2(bf_hi(kk.x), bf_hi(kk.y))};
                    const C2 K1{make_float2(bf_lo(kk.z), bf_lo(kk.w)), make_float2(bf_hi(kk.z), bf_hi(kk.w))};
                    const C2 v0 = cmul2(c2_at(d, 2 * (q4 & 1)), K0);
                    const C2 v1 = cmul2(c2_at(d, 2 * (q4 & 1) + 1), K1);
                    sts128(A, tc::chunk_off(row, 4 * hh + q4, kSBO64s), pack_bf16(v0.re.x, -v0.im.x),
                           pack_bf16(v0.re.y, -v0.im.y), pack_bf16(v1.re.x, -v1.im.x), pack_bf16(v1.re.y, -v1.im.y));
                }
            }
        }
        // ---------------- stage 2' (inverse, on conj)
        stage_issue(a_addr, kSBO64s, b32_addr, kSBO64, 4, 4, tc::idesc_bf16(128, 64), tmem, 64, &mbar, ok && issue_mma);
        pass2i_512(A, w512, tl, Q, hh, lane, &mbar, phase, ok, wait_budget_ns);
        // ---------------- stage 1': 8 tiles x (K 32 -> N 16), outputs s < 8 only
        stage_issue(a_addr, kSBO32, b1i_addr, kSBO32, 8, 2, tc::idesc_bf16(128, 16), tmem, 16, &mbar, ok && issue_mma);
        ok = stage_wait(&mbar, phase, ok, wait_budget_ns);
        // result conj(D1') at row a_tc = c + 32 a, output s -> Vs[c][a + 32 s], then the
        // task's 32 columns (contiguous in the workspace) in 16-byte stores
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int atc = 128 * (4 * hh + j) + 32 * Q + lane;
            float d[16];
            tc::tmem_ld16(tl + uint32_t(16 * (4 * hh + j)), d);
            tc::tmem_ld_wait();
            const int cc = atc & 31, aa = atc >> 5;
#pragma unroll
            for (int s8 = 0; s8 < 8; ++s8) {
                // a warp's lanes are 32 columns (1 KB apart): word p of column cc sits at
                // p ^ cc, so that they fall in 32 different banks
                const int col = 4 * (s8 >> 1) + (s8 & 1);                 // re at col, im at col + 2
                Vs[cc * MH + ((aa + 32 * s8) ^ cc)] = ok ? pack_bf16(d[col], -d[col + 2]) : 0x7fc07fc0u;
            }
        }
        tc::fence_before_sync();
        __syncthreads();
        {
            // 16-byte group g of column cc (words 4g .. 4g+3) is group g ^ (cc >> 2) with its
            // words permuted by cc & 3; cc is the same for the 32 lanes of a warp
            uint4* dst = reinterpret_cast<uint4*>(col0);
#pragma unroll
            for (int k = 0; k < NCOL * MH / 4 / NT; ++k) {
                const int gi = t + NT * k, cc = gi >> 6, g = gi & 63;
                uint4 v = *reinterpret_cast<const uint4*>(Vs + cc * MH + 4 * (g ^ (cc >> 2)));
                if (cc & 1) v = make_uint4(v.y, v.x, v.w, v.z);
                if (cc & 2) v = make_uint4(v.z, v.w, v.x, v.y);
                dst[gi] = v;
            }
        }
        if (__syncthreads_or(!ok)) {                    // a tensor-core wait ran out (uniform decision)
            if (t == 0) report_status(status, kStatusTimeout);
            break;
        }
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");   // the next kernel may start its setup
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, kTmemCols);
}


// ---------------------------------------------------------------------------
// Paired images: the two images (b0, b0 + 1) of a channel share the real
// filter, so they travel as one complex image z = g[b0] + i g[b0 + 1] (g the
// gated input), and every pass is a plain 512-point complex transform with
// 256 non-zero inputs: rows forward (here), the column kernel above over all
// 2W = 512 bin columns, rows inverse with the output gate (below).  The
// workspace of a pair holds Z[k][row] (k < 512 bins, 256 rows, bf16 pairs).
// With the unnormalised transforms both ways the spectrum must be
// (DFT(k) + D) / (4HW), twice the stored (DFT(k) + D) / (8HW), whose other
// factor two belongs to the packed-real row passes of the unpaired path.
// ---------------------------------------------------------------------------

constexpr int W2 = 256;           // image width of the paired path (row transform 512)
constexpr int NROW = 32;          // image rows per task

// Raw input rows of a task (32 rows of both images of a pair), held in
// registers between their loads and the staging: x, and v when GATE.
constexpr int kRowIt = NROW * W2 / 8 / NT;   // 16-byte groups of a row image per thread
template <bool GATE>
struct PairRows {
    uint4 x[kRowIt][2];
    uint4 v[GATE ? kRowIt : 1][2];
};
template <bool GATE>
__device__ __forceinline__ void load_pair_rows(PairRows<GATE>& in, const bf16* __restrict__ x_b0,
                                               const bf16* __restrict__ x_b1, const bf16* __restrict__ v_b0,
                                               const bf16* __restrict__ v_b1, int t) {
#pragma unroll
    for (int jj = 0; jj < kRowIt; ++jj) {
        const int ci = t + NT * jj, r = ci >> 5, n0 = 8 * (ci & 31);
        const int64_t off = int64_t(r) * W2 + n0;
        in.x[jj][0] = __ldg(reinterpret_cast<const uint4*>(x_b0 + off));
        in.x[jj][1] = __ldg(reinterpret_cast<const uint4*>(x_b1 + off));
        if constexpr (GATE) {
            in.v[jj][0] = __ldg(reinterpret_cast<const uint4*>(v_b0 + off));
            in.v[jj][1] = __ldg(reinterpret_cast<const uint4*>(v_b1 + off));
        }
    }
}
// z of the task's rows -> staging Zs[r][n ^ (8 (r >> 3))] (bf16 pairs (z[b0], z[b1])):
// the XOR lets the stage-1 gathers read 32 different banks.  GATE: z = x v (the
// first order step), else z = x (a later step's input, already gated by the
// previous step's inverse pass).
template <bool GATE>
__device__ __forceinline__ void store_pair_rows(uint32_t* Zs, const PairRows<GATE>& in, int t) {
#pragma unroll
    for (int jj = 0; jj < kRowIt; ++jj) {
        const int ci = t + NT * jj, r = ci >> 5, n0 = 8 * (ci & 31);
        const uint4 xa = in.x[jj][0], xb = in.x[jj][1];
        const uint32_t xw[2][4] = {{xa.x, xa.y, xa.z, xa.w}, {xb.x, xb.y, xb.z, xb.w}};
        uint32_t o[8];
        if constexpr (GATE) {
            const uint4 va = in.v[jj][0], vb = in.v[jj][1];
            const uint32_t vw[2][4] = {{va.x, va.y, va.z, va.w}, {vb.x, vb.y, vb.z, vb.w}};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                // samples 2q, 2q+1 of both images: (g[b0], g[b1]) at each
                const float2 lo = __fmul2_rn(make_float2(bf_lo(xw[0][q]), bf_lo(xw[1][q])),
                                             make_float2(bf_lo(vw[0][q]), bf_lo(vw[1][q])));
                const float2 hi = __fmul2_rn(make_float2(bf_hi(xw[0][q]), bf_hi(xw[1][q])),
                                             make_float2(bf_hi(vw[0][q]), bf_hi(vw[1][q])));
                o[2 * q] = pack_bf16(lo.x, lo.y);
                o[2 * q + 1] = pack_bf16(hi.x, hi.y);
            }
        } else {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                // the two images' samples interleaved: (z[b0], z[b1]) per sample
                o[2 * q] = __byte_perm(xw[0][q], xw[1][q], 0x5410);
                o[2 * q + 1] = __byte_perm(xw[0][q], xw[1][q], 0x7632);
            }
        }
        uint32_t* dst = Zs + r * W2 + (n0 ^ (8 * (r >> 3)));
        *reinterpret_cast<uint4*>(dst) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4*>(dst + 4) = make_uint4(o[4], o[5], o[6], o[7]);
    }
}
template <bool GATE>
__device__ __forceinline__ void stage_pair_rows(uint32_t* Zs, const bf16* __restrict__ x_b0, const bf16* __restrict__ x_b1,
                                                const bf16* __restrict__ v_b0, const bf16* __restrict__ v_b1, int t) {
    PairRows<GATE> in;
    load_pair_rows<GATE>(in, x_b0, x_b1, v_b0, v_b1, t);
    store_pair_rows<GATE>(Zs, in, t);
}

// Output gate of 32 rows of a pair: the gate rows x_b0 / x_b1 (loaded into
// gx first, so that their loads can be issued early), times the staged result
// Ys[r][n ^ r] (bf16 pairs (image b0, image b1)), stored to y_b0 / y_b1 (rows of
// W2 samples), 8 columns of a row per step; NaN once a wait ran out.
__device__ __forceinline__ void load_gate_rows(uint4 (&gx)[kRowIt][2], const bf16* __restrict__ xa,
                                               const bf16* __restrict__ xb, int t) {
#pragma unroll
    for (int jj = 0; jj < kRowIt; ++jj) {
        const int ci = t + NT * jj, r = ci >> 5, n0 = 8 * (ci & 31);
        const int64_t off = int64_t(r) * W2 + n0;
        gx[jj][0] = __ldg(reinterpret_cast<const uint4*>(xa + off));
        gx[jj][1] = __ldg(reinterpret_cast<const uint4*>(xb + off));
    }
}
__device__ __forceinline__ void apply_gate_rows(const uint32_t* Ys, const uint4 (&gx)[kRowIt][2], bf16* __restrict__ ya,
                                                bf16* __restrict__ yb, int t, bool ok) {
#pragma unroll
    for (int jj = 0; jj < kRowIt; ++jj) {
        const int ci = t + NT * jj, r = ci >> 5, n0 = 8 * (ci & 31);
        const int64_t off = int64_t(r) * W2 + n0;
        const uint4 x0a = gx[jj][0], x0b = gx[jj][1];
        // word n0 + i sits at (n0 ^ (r & 24)) + (i ^ (r & 7))
        const uint32_t* src = Ys + r * W2 + (n0 ^ (r & 24));
        const uint4 g0 = *reinterpret_cast<const uint4*>(src);
        const uint4 g1 = *reinterpret_cast<const uint4*>(src + 4);
        uint32_t w[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
        const int m = r & 7;
        if (m & 1) {
#pragma unroll
            for (int i = 0; i < 8; i += 2) { const uint32_t tmp = w[i]; w[i] = w[i + 1]; w[i + 1] = tmp; }
        }
        if (m & 2) {
#pragma unroll
            for (int i = 0; i < 8; i += 4) {
                uint32_t tmp = w[i]; w[i] = w[i + 2]; w[i + 2] = tmp;
                tmp = w[i + 1]; w[i + 1] = w[i + 3]; w[i + 3] = tmp;
            }
        }
        if (m & 4) {
#pragma unroll
            for (int i = 0; i < 4; ++i) { const uint32_t tmp = w[i]; w[i] = w[i + 4]; w[i + 4] = tmp; }
        }
        const uint32_t xaw[4] = {x0a.x, x0a.y, x0a.z, x0a.w}, xbw[4] = {x0b.x, x0b.y, x0b.z, x0b.w};
        uint32_t oa[4], ob[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float2 lo = __fmul2_rn(make_float2(bf_lo(xaw[q]), bf_lo(xbw[q])),
                                         make_float2(bf_lo(w[2 * q]), bf_hi(w[2 * q])));
            const float2 hi = __fmul2_rn(make_float2(bf_hi(xaw[q]), bf_hi(xbw[q])),
                                         make_float2(bf_lo(w[2 * q + 1]), bf_hi(w[2 * q + 1])));
            oa[q] = pack_bf16(lo.x, hi.x);
            ob[q] = pack_bf16(lo.y, hi.y);
        }
        const uint4 nan4 = make_uint4(0x7fc07fc0u, 0x7fc07fc0u, 0x7fc07fc0u, 0x7fc07fc0u);
        *reinterpret_cast<uint4*>(ya + off) = ok ? make_uint4(oa[0], oa[1], oa[2], oa[3]) : nan4;
        *reinterpret_cast<uint4*>(yb + off) = ok ? make_uint4(ob[0], ob[1], ob[2], ob[3]) : nan4;
    }
}
__device__ __forceinline__ void gate_store_pair_rows(const uint32_t* Ys, const bf16* __restrict__ xa,
                                                     const bf16* __restrict__ xb, bf16* __restrict__ ya,
                                                     bf16* __restrict__ yb, int t, bool ok) {
    uint4 gx[kRowIt][2];
    load_gate_rows(gx, xa, xb, t);
    apply_gate_rows(Ys, gx, ya, yb, t, ok);
}

__global__ void __launch_bounds__(NT, 2)
k_2d_rows_fwd_tc(const bf16* __restrict__ u, const bf16* __restrict__ zsrc, __nv_bfloat162* __restrict__ ws,
                 const uint8_t* __restrict__ spectrum, int64_t B, int64_t C, int order, int64_t pair0, int npairs,
                 int64_t ws_pair_stride,
                 uint64_t wait_budget_ns, int issue_mma, uint32_t* status) {
    extern __shared__ __align__(1024) uint8_t smem_rf[];
    __shared__ __align__(8) uint64_t mbar;
    __shared__ uint32_t tmem_base;
    uint8_t* A = smem_rf;
    uint8_t* A1 = smem_rf + kOffA1;
    uint32_t* Zs = reinterpret_cast<uint32_t*>(smem_rf);     // gated rows, then the output staging
    float2* w512 = reinterpret_cast<float2*>(smem_rf + kOffW512);
    const int t = threadIdx.x;
    const int warp = t >> 5, lane = t & 31;
    const int Q = warp & 3, hh = warp >> 2;
    setup_tables<true, true, false>(smem_rf, w512);
    asm volatile("griddepcontrol.wait;" ::: "memory");   // as in k_2d_cols_tc
    const SpecHeader hv = *reinterpret_cast<const SpecHeader*>(spectrum);
    const bool hdr_ok = (hv.magic == kSpecMagic) & (hv.path == PATH_GRID_2D) & (hv.H == MH) & (hv.W == W2);
    if (!hdr_ok) {
        if (t == 0) report_status(status, kStatusSpectrumMismatch);
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
    const uint32_t a1_addr = tc::smem_u32(A1);
    const uint32_t b1_addr = tc::smem_u32(smem_rf + kOffB1);
    const uint32_t b32_addr = tc::smem_u32(smem_rf + kOffB32);
    uint32_t phase = 0;
    bool ok = true;
    const int64_t nb2 = B / 2, Ctot = int64_t(order + 1) * C, n_img = int64_t(MH) * W2;
    const int ntasks = npairs * (MH / NROW);

    for (int task = blockIdx.x; task < ntasks; task += gridDim.x) {
        const int lp = task / (MH / NROW), rg = task - lp * (MH / NROW);
        const int64_t pr = pair0 + lp, c = pr / nb2, b0 = 2 * (pr - c * nb2);
        const int64_t rowoff = int64_t(NROW * rg) * W2;
        if (zsrc == nullptr) {
            // first order step: z = x_{order-1} v
            const bf16* x0 = u + (b0 * Ctot + int64_t(order - 1) * C + c) * n_img + rowoff;
            const bf16* v0 = u + (b0 * Ctot + int64_t(order) * C + c) * n_img + rowoff;
            stage_pair_rows<true>(Zs, x0, x0 + Ctot * n_img, v0, v0 + Ctot * n_img, t);
        } else {
            // later steps: z written by the previous step's inverse pass ([B, C, H, W])
            const bf16* z0 = zsrc + (b0 * C + c) * n_img + rowoff;
            stage_pair_rows<false>(Zs, z0, z0 + C * n_img, nullptr, nullptr, t);
        }
        __syncthreads();
        // ---------------- stage-1 operand: rows a_tc = r + 32 a, slots s < 8 (z[r][a + 32 s])
        build_stage1(A1, [&](int r, int aa, int sl) { return Zs[r * W2 + ((aa + 32 * sl) ^ (8 * (r >> 3)))]; });
        stage_issue(a1_addr, kSBO16, b1_addr, kSBO16, 8, 1, tc::idesc_bf16(128, 32), tmem, 32, &mbar, ok && issue_mma);
        // ---------------- pass 1: twiddle w512^(q k1), rows of stage 2 (k1, b = r)
        pass1_512(A, w512, tl, Q, hh, lane, &mbar, phase, ok, wait_budget_ns);
        // ---------------- stage 2 (over a): Z[k1 + 16 k2] of row r
        stage_issue(a_addr, kSBO64, b32_addr, kSBO64, 4, 4, tc::idesc_bf16(128, 64), tmem, 64, &mbar, ok && issue_mma);
        ok = stage_wait(&mbar, phase, ok, wait_budget_ns);
        // rows (k1 = 4 Q + lane / 8, r = 4 (lane & 7) + T), bins k2 = 16 h + ..: staging
        // Os[k][r ^ (k & 3)] (the 32 lanes of a store hit 32 banks), then 128-byte rows
        // Z[k][32 rg .. 32 rg + 31] of the workspace
        {
            uint32_t* Os = reinterpret_cast<uint32_t*>(smem_rf);
            const int k1 = 4 * Q + (lane >> 3);
#pragma unroll
            for (int TH = 0; TH < 8; ++TH) {
                const int T = TH >> 1;
                float d[16];
                tc::tmem_ld16(tl + uint32_t(64 * T + 32 * hh + 16 * (TH & 1)), d);
                tc::tmem_ld_wait();
                const int r = 4 * (lane & 7) + T;
#pragma unroll
                for (int pcol = 0; pcol < 4; ++pcol) {
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int k2 = 16 * hh + 8 * (TH & 1) + 2 * pcol + e;
                        const int k = k1 + 16 * k2;
                        Os[k * NROW + (r ^ (k & 3))] = ok ? pack_bf16(d[4 * pcol + e], d[4 * pcol + 2 + e]) : 0x7fc07fc0u;
                    }
                }
            }
            tc::fence_before_sync();
            __syncthreads();
            uint32_t* wsp = reinterpret_cast<uint32_t*>(ws + int64_t(lp) * ws_pair_stride) + NROW * rg;
#pragma unroll 4
            for (int kk = 0; kk < 512 * NROW / 4 / NT; ++kk) {
                const int gi = t + NT * kk, k = gi >> 3, g4 = gi & 7;
                uint4 v = *reinterpret_cast<const uint4*>(Os + k * NROW + 4 * g4);
                const int m = k & 3;                  // word r sits at r ^ m inside its group of 4
                if (m & 1) v = make_uint4(v.y, v.x, v.w, v.z);
                if (m & 2) v = make_uint4(v.z, v.w, v.x, v.y);
                *reinterpret_cast<uint4*>(wsp + int64_t(k) * MH + 4 * g4) = v;
            }
        }
        if (__syncthreads_or(!ok)) {
            if (t == 0) report_status(status, kStatusTimeout);
            break;
        }
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");   // the next kernel may start its setup
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, kTmemCols);
}

__global__ void __launch_bounds__(NT, 2)
k_2d_rows_inv_tc(const bf16* __restrict__ u, bf16* __restrict__ y, const __nv_bfloat162* __restrict__ ws,
                 const uint8_t* __restrict__ spectrum, int64_t B, int64_t C, int order, int gchunk, int64_t pair0,
                 int npairs,
                 int64_t ws_pair_stride, uint64_t wait_budget_ns, int issue_mma, uint32_t* status) {
    extern __shared__ __align__(1024) uint8_t smem_ri[];
    __shared__ __align__(8) uint64_t mbar;
    __shared__ uint32_t tmem_base;
    uint8_t* A = smem_ri;
    uint32_t* Ys = reinterpret_cast<uint32_t*>(smem_ri);      // output staging [r][n ^ r]
    float2* w512 = reinterpret_cast<float2*>(smem_ri + kOffW512);
    const int t = threadIdx.x;
    const int warp = t >> 5, lane = t & 31;
    const int Q = warp & 3, hh = warp >> 2;
    setup_tables<false, true, true>(smem_ri, w512);
    asm volatile("griddepcontrol.wait;" ::: "memory");   // as in k_2d_cols_tc
    const SpecHeader hv = *reinterpret_cast<const SpecHeader*>(spectrum);
    const bool hdr_ok = (hv.magic == kSpecMagic) & (hv.path == PATH_GRID_2D) & (hv.H == MH) & (hv.W == W2);
    if (!hdr_ok) {
        if (t == 0) report_status(status, kStatusSpectrumMismatch);
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
    const uint32_t b32_addr = tc::smem_u32(smem_ri + kOffB32);
    const uint32_t b1i_addr = tc::smem_u32(smem_ri + kOffB1i);
    uint32_t phase = 0;
    bool ok = true;
    const int64_t nb2 = B / 2, Ctot = int64_t(order + 1) * C, n_img = int64_t(MH) * W2;
    const int ntasks = npairs * (MH / NROW);

    for (int task = blockIdx.x; task < ntasks; task += gridDim.x) {
        const int lp = task / (MH / NROW), rg = task - lp * (MH / NROW);
        const int64_t pr = pair0 + lp, c = pr / nb2, b0 = 2 * (pr - c * nb2);
        // ---------------- stage-2' operand: conj Y[k1 + 16 k2][r] at row 128 (k1 & 3) +
        // 32 (k1 >> 2) + r, chunk k2 / 4 (row groups kSBO64s apart); lane = r
        {
            const uint32_t* wsp = reinterpret_cast<const uint32_t*>(ws + int64_t(lp) * ws_pair_stride) + NROW * rg + lane;
            // all 64 loads of the thread in flight together (they wait on L2, not on
            // each other)
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                const int ci = warp + 8 * m, k1 = ci & 15, ch = ci >> 4;
                uint32_t q[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) q[e] = wsp[int64_t(k1 + 16 * (4 * ch + e)) * MH] ^ 0x80000000u;
                const int row = 128 * (k1 & 3) + 32 * (k1 >> 2) + lane;
                sts128(A, tc::chunk_off(row, ch, kSBO64s), q[0], q[1], q[2], q[3]);
            }
        }
        stage_issue(a_addr, kSBO64s, b32_addr, kSBO64, 4, 4, tc::idesc_bf16(128, 64), tmem, 64, &mbar, ok && issue_mma);
        // ---------------- pass 2' (twiddle w512^(q k1)) -> stage-1' rows r + 32 q
        pass2i_512(A, w512, tl, Q, hh, lane, &mbar, phase, ok, wait_budget_ns);
        // ---------------- stage 1': outputs s < 8 (n = a + 32 s < 256)
        stage_issue(a_addr, kSBO32, b1i_addr, kSBO32, 8, 2, tc::idesc_bf16(128, 16), tmem, 16, &mbar, ok && issue_mma);
        ok = stage_wait(&mbar, phase, ok, wait_budget_ns);
        // 2 conj(D1') at row a_tc = r + 32 a, output s: (image b0, image b1) of row r,
        // column n = a + 32 s -> Ys[r][n ^ r]
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int atc = 128 * (4 * hh + j) + 32 * Q + lane;
            float d[16];
            tc::tmem_ld16(tl + uint32_t(16 * (4 * hh + j)), d);
            tc::tmem_ld_wait();
            const int r = atc & 31, aa = atc >> 5;
#pragma unroll
            for (int s8 = 0; s8 < 8; ++s8) {
                const int col = 4 * (s8 >> 1) + (s8 & 1);
                Ys[r * W2 + ((aa + 32 * s8) ^ r)] = pack_bf16(2.0f * d[col], -2.0f * d[col + 2]);
            }
        }
        tc::fence_before_sync();
        __syncthreads();
        // gate: y = x_gchunk * conv for both images (x0 at the last order step,
        // else the next step's input)
        {
            const int64_t rowoff = int64_t(NROW * rg) * W2;
            const bf16* xa = u + (b0 * Ctot + int64_t(gchunk) * C + c) * n_img + rowoff;
            bf16* ya = y + (b0 * C + c) * n_img + rowoff;
            gate_store_pair_rows(Ys, xa, xa + Ctot * n_img, ya, ya + C * n_img, t, ok);
        }
        if (__syncthreads_or(!ok)) {
            if (t == 0) report_status(status, kStatusTimeout);
            break;
        }
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");   // the next kernel may start its setup
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, kTmemCols);
}


// ---------------------------------------------------------------------------
// The circular 2-D form ([P5] "Native Multi-Dimensional Subquadratic
// Operators", 方法论: the N-D FFT convolution; without the zero padding the
// product of the transforms is the periodic convolution) at 256 x 256 with
// bf16 storage, the two images of a channel paired as above.  Every line
// transform is a 256-point complex DFT, n = n1 + 16 n2, k = k1 + 16 k2:
//   X[k1 + 16 k2] = sum_n1 w16^(n1 k2) w256^(n1 k1) sum_n2 x[n1 + 16 n2] w16^(n2 k1)
// two stages with the real form of the full 16-point DFT matrix (K 32 -> N
// 32) and the twiddle w256^(n1 k1) between them.  The inverse runs on conj
// through the same matrix and twiddle: a stage over k2 (-> n1), the twiddle
// w256^(k1 n1), a stage over k1 (-> n2).  A task is 32 lines (8192 points,
// four tiles of 128 rows); the vector (line l, index i) of every stage sits at
//   R(l, i) = 128 (i & 3) + 32 (i >> 2) + l,
// so that thread (lane quarter Q, lane l) holds i = 4 Q + T in tile T and the
// four slots of each 16-byte chunk it writes.  Three kernels per order step,
// as for the padded pairs: rows forward (gates, Z[k][row] to the workspace),
// columns (forward, spectrum product, inverse; in place), rows inverse (output
// gate).  The spectrum is the full 256 x 256 plane (bf16 pairs) in the column
// pass's thread order, completed from the stored W/2 + 1 columns by the
// symmetry of a real filter's transform.  Each kernel copies the next task's
// inputs into shared memory with cp.async while the current task is
// transformed; its output staging reuses the operand area, which is free once
// the last stage is done.
// ---------------------------------------------------------------------------

constexpr int CN = int(kTc2dH);                  // H = W of the circular tensor-core path
constexpr uint32_t kSBOc = kSBO32;               // operand rows of K 32 (16 complex slots)
constexpr uint32_t kAc = 64 * kSBOc;             // 512 rows
constexpr uint32_t kOffStC = kAc;                // staging: 32 lines x 256 bf16 pairs
constexpr uint32_t kOffBc = kOffStC + NROW * CN * 4;
constexpr uint32_t kOffW256 = kOffBc + 4 * kSBOc;   // after the N 32 x K 32 DFT matrix
constexpr size_t kSmemC = size_t(kOffW256) + CN * sizeof(float2);
constexpr uint32_t kTmemColsC = 128;             // 4 tiles x 32 columns
constexpr int kPlaneTaskC = NROW * CN;           // bf16 pairs of the plane per column task
static_assert(kOffStC % 16 == 0 && kOffW256 % 16 == 0, "table alignment");
// the rows-forward kernel stages the raw rows of x and v of both images (four
// 16 KB planes) in place of the 32 KB staging, its tables after them
constexpr uint32_t kRawPlane = NROW * CN * 2;
constexpr uint32_t kOffBcF = kOffStC + 4 * kRawPlane;
constexpr uint32_t kOffW256F = kOffBcF + 4 * kSBOc;
constexpr size_t kSmemCF = size_t(kOffW256F) + CN * sizeof(float2);
static_assert(2 * (kSmemCF + 2048) <= 227 * 1024, "two rows-forward CTAs per SM");

__device__ __forceinline__ int rowc(int l, int i) { return 128 * (i & 3) + 32 * (i >> 2) + l; }

// Plane entry e of uint4 idx4 of a column task: idx4 = ((Q * 2 + h) * 8 + 2 T +
// half) * 32 + lane holds, for column f = 32 fg + lane, bins k = k1 + 16 k2 with
// k1 = 4 Q + T and k2 = 8 h + 4 half + e.
__device__ __forceinline__ void plane_entry_c(int idx4, int e, int& l, int& k) {
    l = idx4 & 31;
    const int i = (idx4 >> 5) & 7, qh = idx4 >> 8;
    const int k1 = 4 * (qh >> 1) + (i >> 1);
    k = k1 + 16 * (8 * (qh & 1) + 4 * (i & 1) + e);
}

// The plane from the complex64 spectrum rows of the circular form: bin k of a
// stored column f <= W/2 sits at f * H + the slot of the register engine's
// position fft_bin_pos(k) (see the circular spectrum build); the columns f >
// W/2 follow from K~[k][f] = conj K~[-k mod H][W - f].
__global__ void k_2dc_plane_tc(const float2* __restrict__ rows, uint4* __restrict__ plane, int64_t nrows,
                               int64_t row_stride) {
    constexpr int per_task = kPlaneTaskC / 4;
    const int64_t per_row = int64_t(CN / NROW) * per_task;
    for (int64_t g = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; g < nrows * per_row;
         g += int64_t(gridDim.x) * blockDim.x) {
        const int64_t r = g / per_row;
        const int rem = int(g - r * per_row);
        const int fg = rem / per_task, idx4 = rem - fg * per_task;
        uint32_t v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            int l, k;
            plane_entry_c(idx4, e, l, k);
            const int f = NROW * fg + l;
            const bool mirror = f > CN / 2;
            const int fs = mirror ? CN - f : f, ks = mirror ? (CN - k) & (CN - 1) : k;
            const int pos = fft_bin_pos<CN>(ks);
            const float2 K = rows[r * row_stride + int64_t(fs) * CN + (pos & 15) * (CN / 16) + (pos >> 4)];
            v[e] = pack_bf16(K.x, mirror ? -K.y : K.y);
        }
        plane[g] = make_uint4(v[0], v[1], v[2], v[3]);
    }
}

// Tables: the real form of the 16-point DFT matrix (B operand) and w256^e.
template <uint32_t OFF_B>
__device__ __forceinline__ void setup_tables_c(uint8_t* smem, float2* w256) {
    float2* w32 = reinterpret_cast<float2*>(smem);
    fill_w32(w32);
    for (int e = threadIdx.x; e < CN; e += NT) {
        float sv, cv;
        sincospif(float(e) * (1.0f / 128.0f), &sv, &cv);   // w256^e = exp(-2 pi i e / 256)
        w256[e] = make_float2(cv, -sv);
    }
    __syncthreads();
    fill_dft<16, 16, 16, kSBOc>(smem + OFF_B, w32);
}

// First operand of a forward transform from the staging Zs[l][n ^ 8 (l >> 3)]
// (32 lines of 256 bf16 pairs): row R(l, n1), chunk c = slots n2 = 4 c .. 4 c + 3.
// Thread (warp w, lane l) takes n1 = ((l + w) & 7) + 8 h: the 32 lanes of a
// gather read 32 banks, and each 8 lanes store 8 rows of one row group.
__device__ __forceinline__ void build_c(uint8_t* A, const uint32_t* Zs, int warp, int lane) {
    const uint32_t* zl = Zs + lane * CN;
    const int sw = 8 * (lane >> 3);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int n1 = ((lane + warp) & 7) + 8 * h;
        const int row = rowc(lane, n1);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            uint32_t q[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) q[e] = zl[(n1 + 16 * (4 * c + e)) ^ sw];
            sts128(A, tc::chunk_off(row, c, kSBOc), q[0], q[1], q[2], q[3]);
        }
    }
}

// Wait for a stage, then the twiddle pass: row R(l, i) (l = lane, i = 4 Q + T in
// tile T), outputs j = 8 h .. 8 h + 7 (columns 16 h ..): value x w256^(i j) ->
// row R(l, j), chunk Q (slots i = 4 Q .. 4 Q + 3).  The table reads are the same
// address for the whole warp.
__device__ __forceinline__ void pass_c(uint8_t* A, const float2* w256, uint32_t tl, int Q, int hh, int lane,
                                       uint64_t* mbar, uint32_t& phase, bool& ok, uint64_t budget) {
    ok = stage_wait(mbar, phase, ok, budget);
    float d[4][16];
#pragma unroll
    for (int T = 0; T < 4; ++T) tc::tmem_ld16(tl + uint32_t(32 * T + 16 * hh), d[T]);
    tc::tmem_ld_wait();
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const int j = 8 * hh + 2 * p;
        C2 v[4];
#pragma unroll
        for (int T = 0; T < 4; ++T) {
            const int i = 4 * Q + T;
            v[T] = cmul2(c2_at(d[T], p), c2_of(w256[(i * j) & (CN - 1)], w256[(i * (j + 1)) & (CN - 1)]));
        }
        sts128(A, tc::chunk_off(rowc(lane, j), Q, kSBOc), pack_bf16(v[0].re.x, v[0].im.x),
               pack_bf16(v[1].re.x, v[1].im.x), pack_bf16(v[2].re.x, v[2].im.x), pack_bf16(v[3].re.x, v[3].im.x));
        sts128(A, tc::chunk_off(rowc(lane, j + 1), Q, kSBOc), pack_bf16(v[0].re.y, v[0].im.y),
               pack_bf16(v[1].re.y, v[1].im.y), pack_bf16(v[2].re.y, v[2].im.y), pack_bf16(v[3].re.y, v[3].im.y));
    }
}

// One DFT16 stage over the four tiles (K 32 -> N 32 each).
__device__ __forceinline__ void issue_c(uint32_t a_addr, uint32_t b_addr, uint32_t tmem, uint64_t* mbar, bool go) {
    stage_issue(a_addr, kSBOc, b_addr, kSBOc, 4, 2, tc::idesc_bf16(128, 32), tmem, 32, mbar, go);
}

__device__ __forceinline__ bool header_c(const uint8_t* spectrum, bool check_plane, int64_t plane_off) {
    const SpecHeader hv = *reinterpret_cast<const SpecHeader*>(spectrum);
    return (hv.magic == kSpecMagic) & (hv.path == PATH_GRID_2D_CIRC) & (hv.H == CN) & (hv.W == CN) &
           (!check_plane | (hv.reserved[1] == plane_off));
}

// Common prologue of the circular kernels: tables (no global memory), then the
// wait for the grids this launch depends on (the kernels are launched with
// programmatic stream serialisation: the tables are built while the previous
// kernel finishes), the header check, barrier and tensor memory.  Returns false
// (status reported) on a header mismatch.
template <uint32_t OFF_B = kOffBc>
__device__ __forceinline__ bool prologue_c(uint8_t* smem, float2* w256, const uint8_t* spectrum, bool check_plane,
                                           int64_t plane_off, uint64_t* mbar, uint32_t* tmem_base,
                                           uint32_t* status) {
    setup_tables_c<OFF_B>(smem, w256);
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const bool hdr_ok = header_c(spectrum, check_plane, plane_off);
    if (!hdr_ok) {
        if (threadIdx.x == 0) report_status(status, kStatusSpectrumMismatch);
        return false;
    }
    if (threadIdx.x == 0) tc::mbar_init(mbar, 1);
    if ((threadIdx.x >> 5) == 0) tc::tmem_alloc(tmem_base, kTmemColsC);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    return true;
}

// GATE: the first order step (z = x_{order-1} v from u); else z from zsrc.
template <bool GATE>
__global__ void __launch_bounds__(NT, 2)
k_2dc_rows_fwd_tc(const bf16* __restrict__ u, const bf16* __restrict__ zsrc, __nv_bfloat162* __restrict__ ws,
                  const uint8_t* __restrict__ spectrum, int64_t B, int64_t C, int order, int64_t pair0, int npairs,
                  int64_t ws_pair_stride, uint64_t wait_budget_ns, int issue_mma, uint32_t* status) {
    extern __shared__ __align__(1024) uint8_t smem_cf[];
    __shared__ __align__(8) uint64_t mbar;
    __shared__ uint32_t tmem_base;
    uint8_t* A = smem_cf;
    uint8_t* Rw = smem_cf + kOffStC;                                 // raw rows: x_b0, x_b1 (, v_b0, v_b1)
    uint32_t* Zs = reinterpret_cast<uint32_t*>(Rw);                  // gated rows (over the raw ones)
    uint32_t* Os = reinterpret_cast<uint32_t*>(smem_cf);             // output staging (the operand area)
    float2* w256 = reinterpret_cast<float2*>(smem_cf + kOffW256F);
    const int t = threadIdx.x;
    const int warp = t >> 5, lane = t & 31;
    const int Q = warp & 3, hh = warp >> 2;
    if (!prologue_c<kOffBcF>(smem_cf, w256, spectrum, false, 0, &mbar, &tmem_base, status)) return;
    const uint32_t tmem = tmem_base;
    const uint32_t tl = tmem + (uint32_t(32 * Q) << 16);
    const uint32_t a_addr = tc::smem_u32(A);
    const uint32_t b_addr = tc::smem_u32(smem_cf + kOffBcF);
    uint32_t phase = 0;
    bool ok = true;
    const int64_t nb2 = B / 2, Ctot = int64_t(order + 1) * C, n_img = int64_t(CN) * CN;
    const int ntasks = npairs * (CN / NROW);
    // a task's raw rows (each plane 16 KB contiguous) into Rw by cp.async: the next
    // task's are copied while this one is transformed
    constexpr int kPlanes = GATE ? 4 : 2;
    auto stage_raw = [&](int task) {
        const int lp = task / (CN / NROW), rg = task - lp * (CN / NROW);
        const int64_t pr = pair0 + lp, c = pr / nb2, b0 = 2 * (pr - c * nb2);
        const int64_t rowoff = int64_t(NROW * rg) * CN;
        const bf16* x0 = GATE ? u + (b0 * Ctot + int64_t(order - 1) * C + c) * n_img + rowoff
                              : zsrc + (b0 * C + c) * n_img + rowoff;
        const int64_t xs = GATE ? Ctot * n_img : C * n_img;                  // image b0 -> b0 + 1
        const bf16* v0 = u + (b0 * Ctot + int64_t(order) * C + c) * n_img + rowoff;
#pragma unroll
        for (int pl = 0; pl < kPlanes; ++pl) {
            const bf16* src = (pl < 2 ? x0 : v0) + (pl & 1) * xs;
#pragma unroll
            for (int kk = 0; kk < int(kRawPlane / 16) / NT; ++kk) {
                const int gi = t + NT * kk;
                cp_async_bytes16(Rw + pl * kRawPlane + 16 * gi, reinterpret_cast<const uint4*>(src) + gi);
            }
        }
        cp_async_commit();
    };
    if (int(blockIdx.x) < ntasks) stage_raw(blockIdx.x);

    for (int task = blockIdx.x; task < ntasks; task += gridDim.x) {
        const int lp = task / (CN / NROW), rg = task - lp * (CN / NROW);
        cp_async_wait_all();
        __syncthreads();
        {
            // this thread's raw values into registers, then (every thread done reading) the
            // gated rows over them
            PairRows<GATE> in;
#pragma unroll
            for (int jj = 0; jj < kRowIt; ++jj) {
                const int ci = t + NT * jj;                 // 16-byte group ci of a plane
#pragma unroll
                for (int im = 0; im < 2; ++im) {
                    in.x[jj][im] = *reinterpret_cast<const uint4*>(Rw + im * kRawPlane + 16 * ci);
                    if constexpr (GATE) in.v[jj][im] = *reinterpret_cast<const uint4*>(Rw + (2 + im) * kRawPlane + 16 * ci);
                }
            }
            __syncthreads();
            store_pair_rows<GATE>(Zs, in, t);
        }
        __syncthreads();
        build_c(A, Zs, warp, lane);
        issue_c(a_addr, b_addr, tmem, &mbar, ok && issue_mma);   // every thread is past its build: Rw is free
        if (task + int(gridDim.x) < ntasks) stage_raw(task + int(gridDim.x));
        pass_c(A, w256, tl, Q, hh, lane, &mbar, phase, ok, wait_budget_ns);
        issue_c(a_addr, b_addr, tmem, &mbar, ok && issue_mma);
        ok = stage_wait(&mbar, phase, ok, wait_budget_ns);
        // rows R(r, k1 = 4 Q + T), bins k2 = 8 h + ..: staging Os[k][r] (a warp's 32
        // lanes are 32 consecutive words), then 128-byte rows Z[k][32 rg .. 32 rg + 31]
#pragma unroll
        for (int T = 0; T < 4; ++T) {
            float d[16];
            tc::tmem_ld16(tl + uint32_t(32 * T + 16 * hh), d);
            tc::tmem_ld_wait();
            const int k1 = 4 * Q + T;
#pragma unroll
            for (int p = 0; p < 4; ++p)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int k = k1 + 16 * (8 * hh + 2 * p + e);
                    Os[k * NROW + lane] = ok ? pack_bf16(d[4 * p + e], d[4 * p + 2 + e]) : 0x7fc07fc0u;
                }
        }
        tc::fence_before_sync();
        __syncthreads();
        uint32_t* wsp = reinterpret_cast<uint32_t*>(ws + int64_t(lp) * ws_pair_stride) + NROW * rg;
#pragma unroll 4
        for (int kk = 0; kk < CN * NROW / 4 / NT; ++kk) {
            const int gi = t + NT * kk, k = gi >> 3, g4 = gi & 7;
            *reinterpret_cast<uint4*>(wsp + int64_t(k) * CN + 4 * g4) =
                *reinterpret_cast<const uint4*>(Os + k * NROW + 4 * g4);
        }
        if (__syncthreads_or(!ok)) {
            if (t == 0) report_status(status, kStatusTimeout);
            break;
        }
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");   // the next kernel may start its setup
    cp_async_wait_all();   // no copy into this CTA's shared memory outlives it
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, kTmemColsC);
}

__global__ void __launch_bounds__(NT, 2)
k_2dc_cols_tc(__nv_bfloat162* __restrict__ ws, const uint8_t* __restrict__ spectrum, int64_t nb2, int step,
              int64_t pair0, int npairs, int64_t ws_pair_stride, int64_t plane_off, int64_t SC,
              uint64_t wait_budget_ns, int issue_mma, uint32_t* status) {
    extern __shared__ __align__(1024) uint8_t smem_cc[];
    __shared__ __align__(8) uint64_t mbar;
    __shared__ uint32_t tmem_base;
    uint8_t* A = smem_cc;
    uint32_t* Zs = reinterpret_cast<uint32_t*>(smem_cc + kOffStC);   // input columns
    uint32_t* Vs = reinterpret_cast<uint32_t*>(smem_cc);             // output staging (the operand area)
    float2* w256 = reinterpret_cast<float2*>(smem_cc + kOffW256);
    const int t = threadIdx.x;
    const int warp = t >> 5, lane = t & 31;
    const int Q = warp & 3, hh = warp >> 2;
    if (!prologue_c(smem_cc, w256, spectrum, true, plane_off, &mbar, &tmem_base, status)) return;
    const uint32_t tmem = tmem_base;
    const uint32_t tl = tmem + (uint32_t(32 * Q) << 16);
    const uint32_t a_addr = tc::smem_u32(A);
    const uint32_t b_addr = tc::smem_u32(smem_cc + kOffBc);
    const uint4* plane = reinterpret_cast<const uint4*>(spectrum + plane_off);
    uint32_t phase = 0;
    bool ok = true;
    const int ntasks = npairs * (CN / NROW);

    // a task's 32 columns (contiguous in the workspace) -> Zs[l][m ^ 8 (l >> 3)] by
    // cp.async: the next task's are copied while this one is transformed
    auto stage_cols = [&](int task) {
        const int lp = task / (CN / NROW), fg = task - lp * (CN / NROW);
        const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const uint32_t*>(
                                                              ws + int64_t(lp) * ws_pair_stride) +
                                                          int64_t(NROW * fg) * CN);
#pragma unroll
        for (int kk = 0; kk < NROW * CN / 4 / NT; ++kk) {
            const int gi = t + NT * kk, l = gi >> 6, m0 = 4 * (gi & 63);
            cp_async_bytes16(Zs + l * CN + (m0 ^ (8 * (l >> 3))), src + gi);
        }
        cp_async_commit();
    };
    if (int(blockIdx.x) < ntasks) stage_cols(blockIdx.x);

    for (int task = blockIdx.x; task < ntasks; task += gridDim.x) {
        const int lp = task / (CN / NROW), fg = task - lp * (CN / NROW);
        const int64_t c = (pair0 + lp) / nb2;
        uint32_t* col0 = reinterpret_cast<uint32_t*>(ws + int64_t(lp) * ws_pair_stride) + int64_t(NROW * fg) * CN;
        const uint4* kq = plane + ((int64_t(step) * SC + c) * (CN / NROW) + fg) * (kPlaneTaskC / 4) +
                          (Q * 2 + hh) * 256 + lane;
        cp_async_wait_all();
        __syncthreads();
        build_c(A, Zs, warp, lane);
        issue_c(a_addr, b_addr, tmem, &mbar, ok && issue_mma);   // every thread is past its build: Zs is free
        if (task + int(gridDim.x) < ntasks) stage_cols(task + int(gridDim.x));
        pass_c(A, w256, tl, Q, hh, lane, &mbar, phase, ok, wait_budget_ns);
        issue_c(a_addr, b_addr, tmem, &mbar, ok && issue_mma);
        {
            // rows R(l, k1 = 4 Q + T), bins k2 = 8 h + 4 half + e: conj(X K~) to the same
            // row, chunk 2 h + half (the operand of the inverse stage over k2)
            uint4 kv[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) kv[i] = __ldg(kq + 32 * i);
            ok = stage_wait(&mbar, phase, ok, wait_budget_ns);
#pragma unroll
            for (int T = 0; T < 4; ++T) {
                float d[16];
                tc::tmem_ld16(tl + uint32_t(32 * T + 16 * hh), d);
                tc::tmem_ld_wait();
                const int row = rowc(lane, 4 * Q + T);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const uint4 kk = kv[2 * T + half];
                    const C2 K0{make_float2(bf_lo(kk.x), bf_lo(kk.y)), make_float2(bf_hi(kk.x), bf_hi(kk.y))};
                    const C2 K1{make_float2(bf_lo(kk.z), bf_lo(kk.w)), make_float2(bf_hi(kk.z), bf_hi(kk.w))};
                    const C2 v0 = cmul2(c2_at(d, 2 * half), K0);
                    const C2 v1 = cmul2(c2_at(d, 2 * half + 1), K1);
                    sts128(A, tc::chunk_off(row, 2 * hh + half, kSBOc), pack_bf16(v0.re.x, -v0.im.x),
                           pack_bf16(v0.re.y, -v0.im.y), pack_bf16(v1.re.x, -v1.im.x), pack_bf16(v1.re.y, -v1.im.y));
                }
            }
        }
        issue_c(a_addr, b_addr, tmem, &mbar, ok && issue_mma);
        pass_c(A, w256, tl, Q, hh, lane, &mbar, phase, ok, wait_budget_ns);
        issue_c(a_addr, b_addr, tmem, &mbar, ok && issue_mma);
        ok = stage_wait(&mbar, phase, ok, wait_budget_ns);
        // conj of the result at row R(l, n1 = 4 Q + T), output n2: word m = n1 + 16 n2 of
        // line l at Vs[l][m ^ l] (32 banks for the 32 lanes), then the 32 columns back
#pragma unroll
        for (int T = 0; T < 4; ++T) {
            float d[16];
            tc::tmem_ld16(tl + uint32_t(32 * T + 16 * hh), d);
            tc::tmem_ld_wait();
            const int n1 = 4 * Q + T;
#pragma unroll
            for (int p = 0; p < 4; ++p)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int m = n1 + 16 * (8 * hh + 2 * p + e);
                    Vs[lane * CN + (m ^ lane)] = ok ? pack_bf16(d[4 * p + e], -d[4 * p + 2 + e]) : 0x7fc07fc0u;
                }
        }
        tc::fence_before_sync();
        __syncthreads();
        {
            // 16-byte group g of line l is group g ^ (l >> 2) with its words permuted by l & 3
            uint4* dst = reinterpret_cast<uint4*>(col0);
#pragma unroll
            for (int kk = 0; kk < NROW * CN / 4 / NT; ++kk) {
                const int gi = t + NT * kk, l = gi >> 6, g = gi & 63;
                uint4 v = *reinterpret_cast<const uint4*>(Vs + l * CN + 4 * (g ^ (l >> 2)));
                if (l & 1) v = make_uint4(v.y, v.x, v.w, v.z);
                if (l & 2) v = make_uint4(v.z, v.w, v.x, v.y);
                dst[gi] = v;
            }
        }
        if (__syncthreads_or(!ok)) {
            if (t == 0) report_status(status, kStatusTimeout);
            break;
        }
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");   // the next kernel may start its setup
    cp_async_wait_all();   // no copy into this CTA's shared memory outlives it
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, kTmemColsC);
}

__global__ void __launch_bounds__(NT, 2)
k_2dc_rows_inv_tc(const bf16* __restrict__ u, bf16* __restrict__ y, const __nv_bfloat162* __restrict__ ws,
                  const uint8_t* __restrict__ spectrum, int64_t B, int64_t C, int order, int gchunk, int64_t pair0,
                  int npairs, int64_t ws_pair_stride, uint64_t wait_budget_ns, int issue_mma, uint32_t* status) {
    extern __shared__ __align__(1024) uint8_t smem_ci[];
    __shared__ __align__(8) uint64_t mbar;
    __shared__ uint32_t tmem_base;
    uint8_t* A = smem_ci;
    uint32_t* Ws = reinterpret_cast<uint32_t*>(smem_ci + kOffStC);   // the task's Y[k][32 rows]
    uint32_t* Ys = reinterpret_cast<uint32_t*>(smem_ci);             // output staging [r][n ^ r] (operand area)
    float2* w256 = reinterpret_cast<float2*>(smem_ci + kOffW256);
    const int t = threadIdx.x;
    const int warp = t >> 5, lane = t & 31;
    const int Q = warp & 3, hh = warp >> 2;
    if (!prologue_c(smem_ci, w256, spectrum, false, 0, &mbar, &tmem_base, status)) return;
    const uint32_t tmem = tmem_base;
    const uint32_t tl = tmem + (uint32_t(32 * Q) << 16);
    const uint32_t a_addr = tc::smem_u32(A);
    const uint32_t b_addr = tc::smem_u32(smem_ci + kOffBc);
    uint32_t phase = 0;
    bool ok = true;
    const int64_t nb2 = B / 2, Ctot = int64_t(order + 1) * C, n_img = int64_t(CN) * CN;
    const int ntasks = npairs * (CN / NROW);

    // a task's Y[k][32 rg .. 32 rg + 31] (256 rows of 128 bytes in the workspace) ->
    // Ws[k][r] by cp.async: the next task's are copied while this one is transformed
    auto stage_rows = [&](int task) {
        const int lp = task / (CN / NROW), rg = task - lp * (CN / NROW);
        const uint32_t* wsp = reinterpret_cast<const uint32_t*>(ws + int64_t(lp) * ws_pair_stride) + NROW * rg;
#pragma unroll
        for (int kk = 0; kk < CN * NROW / 4 / NT; ++kk) {
            const int gi = t + NT * kk, k = gi >> 3, g4 = gi & 7;
            cp_async_bytes16(Ws + k * NROW + 4 * g4, wsp + int64_t(k) * CN + 4 * g4);
        }
        cp_async_commit();
    };
    if (int(blockIdx.x) < ntasks) stage_rows(blockIdx.x);

    for (int task = blockIdx.x; task < ntasks; task += gridDim.x) {
        const int lp = task / (CN / NROW), rg = task - lp * (CN / NROW);
        const int64_t pr = pair0 + lp, c = pr / nb2, b0 = 2 * (pr - c * nb2);
        cp_async_wait_all();
        __syncthreads();
        {
            // conj Y[k1 + 16 k2][r] at row R(r, k1), chunk k2 / 4; lane = r (a warp reads
            // 32 consecutive words)
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const int ci = warp + 8 * m, k1 = ci & 15, ch = ci >> 4;
                uint32_t q[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) q[e] = Ws[(k1 + 16 * (4 * ch + e)) * NROW + lane] ^ 0x80000000u;
                sts128(A, tc::chunk_off(rowc(lane, k1), ch, kSBOc), q[0], q[1], q[2], q[3]);
            }
        }
        issue_c(a_addr, b_addr, tmem, &mbar, ok && issue_mma);   // every thread is past its build: Ws is free
        if (task + int(gridDim.x) < ntasks) stage_rows(task + int(gridDim.x));
        pass_c(A, w256, tl, Q, hh, lane, &mbar, phase, ok, wait_budget_ns);
        issue_c(a_addr, b_addr, tmem, &mbar, ok && issue_mma);
        // the gate rows (x_gchunk of both images) are on their way while the last stage runs
        const int64_t rowoff = int64_t(NROW * rg) * CN;
        const bf16* xa = u + (b0 * Ctot + int64_t(gchunk) * C + c) * n_img + rowoff;
        uint4 gx[kRowIt][2];
        load_gate_rows(gx, xa, xa + Ctot * n_img, t);
        ok = stage_wait(&mbar, phase, ok, wait_budget_ns);
        // 2 conj(D) at row R(r, n1 = 4 Q + T), output n2: (image b0, image b1) of row r,
        // column n = n1 + 16 n2 -> Ys[r][n ^ r]
#pragma unroll
        for (int T = 0; T < 4; ++T) {
            float d[16];
            tc::tmem_ld16(tl + uint32_t(32 * T + 16 * hh), d);
            tc::tmem_ld_wait();
            const int n1 = 4 * Q + T;
#pragma unroll
            for (int p = 0; p < 4; ++p)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int n = n1 + 16 * (8 * hh + 2 * p + e);
                    Ys[lane * CN + (n ^ lane)] = pack_bf16(2.0f * d[4 * p + e], -2.0f * d[4 * p + 2 + e]);
                }
        }
        tc::fence_before_sync();
        __syncthreads();
        {
            bf16* ya = y + (b0 * C + c) * n_img + rowoff;
            apply_gate_rows(Ys, gx, ya, ya + C * n_img, t, ok);
        }
        if (__syncthreads_or(!ok)) {
            if (t == 0) report_status(status, kStatusTimeout);
            break;
        }
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");   // the next kernel may start its setup
    cp_async_wait_all();   // no copy into this CTA's shared memory outlives it
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, kTmemColsC);
}

}  // namespace

// Orders above kMaxOrderTc keep the fp32 passes, as in 1-D: every order step
// adds the bf16 roundings of its stage operands (image error ~6e-3, 1e-2 and
// 1.4e-2 at orders 2, 3 and 4 with the paired passes).
bool cols_2d_tc_path(const Plan& p, const ConvArgs& a) {
    return p.path == PATH_GRID_2D && p.H == kTc2dH && p.W % NCOL == 0 && a.g2_plane_off != 0 &&
           a.dtype == DT_BF16 && !a.fp32_transform && p.order <= kMaxOrderTc;
}

cudaError_t launch_spectrum_2d_tc_plane(const Plan& p, const uint8_t* spectrum_rows, uint8_t* plane, int64_t nrows,
                                        cudaStream_t s) {
    const int64_t n = nrows * int64_t(2 * p.W / NCOL) * (kPlaneTask / 4);
    int64_t blocks = (n + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    k_2d_plane_tc<<<unsigned(blocks), 256, 0, s>>>(reinterpret_cast<const float2*>(spectrum_rows),
                                                   reinterpret_cast<uint4*>(plane), nrows, int(p.W),
                                                   int64_t(p.spec_row_bytes / sizeof(float2)));
    return cudaGetLastError();
}

cudaError_t launch_cols_2d_tc(const Plan& p, const ConvArgs& a, void* ws, int64_t img0, int64_t nimg, int step,
                              int64_t ws_img_stride, cudaStream_t s) {
    auto kern = k_2d_cols_tc;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmem));
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t ntasks = nimg * (p.W / NCOL);
    if (ntasks > INT32_MAX || nimg > INT32_MAX) return cudaErrorInvalidValue;
    int64_t grid = int64_t(2) * sms;
    if (grid > ntasks) grid = ntasks;
    kern<<<unsigned(grid), NT, kSmem, s>>>(static_cast<__nv_bfloat162*>(ws), a.spectrum, int(p.C), int(p.W), a.B, step,
                                           img0, int(nimg), ws_img_stride, int64_t(a.g2_plane_off), a.spec_C,
                                           a.spec_per_b, int(p.W), a.wait_budget_ns, a.issue_mma, a.status);
    return cudaGetLastError();
}

bool pairs_2d_tc_path(const Plan& p, const ConvArgs& a) {
    return cols_2d_tc_path(p, a) && p.W == W2 && a.B % 2 == 0 && a.spec_per_b == 0;
}

cudaError_t launch_conv_2d_pairs_tc(const Plan& p, const ConvArgs& a, void* ws, int64_t img0, int64_t nimg,
                                    int64_t ws_img_stride, cudaStream_t s) {
    if (img0 % 2 != 0 || nimg % 2 != 0) return cudaErrorInvalidValue;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t npairs = nimg / 2, pair0 = img0 / 2, pstride = 2 * ws_img_stride;
    const int64_t ntasks = npairs * (MH / NROW);
    if (ntasks > INT32_MAX || npairs * (2 * W2 / NCOL) > INT32_MAX) return cudaErrorInvalidValue;
    const unsigned grid = unsigned(ntasks < 2 * sms ? ntasks : 2 * sms);
    const bf16* u = static_cast<const bf16*>(a.u);
    __nv_bfloat162* w = static_cast<__nv_bfloat162*>(ws);
    cudaError_t e = cudaFuncSetAttribute(k_2d_rows_fwd_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmem));
    if (e == cudaSuccess) e = cudaFuncSetAttribute(k_2d_cols_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmem));
    if (e == cudaSuccess) e = cudaFuncSetAttribute(k_2d_rows_inv_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmem));
    if (e != cudaSuccess) return e;
    bf16* y = static_cast<bf16*>(a.y);
    const int64_t ctasks = npairs * (2 * W2 / NCOL);
    // programmatic stream serialisation, as for the circular passes
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    auto cfg = [&](unsigned g) {
        cudaLaunchConfig_t c = {};
        c.gridDim = dim3(g);
        c.blockDim = dim3(NT);
        c.dynamicSmemBytes = kSmem;
        c.stream = s;
        c.attrs = pdl;
        c.numAttrs = 1;
        return c;
    };
    const cudaLaunchConfig_t cr = cfg(grid), ccl = cfg(unsigned(ctasks < 2 * sms ? ctasks : 2 * sms));
    for (int st = 1; st < p.order && e == cudaSuccess; ++st) {
        // step st gates with x_{order-st}: the first step's input is x_{order-1} v, a later
        // step's is x_{order-st} times the previous step's result, which that step's
        // inverse pass left in y; the last inverse pass applies x0
        e = cudaLaunchKernelEx(&cr, k_2d_rows_fwd_tc, u, st == 1 ? static_cast<const bf16*>(nullptr) : y, w,
                               a.spectrum, a.B, p.C, p.order, pair0, int(npairs), pstride, a.wait_budget_ns,
                               a.issue_mma, a.status);
        // every bin column of a pair (2W), spectrum row (st - 1) C + c, c = pair / (B/2)
        if (e == cudaSuccess)
            e = cudaLaunchKernelEx(&ccl, k_2d_cols_tc, w, a.spectrum, int(p.C), 2 * W2, a.B / 2, st - 1, pair0,
                                   int(npairs), pstride, int64_t(a.g2_plane_off), a.spec_C, int64_t(0), W2,
                                   a.wait_budget_ns, a.issue_mma, a.status);
        if (e == cudaSuccess)
            e = cudaLaunchKernelEx(&cr, k_2d_rows_inv_tc, u, y, static_cast<const __nv_bfloat162*>(w), a.spectrum,
                                   a.B, p.C, p.order, st == p.order - 1 ? 0 : p.order - st - 1, pair0, int(npairs),
                                   pstride, a.wait_budget_ns, a.issue_mma, a.status);
    }
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}


bool pairs_2dc_tc_path(const Plan& p, const ConvArgs& a) {
    return p.path == PATH_GRID_2D_CIRC && p.H == CN && p.W == CN && a.g2_plane_off != 0 && a.dtype == DT_BF16 &&
           !a.fp32_transform && p.order <= kMaxOrderTc && a.B % 2 == 0 && a.spec_per_b == 0;
}

cudaError_t launch_spectrum_2dc_tc_plane(const Plan& p, const uint8_t* spectrum_rows, uint8_t* plane, int64_t nrows,
                                         cudaStream_t s) {
    const int64_t n = nrows * int64_t(CN / NROW) * (kPlaneTaskC / 4);
    int64_t blocks = (n + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    k_2dc_plane_tc<<<unsigned(blocks), 256, 0, s>>>(reinterpret_cast<const float2*>(spectrum_rows),
                                                    reinterpret_cast<uint4*>(plane), nrows,
                                                    int64_t(p.spec_row_bytes / sizeof(float2)));
    return cudaGetLastError();
}

cudaError_t launch_conv_2dc_pairs_tc(const Plan& p, const ConvArgs& a, void* ws, int64_t img0, int64_t nimg,
                                     int64_t ws_img_stride, cudaStream_t s) {
    if (img0 % 2 != 0 || nimg % 2 != 0) return cudaErrorInvalidValue;
    if (2 * ws_img_stride < int64_t(CN) * CN) return cudaErrorInvalidValue;   // a pair's Z[k][row]
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t npairs = nimg / 2, pair0 = img0 / 2, pstride = 2 * ws_img_stride;
    const int64_t ntasks = npairs * (CN / NROW);
    if (ntasks > INT32_MAX) return cudaErrorInvalidValue;
    const unsigned grid = unsigned(ntasks < 2 * sms ? ntasks : 2 * sms);
    cudaError_t e = cudaFuncSetAttribute(k_2dc_rows_fwd_tc<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmemCF));
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k_2dc_rows_fwd_tc<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmemCF));
    if (e == cudaSuccess) e = cudaFuncSetAttribute(k_2dc_cols_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmemC));
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k_2dc_rows_inv_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmemC));
    if (e != cudaSuccess) return e;
    const bf16* u = static_cast<const bf16*>(a.u);
    bf16* y = static_cast<bf16*>(a.y);
    __nv_bfloat162* w = static_cast<__nv_bfloat162*>(ws);
    // programmatic stream serialisation: each kernel sets up its tables while the one
    // before it finishes, and waits for it (griddepcontrol.wait) before its first read
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    auto cfg = [&](size_t smem) {
        cudaLaunchConfig_t c = {};
        c.gridDim = dim3(grid);
        c.blockDim = dim3(NT);
        c.dynamicSmemBytes = smem;
        c.stream = s;
        c.attrs = pdl;
        c.numAttrs = 1;
        return c;
    };
    const cudaLaunchConfig_t cf = cfg(kSmemCF), cc = cfg(kSmemC);
    for (int st = 1; st < p.order && e == cudaSuccess; ++st) {
        // as for the padded pairs: step st gates with x_{order-st}; a later step reads
        // its input from y, where the previous step's inverse pass left it
        e = cudaLaunchKernelEx(&cf, st == 1 ? k_2dc_rows_fwd_tc<true> : k_2dc_rows_fwd_tc<false>, u,
                               static_cast<const bf16*>(y), w, a.spectrum, a.B, p.C, p.order, pair0, int(npairs),
                               pstride, a.wait_budget_ns, a.issue_mma, a.status);
        if (e == cudaSuccess)
            e = cudaLaunchKernelEx(&cc, k_2dc_cols_tc, w, a.spectrum, a.B / 2, st - 1, pair0, int(npairs), pstride,
                                   int64_t(a.g2_plane_off), a.spec_C, a.wait_budget_ns, a.issue_mma, a.status);
        if (e == cudaSuccess)
            e = cudaLaunchKernelEx(&cc, k_2dc_rows_inv_tc, u, y, static_cast<const __nv_bfloat162*>(w), a.spectrum,
                                   a.B, p.C, p.order, st == p.order - 1 ? 0 : p.order - st - 1, pair0, int(npairs),
                                   pstride, a.wait_budget_ns, a.issue_mma, a.status);
    }
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace hyena
