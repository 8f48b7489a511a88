// plan.h -- host-side planning for the Hyena gated FFT long convolution.
//
// A plan is a pure function of (C, ndim, sizes, order).  It fixes the kernel
// path, the FFT factorisations, and the byte layout of the caller-owned
// spectrum buffer:
//
//   [0, 256)               SpecHeader (magic, shape, layout offsets)
//   [256, spec_off)        twiddle tables (float2, double-precision values
//                          rounded to fp32), described by TableSpec entries
//   [spec_off, total)      filter spectra, [order-1][C] rows of spec_row_bytes
//
// Paths (N = 2L zero-padded transform, computed as two M = L/2-point chains):
//   PATH_ONCHIP_1D    16 <= L <= 16384: one CTA per (b, c) row, everything in
//                     shared memory.  Spectrum row = (M+1) float4 pair entries;
//                     L = 8192: all 2L bins, complex64, in the position
//                     order of the tensor-core kernel (onchip_tc.cu).
//   PATH_MULTIPASS_1D 32768 <= L <= 2^20: four-step M = M1 x M2 with three
//                     passes through a caller workspace (rows processed in
//                     groups that fit it; by default the whole batch up to
//                     4 GiB).  Spectrum row = M1 units of M2 float4 pair
//                     entries.  L = 65536 adds, after the rows, the cluster
//                     plane (cluster.cu): per (step, c) all 2L bins of K~ as
//                     bf16 (re, im), eight sub-planes of 16384 in the
//                     tensor-core kernel's position order (header
//                     reserved[0] holds its offset).
//   PATH_GRID_2D      2-D H x W (16..512 each), zero-padded to 2H x 2W: a row
//                     pass (packed real FFT of each image row), a column pass
//                     (2H-point FFT, spectrum multiply, inverse) and an
//                     inverse row pass.  Spectrum per channel = (W+1) columns
//                     x 2H complex64 in the column pass's position order.
//   PATH_GRID_2D_CIRC 2-D circular (ndim = 2 | kCircularFlag): no padding, the
//                     W-point row FFT (packed, one W/2-point chain) and the
//                     H-point column FFT.  Spectrum per channel = (W/2+1)
//                     columns x H complex64.
//   PATH_GRID_3D      3-D N1 x H x W (16..128 each), zero padded on every
//                     axis: the 2-D row passes over N1 H rows, a forward and
//                     an inverse column pass (2H points) and a depth pass
//                     (2N1 points, spectrum multiply) between them.  Spectrum
//                     per channel = (W+1) 2H depth lines x 2N1 complex64.
//                     N1 is kept in the L field.
#pragma once
#include <stddef.h>
#include <stdint.h>

#include <string>

namespace hyena {

enum Path {
    PATH_NONE = 0, PATH_ONCHIP_1D = 1, PATH_MULTIPASS_1D = 2, PATH_GRID_2D = 3, PATH_GRID_2D_CIRC = 4, PATH_GRID_3D = 5
};

// OR-ed into ndim (2-D only): the circular (periodic) form (HYENA_CIRCULAR).
constexpr int kCircularFlag = 0x100;

constexpr uint32_t kSpecMagic = 0x4853504Eu;  // "NPSH"
constexpr uint32_t kSpecVersion = 2;
constexpr size_t kHeaderBytes = 256;
constexpr int kMaxTableSpecs = 24;

constexpr int64_t kOnchipMaxL = 16384;
// L served by the cluster kernel (bf16 storage): 2L = kClusterR x 16384
constexpr int64_t kClusterL = 65536;
constexpr int kClusterR = 8;
// 2-D column length served by the tensor-core column pass (bf16 storage): a
// 2H = 512-point transform per column, 32 columns per 16384-point task
constexpr int64_t kTc2dH = 256;
constexpr int64_t kMaxL = int64_t(1) << 20;
constexpr int64_t kMin1D = 16;
constexpr int64_t kMin2D = 16;
constexpr int64_t kMax2D = 512;
constexpr int64_t kMin3D = 16;
constexpr int64_t kMax3D = 128;
constexpr int kMaxOrder = 8;

struct SpecHeader {
    uint32_t magic, version;
    int32_t ndim, order, path, reserved0;
    int64_t C, L, H, W, M, M1, M2;
    int64_t tables_off, tables_count, spec_off, spec_row_bytes, total_bytes;
    uint32_t reserved1, reserved2;
    int64_t reserved[16];
};
static_assert(sizeof(SpecHeader) == kHeaderBytes, "header must be 256 bytes");

// entry[i][j] (i < na, j < nb) = w_N^(((a0 + i) (b0 + j) mult + add) mod N),
// w_N = exp(-2 pi i / N), stored at tables[dst + i * nb + j].
struct TableSpec {
    int64_t dst, N, a0, na, b0, nb, mult, add;
};
struct TableSpecs {
    TableSpec s[kMaxTableSpecs];
    int n;
    int64_t total;
};

struct Plan {
    int ndim = 0, order = 0, path = PATH_NONE;
    int64_t C = 0, L = 0, H = 0, W = 0;
    int64_t M = 0, M1 = 0, M2 = 0;   // chain size; multi-pass factors; 2-D: M1 = W/2, M2 = H
    int64_t n = 0;                   // samples per row (L or H*W)
    // table offsets in float2 units from the start of the tables
    int64_t t_fft_a = 0, t_fft_b = 0, t_twist = 0, t_untangle = 0, t_four = 0;
    int64_t t_twist_hi = 0, t_twist_lo = 0, t_unt1 = 0, t_unt2 = 0, t_unt_c = 0, t_twist_h = 0;
    int64_t t_fft_d = 0, t_twist_d = 0;   // 3-D depth axis
    // L = kClusterL: CTA FFT of 16384 points, w_2L^a (a < 16384), and the
    // even / odd powers w_16384^(2j), w_16384^(2j+1) (j < 2048)
    int64_t t_cl_fft = 0, t_cl_wa = 0, t_cl_even = 0, t_cl_odd = 0;
    size_t cl_plane_off = 0;               // 0: no cluster plane
    // 2-D form with H = 256 and W a multiple of 32: the tensor-core passes'
    // spectrum plane (bf16 (re, im), per filter 2W/32 blocks of 32 columns
    // x 512 bins of the 2H x 2W transform, in the column kernel's thread
    // order); 0: none
    size_t g2_plane_off = 0;
    TableSpecs specs{};
    size_t tables_off = kHeaderBytes;
    size_t spec_off = 0;
    size_t spec_row_bytes = 0;
    size_t total_bytes = 0;
    // workspace (multi-pass and 2-D): bytes per (b, c) row in flight
    size_t ws_row_bytes = 0;
};

// Returns false (and a reason) for unsupported shapes / orders.
bool make_plan(int64_t C, int ndim, const int64_t* sizes, int order, Plan* p, std::string* why);

// Default number of rows processed per group on the workspace paths.
int64_t default_group_rows(const Plan& p, int64_t rows);

}  // namespace hyena
