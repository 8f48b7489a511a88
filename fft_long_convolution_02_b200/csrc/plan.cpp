// plan.cpp -- see plan.h.
#include "plan.h"

#include "plan_common.h"

namespace hyena {

namespace {

bool is_pow2(int64_t x) { return x > 0 && (x & (x - 1)) == 0; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct TableBuilder {
    TableSpecs* specs;
    int64_t cursor = 0;
    bool ok = true;

    int64_t add(int64_t N, int64_t a0, int64_t na, int64_t b0, int64_t nb, int64_t mult = 1,
                int64_t addc = 0) {
        int64_t at = cursor;
        if (na * nb == 0) return at;
        if (specs->n >= kMaxTableSpecs) { ok = false; return at; }
        specs->s[specs->n++] = TableSpec{at, N, a0, na, b0, nb, mult, addc};
        cursor += na * nb;
        return at;
    }
    // Per-stage twiddles of an M-point CTA FFT: stage i, entry (s'-1)*P + p = w_len^(p s').
    int64_t add_fft(int M) {
        int64_t at = cursor;
        for (int i = 0; i < fft_nstages(M); ++i) {
            const int R = fft_stage_radix(M, i), P = fft_stage_stride(M, i);
            if (P > 1) add(fft_stage_len(M, i), 1, R - 1, 0, P);
        }
        return at;
    }
    // Pair twiddles w_2Lp^f of the packed-real untangle for a length-Lp real
    // axis (chain size Mp = Lp/2): chain e pairs j = 0..Mp/2 use f = 2j,
    // chain o pairs j = 0..Mp/2-1 use f = 2j+1.
    int64_t add_untangle(int64_t Lp) {
        int64_t at = cursor;
        const int64_t Mp = Lp / 2;
        add(Lp, 0, Mp / 2 + 1, 1, 1);            // w_Lp^j = w_2Lp^(2j)
        add(2 * Lp, 0, Mp / 2, 2, 1, 1, 1);      // w_2Lp^(2j+1)
        return at;
    }
};

}  // namespace

bool make_plan(int64_t C, int ndim, const int64_t* sizes, int order, Plan* p, std::string* why) {
    *p = Plan{};
    if (C < 1) { *why = "C must be >= 1"; return false; }
    if (order < 2 || order > kMaxOrder) { *why = "order must be in [2, 8]"; return false; }
    if (!sizes) { *why = "sizes is NULL"; return false; }
    const bool circular = (ndim & kCircularFlag) != 0;
    ndim &= ~kCircularFlag;
    if (circular && ndim != 2) { *why = "the circular form is 2-D only"; return false; }
    p->C = C;
    p->ndim = ndim;
    p->order = order;
    TableBuilder tb{&p->specs};
    const int64_t S = order - 1;
    if (ndim == 1) {
        const int64_t L = sizes[0];
        if (!is_pow2(L) || L < kMin1D || L > kMaxL) {
            *why = "1-D length must be a power of two in [16, 2^20]";
            return false;
        }
        p->L = L;
        p->H = 1;
        p->W = L;
        p->n = L;
        p->M = L / 2;
        if (L <= kOnchipMaxL) {
            p->path = PATH_ONCHIP_1D;
            p->t_fft_a = tb.add_fft(int(p->M));
            p->t_twist = tb.add(L, 0, p->M, 1, 1);                  // w_L^n, n < M
            p->t_untangle = tb.add_untangle(L);
            // L = 8192: all 2L bins of the zero-padded transform (complex64, in
            // the position order of its tensor-core kernel); other lengths the
            // pair layout ((M+1) float4 entries)
            p->spec_row_bytes = (L == 8192) ? size_t(16 * L) : size_t(p->M + 1) * 16;
        } else {
            p->path = PATH_MULTIPASS_1D;
            p->M1 = (p->M >= (int64_t(1) << 16)) ? 256 : 128;
            p->M2 = p->M / p->M1;
            p->t_fft_a = tb.add_fft(int(p->M1));
            p->t_fft_b = tb.add_fft(int(p->M2));
            p->t_four = tb.add(p->M, 0, p->M1, 0, p->M2);             // w_M^(m1 n2), [m1][n2]
            p->t_twist_hi = tb.add(L, 0, p->M1, p->M2, 1);            // w_L^(M2 n1)
            p->t_twist_lo = tb.add(L, 0, p->M2, 1, 1);                // w_L^(n2)
            // pair twiddle w_2L^(2m) = w_L^m = w_L^(m1) * w_(2 M2)^(m2), m = m1 + M1 m2
            p->t_unt1 = tb.add(L, 0, p->M1, 1, 1);                    // w_L^(m1)
            p->t_unt2 = tb.add(2 * p->M2, 0, p->M2, 1, 1);            // w_(2 M2)^(m2)
            p->t_unt_c = tb.add(2 * L, 1, 1, 1, 1);                   // w_2L^1
            p->spec_row_bytes = size_t(p->M) * 16;                   // M1 units x M2 float4
            p->ws_row_bytes = size_t(2 * p->M) * 8;                  // two chains of M complex
            if (L == kClusterL) {
                p->t_cl_fft = tb.add_fft(16384);
                p->t_cl_wa = tb.add(2 * L, 0, 16384, 1, 1);              // w_2L^a
                p->t_cl_even = tb.add(16384, 0, 2048, 1, 1, 2, 0);       // w_16384^(2j)
                p->t_cl_odd = tb.add(16384, 0, 2048, 1, 1, 2, 1);        // w_16384^(2j+1)
            }
        }
    } else if (ndim == 2) {
        const int64_t H = sizes[0], W = sizes[1];
        if (!is_pow2(H) || !is_pow2(W) || H < kMin2D || W < kMin2D || H > kMax2D || W > kMax2D) {
            *why = "2-D sizes must be powers of two in [16, 512]";
            return false;
        }
        p->path = circular ? PATH_GRID_2D_CIRC : PATH_GRID_2D;
        p->H = H;
        p->W = W;
        p->L = 0;
        p->n = H * W;
        p->M1 = W / 2;   // row chain size
        p->M2 = H;       // column chain size
        p->t_fft_a = tb.add_fft(int(p->M1));
        p->t_fft_b = tb.add_fft(int(p->M2));
        p->t_twist = tb.add(W, 0, p->M1, 1, 1);                        // w_W^n, n < W/2
        p->t_untangle = tb.add_untangle(W);
        p->t_twist_h = tb.add(2 * H, 0, H, 1, 1);                      // w_2H^p, p < H
        if (circular) {
            p->spec_row_bytes = size_t(W / 2 + 1) * size_t(H) * 8;
            p->ws_row_bytes = size_t(W / 2 + 1) * size_t(H) * 8;
        } else {
            p->spec_row_bytes = size_t(W + 1) * size_t(2 * H) * 8;
            p->ws_row_bytes = size_t(W + 1) * size_t(H) * 8;
        }
    } else if (ndim == 3) {
        const int64_t N1 = sizes[0], H = sizes[1], W = sizes[2];
        if (!is_pow2(N1) || !is_pow2(H) || !is_pow2(W) || N1 < kMin3D || H < kMin3D || W < kMin3D ||
            N1 > kMax3D || H > kMax3D || W > kMax3D) {
            *why = "3-D sizes must be powers of two in [16, 128]";
            return false;
        }
        p->path = PATH_GRID_3D;
        p->L = N1;
        p->H = H;
        p->W = W;
        p->n = N1 * H * W;
        p->M1 = W / 2;
        p->M2 = H;
        p->t_fft_a = tb.add_fft(int(p->M1));
        p->t_fft_b = tb.add_fft(int(p->M2));
        p->t_twist = tb.add(W, 0, p->M1, 1, 1);                        // w_W^n, n < W/2
        p->t_untangle = tb.add_untangle(W);
        p->t_twist_h = tb.add(2 * H, 0, H, 1, 1);                      // w_2H^p, p < H
        p->t_fft_d = tb.add_fft(int(N1));
        p->t_twist_d = tb.add(2 * N1, 0, N1, 1, 1);                    // w_2N1^d, d < N1
        p->spec_row_bytes = size_t(W + 1) * size_t(2 * H) * size_t(2 * N1) * 8;
        p->ws_row_bytes = size_t(3) * size_t(W + 1) * size_t(H) * size_t(N1) * 8;   // ws1 + ws2
    } else {
        *why = "ndim must be 1, 2 or 3";
        return false;
    }
    if (!tb.ok) { *why = "internal: too many twiddle tables"; return false; }
    p->specs.total = tb.cursor;
    p->tables_off = kHeaderBytes;
    p->spec_off = align_up(p->tables_off + size_t(tb.cursor) * 8, 256);
    p->total_bytes = p->spec_off + size_t(S) * size_t(C) * p->spec_row_bytes;
    if (p->path == PATH_MULTIPASS_1D && p->L == kClusterL) {
        p->cl_plane_off = align_up(p->total_bytes, 256);
        p->total_bytes = p->cl_plane_off + size_t(S) * size_t(C) * size_t(2 * p->L) * 4;
    }
    if (p->path == PATH_GRID_2D && p->H == kTc2dH && p->W % 32 == 0) {
        p->g2_plane_off = align_up(p->total_bytes, 256);
        p->total_bytes = p->g2_plane_off + size_t(S) * size_t(C) * size_t(2 * p->W) * size_t(2 * p->H) * 4;
    }
    if (p->path == PATH_GRID_2D_CIRC && p->H == kTc2dH && p->W == kTc2dH) {
        // the full H x W plane of the circular transform (bf16 pairs)
        p->g2_plane_off = align_up(p->total_bytes, 256);
        p->total_bytes = p->g2_plane_off + size_t(S) * size_t(C) * size_t(p->W) * size_t(p->H) * 4;
    }
    return true;
}

int64_t default_group_rows(const Plan& p, int64_t rows) {
    if (p.ws_row_bytes == 0) return rows;
    // rows per workspace group: the whole batch, up to 4 GiB of workspace.
    // Fewer, larger groups mean fewer launches and fewer partly filled last
    // waves; measured per call on B200 (group rows: ms):
    //   L = 2^20, B*C = 256:        12: 4.51  37: 3.91  128: 3.72  256: 3.67
    //   L = 65536, B*C = 4096 (o3): 192: 6.58  592: 5.93  2048: 5.72  4096: 5.68
    //   256 x 256, B*C = 512:       95: 0.76  256: 0.67  512: 0.64
    const size_t target = size_t(4) << 30;
    int64_t g = int64_t(target / p.ws_row_bytes);
    if (g < 1) g = 1;
    if (g > rows) g = rows;
    return g;
}

}  // namespace hyena
