// tables.cu -- writes the spectrum-buffer header and fills the twiddle
// tables of a plan.  Each entry w_N^e = exp(-2 pi i e / N) is evaluated in
// double precision (sincospi of the exactly reduced fraction e / N) and
// rounded once to fp32.  Cold path: runs inside hyena_filter_spectrum.
#include "kernels.h"

namespace hyena {

namespace {

__global__ void k_write_header(SpecHeader* dst, SpecHeader h) {
    if (threadIdx.x == 0 && blockIdx.x == 0) *dst = h;
}

__global__ void k_fill_tables(float2* __restrict__ tables, TableSpecs specs) {
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    for (int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; idx < specs.total; idx += stride) {
        int si = 0;
        int64_t off = idx;
        while (si < specs.n - 1 && off >= specs.s[si].na * specs.s[si].nb) {
            off -= specs.s[si].na * specs.s[si].nb;
            ++si;
        }
        const TableSpec t = specs.s[si];
        const int64_t i = off / t.nb, j = off - (off / t.nb) * t.nb;
        const int64_t prod = ((t.a0 + i) % t.N) * ((t.b0 + j) % t.N) % t.N;
        const int64_t e = (prod * (t.mult % t.N) % t.N + t.add) % t.N;
        double sn, cs;
        sincospi(-2.0 * double(e) / double(t.N), &sn, &cs);
        tables[t.dst + off] = make_float2(float(cs), float(sn));
    }
}

}  // namespace

cudaError_t launch_header_and_tables(const Plan& p, uint8_t* spectrum, cudaStream_t s) {
    SpecHeader h{};
    h.magic = kSpecMagic;
    h.version = kSpecVersion;
    h.ndim = p.ndim;
    h.order = p.order;
    h.path = p.path;
    h.C = p.C;
    h.L = p.L;
    h.H = p.H;
    h.W = p.W;
    h.M = p.M;
    h.M1 = p.M1;
    h.M2 = p.M2;
    h.tables_off = int64_t(p.tables_off);
    h.tables_count = p.specs.total;
    h.spec_off = int64_t(p.spec_off);
    h.spec_row_bytes = int64_t(p.spec_row_bytes);
    h.total_bytes = int64_t(p.total_bytes);
    h.reserved[0] = int64_t(p.cl_plane_off);
    h.reserved[1] = int64_t(p.g2_plane_off);
    k_write_header<<<1, 32, 0, s>>>(reinterpret_cast<SpecHeader*>(spectrum), h);
    if (p.specs.total > 0) {
        int blocks = int((p.specs.total + 255) / 256);
        if (blocks > 4096) blocks = 4096;
        k_fill_tables<<<blocks, 256, 0, s>>>(reinterpret_cast<float2*>(spectrum + p.tables_off), p.specs);
    }
    return cudaGetLastError();
}

}  // namespace hyena
