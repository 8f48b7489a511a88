"""Planted mistakes in the oracle must each fail at least one pin.

Each case copies hyena_oracle.c, applies one textual change that a careless
implementation could plausibly contain, compiles it with gcc into a
temporary directory and runs every pin against it.  The committed oracle is
never modified.  This shows the pins constrain every part of the oracle.
"""
import os
import tempfile

import pytest

import oracle
import oracle_pins

MUTATIONS = {
    "shortconv taps reversed": ("out[t] = w[0] * um2 + w[1] * um1 + w[2] * u[t] + bias;",
                                "out[t] = w[2] * um2 + w[1] * um1 + w[0] * u[t] + bias;"),
    "shortconv bias dropped": ("out[t] = w[0] * um2 + w[1] * um1 + w[2] * u[t] + bias;",
                               "out[t] = w[0] * um2 + w[1] * um1 + w[2] * u[t];"),
    "conv skip D dropped": ("out[t] = acc + D * x[t];", "out[t] = acc;"),
    "conv not causal-inclusive": ("for (int64_t tau = 0; tau <= t; ++tau)",
                                  "for (int64_t tau = 0; tau < t; ++tau)"),
    "fft sign flipped": ("sw[j] = sin(a) * (double)sign;", "sw[j] = -sin(a) * (double)sign;"),
    "fft twiddle stride": ("double wr = cw[j * step], wi = sw[j * step];",
                           "double wr = cw[j], wi = sw[j];"),
    "fft conv circular (no padding)": ("int64_t n = next_pow2(2 * L);", "int64_t n = next_pow2(L);"),
    "fft conv skip dropped": ("out[t] = xr[t] / (double)n + D * x[t];", "out[t] = xr[t] / (double)n;"),
    "2-D kernel transposed": ("acc += K[i * W + j] * x[(p - i) * W + (q - j)];",
                              "acc += K[j * W + i] * x[(p - i) * W + (q - j)];"),
    "2-D fft conv circular": ("int64_t nh = next_pow2(2 * H), nw = next_pow2(2 * W);",
                              "int64_t nh = next_pow2(H), nw = next_pow2(W);"),
    "gate order not reversed": ("const double *gate = x + (int64_t)(order - s) * n;",
                                "const double *gate = x + (int64_t)s * n;"),
    "filters in reverse step order": ("const double *ks = k_row + (int64_t)(s - 1) * n;",
                                      "const double *ks = k_row + (int64_t)(order - 1 - s) * n;"),
    "skip from the wrong step": ("double Ds = D_row[s - 1];", "double Ds = D_row[order - 1 - s];"),
    "output gated by x1": ("for (int64_t t = 0; t < n; ++t) y_row[t] = x[t] * v[t];",
                           "for (int64_t t = 0; t < n; ++t) y_row[t] = x[n + t] * v[t];"),
    "value chunk taken first": ("double *v = x + (int64_t)order * n;", "double *v = x;"),
    "2-D circular index not wrapped": ("acc += K[i * W + j] * x[((p - i + H) % H) * W + ((q - j + W) % W)];",
                                       "acc += K[i * W + j] * x[((p + i) % H) * W + ((q + j) % W)];"),
    "2-D circular fft skip dropped": ("for (size_t t = 0; t < n; ++t) out[t] = xr[t] * scale + D * x[t];",
                                      "for (size_t t = 0; t < n; ++t) out[t] = xr[t] * scale;"),
    "3-D kernel axes swapped": ("acc += K[(h * N2 + i) * N3 + j] * x[((a - h) * N2 + (p - i)) * N3 + (q - j)];",
                                "acc += K[(i * N2 + h) * N3 + j] * x[((a - h) * N2 + (p - i)) * N3 + (q - j)];"),
    "3-D fft depth axis not padded": ("int64_t n1 = next_pow2(2 * N1), n2 = next_pow2(2 * N2), n3 = next_pow2(2 * N3);",
                                      "int64_t n1 = next_pow2(N1), n2 = next_pow2(2 * N2), n3 = next_pow2(2 * N3);"),
    "3-D operator gates with v's chunk": ("const double *g = x + (int64_t)(order - s) * n;",
                                          "const double *g = x + (int64_t)order * n;"),
    "split interleaved (chunk j of c at c*(order+1) + j)": ("const int64_t ch = (int64_t)j * C + c;",
                                                            "const int64_t ch = c * (int64_t)(order + 1) + j;"),
    "split batch stride of one chunk": ("const int64_t src = (b * Ctot + ch) * n;",
                                        "const int64_t src = (b * C + ch) * n;"),
    "split taps of the row's first chunk": ("scw_rows[(i * (order + 1) + j) * 3 + m] = sc_w[ch * 3 + m];",
                                            "scw_rows[(i * (order + 1) + j) * 3 + m] = sc_w[c * 3 + m];"),
    "split bias of the row's first chunk": ("scb_rows[i * (order + 1) + j] = sc_b ? sc_b[ch] : 0.0;",
                                            "scb_rows[i * (order + 1) + j] = sc_b ? sc_b[c] : 0.0;"),
    "split per-sample filter index transposed": ("const int64_t f = per_sample ? b * C + c : c;",
                                                 "const int64_t f = per_sample ? c * B + b : c;"),
    "split filters indexed by batch": ("const int64_t f = per_sample ? b * C + c : c;",
                                       "const int64_t f = per_sample ? b * C + c : (c + b) % C;"),
    "bf16 bits read as the low half": ("uint32_t bits = (uint32_t)((const uint16_t *)base)[i] << 16;",
                                       "uint32_t bits = (uint32_t)((const uint16_t *)base)[i];"),
    "in_proj weight transposed": ("for (int64_t i = 0; i < D; ++i) acc += x[(b * L + l) * D + i] * W[j * D + i];",
                                  "for (int64_t i = 0; i < D; ++i) acc += x[(b * L + l) * D + i] * W[i * J + j];"),
    "in_proj not rearranged": ("u[(b * J + j) * L + l] = acc;", "u[(b * L + l) * J + j] = acc;"),
    "out_proj reads y unrearranged": ("for (int64_t i = 0; i < D; ++i) acc += y[(b * D + i) * L + l] * W[j * D + i];",
                                      "for (int64_t i = 0; i < D; ++i) acc += y[(b * L + l) * D + i] * W[j * D + i];"),
    "out_proj bias dropped": ("                double acc = bias ? bias[j] : 0.0;\n                for (int64_t i = 0; i < D; ++i) acc += y",
                              "                double acc = 0.0;\n                for (int64_t i = 0; i < D; ++i) acc += y"),
    "2-D circular form runs padded": ("if (direct) oracle_conv2d_circ_direct(ks, Ds, w, vn, H, W);",
                                      "if (direct) oracle_conv2d_direct(ks, Ds, w, vn, H, W);"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name):
    old, new = MUTATIONS[name]
    src = open(os.path.join(os.path.dirname(oracle.__file__), "hyena_oracle.c")).read()
    assert src.count(old) == 1, f"mutation anchor not found exactly once: {old!r}"
    with tempfile.TemporaryDirectory() as d:
        path = os.path.join(d, "mutant.c")
        with open(path, "w") as f:
            f.write(src.replace(old, new))
        mutant = oracle.Oracle(oracle.build(force=True, src=path, out=os.path.join(d, "libmutant.so")))
        failed = []
        for pin in oracle_pins.ALL_PINS:
            try:
                pin(mutant)
            except AssertionError:
                failed.append(pin.__name__)
        assert failed, f"no pin catches the planted mistake '{name}'"
