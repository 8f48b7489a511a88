"""CPU tests of the C ABI: the library loads, exports every declared symbol,
and rejects bad arguments before launching anything (no GPU needed)."""
import ctypes
import os
import re

import pytest

from fft_long_convolution_02_b200 import binding as hb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from fft_long_convolution_02_b200 import build
    build.build()
    return hb.load()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "hyena.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(hyena_\w+)\s*\(", src)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(hb.EXPORTS) == names


def test_version_and_status_strings(lib):
    assert lib.hyena_version() == 101
    for code, name in hb.STATUS.items():
        assert lib.hyena_status_string(code).decode() == name


def _sz(*s):
    return (ctypes.c_int64 * len(s))(*s)


def test_spectrum_bytes_and_workspace(lib):
    # on-chip: header + tables + (order-1) C (L/2+1) 16 bytes
    b = lib.hyena_spectrum_bytes(768, 1, _sz(1024), 2)
    assert 768 * (512 + 1) * 16 <= b < 768 * (512 + 1) * 16 + (1 << 20)
    # L = 8192: all 2L bins, 16L bytes per channel
    b = lib.hyena_spectrum_bytes(768, 1, _sz(8192), 2)
    assert 768 * 16 * 8192 <= b < 768 * 16 * 8192 + (1 << 20)
    assert lib.hyena_gated_fftconv_workspace_bytes(4, 768, 1, _sz(8192), 2) == 0
    # multi-pass: spectrum rows of 8L bytes, workspace 8L bytes per row
    L = 1 << 20
    b = lib.hyena_spectrum_bytes(256, 1, _sz(L), 2)
    assert 256 * 8 * L <= b < 256 * 8 * L + (64 << 20)
    assert lib.hyena_gated_fftconv_workspace_min_bytes(256, 1, _sz(L), 2) == 8 * L
    # 2-D: (W+1) * 2H complex64 per channel, and at H = 256 the tensor-core
    # passes' plane, 2W * 2H bf16 pairs per channel
    b = lib.hyena_spectrum_bytes(256, 2, _sz(256, 256), 2)
    assert 256 * (257 * 512 * 8 + 512 * 512 * 4) <= b < 256 * (257 * 512 * 8 + 512 * 512 * 4) + (1 << 20)
    b = lib.hyena_spectrum_bytes(256, 2, _sz(128, 256), 2)
    assert 256 * 257 * 256 * 8 <= b < 256 * 257 * 256 * 8 + (1 << 20)
    # 2-D circular: (W/2+1) * H complex64 per channel; 1-D circular is refused
    circ = 2 | 0x100
    b = lib.hyena_spectrum_bytes(256, circ, _sz(256, 128), 2)
    assert 256 * 65 * 256 * 8 <= b < 256 * 65 * 256 * 8 + (1 << 20)
    assert lib.hyena_gated_fftconv_workspace_min_bytes(256, circ, _sz(256, 128), 2) == 65 * 256 * 8
    # at 256 x 256 also the full H x W bf16 plane of the tensor-core passes
    b = lib.hyena_spectrum_bytes(256, circ, _sz(256, 256), 2)
    assert 256 * (129 * 256 * 8 + 256 * 256 * 4) <= b < 256 * (129 * 256 * 8 + 256 * 256 * 4) + (1 << 20)
    assert lib.hyena_spectrum_bytes(64, 1 | 0x100, _sz(1024), 2) == 0
    # 3-D: (W+1) 2H depth lines x 2 N1 complex64 per channel; workspace 3 (W+1) H N1 complex64
    b = lib.hyena_spectrum_bytes(8, 3, _sz(16, 32, 64), 2)
    assert 8 * 65 * 64 * 32 * 8 <= b < 8 * 65 * 64 * 32 * 8 + (1 << 20)
    assert lib.hyena_gated_fftconv_workspace_min_bytes(8, 3, _sz(16, 32, 64), 2) == 3 * 65 * 32 * 16 * 8
    assert lib.hyena_spectrum_bytes(8, 3, _sz(8, 32, 64), 2) == 0
    assert lib.hyena_spectrum_bytes(8, 3, _sz(16, 32, 256), 2) == 0
    # unsupported shapes
    for bad in [(1, _sz(12), 2), (1, _sz(8), 2), (1, _sz(1 << 21), 2), (2, _sz(16, 1024), 2),
                (1, _sz(1024), 1), (1, _sz(1024), 9)]:
        assert lib.hyena_spectrum_bytes(64, *bad) == 0


def _detail(lib):
    return lib.hyena_last_error_detail().decode()


def test_validation_errors_before_launch(lib):
    fake = 1 << 20            # never dereferenced: validation fails first
    sizes = _sz(1024)
    nbytes = lib.hyena_spectrum_bytes(64, 1, sizes, 2)
    gf = lib.hyena_gated_fftconv
    # NULL tensors
    assert gf(None, fake, fake, nbytes, None, None, 1, 64, 1, sizes, 2, 0, None, 0, None) == 1
    # bad dtype
    assert gf(fake, fake * 4, fake * 8, nbytes, None, None, 1, 64, 1, sizes, 2, 7, None, 0, None) == 1
    # unsupported length / order
    assert gf(fake, fake * 4, fake * 8, nbytes, None, None, 1, 64, 1, _sz(1000), 2, 0, None, 0, None) == 2
    assert gf(fake, fake * 4, fake * 8, nbytes, None, None, 1, 64, 1, sizes, 1, 0, None, 0, None) == 2
    # misaligned pointers
    assert gf(fake + 4, fake * 4, fake * 8, nbytes, None, None, 1, 64, 1, sizes, 2, 0, None, 0, None) == 3
    assert "16-byte" in _detail(lib)
    # spectrum size mismatch
    assert gf(fake, fake * 4, fake * 8, nbytes + 16, None, None, 1, 64, 1, sizes, 2, 0, None, 0, None) == 4
    # overlapping u and y
    assert gf(fake, fake + 64, fake * 8, nbytes, None, None, 1, 64, 1, sizes, 2, 0, None, 0, None) == 1
    # 2-D with a short conv
    s2 = _sz(32, 32)
    n2 = lib.hyena_spectrum_bytes(8, 2, s2, 2)
    ws = lib.hyena_gated_fftconv_workspace_bytes(1, 8, 2, s2, 2)
    assert gf(fake, fake * 4, fake * 8, n2, fake * 16, None, 1, 8, 2, s2, 2, 0, fake * 32, ws, None) == 1
    # workspace too small on a workspace path
    assert gf(fake, fake * 4, fake * 8, n2, None, None, 1, 8, 2, s2, 2, 0, None, 0, None) == 5
    # B < 1
    assert gf(fake, fake * 4, fake * 8, nbytes, None, None, 0, 64, 1, sizes, 2, 0, None, 0, None) == 1
    # per-sample filters: the spectrum must hold B*C rows per step
    ps = lib.hyena_gated_fftconv_per_sample
    assert ps(fake, fake * 4, fake * 8, nbytes, None, None, 2, 64, 1, sizes, 2, 0, None, 0, None) == 4
    assert "B*C" in _detail(lib)
    assert ps(fake, fake * 4, fake * 8, nbytes, None, None, 0, 64, 1, sizes, 2, 0, None, 0, None) == 1
    # filter spectrum: size mismatch and NULLs
    fs = lib.hyena_filter_spectrum
    assert fs(fake, 0, None, 64, 1, sizes, 2, fake * 8, nbytes - 16, None) == 4
    assert fs(None, 0, None, 64, 1, sizes, 2, fake * 8, nbytes, None) == 1
    # short conv
    sc = lib.hyena_shortconv
    assert sc(fake, fake * 4, None, None, 1, 3, 64, 0, None) == 1
    assert sc(fake, fake * 4, fake * 8, None, 1, 3, 63, 0, None) == 2
    assert sc(fake, fake + 16, fake * 8, None, 1, 3, 64, 0, None) == 1
    # host-buffer pipeline: device-side checks first, then the host pointers and chunk size
    hp = lib.hyena_gated_fftconv_host
    assert hp(fake, fake * 2, fake * 4 + 4, fake * 6, fake * 8, nbytes, None, None, 1, 64, 1, sizes, 2, 0,
              None, 0, 0, None) == 3
    assert hp(None, fake * 2, fake * 4, fake * 6, fake * 8, nbytes, None, None, 1, 64, 1, sizes, 2, 0,
              None, 0, 0, None) == 1
    assert hp(fake, fake * 2, fake * 4, fake * 6, fake * 8, nbytes, None, None, 1, 64, 1, sizes, 2, 0,
              None, 0, -1, None) == 1
    # tensor-core wait test hook: L = 8192 bf16 only, order <= 3, budget > 0
    dg = lib.hyena_debug_conv_tc
    n8 = lib.hyena_spectrum_bytes(4, 1, _sz(8192), 2)
    n8o4 = lib.hyena_spectrum_bytes(4, 1, _sz(8192), 4)
    big = 1 << 32
    assert dg(None, big, big * 2, n8, None, None, 2, 4, 2, 1000, 0, None) == 1
    assert dg(big, big * 2, big * 3, n8o4, None, None, 2, 4, 4, 1000, 0, None) == 2
    assert dg(big, big * 2, big * 3, n8, None, None, 2, 4, 2, 0, 0, None) == 1
    assert dg(big, big * 2, big * 3, n8 + 16, None, None, 2, 4, 2, 1000, 0, None) == 4
    # projections: NULLs, shapes, order, alignment, overlap (no launch)
    ip, op = lib.hyena_in_proj, lib.hyena_out_proj
    assert ip(None, fake, None, fake * 4, 1, 64, 64, 2, None) == 1
    assert ip(fake, fake * 2, None, fake * 4, 1, 64, 60, 2, None) == 2          # D not a multiple of 8
    assert ip(fake, fake * 2, None, fake * 4, 1, 60, 64, 2, None) == 2          # L not a multiple of 8
    assert ip(fake, fake * 2, None, fake * 4, 1, 64, 64, 9, None) == 2          # order
    assert ip(fake + 8, fake * 2, None, fake * 4, 1, 64, 64, 2, None) == 3
    assert ip(fake, fake * 2, None, fake + 64, 1, 64, 64, 2, None) == 1          # u overlaps x
    assert op(fake, fake * 2, fake * 3 + 2, fake * 4, 1, 64, 64, None) == 3      # bias misaligned
    assert op(fake, fake * 2, None, fake + 16, 1, 64, 64, None) == 1             # out overlaps y
    assert op(fake, fake * 2, None, fake * 4, 0, 64, 64, None) == 1
    # implicit filters: parameter checks before any launch
    assert lib.hyena_implicit_filter_workspace_bytes(8192, 64) == 8192 * 64 * 4
    assert lib.hyena_implicit_filter_workspace_bytes(8192, 129) == 0
    fi = lib.hyena_filter_spectrum_implicit
    assert fi(None, None, 4, 1024, 2, fake, nbytes, fake, 1 << 20, None, None) == 1
    prm = hb.ImplicitFilter(3, 64, 2, fake, fake, fake, fake, fake, fake, fake)
    n1 = lib.hyena_spectrum_bytes(4, 1, _sz(1024), 2)
    bad = hb.ImplicitFilter(4, 64, 2, fake, fake, fake, fake, fake, fake, fake)
    assert fi(ctypes.byref(bad), None, 4, 1024, 2, fake, n1, fake, 1024 * 64 * 4, None, None) == 1
    noinner = hb.ImplicitFilter(3, 64, 2, fake, fake, None, None, fake, fake, fake)
    assert fi(ctypes.byref(noinner), None, 4, 1024, 2, fake, n1, fake, 1024 * 64 * 4, None, None) == 1
    assert fi(ctypes.byref(prm), None, 4, 1024, 2, fake, n1, fake, 1024 * 64 * 4 - 4, None, None) == 5
    assert fi(ctypes.byref(prm), None, 4, 1024, 2, fake, n1 + 16, fake, 1024 * 64 * 4, None, None) == 4
    assert fi(ctypes.byref(prm), None, 4, 1 << 15, 2, fake, n1, fake, 1 << 30, None, None) == 2
    # flags entry point: unknown bits first, then the same checks as hyena_gated_fftconv
    gx = lib.hyena_gated_fftconv_ex
    assert gx(fake, fake * 4, fake * 8, nbytes, None, None, 1, 64, 1, sizes, 2, 0, None, 0, 0x2, None) == 1
    assert "flag" in _detail(lib)
    assert gx(fake, fake * 4, fake * 8, nbytes + 16, None, None, 1, 64, 1, sizes, 2, 0, None, 0, 0x1, None) == 4


def test_status_strings(lib):
    assert lib.hyena_status_string(8) == b"HYENA_ERR_TIMEOUT"
    assert lib.hyena_status_string(0) == b"HYENA_OK"


def test_spectrum_and_workspace_sizes_every_path(lib):
    """Byte counts of every path against their closed forms (header + tables
    below 1 MiB), and the shapes each path refuses."""
    hdr = 1 << 20
    C, order = 4, 3
    S = order - 1

    def spec(nd, *sizes):
        return lib.hyena_spectrum_bytes(C, nd, _sz(*sizes), order)

    def wsmin(nd, *sizes):
        return lib.hyena_gated_fftconv_workspace_min_bytes(C, nd, _sz(*sizes), order)

    for L in (16, 64, 1024, 4096, 16384):                      # on-chip pair layout
        assert S * C * (L // 2 + 1) * 16 <= spec(1, L) < S * C * (L // 2 + 1) * 16 + hdr
        assert wsmin(1, L) == 0
    assert S * C * 16 * 8192 <= spec(1, 8192) < S * C * 16 * 8192 + hdr   # two planes at L = 8192
    for L in (1 << 15, 1 << 17, 1 << 20):                      # four-step
        assert S * C * 8 * L <= spec(1, L) < S * C * 8 * L + (64 << 20)
        assert wsmin(1, L) == 8 * L
    for H, W in ((16, 16), (512, 32), (32, 512)):              # 2-D padded and circular
        assert S * C * (W + 1) * 2 * H * 8 <= spec(2, H, W) < S * C * (W + 1) * 2 * H * 8 + hdr
        assert wsmin(2, H, W) == (W + 1) * H * 8
        circ = 2 | 0x100
        assert S * C * (W // 2 + 1) * H * 8 <= spec(circ, H, W) < S * C * (W // 2 + 1) * H * 8 + hdr
        assert wsmin(circ, H, W) == (W // 2 + 1) * H * 8
    for N1, H, W in ((16, 16, 16), (128, 16, 32)):             # 3-D
        lines = (W + 1) * 2 * H
        assert S * C * lines * 2 * N1 * 8 <= spec(3, N1, H, W) < S * C * lines * 2 * N1 * 8 + hdr
        assert wsmin(3, N1, H, W) == 3 * (W + 1) * H * N1 * 8
    refused = [(1, (8,)), (1, (48,)), (1, (1 << 21,)), (2, (8, 16)), (2, (16, 1024)), (2, (24, 16)),
               (3, (8, 16, 16)), (3, (16, 256, 16)), (1 | 0x100, (1024,)),
               (3 | 0x100, (16, 16, 16)), (4, (16, 16, 16, 16))]
    for nd, sizes in refused:
        assert lib.hyena_spectrum_bytes(C, nd, _sz(*sizes), order) == 0, (nd, sizes)
