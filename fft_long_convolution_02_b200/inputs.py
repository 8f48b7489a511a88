"""Seeded synthetic inputs for the Hyena gated long convolution.

This module is shared by the tests, the benchmark and the oracle checks.  It
holds none of the operator's arithmetic: it only draws random numbers and
rounds them to the storage type, producing tensors in the layouts of the C
ABI (u [B, (order+1)*C, ...], k [order-1, FC, ...], D [order-1, FC], taps
[(order+1)*C, 3]).  How a (b, c) row reads its chunks from them (the split)
is part of the operator and lives in the oracle.

Every row of every tensor has its own counter-keyed numpy PCG64 stream,
``SeedSequence([seed, tag, i, j])``, so any row can be produced without
materialising the whole tensor (the oracle checks large shapes on a sample
of rows).  Tags: 1 = u, 2 = k, 3 = D, 4 = short-conv taps, 5 = tokens,
6 = embedding table, 7 = short-conv bias.

Workload recipes (shapes and distributions of the Hyena operator at the
widths and lengths the pages discuss):

* ``tiny``     B=1 C=64 L=1024 order 2, fp32.  u ~ N(0,1); k[c,t] =
  N(0,1) exp(-a_c t/L), a_c ~ U[1,8]; D ~ N(0,1); taps ~ N(0, 1/3).
* ``d768_l8k`` B=4 C=768 L=8192 order 2, bf16.  As ``tiny`` with
  a_c ~ U[0.5,6]; short conv on all 3C channels.
* ``dna_1m``   B=1 C=256 L=2^20 order 2, bf16.  Tokens uniform over
  {A,C,G,T}, embedded by a seeded N(0,1) 4x768 table; channels 0..255 ->
  x0, 256..511 -> x1, 512..767 -> v.  a_c ~ U[0.1,4].
* ``order3``   B=2 C=2048 L=65536 order 3, bf16.  a_c ~ U[0.5,8].
* ``grid2d``   B=2 C=256 256x256 order 2, bf16, no short conv.
  K[c,i,j] = N(0,1) exp(-(i^2+j^2)/(2 s_c^2)), s_c ~ U[8,128].
* ``grid2d_circ`` as ``grid2d`` in the circular (periodic) 2-D form; the
  filter is the same Gaussian-windowed N(0,1) field on the H x W grid.
* ``vol3d``    B=2 C=32 64x64x64 order 2, bf16, no short conv (3-D volumes).
  K[c,a,i,j] = N(0,1) exp(-(a^2+i^2+j^2)/(2 s_c^2)), s_c ~ U[4,32].
* ``d768_l8k_ps`` as ``d768_l8k`` with per-sample (input-dependent) filters:
  k and D drawn for every (b, c) row, filter index b*C + c.

"N(0, 1/3)" is read as variance 1/3 (standard deviation sqrt(1/3)).
bf16 values are produced once here by round-to-nearest-even from float32,
and both the CUDA path and the oracle consume exactly those values.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np

TAG_U, TAG_K, TAG_D, TAG_SCW, TAG_TOK, TAG_EMB, TAG_SCB = 1, 2, 3, 4, 5, 6, 7
TAG_X, TAG_WIN, TAG_BIN, TAG_WOUT, TAG_BOUT = 8, 9, 10, 11, 12
TAG_FILT = 13


@dataclass(frozen=True)
class Problem:
    name: str
    B: int
    C: int
    order: int
    dtype: str                 # "f32" or "bf16" storage of u, k and y
    L: int = 0                 # 1-D length (0 for 2-D / 3-D)
    H: int = 0                 # 2-D grid (0 for 1-D); 3-D: second axis
    W: int = 0
    N1: int = 0                # 3-D: first axis (0 otherwise)
    shortconv: bool = True
    decay: tuple = (1.0, 8.0)  # a_c range (1-D)
    sigma: tuple = (8.0, 128.0)  # s_c range (2-D)
    u_kind: str = "normal"     # "normal" or "acgt"
    sc_bias: bool = False
    per_sample: bool = False   # one long filter (and D) per (b, c) row
    circular: bool = False     # 2-D only: periodic boundary, no padding
    seed: int = 20260000

    @property
    def ndim(self) -> int:
        return 3 if self.N1 else (2 if self.H else 1)

    @property
    def n(self) -> int:
        return self.N1 * self.H * self.W if self.N1 else (self.H * self.W if self.H else self.L)

    @property
    def shape(self) -> tuple:
        if self.N1:
            return (self.N1, self.H, self.W)
        return (self.H, self.W) if self.H else (self.L,)

    @property
    def Ctot(self) -> int:
        return (self.order + 1) * self.C

    @property
    def FC(self) -> int:
        """Filter channels: C, or B*C with per-sample filters (index b*C + c)."""
        return self.B * self.C if self.per_sample else self.C

    def with_(self, **kw) -> "Problem":
        return replace(self, **kw)


WORKLOADS = {
    "tiny": Problem("tiny", B=1, C=64, L=1024, order=2, dtype="f32",
                    decay=(1.0, 8.0), seed=20260000),
    "d768_l8k": Problem("d768_l8k", B=4, C=768, L=8192, order=2, dtype="bf16",
                        decay=(0.5, 6.0), seed=20260001),
    "dna_1m": Problem("dna_1m", B=1, C=256, L=1 << 20, order=2, dtype="bf16",
                      decay=(0.1, 4.0), u_kind="acgt", seed=20260002),
    "order3": Problem("order3", B=2, C=2048, L=65536, order=3, dtype="bf16",
                      decay=(0.5, 8.0), seed=20260003),
    "grid2d": Problem("grid2d", B=2, C=256, H=256, W=256, order=2, dtype="bf16",
                      shortconv=False, sigma=(8.0, 128.0), seed=20260004),
    "grid2d_circ": Problem("grid2d_circ", B=2, C=256, H=256, W=256, order=2, dtype="bf16",
                           shortconv=False, sigma=(8.0, 128.0), circular=True, seed=20260006),
    "vol3d": Problem("vol3d", B=2, C=32, N1=64, H=64, W=64, order=2, dtype="bf16",
                     shortconv=False, sigma=(4.0, 32.0), seed=20260007),
    "d768_l8k_ps": Problem("d768_l8k_ps", B=4, C=768, L=8192, order=2, dtype="bf16",
                           decay=(0.5, 6.0), per_sample=True, seed=20260005),
}


def _rng(p: Problem, tag: int, i: int = 0, j: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([p.seed, tag, i, j])))


# ---------------------------------------------------------------- storage ---
def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest even."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def store(p: Problem, x: np.ndarray) -> np.ndarray:
    """Round float data to the problem's storage type (float32 or bf16 bits)."""
    x = np.asarray(x, dtype=np.float32)
    return to_bf16_bits(x) if p.dtype == "bf16" else np.ascontiguousarray(x)


def stored_values(p: Problem, s: np.ndarray) -> np.ndarray:
    """Exact float64 values of stored data."""
    if p.dtype == "bf16":
        return bf16_bits_to_f32(s).astype(np.float64)
    return np.asarray(s, dtype=np.float64)


# ------------------------------------------------------------------- rows ---
def _tokens(p: Problem) -> np.ndarray:
    return _rng(p, TAG_TOK).integers(0, 4, size=p.n, dtype=np.int64)


def _embedding(p: Problem) -> np.ndarray:
    return _rng(p, TAG_EMB).standard_normal((4, p.Ctot), dtype=np.float32)


def u_row(p: Problem, b: int, ch: int, _cache: dict | None = None) -> np.ndarray:
    """Float32 values of u[b, ch, ...] before storage rounding (flat, length n)."""
    if p.u_kind == "acgt":
        if _cache is not None:
            if "tok" not in _cache:
                _cache["tok"] = _tokens(p)
                _cache["emb"] = _embedding(p)
            tok, emb = _cache["tok"], _cache["emb"]
        else:
            tok, emb = _tokens(p), _embedding(p)
        return emb[tok, ch].astype(np.float32)
    return _rng(p, TAG_U, b, ch).standard_normal(p.n, dtype=np.float32)


def k_row(p: Problem, s: int, c: int) -> np.ndarray:
    """Float32 values of the long filter of step s (0-based), channel c (flat)."""
    g = _rng(p, TAG_K, s, c)
    if p.ndim == 1:
        a = g.uniform(p.decay[0], p.decay[1])
        t = np.arange(p.L, dtype=np.float64)
        env = np.exp(-a * t / p.L)
        return (g.standard_normal(p.L) * env).astype(np.float32)
    sig = g.uniform(p.sigma[0], p.sigma[1])
    if p.ndim == 3:
        a = np.arange(p.N1, dtype=np.float64)[:, None, None]
        i = np.arange(p.H, dtype=np.float64)[None, :, None]
        j = np.arange(p.W, dtype=np.float64)[None, None, :]
        env = np.exp(-(a * a + i * i + j * j) / (2.0 * sig * sig))
        return (g.standard_normal(p.shape) * env).astype(np.float32).reshape(-1)
    i = np.arange(p.H, dtype=np.float64)[:, None]
    j = np.arange(p.W, dtype=np.float64)[None, :]
    env = np.exp(-(i * i + j * j) / (2.0 * sig * sig))
    return (g.standard_normal((p.H, p.W)) * env).astype(np.float32).reshape(-1)


def D_all(p: Problem) -> np.ndarray:
    """[order-1, FC] float32 skip values."""
    return _rng(p, TAG_D).standard_normal((p.order - 1, p.FC), dtype=np.float32)


def sc_w_all(p: Problem) -> np.ndarray | None:
    """[(order+1)*C, 3] float32 short-conv taps, or None when disabled."""
    if not p.shortconv:
        return None
    return (_rng(p, TAG_SCW).standard_normal((p.Ctot, 3)) * np.sqrt(1.0 / 3.0)).astype(np.float32)


def sc_b_all(p: Problem) -> np.ndarray | None:
    if not (p.shortconv and p.sc_bias):
        return None
    return (_rng(p, TAG_SCB).standard_normal(p.Ctot) * np.sqrt(1.0 / 3.0)).astype(np.float32)


# ------------------------------------------------------------ full tensors ---
def make_u(p: Problem) -> np.ndarray:
    """Stored u: [B, (order+1)*C, *shape] (float32 or bf16 bits)."""
    out = np.empty((p.B, p.Ctot) + p.shape, dtype=np.uint16 if p.dtype == "bf16" else np.float32)
    cache: dict = {}
    for b in range(p.B):
        for ch in range(p.Ctot):
            out[b, ch] = store(p, u_row(p, b, ch, cache)).reshape(p.shape)
    return out


def make_k(p: Problem) -> np.ndarray:
    """Stored k: [order-1, FC, *shape] (FC = B*C, index b*C + c, with per-sample filters)."""
    out = np.empty((p.order - 1, p.FC) + p.shape, dtype=np.uint16 if p.dtype == "bf16" else np.float32)
    for s in range(p.order - 1):
        for c in range(p.FC):
            out[s, c] = store(p, k_row(p, s, c)).reshape(p.shape)
    return out


def make_layer(p: Problem) -> dict:
    """Inputs of the layer around the operator (1-D, width D = C): the token
    stream x [B, L, D] ~ N(0, 1), and the in/out projections with the default
    nn.Linear initialisation ranges, weights and biases U(-1/sqrt(D), 1/sqrt(D)):
    W_in [(order+1) D, D], b_in [(order+1) D], W_out [D, D], b_out [D].  x and
    the weights in the problem's storage type, the biases float32."""
    D, J = p.C, p.Ctot
    r = 1.0 / np.sqrt(D)
    x = np.empty((p.B, p.L, D), dtype=np.uint16 if p.dtype == "bf16" else np.float32)
    for b in range(p.B):
        x[b] = store(p, _rng(p, TAG_X, b).standard_normal((p.L, D), dtype=np.float32))
    W_in = store(p, _rng(p, TAG_WIN).uniform(-r, r, (J, D)).astype(np.float32))
    b_in = _rng(p, TAG_BIN).uniform(-r, r, J).astype(np.float32)
    W_out = store(p, _rng(p, TAG_WOUT).uniform(-r, r, (D, D)).astype(np.float32))
    b_out = _rng(p, TAG_BOUT).uniform(-r, r, D).astype(np.float32)
    return {"x": x, "W_in": W_in, "b_in": b_in, "W_out": W_out, "b_out": b_out}


def implicit_filter_params(p: Problem, width: int = 64, emb_dim: int = 3, num_inner: int = 2) -> dict:
    """Synthetic parameters of the implicit filter (HyenaFilter) for the
    (order-1) C filters of problem p: the default nn.Linear ranges
    U(-1/sqrt(fan_in), 1/sqrt(fan_in)) for weights and biases, Sin
    frequencies w ~ U[0.5, 2] around the default 1, decay rates alpha over
    the workload's range p.decay (float32 arrays)."""
    g = _rng(p, TAG_FILT)
    dm = (p.order - 1) * p.C
    u = lambda fan, shape: g.uniform(-1 / np.sqrt(fan), 1 / np.sqrt(fan), shape).astype(np.float32)
    return {"emb_dim": emb_dim, "width": width, "num_inner": num_inner,
            "W_in": u(emb_dim, (width, emb_dim)), "b_in": u(emb_dim, width),
            "W_inner": u(width, (num_inner, width, width)), "b_inner": u(width, (num_inner, width)),
            "W_out": u(width, (dm, width)), "w": g.uniform(0.5, 2.0, width).astype(np.float32),
            "alpha": g.uniform(p.decay[0], p.decay[1], dm).astype(np.float32)}


def make_all(p: Problem) -> dict:
    return {"u": make_u(p), "k": make_k(p), "D": D_all(p), "sc_w": sc_w_all(p), "sc_b": sc_b_all(p)}
