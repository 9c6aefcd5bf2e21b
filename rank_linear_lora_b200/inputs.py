"""Seeded synthetic inputs for the LoRA linear layer.

This module draws the tensors that both the fp64 oracle and the CUDA path consume.
It holds none of the layer's arithmetic: it only produces random numbers, rounds them
to the storage formats (bf16, or the 4-bit blockwise code for a frozen weight) and
describes the five workloads.

Random numbers come from a counter-based generator so that a tensor's values do not
depend on the shapes of the other tensors, and so any element can be regenerated
from (seed, tensor id, flat index):

* 64-bit words: the splitmix64 output function (Steele, Lea and Flood, "Fast
  splittable pseudorandom number generators", OOPSLA 2014), applied to
  ``key + (index + 1) * 0x9E3779B97F4A7C15`` where ``key`` mixes the seed with the
  tensor id.
* uniforms in (0, 1): the top 53 bits of a word, offset by half an ulp so 0 never
  occurs.
* normals: the Box-Muller transform (cosine branch) of the uniforms at counters
  2*i and 2*i + 1.

Values are drawn in fp64, rounded to fp32, then to bf16 with round-to-nearest-even.
The arrays handed out are raw bf16 bit patterns (``uint16``) so both sides read
exactly the same bits.

Value distributions per tensor (the workloads' own recipe):
x, dY ~ N(0, 1); W ~ N(0, 1/d_in); A ~ U(-1/sqrt(d_in), +1/sqrt(d_in)); B ~ N(0, 0.02^2).
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_TWO_NEG53 = 2.0 ** -53
_CHUNK = 1 << 22

# Tensor ids of the counter-based streams.  A multi-layer workload offsets them by
# 16 * layer so every layer has its own streams.
TID_X, TID_W, TID_A, TID_B, TID_DY = 1, 2, 3, 4, 5


def _mix(z: np.ndarray) -> np.ndarray:
    """splitmix64 output function on a uint64 array (wrapping arithmetic)."""
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, tensor_id: int) -> np.uint64:
    with np.errstate(over="ignore"):
        t = _mix(np.array([tensor_id], dtype=np.uint64) + _GOLDEN)
        k = _mix(np.array([seed], dtype=np.uint64) ^ t)
    return k[0]


def _words(key: np.uint64, idx: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return _mix(key + (idx + np.uint64(1)) * _GOLDEN)


def _uniform01(key: np.uint64, idx: np.ndarray) -> np.ndarray:
    w = _words(key, idx)
    return ((w >> np.uint64(11)).astype(np.float64) + 0.5) * _TWO_NEG53


def _draw_chunk(kind: str, key: np.uint64, lo: int, hi: int, p0: float) -> np.ndarray:
    i = np.arange(lo, hi, dtype=np.uint64)
    if kind == "normal":
        u1 = _uniform01(key, i * np.uint64(2))
        u2 = _uniform01(key, i * np.uint64(2) + np.uint64(1))
        return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2) * p0
    if kind == "uniform":
        u = _uniform01(key, i)
        return (2.0 * u - 1.0) * p0
    raise ValueError(kind)


def draw(kind: str, seed: int, tensor_id: int, n: int, p0: float) -> np.ndarray:
    """n fp64 draws: ``normal`` with std p0, or ``uniform`` on (-p0, p0)."""
    key = stream_key(seed, tensor_id)
    if n <= _CHUNK:
        return _draw_chunk(kind, key, 0, n, p0)
    out = np.empty(n, dtype=np.float64)
    bounds = [(lo, min(n, lo + _CHUNK)) for lo in range(0, n, _CHUNK)]

    def work(b):
        out[b[0]:b[1]] = _draw_chunk(kind, key, b[0], b[1], p0)

    with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
        list(ex.map(work, bounds))
    return out


def f32_to_bf16_bits(a32: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(a32, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def to_bf16_bits(a64: np.ndarray) -> np.ndarray:
    return f32_to_bf16_bits(a64.astype(np.float32))


Q4_BLOCK = 64


def quantise_q4(w32: np.ndarray):
    """4-bit blockwise code of a frozen weight [d_out, d_in] (fp32 draws).

    Per block of 64 consecutive d_in elements: absmax = max |w| (fp32);
    q = clamp(round_half_away(7 * w / absmax) + 8, 1, 15) (a block with absmax 0
    gets q = 8); the stored scale is bf16(absmax) (nearest-even).  Two codes per
    byte along d_in: the low nibble holds the even index.  Returns (packed uint8
    [d_out, d_in/2], scale bf16 bits [d_out, d_in/64]).
    """
    d_out, d_in = w32.shape
    assert d_in % Q4_BLOCK == 0
    out_q = np.empty((d_out, d_in // 2), dtype=np.uint8)
    out_s = np.empty((d_out, d_in // Q4_BLOCK), dtype=np.uint16)
    rows = max(1, (1 << 22) // d_in)

    def work(r0):
        r1 = min(d_out, r0 + rows)
        wb = w32[r0:r1].reshape(r1 - r0, d_in // Q4_BLOCK, Q4_BLOCK)
        amax = np.abs(wb).max(axis=2).astype(np.float32)
        safe = np.where(amax > 0, amax, np.float32(1)).astype(np.float64)
        t = 7.0 * wb.astype(np.float64) / safe[:, :, None]
        q = np.sign(t) * np.floor(np.abs(t) + 0.5) + 8.0
        q = np.clip(q, 1, 15)
        q = np.where(amax[:, :, None] > 0, q, 8.0).astype(np.uint8).reshape(r1 - r0, d_in)
        out_q[r0:r1] = (q[:, 0::2] & 0x0F) | (q[:, 1::2] << 4)
        out_s[r0:r1] = f32_to_bf16_bits(amax)

    with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
        list(ex.map(work, range(0, d_out, rows)))
    return out_q, out_s


def unpack_q4_codes(packed: np.ndarray) -> np.ndarray:
    """Inverse of the nibble packing only (codes 0..15, no scaling)."""
    d_out, half = packed.shape
    q = np.empty((d_out, half * 2), dtype=np.uint8)
    q[:, 0::2] = packed & 0x0F
    q[:, 1::2] = packed >> 4
    return q


def nf4_codebook() -> np.ndarray:
    """The 16 values of the 4-bit NormalFloat data type (QLoRA; the format of BNB-style
    4-bit weights), in increasing order, fp64.

    Construction: codes split the standard normal into equal-probability bins on each
    side of an exact zero, each side scaled so its extreme value is 1.  The positive
    side takes the quantiles Phi^-1(p) at 8 evenly spaced probabilities p from 1 - delta
    down to 1/2 (1/2 excluded), the negative side -Phi^-1(p) at 7 such probabilities,
    and zero joins them: 7 negative values, 0, 8 positive values.  delta, the tail
    probability beyond the outermost value, is the midpoint of 1/(2*15) and 1/(2*16)
    (half a bin of the 15- and 16-bin grids), which keeps the extreme quantiles finite.
    """
    from scipy.special import ndtri
    delta = 0.5 * (1.0 / 30.0 + 1.0 / 32.0)
    pos = ndtri(np.linspace(1.0 - delta, 0.5, 9)[:-1])
    neg = -ndtri(np.linspace(1.0 - delta, 0.5, 8)[:-1])
    return np.sort(np.concatenate([neg / np.abs(neg).max(), [0.0], pos / pos.max()]))


def quantise_codebook(w32: np.ndarray, codebook: np.ndarray):
    """4-bit codebook code of a frozen weight [d_out, d_in] (fp32 draws).

    Per block of 64 consecutive d_in elements: absmax = max |w| (fp32), stored as
    bf16(absmax) (nearest-even); each weight's code is the index of the codebook value
    nearest to w / stored scale (fp64; ties to the lower index); a block with absmax 0
    gets the code of the value nearest 0.  Packing as quantise_q4 (low nibble = even
    index).  Returns (packed uint8 [d_out, d_in/2], scale bf16 bits [d_out, d_in/64]).
    """
    d_out, d_in = w32.shape
    assert d_in % Q4_BLOCK == 0
    cb = np.asarray(codebook, dtype=np.float64)
    assert cb.shape == (16,) and np.all(np.diff(cb) > 0)
    mids = 0.5 * (cb[1:] + cb[:-1])  # decision boundaries; value == boundary -> lower index
    out_q = np.empty((d_out, d_in // 2), dtype=np.uint8)
    out_s = np.empty((d_out, d_in // Q4_BLOCK), dtype=np.uint16)
    rows = max(1, (1 << 22) // d_in)

    def work(r0):
        r1 = min(d_out, r0 + rows)
        wb = w32[r0:r1].reshape(r1 - r0, d_in // Q4_BLOCK, Q4_BLOCK)
        amax = np.abs(wb).max(axis=2).astype(np.float32)
        sbits = f32_to_bf16_bits(amax)
        sc = bf16_bits_to_f32(sbits).astype(np.float64)
        safe = np.where(sc > 0, sc, 1.0)
        t = np.where(sc[:, :, None] > 0, wb.astype(np.float64) / safe[:, :, None], 0.0)
        q = np.searchsorted(mids, t, side="left").astype(np.uint8).reshape(r1 - r0, d_in)
        out_q[r0:r1] = (q[:, 0::2] & 0x0F) | (q[:, 1::2] << 4)
        out_s[r0:r1] = sbits

    with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
        list(ex.map(work, range(0, d_out, rows)))
    return out_q, out_s


E4M3_MAX = 448.0


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """FP8 E4M3 codes (OCP 8-bit floating point specification: sign, 4 exponent bits
    with bias 7, 3 mantissa bits, no infinities) of finite values |v| <= 448, rounded
    to the nearest representable value, ties to even.

    In the binade [2^e, 2^(e+1)), e = -6 .. 8, representable values are 2^(e-3) apart;
    below 2^-6 (the subnormals) they are 2^-9 apart, the spacing of the lowest binade.
    So a value is k * 2^(e-3) for an integer k, with k in 8..15 for a normal value
    (exponent field e + 7, mantissa k - 8) and k in 0..7 for a subnormal one
    (exponent field 0, mantissa k).  The sign of -0.0 is kept.
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    if not np.all(a <= E4M3_MAX):
        raise ValueError("e4m3_encode: values must be finite with |v| <= 448")
    _, E = np.frexp(a)                      # a = f * 2^E, f in [0.5, 1)
    e = np.clip(E - 1, -6, 8)               # binade exponent; subnormals share -6
    k = np.rint(np.ldexp(a, 3 - e))         # spacing multiples, ties to even (exact scaling)
    carry = k >= 16                         # rounded up into the next binade
    e = np.where(carry, e + 1, e)
    k = np.where(carry, 8, k).astype(np.int64)
    normal = k >= 8
    code = np.where(normal, ((e + 7) << 3) | (k - 8), k)
    return (code | (np.signbit(v).astype(np.int64) << 7)).astype(np.uint8)


def quantise_fp8(w32: np.ndarray):
    """FP8 E4M3 code of a frozen weight [d_out, d_in] (fp32 draws), one scale per row.

    absmax = max |w| over the row (fp32); the stored scale is bf16(absmax / 448)
    (fp32 quotient, then nearest-even); each code is e4m3_encode of w / scale (the
    stored scale, quotient in fp64), clamped to +-448 since the rounded scale may sit
    just below absmax / 448.  A row with absmax 0 gets scale 0 and codes 0.  Returns
    (codes uint8 [d_out, d_in], scale bf16 bits [d_out]).
    """
    d_out, d_in = w32.shape
    out_q = np.empty((d_out, d_in), dtype=np.uint8)
    out_s = np.empty(d_out, dtype=np.uint16)
    rows = max(1, (1 << 22) // d_in)

    def work(r0):
        r1 = min(d_out, r0 + rows)
        wb = w32[r0:r1]
        amax = np.abs(wb).max(axis=1).astype(np.float32)
        sbits = f32_to_bf16_bits((amax / np.float32(E4M3_MAX)).astype(np.float32))
        sc = bf16_bits_to_f32(sbits).astype(np.float64)
        safe = np.where(sc > 0, sc, 1.0)
        t = np.clip(wb.astype(np.float64) / safe[:, None], -E4M3_MAX, E4M3_MAX)
        q = e4m3_encode(t)
        q[sc == 0] = 0
        out_q[r0:r1] = q
        out_s[r0:r1] = sbits

    with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
        list(ex.map(work, range(0, d_out, rows)))
    return out_q, out_s


@dataclass
class LayerSpec:
    """One LoRA linear: M tokens, d_in -> d_out, rank r, scale alpha/r.

    ``proj`` > 1 describes that many projections of one x stacked into one layer
    (equal sizes d_out/proj and r/proj each, scale alpha/r = (alpha/proj)/(r/proj)):
    W and A stacked by rows, B block-diagonal [d_out, r] with projection p's rank
    columns p*r/proj.. used only by its own rows.
    """
    name: str
    M: int
    d_in: int
    d_out: int
    r: int
    alpha: float
    q4: bool = False
    seed: int = 0
    layer: int = 0
    proj: int = 1
    fp8: bool = False
    nf4: bool = False   # frozen weight as 4-bit NormalFloat codes (codebook input)

    @property
    def s(self) -> float:
        return self.alpha / self.r

    @property
    def flops(self) -> float:
        """Algorithmic fwd+bwd FLOPs: 4*M*d_in*d_out + 6*M*r*(d_in+d_out) per projection,
        summed over the ``proj`` projections (the zero blocks of a stacked B are no work)."""
        rp = self.r // self.proj
        return 4.0 * self.M * self.d_in * self.d_out + 6.0 * self.M * rp * (self.proj * self.d_in + self.d_out)

    def with_(self, **kw) -> "LayerSpec":
        d = dict(self.__dict__)
        d.update(kw)
        return LayerSpec(**d)


@dataclass
class Workload:
    name: str
    layers: list = field(default_factory=list)


def workload(idx: int, r: int | None = None) -> Workload:
    """The five workloads (seed 0x5EED0000 + index).

    0: tiny, M=64, 256->256, r=8, alpha=16.
    1: attention projection, M=4096 (2 x 2048), 4096->4096, r=8, alpha=32.
    2: one 7B MLP set, M=8192: gate 4096->11008, up 4096->11008, down 11008->4096, r=16, alpha=32;
       layer 3 is gate and up on one x stacked into one layer (4096->22016, 2 x r16).
    3: rank sweep, M=16384 (2 x 8192), 4096->4096, r in {8,16,64,128}, alpha=16.
    4: 4-bit frozen W, up projection 8192->28672, r=16, alpha=32, M=4096.
    """
    seed = 0x5EED0000 + idx
    if idx == 0:
        return Workload("tiny M64 256x256 r8", [LayerSpec("tiny", 64, 256, 256, 8, 16.0, seed=seed)])
    if idx == 1:
        return Workload("attn-proj M4096 4096x4096 r8",
                        [LayerSpec("q_proj", 4096, 4096, 4096, 8, 32.0, seed=seed)])
    if idx == 2:
        return Workload("mlp-set M8192 4096<->11008 r16", [
            LayerSpec("gate_proj", 8192, 4096, 11008, 16, 32.0, seed=seed, layer=0),
            LayerSpec("up_proj", 8192, 4096, 11008, 16, 32.0, seed=seed, layer=1),
            LayerSpec("down_proj", 8192, 11008, 4096, 16, 32.0, seed=seed, layer=2),
            LayerSpec("gate_up_proj", 8192, 4096, 22016, 32, 64.0, seed=seed, layer=3, proj=2),
        ])
    if idx == 3:
        rr = 8 if r is None else r
        return Workload(f"rank-sweep M16384 4096x4096 r{rr}",
                        [LayerSpec(f"proj_r{rr}", 16384, 4096, 4096, rr, 16.0, seed=seed)])
    if idx == 4:
        return Workload("q4 up-proj M4096 8192->28672 r16",
                        [LayerSpec("up_proj_q4", 4096, 8192, 28672, 16, 32.0, q4=True, seed=seed)])
    raise ValueError(idx)


@dataclass
class LayerInputs:
    spec: LayerSpec
    x: np.ndarray            # bf16 bits [M, d_in]
    A: np.ndarray            # bf16 bits [r, d_in]
    B: np.ndarray            # bf16 bits [d_out, r]
    dY: np.ndarray           # bf16 bits [M, d_out]
    W: np.ndarray | None     # bf16 bits [d_out, d_in] (None for q4)
    Wq: np.ndarray | None    # uint8 [d_out, d_in/2] (q4 only)
    Wscale: np.ndarray | None  # bf16 bits [d_out, d_in/64] (q4 only)
    W8: np.ndarray | None = None       # uint8 E4M3 codes [d_out, d_in] (fp8 only)
    W8scale: np.ndarray | None = None  # bf16 bits [d_out] (fp8 only)
    codebook: np.ndarray | None = None  # fp64 [16] (nf4 only; Wq, Wscale hold its codes)


def make_inputs(spec: LayerSpec, *, zero_A: bool = False, zero_B: bool = False) -> LayerInputs:
    """Draw every input of one layer from its seeded streams."""
    seed, off = spec.seed, 16 * spec.layer
    M, di, do, r = spec.M, spec.d_in, spec.d_out, spec.r
    x = to_bf16_bits(draw("normal", seed, TID_X + off, M * di, 1.0)).reshape(M, di)
    dY = to_bf16_bits(draw("normal", seed, TID_DY + off, M * do, 1.0)).reshape(M, do)
    bound = 1.0 / math.sqrt(di)
    A = to_bf16_bits(draw("uniform", seed, TID_A + off, r * di, bound)).reshape(r, di)
    B = to_bf16_bits(draw("normal", seed, TID_B + off, do * r, 0.02)).reshape(do, r)
    if spec.proj > 1:  # stacked projections: keep only the diagonal blocks of B
        P = spec.proj
        own = (np.arange(do)[:, None] // (do // P)) == (np.arange(r)[None, :] // (r // P))
        B = np.where(own, B, np.uint16(0)).astype(np.uint16)
    if zero_A:
        A = np.zeros_like(A)
    if zero_B:
        B = np.zeros_like(B)
    w32 = draw("normal", seed, TID_W + off, do * di, 1.0 / math.sqrt(di)).astype(np.float32).reshape(do, di)
    if spec.q4:
        Wq, Ws = quantise_q4(w32)
        return LayerInputs(spec, x, A, B, dY, None, Wq, Ws)
    if spec.fp8:
        W8, W8s = quantise_fp8(w32)
        return LayerInputs(spec, x, A, B, dY, None, None, None, W8, W8s)
    if spec.nf4:
        cb = nf4_codebook()
        Wq, Ws = quantise_codebook(w32, cb)
        return LayerInputs(spec, x, A, B, dY, None, Wq, Ws, codebook=cb)
    return LayerInputs(spec, x, A, B, dY, f32_to_bf16_bits(w32), None, None)
