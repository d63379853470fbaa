"""Seeded synthetic inputs for NSNQuant encode / dequant / decode attention.

This module is the only code shared by the CPU oracle and the GPU path. It holds
no NSNQuant arithmetic: it draws random numbers and shapes them into the
workloads (key/value activations with outlier channels, queries, k-means
training samples). Everything the method computes lives elsewhere.

Random numbers come from a counter-based SplitMix64 (S. Vigna, "SplitMix64",
public domain reference generator: state advance by the golden-ratio constant,
then the two xor-shift-multiply finalisation rounds). Output number ``i`` of a
stream is the finaliser applied to ``base + (i + 1) * GAMMA``, so any slice of
any tensor can be drawn independently. Uniforms take the top 53 bits; normals
use the Box-Muller transform (G. Box and M. Muller, 1958) in fp64, both outputs
of each pair.

Workload shapes follow the five configurations the decode-attention study is
quoted on (tiny correctness; Llama-3-8B layer encode; GQA 4:1 decode over a
32k context; 128k long context; Llama-3-70B serving mix). Distributions:
  K[t, c] = (z[t, c] + bias[c]) * s_t,  z ~ N(0, 1),  s_t = exp(sigma * N(0, 1))
with |bias| = 8 on 4 channels (sigma 0.5) or |bias| = 12 on 8 channels
(sigma 1.0, the long-context early-layer outlier case); V ~ N(0, 1);
q ~ N(0, 1).
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# Stream ids: independent sub-streams of one configuration seed.
STREAM_K = 0
STREAM_V = 1
STREAM_Q = 2
STREAM_CODEBOOK = 3
STREAM_SCALE_K = 4
STREAM_APPEND_K = 5
STREAM_APPEND_V = 6
STREAM_EXTRA = 7


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_base(seed: int, stream: int) -> np.uint64:
    """Starting state of sub-stream ``stream`` of configuration seed ``seed``."""
    with np.errstate(over="ignore"):
        s = np.array([(int(seed) << 20) ^ int(stream)], dtype=np.uint64)
        return _mix(s * GAMMA + np.uint64(0x632BE59BD9B4E019))[0]


def raw_u64(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    """SplitMix64 outputs ``start .. start+count-1`` of one sub-stream."""
    base = stream_base(seed, stream)
    with np.errstate(over="ignore"):
        idx = np.arange(start + 1, start + count + 1, dtype=np.uint64)
        return _mix(base + idx * GAMMA)


def uniform(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    """fp64 uniforms in [0, 1) from the top 53 bits."""
    return (raw_u64(seed, stream, start, count) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def normal(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    """fp64 N(0, 1) values ``start .. start+count-1`` (Box-Muller, both outputs)."""
    if count <= 0:
        return np.zeros(0, dtype=np.float64)
    p0 = start // 2
    p1 = (start + count + 1) // 2
    u = uniform(seed, stream, 2 * p0, 2 * (p1 - p0))
    u1 = 1.0 - u[0::2]  # (0, 1]
    u2 = u[1::2]
    r = np.sqrt(-2.0 * np.log(u1))
    th = 2.0 * np.pi * u2
    out = np.empty(2 * (p1 - p0), dtype=np.float64)
    out[0::2] = r * np.cos(th)
    out[1::2] = r * np.sin(th)
    off = start - 2 * p0
    return out[off:off + count]


def round_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even); returns uint16 bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rnd = np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))
    return ((b + rnd) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclasses.dataclass(frozen=True)
class KDist:
    """Outlier structure of the key activations."""
    bias: float          # |bias| on the outlier channels (signs alternate +, -, +, ...)
    n_outlier: int       # number of outlier channels, evenly spaced over head_dim
    sigma: float         # per-token scale = exp(sigma * N(0, 1))

    def channels(self, d: int):
        step = d // self.n_outlier
        chans = [i * step for i in range(self.n_outlier)]
        signs = [1.0 if i % 2 == 0 else -1.0 for i in range(self.n_outlier)]
        return chans, signs


K_MODERATE = KDist(bias=8.0, n_outlier=4, sigma=0.5)
K_STRONG = KDist(bias=12.0, n_outlier=8, sigma=1.0)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hkv: int
    Hq: int
    T: int
    d: int
    sub_dim: int         # 8 -> 1 bit/coord, 4 -> 2 bit/coord
    dtype: str           # "f32" or "bf16" for K/V/q I/O
    kdist: KDist
    seed: int
    decode_steps: int = 0
    prefill_seqs: int = 0
    prefill_len: int = 0


WORKLOADS = {
    "tiny": Workload("tiny", B=1, Hkv=1, Hq=1, T=256, d=128, sub_dim=8, dtype="f32",
                     kdist=K_MODERATE, seed=0),
    "encode-8x4096": Workload("encode-8x4096", B=8, Hkv=8, Hq=32, T=4096, d=128, sub_dim=4,
                              dtype="bf16", kdist=K_MODERATE, seed=1),
    "decode-16x32k-2b": Workload("decode-16x32k-2b", B=16, Hkv=8, Hq=32, T=32768, d=128,
                                 sub_dim=4, dtype="bf16", kdist=K_MODERATE, seed=2),
    "decode-16x32k-1b": Workload("decode-16x32k-1b", B=16, Hkv=8, Hq=32, T=32768, d=128,
                                 sub_dim=8, dtype="bf16", kdist=K_MODERATE, seed=2),
    "long-128k": Workload("long-128k", B=1, Hkv=8, Hq=32, T=131072, d=128, sub_dim=4,
                          dtype="bf16", kdist=K_STRONG, seed=3, decode_steps=64),
    "serving-64x8k": Workload("serving-64x8k", B=64, Hkv=8, Hq=64, T=8192, d=128, sub_dim=4,
                              dtype="bf16", kdist=K_MODERATE, seed=4, prefill_seqs=4,
                              prefill_len=2048),
}


def _slice_index(w: Workload, b: int, h: int, t0: int, H: int, T: int) -> int:
    return ((b * H + h) * T + t0) * w.d


def keys(w: Workload, b0: int = 0, b1: Optional[int] = None, t0: int = 0,
         t1: Optional[int] = None, stream: int = STREAM_K, scale_stream: int = STREAM_SCALE_K,
         T_total: Optional[int] = None) -> np.ndarray:
    """Key activations [b1-b0][Hkv][t1-t0][d] as fp64 (before any I/O rounding).

    Element (b, h, t, c) is drawn at counter ((b*Hkv + h)*T + t)*d + c, so any
    sub-block equals the same block of the full tensor.
    """
    b1 = w.B if b1 is None else b1
    T = w.T if T_total is None else T_total
    t1 = T if t1 is None else t1
    chans, signs = w.kdist.channels(w.d)
    bias = np.zeros(w.d)
    for c, s in zip(chans, signs):
        bias[c] = s * w.kdist.bias
    out = np.empty((b1 - b0, w.Hkv, t1 - t0, w.d), dtype=np.float64)
    for bi, b in enumerate(range(b0, b1)):
        for h in range(w.Hkv):
            n = normal(w.seed, stream, _slice_index(w, b, h, t0, w.Hkv, T), (t1 - t0) * w.d)
            z = n.reshape(t1 - t0, w.d)
            ts = normal(w.seed, scale_stream, (b * w.Hkv + h) * T + t0, t1 - t0)
            s = np.exp(w.kdist.sigma * ts)
            out[bi, h] = (z + bias[None, :]) * s[:, None]
    return out


def values(w: Workload, b0: int = 0, b1: Optional[int] = None, t0: int = 0,
           t1: Optional[int] = None, stream: int = STREAM_V,
           T_total: Optional[int] = None) -> np.ndarray:
    """Value activations [b1-b0][Hkv][t1-t0][d], N(0, 1), fp64."""
    b1 = w.B if b1 is None else b1
    T = w.T if T_total is None else T_total
    t1 = T if t1 is None else t1
    out = np.empty((b1 - b0, w.Hkv, t1 - t0, w.d), dtype=np.float64)
    for bi, b in enumerate(range(b0, b1)):
        for h in range(w.Hkv):
            n = normal(w.seed, stream, _slice_index(w, b, h, t0, w.Hkv, T), (t1 - t0) * w.d)
            out[bi, h] = n.reshape(t1 - t0, w.d)
    return out


def queries(w: Workload, step: int = 0, B: Optional[int] = None) -> np.ndarray:
    """One query token per sequence: [B][Hq][d], N(0, 1), fp64."""
    B = w.B if B is None else B
    n = B * w.Hq * w.d
    return normal(w.seed, STREAM_Q, step * n, n).reshape(B, w.Hq, w.d)


def codebook_samples(sub_dim: int, n: int = 1 << 16, seed: int = 0) -> np.ndarray:
    """k-means training set: n seeded N(0, I) vectors of dimension sub_dim."""
    return normal(seed, STREAM_CODEBOOK + 16 * sub_dim, 0, n * sub_dim).reshape(n, sub_dim)


def to_io(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round fp64 activations to the I/O type: fp32 array, or uint16 bf16 bits."""
    if dtype == "f32":
        return np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "bf16":
        return round_to_bf16_bits(np.asarray(x, dtype=np.float32))
    raise ValueError(dtype)


def io_to_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    """Exact fp64 value of an I/O array produced by ``to_io``."""
    if dtype == "f32":
        return np.asarray(a, dtype=np.float32).astype(np.float64)
    return bf16_bits_to_f32(a).astype(np.float64)
