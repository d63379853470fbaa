"""B200-native NSNQuant KV-cache quantization and quantized decode attention.

Thin Python binding over the C ABI in include/nsnq.h (libnsnq.so): argument
marshalling only. Every step of the path runs in the library's sm_100a CUDA
kernels; PyTorch supplies device memory and the current stream. There is no
CPU fallback: if the library is missing, loading raises.

    cb    = Codebook(centroids_fp32_256xg.cuda())
    cache = Cache.empty(B, H, cap, sub_dim=cb.sub_dim, device="cuda")
    nsnq_encode(x, cb, cache)                      # prompt: shift computed
    nsnq_encode(x_new, cb, cache, t_offset=T, shift_mode=SHIFT_GIVEN)
    nsnq_encode_kv(k, v, cb, k_cache, v_cache)     # keys and values in one call
    out = nsnq_attn_decode(q, k_cache, v_cache, k_cb, v_cb, seq_lens, max_len)

With a full-precision residual window of R recent tokens (DecodeCache does
the bookkeeping for sequences decoded in lock-step):

    dc = DecodeCache(B, Hkv, cap, k_cb, v_cb, window=R)
    dc.prefill(k_prompt, v_prompt)
    dc.append(k_new, v_new)          # flushes (quantizes) a full window
    out = dc.attend(q)
"""
from __future__ import annotations

import collections
import ctypes
import dataclasses
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_build", "libnsnq.so")

NSNQ_OK, NSNQ_ERR_INVALID_ARG, NSNQ_ERR_UNSUPPORTED, NSNQ_ERR_WORKSPACE, NSNQ_ERR_CUDA = range(5)
NSNQ_F32, NSNQ_BF16 = 0, 1
SHIFT_COMPUTE, SHIFT_GIVEN = 0, 1
ENCODE_DEFAULT, ENCODE_ADAPTIVE_SCALE, ENCODE_DOUBLE_QUANT, ENCODE_TC_SEARCH = 0, 1, 2, 4
HEAD_DIM = 128
N_CENTROIDS = 256

EXPORTED = ("nsnq_status_string", "nsnq_last_error", "nsnq_codebook_index_bytes",
            "nsnq_codebook_index_build", "nsnq_encode_workspace", "nsnq_encode", "nsnq_dequant",
            "nsnq_attn_workspace", "nsnq_attn_decode", "nsnq_attn_decode_res",
            "nsnq_attn_decode_rope", "nsnq_residual_write", "nsnq_attn_decode_noalloc",
            "nsnq_codebook_quantize4", "nsnq_encode_kv_workspace", "nsnq_encode_kv")


class NSNQError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"{_status_name(status)}: {detail}")
        self.status = status


class _Codebook(ctypes.Structure):
    _fields_ = [("centroids", ctypes.c_void_p), ("n_centroids", ctypes.c_int),
                ("sub_dim", ctypes.c_int), ("index", ctypes.c_void_p)]


class _Cache(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("shift", ctypes.c_void_p), ("cap", ctypes.c_int64),
                ("s1_grid", ctypes.c_void_p), ("s1_levels", ctypes.c_void_p)]


class _Residual(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("dtype", ctypes.c_int),
                ("lens", ctypes.c_void_p), ("cap", ctypes.c_int64)]


_lib = None


def load(path: str = LIB_PATH):
    """Load libnsnq.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m attention_decode_b200.build`"
                           " (the library has no CPU fallback)")
    L = ctypes.CDLL(path)
    vp, i64, ci, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    L.nsnq_status_string.argtypes = [ci]
    L.nsnq_status_string.restype = ctypes.c_char_p
    L.nsnq_last_error.argtypes = []
    L.nsnq_last_error.restype = ctypes.c_char_p
    L.nsnq_codebook_index_bytes.argtypes = [ci]
    L.nsnq_codebook_index_bytes.restype = sz
    L.nsnq_codebook_index_build.argtypes = [_Codebook, vp, sz, vp]
    L.nsnq_codebook_index_build.restype = ci
    L.nsnq_encode_workspace.argtypes = [ci, ci, i64, ci]
    L.nsnq_encode_workspace.restype = sz
    L.nsnq_encode.argtypes = [vp, ci, ci, ci, i64, ci, i64, i64, i64, i64, ci, ctypes.c_uint,
                              _Codebook, _Cache, vp, sz, vp]
    L.nsnq_encode.restype = ci
    L.nsnq_encode_kv_workspace.argtypes = [ci, ci, i64, ci]
    L.nsnq_encode_kv_workspace.restype = sz
    L.nsnq_encode_kv.argtypes = [vp, vp, ci, ci, ci, i64, ci, i64, i64, i64, i64, ci, ctypes.c_uint,
                                 _Codebook, _Cache, _Cache, vp, sz, vp]
    L.nsnq_encode_kv.restype = ci
    L.nsnq_dequant.argtypes = [_Cache, _Codebook, ci, ci, i64, i64, ci, vp, vp]
    L.nsnq_dequant.restype = ci
    L.nsnq_attn_workspace.argtypes = [ci, ci, ci, ci, i64]
    L.nsnq_attn_workspace.restype = sz
    L.nsnq_attn_decode.argtypes = [vp, ci, _Cache, _Cache, _Codebook, _Codebook, vp, i64, ci, ci,
                                   ci, ci, ctypes.c_float, vp, ci, vp, sz, vp]
    L.nsnq_attn_decode.restype = ci
    L.nsnq_attn_decode_res.argtypes = [vp, ci, _Cache, _Cache, _Codebook, _Codebook, vp, i64,
                                       _Residual, ci, ci, ci, ci, ctypes.c_float, vp, ci, vp, sz,
                                       vp]
    L.nsnq_attn_decode_res.restype = ci
    L.nsnq_attn_decode_rope.argtypes = [vp, ci, _Cache, _Cache, _Codebook, _Codebook, vp, i64,
                                        ctypes.c_double, ci, ci, ci, ci, ctypes.c_float, vp, ci, vp,
                                        sz, vp]
    L.nsnq_attn_decode_rope.restype = ci
    L.nsnq_residual_write.argtypes = [vp, ci, ci, ci, i64, ci, i64, i64, i64, i64, vp, ci, i64, vp]
    L.nsnq_residual_write.restype = ci
    L.nsnq_attn_decode_noalloc.argtypes = [vp, ci, _Cache, _Cache, _Codebook, _Codebook, vp, i64,
                                           ci, ci, ci, ci, ctypes.c_float, vp, ci, vp]
    L.nsnq_attn_decode_noalloc.restype = ci
    L.nsnq_codebook_quantize4.argtypes = [vp, vp, vp, vp, ci, ci, vp]
    L.nsnq_codebook_quantize4.restype = ci
    _lib = L
    return L


def _status_name(s: int) -> str:
    try:
        return load().nsnq_status_string(s).decode()
    except Exception:
        return f"status {s}"


def _check(status: int):
    if status != NSNQ_OK:
        raise NSNQError(status, load().nsnq_last_error().decode())


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return NSNQ_F32
    if t.dtype == torch.bfloat16:
        return NSNQ_BF16
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


@dataclasses.dataclass
class Codebook:
    """Global codebook: [256][sub_dim] fp32 on the device. A 2-bit
    (sub_dim 4) codebook also carries its search index, built on first use
    by nsnq_codebook_index_build, unless no_index is set (then every encode
    with it must pass ENCODE_TC_SEARCH)."""
    centroids: torch.Tensor
    index: Optional[torch.Tensor] = None
    no_index: bool = False

    @property
    def sub_dim(self) -> int:
        return int(self.centroids.shape[1])

    def prepare(self, stream=None) -> "Codebook":
        if self.sub_dim == 4 and self.index is None:
            n = int(load().nsnq_codebook_index_bytes(4))
            idx = torch.empty(n, dtype=torch.uint8, device=self.centroids.device)
            raw = _Codebook(_ptr(self.centroids), int(self.centroids.shape[0]), 4, None)
            _check(load().nsnq_codebook_index_build(raw, _ptr(idx), n, _stream(stream)))
            self.index = idx
        return self

    def __setattr__(self, name, value):
        object.__setattr__(self, name, value)
        if name != "_cstruct":
            object.__setattr__(self, "_cstruct", None)  # the C view no longer matches

    def _c(self) -> _Codebook:
        c = getattr(self, "_cstruct", None)
        if c is None:
            if self.sub_dim == 4 and self.index is None and self.centroids.is_cuda and not self.no_index:
                self.prepare()
            c = _Codebook(_ptr(self.centroids), int(self.centroids.shape[0]), self.sub_dim,
                          _ptr(self.index))
            object.__setattr__(self, "_cstruct", c)
        return c


def codebook_quantize4(centroids: torch.Tensor, stream=None, want_levels: bool = False):
    """The double-quantized codebook (16 shared uniform levels, Methodology §3):
    a new [256][g] fp32 tensor, plus (levels [256*g/2] uint8, grid (lo, step)
    fp64) when want_levels."""
    if centroids.dtype != torch.float32 or not centroids.is_contiguous():
        raise TypeError("centroids must be contiguous float32")
    n, g = int(centroids.shape[0]), int(centroids.shape[1])
    out = torch.empty_like(centroids)
    levels = torch.empty(n * g // 2, dtype=torch.uint8, device=centroids.device) if want_levels else None
    grid = torch.empty(2, dtype=torch.float64, device=centroids.device) if want_levels else None
    _check(load().nsnq_codebook_quantize4(_ptr(centroids), _ptr(out), _ptr(levels), _ptr(grid), n,
                                          g, _stream(stream)))
    return (out, levels, grid) if want_levels else out


@dataclasses.dataclass
class Cache:
    """One quantized tensor (K or V): codes [B][H][cap][D/g] uint8,
    scales [B][H][cap][2] fp32 (s1, s2), shift [B][H][D] fp32 (o) and, for
    double quantization, s1_grid [B][H][2] fp32 (lo, step of the log2 grid).
    The packed double-quantized form (Cache.empty(..., packed=True)) keeps s1
    as 4-bit levels, s1_levels [B][H][(cap+7)/8] int32, and scales holds s2
    alone, [B][H][cap] fp32 (sign bit set for a token with s1 = 0)."""
    codes: torch.Tensor
    scales: torch.Tensor
    shift: torch.Tensor
    s1_grid: Optional[torch.Tensor] = None
    s1_levels: Optional[torch.Tensor] = None

    @property
    def cap(self) -> int:
        return int(self.codes.shape[2])

    @property
    def packed(self) -> bool:
        return self.s1_levels is not None

    @classmethod
    def empty(cls, B: int, H: int, cap: int, sub_dim: int, device="cuda", D: int = HEAD_DIM,
              packed: bool = False):
        scales = (torch.zeros(B, H, cap, dtype=torch.float32, device=device) if packed else
                  torch.zeros(B, H, cap, 2, dtype=torch.float32, device=device))
        levels = (torch.zeros(B, H, (cap + 7) // 8, dtype=torch.int32, device=device)
                  if packed else None)
        return cls(torch.zeros(B, H, cap, D // sub_dim, dtype=torch.uint8, device=device),
                   scales, torch.zeros(B, H, D, dtype=torch.float32, device=device),
                   torch.zeros(B, H, 2, dtype=torch.float32, device=device), levels)

    def view(self, b0: int, b1: int) -> "Cache":
        """The sequences [b0, b1) of this cache (shared storage)."""
        return Cache(self.codes[b0:b1], self.scales[b0:b1], self.shift[b0:b1],
                     None if self.s1_grid is None else self.s1_grid[b0:b1],
                     None if self.s1_levels is None else self.s1_levels[b0:b1])

    def __setattr__(self, name, value):
        object.__setattr__(self, name, value)
        if name != "_cstruct":
            object.__setattr__(self, "_cstruct", None)  # the C view no longer matches

    def _c(self) -> _Cache:
        # The C view is built once per set of tensors (in-place updates keep
        # their storage): a decode loop calls the library many times per second.
        c = getattr(self, "_cstruct", None)
        if c is None:
            c = _Cache(_ptr(self.codes), _ptr(self.scales), _ptr(self.shift), self.cap,
                       _ptr(self.s1_grid), _ptr(self.s1_levels))
            object.__setattr__(self, "_cstruct", c)
        return c


def nsnq_encode_workspace(B: int, H: int, T: int, D: int = HEAD_DIM) -> int:
    return int(load().nsnq_encode_workspace(B, H, T, D))


def nsnq_attn_workspace(B: int, Hq: int, Hkv: int, max_len: int, D: int = HEAD_DIM) -> int:
    return int(load().nsnq_attn_workspace(B, Hq, Hkv, D, max_len))


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def nsnq_encode(x: torch.Tensor, cb: Codebook, cache: Cache, t_offset: int = 0,
                shift_mode: int = SHIFT_COMPUTE, workspace: Optional[torch.Tensor] = None,
                stream=None, flags: int = ENCODE_DEFAULT) -> torch.Tensor:
    """Encode x [B][H][T][D] (fp32 or bf16; channels contiguous) into cache
    positions [t_offset, t_offset + T). Returns the workspace (its first two
    uint64 hold the near-tie counters)."""
    B, H, T, D = x.shape
    if x.stride(3) != 1:
        raise ValueError("x must have contiguous channels")
    if workspace is None:  # (a given workspace is checked by the library)
        workspace = _workspace(nsnq_encode_workspace(B, H, T, D), x.device)
    _check(load().nsnq_encode(_ptr(x), _dtype_code(x), B, H, T, D, x.stride(0), x.stride(1),
                              x.stride(2), t_offset, shift_mode, flags, cb._c(), cache._c(),
                              _ptr(workspace), workspace.numel() * workspace.element_size(),
                              _stream(stream)))
    return workspace


def nsnq_encode_kv_workspace(B: int, H: int, T: int, D: int = HEAD_DIM) -> int:
    return int(load().nsnq_encode_kv_workspace(B, H, T, D))


def nsnq_encode_kv(k: torch.Tensor, v: torch.Tensor, cb: Codebook, k_cache: Cache, v_cache: Cache,
                   t_offset: int = 0, shift_mode: int = SHIFT_COMPUTE,
                   workspace: Optional[torch.Tensor] = None, stream=None,
                   flags: int = ENCODE_DEFAULT) -> torch.Tensor:
    """nsnq_encode of keys k and values v (same shape, dtype and strides) with
    one codebook, in one call: both tensors share the call's launches.
    Returns the workspace (its counters cover both tensors)."""
    B, H, T, D = k.shape
    if tuple(v.shape) != (B, H, T, D) or v.dtype != k.dtype or v.stride() != k.stride():
        raise ValueError("k and v must have the same shape, dtype and strides")
    if k.stride(3) != 1:
        raise ValueError("k and v must have contiguous channels")
    if workspace is None:
        workspace = _workspace(nsnq_encode_kv_workspace(B, H, T, D), k.device)
    _check(load().nsnq_encode_kv(_ptr(k), _ptr(v), _dtype_code(k), B, H, T, D, k.stride(0),
                                 k.stride(1), k.stride(2), t_offset, shift_mode, flags, cb._c(),
                                 k_cache._c(), v_cache._c(), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream)))
    return workspace


EncodeStats = collections.namedtuple(
    "EncodeStats", ("fp64_token_heads", "fp64_subvectors", "index_mismatch", "mma_timeout"))
EncodeStats.__doc__ = """Counters of the last nsnq_encode that used a workspace (its first 64
bytes): token-heads and sub-vectors decided on the fp64 near-tie path,
whether the codebook index did not match the centroids, and whether a
tensor-core scoring round timed out (that call's codes are then void)."""


def encode_stats(workspace: torch.Tensor) -> EncodeStats:
    """Read the counters of the last encode from its workspace (synchronises
    with the device): (fp64 token-heads, fp64 sub-vectors, index mismatch,
    MMA timeout)."""
    v = workspace[:40].cpu().view(torch.int64)
    return EncodeStats(int(v[0]), int(v[1]), int(v[2]), int(v[4]))


def nsnq_dequant(cache: Cache, cb: Codebook, B: int, H: int, t0: int, T: int,
                 out: Optional[torch.Tensor] = None, D: int = HEAD_DIM, stream=None) -> torch.Tensor:
    """Reconstruct tokens [t0, t0+T): returns fp32 [B][H][T][D]."""
    if out is None:
        out = torch.empty(B, H, T, D, dtype=torch.float32, device=cache.codes.device)
    _check(load().nsnq_dequant(cache._c(), cb._c(), B, H, t0, T, D, _ptr(out), _stream(stream)))
    return out


def nsnq_attn_decode(q: torch.Tensor, k_cache: Cache, v_cache: Cache, k_cb: Codebook,
                     v_cb: Codebook, seq_lens: torch.Tensor, max_len: int, Hkv: int,
                     softmax_scale: float = 0.0, out_dtype: torch.dtype = torch.bfloat16,
                     out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """One decode step: q [B][Hq][D] -> out [B][Hq][D] over the quantized caches."""
    B, Hq, D = q.shape
    if out is None:
        out = torch.empty(B, Hq, D, dtype=out_dtype, device=q.device)
    if workspace is None:
        workspace = _workspace(nsnq_attn_workspace(B, Hq, Hkv, max_len, D), q.device)
    if seq_lens.dtype != torch.int32:
        raise TypeError("seq_lens must be int32")
    _check(load().nsnq_attn_decode(_ptr(q), _dtype_code(q), k_cache._c(), v_cache._c(), k_cb._c(),
                                   v_cb._c(), _ptr(seq_lens), max_len, B, Hq, Hkv, D,
                                   float(softmax_scale), _ptr(out), _dtype_code(out),
                                   _ptr(workspace), workspace.numel() * workspace.element_size(),
                                   _stream(stream)))
    return out


def nsnq_attn_decode_noalloc(q: torch.Tensor, k_cache: Cache, v_cache: Cache, k_cb: Codebook,
                             v_cb: Codebook, seq_lens: torch.Tensor, max_len: int, Hkv: int,
                             softmax_scale: float = 0.0, out_dtype: torch.dtype = torch.bfloat16,
                             out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """nsnq_attn_decode without a workspace: the split partials live in the
    library's fixed 4 MiB device array (for callers that cannot allocate).
    Calls on one device must not overlap on the GPU."""
    B, Hq, D = q.shape
    if out is None:
        out = torch.empty(B, Hq, D, dtype=out_dtype, device=q.device)
    if seq_lens.dtype != torch.int32:
        raise TypeError("seq_lens must be int32")
    _check(load().nsnq_attn_decode_noalloc(_ptr(q), _dtype_code(q), k_cache._c(), v_cache._c(),
                                           k_cb._c(), v_cb._c(), _ptr(seq_lens), max_len, B, Hq,
                                           Hkv, D, float(softmax_scale), _ptr(out),
                                           _dtype_code(out), _stream(stream)))
    return out


@dataclasses.dataclass
class Residual:
    """Full-precision residual window: k, v [B][Hkv][cap][D] (fp32 or bf16)
    and lens int32 [B] (tokens held per sequence)."""
    k: torch.Tensor
    v: torch.Tensor
    lens: torch.Tensor

    @property
    def cap(self) -> int:
        return int(self.k.shape[2])

    @classmethod
    def empty(cls, B: int, H: int, cap: int, dtype=torch.bfloat16, device="cuda",
              D: int = HEAD_DIM):
        return cls(torch.zeros(B, H, cap, D, dtype=dtype, device=device),
                   torch.zeros(B, H, cap, D, dtype=dtype, device=device),
                   torch.zeros(B, dtype=torch.int32, device=device))

    def _c(self) -> _Residual:
        return _Residual(_ptr(self.k), _ptr(self.v), _dtype_code(self.k), _ptr(self.lens),
                         self.cap)


def nsnq_residual_write(x: torch.Tensor, buf: torch.Tensor, t_offset: int, stream=None):
    """Copy x [B][H][T][D] into rows [t_offset, t_offset + T) of buf [B][H][cap][D]."""
    B, H, T, D = x.shape
    if x.stride(3) != 1 or not buf.is_contiguous():
        raise ValueError("x must have contiguous channels and buf must be contiguous")
    if tuple(buf.shape[:2]) != (B, H) or buf.shape[3] != D:
        raise ValueError(f"buf shape {tuple(buf.shape)} does not match x {tuple(x.shape)}")
    _check(load().nsnq_residual_write(_ptr(x), _dtype_code(x), B, H, T, D, x.stride(0),
                                      x.stride(1), x.stride(2), t_offset, _ptr(buf),
                                      _dtype_code(buf), int(buf.shape[2]), _stream(stream)))


def nsnq_attn_decode_res(q: torch.Tensor, k_cache: Cache, v_cache: Cache, k_cb: Codebook,
                         v_cb: Codebook, seq_lens: torch.Tensor, max_len: int, Hkv: int,
                         res: Optional[Residual], softmax_scale: float = 0.0,
                         out_dtype: torch.dtype = torch.bfloat16,
                         out: Optional[torch.Tensor] = None,
                         workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Decode step over [quantized tokens || residual window tokens]."""
    B, Hq, D = q.shape
    if out is None:
        out = torch.empty(B, Hq, D, dtype=out_dtype, device=q.device)
    if workspace is None:
        workspace = _workspace(nsnq_attn_workspace(B, Hq, Hkv, max_len, D), q.device)
    if seq_lens.dtype != torch.int32 or (res is not None and res.lens.dtype != torch.int32):
        raise TypeError("seq_lens and res.lens must be int32")
    rc = res._c() if res is not None else _Residual(None, None, NSNQ_BF16, None, 0)
    _check(load().nsnq_attn_decode_res(_ptr(q), _dtype_code(q), k_cache._c(), v_cache._c(),
                                       k_cb._c(), v_cb._c(), _ptr(seq_lens), max_len, rc, B, Hq,
                                       Hkv, D, float(softmax_scale), _ptr(out), _dtype_code(out),
                                       _ptr(workspace),
                                       workspace.numel() * workspace.element_size(),
                                       _stream(stream)))
    return out


class DecodeCache:
    """Quantized K/V caches plus a full-precision residual window of `window`
    tokens, for sequences decoded in lock-step (one length for the batch).

    prefill() quantizes the whole prompt (shift computed over it); append()
    puts the new token in the window and, once the window holds `window`
    tokens, flushes it: the window is quantized with the stored shift and
    appended to the caches, and the window empties. attend() runs one
    decode step over [quantized || window]. Bookkeeping only: every step
    runs in the library's kernels."""

    def __init__(self, B: int, Hkv: int, cap: int, k_cb: Codebook, v_cb: Codebook, window: int,
                 res_dtype=torch.bfloat16, device="cuda", flags: int = ENCODE_DEFAULT):
        if window <= 0:
            raise ValueError("window must be positive")
        self.B, self.Hkv, self.window, self.flags = B, Hkv, window, flags
        self.k_cb, self.v_cb = k_cb, v_cb
        self.k = Cache.empty(B, Hkv, cap, k_cb.sub_dim, device)
        self.v = Cache.empty(B, Hkv, cap, v_cb.sub_dim, device)
        self.res = Residual.empty(B, Hkv, window, res_dtype, device)
        self.seq_lens = torch.zeros(B, dtype=torch.int32, device=device)
        self.n_quant = 0
        self.n_res = 0
        self._prefilled = False

    def prefill(self, k: torch.Tensor, v: torch.Tensor, stream=None):
        if self._prefilled:
            raise RuntimeError("prefill() was already called")
        T = int(k.shape[2])
        self._encode(k, v, 0, SHIFT_COMPUTE, stream)
        self.n_quant = T
        self.seq_lens.fill_(T)
        self._prefilled = True

    def _encode(self, k: torch.Tensor, v: torch.Tensor, t_offset: int, mode: int, stream):
        # one call for both caches when they share a codebook and the inputs a layout
        if self.k_cb is self.v_cb and v.dtype == k.dtype and v.stride() == k.stride():
            nsnq_encode_kv(k, v, self.k_cb, self.k, self.v, t_offset=t_offset, shift_mode=mode,
                           stream=stream, flags=self.flags)
        else:
            nsnq_encode(k, self.k_cb, self.k, t_offset=t_offset, shift_mode=mode, stream=stream,
                        flags=self.flags)
            nsnq_encode(v, self.v_cb, self.v, t_offset=t_offset, shift_mode=mode, stream=stream,
                        flags=self.flags)

    def append(self, k_new: torch.Tensor, v_new: torch.Tensor, stream=None):
        """k_new, v_new [B][Hkv][D] or [B][Hkv][1][D]: one token per sequence."""
        if not self._prefilled:
            raise RuntimeError("prefill() first: the window is quantized with the prompt's shift")
        if k_new.dim() == 3:
            k_new, v_new = k_new.unsqueeze(2), v_new.unsqueeze(2)
        nsnq_residual_write(k_new, self.res.k, self.n_res, stream)
        nsnq_residual_write(v_new, self.res.v, self.n_res, stream)
        self.n_res += 1
        if self.n_res == self.window:
            self.flush(stream)
        else:
            self.res.lens.fill_(self.n_res)

    def flush(self, stream=None):
        if self.n_res == 0:
            return
        if self.n_quant + self.n_res > self.k.cap:
            raise RuntimeError("quantized cache is full")
        n = self.n_res
        self._encode(self.res.k[:, :, :n], self.res.v[:, :, :n], self.n_quant, SHIFT_GIVEN, stream)
        self.n_quant += n
        self.n_res = 0
        self.seq_lens.fill_(self.n_quant)
        self.res.lens.fill_(0)

    def attend(self, q: torch.Tensor, softmax_scale: float = 0.0,
               out_dtype: torch.dtype = torch.bfloat16, stream=None) -> torch.Tensor:
        return nsnq_attn_decode_res(q, self.k, self.v, self.k_cb, self.v_cb, self.seq_lens,
                                    self.n_quant, self.Hkv, self.res, softmax_scale, out_dtype,
                                    stream=stream)


def nsnq_attn_decode_rope(q: torch.Tensor, k_cache: Cache, v_cache: Cache, k_cb: Codebook,
                          v_cb: Codebook, seq_lens: torch.Tensor, max_len: int, Hkv: int,
                          rope_base: float = 10000.0, softmax_scale: float = 0.0,
                          out_dtype: torch.dtype = torch.bfloat16,
                          out: Optional[torch.Tensor] = None,
                          workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Decode step over keys quantized before RoPE: key t is rotated to position t
    in the kernel; q [B][Hq][D] is already rotated at its own position."""
    B, Hq, D = q.shape
    if out is None:
        out = torch.empty(B, Hq, D, dtype=out_dtype, device=q.device)
    if workspace is None:
        workspace = _workspace(nsnq_attn_workspace(B, Hq, Hkv, max_len, D), q.device)
    if seq_lens.dtype != torch.int32:
        raise TypeError("seq_lens must be int32")
    _check(load().nsnq_attn_decode_rope(_ptr(q), _dtype_code(q), k_cache._c(), v_cache._c(),
                                        k_cb._c(), v_cb._c(), _ptr(seq_lens), max_len,
                                        float(rope_base), B, Hq, Hkv, D, float(softmax_scale),
                                        _ptr(out), _dtype_code(out), _ptr(workspace),
                                        workspace.numel() * workspace.element_size(),
                                        _stream(stream)))
    return out
