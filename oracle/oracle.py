"""Python face of the CPU oracle (ctypes over oracle/nsnq_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
benchmark's CPU-baseline leg, never by the product package. Everything here is
argument marshalling and per-slice looping; the arithmetic is in the C file,
single-threaded fp64.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        fp = ctypes.POINTER(ctypes.c_float)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        i64p = ctypes.POINTER(ctypes.c_int64)
        L.oracle_hadamard.argtypes = [ctypes.c_int, dp]
        L.oracle_kmeans.argtypes = [dp, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                    dp, i64p]
        L.oracle_encode_head.argtypes = [dp, ctypes.c_int64, ctypes.c_int, ctypes.c_int, fp,
                                         ctypes.c_int, ctypes.c_int, dp, ctypes.c_int, ctypes.c_int,
                                         dp, u8p, dp, dp, dp, dp]
        L.oracle_quantize4.argtypes = [dp, ctypes.c_int64, dp]
        L.oracle_dequant_head.argtypes = [u8p, fp, fp, fp, ctypes.c_int64, ctypes.c_int,
                                          ctypes.c_int, fp, ctypes.c_int, dp]
        L.oracle_attention_head.argtypes = [dp, ctypes.c_int, dp, dp, ctypes.c_int64,
                                            ctypes.c_int, ctypes.c_double, dp]
        L.oracle_rope.argtypes = [dp, ctypes.c_int64, ctypes.c_int, i64p, ctypes.c_double]
        for f in ("oracle_hadamard", "oracle_kmeans", "oracle_encode_head",
                  "oracle_dequant_head", "oracle_attention_head", "oracle_rope",
                  "oracle_quantize4"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def _p(a: Optional[np.ndarray], ct):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.POINTER(ct))


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


def hadamard(d: int) -> np.ndarray:
    H = np.empty((d, d), dtype=np.float64)
    _check(lib().oracle_hadamard(d, _p(H, ctypes.c_double)), "hadamard")
    return H


def kmeans(X: np.ndarray, k: int, iters: int):
    """Lloyd k-means from the first k samples; returns (fp64 centroids, counts)."""
    X = np.ascontiguousarray(X, dtype=np.float64)
    n, g = X.shape
    C = np.empty((k, g), dtype=np.float64)
    counts = np.zeros(k, dtype=np.int64)
    _check(lib().oracle_kmeans(_p(X, ctypes.c_double), n, g, k, iters, _p(C, ctypes.c_double),
                               _p(counts, ctypes.c_int64)), "kmeans")
    return C, counts


def encode(x: np.ndarray, codebook: np.ndarray, shift: Optional[np.ndarray] = None,
           want_w: bool = False, adaptive_scale: bool = False, double_quant: bool = False,
           s1_grid: Optional[np.ndarray] = None):
    """Encode x [B][H][T][d] (exact fp64 values of the I/O type).

    shift None -> the shift is computed per (b, h) over the T tokens;
    else shift [B][H][d] is used as given. adaptive_scale -> s2 carries the
    scale adjustment ||w||^2 / (w . w_hat). double_quant -> s1 on the
    head's 4-bit log2 grid (s1_grid [B][H][2] = (lo, step), given together
    with the shift, else computed) and a computed o on 16 uniform levels.
    Returns dict with codes uint8 [B][H][T][d/g], s1, s2 fp64 [B][H][T],
    o fp64 [B][H][d], s1_grid fp64 [B][H][2] and (optionally) w fp64
    [B][H][T][d].
    """
    x = np.ascontiguousarray(x, dtype=np.float64)
    B, H, T, d = x.shape
    C = np.ascontiguousarray(codebook, dtype=np.float32)
    K, g = C.shape
    J = d // g
    codes = np.zeros((B, H, T, J), dtype=np.uint8)
    s1 = np.zeros((B, H, T))
    s2 = np.zeros((B, H, T))
    o = np.zeros((B, H, d))
    w = np.zeros((B, H, T, d)) if want_w else None
    grid = np.zeros((B, H, 2))
    if s1_grid is not None:
        grid[...] = np.asarray(s1_grid, dtype=np.float64)
    for b in range(B):
        for h in range(H):
            oin = None
            if shift is not None:
                oin = np.ascontiguousarray(shift[b, h], dtype=np.float64)
            gb = np.ascontiguousarray(grid[b, h])
            ob = np.zeros(d)
            cb = np.zeros((T, J), dtype=np.uint8)
            s1b = np.zeros(T)
            s2b = np.zeros(T)
            wb = np.zeros((T, d)) if want_w else None
            _check(lib().oracle_encode_head(
                _p(np.ascontiguousarray(x[b, h]), ctypes.c_double), T, d, g,
                _p(C, ctypes.c_float), K, 1 if shift is not None else 0,
                _p(oin, ctypes.c_double), 1 if adaptive_scale else 0, 1 if double_quant else 0,
                _p(gb, ctypes.c_double), _p(cb, ctypes.c_uint8), _p(s1b, ctypes.c_double),
                _p(s2b, ctypes.c_double), _p(ob, ctypes.c_double), _p(wb, ctypes.c_double)),
                "encode")
            codes[b, h] = cb
            s1[b, h] = s1b
            s2[b, h] = s2b
            o[b, h] = ob
            grid[b, h] = gb
            if want_w:
                w[b, h] = wb
    return {"codes": codes, "s1": s1, "s2": s2, "o": o, "w": w, "s1_grid": grid}


def quantize4(x: np.ndarray) -> np.ndarray:
    """4-bit asymmetric uniform quantization of all entries of x (16 levels
    from min to max), fp64; for a codebook, its double-quantized entries."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty_like(x)
    _check(lib().oracle_quantize4(_p(x.reshape(-1), ctypes.c_double), x.size,
                                  _p(out.reshape(-1), ctypes.c_double)), "quantize4")
    return out


def dequant(codes: np.ndarray, s1: np.ndarray, s2: np.ndarray, o: np.ndarray,
            codebook: np.ndarray) -> np.ndarray:
    """x_hat [B][H][T][d] fp64 from codes [B][H][T][J] and stored fp32 s1, s2, o."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    B, H, T, J = codes.shape
    C = np.ascontiguousarray(codebook, dtype=np.float32)
    K, g = C.shape
    d = J * g
    s1 = np.asarray(s1, dtype=np.float32)
    s2 = np.asarray(s2, dtype=np.float32)
    o = np.asarray(o, dtype=np.float32)
    out = np.zeros((B, H, T, d))
    for b in range(B):
        for h in range(H):
            ob = np.zeros((T, d))
            _check(lib().oracle_dequant_head(
                _p(np.ascontiguousarray(codes[b, h]), ctypes.c_uint8),
                _p(np.ascontiguousarray(s1[b, h]), ctypes.c_float),
                _p(np.ascontiguousarray(s2[b, h]), ctypes.c_float),
                _p(np.ascontiguousarray(o[b, h]), ctypes.c_float), T, d, g,
                _p(C, ctypes.c_float), K, _p(ob, ctypes.c_double)), "dequant")
            out[b, h] = ob
    return out


def attention(q: np.ndarray, Khat: np.ndarray, Vhat: np.ndarray, seq_lens=None,
              scale: Optional[float] = None) -> np.ndarray:
    """Decode attention: q [B][Hq][d], Khat/Vhat [B][Hkv][T][d] (dense dequantized),
    query head h reads kv-head h // (Hq/Hkv); sequence b attends to its first
    seq_lens[b] tokens. Returns fp64 [B][Hq][d]."""
    q = np.ascontiguousarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    Hkv, T = Khat.shape[1], Khat.shape[2]
    G = Hq // Hkv
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    out = np.zeros((B, Hq, d))
    for b in range(B):
        L = T if seq_lens is None else int(seq_lens[b])
        for kh in range(Hkv):
            Kb = np.ascontiguousarray(Khat[b, kh, :L], dtype=np.float64)
            Vb = np.ascontiguousarray(Vhat[b, kh, :L], dtype=np.float64)
            qb = np.ascontiguousarray(q[b, kh * G:(kh + 1) * G])
            ob = np.zeros((G, d))
            _check(lib().oracle_attention_head(
                _p(qb, ctypes.c_double), G, _p(Kb, ctypes.c_double), _p(Vb, ctypes.c_double),
                L, d, scale, _p(ob, ctypes.c_double)), "attention")
            out[b, kh * G:(kh + 1) * G] = ob
    return out


def stored(enc: dict):
    """The fp32 values an encoder stores for (s1, s2, o)."""
    return (enc["s1"].astype(np.float32), enc["s2"].astype(np.float32),
            enc["o"].astype(np.float32))


def attention_with_residual(q: np.ndarray, Khat: np.ndarray, Vhat: np.ndarray, seq_lens,
                            Kres: np.ndarray, Vres: np.ndarray, res_lens,
                            scale: Optional[float] = None) -> np.ndarray:
    """Decode attention over [quantized part || full-precision residual]
    (Methodology §4, Implementation Details, Residuals: the cache is a
    quantized part plus a full-precision residual of recent tokens).

    Khat/Vhat [B][Hkv][T][d] dense dequantized, sequence b uses its first
    seq_lens[b] rows; Kres/Vres [B][Hkv][R][d] the residual tokens as stored,
    sequence b uses its first res_lens[b] rows, which come after its quantized
    tokens. One softmax over both parts. Returns fp64 [B][Hq][d]."""
    B, Hq, d = q.shape
    out = np.zeros((B, Hq, d))
    for b in range(B):
        L, r = int(seq_lens[b]), int(res_lens[b])
        Kb = np.concatenate([np.asarray(Khat[b:b + 1, :, :L], dtype=np.float64),
                             np.asarray(Kres[b:b + 1, :, :r], dtype=np.float64)], axis=2)
        Vb = np.concatenate([np.asarray(Vhat[b:b + 1, :, :L], dtype=np.float64),
                             np.asarray(Vres[b:b + 1, :, :r], dtype=np.float64)], axis=2)
        out[b:b + 1] = attention(q[b:b + 1], Kb, Vb, scale=scale)
    return out


def decode_with_residual(k_prompt: np.ndarray, v_prompt: np.ndarray, k_new: np.ndarray,
                         v_new: np.ndarray, queries: np.ndarray, Ck: np.ndarray, Cv: np.ndarray,
                         R: int, scale: Optional[float] = None, adaptive_scale: bool = False):
    """The serving loop with a residual window of R tokens (Methodology §4,
    Implementation Details, Residuals), every sequence in lock-step.

    Readings: the prompt [B][Hkv][T][d] is quantized whole, its shift o
    computed over its T tokens; decode step s appends token s of
    k_new/v_new [B][Hkv][S][d] to the residual; when the residual then holds
    R tokens it is flushed: encoded with the stored o (not refreshed) and
    appended to the quantized cache, and the residual is emptied; the step's
    query queries[s] [B][Hq][d] then attends over [quantized || residual].
    Inputs are the exact values of the I/O type. Returns (outputs fp64
    [S][B][Hq][d], final state dict: codes/s1/s2 per tensor over the
    quantized tokens, o, number of quantized and residual tokens).
    adaptive_scale applies the scale adjustment at every encode."""
    B, Hkv, T, d = k_prompt.shape
    S = k_new.shape[2]
    enc = {"K": encode(k_prompt, Ck, adaptive_scale=adaptive_scale),
           "V": encode(v_prompt, Cv, adaptive_scale=adaptive_scale)}
    o = {n: enc[n]["o"] for n in enc}
    codes = {n: [enc[n]["codes"]] for n in enc}
    s1 = {n: [enc[n]["s1"]] for n in enc}
    s2 = {n: [enc[n]["s2"]] for n in enc}
    C = {"K": Ck, "V": Cv}
    res = {"K": k_new[:, :, :0], "V": v_new[:, :, :0]}
    new = {"K": k_new, "V": v_new}
    outs = np.zeros((S,) + queries.shape[1:])
    for s in range(S):
        for n in res:
            res[n] = np.concatenate([res[n], new[n][:, :, s:s + 1]], axis=2)
        if res["K"].shape[2] == R:
            for n in res:
                e = encode(res[n], C[n], shift=o[n], adaptive_scale=adaptive_scale)
                codes[n].append(e["codes"])
                s1[n].append(e["s1"])
                s2[n].append(e["s2"])
                res[n] = res[n][:, :, :0]
        hat = {}
        for n in res:
            cs = np.concatenate(codes[n], axis=2)
            a1 = np.concatenate(s1[n], axis=2)
            a2 = np.concatenate(s2[n], axis=2)
            hat[n] = dequant(cs, a1.astype(np.float32), a2.astype(np.float32),
                             o[n].astype(np.float32), C[n])
        nq = hat["K"].shape[2]
        nr = res["K"].shape[2]
        outs[s] = attention_with_residual(queries[s], hat["K"], hat["V"], [nq] * B,
                                          res["K"], res["V"], [nr] * B, scale=scale)
    state = {"n_quant": T + (S // R) * R if R > 0 else T, "n_res": S % R}
    for n in res:
        state[n] = {"codes": np.concatenate(codes[n], axis=2),
                    "s1": np.concatenate(s1[n], axis=2), "s2": np.concatenate(s2[n], axis=2),
                    "o": o[n]}
    return outs, state


def rope(x: np.ndarray, positions, base: float = 10000.0) -> np.ndarray:
    """Rotary embedding of x [..., T, d] at positions [T] (half-split pairing,
    angle pos * base^(-2i/d)); returns a new fp64 array."""
    x = np.array(x, dtype=np.float64, copy=True)
    d = x.shape[-1]
    T = x.shape[-2]
    pos = np.ascontiguousarray(np.broadcast_to(np.asarray(positions, dtype=np.int64), (T,)))
    flat = x.reshape(-1, T, d)
    for i in range(flat.shape[0]):
        row = np.ascontiguousarray(flat[i])
        _check(lib().oracle_rope(_p(row, ctypes.c_double), T, d, _p(pos, ctypes.c_int64),
                                 float(base)), "rope")
        flat[i] = row
    return flat.reshape(x.shape)


def attention_rope(q: np.ndarray, Khat: np.ndarray, Vhat: np.ndarray, seq_lens=None,
                   base: float = 10000.0, scale: Optional[float] = None) -> np.ndarray:
    """Decode attention with keys quantized before RoPE (Methodology §4,
    Implementation Details): key t of the cache (dequantized, Khat) is
    rotated to position t before the dot product; q is the query already
    rotated at its own position."""
    T = Khat.shape[2]
    return attention(q, rope(Khat, np.arange(T), base), Vhat, seq_lens, scale)
