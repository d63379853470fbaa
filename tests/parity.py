"""Helpers shared by the GPU parity tests: move seeded inputs and oracle
outputs to the device, and apply the comparison rules.

Comparison rules (the tolerances the GPU path is held to):
  codes   bit-exact, except where the oracle's fp64 relative distance gap
          (d(w, C_gpu) - d(w, C_oracle)) / max(d(w, C_oracle), 1e-30) < 1e-6
  s1, s2  within 2e-6 relative of the oracle's fp64 value (fp32 storage)
  o       within 1 fp32 ulp of the oracle's fp64 value, rounded
  dequant |gpu - oracle| <= 1e-5 * max(1, |oracle|), same codes/scales/o
  attn    per (batch, head) row: max|gpu - oracle| <= 2e-3 * max|oracle row|,
          plus the bf16 rounding of each output element when the output is bf16
"""
from __future__ import annotations

import numpy as np
import torch

import attention_decode_b200 as nsnq
import nsnq_synth as S

GAP_TOL = 1e-6
ATTN_TOL = 2e-3


def to_dev(io: np.ndarray, dtype: str) -> torch.Tensor:
    if dtype == "f32":
        return torch.from_numpy(np.ascontiguousarray(io, dtype=np.float32)).cuda()
    return torch.from_numpy(np.ascontiguousarray(io).view(np.int16)).cuda().view(torch.bfloat16)


def codebook(C: np.ndarray) -> nsnq.Codebook:
    return nsnq.Codebook(torch.from_numpy(np.ascontiguousarray(C, dtype=np.float32)).cuda())


def cache_from_oracle(enc: dict, cap: int = None, t_offset: int = 0) -> nsnq.Cache:
    codes = enc["codes"]
    B, H, T, J = codes.shape
    cap = T + t_offset if cap is None else cap
    c = nsnq.Cache.empty(B, H, cap, sub_dim=128 // J)
    c.codes[:, :, t_offset:t_offset + T] = torch.from_numpy(codes).cuda()
    sc = np.stack([enc["s1"], enc["s2"]], -1).astype(np.float32)
    c.scales[:, :, t_offset:t_offset + T] = torch.from_numpy(sc).cuda()
    c.shift.copy_(torch.from_numpy(enc["o"].astype(np.float32)))
    return c


def code_report(gpu_codes: np.ndarray, ora_codes: np.ndarray, w: np.ndarray, C: np.ndarray):
    """(mismatches, mismatches outside the tie tolerance, largest relative gap)."""
    g = C.shape[1]
    mism = np.argwhere(gpu_codes != ora_codes)
    bad, worst = 0, 0.0
    C64 = C.astype(np.float64)
    for idx in mism:
        *lead, j = idx
        sub = w[tuple(lead)][j * g:(j + 1) * g]
        dg = ((sub - C64[gpu_codes[tuple(idx)]]) ** 2).sum()
        do = ((sub - C64[ora_codes[tuple(idx)]]) ** 2).sum()
        gap = (dg - do) / max(do, 1e-30)
        worst = max(worst, gap)
        if gap >= GAP_TOL:
            bad += 1
    return len(mism), bad, worst


def check_scales(gpu_scales: np.ndarray, enc: dict):
    for k, name in ((0, "s1"), (1, "s2")):
        ref = enc[name]
        got = gpu_scales[..., k].astype(np.float64)
        err = np.abs(got - ref)
        assert (err <= 2e-6 * np.abs(ref) + 1e-30).all(), (name, float((err / (np.abs(ref) + 1e-30)).max()))


def check_shift(gpu_shift: np.ndarray, o: np.ndarray):
    ref32 = o.astype(np.float32)
    ulp = np.spacing(np.abs(ref32)).astype(np.float64)
    err = np.abs(gpu_shift.astype(np.float64) - ref32.astype(np.float64))
    assert (err <= ulp).all(), float((err / np.maximum(ulp, 1e-45)).max())


def check_dequant(got: np.ndarray, ref: np.ndarray):
    err = np.abs(got.astype(np.float64) - ref)
    lim = 1e-5 * np.maximum(1.0, np.abs(ref))
    assert (err <= lim).all(), float((err / lim).max())


def attn_errors(got: np.ndarray, ref: np.ndarray, bf16_out: bool):
    """Per-row normalised error: max|gpu-oracle| / (2e-3 * max|oracle row|) (must be <= 1)."""
    got = got.astype(np.float64)
    rowmax = np.abs(ref).max(-1, keepdims=True)
    allow = ATTN_TOL * rowmax
    if bf16_out:
        allow = allow + np.abs(ref) * 2.0 ** -8
    err = np.abs(got - ref)
    return (err / np.maximum(allow, 1e-30)).max(-1), err


def out_to_np(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy()
