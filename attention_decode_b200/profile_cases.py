"""Run one named workload through the library a few times (for profilers).

    python -m attention_decode_b200.profile_cases <case> [--reps N]

Cases (seeded synthetic inputs generated on the device):
  encode-16x8x4096     encode one bf16 tensor, 16 x 8 kv-heads x 4096 tokens, 2 bit
                       (134 MB of input: larger than L2)
  encode-8x8x4096      the benchmark's per-tensor encode (67 MB)
  encode-kv-8x8x4096   the benchmark step's encode: keys and values of 8 x 8 kv-heads x
                       4096 tokens in one nsnq_encode_kv call (134 MB)
  encode-tc-8x8x4096   the same with the tensor-core search (ENCODE_TC_SEARCH, no index)
  encode1-16x8x4096    1-bit encode (tensor-core scoring), 16 x 8 kv-heads x 4096 tokens
  encode1-8x8x4096     1-bit encode, 8 x 8 kv-heads x 4096 tokens
  attn-16x32k-2b       decode attention, B 16, Hq 32, Hkv 8, 32768 tokens, 2 bit
  attn-16x32k-1b       the same with 1-bit K and V
  attn-64x8k-gqa8      decode attention, B 64, Hq 64, Hkv 8, 8192 tokens, 2 bit
  attn-8x4k-2b         decode attention of the benchmark step: B 8, Hq 32, Hkv 8, 4096 tokens
  attn-1x128k-2b       long-context decode attention: B 1, Hq 32, Hkv 8, 131072 tokens, 2 bit
  attn-rope-16x32k-2b  attn-16x32k-2b with the keys read as quantized before RoPE
"""
from __future__ import annotations

import argparse
import os

import numpy as np
import torch

import attention_decode_b200 as nsnq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _codebook(g, dev):
    path = os.path.join(ROOT, "tests", "golden", f"codebook_g{g}.f32")
    return nsnq.Codebook(torch.from_numpy(np.fromfile(path, dtype="<f4").reshape(256, g)).to(dev))


def _keys(gen, B, H, T, dev):
    bias = torch.zeros(128, device=dev)
    bias[[0, 32, 64, 96]] = torch.tensor([8.0, -8.0, 8.0, -8.0], device=dev)
    z = torch.randn(B, H, T, 128, generator=gen, device=dev)
    s = torch.exp(0.5 * torch.randn(B, H, T, 1, generator=gen, device=dev))
    return ((z + bias) * s).to(torch.bfloat16)


def encode_case(B, H, T, reps, dev, sub=4, flags=nsnq.ENCODE_DEFAULT):
    gen = torch.Generator(device=dev)
    gen.manual_seed(0)
    cb = _codebook(sub, dev)
    cb.no_index = bool(flags & nsnq.ENCODE_TC_SEARCH)
    x = _keys(gen, B, H, T, dev)
    cache = nsnq.Cache.empty(B, H, T, sub, device=dev)
    ws = torch.empty(nsnq.nsnq_encode_workspace(B, H, T), dtype=torch.uint8, device=dev)
    if not cb.no_index:
        cb.prepare()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(reps):
        e0.record()
        nsnq.nsnq_encode(x, cb, cache, workspace=ws, flags=flags)
        e1.record()
    torch.cuda.synchronize()
    th, sv, mism, tmo = nsnq.encode_stats(ws)
    print(f"last call {e0.elapsed_time(e1):.3f} ms; fp64 path: {th} of {B * H * T} token-heads, "
          f"{sv} sub-vectors; index mismatch {mism}; MMA timeout {tmo}")


def encode_kv_case(B, H, T, reps, dev, sub=4):
    gen = torch.Generator(device=dev)
    gen.manual_seed(0)
    cb = _codebook(sub, dev).prepare()
    k = _keys(gen, B, H, T, dev)
    v = torch.randn(B, H, T, 128, generator=gen, device=dev).to(torch.bfloat16)
    kc = nsnq.Cache.empty(B, H, T, sub, device=dev)
    vc = nsnq.Cache.empty(B, H, T, sub, device=dev)
    ws = torch.empty(nsnq.nsnq_encode_kv_workspace(B, H, T), dtype=torch.uint8, device=dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(reps):
        e0.record()
        nsnq.nsnq_encode_kv(k, v, cb, kc, vc, workspace=ws)
        e1.record()
    torch.cuda.synchronize()
    th, sv, mism, tmo = nsnq.encode_stats(ws)
    print(f"last call {e0.elapsed_time(e1):.3f} ms; fp64 path: {th} of {2 * B * H * T} token-heads, "
          f"{sv} sub-vectors; index mismatch {mism}; MMA timeout {tmo}")


def append_case(B, H, sub, reps, dev):
    """A decode step's appends: one token per (sequence, kv-head) encoded with
    the stored shift (the small-call pass 2) after a 1024-token prompt."""
    gen = torch.Generator(device=dev)
    gen.manual_seed(0)
    cb = _codebook(sub, dev)
    T = 1024
    cache = nsnq.Cache.empty(B, H, T + reps, sub, device=dev)
    ws = torch.empty(nsnq.nsnq_encode_workspace(B, H, T), dtype=torch.uint8, device=dev)
    cb.prepare()
    nsnq.nsnq_encode(_keys(gen, B, H, T, dev), cb, cache, workspace=ws)
    xn = _keys(gen, B, H, reps, dev)
    for i in range(reps):
        nsnq.nsnq_encode(xn[:, :, i:i + 1], cb, cache, t_offset=T + i,
                         shift_mode=nsnq.SHIFT_GIVEN, workspace=ws)
    torch.cuda.synchronize()


def attn_case(B, Hq, Hkv, T, sub, reps, dev, rope=False):
    gen = torch.Generator(device=dev)
    gen.manual_seed(1)
    cb = _codebook(sub, dev)
    kc = nsnq.Cache.empty(B, Hkv, T, sub, device=dev)
    vc = nsnq.Cache.empty(B, Hkv, T, sub, device=dev)
    for c in (kc, vc):
        c.codes.copy_(torch.randint(0, 256, c.codes.shape, generator=gen, device=dev,
                                    dtype=torch.int32).to(torch.uint8))
        c.scales.copy_(torch.rand(c.scales.shape, generator=gen, device=dev) + 0.5)
        c.shift.copy_(torch.randn(c.shift.shape, generator=gen, device=dev))
    q = torch.randn(B, Hq, 128, generator=gen, device=dev).to(torch.bfloat16)
    seq = torch.full((B,), T, dtype=torch.int32, device=dev)
    ws = torch.empty(nsnq.nsnq_attn_workspace(B, Hq, Hkv, T), dtype=torch.uint8, device=dev)
    out = torch.empty(B, Hq, 128, dtype=torch.bfloat16, device=dev)
    run = nsnq.nsnq_attn_decode_rope if rope else nsnq.nsnq_attn_decode
    for _ in range(reps):
        run(q, kc, vc, cb, cb, seq, T, Hkv=Hkv, out=out, workspace=ws)
    torch.cuda.synchronize()


CASES = {
    "encode-16x8x4096": lambda r, d: encode_case(16, 8, 4096, r, d),
    "encode-8x8x4096": lambda r, d: encode_case(8, 8, 4096, r, d),
    "encode-kv-8x8x4096": lambda r, d: encode_kv_case(8, 8, 4096, r, d),
    "encode-tc-8x8x4096": lambda r, d: encode_case(8, 8, 4096, r, d, flags=nsnq.ENCODE_TC_SEARCH),
    "encode1-16x8x4096": lambda r, d: encode_case(16, 8, 4096, r, d, sub=8),
    "encode1-8x8x4096": lambda r, d: encode_case(8, 8, 4096, r, d, sub=8),
    "attn-16x32k-2b": lambda r, d: attn_case(16, 32, 8, 32768, 4, r, d),
    "attn-16x32k-1b": lambda r, d: attn_case(16, 32, 8, 32768, 8, r, d),
    "attn-rope-16x32k-2b": lambda r, d: attn_case(16, 32, 8, 32768, 4, r, d, rope=True),
    "attn-64x8k-gqa8": lambda r, d: attn_case(64, 64, 8, 8192, 4, r, d),
    "attn-8x4k-2b": lambda r, d: attn_case(8, 32, 8, 4096, 4, r, d),
    "attn-1x128k-2b": lambda r, d: attn_case(1, 32, 8, 131072, 4, r, d),
    "append-64x8-2b": lambda r, d: append_case(64, 8, 4, r, d),
}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=sorted(CASES))
    ap.add_argument("--reps", type=int, default=3)
    a = ap.parse_args()
    from attention_decode_b200 import build as nbuild
    nbuild.build()
    CASES[a.case](a.reps, torch.device("cuda", 0))
    print(f"{a.case}: {a.reps} calls done")


if __name__ == "__main__":
    main()
