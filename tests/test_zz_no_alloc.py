"""nsnq_attn_decode_noalloc: decode attention for callers that cannot
allocate device memory (an engine-owned memory pool, a loop where an
allocation is not allowed, a C caller without an allocator). Its split
partials live in the library's fixed 4 MiB device array instead of a
caller workspace. Checked through the C ABI against nsnq_attn_decode on
two calls in a row (the array is shared and keeps the previous call's
contents), for the rejection of shapes that do not fit, and for a call
captured into a CUDA graph after a warm-up call.

Kept in a file of its own that is collected last."""
import os

import numpy as np
import pytest
import torch

import attention_decode_b200 as nsnq
from attention_decode_b200 import build as nbuild
from tests import parity as P
from tests.conftest import load_codebook

pytestmark = pytest.mark.gpu


def _random_inputs(B, Hq, Hkv, T, sub, seed):
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)
    caches = []
    for _ in range(2):
        c = nsnq.Cache.empty(B, Hkv, T, sub)
        c.codes.copy_(torch.randint(0, 256, c.codes.shape, generator=gen, device="cuda",
                                    dtype=torch.int32).to(torch.uint8))
        c.scales.copy_(torch.rand(c.scales.shape, generator=gen, device="cuda") + 0.5)
        c.shift.copy_(torch.randn(c.shift.shape, generator=gen, device="cuda"))
        caches.append(c)
    q = torch.randn(B, Hq, 128, generator=gen, device="cuda").to(torch.bfloat16)
    lens = torch.randint(0, T + 1, (B,), generator=gen, device="cuda", dtype=torch.int32)
    return caches, q, lens


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    nbuild.build()
    cb = nsnq.Codebook(torch.from_numpy(load_codebook(4)).cuda())
    shapes = [(4, 32, 8, 3000, 1), (2, 8, 2, 700, 2)]  # different shapes: the array is reused
    for B, Hq, Hkv, T, seed in shapes:
        (kc, vc), q, lens = _random_inputs(B, Hq, Hkv, T, 4, seed)
        ref = nsnq.nsnq_attn_decode(q, kc, vc, cb, cb, lens, T, Hkv=Hkv, out_dtype=torch.float32)
        got = nsnq.nsnq_attn_decode_noalloc(q, kc, vc, cb, cb, lens, T, Hkv=Hkv,
                                            out_dtype=torch.float32)
        torch.cuda.synchronize()
        r, g = ref.cpu().numpy().astype(np.float64), got.cpu().numpy()
        e, _ = P.attn_errors(g, r, False)
        assert (e <= 1.0).all(), e.max()


def test_noalloc_rejects_shapes_beyond_its_array():
    nbuild.build()
    cb = nsnq.Codebook(torch.from_numpy(load_codebook(4)).cuda())
    B, Hq, Hkv, T = 256, 64, 8, 16  # 256 x 64 partial rows of 528 B = 8.6 MB > 4 MiB
    assert nsnq.nsnq_attn_workspace(B, Hq, Hkv, T) > 4 * 1024 * 1024
    (kc, vc), q, lens = _random_inputs(B, Hq, Hkv, T, 4, 3)
    with pytest.raises(nsnq.NSNQError) as ei:
        nsnq.nsnq_attn_decode_noalloc(q, kc, vc, cb, cb, lens, T, Hkv=Hkv)
    assert ei.value.status == nsnq.NSNQ_ERR_WORKSPACE
    assert "fixed device array" in str(ei.value)


def test_noalloc_call_captured_in_a_cuda_graph():
    """The documented use: one call outside capture (it looks up the array),
    then calls captured into a CUDA graph; a replay reads the inputs' current
    contents and matches nsnq_attn_decode on them."""
    nbuild.build()
    cb = nsnq.Codebook(torch.from_numpy(load_codebook(4)).cuda())
    B, Hq, Hkv, T = 4, 32, 8, 2000
    (kc, vc), q, lens = _random_inputs(B, Hq, Hkv, T, 4, 5)
    out = torch.empty(B, Hq, 128, dtype=torch.float32, device="cuda")
    nsnq.nsnq_attn_decode_noalloc(q, kc, vc, cb, cb, lens, T, Hkv=Hkv, out=out)  # warm-up
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        nsnq.nsnq_attn_decode_noalloc(q, kc, vc, cb, cb, lens, T, Hkv=Hkv, out=out)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(6)
    q.copy_(torch.randn(q.shape, generator=gen, device="cuda").to(q.dtype))  # new query, same buffer
    out.zero_()
    graph.replay()
    ref = nsnq.nsnq_attn_decode(q, kc, vc, cb, cb, lens, T, Hkv=Hkv, out_dtype=torch.float32)
    torch.cuda.synchronize()
    e, _ = P.attn_errors(out.cpu().numpy(), ref.cpu().numpy().astype(np.float64), False)
    assert (e <= 1.0).all(), e.max()
    del graph
