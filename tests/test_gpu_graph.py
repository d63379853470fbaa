"""A decode step captured in a CUDA graph: one-token appends of K and V
(shift given) followed by decode attention, and a prompt encode followed by
attention. The encode kernels and the attention split kernel are chained by
programmatic dependent launches; captured, they become programmatic graph
edges. A replay must give the same caches and output as the same calls made
eagerly."""
import numpy as np
import pytest
import torch

import attention_decode_b200 as nsnq
import nsnq_synth as S
from tests import parity as P

pytestmark = pytest.mark.gpu

D = 128


def _kv(B, H, T, seed):
    w = S.Workload("case", B=B, Hkv=H, Hq=4 * H, T=T, d=D, sub_dim=4, dtype="bf16",
                   kdist=S.K_MODERATE, seed=seed)
    return (P.to_dev(S.to_io(S.keys(w), "bf16"), "bf16"),
            P.to_dev(S.to_io(S.values(w), "bf16"), "bf16"))


def _step(cb, kc, vc, k, v, q, seq, T, out, t_offset=None, ws_e=None, ws_a=None):
    mode = nsnq.SHIFT_COMPUTE if t_offset is None else nsnq.SHIFT_GIVEN
    off = 0 if t_offset is None else t_offset
    nsnq.nsnq_encode(k, cb, kc, t_offset=off, shift_mode=mode, workspace=ws_e)
    nsnq.nsnq_encode(v, cb, vc, t_offset=off, shift_mode=mode, workspace=ws_e)
    nsnq.nsnq_attn_decode(q, kc, vc, cb, cb, seq, T, Hkv=kc.codes.shape[1], out=out,
                          out_dtype=torch.float32, workspace=ws_a)


@pytest.mark.parametrize("kind", ["prompt", "append"])
def test_captured_step_equals_eager(codebooks, kind):
    B, H, T = 2, 4, 3000
    cb = P.codebook(codebooks[4])
    k, v = _kv(B, H, T, seed=21)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(22)
    q = torch.randn(B, 4 * H, D, generator=gen, device="cuda").to(torch.bfloat16)
    caches = {}
    for name in ("eager", "graph"):
        kc = nsnq.Cache.empty(B, H, T + 1, 4)
        vc = nsnq.Cache.empty(B, H, T + 1, 4)
        caches[name] = (kc, vc)
    ws_e = torch.empty(nsnq.nsnq_encode_workspace(B, H, T), dtype=torch.uint8, device="cuda")
    ws_a = torch.empty(nsnq.nsnq_attn_workspace(B, 4 * H, H, T + 1), dtype=torch.uint8, device="cuda")
    outs = {n: torch.zeros(B, 4 * H, D, device="cuda") for n in caches}
    if kind == "prompt":
        seq = torch.full((B,), T, dtype=torch.int32, device="cuda")
        args = dict(k=k, v=v, T=T, t_offset=None)
    else:
        for kc, vc in caches.values():  # same prompt in both, then one appended token
            nsnq.nsnq_encode(k, cb, kc, workspace=ws_e)
            nsnq.nsnq_encode(v, cb, vc, workspace=ws_e)
        seq = torch.full((B,), T + 1, dtype=torch.int32, device="cuda")
        kn, vn = _kv(B, H, 1, seed=23)
        args = dict(k=kn, v=vn, T=T + 1, t_offset=T)
    cb._c()  # index built outside the capture
    kc, vc = caches["eager"]
    _step(cb, kc, vc, q=q, seq=seq, out=outs["eager"], ws_e=ws_e, ws_a=ws_a, **args)
    torch.cuda.synchronize()
    kc, vc = caches["graph"]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        _step(cb, kc, vc, q=q, seq=seq, out=outs["graph"], ws_e=ws_e, ws_a=ws_a, **args)
    for _ in range(2):  # replays repeat the same step
        graph.replay()
    torch.cuda.synchronize()
    del graph
    (ke, ve), (kg, vg) = caches["eager"], caches["graph"]
    assert torch.equal(ke.codes, kg.codes) and torch.equal(ve.codes, vg.codes)
    assert torch.equal(ke.scales, kg.scales) and torch.equal(ve.scales, vg.scales)
    assert torch.equal(ke.shift, kg.shift) and torch.equal(ve.shift, vg.shift)
    assert torch.equal(outs["eager"], outs["graph"])


@pytest.mark.parametrize("order,T", [("vk", 3000), ("vk", 100), ("kv", 100)])
def test_attention_right_after_either_encode(codebooks, order, T):
    """Attention launched right after the encode of K (V encoded before it),
    or after a small-call encode: the attention kernel starts under the
    encode (programmatic dependent launch) and must still read the finished
    caches. Compared with the same attention after a device synchronize."""
    B, H = 2, 4
    cb = P.codebook(codebooks[4])
    k, v = _kv(B, H, T, seed=31)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(32)
    q = torch.randn(B, 4 * H, D, generator=gen, device="cuda").to(torch.bfloat16)
    seq = torch.full((B,), T, dtype=torch.int32, device="cuda")
    kc = nsnq.Cache.empty(B, H, T, 4)
    vc = nsnq.Cache.empty(B, H, T, 4)
    cb._c()
    first, second = ((v, vc), (k, kc)) if order == "vk" else ((k, kc), (v, vc))
    nsnq.nsnq_encode(first[0], cb, first[1])
    nsnq.nsnq_encode(second[0], cb, second[1])
    out = nsnq.nsnq_attn_decode(q, kc, vc, cb, cb, seq, T, Hkv=H, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref = nsnq.nsnq_attn_decode(q, kc, vc, cb, cb, seq, T, Hkv=H, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
