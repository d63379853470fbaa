"""GPU parity of double quantization (NSNQuant Technical Summary,
Methodology §3, Double Quantization): s1 on the head's 4-bit log2 grid, a
computed o on 16 uniform levels, and a 4-bit codebook, each against the CPU
oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

import attention_decode_b200 as nsnq
import nsnq_synth as S
from oracle import oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu

D = 128
DQ = nsnq.ENCODE_DOUBLE_QUANT


def _w(B, H, T, dtype, sub, kdist=S.K_MODERATE, seed=17):
    return S.Workload("dq", B=B, Hkv=H, Hq=H, T=T, d=D, sub_dim=sub, dtype=dtype, kdist=kdist,
                      seed=seed)


def _check_grid(gpu: np.ndarray, ref: np.ndarray):
    ulp = np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64)
    assert (np.abs(gpu.astype(np.float64) - ref) <= ulp).all(), (gpu, ref)


@pytest.mark.parametrize("sub,T,dtype,kdist,flags", [
    (4, 700, "bf16", S.K_MODERATE, DQ),
    (4, 513, "f32", S.K_STRONG, DQ),
    (8, 300, "bf16", S.K_MODERATE, DQ),
    (4, 400, "bf16", S.K_MODERATE, DQ | nsnq.ENCODE_ADAPTIVE_SCALE),
    (8, 257, "f32", S.K_STRONG, DQ | nsnq.ENCODE_ADAPTIVE_SCALE),
])
def test_double_quant_encode_matches_oracle(codebooks, sub, T, dtype, kdist, flags):
    w = _w(2, 2, T, dtype, sub, kdist)
    io = S.to_io(S.keys(w), dtype)
    x64 = S.io_to_f64(io, dtype)
    C = codebooks[sub]
    ora = O.encode(x64, C, want_w=True, double_quant=True,
                   adaptive_scale=bool(flags & nsnq.ENCODE_ADAPTIVE_SCALE))
    cache = nsnq.Cache.empty(2, 2, T, sub)
    nsnq.nsnq_encode(P.to_dev(io, dtype), P.codebook(C), cache, flags=flags)
    torch.cuda.synchronize()
    _check_grid(cache.s1_grid.cpu().numpy(), ora["s1_grid"])
    P.check_shift(cache.shift.cpu().numpy(), ora["o"])
    _, n_bad, worst = P.code_report(cache.codes.cpu().numpy(), ora["codes"], ora["w"], C)
    assert n_bad == 0, worst
    P.check_scales(cache.scales.cpu().numpy(), ora)


@pytest.mark.parametrize("sub", [4, 8])
def test_double_quant_append_uses_the_stored_grid(codebooks, sub):
    """Prompt in shift-compute mode, then appended tokens (some far outside
    the prompt's s1 range) in shift-given mode on the stored grid and o."""
    w = _w(1, 2, 600, "bf16", sub)
    x = S.to_io(S.keys(w), "bf16")
    x[:, :, 590:] = S.to_io(S.io_to_f64(x[:, :, 590:], "bf16") * 30.0, "bf16")  # above the grid
    x64 = S.io_to_f64(x, "bf16")
    C = codebooks[sub]
    cb = P.codebook(C)
    cache = nsnq.Cache.empty(1, 2, 600, sub)
    xd = P.to_dev(x, "bf16")
    nsnq.nsnq_encode(xd[:, :, :500], cb, cache, flags=DQ)
    nsnq.nsnq_encode(xd[:, :, 500:], cb, cache, t_offset=500, shift_mode=nsnq.SHIFT_GIVEN, flags=DQ)
    torch.cuda.synchronize()
    grid = cache.s1_grid.cpu().numpy().astype(np.float64)
    o = cache.shift.cpu().numpy().astype(np.float64)
    pre = O.encode(x64[:, :, :500], C, double_quant=True)
    _check_grid(grid, pre["s1_grid"])
    app = O.encode(x64[:, :, 500:], C, shift=o, want_w=True, double_quant=True, s1_grid=grid)
    _, n_bad, worst = P.code_report(cache.codes[:, :, 500:].cpu().numpy(), app["codes"], app["w"], C)
    assert n_bad == 0, worst
    P.check_scales(cache.scales[:, :, 500:].cpu().numpy(), app)


@pytest.mark.parametrize("ksub,vsub", [(4, 4), (8, 8)])
def test_double_quant_codebooks_through_encode_and_attention(codebooks, ksub, vsub):
    """4-bit codebooks (16 levels over all entries) with double-quantized
    byproducts: GPU encode, then decode attention over the GPU caches,
    against the oracle's encode -> dequant -> attention."""
    B, H, Hq, T = 2, 2, 8, 640
    w = S.Workload("dqa", B=B, Hkv=H, Hq=Hq, T=T, d=D, sub_dim=4, dtype="bf16",
                   kdist=S.K_MODERATE, seed=23)
    # the 4-bit codebooks come from the library's own transform (checked
    # against the oracle's in test_codebook_quantize4_matches_oracle)
    Ck = nsnq.codebook_quantize4(torch.from_numpy(codebooks[ksub]).cuda()).cpu().numpy()
    Cv = nsnq.codebook_quantize4(torch.from_numpy(codebooks[vsub]).cuda()).cpu().numpy()
    assert len(np.unique(Ck)) <= 16
    k_io, v_io = S.to_io(S.keys(w), "bf16"), S.to_io(S.values(w), "bf16")
    ok = O.encode(S.io_to_f64(k_io, "bf16"), Ck, want_w=True, double_quant=True)
    ov = O.encode(S.io_to_f64(v_io, "bf16"), Cv, want_w=True, double_quant=True)
    kc, vc = nsnq.Cache.empty(B, H, T, ksub), nsnq.Cache.empty(B, H, T, vsub)
    kcb, vcb = P.codebook(Ck), P.codebook(Cv)
    nsnq.nsnq_encode(P.to_dev(k_io, "bf16"), kcb, kc, flags=DQ)
    nsnq.nsnq_encode(P.to_dev(v_io, "bf16"), vcb, vc, flags=DQ)
    torch.cuda.synchronize()
    for cache, ora, C in ((kc, ok, Ck), (vc, ov, Cv)):
        _, n_bad, worst = P.code_report(cache.codes.cpu().numpy(), ora["codes"], ora["w"], C)
        assert n_bad == 0, worst
    q_io = S.to_io(S.queries(w), "bf16")
    lens = [T, 401]
    out = nsnq.nsnq_attn_decode(P.to_dev(q_io, "bf16"), kc, vc, kcb, vcb,
                                torch.tensor(lens, dtype=torch.int32, device="cuda"), T, Hkv=H,
                                out_dtype=torch.float32)
    torch.cuda.synchronize()
    # the oracle's attention over the GPU's stored byproducts (its own codes)
    Kh = O.dequant(kc.codes.cpu().numpy(), kc.scales[..., 0].cpu().numpy(),
                   kc.scales[..., 1].cpu().numpy(), kc.shift.cpu().numpy(), Ck)
    Vh = O.dequant(vc.codes.cpu().numpy(), vc.scales[..., 0].cpu().numpy(),
                   vc.scales[..., 1].cpu().numpy(), vc.shift.cpu().numpy(), Cv)
    ref = O.attention(S.io_to_f64(q_io, "bf16"), Kh, Vh, lens)
    e, _ = P.attn_errors(P.out_to_np(out), ref, False)
    assert (e <= 1.0).all(), e.max()


@pytest.mark.parametrize("g", [4, 8])
def test_codebook_quantize4_matches_oracle(codebooks, g):
    """The library's 4-bit codebook transform: values equal the oracle's
    fp64 levels rounded to fp32, the 4-bit indices and the grid rebuild
    them, and the transform works in place."""
    C = codebooks[g]
    ref = O.quantize4(C)
    dev = torch.from_numpy(C).cuda()
    out, levels, grid = nsnq.codebook_quantize4(dev, want_levels=True)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), ref.astype(np.float32))
    lo, step = grid.cpu().numpy()
    assert lo == C.min() and abs(lo + 15 * step - C.max()) <= 1e-12 * abs(C.max())
    nib = levels.cpu().numpy()
    k = np.stack([nib & 15, nib >> 4], -1).reshape(-1).astype(np.float64)
    assert np.array_equal((lo + k * step).astype(np.float32), out.cpu().numpy().reshape(-1))
    inplace = dev.clone()
    nsnq.load().nsnq_codebook_quantize4(inplace.data_ptr(), inplace.data_ptr(), None, None, 256,
                                        g, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert torch.equal(inplace, out)
    # a constant codebook keeps its value (step 0)
    flat = torch.full((256, g), 0.75, device="cuda")
    assert torch.equal(nsnq.codebook_quantize4(flat), flat)


# ------------------------------------------------------------- packed form --
def unpack(cache):
    """(s1, s2, level, zero) of a packed cache, read back independently of the
    library: level k of token t sits in bits 4(t%8).. of word t/8, s1 =
    2^(lo + k step) evaluated in fp64 and rounded to fp32, and a set sign bit
    of the stored s2 marks a token with s1 = 0."""
    lev = cache.s1_levels.cpu().numpy().view(np.uint32)
    B, H, W = lev.shape
    nib = (lev[..., None] >> (4 * np.arange(8, dtype=np.uint32))) & np.uint32(15)
    k = nib.reshape(B, H, W * 8)[:, :, :cache.cap].astype(np.float64)
    grid = cache.s1_grid.cpu().numpy().astype(np.float64)
    raw = cache.scales.cpu().numpy()
    zero = np.signbit(raw)
    s1 = (2.0 ** (grid[..., 0:1] + k * grid[..., 1:2])).astype(np.float32)
    return np.where(zero, np.float32(0), s1), np.abs(raw), k, zero


@pytest.mark.parametrize("sub,dtype", [(4, "bf16"), (8, "bf16"), (4, "f32")])
def test_packed_double_quant_encode(codebooks, sub, dtype):
    """Packed double-quantized caches (4-bit s1 levels, s2 alone): the same
    codes, grid and shift as the unpacked form, s1 and s2 that unpack to the
    unpacked cache's values bit for bit, levels equal to the oracle's, and
    byte-sharing appends (one token at a time at odd positions) that leave
    their neighbours' levels intact. All-zero tokens (s1 = 0) included."""
    B, H, T, extra = 2, 2, 501, 5  # odd lengths: partial level words
    w = _w(B, H, T + extra, dtype, sub)
    io = S.to_io(S.keys(w), dtype)
    io[:, :, [3, 17, T + 1]] = 0  # zero tokens in the prompt and among the appends
    x64 = S.io_to_f64(io, dtype)
    C = codebooks[sub]
    cb = P.codebook(C)
    x = P.to_dev(io, dtype)
    caches = {}
    for packed in (True, False):
        c = nsnq.Cache.empty(B, H, T + extra, sub, packed=packed)
        nsnq.nsnq_encode(x[:, :, :T], cb, c, flags=DQ)
        for i in range(extra):
            nsnq.nsnq_encode(x[:, :, T + i:T + i + 1], cb, c, t_offset=T + i,
                             shift_mode=nsnq.SHIFT_GIVEN, flags=DQ)
        caches[packed] = c
    torch.cuda.synchronize()
    pk, pl = caches[True], caches[False]
    assert torch.equal(pk.codes, pl.codes)
    assert torch.equal(pk.shift, pl.shift) and torch.equal(pk.s1_grid, pl.s1_grid)
    s1, s2, k, zero = unpack(pk)
    ref = pl.scales.cpu().numpy()
    assert np.array_equal(s1, ref[..., 0]) and np.array_equal(s2, ref[..., 1])
    assert zero[:, :, [3, 17, T + 1]].all() and zero.sum() == 3 * B * H
    ora = O.encode(x64[:, :, :T], C, want_w=True, double_quant=True)
    lo, step = pl.s1_grid.cpu().numpy().astype(np.float64)[..., 0], \
        pl.s1_grid.cpu().numpy().astype(np.float64)[..., 1]
    with np.errstate(divide="ignore"):
        k_ora = np.clip(np.round((np.log2(ora["s1"]) - lo[..., None]) / step[..., None]), 0, 15)
    nz = ora["s1"] > 0
    assert np.array_equal(k[:, :, :T][nz], k_ora[nz])
    P.check_scales(np.stack([s1[:, :, :T], s2[:, :, :T]], -1), ora)


@pytest.mark.parametrize("sub", [4, 8])
def test_packed_caches_through_dequant_and_attention(codebooks, sub):
    """Dequant, decode attention and attention over keys before RoPE read a
    packed cache exactly as the unpacked one (same values, bit for bit), and
    agree with the oracle's attention over the unpacked byproducts."""
    B, H, Hq, T = 2, 2, 8, 640
    w = S.Workload("dqp", B=B, Hkv=H, Hq=Hq, T=T, d=D, sub_dim=sub, dtype="bf16",
                   kdist=S.K_MODERATE, seed=29)
    C = codebooks[sub]
    cb = P.codebook(C)
    k_io, v_io = S.to_io(S.keys(w), "bf16"), S.to_io(S.values(w), "bf16")
    k_io[0, 1, 100] = 0
    c = {}
    for packed in (True, False):
        kc = nsnq.Cache.empty(B, H, T, sub, packed=packed)
        vc = nsnq.Cache.empty(B, H, T, sub, packed=packed)
        nsnq.nsnq_encode(P.to_dev(k_io, "bf16"), cb, kc, flags=DQ)
        nsnq.nsnq_encode(P.to_dev(v_io, "bf16"), cb, vc, flags=DQ)
        c[packed] = (kc, vc)
    q = P.to_dev(S.to_io(S.queries(w), "bf16"), "bf16")
    lens = torch.tensor([T, 333], dtype=torch.int32, device="cuda")
    outs = {}
    for packed in (True, False):
        kc, vc = c[packed]
        outs[packed] = (
            nsnq.nsnq_dequant(kc, cb, B, H, 0, T),
            nsnq.nsnq_attn_decode(q, kc, vc, cb, cb, lens, T, Hkv=H, out_dtype=torch.float32),
            nsnq.nsnq_attn_decode_rope(q, kc, vc, cb, cb, lens, T, Hkv=H,
                                       out_dtype=torch.float32))
    torch.cuda.synchronize()
    for a, b in zip(outs[True], outs[False]):
        assert torch.equal(a, b)
    kc, vc = c[False]
    Kh = O.dequant(kc.codes.cpu().numpy(), kc.scales[..., 0].cpu().numpy(),
                   kc.scales[..., 1].cpu().numpy(), kc.shift.cpu().numpy(), C)
    Vh = O.dequant(vc.codes.cpu().numpy(), vc.scales[..., 0].cpu().numpy(),
                   vc.scales[..., 1].cpu().numpy(), vc.shift.cpu().numpy(), C)
    ref = O.attention(S.io_to_f64(S.to_io(S.queries(w), "bf16"), "bf16"), Kh, Vh, [T, 333])
    e, _ = P.attn_errors(P.out_to_np(outs[True][1]), ref, False)
    assert (e <= 1.0).all(), e.max()
