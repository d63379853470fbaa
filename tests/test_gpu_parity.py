"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs, at sizes the oracle finishes in seconds, spanning several
tiles and ragged tails, plus the degenerate cases of the method."""
import numpy as np
import pytest
import torch

import attention_decode_b200 as nsnq
import nsnq_synth as S
from oracle import oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu

D = 128


def _workload(B, H, T, dtype, sub, kdist=S.K_MODERATE, seed=7, Hq=None):
    return S.Workload("case", B=B, Hkv=H, Hq=Hq or H, T=T, d=D, sub_dim=sub, dtype=dtype,
                      kdist=kdist, seed=seed)


def _inputs(w, which):
    x = S.keys(w) if which == "K" else S.values(w)
    io = S.to_io(x, w.dtype)
    return io, S.io_to_f64(io, w.dtype)


ENCODE_CASES = [
    # name, B, H, T, dtype, sub, kdist, tensor
    ("tiny-K-1bit-f32", 1, 1, 256, "f32", 8, S.K_MODERATE, "K"),
    ("tiny-V-1bit-f32", 1, 1, 256, "f32", 8, S.K_MODERATE, "V"),
    ("K-2bit-bf16-ragged", 2, 3, 1000, "bf16", 4, S.K_MODERATE, "K"),
    ("V-2bit-bf16-ragged", 2, 2, 777, "bf16", 4, S.K_MODERATE, "V"),
    ("K-1bit-bf16-ragged", 2, 2, 545, "bf16", 8, S.K_MODERATE, "K"),
    ("K-2bit-f32-strong-outliers", 1, 2, 1100, "f32", 4, S.K_STRONG, "K"),
    ("K-2bit-bf16-single-token", 1, 2, 1, "bf16", 4, S.K_MODERATE, "K"),
    # above the small-call size (1024 token-heads): the tensor-core 1-bit path with fp32 input
    ("K-1bit-f32-ragged", 2, 2, 300, "f32", 8, S.K_MODERATE, "K"),
    # one token-head past the small-call size: the persistent kernels on a single head
    ("K-2bit-bf16-1025", 1, 1, 1025, "bf16", 4, S.K_STRONG, "K"),
    ("K-1bit-bf16-1025", 1, 1, 1025, "bf16", 8, S.K_MODERATE, "K"),
]


@pytest.mark.parametrize("case", ENCODE_CASES, ids=[c[0] for c in ENCODE_CASES])
def test_encode_matches_oracle(codebooks, case):
    _, B, H, T, dtype, sub, kdist, which = case
    w = _workload(B, H, T, dtype, sub, kdist)
    io, x64 = _inputs(w, which)
    C = codebooks[sub]
    ora = O.encode(x64, C, want_w=True)
    cb = P.codebook(C)
    cache = nsnq.Cache.empty(B, H, T, sub)
    ws = nsnq.nsnq_encode(P.to_dev(io, dtype), cb, cache)
    torch.cuda.synchronize()
    n_mis, n_bad, worst = P.code_report(cache.codes.cpu().numpy(), ora["codes"], ora["w"], C)
    assert n_bad == 0, (n_mis, n_bad, worst)
    P.check_scales(cache.scales.cpu().numpy(), ora)
    P.check_shift(cache.shift.cpu().numpy(), ora["o"])
    th, sv, mismatch, timeout = nsnq.encode_stats(ws)
    assert mismatch == 0 and timeout == 0
    assert th <= max(4, B * H * T // 50)


def test_encode_given_shift_and_offset(codebooks):
    """Shift-given mode appends at an offset and reuses the stored o."""
    w = _workload(2, 2, 300, "bf16", 4)
    io, x64 = _inputs(w, "K")
    C = codebooks[4]
    o_given = (np.random.default_rng(1).standard_normal((2, 2, D)) * 0.3).astype(np.float32)
    ora = O.encode(x64, C, shift=o_given.astype(np.float64), want_w=True)
    cache = nsnq.Cache.empty(2, 2, 310, 4)
    cache.shift.copy_(torch.from_numpy(o_given))
    nsnq.nsnq_encode(P.to_dev(io, "bf16"), P.codebook(C), cache, t_offset=7,
                     shift_mode=nsnq.SHIFT_GIVEN)
    torch.cuda.synchronize()
    codes = cache.codes.cpu().numpy()
    _, n_bad, worst = P.code_report(codes[:, :, 7:307], ora["codes"], ora["w"], C)
    assert n_bad == 0, worst
    assert (codes[:, :, :7] == 0).all() and (codes[:, :, 307:] == 0).all()
    P.check_scales(cache.scales.cpu().numpy()[:, :, 7:307], ora)
    assert np.array_equal(cache.shift.cpu().numpy(), o_given)


def test_encode_strided_input(codebooks):
    """x given as a [B][T][H][D] buffer viewed as [B][H][T][D] (non-default strides)."""
    w = _workload(2, 4, 200, "bf16", 4)
    io, x64 = _inputs(w, "K")
    C = codebooks[4]
    dev = P.to_dev(io, "bf16").permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)
    assert dev.stride(2) == 4 * D
    ora = O.encode(x64, C, want_w=True)
    cache = nsnq.Cache.empty(2, 4, 200, 4)
    nsnq.nsnq_encode(dev, P.codebook(C), cache)
    torch.cuda.synchronize()
    _, n_bad, worst = P.code_report(cache.codes.cpu().numpy(), ora["codes"], ora["w"], C)
    assert n_bad == 0, worst


def test_encode_zero_tokens(codebooks):
    """All-zero tokens: s1 = 0, y = 0, z = -o (oracle reading for zero norm)."""
    w = _workload(1, 2, 64, "f32", 4)
    io, x64 = _inputs(w, "K")
    io[0, 0, 5] = 0.0
    io[0, 1, 0:3] = 0.0
    x64 = S.io_to_f64(io, "f32")
    C = codebooks[4]
    ora = O.encode(x64, C, want_w=True)
    cache = nsnq.Cache.empty(1, 2, 64, 4)
    nsnq.nsnq_encode(P.to_dev(io, "f32"), P.codebook(C), cache)
    torch.cuda.synchronize()
    _, n_bad, worst = P.code_report(cache.codes.cpu().numpy(), ora["codes"], ora["w"], C)
    assert n_bad == 0, worst
    sc = cache.scales.cpu().numpy()
    assert sc[0, 0, 5, 0] == 0 and (sc[0, 1, 0:3, 0] == 0).all()
    P.check_scales(sc, ora)


DEQUANT_CASES = [
    ("1bit", 1, 1, 256, "f32", 8, S.K_MODERATE),
    ("2bit-ragged", 2, 3, 333, "bf16", 4, S.K_MODERATE),
    ("2bit-strong", 1, 2, 500, "bf16", 4, S.K_STRONG),
]


@pytest.mark.parametrize("case", DEQUANT_CASES, ids=[c[0] for c in DEQUANT_CASES])
def test_dequant_matches_oracle(codebooks, case):
    _, B, H, T, dtype, sub, kdist = case
    w = _workload(B, H, T, dtype, sub, kdist)
    _, x64 = _inputs(w, "K")
    C = codebooks[sub]
    ora = O.encode(x64, C)
    s1, s2, o = O.stored(ora)
    ref = O.dequant(ora["codes"], s1, s2, o, C)
    cache = P.cache_from_oracle(ora, cap=T + 9, t_offset=4)
    out = nsnq.nsnq_dequant(cache, P.codebook(C), B, H, 4, T)
    torch.cuda.synchronize()
    P.check_dequant(out.cpu().numpy(), ref)
    part = nsnq.nsnq_dequant(cache, P.codebook(C), B, H, 4 + T // 3, T // 2)
    torch.cuda.synchronize()
    P.check_dequant(part.cpu().numpy(), ref[:, :, T // 3:T // 3 + T // 2])


ATTN_CASES = [
    # name, B, Hq, Hkv, T, ksub, vsub, q dtype, out dtype, seq_lens
    ("tiny-1bit", 1, 1, 1, 256, 8, 8, "f32", torch.float32, [256]),
    ("gqa4-2bit", 2, 8, 2, 700, 4, 4, "bf16", torch.bfloat16, [700, 333]),
    ("gqa8-2bit", 2, 16, 2, 600, 4, 4, "bf16", torch.float32, [600, 1]),
    ("gqa4-1bit", 2, 8, 2, 640, 8, 8, "bf16", torch.float32, [640, 639]),
    ("mixed-k2-v1-empty", 2, 4, 2, 513, 4, 8, "f32", torch.float32, [0, 513]),
    ("mixed-k1-v2", 1, 6, 3, 300, 8, 4, "f32", torch.float32, [300]),
    ("gqa2-many-splits", 1, 4, 2, 5000, 4, 4, "bf16", torch.float32, [4999]),
    ("mha", 2, 3, 3, 257, 4, 4, "bf16", torch.bfloat16, [257, 31]),
]


@pytest.mark.parametrize("case", ATTN_CASES, ids=[c[0] for c in ATTN_CASES])
def test_attention_matches_oracle(codebooks, case):
    _, B, Hq, Hkv, T, ksub, vsub, qdt, odt, lens = case
    w = _workload(B, Hkv, T, "bf16", 4, Hq=Hq)
    _, k64 = _inputs(w, "K")
    _, v64 = _inputs(w, "V")
    Ck, Cv = codebooks[ksub], codebooks[vsub]
    ok, ov = O.encode(k64, Ck), O.encode(v64, Cv)
    Kh = O.dequant(ok["codes"], *O.stored(ok), Ck)
    Vh = O.dequant(ov["codes"], *O.stored(ov), Cv)
    q_io = S.to_io(S.queries(w), qdt)
    q64 = S.io_to_f64(q_io, qdt)
    ref = O.attention(q64, Kh, Vh, lens)
    kc = P.cache_from_oracle(ok, cap=T + 5)
    vc = P.cache_from_oracle(ov, cap=T + 3)
    seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
    out = nsnq.nsnq_attn_decode(P.to_dev(q_io, qdt), kc, vc, P.codebook(Ck), P.codebook(Cv), seq,
                                max_len=T, Hkv=Hkv, out_dtype=odt)
    torch.cuda.synchronize()
    e, _ = P.attn_errors(P.out_to_np(out), ref, odt == torch.bfloat16)
    assert (e <= 1.0).all(), e.max()
    for b, L in enumerate(lens):
        if L == 0:
            assert (out[b] == 0).all()


def test_attention_single_token_is_value(codebooks):
    """A one-token context returns that token's dequantized value exactly-ish."""
    w = _workload(1, 2, 40, "bf16", 4, Hq=8)
    _, k64 = _inputs(w, "K")
    _, v64 = _inputs(w, "V")
    C = codebooks[4]
    ok, ov = O.encode(k64, C), O.encode(v64, C)
    Vh = O.dequant(ov["codes"], *O.stored(ov), C)
    q = torch.randn(1, 8, D, device="cuda")
    out = nsnq.nsnq_attn_decode(q, P.cache_from_oracle(ok), P.cache_from_oracle(ov),
                                P.codebook(C), P.codebook(C),
                                torch.tensor([1], dtype=torch.int32, device="cuda"), 40, Hkv=2,
                                out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref = np.repeat(Vh[0, :, 0], 4, axis=0)
    assert np.abs(out[0].cpu().numpy() - ref).max() < 1e-5 * np.abs(ref).max()


def test_pipeline_tiny_config(codebooks):
    """Tiny correctness config end to end on the GPU (encode K/V, one-query
    attention) against the oracle's encode -> dequant -> attention."""
    w = S.WORKLOADS["tiny"]
    C = codebooks[8]
    k_io = S.to_io(S.keys(w), "f32")
    v_io = S.to_io(S.values(w), "f32")
    q_io = S.to_io(S.queries(w), "f32")
    ok = O.encode(S.io_to_f64(k_io, "f32"), C)
    ov = O.encode(S.io_to_f64(v_io, "f32"), C)
    ref = O.attention(S.io_to_f64(q_io, "f32"), O.dequant(ok["codes"], *O.stored(ok), C),
                      O.dequant(ov["codes"], *O.stored(ov), C))
    cb = P.codebook(C)
    kc, vc = nsnq.Cache.empty(1, 1, 256, 8), nsnq.Cache.empty(1, 1, 256, 8)
    nsnq.nsnq_encode(P.to_dev(k_io, "f32"), cb, kc)
    nsnq.nsnq_encode(P.to_dev(v_io, "f32"), cb, vc)
    out = nsnq.nsnq_attn_decode(P.to_dev(q_io, "f32"), kc, vc, cb, cb,
                                torch.tensor([256], dtype=torch.int32, device="cuda"), 256, Hkv=1,
                                out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert np.array_equal(kc.codes.cpu().numpy(), ok["codes"])
    assert np.array_equal(vc.codes.cpu().numpy(), ov["codes"])
    e, _ = P.attn_errors(P.out_to_np(out), ref, False)
    assert (e <= 1.0).all(), e.max()


def _parse_index(idx: np.ndarray):
    hdr = idx[:64].view(np.uint32)
    n_cells = int(hdr[3])
    offs = idx[64:64 + 2 * (n_cells + 1)].view(np.uint16).astype(np.int64)
    start = 64 + ((2 * (n_cells + 1) + 15) // 16) * 16
    ents = idx[start:start + 4 * int(hdr[1])].view(np.uint16)   # pairs of entries
    return hdr, 2 * offs, ents


def _bins(x: np.ndarray) -> np.ndarray:
    """The index's binning of one coordinate: the number of edges (0, +-10/32, +-22/32,
    +-35/32, +-53/32) at or below it."""
    x = x.astype(np.float32)
    edges = (0.3125, 0.6875, 1.09375, 1.65625)
    return sum((x >= np.float32(e)).astype(np.int64) for e in sorted([-e for e in edges] + [0.0] + list(edges)))


def test_codebook_index_lists_contain_the_nearest(codebooks):
    """Grid-cell candidate lists of the 2-bit search index: for sampled points
    (standard normal, and heavy-tailed) the true nearest codeword (brute
    force) is in the point's cell list, each list is sorted by a valid lower
    bound of the distance over the cell, and the entry padding an odd list
    is farther than the nearest codeword."""
    C = codebooks[4]
    cb = P.codebook(C).prepare()
    idx = cb.index.cpu().numpy()
    hdr, offs, ents = _parse_index(idx)
    assert hdr[0] == 0x4E534E52 and hdr[2] == 0
    nb = 10
    assert hdr[3] == nb ** 4
    rng = np.random.default_rng(5)
    pts = np.concatenate([rng.standard_normal((20000, 4)), 3 * rng.standard_t(3, (5000, 4))])
    pts = np.clip(pts, -11.3, 11.3)
    b = _bins(pts)
    cell = ((b[:, 0] * nb + b[:, 1]) * nb + b[:, 2]) * nb + b[:, 3]
    d2 = ((pts[:, None, :] - C[None].astype(np.float64)) ** 2).sum(-1)
    nearest = d2.argmin(1)
    for i in range(len(pts)):
        lst = ents[offs[cell[i]]:offs[cell[i] + 1]]
        assert len(lst) % 2 == 0 and len(lst) > 0
        codes, lbq = lst & 0xFF, lst >> 8
        assert nearest[i] in codes, i
        assert (np.diff(lbq.astype(np.int64)) >= 0).all()
        assert (lbq[:-1] / 64.0 <= d2[i, codes[:-1]] + 1e-9).all()
        # the last entry is a listed codeword (valid bound) or the padding
        # (lbq 255, a codeword farther than the nearest everywhere in the cell)
        last = d2[i, codes[-1]]
        assert lbq[-1] / 64.0 <= last + 1e-9 or (lbq[-1] == 255 and last > d2[i, nearest[i]])


def test_encode_detects_index_of_another_codebook(codebooks):
    C = codebooks[4]
    other = P.codebook((C * np.float32(1.01)).astype(np.float32)).prepare()
    good = P.codebook(C)
    w = _workload(1, 2, 600, "bf16", 4)  # above the small-call size: the indexed search
    io, _ = _inputs(w, "K")
    x = P.to_dev(io, "bf16")
    cache = nsnq.Cache.empty(1, 2, 600, 4)
    ws = nsnq.nsnq_encode(x, nsnq.Codebook(good.centroids, other.index), cache)
    assert nsnq.encode_stats(ws)[2] != 0
    ws = nsnq.nsnq_encode(x, good, cache)
    assert nsnq.encode_stats(ws)[2] == 0


@pytest.mark.parametrize("sub,T,dtype,kdist", [(4, 700, "bf16", S.K_MODERATE), (8, 300, "f32", S.K_MODERATE),
                                                (4, 400, "bf16", S.K_STRONG)])
def test_encode_adaptive_scale_matches_oracle(codebooks, sub, T, dtype, kdist):
    """Scale adjustment (Methodology §3): same codes, s2 multiplied by
    ||w||^2 / (w . w_hat), against the oracle's fp64 value."""
    w = _workload(2, 2, T, dtype, sub, kdist)
    io, x64 = _inputs(w, "K")
    C = codebooks[sub]
    ora = O.encode(x64, C, want_w=True, adaptive_scale=True)
    cache = nsnq.Cache.empty(2, 2, T, sub)
    nsnq.nsnq_encode(P.to_dev(io, dtype), P.codebook(C), cache, flags=nsnq.ENCODE_ADAPTIVE_SCALE)
    torch.cuda.synchronize()
    _, n_bad, worst = P.code_report(cache.codes.cpu().numpy(), ora["codes"], ora["w"], C)
    assert n_bad == 0, worst
    P.check_scales(cache.scales.cpu().numpy(), ora)
    P.check_shift(cache.shift.cpu().numpy(), ora["o"])


@pytest.mark.parametrize("sub", [4, 8])
def test_encode_adaptive_scale_given_shift(codebooks, sub):
    """Scale adjustment with a given shift (the append path), a far-off shift
    included so that some tokens take the fp64 path."""
    w = _workload(1, 2, 600, "bf16", sub)  # above the small-call size
    io, x64 = _inputs(w, "K")
    C = codebooks[sub]
    o_given = (np.random.default_rng(3).standard_normal((1, 2, D)) * 0.3).astype(np.float32)
    ora = O.encode(x64, C, shift=o_given.astype(np.float64), want_w=True, adaptive_scale=True)
    cache = nsnq.Cache.empty(1, 2, 600, sub)
    cache.shift.copy_(torch.from_numpy(o_given))
    nsnq.nsnq_encode(P.to_dev(io, "bf16"), P.codebook(C), cache, shift_mode=nsnq.SHIFT_GIVEN,
                     flags=nsnq.ENCODE_ADAPTIVE_SCALE)
    torch.cuda.synchronize()
    _, n_bad, worst = P.code_report(cache.codes.cpu().numpy(), ora["codes"], ora["w"], C)
    assert n_bad == 0, worst
    P.check_scales(cache.scales.cpu().numpy(), ora)


ADAPT, DQF = nsnq.ENCODE_ADAPTIVE_SCALE, nsnq.ENCODE_DOUBLE_QUANT


@pytest.mark.parametrize("sub,dtype,B,H,T,flags,given", [
    (4, "bf16", 64, 8, 1, 0, True),        # one decode step's appends, 64 sequences
    (8, "bf16", 64, 8, 1, 0, True),
    (4, "f32", 1, 2, 300, 0, False),
    (8, "f32", 2, 2, 200, ADAPT, False),
    (4, "bf16", 2, 2, 200, DQF | ADAPT, False),
    (8, "bf16", 1, 4, 256, DQF, False),
    (4, "bf16", 4, 8, 32, ADAPT, True),     # exactly the small-call size
])
def test_small_call_encode_matches_oracle(codebooks, sub, dtype, B, H, T, flags, given):
    """Calls of at most 1024 token-heads take the one-warp-per-token-head fp64
    pass 2; codes, scales and (shift-compute mode) the shift against the
    oracle, for both bit rates, both input types, the scale adjustment and
    double quantization."""
    w = _workload(B, H, T, dtype, sub, S.K_STRONG if sub == 4 else S.K_MODERATE, seed=11)
    io, x64 = _inputs(w, "K")
    C = codebooks[sub]
    o_given = None
    if given:
        o_given = (np.random.default_rng(5).standard_normal((B, H, D)) * 0.3).astype(np.float32)
    ora = O.encode(x64, C, shift=None if o_given is None else o_given.astype(np.float64), want_w=True,
                   adaptive_scale=bool(flags & ADAPT), double_quant=bool(flags & DQF))
    cache = nsnq.Cache.empty(B, H, T, sub)
    if given:
        cache.shift.copy_(torch.from_numpy(o_given))
    nsnq.nsnq_encode(P.to_dev(io, dtype), P.codebook(C), cache,
                     shift_mode=nsnq.SHIFT_GIVEN if given else nsnq.SHIFT_COMPUTE, flags=flags)
    torch.cuda.synchronize()
    _, n_bad, worst = P.code_report(cache.codes.cpu().numpy(), ora["codes"], ora["w"], C)
    assert n_bad == 0, worst
    P.check_scales(cache.scales.cpu().numpy(), ora)
    if not given:
        P.check_shift(cache.shift.cpu().numpy(), ora["o"])


def test_small_given_call_resets_the_stats(codebooks):
    """A small shift-given call (no workspace memset) still leaves the
    workspace's counters zeroed for encode_stats()."""
    C = codebooks[4]
    other = P.codebook((C * np.float32(1.01)).astype(np.float32)).prepare()
    good = P.codebook(C)
    w = _workload(1, 2, 600, "bf16", 4)
    io, _ = _inputs(w, "K")
    x = P.to_dev(io, "bf16")
    cache = nsnq.Cache.empty(1, 2, 601, 4)
    ws = nsnq.nsnq_encode(x, nsnq.Codebook(good.centroids, other.index), cache)
    assert nsnq.encode_stats(ws)[2] != 0
    nsnq.nsnq_encode(x[:, :, :1], good, cache, t_offset=600, shift_mode=nsnq.SHIFT_GIVEN, workspace=ws)
    torch.cuda.synchronize()
    assert tuple(nsnq.encode_stats(ws)) == (0, 0, 0, 0)


@pytest.mark.parametrize("fill", [0xFF, 0x00, "random"])
def test_encode_with_a_garbage_index_completes_and_is_flagged(codebooks, fill):
    """An index buffer that is not an index (offsets past the lists, a wrong
    magic and hash) must not take the walk outside shared memory: the call
    completes, the mismatch flag is set, and a later call with the right
    index is exact again."""
    C = codebooks[4]
    good = P.codebook(C)
    n = int(nsnq.load().nsnq_codebook_index_bytes(4))
    if fill == "random":
        junk = torch.randint(0, 256, (n,), dtype=torch.int32, device="cuda",
                             generator=torch.Generator(device="cuda").manual_seed(9)).to(torch.uint8)
    else:
        junk = torch.full((n,), fill, dtype=torch.uint8, device="cuda")
    w = _workload(1, 2, 600, "bf16", 4)
    io, x64 = _inputs(w, "K")
    x = P.to_dev(io, "bf16")
    cache = nsnq.Cache.empty(1, 2, 600, 4)
    ws = nsnq.nsnq_encode(x, nsnq.Codebook(good.centroids, junk), cache)
    torch.cuda.synchronize()
    assert nsnq.encode_stats(ws)[2] != 0
    nsnq.nsnq_encode(x, good, cache, workspace=ws)
    torch.cuda.synchronize()
    assert nsnq.encode_stats(ws)[2] == 0
    ora = O.encode(x64, C, want_w=True)
    _, n_bad, worst = P.code_report(cache.codes.cpu().numpy(), ora["codes"], ora["w"], C)
    assert n_bad == 0, worst
