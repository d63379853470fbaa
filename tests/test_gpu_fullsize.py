"""Parity at the full workload sizes, in the launch configuration the
benchmark times: the whole tensor goes through the CUDA path, and sampled
(batch, kv-head) slices are checked against the oracle, which computes them
one by one."""
import numpy as np
import pytest
import torch

import attention_decode_b200 as nsnq
import nsnq_synth as S
from oracle import oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu


def _check_encode_slice(cache, b, h, x64_slice, C, o_given=None):
    ora = O.encode(x64_slice, C, shift=o_given, want_w=True)
    T = x64_slice.shape[2]
    codes = cache.codes[b:b + 1, h:h + 1, :T].cpu().numpy()
    n_mis, n_bad, worst = P.code_report(codes, ora["codes"], ora["w"], C)
    assert n_bad == 0, (b, h, n_mis, worst)
    P.check_scales(cache.scales[b:b + 1, h:h + 1, :T].cpu().numpy(), ora)
    if o_given is None:
        P.check_shift(cache.shift[b:b + 1, h:h + 1].cpu().numpy(), ora["o"])
    return ora, n_mis


def test_fullsize_encode_llama3_8b_layer(codebooks):
    """8 sequences x 8 kv-heads x 4096 prompt tokens, bf16, 2 bit."""
    w = S.WORKLOADS["encode-8x4096"]
    C = codebooks[4]
    cb = P.codebook(C)
    for which in ("K", "V"):
        x64 = S.keys(w) if which == "K" else S.values(w)
        io = S.to_io(x64, "bf16")
        x64 = S.io_to_f64(io, "bf16")
        cache = nsnq.Cache.empty(w.B, w.Hkv, w.T, 4)
        nsnq.nsnq_encode(P.to_dev(io, "bf16"), cb, cache)
        torch.cuda.synchronize()
        for b, h in ((0, 0), (5, 3), (7, 7)):
            _check_encode_slice(cache, b, h, x64[b:b + 1, h:h + 1], C)


def _random_cache(B, H, cap, sub, gen):
    c = nsnq.Cache.empty(B, H, cap, sub)
    c.codes.copy_(torch.randint(0, 256, c.codes.shape, generator=gen, device="cuda",
                                dtype=torch.int32).to(torch.uint8))
    s1 = torch.exp(0.5 * torch.randn(B, H, cap, generator=gen, device="cuda")) * 1.7
    s2 = 0.4 + 0.3 * torch.rand(B, H, cap, generator=gen, device="cuda")
    c.scales.copy_(torch.stack([s1, s2], -1))
    c.shift.copy_(torch.randn(B, H, 128, generator=gen, device="cuda"))
    return c


def _attention_case(w, codebooks, samples, ksub, vsub):
    """Full-size caches (random codes everywhere except the sampled slices,
    which hold the oracle's encoding of the seeded K/V); full-size launch;
    the sampled heads' outputs are compared with the oracle's attention."""
    gen = torch.Generator(device="cuda")
    gen.manual_seed(w.seed)
    Ck, Cv = codebooks[ksub], codebooks[vsub]
    kc = _random_cache(w.B, w.Hkv, w.T, ksub, gen)
    vc = _random_cache(w.B, w.Hkv, w.T, vsub, gen)
    refs = {}
    for b, h in samples:
        k64 = S.io_to_f64(S.to_io(S.keys(w, b0=b, b1=b + 1)[:, h:h + 1], "bf16"), "bf16")
        v64 = S.io_to_f64(S.to_io(S.values(w, b0=b, b1=b + 1)[:, h:h + 1], "bf16"), "bf16")
        ok, ov = O.encode(k64, Ck), O.encode(v64, Cv)
        for cache, enc in ((kc, ok), (vc, ov)):
            cache.codes[b, h] = torch.from_numpy(enc["codes"][0, 0]).cuda()
            cache.scales[b, h] = torch.from_numpy(
                np.stack([enc["s1"][0, 0], enc["s2"][0, 0]], -1).astype(np.float32)).cuda()
            cache.shift[b, h] = torch.from_numpy(enc["o"][0, 0].astype(np.float32)).cuda()
        refs[(b, h)] = (O.dequant(ok["codes"], *O.stored(ok), Ck),
                        O.dequant(ov["codes"], *O.stored(ov), Cv))
    q_io = S.to_io(S.queries(w), "bf16")
    q64 = S.io_to_f64(q_io, "bf16")
    seq = torch.full((w.B,), w.T, dtype=torch.int32, device="cuda")
    out = nsnq.nsnq_attn_decode(P.to_dev(q_io, "bf16"), kc, vc, P.codebook(Ck), P.codebook(Cv),
                                seq, w.T, Hkv=w.Hkv, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    got = P.out_to_np(out)
    G = w.Hq // w.Hkv
    for (b, h), (Kh, Vh) in refs.items():
        ref = O.attention(q64[b:b + 1, h * G:(h + 1) * G], Kh, Vh)
        e, _ = P.attn_errors(got[b:b + 1, h * G:(h + 1) * G], ref, True)
        assert (e <= 1.0).all(), (b, h, e.max())


@pytest.mark.parametrize("name,ksub", [("decode-16x32k-2b", 4), ("decode-16x32k-1b", 8)])
def test_fullsize_attention_gqa4_32k(codebooks, name, ksub):
    _attention_case(S.WORKLOADS[name], codebooks, [(3, 5), (15, 0)], ksub, ksub)


def test_fullsize_attention_serving_gqa8(codebooks):
    _attention_case(S.WORKLOADS["serving-64x8k"], codebooks, [(10, 2), (63, 7)], 4, 4)


def test_fullsize_long_context_encode_and_append(codebooks):
    """128k-token prompt (strong outliers) encoded in one call, then decode
    steps that append one token each with the prompt's shift, then attention
    over prompt + appended tokens for one sampled kv-head."""
    w = S.WORKLOADS["long-128k"]
    C = codebooks[4]
    cb = P.codebook(C)
    steps = 3
    cap = w.T + steps
    h = 6
    caches, refs = [], []
    for which in ("K", "V"):
        x64 = S.keys(w) if which == "K" else S.values(w)
        io = S.to_io(x64, "bf16")
        cache = nsnq.Cache.empty(1, w.Hkv, cap, 4)
        nsnq.nsnq_encode(P.to_dev(io, "bf16"), cb, cache)
        torch.cuda.synchronize()
        x_h = S.io_to_f64(io[:, h:h + 1], "bf16")
        del x64, io
        ora, _ = _check_encode_slice(cache, 0, h, x_h, C)
        # From here on the sampled head holds the oracle's prompt encoding, so
        # the appended tokens on both sides use the same stored shift.
        o32 = ora["o"].astype(np.float32)
        cache.codes[0, h, :w.T] = torch.from_numpy(ora["codes"][0, 0]).cuda()
        cache.scales[0, h, :w.T] = torch.from_numpy(
            np.stack([ora["s1"][0, 0], ora["s2"][0, 0]], -1).astype(np.float32)).cuda()
        cache.shift[0, h] = torch.from_numpy(o32[0, 0]).cuda()
        # decode steps: one new token per call, shift given (the prompt's stored o)
        if which == "K":
            new = S.keys(w, T_total=cap, t0=w.T, t1=cap, stream=S.STREAM_APPEND_K)
        else:
            new = S.values(w, T_total=cap, t0=w.T, t1=cap, stream=S.STREAM_APPEND_V)
        new_io = S.to_io(new, "bf16")
        for s in range(steps):
            nsnq.nsnq_encode(P.to_dev(np.ascontiguousarray(new_io[:, :, s:s + 1]), "bf16"), cb,
                             cache, t_offset=w.T + s, shift_mode=nsnq.SHIFT_GIVEN)
        torch.cuda.synchronize()
        ora_new = O.encode(S.io_to_f64(new_io[:, h:h + 1], "bf16"), C,
                           shift=o32.astype(np.float64), want_w=True)
        _, n_bad, worst = P.code_report(cache.codes[0:1, h:h + 1, w.T:cap].cpu().numpy(),
                                        ora_new["codes"], ora_new["w"], C)
        assert n_bad == 0, worst
        P.check_scales(cache.scales[0:1, h:h + 1, w.T:cap].cpu().numpy(), ora_new)
        full = {k: np.concatenate([ora[k], ora_new[k]], axis=2) for k in ("codes", "s1", "s2")}
        full["o"] = ora["o"]
        cache.codes[0, h] = torch.from_numpy(full["codes"][0, 0]).cuda()
        cache.scales[0, h] = torch.from_numpy(
            np.stack([full["s1"][0, 0], full["s2"][0, 0]], -1).astype(np.float32)).cuda()
        caches.append(cache)
        refs.append(O.dequant(full["codes"], *O.stored(full), C))
    q_io = S.to_io(S.queries(w), "bf16")
    out = nsnq.nsnq_attn_decode(P.to_dev(q_io, "bf16"), caches[0], caches[1], cb, cb,
                                torch.tensor([cap], dtype=torch.int32, device="cuda"), cap,
                                Hkv=w.Hkv, out_dtype=torch.float32)
    torch.cuda.synchronize()
    G = w.Hq // w.Hkv
    ref = O.attention(S.io_to_f64(q_io, "bf16")[:, h * G:(h + 1) * G], refs[0], refs[1])
    e, _ = P.attn_errors(P.out_to_np(out)[:, h * G:(h + 1) * G], ref, False)
    assert (e <= 1.0).all(), e.max()


def test_fullsize_encode_1bit_tensor_core_loop(codebooks):
    """8 sequences x 8 kv-heads x 4096 tokens, bf16, 1 bit (g = 8): 32768
    tiles of the tensor-core kernel, so every CTA of its persistent grid runs
    dozens of tiles (mbarrier phase, TMEM reuse and A-operand overwrite carried
    from tile to tile). Sampled heads from the first, middle and last tiles of
    the grid's loop against the oracle; the MMA-timeout flag must stay 0."""
    w = S.WORKLOADS["encode-8x4096"]
    C = codebooks[8]
    cb = P.codebook(C)
    for which in ("K", "V"):
        x64 = S.keys(w) if which == "K" else S.values(w)
        io = S.to_io(x64, "bf16")
        x64 = S.io_to_f64(io, "bf16")
        cache = nsnq.Cache.empty(w.B, w.Hkv, w.T, 8)
        ws = nsnq.nsnq_encode(P.to_dev(io, "bf16"), cb, cache)
        torch.cuda.synchronize()
        st = nsnq.encode_stats(ws)
        assert st.mma_timeout == 0 and st.index_mismatch == 0, st
        for b, h in ((0, 0), (3, 6), (7, 7)):
            _check_encode_slice(cache, b, h, x64[b:b + 1, h:h + 1], C)


@pytest.mark.parametrize("name,sub", [("decode-16x32k-1b", 8), ("decode-16x32k-2b", 4)])
def test_fullsize_attention_over_gpu_encoded_cache(codebooks, name, sub):
    """decode-16x32k with the cache built by the GPU encode: K and V
    (16 x 8 kv-heads x 32768 tokens each, drawn on the device) are encoded in
    one call per tensor (4.2 M token-heads; at 1 bit the tensor-core kernel's
    full persistent loop), then decode attention runs over them. For sampled
    (sequence, kv-head) slices the GPU codes, scales and shift are checked
    against the oracle's encoding of the same bf16 inputs, and the attention
    output against the oracle's attention over the GPU's own codes, scales
    and shift."""
    w = S.WORKLOADS[name]
    C = codebooks[sub]
    cb = P.codebook(C)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(w.seed)
    chans, signs = w.kdist.channels(128)
    bias = torch.zeros(128, device="cuda")
    bias[chans] = torch.tensor(signs, device="cuda") * w.kdist.bias
    samples = [(2, 1), (15, 7)]
    caches, slices = {}, {}
    for which in ("K", "V"):
        z = torch.randn(w.B, w.Hkv, w.T, 128, generator=gen, device="cuda")
        if which == "K":
            s = torch.exp(w.kdist.sigma * torch.randn(w.B, w.Hkv, w.T, 1, generator=gen,
                                                      device="cuda"))
            z = (z + bias) * s
        x = z.to(torch.bfloat16)
        del z
        cache = nsnq.Cache.empty(w.B, w.Hkv, w.T, sub)
        ws = nsnq.nsnq_encode(x, cb, cache)
        torch.cuda.synchronize()
        st = nsnq.encode_stats(ws)
        assert st.mma_timeout == 0 and st.index_mismatch == 0, st
        for b, h in samples:
            slices[(which, b, h)] = x[b:b + 1, h:h + 1].float().cpu().numpy().astype(np.float64)
        del x
        caches[which] = cache
    q = torch.randn(w.B, w.Hq, 128, generator=gen, device="cuda").to(torch.bfloat16)
    seq = torch.full((w.B,), w.T, dtype=torch.int32, device="cuda")
    out = nsnq.nsnq_attn_decode(q, caches["K"], caches["V"], cb, cb, seq, w.T, Hkv=w.Hkv,
                                out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    got = P.out_to_np(out)
    q64 = q.float().cpu().numpy().astype(np.float64)
    G = w.Hq // w.Hkv
    for b, h in samples:
        deq = []
        for which in ("K", "V"):
            cache = caches[which]
            _check_encode_slice(cache, b, h, slices[(which, b, h)], C)
            codes = cache.codes[b:b + 1, h:h + 1].cpu().numpy()
            sc = cache.scales[b:b + 1, h:h + 1].cpu().numpy()
            o = cache.shift[b:b + 1, h:h + 1].cpu().numpy()
            deq.append(O.dequant(codes, sc[..., 0], sc[..., 1], o, C))
        ref = O.attention(q64[b:b + 1, h * G:(h + 1) * G], deq[0], deq[1])
        e, _ = P.attn_errors(got[b:b + 1, h * G:(h + 1) * G], ref, True)
        assert (e <= 1.0).all(), (b, h, e.max())
