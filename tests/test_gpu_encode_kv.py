"""GPU parity of the two-tensor encode (nsnq_encode_kv: a layer's keys and
values with the one global codebook of NSNQuant's Technical Summary,
Methodology §3, sharing the call's launches). Each tensor against the CPU
oracle on the same seeded inputs, over the paths a call can take (index walk,
tensor-core search, 1 bit, the small-call kernel, shift given at an offset,
double quantization, packed caches), and at the full benchmark size."""
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


def _w(B, H, T, dtype, sub, kdist=S.K_MODERATE, seed=23):
    return S.Workload("kv", B=B, Hkv=H, Hq=H, T=T, d=D, sub_dim=sub, dtype=dtype, kdist=kdist,
                      seed=seed)


def _kv_io(w):
    return S.to_io(S.keys(w), w.dtype), S.to_io(S.values(w), w.dtype)


def _check(cache, io, dtype, C, flags=0, o_given=None, t0=0):
    T = io.shape[2]
    ora = O.encode(S.io_to_f64(io, dtype), C, want_w=True, shift=o_given,
                   double_quant=bool(flags & DQ),
                   adaptive_scale=bool(flags & nsnq.ENCODE_ADAPTIVE_SCALE))
    codes = cache.codes[:, :, t0:t0 + T].cpu().numpy()
    n_mis, n_bad, worst = P.code_report(codes, ora["codes"], ora["w"], C)
    assert n_bad == 0, (n_mis, worst)
    if not cache.packed:
        P.check_scales(cache.scales[:, :, t0:t0 + T].cpu().numpy(), ora)
    if o_given is None:
        P.check_shift(cache.shift.cpu().numpy(), ora["o"])
    return ora


KV_CASES = [
    # name, B, H, T, dtype, sub, flags, kdist
    ("2bit-walk-bf16-ragged", 2, 3, 1000, "bf16", 4, 0, S.K_MODERATE),
    ("2bit-tc-search-bf16", 2, 2, 777, "bf16", 4, nsnq.ENCODE_TC_SEARCH, S.K_MODERATE),
    ("1bit-bf16-ragged", 2, 2, 545, "bf16", 8, 0, S.K_MODERATE),
    ("2bit-f32-strong-outliers", 1, 2, 1100, "f32", 4, 0, S.K_STRONG),
    ("2bit-adaptive", 2, 2, 400, "bf16", 4, nsnq.ENCODE_ADAPTIVE_SCALE, S.K_MODERATE),
    # 2 x 1 x 2 x 200 = 800 token-heads: the small-call kernel after pass 1
    ("2bit-small-call", 1, 2, 200, "bf16", 4, 0, S.K_STRONG),
    ("1bit-small-call", 1, 2, 100, "f32", 8, 0, S.K_MODERATE),
    # 2 x 513 token-heads: just above the small-call size, one head per tensor
    ("2bit-1026", 1, 1, 513, "bf16", 4, 0, S.K_STRONG),
]


@pytest.mark.parametrize("case", KV_CASES, ids=[c[0] for c in KV_CASES])
def test_encode_kv_matches_oracle(codebooks, case):
    _, B, H, T, dtype, sub, flags, kdist = case
    w = _w(B, H, T, dtype, sub, kdist)
    k_io, v_io = _kv_io(w)
    C = codebooks[sub]
    cb = P.codebook(C)
    if flags & nsnq.ENCODE_TC_SEARCH:
        cb = nsnq.Codebook(cb.centroids, no_index=True)
    kc, vc = nsnq.Cache.empty(B, H, T, sub), nsnq.Cache.empty(B, H, T, sub)
    ws = nsnq.nsnq_encode_kv(P.to_dev(k_io, dtype), P.to_dev(v_io, dtype), cb, kc, vc, flags=flags)
    torch.cuda.synchronize()
    _check(kc, k_io, dtype, C, flags)
    _check(vc, v_io, dtype, C, flags)
    th, sv, mismatch, timeout = nsnq.encode_stats(ws)
    assert mismatch == 0 and timeout == 0
    assert th <= max(8, 2 * B * H * T // 50)


def test_encode_kv_equals_two_calls(codebooks):
    """The pair call and two single calls give the same caches: codes equal
    (up to near ties, decided from o sums grouped by a different chunk plan),
    s1 and s2 equal to fp32 rounding, o within one fp32 ulp."""
    B, H, T = 3, 2, 2000
    w = _w(B, H, T, "bf16", 4, S.K_STRONG, seed=41)
    k_io, v_io = _kv_io(w)
    cb = P.codebook(codebooks[4])
    k, v = P.to_dev(k_io, "bf16"), P.to_dev(v_io, "bf16")
    kc, vc = nsnq.Cache.empty(B, H, T, 4), nsnq.Cache.empty(B, H, T, 4)
    nsnq.nsnq_encode_kv(k, v, cb, kc, vc)
    ks, vs = nsnq.Cache.empty(B, H, T, 4), nsnq.Cache.empty(B, H, T, 4)
    nsnq.nsnq_encode(k, cb, ks)
    nsnq.nsnq_encode(v, cb, vs)
    torch.cuda.synchronize()
    for a, b in ((kc, ks), (vc, vs)):
        agree = (a.codes == b.codes).float().mean().item()
        assert agree >= 1.0 - 1e-5, agree
        np.testing.assert_allclose(a.scales.cpu().numpy(), b.scales.cpu().numpy(), rtol=2e-6)
        sa, sb = a.shift.cpu().numpy(), b.shift.cpu().numpy()
        assert (np.abs(sa - sb) <= np.spacing(np.abs(sb))).all()


@pytest.mark.parametrize("T,sub", [(1, 4), (3, 8), (300, 4)])
def test_encode_kv_given_shift_at_offset(codebooks, T, sub):
    """Shift-given appends at an offset (a decode step's, T = 1, and a
    window flush): each tensor with its own stored o."""
    B, H, off = 2, 2, 11
    w = _w(B, H, T, "bf16", sub, seed=5)
    k_io, v_io = _kv_io(w)
    C = codebooks[sub]
    rng = np.random.default_rng(3)
    ok, ov = [(rng.standard_normal((B, H, D)) * s).astype(np.float32) for s in (0.4, 0.1)]
    kc, vc = nsnq.Cache.empty(B, H, off + T, sub), nsnq.Cache.empty(B, H, off + T, sub)
    kc.shift.copy_(torch.from_numpy(ok))
    vc.shift.copy_(torch.from_numpy(ov))
    nsnq.nsnq_encode_kv(P.to_dev(k_io, "bf16"), P.to_dev(v_io, "bf16"), P.codebook(C), kc, vc,
                        t_offset=off, shift_mode=nsnq.SHIFT_GIVEN)
    torch.cuda.synchronize()
    _check(kc, k_io, "bf16", C, o_given=ok.astype(np.float64), t0=off)
    _check(vc, v_io, "bf16", C, o_given=ov.astype(np.float64), t0=off)
    assert torch.equal(kc.shift.cpu(), torch.from_numpy(ok))
    assert torch.equal(vc.shift.cpu(), torch.from_numpy(ov))


@pytest.mark.parametrize("sub,packed", [(4, False), (4, True), (8, True)])
def test_encode_kv_double_quant(codebooks, sub, packed):
    """Double quantization: each tensor's own s1 grid and o levels; the packed
    form holds the same codes and grids as the unpacked one."""
    B, H, T = 2, 2, 701
    w = _w(B, H, T, "bf16", sub, seed=9)
    k_io, v_io = _kv_io(w)
    C = codebooks[sub]
    kc = nsnq.Cache.empty(B, H, T, sub, packed=packed)
    vc = nsnq.Cache.empty(B, H, T, sub, packed=packed)
    nsnq.nsnq_encode_kv(P.to_dev(k_io, "bf16"), P.to_dev(v_io, "bf16"), P.codebook(C), kc, vc,
                        flags=DQ)
    torch.cuda.synchronize()
    for cache, io in ((kc, k_io), (vc, v_io)):
        ora = _check(cache, io, "bf16", C, flags=DQ)
        g = cache.s1_grid.cpu().numpy().astype(np.float64)
        ulp = np.spacing(np.abs(ora["s1_grid"]).astype(np.float32)).astype(np.float64)
        assert (np.abs(g - ora["s1_grid"]) <= ulp).all()


def test_encode_kv_fullsize(codebooks):
    """The benchmark's step: keys and values of 8 sequences x 8 kv-heads x
    4096 tokens (bf16, 2 bit) in one call; sampled heads of both tensors
    against the oracle."""
    w = S.WORKLOADS["encode-8x4096"]
    C = codebooks[4]
    k_io, v_io = S.to_io(S.keys(w), "bf16"), S.to_io(S.values(w), "bf16")
    kc, vc = nsnq.Cache.empty(w.B, w.Hkv, w.T, 4), nsnq.Cache.empty(w.B, w.Hkv, w.T, 4)
    ws = nsnq.nsnq_encode_kv(P.to_dev(k_io, "bf16"), P.to_dev(v_io, "bf16"), P.codebook(C), kc, vc)
    torch.cuda.synchronize()
    for cache, io in ((kc, k_io), (vc, v_io)):
        for b, h in ((0, 0), (4, 6), (7, 7)):
            sl = io[b:b + 1, h:h + 1]
            one = nsnq.Cache(cache.codes[b:b + 1, h:h + 1], cache.scales[b:b + 1, h:h + 1],
                             cache.shift[b:b + 1, h:h + 1])
            _check(one, sl, "bf16", C)
    assert nsnq.encode_stats(ws).mma_timeout == 0


def test_decode_cache_with_one_codebook(codebooks):
    """DecodeCache with one codebook for keys and values encodes both caches
    with the pair call (prefill and window flushes): the caches equal those of
    a DecodeCache whose codebooks are distinct objects (two calls each)."""
    B, Hkv, T, steps, window = 2, 2, 300, 9, 4
    w = S.Workload("dc", B=B, Hkv=Hkv, Hq=8, T=T, d=D, sub_dim=4, dtype="bf16",
                   kdist=S.K_MODERATE, seed=12)
    kp, vp = (P.to_dev(S.to_io(f(w, T_total=T + steps, t1=T), "bf16"), "bf16")
              for f in (S.keys, S.values))
    kn, vn = (P.to_dev(S.to_io(f(w, T_total=T + steps, t0=T), "bf16"), "bf16")
              for f in (S.keys, S.values))
    cb = P.codebook(codebooks[4])
    caches = []
    for k_cb, v_cb in ((cb, cb), (cb, P.codebook(codebooks[4]))):
        dc = nsnq.DecodeCache(B, Hkv, T + steps, k_cb, v_cb, window=window)
        dc.prefill(kp, vp)
        for s in range(steps):
            dc.append(kn[:, :, s], vn[:, :, s])
        caches.append(dc)
    torch.cuda.synchronize()
    one, two = caches
    assert one.n_quant == two.n_quant == T + (steps // window) * window
    n = one.n_quant
    for a, b in ((one.k, two.k), (one.v, two.v)):
        agree = (a.codes[:, :, :n] == b.codes[:, :, :n]).float().mean().item()
        assert agree >= 1.0 - 1e-5, agree
        np.testing.assert_allclose(a.scales[:, :, :n].cpu().numpy(), b.scales[:, :, :n].cpu().numpy(),
                                   rtol=2e-6)
