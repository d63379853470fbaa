"""GPU parity of the full-precision residual window (NSNQuant Technical
Summary, Methodology §4, Implementation Details, Residuals): the window
write, attention over [quantized || residual], and the lock-step decode loop
with flushes, each against the CPU oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

import attention_decode_b200 as nsnq
import nsnq_synth as S
from oracle import oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu

D = 128


def _w(B, Hkv, Hq, T, seed=11, dtype="bf16"):
    return S.Workload("res", B=B, Hkv=Hkv, Hq=Hq, T=T, d=D, sub_dim=4, dtype=dtype,
                      kdist=S.K_MODERATE, seed=seed)


def _torch_dtype(dt):
    return torch.bfloat16 if dt == "bf16" else torch.float32


@pytest.mark.parametrize("xdt,bdt", [("bf16", "bf16"), ("f32", "bf16"), ("f32", "f32"),
                                     ("bf16", "f32")])
def test_residual_write_is_an_exact_copy(xdt, bdt):
    """Rows land at [t_offset, t_offset + T) of every (batch, head); fp32 to
    bf16 rounds to nearest even (torch's conversion), other pairs are exact;
    rows outside the range stay untouched. x is read through [B][T][H][D]
    strides."""
    w = _w(3, 4, 4, 5)
    x = P.to_dev(S.to_io(S.keys(w), xdt), xdt)            # [B][H][T][D]
    xs = x.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)  # strided view
    buf = torch.full((3, 4, 12, D), 7.0, dtype=_torch_dtype(bdt), device="cuda")
    nsnq.nsnq_residual_write(xs, buf, t_offset=6)
    torch.cuda.synchronize()
    ref = x.to(_torch_dtype(bdt))
    assert torch.equal(buf[:, :, 6:11], ref)
    assert (buf[:, :, :6] == 7).all() and (buf[:, :, 11:] == 7).all()


RES_CASES = [
    # name, B, Hq, Hkv, T (quantized cap), quantized lens, residual cap, residual lens, ksub, vsub
    ("gqa4-ragged", 5, 8, 2, 400, [400, 0, 77, 0, 311], 16, [0, 16, 5, 0, 9], 4, 4),
    ("mha-chunked-window", 2, 4, 4, 300, [300, 123], 300, [290, 257], 4, 8),
    ("gqa8-1bit", 2, 16, 2, 500, [500, 1], 64, [64, 63], 8, 8),
]


@pytest.mark.parametrize("rdt", ["bf16", "f32"])
@pytest.mark.parametrize("case", RES_CASES, ids=[c[0] for c in RES_CASES])
def test_attention_with_residual_matches_oracle(codebooks, case, rdt):
    _, B, Hq, Hkv, T, lens, R, rlens, ksub, vsub = case
    w = _w(B, Hkv, Hq, T)
    Ck, Cv = codebooks[ksub], codebooks[vsub]
    ok = O.encode(S.io_to_f64(S.to_io(S.keys(w), "bf16"), "bf16"), Ck)
    ov = O.encode(S.io_to_f64(S.to_io(S.values(w), "bf16"), "bf16"), Cv)
    Kh = O.dequant(ok["codes"], *O.stored(ok), Ck)
    Vh = O.dequant(ov["codes"], *O.stored(ov), Cv)
    # residual tokens: the next R tokens of the same streams
    kr_io = S.to_io(S.keys(w, t0=T, t1=T + R, T_total=T + R), rdt)
    vr_io = S.to_io(S.values(w, t0=T, t1=T + R, T_total=T + R), rdt)
    q_io = S.to_io(S.queries(w), "bf16")
    ref = O.attention_with_residual(S.io_to_f64(q_io, "bf16"), Kh, Vh, lens,
                                    S.io_to_f64(kr_io, rdt), S.io_to_f64(vr_io, rdt), rlens)
    res = nsnq.Residual(P.to_dev(kr_io, rdt), P.to_dev(vr_io, rdt),
                        torch.tensor(rlens, dtype=torch.int32, device="cuda"))
    out = nsnq.nsnq_attn_decode_res(P.to_dev(q_io, "bf16"), P.cache_from_oracle(ok),
                                    P.cache_from_oracle(ov), P.codebook(Ck), P.codebook(Cv),
                                    torch.tensor(lens, dtype=torch.int32, device="cuda"), T, Hkv,
                                    res, out_dtype=torch.float32)
    torch.cuda.synchronize()
    e, _ = P.attn_errors(P.out_to_np(out), ref, False)
    assert (e <= 1.0).all(), e.max()
    for b in range(B):
        if lens[b] == 0 and rlens[b] == 0:
            assert (out[b] == 0).all()


def test_residual_lengths_are_clamped_to_the_window(codebooks):
    """A residual length outside [0, cap] reads as its nearest end."""
    w = _w(2, 1, 2, 50)
    C = codebooks[4]
    ok = O.encode(S.io_to_f64(S.to_io(S.keys(w), "bf16"), "bf16"), C)
    ov = O.encode(S.io_to_f64(S.to_io(S.values(w), "bf16"), "bf16"), C)
    kr = P.to_dev(S.to_io(S.keys(w, t0=50, t1=58, T_total=58), "bf16"), "bf16")
    vr = P.to_dev(S.to_io(S.values(w, t0=50, t1=58, T_total=58), "bf16"), "bf16")
    q = P.to_dev(S.to_io(S.queries(w), "bf16"), "bf16")
    args = (P.cache_from_oracle(ok), P.cache_from_oracle(ov), P.codebook(C), P.codebook(C),
            torch.tensor([50, 50], dtype=torch.int32, device="cuda"), 50, 1)
    a = nsnq.nsnq_attn_decode_res(q, *args, nsnq.Residual(kr, vr, torch.tensor(
        [100, -3], dtype=torch.int32, device="cuda")), out_dtype=torch.float32)
    b = nsnq.nsnq_attn_decode_res(q, *args, nsnq.Residual(kr, vr, torch.tensor(
        [8, 0], dtype=torch.int32, device="cuda")), out_dtype=torch.float32)
    c = nsnq.nsnq_attn_decode(q, *args, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert torch.equal(b[1], c[1])  # an empty window is the plain path, bit for bit


@pytest.mark.parametrize("window,steps,flags", [(8, 19, nsnq.ENCODE_DEFAULT),
                                                (5, 11, nsnq.ENCODE_ADAPTIVE_SCALE)])
def test_decode_loop_matches_oracle(codebooks, window, steps, flags):
    """Prefill, then `steps` decode steps with a window of `window` tokens:
    every step's output and the final caches (flushed tokens included)
    against the oracle's serving loop."""
    B, Hkv, Hq, T = 2, 2, 8, 100
    w = _w(B, Hkv, Hq, T, seed=5)
    Ck, Cv = codebooks[4], codebooks[8]
    kp = S.to_io(S.keys(w, T_total=T + steps, t1=T), "bf16")
    vp = S.to_io(S.values(w, T_total=T + steps, t1=T), "bf16")
    kn = S.to_io(S.keys(w, T_total=T + steps, t0=T), "bf16")
    vn = S.to_io(S.values(w, T_total=T + steps, t0=T), "bf16")
    qs = [S.to_io(S.queries(w, step=s), "bf16") for s in range(steps)]
    f = lambda a: S.io_to_f64(a, "bf16")
    adaptive = flags == nsnq.ENCODE_ADAPTIVE_SCALE
    outs, st = O.decode_with_residual(f(kp), f(vp), f(kn), f(vn), np.stack([f(q) for q in qs]),
                                      Ck, Cv, R=window, adaptive_scale=adaptive)
    dc = nsnq.DecodeCache(B, Hkv, T + steps, P.codebook(Ck), P.codebook(Cv), window=window,
                          flags=flags)
    dc.prefill(P.to_dev(kp, "bf16"), P.to_dev(vp, "bf16"))
    kn_d, vn_d = P.to_dev(kn, "bf16"), P.to_dev(vn, "bf16")
    got = []
    for s in range(steps):
        dc.append(kn_d[:, :, s], vn_d[:, :, s])
        got.append(P.out_to_np(dc.attend(P.to_dev(qs[s], "bf16"), out_dtype=torch.float32)))
    torch.cuda.synchronize()
    assert dc.n_quant == T + (steps // window) * window and dc.n_res == steps % window
    for s in range(steps):
        e, _ = P.attn_errors(got[s], outs[s], False)
        assert (e <= 1.0).all(), (s, e.max())
    nq = dc.n_quant
    for name, cache, C, x in (("K", dc.k, Ck, np.concatenate([kp, kn], 2)),
                              ("V", dc.v, Cv, np.concatenate([vp, vn], 2))):
        wref = np.concatenate([O.encode(f(x[:, :, :T]), C, want_w=True)["w"],
                               O.encode(f(x[:, :, T:nq]), C, shift=st[name]["o"],
                                        want_w=True)["w"]], 2)
        _, n_bad, worst = P.code_report(cache.codes[:, :, :nq].cpu().numpy(), st[name]["codes"],
                                        wref, C)
        assert n_bad == 0, (name, worst)
        P.check_scales(cache.scales[:, :, :nq].cpu().numpy(), st[name])
