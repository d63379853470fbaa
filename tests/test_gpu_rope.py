"""GPU parity of decode attention over keys quantized before RoPE (NSNQuant
Technical Summary, Methodology §4, Implementation Details): the kernel
dequantizes and rotates every key to its position; the oracle rotates its
dequantized keys and runs plain attention."""
import numpy as np
import pytest
import torch

import attention_decode_b200 as nsnq
import nsnq_synth as S
from oracle import oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu

D = 128

CASES = [
    # name, B, Hq, Hkv, T, ksub, vsub, q dtype, out dtype, seq_lens, rope base
    ("gqa4-2bit", 2, 8, 2, 700, 4, 4, "bf16", torch.float32, [700, 333], 10000.0),
    ("gqa8-1bit-keys", 2, 16, 2, 600, 8, 4, "bf16", torch.float32, [600, 1], 500000.0),
    ("mha-mixed", 2, 3, 3, 257, 4, 8, "f32", torch.bfloat16, [257, 31], 10000.0),
    ("gqa2-empty", 2, 4, 2, 300, 4, 4, "bf16", torch.float32, [0, 300], 10000.0),
    ("gqa4-many-splits", 1, 4, 1, 5000, 4, 4, "bf16", torch.float32, [4999], 10000.0),
    ("gqa4-32k-positions", 1, 4, 1, 32768, 4, 4, "bf16", torch.float32, [32768], 500000.0),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_rope_attention_matches_oracle(codebooks, case):
    _, B, Hq, Hkv, T, ksub, vsub, qdt, odt, lens, base = case
    w = S.Workload("rope", B=B, Hkv=Hkv, Hq=Hq, T=T, d=D, sub_dim=4, dtype="bf16",
                   kdist=S.K_MODERATE, seed=13)
    Ck, Cv = codebooks[ksub], codebooks[vsub]
    ok = O.encode(S.io_to_f64(S.to_io(S.keys(w), "bf16"), "bf16"), Ck)
    ov = O.encode(S.io_to_f64(S.to_io(S.values(w), "bf16"), "bf16"), Cv)
    Kh = O.dequant(ok["codes"], *O.stored(ok), Ck)
    Vh = O.dequant(ov["codes"], *O.stored(ov), Cv)
    q_io = S.to_io(S.queries(w), qdt)
    ref = O.attention_rope(S.io_to_f64(q_io, qdt), Kh, Vh, lens, base=base)
    out = nsnq.nsnq_attn_decode_rope(P.to_dev(q_io, qdt), P.cache_from_oracle(ok, cap=T + 3),
                                     P.cache_from_oracle(ov, cap=T + 1), P.codebook(Ck),
                                     P.codebook(Cv), torch.tensor(lens, dtype=torch.int32,
                                                                  device="cuda"),
                                     T, Hkv=Hkv, rope_base=base, out_dtype=odt)
    torch.cuda.synchronize()
    e, _ = P.attn_errors(P.out_to_np(out), ref, odt == torch.bfloat16)
    assert (e <= 1.0).all(), e.max()
    for b, L in enumerate(lens):
        if L == 0:
            assert (out[b] == 0).all()


def test_rope_at_position_zero_only_is_the_plain_kernel(codebooks):
    """A one-token context sits at position 0, where the rotation is the
    identity: the output is that token's value, as in the plain kernel."""
    w = S.Workload("rope0", B=1, Hkv=2, Hq=8, T=40, d=D, sub_dim=4, dtype="bf16",
                   kdist=S.K_MODERATE, seed=3)
    C = codebooks[4]
    ok = O.encode(S.io_to_f64(S.to_io(S.keys(w), "bf16"), "bf16"), C)
    ov = O.encode(S.io_to_f64(S.to_io(S.values(w), "bf16"), "bf16"), C)
    q = torch.randn(1, 8, D, device="cuda")
    args = (q, P.cache_from_oracle(ok), P.cache_from_oracle(ov), P.codebook(C), P.codebook(C),
            torch.tensor([1], dtype=torch.int32, device="cuda"), 40)
    a = nsnq.nsnq_attn_decode_rope(*args, Hkv=2, out_dtype=torch.float32)
    b = nsnq.nsnq_attn_decode(*args, Hkv=2, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.allclose(a, b, rtol=1e-5, atol=1e-6)
