"""2-bit encode with the nearest codeword found by scoring all 256 codewords
on the tensor cores (ENCODE_TC_SEARCH, no search index): parity with the
oracle's fp64 argmin on ragged shapes and both input types, with the scale
adjustment and double quantization, and the same codes as the index walk at
the benchmark's full size."""
import numpy as np
import pytest
import torch

import attention_decode_b200 as nsnq
import nsnq_synth as S
from oracle import oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu

D = 128
TC = nsnq.ENCODE_TC_SEARCH


def _index_free(C):
    return nsnq.Codebook(torch.from_numpy(np.ascontiguousarray(C, dtype=np.float32)).cuda(), no_index=True)


CASES = [
    # name, B, H, T, dtype, kdist, tensor, extra flags
    ("K-bf16-ragged", 2, 3, 1000, "bf16", S.K_MODERATE, "K", 0),
    ("V-bf16-ragged", 2, 2, 777, "bf16", S.K_MODERATE, "V", 0),
    ("K-f32-strong-outliers", 1, 2, 1100, "f32", S.K_STRONG, "K", 0),
    ("K-bf16-1025", 1, 1, 1025, "bf16", S.K_STRONG, "K", 0),
    ("K-bf16-adaptive", 2, 2, 700, "bf16", S.K_MODERATE, "K", nsnq.ENCODE_ADAPTIVE_SCALE),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_tc_search_matches_oracle(codebooks, case):
    _, B, H, T, dtype, kdist, which, extra = case
    w = S.Workload("case", B=B, Hkv=H, Hq=H, T=T, d=D, sub_dim=4, dtype=dtype, kdist=kdist, seed=11)
    x = S.keys(w) if which == "K" else S.values(w)
    io = S.to_io(x, dtype)
    C = codebooks[4]
    ora = O.encode(S.io_to_f64(io, dtype), C, want_w=True,
                   adaptive_scale=bool(extra & nsnq.ENCODE_ADAPTIVE_SCALE))
    cache = nsnq.Cache.empty(B, H, T, 4)
    ws = nsnq.nsnq_encode(P.to_dev(io, dtype), _index_free(C), cache, flags=TC | extra)
    torch.cuda.synchronize()
    n_mis, n_bad, worst = P.code_report(cache.codes.cpu().numpy(), ora["codes"], ora["w"], C)
    assert n_bad == 0, (n_mis, n_bad, worst)
    P.check_scales(cache.scales.cpu().numpy(), ora)
    P.check_shift(cache.shift.cpu().numpy(), ora["o"])
    st = nsnq.encode_stats(ws)
    assert st.mma_timeout == 0 and st.index_mismatch == 0


def test_tc_search_with_double_quantization(codebooks):
    """Double quantization: s1 on the head's 16-level grid, the same as the
    walk path's (both are checked against the oracle elsewhere)."""
    B, H, T = 2, 2, 900
    w = S.Workload("case", B=B, Hkv=H, Hq=H, T=T, d=D, sub_dim=4, dtype="bf16", kdist=S.K_MODERATE, seed=12)
    x = P.to_dev(S.to_io(S.keys(w), "bf16"), "bf16")
    C = codebooks[4]
    caches = []
    for flags, cb in ((nsnq.ENCODE_DOUBLE_QUANT, P.codebook(C)), (nsnq.ENCODE_DOUBLE_QUANT | TC, _index_free(C))):
        c = nsnq.Cache.empty(B, H, T, 4)
        nsnq.nsnq_encode(x, cb, c, flags=flags)
        caches.append(c)
    torch.cuda.synchronize()
    assert torch.equal(caches[0].codes, caches[1].codes)
    assert torch.equal(caches[0].shift, caches[1].shift)
    # s1 is the same grid level; s2 is an fp32 norm summed in another order
    assert torch.equal(caches[0].scales[..., 0], caches[1].scales[..., 0])
    torch.testing.assert_close(caches[0].scales[..., 1], caches[1].scales[..., 1], rtol=2e-6, atol=0)


def test_tc_search_equals_index_walk_at_full_size(codebooks):
    """8 x 8 kv-heads x 4096 bf16 keys: both searches are exact (fp64
    re-decision of near ties), so the codes agree; the scales agree to the
    fp32 rounding of norms summed in another order."""
    w = S.WORKLOADS["encode-8x4096"]
    x = P.to_dev(S.to_io(S.keys(w), "bf16"), "bf16")
    B, H, T = w.B, w.Hkv, w.T
    C = codebooks[4]
    out = []
    for flags, cb in ((0, P.codebook(C)), (TC, _index_free(C))):
        c = nsnq.Cache.empty(B, H, T, 4)
        ws = nsnq.nsnq_encode(x, cb, c, flags=flags)
        torch.cuda.synchronize()
        st = nsnq.encode_stats(ws)
        assert st.mma_timeout == 0 and st.index_mismatch == 0
        out.append(c)
    n_diff = int((out[0].codes != out[1].codes).sum())
    assert n_diff == 0, n_diff
    torch.testing.assert_close(out[0].scales, out[1].scales, rtol=2e-6, atol=0)


def test_index_free_codebook_needs_the_flag(codebooks):
    cache = nsnq.Cache.empty(1, 2, 1500, 4)
    x = torch.randn(1, 2, 1500, D, device="cuda")
    with pytest.raises(nsnq.NSNQError) as ei:
        nsnq.nsnq_encode(x, _index_free(codebooks[4]), cache)
    assert ei.value.status == nsnq.NSNQ_ERR_INVALID_ARG
    assert "ENCODE_TC_SEARCH" in str(ei.value)
