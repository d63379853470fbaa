"""GPU parity on inputs built to sit on Voronoi boundaries of the codebook.

Each token is constructed backwards from a target transformed vector w: one
sub-vector is put at the midpoint of two neighbouring codewords (a pair whose
midpoint has exactly those two as its nearest codewords) plus an offset along
their difference of 1e-7 .. 1e-3 of its length, some tokens also carry a
coordinate near +-11 in another sub-vector, and the remaining coordinates fill
|w| up to sqrt(d). Then x = s1 (s2 H w + o) for a fixed stored shift o. The
GPU codes must equal the oracle's fp64 argmin of the same fp32 input except
where the oracle's own relative gap is below the 1e-6 tie rule; with offsets
on both sides of that rule this exercises the fp32 decision, the near-tie
band and the fp64 re-decision of every encode path (small calls, the 2-bit
indexed walk, the 1-bit and 2-bit tensor-core scores)."""
import numpy as np
import pytest
import scipy.linalg
import torch

import attention_decode_b200 as nsnq
from oracle import oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu

D = 128


def _boundary_pairs(C: np.ndarray, rng, n: int):
    """Codeword pairs (a, b) whose midpoint has a and b as its two nearest codewords."""
    C64 = C.astype(np.float64)
    out = []
    for a in rng.permutation(len(C)):
        d = ((C64 - C64[a]) ** 2).sum(1)
        d[a] = np.inf
        b = int(np.argmin(d))
        m = 0.5 * (C64[a] + C64[b])
        dm = ((C64 - m) ** 2).sum(1)
        order = np.argsort(dm)
        if set(order[:2]) == {a, b} and dm[order[2]] > dm[order[0]] * (1 + 1e-2):
            out.append((int(a), b))
        if len(out) == n:
            break
    return out


def _near_tie_tokens(C: np.ndarray, n_tok: int, seed: int):
    """fp32 tokens [n_tok][D] and the fixed shift o [D] they were built for."""
    g = C.shape[1]
    J = D // g
    rng = np.random.default_rng(seed)
    H = scipy.linalg.hadamard(D).astype(np.float64) / np.sqrt(D)
    o = 0.25 * rng.standard_normal(D)
    pairs = _boundary_pairs(C, rng, 64)
    offsets = [s * 10.0 ** e for e in (-7, -6.5, -6, -5.5, -5, -4, -3) for s in (1, -1)]
    xs = []
    for t in range(n_tok):
        a, b = pairs[t % len(pairs)]
        ca, cb = C[a].astype(np.float64), C[b].astype(np.float64)
        dirn = (cb - ca) / np.linalg.norm(cb - ca)
        eps = offsets[t % len(offsets)] * np.linalg.norm(cb - ca)
        w = rng.standard_normal(D)
        j = int(rng.integers(J))
        w[j * g:(j + 1) * g] = 0.5 * (ca + cb) + eps * dirn
        fixed = np.zeros(D, dtype=bool)
        fixed[j * g:(j + 1) * g] = True
        if t % 3 == 0:  # an outlier coordinate in another sub-vector
            k = int((j * g + g + rng.integers(D - g)) % D)
            w[k] = 11.0 * (1 if rng.random() < 0.5 else -1)
            fixed[k] = True
        rest = D - (w[fixed] ** 2).sum()
        assert rest > 0
        w[~fixed] *= np.sqrt(rest / (w[~fixed] ** 2).sum())
        u = H @ w                        # H is symmetric and orthonormal: w = H u
        # s2 > 0 with |s2 u + o| = sqrt(D), so that y = s2 u + o has the norm of x / s1
        uo = u @ o
        s2 = (-uo + np.sqrt(uo * uo - D * ((o @ o) - D))) / D
        s1 = float(np.exp(rng.standard_normal()))
        xs.append(s1 * (s2 * u + o))
    return np.asarray(xs, dtype=np.float32), o.astype(np.float32)


@pytest.mark.parametrize("g,tc,T", [(4, False, 1), (8, False, 1), (4, False, 1500),
                                      (8, False, 1500), (4, True, 1500)])
def test_encode_near_voronoi_boundaries(codebooks, g, tc, T):
    """T = 1: one token per (sequence, head), a decode step's appends (small
    calls); T = 1500: the persistent 2-bit walk, the 1-bit tensor-core kernel
    or (tc) the 2-bit tensor-core search."""
    C = codebooks[g]
    B, H = (1, 512) if T == 1 else (1, 2)
    n = B * H * T
    x, o = _near_tie_tokens(C, n, seed=100 + g + T)
    x = x.reshape(B, H, T, D)
    shift = np.broadcast_to(o, (B, H, D)).copy()
    ora = O.encode(x.astype(np.float64), C, shift=shift.astype(np.float64), want_w=True)
    cache = nsnq.Cache.empty(B, H, T, g)
    cache.shift.copy_(torch.from_numpy(shift))
    ws = nsnq.nsnq_encode(P.to_dev(x, "f32"), P.codebook(C), cache, shift_mode=nsnq.SHIFT_GIVEN,
                          flags=nsnq.ENCODE_TC_SEARCH if tc else nsnq.ENCODE_DEFAULT)
    torch.cuda.synchronize()
    n_mis, n_bad, worst = P.code_report(cache.codes.cpu().numpy(), ora["codes"], ora["w"], C)
    assert n_bad == 0, (n_mis, worst)
    P.check_scales(cache.scales.cpu().numpy(), ora)
    st = nsnq.encode_stats(ws)
    assert st.mma_timeout == 0 and st.index_mismatch == 0
    if T > 1:  # the boundary tokens did reach the fp64 re-decision
        assert st.fp64_subvectors > 0
