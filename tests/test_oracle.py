"""Pins for the CPU oracle: each test checks it against something other than
itself (library routines, closed forms, textbook quantizers, invariants the
method's definition fixes, brute force on tiny inputs)."""
import hashlib
import json
import os

import numpy as np
import pytest
import scipy.linalg
import scipy.spatial.distance
import torch

import nsnq_synth as S
from oracle import oracle as O
from tests.conftest import GOLDEN

D = 128


# ---------------------------------------------------------------- Hadamard --
@pytest.mark.parametrize("d", [1, 2, 4, 8, 16, 64, 128, 256])
def test_hadamard_is_scipy_sylvester(d):
    """NSNQuant Methodology §2 (naive Hadamard): the oracle's matrix equals
    SciPy's Sylvester construction, normalised to be orthonormal."""
    H = O.hadamard(d)
    ref = scipy.linalg.hadamard(d).astype(np.float64) / np.sqrt(d)
    assert np.array_equal(H, ref)
    assert np.abs(H @ H - np.eye(d)).max() < 1e-12        # symmetric and H^2 = I
    v = np.random.default_rng(d).standard_normal(d)
    assert abs(np.linalg.norm(H @ v) - np.linalg.norm(v)) < 1e-12


# ------------------------------------------------------------------ k-means --
@pytest.mark.parametrize("k,centroids,mse", [
    # J. Max, "Quantizing for minimum distortion" (1960), Gaussian source:
    # 2 levels at +-sqrt(2/pi), MSE 1 - 2/pi; 4 levels at +-0.4528, +-1.5104, MSE 0.1175.
    (2, [-0.7979, 0.7979], 0.3634),
    (4, [-1.5104, -0.4528, 0.4528, 1.5104], 0.1175),
])
def test_kmeans_reaches_lloyd_max(k, centroids, mse):
    X = S.normal(11, S.STREAM_EXTRA, 0, 1 << 17).reshape(-1, 1)
    C, counts = O.kmeans(X, k, 300)
    c = np.sort(C[:, 0])
    assert np.allclose(c, centroids, rtol=0.015, atol=0.01), c
    d2 = ((X - C[:, 0][None, :]) ** 2).min(1).mean()
    assert abs(d2 - mse) < 0.01 * mse + 2e-3, d2
    assert counts.sum() == X.shape[0]


def test_kmeans_matches_sklearn_lloyd():
    """Same recipe (init = first k samples, 25 Lloyd iterations) through
    scikit-learn's independent implementation."""
    from sklearn.cluster import KMeans
    X = S.codebook_samples(4, 1 << 13, seed=5)
    C, counts = O.kmeans(X, 64, 25)
    assert counts.min() > 0  # no empty cluster, so the relocation rules cannot differ
    km = KMeans(n_clusters=64, init=X[:64].copy(), n_init=1, max_iter=25, tol=0.0,
                algorithm="lloyd").fit(X)
    assert np.abs(km.cluster_centers_ - C).max() < 1e-9


def test_kmeans_empty_cluster_keeps_centroid():
    # Two identical seeds: in the first assignment every tie goes to index 0,
    # so cluster 1 is empty and keeps its value; centroid 0 moves to the mean.
    X = np.array([[0.0], [0.0], [1.0], [1.2]])
    C, counts = O.kmeans(X, 2, 1)
    assert C[1, 0] == 0.0 and counts[1] == 0
    assert abs(C[0, 0] - 2.2 / 4) < 1e-15
    # second iteration: the two zeros now prefer centroid 1
    C, counts = O.kmeans(X, 2, 2)
    assert list(counts) == [2, 2] and C[1, 0] == 0.0 and abs(C[0, 0] - 1.1) < 1e-15


def test_codebook_files_are_the_recipe():
    meta = json.load(open(os.path.join(GOLDEN, "codebooks.json")))
    import oracle.make_codebooks as M
    for g in (8, 4):
        _, C, _ = M.make(g)
        sha = hashlib.sha256(C.astype("<f4").tobytes()).hexdigest()
        assert sha == meta["files"][f"codebook_g{g}.f32"]["sha256"]


@pytest.mark.parametrize("g,lo,hi", [
    # held-out distortion per coordinate lies between the Gaussian Shannon bound
    # 2^(-2R) and the scalar Lloyd-Max quantizer at the same rate R = 8/g bits.
    (8, 0.25, 0.3634),
    (4, 0.0625, 0.1175),
])
def test_codebook_distortion_between_bounds(codebooks, g, lo, hi):
    C = codebooks[g].astype(np.float64)
    X = S.normal(21, S.STREAM_EXTRA, 0, 20000 * g).reshape(-1, g)
    d2 = scipy.spatial.distance.cdist(X, C, "sqeuclidean").min(1).mean() / g
    assert lo < d2 < hi, d2


# ----------------------------------------------------------- NSN + encode --
def _tiny_keys(T=256, seed=0):
    w = S.WORKLOADS["tiny"]
    return S.io_to_f64(S.to_io(S.keys(w, T_total=T, t1=T), "f32"), "f32")


@pytest.mark.parametrize("g", [8, 4])
def test_encode_nsn_invariants(codebooks, g):
    """Methodology §1: after the shift the channel mean is 0, after the second
    normalize every token has norm sqrt(d), and the byproducts (s1, o, s2)
    rebuild the token exactly from the transformed vector."""
    x = _tiny_keys()
    enc = O.encode(x, codebooks[g], want_w=True)
    H = scipy.linalg.hadamard(D) / np.sqrt(D)
    w = enc["w"][0, 0]
    u = w @ H  # H symmetric, H^2 = I
    s1, s2, o = enc["s1"][0, 0], enc["s2"][0, 0], enc["o"][0, 0]
    assert np.abs(np.linalg.norm(w, axis=1) - np.sqrt(D)).max() < 1e-12
    assert np.abs(np.linalg.norm(u, axis=1) - np.sqrt(D)).max() < 1e-12
    z = s2[:, None] * u
    assert np.abs(z.mean(0)).max() < 1e-12 * np.abs(o).max()
    rebuilt = s1[:, None] * (z + o[None, :])
    assert np.abs(rebuilt - x[0, 0]).max() < 1e-12 * np.abs(x).max()
    # the mean is taken over normalised tokens: o = mean of x / s1
    assert np.abs(o - (x[0, 0] / s1[:, None]).mean(0)).max() < 1e-12


@pytest.mark.parametrize("g", [8, 4])
def test_encode_codes_are_nearest_codewords(codebooks, g):
    """Methodology §3: every sub-vector maps to its nearest codeword (SciPy's
    cdist + first-index argmin as the independent brute force)."""
    x = _tiny_keys(T=32)
    C = codebooks[g]
    enc = O.encode(x, C, want_w=True)
    sub = enc["w"][0, 0].reshape(-1, g)
    dist = scipy.spatial.distance.cdist(sub, C.astype(np.float64), "sqeuclidean")
    assert np.array_equal(enc["codes"][0, 0].reshape(-1), dist.argmin(1).astype(np.uint8))


def test_encode_given_shift_uses_it(codebooks):
    x = _tiny_keys(T=16)
    o = np.random.default_rng(3).standard_normal((1, 1, D)) * 0.1
    enc = O.encode(x, codebooks[4], shift=o, want_w=True)
    assert np.array_equal(enc["o"], o)
    H = scipy.linalg.hadamard(D) / np.sqrt(D)
    u = enc["w"][0, 0] @ H
    rebuilt = enc["s1"][0, 0][:, None] * (enc["s2"][0, 0][:, None] * u + o[0, 0][None, :])
    assert np.abs(rebuilt - x[0, 0]).max() < 1e-12 * np.abs(x).max()


def test_encode_degenerate_tokens():
    """Zero token -> s1 = 0; a single token in compute mode -> z = 0, s2 = 0,
    w = 0, so every code is the codeword of least norm (lowest index on ties)."""
    C = np.full((256, 4), 3.0, dtype=np.float32)
    C[5] = [1, 0, 0, 0]
    C[9] = [0, 1, 0, 0]  # same norm as C[5]: the tie goes to index 5
    x = np.zeros((1, 1, 1, D))
    enc = O.encode(x, C)
    assert enc["s1"][0, 0, 0] == 0 and enc["s2"][0, 0, 0] == 0
    assert (enc["codes"] == 5).all()
    x = np.random.default_rng(0).standard_normal((1, 1, 1, D))
    enc = O.encode(x, C)
    assert enc["s1"][0, 0, 0] > 0 and enc["s2"][0, 0, 0] == 0
    assert (enc["codes"] == 5).all()
    # identical tokens: o equals every y, the residual vanishes (rounding-level
    # leftovers of the mean count as zero), so s2 = 0 for each of them
    x = np.repeat(np.random.default_rng(1).standard_normal((1, 1, 1, D)), 3, axis=2)
    enc = O.encode(x, C)
    assert (enc["s2"] == 0).all() and (enc["codes"] == 5).all()
    enc0 = O.encode(np.zeros((1, 1, 0, D)), C)
    assert enc0["codes"].shape == (1, 1, 0, D // 4) and (enc0["o"] == 0).all()


@pytest.mark.parametrize("g,T", [(8, 16), (4, 8)])
def test_roundtrip_with_planted_codebook(g, T):
    """Plant the transformed sub-vectors themselves as codewords (in shuffled
    order): encode must pick exactly those indices, and dequant must give
    back the input up to fp32 storage rounding of codebook, s1, s2, o."""
    x = _tiny_keys(T=T)
    rng = np.random.default_rng(7)
    probe = rng.standard_normal((256, g)).astype(np.float32)
    w = O.encode(x, probe, want_w=True)["w"][0, 0]
    sub = w.reshape(-1, g)
    assert sub.shape[0] == 256
    perm = rng.permutation(256)
    C = np.empty((256, g), dtype=np.float32)
    C[perm] = sub.astype(np.float32)  # sub-vector i becomes codeword perm[i]
    enc = O.encode(x, C)
    assert np.array_equal(enc["codes"][0, 0].reshape(-1), perm.astype(np.uint8))
    s1, s2, o = O.stored(enc)
    xh = O.dequant(enc["codes"], s1, s2, o, C)
    assert np.abs(xh - x).max() < 2e-6 * np.abs(x).max()


def test_dequant_closed_form():
    """All codes 0 with C_0 = e_0 (g = 4): w_hat has ones at coordinates 4j, and
    by Walsh-function orthogonality H w_hat = (32/sqrt(128)) on coordinates
    0..3 and 0 elsewhere."""
    C = np.zeros((256, 4), dtype=np.float32)
    C[0, 0] = 1.0
    T = 3
    codes = np.zeros((1, 1, T, 32), dtype=np.uint8)
    s1 = np.array([[[1.0, 2.0, 0.5]]], dtype=np.float32)
    s2 = np.array([[[1.0, 0.25, 3.0]]], dtype=np.float32)
    o = np.linspace(-1, 1, D, dtype=np.float32).reshape(1, 1, D)
    xh = O.dequant(codes, s1, s2, o, C)[0, 0]
    hw = np.zeros(D)
    hw[:4] = 32 / np.sqrt(D)
    for t in range(T):
        ref = float(s1[0, 0, t]) * (float(s2[0, 0, t]) * hw + o[0, 0].astype(np.float64))
        assert np.abs(xh[t] - ref).max() < 1e-12


def test_transformed_channels_are_near_standard_normal(codebooks):
    """Methodology §1-§2 (Lemma 1 and the CLT argument): after NSN and the
    Hadamard transform every channel has mean ~0 and variance ~1."""
    w = S.WORKLOADS["encode-8x4096"]
    x = S.io_to_f64(S.to_io(S.keys(w, b0=0, b1=1)[:, :2], "bf16"), "bf16")
    enc = O.encode(x, codebooks[4], want_w=True)
    for h in range(2):
        wt = enc["w"][0, h]
        T = wt.shape[0]
        assert np.abs(wt.mean(0)).max() < 6 / np.sqrt(T)
        assert np.abs(wt.var(0) - 1).max() < 0.1


# --------------------------------------------------------------- attention --
def _sdpa(q, K, V, scale):
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(K)[None], torch.from_numpy(V)[None],
        scale=scale)[0].numpy()


def test_attention_matches_torch_sdpa_with_gqa_and_lengths():
    rng = np.random.default_rng(1)
    B, Hq, Hkv, T = 3, 8, 2, 37
    q = rng.standard_normal((B, Hq, D))
    K = rng.standard_normal((B, Hkv, T, D)) * 1.5
    V = rng.standard_normal((B, Hkv, T, D))
    lens = np.array([37, 1, 20])
    out = O.attention(q, K, V, lens)
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            L = lens[b]
            ref = _sdpa(q[b, h][None], K[b, h // G, :L], V[b, h // G, :L], 1 / np.sqrt(D))[0]
            assert np.abs(out[b, h] - ref).max() < 1e-12


def test_attention_special_cases():
    rng = np.random.default_rng(2)
    K = rng.standard_normal((1, 1, 50, D))
    V = rng.standard_normal((1, 1, 50, D))
    out = O.attention(np.zeros((1, 1, D)), K, V)       # q = 0 -> mean of v
    assert np.abs(out[0, 0] - V[0, 0].mean(0)).max() < 1e-12
    out = O.attention(rng.standard_normal((1, 1, D)), K, V, [1])  # one token -> v_0
    assert np.abs(out[0, 0] - V[0, 0, 0]).max() < 1e-15
    out = O.attention(rng.standard_normal((1, 1, D)), K, V, [0])  # empty -> 0
    assert (out == 0).all()


# ------------------------------------------------------------ input recipe --
def test_synthetic_normals_are_standard_normal():
    import scipy.stats
    n = S.normal(123, 0, 0, 200000)
    assert abs(n.mean()) < 0.01 and abs(n.var() - 1) < 0.01
    assert scipy.stats.kstest(n, "norm").pvalue > 1e-3
    # counter-based: any slice equals the same slice of the whole stream
    assert np.array_equal(S.normal(123, 0, 1001, 77), n[1001:1078])


def test_synthetic_keys_have_outlier_channels():
    w = S.WORKLOADS["tiny"]
    K = S.keys(w)
    chans, signs = w.kdist.channels(D)
    assert chans == [0, 32, 64, 96]
    m = np.abs(K[0, 0]).mean(0)
    assert all(m[c] > 5 for c in chans) and np.median(m) < 2
    sub = S.keys(w, t0=100, t1=120, T_total=256)
    assert np.array_equal(sub[0, 0], K[0, 0, 100:120])


@pytest.mark.parametrize("g", [8, 4])
def test_adaptive_scale_leaves_error_orthogonal_to_the_token(codebooks, g):
    """Methodology §3, scale adjustment: the scaled quantized vector keeps the
    component along the original, so after removing the shift the
    reconstruction error is orthogonal to the original token, and the codes
    are those of the plain encoding."""
    x = _tiny_keys(T=64)
    C = codebooks[g]
    plain = O.encode(x, C)
    adj = O.encode(x, C, adaptive_scale=True)
    assert np.array_equal(plain["codes"], adj["codes"])
    assert np.array_equal(plain["s1"], adj["s1"]) and np.array_equal(plain["o"], adj["o"])
    # no float32 storage here: rebuild with the exact byproducts
    H = scipy.linalg.hadamard(D) / np.sqrt(D)
    wh = C[adj["codes"][0, 0]].reshape(64, D).astype(np.float64)
    s1, s2, o = adj["s1"][0, 0], adj["s2"][0, 0], adj["o"][0, 0]
    xr = s1[:, None] * (s2[:, None] * (wh @ H) + o[None, :])
    xc = x[0, 0] - s1[:, None] * o[None, :]          # original minus shift part
    err = xr - x[0, 0]
    cos = (err * xc).sum(1) / (np.linalg.norm(err, axis=1) * np.linalg.norm(xc, axis=1))
    assert np.abs(cos).max() < 1e-10
    # the plain encoding's error is not orthogonal
    whp = wh
    xp = plain["s1"][0, 0][:, None] * (plain["s2"][0, 0][:, None] * (whp @ H) + o[None, :])
    ep = xp - x[0, 0]
    assert np.abs((ep * xc).sum(1)).max() > 1e-3
    ratio = adj["s2"][0, 0] / plain["s2"][0, 0]
    assert (ratio > 0.5).all() and (ratio < 2.0).all()


# --------------------------------------------------------- residual window --
def test_residual_attention_matches_sdpa_over_concatenation():
    """Methodology §4 (Residuals): one softmax over the quantized tokens and
    the full-precision residual, each sequence with its own two lengths
    (empty parts included), checked against torch SDPA over the
    concatenated rows."""
    rng = np.random.default_rng(4)
    B, Hq, Hkv, T, R = 4, 4, 2, 23, 9
    q = rng.standard_normal((B, Hq, D))
    K = rng.standard_normal((B, Hkv, T, D)) * 1.3
    V = rng.standard_normal((B, Hkv, T, D))
    Kr = rng.standard_normal((B, Hkv, R, D)) * 1.3 + 0.5
    Vr = rng.standard_normal((B, Hkv, R, D)) - 0.7
    lens, rlens = [23, 0, 5, 0], [0, 9, 4, 0]
    out = O.attention_with_residual(q, K, V, lens, Kr, Vr, rlens)
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            Kc = np.concatenate([K[b, h // G, :lens[b]], Kr[b, h // G, :rlens[b]]])
            Vc = np.concatenate([V[b, h // G, :lens[b]], Vr[b, h // G, :rlens[b]]])
            if Kc.shape[0] == 0:
                assert (out[b, h] == 0).all()
                continue
            ref = _sdpa(q[b, h][None], Kc, Vc, 1 / np.sqrt(D))[0]
            assert np.abs(out[b, h] - ref).max() < 1e-12


def _loop_inputs(B=2, Hkv=2, Hq=4, T=40, S_=11, seed=3):
    rng = np.random.default_rng(seed)
    mk = lambda *s: rng.standard_normal(s).astype(np.float32).astype(np.float64)
    kp = mk(B, Hkv, T, D) + np.where(np.arange(D) % 32 == 0, 4.0, 0.0)
    return kp, mk(B, Hkv, T, D), mk(B, Hkv, S_, D) * 1.2, mk(B, Hkv, S_, D), mk(S_, B, Hq, D)


def test_decode_loop_flushes_equal_a_one_shot_encode_with_the_stored_shift(codebooks):
    """Residual window R = 4 over 11 decode steps: two flushes. Every flushed
    token is encoded with the prompt's shift, so the cache equals a one-shot
    encoding of the first 8 new tokens with that shift; 3 tokens stay."""
    kp, vp, kn, vn, qs = _loop_inputs()
    C = codebooks[4]
    outs, st = O.decode_with_residual(kp, vp, kn, vn, qs, C, C, R=4)
    assert st["n_quant"] == 40 + 8 and st["n_res"] == 3
    for n, x in (("K", kn), ("V", vn)):
        prompt = O.encode(kp if n == "K" else vp, C)
        one = O.encode(x[:, :, :8], C, shift=prompt["o"])
        assert np.array_equal(st[n]["codes"][:, :, :40], prompt["codes"])
        assert np.array_equal(st[n]["codes"][:, :, 40:], one["codes"])
        assert np.array_equal(st[n]["s2"][:, :, 40:], one["s2"])
        assert np.array_equal(st[n]["o"], prompt["o"])


def test_decode_loop_without_a_flush_attends_to_the_raw_new_tokens(codebooks):
    """R above the number of steps: the new tokens stay at full precision, so
    step s is SDPA over [dequantized prompt || the first s + 1 raw tokens]."""
    kp, vp, kn, vn, qs = _loop_inputs(S_=5)
    C = codebooks[8]
    outs, st = O.decode_with_residual(kp, vp, kn, vn, qs, C, C, R=64)
    assert st["n_res"] == 5
    eK, eV = O.encode(kp, C), O.encode(vp, C)
    Kh = O.dequant(eK["codes"], *O.stored(eK), C)
    Vh = O.dequant(eV["codes"], *O.stored(eV), C)
    G = qs.shape[2] // kp.shape[1]
    for s in range(5):
        for b in range(2):
            for h in range(4):
                Kc = np.concatenate([Kh[b, h // G], kn[b, h // G, :s + 1]])
                Vc = np.concatenate([Vh[b, h // G], vn[b, h // G, :s + 1]])
                ref = _sdpa(qs[s, b, h][None], Kc, Vc, 1 / np.sqrt(D))[0]
                assert np.abs(outs[s, b, h] - ref).max() < 1e-12


def test_decode_loop_with_a_one_token_window_quantizes_every_token(codebooks):
    """R = 1: each new token is flushed at once, so every step attends over a
    fully quantized cache with no residual."""
    kp, vp, kn, vn, qs = _loop_inputs(S_=3)
    C = codebooks[4]
    outs, st = O.decode_with_residual(kp, vp, kn, vn, qs, C, C, R=1)
    assert st["n_res"] == 0 and st["n_quant"] == 43
    eK, eV = O.encode(kp, C), O.encode(vp, C)
    for s in range(3):
        fK = O.encode(kn[:, :, :s + 1], C, shift=eK["o"])
        fV = O.encode(vn[:, :, :s + 1], C, shift=eV["o"])
        cat = lambda a, b, k: np.concatenate([a[k], b[k]], axis=2)
        Kh = O.dequant(cat(eK, fK, "codes"), cat(eK, fK, "s1").astype(np.float32),
                       cat(eK, fK, "s2").astype(np.float32), eK["o"].astype(np.float32), C)
        Vh = O.dequant(cat(eV, fV, "codes"), cat(eV, fV, "s1").astype(np.float32),
                       cat(eV, fV, "s2").astype(np.float32), eV["o"].astype(np.float32), C)
        ref = O.attention(qs[s], Kh, Vh)
        assert np.abs(outs[s] - ref).max() < 1e-12


# ----------------------------------------------------------------- RoPE --
def test_rope_matches_the_complex_rotation():
    """The rotary embedding as complex multiplication: channel pair
    (x_i, x_{i+64}) as x_i + 1j x_{i+64}, times exp(1j pos base^(-2i/d))
    (an independent formulation of the same rotation)."""
    rng = np.random.default_rng(7)
    x = rng.standard_normal((3, 11, D))
    pos = np.array([0, 1, 2, 5, 17, 100, 1000, 4095, 32767, 131071, 7])
    for base in (10000.0, 500000.0):
        y = O.rope(x, pos, base)
        i = np.arange(D // 2)
        ang = pos[:, None] * base ** (-2.0 * i / D)
        z = (x[..., :D // 2] + 1j * x[..., D // 2:]) * np.exp(1j * ang)
        ref = np.concatenate([z.real, z.imag], axis=-1)
        assert np.abs(y - ref).max() < 1e-9 * np.abs(x).max()


def test_rope_is_a_rotation_with_relative_positions():
    """Norm preserved, position 0 is the identity, and the dot product of a
    query at m with a key at n depends only on m - n."""
    rng = np.random.default_rng(8)
    q = rng.standard_normal((1, D))
    k = rng.standard_normal((1, D))
    assert np.array_equal(O.rope(k, [0]), k)
    for m, n in ((5, 3), (1000, 10), (77, 77), (3, 9)):
        lhs = (O.rope(q, [m]) * O.rope(k, [n])).sum()
        rhs = (O.rope(q, [m - n]) * k).sum()
        assert abs(lhs - rhs) < 1e-10 * np.abs(q).sum() * np.abs(k).sum()
        assert abs(np.linalg.norm(O.rope(k, [n])) - np.linalg.norm(k)) < 1e-12


def test_attention_rope_is_sdpa_over_rotated_keys():
    """Keys quantized before RoPE: attention rotates key t to position t,
    checked against torch SDPA over keys rotated by the complex formulation."""
    rng = np.random.default_rng(9)
    B, Hq, Hkv, T = 2, 4, 2, 40
    q = rng.standard_normal((B, Hq, D))
    K = rng.standard_normal((B, Hkv, T, D)) * 1.2
    V = rng.standard_normal((B, Hkv, T, D))
    lens = [40, 13]
    out = O.attention_rope(q, K, V, lens, base=10000.0)
    i = np.arange(D // 2)
    ang = np.arange(T)[:, None] * 10000.0 ** (-2.0 * i / D)
    z = (K[..., :D // 2] + 1j * K[..., D // 2:]) * np.exp(1j * ang)
    Kr = np.concatenate([z.real, z.imag], axis=-1)
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            ref = _sdpa(q[b, h][None], Kr[b, h // G, :lens[b]], V[b, h // G, :lens[b]], 1 / np.sqrt(D))[0]
            assert np.abs(out[b, h] - ref).max() < 1e-12


# ----------------------------------------------------- double quantization --
def test_quantize4_is_a_16_level_uniform_grid():
    """Methodology §3 (Double Quantization), 4-bit reading: 16 uniform levels
    from the minimum to the maximum, each value on its nearest level."""
    rng = np.random.default_rng(10)
    x = rng.standard_normal(1000) * 3 + 1
    xq = O.quantize4(x)
    lo, hi = x.min(), x.max()
    step = (hi - lo) / 15
    k = (xq - lo) / step
    assert np.abs(k - np.round(k)).max() < 1e-9 and k.min() > -1e-9 and k.max() < 15 + 1e-9
    assert len(np.unique(np.round(k))) <= 16
    assert np.abs(x - xq).max() <= step / 2 + 1e-12
    assert xq.min() == lo and abs(xq.max() - hi) < 1e-12
    assert np.array_equal(O.quantize4(np.full(7, 2.5)), np.full(7, 2.5))
    C = np.random.default_rng(11).standard_normal((256, 4)).astype(np.float32)
    assert len(np.unique(O.quantize4(C))) <= 16


@pytest.mark.parametrize("g", [8, 4])
def test_double_quant_byproducts_and_reconstruction(codebooks, g):
    """Double quantization: s1 on the head's 16-level log2 grid (the nearest
    level of log2 of the exact s1, grid from the tokens' least to largest),
    o on 16 uniform levels, and the byproducts still rebuild the token
    exactly from the transformed vector (s2 absorbs the quantized s1)."""
    x = _tiny_keys(T=64)
    C = codebooks[g]
    enc = O.encode(x, C, want_w=True, double_quant=True)
    s1_exact = np.linalg.norm(x[0, 0], axis=1) / np.sqrt(D)
    lg = np.log2(s1_exact)
    lo, step = enc["s1_grid"][0, 0]
    # the grid: fp32 values spanning the tokens' log2 s1 (up to fp32 rounding)
    assert np.float32(lo) == lo and np.float32(step) == step and step > 0
    assert abs(lo - lg.min()) <= 2.0 ** -23 * abs(lg.min()) + 1e-30
    assert abs(lo + 15 * step - lg.max()) <= 16 * 2.0 ** -23 * max(abs(lg.max()), abs(lo))
    # every stored s1 is one of the 16 levels 2^(lo + j step) ...
    lq = np.log2(enc["s1"][0, 0])
    k = (lq - lo) / step
    assert np.abs(k - np.round(k)).max() < 1e-9 and k.min() > -1e-9 and k.max() < 15 + 1e-9
    # ... the nearest one in the log2 domain (brute force over the 16 levels)
    levels = lo + step * np.arange(16)
    best = np.abs(lg[:, None] - levels[None, :]).min(1)
    assert (np.abs(lq - lg) <= best + 1e-12).all()
    assert (np.abs(lq - lg) <= step / 2 + 1e-12).all()
    # the extreme tokens take the extreme levels
    assert round(k[np.argmin(lg)]) == 0 and round(k[np.argmax(lg)]) == 15
    o = enc["o"][0, 0]
    assert len(np.unique(np.round((o - o.min()) / ((o.max() - o.min()) / 15), 9))) <= 16
    H = scipy.linalg.hadamard(D) / np.sqrt(D)
    u = enc["w"][0, 0] @ H
    rebuilt = enc["s1"][0, 0][:, None] * (enc["s2"][0, 0][:, None] * u + o[None, :])
    assert np.abs(rebuilt - x[0, 0]).max() < 1e-12 * np.abs(x).max()
    plain = O.encode(x, C)
    assert not np.array_equal(plain["s1"], enc["s1"])
    assert np.array_equal(plain["codes"], O.encode(x, C, double_quant=False)["codes"])


def test_double_quant_append_uses_the_stored_grid(codebooks):
    """Appended tokens (shift given) are quantized on the prompt's stored s1
    grid, clamped to its 16 levels, with the stored o as the shift."""
    x = _tiny_keys(T=80)
    C = codebooks[4]
    pre = O.encode(x[:, :, :48], C, double_quant=True)
    new = np.concatenate([x[:, :, 48:], 40 * x[:, :, 48:50]], axis=2)  # two far above the grid
    app = O.encode(new, C, shift=pre["o"], double_quant=True, s1_grid=pre["s1_grid"])
    lo, step = pre["s1_grid"][0, 0]
    k = (np.log2(app["s1"][0, 0]) - lo) / step
    assert np.abs(k - np.round(k)).max() < 1e-9 and k.min() > -1e-9 and k.max() < 15 + 1e-9
    assert np.allclose(app["s1"][0, 0, -2:], 2.0 ** (lo + 15 * step))
    assert np.array_equal(app["o"], pre["o"]) and np.array_equal(app["s1_grid"], pre["s1_grid"])


# ------------------------------------------------- rotated-query identities --
@pytest.mark.parametrize("g", [4, 8])
def test_lut_scores_equal_dense_scores(codebooks, g):
    """Methodology §4: with x_hat = s1 (s2 H w_hat + o) and H symmetric
    orthonormal, q . x_hat = s1 (s2 sum_j L[j][code_j] + q . o) where
    L[j][c] = (H q)_j . C_c. The left side uses the oracle's dense dequant;
    the right side is assembled here from the table, so a wrong sign, index
    or transpose in either form breaks the equality."""
    w = S.Workload("lut", B=1, Hkv=2, Hq=2, T=64, d=D, sub_dim=g, dtype="f32",
                   kdist=S.K_MODERATE, seed=31)
    x = S.keys(w)
    C = codebooks[g]
    enc = O.encode(x, C)
    s1, s2, o = O.stored(enc)
    xh = O.dequant(enc["codes"], s1, s2, o, C)
    rng = np.random.default_rng(7)
    H = scipy.linalg.hadamard(D).astype(np.float64) / np.sqrt(D)
    for h in range(2):
        q = rng.standard_normal(D)
        qr = H @ q
        L = qr.reshape(D // g, g) @ C.astype(np.float64).T  # [j][c]
        codes = enc["codes"][0, h].astype(np.int64)           # [T][j]
        table = L[np.arange(D // g)[None, :], codes].sum(-1)  # [T]
        lut = s1[0, h].astype(np.float64) * (s2[0, h].astype(np.float64) * table
                                             + q @ o[0, h].astype(np.float64))
        dense = xh[0, h] @ q
        assert np.abs(lut - dense).max() <= 1e-10 * np.abs(dense).max()


def test_rotated_domain_value_sum_equals_dense(codebooks):
    """Methodology §4: sum_t p_t v_hat_t = H (sum_t p_t s1_t s2_t w_hat_t)
    + (sum_t p_t s1_t) o, i.e. values can be accumulated in the Hadamard
    domain and rotated once."""
    g = 4
    w = S.Workload("vsum", B=1, Hkv=1, Hq=1, T=50, d=D, sub_dim=g, dtype="f32",
                   kdist=S.K_MODERATE, seed=32)
    v = S.values(w)
    C = codebooks[g]
    enc = O.encode(v, C)
    s1, s2, o = O.stored(enc)
    vh = O.dequant(enc["codes"], s1, s2, o, C)[0, 0]
    p = np.random.default_rng(8).random(50)
    H = scipy.linalg.hadamard(D).astype(np.float64) / np.sqrt(D)
    what = C.astype(np.float64)[enc["codes"][0, 0].astype(np.int64)].reshape(50, D)
    a = (p * s1[0, 0] * s2[0, 0]) @ what
    beta = (p * s1[0, 0]).sum()
    rotated = H @ a + beta * o[0, 0].astype(np.float64)
    dense = p @ vh
    assert np.abs(rotated - dense).max() <= 1e-10 * np.abs(dense).max()
