"""Write the two global NSNQuant codebooks used by the tests and the benchmark.

Recipe (gist.science "NSNQuant ...", Technical Summary, Methodology §3: the
codebook is K-Means on synthetic standard-normal data, built once and reused
for any model): 2^16 seeded N(0, I) samples of dimension g, 256 centroids,
25 Lloyd iterations from the first 256 samples, fp64 arithmetic, rounded to
fp32 at the end. g = 8 gives 1 bit per coordinate, g = 4 gives 2 bits.

Calls only the oracle (and the shared seeded-sample generator). Output:
tests/golden/codebook_g{8,4}.f32 (little-endian fp32, [256][g]) and
tests/golden/codebooks.json (recipe, sha256, k-means distortion).
"""
from __future__ import annotations

import hashlib
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import nsnq_synth as S  # noqa: E402
from oracle import oracle as O  # noqa: E402

GOLDEN = os.path.join(ROOT, "tests", "golden")
N_SAMPLES = 1 << 16
N_CENTROIDS = 256
ITERS = 25


def make(g: int):
    X = S.codebook_samples(g, N_SAMPLES, seed=0)
    C64, counts = O.kmeans(X, N_CENTROIDS, ITERS)
    C32 = C64.astype(np.float32)
    return X, C32, counts


def main():
    os.makedirs(GOLDEN, exist_ok=True)
    meta = {"recipe": {"samples": N_SAMPLES, "centroids": N_CENTROIDS, "iters": ITERS,
                       "init": "first 256 samples", "rng": "nsnq_synth.codebook_samples(g, 2^16, seed=0)",
                       "precision": "fp64 k-means, rounded to fp32"},
            "source": "gist.science NSNQuant, Technical Summary, Methodology §3 (K-Means on standard normal data)",
            "files": {}}
    for g in (8, 4):
        X, C, counts = make(g)
        path = os.path.join(GOLDEN, f"codebook_g{g}.f32")
        C.astype("<f4").tofile(path)
        sha = hashlib.sha256(C.astype("<f4").tobytes()).hexdigest()
        d2 = ((X[:, None, :] - C[None, :, :].astype(np.float64)) ** 2).sum(-1).min(1)
        meta["files"][f"codebook_g{g}.f32"] = {
            "sub_dim": g, "bits_per_coord": 8 // g, "sha256": sha,
            "train_mse_per_coord": float(d2.mean() / g),
            "min_cluster": int(counts.min()), "max_cluster": int(counts.max())}
        print(g, sha, d2.mean() / g, counts.min(), counts.max())
    with open(os.path.join(GOLDEN, "codebooks.json"), "w") as f:
        json.dump(meta, f, indent=1, sort_keys=True)
        f.write("\n")


if __name__ == "__main__":
    main()
