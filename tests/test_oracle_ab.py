"""Pins of the oracle's AB-Attention functions (news page "AB-Attention
acelera a geracao de video em ate 2,23x e pula 92% da atencao", section
"Os tres recursos do AB-Attention") against what the page and the
mathematics fix:

* key-block means: the fp64 mean of 4 tokens;
* IBCS clustering: recovery of well-separated clusters; every centroid the
  mean of its queries; every query at its nearest centroid of the last
  assignment; the within-cluster sum of squares never grows with more
  iterations; weights sum to one;
* block scores: an fp64 restatement of the centroid-weighted softmax,
  sum one, the single-cluster case;
* SIP inclusion: sum(pi) = budget, pi proportional to the score below the
  cap, an exact-rational restatement;
* Horvitz-Thompson: over every possible sample of a small case, weighted by
  its probability, the expected numerator and normaliser of the shifted
  attention equal the full ones (exact enumeration);
* every block sampled with pi = 1: dense attention.
"""
import itertools
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

from block_sparse_attention_flatten_b200 import inputs


def f64(bits) -> np.ndarray:
    if isinstance(bits, torch.Tensor):
        return bits.to(torch.float64).numpy()
    return bits.astype(np.uint32).__lshift__(16).view(np.float32).astype(np.float64)


def bf16(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


@pytest.fixture(scope="module")
def tiny(oracle_lib):
    w = inputs.AB_TINY
    q, k, v = inputs.make_qkv(w.base)
    return w, q, k, v


def test_key_means_are_block_means(oracle_lib, tiny):
    w, q, k, v = tiny
    kbar = oracle_lib.ab_key_means(k)
    ref = f64(k).reshape(1, w.nkb, 4, w.base.Hh, w.base.D).mean(axis=2).transpose(0, 2, 1, 3)
    np.testing.assert_allclose(kbar, ref, rtol=0, atol=1e-6)


def test_kmeans_recovers_separated_clusters(oracle_lib):
    rng = np.random.default_rng(3)
    D, Hh = 64, 1
    centers = rng.standard_normal((8, D)) * 8.0
    # the starting queries (positions 0, 16, ..., 112) come one from each
    # cluster, the rest of the block is shuffled
    rest = rng.permutation(np.repeat(np.arange(8), 15))
    labels = np.empty(128, dtype=np.int64)
    labels[::16] = np.arange(8)
    labels[np.arange(128) % 16 != 0] = rest
    x = centers[labels] + 0.01 * rng.standard_normal((128, D))
    q = bf16(x.reshape(1, 128, Hh, D))
    cent, counts, assign = oracle_lib.ab_kmeans(q, iters=4)
    a = assign[0, 0]
    # same partition up to the cluster labels
    for c in range(8):
        members = set(np.nonzero(a == c)[0].tolist())
        assert members in [set(np.nonzero(labels == t)[0].tolist()) for t in range(8)]
    assert counts.sum() == 128 and np.all(counts == 16)
    for c in range(8):
        np.testing.assert_allclose(cent[0, 0, 0, c], f64(q)[0, a == c, 0].mean(axis=0), atol=1e-5)


def test_kmeans_centroids_assignment_and_descent(oracle_lib, tiny):
    w, q, k, v = tiny
    qd = f64(q)[0]  # [S, Hh, D]
    sse_prev = None
    for iters in (1, 2, 3, 4, 6):
        cent, counts, assign = oracle_lib.ab_kmeans(q, iters=iters)
        sse = 0.0
        for h in range(w.base.Hh):
            for I in range(w.nqb):
                xs = qd[I * 128:(I + 1) * 128, h]
                a = assign[0, h, I * 128:(I + 1) * 128]
                assert counts[0, h, I].sum() == 128
                for c in range(8):
                    assert counts[0, h, I, c] == np.sum(a == c)
                    if counts[0, h, I, c] > 0:
                        np.testing.assert_allclose(cent[0, h, I, c], xs[a == c].mean(axis=0), atol=1e-5)
                        sse += float(((xs[a == c] - xs[a == c].mean(axis=0)) ** 2).sum())
        if sse_prev is not None:
            assert sse <= sse_prev * (1 + 1e-9)
        sse_prev = sse
    # with one more iteration the assignment is that to the nearest centroid
    cent4, _, _ = oracle_lib.ab_kmeans(q, iters=4)
    _, _, assign5 = oracle_lib.ab_kmeans(q, iters=5)
    for h in range(w.base.Hh):
        for I in range(w.nqb):
            xs = qd[I * 128:(I + 1) * 128, h]
            d2 = ((xs[:, None, :] - cent4[0, h, I][None].astype(np.float64)) ** 2).sum(-1)
            a5 = assign5[0, h, I * 128:(I + 1) * 128]
            best = d2.min(axis=1)
            assert np.all(d2[np.arange(128), a5] <= best * (1 + 1e-5) + 1e-9)


def test_scores_restated_in_fp64(oracle_lib, tiny):
    w, q, k, v = tiny
    cent, counts, _ = oracle_lib.ab_kmeans(q, iters=4)
    kbar = oracle_lib.ab_key_means(k)
    scale = 1.0 / math.sqrt(w.base.D)
    s = oracle_lib.ab_scores(cent, counts, kbar, scale)
    for h in range(w.base.Hh):
        for I in range(w.nqb):
            l = cent[0, h, I].astype(np.float64) @ kbar[0, h].astype(np.float64).T * scale  # [8, NKB]
            a = np.exp(l - l.max(axis=1, keepdims=True))
            a /= a.sum(axis=1, keepdims=True)
            ref = (counts[0, h, I].astype(np.float64) / 128.0) @ a
            np.testing.assert_allclose(s[0, h, I], ref, rtol=2e-5, atol=1e-12)
            assert abs(s[0, h, I].sum() - 1.0) < 1e-12


def test_single_cluster_score_is_one_softmax(oracle_lib):
    rng = np.random.default_rng(5)
    D = 64
    qrow = rng.standard_normal(D)
    q = bf16(np.tile(qrow, (128, 1)).reshape(1, 128, 1, D))  # every query equal
    k = bf16(rng.standard_normal((1, 128, 1, D)))
    cent, counts, _ = oracle_lib.ab_kmeans(q, iters=3)
    assert counts[0, 0, 0].max() == 128  # all in one cluster (ties go to the lowest index)
    kbar = oracle_lib.ab_key_means(k)
    s = oracle_lib.ab_scores(cent, counts, kbar, 0.125)
    l = f64(q)[0, 0, 0] @ kbar[0, 0].astype(np.float64).T * 0.125
    ref = np.exp(l - l.max())
    np.testing.assert_allclose(s[0, 0, 0], ref / ref.sum(), rtol=2e-5)


def exact_inclusion(s, budget):
    """Water-filling in exact rationals: pi = min(1, lam * s), sum pi = budget."""
    fr = [Fraction(float(x)) for x in s]
    order = sorted(range(len(s)), key=lambda j: -fr[j])
    pos = [j for j in order if fr[j] > 0]
    b = Fraction(float(budget))
    if b >= len(pos):
        return [Fraction(1) if fr[j] > 0 else Fraction(0) for j in range(len(s))], None
    for m in range(len(pos)):
        rest = sum(fr[j] for j in pos[m:])
        lam = (b - m) / rest
        if lam * fr[pos[m]] < 1:
            out = [Fraction(0)] * len(s)
            for i, j in enumerate(pos):
                out[j] = Fraction(1) if i < m else lam * fr[j]
            return out, lam
    raise AssertionError("no solution")


@pytest.mark.parametrize("seed,n,budget", [(1, 40, 4.0), (2, 64, 10.0), (3, 17, 16.0), (4, 30, 30.0), (5, 50, 1.0)])
def test_inclusion_probabilities(oracle_lib, seed, n, budget):
    rng = np.random.default_rng(seed)
    s = rng.pareto(1.2, size=n) + 1e-3  # heavy-tailed: some blocks capped at 1
    s[rng.integers(0, n)] = 0.0 if n > 20 else s[0]
    s /= s.sum()
    pi, lam = oracle_lib.ab_inclusion_row(s, budget)
    ref, _ = exact_inclusion(s, budget)
    np.testing.assert_allclose(pi, [float(x) for x in ref], rtol=1e-12, atol=1e-15)
    npos = int((s > 0).sum())
    assert abs(pi.sum() - min(budget, npos)) < 1e-9
    assert np.all((pi >= 0) & (pi <= 1))
    below = (pi < 1) & (s > 0)
    if below.any() and math.isfinite(lam):
        np.testing.assert_allclose(pi[below] / s[below], lam, rtol=1e-12)
        assert np.all(lam * s[pi == 1] >= 1 - 1e-12)


def test_horvitz_thompson_unbiased_by_enumeration(oracle_lib):
    """One query block of 128 tokens over 6 key blocks (24 tokens): for every
    one of the 2^6 samples, the oracle's shifted attention gives
    N_hat = O * exp(LSE) and D_hat = exp(LSE); their expectations under the
    inclusion probabilities equal the full numerator and normaliser."""
    rng = np.random.default_rng(9)
    D, S = 64, 128
    q = bf16(rng.standard_normal((1, S, 1, D)) * 0.5)
    k = bf16(rng.standard_normal((1, S, 1, D)) * 0.5)
    v = bf16(rng.standard_normal((1, S, 1, D)))
    nkb = S // 4
    blocks = [0, 3, 7, 12, 20, 31]
    pis = np.array([1.0, 0.9, 0.5, 0.25, 0.6, 0.1])
    scale = 0.125
    qd, kd, vd = f64(q)[0, :, 0], f64(k)[0, :, 0], f64(v)[0, :, 0]
    toks = np.concatenate([np.arange(4 * J, 4 * J + 4) for J in blocks])
    l = qd @ kd[toks].T * scale
    N_full = np.exp(l) @ vd[toks]
    D_full = np.exp(l).sum(axis=1)
    EN = np.zeros_like(N_full)
    ED = np.zeros_like(D_full)
    for pattern in itertools.product([0, 1], repeat=len(blocks)):
        prob = float(np.prod([p if x else 1 - p for p, x in zip(pis, pattern)]))
        if prob == 0.0:
            continue
        sel = [i for i, x in enumerate(pattern) if x]
        if not sel:
            continue  # the empty sample contributes zero to both
        cnt = np.array([[[len(sel)]]], dtype=np.int32)
        idx = np.full((1, 1, 1, nkb), -1, dtype=np.int32)
        shift = np.zeros((1, 1, 1, nkb))
        idx[0, 0, 0, :len(sel)] = [blocks[i] for i in sel]
        shift[0, 0, 0, :len(sel)] = [-math.log(pis[i]) for i in sel]
        out, lse = oracle_lib.ab_attention(q, k, v, cnt, idx, shift, scale)
        Dh = np.exp(lse[0, 0])
        EN += prob * out[0, :, 0] * Dh[:, None]
        ED += prob * Dh
    np.testing.assert_allclose(EN, N_full, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(ED, D_full, rtol=1e-10)


def test_full_sample_equals_dense_attention(oracle_lib, tiny):
    w, q, k, v = tiny
    B, S, Hh, D = q.shape
    nkb = w.nkb
    cnt = np.full((B, Hh, w.nqb), nkb, dtype=np.int32)
    idx = np.broadcast_to(np.arange(nkb, dtype=np.int32), (B, Hh, w.nqb, nkb)).copy()
    shift = np.zeros((B, Hh, w.nqb, nkb))
    out, lse = oracle_lib.ab_attention(q, k, v, cnt, idx, shift, 1.0 / math.sqrt(D), qblocks=[0, 5])
    qd, kd, vd = f64(q)[0], f64(k)[0], f64(v)[0]
    for h in range(Hh):
        for n, I in enumerate((0, 5)):
            l = qd[I * 128:(I + 1) * 128, h] @ kd[:, h].T / math.sqrt(D)
            p = np.exp(l - l.max(axis=1, keepdims=True))
            ref = (p / p.sum(axis=1, keepdims=True)) @ vd[:, h]
            np.testing.assert_allclose(out[0, n * 128:(n + 1) * 128, h], ref, atol=1e-10)
