"""Pins of the CPU oracle against what the method and the mathematics fix.

Each test checks one oracle function against something other than itself:
an independent formulation, a closed form, an exact-arithmetic restatement,
an invariant, or a special case that reduces to a textbook routine.  The
steps follow the NABLA technical summary (gist.science, paper 2507.13546),
section "Metodologia: NABLA".
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from block_sparse_attention_flatten_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
BLOCK = 64


def f32(x):
    return np.float32(x)


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).numpy()


# ----------------------------------------------------------------------------
# Fractal flattening (Metodologia item 1)
# ----------------------------------------------------------------------------
def reshape_flatten(x: np.ndarray, T, H, W, P=8):
    """Independent formulation: split H and W into (patch, within) and move the
    patch axes in front of the within-patch axes."""
    B = x.shape[0]
    R = int(np.prod(x.shape[2:]))
    g = x.reshape(B, T, H // P, P, W // P, P, R)
    g = g.transpose(0, 1, 2, 4, 3, 5, 6)
    return np.ascontiguousarray(g).reshape(B, T * H * W, R)


@pytest.mark.parametrize("T,H,W,R", [(4, 16, 16, 128), (3, 8, 24, 8), (2, 48, 80, 16), (1, 8, 8, 8), (5, 16, 8, 24)])
def test_flatten_matches_reshape_formulation(oracle_lib, T, H, W, R):
    rng = np.random.default_rng(T * 1000 + H + W)
    x = rng.integers(0, 65535, size=(2, T * H * W, R), dtype=np.uint16)
    got = oracle_lib.flatten(x, T, H, W)
    assert np.array_equal(got, reshape_flatten(x, T, H, W))


def test_flatten_is_bijection_and_inverse(oracle_lib):
    T, H, W = 4, 16, 24
    S = T * H * W
    ids = np.arange(S, dtype=np.uint16).reshape(1, S, 1)
    ids8 = np.repeat(ids, 8, axis=2)  # rows of 16 bytes
    f = oracle_lib.flatten(ids8, T, H, W)
    perm = f[0, :, 0].astype(np.int64)
    assert np.array_equal(np.sort(perm), np.arange(S))
    back = oracle_lib.unflatten(f, T, H, W)
    assert np.array_equal(back, ids8)


def test_flatten_identity_when_one_patch_per_frame(oracle_lib):
    rng = np.random.default_rng(7)
    x = rng.integers(0, 65535, size=(1, 3 * 64, 8), dtype=np.uint16)
    assert np.array_equal(oracle_lib.flatten(x, 3, 8, 8), x)


def test_flatten_first_patch_listing(oracle_lib):
    """First flattened block of a 1x16x16 grid = grid rows 0..7, columns 0..7."""
    T, H, W = 1, 16, 16
    ids = np.arange(T * H * W, dtype=np.uint16).reshape(1, -1, 1).repeat(8, axis=2)
    perm = oracle_lib.flatten(ids, T, H, W)[0, :, 0].astype(int)
    expect0 = [h * 16 + w for h in range(8) for w in range(8)]
    expect1 = [h * 16 + w for h in range(8) for w in range(8, 16)]
    expect2 = [h * 16 + w for h in range(8, 16) for w in range(8)]
    assert perm[:64].tolist() == expect0
    assert perm[64:128].tolist() == expect1
    assert perm[128:192].tolist() == expect2


# ----------------------------------------------------------------------------
# Pooling and reduced attention (Metodologia item 2)
# ----------------------------------------------------------------------------
@pytest.fixture(scope="module")
def tiny_flat(oracle_lib):
    w = inputs.TINY
    q, k, v = inputs.make_qkv(w)
    qf = oracle_lib.flatten(q, w.T, w.H, w.W).reshape(q.shape)
    kf = oracle_lib.flatten(k, w.T, w.H, w.W).reshape(k.shape)
    vf = oracle_lib.flatten(v, w.T, w.H, w.W).reshape(v.shape)
    return w, (q, k, v), (qf, kf, vf)


def bits_to_f64(a: np.ndarray) -> np.ndarray:
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_pool_is_block_mean(oracle_lib, tiny_flat):
    w, _, (qf, kf, vf) = tiny_flat
    qbar = oracle_lib.pool(qf)
    x = bits_to_f64(qf)  # [B,S,Hh,D]
    ref = x.reshape(w.B, w.Nb, BLOCK, w.Hh, w.D).mean(axis=2).transpose(0, 2, 1, 3)
    np.testing.assert_allclose(qbar, ref, rtol=0, atol=2e-6)


def test_pool_bilinearity_gives_mean_token_logit(oracle_lib, tiny_flat):
    """qbar_i . kbar_j equals the mean of the 64x64 tile of token dot products."""
    w, _, (qf, kf, vf) = tiny_flat
    qbar = oracle_lib.pool(qf).astype(np.float64)
    kbar = oracle_lib.pool(kf).astype(np.float64)
    q = bits_to_f64(qf)[0]
    k = bits_to_f64(kf)[0]
    for hd in range(w.Hh):
        logits = q[:, hd, :] @ k[:, hd, :].T  # [S,S]
        tile_mean = logits.reshape(w.Nb, BLOCK, w.Nb, BLOCK).mean(axis=(1, 3))
        np.testing.assert_allclose(qbar[0, hd] @ kbar[0, hd].T, tile_mean, rtol=1e-5, atol=1e-5)


def test_block_probs_is_softmax_of_scaled_tile_means(oracle_lib, tiny_flat):
    w, _, (qf, kf, vf) = tiny_flat
    qbar = oracle_lib.pool(qf)
    kbar = oracle_lib.pool(kf)
    q = bits_to_f64(qf)[0]
    k = bits_to_f64(kf)[0]
    for hd in range(w.Hh):
        tile_mean = (q[:, hd, :] @ k[:, hd, :].T).reshape(w.Nb, BLOCK, w.Nb, BLOCK).mean(axis=(1, 3))
        s = tile_mean / math.sqrt(w.D)
        ref = np.exp(s - s.max(axis=1, keepdims=True))
        ref /= ref.sum(axis=1, keepdims=True)
        for i in range(w.Nb):
            p = oracle_lib.block_probs_row(qbar[0, hd], kbar[0, hd], i, w.scale)
            np.testing.assert_allclose(p, ref[i], rtol=2e-5, atol=1e-9)
            assert abs(float(np.sum(p.astype(np.float64))) - 1.0) <= w.Nb * 2.0 ** -24
            assert np.all(p >= 0)


def test_equal_scores_give_exact_uniform_probabilities(oracle_lib):
    rng = np.random.default_rng(3)
    kbar = rng.standard_normal((16, 64)).astype(np.float32)
    qbar = np.zeros((16, 64), dtype=np.float32)
    p = oracle_lib.block_probs_row(qbar, kbar, 5, 0.125)
    assert np.all(p == np.float32(1.0 / 16.0))


# ----------------------------------------------------------------------------
# CDF thresholding
# ----------------------------------------------------------------------------
def read_uniform_cases():
    cases = []
    with open(os.path.join(GOLDEN, "uniform16.txt")) as fh:
        for line in fh:
            if line.startswith("#") or not line.strip():
                continue
            thr, kept = line.split()
            cases.append((float(thr), [int(x) for x in kept.split(",")]))
    return cases


@pytest.mark.parametrize("thr,kept", read_uniform_cases())
def test_uniform_worked_case(oracle_lib, thr, kept):
    rng = np.random.default_rng(11)
    kbar = rng.standard_normal((1, 1, 16, 64)).astype(np.float32)
    qbar = np.zeros((1, 1, 16, 64), dtype=np.float32)
    cnt, idx, status, _ = oracle_lib.build_mask(qbar, kbar, thr, 0.125, nbh=2, nbw=2)
    for i in range(16):
        assert idx[0, 0, i, : cnt[0, 0, i]].tolist() == kept


def exact_top_p(w: np.ndarray, thr: float):
    """Nucleus selection in exact rational arithmetic on a row of weights w
    (probabilities up to a common factor): the smallest set of the largest
    weights (ties: higher index first) whose complement holds at most 1 - thr
    of the total; the arg-max always belongs to it."""
    n = w.shape[0]
    order = sorted(range(n), key=lambda j: (float(w[j]), j), reverse=True)
    fr = [Fraction(float(w[j])) for j in order]
    total = sum(fr)
    tau = (Fraction(1) - Fraction(float(np.float32(thr)))) * total
    rest = total
    kept = set()
    if thr >= 1.0:
        return set(range(n))
    for m in range(1, n + 1):
        rest -= fr[m - 1]
        kept.add(order[m - 1])
        if rest <= tau:
            break
    return kept


@pytest.mark.parametrize("thr", [0.3, 0.5, 0.7, 0.9, 0.95, 0.99])
def test_cdf_rule_equals_exact_top_p(oracle_lib, thr):
    """The oracle's CDF rule on the softmax numerators of real rows equals
    exact top-p selection; rows whose cumulative mass comes within 1e-12 of
    the threshold (where fp64 rounding could decide) are skipped."""
    w = inputs.Workload("pin", 1, 3, 64, 4, 16, 24, 1.0, thr, seed=21)
    q, k, _ = inputs.make_qkv(w)
    qbar = oracle_lib.pool(oracle_lib.flatten(q, w.T, w.H, w.W).reshape(q.shape))
    kbar = oracle_lib.pool(oracle_lib.flatten(k, w.T, w.H, w.W).reshape(k.shape))
    checked = 0
    for hd in range(w.Hh):
        for i in range(w.Nb):
            e = oracle_lib.block_numerators_row(qbar[0, hd], kbar[0, hd], i, w.scale)
            keep, cum, band, argmax = oracle_lib.cdf_keep(e, thr)
            if np.any(np.abs(cum - (1.0 - float(np.float32(thr)))) < 1e-12):
                continue
            assert set(np.nonzero(keep)[0].tolist()) == exact_top_p(e, thr)
            assert keep[int(np.argmax(e))]
            checked += 1
    assert checked >= w.Hh * w.Nb - 2


def test_numerators_are_the_unnormalised_probabilities(oracle_lib, tiny_flat):
    """e_j = exp(s_j - max s) with the maximum exactly 1, and e / sum(e)
    rounded to fp32 is the probability row."""
    w, _, (qf, kf, vf) = tiny_flat
    qbar, kbar = oracle_lib.pool(qf), oracle_lib.pool(kf)
    for hd in range(w.Hh):
        for i in range(w.Nb):
            e = oracle_lib.block_numerators_row(qbar[0, hd], kbar[0, hd], i, w.scale)
            p = oracle_lib.block_probs_row(qbar[0, hd], kbar[0, hd], i, w.scale)
            assert e.max() == np.float32(1.0) and np.all(e > 0)
            Z = float(np.sum(e.astype(np.float64)))
            assert np.array_equal((e.astype(np.float64) / Z).astype(np.float32), p)


def test_mask_invariants_mass_and_minimality(oracle_lib):
    w = inputs.Workload("pin", 1, 4, 64, 4, 16, 32, 1.0, 0.8, seed=5)
    q, k, _ = inputs.make_qkv(w)
    qbar = oracle_lib.pool(oracle_lib.flatten(q, w.T, w.H, w.W).reshape(q.shape))
    kbar = oracle_lib.pool(oracle_lib.flatten(k, w.T, w.H, w.W).reshape(k.shape))
    cnt, idx, status, probs = oracle_lib.build_mask(qbar, kbar, w.thr, w.scale, w.nbh, w.nbw, want_probs=True)
    for hd in range(w.Hh):
        for i in range(w.Nb):
            lst = idx[0, hd, i, : cnt[0, hd, i]]
            assert np.all(np.diff(lst) > 0)
            p = probs[0, hd, i].astype(np.float64)
            kept_mass = math.fsum(p[lst])
            # the rule runs on the exact quotients e / Z; p holds them
            # rounded to fp32, each within 2^-24 relative
            tol = 2.0 ** -23
            assert kept_mass >= w.thr - tol
            # arg-max kept
            assert int(np.argmax(p)) in set(lst.tolist())
            # minimality: dropping the smallest kept block leaves less than thr
            if len(lst) > 1:
                assert kept_mass - p[lst].min() < w.thr + tol
            assert np.array_equal(np.nonzero(status[0, hd, i] & 1)[0], lst)


def test_thr_one_keeps_all_and_thr_zero_keeps_argmax(oracle_lib, tiny_flat):
    w, _, (qf, kf, vf) = tiny_flat
    qbar, kbar = oracle_lib.pool(qf), oracle_lib.pool(kf)
    cnt, idx, _, probs = oracle_lib.build_mask(qbar, kbar, 1.0, w.scale, w.nbh, w.nbw, want_probs=True)
    assert np.all(cnt == w.Nb)
    cnt0, idx0, _, _ = oracle_lib.build_mask(qbar, kbar, 0.0, w.scale, w.nbh, w.nbw)
    assert np.all(cnt0 == 1)
    assert np.array_equal(idx0[..., 0], np.argmax(probs, axis=-1))


# ----------------------------------------------------------------------------
# STA union (Metodologia item 3)
# ----------------------------------------------------------------------------
def read_sta_counts():
    rows = []
    with open(os.path.join(GOLDEN, "sta_counts.txt")) as fh:
        for line in fh:
            if line.startswith("#") or not line.strip():
                continue
            rows.append(tuple(int(x) for x in line.split()))
    return rows


@pytest.mark.parametrize("nt,nh,nw,total", read_sta_counts())
def test_sta_closed_form_counts(oracle_lib, nt, nh, nw, total):
    Nb = nt * nh * nw
    # per-row closed form
    def axis(x, n):
        return min(x + 1, n - 1) - max(x - 1, 0) + 1
    grand = 0
    sample_rows = range(Nb) if Nb <= 1000 else range(0, Nb, 37)
    for i in sample_rows:
        t, h, w_ = i // (nh * nw), (i % (nh * nw)) // nw, i % nw
        expect = axis(t, nt) * axis(h, nh) * axis(w_, nw)
        # count only the candidate neighbourhood (+-1 in each coordinate)
        got = 0
        for dt in (-1, 0, 1):
            for dh in (-1, 0, 1):
                for dw in (-1, 0, 1):
                    tt, hh, ww = t + dt, h + dh, w_ + dw
                    if 0 <= tt < nt and 0 <= hh < nh and 0 <= ww < nw:
                        j = (tt * nh + hh) * nw + ww
                        got += oracle_lib.sta(i, j, nh, nw)
        assert got == expect
        if Nb <= 1000:
            assert sum(oracle_lib.sta(i, j, nh, nw) for j in range(Nb)) == expect
    # closed-form total
    assert (3 * nt - 2) * (3 * nh - 2) * (3 * nw - 2) == total


def test_sta_symmetric_and_far_blocks_excluded(oracle_lib):
    nh, nw = 6, 10
    rng = np.random.default_rng(0)
    for _ in range(500):
        i, j = rng.integers(0, 16 * nh * nw, size=2)
        assert oracle_lib.sta(int(i), int(j), nh, nw) == oracle_lib.sta(int(j), int(i), nh, nw)
    # two frames apart is outside a 3-frame window
    assert not oracle_lib.sta(0, 2 * nh * nw, nh, nw)
    assert oracle_lib.sta(0, 1 * nh * nw + nw + 1, nh, nw)


def test_sta_union_is_superset(oracle_lib):
    w = inputs.Workload("pin", 1, 2, 64, 4, 16, 24, 1.0, 0.7, sta=(3, 3, 3), seed=9)
    q, k, _ = inputs.make_qkv(w)
    qbar = oracle_lib.pool(oracle_lib.flatten(q, w.T, w.H, w.W).reshape(q.shape))
    kbar = oracle_lib.pool(oracle_lib.flatten(k, w.T, w.H, w.W).reshape(k.shape))
    _, _, st_u, _ = oracle_lib.build_mask(qbar, kbar, w.thr, w.scale, w.nbh, w.nbw, sta_window=(3, 3, 3))
    _, _, st_n, _ = oracle_lib.build_mask(qbar, kbar, w.thr, w.scale, w.nbh, w.nbw)
    union = (st_u & 1).astype(bool)
    nabla = (st_n & 1).astype(bool)
    assert np.all(union >= nabla)
    for i in range(w.Nb):
        for j in range(w.Nb):
            if oracle_lib.sta(i, j, w.nbh, w.nbw):
                assert union[0, :, i, j].all()
    assert np.array_equal(union, nabla | np.array(
        [[oracle_lib.sta(i, j, w.nbh, w.nbw) for j in range(w.Nb)] for i in range(w.Nb)])[None, None])


def sta_window_by_coordinates(i, nt, nh, nw, window):
    """Independent formulation of one row of the static window: walk the
    window's (frame, patch row, patch column) offsets in nested order, keep
    those inside the grid and map them to flattened block indices."""
    rt, rh, rw = (x // 2 for x in window)
    t, h, w_ = i // (nh * nw), (i // nw) % nh, i % nw
    out = []
    for tt in range(t - rt, t + rt + 1):
        for hh in range(h - rh, h + rh + 1):
            for ww in range(w_ - rw, w_ + rw + 1):
                if 0 <= tt < nt and 0 <= hh < nh and 0 <= ww < nw:
                    out.append((tt * nh + hh) * nw + ww)
    return out


@pytest.mark.parametrize("nt,nh,nw,total", read_sta_counts())
def test_sta_lists_golden_totals(oracle_lib, nt, nh, nw, total):
    cnt, idx = oracle_lib.sta_lists(nt, nh, nw, (3, 3, 3))
    assert int(cnt.sum()) == total
    Nb = nt * nh * nw
    for i in (range(Nb) if Nb <= 200 else range(0, Nb, 13)):
        assert list(idx[i, :cnt[i]]) == sta_window_by_coordinates(i, nt, nh, nw, (3, 3, 3))
        assert np.all(idx[i, cnt[i]:] == -1)


@pytest.mark.parametrize("window", [(1, 3, 5), (5, 1, 3), (3, 5, 1), (7, 7, 7)])
def test_sta_lists_other_windows(oracle_lib, window):
    nt, nh, nw = 5, 4, 6
    cnt, idx = oracle_lib.sta_lists(nt, nh, nw, window)
    rt, rh, rw = (x // 2 for x in window)

    def axis(x, n, r):
        return min(x + r, n - 1) - max(x - r, 0) + 1
    for i in range(nt * nh * nw):
        t, h, w_ = i // (nh * nw), (i // nw) % nh, i % nw
        assert cnt[i] == axis(t, nt, rt) * axis(h, nh, rh) * axis(w_, nw, rw)
        assert list(idx[i, :cnt[i]]) == sta_window_by_coordinates(i, nt, nh, nw, window)


def test_sta_lists_degenerate_windows(oracle_lib):
    nt, nh, nw = 3, 2, 5
    Nb = nt * nh * nw
    # 1x1x1: every block attends to itself only (tile-local attention)
    cnt, idx = oracle_lib.sta_lists(nt, nh, nw, (1, 1, 1))
    assert np.all(cnt == 1) and np.array_equal(idx[:, 0], np.arange(Nb))
    # a window reaching across the whole grid from any block: dense lists
    cnt, idx = oracle_lib.sta_lists(nt, nh, nw, (2 * nt - 1, 2 * nh - 1, 2 * nw - 1))
    assert np.all(cnt == Nb)
    assert np.array_equal(idx, np.broadcast_to(np.arange(Nb), (Nb, Nb)))


# ----------------------------------------------------------------------------
# Attention on kept tiles
# ----------------------------------------------------------------------------
def dense_attention_grid(q, k, v, scale):
    """Plain dense softmax attention in grid order, fp64, numpy."""
    qd, kd, vd = bf16_to_f64(q), bf16_to_f64(k), bf16_to_f64(v)
    B, S, Hh, D = qd.shape
    out = np.zeros((B, S, Hh, D))
    lse = np.zeros((B, Hh, S))
    for b in range(B):
        for h in range(Hh):
            l = (qd[b, :, h] @ kd[b, :, h].T) * scale
            m = l.max(axis=1, keepdims=True)
            e = np.exp(l - m)
            z = e.sum(axis=1, keepdims=True)
            out[b, :, h] = (e @ vd[b, :, h]) / z
            lse[b, h] = (m + np.log(z))[:, 0]
    return out, lse


def test_thr_one_equals_dense_attention(oracle_lib, tiny_flat):
    w, (q, k, v), (qf, kf, vf) = tiny_flat
    qbar, kbar = oracle_lib.pool(qf), oracle_lib.pool(kf)
    cnt, idx, _, _ = oracle_lib.build_mask(qbar, kbar, 1.0, w.scale, w.nbh, w.nbw, want_status=False)
    out_f, lse_f = oracle_lib.attention(qf, kf, vf, cnt, idx, w.scale)
    ref, ref_lse = dense_attention_grid(q, k, v, w.scale)
    # bring the oracle's flattened-order rows back to grid order (attention is
    # permutation-equivariant over tokens)
    perm = oracle_lib.flatten(np.arange(w.S, dtype=np.uint16).reshape(1, -1, 1).repeat(8, 2), w.T, w.H, w.W)[0, :, 0]
    perm = perm.astype(np.int64)
    np.testing.assert_allclose(out_f[:, :, :, :], ref[:, perm], rtol=0, atol=1e-10)
    np.testing.assert_allclose(lse_f, ref_lse[:, :, perm], rtol=0, atol=1e-10)


def test_attention_special_cases(oracle_lib):
    B, Hh, D, S = 1, 2, 64, 256
    Nb = S // BLOCK
    g = torch.Generator().manual_seed(17)
    q = torch.randn(B, S, Hh, D, generator=g).to(torch.bfloat16)
    k = torch.randn(B, S, Hh, D, generator=g).to(torch.bfloat16)
    v = torch.randn(B, S, Hh, D, generator=g).to(torch.bfloat16)
    # own block only -> tile-local attention
    cnt = np.ones((B, Hh, Nb), dtype=np.int32)
    idx = np.full((B, Hh, Nb, Nb), -1, dtype=np.int32)
    for i in range(Nb):
        idx[:, :, i, 0] = i
    out, lse = oracle_lib.attention(q, k, v, cnt, idx, 0.125)
    qd, kd, vd = bf16_to_f64(q), bf16_to_f64(k), bf16_to_f64(v)
    for i in range(Nb):
        sl = slice(i * BLOCK, (i + 1) * BLOCK)
        for h in range(Hh):
            l = qd[0, sl, h] @ kd[0, sl, h].T * 0.125
            e = np.exp(l - l.max(axis=1, keepdims=True))
            ref = e @ vd[0, sl, h] / e.sum(axis=1, keepdims=True)
            np.testing.assert_allclose(out[0, sl, h], ref, atol=1e-12)
    # constant V -> constant output
    vc = torch.full((B, S, Hh, D), 0.75, dtype=torch.bfloat16)
    cnt2 = np.array([[[2, 1, 3, 4]] * Hh], dtype=np.int32)
    idx2 = np.full((B, Hh, Nb, Nb), -1, dtype=np.int32)
    idx2[:, :, 0, :2] = [0, 3]
    idx2[:, :, 1, :1] = [2]
    idx2[:, :, 2, :3] = [0, 1, 2]
    idx2[:, :, 3, :4] = [0, 1, 2, 3]
    out2, _ = oracle_lib.attention(q, k, vc, cnt2, idx2, 0.125)
    np.testing.assert_allclose(out2, 0.75, atol=1e-13)
    # Q = 0 -> uniform weights -> mean of V over kept tokens
    q0 = torch.zeros_like(q)
    out3, lse3 = oracle_lib.attention(q0, k, v, cnt2, idx2, 0.125)
    for i in range(Nb):
        toks = np.concatenate([np.arange(j * BLOCK, (j + 1) * BLOCK) for j in idx2[0, 0, i, : cnt2[0, 0, i]]])
        ref = vd[0, toks].mean(axis=0)  # [Hh, D]
        np.testing.assert_allclose(out3[0, i * BLOCK:(i + 1) * BLOCK], np.broadcast_to(ref, (BLOCK, Hh, D)), atol=1e-12)
        np.testing.assert_allclose(lse3[0, :, i * BLOCK:(i + 1) * BLOCK], math.log(len(toks)), atol=1e-12)
    # empty row -> zeros and -inf
    cnt4 = np.zeros((B, Hh, Nb), dtype=np.int32)
    out4, lse4 = oracle_lib.attention(q, k, v, cnt4, idx, 0.125)
    assert np.all(out4 == 0) and np.all(np.isneginf(lse4))


# ----------------------------------------------------------------------------
# Gradient of the attention on kept tiles (backward pass for training)
# ----------------------------------------------------------------------------
def random_lists(rng, B, Hh, Nb, p_keep, empty_rows=(), unkept_col=None):
    cnt = np.zeros((B, Hh, Nb), dtype=np.int32)
    idx = np.full((B, Hh, Nb, Nb), -1, dtype=np.int32)
    for b in range(B):
        for h in range(Hh):
            for i in range(Nb):
                if i in empty_rows:
                    continue
                keep = np.nonzero(rng.random(Nb) < p_keep)[0]
                if unkept_col is not None:
                    keep = keep[keep != unkept_col]
                if keep.size == 0:
                    keep = np.array([i if i != unkept_col else (i + 1) % Nb])
                cnt[b, h, i] = keep.size
                idx[b, h, i, :keep.size] = np.sort(keep)
    return cnt, idx


def autograd_masked_attention(q, k, v, do, cnt, idx, scale):
    """Independent formulation: token-level masked softmax attention in fp64
    torch, differentiated by autograd.  Rows with no kept block are left out
    of the loss (their output is defined as 0)."""
    B, S, Hh, D = q.shape
    Nb = S // BLOCK
    blk = np.zeros((B, Hh, Nb, Nb), dtype=bool)
    for b in range(B):
        for h in range(Hh):
            for i in range(Nb):
                blk[b, h, i, idx[b, h, i, :cnt[b, h, i]]] = True
    tok = torch.from_numpy(blk).repeat_interleave(BLOCK, 2).repeat_interleave(BLOCK, 3)  # [B,Hh,S,S]
    qt, kt, vt = (x.to(torch.float64).permute(0, 2, 1, 3).clone().requires_grad_(True) for x in (q, k, v))
    logits = (qt @ kt.transpose(-1, -2)) * scale
    rows = tok.any(-1)
    p = torch.softmax(logits.masked_fill(~tok, float("-inf")), -1)
    p = torch.where(rows.unsqueeze(-1), p, torch.zeros_like(p))
    out = p @ vt
    (out * do.to(torch.float64).permute(0, 2, 1, 3)).sum().backward()
    return tuple(x.grad.permute(0, 2, 1, 3).numpy() for x in (qt, kt, vt))


@pytest.mark.parametrize("D,p_keep,empty", [(64, 0.5, ()), (128, 0.3, (2,)), (64, 1.0, ())])
def test_attention_bwd_equals_autograd(oracle_lib, D, p_keep, empty):
    rng = np.random.default_rng(7 + D)
    B, Hh, Nb = 2, 2, 5
    S = Nb * BLOCK
    q, k, v, do = (inputs.randn_bf16((B, S, Hh, D), seed=s) for s in (11, 12, 13, 14))
    cnt, idx = random_lists(rng, B, Hh, Nb, p_keep, empty_rows=empty, unkept_col=3 if p_keep < 1 else None)
    scale = 1.0 / math.sqrt(D)
    dq, dk, dv = oracle_lib.attention_bwd(q, k, v, do, cnt, idx, scale)
    rq, rk, rv = autograd_masked_attention(q, k, v, do, cnt, idx, scale)
    for got, ref in ((dq, rq), (dk, rk), (dv, rv)):
        assert np.abs(got - ref).max() <= 1e-10 * max(1.0, np.abs(ref).max())


def test_attention_bwd_sampled_equals_autograd_on_listed_blocks(oracle_lib):
    rng = np.random.default_rng(5)
    B, Hh, Nb, D = 2, 2, 6, 64
    S = Nb * BLOCK
    q, k, v, do = (inputs.randn_bf16((B, S, Hh, D), seed=s) for s in (31, 32, 33, 34))
    cnt, idx = random_lists(rng, B, Hh, Nb, 0.45, empty_rows=(1,), unkept_col=4)
    rq, rk, rv = autograd_masked_attention(q, k, v, do, cnt, idx, 0.125)
    qb, kb = np.array([5, 0, 1]), np.array([2, 4, 3])
    dq, dk, dv = oracle_lib.attention_bwd_sampled(q, k, v, do, cnt, idx, 0.125, qb, kb)
    rows = lambda blocks: np.concatenate([np.arange(j * BLOCK, (j + 1) * BLOCK) for j in blocks])  # noqa: E731
    for got, ref in ((dq, rq[:, rows(qb)]), (dk, rk[:, rows(kb)]), (dv, rv[:, rows(kb)])):
        assert np.abs(got - ref).max() <= 1e-10 * max(1.0, np.abs(ref).max())
    empty = oracle_lib.attention_bwd_sampled(q, k, v, do, cnt, idx, 0.125, np.array([], np.int32), kb)
    assert empty[0].shape == (B, 0, Hh, D)


def test_attention_bwd_invariants(oracle_lib):
    rng = np.random.default_rng(3)
    B, Hh, Nb, D = 1, 3, 6, 64
    S = Nb * BLOCK
    q, k, v, do = (inputs.randn_bf16((B, S, Hh, D), seed=s) for s in (21, 22, 23, 24))
    cnt, idx = random_lists(rng, B, Hh, Nb, 0.4, empty_rows=(4,), unkept_col=1)
    dq, dk, dv = oracle_lib.attention_bwd(q, k, v, do, cnt, idx, 0.125)
    # the softmax Jacobian's rows sum to zero, so the key gradients of one
    # head sum to zero over all key tokens
    assert np.abs(dk.sum(axis=1)).max() < 1e-9
    # each kept row's probabilities sum to one: the value gradients sum to
    # the output gradients of the rows that keep anything
    live = np.repeat(cnt > 0, BLOCK, axis=2).transpose(0, 2, 1)  # [B,S,Hh]
    dof = do.to(torch.float64).numpy() * live[..., None]
    assert np.abs(dv.sum(axis=1) - dof.sum(axis=1)).max() < 1e-9
    # a key block no row keeps, and a row that keeps nothing, get zeros
    assert not np.any(dk[:, 64:128]) and not np.any(dv[:, 64:128])
    assert not np.any(dq[:, 4 * 64:5 * 64])


# ----------------------------------------------------------------------------
# Radial window (Radial Attention article, "Zastosowanie zasad rozkladu
# energii"): half-width floor(r0 / 2^floor(log2(dt + 1))) at temporal
# distance dt
# ----------------------------------------------------------------------------
def radial_rho(dt: int, r0: int) -> int:
    """Restated with floating-point log2 (independent of the oracle's bit loop)."""
    return int(r0 // (2 ** math.floor(math.log2(dt + 1))))


def radial_enumerate(nbt, nbh, nbw, r0):
    """Row lists by walking each frame's clipped box in (frame, row, column)
    order, which is ascending flattened order."""
    per_t = nbh * nbw
    rows = []
    for i in range(nbt * per_t):
        ti, hi, wi = i // per_t, (i % per_t) // nbw, i % nbw
        out = []
        for tj in range(nbt):
            rho = radial_rho(abs(ti - tj), r0)
            for hj in range(max(0, hi - rho), min(nbh - 1, hi + rho) + 1):
                for wj in range(max(0, wi - rho), min(nbw - 1, wi + rho) + 1):
                    out.append((tj * nbh + hj) * nbw + wj)
        rows.append(out)
    return rows


RADIAL_GRIDS = [(16, 6, 10, 4), (9, 3, 5, 1), (20, 2, 2, 7), (4, 6, 10, 100), (1, 1, 1, 1), (33, 6, 10, 2)]


@pytest.mark.parametrize("nbt,nbh,nbw,r0", RADIAL_GRIDS)
def test_radial_lists_equal_enumeration_and_closed_form(oracle_lib, nbt, nbh, nbw, r0):
    cnt, idx = oracle_lib.radial_lists(nbt, nbh, nbw, r0)
    ref = radial_enumerate(nbt, nbh, nbw, r0)
    per_t = nbh * nbw
    for i, lst in enumerate(ref):
        assert idx[i, : cnt[i]].tolist() == lst
        ti, hi, wi = i // per_t, (i % per_t) // nbw, i % nbw
        closed = sum((min(hi + radial_rho(abs(ti - tj), r0), nbh - 1) - max(hi - radial_rho(abs(ti - tj), r0), 0) + 1) *
                     (min(wi + radial_rho(abs(ti - tj), r0), nbw - 1) - max(wi - radial_rho(abs(ti - tj), r0), 0) + 1)
                     for tj in range(nbt))
        assert cnt[i] == closed


def test_radial_symmetric_and_shrinking(oracle_lib):
    nbt, nbh, nbw, r0 = 12, 6, 10, 5
    per_t = nbh * nbw
    Nb = nbt * per_t
    rng = np.random.default_rng(17)
    for _ in range(3000):
        i, j = (int(x) for x in rng.integers(0, Nb, size=2))
        assert oracle_lib.radial(i, j, nbh, nbw, r0) == oracle_lib.radial(j, i, nbh, nbw, r0)
    # a spatial offset kept at temporal distance dt is kept at every smaller one
    i = 5 * per_t + 2 * nbw + 4
    for dh in range(-3, 4):
        for dw in range(-5, 6):
            kept = [oracle_lib.radial(i, tj * per_t + (2 + dh) * nbw + 4 + dw, nbh, nbw, r0)
                    for tj in range(5, nbt) if 0 <= 2 + dh < nbh and 0 <= 4 + dw < nbw]
            assert kept == sorted(kept, reverse=True)
    # co-located blocks of every frame are kept; nothing is kept when off
    assert all(oracle_lib.radial(i, tj * per_t + 2 * nbw + 4, nbh, nbw, r0) for tj in range(nbt))
    assert not any(oracle_lib.radial(i, j, nbh, nbw, 0) for j in range(Nb))


def test_radial_union_is_superset(oracle_lib):
    w = inputs.Workload("pin", 1, 2, 64, 8, 16, 24, 1.0, 0.7, seed=19)
    q, k, _ = inputs.make_qkv(w)
    qbar = oracle_lib.pool(oracle_lib.flatten(q, w.T, w.H, w.W).reshape(q.shape))
    kbar = oracle_lib.pool(oracle_lib.flatten(k, w.T, w.H, w.W).reshape(k.shape))
    cnt_a, idx_a, _, _ = oracle_lib.build_mask(qbar, kbar, w.thr, w.scale, w.nbh, w.nbw)
    cnt_u, idx_u, status, _ = oracle_lib.build_mask(qbar, kbar, w.thr, w.scale, w.nbh, w.nbw, radial_r0=2)
    cnt_r, idx_r = oracle_lib.radial_lists(w.T, w.nbh, w.nbw, 2)
    for hd in range(w.Hh):
        for i in range(w.Nb):
            u = set(idx_u[0, hd, i, : cnt_u[0, hd, i]].tolist())
            a = set(idx_a[0, hd, i, : cnt_a[0, hd, i]].tolist())
            r = set(idx_r[i, : cnt_r[i]].tolist())
            assert u == a | r
            # window blocks are forced, never band
            assert not any(status[0, hd, i, j] & 2 for j in r)


def test_generator_is_deterministic_and_shaped():
    w = inputs.Workload("g", 1, 2, 64, 2, 8, 16, 1.0, 0.9, seed=3)
    a = inputs.make_qkv(w)
    b = inputs.make_qkv(w)
    for x, y in zip(a, b):
        assert x.dtype == torch.bfloat16 and x.shape == (1, w.S, 2, 64)
        assert torch.equal(x, y)
    idx = inputs.sample_query_blocks(960)
    assert len(idx) == 64 and len(set(idx.tolist())) == 64 and np.all(np.diff(idx) > 0)


def test_band_marks_only_blocks_near_the_threshold(oracle_lib):
    """Band blocks are exactly those whose cumulative mass lies within 1e-5
    of 1 - thr; probabilities one ulp apart are ordered by value (the larger
    one is kept), not banded."""
    one_ulp_up = np.nextafter(np.float32(0.06), np.float32(1.0))
    # ascending: 0.06 (c = 0.06 <= 0.1), then 0.06 + 1 ulp (c = 0.12 > 0.1)
    p = np.array([0.8, 0.06, one_ulp_up, 0.2], dtype=np.float32)
    p = p / p.astype(np.float64).sum()  # weights: the rule normalises anyway
    keep, cum, band, argmax = oracle_lib.cdf_keep(p.astype(np.float32), 0.9)
    assert keep.tolist() == [True, False, True, True]
    assert not band.any()
    # the same with the two near-equal weights swapped between blocks
    p_sw = np.array([0.8, one_ulp_up, 0.06, 0.2], dtype=np.float32)
    keep_sw, _, band_sw, _ = oracle_lib.cdf_keep(p_sw, 0.9)
    assert keep_sw.tolist() == [True, True, False, True] and not band_sw.any()
    # exactly equal weights across the threshold: the higher index is kept
    p_eq = np.array([0.8, 0.06, 0.06, 0.2], dtype=np.float32)
    keep_eq, _, band_eq, _ = oracle_lib.cdf_keep(p_eq, 0.9)
    assert keep_eq.tolist() == [True, False, True, True] and not band_eq.any()
    # a block whose cumulative mass sits 5e-6 above the threshold
    tau = 1.0 - float(np.float32(0.9))
    p3 = np.array([0.6, np.float32(tau + 5e-6), 0.3 - 5e-6], dtype=np.float32)  # sums to 1
    keep3, cum3, band3, _ = oracle_lib.cdf_keep(p3, 0.9)
    assert keep3.tolist() == [True, True, True]
    assert band3.tolist() == [False, True, False]


def test_arg_max_of_near_equal_maxima_is_the_larger(oracle_lib):
    top = np.float32(0.4)
    p = np.array([0.2, np.nextafter(top, np.float32(1.0)), top, 0.0001], dtype=np.float32)
    keep, cum, band, argmax = oracle_lib.cdf_keep(p, 0.0)  # thr 0: only the arg-max is kept
    assert argmax == 1 and keep.tolist() == [False, True, False, False]
    p2 = np.array([0.2, top, top, 0.0001], dtype=np.float32)  # exact tie: the higher index
    _, _, _, argmax2 = oracle_lib.cdf_keep(p2, 0.0)
    assert argmax2 == 2


def test_parity_helper_flat_order_matches_oracle_flatten(oracle_lib):
    """The tests' own flat->grid row index (used to compare grid-order
    attention outputs) agrees with the oracle's flattening."""
    from _parity import flat_order
    for T, H, W in ((1, 8, 8), (2, 16, 24), (3, 24, 16)):
        S = T * H * W
        ids = np.arange(S, dtype=np.uint16).reshape(1, S, 1)
        flat = oracle_lib.flatten(ids, T, H, W).reshape(-1)
        assert np.array_equal(flat, flat_order(T, H, W).astype(np.uint16))


def test_parity_helper_sampled_gradient_errors(oracle_lib):
    """The GPU tests' sampled-gradient comparison, fed the full oracle
    gradient in place of the GPU's: zero error on the listed blocks, and a
    planted error in a listed block is seen."""
    import sys
    sys.path.insert(0, os.path.dirname(__file__))
    from _parity import sampled_gradient_errors
    rng = np.random.default_rng(8)
    B, Hh, Nb, D = 1, 2, 7, 64
    S = Nb * BLOCK
    q, k, v, do = (inputs.randn_bf16((B, S, Hh, D), seed=s) for s in (41, 42, 43, 44))
    cnt, idx = random_lists(rng, B, Hh, Nb, 0.4)
    full = [torch.from_numpy(x) for x in oracle_lib.attention_bwd(q, k, v, do, cnt, idx, 0.125)]
    qb, kb = np.array([6, 2]), np.array([0, 5, 3])
    ref = oracle_lib.attention_bwd_sampled(q, k, v, do, cnt, idx, 0.125, qb, kb)
    for mx, mean in sampled_gradient_errors(*full, ref, qb, kb):
        assert mx < 1e-12 and mean < 1e-12
    full[1][:, 5 * BLOCK + 3, 1, 7] += 1.0  # key block 5 is listed
    errs = sampled_gradient_errors(*full, ref, qb, kb)
    assert errs[1][0] > 1e-3 and errs[0][0] < 1e-12 and errs[2][0] < 1e-12
