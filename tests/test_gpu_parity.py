"""GPU parity of every stage against the CPU oracle, through the C ABI.

Small and edge-case shapes: the tiny layer in full, odd block counts (a
query-block pair with one half missing), a single block, D = 64 and 128,
thr = 0 and 1, hand-built block lists whose two paired query blocks
disagree, empty rows, corrupted lists, and inputs whose logits grow along
the walk so the lazy O rescale runs.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from _parity import (Case, LSE_ABS, MAX_ABS, MEAN_ABS, check_attention, compare_masks, flat_to_grid_rows,
                     grid_to_flat_rows, oracle_masks)
from block_sparse_attention_flatten_b200 import inputs
from block_sparse_attention_flatten_b200 import nabla

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from block_sparse_attention_flatten_b200 import build
    build.build()
    assert torch.cuda.is_available()
    oracle.build()
    yield
    torch.cuda.synchronize()


SMALL = [
    inputs.TINY,
    inputs.Workload("odd Nb=3 D64", 1, 2, 64, 3, 8, 8, 0.0, 0.9, seed=31),
    inputs.Workload("odd Nb=3 D128", 1, 3, 128, 1, 8, 24, 1.0, 0.7, seed=32),
    inputs.Workload("single block", 1, 2, 128, 1, 8, 8, 0.0, 0.9, seed=33),
    inputs.Workload("Nb=45 D128 STA", 2, 2, 128, 5, 24, 24, 1.0, 0.8, sta=(3, 3, 3), seed=34),
    inputs.Workload("Nb=24 D64 dense", 1, 4, 64, 2, 16, 48, 1.0, 1.0, seed=35),
    inputs.Workload("Nb=24 thr0", 1, 2, 128, 2, 16, 48, 1.0, 0.0, seed=36),
    inputs.Workload("Nb=35 D64 STA 5x3x1", 1, 2, 64, 5, 8, 56, 1.0, 0.6, sta=(5, 3, 1), seed=37),
    inputs.Workload("Nb=45 D64 thr0 STA", 1, 2, 64, 5, 24, 24, 1.0, 0.0, sta=(3, 3, 3), seed=38),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_small_layers_end_to_end(w):
    case = Case(w)
    qf_h, kf_h, vf_h = case.host_flat()
    # flattening is bit-exact
    case.assert_flatten_matches_oracle()
    # pooling: same fp32 sum order as the oracle -> bit-exact
    qbar, kbar, cnt_o, idx_o, status = oracle_masks(case, qf_h, kf_h)
    qg, kg = nabla.pooled_from_workspace(case.ws, w.B, w.Hh, w.Nb, w.D)
    assert np.array_equal(qg.cpu().numpy(), qbar)
    assert np.array_equal(kg.cpu().numpy(), kbar)
    # masks: bit-exact outside the band
    bad, in_band, nband = compare_masks(case, status)
    assert bad == 0, f"{bad} mask mismatches outside the band ({in_band} inside, {nband} band blocks)"
    # attention on every query block, against the oracle on the GPU's lists,
    # through both entry points (pairs 2p, 2p+1 and the grid-aware pairing)
    for grid in (False, True):
        out, lse = case.attention(grid=grid)
        mx, mean, lse_err = check_attention(case, out, lse, np.arange(w.Nb), (qf_h, kf_h, vf_h))
        assert mx <= MAX_ABS and mean <= MEAN_ABS and lse_err <= LSE_ABS, (grid, mx, mean, lse_err)
    # unflatten brings the output back to grid order bit-exactly
    o_grid = nabla.unflatten(out, w.T, w.H, w.W)
    ref = oracle.unflatten(out.cpu(), w.T, w.H, w.W).reshape(out.shape)
    assert np.array_equal(o_grid.cpu().view(torch.int16).numpy().view(np.uint16), ref)


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_fused_flatten_pool_and_pooled_mask(w):
    """nabla_flatten_pool_qk writes the oracle's flattening (bit-exact) and its
    pooled means (bit-exact, same fp32 order); nabla_build_mask_pooled on that
    workspace gives the same block lists as nabla_build_mask."""
    q, k, _ = inputs.make_qkv(w)
    qd, kd = q.cuda(), k.cuda()
    qf, kf, ws = nabla.flatten_pool_qk(qd, kd, w.T, w.H, w.W, thr=w.thr, sta=w.sta)
    cnt, idx = nabla.build_mask_pooled(ws, w.B, w.Hh, w.D, w.T, w.H, w.W, w.thr, w.sta)
    torch.cuda.synchronize()
    assert nabla.get_status() == 0
    qf_ref = oracle.flatten(q, w.T, w.H, w.W).reshape(q.shape)
    kf_ref = oracle.flatten(k, w.T, w.H, w.W).reshape(k.shape)
    assert np.array_equal(qf.cpu().view(torch.int16).numpy().view(np.uint16), qf_ref)
    assert np.array_equal(kf.cpu().view(torch.int16).numpy().view(np.uint16), kf_ref)
    qg, kg = nabla.pooled_from_workspace(ws, w.B, w.Hh, w.Nb, w.D)
    assert np.array_equal(qg.cpu().numpy(), oracle.pool(qf_ref))
    assert np.array_equal(kg.cpu().numpy(), oracle.pool(kf_ref))
    cnt2, idx2, _ = nabla.build_mask(qf, kf, w.T, w.H, w.W, w.thr, w.sta)
    cnt3, idx3, ws3 = nabla.build_mask_grid(qd, kd, w.T, w.H, w.W, w.thr, w.sta)  # straight from grid order
    torch.cuda.synchronize()
    for a_, b_ in zip(nabla.pooled_from_workspace(ws3, w.B, w.Hh, w.Nb, w.D), (qg, kg)):
        assert torch.equal(a_, b_)  # the pooled vectors (the workspace's padding columns are never written)
    valid = torch.arange(w.Nb, device="cuda").view(1, 1, 1, -1) < cnt.unsqueeze(-1)
    for c_, i_ in ((cnt2, idx2), (cnt3, idx3)):
        assert torch.equal(cnt, c_)
        assert torch.equal(torch.where(valid, idx, -1), torch.where(valid, i_, -1))


def dense_grid(q, k, v, scale):
    qd, kd, vd = q.double(), k.double(), v.double()
    B, S, Hh, D = qd.shape
    out = torch.empty_like(qd)
    for b in range(B):
        for h in range(Hh):
            l = qd[b, :, h] @ kd[b, :, h].T * scale
            out[b, :, h] = torch.softmax(l, dim=-1) @ vd[b, :, h]
    return out


def test_thr_one_full_path_equals_dense_attention():
    """flatten -> mask(thr=1) -> sparse attention -> unflatten == dense attention."""
    w = inputs.Workload("dense", 1, 3, 128, 3, 16, 24, 1.0, 1.0, seed=41)
    case = Case(w)
    assert torch.all(case.kv_count == w.Nb)
    out, _ = case.attention()
    o = nabla.unflatten(out, w.T, w.H, w.W).double().cpu()
    ref = dense_grid(case.q, case.k, case.v, w.scale)
    err = (o - ref).abs()
    assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS


def test_unflatten_inverts_flatten_other_row_widths():
    g = torch.Generator().manual_seed(5)
    for (T, H, W, row) in [(2, 8, 16, 8), (3, 24, 16, 24), (1, 48, 80, 3072), (7, 8, 8, 64)]:
        x = torch.randn(2, T * H * W, row, generator=g).to(torch.bfloat16).cuda()
        f = nabla.flatten(x, T, H, W)
        ref = oracle.flatten(x.cpu(), T, H, W)
        assert np.array_equal(f.cpu().view(torch.int16).numpy().view(np.uint16), ref)
        assert torch.equal(nabla.unflatten(f, T, H, W), x)


def random_lists(B, Hh, Nb, rng, pmax=0.6):
    cnt = np.zeros((B, Hh, Nb), dtype=np.int32)
    idx = np.full((B, Hh, Nb, Nb), -1, dtype=np.int32)
    for b in range(B):
        for h in range(Hh):
            for i in range(Nb):
                p = rng.uniform(0.05, pmax)
                sel = np.nonzero(rng.random(Nb) < p)[0]
                if sel.size == 0:
                    sel = np.array([rng.integers(Nb)])
                cnt[b, h, i] = sel.size
                idx[b, h, i, : sel.size] = sel
    return cnt, idx


@pytest.mark.parametrize("D,Nb_t,logit_scale", [(128, 5, 1.0), (64, 4, 1.0), (128, 3, 6.0), (64, 5, 6.0)])
def test_hand_built_lists_pairs_disagree(D, Nb_t, logit_scale):
    """Random lists per query block (the two halves of a pair differ), and
    large logits so the running max moves and O is rescaled."""
    rng = np.random.default_rng(D * 10 + Nb_t)
    T, H, W, Hh, B = Nb_t, 8, 40, 2, 1  # Nb = 5 * Nb_t blocks
    S = T * H * W
    Nb = S // 64
    g = torch.Generator().manual_seed(D + Nb_t)
    q = (torch.randn(B, S, Hh, D, generator=g) * logit_scale).to(torch.bfloat16)
    k = torch.randn(B, S, Hh, D, generator=g).to(torch.bfloat16)
    # With peaked softmax rows the output approaches single V entries (|v| up
    # to ~4.5), where one bf16 output ulp alone is 2^-5; V is scaled so the
    # fixed 2e-2 bound tests the rescaling arithmetic, not bf16 quantisation.
    v = (torch.randn(B, S, Hh, D, generator=g) / logit_scale).to(torch.bfloat16)
    cnt, idx = random_lists(B, Hh, Nb, rng)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    cnt_d = torch.from_numpy(cnt).cuda()
    idx_d = torch.from_numpy(idx).cuda()
    out, lse = nabla.sparse_attn_fwd(qd, kd, vd, cnt_d, idx_d)
    torch.cuda.synchronize()
    assert nabla.get_status() == 0
    ref, ref_lse = oracle.attention(q, k, v, cnt, idx, 1.0 / math.sqrt(D))
    err = np.abs(out.double().cpu().numpy() - ref)
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
    assert np.abs(lse.double().cpu().numpy() - ref_lse).max() <= LSE_ABS * max(1.0, logit_scale)


@pytest.mark.parametrize("grid", [None, (12, 16, 64)], ids=["pairs", "grid"])
def test_long_lists(grid):
    """Lists longer than the 32 entries the kernel reads ahead of their count
    (and longer than a CTA's thread count), with the two paired halves
    disagreeing."""
    rng = np.random.default_rng(77)
    T, H, W, Hh, B, D = 12, 16, 64, 1, 1, 64  # Nb = 192
    S = T * H * W
    Nb = S // 64
    g = torch.Generator().manual_seed(78)
    q, k, v = (torch.randn(B, S, Hh, D, generator=g).to(torch.bfloat16) for _ in range(3))
    cnt = np.zeros((B, Hh, Nb), dtype=np.int32)
    idx = np.full((B, Hh, Nb, Nb), -1, dtype=np.int32)
    for i in range(Nb):
        n = int(rng.choice([5, 33, 64, 150, Nb]))
        sel = np.sort(rng.choice(Nb, size=n, replace=False))
        cnt[0, 0, i] = n
        idx[0, 0, i, :n] = sel
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    cnt_d, idx_d = torch.from_numpy(cnt).cuda(), torch.from_numpy(idx).cuda()
    if grid is None:
        out, lse = nabla.sparse_attn_fwd(qd, kd, vd, cnt_d, idx_d)
    else:
        qg, kg, vg = (flat_to_grid_rows(x, *grid, 1) for x in (qd, kd, vd))
        out, lse = nabla.sparse_attn_fwd(qg, kg, vg, cnt_d, idx_d, grid=grid)
        out, lse = grid_to_flat_rows(out, *grid, 1), grid_to_flat_rows(lse, *grid, 2)
    torch.cuda.synchronize()
    assert nabla.get_status() == 0
    ref, ref_lse = oracle.attention(q, k, v, cnt, idx, 1.0 / math.sqrt(D))
    err = np.abs(out.double().cpu().numpy() - ref)
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
    assert np.abs(lse.double().cpu().numpy() - ref_lse).max() <= LSE_ABS


def grouped_lists(T, nbh, nbw, Hh, rng):
    """Block lists on a T x nbh x nbw block grid whose 2 x 2 (w, t) groups
    push the grid-aware pairing both ways: in 'w' groups the two horizontal
    neighbours share their list and the frames differ, in 't' groups the two
    frames share it and the neighbours differ; 'e' groups hold empty rows and
    'r' groups random lists."""
    Nb = T * nbh * nbw
    F = nbh * nbw
    cnt = np.zeros((1, Hh, Nb), dtype=np.int32)
    idx = np.full((1, Hh, Nb, Nb), -1, dtype=np.int32)
    kinds = []

    def put(h, i, sel):
        sel = np.unique(sel)
        cnt[0, h, i] = sel.size
        idx[0, h, i, :sel.size] = sel

    for h in range(Hh):
        for t in range(0, T, 2):
            for bh in range(nbh):
                for bw in range(0, nbw, 2):
                    a = t * F + bh * nbw + bw
                    g = [a, a + 1, a + F, a + F + 1]
                    kind = "wter"[rng.integers(4)]
                    kinds.append(kind)
                    lists = [rng.choice(Nb, size=rng.integers(1, Nb // 3), replace=False) for _ in range(4)]
                    if kind == "w":
                        lists[1], lists[3] = lists[0], lists[2]
                    elif kind == "t":
                        lists[2], lists[3] = lists[0], lists[1]
                    elif kind == "e":
                        lists[rng.integers(4)] = np.array([], dtype=np.int64)
                    for i, sel in zip(g, lists):
                        put(h, i, sel)
    return cnt, idx, kinds


@pytest.mark.parametrize("D", [64, 128])
def test_grid_pairing_takes_both_decisions(D):
    """The grid-aware entry point splits some groups along w and others along
    t (and handles groups with an empty row); every query block must still
    attend exactly to its own list."""
    rng = np.random.default_rng(500 + D)
    T, H, W, Hh, B = 4, 16, 32, 3, 1  # block grid 4 x 2 x 4, Nb = 32
    S = T * H * W
    nbh, nbw = H // 8, W // 8
    g = torch.Generator().manual_seed(600 + D)
    q, k, v = (torch.randn(B, S, Hh, D, generator=g).to(torch.bfloat16) for _ in range(3))
    cnt, idx, kinds = grouped_lists(T, nbh, nbw, Hh, rng)
    assert {"w", "t"} <= set(kinds)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    cnt_d = torch.from_numpy(cnt).cuda()
    idx_d = torch.from_numpy(idx).cuda()
    ref, ref_lse = oracle.attention(q, k, v, cnt, idx, 1.0 / math.sqrt(D))
    for grid in (None, (T, H, W)):
        if grid is None:  # q, k, v taken as flattened tensors
            out, lse = nabla.sparse_attn_fwd(qd, kd, vd, cnt_d, idx_d)
        else:  # the same tensors in grid order; outputs back to flattened rows
            qg, kg, vg = (flat_to_grid_rows(x, T, H, W, 1) for x in (qd, kd, vd))
            out, lse = nabla.sparse_attn_fwd(qg, kg, vg, cnt_d, idx_d, grid=grid)
            out, lse = grid_to_flat_rows(out, T, H, W, 1), grid_to_flat_rows(lse, T, H, W, 2)
        torch.cuda.synchronize()
        assert nabla.get_status() == 0
        err = np.abs(out.double().cpu().numpy() - ref)
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (grid, err.max(), err.mean())
        got_lse = lse.double().cpu().numpy()
        finite = np.isfinite(ref_lse)
        assert np.array_equal(finite, np.isfinite(got_lse))
        assert np.abs(got_lse[finite] - ref_lse[finite]).max() <= LSE_ABS
        # empty rows: exactly zero output
        empty = np.nonzero(cnt[0] == 0)
        o = out.float().cpu()
        for h, i in zip(*empty):
            assert torch.all(o[0, i * 64:(i + 1) * 64, h] == 0)


def test_grid_entry_point_rejects_bad_grids():
    x = torch.zeros(1, 1024, 1, 64, dtype=torch.bfloat16, device="cuda")
    cnt = torch.ones(1, 1, 16, dtype=torch.int32, device="cuda")
    idx = torch.zeros(1, 1, 16, 16, dtype=torch.int32, device="cuda")
    with pytest.raises(ValueError):
        nabla.sparse_attn_fwd(x, x, x, cnt, idx, grid=(4, 16, 8))  # 512 tokens, not 1024
    with pytest.raises(nabla.NablaError):
        nabla.sparse_attn_fwd(x, x, x, cnt, idx, grid=(4, 4, 64))  # H not a multiple of 8
    assert nabla.get_status() == 0


def test_empty_rows_give_zero_output_and_neg_inf_lse():
    B, Hh, D, S = 1, 2, 128, 512
    Nb = S // 64
    g = torch.Generator().manual_seed(8)
    q, k, v = (torch.randn(B, S, Hh, D, generator=g).to(torch.bfloat16).cuda() for _ in range(3))
    cnt = torch.zeros(B, Hh, Nb, dtype=torch.int32)
    idx = torch.zeros(B, Hh, Nb, Nb, dtype=torch.int32)
    cnt[0, 0, 2] = 2  # block 2 of head 0 attends blocks 1 and 5; its pair partner (3) has nothing
    idx[0, 0, 2, :2] = torch.tensor([1, 5])
    out, lse = nabla.sparse_attn_fwd(q, k, v, cnt.cuda(), idx.cuda())
    torch.cuda.synchronize()
    assert nabla.get_status() == 0
    o = out.float().cpu()
    l = lse.cpu()
    assert torch.all(o[0, 3 * 64:4 * 64] == 0)
    assert torch.all(o[0, :, 1] == 0) and torch.all(torch.isneginf(l[0, 1]))
    assert torch.all(torch.isneginf(l[0, 0, 3 * 64:4 * 64]))
    assert torch.all(torch.isfinite(l[0, 0, 2 * 64:3 * 64]))


def test_corrupted_lists_are_reported_not_faulted():
    B, Hh, D, S = 1, 1, 64, 256
    Nb = S // 64
    g = torch.Generator().manual_seed(9)
    q, k, v = (torch.randn(B, S, Hh, D, generator=g).to(torch.bfloat16).cuda() for _ in range(3))
    cnt = torch.full((B, Hh, Nb), 2, dtype=torch.int32)
    idx = torch.zeros(B, Hh, Nb, Nb, dtype=torch.int32)
    idx[..., 0] = 0
    idx[..., 1] = 1
    idx[0, 0, 3, 1] = Nb + 7  # out of range: skipped by the kernel and reported
    assert nabla.validate_mask(cnt.cuda(), idx.cuda()) == 1
    out, _ = nabla.sparse_attn_fwd(q, k, v, cnt.cuda(), idx.cuda())
    assert nabla.get_status() == nabla.NABLA_ERR_DEVICE_BOUNDS
    assert nabla.get_status() == 0  # cleared
    # the row that lost its bad entry attends block 0 only
    cnt_ref = cnt.numpy().copy()
    cnt_ref[0, 0, 3] = 1
    ref, _ = oracle.attention(q.cpu(), k.cpu(), v.cpu(), cnt_ref, idx.numpy(), 0.125)
    err = np.abs(out.double().cpu().numpy() - ref)
    assert err.max() <= MAX_ABS


def test_stream_argument_is_honoured():
    w = inputs.TINY
    q, k, v = inputs.make_qkv(w)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
        qf = nabla.flatten(qd, w.T, w.H, w.W)
        kf = nabla.flatten(kd, w.T, w.H, w.W)
        vf = nabla.flatten(vd, w.T, w.H, w.W)
        cnt, idx, _ = nabla.build_mask(qf, kf, w.T, w.H, w.W, w.thr)
        out, lse = nabla.sparse_attn_fwd(qf, kf, vf, cnt, idx)
    s.synchronize()
    case = Case(w, q, k, v)
    out2, _ = case.attention()
    assert torch.equal(out, out2) and torch.equal(cnt, case.kv_count)


def test_bounded_wait_times_out_without_faulting():
    """A wait on a barrier nothing completes gives up after its limit, records
    NABLA_ERR_DEVICE_TIMEOUT, and leaves the context usable."""
    assert nabla.get_status() == 0
    assert nabla.selftest_wait_timeout(2_000_000) == nabla.NABLA_ERR_DEVICE_TIMEOUT
    assert nabla.get_status() == 0  # read-and-clear
    w = inputs.Workload("after timeout", 1, 2, 64, 1, 8, 16, 0.0, 0.9, seed=51)
    case = Case(w)
    out, lse = case.attention()
    assert torch.isfinite(out.float()).all()
