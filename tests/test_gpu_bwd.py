"""GPU parity of the backward pass (nabla_transpose_lists,
nabla_sparse_attn_bwd and its grid-order form) against the CPU oracle.

* The transposed block lists are integer work: bit-exact against a plain
  transposition of the row lists.
* dQ, dK, dV (bf16) against the fp64 oracle gradient on the GPU's own lists:
  the products round P and dS to bf16 (relative error <= 2^-9 each) and the
  outputs are rounded to bf16 (<= 2^-9); with cancellation inside dK and dQ
  the error is bounded relative to the gradient's scale, not per element:
  max |err| <= 2e-2 * max |ref| and mean |err| <= 1e-2 * mean |ref| (about
  five times the largest single rounding).
"""
import numpy as np
import pytest
import torch

import oracle
from _parity import Case, grid_to_flat_rows, sampled_gradient_errors
from block_sparse_attention_flatten_b200 import inputs
from block_sparse_attention_flatten_b200 import nabla

pytestmark = pytest.mark.gpu

MAX_REL = 2e-2
MEAN_REL = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _built():
    from block_sparse_attention_flatten_b200 import build
    build.build()
    assert torch.cuda.is_available()
    oracle.build()
    yield
    torch.cuda.synchronize()


def transpose_host(cnt: np.ndarray, idx: np.ndarray):
    B, Hh, Nb = cnt.shape
    qc = np.zeros_like(cnt)
    qi = np.full_like(idx, -1)
    for b in range(B):
        for h in range(Hh):
            cols = [[] for _ in range(Nb)]
            for i in range(Nb):
                for j in idx[b, h, i, :cnt[b, h, i]]:
                    cols[j].append(i)
            for j in range(Nb):
                qc[b, h, j] = len(cols[j])
                qi[b, h, j, :len(cols[j])] = cols[j]
    return qc, qi


def check_transpose(kv_count, kv_idx):
    qc, qi = nabla.transpose_lists(kv_count, kv_idx)
    torch.cuda.synchronize()
    assert nabla.get_status() == 0
    rc, ri = transpose_host(kv_count.cpu().numpy(), kv_idx.cpu().numpy())
    assert np.array_equal(qc.cpu().numpy(), rc)
    Nb = kv_count.shape[-1]
    valid = np.arange(Nb)[None, None, None, :] < rc[..., None]
    assert np.array_equal(np.where(valid, qi.cpu().numpy(), -1), ri)
    return qc, qi


def hand_lists(B, Hh, Nb, seed, p_keep=0.4, empty_row=None, unkept_col=None):
    rng = np.random.default_rng(seed)
    cnt = np.zeros((B, Hh, Nb), dtype=np.int32)
    idx = np.full((B, Hh, Nb, Nb), -1, dtype=np.int32)
    for b in range(B):
        for h in range(Hh):
            for i in range(Nb):
                if i == empty_row:
                    continue
                keep = np.nonzero(rng.random(Nb) < p_keep)[0]
                keep = keep[keep != unkept_col] if unkept_col is not None else keep
                if keep.size == 0:
                    keep = np.array([i if i != unkept_col else (i + 1) % Nb])
                cnt[b, h, i] = keep.size
                idx[b, h, i, :keep.size] = keep
    return torch.from_numpy(cnt).cuda(), torch.from_numpy(idx).cuda()


def rel_errors(got: torch.Tensor, ref: np.ndarray):
    err = np.abs(got.double().cpu().numpy() - ref)
    scale_max, scale_mean = np.abs(ref).max(), np.abs(ref).mean()
    return err.max() / max(scale_max, 1e-30), err.mean() / max(scale_mean, 1e-30)


def run_backward(w: inputs.Workload, grid: bool, lists=None, seed_do: int = 99):
    """Forward + backward through the C ABI; returns the flattened-order
    gradients and the oracle's."""
    case = Case(w)
    if lists is not None:
        case.kv_count, case.kv_idx = lists
    kv_count, kv_idx = case.kv_count, case.kv_idx
    do = inputs.randn_bf16((w.B, w.S, w.Hh, w.D), seed=seed_do)  # output gradient, grid order
    dod = do.cuda()
    q_lists = check_transpose(kv_count, kv_idx)
    if grid:
        out, lse = nabla.sparse_attn_fwd(case.qd, case.kd, case.vd, kv_count, kv_idx, grid=(w.T, w.H, w.W))
        dq, dk, dv = nabla.sparse_attn_bwd(case.qd, case.kd, case.vd, out, dod, lse, kv_count, kv_idx,
                                           q_lists=q_lists, grid=(w.T, w.H, w.W))
        dq, dk, dv = (grid_to_flat_rows(x, w.T, w.H, w.W, 1) for x in (dq, dk, dv))
    else:
        dof = nabla.flatten(dod, w.T, w.H, w.W)
        out, lse = nabla.sparse_attn_fwd(case.qf, case.kf, case.vf, kv_count, kv_idx)
        dq, dk, dv = nabla.sparse_attn_bwd(case.qf, case.kf, case.vf, out, dof, lse, kv_count, kv_idx,
                                           q_lists=q_lists)
    torch.cuda.synchronize()
    assert nabla.get_status() == 0
    qf, kf, vf = case.host_flat()
    dof_h = oracle.flatten(do, w.T, w.H, w.W).reshape(do.shape)
    ref = oracle.attention_bwd(qf, kf, vf, dof_h, kv_count.cpu().numpy(), kv_idx.cpu().numpy(), w.scale)
    return (dq, dk, dv), ref, case


BWD_CASES = [
    inputs.TINY,
    inputs.Workload("odd Nb=3 D128", 1, 3, 128, 1, 8, 24, 1.0, 0.7, seed=32),
    inputs.Workload("Nb=45 D128 STA B2", 2, 2, 128, 5, 24, 24, 1.0, 0.8, sta=(3, 3, 3), seed=34),
    inputs.Workload("Nb=24 D64 dense", 1, 4, 64, 2, 16, 48, 1.0, 1.0, seed=35),
    inputs.Workload("Nb=24 thr0", 1, 2, 128, 2, 16, 48, 1.0, 0.0, seed=36),
    inputs.Workload("Nb=35 D64 STA 5x3x1", 1, 2, 64, 5, 8, 56, 1.0, 0.6, sta=(5, 3, 1), seed=37),
    inputs.Workload("Nb=240 D128 Wan-like 4x48x80", 1, 3, 128, 4, 48, 80, 1.0, 0.7, seed=2),
]


@pytest.mark.parametrize("grid", [False, True], ids=["flat", "grid"])
@pytest.mark.parametrize("w", BWD_CASES, ids=lambda w: w.name)
def test_backward_matches_oracle(w, grid):
    got, ref, _ = run_backward(w, grid)
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        mx, mean = rel_errors(g, r)
        print(f"\n{w.name} {'grid' if grid else 'flat'} {name}: max/max|ref| {mx:.2e}, mean/mean|ref| {mean:.2e}")
        assert mx <= MAX_REL and mean <= MEAN_REL, (name, mx, mean)


@pytest.mark.parametrize("D", [64, 128])
def test_backward_empty_rows_and_unkept_blocks(D):
    w = inputs.Workload(f"hand lists D{D}", 1, 2, D, 3, 16, 16, 0.0, 0.9, seed=51)  # Nb = 12
    lists = hand_lists(w.B, w.Hh, w.Nb, seed=52, empty_row=5, unkept_col=7)
    (dq, dk, dv), ref, _ = run_backward(w, grid=False, lists=lists)
    for g, r in zip((dq, dk, dv), ref):
        mx, mean = rel_errors(g, r)
        assert mx <= MAX_REL and mean <= MEAN_REL
    assert not bool(dq[:, 5 * 64:6 * 64].any())                     # empty row: dQ = 0
    assert not bool(dk[:, 7 * 64:8 * 64].any()) and not bool(dv[:, 7 * 64:8 * 64].any())  # unkept block


def test_backward_is_deterministic():
    w = inputs.Workload("determinism", 1, 2, 128, 2, 16, 48, 1.0, 0.9, seed=53)
    case = Case(w)
    do = inputs.randn_bf16((w.B, w.S, w.Hh, w.D), seed=54).cuda()
    out, lse = nabla.sparse_attn_fwd(case.qd, case.kd, case.vd, case.kv_count, case.kv_idx, grid=(w.T, w.H, w.W))
    g1 = nabla.sparse_attn_bwd(case.qd, case.kd, case.vd, out, do, lse, case.kv_count, case.kv_idx,
                               grid=(w.T, w.H, w.W))
    g2 = nabla.sparse_attn_bwd(case.qd, case.kd, case.vd, out, do, lse, case.kv_count, case.kv_idx,
                               grid=(w.T, w.H, w.W))
    torch.cuda.synchronize()
    for a_, b_ in zip(g1, g2):
        assert torch.equal(a_, b_)


def test_backward_full_size_properties():
    """Wan-1.3B-like layer at full size (about 1.2e12 algorithmic FLOP per
    backward: minutes of the scalar fp64 oracle per run, so it is not
    compared element by element here): the transposed lists bit-exact,
    and two identities of the exact gradient that hold at any size -- the
    key gradients of a head sum to zero over all key tokens, and the value
    gradients sum to the output gradients of the rows (every row keeps a
    block).  Measured against the sums of magnitudes, with the bf16 bound."""
    w = inputs.WAN13B
    q, k, v = inputs.make_qkv(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    kv_count, kv_idx, _ = nabla.build_mask_grid(qd, kd, w.T, w.H, w.W, w.thr, w.sta)
    q_lists = check_transpose(kv_count, kv_idx)
    do = inputs.randn_bf16((w.B, w.S, w.Hh, w.D), seed=98).cuda()
    out, lse = nabla.sparse_attn_fwd(qd, kd, vd, kv_count, kv_idx, grid=(w.T, w.H, w.W))
    dq, dk, dv = nabla.sparse_attn_bwd(qd, kd, vd, out, do, lse, kv_count, kv_idx, q_lists=q_lists,
                                       grid=(w.T, w.H, w.W))
    torch.cuda.synchronize()
    assert nabla.get_status() == 0
    assert bool((kv_count > 0).all())
    for x in (dq, dk, dv):
        assert bool(torch.isfinite(x.float()).all())
    sum_dk = dk.double().sum(dim=1)                      # [B, Hh, D]
    mag_dk = dk.double().abs().sum(dim=1)
    assert float((sum_dk.abs() / mag_dk).max()) <= 1e-2
    sum_dv = dv.double().sum(dim=1)
    sum_do = do.double().sum(dim=1)
    mag_dv = dv.double().abs().sum(dim=1)
    assert float(((sum_dv - sum_do).abs() / mag_dv).max()) <= 1e-2
    # timing (printed, not asserted): transposition + backward, L2 warm
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    for _ in range(3):
        nabla.sparse_attn_bwd(qd, kd, vd, out, do, lse, kv_count, kv_idx, q_lists=q_lists, dq=dq, dk=dk, dv=dv,
                              grid=(w.T, w.H, w.W))
    ev[0].record()
    ql = nabla.transpose_lists(kv_count, kv_idx)
    ev[1].record()
    nabla.sparse_attn_bwd(qd, kd, vd, out, do, lse, kv_count, kv_idx, q_lists=ql, dq=dq, dk=dk, dv=dv,
                          grid=(w.T, w.H, w.W))
    ev[2].record()
    torch.cuda.synchronize()
    kept = float(kv_count.double().sum())
    t_bwd = ev[1].elapsed_time(ev[2])
    print(f"\nWan-like backward: transpose {ev[0].elapsed_time(ev[1]):.3f} ms, backward {t_bwd:.3f} ms, "
          f"{10 * 64 * 64 * w.D * kept / (t_bwd * 1e-3) / 1e12:.1f} TFLOP/s (algorithmic, 5 products per tile)")


def test_backward_full_size_sampled_against_oracle():
    """Wan-1.3B-like layer at full size in grid order (the layout bench.py
    times): dQ of 8 seeded query blocks and dK, dV of 4 seeded key blocks,
    all heads, element by element against the oracle's gradient restricted
    to those blocks (evaluated on the GPU's own lists)."""
    w = inputs.WAN13B
    q, k, v = inputs.make_qkv(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    kv_count, kv_idx, _ = nabla.build_mask_grid(qd, kd, w.T, w.H, w.W, w.thr, w.sta)
    do = inputs.randn_bf16((w.B, w.S, w.Hh, w.D), seed=97)
    out, lse = nabla.sparse_attn_fwd(qd, kd, vd, kv_count, kv_idx, grid=(w.T, w.H, w.W))
    dq, dk, dv = nabla.sparse_attn_bwd(qd, kd, vd, out, do.cuda(), lse, kv_count, kv_idx, grid=(w.T, w.H, w.W))
    torch.cuda.synchronize()
    assert nabla.get_status() == 0
    grads = [grid_to_flat_rows(x, w.T, w.H, w.W, 1) for x in (dq, dk, dv)]
    del out, lse, dq, dk, dv
    qb = inputs.sample_query_blocks(w.Nb, 8, seed=1234)
    kb = inputs.sample_query_blocks(w.Nb, 4, seed=4321)
    flat = [oracle.flatten(x, w.T, w.H, w.W).reshape(x.shape) for x in (q, k, v, do)]
    ref = oracle.attention_bwd_sampled(*flat, kv_count.cpu().numpy(), kv_idx.cpu().numpy(), w.scale, qb, kb)
    for name, (mx, mean) in zip(("dq", "dk", "dv"), sampled_gradient_errors(*grads, ref, qb, kb)):
        print(f"\nWan-like full size, sampled {name}: max/max|ref| {mx:.2e}, mean/mean|ref| {mean:.2e}")
        assert mx <= MAX_REL and mean <= MEAN_REL, (name, mx, mean)
