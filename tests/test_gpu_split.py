"""The key-range split of the attention (nabla_sparse_attn_fwd_grid_split):
outputs and LSE against the fp64 oracle on the GPU's own block lists, and
against the unsplit kernel, on hand-built lists that put kept blocks in
every range, rows whose kept blocks all fall in one range (the others have
no block: weight 0), empty rows, odd block counts and batch 2; repeated
runs on one workspace; plus the argument checks."""
import math

import numpy as np
import pytest
import torch

import oracle
from _parity import LSE_ABS, MAX_ABS, MEAN_ABS, flat_to_grid_rows, grid_to_flat_rows
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


def _lists(B, Hh, Nb, rng, kind):
    cnt = np.zeros((B, Hh, Nb), dtype=np.int32)
    idx = np.full((B, Hh, Nb, Nb), -1, dtype=np.int32)
    for b in range(B):
        for h in range(Hh):
            for i in range(Nb):
                if kind == "spread":
                    n = min(Nb, int(rng.choice([1, 5, 33, Nb // 2, Nb])))
                    sel = np.sort(rng.choice(Nb, size=n, replace=False))
                elif kind == "one_range":  # all kept blocks below Nb / 4
                    hi = max(1, Nb // 4)
                    n = int(rng.integers(1, hi + 1))
                    sel = np.sort(rng.choice(hi, size=n, replace=False))
                else:  # "with_empty": every third row empty
                    if i % 3 == 0:
                        continue
                    n = int(rng.integers(1, Nb + 1))
                    sel = np.sort(rng.choice(Nb, size=n, replace=False))
                cnt[b, h, i] = len(sel)
                idx[b, h, i, :len(sel)] = sel
    return cnt, idx


# Ranges are multiples of 32 blocks, so the grids hold 96-128 blocks (the
# last case, 12 blocks, leaves every range but the first empty).
@pytest.mark.parametrize("B,Hh,D,grid,split,kind", [
    (1, 2, 128, (4, 32, 48), 2, "spread"),
    (1, 2, 128, (4, 32, 48), 3, "spread"),
    (2, 1, 64, (2, 64, 64), 4, "spread"),
    (1, 2, 128, (4, 32, 64), 2, "one_range"),
    (1, 1, 128, (6, 32, 32), 3, "with_empty"),
    (1, 3, 64, (5, 24, 48), 2, "spread"),
    (1, 2, 128, (3, 16, 16), 2, "spread"),
    (1, 2, 128, (4, 48, 64), 5, "spread"),  # the merge's any-count path; ranges 4 and 5 empty
])
def test_split_against_oracle_and_unsplit(B, Hh, D, grid, split, kind):
    T, H, W = grid
    S = T * H * W
    Nb = S // 64
    rng = np.random.default_rng(91 + split)
    g = torch.Generator().manual_seed(92)
    q, k, v = (torch.randn(B, S, Hh, D, generator=g).to(torch.bfloat16) for _ in range(3))
    cnt, idx = _lists(B, Hh, Nb, rng, kind)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    cnt_d, idx_d = torch.from_numpy(cnt).cuda(), torch.from_numpy(idx).cuda()
    qg, kg, vg = (flat_to_grid_rows(x, T, H, W, 1) for x in (qd, kd, vd))
    out_s, lse_s = nabla.sparse_attn_fwd(qg, kg, vg, cnt_d, idx_d, grid=grid, split=split)
    out_1, lse_1 = nabla.sparse_attn_fwd(qg, kg, vg, cnt_d, idx_d, grid=grid)
    torch.cuda.synchronize()
    assert nabla.get_status() == 0
    out_f, lse_f = grid_to_flat_rows(out_s, T, H, W, 1), grid_to_flat_rows(lse_s, T, H, W, 2)
    ref, ref_lse = oracle.attention(q, k, v, cnt, idx, 1.0 / math.sqrt(D))
    err = np.abs(out_f.double().cpu().numpy() - ref)
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
    got_lse = lse_f.double().cpu().numpy()
    finite = np.isfinite(ref_lse)
    assert np.array_equal(finite, np.isfinite(got_lse))
    assert np.abs(got_lse[finite] - ref_lse[finite]).max() <= LSE_ABS
    # empty rows: zero output
    empty = cnt == 0
    if empty.any():
        o = out_f.float().cpu().numpy()  # [B][S][Hh][D], flattened order
        for b, h, i in zip(*np.nonzero(empty)):
            assert not o[b, 64 * i:64 * (i + 1), h].any()
    # against the unsplit kernel: the same attention up to the rounding of
    # the range outputs to bf16 before the merge
    d = (out_s.float() - out_1.float()).abs()
    assert float(d.max()) <= MAX_ABS and float(d.mean()) <= MEAN_ABS
    fin = torch.isfinite(lse_1)
    assert torch.equal(fin, torch.isfinite(lse_s))
    assert float((lse_s[fin] - lse_1[fin]).abs().max()) <= LSE_ABS


@pytest.mark.parametrize("grid,split", [((4, 32, 48), 2), ((2, 64, 64), 4), ((12, 48, 80), 2)])
def test_split_is_deterministic_on_a_reused_workspace(grid, split):
    """Five runs on one workspace, filled with 0xFF before each (stale range
    outputs and LSE), give bit-identical O and LSE, equal to the unsplit
    kernel's up to the rounding of the range outputs."""
    T, H, W = grid
    B, Hh, D = 1, 2, 128
    S = T * H * W
    Nb = S // 64
    rng = np.random.default_rng(7)
    g = torch.Generator().manual_seed(8)
    q, k, v = (torch.randn(B, S, Hh, D, generator=g).to(torch.bfloat16).cuda() for _ in range(3))
    cnt, idx = _lists(B, Hh, Nb, rng, "spread")
    cnt_d, idx_d = torch.from_numpy(cnt).cuda(), torch.from_numpy(idx).cuda()
    ws = torch.empty(nabla.attn_split_workspace_bytes(B, Hh, D, T, H, W, split), dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(5):
        ws.fill_(255)
        outs.append(nabla.sparse_attn_fwd(q, k, v, cnt_d, idx_d, grid=grid, split=split, workspace=ws))
    torch.cuda.synchronize()
    assert nabla.get_status() == 0
    for o, l in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0][0].view(torch.int16))
        assert torch.equal(l.view(torch.int32), outs[0][1].view(torch.int32))
    out_1, _ = nabla.sparse_attn_fwd(q, k, v, cnt_d, idx_d, grid=grid)
    d = (outs[0][0].float() - out_1.float()).abs()
    assert float(d.max()) <= MAX_ABS and float(d.mean()) <= MEAN_ABS


def test_split_on_the_adaptive_mask_of_a_layer():
    """The Wan-1.3B-like layer's own mask, split in 4: sampled query blocks
    against the oracle, the whole output against the unsplit kernel."""
    w = inputs.WAN13B
    q, k, v = inputs.make_qkv(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    cnt, idx, _ = nabla.build_mask_grid(qd, kd, w.T, w.H, w.W, thr=w.thr, sta=w.sta)
    out_s, lse_s = nabla.sparse_attn_fwd(qd, kd, vd, cnt, idx, grid=(w.T, w.H, w.W), split=4)
    out_1, lse_1 = nabla.sparse_attn_fwd(qd, kd, vd, cnt, idx, grid=(w.T, w.H, w.W))
    torch.cuda.synchronize()
    assert nabla.get_status() == 0
    d = (out_s.float() - out_1.float()).abs()
    assert float(d.max()) <= MAX_ABS and float(d.mean()) <= MEAN_ABS
    assert float((lse_s - lse_1).abs().max()) <= LSE_ABS
    # sampled blocks against the oracle (its own flattening of the host tensors)
    qf = oracle.flatten(q, w.T, w.H, w.W).reshape(q.shape)
    kf = oracle.flatten(k, w.T, w.H, w.W).reshape(k.shape)
    vf = oracle.flatten(v, w.T, w.H, w.W).reshape(v.shape)
    rng = np.random.default_rng(1234)
    qblocks = np.sort(rng.choice(w.Nb, size=16, replace=False))
    cnt_h, idx_h = cnt.cpu().numpy(), idx.cpu().numpy()
    ref, ref_lse = oracle.attention(qf, kf, vf, cnt_h, idx_h, w.scale, qblocks=qblocks)
    of = grid_to_flat_rows(out_s, w.T, w.H, w.W, 1).float().cpu().numpy()
    rows = np.concatenate([np.arange(j * 64, (j + 1) * 64) for j in qblocks])
    got = of[:, rows]
    err = np.abs(got - ref)
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())


def test_split_argument_checks():
    x = torch.zeros(1, 1024, 2, 64, dtype=torch.bfloat16, device="cuda")
    cnt = torch.ones(1, 2, 16, dtype=torch.int32, device="cuda")
    idx = torch.zeros(1, 2, 16, 16, dtype=torch.int32, device="cuda")
    with pytest.raises(ValueError):
        nabla.attn_split_workspace_bytes(1, 2, 64, 4, 16, 16, 1)  # split < 2
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    L = nabla.lib()
    rc = L.nabla_sparse_attn_fwd_grid_split(*(nabla._dev(t, t.dtype, "t") for t in (x, x, x, cnt, idx)), 1, 2, 64,
                                            4, 16, 16, 0.0, 1, nabla._dev(ws, torch.uint8, "ws"),
                                            nabla._dev(x, torch.bfloat16, "out"), None, None)
    assert rc == nabla.NABLA_ERR_INVALID  # nsplit = 1
    rc = L.nabla_sparse_attn_fwd_grid_split(*(nabla._dev(t, t.dtype, "t") for t in (x, x, x, cnt, idx)), 1, 2, 64,
                                            4, 16, 16, 0.0, 2, None, nabla._dev(x, torch.bfloat16, "out"), None,
                                            None)
    assert rc == nabla.NABLA_ERR_INVALID  # no workspace
