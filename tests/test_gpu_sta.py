"""GPU parity of the static sliding-tile mask (nabla_build_mask_sta) and of
attention on it, through the C ABI, against the CPU oracle.

The lists are integer work and must be bit-exact for every row of every
(batch, head) copy; entries past a row's count are never compared.
Attention on the static lists follows the usual tolerances against the fp64
oracle run on the oracle's own lists.
"""
import numpy as np
import pytest
import torch

import oracle
from _parity import LSE_ABS, MAX_ABS, MEAN_ABS, attention_rows, grid_to_flat_rows, lse_rows
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


# (B, Hh, T, H, W, window)
LIST_CASES = [
    (1, 2, 4, 16, 16, (3, 3, 3)),        # tiny layer grid, 2 x 2 patches
    (2, 3, 16, 48, 80, (3, 3, 3)),       # Wan-1.3B-like grid
    (1, 2, 64, 48, 80, (3, 3, 3)),       # long-video grid (3,840 blocks)
    (1, 2, 5, 24, 56, (5, 3, 1)),        # anisotropic window
    (1, 1, 3, 8, 8, (1, 1, 1)),          # one patch per frame, window = the block itself
    (2, 2, 7, 40, 24, (9, 65535, 3)),    # window wider than the grid along h
    (1, 1, 1, 8, 8, (3, 3, 3)),          # a single block
    (2, 35000, 4, 16, 16, (3, 3, 3)),    # more (b, head) copies than one grid dimension holds
]


def expect_lists(T, H, W, window, device):
    cnt_o, idx_o = oracle.sta_lists(T, H // 8, W // 8, window)
    return torch.from_numpy(cnt_o).to(device), torch.from_numpy(idx_o).to(device)


@pytest.mark.parametrize("B,Hh,T,H,W,window", LIST_CASES,
                         ids=lambda x: "x".join(map(str, x)) if isinstance(x, tuple) else str(x))
def test_sta_lists_bit_exact(B, Hh, T, H, W, window):
    Nb = T * H * W // 64
    kv_count = torch.full((B, Hh, Nb), -7, dtype=torch.int32, device="cuda")
    kv_idx = torch.full((B, Hh, Nb, Nb), -7, dtype=torch.int32, device="cuda")
    nabla.build_mask_sta(B, Hh, T, H, W, window, kv_count=kv_count, kv_idx=kv_idx)
    torch.cuda.synchronize()
    assert nabla.get_status() == 0
    cnt_o, idx_o = expect_lists(T, H, W, window, kv_count.device)
    assert torch.equal(kv_count, cnt_o.expand(B, Hh, Nb))
    e = torch.arange(Nb, device=kv_idx.device, dtype=torch.int32)
    valid = e.view(1, 1, 1, Nb) < kv_count.unsqueeze(-1)
    assert torch.equal(torch.where(valid, kv_idx, -1), idx_o.expand(B, Hh, Nb, Nb))
    # nothing past the count is written
    assert bool((kv_idx[~valid] == -7).all())
    assert nabla.validate_mask(kv_count, kv_idx) == 0


def test_sta_lists_equal_the_window_part_of_the_union():
    # thr = 0 keeps only the arg-max from the CDF, so the union with the
    # window is the window plus at most one block per row
    w = inputs.Workload("sta union", 1, 2, 64, 6, 16, 32, 1.0, 0.0, sta=(3, 3, 3), seed=43)
    q, k, _ = inputs.make_qkv(w)
    qd, kd = q.cuda(), k.cuda()
    cnt_u, idx_u, _ = nabla.build_mask_grid(qd, kd, w.T, w.H, w.W, w.thr, w.sta)
    cnt_s, idx_s = nabla.build_mask_sta(w.B, w.Hh, w.T, w.H, w.W, w.sta)
    torch.cuda.synchronize()
    d = (cnt_u - cnt_s).cpu().numpy()
    assert d.min() >= 0 and d.max() <= 1
    cu, iu, cs, is_ = (x.cpu().numpy() for x in (cnt_u, idx_u, cnt_s, idx_s))
    for hd in range(w.Hh):
        for i in range(w.Nb):
            assert set(is_[0, hd, i, :cs[0, hd, i]]) <= set(iu[0, hd, i, :cu[0, hd, i]])


STA_ATTN = [
    inputs.Workload("sta-only D128 8x32x48", 1, 4, 128, 8, 32, 48, 1.0, 1.0, sta=(3, 3, 3), seed=41),
    inputs.Workload("sta-only D64 odd t 5x24x40", 2, 2, 64, 5, 24, 40, 1.0, 1.0, sta=(3, 3, 5), seed=42),
    inputs.Workload("sta-only Hunyuan-like 32x48x80", 1, 24, 128, 32, 48, 80, 1.0, 1.0, sta=(3, 3, 3), seed=3),
]


@pytest.mark.parametrize("w", STA_ATTN, ids=lambda w: w.name)
def test_attention_on_sta_lists(w):
    q, k, v = inputs.make_qkv(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    kv_count, kv_idx = nabla.build_mask_sta(w.B, w.Hh, w.T, w.H, w.W, w.sta)
    out, lse = nabla.sparse_attn_fwd(qd, kd, vd, kv_count, kv_idx, grid=(w.T, w.H, w.W))
    torch.cuda.synchronize()
    assert nabla.get_status() == 0
    out_f = grid_to_flat_rows(out, w.T, w.H, w.W, 1)
    lse_f = grid_to_flat_rows(lse, w.T, w.H, w.W, 2)
    del out, lse
    qblocks = inputs.sample_query_blocks(w.Nb, min(64, w.Nb), seed=1234)
    cnt_o, idx_o = oracle.sta_lists(w.T, w.nbh, w.nbw, w.sta)
    cnt = np.ascontiguousarray(np.broadcast_to(cnt_o[qblocks], (w.B, w.Hh, len(qblocks))))
    idx = np.ascontiguousarray(np.broadcast_to(idx_o[qblocks], (w.B, w.Hh, len(qblocks), w.Nb)))
    qf = oracle.flatten(q, w.T, w.H, w.W).reshape(q.shape)
    kf = oracle.flatten(k, w.T, w.H, w.W).reshape(k.shape)
    vf = oracle.flatten(v, w.T, w.H, w.W).reshape(v.shape)
    ref, ref_lse = oracle.attention(qf, kf, vf, cnt, idx, w.scale, qblocks=qblocks)
    err = np.abs(attention_rows(out_f, qblocks) - ref)
    lse_err = float(np.abs(lse_rows(lse_f, qblocks) - ref_lse).max())
    print(f"\n{w.name}: kept fraction {cnt_o.sum() / w.Nb ** 2:.4f}; attention max {err.max():.3e} "
          f"mean {err.mean():.3e} lse {lse_err:.3e}")
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS and lse_err <= LSE_ABS
