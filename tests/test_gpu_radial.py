"""The radial decay window (the Radial Attention article's static mask,
"Zastosowanie zasad rozkladu energii") on the GPU, against the oracle.

* nabla_build_mask_radial: the window's lists bit-exact, every row of every
  (batch, head) copy, on several grids and half-widths, entries past the
  count untouched;
* the window OR-ed into the adaptive mask (nabla_params.radial): lists
  bit-exact outside the 1e-5 band, a superset of the window's lists;
* attention on the window's lists against the oracle on sampled blocks.
"""
import numpy as np
import pytest
import torch

import oracle
from _parity import Case, LSE_ABS, MAX_ABS, MEAN_ABS, check_attention, compare_masks
from block_sparse_attention_flatten_b200 import inputs
from block_sparse_attention_flatten_b200 import nabla

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from block_sparse_attention_flatten_b200 import build
    build.build()
    assert torch.cuda.is_available()
    oracle.build()


@pytest.mark.parametrize("T,H,W,r0,B,Hh", [
    (16, 48, 80, 4, 1, 3),
    (9, 24, 40, 1, 2, 2),
    (33, 48, 80, 2, 1, 2),
    (64, 48, 80, 2, 1, 24),  # the long-video grid, every head
    (4, 48, 80, 100, 1, 1),  # window wider than the grid at distance 0
    (1, 8, 8, 1, 3, 1),      # a single block
])
def test_radial_lists_bit_exact(T, H, W, r0, B, Hh):
    Nb = T * H * W // 64
    cnt = torch.full((B, Hh, Nb), -5, dtype=torch.int32, device="cuda")
    idx = torch.full((B, Hh, Nb, Nb), -5, dtype=torch.int32, device="cuda")
    nabla.build_mask_radial(B, Hh, T, H, W, r0, kv_count=cnt, kv_idx=idx)
    torch.cuda.synchronize()
    assert nabla.get_status() == 0
    ref_c, ref_i = oracle.radial_lists(T, H // 8, W // 8, r0)
    ref_i = torch.from_numpy(ref_i).cuda()
    ref_c = torch.from_numpy(ref_c).cuda()
    for b in range(B):
        for h in range(Hh):
            assert torch.equal(cnt[b, h], ref_c)
            valid = torch.arange(Nb, device="cuda").view(1, -1) < ref_c.view(-1, 1)
            # written entries equal the oracle's; the rest untouched
            assert torch.equal(torch.where(valid, idx[b, h], -1), torch.where(valid, ref_i, -1))
            assert torch.all(torch.where(valid, 0, idx[b, h] + 5) == 0)


UNION_CASES = [
    inputs.Workload("radial union Nb=240", 1, 3, 128, 4, 48, 80, 1.0, 0.7, seed=51, radial=3),
    inputs.Workload("radial union + STA Nb=45 D64", 2, 2, 64, 5, 24, 24, 1.0, 0.8, sta=(3, 3, 3), seed=52, radial=1),
    inputs.Workload("radial union thr0", 1, 2, 128, 8, 24, 40, 1.0, 0.0, seed=53, radial=2),
    inputs.HUNYUAN_RADIAL,
]


@pytest.mark.parametrize("w", UNION_CASES, ids=lambda w: w.name)
def test_radial_union_mask_and_attention(w):
    case = Case(w)
    qf_h, kf_h, vf_h = case.host_flat()
    qbar, kbar = oracle.pool(qf_h), oracle.pool(kf_h)
    _, _, status, _ = oracle.build_mask(qbar, kbar, w.thr, w.scale, w.nbh, w.nbw, sta_window=w.sta,
                                        radial_r0=w.radial)
    bad, in_band, nband = compare_masks(case, status)
    print(f"\n{w.name}: mismatches outside band {bad}, inside {in_band}, band blocks {nband}")
    assert bad == 0
    # superset of the window alone
    rc, ri = nabla.build_mask_radial(w.B, w.Hh, w.T, w.H, w.W, w.radial)
    from _parity import keep_matrix_gpu
    keep_u = keep_matrix_gpu(case.kv_count, case.kv_idx)
    keep_r = keep_matrix_gpu(rc, ri)
    assert torch.all(keep_u | ~keep_r)
    # attention on the union lists
    qblocks = inputs.sample_query_blocks(w.Nb, min(w.Nb, 32), seed=1234)
    out, lse = case.attention()
    mx, mean, lse_err = check_attention(case, out, lse, qblocks, (qf_h, kf_h, vf_h))
    assert mx <= MAX_ABS and mean <= MEAN_ABS and lse_err <= LSE_ABS


def test_attention_on_radial_lists():
    w = inputs.Workload("radial only Nb=240", 1, 4, 128, 4, 48, 80, 1.0, 1.0, seed=54, radial=2)
    case = Case(w)
    case.kv_count, case.kv_idx = nabla.build_mask_radial(w.B, w.Hh, w.T, w.H, w.W, w.radial)
    out, lse = case.attention()
    mx, mean, lse_err = check_attention(case, out, lse, np.arange(w.Nb))
    assert mx <= MAX_ABS and mean <= MEAN_ABS and lse_err <= LSE_ABS
